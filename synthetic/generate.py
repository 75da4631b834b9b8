"""Seeded generators for LLSA inputs (CPU, torch).

Recipe (the same for the CUDA path and the CPU oracle):

* Every tensor draws from its own ``torch.Generator`` seeded with
  ``1000 * seed_base + t`` where t = 0 for Q, 1 for K, 2 for V and 3 for dO.
* ``"normal"`` tensors are i.i.d. N(0, 1).
* ``"smooth"`` tensors are, for each (b, h, channel d), a field on a G x G pixel
  grid: f(r, c) = sum_{m=1..8} a_m sin(2 pi (fx_m c + fy_m r) / G + phi_m) + 0.1 eps(r, c),
  with a_m ~ N(0, 0.5^2), (fx_m, fy_m) uniform over the 48 integer pairs in
  [-3, 3]^2 other than (0, 0), phi_m ~ U[0, 2 pi) and eps ~ N(0, 1).  This stands
  in for the image-like pixel-DiT activations the pages train on (FFHQ faces),
  which are not available here; no item of that dataset is reproduced.
* Tokens are placed in quadtree (Z) order: sequence position z holds pixel
  (r, c) with z = sum_b (2 r_b + c_b) 4^b, so every aligned run of 4^j tokens is
  a 2^j x 2^j square of pixels ("LLSA GitHub README", token reordering example).
* Values are generated in fp32 and then rounded to nearest-even into the
  requested dtype, so both sides receive identical bits.
"""
from __future__ import annotations

import math

import numpy as np
import torch

TENSOR_SLOT = {"q": 0, "k": 1, "v": 2, "do": 3}


def morton_order(G: int) -> np.ndarray:
    """Raster index (r*G + c) of the pixel at each Z-order sequence position.

    Closed form: split the bits of z into pairs; in pair b the higher bit is bit b
    of the row and the lower bit is bit b of the column.
    """
    assert G > 0 and G & (G - 1) == 0, "grid side must be a power of two"
    z = np.arange(G * G, dtype=np.int64)
    r = np.zeros_like(z)
    c = np.zeros_like(z)
    nbits = int(math.log2(G))
    for b in range(nbits):
        c |= ((z >> (2 * b)) & 1) << b
        r |= ((z >> (2 * b + 1)) & 1) << b
    return r * G + c


def quadtree_order_recursive(G: int) -> np.ndarray:
    """Same ordering built a second, independent way: visit the four quadrants
    top-left, top-right, bottom-left, bottom-right and recurse into each."""
    out = []

    def visit(r0: int, c0: int, size: int) -> None:
        if size == 1:
            out.append(r0 * G + c0)
            return
        h = size // 2
        visit(r0, c0, h)
        visit(r0, c0 + h, h)
        visit(r0 + h, c0, h)
        visit(r0 + h, c0 + h, h)

    visit(0, 0, G)
    return np.asarray(out, dtype=np.int64)


_NONZERO_PAIRS = torch.tensor([(fx, fy) for fx in range(-3, 4) for fy in range(-3, 4)
                               if (fx, fy) != (0, 0)], dtype=torch.float32)


def smooth_field_tokens(B: int, H: int, N: int, D: int, gen: torch.Generator) -> torch.Tensor:
    """[B, H, N, D] fp32 smooth fields in Z order (see module docstring)."""
    G = int(round(math.sqrt(N)))
    assert G * G == N, "smooth fields need a square token grid"
    M = 8
    amp = torch.randn(B, H, D, M, generator=gen) * 0.5
    pair = torch.randint(0, _NONZERO_PAIRS.shape[0], (B, H, D, M), generator=gen)
    phase = torch.rand(B, H, D, M, generator=gen) * (2.0 * math.pi)
    noise = torch.randn(B, H, D, G, G, generator=gen)
    fx = _NONZERO_PAIRS[pair, 0]
    fy = _NONZERO_PAIRS[pair, 1]
    coord = torch.arange(G, dtype=torch.float32)
    field = 0.1 * noise
    two_pi_over_g = 2.0 * math.pi / G
    for m in range(M):
        arg = (two_pi_over_g * (fx[..., m, None, None] * coord[None, :]
                                + fy[..., m, None, None] * coord[:, None])
               + phase[..., m, None, None])
        field = field + amp[..., m, None, None] * torch.sin(arg)
    flat = field.reshape(B, H, D, N)                       # raster order
    zpos = torch.from_numpy(morton_order(G))
    tokens = flat[..., zpos]                                # Z order
    return tokens.permute(0, 1, 3, 2).contiguous()         # [B, H, N, D]


def _torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16, "f64": torch.float64}[dtype]


def make_tensor(kind: str, B: int, H: int, N: int, D: int, dtype: str, seed: int) -> torch.Tensor:
    gen = torch.Generator().manual_seed(seed)
    if kind == "normal":
        x = torch.randn(B, H, N, D, generator=gen)
    elif kind == "smooth":
        x = smooth_field_tokens(B, H, N, D, gen)
    else:
        raise ValueError(kind)
    return x.to(_torch_dtype(dtype)).contiguous()


def make_inputs(B: int, H: int, N: int, D: int, dtype: str, qk_kind: str, seed_base: int,
                with_do: bool = True) -> dict:
    """q, k, v (and dO) as CPU torch tensors in ``dtype``; V and dO are always N(0, 1)."""
    out = {
        "q": make_tensor(qk_kind, B, H, N, D, dtype, 1000 * seed_base + TENSOR_SLOT["q"]),
        "k": make_tensor(qk_kind, B, H, N, D, dtype, 1000 * seed_base + TENSOR_SLOT["k"]),
        "v": make_tensor("normal", B, H, N, D, dtype, 1000 * seed_base + TENSOR_SLOT["v"]),
    }
    if with_do:
        out["do"] = make_tensor("normal", B, H, N, D, dtype, 1000 * seed_base + TENSOR_SLOT["do"])
    return out


def make_config_inputs(cfg, with_do: bool | None = None) -> dict:
    """Inputs of one of the named workloads (seed base = its number)."""
    if with_do is None:
        with_do = cfg.backward
    return make_inputs(cfg.B, cfg.H, cfg.N, cfg.D, cfg.dtype, cfg.qk_kind, cfg.seed_base, with_do)


def to_f64_numpy(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32 tensor to a float64 numpy array."""
    return t.detach().to(torch.float64).cpu().numpy()


def to_f32_numpy(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/fp32 tensor to a float32 numpy array."""
    return t.detach().to(torch.float32).cpu().numpy()
