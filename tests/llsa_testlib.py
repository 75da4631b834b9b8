"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and compare with
the CPU oracle on identical seeded inputs.

Protocol (selection near-ties): the pyramid must be bit-identical; the GPU's selection is
checked level by level against the oracle's fp64 scores (a row passes if it is the
oracle's Top-K, or a valid Top-K within the tie window); then attention outputs and
gradients are compared with the oracle re-run on the GPU's checked indices ("replay").
"""
from __future__ import annotations

import numpy as np
import torch

from log_linear_hierarchical_b200 import api
from oracle import llsa_oracle as orc
from synthetic import make_inputs, to_f32_numpy, to_f64_numpy

# Tolerances stated for the path: max-abs 1e-4 (fp32) and 2e-2 (bf16) on O, dQ, dK, dV.
TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def run_gpu(B, H, N, D, topk, levels, dtype, inputs, backward=True, device="cuda", log_bias=False, all_top=False,
            level1=False, n_valid=0, grid_order=False, causal=False):
    """All five calls on one stream; returns CPU tensors of every output."""
    tdt = TORCH_DTYPE[dtype]
    shape = api.make_shape(B, H, N, D, topk, levels, tdt, log_bias=log_bias, all_top=all_top,
                           level1=level1, n_valid=n_valid, grid_order=grid_order, causal=causal)
    dev = {k: v.to(device) for k, v in inputs.items()}
    buf = api.LLSABuffers.allocate(shape, device, tdt)
    assert api.llsa_device_status() == 0
    api.llsa_forward_path(shape, dev["q"], dev["k"], dev["v"], buf)
    if backward:
        api.llsa_backward_path(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    else:
        api.llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose)
    torch.cuda.synchronize()
    status = api.llsa_device_status()
    out = {
        "status": status,
        "q_pyr": [t.cpu().numpy() for t in buf.pyramid_levels(buf.q_pyr)],
        "k_pyr": [t.cpu().numpy() for t in buf.pyramid_levels(buf.k_pyr)],
        "v_pyr": [t.cpu().numpy() for t in buf.pyramid_levels(buf.v_pyr)],
        "idx": [t.cpu().numpy() for t in buf.idx_levels()],
        "row_ptr": [t.cpu().numpy() for t in buf.csr_levels()[0]],
        "col": [t.cpu().numpy() for t in buf.csr_levels()[1]],
        "o": buf.o.float().cpu().numpy(),
        "lse": buf.lse.cpu().numpy(),
    }
    if backward:
        out["dq"] = buf.dq.float().cpu().numpy()
        out["dk"] = buf.dk.float().cpu().numpy()
        out["dv"] = buf.dv.float().cpu().numpy()
    return out


def check_pyramid_bitexact(inputs, gpu, levels):
    for name in ("q", "k", "v"):
        ref = orc.build_pyramid(to_f32_numpy(inputs[name]), levels)
        for lev in range(levels):
            got = gpu[f"{name}_pyr"][lev]
            assert got.shape == ref[lev].shape
            if not np.array_equal(got.view(np.uint32), ref[lev].view(np.uint32)):
                bad = np.argwhere(got.view(np.uint32) != ref[lev].view(np.uint32))[:3]
                raise AssertionError(f"{name} pyramid level {lev + 1} differs at {bad.tolist()}")


# Rows whose selection needed the fp32 error bound of a pair (beyond the stated 1e-5
# relative window) may be at most this fraction of all rows, plus FLOOR_ROWS_SLACK.
FLOOR_ROWS_FRACTION = 1e-3
FLOOR_ROWS_SLACK = 2


def check_selection(gpu, topk):
    """Selection parity: no bad row, and few rows that lean on the fp32 bound."""
    res = orc.check_selection(gpu["q_pyr"], gpu["k_pyr"], gpu["idx"], topk)
    assert res["bad"] == 0, res
    assert res["floor_used"] <= FLOOR_ROWS_FRACTION * res["rows"] + FLOOR_ROWS_SLACK, res
    print("selection rows", res["rows"], "exact", res["exact"], "tie window", res["tie_window"],
          "fp32 bound", res["floor_used"])
    return res


def check_transpose_bitexact(gpu):
    rps, cols = orc.index_transpose_all(gpu["idx"])
    for lev, (rp, cl) in enumerate(zip(rps, cols)):
        assert np.array_equal(gpu["row_ptr"][lev], rp), f"row_ptr level {lev + 1}"
        assert np.array_equal(gpu["col"][lev], cl), f"col level {lev + 1}"


def replay(inputs, gpu, backward=True, heads=None, log_bias=False, all_top=False, level1=False):
    """Oracle forward (and backward) on the GPU's indices; ``heads`` = (b, h slice) subset."""
    def sl(x):
        return x if heads is None else x[heads[0]:heads[0] + 1, heads[1]]
    q, k, v = (sl(to_f64_numpy(inputs[n])) for n in ("q", "k", "v"))
    kp = [sl(x) for x in gpu["k_pyr"]]
    vp = [sl(x) for x in gpu["v_pyr"]]
    idx = [sl(x) for x in gpu["idx"]]
    o, lse = orc.forward(q, k, v, kp, vp, idx, log_bias=log_bias, all_top=all_top, level1=level1)
    out = {"o": o, "lse": lse}
    if backward:
        do = sl(to_f64_numpy(inputs["do"]))
        out["dq"], out["dk"], out["dv"] = orc.backward(q, k, v, o, lse, do, kp, vp, idx, log_bias=log_bias,
                                                           all_top=all_top, level1=level1)
    return out


def max_err(a, b):
    return float(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)).max())


def bf16_half_ulp(x):
    """Half a unit in the last place of bf16 (8 significant bits) at |x|: the most that
    storing an exact value in the output format changes it, 2^(floor(log2 |x|) - 8)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


# From |ref| = 8 on, the bf16 output store alone can change a value by 2^-5 > 2e-2.
BF16_STORE_FROM = 8.0


def output_limit(ref, dtype, name):
    """Per-element bound of |gpu - ref|.  fp32 outputs: 1e-4.  bf16 outputs: 2e-2, plus the
    bf16 store's half-ulp where |ref| >= 8 (there the rounding of the stored result alone
    exceeds 2e-2).  LSE is fp32 in both dtypes: 1e-4, or 1e-2 on the bf16 path (coarse K/V
    rows are rounded to bf16 before the score products)."""
    r = np.asarray(ref, np.float64)
    if name == "lse":
        return np.full_like(r, 1e-4 if dtype == "f32" else 1e-2)
    if dtype == "bf16":
        return TOL["bf16"] + np.where(np.abs(r) >= BF16_STORE_FROM, bf16_half_ulp(r), 0.0)
    return np.full_like(r, TOL[dtype])


def compare_outputs(gpu, ref, dtype, names, heads=None):
    """Element-wise check |gpu - ref| <= output_limit.  The report records, per output, the
    largest error, the largest |ref|, the worst excess over the bound, and how many elements
    exceed the plain stated tolerance (2e-2 bf16, 1e-4 fp32) -- only elements with
    |ref| >= 8 can do so and still pass."""
    report = {}
    for n in names:
        g = np.asarray(gpu[n] if heads is None else gpu[n][heads[0]:heads[0] + 1, heads[1]], np.float64)
        r = np.asarray(ref[n], np.float64)
        err = np.abs(g - r)
        lim = output_limit(r, dtype, n)
        plain = 1e-2 if (n == "lse" and dtype == "bf16") else (1e-4 if n == "lse" else TOL[dtype])
        worst = np.unravel_index(np.argmax(err - lim), err.shape)
        report[n] = dict(max_abs=float(err.max()), max_ref=float(np.abs(r).max()),
                         worst_excess=float((err - lim)[worst]), over_plain=int(np.count_nonzero(err > plain)),
                         ok=bool(np.all(err <= lim)))
    print("outputs", {n: (round(v["max_abs"], 6), round(v["max_ref"], 3), v["over_plain"]) for n, v in report.items()})
    for n, rep in report.items():
        assert rep["ok"], f"{n}: error exceeds tolerance by {rep['worst_excess']:.3g}; all: {report}"
    return report


def inputs_for(B, H, N, D, dtype, qk_kind, seed):
    return make_inputs(B, H, N, D, dtype, qk_kind, seed)
