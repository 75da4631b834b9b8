"""The synthetic LLSA workloads, by shape.

Each workload is a non-causal multi-head attention problem over a square pixel
grid whose tokens are laid out in quadtree (Z) order, as the LLSA README's token
reordering example recommends for images ("LLSA GitHub README", section on
non-sequential data).  Pixel-space DiT sequences (no patchification) give one
token per pixel, so a G x G image has N = G*G tokens.
"""
from dataclasses import dataclass


@dataclass(frozen=True)
class WorkloadConfig:
    seed_base: int      # inputs are drawn with seed 1000 * seed_base + tensor slot
    name: str
    B: int
    H: int
    N: int
    D: int
    levels: int
    topk: int
    dtype: str          # "f32" or "bf16": the dtype of q, k, v, dO and of the outputs
    qk_kind: str        # "normal" or "smooth"
    backward: bool      # whether the workload's step includes the backward pass
    block: int = 16

    @property
    def grid(self) -> int:
        g = int(round(self.N ** 0.5))
        assert g * g == self.N
        return g

    def level_sizes(self):
        """n_l = N / 16^l tokens at level l = 0..L."""
        return [self.N // self.block ** l for l in range(self.levels + 1)]

    @property
    def kv_len(self) -> int:
        """Entries per query block's KV list: 16*K fine tokens plus K coarse tokens per level 2..L."""
        return self.block * self.topk + (self.levels - 1) * self.topk

    def describe(self) -> str:
        return (f"B={self.B} H={self.H} N={self.N} ({self.grid}x{self.grid} Z-order) D={self.D} "
                f"block={self.block} L={self.levels} topk={self.topk} {self.dtype} q/k={self.qk_kind}")


WORKLOADS = {w.name: w for w in (
    WorkloadConfig(1, "tiny-f32", B=1, H=2, N=1024, D=64, levels=1, topk=8, dtype="f32",
                   qk_kind="normal", backward=True),
    WorkloadConfig(2, "dit-s-4096", B=4, H=6, N=4096, D=64, levels=1, topk=16, dtype="bf16",
                   qk_kind="smooth", backward=True),
    WorkloadConfig(3, "two-level-16384", B=2, H=6, N=16384, D=64, levels=2, topk=8, dtype="bf16",
                   qk_kind="smooth", backward=True),
    WorkloadConfig(4, "headline-65536", B=1, H=6, N=65536, D=64, levels=3, topk=8, dtype="bf16",
                   qk_kind="smooth", backward=True),
    WorkloadConfig(5, "scaleout-262144", B=1, H=6, N=262144, D=64, levels=3, topk=16, dtype="bf16",
                   qk_kind="smooth", backward=False),
    # the headline geometry with 128-channel heads (DiT-B/L/XL-class head width)
    WorkloadConfig(6, "headline-65536-d128", B=1, H=6, N=65536, D=128, levels=3, topk=8, dtype="bf16",
                   qk_kind="smooth", backward=True),
)}


def workload(name: str) -> WorkloadConfig:
    """The workload of that name (tiny-f32, dit-s-4096, two-level-16384, headline-65536,
    scaleout-262144, headline-65536-d128)."""
    return WORKLOADS[name]
