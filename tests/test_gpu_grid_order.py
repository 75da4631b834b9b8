"""Token order fused into the path (LLSA GitHub README, token reordering example): with
LLSA_FLAG_GRID_ORDER the inputs and outputs are in the row-major order of the square token
grid and the kernels read and write them through the quadtree (Z) order, with no permutation
pass.  A grid-order call must give exactly (bit for bit) what the same call gives on the
Z-ordered tokens, with its outputs put back in grid order; the Z-order call is itself checked
against the oracle by the other GPU tests, and one case here checks it again directly."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import TORCH_DTYPE, compare_outputs, inputs_for, replay, run_gpu
from oracle import llsa_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert api.llsa_device_status() == 0
    yield
    assert api.llsa_device_status() == 0


def to_grid(t: torch.Tensor) -> torch.Tensor:
    """[B, H, N, D] in Z order -> row-major grid order (the oracle's permutation)."""
    N = t.shape[2]
    side = int(round(N ** 0.5))
    z = torch.from_numpy(orc.zorder_index(side))        # z index of each row-major position
    return t[:, :, z].contiguous()


def grid_vs_z(B, H, N, D, topk, levels, dtype, seed, **variants):
    kind = "smooth" if dtype == "bf16" else "normal"
    inputs = inputs_for(B, H, N, D, dtype, kind, seed)            # Z order
    zres = run_gpu(B, H, N, D, topk, levels, dtype, inputs, **variants)
    ginputs = {k: to_grid(v) for k, v in inputs.items()}
    gres = run_gpu(B, H, N, D, topk, levels, dtype, ginputs, grid_order=True, **variants)
    assert zres["status"] == 0 and gres["status"] == 0
    for name in ("q_pyr", "k_pyr", "v_pyr", "idx", "row_ptr", "col"):
        for a, b in zip(zres[name], gres[name]):
            assert np.array_equal(np.asarray(a).view(np.uint32), np.asarray(b).view(np.uint32)), name
    for name in ("o", "dq", "dk", "dv"):
        want = to_grid(torch.from_numpy(zres[name])).numpy()
        assert np.array_equal(gres[name], want), name
    lse_want = to_grid(torch.from_numpy(zres["lse"])[..., None]).numpy()[..., 0]
    assert np.array_equal(gres["lse"], lse_want)
    return inputs, zres, gres


@pytest.mark.parametrize("B,H,N,topk,levels,D,dtype", [
    (1, 2, 1024, 8, 1, 64, "f32"),
    (2, 1, 4096, 16, 1, 64, "bf16"),
    (1, 2, 4096, 4, 2, 64, "bf16"),
    (1, 2, 4096, 4, 2, 128, "bf16"),
    (1, 1, 4096, 4, 2, 128, "f32"),
    (1, 1, 65536, 8, 3, 64, "bf16"),     # the headline geometry
])
def test_grid_order_equals_z_order(B, H, N, topk, levels, D, dtype):
    grid_vs_z(B, H, N, D, topk, levels, dtype, seed=160)


def test_grid_order_with_enrichment_variants():
    grid_vs_z(1, 1, 16384, 64, 8, 2, "bf16", seed=161, log_bias=True, all_top=True, level1=True)


def test_grid_order_against_the_oracle():
    inputs, zres, gres = grid_vs_z(1, 2, 4096, 64, 4, 2, "bf16", seed=162)
    ref = replay(inputs, zres)
    back = {n: orc.to_z_order(gres[n]) for n in ("o", "dq", "dk", "dv")}
    back["lse"] = orc.to_z_order(gres["lse"][..., None])[..., 0]
    compare_outputs(back, ref, "bf16", ["o", "lse", "dq", "dk", "dv"])


@pytest.mark.parametrize("one_launch,D,variants", [
    (False, 64, {}),
    (True, 64, {}),                                    # the flag changes nothing under grid order
    (False, 128, {}),
    (False, 64, dict(log_bias=True, level1=True)),
])
def test_grid_order_step_and_plan_match_separate_calls(one_launch, D, variants):
    """The one-call step and a plan read quadtree-ordered copies of q, k, v, dO (made by the
    pyramid launch) and write every output to its grid row; the separate calls read the grid
    through patch maps.  Both must give the same bits."""
    B, H, N, K, L = 1, 2, 16384, 8, 2
    ginputs = {k: to_grid(v) for k, v in inputs_for(B, H, N, D, "bf16", "smooth", 163).items()}
    ref = run_gpu(B, H, N, D, K, L, "bf16", ginputs, grid_order=True, **variants)
    tdt = TORCH_DTYPE["bf16"]
    shape = api.make_shape(B, H, N, D, K, L, tdt, grid_order=True, one_launch_select=one_launch, **variants)
    dev = {k: v.cuda() for k, v in ginputs.items()}
    buf = api.LLSABuffers.allocate(shape, "cuda", tdt)
    api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    for n in ("o", "dq", "dk", "dv"):
        assert np.array_equal(getattr(buf, n).float().cpu().numpy(), ref[n]), n
    assert np.array_equal(buf.lse.cpu().numpy(), ref["lse"])
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=2)
    buf.dk.zero_()
    plan.launch()
    torch.cuda.synchronize()
    assert np.array_equal(buf.dk.float().cpu().numpy(), ref["dk"])
    plan.close()


def test_grid_order_headline_step_matches_separate_calls():
    """The benchmarked geometry with row-major grid tensors: the step (quadtree-ordered copies,
    outputs to grid rows) against the separate calls (4 x 4-pixel boxes), bit for bit."""
    B, H, N, K, L = 1, 6, 65536, 8, 3
    ginputs = {k: to_grid(v) for k, v in inputs_for(B, H, N, 64, "bf16", "smooth", 164).items()}
    ref = run_gpu(B, H, N, 64, K, L, "bf16", ginputs, grid_order=True)
    tdt = TORCH_DTYPE["bf16"]
    shape = api.make_shape(B, H, N, 64, K, L, tdt, grid_order=True)
    dev = {k: v.cuda() for k, v in ginputs.items()}
    buf = api.LLSABuffers.allocate(shape, "cuda", tdt)
    api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    for n in ("o", "dq", "dk", "dv"):
        assert np.array_equal(getattr(buf, n).float().cpu().numpy(), ref[n]), n
    assert np.array_equal(buf.lse.cpu().numpy(), ref["lse"])
