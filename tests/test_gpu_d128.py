"""Head width D = 128 (the README usage section makes LLSA a drop-in for
scaled_dot_product_attention, whose heads are 64 or 128 wide in DiT-B/L/XL-class models):
every stage of the CUDA path against the oracle at D = 128, in bf16 and fp32, across several
tiles with ragged tails, with the enrichment variants, at the headline geometry, and through
the one-call step and a plan."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import (TORCH_DTYPE, check_pyramid_bitexact, check_selection, check_transpose_bitexact,
                          compare_outputs, inputs_for, replay, run_gpu)

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(autouse=True)
def _status_clean():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert api.llsa_device_status() == 0
    yield
    assert api.llsa_device_status() == 0


def full_check(B, H, N, topk, levels, dtype, seed, heads=None, **variants):
    kind = "smooth" if (dtype == "bf16" and int(round(N ** 0.5)) ** 2 == N) else "normal"
    inputs = inputs_for(B, H, N, D, dtype, kind, seed)
    gpu = run_gpu(B, H, N, D, topk, levels, dtype, inputs, **variants)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, levels)
    check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    for hs in (heads or [None]):
        ref = replay(inputs, gpu, heads=hs, **variants)
        compare_outputs(gpu, ref, dtype, ["o", "lse", "dq", "dk", "dv"], heads=hs)
    return inputs, gpu


@pytest.mark.parametrize("B,H,N,topk,levels", [
    (1, 2, 1024, 8, 1),      # the tiny workload's geometry
    (2, 3, 4096, 4, 1),
    (1, 2, 4096, 2, 2),      # one padded coarse tile
    (1, 1, 8192, 2, 3),      # three levels
    (2, 1, 16384, 8, 2),     # the two-level geometry
    (1, 1, 12288, 6, 2),     # N and K not powers of two
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_d128_matches_oracle(B, H, N, topk, levels, dtype):
    full_check(B, H, N, topk, levels, dtype, seed=128)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_d128_enrichment_variants(dtype):
    full_check(1, 2, 4096, 4, 2, dtype, seed=129, log_bias=True, all_top=True, level1=True)


def test_d128_headline_geometry():
    """B=1 H=2 N=65536 L=3 K=8 bf16 at D = 128: every stage, both heads."""
    full_check(1, 2, 65536, 8, 3, "bf16", seed=130, heads=[(0, slice(0, 1)), (0, slice(1, 2))])


def test_d128_step_and_plan_match_separate_calls():
    B, H, N, K, L = 1, 2, 16384, 8, 2
    inputs = inputs_for(B, H, N, D, "bf16", "smooth", 131)
    ref = run_gpu(B, H, N, D, K, L, "bf16", inputs)
    tdt = TORCH_DTYPE["bf16"]
    shape = api.make_shape(B, H, N, D, K, L, tdt)
    dev = {k: v.cuda() for k, v in inputs.items()}
    buf = api.LLSABuffers.allocate(shape, "cuda", tdt)
    api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    for n in ("o", "dq", "dk", "dv"):
        assert np.array_equal(getattr(buf, n).float().cpu().numpy(), ref[n]), n
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=2)
    buf.dk.zero_()
    plan.launch()
    torch.cuda.synchronize()
    assert np.array_equal(buf.dk.float().cpu().numpy(), ref["dk"])
    plan.close()


def test_d128_autograd_op():
    from log_linear_hierarchical_b200 import llsa_attention
    inputs = inputs_for(1, 2, 4096, D, "bf16", "smooth", 132)
    q, k, v, do = (inputs[n].cuda() for n in ("q", "k", "v", "do"))
    for t in (q, k, v):
        t.requires_grad_(True)
    o = llsa_attention(q, k, v, topk=4, levels=2)
    o.backward(do)
    gpu = run_gpu(1, 2, 4096, D, 4, 2, "bf16", inputs)
    assert np.array_equal(o.detach().float().cpu().numpy(), gpu["o"])
    assert np.array_equal(k.grad.float().cpu().numpy(), gpu["dk"])
