"""Shapes outside the powers of two: any topk, and any N that 16^L divides (n_l need not be
powers of two; with L = 1, n_1 need not be a multiple of 16, so a CTA's query blocks can
straddle two heads).  GPU against the oracle on the GPU's validated selection, through the
five calls, the step and a plan, with and without the enrichment variants."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import (TORCH_DTYPE, check_pyramid_bitexact, check_selection, check_transpose_bitexact,
                          compare_outputs, inputs_for, replay, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    assert api.llsa_device_status() == 0
    yield
    assert api.llsa_device_status() == 0


@pytest.mark.parametrize("B,H,N,topk,levels,dtype,variants", [
    (1, 2, 12288, 8, 2, "bf16", {}),                   # n_1 = 768, n_2 = 48
    (1, 1, 12288, 3, 3, "bf16", {}),                   # n_3 = 3, K = 3
    (2, 1, 1040, 5, 1, "bf16", {}),                    # n_1 = 65: blocks of a CTA span two heads
    (2, 1, 1040, 5, 1, "f32", {}),
    (1, 1, 20480, 6, 2, "f32", {}),                    # n_2 = 80, K = 6
    (1, 1, 61440, 12, 3, "bf16", {}),                  # n_3 = 15, K = 12, (L-1) K = 24
    (1, 1, 12288, 3, 3, "bf16", dict(log_bias=True, all_top=True, level1=True)),
    (1, 2, 20480, 7, 2, "bf16", dict(level1=True)),
])
def test_general_shapes_match_oracle(B, H, N, topk, levels, dtype, variants):
    inputs = inputs_for(B, H, N, 64, dtype, "normal", 61)
    gpu = run_gpu(B, H, N, 64, topk, levels, dtype, inputs, **variants)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, levels)
    check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu, **variants)
    compare_outputs(gpu, ref, dtype, ["o", "lse", "dq", "dk", "dv"])


def test_general_shape_step_and_plan_match_separate_calls():
    B, H, N, K, L = 2, 3, 12288, 6, 2
    inputs = inputs_for(B, H, N, 64, "bf16", "normal", 62)
    ref = run_gpu(B, H, N, 64, K, L, "bf16", inputs)
    tdt = TORCH_DTYPE["bf16"]
    shape = api.make_shape(B, H, N, 64, K, L, tdt)
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


@pytest.mark.parametrize("topk", [2, 4])
def test_four_levels_with_register_resident_selection_at_every_sparse_level(topk):
    # L = 4 with K in {2, 4} at N = 2^20 (a 1024 x 1024 grid) with smooth Q/K fields: levels
    # 3, 2 and 1 all take the register-resident children selection, and the most popular
    # key blocks gather hundreds of query blocks, the hardest case for dK (it sums dS q over
    # every query that selected the key, terms that cancel).
    B, H, N, L = 1, 1, 1 << 20, 4
    inputs = inputs_for(B, H, N, 64, "bf16", "smooth", 63)
    gpu = run_gpu(B, H, N, 64, topk, L, "bf16", inputs)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, L)
    check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu)
    rep = compare_outputs(gpu, ref, "bf16", ["o", "lse", "dq", "dk", "dv"])
    popular = max(int(np.diff(rp[0, 0]).max()) for rp in gpu["row_ptr"][:1])
    print("longest level-1 CSR row", popular, "query blocks")
