"""The all-coarsest enrichment variant (LLSA_FLAG_ALL_TOP: every query block's list ends with
all n_L coarsest tokens) on the GPU against the oracle run with ``all_top=True`` on the GPU's
validated selection (replay protocol), in bf16 and fp32, alone and with the log-count bias,
through the five calls, the one-call step and a plan."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import (TORCH_DTYPE, check_pyramid_bitexact, check_selection, check_transpose_bitexact,
                          compare_outputs, inputs_for, replay, run_gpu)
from synthetic import WORKLOADS, make_config_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    assert api.llsa_device_status() == 0
    yield
    assert api.llsa_device_status() == 0


def _kind(N):
    return "smooth" if int(round(N ** 0.5)) ** 2 == N else "normal"  # smooth fields need a square grid


@pytest.mark.parametrize("B,H,N,topk,levels,dtype,log_bias", [
    (1, 2, 4096, 4, 2, "bf16", False),     # C = 16: one coarse tile
    (1, 2, 4096, 4, 2, "f32", False),
    (1, 1, 16384, 2, 3, "bf16", False),    # C = 2 + 4
    (1, 1, 32768, 2, 3, "f32", True),      # C = 2 + 8
    (2, 1, 16384, 8, 2, "bf16", False),    # C = 64: four coarse tiles
    (1, 2, 4096, 4, 2, "bf16", True),
    (1, 1, 65536, 8, 3, "bf16", False),    # the headline geometry: C = 8 + 16
])
def test_all_top_matches_oracle(B, H, N, topk, levels, dtype, log_bias):
    inputs = inputs_for(B, H, N, 64, dtype, _kind(N), 31)
    gpu = run_gpu(B, H, N, 64, topk, levels, dtype, inputs, log_bias=log_bias, all_top=True)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, levels)
    check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu, log_bias=log_bias, all_top=True)
    compare_outputs(gpu, ref, dtype, ["o", "lse", "dq", "dk", "dv"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_all_top_is_the_default_when_k_covers_the_coarsest_level(dtype):
    # K = n_L = 16: the level-L selection is every coarsest token in index order, so the two
    # lists are the same entries in the same order and the kernels give identical bits
    inputs = inputs_for(1, 2, 4096, 64, dtype, "smooth", 32)
    a = run_gpu(1, 2, 4096, 64, 16, 2, dtype, inputs)
    b = run_gpu(1, 2, 4096, 64, 16, 2, dtype, inputs, all_top=True)
    for n in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[n], b[n]), n


def test_all_top_changes_nothing_at_one_level_and_something_above():
    inputs = inputs_for(1, 2, 1024, 64, "bf16", "smooth", 33)
    a = run_gpu(1, 2, 1024, 64, 8, 1, "bf16", inputs)
    b = run_gpu(1, 2, 1024, 64, 8, 1, "bf16", inputs, all_top=True)
    for n in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[n], b[n]), n
    inputs = inputs_for(1, 1, 16384, 64, "bf16", "smooth", 34)   # n_3 = 4 > K = 2
    a = run_gpu(1, 1, 16384, 64, 2, 3, "bf16", inputs)
    b = run_gpu(1, 1, 16384, 64, 2, 3, "bf16", inputs, all_top=True)
    assert not np.array_equal(a["o"], b["o"])
    for x, y in zip(a["idx"], b["idx"]):  # the selection does not depend on the enrichment
        assert np.array_equal(x, y)


def test_all_top_step_and_plan_match_separate_calls():
    cfg = WORKLOADS["headline-65536"]
    inputs = make_config_inputs(cfg)
    ref = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs, all_top=True)
    tdt = TORCH_DTYPE[cfg.dtype]
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, tdt, all_top=True)
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
