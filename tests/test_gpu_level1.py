"""The level-1 enrichment variant (LLSA_FLAG_LEVEL1: each selected block's level-1 pooled token
joins the list) on the GPU against the oracle run with ``level1=True`` on the GPU's validated
selection (replay protocol).  The oracle attends the pyramid's level-1 rows as extra entries;
the bf16 kernels fold each pooled entry into its block's fine tile, so the two agree only if
the fold is right.  bf16 and fp32, with the other variants, through the five calls, the
one-call step and a plan."""
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


@pytest.mark.parametrize("B,H,N,topk,levels,dtype,log_bias,all_top", [
    (1, 2, 1024, 8, 1, "bf16", False, False),    # L = 1: the pooled entries are the only extra ones
    (1, 2, 1024, 8, 1, "f32", False, False),
    (1, 2, 4096, 4, 2, "bf16", False, False),
    (1, 2, 4096, 4, 2, "f32", True, False),
    (1, 1, 16384, 2, 3, "bf16", True, False),
    (2, 1, 16384, 8, 2, "bf16", False, True),
    (1, 1, 32768, 2, 3, "f32", True, True),
    (1, 1, 65536, 8, 3, "bf16", False, False),   # the headline geometry
    (1, 1, 4096, 16, 1, "bf16", True, False),    # K = 16: sixteen folds per query block
])
def test_level1_matches_oracle(B, H, N, topk, levels, dtype, log_bias, all_top):
    inputs = inputs_for(B, H, N, 64, dtype, _kind(N), 51)
    gpu = run_gpu(B, H, N, 64, topk, levels, dtype, inputs, log_bias=log_bias, all_top=all_top, level1=True)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, levels)
    check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu, log_bias=log_bias, all_top=all_top, level1=True)
    compare_outputs(gpu, ref, dtype, ["o", "lse", "dq", "dk", "dv"])


def test_level1_changes_the_result_but_not_the_selection():
    inputs = inputs_for(1, 1, 16384, 64, "bf16", "smooth", 52)
    a = run_gpu(1, 1, 16384, 64, 2, 3, "bf16", inputs)
    b = run_gpu(1, 1, 16384, 64, 2, 3, "bf16", inputs, level1=True)
    for n in ("o", "dq", "dk", "dv"):
        assert not np.array_equal(a[n], b[n]), n
    for x, y in zip(a["idx"], b["idx"]):
        assert np.array_equal(x, y)


def test_level1_step_and_plan_match_separate_calls():
    cfg = WORKLOADS["headline-65536"]
    inputs = make_config_inputs(cfg)
    ref = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs, level1=True)
    tdt = TORCH_DTYPE[cfg.dtype]
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, tdt, level1=True)
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
