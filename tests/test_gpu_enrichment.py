"""The log-count enrichment variant (LLSA_FLAG_LOG_BIAS) on the GPU against the oracle run
with ``log_bias=True`` on the GPU's validated selection (replay protocol), in bf16 and fp32,
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


@pytest.mark.parametrize("B,H,N,topk,levels,dtype", [
    (1, 2, 4096, 4, 2, "bf16"),
    (1, 2, 4096, 4, 2, "f32"),
    (1, 1, 8192, 2, 3, "bf16"),
    (1, 1, 8192, 2, 3, "f32"),
    (2, 1, 16384, 8, 2, "bf16"),
    (1, 2, 1024, 8, 1, "bf16"),   # L = 1: no coarse entries, the flag changes nothing
])
def test_log_bias_matches_oracle(B, H, N, topk, levels, dtype):
    kind = "smooth" if int(round(N ** 0.5)) ** 2 == N else "normal"  # smooth fields need a square grid
    inputs = inputs_for(B, H, N, 64, dtype, kind, 21)
    gpu = run_gpu(B, H, N, 64, topk, levels, dtype, inputs, log_bias=True)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, levels)
    check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu, log_bias=True)
    compare_outputs(gpu, ref, dtype, ["o", "lse", "dq", "dk", "dv"])


def test_log_bias_changes_the_result_when_there_are_coarse_tokens():
    inputs = inputs_for(1, 1, 8192, 64, "bf16", "normal", 22)
    a = run_gpu(1, 1, 8192, 64, 2, 3, "bf16", inputs)
    b = run_gpu(1, 1, 8192, 64, 2, 3, "bf16", inputs, log_bias=True)
    assert not np.array_equal(a["o"], b["o"])
    for x, y in zip(a["idx"], b["idx"]):  # the selection does not depend on the weighting
        assert np.array_equal(x, y)


def test_log_bias_step_and_plan_match_separate_calls():
    cfg = WORKLOADS["headline-65536"]
    inputs = make_config_inputs(cfg)
    ref = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs, log_bias=True)
    tdt = TORCH_DTYPE[cfg.dtype]
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, tdt, log_bias=True)
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
