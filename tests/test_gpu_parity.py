"""Parity of the CUDA path (through the C ABI) with the CPU oracle on seeded inputs.

Every stage is checked: pyramid bit-exact, selection exact outside the tie window, CSR
transpose bit-exact, and O / LSE / dQ / dK / dV within the stated tolerances against the
oracle replayed on the GPU's indices.  Every call must leave the device status word clear.
"""
import numpy as np
import pytest
import torch

from synthetic import WORKLOADS, make_config_inputs

from llsa_testlib import (check_pyramid_bitexact, check_selection, check_transpose_bitexact, compare_outputs,
                          inputs_for, replay, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def full_check(B, H, N, D, topk, levels, dtype, qk_kind, seed, backward=True):
    inputs = inputs_for(B, H, N, D, dtype, qk_kind, seed)
    gpu = run_gpu(B, H, N, D, topk, levels, dtype, inputs, backward=backward)
    assert gpu["status"] == 0, f"device status {gpu['status']}"
    check_pyramid_bitexact(inputs, gpu, levels)
    sel = check_selection(gpu, topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu, backward=backward)
    names = ["o", "lse"] + (["dq", "dk", "dv"] if backward else [])
    rep = compare_outputs(gpu, ref, dtype, names)
    return sel, rep


# Small cases that span several tiles and CTAs and end in ragged tails, for both dtypes.
@pytest.mark.parametrize("B,H,N,topk,levels", [
    (1, 2, 1024, 8, 1),      # the tiny workload's shape
    (2, 3, 4096, 4, 1),
    (1, 2, 4096, 2, 2),      # n_2 = 16, coarse entries = 2 (one padded coarse tile)
    (1, 1, 8192, 2, 3),      # three levels, n_3 = 2
    (2, 1, 16384, 8, 2),
    (1, 1, 65536, 1, 4),     # four levels, n_4 = 1, K = 1
    (1, 2, 8192, 4, 1),      # coarsest level of 512 keys: scored in two passes of 256
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_shapes(B, H, N, topk, levels, dtype):
    square = int(round(N ** 0.5)) ** 2 == N
    kind = "smooth" if (dtype == "bf16" and square) else "normal"
    sel, rep = full_check(B, H, N, 64, topk, levels, dtype, kind, seed=77)
    print(dtype, (B, H, N, topk, levels), sel["exact"], "/", sel["rows"], rep)


@pytest.mark.parametrize("B,H,N,topk,levels", [
    (1, 1, 16, 1, 1),        # a single block
    (1, 3, 64, 4, 1),        # 4 query blocks: every key block selected
    (3, 1, 256, 16, 1),      # K = n_1: dense attention
    (1, 2, 256, 1, 2),       # n_2 = 1
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_degenerate_shapes(B, H, N, topk, levels, dtype):
    full_check(B, H, N, 64, topk, levels, dtype, "normal", seed=5)


def test_tiny_workload_f32():
    cfg = WORKLOADS["tiny-f32"]
    sel, rep = full_check(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, cfg.qk_kind, seed=cfg.seed_base)
    assert sel["exact"] == sel["rows"]


@pytest.mark.parametrize("name", ["dit-s-4096", "two-level-16384"])
def test_mid_workloads(name):
    cfg = WORKLOADS[name]
    inputs = make_config_inputs(cfg)
    gpu = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, cfg.levels)
    check_selection(gpu, cfg.topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu)
    compare_outputs(gpu, ref, cfg.dtype, ["o", "lse", "dq", "dk", "dv"])


def test_headline_workload_full_size():
    """B=1 H=6 N=65536 L=3 K=8 bf16, the benchmarked step: every stage, every head."""
    cfg = WORKLOADS["headline-65536"]
    inputs = make_config_inputs(cfg)
    gpu = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, cfg.levels)
    check_selection(gpu, cfg.topk)
    check_transpose_bitexact(gpu)
    for h in range(cfg.H):
        ref = replay(inputs, gpu, heads=(0, slice(h, h + 1)))
        compare_outputs(gpu, ref, cfg.dtype, ["o", "lse", "dq", "dk", "dv"], heads=(0, slice(h, h + 1)))


def test_scaleout_workload_full_size():
    """B=1 H=6 N=262144 L=3 K=16 bf16: pyramid, selection and CSR on every head; forward and
    backward outputs on one full head (the backward at this geometry is measured too)."""
    cfg = WORKLOADS["scaleout-262144"]
    inputs = make_config_inputs(cfg, with_do=True)
    gpu = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, cfg.levels)
    check_selection(gpu, cfg.topk)
    check_transpose_bitexact(gpu)
    ref = replay(inputs, gpu, heads=(0, slice(3, 4)))
    compare_outputs(gpu, ref, cfg.dtype, ["o", "lse", "dq", "dk", "dv"], heads=(0, slice(3, 4)))


def test_repeat_calls_are_deterministic():
    cfg = WORKLOADS["two-level-16384"]
    inputs = make_config_inputs(cfg)
    a = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs)
    b = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs)
    for key in ("idx", "row_ptr", "col"):
        for x, y in zip(a[key], b[key]):
            assert np.array_equal(x, y)
    for key in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[key], b[key]), key


def test_out_of_range_index_is_recorded_not_dereferenced():
    """A corrupted selection entry must not fault: kernels clamp it and set the status."""
    from log_linear_hierarchical_b200 import api
    B, H, N, topk, levels = 1, 1, 4096, 4, 2
    inputs = inputs_for(B, H, N, 64, "bf16", "normal", 3)
    shape = api.make_shape(B, H, N, 64, topk, levels, torch.bfloat16)
    dev = {k: v.cuda() for k, v in inputs.items()}
    buf = api.LLSABuffers.allocate(shape, "cuda", torch.bfloat16)
    api.llsa_forward_path(shape, dev["q"], dev["k"], dev["v"], buf)
    assert api.llsa_device_status() == 0
    buf.idx[3] = 1 << 20        # level-1 entry far outside [0, 256)
    api.llsa_forward(shape, dev["q"], dev["k"], dev["v"], buf.k_pyr, buf.v_pyr, buf.idx, buf.o, buf.lse)
    api.llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose)
    assert api.llsa_device_status() == 5   # LLSA_ERR_INTERNAL
    assert api.llsa_device_status() == 0   # cleared by the read


@pytest.mark.parametrize("variants", [{}, dict(log_bias=True, all_top=True, level1=True)])
def test_autograd_op_matches_buffers_path(variants):
    from log_linear_hierarchical_b200 import llsa_attention
    inputs = inputs_for(1, 2, 4096, 64, "bf16", "smooth", 9)
    q, k, v, do = (inputs[n].cuda() for n in ("q", "k", "v", "do"))
    q.requires_grad_(True)
    k.requires_grad_(True)
    v.requires_grad_(True)
    o = llsa_attention(q, k, v, topk=4, levels=2, **variants)
    o.backward(do)
    gpu = run_gpu(1, 2, 4096, 64, 4, 2, "bf16", inputs, **variants)
    assert np.array_equal(o.detach().float().cpu().numpy(), gpu["o"])
    assert np.array_equal(q.grad.float().cpu().numpy(), gpu["dq"])
    assert np.array_equal(k.grad.float().cpu().numpy(), gpu["dk"])


def test_single_level_long_sequence():
    """L = 1 at N = 65536: the coarsest level is 4096 keys (16 scoring passes, 4 queries per
    CTA), and the CSR rows are long."""
    sel, rep = full_check(1, 1, 65536, 64, 8, 1, "bf16", "smooth", seed=41)
    print(sel, rep)
