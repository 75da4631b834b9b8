"""Causal LLSA (LLSA_FLAG_CAUSAL) on the GPU against the causal oracle
(``oracle/llsa_causal.py``): the pyramid bit-exact, the selection row by row under the
causal candidate rule (exact, or a near tie), the index transposes bit-exact with the empty
slots of short lists dropped, and O, LSE, dQ, dK, dV within the bf16 bound of the oracle
replayed on the GPU's own selection.  One level with K = n_1 is dense causal attention, so
that case is also checked against torch's SDPA with is_causal=True."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from log_linear_hierarchical_b200 import _lib, api
from llsa_testlib import (TORCH_DTYPE, check_pyramid_bitexact, compare_outputs, inputs_for, max_err, run_gpu)
from oracle import llsa_causal as oc
from synthetic import to_f64_numpy

pytestmark = pytest.mark.gpu

KEYS = ("o", "dq", "dk", "dv")


@pytest.fixture(autouse=True)
def _status_clean():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert api.llsa_device_status() == 0
    yield
    assert api.llsa_device_status() == 0


def replay_causal(inputs, gpu):
    q, k, v, do = (to_f64_numpy(inputs[n]) for n in ("q", "k", "v", "do"))
    o, lse = oc.forward_causal(q, k, v, gpu["k_pyr"], gpu["v_pyr"], gpu["idx"])
    dq, dk, dv = oc.backward_causal(q, k, v, o, lse, do, gpu["k_pyr"], gpu["v_pyr"], gpu["idx"])
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


def check_causal(B, H, N, D, topk, levels, seed):
    inputs = inputs_for(B, H, N, D, "bf16", "smooth", seed)
    gpu = run_gpu(B, H, N, D, topk, levels, "bf16", inputs, causal=True)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, levels)
    res = oc.check_selection_causal(gpu["q_pyr"], gpu["k_pyr"], gpu["idx"], topk)
    print("causal selection rows", res["rows"], "exact", res["exact"], "tie window", res["tie_window"],
          "fp32 bound", res["floor_used"])
    assert res["bad"] == 0, res
    assert res["floor_used"] <= 1e-3 * res["rows"] + 2, res
    for lev, lv in enumerate(gpu["idx"]):
        for b in range(B):
            for h in range(H):
                rp, cl = oc.index_transpose_causal(lv[b, h], lv.shape[2])
                assert np.array_equal(gpu["row_ptr"][lev][b, h], rp), (lev, b, h)
                assert np.array_equal(gpu["col"][lev][b, h][:rp[-1]], cl), (lev, b, h)
    compare_outputs(gpu, replay_causal(inputs, gpu), "bf16", ["o", "lse", "dq", "dk", "dv"])
    return inputs, gpu


@pytest.mark.parametrize("B,H,N,topk,levels,D", [
    (1, 2, 1024, 8, 1, 64),        # one level: the first blocks have short lists
    (2, 1, 4096, 4, 2, 64),
    (1, 2, 16384, 8, 2, 64),
    (1, 1, 65536, 8, 3, 64),       # the headline geometry, one head
    (1, 1, 65536, 3, 3, 64),       # K = 3: the generic selection kernel
    (1, 1, 1 << 18, 2, 4, 64),     # four levels
    (1, 2, 4096, 4, 2, 128),       # 128-channel heads
])
def test_causal_matches_oracle(B, H, N, topk, levels, D):
    check_causal(B, H, N, D, topk, levels, seed=170 + levels)


def test_one_level_every_past_block_is_sdpa_causal():
    B, H, N, D = 1, 2, 1024, 64                   # K = n_1 = 64
    inputs, gpu = check_causal(B, H, N, D, N // 16, 1, seed=180)
    q, k, v = (inputs[n].float().requires_grad_(True) for n in ("q", "k", "v"))
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
    o.backward(inputs["do"].float())
    assert max_err(gpu["o"], o.detach().numpy()) < 2e-2
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        assert max_err(gpu[name], t.grad.numpy()) < 2e-2, name


def test_short_lists_end_in_no_pick():
    B, H, N, K, L = 1, 1, 4096, 8, 2
    gpu = run_gpu(B, H, N, 64, K, L, "bf16", inputs_for(B, H, N, 64, "bf16", "smooth", 181), backward=False,
                  causal=True)
    top = gpu["idx"][1][0, 0]                     # level 2: query a has a + 1 candidates
    for a in range(16):
        assert np.count_nonzero(top[a] == _lib.LLSA_NO_PICK) == max(0, K - (a + 1))
    for lv in gpu["idx"]:                        # real picks strictly ascending, then only NO_PICK
        real = lv != _lib.LLSA_NO_PICK
        assert np.all(real[..., :-1] >= real[..., 1:])
        d = np.diff(lv.astype(np.int64), axis=-1)
        assert np.all((d > 0) | ~real[..., 1:])


def test_causal_step_and_plan_match_separate_calls():
    B, H, N, K, L = 1, 2, 16384, 8, 2
    inputs = inputs_for(B, H, N, 64, "bf16", "smooth", 182)
    ref = run_gpu(B, H, N, 64, K, L, "bf16", inputs, causal=True)
    tdt = TORCH_DTYPE["bf16"]
    shape = api.make_shape(B, H, N, 64, K, L, tdt, causal=True)
    dev = {k: v.cuda() for k, v in inputs.items()}
    buf = api.LLSABuffers.allocate(shape, "cuda", tdt)
    api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    for n in KEYS:
        assert np.array_equal(getattr(buf, n).float().cpu().numpy(), ref[n]), n
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=2)
    buf.dk.zero_()
    plan.launch()
    torch.cuda.synchronize()
    assert np.array_equal(buf.dk.float().cpu().numpy(), ref["dk"])
    plan.close()


def test_autograd_is_causal_matches_the_calls():
    B, H, N, K = 1, 2, 4096, 4
    inputs = inputs_for(B, H, N, 64, "bf16", "smooth", 183)
    ref = run_gpu(B, H, N, 64, K, 2, "bf16", inputs, causal=True)
    q, k, v = (inputs[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
    o = api.llsa_l2(q, k, v, topk=K, is_causal=True)
    o.backward(inputs["do"].cuda())
    assert np.array_equal(o.detach().float().cpu().numpy(), ref["o"])
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        assert np.array_equal(t.grad.float().cpu().numpy(), ref[name]), name


def test_causal_headline_workload_all_heads():
    """The benchmarked geometry (B=1 H=6 N=65536 L=3 K=8) under the causal mask: every stage
    of every head against the causal oracle."""
    from synthetic import WORKLOADS, make_config_inputs
    cfg = WORKLOADS["headline-65536"]
    inputs = make_config_inputs(cfg, with_do=True)
    gpu = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs, causal=True)
    assert gpu["status"] == 0
    check_pyramid_bitexact(inputs, gpu, cfg.levels)
    res = oc.check_selection_causal(gpu["q_pyr"], gpu["k_pyr"], gpu["idx"], cfg.topk)
    assert res["bad"] == 0 and res["floor_used"] <= 1e-3 * res["rows"] + 2, res
    for h in range(cfg.H):
        one = {k: v[:, h:h + 1] for k, v in inputs.items()}
        sub = {n: [x[:, h:h + 1] for x in gpu[n]] for n in ("k_pyr", "v_pyr", "idx")}
        ref = replay_causal(one, sub)
        got = {n: gpu[n][:, h:h + 1] for n in ("o", "lse", "dq", "dk", "dv")}
        compare_outputs(got, ref, "bf16", ["o", "lse", "dq", "dk", "dv"])
