"""The one-call step (llsa_train_step, transpose on a second stream) and its CUDA-graph
plan give the same bits as the five calls made one after another on one stream."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import TORCH_DTYPE, run_gpu
from synthetic import WORKLOADS, make_config_inputs, make_inputs

pytestmark = pytest.mark.gpu

KEYS = ("o", "lse", "dq", "dk", "dv")


def outputs(buf):
    out = {k: getattr(buf, k).float().cpu().numpy() for k in KEYS}
    out["idx"] = buf.idx.cpu().numpy()
    out["row_ptr"] = buf.row_ptr.cpu().numpy()
    out["col"] = buf.col.cpu().numpy()
    return out


def assert_same(a, b):
    for x, y in zip(a["idx"], b["idx"]):
        assert np.array_equal(x, y)
    for x, y in zip(a["col"], b["col"]):
        assert np.array_equal(x, y)
    for x, y in zip(a["row_ptr"], b["row_ptr"]):
        assert np.array_equal(x, y)
    for k in KEYS:
        assert np.array_equal(a[k], b[k]), k


def separate_calls(cfg, inputs):
    ref = run_gpu(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, cfg.dtype, inputs)
    ref["idx"] = np.concatenate([x.ravel() for x in ref["idx"]])
    ref["row_ptr"] = np.concatenate([x.ravel() for x in ref["row_ptr"]])
    ref["col"] = np.concatenate([x.ravel() for x in ref["col"]])
    return ref


def setup(cfg, inputs):
    tdt = TORCH_DTYPE[cfg.dtype]
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, tdt)
    dev = {k: v.cuda() for k, v in inputs.items()}
    return shape, dev, api.LLSABuffers.allocate(shape, "cuda", tdt)


def flat(out):
    return {k: (v.ravel() if k in ("idx", "row_ptr", "col") else v) for k, v in out.items()}


@pytest.mark.parametrize("name", ["tiny-f32", "two-level-16384"])
def test_train_step_matches_separate_calls(name):
    cfg = WORKLOADS[name]
    inputs = make_config_inputs(cfg)
    ref = separate_calls(cfg, inputs)
    shape, dev, buf = setup(cfg, inputs)
    api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    assert api.llsa_device_status() == 0
    assert_same(flat(outputs(buf)), ref)


def test_train_step_without_side_stream():
    cfg = WORKLOADS["two-level-16384"]
    inputs = make_config_inputs(cfg)
    ref = separate_calls(cfg, inputs)
    shape, dev, buf = setup(cfg, inputs)
    s = torch.cuda.current_stream()
    api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, side=s)
    torch.cuda.synchronize()
    assert_same(flat(outputs(buf)), ref)


def test_plan_replays_match_separate_calls():
    cfg = WORKLOADS["two-level-16384"]
    inputs = make_config_inputs(cfg)
    ref = separate_calls(cfg, inputs)
    shape, dev, buf = setup(cfg, inputs)
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=2)
    for _ in range(2):
        for t in (buf.o, buf.dq, buf.dk, buf.dv):
            t.zero_()
        plan.launch()
        torch.cuda.synchronize()
        assert api.llsa_device_status() == 0
        assert_same(flat(outputs(buf)), ref)
    # the plan reads its inputs at launch time: new inputs in the same buffers, new results
    other = make_inputs(cfg.B, cfg.H, cfg.N, cfg.D, cfg.dtype, cfg.qk_kind, cfg.seed_base + 100)
    ref2 = separate_calls(cfg, other)
    for k in ("q", "k", "v", "do"):
        dev[k].copy_(other[k].cuda())
    plan.launch()
    torch.cuda.synchronize()
    assert_same(flat(outputs(buf)), ref2)
    plan.close()


def test_plan_is_traced_at_every_launch():
    cfg = WORKLOADS["two-level-16384"]
    inputs = make_config_inputs(cfg)
    shape, dev, buf = setup(cfg, inputs)
    with api.LaunchTrace(64) as eager:
        api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    per_step = eager.used
    assert per_step >= 10
    tr = api.LaunchTrace(64)
    with tr:
        plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=3)
    assert tr.used == 3 * per_step
    plan.launch()
    times = tr.launches()
    assert [n for n, _ in times] == [n for n, _ in eager.launches()] * 3
    assert all(ms > 0 for _, ms in times)
    plan.close()


def test_plan_headline_matches_serialized_calls():
    """Full headline size: the plan (kernels chained by programmatic dependent launch, dK/dV
    overlapping the coarse reduction) against the five calls run with trace events between
    every kernel, which serialises them; bit for bit over three replays."""
    cfg = WORKLOADS["headline-65536"]
    inputs = make_config_inputs(cfg)
    shape, dev, buf = setup(cfg, inputs)
    with api.LaunchTrace(64):
        api.llsa_forward_path(shape, dev["q"], dev["k"], dev["v"], buf)
        api.llsa_backward_path(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    torch.cuda.synchronize()
    assert api.llsa_device_status() == 0
    ref = outputs(buf)
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=3)
    for _ in range(3):
        for t in (buf.o, buf.lse, buf.dq, buf.dk, buf.dv, buf.ws_backward, buf.row_ptr, buf.col):
            t.fill_(7)
        plan.launch()
        torch.cuda.synchronize()
        assert api.llsa_device_status() == 0
        assert_same(outputs(buf), ref)
    plan.close()


@pytest.mark.parametrize("B,H,N,K,L,D", [
    (1, 2, 65536, 8, 3, 64),     # the headline geometry: levels 3 pooled with the coarsest Top-K
    (1, 1, 1 << 18, 2, 4, 64),   # four levels, n_4 = 4
    (2, 1, 16384, 16, 2, 128),   # two levels, D = 128, K = 16
    (1, 2, 4096, 2, 2, 64),      # n_2 = 16
])
def test_fused_pyramid_and_selection_equal_the_separate_launches(B, H, N, K, L, D):
    """With LLSA_FLAG_ONE_LAUNCH_SELECT a step runs the pyramid and every selection level as
    one cooperative launch (pyramid_select); its pyramid, selection and all results are
    bit-identical to the separate pyramid and selection kernels of the five calls."""
    inputs = make_inputs(B, H, N, D, "bf16", "smooth", 150 + L)
    ref = run_gpu(B, H, N, D, K, L, "bf16", inputs)
    shape = api.make_shape(B, H, N, D, K, L, torch.bfloat16, one_launch_select=True)
    dev = {k: v.cuda() for k, v in inputs.items()}
    buf = api.LLSABuffers.allocate(shape, "cuda", torch.bfloat16)
    with api.LaunchTrace(64) as tr:
        api.llsa_train_step(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    names = [n for n, _ in tr.launches()]
    assert api.llsa_device_status() == 0
    assert names[0] == "pyramid_select" and "select" not in names and "pyramid_l12" not in names, names
    for name, got in (("q_pyr", buf.q_pyr), ("k_pyr", buf.k_pyr), ("v_pyr", buf.v_pyr)):
        want = np.concatenate([x.ravel() for x in ref[name]])
        assert np.array_equal(got.cpu().numpy().view(np.uint32), want.view(np.uint32)), name
    assert np.array_equal(buf.idx.cpu().numpy(), np.concatenate([x.ravel() for x in ref["idx"]]))
    for k in KEYS:
        assert np.array_equal(getattr(buf, k).float().cpu().numpy(), ref[k]), k
    plan = api.LLSAPlan(shape, dev["q"], dev["k"], dev["v"], dev["do"], buf, repeat=2)
    for k in KEYS:
        getattr(buf, k).zero_()
    plan.launch()
    torch.cuda.synchronize()
    assert api.llsa_device_status() == 0
    for k in KEYS:
        assert np.array_equal(getattr(buf, k).float().cpu().numpy(), ref[k]), k
    plan.close()
    # without the flag the same step takes the separate launches
    plain = api.make_shape(B, H, N, D, K, L, torch.bfloat16)
    with api.LaunchTrace(64) as tr:
        api.llsa_train_step(plain, dev["q"], dev["k"], dev["v"], dev["do"], buf)
    names = [n for n, _ in tr.launches()]
    assert names[0] == "pyramid_l12" and "pyramid_select" not in names, names
