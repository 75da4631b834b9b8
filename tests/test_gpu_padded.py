"""Padded sequences on the GPU (the LLSA GitHub README's usage section: the released kernels
need a power-of-two token length, to be lifted later): a sequence of n_valid real tokens run
on a grid of N positions, N a multiple of 16^L, positions n_valid.. being padding.  Every
stage against the padded-sequence oracle (``oracle/llsa_padded.py``) on the GPU's own
selection: pyramid bit-exact, selection among real tokens only, CSR bit-exact, outputs and
gradients within the tolerances, padding outputs exactly zero, and results that do not
depend on what the padding holds (NaN included)."""
import math

import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from llsa_testlib import TORCH_DTYPE, check_transpose_bitexact, compare_outputs, inputs_for, run_gpu
from oracle import llsa_oracle as orc
from oracle import llsa_padded as opad
from synthetic import to_f32_numpy, to_f64_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert api.llsa_device_status() == 0
    yield
    assert api.llsa_device_status() == 0


def padded_check(B, H, N, D, topk, levels, dtype, n_valid, seed, junk=None):
    kind = "smooth" if (dtype == "bf16" and int(round(N ** 0.5)) ** 2 == N) else "normal"
    inputs = inputs_for(B, H, N, D, dtype, kind, seed)
    if junk is not None:          # overwrite the padding (the oracle zeroes it itself)
        for name in ("q", "k", "v", "do"):
            inputs[name][:, :, n_valid:] = junk
    gpu = run_gpu(B, H, N, D, topk, levels, dtype, inputs, n_valid=n_valid)
    assert gpu["status"] == 0
    # pyramid: bit-exact against the padded oracle
    for name in ("q", "k", "v"):
        ref = opad.build_pyramid_padded(to_f32_numpy(inputs[name]), levels, n_valid)
        for lev in range(levels):
            got = gpu[f"{name}_pyr"][lev]
            assert np.array_equal(got.view(np.uint32), ref[lev].view(np.uint32)), (name, lev + 1)
    sel = orc.check_selection(gpu["q_pyr"], gpu["k_pyr"], gpu["idx"], topk, n_valid=n_valid)
    assert sel["bad"] == 0, sel
    for lev in range(levels):                       # real tokens only
        assert gpu["idx"][lev].max() < math.ceil(n_valid / 16 ** (lev + 1))
    check_transpose_bitexact(gpu)
    q, k, v, do = (to_f64_numpy(inputs[n]) for n in ("q", "k", "v", "do"))
    for x in (q, k, v, do):
        x[:, :, n_valid:] = 0.0
    kp, vp, idx = gpu["k_pyr"], gpu["v_pyr"], gpu["idx"]
    o, lse = opad.forward_padded(q, k, v, kp, vp, idx, n_valid)
    dq, dk, dv = opad.backward_padded(q, k, v, o, lse, do, kp, vp, idx, n_valid)
    rep = compare_outputs(gpu, dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv), dtype, ["o", "lse", "dq", "dk", "dv"])
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert not np.any(gpu[name][:, :, n_valid:]), name   # padding outputs are exactly 0
    return gpu, rep


@pytest.mark.parametrize("B,H,N,topk,levels,n_valid", [
    (1, 2, 1024, 8, 1, 1000),      # partial last block
    (1, 2, 1024, 8, 1, 1009),
    (2, 1, 4096, 4, 2, 3000),      # partial level-2 token, empty level-1 blocks
    (1, 2, 4096, 2, 2, 2600),      # 11 real level-2 tokens of 16
    (1, 1, 8192, 2, 3, 4097),      # one real token in the second level-3 token
    (1, 1, 16384, 8, 2, 16000),
    (1, 1, 65536, 8, 3, 60001),    # the headline geometry, cut
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_padded_matches_oracle(B, H, N, topk, levels, n_valid, dtype):
    padded_check(B, H, N, 64, topk, levels, dtype, n_valid, seed=140)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_padded_head_width_128(dtype):
    padded_check(1, 2, 4096, 128, 4, 2, dtype, 3001, seed=141)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_padding_contents_do_not_matter(dtype):
    a, _ = padded_check(1, 2, 4096, 64, 4, 2, dtype, 2999, seed=142)
    b, _ = padded_check(1, 2, 4096, 64, 4, 2, dtype, 2999, seed=142, junk=float("nan"))
    c, _ = padded_check(1, 2, 4096, 64, 4, 2, dtype, 2999, seed=142, junk=1e4)
    for name in ("q_pyr", "k_pyr", "v_pyr", "idx"):
        for x, y, z in zip(a[name], b[name], c[name]):
            assert np.array_equal(x, y) and np.array_equal(x, z), name
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[name], b[name]) and np.array_equal(a[name], c[name]), name


def test_unpadded_n_valid_is_the_plain_path():
    inputs = inputs_for(1, 2, 4096, 64, "bf16", "smooth", 143)
    a = run_gpu(1, 2, 4096, 64, 4, 2, "bf16", inputs)
    b = run_gpu(1, 2, 4096, 64, 4, 2, "bf16", inputs, n_valid=4096)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[name], b[name]), name


@pytest.mark.parametrize("one_launch", [False, True])
def test_padded_step_and_plan_match_separate_calls(one_launch):
    B, H, N, K, L, nv = 1, 2, 16384, 8, 2, 15000
    inputs = inputs_for(B, H, N, 64, "bf16", "smooth", 144)
    ref = run_gpu(B, H, N, 64, K, L, "bf16", inputs, n_valid=nv)
    tdt = TORCH_DTYPE["bf16"]
    shape = api.make_shape(B, H, N, 64, K, L, tdt, n_valid=nv, one_launch_select=one_launch)
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
