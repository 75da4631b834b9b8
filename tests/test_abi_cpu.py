"""The C-ABI library on a machine without a GPU: it loads, exports every symbol the header
declares, and its host-side checks and size queries behave as documented.  No call here
reaches a kernel launch."""
import ctypes
import os
import re

import pytest
import torch

from log_linear_hierarchical_b200 import _lib
from log_linear_hierarchical_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "llsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(llsa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from log_linear_hierarchical_b200 import build
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert "llsa_forward" in names and "llsa_backward" in names
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(_lib.SIGNATURES), "binding and header declare different functions"


def shape(**kw):
    base = dict(B=1, H=6, N=65536, D=64, topk=8, levels=3, dtype=0)
    base.update(kw)
    return api.make_shape(base["B"], base["H"], base["N"], base["D"], base["topk"], base["levels"],
                          base["dtype"], block=base.get("block", 16))


@pytest.mark.parametrize("kw,status", [
    ({}, 0),
    (dict(levels=1, N=1024, topk=8, dtype=1, H=2), 0),
    (dict(N=3000), 1),                 # not a multiple of 16^L
    (dict(N=3840), 1),                 # 15 * 256: not a multiple of 16^3
    (dict(N=61440), 0),                # 15 * 4096: n_L = 15
    (dict(N=12 * 4096), 0),            # a multiple of 16^L that is not a power of two: n_L = 12
    (dict(levels=1, N=16 * 65, topk=5), 0),   # n_1 = 65, K = 5
    (dict(topk=6), 0),                 # K need not be a power of two
    (dict(topk=17), 1),                # topk > n_L = 16
    (dict(topk=32), 1),                # topk > n_L = 16
    (dict(N=2048), 1),                 # N < 16^L
    (dict(B=0), 1),
    (dict(dtype=7), 1),
    (dict(D=128), 0),                  # D = 128 is built
    (dict(D=96), 2),                   # other head widths: legal, not built
    (dict(block=32), 2),
    (dict(levels=5, N=1 << 20, topk=1), 2),
    (dict(N=1 << 21), 2),
    (dict(levels=3, N=262144, topk=16), 0),
    (dict(levels=3, N=1 << 20, topk=32), 2),   # (L-1) K = 64 coarse entries: above the 32 built
])
def test_validation(lib, kw, status):
    assert api.llsa_validate_shape(shape(**kw)) == status


@pytest.mark.parametrize("B,H,N,K,L", [(2, 3, 12288, 6, 2), (1, 2, 1040, 5, 1), (1, 1, 61440, 12, 3)])
def test_sizes_match_layout_at_general_shapes(lib, B, H, N, K, L):
    # n_l = N / 16^l need not be powers of two, nor K
    s = api.make_shape(B, H, N, 64, K, L, 0)
    assert api.llsa_validate_shape(s) == 0
    n = [N // 16 ** l for l in range(1, L + 1)]
    assert api.llsa_pyramid_elems(s) == B * H * 64 * sum(n)
    assert api.llsa_index_elems(s) == B * H * K * sum(n)
    assert api.llsa_row_ptr_elems(s) == B * H * sum(x + 1 for x in n)
    assert api.llsa_transpose_workspace_bytes(s) >= 4 * B * H * K * sum(n)
    assert api.llsa_backward_workspace_bytes(s) >= 4 * B * H * N


def test_sizes_match_layout(lib):
    s = shape()
    n = [4096, 256, 16]
    assert api.llsa_pyramid_elems(s) == 6 * 64 * sum(n)
    assert api.llsa_index_elems(s) == 6 * 8 * sum(n)
    assert api.llsa_row_ptr_elems(s) == 6 * sum(x + 1 for x in n)
    assert api.llsa_transpose_workspace_bytes(s) >= 4 * 6 * 8 * sum(n)
    # delta + partials + coarse grads
    assert api.llsa_backward_workspace_bytes(s) >= 4 * (6 * 65536 + 2 * 6 * 256 * 16 * 64 + 2 * 6 * (256 + 16) * 64)
    bad = shape(N=3000)
    assert api.llsa_pyramid_elems(bad) == 0 and api.llsa_backward_workspace_bytes(bad) == 0


def test_null_and_misaligned_pointers_rejected_before_launch(lib):
    s = shape()
    null = None
    assert lib.llsa_build_pyramid(ctypes.byref(s), null, null, null, null, null, null, null) == 1
    assert lib.llsa_select(ctypes.byref(s), 16, 32, 49, null) == 1    # idx misaligned
    assert lib.llsa_forward(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 17, 16, null) == 1   # o misaligned
    ws = api.llsa_transpose_workspace_bytes(s)
    assert lib.llsa_index_transpose(ctypes.byref(s), 16, 16, 16, 16, ws - 1, null) == 3  # workspace too small
    assert lib.llsa_status_string(3).decode() == "workspace too small"


def test_status_error_message(lib):
    err = api.LLSAError("llsa_select", 2)
    assert "LLSA_ERR_UNSUPPORTED" in str(err)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(_lib.LLSAExtensionMissing):
        _lib.load(str(tmp_path / "nope.so"))


def test_step_and_plan_rejected_before_launch(lib):
    """llsa_train_step and llsa_plan_create check every buffer before any CUDA call."""
    s = shape()
    empty = _lib.LLSAStepBuffers()
    assert lib.llsa_train_step(ctypes.byref(s), ctypes.byref(empty), None, None) == 1
    assert lib.llsa_train_step(ctypes.byref(s), None, None, None) == 1
    ptrs = {n: 256 for n, _ in _lib.LLSAStepBuffers._fields_ if not n.endswith("_bytes")}
    small_ws = _lib.LLSAStepBuffers(**ptrs, transpose_workspace_bytes=api.llsa_transpose_workspace_bytes(s) - 1,
                                    backward_workspace_bytes=api.llsa_backward_workspace_bytes(s))
    assert lib.llsa_train_step(ctypes.byref(s), ctypes.byref(small_ws), None, None) == 3
    misaligned = _lib.LLSAStepBuffers(**dict(ptrs, lse=260), transpose_workspace_bytes=1 << 30,
                                      backward_workspace_bytes=1 << 30)
    assert lib.llsa_train_step(ctypes.byref(s), ctypes.byref(misaligned), None, None) == 1
    handle = ctypes.c_void_p(1234)
    assert lib.llsa_plan_create(ctypes.byref(s), ctypes.byref(small_ws), 1, ctypes.byref(handle)) == 3
    assert not handle.value
    assert lib.llsa_plan_create(ctypes.byref(s), ctypes.byref(small_ws), 0, ctypes.byref(handle)) == 1
    assert lib.llsa_plan_create(ctypes.byref(s), ctypes.byref(small_ws), 1, None) == 1
    assert lib.llsa_plan_launch(None, None) == 1
    lib.llsa_plan_destroy(None)


def test_flags_validated(lib):
    s = shape()
    # any combination of LOG_BIAS (1), ALL_TOP (2), LEVEL1 (4), GRID_ORDER (8), ONE_LAUNCH_SELECT (16);
    # CAUSAL (32) has its own rules below
    for good in range(1, 32):
        s.flags = good
        assert lib.llsa_validate_shape(ctypes.byref(s)) == 0, good
    for bad in (64, 128, 1 << 30, -1):
        s.flags = bad
        assert lib.llsa_validate_shape(ctypes.byref(s)) == 1, bad


def test_causal_rules(lib):
    causal = _lib.LLSA_FLAG_CAUSAL
    s = shape()
    for ok in (causal, causal | _lib.LLSA_FLAG_ONE_LAUNCH_SELECT):
        s.flags = ok
        assert lib.llsa_validate_shape(ctypes.byref(s)) == 0, ok
    for other in (_lib.LLSA_FLAG_LOG_BIAS, _lib.LLSA_FLAG_ALL_TOP, _lib.LLSA_FLAG_LEVEL1, _lib.LLSA_FLAG_GRID_ORDER):
        s.flags = causal | other
        assert lib.llsa_validate_shape(ctypes.byref(s)) == 2, other     # UNSUPPORTED
    f32 = shape(dtype=1)
    f32.flags = causal
    assert lib.llsa_validate_shape(ctypes.byref(f32)) == 2
    padded = api.make_shape(1, 2, 4096, 64, 4, 2, 0, n_valid=3000, causal=True)
    assert lib.llsa_validate_shape(ctypes.byref(padded)) == 2
    assert api.make_shape(1, 2, 4096, 64, 4, 2, 0, causal=True).flags == causal == 32
    assert _lib.LLSA_NO_PICK == 2 ** 31 - 1
    assert api.make_shape(1, 6, 65536, 64, 8, 3, 0, log_bias=True).flags == _lib.LLSA_FLAG_LOG_BIAS
    assert api.make_shape(1, 6, 65536, 64, 8, 3, 0, log_bias=True, all_top=True).flags == 3
    assert api.make_shape(1, 6, 65536, 64, 8, 3, 0, level1=True).flags == _lib.LLSA_FLAG_LEVEL1 == 4


def test_all_top_coarse_limit(lib):
    # C = (L-2) K + n_L coarse entries; more than 96 is unsupported
    cases = [((262144, 3, 16), 0),    # C = 16 + 64
             ((16384, 2, 8), 0),      # C = 64
             ((65536, 2, 8), 2),      # C = 256
             ((1 << 20, 3, 16), 2),   # C = 16 + 256
             ((1 << 20, 4, 8), 0),    # C = 16 + 16
             ((4096, 1, 8), 0)]       # L = 1: no coarse entries
    for (N, L, K), want in cases:
        s = api.make_shape(1, 1, N, 64, K, L, 0, all_top=True)
        assert lib.llsa_validate_shape(ctypes.byref(s)) == want, (N, L, K)
        s.flags = 0
        assert lib.llsa_validate_shape(ctypes.byref(s)) == 0, (N, L, K)


def test_token_permute_rejected_before_launch(lib):
    s = shape(levels=1, N=2048, topk=8)   # 2048 is not a square grid
    assert lib.llsa_token_permute(ctypes.byref(s), 256, 512, 1, None) == 1
    s = shape(levels=1, N=4096, topk=8)
    assert lib.llsa_token_permute(ctypes.byref(s), 256, 256, 1, None) == 1   # in place
    assert lib.llsa_token_permute(ctypes.byref(s), None, 256, 0, None) == 1
    assert lib.llsa_token_permute(ctypes.byref(s), 264, 512, 0, None) == 1   # misaligned


def test_variant_flags_change_only_the_backward_workspace(lib):
    base = api.make_shape(1, 6, 65536, 64, 8, 3, 0)
    for kw in (dict(log_bias=True), dict(level1=True), dict(all_top=True), dict(all_top=True, level1=True)):
        s = api.make_shape(1, 6, 65536, 64, 8, 3, 0, **kw)
        for fn in (api.llsa_pyramid_elems, api.llsa_index_elems, api.llsa_row_ptr_elems,
                   api.llsa_transpose_workspace_bytes):
            assert fn(s) == fn(base), (kw, fn.__name__)
        ws, ws0 = api.llsa_backward_workspace_bytes(s), api.llsa_backward_workspace_bytes(base)
        if kw.get("all_top"):
            # coarse partials [B*H*n_2][C][64] for dK and dV: C goes from (L-1) K = 16 to
            # (L-2) K + n_L = 24
            assert ws - ws0 >= 2 * 4 * 6 * 256 * (24 - 16) * 64
        else:
            assert ws == ws0
    one = api.make_shape(1, 2, 4096, 64, 8, 1, 0)
    assert api.llsa_backward_workspace_bytes(api.make_shape(1, 2, 4096, 64, 8, 1, 0, all_top=True)) == \
        api.llsa_backward_workspace_bytes(one)   # L = 1: no coarse entries either way


def test_binding_refuses_tensors_the_kernels_would_misread():
    # wrong dtype, wrong size or host memory is refused before anything is launched
    B, H, N, K, L = 1, 2, 4096, 4, 2
    shape = api.make_shape(B, H, N, 64, K, L, torch.bfloat16)
    act = lambda dt=torch.bfloat16, n=B * H * N * 64: torch.zeros(n, dtype=dt)  # noqa: E731
    pyr = torch.zeros(api.llsa_pyramid_elems(shape), dtype=torch.float32)
    idx = torch.zeros(api.llsa_index_elems(shape), dtype=torch.int32)
    lse = torch.zeros(B * H * N, dtype=torch.float32)
    cases = [
        (dict(q=act(torch.float32)), "q: dtype"),            # fp32 under a bf16 shape
        (dict(k=act(n=B * H * N * 64 - 64)), "k: "),          # one token short
        (dict(idx=idx.float()), "idx: dtype"),
        (dict(k_pyr=pyr[:-1]), "k_pyr: "),                    # pyramid too small
        (dict(lse=lse[: B * H * N // 2]), "lse: "),
        ({}, "CUDA"),                                         # everything right but on the host
    ]
    for override, msg in cases:
        args = dict(q=act(), k=act(), v=act(), k_pyr=pyr, v_pyr=pyr, idx=idx, o=act(), lse=lse)
        args.update(override)
        with pytest.raises(ValueError, match=msg):
            api.llsa_forward(shape, **args)
    with pytest.raises(ValueError, match="dst: dtype"):
        api.llsa_token_permute(shape, act(), act(torch.float32))


@pytest.mark.parametrize("limit", [0, -5, 4_000_000_001])
def test_bounded_wait_check_rejects_limits_outside_range(lib, limit):
    assert lib.llsa_check_bounded_wait(limit, None) == 1   # LLSA_ERR_INVALID_ARG, nothing launched


def test_buffer_sizes_scale_with_head_width(lib):
    s64 = api.make_shape(1, 6, 65536, 64, 8, 3, 0)
    s128 = api.make_shape(1, 6, 65536, 128, 8, 3, 0)
    assert api.llsa_pyramid_elems(s128) == 2 * api.llsa_pyramid_elems(s64) == 2 * 6 * (4096 + 256 + 16) * 64
    assert api.llsa_index_elems(s128) == api.llsa_index_elems(s64)
    assert api.llsa_transpose_workspace_bytes(s128) == api.llsa_transpose_workspace_bytes(s64)
    # Delta and the dK/dV order do not grow with D; the coarse partials and gradients double
    assert api.llsa_backward_workspace_bytes(s128) > api.llsa_backward_workspace_bytes(s64)


def test_grid_order_workspace_holds_the_step_copies(lib):
    # bf16 under grid order: room for quadtree-ordered q, k, v, dO (bf16) and LSE (fp32)
    B, H, N, D = 1, 6, 65536, 64
    plain = api.llsa_backward_workspace_bytes(api.make_shape(B, H, N, D, 8, 3, 0))
    grid = api.llsa_backward_workspace_bytes(api.make_shape(B, H, N, D, 8, 3, 0, grid_order=True))
    copies = 4 * B * H * N * D * 2 + B * H * N * 4
    assert copies <= grid - plain < copies + 256
    f32 = api.llsa_backward_workspace_bytes(api.make_shape(B, H, N, D, 8, 3, 1, grid_order=True))
    assert f32 == api.llsa_backward_workspace_bytes(api.make_shape(B, H, N, D, 8, 3, 1))


def test_grid_order_and_padding_rules(lib):
    grid = _lib.LLSA_FLAG_GRID_ORDER
    ok = api.make_shape(1, 2, 4096, 64, 4, 2, 0, grid_order=True)
    assert lib.llsa_validate_shape(ctypes.byref(ok)) == 0
    assert lib.llsa_validate_shape(ctypes.byref(api.make_shape(1, 2, 12288, 64, 4, 2, 0, grid_order=True))) == 1
    assert lib.llsa_validate_shape(ctypes.byref(api.make_shape(1, 2, 8192, 64, 4, 2, 0, grid_order=True))) == 1
    assert lib.llsa_validate_shape(ctypes.byref(api.make_shape(1, 2, 64, 64, 2, 1, 0, grid_order=True))) == 2
    padded = api.make_shape(1, 2, 4096, 64, 4, 2, 0, n_valid=3000)
    assert lib.llsa_validate_shape(ctypes.byref(padded)) == 0
    padded.flags = grid
    assert lib.llsa_validate_shape(ctypes.byref(padded)) == 2        # padding takes no variant flag
    padded.flags = _lib.LLSA_FLAG_ONE_LAUNCH_SELECT                  # only the launch-shape one
    assert lib.llsa_validate_shape(ctypes.byref(padded)) == 0
    assert api.make_shape(1, 2, 4096, 64, 4, 2, 0, one_launch_select=True).flags == 16
    assert lib.llsa_validate_shape(ctypes.byref(api.make_shape(1, 2, 4096, 64, 13, 2, 0, n_valid=2900))) == 1
    assert lib.llsa_validate_shape(ctypes.byref(api.make_shape(1, 2, 4096, 64, 4, 2, 0, n_valid=5000))) == 1
    assert lib.llsa_validate_shape(ctypes.byref(api.make_shape(1, 2, 4096, 64, 4, 2, 0, n_valid=-1))) == 1
