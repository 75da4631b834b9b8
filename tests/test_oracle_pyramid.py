"""Pins for the oracle's pyramid (CPU): closed forms, the rounding order, and the
error bound against the exact mean."""
import numpy as np
import pytest

from oracle.llsa_oracle import build_pyramid, level_sizes


def test_constant_input_is_a_fixed_point():
    x = np.full((1, 2, 4096, 64), 0.375, dtype=np.float32)
    pyr = build_pyramid(x, 3)
    assert [p.shape[2] for p in pyr] == level_sizes(4096, 3)[1:]
    for p in pyr:
        assert p.dtype == np.float32
        assert np.all(p == np.float32(0.375))


def test_ramp_gives_contiguous_block_means():
    # x[t] = t: level-1 token j is the mean of tokens 16j..16j+15 = 16j + 7.5, and
    # level-2 token j the mean of 256j..256j+255 = 256j + 127.5 (all exact in fp32).
    # A strided grouping (token j + n/16 * r) would give other values.
    N = 4096
    t = np.arange(N, dtype=np.float32)
    x = np.broadcast_to(t[None, None, :, None], (1, 1, N, 4)).copy()
    l1, l2, l3 = build_pyramid(x, 3)
    j1 = np.arange(N // 16, dtype=np.float64)
    j2 = np.arange(N // 256, dtype=np.float64)
    assert np.array_equal(l1[0, 0, :, 0], (16 * j1 + 7.5).astype(np.float32))
    assert np.array_equal(l2[0, 0, :, 0], (256 * j2 + 127.5).astype(np.float32))
    assert l3[0, 0, 0, 0] == np.float32(2047.5)


def test_sequential_fp32_order_from_zero():
    # The reading fixes the order: ((0 + x0) + x1) + ... + x15, each sum rounded to fp32.
    # With x0 = 2^24 and fifteen 1.0s, every "+1" rounds back to 2^24 (ties to even), so
    # the level-1 value is 2^24 / 16 = 2^20, not the exact mean (2^24 + 15) / 16.
    x = np.ones((1, 1, 16, 1), dtype=np.float32)
    x[0, 0, 0, 0] = 2.0 ** 24
    (l1,) = build_pyramid(x, 1)
    assert l1[0, 0, 0, 0] == np.float32(2.0 ** 20)
    # Putting the big value last adds the fifteen ones exactly first: (15 + 2^24) rounds
    # to 2^24 + 16 (ties to even), and / 16 gives 2^20 + 1.
    y = np.ones((1, 1, 16, 1), dtype=np.float32)
    y[0, 0, 15, 0] = 2.0 ** 24
    (m1,) = build_pyramid(y, 1)
    assert m1[0, 0, 0, 0] == np.float32(2.0 ** 20 + 1)


@pytest.mark.parametrize("levels", [1, 2, 3])
def test_close_to_exact_mean(levels):
    rng = np.random.default_rng(5)
    N = 16 ** levels * 2
    x = rng.standard_normal((2, 3, N, 8)).astype(np.float32)
    pyr = build_pyramid(x, levels)
    maxabs = np.abs(x).max()
    u = 2.0 ** -24
    for lev in range(1, levels + 1):
        span = 16 ** lev
        exact = x.astype(np.float64).reshape(2, 3, N // span, span, 8).mean(axis=3)
        err = np.abs(pyr[lev - 1].astype(np.float64) - exact).max()
        # 16 rounded additions per level, each within u of a partial sum bounded by 16 max|x|
        assert err <= lev * 16 * u * maxabs * 1.01, (lev, err)


def test_fp64_mode_matches_exact_mean():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 1, 4096, 4))
    pyr = build_pyramid(x, 2, acc_dtype=np.float64)
    exact2 = x.reshape(1, 1, 16, 256, 4).mean(axis=3)
    assert np.abs(pyr[1] - exact2).max() < 1e-14
