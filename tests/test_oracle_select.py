"""Pins for the oracle's hierarchical Top-K (CPU): brute-force enumeration of key
sets on tiny inputs, with integer-valued vectors so that scores and ties are exact."""
import itertools

import numpy as np
import pytest

from oracle.llsa_oracle import build_pyramid, check_selection, select


def brute_force_topk(scores, cand, K):
    """Best K-subset by total score; among equal totals the lexicographically smallest
    sorted key tuple.  Enumerates every subset."""
    best_sum, best = None, None
    for sub in itertools.combinations(range(len(cand)), K):
        tot = sum(scores[i] for i in sub)
        keys = tuple(sorted(int(cand[i]) for i in sub))
        if best is None or tot > best_sum or (tot == best_sum and keys < best):
            best_sum, best = tot, keys
    return list(best)


def int_vectors(rng, shape, lo=-2, hi=2):
    return rng.integers(lo, hi + 1, size=shape).astype(np.float32)


@pytest.mark.parametrize("K", [1, 2, 3, 4, 5])   # K need not be a power of two
def test_single_level_equals_brute_force(K):
    rng = np.random.default_rng(100 + K)
    n, D = 16, 8
    q1 = int_vectors(rng, (1, 2, n, D))
    k1 = int_vectors(rng, (1, 2, n, D), -1, 1)   # narrow range: many exact ties
    (idx,) = select([q1], [k1], K)
    ties_seen = 0
    for h in range(2):
        for a in range(n):
            s = (q1[0, h, a].astype(np.int64) @ k1[0, h].astype(np.int64).T).tolist()
            ties_seen += len(s) - len(set(s))
            assert idx[0, h, a].tolist() == brute_force_topk(s, np.arange(n), K)
    assert ties_seen > 0


def test_two_levels_equal_brute_force():
    # N = 4096, L = 2 (16 level-2 tokens, 256 level-1 tokens), K = 2.  The brute force
    # rebuilds each level-1 query's candidates from the level-2 choice of its parent:
    # every level-1 token whose level-2 parent (token // 16) was chosen.
    rng = np.random.default_rng(7)
    K, D = 2, 8
    q1 = int_vectors(rng, (1, 1, 256, D))
    k1 = int_vectors(rng, (1, 1, 256, D))
    q2 = int_vectors(rng, (1, 1, 16, D))
    k2 = int_vectors(rng, (1, 1, 16, D))
    idx1, idx2 = select([q1, q2], [k1, k2], K)
    for a in range(16):
        s = (q2[0, 0, a].astype(np.int64) @ k2[0, 0].astype(np.int64).T).tolist()
        assert idx2[0, 0, a].tolist() == brute_force_topk(s, np.arange(16), K)
    for a in range(256):
        chosen_parents = set(idx2[0, 0, a // 16].tolist())
        cand = np.array([t for t in range(256) if t // 16 in chosen_parents])
        s = (q1[0, 0, a].astype(np.int64) @ k1[0, 0, cand].astype(np.int64).T).tolist()
        assert idx1[0, 0, a].tolist() == brute_force_topk(s, cand, K)


def test_topk_equal_to_level_size_selects_everything():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 3, 64, 16)).astype(np.float32)
    k = rng.standard_normal((2, 3, 64, 16)).astype(np.float32)
    (idx,) = select([q], [k], 64)
    assert np.all(idx == np.arange(64))


def test_selection_ignores_positive_query_scale_and_prefers_aligned_keys():
    rng = np.random.default_rng(11)
    k = rng.standard_normal((1, 1, 32, 16)).astype(np.float32)
    q = k[:, :, ::-1].copy() * 3.0          # query a is 3x key 31 - a
    (idx,) = select([q], [k], 1)
    (idx2,) = select([q * 0.5], [k], 1)
    assert np.array_equal(idx, idx2)
    # Each query's best key by dot product; here pinned by direct argmax of the scores
    s = q[0, 0] @ k[0, 0].T
    assert np.array_equal(idx[0, 0, :, 0], s.argmax(axis=1))


def test_output_rows_ascending_and_distinct():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 2, 4096, 16)).astype(np.float32)
    y = rng.standard_normal((1, 2, 4096, 16)).astype(np.float32)
    idx = select(build_pyramid(x, 2), build_pyramid(y, 2), 4)
    for lv in idx:
        assert lv.dtype == np.int32
        assert np.all(np.diff(lv, axis=-1) > 0)


def test_check_selection_accepts_own_and_rejects_planted_swap():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((1, 1, 4096, 16)).astype(np.float32)
    y = rng.standard_normal((1, 1, 4096, 16)).astype(np.float32)
    qp, kp = build_pyramid(x, 2), build_pyramid(y, 2)
    idx = select(qp, kp, 4)
    res = check_selection(qp, kp, idx, 4)
    assert res["bad"] == 0 and res["exact"] == res["rows"]
    # Replace one selected level-1 key by the worst candidate of the same row.
    bad = [lv.copy() for lv in idx]
    a = 37
    parents = idx[1][0, 0, a // 16]
    cand = (16 * parents[:, None] + np.arange(16)).ravel()
    s = qp[0][0, 0, a].astype(np.float64) @ kp[0][0, 0, cand].astype(np.float64).T
    worst = int(cand[np.argmin(s)])
    row = sorted(set(bad[0][0, 0, a].tolist()[1:]) | {worst})
    bad[0][0, 0, a] = row
    res = check_selection(qp, kp, bad, 4)
    assert res["bad"] == 1


def test_check_selection_tie_window():
    # Two keys whose scores differ by far less than 1e-5 relative: either may be chosen.
    k = np.zeros((1, 1, 4, 2), dtype=np.float32)
    k[0, 0, :, 0] = [1.0, 0.5, np.float32(1.0) + np.float32(2.0 ** -22), -1.0]
    q = np.zeros((1, 1, 4, 2), dtype=np.float32)
    q[0, 0, :, 0] = 1.0
    (idx,) = select([q], [k], 1)
    assert idx[0, 0, 0, 0] == 2
    swapped = idx.copy()
    swapped[0, 0, :, 0] = 0
    res = check_selection([q], [k], [swapped], 1)
    assert res["bad"] == 0 and res["tie_window"] == 4
    worse = idx.copy()
    worse[0, 0, :, 0] = 1
    assert check_selection([q], [k], [worse], 1)["bad"] == 4


def test_rejects_topk_above_coarsest_level_size():
    q = np.zeros((1, 1, 1, 4), dtype=np.float32)
    with pytest.raises(ValueError):
        select([q], [q], 2)


# ----------------------------------------------------------------------------- fp32 error floor
# The selection kernels rank fp32 dot products of the fp32 pyramid rows, so two keys whose
# fp64 scores differ by less than the rounding error of those dot products may come out in
# either order.  The checker therefore accepts an inverted pair when its fp64 gap is below
# the sum of the two scores' fp32 error bounds.  These pins tie that bound to real fp32
# arithmetic (it must cover what an fp32 summation actually does) and keep it from being
# loose (a swap well beyond it must fail), with each pair judged on its own bound.

D64 = 64
BIG = np.float32(2.0 ** 24)


def _cancelling_key(small):
    """[2^24, small x 62, -2^24]: the fp64 dot with a ones query is 62 * small, while an fp32
    running sum starting at 2^24 rounds every small term (below one ulp) away."""
    k = np.full(D64, np.float32(small), dtype=np.float32)
    k[0], k[-1] = BIG, -BIG
    return k


def _fp32_sequential_dot(q, k):
    acc = np.float32(0.0)
    for a, b in zip(q.astype(np.float32), k.astype(np.float32)):
        acc = np.float32(acc + np.float32(a * b))
    return float(acc)


def _rows(keys):
    k = np.stack(keys).astype(np.float32)[None, None]          # [1, 1, n, D]
    q = np.ones_like(k)                                          # every query row is all ones
    return q, k


def test_floor_accepts_an_inversion_that_fp32_summation_makes():
    x = _cancelling_key(1.0)                  # fp64 score 62/8 = 7.75; fp32 running sum 0
    y = np.zeros(D64, np.float32)
    y[0] = 0.5                                # score 0.0625 in both precisions
    bad1 = np.full(D64, -1.0, np.float32)
    bad2 = np.full(D64, -2.0, np.float32)
    q, k = _rows([x, y, bad1, bad2])
    fp32 = [_fp32_sequential_dot(q[0, 0, 0], k[0, 0, j]) for j in range(4)]
    assert fp32[0] == 0.0 and fp32[1] == 0.5          # fp32 ranks y above x
    gpu_like = np.full((1, 1, 4, 1), int(np.argmax(fp32)), dtype=np.int32)
    assert gpu_like[0, 0, 0, 0] == 1
    (want,) = select([q], [k], 1)
    assert want[0, 0, 0, 0] == 0                       # fp64 ranks x first
    res = check_selection([q], [k], [gpu_like], 1)
    # the gap (61.5 / 8) is far outside 1e-5 relative, inside the fp32 bound of x (about 16)
    assert res["bad"] == 0 and res["floor_used"] == 4, res


def test_floor_rejects_a_swap_beyond_the_pair_bound():
    w = _cancelling_key(3.0)                  # fp64 score 186 / 8 = 23.25, bound about 16.0
    y = np.zeros(D64, np.float32)
    y[0] = 0.5
    q, k = _rows([w, y, np.full(D64, -1.0, np.float32), np.full(D64, -2.0, np.float32)])
    planted = np.full((1, 1, 4, 1), 1, dtype=np.int32)   # y kept, w rejected: gap 23.19
    assert check_selection([q], [k], [planted], 1)["bad"] == 4


def test_floor_is_judged_per_pair_not_per_row():
    # Key z has a huge sum |q_d k_d| (so a huge fp32 bound) and the lowest score; the planted
    # swap is between a and b, whose own bounds are tiny.  A row-wide bound would hide it.
    a = np.zeros(D64, np.float32)
    a[0] = 1.0
    b = np.zeros(D64, np.float32)
    b[0] = 0.999
    z = np.zeros(D64, np.float32)
    z[0], z[1], z[2] = 2.0 ** 30, -(2.0 ** 30), -1.0
    q, k = _rows([a, b, z, np.full(D64, -3.0, np.float32)])
    planted = np.full((1, 1, 4, 1), 1, dtype=np.int32)   # b instead of a: gap 1.25e-4
    assert check_selection([q], [k], [planted], 1)["bad"] == 4
    honest = np.full((1, 1, 4, 1), 0, dtype=np.int32)
    assert check_selection([q], [k], [honest], 1)["exact"] == 4


def test_floor_covers_fp32_summation_orders_and_is_not_loose():
    # Cancellation-heavy rows: the realised fp32 error of several summation orders (running
    # sum, reversed, pairwise tree, fused multiply-add chain emulated exactly) never exceeds
    # the bound, and the worst case is not far below it (a bound 8x too large, as with a
    # dropped 1/sqrt(D), would put every ratio under 0.015).
    from oracle.llsa_oracle import dot_error_floor
    rng = np.random.default_rng(2024)
    worst = 0.0
    for trial in range(300):
        big = np.float32(2.0 ** rng.integers(8, 30))
        k = (rng.standard_normal(D64) * rng.choice([1e-3, 1.0, 50.0])).astype(np.float32)
        k[rng.integers(0, D64)] += big
        k[rng.integers(0, D64)] -= big
        q = rng.choice([1.0, -1.0], D64).astype(np.float32) * np.float32(rng.uniform(0.5, 2.0))
        exact = float(q.astype(np.float64) @ k.astype(np.float64)) / 8.0
        bound = float(dot_error_floor(q[None], k[None])[0, 0])
        prods = (q * k).astype(np.float32)                      # each product rounded once
        orders = [prods, prods[::-1]]
        sums = [float(np.float32(np.cumsum(o, dtype=np.float32)[-1])) for o in orders]
        tree = prods.copy()
        while tree.size > 1:
            tree = (tree[0::2] + tree[1::2]).astype(np.float32)
        sums.append(float(tree[0]))
        acc = np.float64(0.0)                                   # fma: product exact, one rounding
        for a, b in zip(q.astype(np.float64), k.astype(np.float64)):
            acc = np.float64(np.float32(acc + a * b))
        sums.append(float(acc))
        for s in sums:
            err = abs(s / 8.0 - exact)
            assert err <= bound, (trial, err, bound)
            worst = max(worst, err / bound)
    assert worst > 0.05, worst
