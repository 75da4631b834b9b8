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
