"""Pins for the oracle's sparse index transpose (CPU): the dense-mask transpose on
small inputs and the CSR invariants."""
import numpy as np
import pytest

from oracle.llsa_oracle import index_transpose, index_transpose_all


def random_lists(rng, n_q, n_k, K):
    return np.stack([np.sort(rng.choice(n_k, size=K, replace=False)) for _ in range(n_q)]).astype(np.int32)


def dense_mask_transpose(idx, n_k):
    """Build the n_q x n_k boolean mask, transpose it, and read the rows off."""
    n_q = idx.shape[0]
    mask = np.zeros((n_q, n_k), dtype=bool)
    for a in range(n_q):
        mask[a, idx[a]] = True
    mt = mask.T
    row_ptr = [0]
    col = []
    for j in range(n_k):
        qs = np.nonzero(mt[j])[0]
        col.extend(qs.tolist())
        row_ptr.append(row_ptr[-1] + len(qs))
    return np.array(row_ptr, dtype=np.int32), np.array(col, dtype=np.int32)


@pytest.mark.parametrize("n,K", [(16, 1), (16, 4), (64, 8), (256, 16), (64, 64), (48, 3), (80, 6)])
def test_equals_dense_mask_transpose(n, K):
    rng = np.random.default_rng(n * 100 + K)
    idx = random_lists(rng, n, n, K)
    rp, col = index_transpose(idx, n)
    rp_d, col_d = dense_mask_transpose(idx, n)
    assert np.array_equal(rp, rp_d)
    assert np.array_equal(col, col_d)


def test_skewed_popularity():
    # Every query picks key 0 and key 5; the other keys are never picked.
    n, K = 32, 2
    idx = np.tile(np.array([0, 5], dtype=np.int32), (n, 1))
    rp, col = index_transpose(idx, n)
    assert rp[1] == n and rp[6] == 2 * n and rp[-1] == 2 * n
    assert np.array_equal(col[:n], np.arange(n)) and np.array_equal(col[n:], np.arange(n))
    assert np.all(np.diff(rp[6:]) == 0)


def test_invariants_on_all_levels():
    rng = np.random.default_rng(2)
    idx = [random_lists(rng, 256, 256, 8)[None, None], random_lists(rng, 16, 16, 8)[None, None]]
    rps, cols = index_transpose_all(idx)
    for lv, rp, cl in zip(idx, rps, cols):
        n, K = lv.shape[2], lv.shape[3]
        rp, cl = rp[0, 0], cl[0, 0]
        assert rp[0] == 0 and rp[-1] == n * K
        assert np.all(np.diff(rp) >= 0)
        for j in range(n):
            seg = cl[rp[j]:rp[j + 1]]
            assert np.all(np.diff(seg) > 0)            # strictly ascending queries
            for a in seg:
                assert j in lv[0, 0, a]
        # every (query, key) entry appears exactly once
        assert sorted(zip(np.repeat(np.arange(n + 1)[:-1], np.diff(rp)).tolist(), cl.tolist())) == \
            sorted((int(j), a) for a in range(n) for j in lv[0, 0, a])
