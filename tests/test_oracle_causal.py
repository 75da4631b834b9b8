"""Pins for the causal-LLSA oracle (``oracle/llsa_causal.py``), on the CPU.

The references are independent of the oracle's per-block list formulation: torch's
``scaled_dot_product_attention`` with ``is_causal=True`` (fp64) and its autograd; the same
with a dense boolean mask built per query token over every level's tokens; brute-force
enumeration of K-subsets for the selection; the dense-mask transpose; fp64 central finite
differences; and the causality property itself (with the selection fixed, output i does not
change when keys and values after position i change, pyramid included).  Planted oracle
mistakes must fail these pins.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import llsa_causal as oc
from oracle.llsa_oracle import build_pyramid

NP = oc.NO_PICK


def rand(rng, *shape):
    return rng.standard_normal(shape)


def full_causal_idx(B, H, n):
    """Every block j <= p for block p (what K = n_1 selects at one level), NO_PICK-padded."""
    idx = np.full((B, H, n, n), NP, dtype=np.int32)
    for p in range(n):
        idx[:, :, p, :p + 1] = np.arange(p + 1)
    return [idx]


@pytest.mark.parametrize("N,D", [(256, 16), (512, 8)])
def test_one_level_every_past_block_is_sdpa_causal(N, D):
    rng = np.random.default_rng(0)
    B, H = 1, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    kp, vp = build_pyramid(k, 1, np.float64), build_pyramid(v, 1, np.float64)
    idx = full_causal_idx(B, H, N // 16)
    o, lse = oc.forward_causal(q, k, v, kp, vp, idx)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    to = F.scaled_dot_product_attention(tq, tk, tv, dropout_p=0.0, is_causal=True)
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    z = tq @ tk.transpose(-1, -2) / math.sqrt(D)
    z = z.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    assert np.abs(lse - torch.logsumexp(z, dim=-1).detach().numpy()).max() < 1e-12
    to.backward(torch.tensor(do))
    dq, dk, dv = oc.backward_causal(q, k, v, o, lse, do, kp, vp, idx)
    for got, ref in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - ref.grad.numpy()).max() < 1e-11


def test_selection_with_K_at_least_n1_takes_every_past_block():
    rng = np.random.default_rng(1)
    B, H, N, D = 1, 1, 256, 8
    q, k = rand(rng, B, H, N, D), rand(rng, B, H, N, D)
    qp, kp = build_pyramid(q, 1), build_pyramid(k, 1)
    idx = oc.select_causal(qp, kp, 16)
    assert np.array_equal(idx[0], full_causal_idx(B, H, 16)[0])


def brute_force_topk(scores, cand, K):
    """Best K-subset of ``cand`` by score sum, ties to the lexicographically lowest subset
    of positions (that is, lower indices win), padded with NO_PICK."""
    m = min(K, len(cand))
    best, best_key = None, None
    for sub in itertools.combinations(range(len(cand)), m):
        key = (-sum(scores[list(sub)]), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    out = [int(cand[s]) for s in best] + [NP] * (K - m)
    return out


@pytest.mark.parametrize("K", [1, 2, 4])
def test_one_level_selection_is_brute_force_over_past_blocks(K):
    rng = np.random.default_rng(2 + K)
    B, H, N, D = 1, 2, 256, 4
    # small integer vectors: many exact ties, so the tie-break is exercised
    q = rng.integers(-2, 3, (B, H, N, D)).astype(np.float64)
    k = rng.integers(-2, 3, (B, H, N, D)).astype(np.float64)
    qp, kp = build_pyramid(q, 1), build_pyramid(k, 1)
    idx = oc.select_causal(qp, kp, K)[0]
    for b in range(B):
        for h in range(H):
            s_all = qp[0][b, h].astype(np.float64) @ kp[0][b, h].astype(np.float64).T
            for a in range(16):
                cand = np.arange(a + 1)
                assert idx[b, h, a].tolist() == brute_force_topk(s_all[a, cand], cand, K), (b, h, a)


def test_two_level_selection_is_brute_force_under_the_hierarchical_rule():
    rng = np.random.default_rng(7)
    B, H, N, D, K = 1, 1, 4096, 4, 2
    q = rng.integers(-2, 3, (B, H, N, D)).astype(np.float64)
    k = rng.integers(-2, 3, (B, H, N, D)).astype(np.float64)
    qp, kp = build_pyramid(q, 2), build_pyramid(k, 2)
    idx = oc.select_causal(qp, kp, K)
    s2 = qp[1][0, 0].astype(np.float64) @ kp[1][0, 0].astype(np.float64).T
    for a in range(16):
        assert idx[1][0, 0, a].tolist() == brute_force_topk(s2[a, :a + 1], np.arange(a + 1), K)
    s1 = qp[0][0, 0].astype(np.float64) @ kp[0][0, 0].astype(np.float64).T
    for a in range(256):
        parents = [c for c in idx[1][0, 0, a // 16] if c != NP]
        cand = np.array(sorted(16 * c + r for c in parents for r in range(16) if 16 * c + r <= a))
        assert idx[0][0, 0, a].tolist() == brute_force_topk(s1[a, cand], cand, K), a
    # real picks strictly ascending, then only NO_PICK
    for lv in idx:
        real = lv != NP
        assert np.all(real[..., :-1] >= real[..., 1:])
        assert np.all((np.diff(lv.astype(np.int64), axis=-1) > 0) | ~real[..., 1:])


def dense_causal_mask(N, idx):
    """Boolean [B, H, N, N + sum_{l>=2} n_l] over [input tokens ; level 2 ; ... ; level L],
    per query token i from the definition: input token t if its block is in S_1(i // 16)
    and t <= i; level-l token j if j is in S_l(a) for a = i // 16^l (the level-l token
    covering i) and j < a."""
    L = len(idx)
    B, H = idx[0].shape[:2]
    sizes = [N // 16 ** lev for lev in range(2, L + 1)]
    m = np.zeros((B, H, N, N + sum(sizes)), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                for j in idx[0][b, h, i // 16]:
                    if j != NP:
                        for t in range(16 * int(j), 16 * int(j) + 16):
                            m[b, h, i, t] = t <= i
                off = N
                for lev in range(2, L + 1):
                    a = i // 16 ** lev
                    for j in idx[lev - 1][b, h, a]:
                        if j != NP and j < a:
                            m[b, h, i, off + int(j)] = True
                    off += N // 16 ** lev
    return m


def test_three_levels_equal_dense_masked_attention_with_pool_autograd():
    rng = np.random.default_rng(11)
    B, H, N, D, K = 1, 1, 8192, 4, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    qp = build_pyramid(q, 3, np.float64)
    kp, vp = build_pyramid(k, 3, np.float64), build_pyramid(v, 3, np.float64)
    idx = oc.select_causal(qp, kp, K)
    o, lse = oc.forward_causal(q, k, v, kp, vp, idx)
    dq, dk, dv = oc.backward_causal(q, k, v, o, lse, do, kp, vp, idx)
    mask = torch.tensor(dense_causal_mask(N, idx))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    pool = lambda x, s: x.reshape(B, H, N // s, s, D).mean(dim=3)
    kk = torch.cat([tk, pool(tk, 256), pool(tk, 4096)], dim=2)
    vv = torch.cat([tv, pool(tv, 256), pool(tv, 4096)], dim=2)
    to = F.scaled_dot_product_attention(tq, kk, vv, attn_mask=mask, dropout_p=0.0)
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    to.backward(torch.tensor(do))
    for got, ref in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - ref.grad.numpy()).max() < 1e-11


def test_outputs_before_a_position_ignore_keys_and_values_after_it():
    rng = np.random.default_rng(13)
    B, H, N, D, K, L = 1, 2, 4096, 8, 2, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    idx = oc.select_causal(build_pyramid(q, L), build_pyramid(k, L), K)
    kp, vp = build_pyramid(k, L), build_pyramid(v, L)
    o, lse = oc.forward_causal(q, k, v, kp, vp, idx)
    for i0 in (5, 16 * 37 + 9, 2000, 16 * 255 + 15):
        k2, v2 = k.copy(), v.copy()
        k2[:, :, i0 + 1:] = rand(rng, B, H, N - i0 - 1, D)
        v2[:, :, i0 + 1:] = rand(rng, B, H, N - i0 - 1, D)
        o2, lse2 = oc.forward_causal(q, k2, v2, build_pyramid(k2, L), build_pyramid(v2, L), idx)
        assert np.array_equal(o2[:, :, :i0 + 1], o[:, :, :i0 + 1]), i0
        assert np.array_equal(lse2[:, :, :i0 + 1], lse[:, :, :i0 + 1]), i0


def test_finite_differences_with_the_selection_fixed():
    rng = np.random.default_rng(17)
    B, H, N, D, K, L = 1, 1, 512, 4, 2, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    idx = oc.select_causal(build_pyramid(q, L), build_pyramid(k, L), K)

    def loss(q_, k_, v_):
        o_, _ = oc.forward_causal(q_, k_, v_, build_pyramid(k_, L, np.float64), build_pyramid(v_, L, np.float64), idx)
        return float((o_ * do).sum())

    kp, vp = build_pyramid(k, L, np.float64), build_pyramid(v, L, np.float64)
    o, lse = oc.forward_causal(q, k, v, kp, vp, idx)
    grads = oc.backward_causal(q, k, v, o, lse, do, kp, vp, idx)
    eps = 1e-6
    for which, g in zip(range(3), grads):
        for pos in [(0, 0, 3, 1), (0, 0, 200, 0), (0, 0, 300, 3), (0, 0, 511, 2), (0, 0, 17, 2)]:
            args = [q.copy(), k.copy(), v.copy()]
            args[which][pos] += eps
            up = loss(*args)
            args[which][pos] -= 2 * eps
            dn = loss(*args)
            assert abs((up - dn) / (2 * eps) - g[pos]) < 1e-6, (which, pos)


def test_sum_invariants():
    rng = np.random.default_rng(19)
    B, H, N, D, K, L = 1, 1, 4096, 8, 3, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    out = oc.llsa_step_causal(q, k, v, do, L, K)
    assert np.abs(out["dv"].sum(axis=2) - do.sum(axis=2)).max() < 1e-9
    assert np.abs(out["dk"].sum(axis=2)).max() < 1e-9


def test_transpose_drops_no_pick_entries():
    rng = np.random.default_rng(23)
    n, K = 40, 3
    idx = np.full((n, K), NP, dtype=np.int32)
    for a in range(n):
        m = min(K, a + 1)
        idx[a, :m] = np.sort(rng.choice(a + 1, m, replace=False))
    row_ptr, col = oc.index_transpose_causal(idx, n)
    dense = np.zeros((n, n), dtype=bool)
    for a in range(n):
        for j in idx[a]:
            if j != NP:
                dense[a, j] = True
    assert row_ptr[-1] == dense.sum() == np.count_nonzero(idx != NP)
    for j in range(n):
        assert col[row_ptr[j]:row_ptr[j + 1]].tolist() == np.nonzero(dense[:, j])[0].tolist()


def test_planted_mistakes_fail_the_pins(monkeypatch):
    rng = np.random.default_rng(29)
    B, H, N, D = 1, 1, 256, 8
    q, k, v = (rand(rng, B, H, N, D) for _ in range(3))
    kp, vp = build_pyramid(k, 1, np.float64), build_pyramid(v, 1, np.float64)
    idx = full_causal_idx(B, H, N // 16)
    ref = F.scaled_dot_product_attention(*(torch.tensor(a) for a in (q, k, v)), is_causal=True).numpy()
    orig = oc.kv_list_causal

    def strict_diagonal(p, bh, idx_, offsets):   # keys t < i instead of t <= i
        rows, vis = orig(p, bh, idx_, offsets)
        return rows, vis & (rows[None, :] != (16 * p + np.arange(16))[:, None])

    monkeypatch.setattr(oc, "kv_list_causal", strict_diagonal)
    with np.errstate(invalid="ignore"):
        o, _ = oc.forward_causal(q, k, v, kp, vp, idx)
    assert not np.allclose(o, ref, atol=1e-6, equal_nan=False)
    monkeypatch.setattr(oc, "kv_list_causal", orig)

    # attending the block's own level-2 ancestor breaks causality
    N2, L = 4096, 2
    q, k, v = (rand(rng, B, H, N2, D) for _ in range(3))
    idx2 = oc.select_causal(build_pyramid(q, L), build_pyramid(k, L), 2)

    def with_ancestor(p, bh, idx_, offsets):
        rows, vis = orig(p, bh, idx_, offsets)
        anc = p // 16
        return np.concatenate([rows, [offsets[2] + anc]]), np.concatenate([vis, np.ones((16, 1), bool)], axis=1)

    monkeypatch.setattr(oc, "kv_list_causal", with_ancestor)
    o1, _ = oc.forward_causal(q, k, v, build_pyramid(k, L), build_pyramid(v, L), idx2)
    v2 = v.copy()
    v2[:, :, 101:] += 1.0
    o2, _ = oc.forward_causal(q, k, v2, build_pyramid(k, L), build_pyramid(v2, L), idx2)
    assert not np.array_equal(o1[:, :, :101], o2[:, :, :101])
