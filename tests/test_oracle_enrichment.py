"""Pins for the oracle's log-count enrichment variant (``log_bias``), on CPU.

The variant adds ln(16^l) to the scaled score of every level-l coarse token.  The pin does
not restate that formula: when every key and value inside each coarsest-level group is the
same vector, a level-l pooled token equals each of the 16^l input tokens it averages, so
attention over the biased list must equal plain softmax attention (torch, fp64) over the
explicit multiset in which each coarse token is repeated 16^l times.  Finite differences
check the backward with the bias on.

The all-coarsest variant (``all_top``) is pinned three ways: with K = n_L the level-L
selection is already every coarsest token, so the variant must change nothing; with the
bias and grouped K/V its level-L part stands for every input token, so the result is
dense attention over the whole sequence plus the finer picks; finite differences and the
sum invariants (sum dV = sum dO, sum dK = 0) check its backward.

The level-1 variant (``level1``: each selected block's pooled token joins the list) is
pinned by dense attention over the tokens and the block means when every block is
selected (L = 1, K = n_1), by the multiset in which, with the bias, each selected block
counts twice, and by finite differences and the sum invariants, alone and with both other
variants.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.llsa_oracle import (BLOCK, backward, build_pyramid, forward, kv_index, kv_sources, llsa_step,
                                 select)


def grouped(rng, B, H, N, D, group):
    """[B, H, N, D] with all tokens inside each run of `group` tokens equal."""
    g = rng.standard_normal((B, H, N // group, D))
    return np.repeat(g, group, axis=2)


@pytest.mark.parametrize("N,L,K", [(4096, 2, 2), (8192, 3, 2)])
def test_log_bias_equals_attention_over_repeated_coarse_tokens(N, L, K):
    rng = np.random.default_rng(11)
    B, H, D = 1, 1, 8
    group = BLOCK ** L  # constant over every coarsest-level group, hence over all levels below
    q = rng.standard_normal((B, H, N, D))
    k = grouped(rng, B, H, N, D, group)
    v = grouped(rng, B, H, N, D, group)
    qp, kp, vp = (build_pyramid(x, L, np.float64) for x in (q, k, v))
    idx = select(qp, kp, K)
    o, lse = forward(q, k, v, kp, vp, idx, log_bias=True)
    ksrc, offsets = kv_sources(k, kp)
    vsrc, _ = kv_sources(v, vp)
    n1 = N // BLOCK
    for p in range(0, n1, max(1, n1 // 16)):
        rows = kv_index(p, (0, 0), idx, offsets)
        reps = np.ones(len(rows), dtype=np.int64)
        for lev in range(2, L + 1):  # the K level-l entries follow the 16K fine ones, levels in order
            start = BLOCK * K + (lev - 2) * K
            reps[start:start + K] = BLOCK ** lev
        km = torch.tensor(np.repeat(ksrc[0, 0][rows], reps, axis=0))[None, None]
        vm = torch.tensor(np.repeat(vsrc[0, 0][rows], reps, axis=0))[None, None]
        qb = torch.tensor(q[0, 0, p * BLOCK:(p + 1) * BLOCK])[None, None]
        ref = F.scaled_dot_product_attention(qb, km, vm)[0, 0].numpy()
        ref_lse = torch.logsumexp(qb @ km.transpose(-1, -2) / math.sqrt(D), dim=-1)[0, 0].numpy()
        assert np.abs(o[0, 0, p * BLOCK:(p + 1) * BLOCK] - ref).max() < 1e-12
        assert np.abs(lse[0, 0, p * BLOCK:(p + 1) * BLOCK] - ref_lse).max() < 1e-11


def test_log_bias_changes_only_coarse_weights():
    # L = 1 has no coarse entries: the variant must be the identity there
    rng = np.random.default_rng(12)
    B, H, N, D = 1, 1, 1024, 8
    q, k, v = (rng.standard_normal((B, H, N, D)) for _ in range(3))
    qp, kp, vp = (build_pyramid(x, 1, np.float64) for x in (q, k, v))
    idx = select(qp, kp, 4)
    a = forward(q, k, v, kp, vp, idx)
    b = forward(q, k, v, kp, vp, idx, log_bias=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_log_bias_finite_differences_with_frozen_selection():
    rng = np.random.default_rng(13)
    B, H, N, D, K, L = 1, 1, 8192, 4, 2, 3
    q, k, v, do = (rng.standard_normal((B, H, N, D)) for _ in range(4))
    idx = select(build_pyramid(q, L, np.float64), build_pyramid(k, L, np.float64), K)

    def loss(q_, k_, v_):
        kp, vp = build_pyramid(k_, L, np.float64), build_pyramid(v_, L, np.float64)
        o, _ = forward(q_, k_, v_, kp, vp, idx, log_bias=True)
        return float((o * do).sum())

    kp, vp = build_pyramid(k, L, np.float64), build_pyramid(v, L, np.float64)
    o, lse = forward(q, k, v, kp, vp, idx, log_bias=True)
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx, log_bias=True)
    eps = 1e-6
    picks = [(0, 0, 7, 1), (0, 0, 2049, 3), (0, 0, 8190, 0), (0, 0, 5000, 2)]
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for pos in picks:
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][pos] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][pos] -= 2 * eps
            dn = loss(args["q"], args["k"], args["v"])
            fd = (up - dn) / (2 * eps)
            assert abs(fd - grad[pos]) < 1e-7 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


# ---------------------------------------------------------------- all-coarsest variant

def test_all_top_equals_default_when_every_coarsest_token_is_selected():
    # K = n_L: the level-L selection is already every coarsest token in index order
    rng = np.random.default_rng(21)
    B, H, N, D, L = 1, 2, 4096, 8, 2
    K = N // BLOCK ** L
    q, k, v, do = (rng.standard_normal((B, H, N, D)) for _ in range(4))
    a = llsa_step(q, k, v, do, L, K)
    b = llsa_step(q, k, v, do, L, K, all_top=True)
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[name], b[name]), name


@pytest.mark.parametrize("N,L,K", [(4096, 2, 2), (16384, 3, 2)])   # n_L = 16, 4 > K
def test_all_top_with_log_bias_is_dense_attention_plus_the_finer_picks(N, L, K):
    # K and V constant over each coarsest-level group: a level-l token stands for 16^l equal
    # input tokens, so with the bias the list is the multiset {selected fine tokens} +
    # {each selected level-l token 16^l times, l < L} + {every input token} (all of level L)
    rng = np.random.default_rng(22)
    B, H, D = 1, 1, 8
    group = BLOCK ** L
    q = rng.standard_normal((B, H, N, D))
    k = grouped(rng, B, H, N, D, group)
    v = grouped(rng, B, H, N, D, group)
    qp, kp, vp = (build_pyramid(x, L, np.float64) for x in (q, k, v))
    idx = select(qp, kp, K)
    o, lse = forward(q, k, v, kp, vp, idx, log_bias=True, all_top=True)
    ksrc, offsets = kv_sources(k, kp)
    vsrc, _ = kv_sources(v, vp)
    for p in range(0, N // BLOCK, max(1, N // BLOCK // 16)):
        fine = kv_index(p, (0, 0), idx, offsets)[:BLOCK * K]
        parts_k, parts_v = [ksrc[0, 0][fine], k[0, 0]], [vsrc[0, 0][fine], v[0, 0]]
        for lev in range(2, L):
            rows = offsets[lev] + idx[lev - 1][0, 0, p // BLOCK ** (lev - 1)]
            parts_k.append(np.repeat(ksrc[0, 0][rows], BLOCK ** lev, axis=0))
            parts_v.append(np.repeat(vsrc[0, 0][rows], BLOCK ** lev, axis=0))
        km = torch.tensor(np.concatenate(parts_k))[None, None]
        vm = torch.tensor(np.concatenate(parts_v))[None, None]
        qb = torch.tensor(q[0, 0, p * BLOCK:(p + 1) * BLOCK])[None, None]
        ref = F.scaled_dot_product_attention(qb, km, vm)[0, 0].numpy()
        ref_lse = torch.logsumexp(qb @ km.transpose(-1, -2) / math.sqrt(D), dim=-1)[0, 0].numpy()
        assert np.abs(o[0, 0, p * BLOCK:(p + 1) * BLOCK] - ref).max() < 1e-12
        assert np.abs(lse[0, 0, p * BLOCK:(p + 1) * BLOCK] - ref_lse).max() < 1e-11


@pytest.mark.parametrize("log_bias", [False, True])
def test_all_top_finite_differences_and_sums(log_bias):
    rng = np.random.default_rng(23)
    B, H, N, D, K, L = 1, 1, 16384, 4, 2, 3   # n_3 = 4 > K: the variant's list differs
    q, k, v, do = (rng.standard_normal((B, H, N, D)) for _ in range(4))
    idx = select(build_pyramid(q, L, np.float64), build_pyramid(k, L, np.float64), K)
    kw = dict(log_bias=log_bias, all_top=True)

    def loss(q_, k_, v_):
        kp, vp = build_pyramid(k_, L, np.float64), build_pyramid(v_, L, np.float64)
        o, _ = forward(q_, k_, v_, kp, vp, idx, **kw)
        return float((o * do).sum())

    kp, vp = build_pyramid(k, L, np.float64), build_pyramid(v, L, np.float64)
    o, lse = forward(q, k, v, kp, vp, idx, **kw)
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx, **kw)
    # rows of P sum to 1 and the pooled adjoint keeps sums: sum dV = sum dO; sum_e dS = 0
    assert np.abs(dv.sum(axis=2) - do.sum(axis=2)).max() < 1e-9
    assert np.abs(dk.sum(axis=2)).max() < 1e-9
    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for pos in [(0, 0, 7, 1), (0, 0, 2049, 3), (0, 0, 16380, 0), (0, 0, 9000, 2)]:
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][pos] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][pos] -= 2 * eps
            dn = loss(args["q"], args["k"], args["v"])
            fd = (up - dn) / (2 * eps)
            assert abs(fd - grad[pos]) < 1e-7 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


# ---------------------------------------------------------------- level-1 pooled tokens

def test_level1_with_every_block_selected_is_dense_attention_over_tokens_and_block_means():
    # L = 1 and K = n_1: every block is selected, so the list is every input token plus
    # every level-1 pooled token: dense attention over the concatenation [K; K^(1)]
    rng = np.random.default_rng(41)
    B, H, N, D = 1, 2, 256, 8
    K = N // BLOCK
    q, k, v = (rng.standard_normal((B, H, N, D)) for _ in range(3))
    out = llsa_step(q, k, v, None, 1, K, level1=True)
    for h in range(H):
        kc = torch.tensor(np.concatenate([k[0, h], out["k_pyr"][0][0, h].astype(np.float64)]))[None, None]
        vc = torch.tensor(np.concatenate([v[0, h], out["v_pyr"][0][0, h].astype(np.float64)]))[None, None]
        qt = torch.tensor(q[0, h])[None, None]
        ref = F.scaled_dot_product_attention(qt, kc, vc)[0, 0].numpy()
        ref_lse = torch.logsumexp(qt @ kc.transpose(-1, -2) / math.sqrt(D), dim=-1)[0, 0].numpy()
        assert np.abs(out["o"][0, h] - ref).max() < 1e-12
        assert np.abs(out["lse"][0, h] - ref_lse).max() < 1e-11


@pytest.mark.parametrize("N,L,K", [(4096, 2, 2), (16384, 3, 2)])
def test_level1_with_log_bias_counts_each_selected_block_twice(N, L, K):
    # K and V constant over each coarsest-level group: a selected block's pooled token equals
    # each of its 16 tokens, so with + ln 16 it weighs as those 16 tokens once more
    rng = np.random.default_rng(42)
    B, H, D = 1, 1, 8
    q = rng.standard_normal((B, H, N, D))
    k = grouped(rng, B, H, N, D, BLOCK ** L)
    v = grouped(rng, B, H, N, D, BLOCK ** L)
    qp, kp, vp = (build_pyramid(x, L, np.float64) for x in (q, k, v))
    idx = select(qp, kp, K)
    o, lse = forward(q, k, v, kp, vp, idx, log_bias=True, level1=True)
    ksrc, offsets = kv_sources(k, kp)
    vsrc, _ = kv_sources(v, vp)
    for p in range(0, N // BLOCK, max(1, N // BLOCK // 16)):
        rows = kv_index(p, (0, 0), idx, offsets)        # the default list
        reps = np.ones(len(rows), dtype=np.int64)
        reps[:BLOCK * K] = 2
        for lev in range(2, L + 1):
            start = BLOCK * K + (lev - 2) * K
            reps[start:start + K] = BLOCK ** lev
        km = torch.tensor(np.repeat(ksrc[0, 0][rows], reps, axis=0))[None, None]
        vm = torch.tensor(np.repeat(vsrc[0, 0][rows], reps, axis=0))[None, None]
        qb = torch.tensor(q[0, 0, p * BLOCK:(p + 1) * BLOCK])[None, None]
        ref = F.scaled_dot_product_attention(qb, km, vm)[0, 0].numpy()
        ref_lse = torch.logsumexp(qb @ km.transpose(-1, -2) / math.sqrt(D), dim=-1)[0, 0].numpy()
        assert np.abs(o[0, 0, p * BLOCK:(p + 1) * BLOCK] - ref).max() < 1e-12
        assert np.abs(lse[0, 0, p * BLOCK:(p + 1) * BLOCK] - ref_lse).max() < 1e-11


@pytest.mark.parametrize("log_bias,all_top", [(False, False), (True, True)])
def test_level1_finite_differences_and_sums(log_bias, all_top):
    rng = np.random.default_rng(43)
    B, H, N, D, K, L = 1, 1, 16384, 4, 2, 3
    q, k, v, do = (rng.standard_normal((B, H, N, D)) for _ in range(4))
    idx = select(build_pyramid(q, L, np.float64), build_pyramid(k, L, np.float64), K)
    kw = dict(log_bias=log_bias, all_top=all_top, level1=True)

    def loss(q_, k_, v_):
        kp, vp = build_pyramid(k_, L, np.float64), build_pyramid(v_, L, np.float64)
        o, _ = forward(q_, k_, v_, kp, vp, idx, **kw)
        return float((o * do).sum())

    kp, vp = build_pyramid(k, L, np.float64), build_pyramid(v, L, np.float64)
    o, lse = forward(q, k, v, kp, vp, idx, **kw)
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx, **kw)
    assert np.abs(dv.sum(axis=2) - do.sum(axis=2)).max() < 1e-9
    assert np.abs(dk.sum(axis=2)).max() < 1e-9
    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for pos in [(0, 0, 7, 1), (0, 0, 2049, 3), (0, 0, 16380, 0), (0, 0, 9000, 2)]:
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][pos] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][pos] -= 2 * eps
            dn = loss(args["q"], args["k"], args["v"])
            fd = (up - dn) / (2 * eps)
            assert abs(fd - grad[pos]) < 1e-7 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])
