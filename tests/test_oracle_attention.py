"""Pins for the oracle's block-sparse attention forward and backward (CPU).

The references here are independent of the oracle's gather formulation: torch's
``scaled_dot_product_attention`` (fp64, with and without a dense boolean mask) and its
autograd, fp64 central finite differences, and closed-form invariants.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.llsa_oracle import backward, build_pyramid, forward, select


def rand(rng, *shape):
    return rng.standard_normal(shape)


def sdpa64(q, k, v, mask=None):
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, dropout_p=0.0, is_causal=False)


def full_idx(B, H, n_q, n_k):
    return np.broadcast_to(np.arange(n_k, dtype=np.int32), (B, H, n_q, n_k)).copy()


@pytest.mark.parametrize("N,D", [(256, 16), (768, 16), (256, 128)])   # 768: n_1 = 48; D = 128 for wider heads
def test_single_level_all_blocks_is_dense_attention(N, D):
    rng = np.random.default_rng(0)
    B, H = 1, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    kp, vp = build_pyramid(k, 1, np.float64), build_pyramid(v, 1, np.float64)
    idx = [full_idx(B, H, N // 16, N // 16)]
    o, lse = forward(q, k, v, kp, vp, idx)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    to = sdpa64(tq, tk, tv)
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    lse_ref = torch.logsumexp(tq @ tk.transpose(-1, -2) / math.sqrt(D), dim=-1)
    assert np.abs(lse - lse_ref.detach().numpy()).max() < 1e-12
    to.backward(torch.tensor(do))
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx)
    assert np.abs(dq - tq.grad.numpy()).max() < 1e-11
    assert np.abs(dk - tk.grad.numpy()).max() < 1e-11
    assert np.abs(dv - tv.grad.numpy()).max() < 1e-11


def test_two_levels_all_tokens_is_dense_attention_over_input_and_level2():
    # With every fine block and every level-2 token in each list, LLSA is dense
    # attention over [K ; mean-pool_256(K)] and [V ; mean-pool_256(V)]; autograd through
    # the pool gives the input-token gradient of the coarse entries.
    rng = np.random.default_rng(1)
    B, H, N, D = 1, 1, 1024, 8
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    kp, vp = build_pyramid(k, 2, np.float64), build_pyramid(v, 2, np.float64)
    idx = [full_idx(B, H, N // 16, N // 16), full_idx(B, H, N // 256, N // 256)]
    o, lse = forward(q, k, v, kp, vp, idx)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    pool = lambda x: x.reshape(B, H, N // 256, 256, D).mean(dim=3)
    kk = torch.cat([tk, pool(tk)], dim=2)
    vv = torch.cat([tv, pool(tv)], dim=2)
    to = sdpa64(tq, kk, vv)
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    to.backward(torch.tensor(do))
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx)
    assert np.abs(dq - tq.grad.numpy()).max() < 1e-11
    assert np.abs(dk - tk.grad.numpy()).max() < 1e-11
    assert np.abs(dv - tv.grad.numpy()).max() < 1e-11


def dense_mask(N, idx):
    """Boolean [B, H, N, N + sum_l n_l] mask over [input tokens ; level 2 ; ... ; level L],
    built per query token i from the definition: the tokens of the level-1 blocks chosen
    for i's block, and the level-l tokens chosen for the level-l token covering i (i // 16^l)."""
    L = len(idx)
    B, H = idx[0].shape[:2]
    sizes = [N // 16 ** lev for lev in range(2, L + 1)]
    cols = N + sum(sizes)
    m = np.zeros((B, H, N, cols), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                for blk in idx[0][b, h, i // 16]:
                    m[b, h, i, 16 * blk:16 * blk + 16] = True
                off = N
                for lev in range(2, L + 1):
                    m[b, h, i, off + idx[lev - 1][b, h, i // 16 ** lev]] = True
                    off += N // 16 ** lev
    return m


def test_three_levels_equals_masked_dense_attention():
    rng = np.random.default_rng(2)
    B, H, N, D, K = 1, 2, 8192, 8, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    qp = build_pyramid(q, 3, np.float64)
    kp, vp = build_pyramid(k, 3, np.float64), build_pyramid(v, 3, np.float64)
    idx = select(qp, kp, K)
    o, lse = forward(q, k, v, kp, vp, idx)
    mask = torch.tensor(dense_mask(N, idx))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    kk = torch.cat([tk] + [tk.reshape(B, H, N // 16 ** l, 16 ** l, D).mean(3) for l in (2, 3)], dim=2)
    vv = torch.cat([tv] + [tv.reshape(B, H, N // 16 ** l, 16 ** l, D).mean(3) for l in (2, 3)], dim=2)
    to = sdpa64(tq, kk, vv, mask)
    assert np.abs(o - to.detach().numpy()).max() < 1e-12
    to.backward(torch.tensor(do))
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx)
    assert np.abs(dq - tq.grad.numpy()).max() < 1e-11
    assert np.abs(dk - tk.grad.numpy()).max() < 1e-11
    assert np.abs(dv - tv.grad.numpy()).max() < 1e-11


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(3)
    B, H, N, D = 1, 1, 4096, 8
    q, k = rand(rng, B, H, N, D), rand(rng, B, H, N, D)
    v = np.full((B, H, N, D), 2.5)
    qp, kp, vp = (build_pyramid(x, 2) for x in (q, k, v))
    idx = select(qp, kp, 4)
    o, _ = forward(q, k, v, kp, vp, idx)
    assert np.abs(o - 2.5).max() < 1e-13


def test_finite_differences_with_frozen_selection():
    rng = np.random.default_rng(4)
    B, H, N, D, K, L = 1, 1, 8192, 4, 2, 3
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    qp = build_pyramid(q, L, np.float64)
    idx = select(qp, build_pyramid(k, L, np.float64), K)

    def loss(q_, k_, v_):
        kp, vp = build_pyramid(k_, L, np.float64), build_pyramid(v_, L, np.float64)
        o, _ = forward(q_, k_, v_, kp, vp, idx)
        return float((o * do).sum())

    kp, vp = build_pyramid(k, L, np.float64), build_pyramid(v, L, np.float64)
    o, lse = forward(q, k, v, kp, vp, idx)
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx)
    eps = 1e-6
    picks = [(0, 0, 5, 1), (0, 0, 1000, 3), (0, 0, 8191, 0), (0, 0, 6222, 2)]
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for pos in picks:
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][pos] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][pos] -= 2 * eps
            dn = loss(args["q"], args["k"], args["v"])
            fd = (up - dn) / (2 * eps)
            assert abs(fd - grad[pos]) < 1e-7 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_gradient_sum_invariants():
    rng = np.random.default_rng(5)
    B, H, N, D = 1, 2, 4096, 8
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    qp, kp, vp = (build_pyramid(x, 2, np.float64) for x in (q, k, v))
    idx = select(qp, kp, 4)
    o, lse = forward(q, k, v, kp, vp, idx)
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx)
    # Rows of P sum to one and the pool adjoint keeps sums: sum_t dV_t = sum_i dO_i.
    assert np.abs(dv.sum(axis=2) - do.sum(axis=2)).max() < 1e-10
    # Each row of dS sums to zero, so the K gradients cancel in total.
    assert np.abs(dk.sum(axis=2)).max() < 1e-10


@pytest.mark.parametrize("seed", [6, 7])
def test_list_order_does_not_matter(seed):
    # Reordering a block's fine list (keeping it a set) must not change O beyond rounding.
    rng = np.random.default_rng(seed)
    B, H, N, D = 1, 1, 1024, 8
    q, k, v = (rand(rng, B, H, N, D) for _ in range(3))
    qp, kp, vp = (build_pyramid(x, 2, np.float64) for x in (q, k, v))
    idx = select(qp, kp, 4)
    o1, l1 = forward(q, k, v, kp, vp, idx)
    rev = [idx[0][..., ::-1].copy(), idx[1]]
    o2, l2 = forward(q, k, v, kp, vp, rev)
    assert np.abs(o1 - o2).max() < 1e-13 and np.abs(l1 - l2).max() < 1e-13


def test_block_subset_matches_full_run():
    rng = np.random.default_rng(8)
    B, H, N, D = 1, 2, 4096, 8
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    qp, kp, vp = (build_pyramid(x, 2) for x in (q, k, v))
    idx = select(qp, kp, 4)
    o, lse = forward(q, k, v, kp, vp, idx)
    blocks = np.array([0, 17, 18, 255])
    o2, l2 = forward(q, k, v, kp, vp, idx, blocks=blocks)
    rows = (16 * blocks[:, None] + np.arange(16)).ravel()
    assert np.abs(o2[:, :, rows] - o[:, :, rows]).max() < 1e-13
    assert np.isnan(o2[:, :, 16]).all()
    dq, dk, dv = backward(q, k, v, o, lse, do, kp, vp, idx)
    dq2, dk2, dv2 = backward(q, k, v, o, lse, do, kp, vp, idx, blocks=np.arange(N // 16))
    assert np.abs(dq2 - dq).max() < 1e-13 and np.abs(dk2 - dk).max() < 1e-13 and np.abs(dv2 - dv).max() < 1e-13
