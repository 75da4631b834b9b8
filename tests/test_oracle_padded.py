"""Pins for the padded-sequence oracle (``oracle/llsa_padded.py``), on CPU.

Nothing here restates the module's formulas: an unpadded sequence must give exactly what the
main oracle gives; with one level and every real block selected the result must be dense
softmax attention (torch SDPA and its autograd, fp64) over the real tokens alone; the
padding's contents must not matter; partial pooled tokens must be fp64 means of their real
tokens; finite differences and the sum invariants check the backward.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import llsa_oracle as orc
from oracle.llsa_padded import (backward_padded, build_pyramid_padded, forward_padded, llsa_step_padded,
                                select_padded, valid_counts)


def rand(rng, *shape):
    return rng.standard_normal(shape)


def test_unpadded_sequence_equals_the_main_oracle():
    rng = np.random.default_rng(71)
    B, H, N, D, K, L = 1, 2, 4096, 8, 2, 2
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    a = orc.llsa_step(q, k, v, do, L, K)
    b = llsa_step_padded(q, k, v, do, L, K, n_valid=N)
    for lev in range(L):
        for name in ("q_pyr", "k_pyr", "v_pyr"):
            assert np.array_equal(a[name][lev].view(np.uint32), b[name][lev].view(np.uint32)), (name, lev)
        assert np.array_equal(a["idx"][lev], b["idx"][lev])
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.abs(a[name] - b[name]).max() < 1e-12, name


@pytest.mark.parametrize("n_valid", [1000, 1009, 1023])
def test_one_level_all_real_blocks_is_dense_attention_over_the_real_tokens(n_valid):
    rng = np.random.default_rng(n_valid)
    B, H, D = 1, 2, 8
    N = 16 * math.ceil(n_valid / 16)
    K = N // 16                               # every block is real here: m_1 = n_1
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    out = llsa_step_padded(q, k, v, do, 1, K, n_valid)
    tq, tk, tv = (torch.tensor(x[:, :, :n_valid], requires_grad=True) for x in (q, k, v))
    ref = F.scaled_dot_product_attention(tq, tk, tv)
    ref.backward(torch.tensor(do[:, :, :n_valid]))
    lse = torch.logsumexp(tq @ tk.transpose(-1, -2) / math.sqrt(D), dim=-1)
    assert np.abs(out["o"][:, :, :n_valid] - ref.detach().numpy()).max() < 1e-12
    assert np.abs(out["lse"][:, :, :n_valid] - lse.detach().numpy()).max() < 1e-12
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        assert np.abs(out[name][:, :, :n_valid] - t.grad.numpy()).max() < 1e-11, name
        assert not out[name][:, :, n_valid:].any(), name   # padding receives nothing
    assert not out["o"][:, :, n_valid:].any()


@pytest.mark.parametrize("n_valid,L,K", [(3000, 2, 4), (1000, 1, 8), (4097, 3, 1)])
def test_padding_contents_do_not_matter(n_valid, L, K):
    rng = np.random.default_rng(72)
    B, H, D = 1, 1, 8
    N = 16 ** L * math.ceil(n_valid / 16 ** L)
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    a = llsa_step_padded(q, k, v, do, L, K, n_valid)
    junk = [x.copy() for x in (q, k, v, do)]
    for x in junk:
        x[:, :, n_valid:] = rng.standard_normal(x[:, :, n_valid:].shape) * 1e3
    b = llsa_step_padded(*junk, L, K, n_valid)
    for lev in range(L):
        assert np.array_equal(a["idx"][lev], b["idx"][lev])
    for name in ("o", "lse", "dq", "dk", "dv"):
        assert np.array_equal(a[name], b[name]), name


def test_partial_pooled_tokens_are_means_of_their_real_tokens():
    rng = np.random.default_rng(73)
    B, H, D, L, n_valid = 1, 2, 8, 2, 3000
    N = 256 * math.ceil(n_valid / 256)
    x = rand(rng, B, H, N, D).astype(np.float32)
    pyr = build_pyramid_padded(x, L, n_valid)
    counts = valid_counts(N, n_valid, L)
    for lev in range(1, L + 1):
        span = 16 ** lev
        for j in range(N // span):
            c = int(counts[lev - 1][j])
            got = pyr[lev - 1][:, :, j].astype(np.float64)
            if c == 0:
                assert not got.any()
                continue
            want = x[:, :, j * span:j * span + c].astype(np.float64).mean(axis=2)
            assert np.abs(got - want).max() < 1e-5 * max(1.0, np.abs(want).max()), (lev, j)
    assert int(counts[0][-1]) == 0 and int(counts[1][-1]) == n_valid - 256 * (N // 256 - 1)


def test_selection_never_picks_empty_tokens():
    rng = np.random.default_rng(74)
    B, H, D, L, K, n_valid = 1, 2, 8, 2, 3, 2600     # m_2 = 11 real level-2 tokens of 12
    N = 256 * math.ceil(n_valid / 256)
    q, k = (rand(rng, B, H, N, D) for _ in range(2))
    qp = build_pyramid_padded(q, L, n_valid)
    kp = build_pyramid_padded(k, L, n_valid)
    idx = select_padded(qp, kp, K, n_valid)
    assert idx[1].max() < 11 and idx[0].max() < math.ceil(n_valid / 16)
    for lev in range(L):                               # lists stay ascending and distinct
        assert np.all(np.diff(idx[lev], axis=-1) > 0)
    with pytest.raises(ValueError):
        select_padded(qp, kp, 12, n_valid)             # more than the 11 real coarsest tokens
    # every real score negative: an empty token (zero mean, score 0) would win if it were a
    # candidate, so this pins that the finer levels drop a partial parent's empty children
    q = np.abs(q) + 0.1
    k = -np.abs(k) - 0.1
    idx = select_padded(build_pyramid_padded(q, L, n_valid), build_pyramid_padded(k, L, n_valid), K, n_valid)
    assert idx[1].max() < 11 and idx[0].max() < math.ceil(n_valid / 16)
    assert (idx[1] == 10).any()                       # the partial level-2 token is picked somewhere


def test_padded_finite_differences_and_sums():
    rng = np.random.default_rng(75)
    B, H, D, L, K, n_valid = 1, 1, 4, 2, 2, 700
    N = 256 * math.ceil(n_valid / 256)
    q, k, v, do = (rand(rng, B, H, N, D) for _ in range(4))
    idx = select_padded(build_pyramid_padded(q, L, n_valid), build_pyramid_padded(k, L, n_valid), K, n_valid)

    def loss(q_, k_, v_):
        kp, vp = build_pyramid_padded(k_, L, n_valid), build_pyramid_padded(v_, L, n_valid)
        o, _ = forward_padded(q_, k_, v_, [x.astype(np.float64) for x in kp], [x.astype(np.float64) for x in vp],
                              idx, n_valid)
        return float((o * do).sum())

    # fp64 pyramids for the finite differences (the fp32 sums would swallow the step)
    def pyr64(x):
        return [p.astype(np.float64) for p in build_pyramid_padded(x, L, n_valid)]

    kp, vp = pyr64(k), pyr64(v)
    o, lse = forward_padded(q, k, v, kp, vp, idx, n_valid)
    dq, dk, dv = backward_padded(q, k, v, o, lse, do, kp, vp, idx, n_valid)
    dor = do.copy()
    dor[:, :, n_valid:] = 0.0
    assert np.abs(dv.sum(axis=2) - dor.sum(axis=2)).max() < 1e-9
    assert np.abs(dk.sum(axis=2)).max() < 1e-9
    eps = 1e-3
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for pos in [(0, 0, 5, 1), (0, 0, 300, 3), (0, 0, 699, 0), (0, 0, 650, 2)]:
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][pos] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][pos] -= 2 * eps
            dn = loss(args["q"], args["k"], args["v"])
            fd = (up - dn) / (2 * eps)
            assert abs(fd - grad[pos]) < 1e-4 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])
