"""LLSA over a padded sequence: the oracle for a reading the pages do not define.

TEST INFRASTRUCTURE ONLY, under the same rules as ``llsa_oracle``: only ``tests/`` may
import it; it shares no code with the CUDA path and imports nothing from it.

The LLSA GitHub README's usage section states that the released kernels need the token
length to be a power of two and that later updates will lift that limit.  A sequence whose
length n_valid is not a multiple of 16^L can still run on a grid of N = 16^L * ceil(n_valid
/ 16^L) positions if the positions from n_valid on are padding that takes no part in the
result.  This module fixes what that means (parity unpinned against the pages, which say
nothing about it; pinned below by closed forms):

* Pooling: level-l token j averages only the real tokens of its span; its count c_{l,j} is
  the number of them, and a token with c = 0 is empty (its value is 0).  Each level is made
  from the stored level below, in fp32: level 1 adds the c real tokens in index order and
  divides by c; level l >= 2 adds, in index order, each child's count times its stored mean
  (c_{l-1} * mean, rounded), then divides by c_{l,j}.  So a level is always a function of the
  level below, as in the unpadded pyramid.  For a full token the products are exact (powers
  of two), and a sequence without padding gives results bit-identical to
  ``llsa_oracle.build_pyramid`` (scaling by a power of two commutes with rounding).
* Selection: empty tokens are never candidates.  The real tokens of every level form a
  prefix [0, m_l) with m_l = ceil(n_valid / 16^l); K <= m_L keeps every list full (each
  picked parent has a real child).  Queries of empty tokens select from their zero mean.
* Attention: the KV lists are ``llsa_oracle``'s; padding keys (positions >= n_valid) are
  masked out.  Padding queries output 0 (LSE 0) and send no gradient anywhere.
* Gradients: a pooled token's gradient reaches each of its c real tokens with weight 1/c.
"""
from __future__ import annotations

import math

import numpy as np

from .llsa_oracle import (BLOCK, children, index_transpose_all, kv_index_table, kv_sources, selection_scores,
                          topk_positions)


def valid_counts(N: int, n_valid: int, levels: int) -> list[np.ndarray]:
    """c_{l,j} for l = 1..L: the number of positions < n_valid in level-l token j's span."""
    if not 1 <= n_valid <= N:
        raise ValueError("need 1 <= n_valid <= N")
    out = []
    for lev in range(1, levels + 1):
        span = BLOCK ** lev
        start = np.arange(N // span, dtype=np.int64) * span
        out.append(np.clip(n_valid - start, 0, span))
    return out


def build_pyramid_padded(x: np.ndarray, levels: int, n_valid: int) -> list[np.ndarray]:
    """Means over the real tokens of every span (see the module header), fp32."""
    B, H, N, D = x.shape
    counts = valid_counts(N, n_valid, levels)
    real = np.asarray(x, dtype=np.float32).copy()
    real[:, :, n_valid:] = 0.0  # padding contributes nothing to the sums
    out = []
    prev = real                                          # level 0: the tokens, count 1 or 0
    prev_count = np.ones(N, dtype=np.float32)
    for lev in range(levels):
        groups = prev.reshape(B, H, -1, BLOCK, D)
        cnt = prev_count.reshape(-1, BLOCK)
        s = np.zeros(groups.shape[:3] + (D,), dtype=np.float32)
        for r in range(BLOCK):
            term = groups[:, :, :, r, :] if lev == 0 else (cnt[None, None, :, r, None] * groups[:, :, :, r, :])
            s = s + term.astype(np.float32)
        c = counts[lev].astype(np.float32)[None, None, :, None]
        mean = np.where(c > 0, s / np.where(c > 0, c, np.float32(1.0)), np.float32(0.0)).astype(np.float32)
        out.append(mean)
        prev = mean
        prev_count = counts[lev].astype(np.float32)
    return out


def select_padded(q_pyr: list[np.ndarray], k_pyr: list[np.ndarray], topk: int, n_valid: int) -> list[np.ndarray]:
    """Hierarchical Top-K over real tokens only: candidates at level L are [0, m_L); at a
    finer level the children of the parent's picks that are real."""
    L = len(q_pyr)
    B, H, nL, _ = q_pyr[L - 1].shape
    m = [math.ceil(n_valid / BLOCK ** lev) for lev in range(1, L + 1)]
    if not 1 <= topk <= m[L - 1]:
        raise ValueError(f"topk={topk} must be in [1, m_L={m[L - 1]}]: the coarsest real tokens must hold K")
    idx: list[np.ndarray | None] = [None] * L
    out = np.empty((B, H, nL, topk), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            s = selection_scores(q_pyr[L - 1][b, h], k_pyr[L - 1][b, h, :m[L - 1]])
            out[b, h] = topk_positions(s, topk)
    idx[L - 1] = out
    for lev in range(L - 1, 0, -1):
        n = q_pyr[lev - 1].shape[2]
        out = np.empty((B, H, n, topk), dtype=np.int32)
        for b in range(B):
            for h in range(H):
                qs, ks = q_pyr[lev - 1][b, h], k_pyr[lev - 1][b, h]
                for g in range(n // BLOCK):
                    cand = children(idx[lev][b, h, g])
                    cand = cand[cand < m[lev - 1]]            # real children only, still ascending
                    s = selection_scores(qs[BLOCK * g:BLOCK * (g + 1)], ks[cand])
                    out[b, h, BLOCK * g:BLOCK * (g + 1)] = cand[topk_positions(s, topk)]
        idx[lev - 1] = out
    return idx


def _key_mask(rows: np.ndarray, N: int, n_valid: int) -> np.ndarray:
    """Rows of ``kv_sources`` that may be attended: real input tokens and (selected, hence
    real) pooled tokens."""
    return (rows < n_valid) | (rows >= N)


def forward_padded(q, k, v, k_pyr, v_pyr, idx, n_valid: int):
    """O [B, H, N, D] and LSE [B, H, N] (fp64); padding queries give 0 and 0."""
    q = np.asarray(q, dtype=np.float64)
    B, H, N, D = q.shape
    ksrc, offsets = kv_sources(k, k_pyr)
    vsrc, _ = kv_sources(v, v_pyr)
    n1 = N // BLOCK
    scale = 1.0 / math.sqrt(D)
    o = np.zeros((B, H, N, D))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            table = kv_index_table(b, h, idx, offsets)
            qb = q[b, h].reshape(n1, BLOCK, D)
            z = np.einsum("nqd,ntd->nqt", qb, ksrc[b, h][table]) * scale
            z = np.where(_key_mask(table, N, n_valid)[:, None, :], z, -np.inf)
            mx = z.max(axis=-1, keepdims=True)
            e = np.exp(z - mx)
            zs = e.sum(axis=-1, keepdims=True)
            o[b, h] = np.einsum("nqt,ntd->nqd", e / zs, vsrc[b, h][table]).reshape(N, D)
            lse[b, h] = (mx + np.log(zs)).reshape(N)
    o[:, :, n_valid:] = 0.0
    lse[:, :, n_valid:] = 0.0
    return o, lse


def backward_padded(q, k, v, o, lse, do, k_pyr, v_pyr, idx, n_valid: int):
    """dQ, dK, dV (fp64) with the selection fixed; padding queries send no gradient and
    padding positions receive none; a pooled token's gradient is spread over its real
    tokens with weight 1 / count."""
    q = np.asarray(q, dtype=np.float64)
    B, H, N, D = q.shape
    L = len(idx)
    do = np.array(do, dtype=np.float64)
    do[:, :, n_valid:] = 0.0
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    ksrc, offsets = kv_sources(k, k_pyr)
    vsrc, _ = kv_sources(v, v_pyr)
    counts = valid_counts(N, n_valid, L)
    n1 = N // BLOCK
    scale = 1.0 / math.sqrt(D)
    dq = np.zeros((B, H, N, D))
    dk = np.zeros((B, H, N, D))
    dv = np.zeros((B, H, N, D))
    for b in range(B):
        for h in range(H):
            table = kv_index_table(b, h, idx, offsets)
            real_q = (np.arange(N) < n_valid).reshape(n1, BLOCK)[..., None]
            mask = _key_mask(table, N, n_valid)[:, None, :] & real_q   # padding queries take part in nothing
            qb = q[b, h].reshape(n1, BLOCK, D)
            dob = do[b, h].reshape(n1, BLOCK, D)
            ke, ve = ksrc[b, h][table], vsrc[b, h][table]
            z = np.einsum("nqd,ntd->nqt", qb, ke) * scale
            p = np.where(mask, np.exp(np.where(mask, z - lse[b, h].reshape(n1, BLOCK)[..., None], 0.0)), 0.0)
            delta = (dob * o[b, h].reshape(n1, BLOCK, D)).sum(axis=-1)
            ds = p * (np.einsum("nqd,ntd->nqt", dob, ve) - delta[..., None])
            dq[b, h] = (np.einsum("nqt,ntd->nqd", ds, ke) * scale).reshape(N, D)
            dksrc = np.zeros_like(ksrc[b, h])
            dvsrc = np.zeros_like(vsrc[b, h])
            np.add.at(dksrc, table, np.einsum("nqt,nqd->ntd", ds, qb) * scale)
            np.add.at(dvsrc, table, np.einsum("nqt,nqd->ntd", p, dob))
            gk, gv = dksrc[:N].copy(), dvsrc[:N].copy()
            for lev in range(1, L + 1):
                span = BLOCK ** lev
                c = counts[lev - 1]
                w = np.where(c > 0, 1.0 / np.maximum(c, 1), 0.0)[:, None]
                ck = dksrc[offsets[lev]:offsets[lev] + N // span] * w
                cv = dvsrc[offsets[lev]:offsets[lev] + N // span] * w
                gk += np.repeat(ck, span, axis=0)
                gv += np.repeat(cv, span, axis=0)
            gk[n_valid:] = 0.0
            gv[n_valid:] = 0.0
            dk[b, h], dv[b, h] = gk, gv
    dq[:, :, n_valid:] = 0.0
    return dq, dk, dv


def llsa_step_padded(q, k, v, do, levels: int, topk: int, n_valid: int):
    """Pyramid, selection, forward, backward and transposes of a padded sequence."""
    q_pyr = build_pyramid_padded(q, levels, n_valid)
    k_pyr = build_pyramid_padded(k, levels, n_valid)
    v_pyr = build_pyramid_padded(v, levels, n_valid)
    idx = select_padded(q_pyr, k_pyr, topk, n_valid)
    o, lse = forward_padded(q, k, v, k_pyr, v_pyr, idx, n_valid)
    out = dict(q_pyr=q_pyr, k_pyr=k_pyr, v_pyr=v_pyr, idx=idx, o=o, lse=lse)
    if do is not None:
        out["dq"], out["dk"], out["dv"] = backward_padded(q, k, v, o, lse, do, k_pyr, v_pyr, idx, n_valid)
    out["row_ptr"], out["col"] = index_transpose_all(idx)
    return out
