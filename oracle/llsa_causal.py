"""Causal LLSA: the oracle for a reading the pages do not define.

TEST INFRASTRUCTURE ONLY, under the same rules as ``llsa_oracle``: only ``tests/`` may
import it; it shares no code with the CUDA path and imports nothing from it.

The LLSA GitHub README's usage section says the released kernels support only non-causal
attention (they replace ``scaled_dot_product_attention(..., is_causal=False)``) and that a
later update will address it.  This module fixes what a causal LLSA computes, taking the
SDPA meaning of ``is_causal=True`` -- query position i attends only to key positions t <= i
-- and changing as little else as possible (parity unpinned against the pages, which say
nothing about it; pinned below by closed forms and invariants):

* Pyramid: unchanged (``llsa_oracle.build_pyramid``).  Level-l token j spans input
  positions [j 16^l, (j+1) 16^l).
* Selection: top-down as in ``llsa_oracle.select``, but a level-l query token a may only
  pick key tokens j <= a (tokens that start no later than it).  The candidates are those of
  the non-causal rule (all of level L; below, the 16K children of the parent's picks) with
  index <= a.  When fewer than K candidates remain, the list holds the picks in ascending
  order followed by NO_PICK (2^31 - 1, so every list stays ascending).  Scores, the
  tie-break and the pooled queries are the non-causal ones, so a query block's choice of
  keys may depend on the later queries of its coarser spans; the attention below never
  reads a key after its query.
* KV list of query block p: the 16 tokens of each picked level-1 block j (j < p: all
  visible; j = p, the diagonal block: key t visible to query i iff t <= i), then for
  l = 2..L the level-l tokens j picked by p's level-l ancestor a = p // 16^(l-1) with
  j < a (such a token lies wholly before the block).  The ancestor itself (picked so that
  the finer levels can descend into it) and NO_PICK entries are not attended.
* Every query keeps at least one visible key: each level has a candidate (its own token,
  j = a, or a child of its parent's own pick), so block p always picks some j <= p, and a
  pick j < p is wholly visible while the diagonal block shows token 16p to every query.
* Gradients: the non-causal ones restricted to the visible entries; pooled tokens pass
  theirs to the input tokens through the mean-pool adjoint (1/16^l each).
* Index transpose: row j of level l lists the queries a with j in S_l(a), ascending; NO_PICK
  entries are dropped, so row_ptr[n] is the number of real picks.
"""
from __future__ import annotations

import math

import numpy as np

from .llsa_oracle import (BLOCK, build_pyramid, children, dot_error_floor, kv_sources, selection_scores,
                          topk_positions, _row_verdict)

NO_PICK = 2 ** 31 - 1


def _pick(scores: np.ndarray, cand: np.ndarray, topk: int) -> np.ndarray:
    """The K best of ``cand`` (ascending) under (score desc, index asc), ascending, padded
    with NO_PICK when there are fewer than K candidates."""
    out = np.full(topk, NO_PICK, dtype=np.int64)
    if cand.size:
        got = cand[topk_positions(scores[None, :], min(topk, cand.size))[0]]
        out[:got.size] = got
    return out


def select_causal(q_pyr: list[np.ndarray], k_pyr: list[np.ndarray], topk: int) -> list[np.ndarray]:
    """Causal hierarchical Top-K: idx[l-1] [B, H, n_l, K] int32, ascending, NO_PICK-padded."""
    L = len(q_pyr)
    B, H, nL, _ = q_pyr[L - 1].shape
    if not 1 <= topk <= nL:
        raise ValueError(f"topk={topk} must be in [1, n_L={nL}]")
    idx: list[np.ndarray | None] = [None] * L
    for lev in range(L, 0, -1):
        n = q_pyr[lev - 1].shape[2]
        out = np.empty((B, H, n, topk), dtype=np.int64)
        for b in range(B):
            for h in range(H):
                qs, ks = q_pyr[lev - 1][b, h], k_pyr[lev - 1][b, h]
                for a in range(n):
                    if lev == L:
                        cand = np.arange(n)
                    else:
                        parents = idx[lev][b, h, a // BLOCK]
                        cand = children(parents[parents != NO_PICK])
                    cand = cand[cand <= a]
                    s = selection_scores(qs[a:a + 1], ks[cand])[0]
                    out[b, h, a] = _pick(s, cand, topk)
        idx[lev - 1] = out.astype(np.int32)
    return idx  # type: ignore[return-value]


def kv_list_causal(p: int, bh: tuple[int, int], idx: list[np.ndarray], offsets: list[int]):
    """Rows (into ``llsa_oracle.kv_sources``) of query block p's causal KV list and the
    [16, T_p] visibility mask of its 16 queries (see the module header)."""
    b, h = bh
    L = len(idx)
    rows, masks = [], []
    q_pos = BLOCK * p + np.arange(BLOCK)
    for j in idx[0][b, h, p]:
        if j == NO_PICK:
            continue
        t = BLOCK * int(j) + np.arange(BLOCK)
        rows.append(t)
        masks.append(t[None, :] <= q_pos[:, None])       # all True when j < p
    for lev in range(2, L + 1):
        anc = p // BLOCK ** (lev - 1)
        for j in idx[lev - 1][b, h, anc]:
            if j < anc:                                   # NO_PICK and the ancestor itself fail this
                rows.append(np.array([offsets[lev] + int(j)]))
                masks.append(np.ones((BLOCK, 1), dtype=bool))
    return np.concatenate(rows), np.concatenate(masks, axis=1)


def forward_causal(q, k, v, k_pyr, v_pyr, idx):
    """O [B, H, N, D] and LSE [B, H, N] (fp64) of causal attention over each block's list:
    z_e = q_i . k_e / sqrt(D) on the entries visible to query i, softmax, O_i = sum p v,
    LSE_i = natural-log log-sum-exp of the visible z."""
    q = np.asarray(q, dtype=np.float64)
    B, H, N, D = q.shape
    ksrc, offsets = kv_sources(k, k_pyr)
    vsrc, _ = kv_sources(v, v_pyr)
    scale = 1.0 / math.sqrt(D)
    o = np.empty((B, H, N, D))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for p in range(N // BLOCK):
                rows, vis = kv_list_causal(p, (b, h), idx, offsets)
                z = q[b, h, BLOCK * p:BLOCK * (p + 1)] @ ksrc[b, h][rows].T * scale
                z = np.where(vis, z, -np.inf)
                m = z.max(axis=1, keepdims=True)
                e = np.exp(z - m)
                zs = e.sum(axis=1, keepdims=True)
                o[b, h, BLOCK * p:BLOCK * (p + 1)] = (e / zs) @ vsrc[b, h][rows]
                lse[b, h, BLOCK * p:BLOCK * (p + 1)] = (m + np.log(zs))[:, 0]
    return o, lse


def backward_causal(q, k, v, o, lse, do, k_pyr, v_pyr, idx):
    """dQ, dK, dV [B, H, N, D] (fp64) of ``forward_causal`` with the selection held fixed:
    P = softmax over the visible entries (0 elsewhere), Delta_i = dO_i . O_i,
    dS = P (dO v^T - Delta), dQ_i = sum_e dS_ie k_e / sqrt(D), dK_e += dS_ie q_i / sqrt(D),
    dV_e += P_ie dO_i; pooled tokens' gradients spread by the mean-pool adjoint."""
    q = np.asarray(q, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    B, H, N, D = q.shape
    L = len(idx)
    ksrc, offsets = kv_sources(k, k_pyr)
    vsrc, _ = kv_sources(v, v_pyr)
    scale = 1.0 / math.sqrt(D)
    dq = np.empty((B, H, N, D))
    dk = np.empty((B, H, N, D))
    dv = np.empty((B, H, N, D))
    for b in range(B):
        for h in range(H):
            dks = np.zeros_like(ksrc[b, h])
            dvs = np.zeros_like(vsrc[b, h])
            delta = (do[b, h] * o[b, h]).sum(axis=1)
            for p in range(N // BLOCK):
                sl = slice(BLOCK * p, BLOCK * (p + 1))
                rows, vis = kv_list_causal(p, (b, h), idx, offsets)
                ke, ve = ksrc[b, h][rows], vsrc[b, h][rows]
                z = q[b, h, sl] @ ke.T * scale
                pm = np.where(vis, np.exp(z - lse[b, h, sl][:, None]), 0.0)
                ds = pm * (do[b, h, sl] @ ve.T - delta[sl][:, None])
                dq[b, h, sl] = ds @ ke * scale
                np.add.at(dks, rows, ds.T @ q[b, h, sl] * scale)
                np.add.at(dvs, rows, pm.T @ do[b, h, sl])
            gk, gv = dks[:N].copy(), dvs[:N].copy()
            for lev in range(2, L + 1):
                n_l, span = N // BLOCK ** lev, BLOCK ** lev
                gk += np.repeat(dks[offsets[lev]:offsets[lev] + n_l], span, axis=0) / span
                gv += np.repeat(dvs[offsets[lev]:offsets[lev] + n_l], span, axis=0) / span
            dk[b, h], dv[b, h] = gk, gv
    return dq, dk, dv


def index_transpose_causal(idx_level: np.ndarray, n_keys: int) -> tuple[np.ndarray, np.ndarray]:
    """Key -> query lists of one (b, h, level) causal selection [n_q, K], NO_PICK entries
    dropped: row_ptr [n_keys + 1] and col [row_ptr[-1]] (ascending queries per row)."""
    n_q, K = idx_level.shape
    flat = idx_level.reshape(-1).astype(np.int64)
    entries = np.nonzero(flat != NO_PICK)[0]
    keys = flat[entries]
    counts = np.bincount(keys, minlength=n_keys)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    col = (entries[np.argsort(keys, kind="stable")] // K).astype(np.int32)
    return row_ptr, col


def llsa_step_causal(q, k, v, do, levels: int, topk: int) -> dict:
    """Pyramid, causal selection, forward, backward and transposes."""
    q_pyr, k_pyr, v_pyr = build_pyramid(q, levels), build_pyramid(k, levels), build_pyramid(v, levels)
    idx = select_causal(q_pyr, k_pyr, topk)
    o, lse = forward_causal(q, k, v, k_pyr, v_pyr, idx)
    out = dict(q_pyr=q_pyr, k_pyr=k_pyr, v_pyr=v_pyr, idx=idx, o=o, lse=lse)
    if do is not None:
        out["dq"], out["dk"], out["dv"] = backward_causal(q, k, v, o, lse, do, k_pyr, v_pyr, idx)
    return out


def check_selection_causal(q_pyr, k_pyr, idx_test, topk: int, rel_tol: float = 1e-5) -> dict:
    """``llsa_oracle.check_selection`` for the causal rule: level by level from the coarsest
    down, the candidates of query a are the children of its parent's picks in ``idx_test``
    (all tokens at level L) with index <= a; the row must be those candidates' Top-K
    (ascending, NO_PICK-padded), exactly or up to near ties (``_row_verdict``)."""
    L = len(q_pyr)
    res = {"rows": 0, "exact": 0, "tie_window": 0, "floor_used": 0, "bad": 0, "bad_examples": []}
    for lev in range(L, 0, -1):
        test = np.asarray(idx_test[lev - 1]).astype(np.int64)
        B, H, n, K = test.shape
        assert K == topk
        for b in range(B):
            for h in range(H):
                qs, ks = q_pyr[lev - 1][b, h], k_pyr[lev - 1][b, h]
                for a in range(n):
                    if lev == L:
                        cand = np.arange(n)
                    else:
                        parents = np.asarray(idx_test[lev][b, h, a // BLOCK]).astype(np.int64)
                        cand = children(parents[parents != NO_PICK])
                    cand = cand[cand <= a]
                    s = selection_scores(qs[a:a + 1], ks[cand])[0]
                    want = _pick(s, cand, topk)
                    got = test[b, h, a]
                    res["rows"] += 1
                    if np.array_equal(got, want):
                        res["exact"] += 1
                        continue
                    m = min(topk, cand.size)
                    real = got[:m]
                    pos = np.searchsorted(cand, real)
                    valid = (np.all(got[m:] == NO_PICK) and np.all(np.diff(real) > 0) and np.all(pos < cand.size)
                             and np.array_equal(cand[np.minimum(pos, cand.size - 1)], real))
                    verdict = "bad"
                    if valid:
                        selm = np.zeros(cand.size, dtype=bool)
                        selm[pos] = True
                        fl = dot_error_floor(qs[a:a + 1], ks[cand])[0]
                        verdict = _row_verdict(s, fl, cand, selm, rel_tol)
                    if verdict != "bad":
                        res["tie_window"] += 1
                        res["floor_used"] += int(verdict == "floor")
                    else:
                        res["bad"] += 1
                        if len(res["bad_examples"]) < 5:
                            res["bad_examples"].append((lev, b, h, a, got.tolist(), want.tolist()))
    return res
