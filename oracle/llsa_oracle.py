"""LLSA oracle: a plain, slow, obviously correct CPU reference (numpy, fp64).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library and its
Python binding never import it, and it imports nothing from them: the only code
both sides share is the seeded input generator in ``synthetic/``.

What it computes (Log-linear Sparse Attention, non-causal, per batch b and head h):

1. ``build_pyramid`` -- block-wise compression of tokens, 16 tokens per block,
   applied recursively for L levels ("Trainable Log-linear Sparse Attention for
   Efficient Diffusion Transformers", abstract: compressing tokens into block-wise
   representations; skill page "Log Linear Sparse Attention", Core Technique 1;
   ``block_size=16`` from the LLSA GitHub README usage section).
2. ``select`` -- hierarchical Top-K: full block scoring at the coarsest level, and at
   every finer level a sparse Top-K over only the children of the blocks the level
   above selected (skill page, Core Technique 1, "progressively adopting sparse
   Top-K selection with the indices found at the previous level", paraphrased).
3. ``kv_index`` -- hierarchical KV enrichment: each query block attends to its
   selected fine blocks plus coarse tokens taken from the coarser levels (skill
   page, Core Technique 2; abstract: coarse representations from several levels).
4. ``forward`` / ``backward`` -- softmax attention restricted to that KV list, with
   the ``scaled_dot_product_attention`` conventions the README's usage section
   replaces (non-causal, scale 1/sqrt(D), no dropout), and its exact gradient.
5. ``index_transpose`` -- the sparse index transpose: query -> key lists turned into
   key -> query lists without a dense mask (skill page, Core Technique 3).
6. ``to_z_order`` / ``from_z_order`` -- the quadtree token order of a square 2-D token
   grid that the README recommends for images (its token reordering example).

Readings where the pages are silent (each one is also listed in the design notes):

* Levels: level l in 1..L has n_l = N / 16^l tokens; level l token j is the mean
  of the 16 level-(l-1) tokens 16j..16j+15 (so a mean over 16^l input tokens).
* Pyramid arithmetic: fp32, the 16 terms added one after another in index order
  starting from 0.0, then multiplied by 1/16 (exact).  Level l is pooled from the
  stored fp32 level l-1.
* Scores for selection: raw dot products q.k / sqrt(D) in fp64 from the fp32
  pyramid.  Top-K of the logits equals Top-K of their softmax, so no softmax.
* Tie-break: among equal scores the lower key index wins; each list is stored in
  ascending key order.  The same K is used at every level.  A query block's own
  block is not forced into its list.
* Enrichment: for l = 2..L the K level-l tokens selected by the block's level-l
  ancestor are appended after the 16K fine tokens, each as one ordinary KV entry
  (unit weight, no score bias).  Level-1 pooled tokens are not attended.
* Enrichment variant, off by default (``log_bias=True``): a level-l coarse token's
  scaled score gets + ln(16^l), the log of the number of input tokens it averages, so
  that it carries the softmax mass of those tokens when they are all equal.
* Enrichment variant, off by default (``all_top=True``): for L >= 2 the level-L part of
  the list is every one of the n_L coarsest tokens, in index order, instead of the K the
  level-L ancestor selected (levels 2..L-1 are unchanged, and so is the selection).
  With L = 1 there are no coarse entries and the variant changes nothing.
* Enrichment variant, off by default (``level1=True``): the list also holds the level-1
  pooled token of each of the K selected fine blocks (the block's mean K and V), placed
  after the fine tokens; with ``log_bias`` those entries get + ln 16.  Their gradient
  goes back to the block's 16 input tokens through the mean-pool adjoint like any other
  pooled token's.
* Gradients: the selection and the pooled queries carry no gradient; coarse K/V
  tokens pass their gradient back to the input tokens through the mean-pool
  adjoint (each of the 16^l tokens under a level-l token receives 1/16^l of it).
* LSE is the natural-log log-sum-exp of the scaled scores.

Parity unpinned against the paper: no page fixes the enrichment content or weighting or
the pyramid's rounding order, so those follow the readings above.  The oracle is pinned to
those readings by closed forms (dense attention over the concatenated levels, a dense-mask
restatement, finite differences) and to the method's fixed parts by brute force, but not
to the authors' own code, which the pages do not include.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 16


# ----------------------------------------------------------------------------- shapes

def level_sizes(N: int, levels: int) -> list[int]:
    """n_l = N / 16^l for l = 0..L (level 0 is the input sequence)."""
    return [N // BLOCK ** l for l in range(levels + 1)]


def kv_len(topk: int, levels: int) -> int:
    """Length of a query block's KV list: 16K fine tokens and K coarse tokens per level 2..L."""
    return BLOCK * topk + (levels - 1) * topk


# ----------------------------------------------------------------------------- step 1: pyramid

def build_pyramid(x: np.ndarray, levels: int, acc_dtype=np.float32) -> list[np.ndarray]:
    """Mean-pooled pyramid of x [B, H, N, D]; returns [level 1, ..., level L], level l of
    shape [B, H, N / 16^l, D] in ``acc_dtype``.

    Each output value is (((0 + x_0) + x_1) + ... + x_15) * (1/16), every addition
    rounded in ``acc_dtype`` (fp32 by default; fp64 is used by the finite-difference
    test so that small perturbations survive).
    """
    out = []
    prev = np.asarray(x).astype(acc_dtype)
    inv = acc_dtype(1.0 / BLOCK)
    for _ in range(levels):
        B, H, n, D = prev.shape
        assert n % BLOCK == 0
        groups = prev.reshape(B, H, n // BLOCK, BLOCK, D)
        acc = np.zeros((B, H, n // BLOCK, D), dtype=acc_dtype)
        for r in range(BLOCK):
            acc = acc + groups[:, :, :, r, :]
        prev = acc * inv
        out.append(prev)
    return out


# ----------------------------------------------------------------------------- step 2: selection

def selection_scores(q_rows: np.ndarray, k_rows: np.ndarray) -> np.ndarray:
    """fp64 logits q.k / sqrt(D) for every (query row, key row) pair: [Rq, Rk]."""
    D = q_rows.shape[-1]
    return (q_rows.astype(np.float64) @ k_rows.astype(np.float64).T) / math.sqrt(D)


def topk_positions(scores: np.ndarray, topk: int) -> np.ndarray:
    """For each row of ``scores`` (candidates listed in ascending key order), the
    positions of the K largest scores, lower position first among equal scores,
    returned in ascending position order.  A stable sort on the negated scores keeps
    equal scores in ascending position, which is the lower-index tie-break."""
    order = np.argsort(-scores, axis=-1, kind="stable")[..., :topk]
    return np.sort(order, axis=-1)


def children(parent_keys: np.ndarray) -> np.ndarray:
    """Level-l keys under the given level-(l+1) keys: 16c + r for r = 0..15, ascending
    when ``parent_keys`` is ascending."""
    parent_keys = np.asarray(parent_keys, dtype=np.int64)
    return (BLOCK * parent_keys[..., :, None] + np.arange(BLOCK)).reshape(*parent_keys.shape[:-1], -1)


def select(q_pyr: list[np.ndarray], k_pyr: list[np.ndarray], topk: int) -> list[np.ndarray]:
    """Hierarchical Top-K.  Returns idx[l-1] of shape [B, H, n_l, K] (int32, ascending)
    for l = 1..L.

    Coarsest level L: every query token scores every key token.  Level l < L: query a
    scores only the 16K children of the K level-(l+1) keys its parent a // 16 selected.
    """
    L = len(q_pyr)
    B, H, nL, _ = q_pyr[L - 1].shape
    if not 1 <= topk <= nL:
        raise ValueError(f"topk={topk} must be in [1, n_L={nL}]: the coarsest level must hold K keys")
    idx: list[np.ndarray | None] = [None] * L
    out = np.empty((B, H, nL, topk), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            s = selection_scores(q_pyr[L - 1][b, h], k_pyr[L - 1][b, h])
            out[b, h] = topk_positions(s, topk)
    idx[L - 1] = out
    for lev in range(L - 1, 0, -1):
        n = q_pyr[lev - 1].shape[2]
        out = np.empty((B, H, n, topk), dtype=np.int32)
        for b in range(B):
            for h in range(H):
                qs, ks = q_pyr[lev - 1][b, h], k_pyr[lev - 1][b, h]
                for g in range(n // BLOCK):                    # sibling group = one parent
                    cand = children(idx[lev][b, h, g])          # [16K] ascending
                    s = selection_scores(qs[BLOCK * g:BLOCK * (g + 1)], ks[cand])
                    out[b, h, BLOCK * g:BLOCK * (g + 1)] = cand[topk_positions(s, topk)]
        idx[lev - 1] = out
    return idx  # type: ignore[return-value]


# ----------------------------------------------------------------------------- step 3: KV list

def kv_sources(x: np.ndarray, x_pyr: list[np.ndarray]) -> tuple[np.ndarray, list[int]]:
    """Stack, per (b, h), the attended token sources: the input tokens (level 0) followed
    by the pooled levels 1..L.  Returns the stacked [B, H, rows, D] array and the row
    offset of each level (offset[0] = 0, offset[l] for l >= 1)."""
    L = len(x_pyr)
    parts = [np.asarray(x)]
    offsets = [0]
    rows = x.shape[2]
    for lev in range(1, L + 1):
        offsets.append(rows)
        parts.append(x_pyr[lev - 1])
        rows += x_pyr[lev - 1].shape[2]
    return np.concatenate([p.astype(np.float64) for p in parts], axis=2), offsets


def kv_index(p: int, bh: tuple[int, int], idx: list[np.ndarray], offsets: list[int],
             all_top: bool = False, level1: bool = False) -> np.ndarray:
    """Rows (into ``kv_sources``) of query block p's KV list: the 16 tokens of each
    selected level-1 block, then for l = 2..L the K level-l tokens selected by p's
    level-l ancestor p // 16^(l-1).  With ``all_top`` the level-L part is instead every
    level-L token 0..n_L-1; with ``level1`` the level-1 pooled tokens of the K selected
    blocks follow the fine tokens."""
    b, h = bh
    L = len(idx)
    rows = [children(idx[0][b, h, p])]
    if level1:
        rows.append(offsets[1] + idx[0][b, h, p].astype(np.int64))
    for lev in range(2, L + 1):
        if all_top and lev == L:
            rows.append(offsets[lev] + np.arange(idx[lev - 1].shape[2], dtype=np.int64))
            continue
        anc = p // BLOCK ** (lev - 1)
        rows.append(offsets[lev] + idx[lev - 1][b, h, anc].astype(np.int64))
    return np.concatenate(rows)


def kv_index_table(b: int, h: int, idx: list[np.ndarray], offsets: list[int], all_top: bool = False,
                   level1: bool = False) -> np.ndarray:
    """[n_1, T] table of ``kv_index`` for every query block of (b, h)."""
    n1 = idx[0].shape[2]
    return np.stack([kv_index(p, (b, h), idx, offsets, all_top, level1) for p in range(n1)])


def kv_bias(topk: int, levels: int, n_top: int | None = None, level1: bool = False) -> np.ndarray:
    """Additive score bias of each KV-list entry under the log-count enrichment variant:
    0 for the 16K fine tokens, ln(16^l) for each of the K level-l coarse tokens.  With
    ``n_top`` (the all-coarsest variant) the level-L part has n_top entries; with
    ``level1`` the K level-1 pooled entries after the fine tokens get ln 16."""
    parts = [np.zeros(BLOCK * topk)]
    if level1:
        parts.append(np.full(topk, math.log(BLOCK)))
    for lev in range(2, levels + 1):
        count = n_top if (n_top is not None and lev == levels) else topk
        parts.append(np.full(count, lev * math.log(BLOCK)))
    return np.concatenate(parts)


# ----------------------------------------------------------------------------- step 4: attention

def forward(q, k, v, k_pyr, v_pyr, idx, chunk: int = 256, blocks=None, log_bias: bool = False,
            all_top: bool = False, level1: bool = False):
    """Softmax attention of every query over its block's KV list.

    Returns (O [B, H, N, D], LSE [B, H, N]) in fp64.  For query i of block p with
    list E(p): z_e = q_i . k_e / sqrt(D), O_i = sum_e softmax(z)_e v_e,
    LSE_i = max z + ln sum_e exp(z_e - max z).  With ``log_bias`` z_e also gets
    ``kv_bias`` (ln(16^l) for a level-l coarse token).
    ``blocks`` (ascending level-1 block indices) restricts the work to those query
    blocks of every (b, h); the other rows of O and LSE are left as NaN.
    ``all_top`` and ``level1`` select the enrichment variants of ``kv_index``.
    """
    q = np.asarray(q, dtype=np.float64)
    B, H, N, D = q.shape
    ksrc, offsets = kv_sources(k, k_pyr)
    vsrc, _ = kv_sources(v, v_pyr)
    n1 = N // BLOCK
    o = np.full((B, H, N, D), np.nan)
    lse = np.full((B, H, N), np.nan)
    scale = 1.0 / math.sqrt(D)
    n_top = idx[-1].shape[2] if all_top else None
    bias = kv_bias(idx[0].shape[-1], len(idx), n_top, level1) if log_bias else 0.0
    sel_blocks = np.arange(n1) if blocks is None else np.asarray(blocks, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            table = kv_index_table(b, h, idx, offsets, all_top, level1)
            qb = q[b, h].reshape(n1, BLOCK, D)
            for s0 in range(0, len(sel_blocks), chunk):
                sl = sel_blocks[s0:s0 + chunk]
                ke = ksrc[b, h][table[sl]]                   # [nb, T, D]
                ve = vsrc[b, h][table[sl]]
                z = np.einsum("nqd,ntd->nqt", qb[sl], ke) * scale + bias
                m = z.max(axis=-1, keepdims=True)
                e = np.exp(z - m)
                zsum = e.sum(axis=-1, keepdims=True)
                o[b, h].reshape(n1, BLOCK, D)[sl] = np.einsum("nqt,ntd->nqd", e / zsum, ve)
                lse[b, h].reshape(n1, BLOCK)[sl] = (m + np.log(zsum))[..., 0]
    return o, lse


def backward(q, k, v, o, lse, do, k_pyr, v_pyr, idx, chunk: int = 256, blocks=None, log_bias: bool = False,
             all_top: bool = False, level1: bool = False):
    """Exact gradient of the attention above with the selection held fixed.

    With P = softmax(z) on each query's list, Delta_i = sum_d dO_id O_id and
    dS = P * (dO v^T - Delta):  dQ_i = sum_e dS_ie k_e / sqrt(D),
    dK_e += dS_ie q_i / sqrt(D), dV_e += P_ie dO_i.  Gradients that land on coarse
    level-l tokens are then spread over their 16^l input tokens with weight 1/16^l
    (the adjoint of the mean pool).  Returns (dQ, dK, dV) [B, H, N, D] in fp64.
    ``blocks`` restricts the sum to those query blocks (dQ rows of the others are NaN).
    ``log_bias`` as in ``forward`` (a constant bias leaves the gradient formulas as they are);
    ``all_top`` and ``level1`` as in ``forward``.
    """
    q = np.asarray(q, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    B, H, N, D = q.shape
    L = len(idx)
    ksrc, offsets = kv_sources(k, k_pyr)
    vsrc, _ = kv_sources(v, v_pyr)
    n1 = N // BLOCK
    scale = 1.0 / math.sqrt(D)
    n_top = idx[-1].shape[2] if all_top else None
    bias = kv_bias(idx[0].shape[-1], L, n_top, level1) if log_bias else 0.0
    dq = np.full((B, H, N, D), np.nan)
    dk = np.empty((B, H, N, D))
    dv = np.empty((B, H, N, D))
    sel_blocks = np.arange(n1) if blocks is None else np.asarray(blocks, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            table = kv_index_table(b, h, idx, offsets, all_top, level1)
            qb = q[b, h].reshape(n1, BLOCK, D)
            dob = do[b, h].reshape(n1, BLOCK, D)
            delta = (do[b, h] * o[b, h]).sum(axis=-1).reshape(n1, BLOCK)
            lseb = lse[b, h].reshape(n1, BLOCK)
            dksrc = np.zeros_like(ksrc[b, h])
            dvsrc = np.zeros_like(vsrc[b, h])
            for s0 in range(0, len(sel_blocks), chunk):
                sl = sel_blocks[s0:s0 + chunk]
                rows = table[sl]
                ke = ksrc[b, h][rows]
                ve = vsrc[b, h][rows]
                z = np.einsum("nqd,ntd->nqt", qb[sl], ke) * scale + bias
                p = np.exp(z - lseb[sl][..., None])
                dp = np.einsum("nqd,ntd->nqt", dob[sl], ve)
                ds = p * (dp - delta[sl][..., None])
                dq[b, h].reshape(n1, BLOCK, D)[sl] = np.einsum("nqt,ntd->nqd", ds, ke) * scale
                dke = np.einsum("nqt,nqd->ntd", ds, qb[sl]) * scale
                dve = np.einsum("nqt,nqd->ntd", p, dob[sl])
                for i in range(rows.shape[0]):               # rows within one list are distinct
                    dksrc[rows[i]] += dke[i]
                    dvsrc[rows[i]] += dve[i]
            gk = dksrc[:N].copy()
            gv = dvsrc[:N].copy()
            for lev in range(1, L + 1):   # level 1 is attended only under ``level1``
                n_l = N // BLOCK ** lev
                span = BLOCK ** lev
                ck = dksrc[offsets[lev]:offsets[lev] + n_l]
                cv = dvsrc[offsets[lev]:offsets[lev] + n_l]
                gk += np.repeat(ck, span, axis=0) / span
                gv += np.repeat(cv, span, axis=0) / span
            dk[b, h] = gk
            dv[b, h] = gv
    return dq, dk, dv


# ----------------------------------------------------------------------------- step 5: transpose

def index_transpose(idx_level: np.ndarray, n_keys: int) -> tuple[np.ndarray, np.ndarray]:
    """Key -> query lists of one (b, h, level) selection ``idx_level`` [n_q, K].

    Returns (row_ptr [n_keys + 1], col [n_q * K]) int32: row j holds, in ascending
    order, every query a whose list contains key j.  A stable sort of the flattened
    entries by key keeps equal keys in ascending entry order, i.e. ascending query.
    """
    n_q, K = idx_level.shape
    flat = idx_level.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=n_keys)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    col = (np.argsort(flat, kind="stable") // K).astype(np.int32)
    return row_ptr, col


def index_transpose_all(idx: list[np.ndarray]) -> tuple[list[np.ndarray], list[np.ndarray]]:
    """Per level, row_ptr [B, H, n_l + 1] and col [B, H, n_l * K]."""
    rps, cols = [], []
    for lv in idx:
        B, H, n, K = lv.shape
        rp = np.empty((B, H, n + 1), dtype=np.int32)
        cl = np.empty((B, H, n * K), dtype=np.int32)
        for b in range(B):
            for h in range(H):
                rp[b, h], cl[b, h] = index_transpose(lv[b, h], n)
        rps.append(rp)
        cols.append(cl)
    return rps, cols


# ----------------------------------------------------------------------------- token order

def zorder_index(side: int) -> np.ndarray:
    """Quadtree (Z) index of every position of a side x side grid, row-major: position
    (r, c) gets z = sum_b (2 r_b + c_b) 4^b over the bits b of r and c, i.e. at every scale
    the quadrants in the order top-left, top-right, bottom-left, bottom-right (the LLSA
    GitHub README, token reordering example: similar, nearby tokens get adjacent indices)."""
    if side < 1 or side & (side - 1):
        raise ValueError("side must be a power of two")
    r, c = np.divmod(np.arange(side * side, dtype=np.int64), side)
    z = np.zeros_like(r)
    for b in range(int(side).bit_length()):
        z |= ((r >> b) & 1) << (2 * b + 1)
        z |= ((c >> b) & 1) << (2 * b)
    return z


def to_z_order(x: np.ndarray) -> np.ndarray:
    """[..., N, D] in row-major grid order -> Z order (N a power of four)."""
    n = x.shape[-2]
    side = int(round(math.sqrt(n)))
    if side * side != n:
        raise ValueError("N must be a square grid")
    out = np.empty_like(x)
    out[..., zorder_index(side), :] = x
    return out


def from_z_order(x: np.ndarray) -> np.ndarray:
    """Inverse of ``to_z_order``."""
    n = x.shape[-2]
    side = int(round(math.sqrt(n)))
    return x[..., zorder_index(side), :]


# ----------------------------------------------------------------------------- whole path

def llsa_step(q, k, v, do, levels: int, topk: int, log_bias: bool = False, all_top: bool = False,
              level1: bool = False):
    """Pyramid, selection, forward, backward and transposes with the oracle's own
    selection.  Inputs are exact widenings of the device inputs."""
    q_pyr = build_pyramid(q, levels)
    k_pyr = build_pyramid(k, levels)
    v_pyr = build_pyramid(v, levels)
    idx = select(q_pyr, k_pyr, topk)
    o, lse = forward(q, k, v, k_pyr, v_pyr, idx, log_bias=log_bias, all_top=all_top, level1=level1)
    out = dict(q_pyr=q_pyr, k_pyr=k_pyr, v_pyr=v_pyr, idx=idx, o=o, lse=lse)
    if do is not None:
        out["dq"], out["dk"], out["dv"] = backward(q, k, v, o, lse, do, k_pyr, v_pyr, idx, log_bias=log_bias,
                                                   all_top=all_top, level1=level1)
    out["row_ptr"], out["col"] = index_transpose_all(idx)
    return out


# ----------------------------------------------------------------------------- selection check

def dot_error_floor(q_rows: np.ndarray, k_rows: np.ndarray) -> np.ndarray:
    """Forward error bound of one fp32 length-D dot product, in the units of the scaled
    score: gamma_D * sum_d |q_d k_d| / sqrt(D) with gamma_D = D u / (1 - D u) and
    u = 2^-24 (Higham, Accuracy and Stability of Numerical Algorithms, 2nd ed., section 3.1,
    bound (3.5)).  It holds for any summation order, with or without fused multiply-adds.
    Returns one bound per (query row, key row) pair: [Rq, Rk]."""
    D = q_rows.shape[-1]
    u = 2.0 ** -24
    gamma = D * u / (1.0 - D * u)
    return gamma * (np.abs(q_rows.astype(np.float64)) @ np.abs(k_rows.astype(np.float64)).T) / math.sqrt(D)


def _row_verdict(s: np.ndarray, fl: np.ndarray, cand: np.ndarray, selm: np.ndarray, rel_tol: float) -> str:
    """Classify one row whose selected set ``selm`` differs from the oracle's Top-K.

    Every (selected x, rejected y) pair that the oracle orders the other way (s_y > s_x,
    or equal scores with y the lower index) must be a near tie: s_y - s_x below
    rel_tol * max(|s_x|, |s_y|) (the stated window), or else below the sum of the two
    scores' fp32 error bounds fl_x + fl_y (a selection computed in fp32 can only invert
    such a pair).  Returns "tie_window", "floor" (some pair needed the fp32 bound) or "bad".
    """
    sx, sy = s[selm][:, None], s[~selm][None, :]
    ix, iy = cand[selm][:, None], cand[~selm][None, :]
    gap = sy - sx
    inverted = (gap > 0) | ((gap == 0) & (iy < ix))
    if not inverted.any():          # cannot happen for a row that differs from the Top-K
        return "tie_window"
    rel = rel_tol * np.maximum(np.abs(sx), np.abs(sy))
    pair_floor = fl[selm][:, None] + fl[~selm][None, :]
    if np.any(inverted & (gap > np.maximum(rel, pair_floor))):
        return "bad"
    return "floor" if np.any(inverted & (gap > rel)) else "tie_window"


def check_selection(q_pyr, k_pyr, idx_test, topk: int, rel_tol: float = 1e-5, n_valid: int | None = None) -> dict:
    """Check a selection produced elsewhere, level by level from the coarsest down.

    At level l the candidates of query a are taken from ``idx_test`` at level l+1 (so a
    near-tie swap above does not cascade into failures below).  A row passes if it is
    the oracle's Top-K exactly, or if every pair it orders differently from the oracle is
    a near tie (``_row_verdict``): within rel_tol relative, or within the fp32 error bounds
    of the pair's two scores.
    Returns counts: exact rows, rows accepted by the relative window alone
    (``tie_window``), rows that needed the fp32 bound of some pair (``floor_used``, also
    counted in ``tie_window``), bad rows, and the first few bad rows for diagnosis.
    ``n_valid`` (a padded sequence): only the real tokens of each level, index < ceil(n_valid
    / 16^l), are candidates (the padded-sequence reading in ``llsa_padded``).
    """
    L = len(q_pyr)
    res = {"rows": 0, "exact": 0, "tie_window": 0, "floor_used": 0, "bad": 0, "bad_examples": []}
    for lev in range(L, 0, -1):
        test = np.asarray(idx_test[lev - 1])
        B, H, n, K = test.shape
        assert K == topk
        for b in range(B):
            for h in range(H):
                qs = q_pyr[lev - 1][b, h]
                ks = k_pyr[lev - 1][b, h]
                if lev == L:
                    groups = [(np.arange(n), np.arange(n))]
                else:
                    groups = [(np.arange(BLOCK * g, BLOCK * (g + 1)), children(idx_test[lev][b, h, g]))
                              for g in range(n // BLOCK)]
                if n_valid is not None:
                    real = -(-n_valid // BLOCK ** lev)
                    groups = [(qrows, cand[cand < real]) for qrows, cand in groups]
                for qrows, cand in groups:
                    s = selection_scores(qs[qrows], ks[cand])
                    floor = dot_error_floor(qs[qrows], ks[cand])
                    want = cand[topk_positions(s, topk)]
                    for r, a in enumerate(qrows):
                        res["rows"] += 1
                        got = test[b, h, a].astype(np.int64)
                        if np.array_equal(got, want[r]):
                            res["exact"] += 1
                            continue
                        pos = np.searchsorted(cand, got)
                        valid = (np.all(np.diff(got) > 0) and np.all(pos < cand.size)
                                 and np.array_equal(cand[np.minimum(pos, cand.size - 1)], got))
                        verdict = "bad"
                        if valid:
                            selm = np.zeros(cand.size, dtype=bool)
                            selm[pos] = True
                            verdict = _row_verdict(s[r], floor[r], cand, selm, rel_tol)
                        if verdict != "bad":
                            res["tie_window"] += 1
                            res["floor_used"] += int(verdict == "floor")
                        else:
                            res["bad"] += 1
                            if len(res["bad_examples"]) < 5:
                                res["bad_examples"].append((lev, b, h, int(a), got.tolist(), want[r].tolist()))
    return res
