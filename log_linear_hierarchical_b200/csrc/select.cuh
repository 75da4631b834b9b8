// Step 2: hierarchical Top-K block selection (skill page "Log Linear Sparse Attention",
// Core Technique 1: full selection only at the coarsest level, then at each finer level a
// sparse Top-K over the children of the blocks selected one level up).
//
// One CTA scores a group of level-l queries against a shared candidate list:
//   * coarsest level: up to 16 queries, candidates = all n_L keys;
//   * finer levels:   the 16 sibling queries of one parent, candidates = the 16K children
//                     16c + r of the parent's K selected keys c (ascending).
// Scores are fp32 dot products of the fp32 pyramid rows (the 1/sqrt(D) scale does not
// change the order and is not applied).  The K winners come from K warp-wide rounds of
// redux.sync max (score) then min (candidate position); the order is (score desc, key asc),
// so the lower key index wins equal scores.  Output rows are written in ascending key order.
//
// Bound: L2 reads of the candidate key rows (each group's 16K rows are read once and
// reused by its 16 queries); the arithmetic is 16 * 16K * 64 FMA per group.
#pragma once

#include "pyramid.cuh"

namespace llsa {

constexpr int kSelThreads = 256;

// Order-preserving map of an fp32 score to an unsigned key: a larger score gives a larger
// key; -0 and +0 both map to the key of +0 (they compare equal as floats).  Every real
// score maps above 0, so 0 marks a removed candidate.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Candidate rows are staged in shared memory with a padded stride (D + 4 floats: a quarter
// warp's 16-byte reads of 8 consecutive rows hit 8 distinct bank groups).
template <int D>
__host__ __device__ constexpr int sel_row_stride() {
  return D + 4;
}
// Candidates scored per pass (256 rows at D = 64, 128 at D = 128: about 68 KB of staged
// rows); larger candidate sets (the coarsest level) are scored in passes of this many rows.
template <int D>
__host__ __device__ constexpr int sel_chunk() {
  return D == 64 ? 256 : 128;
}

// Top-K of one query's score keys krow[0..nc) by one warp: each lane keeps the best of its
// candidates c = lane + 32 i; redux.sync finds the largest key, then the lowest candidate
// holding it; the owner removes it (key 0) and rescans.  Winners go to wrow[0..K).
__device__ __forceinline__ void warp_topk(uint32_t* krow, int nc, int K, int* wrow) {
  const int lane = lane_id();
  uint32_t bk = 0u;
  int bc = 0x7fffffff;
  for (int c = lane; c < nc; c += 32) {
    const uint32_t k = krow[c];
    if (k > bk) {
      bk = k;
      bc = c;
    }
  }
  for (int r = 0; r < K; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t w = __reduce_min_sync(0xffffffffu, bk == m ? (uint32_t)bc : 0x7fffffffu);
    if (lane == 0) wrow[r] = (int)w;  // 0x7fffffff: no candidate left (a short causal list)
    if (m != 0u && bc == (int)w && bk == m) {  // the owner drops its winner and finds its next best
      krow[w] = 0u;
      bk = 0u;
      bc = 0x7fffffff;
      for (int c = lane; c < nc; c += 32) {
        const uint32_t k = krow[c];
        if (k > bk) {
          bk = k;
          bc = c;
        }
      }
    }
  }
  __syncwarp();
}

// grid.x = B*H * groups; dynamic smem: see select_smem_bytes.
// parent_idx == nullptr selects the coarsest-level mode.
template <int D>
__global__ void __launch_bounds__(kSelThreads) select_kernel(Geometry g, int level, int gq,
                                                             const float* __restrict__ qp,
                                                             const float* __restrict__ kp,
                                                             const int* __restrict__ parent_idx,
                                                             int* __restrict__ out_idx) {
  pdl_enter();
  extern __shared__ __align__(16) float sel_smem[];
  const int n = g.n[level];
  const int K = g.K;
  const bool sparse = parent_idx != nullptr;
  const int nc = sparse ? kBlock * K : n;
  const int groups = (n + gq - 1) / gq;
  const int bh = blockIdx.x / groups;
  const int grp = blockIdx.x - bh * groups;
  const int a0 = grp * gq;
  const int rows = min(gq, n - a0);
  const int chunk = min(nc, sel_chunk<D>());

  constexpr int RS = sel_row_stride<D>();
  float* qs = sel_smem;                                             // [gq][D]
  float* ks = qs + gq * D;                                          // [chunk][D + 4]
  int* cand = reinterpret_cast<int*>(ks + chunk * RS);              // [nc] (sparse only)
  uint32_t* sk = reinterpret_cast<uint32_t*>(cand + (sparse ? nc : 0));  // [gq][nc] score keys
  int* win = reinterpret_cast<int*>(sk + gq * nc);                  // [gq][K]

  const int tid = threadIdx.x;
  const float* qbase = qp + ((long long)bh * n + a0) * D;
  for (int i = tid; i < gq * D; i += kSelThreads) qs[i] = (i < rows * D) ? qbase[i] : 0.0f;
  if (sparse) {
    const int np = g.n[level + 1];
    const int* prow = parent_idx + ((long long)bh * np + a0 / kBlock) * K;
    for (int i = tid; i < nc; i += kSelThreads) {
      const int raw = __ldg(prow + i / kBlock);  // a causal parent list may end in kNoPick: no children
      cand[i] = (g.causal && raw == kNoPick) ? -1 : checked_index(raw, np) * kBlock + (i % kBlock);
    }
  }
  __syncthreads();

  // ---- scores, one chunk of candidate rows at a time.  Thread t computes a tile of 2
  // queries (t / tpq selects the pair) x 4 candidates strided by tpq (t % tpq selects the
  // first) from shared memory.
  const int qgroups = (gq + 1) / 2;
  const int tpq = kSelThreads / qgroups;      // threads per query pair (32 for 16 queries)
  const int qg = tid / tpq;
  const int ct0 = tid - qg * tpq;
  for (int c0 = 0; c0 < nc; c0 += chunk) {
    const int cn = min(chunk, nc - c0);
    // stage rows c0 .. c0+cn-1 (coalesced: 16 threads copy one 256-byte row)
    for (int i = tid; i < cn * (D / 4); i += kSelThreads) {
      const int r = i / (D / 4);
      const int piece = i - r * (D / 4);
      const int key = max(sparse ? cand[c0 + r] : c0 + r, 0);
      const float4 v = __ldg(reinterpret_cast<const float4*>(kp + ((long long)bh * n + key) * D) + piece);
      *reinterpret_cast<float4*>(ks + r * RS + piece * 4) = v;
    }
    __syncthreads();
    for (int c = ct0; c < cn; c += 4 * tpq) {
      float acc[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
      const float4* kr[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) kr[v] = reinterpret_cast<const float4*>(ks + min(c + v * tpq, cn - 1) * RS);
      const float4* qr[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) qr[u] = reinterpret_cast<const float4*>(qs + min(2 * qg + u, gq - 1) * D);
#pragma unroll 4
      for (int i = 0; i < D / 4; ++i) {
        float4 kv[4], qv[2];
#pragma unroll
        for (int v = 0; v < 4; ++v) kv[v] = kr[v][i];
#pragma unroll
        for (int u = 0; u < 2; ++u) qv[u] = qr[u][i];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            acc[u][v] = fmaf(qv[u].x, kv[v].x, acc[u][v]);
            acc[u][v] = fmaf(qv[u].y, kv[v].y, acc[u][v]);
            acc[u][v] = fmaf(qv[u].z, kv[v].z, acc[u][v]);
            acc[u][v] = fmaf(qv[u].w, kv[v].w, acc[u][v]);
          }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int qi = 2 * qg + u;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int cc = c + v * tpq;
          if (qi < gq && cc < cn) {
            // empty tokens of a padded sequence (index >= the level's real count), missing
            // children and, under the causal rule, keys after the query token are never
            // candidates: key 0 marks a removed candidate
            const int key = sparse ? cand[c0 + cc] : c0 + cc;
            const bool ok = key >= 0 && key < g.m[level] && (!g.causal || key <= a0 + qi);
            sk[qi * nc + c0 + cc] = ok ? score_key(acc[u][v]) : 0u;
          }
        }
      }
    }
    __syncthreads();
  }

  // ---- K rounds per query, one warp per query
  const int warp = tid >> 5;
  const int lane = tid & 31;
  for (int qi = warp; qi < rows; qi += kSelThreads / 32) {
    int* wrow = win + qi * K;
    warp_topk(sk + qi * nc, nc, K, wrow);
    // ascending order: each winner's rank is the number of smaller winners
    int* orow = out_idx + ((long long)bh * n + a0 + qi) * K;
    for (int r = lane; r < K; r += 32) {
      const int mine = min(max(wrow[r], 0), nc - 1);
      int rank = 0;  // rounds without a winner (0x7fffffff) rank last, in round order
      for (int r2 = 0; r2 < K; ++r2) rank += wrow[r2] < wrow[r] || (wrow[r2] == wrow[r] && r2 < r);
      orow[rank] = wrow[r] == 0x7fffffff ? kNoPick : (sparse ? cand[mine] : mine);
    }
    __syncwarp();
  }
}

template <int D>
inline size_t select_smem_bytes(int gq, int nc, int K, bool sparse) {
  const int chunk = nc < sel_chunk<D>() ? nc : sel_chunk<D>();
  return sizeof(float) * ((size_t)gq * D + (size_t)chunk * sel_row_stride<D>() + (sparse ? nc : 0) +
                          (size_t)gq * nc + (size_t)gq * K);
}

// Finer levels with 16K = 32 * CPT candidates (K = 2, 4, 8, 16): the 16 sibling queries of
// one parent, 8 warps, warp w scoring queries 2w and 2w + 1 against all candidates.  Lane l
// holds candidates l + 32 j (j < CPT) of both queries in registers, which is the layout the
// warp Top-K walks, so scores never leave registers.  Each lane orders its candidates once
// (score desc, position asc); then K rounds of redux.sync max (score key) then min
// (candidate position) over the lanes' heads, the two queries' rounds interleaved.  The dot products
// accumulate channels 0..63 in order, as in select_kernel, so both give the same scores.
// A load of data that the same launch may have written (RO = false: the coherent path) or
// of data read-only for the whole launch (RO = true: the read-only data cache).
template <bool RO, typename T>
__device__ __forceinline__ T ld_in(const T* p) {
  if constexpr (RO) return __ldg(p);
  else return *p;
}

// One sibling group (unit = (b*H + h) * (n_l / 16) + group) of select_children_kernel;
// `sel_smem` is the CTA's shared buffer (select_children_smem_bytes).  kSelThreads threads.
// RO: the pyramid and the parent selection were written by earlier launches (read through
// the read-only cache); false inside the fused launch that writes them.
template <int D, int CPT, bool RO = true>
__device__ __forceinline__ void select_children_unit(const Geometry& g, int level, const float* __restrict__ qp,
                                                     const float* __restrict__ kp, const int* __restrict__ parent_idx,
                                                     int* __restrict__ out_idx, int unit, float* sel_smem) {
  constexpr int NC = 32 * CPT;
  constexpr int K = 2 * CPT;  // NC = 16 K
  const int n = g.n[level];
  const int groups = n / kBlock;
  const int bh = unit / groups;
  const int grp = unit - bh * groups;
  const int a0 = grp * kBlock;

  constexpr int RS = sel_row_stride<D>();
  constexpr int PR = D / 4;                                      // float4 pieces per row
  float* qs = sel_smem;                                          // [16][D]
  float* ks = qs + kBlock * D;                                   // [NC][D + 4]
  int* cand = reinterpret_cast<int*>(ks + NC * RS);              // [NC]

  const int tid = threadIdx.x;
  const float4* qbase = reinterpret_cast<const float4*>(qp + ((long long)bh * n + a0) * D);
  constexpr int QP = kBlock * PR / kSelThreads;  // query pieces per thread (16 rows x D/4)
  float4 qv[QP];
#pragma unroll
  for (int u = 0; u < QP; ++u) qv[u] = ld_in<RO>(qbase + tid + u * kSelThreads);
  const int np = g.n[level + 1];
  const int* prow = parent_idx + ((long long)bh * np + a0 / kBlock) * K;
  __syncthreads();  // the previous unit's shared rows are no longer read
  for (int i = tid; i < NC; i += kSelThreads) {
    const int raw = ld_in<RO>(prow + i / kBlock);  // a causal parent list may end in kNoPick
    cand[i] = (g.causal && raw == kNoPick) ? -1 : checked_index(raw, np) * kBlock + (i % kBlock);
  }
#pragma unroll
  for (int u = 0; u < QP; ++u) reinterpret_cast<float4*>(qs)[tid + u * kSelThreads] = qv[u];
  __syncthreads();
  // candidate rows: 16 threads copy one 256-byte row; each thread issues all its loads
  // (up to 8 at a time) before storing any, so they share one memory latency
  constexpr int kPer = NC * PR / kSelThreads;  // float4 pieces per thread
  constexpr int kBatch = kPer < 8 ? kPer : 8;
#pragma unroll
  for (int b0 = 0; b0 < kPer; b0 += kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = tid + (b0 + u) * kSelThreads;
      v[u] = ld_in<RO>(reinterpret_cast<const float4*>(kp + ((long long)bh * n + max(cand[i / PR], 0)) * D) + (i % PR));
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = tid + (b0 + u) * kSelThreads;
      *reinterpret_cast<float4*>(ks + (i / PR) * RS + (i % PR) * 4) = v[u];
    }
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const float4* q0 = reinterpret_cast<const float4*>(qs + (2 * warp) * D);
  const float4* q1 = reinterpret_cast<const float4*>(qs + (2 * warp + 1) * D);
  float acc[2][CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) acc[0][j] = acc[1][j] = 0.f;
#pragma unroll 4
  for (int i = 0; i < D / 4; ++i) {
    const float4 a = q0[i], b = q1[i];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const float4 kv = reinterpret_cast<const float4*>(ks + (lane + 32 * j) * RS)[i];
      acc[0][j] = fmaf(a.x, kv.x, acc[0][j]);
      acc[0][j] = fmaf(a.y, kv.y, acc[0][j]);
      acc[0][j] = fmaf(a.z, kv.z, acc[0][j]);
      acc[0][j] = fmaf(a.w, kv.w, acc[0][j]);
      acc[1][j] = fmaf(b.x, kv.x, acc[1][j]);
      acc[1][j] = fmaf(b.y, kv.y, acc[1][j]);
      acc[1][j] = fmaf(b.z, kv.z, acc[1][j]);
      acc[1][j] = fmaf(b.w, kv.w, acc[1][j]);
    }
  }
  uint32_t key[2][CPT];
  uint32_t bk[2] = {0u, 0u};
  int bc[2] = {0x7fffffff, 0x7fffffff};
  // each lane orders its CPT candidates once (score desc, index asc); a winner's owner then
  // only shifts its list
  int ci[2][CPT];
  const int mreal = g.m[level];  // real tokens of the level (all n of them unless padded)
#pragma unroll
  for (int u = 0; u < 2; ++u) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = cand[lane + 32 * j];  // missing children and (causal) keys after the query: none
      key[u][j] = (c >= 0 && c < mreal && (!g.causal || c <= a0 + 2 * warp + u)) ? score_key(acc[u][j]) : 0u;
      ci[u][j] = lane + 32 * j;
    }
#pragma unroll
    for (int pass = 0; pass < CPT; ++pass)
#pragma unroll
      for (int j = pass & 1; j + 1 < CPT; j += 2)
        if (key[u][j + 1] > key[u][j]) {  // indices ascend with j, so equal keys stay in order
          const uint32_t tk = key[u][j];
          key[u][j] = key[u][j + 1];
          key[u][j + 1] = tk;
          const int tc = ci[u][j];
          ci[u][j] = ci[u][j + 1];
          ci[u][j + 1] = tc;
        }
    bk[u] = key[u][0];
    bc[u] = key[u][0] ? ci[u][0] : 0x7fffffff;
  }
  int win[2] = {0, 0};
#pragma unroll 1
  for (int r = 0; r < K; ++r) {
    uint32_t m[2];
    int w[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) m[u] = __reduce_max_sync(0xffffffffu, bk[u]);
#pragma unroll
    for (int u = 0; u < 2; ++u) w[u] = (int)__reduce_min_sync(0xffffffffu, bk[u] == m[u] ? (uint32_t)bc[u] : 0x7fffffffu);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (lane == r) win[u] = w[u];
      if (bc[u] == w[u]) {
#pragma unroll
        for (int j = 0; j + 1 < CPT; ++j) {
          key[u][j] = key[u][j + 1];
          ci[u][j] = ci[u][j + 1];
        }
        key[u][CPT - 1] = 0u;
        ci[u][CPT - 1] = 0x7fffffff;
        bk[u] = key[u][0];
        bc[u] = key[u][0] ? ci[u][0] : 0x7fffffff;
      }
    }
  }
  // ascending order: each winner's rank is the number of smaller winners
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    int rank = 0;  // rounds without a winner (0x7fffffff) rank last, in round order
#pragma unroll
    for (int r2 = 0; r2 < K; ++r2) {
      const int w2 = __shfl_sync(0xffffffffu, win[u], r2);
      rank += w2 < win[u] || (w2 == win[u] && r2 < lane);
    }
    if (lane < K) {
      int* orow = out_idx + ((long long)bh * n + a0 + 2 * warp + u) * K;
      orow[rank] = win[u] == 0x7fffffff ? kNoPick : cand[min(max(win[u], 0), NC - 1)];
    }
  }
}

template <int D, int CPT>
__global__ void __launch_bounds__(kSelThreads) select_children_kernel(Geometry g, int level,
                                                                      const float* __restrict__ qp,
                                                                      const float* __restrict__ kp,
                                                                      const int* __restrict__ parent_idx,
                                                                      int* __restrict__ out_idx) {
  pdl_enter();
  extern __shared__ __align__(16) float sel_smem[];
  select_children_unit<D, CPT>(g, level, qp, kp, parent_idx, out_idx, blockIdx.x, sel_smem);
}

template <int D>
inline size_t select_children_smem_bytes(int nc) {
  return sizeof(float) * ((size_t)kBlock * D + (size_t)nc * sel_row_stride<D>() + (size_t)nc);
}

// Coarsest level with few tokens (n_L <= 64), one CTA per (b, h): optionally first the
// pooled levels 3..L of q, k and v from level 2 (POOL; the same sequential fp32 sums as
// pyramid_up_kernel), then the full Top-K of each of the n_L queries over the n_L keys,
// one warp per query, lane l scoring keys l and l + 32 (channels in order, as in
// select_kernel), K rounds of redux.sync max then min.  This replaces launches of 6..72
// CTAs whose time is all latency.
constexpr int kTopMaxN = 64;

constexpr int kTopThreads = 512;

// Dynamic shared memory: the n_L query and key rows at stride D + 4.
template <int D>
__host__ __device__ constexpr int coarsest_small_smem() {
  return 2 * kTopMaxN * sel_row_stride<D>() * (int)sizeof(float);
}

// One (b, h) of coarsest_small_kernel, by any number of whole warps; `top_smem` is the
// CTA's shared buffer (coarsest_small_smem).
template <int D, bool POOL>
__device__ __forceinline__ void coarsest_small_unit(const Geometry& g, float* __restrict__ q_pyr,
                                                    float* __restrict__ k_pyr, float* __restrict__ v_pyr,
                                                    int* __restrict__ idx, int bh, float* top_smem) {
  constexpr int RS = sel_row_stride<D>();
  constexpr int PR = D / 4;
  float* qs = top_smem;                    // [n_L][D + 4]
  float* ks = top_smem + kTopMaxN * RS;    // [n_L][D + 4]
  const int nth = blockDim.x;
  const int L = g.L, K = g.K, n = g.n[L];
  if (POOL) {
    for (int l = 3; l <= L; ++l) {
      const int nl = g.n[l], np = g.n[l - 1];
      const int items = 3 * nl * D;
      // two values per pass: their 32 loads are issued before the in-order sums
      for (int i0 = threadIdx.x; i0 < items; i0 += 2 * nth) {
        float x[2][kBlock];
        float* dst[2] = {nullptr, nullptr};
        int jj[2] = {0, 0};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u * nth;
          if (i < items) {
            const int t = i / (nl * D);
            const int rem = i - t * nl * D;
            const int j = rem / D, d = rem - j * D;
            jj[u] = j;
            float* pyr = t == 0 ? q_pyr : (t == 1 ? k_pyr : v_pyr);
            const float* src = pyr + g.pyr_off[l - 1] + ((long long)bh * np + (long long)j * kBlock) * D + d;
#pragma unroll
            for (int r = 0; r < kBlock; ++r) x[u][r] = src[r * D];
            dst[u] = pyr + g.pyr_off[l] + ((long long)bh * nl + j) * D + d;
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (!dst[u]) continue;
          *dst[u] = pool_up(g, l, jj[u], x[u]);
        }
      }
      __syncthreads();  // level l is read back by this CTA
    }
  }
  __syncthreads();  // the previous unit's shared rows are no longer read
  const float* qrow = q_pyr + g.pyr_off[L] + (long long)bh * n * D;
  const float* krow = k_pyr + g.pyr_off[L] + (long long)bh * n * D;
  for (int i = threadIdx.x; i < n * PR; i += blockDim.x) {
    const int r = i / PR, piece = i - r * PR;
    *reinterpret_cast<float4*>(qs + r * RS + piece * 4) = reinterpret_cast<const float4*>(qrow + r * D)[piece];
    *reinterpret_cast<float4*>(ks + r * RS + piece * 4) = reinterpret_cast<const float4*>(krow + r * D)[piece];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int a = warp; a < n; a += blockDim.x >> 5) {
    const float4* qa = reinterpret_cast<const float4*>(qs + a * RS);
    float acc[2] = {0.f, 0.f};
#pragma unroll 4
    for (int i = 0; i < D / 4; ++i) {
      const float4 qv = qa[i];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = min(lane + 32 * j, n - 1);
        const float4 kv = reinterpret_cast<const float4*>(ks + c * RS)[i];
        acc[j] = fmaf(qv.x, kv.x, acc[j]);
        acc[j] = fmaf(qv.y, kv.y, acc[j]);
        acc[j] = fmaf(qv.z, kv.z, acc[j]);
        acc[j] = fmaf(qv.w, kv.w, acc[j]);
      }
    }
    uint32_t key[2];
    uint32_t bk = 0u;
    int bc = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = lane + 32 * j;  // real tokens only; under the causal rule none after a
      key[j] = (c < g.m[L] && (!g.causal || c <= a)) ? score_key(acc[j]) : 0u;
      if (key[j] > bk) {
        bk = key[j];
        bc = lane + 32 * j;
      }
    }
    int win = 0;  // lane r < K keeps the r-th winner
    for (int r = 0; r < K; ++r) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
      const int w = (int)__reduce_min_sync(0xffffffffu, bk == m ? (uint32_t)bc : 0x7fffffffu);
      if (lane == r) win = w;
      if (bc == w) {
        bk = 0u;
        bc = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (lane + 32 * j == w) key[j] = 0u;
          if (key[j] > bk) {
            bk = key[j];
            bc = lane + 32 * j;
          }
        }
      }
    }
    int rank = 0;  // rounds without a winner (0x7fffffff) rank last, in round order
    for (int r2 = 0; r2 < K; ++r2) {
      const int w2 = __shfl_sync(0xffffffffu, win, r2);
      rank += w2 < win || (w2 == win && r2 < lane);
    }
    if (lane < K) idx[g.idx_off[L] + ((long long)bh * n + a) * K + rank] = win == 0x7fffffff ? kNoPick : min(max(win, 0), n - 1);
  }
}

template <int D, bool POOL>
__global__ void __launch_bounds__(kTopThreads) coarsest_small_kernel(Geometry g, float* __restrict__ q_pyr,
                                                                     float* __restrict__ k_pyr,
                                                                     float* __restrict__ v_pyr,
                                                                     int* __restrict__ idx) {
  pdl_enter();
  extern __shared__ __align__(16) float top_smem[];
  coarsest_small_unit<D, POOL>(g, q_pyr, k_pyr, v_pyr, idx, blockIdx.x, top_smem);
}

}  // namespace llsa
