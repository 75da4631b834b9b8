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

#include "llsa_common.cuh"

namespace llsa {

constexpr int kSelThreads = 256;

// Order-preserving map of an fp32 score to an unsigned key: a larger score gives a larger
// key; -0 and +0 both map to the key of +0 (they compare equal as floats).  Every real
// score maps above 0, so 0 marks a removed candidate.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Candidate rows are staged in shared memory with a padded stride (68 floats: a quarter
// warp's 16-byte reads of 8 consecutive rows hit 8 distinct bank groups).
constexpr int kSelRowStride = kD + 4;
// Candidates scored per pass; larger candidate sets (coarsest level with n_L > 256) are
// scored in passes of this many rows.
constexpr int kSelChunk = 256;

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
    if (lane == 0) wrow[r] = (int)w;
    if (bc == (int)w && bk == m) {  // the owner drops its winner and finds its next best
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
  const int chunk = min(nc, kSelChunk);

  float* qs = sel_smem;                                             // [gq][64]
  float* ks = qs + gq * kD;                                         // [chunk][68]
  int* cand = reinterpret_cast<int*>(ks + chunk * kSelRowStride);   // [nc] (sparse only)
  uint32_t* sk = reinterpret_cast<uint32_t*>(cand + (sparse ? nc : 0));  // [gq][nc] score keys
  int* win = reinterpret_cast<int*>(sk + gq * nc);                  // [gq][K]

  const int tid = threadIdx.x;
  const float* qbase = qp + ((long long)bh * n + a0) * kD;
  for (int i = tid; i < gq * kD; i += kSelThreads) qs[i] = (i < rows * kD) ? qbase[i] : 0.0f;
  if (sparse) {
    const int np = g.n[level + 1];
    const int* prow = parent_idx + ((long long)bh * np + a0 / kBlock) * K;
    for (int i = tid; i < nc; i += kSelThreads) {
      const int c = checked_index(__ldg(prow + i / kBlock), np);
      cand[i] = c * kBlock + (i % kBlock);
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
    for (int i = tid; i < cn * (kD / 4); i += kSelThreads) {
      const int r = i / (kD / 4);
      const int piece = i - r * (kD / 4);
      const int key = sparse ? cand[c0 + r] : c0 + r;
      const float4 v = __ldg(reinterpret_cast<const float4*>(kp + ((long long)bh * n + key) * kD) + piece);
      *reinterpret_cast<float4*>(ks + r * kSelRowStride + piece * 4) = v;
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
      for (int v = 0; v < 4; ++v) kr[v] = reinterpret_cast<const float4*>(ks + min(c + v * tpq, cn - 1) * kSelRowStride);
      const float4* qr[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) qr[u] = reinterpret_cast<const float4*>(qs + min(2 * qg + u, gq - 1) * kD);
#pragma unroll 4
      for (int i = 0; i < kD / 4; ++i) {
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
          if (qi < gq && cc < cn) sk[qi * nc + c0 + cc] = score_key(acc[u][v]);
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
      int rank = 0;
      for (int r2 = 0; r2 < K; ++r2) rank += wrow[r2] < wrow[r];
      orow[rank] = sparse ? cand[mine] : mine;
    }
    __syncwarp();
  }
}

inline size_t select_smem_bytes(int gq, int nc, int K, bool sparse) {
  const int chunk = nc < kSelChunk ? nc : kSelChunk;
  return sizeof(float) * ((size_t)gq * kD + (size_t)chunk * kSelRowStride + (sparse ? nc : 0) + (size_t)gq * nc +
                          (size_t)gq * K);
}

// Finer levels with 16K = 32 * CPT candidates (K = 2, 4, 8, 16): the 16 sibling queries of
// one parent, 8 warps, warp w scoring queries 2w and 2w + 1 against all candidates.  Lane l
// holds candidates l + 32 j (j < CPT) of both queries in registers, which is the layout the
// warp Top-K walks, so scores never leave registers.  Each lane orders its candidates once
// (score desc, position asc); then K rounds of redux.sync max (score key) then min
// (candidate position) over the lanes' heads, the two queries' rounds interleaved.  The dot products
// accumulate channels 0..63 in order, as in select_kernel, so both give the same scores.
template <int CPT>
__global__ void __launch_bounds__(kSelThreads) select_children_kernel(Geometry g, int level,
                                                                      const float* __restrict__ qp,
                                                                      const float* __restrict__ kp,
                                                                      const int* __restrict__ parent_idx,
                                                                      int* __restrict__ out_idx) {
  pdl_enter();
  constexpr int NC = 32 * CPT;
  constexpr int K = 2 * CPT;  // NC = 16 K
  extern __shared__ __align__(16) float sel_smem[];
  const int n = g.n[level];
  const int groups = n / kBlock;
  const int bh = blockIdx.x / groups;
  const int grp = blockIdx.x - bh * groups;
  const int a0 = grp * kBlock;

  float* qs = sel_smem;                                          // [16][64]
  float* ks = qs + kBlock * kD;                                  // [NC][68]
  int* cand = reinterpret_cast<int*>(ks + NC * kSelRowStride);   // [NC]

  const int tid = threadIdx.x;
  const float4* qbase = reinterpret_cast<const float4*>(qp + ((long long)bh * n + a0) * kD);
  const float4 qv = __ldg(qbase + tid);  // 16 rows x 16 pieces = one per thread
  const int np = g.n[level + 1];
  const int* prow = parent_idx + ((long long)bh * np + a0 / kBlock) * K;
  for (int i = tid; i < NC; i += kSelThreads) cand[i] = checked_index(__ldg(prow + i / kBlock), np) * kBlock + (i % kBlock);
  reinterpret_cast<float4*>(qs)[tid] = qv;
  __syncthreads();
  // candidate rows: 16 threads copy one 256-byte row; each thread issues all its loads
  // (up to 8 at a time) before storing any, so they share one memory latency
  constexpr int kPer = NC * (kD / 4) / kSelThreads;  // float4 pieces per thread
  constexpr int kBatch = kPer < 8 ? kPer : 8;
#pragma unroll
  for (int b0 = 0; b0 < kPer; b0 += kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = tid + (b0 + u) * kSelThreads;
      v[u] = __ldg(reinterpret_cast<const float4*>(kp + ((long long)bh * n + cand[i >> 4]) * kD) + (i & 15));
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = tid + (b0 + u) * kSelThreads;
      *reinterpret_cast<float4*>(ks + (i >> 4) * kSelRowStride + (i & 15) * 4) = v[u];
    }
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const float4* q0 = reinterpret_cast<const float4*>(qs + (2 * warp) * kD);
  const float4* q1 = reinterpret_cast<const float4*>(qs + (2 * warp + 1) * kD);
  float acc[2][CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) acc[0][j] = acc[1][j] = 0.f;
#pragma unroll 4
  for (int i = 0; i < kD / 4; ++i) {
    const float4 a = q0[i], b = q1[i];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const float4 kv = reinterpret_cast<const float4*>(ks + (lane + 32 * j) * kSelRowStride)[i];
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
#pragma unroll
  for (int u = 0; u < 2; ++u) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      key[u][j] = score_key(acc[u][j]);
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
    bc[u] = ci[u][0];
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
    int rank = 0;
#pragma unroll
    for (int r2 = 0; r2 < K; ++r2) rank += __shfl_sync(0xffffffffu, win[u], r2) < win[u];
    if (lane < K) {
      int* orow = out_idx + ((long long)bh * n + a0 + 2 * warp + u) * K;
      orow[rank] = cand[min(max(win[u], 0), NC - 1)];
    }
  }
}

inline size_t select_children_smem_bytes(int nc) {
  return sizeof(float) * ((size_t)kBlock * kD + (size_t)nc * kSelRowStride + (size_t)nc);
}

// Coarsest level with few tokens (n_L <= 64), one CTA per (b, h): optionally first the
// pooled levels 3..L of q, k and v from level 2 (POOL; the same sequential fp32 sums as
// pyramid_up_kernel), then the full Top-K of each of the n_L queries over the n_L keys,
// one warp per query, lane l scoring keys l and l + 32 (channels in order, as in
// select_kernel), K rounds of redux.sync max then min.  This replaces launches of 6..72
// CTAs whose time is all latency.
constexpr int kTopMaxN = 64;

constexpr int kTopThreads = 512;

template <bool POOL>
__global__ void __launch_bounds__(kTopThreads) coarsest_small_kernel(Geometry g, float* __restrict__ q_pyr,
                                                                     float* __restrict__ k_pyr,
                                                                     float* __restrict__ v_pyr,
                                                                     int* __restrict__ idx) {
  pdl_enter();
  __shared__ __align__(16) float qs[kTopMaxN * kSelRowStride];
  __shared__ __align__(16) float ks[kTopMaxN * kSelRowStride];
  const int bh = blockIdx.x;
  const int L = g.L, K = g.K, n = g.n[L];
  if (POOL) {
    for (int l = 3; l <= L; ++l) {
      const int nl = g.n[l], np = g.n[l - 1];
      const int items = 3 * nl * kD;
      // two values per pass: their 32 loads are issued before the in-order sums
      for (int i0 = threadIdx.x; i0 < items; i0 += 2 * kTopThreads) {
        float x[2][kBlock];
        float* dst[2] = {nullptr, nullptr};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u * kTopThreads;
          if (i < items) {
            const int t = i / (nl * kD);
            const int rem = i - t * nl * kD;
            const int j = rem >> 6, d = rem & (kD - 1);
            float* pyr = t == 0 ? q_pyr : (t == 1 ? k_pyr : v_pyr);
            const float* src = pyr + g.pyr_off[l - 1] + ((long long)bh * np + (long long)j * kBlock) * kD + d;
#pragma unroll
            for (int r = 0; r < kBlock; ++r) x[u][r] = src[r * kD];
            dst[u] = pyr + g.pyr_off[l] + ((long long)bh * nl + j) * kD + d;
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (!dst[u]) continue;
          float acc = 0.0f;
#pragma unroll
          for (int r = 0; r < kBlock; ++r) acc = __fadd_rn(acc, x[u][r]);
          *dst[u] = __fmul_rn(acc, 0.0625f);
        }
      }
      __syncthreads();  // level l is read back by this CTA
    }
  }
  const float* qrow = q_pyr + g.pyr_off[L] + (long long)bh * n * kD;
  const float* krow = k_pyr + g.pyr_off[L] + (long long)bh * n * kD;
  for (int i = threadIdx.x; i < n * (kD / 4); i += blockDim.x) {
    const int r = i >> 4, piece = i & 15;
    *reinterpret_cast<float4*>(qs + r * kSelRowStride + piece * 4) = reinterpret_cast<const float4*>(qrow + r * kD)[piece];
    *reinterpret_cast<float4*>(ks + r * kSelRowStride + piece * 4) = reinterpret_cast<const float4*>(krow + r * kD)[piece];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int a = warp; a < n; a += blockDim.x >> 5) {
    const float4* qa = reinterpret_cast<const float4*>(qs + a * kSelRowStride);
    float acc[2] = {0.f, 0.f};
#pragma unroll 4
    for (int i = 0; i < kD / 4; ++i) {
      const float4 qv = qa[i];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = min(lane + 32 * j, n - 1);
        const float4 kv = reinterpret_cast<const float4*>(ks + c * kSelRowStride)[i];
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
      key[j] = lane + 32 * j < n ? score_key(acc[j]) : 0u;
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
    int rank = 0;
    for (int r2 = 0; r2 < K; ++r2) rank += __shfl_sync(0xffffffffu, win, r2) < win;
    if (lane < K) idx[g.idx_off[L] + ((long long)bh * n + a) * K + rank] = min(max(win, 0), n - 1);
  }
}

}  // namespace llsa
