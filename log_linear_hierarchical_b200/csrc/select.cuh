// Step 2: hierarchical Top-K block selection (skill page "Log Linear Sparse Attention",
// Core Technique 1: full selection only at the coarsest level, then at each finer level a
// sparse Top-K over the children of the blocks selected one level up).
//
// One CTA scores a group of level-l queries against a shared candidate list:
//   * coarsest level: up to 16 queries, candidates = all n_L keys;
//   * finer levels:   the 16 sibling queries of one parent, candidates = the 16K children
//                     16c + r of the parent's K selected keys c (ascending).
// Scores are fp32 dot products of the fp32 pyramid rows (the 1/sqrt(D) scale does not
// change the order and is not applied).  The K winners come from K warp-wide argmax
// rounds over the scores held in shared memory; the order is (score desc, key asc), so
// the lower key index wins equal scores.  Output rows are written in ascending key order.
//
// Bound: L2 reads of the candidate key rows (each group's 16K rows are read once and
// reused by its 16 queries); the arithmetic is 16 * 16K * 64 FMA per group.
#pragma once

#include "llsa_common.cuh"

namespace llsa {

constexpr int kSelThreads = 256;

// True if (s1, c1) ranks before (s2, c2): higher score first, then lower candidate position.
__device__ __forceinline__ bool sel_better(float s1, int c1, float s2, int c2) {
  return s1 > s2 || (s1 == s2 && c1 < c2);
}

// grid.x = B*H * groups; dynamic smem = gq*64 + nc + gq*nc + gq*K ints/floats.
// parent_idx == nullptr selects the coarsest-level mode.
__global__ void __launch_bounds__(kSelThreads) select_kernel(Geometry g, int level, int gq,
                                                             const float* __restrict__ qp,
                                                             const float* __restrict__ kp,
                                                             const int* __restrict__ parent_idx,
                                                             int* __restrict__ out_idx) {
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

  float* qs = sel_smem;                          // [gq][64]
  int* cand = reinterpret_cast<int*>(qs + gq * kD);  // [nc] (sparse only)
  float* sc = reinterpret_cast<float*>(cand + (sparse ? nc : 0));  // [gq][nc]
  int* win = reinterpret_cast<int*>(sc + gq * nc);                 // [gq][K]

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

  // ---- scores: thread owns one candidate row (in registers) and a subset of the queries
  const int nsplit = nc >= kSelThreads ? 1 : kSelThreads / nc;
  const int cstep = nc >= kSelThreads ? kSelThreads : nc;
  const int qsub = tid / cstep;
  for (int c = tid % cstep; c < nc; c += cstep) {
    const int key = sparse ? cand[c] : c;
    const float4* krow = reinterpret_cast<const float4*>(kp + ((long long)bh * n + key) * kD);
    float4 kr[kD / 4];
#pragma unroll
    for (int i = 0; i < kD / 4; ++i) kr[i] = __ldg(krow + i);
    for (int qi = qsub; qi < gq; qi += nsplit) {
      const float4* qrow = reinterpret_cast<const float4*>(qs + qi * kD);
      float s = 0.0f;
#pragma unroll
      for (int i = 0; i < kD / 4; ++i) {
        const float4 qv = qrow[i];
        s = fmaf(qv.x, kr[i].x, s);
        s = fmaf(qv.y, kr[i].y, s);
        s = fmaf(qv.z, kr[i].z, s);
        s = fmaf(qv.w, kr[i].w, s);
      }
      sc[qi * nc + c] = s;
    }
  }
  __syncthreads();

  // ---- K argmax rounds per query, one warp per query
  const int warp = tid >> 5;
  const int lane = tid & 31;
  for (int qi = warp; qi < rows; qi += kSelThreads / 32) {
    float* srow = sc + qi * nc;
    int* wrow = win + qi * K;
    for (int r = 0; r < K; ++r) {
      float bs = -INFINITY;
      int bc = 0x7fffffff;
      for (int c = lane; c < nc; c += 32) {
        const float s = srow[c];
        if (sel_better(s, c, bs, bc)) {
          bs = s;
          bc = c;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int oc = __shfl_xor_sync(0xffffffffu, bc, off);
        if (sel_better(os, oc, bs, bc)) {
          bs = os;
          bc = oc;
        }
      }
      if (bc < 0 || bc >= nc) {  // only reachable with NaN scores
        record_error(LLSA_ERR_INTERNAL);
        bc = 0;
      }
      if (lane == (bc & 31)) srow[bc] = -INFINITY;
      if (lane == 0) wrow[r] = bc;
      __syncwarp();
    }
    // ascending order: each winner's rank is the number of smaller winners
    int* orow = out_idx + ((long long)bh * n + a0 + qi) * K;
    for (int r = lane; r < K; r += 32) {
      const int mine = wrow[r];
      int rank = 0;
      for (int r2 = 0; r2 < K; ++r2) rank += wrow[r2] < mine;
      orow[rank] = sparse ? cand[mine] : mine;
    }
    __syncwarp();
  }
}

inline size_t select_smem_bytes(int gq, int nc, int K, bool sparse) {
  return sizeof(float) * ((size_t)gq * kD + (sparse ? nc : 0) + (size_t)gq * nc + (size_t)gq * K);
}

}  // namespace llsa
