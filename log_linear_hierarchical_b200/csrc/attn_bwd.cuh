// Step 4b: gradient of the block-sparse attention with the selection held fixed (the
// pages train LLSA end to end; skill page "Log Linear Sparse Attention", Core Technique 3:
// the sparse index transpose serves the backward pass).
//
// No atomics.  Three kernels:
//   attn_bwd_dq_bf16_kernel      query-major.  Per query block: Delta = rowsum(dO * O),
//                                S = Q K^T, P = exp(S/sqrt(D) - LSE), dP = dO V^T,
//                                dS = P (dP - Delta), dQ = dS K / sqrt(D) over the whole KV list.
//                                A CTA is one level-2 group (16 query blocks), which shares
//                                its coarse KV entries, so the coarse gradients dS^T Q and
//                                P^T dO are summed over the group in shared memory and written
//                                once per (group, coarse slot).
//   coarse_grad_reduce_kernel    per coarse level-l token j: the sum of those partials over
//                                the level-l queries that selected j, read from the level-l CSR.
//   attn_bwd_dkdv_bf16_kernel    key-major.  Per selected fine key block j: the query blocks
//                                of CSR row j, recomputing P^T and dS^T for the 16 x 16 pair and
//                                accumulating dV = P^T dO and dK = dS^T Q / sqrt(D); the
//                                epilogue adds the mean-pool adjoint of every ancestor's coarse
//                                gradient (weight 1/16^l) and writes dK, dV once.
// Gathered tiles arrive by 2-D TMA (128-byte swizzle, no multicast) plus 64-byte bulk copies
// for LSE and Delta; products are mma.sync m16n8k16 bf16 with fp32 accumulation.
#pragma once

#include "attn_fwd.cuh"

namespace llsa {

// Backward workspace layout (fp32, offsets in floats, each 64-float aligned).
struct BwdWorkspace {
  long long delta;          // [B*H*N]
  long long part_k, part_v; // [B*H*n_2][C][64]
  long long cg_k, cg_v;     // coarse gradients, level-major [l=2..L][B*H*n_l][64]
  long long cg_off[kMaxLevels + 1];
  long long total;
};

__host__ __device__ inline BwdWorkspace bwd_workspace_layout(const Geometry& g) {
  auto up = [](long long x) { return (x + 63) & ~63LL; };
  BwdWorkspace w{};
  long long off = 0;
  w.delta = off;
  off = up(off + (long long)g.BH * g.N);
  const long long parts = g.L >= 2 ? (long long)g.BH * g.n[2] * g.coarse * kD : 0;
  w.part_k = off;
  off = up(off + parts);
  w.part_v = off;
  off = up(off + parts);
  long long cg = 0;
  for (int l = 0; l <= kMaxLevels; ++l) w.cg_off[l] = 0;
  for (int l = 2; l <= g.L; ++l) {
    w.cg_off[l] = cg;
    cg += (long long)g.BH * g.n[l] * kD;
  }
  w.cg_k = off;
  off = up(off + cg);
  w.cg_v = off;
  off = up(off + cg);
  w.total = off;
  return w;
}

// fp32 coarse-gradient accumulator tile [rows][64] with an XOR swizzle on 8-float groups so
// that the fragment-layout float2 accesses of a warp hit distinct banks.
__device__ __forceinline__ int cacc_index(int row, int col) { return row * kD + (col ^ ((row & 3) << 3)); }

// acc_smem[16 rows of chunk] += A (16 x 16 fragments) * B (16-row x 64 tile, rows = K).
__device__ __forceinline__ void mma_a_b_smem_acc(float* cacc, int row0, uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t btile) {
  const int lane = lane_id();
  const int brow = (lane & 7) + (((lane >> 3) & 1) << 3);
  const int r0 = row0 + (lane >> 2);
  const int c2 = 2 * (lane & 3);
#pragma unroll
  for (int dc = 0; dc < 4; ++dc) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(btile + swz(brow, 2 * dc + (lane >> 4)), b0, b1, b2, b3);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = (2 * dc + h) * 8 + c2;
      float2* p0 = reinterpret_cast<float2*>(cacc + cacc_index(r0, col));
      float2* p1 = reinterpret_cast<float2*>(cacc + cacc_index(r0 + 8, col));
      const float2 x0 = *p0, x1 = *p1;
      float c[4] = {x0.x, x0.y, x1.x, x1.y};
      if (h == 0) mma_bf16(c, a0, a1, a2, a3, b0, b1);
      else mma_bf16(c, a0, a1, a2, a3, b2, b3);
      *p0 = make_float2(c[0], c[1]);
      *p1 = make_float2(c[2], c[3]);
    }
  }
}

struct DqWarpMap {
  uint32_t qd, ring, ck, cv;
  float* cacc_k;
  float* cacc_v;
  float* lse;   // [2][16]
  int* idx;
  uint32_t bar_qd, bar_kv;
};

template <int STAGES>
__device__ __forceinline__ DqWarpMap dq_warp_map(uint8_t* base, const Geometry& g) {
  DqWarpMap m;
  const uint32_t b = smem_u32(base);
  m.qd = b;                                   // [2][Q tile, dO tile]
  m.ring = b + 4 * kTileBytes;
  m.ck = m.ring + STAGES * 2 * kTileBytes;
  m.cv = m.ck + g.coarse_pad * 128;
  uint8_t* p = base + 4 * kTileBytes + STAGES * 2 * kTileBytes + 2 * g.coarse_pad * 128;
  m.cacc_k = reinterpret_cast<float*>(p);
  m.cacc_v = m.cacc_k + g.coarse_pad * kD;
  p += 2 * g.coarse_pad * kD * 4;
  m.lse = reinterpret_cast<float*>(p);
  p += 2 * kBlock * 4;
  m.idx = reinterpret_cast<int*>(p);
  p += (kUnitBlocks * g.K * 4 + 15) & ~15;
  m.bar_qd = smem_u32(p);
  m.bar_kv = m.bar_qd + 16;
  return m;
}

template <int STAGES>
inline int dq_warp_bytes(const Geometry& g) {
  int bytes = 4 * kTileBytes + STAGES * 2 * kTileBytes + 2 * g.coarse_pad * 128 + 2 * g.coarse_pad * kD * 4 +
              2 * kBlock * 4 + ((kUnitBlocks * g.K * 4 + 15) & ~15) + 8 * (2 + STAGES);
  return (bytes + 1023) & ~1023;
}

// One 16-token chunk of the query-major backward.  Returns dS and P as bf16 fragments in
// (ds_a, p_a) for the coarse-gradient products.
__device__ __forceinline__ void dq_chunk(const uint32_t (&qf)[4][4], const uint32_t (&df)[4][4], uint32_t ktile,
                                         uint32_t vtile, int valid, float scale_log2, const float (&lse2)[2],
                                         const float (&delta)[2], float (&dq)[8][4], uint32_t (&ds_a)[4],
                                         uint32_t (&p_a)[4]) {
  const int lane = lane_id();
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float dp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  mma_a_bt(s, qf, ktile);
  mma_a_bt(dp, df, vtile);
  float p[2][4], ds[2][4];
#pragma unroll
  for (int n = 0; n < 2; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = n * 8 + 2 * (lane & 3) + (e & 1);
      const int r = e >> 1;
      p[n][e] = (col < valid) ? exp2f(s[n][e] * scale_log2 - lse2[r]) : 0.0f;
      ds[n][e] = p[n][e] * (dp[n][e] - delta[r]);
    }
  ds_a[0] = pack_bf16(ds[0][0], ds[0][1]);
  ds_a[1] = pack_bf16(ds[0][2], ds[0][3]);
  ds_a[2] = pack_bf16(ds[1][0], ds[1][1]);
  ds_a[3] = pack_bf16(ds[1][2], ds[1][3]);
  p_a[0] = pack_bf16(p[0][0], p[0][1]);
  p_a[1] = pack_bf16(p[0][2], p[0][3]);
  p_a[2] = pack_bf16(p[1][0], p[1][1]);
  p_a[3] = pack_bf16(p[1][2], p[1][3]);
  mma_a_b(dq, ds_a[0], ds_a[1], ds_a[2], ds_a[3], ktile);
}

template <int STAGES>
__global__ void __launch_bounds__(128) attn_bwd_dq_bf16_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, AttnParams P,
    const float* __restrict__ k_pyr, const float* __restrict__ v_pyr, const int* __restrict__ idx,
    const __nv_bfloat16* __restrict__ o, const float* __restrict__ lse, __nv_bfloat16* __restrict__ dq_out,
    float* __restrict__ ws) {
  extern __shared__ uint8_t dq_smem_raw[];
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n1 = g.n[1];
  const int K = g.K;
  const int total_blocks = g.BH * n1;
  const int first = (blockIdx.x * nwarps + warp) * kUnitBlocks;
  const bool active = first < total_blocks;
  const int nblk = active ? min(kUnitBlocks, total_blocks - first) : 0;
  const DqWarpMap sm = dq_warp_map<STAGES>(align1024(dq_smem_raw) + warp * P.warp_bytes, g);
  const bool has_coarse = g.L >= 2;

  for (int i = lane; i < nblk * K; i += 32)
    sm.idx[i] = checked_index(__ldg(idx + g.idx_off[1] + (long long)first * K + i), n1);
  for (int i = lane; i < 2 * g.coarse_pad * kD; i += 32) sm.cacc_k[i] = 0.0f;  // cacc_k, cacc_v contiguous
  if (lane == 0) {
    for (int b = 0; b < 2 + STAGES; ++b) mbar_init(sm.bar_qd + 8 * b, 1);
    mbar_fence_init();
  }
  __syncwarp();

  const int total_loads = nblk * K;
  auto issue_kv = [&](int seq) {
    const int gb = first + seq / K;
    const int bh = gb / n1;
    const int row = bh * g.N + sm.idx[seq] * kBlock;
    const int stage = seq % STAGES;
    const uint32_t bar = sm.bar_kv + 8 * stage;
    const uint32_t dst = sm.ring + stage * 2 * kTileBytes;
    mbar_expect_tx(bar, 2 * kTileBytes);
    tma_load_2d(dst, &tm_k, 0, row, bar);
    tma_load_2d(dst + kTileBytes, &tm_v, 0, row, bar);
  };
  auto issue_qd = [&](int i) {
    const uint32_t bar = sm.bar_qd + 8 * (i & 1);
    const int row = (first + i) * kBlock;
    const uint32_t dst = sm.qd + (i & 1) * 2 * kTileBytes;
    mbar_expect_tx(bar, 2 * kTileBytes + kBlock * 4);
    tma_load_2d(dst, &tm_q, 0, row, bar);
    tma_load_2d(dst + kTileBytes, &tm_do, 0, row, bar);
    bulk_load(smem_u32(sm.lse + (i & 1) * kBlock), lse + row, kBlock * 4, bar);
  };
  if (lane == 0 && nblk > 0) {
    issue_qd(0);
    for (int s = 0; s < min(STAGES, total_loads); ++s) issue_kv(s);
  }
  if (has_coarse && nblk > 0) {
    const int bh0 = first / n1;
    const int p0 = first - bh0 * n1;
    stage_coarse_rows(g, k_pyr, idx, bh0, p0, sm.ck);
    stage_coarse_rows(g, v_pyr, idx, bh0, p0, sm.cv);
    __syncwarp();
  }

  bool ok = true;
  int next_seq = 0, next_q = 0;
  for (int i = 0; i < nblk && ok; ++i) {
    const int gb = first + i;
    ok = __all_sync(0xffffffffu, mbar_wait(sm.bar_qd + 8 * (i & 1), (i >> 1) & 1));
    if (!ok) break;
    next_q = i + 1;
    // the other buffer was released at the end of block i-1
    if (lane == 0 && i + 1 < nblk) issue_qd(i + 1);
    const uint32_t qt = sm.qd + (i & 1) * 2 * kTileBytes;
    const uint32_t dt = qt + kTileBytes;
    uint32_t qf[4][4], df[4][4];
    load_a_frags(qt, qf);
    load_a_frags(dt, df);
    // Delta_r = sum_d dO[r][d] * O[r][d] (O from global, dO from the staged tile)
    float dlt;
    {
      const int r = lane >> 1;
      const int h = lane & 1;
      const uint4* orow = reinterpret_cast<const uint4*>(o + ((long long)gb * kBlock + r) * kD + h * 32);
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 ov = __ldg(orow + c);
        uint4 dv;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(dv.x), "=r"(dv.y), "=r"(dv.z), "=r"(dv.w)
                     : "r"(dt + swz(r, h * 4 + c)));
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
        const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(dw[e] << 16), acc);
          acc = fmaf(__uint_as_float(ow[e] & 0xffff0000u), __uint_as_float(dw[e] & 0xffff0000u), acc);
        }
      }
      dlt = acc + __shfl_xor_sync(0xffffffffu, acc, 1);
      if (h == 0) ws[W.delta + (long long)gb * kBlock + r] = dlt;
    }
    const int r0 = lane >> 2;
    const float delta[2] = {__shfl_sync(0xffffffffu, dlt, 2 * r0), __shfl_sync(0xffffffffu, dlt, 2 * r0 + 16)};
    const float lse2[2] = {sm.lse[(i & 1) * kBlock + r0] * kLog2e, sm.lse[(i & 1) * kBlock + r0 + 8] * kLog2e};

    float dq[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
    uint32_t ds_a[4], p_a[4];
    for (int s = 0; s < K; ++s) {
      const int seq = i * K + s;
      const int stage = seq % STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(sm.bar_kv + 8 * stage, (seq / STAGES) & 1));
      if (!ok) break;
      next_seq = seq + 1;
      const uint32_t kt = sm.ring + stage * 2 * kTileBytes;
      dq_chunk(qf, df, kt, kt + kTileBytes, kBlock, P.scale_log2, lse2, delta, dq, ds_a, p_a);
      __syncwarp();
      if (lane == 0 && seq + STAGES < total_loads) issue_kv(seq + STAGES);
    }
    if (!ok) break;
    for (int cc = 0; cc < g.coarse_pad / kBlock; ++cc) {
      dq_chunk(qf, df, sm.ck + cc * kTileBytes, sm.cv + cc * kTileBytes, min(kBlock, g.coarse - cc * kBlock),
               P.scale_log2, lse2, delta, dq, ds_a, p_a);
      // transposes (tokens x queries) of dS and P as A operands
      const uint32_t dt0 = movm_t(ds_a[0]), dt1 = movm_t(ds_a[2]), dt2 = movm_t(ds_a[1]), dt3 = movm_t(ds_a[3]);
      mma_a_b_smem_acc(sm.cacc_k, cc * kBlock, dt0, dt1, dt2, dt3, qt);
      const uint32_t pt0 = movm_t(p_a[0]), pt1 = movm_t(p_a[2]), pt2 = movm_t(p_a[1]), pt3 = movm_t(p_a[3]);
      mma_a_b_smem_acc(sm.cacc_v, cc * kBlock, pt0, pt1, pt2, pt3, dt);
    }
    __syncwarp();
    store_tile_bf16(dq, P.scale, P.scale, qt, dq_out + (long long)gb * kBlock * kD);
  }
  if (!ok) {
    for (int seq = next_seq; seq < min(total_loads, next_seq + STAGES); ++seq)
      mbar_wait(sm.bar_kv + 8 * (seq % STAGES), (seq / STAGES) & 1);
    for (int i = next_q; i < min(nblk, next_q + 2); ++i) mbar_wait(sm.bar_qd + 8 * (i & 1), (i >> 1) & 1);
  }
  if (!has_coarse) return;
  // ---- one level-2 group per CTA: sum the warps' coarse partials in a fixed order
  __syncthreads();
  const int group = blockIdx.x;  // = (b*H + h) * n_2 + p / 16
  if (group * kBlock >= total_blocks) return;
  uint8_t* base0 = align1024(dq_smem_raw);
  for (int e = threadIdx.x; e < g.coarse * kD; e += blockDim.x) {
    const int row = e / kD;
    const int col = e - row * kD;
    float sk = 0.f, sv = 0.f;
    for (int w = 0; w < nwarps; ++w) {
      const DqWarpMap mw = dq_warp_map<STAGES>(base0 + w * P.warp_bytes, g);
      sk += mw.cacc_k[cacc_index(row, col)];
      sv += mw.cacc_v[cacc_index(row, col)];
    }
    ws[W.part_k + (long long)group * g.coarse * kD + e] = sk;
    ws[W.part_v + (long long)group * g.coarse * kD + e] = sv;
  }
}

// Per coarse level-l token j (one warp each): sum of the group partials of every level-l
// query a in CSR row j, over the level-2 groups under a, in ascending (a, group) order.
__global__ void __launch_bounds__(128) coarse_grad_reduce_kernel(Geometry g, float scale,
                                                                 const int* __restrict__ idx,
                                                                 const int* __restrict__ row_ptr,
                                                                 const int* __restrict__ col, float* __restrict__ ws) {
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lev = 2;
  for (; lev <= g.L; ++lev) {
    const long long cnt = (long long)g.BH * g.n[lev];
    if (wid < cnt) break;
    wid -= cnt;
  }
  if (lev > g.L) return;
  const int nl = g.n[lev];
  const int K = g.K;
  const int bh = (int)(wid / nl);
  const int j = (int)(wid - (long long)bh * nl);
  int span = 1;  // level-2 groups under one level-l token: 16^(l-2)
  for (int i = 2; i < lev; ++i) span *= kBlock;
  const int* rp = row_ptr + g.rp_off[lev] + (long long)bh * (nl + 1);
  const int E = nl * K;
  int rs = rp[j], re = rp[j + 1];
  if (rs < 0 || re > E || rs > re) {
    record_error(LLSA_ERR_INTERNAL);
    rs = re = 0;
  }
  const int* cl = col + g.idx_off[lev] + (long long)bh * E;
  const int* il = idx + g.idx_off[lev] + (long long)bh * E;
  const long long n2 = g.n[2];
  float2 sk = make_float2(0.f, 0.f), sv = make_float2(0.f, 0.f);
  for (int e = rs; e < re; ++e) {
    const int a = checked_index(__ldg(cl + e), nl);
    // slot of j in the ascending list of a
    int lo = 0, hi = K - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(il + (long long)a * K + mid) < j) lo = mid + 1; else hi = mid;
    }
    if (__ldg(il + (long long)a * K + lo) != j) record_error(LLSA_ERR_INTERNAL);
    const int slot = (lev - 2) * K + lo;
    const long long g0 = (long long)bh * n2 + (long long)a * span;
    for (int gi = 0; gi < span; ++gi) {
      const long long off = ((g0 + gi) * g.coarse + slot) * kD + 2 * lane;
      const float2 x = *reinterpret_cast<const float2*>(ws + W.part_k + off);
      const float2 y = *reinterpret_cast<const float2*>(ws + W.part_v + off);
      sk.x += x.x;
      sk.y += x.y;
      sv.x += y.x;
      sv.y += y.y;
    }
  }
  const long long out = W.cg_off[lev] + ((long long)bh * nl + j) * kD + 2 * lane;
  *reinterpret_cast<float2*>(ws + W.cg_k + out) = make_float2(sk.x * scale, sk.y * scale);
  *reinterpret_cast<float2*>(ws + W.cg_v + out) = sv;
}

struct DkvWarpMap {
  uint32_t kv, ring;
  float* lse;    // [STAGES][16]
  float* delta;  // [STAGES][16]
  uint32_t bar_kv, bar_ring;
};

template <int STAGES>
__device__ __forceinline__ DkvWarpMap dkv_warp_map(uint8_t* base) {
  DkvWarpMap m;
  const uint32_t b = smem_u32(base);
  m.kv = b;
  m.ring = b + 2 * kTileBytes;
  uint8_t* p = base + 2 * kTileBytes + STAGES * 2 * kTileBytes;
  m.lse = reinterpret_cast<float*>(p);
  m.delta = m.lse + STAGES * kBlock;
  p += 2 * STAGES * kBlock * 4;
  m.bar_kv = smem_u32(p);
  m.bar_ring = m.bar_kv + 8;
  return m;
}

template <int STAGES>
inline int dkv_warp_bytes() {
  int bytes = 2 * kTileBytes + STAGES * 2 * kTileBytes + 2 * STAGES * kBlock * 4 + 8 * (1 + STAGES);
  return (bytes + 1023) & ~1023;
}

template <int STAGES>
__global__ void __launch_bounds__(128) attn_bwd_dkdv_bf16_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, AttnParams P,
    const float* __restrict__ lse, const int* __restrict__ row_ptr, const int* __restrict__ col,
    const float* __restrict__ ws, __nv_bfloat16* __restrict__ dk_out, __nv_bfloat16* __restrict__ dv_out) {
  extern __shared__ uint8_t dkv_smem_raw[];
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n1 = g.n[1];
  const int K = g.K;
  const int kb = blockIdx.x * nwarps + warp;  // flat key block (b*H + h) * n_1 + j
  if (kb >= g.BH * n1) return;               // warp-uniform; no CTA-wide barrier here
  const int bh = kb / n1;
  const int j = kb - bh * n1;
  const DkvWarpMap sm = dkv_warp_map<STAGES>(align1024(dkv_smem_raw) + warp * P.warp_bytes);

  const int E = n1 * K;
  const int* rp = row_ptr + g.rp_off[1] + (long long)bh * (n1 + 1);
  int rs = __ldg(rp + j), re = __ldg(rp + j + 1);
  if (rs < 0 || re > E || rs > re) {
    if (lane == 0) record_error(LLSA_ERR_INTERNAL);
    rs = re = 0;
  }
  const int npairs = re - rs;
  const int* cl = col + g.idx_off[1] + (long long)bh * E + rs;

  if (lane == 0) {
    for (int b = 0; b < 1 + STAGES; ++b) mbar_init(sm.bar_kv + 8 * b, 1);
    mbar_fence_init();
  }
  __syncwarp();
  auto issue_pair = [&](int i) {
    const int p = checked_index(__ldg(cl + i), n1);
    const int row = bh * g.N + p * kBlock;
    const int stage = i % STAGES;
    const uint32_t bar = sm.bar_ring + 8 * stage;
    const uint32_t dst = sm.ring + stage * 2 * kTileBytes;
    mbar_expect_tx(bar, 2 * kTileBytes + 2 * kBlock * 4);
    tma_load_2d(dst, &tm_q, 0, row, bar);
    tma_load_2d(dst + kTileBytes, &tm_do, 0, row, bar);
    bulk_load(smem_u32(sm.lse + stage * kBlock), lse + row, kBlock * 4, bar);
    bulk_load(smem_u32(sm.delta + stage * kBlock), ws + W.delta + row, kBlock * 4, bar);
  };
  if (lane == 0) {
    mbar_expect_tx(sm.bar_kv, 2 * kTileBytes);
    tma_load_2d(sm.kv, &tm_k, 0, bh * g.N + j * kBlock, sm.bar_kv);
    tma_load_2d(sm.kv + kTileBytes, &tm_v, 0, bh * g.N + j * kBlock, sm.bar_kv);
    for (int i = 0; i < min(STAGES, npairs); ++i) issue_pair(i);
  }
  float dk[8][4], dv[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  bool ok = __all_sync(0xffffffffu, mbar_wait(sm.bar_kv, 0));
  int next = 0;
  if (ok) {
    uint32_t kf[4][4], vf[4][4];
    load_a_frags(sm.kv, kf);
    load_a_frags(sm.kv + kTileBytes, vf);
    const int c2 = 2 * (lane & 3);
    for (int i = 0; i < npairs; ++i) {
      const int stage = i % STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(sm.bar_ring + 8 * stage, (i / STAGES) & 1));
      if (!ok) break;
      next = i + 1;
      const uint32_t qt = sm.ring + stage * 2 * kTileBytes;
      const uint32_t dt = qt + kTileBytes;
      float st[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float dpt[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      mma_a_bt(st, kf, qt);   // S^T: rows = keys, cols = queries
      mma_a_bt(dpt, vf, dt);  // dP^T
      const float* ls = sm.lse + stage * kBlock;
      const float* dl = sm.delta + stage * kBlock;
      float pt[2][4], dst[2][4];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qcol = n * 8 + c2 + (e & 1);
          pt[n][e] = exp2f(st[n][e] * P.scale_log2 - ls[qcol] * kLog2e);
          dst[n][e] = pt[n][e] * (dpt[n][e] - dl[qcol]);
        }
      mma_a_b(dv, pack_bf16(pt[0][0], pt[0][1]), pack_bf16(pt[0][2], pt[0][3]), pack_bf16(pt[1][0], pt[1][1]),
              pack_bf16(pt[1][2], pt[1][3]), dt);
      mma_a_b(dk, pack_bf16(dst[0][0], dst[0][1]), pack_bf16(dst[0][2], dst[0][3]), pack_bf16(dst[1][0], dst[1][1]),
              pack_bf16(dst[1][2], dst[1][3]), qt);
      __syncwarp();
      if (lane == 0 && i + STAGES < npairs) issue_pair(i + STAGES);
    }
  }
  if (!ok) {
    for (int i = next; i < min(npairs, next + STAGES); ++i) mbar_wait(sm.bar_ring + 8 * (i % STAGES), (i / STAGES) & 1);
    return;
  }
  // epilogue: scale dK, add the mean-pool adjoint of the ancestors' coarse gradients
  const int c2 = 2 * (lane & 3);
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] *= P.scale;
  int span = 1;  // 16^(l-1): level-1 blocks under one level-l token
  float wgt = 1.0f / kBlock;
  for (int lev = 2; lev <= g.L; ++lev) {
    span *= kBlock;
    wgt *= 1.0f / kBlock;  // 1 / 16^l
    const int a = j / span;
    const float* ck = ws + W.cg_k + W.cg_off[lev] + ((long long)bh * g.n[lev] + a) * kD;
    const float* cv = ws + W.cg_v + W.cg_off[lev] + ((long long)bh * g.n[lev] + a) * kD;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float2 xk = *reinterpret_cast<const float2*>(ck + n * 8 + c2);
      const float2 xv = *reinterpret_cast<const float2*>(cv + n * 8 + c2);
      dk[n][0] += wgt * xk.x;
      dk[n][1] += wgt * xk.y;
      dk[n][2] += wgt * xk.x;
      dk[n][3] += wgt * xk.y;
      dv[n][0] += wgt * xv.x;
      dv[n][1] += wgt * xv.y;
      dv[n][2] += wgt * xv.x;
      dv[n][3] += wgt * xv.y;
    }
  }
  const long long row0 = (long long)bh * g.N + (long long)j * kBlock;
  store_tile_bf16(dk, 1.0f, 1.0f, sm.kv, dk_out + row0 * kD);
  store_tile_bf16(dv, 1.0f, 1.0f, sm.kv + kTileBytes, dv_out + row0 * kD);
}

}  // namespace llsa
