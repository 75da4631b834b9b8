// Step 4b: gradient of the block-sparse attention with the selection held fixed (the
// pages train LLSA end to end; skill page "Log Linear Sparse Attention", Core Technique 3:
// the sparse index transpose serves the backward pass).
//
// No atomics.  Three kernels:
//   attn_bwd_dq_bf16_kernel      query-major.  Per query block: Delta = rowsum(dO * O),
//                                S = Q K^T, P = exp(S/sqrt(D) - LSE), dP = dO V^T,
//                                dS = P (dP - Delta), dQ = dS K / sqrt(D) over the whole KV list.
//   attn_bwd_coarse_bf16_kernel  key-major over coarse tokens.  A level-2 group's 16 query
//                                blocks share their coarse KV entries; per (group, 16-token
//                                coarse tile) it sums dS^T Q and P^T dO over the group's 256
//                                queries and writes one fp32 partial per (group, coarse slot).
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
  // bf16 path: per query block [B*H*n_1][32] = its 16 LSE * log2(e) then its 16 Delta, in
  // the block's shared-memory tile-row order (written by dQ; one 128-byte copy per pair in
  // the key-major kernels).  fp32 path: Delta [B*H*N] in the first half.
  long long lsd;
  long long part_k, part_v; // [B*H*n_2][C][64]
  long long cg_k, cg_v;     // coarse gradients, level-major [l=2..L][B*H*n_l][64]
  long long cg_off[kMaxLevels + 1];
  long long order;          // int4 [B*H*n_1] {key block, CSR row start, row end, 0}, longest row first
  long long order_counts;   // int32 [kOrdClasses][order tiles]
  long long order_nonempty; // int32: rows with at least one query block (they come first)
  long long barrier;        // uint32[16]: the grid-barrier counter of the fused pyramid + selection
  long long total;
};

// Longest-first order of the fine key blocks for the key-major dK/dV kernel: its CTAs are
// scheduled roughly in launch order, and a row of up to ~150 query blocks started last would
// run alone long after the rest.  Rows are grouped into classes by floor(log2(length))
// (class 0: >= 128 query blocks, ..., class 7: one, class 8: empty), stable within a class.
constexpr int kOrdClasses = 9;
constexpr int kOrdThreads = 256;
constexpr int kOrdRowsPerThread = 8;
constexpr int kOrdTile = kOrdThreads * kOrdRowsPerThread;

__host__ __device__ inline int order_tiles(const Geometry& g) { return (g.BH * g.n[1] + kOrdTile - 1) / kOrdTile; }

__host__ __device__ inline BwdWorkspace bwd_workspace_layout(const Geometry& g) {
  auto up = [](long long x) { return (x + 63) & ~63LL; };
  BwdWorkspace w{};
  long long off = 0;
  w.lsd = off;
  off = up(off + 2LL * g.BH * g.N);
  const long long parts = g.L >= 2 ? (long long)g.BH * g.n[2] * g.coarse * g.D : 0;
  w.part_k = off;
  off = up(off + parts);
  w.part_v = off;
  off = up(off + parts);
  long long cg = 0;
  for (int l = 0; l <= kMaxLevels; ++l) w.cg_off[l] = 0;
  for (int l = 2; l <= g.L; ++l) {
    w.cg_off[l] = cg;
    cg += (long long)g.BH * g.n[l] * g.D;
  }
  w.cg_k = off;
  off = up(off + cg);
  w.cg_v = off;
  off = up(off + cg);
  w.order = off;
  off = up(off + 4LL * g.BH * g.n[1]);
  w.order_counts = off;
  off = up(off + (long long)kOrdClasses * order_tiles(g));
  w.order_nonempty = off;
  off = up(off + 1);
  w.barrier = off;
  off = up(off + 16);
  w.total = off;
  return w;
}

// bf16 under LLSA_FLAG_GRID_ORDER (g.zcopy) the host places after that layout the one-call
// step's quadtree-ordered copies of q, k, v, dO ([B*H*N][D] bf16 each) and of LSE ([B*H*N]
// fp32).  The kernels get their addresses as arguments, so the layout they compute (every
// thread, at start) stays as small as it was.
inline long long bwd_workspace_floats(const Geometry& g) {
  const long long base = bwd_workspace_layout(g).total;
  if (!g.zcopy) return base;
  const long long zt = (long long)g.BH * g.N * g.D / 2;  // one bf16 tensor, in floats (D is even)
  return base + ((4 * zt + (long long)g.BH * g.N + 63) & ~63LL);
}

// ---------------------------------------------------------------------------- query-major dQ

// At D = 128 dQ keeps one [Q, dO] tile pair per warp and reads the Q and dO operands from it
// at each k-step ("lean"): the pair of buffers took 136 KB of shared memory per CTA (one CTA,
// 4 warps per SM) and the fragments 64 registers; lean, 2 CTAs fit (dQ 331 -> 255 us at the
// 6-head 65536-token shape).  At D = 64 the double buffer and register fragments are faster
// (the lean form measured 126 against 115 us there, even at 16 warps per SM).
template <int D>
__host__ __device__ constexpr bool dq_lean() {
  return D == 128;
}

// The Q and dO operands of dQ's score products: fragments in registers, or (LEAN) the two
// shared-memory tiles, read at each k-step.
template <int D, bool LEAN>
struct QdOps;
template <int D>
struct QdOps<D, false> {
  uint32_t qf[D / 16][4], df[D / 16][4];
  __device__ __forceinline__ void load(uint32_t qt, uint32_t dt, int perm) {
    load_a_frags<D>(qt, qf, perm);
    load_a_frags<D>(dt, df, perm);
  }
  __device__ __forceinline__ void scores(float (&s)[2][4], float (&dp)[2][4], uint32_t ktile, uint32_t vtile,
                                         int bperm) const {
    mma_a_bt<D>(s, qf, ktile, bperm);
    mma_a_bt<D>(dp, df, vtile, bperm);
  }
};
template <int D>
struct QdOps<D, true> {
  uint32_t qt, dt;
  int aperm;
  __device__ __forceinline__ void load(uint32_t q, uint32_t d, int perm) {
    qt = q;
    dt = d;
    aperm = perm;
  }
  __device__ __forceinline__ void scores(float (&s)[2][4], float (&dp)[2][4], uint32_t ktile, uint32_t vtile,
                                         int bperm) const {
    mma_at_bt<D>(s, qt, ktile, aperm, bperm);
    mma_at_bt<D>(dp, dt, vtile, aperm, bperm);
  }
};

template <int D, int STAGES>
__host__ __device__ inline CtaSmem dq_smem(const Geometry& g, int nwarps) {
  CtaSmem c;
  c.coarse_bytes = 2 * g.coarse_pad * D * 2;
  // [2][Q, dO] (one [Q, dO] pair at D = 128, see dq_lean) + ring of [K, V]
  c.warp_tiles = (dq_lean<D>() ? 2 : 4) * tile_bytes<D>() + STAGES * 2 * tile_bytes<D>();
  c.warp_tail = 2 * kBlock * 4 + ((kUnitBlocks * g.K * 4 + 15) & ~15) + ((8 * (2 + STAGES) + 15) & ~15);
  c.nwarps = nwarps;
  return c;
}

// One 16-token chunk of the query-major backward: dQ += dS K with dS = P (dP - Delta).
// POOL (level-1 variant, fine chunks): the block-mean entry has score mean(S) + pool_bias
// and dP mean(dP); its dS, times the mean K row, is dS / 16 added to each of the 16 dS.
// MASK, cmask, CAUSAL and shift as in fwd_chunk (masked entries get P = 0, hence dS = 0).
// ops: the block's Q and dO operands (QdOps).
template <int D, bool MASK, bool POOL = false, bool CAUSAL = false, class Ops>
__device__ __forceinline__ void dq_chunk(const Ops& ops,
                                         uint32_t ktile, uint32_t vtile, int valid, float scale_log2,
                                         const float (&lse2)[2], const float (&delta)[2], float (&dq)[D / 8][4],
                                         const Geometry* bias_g = nullptr, int c0 = 0, float pool_bias = 0.f,
                                         int perm = 0, uint32_t cmask = 0xffffffffu, int shift = 15) {
  const int lane = lane_id();
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float dp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  ops.scores(s, dp, ktile, vtile, perm);
  float pds[2] = {0.f, 0.f};  // pooled entry's dS / 16, rows r0 and r0 + 8
  if (POOL) {
    float t[2], u[2];
    quad_row_sums(s, t[0], t[1]);
    quad_row_sums(dp, u[0], u[1]);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float pb = ex2(fmaf(fmaf(t[r], 1.0f / kBlock, pool_bias), scale_log2, -lse2[r]));
      pds[r] = pb * fmaf(u[r], 1.0f / kBlock, -delta[r]) * (1.0f / kBlock);
    }
  }
  float ds[2][4];
#pragma unroll
  for (int n = 0; n < 2; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = n * 8 + 2 * (lane & 3) + (e & 1);
      const int r = e >> 1;
      float sb = s[n][e];
      if (MASK && bias_g && bias_g->log_bias && col < valid) sb += coarse_log_bias(*bias_g, c0 + col) * sqrt_d<D>();
      const bool vis =
          (!MASK || (col < valid && ((cmask >> col) & 1u))) && (!CAUSAL || col <= (lane >> 2) + 8 * r + shift);
      const float p = vis ? ex2(fmaf(sb, scale_log2, -lse2[r])) : 0.0f;
      ds[n][e] = POOL ? fmaf(p, dp[n][e] - delta[r], pds[r]) : p * (dp[n][e] - delta[r]);
    }
  mma_a_b<D>(dq, pack_bf16(ds[0][0], ds[0][1]), pack_bf16(ds[0][2], ds[0][3]), pack_bf16(ds[1][0], ds[1][1]),
             pack_bf16(ds[1][2], ds[1][3]), ktile, perm);
}

// Same CTA shape as the forward: 4 warps x 4 query blocks, coarse KV staged once per CTA.
// POOL: the level-1 variant (see dq_chunk).  LAYOUT (see Layout): under kPadded the fine
// tile that holds the last real token masks its padding keys; padding queries (zero Q and
// dO rows, O = 0, LSE = 0) get dS = 0 and so dQ = 0 and Delta = 0 without a mask.
template <int D, int STAGES, bool POOL, int LAYOUT>
__global__ void __launch_bounds__(128, D == 64 ? 3 : 2) attn_bwd_dq_bf16_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, AttnParams P,
    const float* __restrict__ k_pyr, const float* __restrict__ v_pyr, const int* __restrict__ idx,
    const __nv_bfloat16* __restrict__ o, const float* __restrict__ lse, __nv_bfloat16* __restrict__ dq_out,
    float* __restrict__ ws) {
  // the coarse tiles come from the pyramid and the coarser selection levels, two or more
  // kernels back, so they are staged before waiting for the kernel ahead (see pdl_wait)
  extern __shared__ uint8_t dq_smem_raw[];
  constexpr bool PAD = LAYOUT == kPadded;
  constexpr bool CAUSAL = LAYOUT == kCausal;
  constexpr int PERM = LAYOUT == kGrid ? 1 : 0;
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n1 = g.n[1];
  const int K = g.K;
  const int total_blocks = g.BH * n1;
  const CtaSmem cs = dq_smem<D, STAGES>(g, nwarps);
  constexpr int TB = tile_bytes<D>();
  uint8_t* base = align1024(dq_smem_raw);
  const uint32_t ck = smem_u32(base);
  const uint32_t cv = ck + g.coarse_pad * D * 2;
  const int cta_first = blockIdx.x * nwarps * kUnitBlocks;
  if (g.L >= 2) {
    const int bh0 = cta_first / n1;
    const int p0 = cta_first - bh0 * n1;
    stage_coarse_rows<D>(g, k_pyr, idx, bh0, p0, ck, threadIdx.x, blockDim.x);
    stage_coarse_rows<D>(g, v_pyr, idx, bh0, p0, cv, threadIdx.x, blockDim.x);
    __syncthreads();
  }
  const uint32_t cmask =
      (CAUSAL && g.L >= 2) ? coarse_visible_mask(g, idx, cta_first / n1, cta_first % n1) : 0xffffffffu;
  const int first = cta_first + warp * kUnitBlocks;
  if (first >= total_blocks) {  // warp-uniform; no CTA-wide barrier after this point
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int nblk = min(kUnitBlocks, total_blocks - first);
  constexpr bool LEAN = dq_lean<D>();
  const uint32_t qd = smem_u32(cs.tiles(base, warp));
  const uint32_t ring = qd + (LEAN ? 2 : 4) * TB;  // after the [Q, dO] pair(s) (dq_smem)
  float* slse = reinterpret_cast<float*>(cs.tail(base, warp));  // [2][16]
  int* srow = reinterpret_cast<int*>(slse + 2 * kBlock);
  const uint32_t bar_qd = smem_u32(srow) + ((kUnitBlocks * K * 4 + 15) & ~15);
  const uint32_t bar_kv = bar_qd + 16;

  for (int i = lane; i < nblk * K; i += 32) {
    // the first K/V row of each load: (b*H + h) * N + 16 j, computed here off the issue path
    // (a causal kNoPick entry: the complement of the block's own first row, as in the forward)
    const int pick = __ldg(idx + g.idx_off[1] + (long long)first * K + i);
    const int qb = first + div_k(g, i);
    if (CAUSAL && pick == kNoPick)
      srow[i] = ~(qb * kBlock);
    else
      srow[i] = div_n1(g, qb) * g.N + checked_index(pick, n1) * kBlock;
  }
  if (lane == 0) {
    for (int b = 0; b < 2 + STAGES; ++b) mbar_init(bar_qd + 8 * b, 1);
    mbar_fence_init();
  }
  __syncwarp();

  const int total_loads = nblk * K;
  auto issue_kv = [&](int seq) {
    const int row = CAUSAL ? max(srow[seq], ~srow[seq]) : srow[seq];
    const int stage = seq % STAGES;
    const uint32_t bar = bar_kv + 8 * stage;
    const uint32_t dst = ring + stage * 2 * TB;
    mbar_expect_tx(bar, 2 * TB);
    tma_load_tile<D, LAYOUT>(dst, &tm_k, g, row, bar);
    tma_load_tile<D, LAYOUT>(dst + TB, &tm_v, g, row, bar);
  };
  // block i's Q/dO tiles: buffer i % 2, or (LEAN) the one buffer, which block i+1's tiles
  // enter once block i has finished with it; the two mbarriers and LSE slots alternate
  auto qd_tiles = [&](int i) { return LEAN ? qd : qd + (i & 1) * 2 * TB; };
  auto issue_qd = [&](int i) {
    const uint32_t bar = bar_qd + 8 * (i & 1);
    const int row = (first + i) * kBlock;
    const uint32_t dst = qd_tiles(i);
    mbar_expect_tx(bar, 2 * TB + kBlock * 4);
    tma_load_tile<D, LAYOUT>(dst, &tm_q, g, row, bar);
    tma_load_tile<D, LAYOUT>(dst + TB, &tm_do, g, row, bar);
    bulk_load_block_rows<LAYOUT>(smem_u32(slse + (i & 1) * kBlock), lse, g, row, bar);
  };
  // the level-1 selection (two kernels back) and K, V are ready: the first K/V tiles are
  // requested before waiting; Q/dO/LSE and O follow the forward, the kernel ahead
  if (lane == 0)
    for (int s = 0; s < min(STAGES, total_loads); ++s) issue_kv(s);
  pdl_wait();
  pdl_launch_dependents();
  if (lane == 0) issue_qd(0);

  bool ok = true;
  int next_seq = 0, next_q = 0, q_issued = 1;
  // O rows of a block (lane: shared-memory tile row lane/2, channels (lane%2) * D/2 onwards;
  // the row's token is tile_row of it).  At D = 64 they are loaded one block ahead; at
  // D = 128 (twice the registers) when the block starts.
  constexpr int OC = D / 16;  // 16-byte chunks per lane
  constexpr bool kPrefetchO = D == 64;
  auto load_o = [&](int i, uint4 (&dst)[OC]) {
    const int bhi = div_n1(g, first + i);
    const long long orow_i = token_row<LAYOUT>(g, bhi, (first + i - bhi * n1) * kBlock + tile_row(lane >> 1, PERM));
    const uint4* orow = reinterpret_cast<const uint4*>(o + orow_i * D + (lane & 1) * (D / 2));
#pragma unroll
    for (int c = 0; c < OC; ++c) dst[c] = __ldg(orow + c);
  };
  uint4 onext[OC];
  if constexpr (kPrefetchO) load_o(0, onext);
  for (int i = 0; i < nblk && ok; ++i) {
    const int gb = first + i;
    uint4 ocur[OC];
    if constexpr (kPrefetchO) {
#pragma unroll
      for (int c = 0; c < OC; ++c) ocur[c] = onext[c];
      if (i + 1 < nblk) load_o(i + 1, onext);
    } else {
      load_o(i, ocur);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(bar_qd + 8 * (i & 1), (i >> 1) & 1));
    if (!ok) break;
    next_q = i + 1;
    // with two buffers the other one was released at the end of block i-1
    if (!LEAN && i + 1 < nblk) {
      if (lane == 0) issue_qd(i + 1);
      q_issued = i + 2;
    }
    const uint32_t qt = qd_tiles(i);
    const uint32_t dt = qt + TB;
    QdOps<D, LEAN> ops;
    ops.load(qt, dt, PERM);
    // Delta_r = sum_d dO[r][d] * O[r][d] (O from registers, dO from the staged tile)
    float dlt;
    {
      const int r = lane >> 1;
      const int h = lane & 1;
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < OC; ++c) {
        const uint4 ov = ocur[c];
        uint4 dv;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(dv.x), "=r"(dv.y), "=r"(dv.z), "=r"(dv.w)
                     : "r"(dt + tswz(r, h * OC + c)));
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
        const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(dw[e] << 16), acc);
          acc = fmaf(__uint_as_float(ow[e] & 0xffff0000u), __uint_as_float(dw[e] & 0xffff0000u), acc);
        }
      }
      dlt = acc + __shfl_xor_sync(0xffffffffu, acc, 1);
      // the block's record for the key-major kernels: lanes 0-15 LSE * log2(e), 16-31 Delta
      const float drow = __shfl_sync(0xffffffffu, dlt, 2 * (lane & 15));
      ws[W.lsd + (long long)gb * 2 * kBlock + lane] = lane < kBlock ? slse[(i & 1) * kBlock + lane] * kLog2e : drow;
    }
    // Delta and LSE are in shared-memory tile-row order: row r0 of the fragments is tile row p0
    const int r0 = lane >> 2;
    const int p0 = tile_row(r0, PERM);
    const float delta[2] = {__shfl_sync(0xffffffffu, dlt, 2 * p0), __shfl_sync(0xffffffffu, dlt, 2 * p0 + 16)};
    const float lse2[2] = {slse[(i & 1) * kBlock + p0] * kLog2e, slse[(i & 1) * kBlock + p0 + 8] * kLog2e};

    float dq[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
#pragma unroll kQmUnroll
    for (int s = 0; s < K; ++s) {
      const int seq = i * K + s;
      const int stage = seq % STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_kv + 8 * stage, (seq / STAGES) & 1));
      if (!ok) break;
      next_seq = seq + 1;
      const uint32_t kt = ring + stage * 2 * TB;
      if (PAD)  // real keys of this tile: 16 except in the one that holds the last real token
        dq_chunk<D, true>(ops, kt, kt + TB, min(kBlock, g.nv - (srow[seq] - div_n1(g, gb) * g.N)), P.scale_log2,
                          lse2, delta, dq);
      else if (CAUSAL) {  // kNoPick: every key masked; the block's own keys: the causal diagonal
        const int r = srow[seq];
        dq_chunk<D, false, false, true>(ops, kt, kt + TB, kBlock, P.scale_log2, lse2, delta, dq, nullptr, 0, 0.f, 0,
                                        0xffffffffu, r < 0 ? -kBlock : (r == gb * kBlock ? 0 : kBlock - 1));
      } else
        dq_chunk<D, false, POOL>(ops, kt, kt + TB, kBlock, P.scale_log2, lse2, delta, dq, nullptr, 0,
                                 pool_log_bias<D>(g), PERM);
      __syncwarp();
      if (lane == 0 && seq + STAGES < total_loads) issue_kv(seq + STAGES);
    }
    if (!ok) break;
    for (int cc = 0; cc < g.coarse_pad / kBlock; ++cc)
      dq_chunk<D, true>(ops, ck + cc * TB, cv + cc * TB, min(kBlock, g.coarse - cc * kBlock), P.scale_log2, lse2,
                        delta, dq, &g, cc * kBlock, 0.f, 0, cmask >> (cc * kBlock));
    __syncwarp();
    {
      const int bhi = div_n1(g, gb);
      store_tile_bf16<D, LAYOUT>(dq, P.scale, P.scale, qt, dq_out, g, bhi, (gb - bhi * n1) * kBlock);
    }
    // LEAN: the one Q/dO buffer (and the staging use above) is done with: request the next
    // block's tiles (store_tile_bf16 ordered its generic accesses before this async copy)
    if (LEAN && i + 1 < nblk) {
      if (lane == 0) issue_qd(i + 1);
      q_issued = i + 2;
    }
  }
  if (!ok) {
    for (int seq = next_seq; seq < min(total_loads, next_seq + STAGES); ++seq)
      mbar_wait(bar_kv + 8 * (seq % STAGES), (seq / STAGES) & 1);
    for (int i = next_q; i < q_issued; ++i) mbar_wait(bar_qd + 8 * (i & 1), (i >> 1) & 1);
  }
}

// ---------------------------------------------------------------------------- key-major pairs

// One (key tile, query block) pair: with the key tile's K and V as A fragments (rows = keys),
// and the query block's Q and dO tiles, LSE and Delta staged:
//   S^T = K Q^T, P^T = exp2(S^T*scale*log2e - LSE*log2e), dP^T = V dO^T,
//   dS^T = P^T (dP^T - Delta), dV += P^T dO, dK += dS^T Q  (dK unscaled; P^T and dS^T as
//   bf16 hi + lo pairs).
// It runs as two phases: kv_scores (S^T, dP^T and the elementwise step) and kv_accumulate
// (the dV, dK products).  At D = 64 the key tile's K and V fragments stay in registers; at
// D = 128 (twice the accumulators) they are read from the staged tile at each k-step.
// BIAS: the key rows are coarse tokens under the log-count variant; kb[0], kb[1] are the
// biases (unscaled-dot units) of this lane's key rows r0 and r0 + 8.
// POOL (level-1 variant; the key rows are a fine block): the block-mean entry, with score
// mean over the 16 keys of S + pool_bias and dP the mean of dP, sends dV_mean = p dO and
// dK_mean = dS q to the block's 16 rows with weight 1/16 each: p / 16 is added to every
// P^T entry of its query column and dS / 16 to every dS^T entry.
template <int D>
__host__ __device__ constexpr bool kv_frags_in_regs() {
  return D == 64;
}

// kvalid < 16: the key tile holds the last real token of a padded sequence, and its rows
// from kvalid on are padding (zero rows) whose P^T and dS^T are masked to 0.
// kvperm, qperm: the tile_row permutations of the key tile and of the query block's tiles.
// kmask: key rows whose bit is clear are not attended (causal coarse entries); diag: the
// causal diagonal pair (key row r is visible to query column c only when r <= c).
// lsd: the query block's record (16 LSE * log2(e), then 16 Delta, in the shared-memory row
// order of its tiles).
template <int D, bool BIAS = false, bool POOL = false>
__device__ __forceinline__ void kv_scores(const uint32_t (&kf)[D / 16][4], const uint32_t (&vf)[D / 16][4],
                                          uint32_t kvtile, uint32_t qt, uint32_t dt, const float* lsd,
                                          float scale_log2, float (&pt)[2][4], float (&dst)[2][4],
                                          const float (&kb)[2], float pool_bias, int kvalid, int kvperm,
                                          int qperm, uint32_t kmask = 0xffffu, bool diag = false) {
  const int c2 = 2 * (lane_id() & 3);
  float st[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float dpt[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  if constexpr (kv_frags_in_regs<D>()) {
    mma_a_bt<D>(st, kf, qt, qperm);   // S^T: rows = keys, cols = queries
    mma_a_bt<D>(dpt, vf, dt, qperm);  // dP^T
  } else {
    mma_at_bt<D>(st, kvtile, qt, kvperm, qperm);
    mma_at_bt<D>(dpt, kvtile + tile_bytes<D>(), dt, kvperm, qperm);
  }
  // this lane's four query columns: c2, c2 + 1 (n = 0) and c2 + 8, c2 + 9 (n = 1); the tile
  // row permutation keeps bit 0, so each pair stays adjacent
  const int pc = tile_row(c2, qperm);
  const float2 l0 = *reinterpret_cast<const float2*>(lsd + pc);
  const float2 l1 = *reinterpret_cast<const float2*>(lsd + 8 + pc);
  const float2 d0 = *reinterpret_cast<const float2*>(lsd + kBlock + pc);
  const float2 d1 = *reinterpret_cast<const float2*>(lsd + kBlock + 8 + pc);
  const float lq[2][2] = {{l0.x, l0.y}, {l1.x, l1.y}};
  const float dq[2][2] = {{d0.x, d0.y}, {d1.x, d1.y}};
  float pa[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, da[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // pooled p/16, dS/16
  if (POOL) {
    // column sums over the 16 key rows: this lane's rows r0, r0 + 8, then the 8 row groups
    float ts[2][2], tp[2][2];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        ts[n][c] = st[n][c] + st[n][2 + c];
        tp[n][c] = dpt[n][c] + dpt[n][2 + c];
      }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1)
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          ts[n][c] += __shfl_xor_sync(0xffffffffu, ts[n][c], off);
          tp[n][c] += __shfl_xor_sync(0xffffffffu, tp[n][c], off);
        }
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float pb = ex2(fmaf(fmaf(ts[n][c], 1.0f / kBlock, pool_bias), scale_log2, -lq[n][c]));
        pa[n][c] = pb * (1.0f / kBlock);
        da[n][c] = pa[n][c] * fmaf(tp[n][c], 1.0f / kBlock, -dq[n][c]);
      }
  }
#pragma unroll
  for (int n = 0; n < 2; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      pt[n][e] = ex2(fmaf(BIAS ? st[n][e] + kb[e >> 1] : st[n][e], scale_log2, -lq[n][e & 1]));
      dst[n][e] = pt[n][e] * (dpt[n][e] - dq[n][e & 1]);
      if (POOL) {
        pt[n][e] += pa[n][e & 1];
        dst[n][e] += da[n][e & 1];
      }
    }
  if (kvalid < kBlock || kmask != 0xffffu || diag) {
    const int r0 = lane_id() >> 2;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kr = r0 + 8 * (e >> 1);  // key row; the query column is n * 8 + c2 + (e & 1)
        if (kr >= kvalid || !((kmask >> kr) & 1u) || (diag && kr > n * 8 + c2 + (e & 1)))
          pt[n][e] = dst[n][e] = 0.0f;
      }
  }
}

// dV += P^T dO and dK += dS^T Q for one pair.  P^T and dS^T enter the products as two bf16
// terms each (value and rounding remainder).  A key's dV and dK sum P dO and dS q over every
// query that selected it; with P and dS rounded once to bf16 (relative error 2^-9 per term)
// the error of a key picked by hundreds of query blocks grew past the output tolerance (for
// dK the terms also cancel: the dS of a query sum to zero, so |dK| stays moderate while its
// error grows).
template <int D>
__device__ __forceinline__ void kv_accumulate(const float (&pt)[2][4], const float (&dst)[2][4], uint32_t qt,
                                              uint32_t dt, float (&dk)[D / 8][4], float (&dv)[D / 8][4], int qperm) {
  uint32_t phi[4], plo[4], dhi[4], dlo[4];
  split_bf16(pt[0][0], pt[0][1], phi[0], plo[0]);
  split_bf16(pt[0][2], pt[0][3], phi[1], plo[1]);
  split_bf16(pt[1][0], pt[1][1], phi[2], plo[2]);
  split_bf16(pt[1][2], pt[1][3], phi[3], plo[3]);
  split_bf16(dst[0][0], dst[0][1], dhi[0], dlo[0]);
  split_bf16(dst[0][2], dst[0][3], dhi[1], dlo[1]);
  split_bf16(dst[1][0], dst[1][1], dhi[2], dlo[2]);
  split_bf16(dst[1][2], dst[1][3], dhi[3], dlo[3]);
  // both high halves first, then both low halves: an accumulator's second product is issued
  // 16 MMAs after its first rather than 8 (same order per accumulator, so the same sums)
  mma_a_b<D>(dv, phi[0], phi[1], phi[2], phi[3], dt, qperm);
  mma_a_b<D>(dk, dhi[0], dhi[1], dhi[2], dhi[3], qt, qperm);
  mma_a_b<D>(dv, plo[0], plo[1], plo[2], plo[3], dt, qperm);
  mma_a_b<D>(dk, dlo[0], dlo[1], dlo[2], dlo[3], qt, qperm);
}

// Per-warp shared memory of the key-major kernels: the key tile's K and V, then a ring of
// STAGES (Q tile, dO tile) stages; the tail holds LSE/Delta of each stage and the mbarriers.
template <int D, int STAGES>
__host__ __device__ inline CtaSmem kv_smem(int nwarps) {
  CtaSmem c;
  c.coarse_bytes = 0;
  c.warp_tiles = 2 * tile_bytes<D>() + STAGES * 2 * tile_bytes<D>();
  c.warp_tail = 2 * STAGES * kBlock * 4 + ((8 * (1 + STAGES) + 15) & ~15);
  c.nwarps = nwarps;
  return c;
}

// Streams the query blocks list[0..npairs) of one key tile through the warp's ring and
// accumulates dK, dV.  `pair_block(i)` gives the flat query-block index of pair i.  If
// `bar_tile` is non-zero the key tile is still arriving on that mbarrier (phase 0) and is
// waited for after the first pair loads are issued.  Returns false (after draining the
// copies in flight) if a wait timed out.  kmask: see kv_scores.  diag_first (kCausal): pair
// 0 is the key block's own query block (a causal CSR row lists only query blocks at or after
// its key block, ascending, so the diagonal pair can only come first).
template <int D, int STAGES, int LAYOUT, bool BIAS = false, bool POOL = false, class PairBlock>
__device__ __forceinline__ bool kv_stream(const Geometry& g, const CUtensorMap* tm_q, const CUtensorMap* tm_do,
                                          const float* __restrict__ lsd, uint32_t kvtile, uint32_t bar_tile,
                                          uint32_t ring, float* slsd,
                                          uint32_t bar_ring, int npairs, PairBlock pair_block, float scale_log2,
                                          float (&dk)[D / 8][4], float (&dv)[D / 8][4],
                                          const float (&kbias)[2] = {0.f, 0.f}, float pool_bias = 0.f,
                                          int kvalid = kBlock, int kvperm = 0, uint32_t kmask = 0xffffu,
                                          bool diag_first = false) {
  constexpr int TB = tile_bytes<D>();
  constexpr int qperm = LAYOUT == kGrid ? 1 : 0;
  const int lane = lane_id();
  // called by the whole warp (pair_block may shuffle); lane 0 issues the copies
  auto issue_pair = [&](int i) {
    const int row = pair_block(i) * kBlock;
    if (lane == 0) {
      const int stage = i % STAGES;
      const uint32_t bar = bar_ring + 8 * stage;
      const uint32_t dst = ring + stage * 2 * TB;
      mbar_expect_tx(bar, 2 * TB + 2 * kBlock * 4);
      tma_load_tile<D, LAYOUT>(dst, tm_q, g, row, bar);
      tma_load_tile<D, LAYOUT>(dst + TB, tm_do, g, row, bar);
      bulk_load(smem_u32(slsd + stage * 2 * kBlock), lsd + 2LL * row, 2 * kBlock * 4, bar);
    }
  };
  for (int i = 0; i < min(STAGES, npairs); ++i) issue_pair(i);
  if (bar_tile != 0u && !__all_sync(0xffffffffu, mbar_wait(bar_tile, 0))) {
    for (int j = 0; j < min(npairs, STAGES); ++j) mbar_wait(bar_ring + 8 * (j % STAGES), (j / STAGES) & 1);
    return false;
  }
  uint32_t kf[D / 16][4], vf[D / 16][4];
  if constexpr (kv_frags_in_regs<D>()) {
    load_a_frags<D>(kvtile, kf, kvperm);
    load_a_frags<D>(kvtile + TB, vf, kvperm);
  }
#pragma unroll kKvUnroll
  for (int i = 0; i < npairs; ++i) {
    const int stage = i % STAGES;
    if (!__all_sync(0xffffffffu, mbar_wait(bar_ring + 8 * stage, (i / STAGES) & 1))) {
      for (int j = i; j < min(npairs, i + STAGES); ++j) mbar_wait(bar_ring + 8 * (j % STAGES), (j / STAGES) & 1);
      return false;
    }
    const uint32_t qt = ring + stage * 2 * TB;
    float pt[2][4], dst[2][4];
    kv_scores<D, BIAS, POOL>(kf, vf, kvtile, qt, qt + TB, slsd + stage * 2 * kBlock, scale_log2, pt, dst, kbias,
                             pool_bias, kvalid, kvperm, qperm, kmask,
                             LAYOUT == kCausal && i == 0 && diag_first);
    kv_accumulate<D>(pt, dst, qt, qt + TB, dk, dv, qperm);
    __syncwarp();
    if (i + STAGES < npairs) issue_pair(i + STAGES);
  }
  return true;
}

// Coarse-token partial gradients.  One warp per (level-2 group, 16-token coarse tile): the
// pairs are the group's 16 query blocks.  Rows >= C of the last tile are padding and are not
// written.  Output: part_k / part_v [group][C][D] fp32 (dK unscaled).  LAYOUT: see Layout.
template <int D, int STAGES, int LAYOUT>
__global__ void __launch_bounds__(32) attn_bwd_coarse_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                  const __grid_constant__ CUtensorMap tm_do,
                                                                  AttnParams P, const float* __restrict__ k_pyr,
                                                                  const float* __restrict__ v_pyr,
                                                                  const int* __restrict__ idx,
                                                                  float* __restrict__ ws) {
  // coarse rows are staged before waiting (two or more kernels back; see pdl_wait)
  extern __shared__ uint8_t co_smem_raw[];
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int tiles = g.coarse_pad / kBlock;
  const int group = blockIdx.x / tiles;  // (b*H + h) * n_2 + a
  const int tile = blockIdx.x - group * tiles;
  const int n1 = g.n[1];
  const int first_block = group * kBlock;  // flat index of the group's first query block
  const int bh = first_block / n1;
  const int p0 = first_block - bh * n1;
  const CtaSmem cs = kv_smem<D, STAGES>(1);
  constexpr int TB = tile_bytes<D>();
  uint8_t* base = align1024(co_smem_raw);
  const uint32_t kvt = smem_u32(cs.tiles(base, 0));
  const uint32_t ring = kvt + 2 * TB;
  float* slsd = reinterpret_cast<float*>(cs.tail(base, 0));  // [STAGES][32] LSE + Delta records
  const uint32_t bar_ring = smem_u32(slsd + STAGES * 2 * kBlock);

  // stage this tile's 16 coarse K and V rows (bf16) like the forward does
  {
    constexpr int CH = D / 8;
    for (int t = lane; t < kBlock * CH; t += 32) {
      const int r = t / CH;
      const int ch = t - r * CH;
      const int row = tile * kBlock + r;
      uint4 pk = make_uint4(0u, 0u, 0u, 0u), pv = make_uint4(0u, 0u, 0u, 0u);
      int lev;
      const int j = row < g.coarse ? coarse_token(g, idx, bh, p0, row, lev) : -1;
      if (j >= 0) {  // entries past C and causal entries that are not attended stay zero
        const int nl = g.n[lev];
        const long long off = g.pyr_off[lev] + ((long long)bh * nl + j) * D + ch * 8;
        const float4 a = __ldg(reinterpret_cast<const float4*>(k_pyr + off));
        const float4 b = __ldg(reinterpret_cast<const float4*>(k_pyr + off) + 1);
        const float4 c = __ldg(reinterpret_cast<const float4*>(v_pyr + off));
        const float4 d = __ldg(reinterpret_cast<const float4*>(v_pyr + off) + 1);
        pk = make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
        pv = make_uint4(pack_bf16(c.x, c.y), pack_bf16(c.z, c.w), pack_bf16(d.x, d.y), pack_bf16(d.z, d.w));
      }
      asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(kvt + tswz(r, ch)), "r"(pk.x), "r"(pk.y),
                   "r"(pk.z), "r"(pk.w)
                   : "memory");
      asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(kvt + TB + tswz(r, ch)), "r"(pv.x),
                   "r"(pv.y), "r"(pv.z), "r"(pv.w)
                   : "memory");
    }
  }
  const uint32_t cmask = LAYOUT == kCausal ? coarse_visible_mask(g, idx, bh, p0) : 0xffffffffu;
  if (lane == 0) {
    for (int b = 0; b < STAGES; ++b) mbar_init(bar_ring + 8 * b, 1);
    mbar_fence_init();
  }
  __syncwarp();
  pdl_wait();  // LSE and Delta (the pairs' inputs) come from the kernels ahead
  pdl_launch_dependents();
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;
  bool ok;
  if (g.log_bias) {  // this lane's key rows are coarse entries tile * 16 + r0 and + 8
    const int r0 = tile * kBlock + (lane >> 2);
    const float kb[2] = {r0 < g.coarse ? coarse_log_bias(g, r0) * sqrt_d<D>() : 0.f,
                         r0 + 8 < g.coarse ? coarse_log_bias(g, r0 + 8) * sqrt_d<D>() : 0.f};
    ok = kv_stream<D, STAGES, LAYOUT, true>(g, &tm_q, &tm_do, ws + W.lsd, kvt, 0u, ring, slsd, bar_ring, kBlock,
                                            [&](int i) { return first_block + i; }, P.scale_log2, dk, dv, kb);
  } else {
    // causal: the tile's entries that the group's blocks attend (the same for all 16)
    const uint32_t kmask = LAYOUT == kCausal ? (cmask >> (tile * kBlock)) & 0xffffu : 0xffffu;
    ok = kv_stream<D, STAGES, LAYOUT>(g, &tm_q, &tm_do, ws + W.lsd, kvt, 0u, ring, slsd, bar_ring, kBlock,
                                      [&](int i) { return first_block + i; }, P.scale_log2, dk, dv, {0.f, 0.f}, 0.f,
                                      kBlock, 0, kmask);
  }
  if (!ok) return;
  const int r0 = lane >> 2;
  const int c2 = 2 * (lane & 3);
  float* pk = ws + W.part_k + (long long)group * g.coarse * D;
  float* pv = ws + W.part_v + (long long)group * g.coarse * D;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = tile * kBlock + r0 + 8 * h;
    if (row < g.coarse) {
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        *reinterpret_cast<float2*>(pk + row * D + n * 8 + c2) = make_float2(dk[n][2 * h], dk[n][2 * h + 1]);
        *reinterpret_cast<float2*>(pv + row * D + n * 8 + c2) = make_float2(dv[n][2 * h], dv[n][2 * h + 1]);
      }
    }
  }
}

// Per coarse level-l token j (one CTA of kReduceWarps warps each): the sum of the group
// partials of every level-l query a in CSR row j, over the 16^(l-2) level-2 groups under a.
// In the level-L part of the all-coarsest variant every level-L query a lists j (at entry
// top_first + j), so the row is a = 0..n_L-1 and the CSR is not read.
// The (a, group) pairs are dealt round-robin to the warps; the warps' sums are added in warp
// order, so the result does not depend on timing.
constexpr int kReduceWarps = 8;

// D/32 consecutive fp32 channels of one lane (a float2 at D = 64, a float4 at D = 128).
template <int D>
struct LaneVec {
  float v[D / 32];
};
template <int D>
__device__ __forceinline__ LaneVec<D> lane_load(const float* p) {
  LaneVec<D> r;
  if constexpr (D == 64) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    r.v[0] = x.x;
    r.v[1] = x.y;
  } else {
    const float4 x = *reinterpret_cast<const float4*>(p);
    r.v[0] = x.x;
    r.v[1] = x.y;
    r.v[2] = x.z;
    r.v[3] = x.w;
  }
  return r;
}
template <int D>
__device__ __forceinline__ void lane_store(float* p, const LaneVec<D>& r, float scale) {
  if constexpr (D == 64) {
    *reinterpret_cast<float2*>(p) = make_float2(r.v[0] * scale, r.v[1] * scale);
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(r.v[0] * scale, r.v[1] * scale, r.v[2] * scale, r.v[3] * scale);
  }
}

template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32) coarse_grad_reduce_kernel(Geometry g, float scale,
                                                                              const int* __restrict__ idx,
                                                                              const int* __restrict__ row_ptr,
                                                                              const int* __restrict__ col,
                                                                              float* __restrict__ ws) {
  // The CSR rows and the selection (two or more kernels back, or joined before this launch) are
  // read before waiting; the partials, written by the kernel ahead, after (see pdl_wait).
  constexpr int V = D / 32;  // channels per lane: V * lane .. V * lane + V - 1
  __shared__ LaneVec<D> red_k[kReduceWarps][32], red_v[kReduceWarps][32];
  __shared__ int slot_of[64];
  __shared__ int anc_of[64];
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int warp = threadIdx.x >> 5;
  long long cid = blockIdx.x;
  int lev = 2;
  for (; lev <= g.L; ++lev) {
    const long long cnt = (long long)g.BH * g.n[lev];
    if (cid < cnt) break;
    cid -= cnt;
  }
  if (lev > g.L) return;  // uniform over the CTA
  const int nl = g.n[lev];
  const int K = g.K;
  const int bh = (int)(cid / nl);
  const int j = (int)(cid - (long long)bh * nl);
  int span = 1;  // level-2 groups under one level-l token: 16^(l-2)
  for (int i = 2; i < lev; ++i) span *= kBlock;
  const bool dense = lev >= g.L && g.top_first < g.coarse;  // all-coarsest level-L part
  const int* rp = row_ptr + g.rp_off[lev] + (long long)bh * (nl + 1);
  const int E = nl * K;
  int rs = dense ? 0 : rp[j], re = dense ? nl : rp[j + 1];
  if (!dense && (rs < 0 || re > E || rs > re)) {
    if (threadIdx.x == 0) record_error(LLSA_ERR_INTERNAL);
    rs = re = 0;
  }
  const int* cl = col + g.idx_off[lev] + (long long)bh * E;
  const int* il = idx + g.idx_off[lev] + (long long)bh * E;
  const long long n2 = g.n[2];
  LaneVec<D> sk, sv;
#pragma unroll
  for (int c = 0; c < V; ++c) sk.v[c] = sv.v[c] = 0.f;
  // CSR rows are processed in chunks of 64 entries: slots first, then the (entry, group) pairs
  bool waited = false;
  for (int c0 = rs; c0 < re; c0 += 64) {
    const int cnt = min(64, re - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
      if (dense) {
        slot_of[e] = g.top_first + j;
        anc_of[e] = c0 + e;
        continue;
      }
      const int a = checked_index(__ldg(cl + c0 + e), nl);
      int lo = 0, hi = K - 1;  // slot of j in the ascending list of a
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(il + (long long)a * K + mid) < j) lo = mid + 1; else hi = mid;
      }
      if (__ldg(il + (long long)a * K + lo) != j) record_error(LLSA_ERR_INTERNAL);
      slot_of[e] = (lev - 2) * K + lo;
      anc_of[e] = a;
    }
    __syncthreads();
    if (!waited) {
      pdl_wait();
      pdl_launch_dependents();
      waited = true;
    }
    const int pairs = cnt * span;
    // four pairs per iteration: their loads are independent, the sums stay in pair order
    for (int p0 = warp * 4; p0 < pairs; p0 += kReduceWarps * 4) {
      LaneVec<D> x[4], y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pi = p0 + u;
#pragma unroll
        for (int c = 0; c < V; ++c) x[u].v[c] = y[u].v[c] = 0.f;
        if (pi < pairs) {
          const int e = pi / span;
          const int gi = pi - e * span;
          const long long grp = (long long)bh * n2 + (long long)anc_of[e] * span + gi;
          const long long off = (grp * g.coarse + slot_of[e]) * D + V * lane;
          x[u] = lane_load<D>(ws + W.part_k + off);
          y[u] = lane_load<D>(ws + W.part_v + off);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int c = 0; c < V; ++c) {
          sk.v[c] += x[u].v[c];
          sv.v[c] += y[u].v[c];
        }
    }
  }
  if (!waited) {  // an empty row: nothing was read from the kernel ahead
    pdl_wait();
    pdl_launch_dependents();
  }
  red_k[warp][lane] = sk;
  red_v[warp][lane] = sv;
  __syncthreads();
  if (warp == 0) {
    LaneVec<D> tk, tv;
#pragma unroll
    for (int c = 0; c < V; ++c) tk.v[c] = tv.v[c] = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w)
#pragma unroll
      for (int c = 0; c < V; ++c) {
        tk.v[c] += red_k[w][lane].v[c];
        tv.v[c] += red_v[w][lane].v[c];
      }
    const long long out = W.cg_off[lev] + ((long long)bh * nl + j) * D + V * lane;
    lane_store<D>(ws + W.cg_k + out, tk, scale);
    lane_store<D>(ws + W.cg_v + out, tv, 1.0f);
  }
}

// ---------------------------------------------------------------------------- dK/dV order

__device__ __forceinline__ int order_class(int len) {
  return len <= 0 ? kOrdClasses - 1 : 7 - min(31 - __clz(len), 7);
}

// CSR extent [rs, re) of flat level-1 row kb = bh * n_1 + j (empty for kb past the end).
__device__ __forceinline__ int2 order_row(const Geometry& g, const int* __restrict__ rp1, int kb) {
  if (kb >= g.BH * g.n[1]) return make_int2(0, 0);
  const int bh = div_n1(g, kb);
  const int* r = rp1 + (long long)bh * (g.n[1] + 1) + (kb - bh * g.n[1]);
  return make_int2(__ldg(r), __ldg(r + 1));
}

__device__ __forceinline__ int order_row_len(const Geometry& g, const int* __restrict__ rp1, int kb) {
  const int2 e = order_row(g, rp1, kb);
  return e.y - e.x;
}

// Per tile of kOrdTile rows: the number of rows of each class (counts[c * tiles + tile]).
__global__ void __launch_bounds__(kOrdThreads) dkdv_order_count_kernel(Geometry g, const int* __restrict__ row_ptr,
                                                                       float* __restrict__ ws) {
  pdl_enter();
  __shared__ int part[kOrdThreads / 32][kOrdClasses];
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int* rp1 = row_ptr + g.rp_off[1];
  const int row0 = blockIdx.x * kOrdTile + threadIdx.x * kOrdRowsPerThread;
  int cnt[kOrdClasses];
#pragma unroll
  for (int c = 0; c < kOrdClasses; ++c) cnt[c] = 0;
  for (int i = 0; i < kOrdRowsPerThread; ++i) {
    if (row0 + i >= g.BH * g.n[1]) break;
    const int c = order_class(order_row_len(g, rp1, row0 + i));
#pragma unroll
    for (int cc = 0; cc < kOrdClasses; ++cc) cnt[cc] += (cc == c);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < kOrdClasses; ++c) {
    int v = cnt[c];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) part[warp][c] = v;
  }
  __syncthreads();
  if (threadIdx.x < kOrdClasses) {
    int v = 0;
    for (int w = 0; w < kOrdThreads / 32; ++w) v += part[w][threadIdx.x];
    reinterpret_cast<int*>(ws + W.order_counts)[threadIdx.x * order_tiles(g) + blockIdx.x] = v;
  }
}

// Writes order[pos] = kb: class by class, tiles in order, rows in order within a tile.
__global__ void __launch_bounds__(kOrdThreads) dkdv_order_scatter_kernel(Geometry g, const int* __restrict__ row_ptr,
                                                                         float* __restrict__ ws) {
  pdl_enter();
  __shared__ int start[kOrdClasses];
  __shared__ int wsum[kOrdThreads / 32][kOrdClasses];
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int tiles = order_tiles(g);
  const int* counts = reinterpret_cast<const int*>(ws + W.order_counts);
  if (threadIdx.x < 32) {
    // start of (class c, this tile) = rows of lower classes + rows of class c in earlier tiles
    const int lane = threadIdx.x;
    int before = 0, mine = 0;
    for (int c = 0; c < kOrdClasses; ++c) {
      int tot = 0, pre = 0;
      for (int t = lane; t < tiles; t += 32) {
        const int v = counts[c * tiles + t];
        tot += v;
        if (t < (int)blockIdx.x) pre += v;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, off);
        pre += __shfl_xor_sync(0xffffffffu, pre, off);
      }
      if (lane == c) mine = before + pre;
      if (c == kOrdClasses - 1 && blockIdx.x == 0 && lane == 0)
        reinterpret_cast<int*>(ws + W.order_nonempty)[0] = before;  // the empty class comes last
      before += tot;
    }
    if (lane < kOrdClasses) start[lane] = mine;
  }
  const int* rp1 = row_ptr + g.rp_off[1];
  const int row0 = blockIdx.x * kOrdTile + threadIdx.x * kOrdRowsPerThread;
  int cls[kOrdRowsPerThread];
  int2 ext[kOrdRowsPerThread];
  int cnt[kOrdClasses];
#pragma unroll
  for (int c = 0; c < kOrdClasses; ++c) cnt[c] = 0;
#pragma unroll
  for (int i = 0; i < kOrdRowsPerThread; ++i) {
    ext[i] = order_row(g, rp1, row0 + i);
    cls[i] = row0 + i < g.BH * g.n[1] ? order_class(ext[i].y - ext[i].x) : -1;
#pragma unroll
    for (int cc = 0; cc < kOrdClasses; ++cc) cnt[cc] += (cc == cls[i]);
  }
  // exclusive scan of the per-thread counts over the CTA, class by class
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int pre[kOrdClasses];
#pragma unroll
  for (int c = 0; c < kOrdClasses; ++c) {
    int v = cnt[c];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    pre[c] = v - cnt[c];
    if (lane == 31) wsum[warp][c] = v;
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < kOrdClasses; ++c) {
    int base = start[c];
    for (int w = 0; w < warp; ++w) base += wsum[w][c];
    pre[c] += base;
  }
  int4* order = reinterpret_cast<int4*>(ws + W.order);
#pragma unroll
  for (int i = 0; i < kOrdRowsPerThread; ++i) {
    const int c = cls[i];
    if (c < 0) continue;
    int pos = 0;
#pragma unroll
    for (int cc = 0; cc < kOrdClasses; ++cc)
      if (cc == c) pos = pre[cc]++;
    order[pos] = make_int4(row0 + i, ext[i].x, ext[i].y, 0);
  }
}

// Fine-token dK, dV.  One warp per CTA and per fine key block (flat (b*H + h) * n_1 + j), so
// a long CSR row never holds other warps' slots.
// coarse_late != 0: the kernel ahead of this one on the stream is coarse_grad_reduce_kernel,
// whose output (the coarse-token gradients) only the epilogue reads; everything the main
// loop reads was complete before that kernel could start, so the wait for it is deferred
// to the epilogue and the main loop overlaps the reduction.
template <int D, int STAGES, bool POOL, int LAYOUT>
__global__ void __launch_bounds__(32) attn_bwd_dkdv_bf16_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, AttnParams P,
    const int* __restrict__ row_ptr, const int* __restrict__ col, const float* __restrict__ ws,
    __nv_bfloat16* __restrict__ dk_out, __nv_bfloat16* __restrict__ dv_out, int coarse_late) {
  if (!coarse_late) pdl_wait();
  pdl_launch_dependents();
  extern __shared__ uint8_t dkv_smem_raw[];
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int n1 = g.n[1];
  const int K = g.K;
  // CTAs past the non-empty rows write the empty rows, 16 per CTA: no query block selected
  // them, so dK and dV are only the mean-pool adjoint of their ancestors' coarse gradients
  // (the same for the 16 keys).  The CTAs beyond those return at once.
  {
    const int ne = min(max(__ldg(reinterpret_cast<const int*>(ws + W.order_nonempty)), 0), g.BH * n1);
    if ((int)blockIdx.x >= ne) {
      const int e0 = ne + ((int)blockIdx.x - ne) * kBlock;
      if (e0 >= g.BH * n1) return;
      if (coarse_late) pdl_wait();
      const int4* order = reinterpret_cast<const int4*>(ws + W.order);
      const int cnt = min(kBlock, g.BH * n1 - e0);
      const int my_kb = lane < cnt ? checked_index(__ldg(&order[e0 + lane].x), g.BH * n1) : 0;
      // four rows at a time: all their coarse-gradient loads are issued before any sum
      constexpr int V = D / 32;  // channels per lane
      for (int r0 = 0; r0 < cnt; r0 += 4) {
        LaneVec<D> xk[4][kMaxLevels], xv[4][kMaxLevels];
        int kbs[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          kbs[u] = __shfl_sync(0xffffffffu, my_kb, min(r0 + u, cnt - 1));
          const int bh = kbs[u] / n1, j = kbs[u] - bh * n1;
          int span = 1, nl = n1;
          long long cg_level = 0;
#pragma unroll
          for (int lev = 2; lev <= kMaxLevels; ++lev) {
#pragma unroll
            for (int c = 0; c < V; ++c) xk[u][lev - 1].v[c] = xv[u][lev - 1].v[c] = 0.f;
            if (lev <= g.L) {
              span *= kBlock;
              nl /= kBlock;
              const long long off = cg_level + ((long long)bh * nl + j / span) * D + V * lane;
              xk[u][lev - 1] = lane_load<D>(ws + W.cg_k + off);
              xv[u][lev - 1] = lane_load<D>(ws + W.cg_v + off);
              cg_level += (long long)g.BH * nl * D;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (r0 + u >= cnt) break;
          const int bh = kbs[u] / n1, j = kbs[u] - bh * n1;
          float ak[V], av[V];  // channels V lane .. V lane + V - 1
#pragma unroll
          for (int c = 0; c < V; ++c) ak[c] = av[c] = 0.f;
          int span = 1;
#pragma unroll
          for (int lev = 2; lev <= kMaxLevels; ++lev) {
            if (lev > g.L) break;
            span *= kBlock;
            // 1 / 16^l, or 1 / (real tokens) of an ancestor a padded sequence cuts
            const int c = pool_count(g, lev, j / span);
            const float wgt = c > 0 ? 1.0f / (float)c : 0.0f;
#pragma unroll
            for (int c = 0; c < V; ++c) {
              ak[c] += wgt * xk[u][lev - 1].v[c];
              av[c] += wgt * xv[u][lev - 1].v[c];
            }
          }
          uint32_t pk[V / 2], pv[V / 2];
#pragma unroll
          for (int c = 0; c < V / 2; ++c) {
            pk[c] = pack_bf16(ak[2 * c], ak[2 * c + 1]);
            pv[c] = pack_bf16(av[2 * c], av[2 * c + 1]);
          }
          const int kvalid = LAYOUT == kPadded ? g.nv - j * kBlock : kBlock;  // padding positions get 0
          const long long row0 = token_row<LAYOUT>(g, bh, j * kBlock);
#pragma unroll
          for (int t = 0; t < kBlock; ++t) {
            const bool real = t < kvalid;
            const long long row = row0 + block_row_offset<LAYOUT>(g, t);
            if constexpr (V == 2) {
              reinterpret_cast<uint32_t*>(dk_out + row * D)[lane] = real ? pk[0] : 0u;
              reinterpret_cast<uint32_t*>(dv_out + row * D)[lane] = real ? pv[0] : 0u;
            } else {
              reinterpret_cast<uint2*>(dk_out + row * D)[lane] = real ? make_uint2(pk[0], pk[1]) : make_uint2(0u, 0u);
              reinterpret_cast<uint2*>(dv_out + row * D)[lane] = real ? make_uint2(pv[0], pv[1]) : make_uint2(0u, 0u);
            }
          }
        }
      }
      return;
    }
  }
  // key blocks are taken longest row first (dkdv_order_*_kernel, complete before this
  // kernel's predecessor started); the entry carries the row's CSR extent
  const int4 ent = __ldg(reinterpret_cast<const int4*>(ws + W.order) + blockIdx.x);
  const int kb = checked_index(ent.x, g.BH * n1);
  const int bh = kb / n1;
  const int j = kb - bh * n1;
  const CtaSmem cs = kv_smem<D, STAGES>(1);
  constexpr int TB = tile_bytes<D>();
  uint8_t* base = align1024(dkv_smem_raw);
  const uint32_t kvt = smem_u32(cs.tiles(base, 0));
  const uint32_t ring = kvt + 2 * TB;
  float* slsd = reinterpret_cast<float*>(cs.tail(base, 0));  // [STAGES][32] LSE + Delta records
  const uint32_t bar_kv = smem_u32(slsd + STAGES * 2 * kBlock);
  const uint32_t bar_ring = bar_kv + 8;

  const int E = n1 * K;
  int rs = ent.y, re = ent.z;
  if (rs < 0 || re > E || rs > re) {
    if (lane == 0) record_error(LLSA_ERR_INTERNAL);
    rs = re = 0;
  }
  const int* cl = col + g.idx_off[1] + (long long)bh * E + rs;

  if (lane == 0) {
    for (int b = 0; b < 1 + STAGES; ++b) mbar_init(bar_kv + 8 * b, 1);
    mbar_fence_init();
  }
  __syncwarp();
  if (lane == 0) {
    mbar_expect_tx(bar_kv, 2 * TB);
    tma_load_tile<D, LAYOUT>(kvt, &tm_k, g, bh * g.N + j * kBlock, bar_kv);
    tma_load_tile<D, LAYOUT>(kvt + TB, &tm_v, g, bh * g.N + j * kBlock, bar_kv);
  }
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;
  const int bh_block0 = bh * n1;
  // the row's query blocks are read 32 at a time by the whole warp and handed to the
  // issuing lane by shuffle, so no load sits on the TMA issue path
  int cached_base = -64, cached = 0;
  auto pair_block = [&](int i) {
    const int base32 = i & ~31;
    if (base32 != cached_base) {
      cached_base = base32;
      const int e = base32 + lane;
      cached = e < re - rs ? checked_index(__ldg(cl + e), n1) : 0;
    }
    return bh_block0 + __shfl_sync(0xffffffffu, cached, i & 31);
  };
  // real keys of this block (16 unless padded)
  const int kvalid = LAYOUT == kPadded ? min(kBlock, g.nv - j * kBlock) : kBlock;
  // causal: whether the row's first query block is the key block itself
  const bool diag_first = LAYOUT == kCausal && re > rs && __ldg(cl) == j;
  const bool ok = kv_stream<D, STAGES, LAYOUT, false, POOL>(g, &tm_q, &tm_do, ws + W.lsd, kvt, bar_kv, ring, slsd,
                                                            bar_ring, re - rs, pair_block, P.scale_log2, dk, dv,
                                                            {0.f, 0.f}, pool_log_bias<D>(g), kvalid,
                                                            LAYOUT == kGrid ? 1 : 0, 0xffffu, diag_first);
  if (!ok) return;
  if (coarse_late) pdl_wait();
  // epilogue: scale dK, add the mean-pool adjoint of the ancestors' coarse gradients
  const int c2 = 2 * (lane & 3);
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] *= P.scale;
  int span = 1;  // 16^(l-1): level-1 blocks under one level-l token
  long long cg_level = 0;  // offset of level l in the coarse-gradient arrays
  int nl = n1;
  for (int lev = 2; lev <= g.L; ++lev) {
    span *= kBlock;
    nl /= kBlock;          // n_l
    const int a = j / span;
    const float wgt = 1.0f / (float)pool_count(g, lev, a);  // 1 / 16^l unless a padded sequence cuts a
    const float* ck = ws + W.cg_k + cg_level + ((long long)bh * nl + a) * D;
    const float* cv = ws + W.cg_v + cg_level + ((long long)bh * nl + a) * D;
    cg_level += (long long)g.BH * nl * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
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
  const int r0 = lane >> 2;  // padding positions of a padded sequence get dK = dV = 0
  const float s0 = r0 < kvalid ? 1.0f : 0.0f, s1 = r0 + 8 < kvalid ? 1.0f : 0.0f;
  store_tile_bf16<D, LAYOUT>(dk, s0, s1, kvt, dk_out, g, bh, j * kBlock);
  store_tile_bf16<D, LAYOUT>(dv, s0, s1, kvt + TB, dv_out, g, bh, j * kBlock);
}

}  // namespace llsa
