// Step 4a: block-sparse attention forward with hierarchical KV enrichment (skill page
// "Log Linear Sparse Attention", Core Technique 2; README usage section: drop-in for
// non-causal scaled_dot_product_attention with block_size=16).
//
// Work unit: one warp owns 4 consecutive query blocks (64 queries).  Those blocks share
// their level-2.. ancestors, so the coarse KV entries are gathered once per unit.  For each
// block the warp streams its KV list -- K selected 16-token blocks of K and V, gathered by
// index with 2-D TMA copies (one 16 x 64 bf16 box per tile, 128-byte swizzle, no multicast)
// through a ring of mbarrier-tracked stages, then the (L-1)K coarse tokens -- and keeps the
// online softmax state (row max, row sum, 16 x 64 fp32 output) in registers:
//   S = Q K^T (mma.sync m16n8k16 bf16, fp32 accumulate), P = exp2(S*scale*log2e - m),
//   O = O*exp2(m_old - m) + P V.
// Coarse rows are fp32 in the pyramid; they are rounded to bf16 as they are staged.
//
// Head width D is 64 or 128 (a template parameter of every kernel).  A 16-token tile of D
// bf16 channels is D/64 sub-tiles of 16 rows x 128 bytes, each one 2-D TMA box with
// 128-byte swizzle (x = 0 and x = 64), stored one after the other.
//
// Bound: the gathered K/V bytes (T * D * 2 * 2 per query block; one head's K and V are
// 16.8 MB at N = 65536, D = 64, so most re-gathers hit L2) against HBM bandwidth, and the
// 4 * 16 * T * D tensor FLOPs per block.
#pragma once

#include "llsa_common.cuh"

namespace llsa {

constexpr int kUnitBlocks = 4;   // query blocks per warp unit
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnParams {
  Geometry g;
  float scale_log2;   // log2(e) / sqrt(D)
  float scale;        // 1 / sqrt(D)
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bytes of one 16-token tile of D bf16 channels, and the byte offset of 16-byte chunk `ch`
// (0 <= ch < D/8) of row `row` in it: sub-tile ch / 8, swizzled chunk ch % 8.
template <int D>
__host__ __device__ constexpr int tile_bytes() {
  return kBlock * D * 2;
}
__device__ __forceinline__ uint32_t tswz(int row, int ch) {
  return static_cast<uint32_t>((ch >> 3) * kSubTileBytes) + swz(row, ch & 7);
}

// Every fragment load below takes `perm` (0 or 1): 1 for a tile that a grid-order TMA box
// brought in (its shared-memory rows are pixel rows, tile_row maps the block's quadtree row to
// them), 0 for a tile whose rows are already in order.

// A-operand fragments of a 16 x D bf16 tile (rows = M, channels = K) for the D/16 k-steps.
template <int D>
__device__ __forceinline__ void load_a_frags(uint32_t tile, uint32_t (&f)[D / 16][4], int perm = 0) {
  const int lane = lane_id();
  const int row = tile_row(lane & 15, perm);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    ldsm_x4(tile + tswz(row, 2 * kk + (lane >> 4)), f[kk][0], f[kk][1], f[kk][2], f[kk][3]);
}

// acc[2][4] (16 x 16) += A (16 x D, fragments) * B^T where B is a 16-row x D tile (rows = N).
template <int D>
__device__ __forceinline__ void mma_a_bt(float (&acc)[2][4], const uint32_t (&a)[D / 16][4], uint32_t btile,
                                         int perm = 0) {
  const int lane = lane_id();
  const int row = tile_row((lane & 7) + ((lane >> 4) << 3), perm);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4(btile + tswz(row, 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
    mma_bf16(acc[0], a[kk][0], a[kk][1], a[kk][2], a[kk][3], b0, b1);
    mma_bf16(acc[1], a[kk][0], a[kk][1], a[kk][2], a[kk][3], b2, b3);
  }
}

// The same with A read from its shared-memory tile one k-step at a time (no A fragments
// held in registers).
template <int D>
__device__ __forceinline__ void mma_at_bt(float (&acc)[2][4], uint32_t atile, uint32_t btile, int aperm = 0,
                                          int bperm = 0) {
  const int lane = lane_id();
  const int row = tile_row((lane & 7) + ((lane >> 4) << 3), bperm);
  const int arow = tile_row(lane & 15, aperm);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
    ldsm_x4(atile + tswz(arow, 2 * kk + (lane >> 4)), a0, a1, a2, a3);
    ldsm_x4(btile + tswz(row, 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
    mma_bf16(acc[0], a0, a1, a2, a3, b0, b1);
    mma_bf16(acc[1], a0, a1, a2, a3, b2, b3);
  }
}

// acc[D/8][4] (16 x D) += A (16 x 16: a0..a3) * B where B is a 16-row x D tile (rows = K).
template <int D>
__device__ __forceinline__ void mma_a_b(float (&acc)[D / 8][4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t btile, int perm = 0) {
  const int lane = lane_id();
  const int row = tile_row((lane & 7) + (((lane >> 3) & 1) << 3), perm);
#pragma unroll
  for (int dc = 0; dc < D / 16; ++dc) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(btile + tswz(row, 2 * dc + (lane >> 4)), b0, b1, b2, b3);
    mma_bf16(acc[2 * dc], a0, a1, a2, a3, b0, b1);
    mma_bf16(acc[2 * dc + 1], a0, a1, a2, a3, b2, b3);
  }
}

// Two fp32 values as a bf16 pair hi (round to nearest) and the pair of their bf16-rounded
// remainders lo, so that hi + lo carries about 16 significant bits of each value.
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  lo = pack_bf16(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

// Stage the C coarse rows of a pyramid (fp32) as bf16 16-row swizzled tiles; padding rows
// (index >= C) and causal entries that are not attended are zero.  Row c is the pyramid row
// of coarse entry c (see coarse_token).
// Threads `tid` = 0..nthreads-1 share the work (a warp or a whole CTA).
template <int D>
__device__ __forceinline__ void stage_coarse_rows(const Geometry& g, const float* __restrict__ pyr,
                                                  const int* __restrict__ idx, int bh, int p, uint32_t dst, int tid,
                                                  int nthreads) {
  constexpr int CH = D / 8;  // 16-byte bf16 chunks per row
  for (int t = tid; t < g.coarse_pad * CH; t += nthreads) {
    const int row = t / CH;
    const int ch = t - row * CH;
    uint4 packed = make_uint4(0u, 0u, 0u, 0u);
    if (row < g.coarse) {
      int lev;
      const int j = coarse_token(g, idx, bh, p, row, lev);
      if (j >= 0) {
        const int nl = g.n[lev];
        const float4* src =
            reinterpret_cast<const float4*>(pyr + g.pyr_off[lev] + ((long long)bh * nl + j) * D + ch * 8);
        const float4 x = __ldg(src);
        const float4 y = __ldg(src + 1);
        packed = make_uint4(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w), pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
      }
    }
    const uint32_t addr = dst + (row >> 4) * tile_bytes<D>() + tswz(row & 15, ch);
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(packed.x), "r"(packed.y), "r"(packed.z),
                 "r"(packed.w)
                 : "memory");
  }
}

// Write a 16 x D fp32 accumulator (fragment layout, already scaled) as the bf16 rows of the
// 16 tokens t0 .. t0 + 15 of head bh of a [B*H*N, D] global array (token_row: in grid order
// each row goes to its pixel), through a swizzled shared staging tile.
template <int D, int LAYOUT>
__device__ __forceinline__ void store_tile_bf16(const float (&acc)[D / 8][4], float s0, float s1, uint32_t stage,
                                                __nv_bfloat16* __restrict__ out, const Geometry& g, int bh, int t0) {
  const int lane = lane_id();
  const int r0 = lane >> 2;
  const uint32_t cb = (lane & 3) * 4;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const uint32_t v0 = pack_bf16(acc[n][0] * s0, acc[n][1] * s0);
    const uint32_t v1 = pack_bf16(acc[n][2] * s1, acc[n][3] * s1);
    asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(stage + tswz(r0, n) + cb), "r"(v0) : "memory");
    asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(stage + tswz(r0 + 8, n) + cb), "r"(v1) : "memory");
  }
  __syncwarp();
  constexpr int CH = D / 8;
  __nv_bfloat16* const base = out + token_row<LAYOUT>(g, bh, t0) * D;
#pragma unroll
  for (int it = 0; it < D / 16; ++it) {
    const int ci = lane + 32 * it;
    const int row = ci / CH;
    const int c = ci - row * CH;
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(stage + tswz(row, c)));
    *reinterpret_cast<uint4*>(base + block_row_offset<LAYOUT>(g, row) * D + c * 8) = v;
  }
  // the staging tile is refilled by TMA later: order these generic accesses before it
  fence_proxy_async();
  __syncwarp();
}

// Loads of the 16-token x D tile that starts at flat token row `row` (= (b*H + h) * N + t):
// D/64 boxes at x = 0, 64 of the flat [B*H*N][D] tensor map, or of the [B*H][n_valid][D]
// one for a padded sequence, whose rows at or past n_valid arrive as zeros.
// Under LLSA_FLAG_GRID_ORDER the map is [B*H*G][G][D] (pixel rows) and the box a 4 x 4 patch: the
// block at quadtree position t / 16 is the patch at block-grid row and column R, C, whose 16
// pixel rows arrive in row-major order (see tile_row).
template <int D, int LAYOUT>
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap* map, const Geometry& g, int row,
                                              uint32_t bar) {
  if constexpr (flat_tile_map(LAYOUT)) {  // the 2-D map (make_tile_map makes the same choice)
#pragma unroll
    for (int h = 0; h < D / 64; ++h) tma_load_2d(dst + h * kSubTileBytes, map, 64 * h, row, bar);
    return;
  }
  const int bh = div_n(g, row);
  const int t = row - bh * g.N;
  if constexpr (LAYOUT == kGrid) {
    const int p = z_to_rowmajor(t >> 4, g.log_g - 2);  // R * (G / 4) + C
    const int R = p >> (g.log_g - 2), C = p & ((1 << (g.log_g - 2)) - 1);
#pragma unroll
    for (int h = 0; h < D / 64; ++h)
      tma_load_3d(dst + h * kSubTileBytes, map, 64 * h, 4 * C, (bh << g.log_g) + 4 * R, bar);
    return;
  }
#pragma unroll
  for (int h = 0; h < D / 64; ++h) tma_load_3d(dst + h * kSubTileBytes, map, 64 * h, t, bh, bar);
}

// The 16 LSE values of the query block whose first token row is `row` (flat), into `dst`
// in the tile's shared-memory row order: one 64-byte bulk copy, or under grid order four
// 16-byte copies of the patch's pixel rows.
template <int LAYOUT>
__device__ __forceinline__ void bulk_load_block_rows(uint32_t dst, const float* src, const Geometry& g, int row,
                                                     uint32_t bar) {
  if constexpr (LAYOUT != kGrid) {
    bulk_load(dst, src + row, kBlock * 4, bar);
    return;
  }
  const int bh = div_n(g, row);
  const int t = row - bh * g.N;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    bulk_load(dst + 16 * r, src + token_row<kGrid>(g, bh, t + 2 * (r & 1) + 8 * (r >> 1)), 16, bar);
}

// sqrt(D): a score bias in units of the unscaled dot product is the scaled bias times this.
template <int D>
__host__ __device__ constexpr float sqrt_d() {
  return D == 64 ? 8.0f : 11.313708498984761f;
}

// Bias of a level-1 pooled entry (level-1 variant) in unscaled-dot units: ln 16 under the
// log-count variant, else 0.
template <int D>
__host__ __device__ inline float pool_log_bias(const Geometry& g) {
  return g.log_bias ? kLn16 * sqrt_d<D>() : 0.0f;
}

// Row sums of a 16 x 16 score fragment (C layout): rows r0 and r0 + 8 of this lane's quad.
__device__ __forceinline__ void quad_row_sums(const float (&s)[2][4], float& t0, float& t1) {
  t0 = (s[0][0] + s[0][1]) + (s[1][0] + s[1][1]);
  t1 = (s[0][2] + s[0][3]) + (s[1][2] + s[1][3]);
  t0 += __shfl_xor_sync(0xffffffffu, t0, 1);
  t0 += __shfl_xor_sync(0xffffffffu, t0, 2);
  t1 += __shfl_xor_sync(0xffffffffu, t1, 1);
  t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
}

// One 16-token chunk of the online softmax.  With MASK (the coarse chunks), columns >=
// `valid` (the padding of the last coarse tile) and columns whose bit of `cmask` is clear
// (causal entries that are not attended) are excluded and, under the log-count variant,
// column c gets the bias of coarse entry c0 + c.  CAUSAL: key column c is visible to query
// row r only when c <= r + `shift` (15: a whole block before the query block, 0: the query
// block's own block, -16: no block, a list's kNoPick slot), one branch-free test per score.  m holds the running row maxima
// of the scaled scores (log2 domain), l the per-lane partial row sums.
// POOL (the level-1 variant, fine chunks only): the chunk's block mean is one more KV
// entry.  Its score is the mean of the 16 scores (q . mean k = mean of q . k), plus
// `pool_bias` (unscaled-dot units), and since its value is the mean of the 16 V rows its
// weight p folds into the chunk as p / 16 added to each of the 16 probabilities.
template <int D, bool MASK, bool POOL = false, bool CAUSAL = false>
__device__ __forceinline__ void fwd_chunk(const uint32_t (&qf)[D / 16][4], uint32_t ktile, uint32_t vtile, int valid,
                                          float scale_log2, float (&m)[2], float (&l)[2], float (&acc)[D / 8][4],
                                          const Geometry* bias_g = nullptr, int c0 = 0, float pool_bias = 0.f,
                                          int perm = 0, uint32_t cmask = 0xffffffffu, int shift = 15) {
  const int lane = lane_id();
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  mma_a_bt<D>(s, qf, ktile, perm);
  float sb0 = 0.f, sb1 = 0.f;  // pooled scores of rows r0, r0 + 8
  if (POOL) {
    quad_row_sums(s, sb0, sb1);
    sb0 = fmaf(sb0, 1.0f / kBlock, pool_bias);
    sb1 = fmaf(sb1, 1.0f / kBlock, pool_bias);
  }
  if (MASK) {
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = n * 8 + 2 * (lane & 3) + (e & 1);
        if (col >= valid || !((cmask >> col) & 1u)) s[n][e] = -INFINITY;
        else if (bias_g && bias_g->log_bias) s[n][e] += coarse_log_bias(*bias_g, c0 + col) * sqrt_d<D>();
      }
  }
  if (CAUSAL) {
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (n * 8 + 2 * (lane & 3) + (e & 1) > (lane >> 2) + 8 * (e >> 1) + shift) s[n][e] = -INFINITY;
  }
  float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
  float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  if (POOL) {
    mx0 = fmaxf(mx0, sb0);
    mx1 = fmaxf(mx1, sb1);
  }
  // the scale is positive, so the maximum of the scaled scores is the scaled maximum
  const float mn0 = fmaxf(m[0], mx0 * scale_log2);
  const float mn1 = fmaxf(m[1], mx1 * scale_log2);
  float p[2][4];
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    p[n][0] = ex2(fmaf(s[n][0], scale_log2, -mn0));
    p[n][1] = ex2(fmaf(s[n][1], scale_log2, -mn0));
    p[n][2] = ex2(fmaf(s[n][2], scale_log2, -mn1));
    p[n][3] = ex2(fmaf(s[n][3], scale_log2, -mn1));
  }
  if (POOL) {
    const float a0 = ex2(fmaf(sb0, scale_log2, -mn0)) * (1.0f / kBlock);
    const float a1 = ex2(fmaf(sb1, scale_log2, -mn1)) * (1.0f / kBlock);
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      p[n][0] += a0;
      p[n][1] += a0;
      p[n][2] += a1;
      p[n][3] += a1;
    }
  }
  // rescale the running sums only when a row maximum moved (decided for the whole warp)
  if (__any_sync(0xffffffffu, mn0 != m[0] || mn1 != m[1])) {
    const float c0 = ex2(m[0] - mn0);
    const float c1 = ex2(m[1] - mn1);
    l[0] *= c0;
    l[1] *= c1;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc[n][0] *= c0;
      acc[n][1] *= c0;
      acc[n][2] *= c1;
      acc[n][3] *= c1;
    }
    m[0] = mn0;
    m[1] = mn1;
  }
  l[0] += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
  l[1] += (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
  mma_a_b<D>(acc, pack_bf16(p[0][0], p[0][1]), pack_bf16(p[0][2], p[0][3]), pack_bf16(p[1][0], p[1][1]),
             pack_bf16(p[1][2], p[1][3]), vtile, perm);
}

// Shared memory of the attention kernels: a CTA region (the group's coarse K and V tiles),
// then per warp a block of 1024-aligned tiles, then per warp a small tail (indices,
// mbarriers).  Offsets are in bytes from the 1024-aligned base.
struct CtaSmem {
  int coarse_bytes;  // 2 * coarse_pad * D * 2
  int warp_tiles;    // bytes of tiles per warp (multiple of 1024)
  int warp_tail;     // bytes of tail per warp (multiple of 16)
  int nwarps;
  __host__ __device__ int total() const { return 1024 + coarse_bytes + nwarps * (warp_tiles + warp_tail); }
  __device__ uint8_t* tiles(uint8_t* base, int w) const { return base + coarse_bytes + w * warp_tiles; }
  __device__ uint8_t* tail(uint8_t* base, int w) const {
    return base + coarse_bytes + nwarps * warp_tiles + w * warp_tail;
  }
};

template <int D, int STAGES>
__host__ __device__ inline CtaSmem fwd_smem(const Geometry& g, int nwarps) {
  CtaSmem c;
  c.coarse_bytes = 2 * g.coarse_pad * D * 2;
  c.warp_tiles = 2 * tile_bytes<D>() + STAGES * 2 * tile_bytes<D>();
  c.warp_tail = ((kUnitBlocks * g.K * 4 + 15) & ~15) + ((8 * (2 + STAGES) + 15) & ~15);
  c.nwarps = nwarps;
  return c;
}

// One CTA = 4 warps = 16 consecutive query blocks (one level-2 group when L >= 2, so the
// coarse KV entries are staged once per CTA).  Each warp owns 4 blocks and streams their
// fine KV tiles through its own ring of STAGES mbarrier-tracked TMA stages.  POOL: the
// level-1 variant (see fwd_chunk).  LAYOUT (see Layout): under kPadded the fine tile that
// holds the last real token masks its padding keys (which arrive as zero rows), and padding
// queries write O = 0 and LSE = 0.
template <int D, int STAGES, bool POOL, int LAYOUT>
__global__ void __launch_bounds__(128, D == 64 ? 4 : 2) attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                            const __grid_constant__ CUtensorMap tm_k,
                                                            const __grid_constant__ CUtensorMap tm_v, AttnParams P,
                                                            const float* __restrict__ k_pyr,
                                                            const float* __restrict__ v_pyr,
                                                            const int* __restrict__ idx, __nv_bfloat16* __restrict__ o,
                                                            float* __restrict__ lse, float* __restrict__ lse_z) {
  // the coarse tiles come from the pyramid and the coarser selection levels, two or more
  // kernels back, so they are staged before waiting for the kernel ahead (see pdl_wait)
  extern __shared__ uint8_t fwd_smem_raw[];
  constexpr bool PAD = LAYOUT == kPadded;
  constexpr bool CAUSAL = LAYOUT == kCausal;
  constexpr int PERM = LAYOUT == kGrid ? 1 : 0;
  const Geometry& g = P.g;
  const int lane = lane_id();
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n1 = g.n[1];
  const int K = g.K;
  const int total_blocks = g.BH * n1;
  const CtaSmem cs = fwd_smem<D, STAGES>(g, nwarps);
  uint8_t* base = align1024(fwd_smem_raw);
  const uint32_t ck = smem_u32(base);
  const uint32_t cv = ck + g.coarse_pad * D * 2;
  const int cta_first = blockIdx.x * nwarps * kUnitBlocks;
  if (g.L >= 2) {  // the CTA's 16 blocks share one ancestor per level (n_1 % 16 == 0 here)
    const int bh0 = cta_first / n1;
    const int p0 = cta_first - bh0 * n1;
    stage_coarse_rows<D>(g, k_pyr, idx, bh0, p0, ck, threadIdx.x, blockDim.x);
    stage_coarse_rows<D>(g, v_pyr, idx, bh0, p0, cv, threadIdx.x, blockDim.x);
    __syncthreads();
  }
  // causal: the coarse entries the CTA's blocks attend (the same ancestors for all 16)
  const uint32_t cmask =
      (CAUSAL && g.L >= 2) ? coarse_visible_mask(g, idx, cta_first / n1, cta_first % n1) : 0xffffffffu;
  pdl_wait();
  pdl_launch_dependents();
  const int first = cta_first + warp * kUnitBlocks;
  if (first >= total_blocks) return;  // warp-uniform; no CTA-wide barrier after this point
  const int nblk = min(kUnitBlocks, total_blocks - first);
  const uint32_t sq = smem_u32(cs.tiles(base, warp));
  constexpr int TB = tile_bytes<D>();
  const uint32_t ring = sq + 2 * TB;
  int* srow = reinterpret_cast<int*>(cs.tail(base, warp));
  const uint32_t bar_q = smem_u32(srow) + ((kUnitBlocks * K * 4 + 15) & ~15);
  const uint32_t bar_kv = bar_q + 16;

  for (int i = lane; i < nblk * K; i += 32) {
    // the first K/V row of each load: (b*H + h) * N + 16 j, computed here off the issue path;
    // a causal list's kNoPick entry loads the block's own rows and is stored as their
    // complement (negative), so that nothing is computed for it
    const int pick = __ldg(idx + g.idx_off[1] + (long long)first * K + i);
    const int qb = first + div_k(g, i);
    if (CAUSAL && pick == kNoPick)
      srow[i] = ~(qb * kBlock);
    else
      srow[i] = div_n1(g, qb) * g.N + checked_index(pick, n1) * kBlock;
  }
  if (lane == 0) {
    for (int b = 0; b < 2 + STAGES; ++b) mbar_init(bar_q + 8 * b, 1);
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
  auto issue_q = [&](int i) {
    const uint32_t bar = bar_q + 8 * (i & 1);
    mbar_expect_tx(bar, TB);
    tma_load_tile<D, LAYOUT>(sq + (i & 1) * TB, &tm_q, g, (first + i) * kBlock, bar);
  };
  if (lane == 0) {
    issue_q(0);
    for (int s = 0; s < min(STAGES, total_loads); ++s) issue_kv(s);
  }

  bool ok = true;
  int next_seq = 0;  // first KV load not yet consumed
  int next_q = 0;    // first Q load not yet consumed
  for (int i = 0; i < nblk && ok; ++i) {
    const int gb = first + i;
    const int bh_i = div_n1(g, gb);
    // real queries of this block (16 unless the sequence is padded)
    const int qvalid = PAD ? g.nv - (gb - bh_i * n1) * kBlock : kBlock;
    ok = __all_sync(0xffffffffu, mbar_wait(bar_q + 8 * (i & 1), (i >> 1) & 1));
    if (!ok) break;
    next_q = i + 1;
    uint32_t qf[D / 16][4];
    load_a_frags<D>(sq + (i & 1) * TB, qf, PERM);
    __syncwarp();
    if (lane == 0 && i + 1 < nblk) issue_q(i + 1);

    float m[2] = {-INFINITY, -INFINITY};
    float l[2] = {0.f, 0.f};
    float acc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

#pragma unroll kQmUnroll
    for (int s = 0; s < K; ++s) {
      const int seq = i * K + s;
      const int stage = seq % STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_kv + 8 * stage, (seq / STAGES) & 1));
      if (!ok) break;
      next_seq = seq + 1;
      const uint32_t kt = ring + stage * 2 * TB;
      if (PAD)  // real keys of this tile: 16 except in the one that holds the last real token
        fwd_chunk<D, true>(qf, kt, kt + TB, min(kBlock, g.nv - (srow[seq] - bh_i * g.N)), P.scale_log2, m, l, acc);
      else if (CAUSAL) {  // kNoPick: every key masked; the block's own keys: the causal diagonal
        const int r = srow[seq];
        fwd_chunk<D, false, false, true>(qf, kt, kt + TB, kBlock, P.scale_log2, m, l, acc, nullptr, 0, 0.f, 0,
                                         0xffffffffu, r < 0 ? -kBlock : (r == gb * kBlock ? 0 : kBlock - 1));
      } else
        fwd_chunk<D, false, POOL>(qf, kt, kt + TB, kBlock, P.scale_log2, m, l, acc, nullptr, 0, pool_log_bias<D>(g),
                                  PERM);
      __syncwarp();
      if (lane == 0 && seq + STAGES < total_loads) issue_kv(seq + STAGES);
    }
    if (!ok) break;
    for (int cc = 0; cc < g.coarse_pad / kBlock; ++cc)
      fwd_chunk<D, true>(qf, ck + cc * TB, cv + cc * TB, min(kBlock, g.coarse - cc * kBlock), P.scale_log2, m, l,
                         acc, &g, cc * kBlock, 0.f, 0, cmask >> (cc * kBlock));

    l[0] += __shfl_xor_sync(0xffffffffu, l[0], 1);
    l[0] += __shfl_xor_sync(0xffffffffu, l[0], 2);
    l[1] += __shfl_xor_sync(0xffffffffu, l[1], 1);
    l[1] += __shfl_xor_sync(0xffffffffu, l[1], 2);
    const int r0 = lane >> 2;
    const bool real0 = !PAD || r0 < qvalid, real1 = !PAD || r0 + 8 < qvalid;
    const int t0 = (gb - bh_i * n1) * kBlock;  // the block's first token in its head
    store_tile_bf16<D, LAYOUT>(acc, real0 ? 1.0f / l[0] : 0.0f, real1 ? 1.0f / l[1] : 0.0f, sq + (i & 1) * TB, o, g,
                               bh_i, t0);
    if ((lane & 3) == 0) {
      const float lse0 = real0 ? (m[0] + log2f(l[0])) * kLn2 : 0.0f;
      const float lse1 = real1 ? (m[1] + log2f(l[1])) * kLn2 : 0.0f;
      const long long lrow = token_row<LAYOUT>(g, bh_i, t0);
      lse[lrow + block_row_offset<LAYOUT>(g, r0)] = lse0;
      lse[lrow + block_row_offset<LAYOUT>(g, r0 + 8)] = lse1;
      if (LAYOUT == kZStore) {  // the quadtree-ordered copy that dQ reads
        lse_z[(long long)gb * kBlock + r0] = lse0;
        lse_z[(long long)gb * kBlock + r0 + 8] = lse1;
      }
    }
  }
  if (!ok) {
    // A copy did not land in time (recorded as LLSA_ERR_TIMEOUT).  Give each copy still in
    // flight one more bounded wait so none lands after this warp has gone.
    for (int seq = next_seq; seq < min(total_loads, next_seq + STAGES); ++seq)
      mbar_wait(bar_kv + 8 * (seq % STAGES), (seq / STAGES) & 1);
    for (int i = next_q; i < min(nblk, next_q + 2); ++i) mbar_wait(bar_q + 8 * (i & 1), (i >> 1) & 1);
  }
}

}  // namespace llsa
