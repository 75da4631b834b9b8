// Shared device helpers and geometry for the LLSA sm_100a kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/llsa.h"

namespace llsa {

constexpr int kBlock = 16;      // tokens per block (README usage section: block_size=16)
constexpr int kMaxD = 128;      // head widths D = 64 and 128 are built (every kernel is templated on D)
constexpr int kMaxLevels = 4;
constexpr int kSubTileBytes = 2048;  // 16 rows x 128 bytes: 64 bf16 channels of a 16-token tile

// TMA ring depths of the attention kernels (forward, query-major dQ, key-major dK/dV).  A
// sweep on B200 at the headline workload preferred 2 stages everywhere: deeper rings cost
// more shared memory per warp than they hide, since occupancy hides the L2 latency better.
#ifndef LLSA_FWD_STAGES
#define LLSA_FWD_STAGES 2
#endif
#ifndef LLSA_DQ_STAGES
#define LLSA_DQ_STAGES 2
#endif
#ifndef LLSA_KV_STAGES
#define LLSA_KV_STAGES 2
#endif
// Unroll of the key-major pair loop and of the query-major fine-tile loops (a sweep on B200
// at the headline workload, 1 -> 4: dK/dV 136.6 -> 131.9 us, forward 100.4 -> 91.6 us,
// dQ 116.6 -> 114.3 us; 8 was slower for the pair loop).
#ifndef LLSA_KV_UNROLL
#define LLSA_KV_UNROLL 4
#endif
#ifndef LLSA_QM_UNROLL
#define LLSA_QM_UNROLL 4
#endif
constexpr int kKvUnroll = LLSA_KV_UNROLL;
constexpr int kQmUnroll = LLSA_QM_UNROLL;

// Per-call geometry: level sizes and the level-major offsets of every packed buffer.
struct Geometry {
  int B, H, N, D, K, L, BH;
  int log_k, log_n1, log_n;              // log2 K, log2 n_1, log2 N where they are powers of two, else -1
  int n[kMaxLevels + 1];                 // n[l] = N / 16^l, l = 0..L
  long long pyr_off[kMaxLevels + 1];     // element offset of level l (1..L) in a pyramid
  long long idx_off[kMaxLevels + 1];     // element offset of level l in idx / col
  long long rp_off[kMaxLevels + 1];      // element offset of level l in row_ptr
  int coarse;                            // C coarse KV entries per query block: (L-1) K,
                                         // or (L-2) K + n_L under LLSA_FLAG_ALL_TOP
  int coarse_pad;                        // C rounded up to a multiple of 16
  int log_bias;                          // LLSA_FLAG_LOG_BIAS: coarse scores + ln(16^l)
  int top_first;                         // LLSA_FLAG_ALL_TOP (L >= 2): (L-2) K, the first
                                         // entry of the level-L part; C (never reached) otherwise
  int pool1;                             // LLSA_FLAG_LEVEL1: each selected fine block's
                                         // level-1 mean is one more KV entry
  int nv;                                // real tokens per sequence (N when not padded)
  int m[kMaxLevels + 1];                 // real tokens of level l: ceil(nv / 16^l)
  int grid;                              // LLSA_FLAG_GRID_ORDER: token rows in memory are in the
                                         // row-major order of a G x G grid (G = 2^log_g); the
                                         // path works in its quadtree (Z) order
  int log_g;
  int causal;                            // LLSA_FLAG_CAUSAL: keys at or before the query only
  int zcopy;                             // bf16 under LLSA_FLAG_GRID_ORDER: the step keeps
                                         // quadtree-ordered copies of q, k, v, dO and LSE
};

// The entry of a causal selection list that holds no pick (a query token with fewer than K
// candidates at or before it); as the largest int it keeps every list ascending.
constexpr int kNoPick = 0x7fffffff;

// Even bits of x, packed: bit 2i of x becomes bit i.
__host__ __device__ inline int compact_even_bits(int x) {
  x &= 0x55555555;
  x = (x | (x >> 1)) & 0x33333333;
  x = (x | (x >> 2)) & 0x0f0f0f0f;
  x = (x | (x >> 4)) & 0x00ff00ff;
  x = (x | (x >> 8)) & 0x0000ffff;
  return x;
}

// Row-major position r * side + c (side = 2^log_side) of quadtree index z, where c takes the
// even bits of z and r the odd ones (z = sum_b (2 r_b + c_b) 4^b: top-left, top-right,
// bottom-left, bottom-right at every scale).
__host__ __device__ inline int z_to_rowmajor(int z, int log_side) {
  return (compact_even_bits(z >> 1) << log_side) | compact_even_bits(z);
}

// Memory row of token t (in the path's Z order) of head bh: (b*H + h) * N + t, or the
// row-major grid position of t under LLSA_FLAG_GRID_ORDER.
__host__ __device__ inline long long token_row(const Geometry& g, int bh, int t) {
  return (long long)bh * g.N + (g.grid ? z_to_rowmajor(t, g.log_g) : t);
}

// How the bf16 attention kernels address q, k, v, dO and their outputs.  A template
// parameter, so the default instantiation carries no per-access test:
//   kFlat:   [B*H*N][D] rows in quadtree order (flat 2-D tensor maps);
//   kPadded: the same with rows at or past n_valid as padding (3-D maps read them as zeros);
//   kGrid:   row-major G x G grids (LLSA_FLAG_GRID_ORDER: 3-D patch maps, the tile_row map);
//   kCausal: flat rows under LLSA_FLAG_CAUSAL (diagonal blocks masked element-wise, lists
//            that may end in kNoPick, coarse entries attended only before the block);
//   kZStore: the one-call step under LLSA_FLAG_GRID_ORDER: q, k, v, dO and LSE are read
//            from quadtree-ordered copies (flat 2-D maps) and every output row is written
//            to its row-major grid position.
enum Layout : int { kFlat = 0, kPadded = 1, kGrid = 2, kCausal = 3, kZStore = 4 };

// The layout of a geometry, and whether its tile tensor map is the flat 2-D [B*H*N][D] view
// (kFlat, kCausal) rather than a 3-D one: the host's tensor map and the kernels' copy
// instruction must agree on the rank.
inline int layout_of(const Geometry& g) { return g.causal ? kCausal : g.grid ? kGrid : (g.nv < g.N ? kPadded : kFlat); }
__host__ __device__ constexpr bool flat_tile_map(int layout) {
  return layout == kFlat || layout == kCausal || layout == kZStore;
}

template <int LAYOUT>
__device__ __forceinline__ long long token_row(const Geometry& g, int bh, int t) {
  return (long long)bh * g.N + ((LAYOUT == kGrid || LAYOUT == kZStore) ? z_to_rowmajor(t, g.log_g) : t);
}

// Memory-row offset of row r (0..15) of a 16-token block from the row of its first token:
// r itself, or under grid order the pixel offset r_y G + r_x of quadtree position
// r = 8 y1 + 4 x1 + 2 y0 + x0 (r_y = 2 y1 + y0, r_x = 2 x1 + x0) -- the same as
// token_row(t0 + r) - token_row(t0) for a block-aligned t0, with a few bit operations.
template <int LAYOUT>
__device__ __forceinline__ long long block_row_offset(const Geometry& g, int r) {
  if constexpr (LAYOUT == kGrid || LAYOUT == kZStore)
    return ((long long)(((r >> 1) & 1) | ((r >> 2) & 2)) << g.log_g) + ((r & 1) | ((r >> 1) & 2));
  return r;
}

// Under LLSA_FLAG_GRID_ORDER a 16-token block is a 4 x 4 pixel patch that a TMA box brings
// in row by row (shared-memory row 4 r + c for pixel (r, c)), while the block's token order
// is the quadtree order (z = 8 r1 + 4 c1 + 2 r0 + c0): row z of the block is shared-memory
// row tile_row(z) (bits 1 and 2 swapped when `perm`, the identity otherwise).
__host__ __device__ inline int tile_row(int z, int perm) {
  const int x = ((z >> 1) ^ (z >> 2)) & perm;
  return z ^ (x * 6);
}

// Real tokens under level-l token j of a sequence with nv real tokens: clamp(nv - j 16^l,
// 0, 16^l) (16^l for every token when the sequence is not padded).
__host__ __device__ inline int pool_count(const Geometry& g, int l, int j) {
  const long long span = 1LL << (4 * l);
  const long long c = (long long)g.nv - (long long)j * span;
  return c <= 0 ? 0 : (c >= span ? (int)span : (int)c);
}

// x / K, x / n_1 and x / N, by a shift when the divisor is a power of two.
__host__ __device__ inline int div_k(const Geometry& g, int x) { return g.log_k >= 0 ? x >> g.log_k : x / g.K; }
__host__ __device__ inline int div_n1(const Geometry& g, int x) { return g.log_n1 >= 0 ? x >> g.log_n1 : x / g.n[1]; }
__host__ __device__ inline int div_n(const Geometry& g, int x) { return g.log_n >= 0 ? x >> g.log_n : x / g.N; }

// Level of coarse entry c (0 <= c < C): 2 + c / K, except that under the all-coarsest
// variant the entries from top_first on are level L.
__host__ __device__ inline int coarse_level(const Geometry& g, int c) {
  return c >= g.top_first ? g.L : 2 + div_k(g, c);
}

// Additive score bias of coarse entry c under the log-count enrichment variant, in units
// of the scaled score: ln(16^l) = l ln 16 for a level-l entry; 0 when it is off.
constexpr float kLn16 = 2.7725887222397811f;
__host__ __device__ inline float coarse_log_bias(const Geometry& g, int c) {
  return g.log_bias ? (float)coarse_level(g, c) * kLn16 : 0.0f;
}

// ---------------------------------------------------------------------------- status word
// One per device (a module global); kernels record the first error, llsa_device_status
// reads and clears it.
__device__ int g_llsa_status;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_llsa_status, 0, code); }

// Range check for every gathered index: an out-of-range value is replaced by 0 (always a
// valid row) and recorded, so a bad index array can never make a kernel read or write
// outside its buffers.
__device__ __forceinline__ int checked_index(int v, int n) {
  if ((unsigned)v >= (unsigned)n) {
    record_error(LLSA_ERR_INTERNAL);
    return 0;
  }
  return v;
}

// Token index (in its level) of coarse entry c of level-1 query block p of head bh: slot
// c % K of the list that p's level-l ancestor selected, or, in the level-L part of the
// all-coarsest variant, token c - top_first.  The index read from `idx` is range-checked.
// Under LLSA_FLAG_CAUSAL an entry is attended only if its token lies wholly before the block,
// i.e. its index is below the ancestor's (kNoPick and the ancestor itself are not); -1 then.
__device__ __forceinline__ int coarse_token(const Geometry& g, const int* __restrict__ idx, int bh, int p, int c,
                                            int& lev) {
  if (c >= g.top_first) {
    lev = g.L;
    return c - g.top_first;
  }
  lev = 2 + div_k(g, c);
  const int nl = g.n[lev];
  const int anc = p >> (4 * (lev - 1));  // p / 16^(l-1)
  const int slot = c - (lev - 2) * g.K;
  const int j = __ldg(idx + g.idx_off[lev] + ((long long)bh * nl + anc) * g.K + slot);
  if (g.causal && j >= anc) return -1;
  return checked_index(j, nl);
}

// Bit c set: coarse entry c of query block p is attended (every entry unless causal).
// Called by a whole warp; C <= 32.
__device__ __forceinline__ uint32_t coarse_visible_mask(const Geometry& g, const int* __restrict__ idx, int bh,
                                                        int p) {
  if (!g.causal) return 0xffffffffu;
  const int lane = threadIdx.x & 31;
  bool vis = false;
  if (lane < g.coarse) {
    int lev;
    vis = coarse_token(g, idx, bh, p, lane, lev) >= 0;
  }
  return __ballot_sync(0xffffffffu, vis);
}

// ---------------------------------------------------------------------------- smem / swizzle
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of (row, 16-byte chunk) in a 16 x 128-byte tile written by a TMA copy with
// CU_TENSOR_MAP_SWIZZLE_128B: the chunk index is XORed with row mod 8 (tile base 1024-aligned).
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------- tensor-core PTX
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A (16x16 bf16, row) * B (16x8 bf16, col) + D, fp32 accumulate.  Registers in and out
// only (no side effects), so the compiler may schedule it like arithmetic.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix held one row-pair per lane (the ldmatrix layout).
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// 2^x by the PTX ex2.approx.ftz.f32 instruction (relative error about 2^-22; subnormal
// results flush to zero, which only affects probabilities below 2^-126).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------- mbarrier / TMA
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Programmatic dependent launch.  Every kernel is launched with programmatic stream
// serialization, so it may be scheduled before the kernel ahead of it on the stream has
// finished.  pdl_wait blocks until that kernel has completed and its writes are visible
// (it returns at once for a kernel launched without the attribute).
// pdl_launch_dependents lets the next kernel's CTAs be scheduled once every CTA of this
// grid has issued it.  Every kernel issues it only after its own pdl_wait, so when a kernel
// starts, the kernel two places ahead of it on the stream has completed.  A kernel may
// therefore read, before its pdl_wait, only data written two or more kernels back or by
// work joined to its stream with an event; each such early read is documented where it is.
// (dK/dV, the last kernel of a step, signals before its deferred wait: the step's first
// kernel reads nothing before its own wait.)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_launch_dependents();
}

// Non-blocking test of the phase with the given parity (no suspend hint), for a thread that
// polls several barriers.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Limit of a bounded wait: about two seconds at the maximum SM clock.
constexpr long long kWaitLimitCycles = 4000000000LL;

// Bounded wait: gives up after `limit` SM cycles, records LLSA_ERR_TIMEOUT and returns
// false, so a copy that never lands cannot hang the GPU.  Once any wait has timed out (the
// status word holds LLSA_ERR_TIMEOUT) the others give up at their next check instead of
// spending their own limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int*>(&g_llsa_status) == LLSA_ERR_TIMEOUT) return false;
      if (clock64() - t0 > limit) {
        record_error(LLSA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Check of the timeout path of mbar_wait, the wait every kernel uses: one thread arms an
// mbarrier for 16 bytes of a transfer that is never issued (so no copy is ever in flight),
// waits on it with a limit of `limit` cycles, and the wait gives up and records
// LLSA_ERR_TIMEOUT.  Nothing else is touched.
__global__ void __launch_bounds__(32) bounded_wait_check_kernel(long long limit) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  mbar_init(b, 1);
  mbar_fence_init();
  mbar_expect_tx(b, 16);
  mbar_wait(b, 0, limit);
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// 4-D tiled TMA load (no multicast) of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}

// 3-D tiled TMA load (no multicast) of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// 2-D tiled TMA load (no multicast) of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Untiled bulk copy global -> shared (both 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

}  // namespace llsa
