// Step 5: the sparse index transpose (skill page "Log Linear Sparse Attention", Core
// Technique 3: the backward pass needs, for every key block, the query blocks that selected
// it, and building a dense query x key mask for that would cost O(n^2)).
//
// For each problem (level l, batch b, head h) the n_l x K list idx becomes a CSR matrix
// (row_ptr, col) of the inverse relation with queries ascending in every row.  It is a
// two-digit stable counting sort of the E = n_l * K entries, with no atomics anywhere:
//
//   1. transpose_hist_kernel    one CTA per 4096-entry tile: per-warp bucket counts
//                               (bucket = key / W, at most 64 buckets) via __match_any_sync,
//                               summed into hist[bucket][tile].
//   2. transpose_scatter_kernel one CTA per tile: bucket offsets from a scan of hist, then a
//                               stable scatter of (key, query) pairs into bucket order.
//   3. transpose_bucket_kernel  one CTA per bucket: per-key counts (warp-private, again via
//                               __match_any_sync), a scan that writes row_ptr, and a stable
//                               scatter of the queries into col.
//
// Every count has exactly one writer per step (the leader lane of each group of equal
// digits in a warp, on warp-private counters), so the result is deterministic.  Warps
// always walk contiguous entry ranges in order, and entries are laid out query-major, so
// equal keys keep ascending query order through both scatters.
// Work is O(E + buckets * tiles) per problem; all levels, batches and heads share each launch.
#pragma once

#include "llsa_common.cuh"

namespace llsa {

constexpr int kTrThreads = 256;
constexpr int kTrWarps = kTrThreads / 32;
constexpr int kTrTile = 4096;                  // entries per tile CTA
constexpr int kTrWarpSeg = kTrTile / kTrWarps;  // 512 entries per warp
constexpr int kTrMaxBuckets = 64;
constexpr int kTrMaxBucketKeys = 1024;          // n_l <= 65536 keys / 64 buckets

struct TransposeLevel {
  int n;            // keys (= queries) at this level
  int E;            // n * K entries per problem
  int tiles;        // ceil(E / kTrTile)
  int nb;           // buckets per problem
  int wshift;       // log2(keys per bucket)
  int cta_tiles;    // first tile-CTA of this level in kernels 1-2
  int cta_buckets;  // first bucket-CTA of this level in kernel 3
  long long hist_off;  // int offset of this level's hist in the workspace
  long long ent_off;   // entry offset of this level (same as idx/col level offset)
  long long rp_off;    // row_ptr offset of this level
};

struct TransposeGeo {
  int L, BH, K;
  TransposeLevel lv[kMaxLevels];
};

__device__ __forceinline__ int tr_level_of(const TransposeGeo& t, int cta, bool buckets) {
  int l = 0;
#pragma unroll
  for (int i = 1; i < kMaxLevels; ++i)
    if (i < t.L && cta >= (buckets ? t.lv[i].cta_buckets : t.lv[i].cta_tiles)) l = i;
  return l;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Per-warp bucket counts of the warp's contiguous segment of one tile.
__device__ __forceinline__ void tr_warp_bucket_counts(const int* __restrict__ keys, int E, int n, int wshift,
                                                      int seg_begin, int seg_end, int* cnt_w) {
  const int lane = lane_id();
  for (int base = seg_begin; base < seg_end; base += 32) {
    const int e = base + lane;
    bool valid = e < seg_end;
    int key = valid ? __ldg(keys + e) : 0;
    if (valid && (unsigned)key >= (unsigned)n) {
      record_error(LLSA_ERR_INTERNAL);
      valid = false;
    }
    const int b = valid ? (key >> wshift) : (-1 - lane);
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    if (valid && lane == __ffs(peers) - 1) cnt_w[b] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kTrThreads) transpose_hist_kernel(TransposeGeo tg, const int* __restrict__ idx,
                                                                    int* __restrict__ ws_hist) {
  pdl_enter();
  __shared__ int cnt[kTrWarps][kTrMaxBuckets];
  const int l = tr_level_of(tg, blockIdx.x, false);
  const TransposeLevel& L = tg.lv[l];
  const int local = blockIdx.x - L.cta_tiles;
  const int bh = local / L.tiles;
  const int t = local - bh * L.tiles;
  for (int i = threadIdx.x; i < kTrWarps * kTrMaxBuckets; i += kTrThreads) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int w = threadIdx.x >> 5;
  const int seg_begin = t * kTrTile + w * kTrWarpSeg;
  const int seg_end = min(L.E, seg_begin + kTrWarpSeg);
  const int* keys = idx + L.ent_off + (long long)bh * L.E;
  tr_warp_bucket_counts(keys, L.E, L.n, L.wshift, seg_begin, seg_end, cnt[w]);
  __syncthreads();
  for (int b = threadIdx.x; b < L.nb; b += kTrThreads) {
    int s = 0;
#pragma unroll
    for (int ww = 0; ww < kTrWarps; ++ww) s += cnt[ww][b];
    ws_hist[L.hist_off + ((long long)bh * L.nb + b) * L.tiles + t] = s;
  }
}

// Exclusive scan of up to 64 values held in smem, by warp 0; also returns the total.
__device__ __forceinline__ void tr_scan64(int* vals, int count, int* total_out) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int a = (2 * lane < count) ? vals[2 * lane] : 0;
    int b = (2 * lane + 1 < count) ? vals[2 * lane + 1] : 0;
    int s = a + b;
    int incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const int excl = incl - s;
    if (2 * lane < count) vals[2 * lane] = excl;
    if (2 * lane + 1 < count) vals[2 * lane + 1] = excl + a;
    if (lane == 31 && total_out) *total_out = incl;
  }
}

__global__ void __launch_bounds__(kTrThreads) transpose_scatter_kernel(TransposeGeo tg, const int* __restrict__ idx,
                                                                       const int* __restrict__ ws_hist,
                                                                       uint32_t* __restrict__ ws_ent) {
  pdl_enter();
  __shared__ int cnt[kTrWarps][kTrMaxBuckets];
  __shared__ int tot[kTrMaxBuckets];
  __shared__ int pre[kTrMaxBuckets];
  const int l = tr_level_of(tg, blockIdx.x, false);
  const TransposeLevel& L = tg.lv[l];
  const int local = blockIdx.x - L.cta_tiles;
  const int bh = local / L.tiles;
  const int t = local - bh * L.tiles;
  const int* hist = ws_hist + L.hist_off + (long long)bh * L.nb * L.tiles;

  for (int i = threadIdx.x; i < kTrWarps * kTrMaxBuckets; i += kTrThreads) (&cnt[0][0])[i] = 0;
  for (int b = threadIdx.x; b < L.nb; b += kTrThreads) {
    int s = 0, p = 0;
    for (int tt = 0; tt < L.tiles; ++tt) {
      const int h = hist[b * L.tiles + tt];
      s += h;
      if (tt < t) p += h;
    }
    tot[b] = s;
    pre[b] = p;
  }
  __syncthreads();
  tr_scan64(tot, L.nb, nullptr);  // tot[b] <- start of bucket b
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int seg_begin = t * kTrTile + w * kTrWarpSeg;
  const int seg_end = min(L.E, seg_begin + kTrWarpSeg);
  const int* keys = idx + L.ent_off + (long long)bh * L.E;
  tr_warp_bucket_counts(keys, L.E, L.n, L.wshift, seg_begin, seg_end, cnt[w]);
  __syncthreads();
  // per-warp write cursors: bucket start + earlier tiles + earlier warps of this tile
  for (int b = threadIdx.x; b < L.nb; b += kTrThreads) {
    int run = tot[b] + pre[b];
#pragma unroll
    for (int ww = 0; ww < kTrWarps; ++ww) {
      const int c = cnt[ww][b];
      cnt[ww][b] = run;
      run += c;
    }
  }
  __syncthreads();
  uint32_t* out = ws_ent + L.ent_off + (long long)bh * L.E;
  const int K = tg.K;
  for (int base = seg_begin; base < seg_end; base += 32) {
    const int e = base + lane;
    bool valid = e < seg_end;
    const int key = valid ? __ldg(keys + e) : 0;
    valid = valid && (unsigned)key < (unsigned)L.n;
    const int b = valid ? (key >> L.wshift) : (-1 - lane);
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    if (valid) {
      const int dst = cnt[w][b] + __popc(peers & lanemask_lt());
      out[dst] = ((uint32_t)key << 16) | (uint32_t)(e / K);
    }
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) cnt[w][b] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kTrThreads) transpose_bucket_kernel(TransposeGeo tg, const uint32_t* __restrict__ ws_ent,
                                                                      const int* __restrict__ ws_hist,
                                                                      int* __restrict__ row_ptr, int* __restrict__ col) {
  pdl_enter();
  __shared__ int kc[kTrWarps][kTrMaxBucketKeys];
  __shared__ int kpre[kTrMaxBucketKeys];
  __shared__ int part[kTrThreads];
  __shared__ int red[kTrWarps][2];
  const int l = tr_level_of(tg, blockIdx.x, true);
  const TransposeLevel& L = tg.lv[l];
  const int local = blockIdx.x - L.cta_buckets;
  const int bh = local / L.nb;
  const int b = local - bh * L.nb;
  const int W = 1 << L.wshift;
  const int tid = threadIdx.x;
  const int w = tid >> 5;
  const int lane = tid & 31;

  // bucket start (all entries of lower buckets) and size, from hist
  const int* hist = ws_hist + L.hist_off + (long long)bh * L.nb * L.tiles;
  int s_before = 0, s_mine = 0;
  for (int i = tid; i < (b + 1) * L.tiles; i += kTrThreads) {
    const int h = hist[i];
    if (i < b * L.tiles) s_before += h; else s_mine += h;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s_before += __shfl_xor_sync(0xffffffffu, s_before, off);
    s_mine += __shfl_xor_sync(0xffffffffu, s_mine, off);
  }
  if (lane == 0) {
    red[w][0] = s_before;
    red[w][1] = s_mine;
  }
  for (int i = tid; i < kTrWarps * W; i += kTrThreads) kc[i / W][i % W] = 0;
  __syncthreads();
  int start = 0, size = 0;
#pragma unroll
  for (int ww = 0; ww < kTrWarps; ++ww) {
    start += red[ww][0];
    size += red[ww][1];
  }

  // per-key counts, warp-private, each warp on a contiguous segment of the bucket
  const uint32_t* ent = ws_ent + L.ent_off + (long long)bh * L.E + start;
  const int seg = (size + kTrWarps - 1) / kTrWarps;
  const int seg_begin = min(size, w * seg);
  const int seg_end = min(size, seg_begin + seg);
  const int kbase = b * W;
  for (int base = seg_begin; base < seg_end; base += 32) {
    const int e = base + lane;
    bool valid = e < seg_end;
    int kl = valid ? (int)(ent[e] >> 16) - kbase : (-1 - lane);
    if (valid && (unsigned)kl >= (unsigned)W) {  // cannot happen for entries written by the scatter
      record_error(LLSA_ERR_INTERNAL);
      valid = false;
      kl = -1 - lane;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, kl);
    if (valid && lane == __ffs(peers) - 1) kc[w][kl] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per key: prefix over warps (in place) and total
  for (int k = tid; k < W; k += kTrThreads) {
    int run = 0;
#pragma unroll
    for (int ww = 0; ww < kTrWarps; ++ww) {
      const int c = kc[ww][k];
      kc[ww][k] = run;
      run += c;
    }
    kpre[k] = run;
  }
  __syncthreads();
  // exclusive scan of kpre over the W keys: each thread scans a run of ceil(W/256) keys
  const int per = (W + kTrThreads - 1) / kTrThreads;
  const int k0 = tid * per;
  int local_sum = 0;
  for (int k = k0; k < min(W, k0 + per); ++k) local_sum += kpre[k];
  part[tid] = local_sum;
  __syncthreads();
  if (tid < 32) {
    int acc = 0;
    for (int i = 0; i < kTrThreads / 32; ++i) acc += part[lane * (kTrThreads / 32) + i];
    int incl = acc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - acc;
    for (int i = 0; i < kTrThreads / 32; ++i) {
      const int v = part[lane * (kTrThreads / 32) + i];
      part[lane * (kTrThreads / 32) + i] = run;
      run += v;
    }
  }
  __syncthreads();
  {
    int run = part[tid];
    for (int k = k0; k < min(W, k0 + per); ++k) {
      const int c = kpre[k];
      kpre[k] = run;
      run += c;
    }
  }
  __syncthreads();
  int* rp = row_ptr + L.rp_off + (long long)bh * (L.n + 1);
  for (int k = tid; k < W && kbase + k < L.n; k += kTrThreads) rp[kbase + k] = start + kpre[k];  // last bucket may be partial
  if (b == L.nb - 1 && tid == 0) rp[L.n] = start + size;
  // scatter queries to their final CSR slots
  for (int k = tid; k < W; k += kTrThreads) {
#pragma unroll
    for (int ww = 0; ww < kTrWarps; ++ww) kc[ww][k] += start + kpre[k];
  }
  __syncthreads();
  int* cl = col + L.ent_off + (long long)bh * L.E;
  for (int base = seg_begin; base < seg_end; base += 32) {
    const int e = base + lane;
    bool valid = e < seg_end;
    const uint32_t v = valid ? ent[e] : 0u;
    int kl = valid ? (int)(v >> 16) - kbase : (-1 - lane);
    if (valid && (unsigned)kl >= (unsigned)W) {
      valid = false;
      kl = -1 - lane;
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, kl);
    if (valid) cl[kc[w][kl] + __popc(peers & lanemask_lt())] = (int)(v & 0xffffu);
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) kc[w][kl] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace llsa
