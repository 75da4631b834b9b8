// Step 5: the sparse index transpose (skill page "Log Linear Sparse Attention", Core
// Technique 3: the backward pass needs, for every key block, the query blocks that selected
// it, and building a dense query x key mask for that would cost O(n^2)).
//
// For each problem (level l, batch b, head h) the n_l x K list idx becomes a CSR matrix
// (row_ptr, col) of the inverse relation with queries ascending in every row; kNoPick
// entries (the empty slots of causal lists) are dropped, so row_ptr[n_l] counts the picks.
// It is a two-digit stable counting sort of the E = n_l * K entries, with no atomics:
//
//   1. transpose_hist_kernel    one CTA per 4096-entry tile: per-warp bucket counts
//                               (bucket = key / W, at most 64 buckets) via __match_any_sync,
//                               summed into hist[bucket][tile].
//   2. transpose_scan_kernel    one CTA per problem: an exclusive scan of hist in (bucket,
//                               tile) order, in place, so hist[bucket][tile] becomes the
//                               first output slot of that tile's entries of that bucket.
//                               Only for problems of more than kTrScanTiles tiles; below
//                               that, kernels 3 and 4 sum the few counts they need.
//   3. transpose_scatter_kernel one CTA per tile: a stable scatter of (key, query) pairs into
//                               bucket order from those offsets.
//   4. transpose_bucket_kernel  one CTA per bucket: per-key counts (warp-private, again via
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
  int cta_tiles;    // first tile-CTA of this level in the hist and scatter kernels
  int cta_buckets;  // first bucket-CTA of this level in the bucket kernel
  int hstride;      // ints of hist per problem: nb * tiles counts, then their total
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
    if (valid && key == kNoPick) valid = false;  // a short causal list's empty slot: no entry
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
    ws_hist[L.hist_off + (long long)bh * L.hstride + b * L.tiles + t] = s;
  }
}

// Exclusive scan of up to 64 values held in smem, by warp 0.
__device__ __forceinline__ void tr_scan64(int* vals, int count) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int a = (2 * lane < count) ? vals[2 * lane] : 0;
    const int b = (2 * lane + 1 < count) ? vals[2 * lane + 1] : 0;
    const int s = a + b;
    int incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const int excl = incl - s;
    if (2 * lane < count) vals[2 * lane] = excl;
    if (2 * lane + 1 < count) vals[2 * lane + 1] = excl + a;
  }
}

// Problems with at most this many tiles per level skip the scan launch: each scatter and
// bucket CTA then sums the few hist entries it needs itself (O(nb * tiles) per CTA, which
// is less than a launch costs at that size).  Larger problems scan hist once.
constexpr int kTrScanTiles = 16;

// Exclusive scan, in place, of the nb * tiles counts of one problem (level, b, h), laid out
// bucket-major: afterwards hist[b][t] is the slot of the first entry of bucket b that tile
// t holds, i.e. (entries of buckets < b) + (entries of bucket b in tiles < t).  Each thread
// scans a contiguous run; the runs' totals are scanned by warp 0.  The total (every entry
// with an in-range key) goes to hist[nb * tiles].  O(nb * tiles) per problem.
__global__ void __launch_bounds__(kTrThreads) transpose_scan_kernel(TransposeGeo tg, int* __restrict__ ws_hist) {
  pdl_enter();
  __shared__ int part[kTrThreads];
  const int l = blockIdx.x / tg.BH;
  const int bh = blockIdx.x - l * tg.BH;
  const TransposeLevel& L = tg.lv[l];
  const int count = L.nb * L.tiles;
  int* hist = ws_hist + L.hist_off + (long long)bh * L.hstride;
  const int tid = threadIdx.x;
  const int per = (count + kTrThreads - 1) / kTrThreads;
  const int i0 = min(count, tid * per);
  const int i1 = min(count, i0 + per);
  int sum = 0;
  for (int i = i0; i < i1; ++i) sum += hist[i];
  part[tid] = sum;
  __syncthreads();
  if (tid < 32) {
    constexpr int kPer = kTrThreads / 32;
    int acc = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc += part[tid * kPer + k];
    int incl = acc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (tid >= off) incl += o;
    }
    int run = incl - acc;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int v = part[tid * kPer + k];
      part[tid * kPer + k] = run;
      run += v;
    }
  }
  __syncthreads();
  int run = part[tid];
  for (int i = i0; i < i1; ++i) {
    const int v = hist[i];
    hist[i] = run;
    run += v;
  }
  if (tid == kTrThreads - 1) hist[count] = run;  // entries with an in-range key
}

// SCANNED: hist was scanned by transpose_scan_kernel; otherwise each CTA sums the raw
// counts it needs (only for problems of at most kTrScanTiles tiles).
template <bool SCANNED>
__global__ void __launch_bounds__(kTrThreads) transpose_scatter_kernel(TransposeGeo tg, const int* __restrict__ idx,
                                                                       const int* __restrict__ ws_hist,
                                                                       uint32_t* __restrict__ ws_ent) {
  pdl_enter();
  __shared__ int cnt[kTrWarps][kTrMaxBuckets];
  __shared__ int start[kTrMaxBuckets];
  __shared__ int lower[kTrMaxBuckets];
  const int l = tr_level_of(tg, blockIdx.x, false);
  const TransposeLevel& L = tg.lv[l];
  const int local = blockIdx.x - L.cta_tiles;
  const int bh = local / L.tiles;
  const int t = local - bh * L.tiles;
  const int* hist = ws_hist + L.hist_off + (long long)bh * L.hstride;

  for (int i = threadIdx.x; i < kTrWarps * kTrMaxBuckets; i += kTrThreads) (&cnt[0][0])[i] = 0;
  if (SCANNED) {
    for (int b = threadIdx.x; b < L.nb; b += kTrThreads) start[b] = hist[b * L.tiles + t];
  } else {
    // start of bucket b in this tile: entries of lower buckets (a scan of the bucket
    // totals) plus entries of bucket b in earlier tiles
    for (int b = threadIdx.x; b < L.nb; b += kTrThreads) {
      int tot = 0, pre = 0;
      for (int tt = 0; tt < L.tiles; ++tt) {
        const int h = hist[b * L.tiles + tt];
        tot += h;
        if (tt < t) pre += h;
      }
      start[b] = tot;
      lower[b] = pre;
    }
    __syncthreads();
    tr_scan64(start, L.nb);
    __syncthreads();
    for (int b = threadIdx.x; b < L.nb; b += kTrThreads) start[b] += lower[b];
  }
  __syncthreads();
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int seg_begin = t * kTrTile + w * kTrWarpSeg;
  const int seg_end = min(L.E, seg_begin + kTrWarpSeg);
  const int* keys = idx + L.ent_off + (long long)bh * L.E;
  tr_warp_bucket_counts(keys, L.E, L.n, L.wshift, seg_begin, seg_end, cnt[w]);
  __syncthreads();
  // per-warp write cursors: this tile's first slot of the bucket + earlier warps of this tile
  for (int b = threadIdx.x; b < L.nb; b += kTrThreads) {
    int run = start[b];
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

template <bool SCANNED>
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

  // bucket start and size: from the scanned hist, its first tile's slot and the next
  // bucket's (the total for the last bucket); from the raw hist, the sums of the counts of
  // the lower buckets and of its own
  const int* hist = ws_hist + L.hist_off + (long long)bh * L.hstride;
  int start, size;
  if (SCANNED) {
    start = hist[b * L.tiles];
    size = hist[(b + 1) * L.tiles] - start;
  } else {
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
    __syncthreads();
    start = size = 0;
#pragma unroll
    for (int ww = 0; ww < kTrWarps; ++ww) {
      start += red[ww][0];
      size += red[ww][1];
    }
  }
  for (int i = tid; i < kTrWarps * W; i += kTrThreads) kc[i / W][i % W] = 0;
  __syncthreads();

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
