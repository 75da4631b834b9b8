// Key-major dK/dV of step 4b on the 5th-generation tensor cores (tcgen05, TMEM accumulators).
//
// All query blocks that selected a fine key block j share its 16 keys, so their work batches:
// a batch is up to 8 of those query blocks (128 queries) and four MMAs cover it:
//   S   [128 x 16] = Q_b  K_j^T        (M = 128 queries, N = 16 keys, K = 64)      -> TMEM
//   dP  [128 x 16] = dO_b V_j^T                                                    -> TMEM
//   (4 warps read one query row each from TMEM: P = exp2(S*scale*log2e - LSE*log2e),
//    dS = P (dP - Delta); rows of missing query blocks are 0; P^T and dS^T go to shared
//    memory as bf16 in the 128-byte-swizzled K-major layout)
//   dV^T[64 x 16] += dO_b^T P          (M = 64 channels, N = 16, K = 128 queries)  -> TMEM
//   dK^T[64 x 16] += Q_b^T  dS
// Roles (one CTA = 6 warps, persistent over the key blocks j = blockIdx.x + i * gridDim.x
// that some query block selected):
//   warp 4     TMA producer: scans the CTA's rows, skips empty ones, publishes each work item
//              in a shared-memory ring and loads K_j/V_j tiles (2 buffers) and the Q/dO
//              tiles + LSE/Delta of each batch (2 stages); no multicast
//   warp 5     allocates TMEM; one thread issues the MMAs, committing to mbarriers
//   warps 0-3  elementwise softmax-gradient step and the epilogue (each warp owns the 32
//              TMEM lanes of its quarter)
// The epilogue adds the mean-pool adjoint of the ancestors' coarse gradients (weight 1/16^l),
// scales dK by 1/sqrt(D) and writes bf16 rows; key blocks no query selected are written by
// dkdv_empty_rows_kernel.  Every wait is bounded; after a timeout each role stops issuing
// work, lets its copies or products in flight complete and leaves; TMEM is freed at the end.
#pragma once

#include "attn_bwd.cuh"

namespace llsa {

constexpr int kTcBatch = 8;                 // query blocks per batch (M = 128)
constexpr int kTcThreads = 192;             // 4 compute warps + producer warp + MMA warp
constexpr int kTcCols = 128;                // TMEM columns per CTA
// TMEM columns: S[2] at 0/16, dP[2] at 32/48, dV^T[2] at 64/80, dK^T[2] at 96/112
constexpr uint32_t kColS = 0, kColDP = 32, kColDV = 64, kColDK = 96;

// Shared-memory map (bytes from the 1024-aligned base).
struct TcMap {
  static constexpr int kv = 0;                       // [2][K tile, V tile]          8 KB
  static constexpr int stage = 8192;                 // [2][Q tiles x8, dO tiles x8] 64 KB
  static constexpr int stage_bytes = 32768;
  static constexpr int pds = stage + 2 * stage_bytes;  // [2][P^T 4 KB, dS^T 4 KB]  16 KB
  static constexpr int pds_bytes = 8192;
  static constexpr int lsed = pds + 2 * pds_bytes;   // [2][128 LSE, 128 Delta] fp32  2 KB
  static constexpr int bars = lsed + 2 * 256 * 4;    // 16 mbarriers
  static constexpr int ring = bars + 16 * 8;       // work items (TcItem x 8)
  static constexpr int taddr = ring + 8 * 16;
  static constexpr int total = taddr + 16;
};
constexpr int kTcSmemBytes = 1024 + TcMap::total;

// mbarrier slots
enum : int { kBarKvFull = 0, kBarKvFree = 2, kBarStFull = 4, kBarStFree = 6, kBarSReady = 8, kBarPdsReady = 10,
             kBarAccReady = 12, kBarAccFree = 14 };

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t sbo) {
  // 128-byte swizzle, version 1, leading byte offset 16 (unused by these swizzled layouts)
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait that ignores the global abort shortcut (used to drain copies in flight).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > 2000000000LL) return;
}

// Work item of the key-major schedule, published by the producer warp in a shared-memory
// ring before the first copy of the item lands; len < 0 ends the schedule.
struct TcItem {
  int bh, j, len, pad;
};
constexpr int kTcRing = 8;  // items in flight are at most 4 apart (2 stages, deferred epilogue)

__global__ void __launch_bounds__(kTcThreads, 1) attn_bwd_dkdv_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, AttnParams P,
    const float* __restrict__ lse, const int* __restrict__ row_ptr, const int* __restrict__ col,
    const float* __restrict__ ws, __nv_bfloat16* __restrict__ dk_out, __nv_bfloat16* __restrict__ dv_out) {
  pdl_enter();
  extern __shared__ uint8_t tc_smem_raw[];
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  uint8_t* base = align1024(tc_smem_raw);
  const uint32_t sb = smem_u32(base);
  const uint32_t bars = sb + TcMap::bars;
  uint32_t* taddr_s = reinterpret_cast<uint32_t*>(base + TcMap::taddr);
  volatile TcItem* ring = reinterpret_cast<volatile TcItem*>(base + TcMap::ring);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n1 = g.n[1];
  const int E = n1 * g.K;
  const int total = g.BH * n1;

  // ---- set-up: barriers, zeroed stage tiles (rows of absent query blocks stay finite), TMEM
  if (threadIdx.x == 0) {
    for (int b = 0; b < 16; ++b) {
      const bool many = (b == kBarPdsReady || b == kBarPdsReady + 1 || b == kBarAccFree || b == kBarAccFree + 1);
      mbar_init(bars + 8 * b, many ? 128 : 1);
    }
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < 2 * TcMap::stage_bytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base + TcMap::stage)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(taddr_s)),
                 "r"(kTcCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *taddr_s;
  bool ok = true;

  if (warp == 4) {
    // ================================================================ TMA producer (whole warp)
    // The CTA's rows j = blockIdx.x + i * gridDim.x are scanned 32 at a time (one row_ptr pair
    // per lane, the next chunk prefetched); empty rows are skipped with a ballot.  A row's
    // query blocks are read 32 at a time, the next row's first 32 prefetched; lane i < nq
    // issues the copies of batch slot i after lane 0 has registered the batch's byte count.
    const int* rp = row_ptr + g.rp_off[1];
    const int* cb = col + g.idx_off[1];
    auto row_of = [&](int i, int& rs, int& len) {
      const int kb = blockIdx.x + i * gridDim.x;
      rs = 0;
      len = 0;
      if (kb < total) {
        const int* r = rp + (long long)(kb >> g.log_n1) * (n1 + 1) + (kb & (n1 - 1));
        const int a = __ldg(r), b = __ldg(r + 1);
        if (a < 0 || b > E || a > b) {
          record_error(LLSA_ERR_INTERNAL);
        } else {
          rs = a;
          len = b - a;
        }
      }
    };
    auto first_cols = [&](int kb, int rs, int len) {
      return lane < len ? __ldg(cb + (long long)(kb >> g.log_n1) * E + rs + lane) : 0;
    };
    int gp = 0, x = 0;
    int issued_st[2] = {-1, -1}, issued_kv[2] = {-1, -1};  // last batch / item issued per buffer
    int c_rs, c_len;
    row_of(lane, c_rs, c_len);
    for (int ci = 0; ok && blockIdx.x + ci * gridDim.x < total; ci += 32) {
      uint32_t mask = __ballot_sync(0xffffffffu, c_len > 0);
      int n_rs, n_len;
      row_of(ci + 32 + lane, n_rs, n_len);
      int mine = 0;
      if (mask) {
        const int src = __ffs(mask) - 1;
        mine = first_cols(blockIdx.x + (ci + src) * gridDim.x, __shfl_sync(0xffffffffu, c_rs, src),
                          __shfl_sync(0xffffffffu, c_len, src));
      }
      while (mask && ok) {
        const int src = __ffs(mask) - 1;
        mask &= mask - 1;
        const int kb = blockIdx.x + (ci + src) * gridDim.x;
        const int rs = __shfl_sync(0xffffffffu, c_rs, src), len = __shfl_sync(0xffffffffu, c_len, src);
        int mine_next = 0;
        if (mask) {
          const int nsrc = __ffs(mask) - 1;
          mine_next = first_cols(blockIdx.x + (ci + nsrc) * gridDim.x, __shfl_sync(0xffffffffu, c_rs, nsrc),
                                 __shfl_sync(0xffffffffu, c_len, nsrc));
        }
        const int bh = kb >> g.log_n1, j = kb & (n1 - 1);
        const int kvb = x & 1;
        if (x >= 2) ok = ok && __all_sync(0xffffffffu, mbar_wait(bars + 8 * (kBarKvFree + kvb), ((x >> 1) - 1) & 1));
        if (ok && lane == 0) {
          const int row = bh * g.N + j * kBlock;
          const uint32_t kvt = sb + TcMap::kv + kvb * 2 * kTileBytes;
          mbar_expect_tx(bars + 8 * (kBarKvFull + kvb), 2 * kTileBytes);
          tma_load_2d(kvt, &tm_k, 0, row, bars + 8 * (kBarKvFull + kvb));
          tma_load_2d(kvt + kTileBytes, &tm_v, 0, row, bars + 8 * (kBarKvFull + kvb));
        }
        if (ok) issued_kv[kvb] = x;
        const int* cl = cb + (long long)bh * E + rs;
        for (int c0 = 0; c0 < len && ok; c0 += 32) {
          const int m = checked_index(c0 == 0 ? mine : (c0 + lane < len ? __ldg(cl + c0 + lane) : 0), n1);
          for (int b0 = c0; b0 < min(len, c0 + 32); b0 += kTcBatch) {
            const int s = gp & 1;
            if (gp >= 2) ok = ok && __all_sync(0xffffffffu, mbar_wait(bars + 8 * (kBarStFree + s), ((gp >> 1) - 1) & 1));
            const int nq = min(kTcBatch, len - b0);
            const int p = __shfl_sync(0xffffffffu, m, (b0 - c0 + lane) & 31);
            if (!ok) break;
            const uint32_t bar = bars + 8 * (kBarStFull + s);
            if (lane == 0) {
              if (b0 == 0) {
                ring[x % kTcRing].bh = bh;
                ring[x % kTcRing].j = j;
                ring[x % kTcRing].len = len;
              }
              mbar_expect_tx(bar, nq * (2 * kTileBytes + 2 * kBlock * 4));
            }
            __syncwarp();
            if (lane < nq) {
              const uint32_t st = sb + TcMap::stage + s * TcMap::stage_bytes;
              float* ls = reinterpret_cast<float*>(base + TcMap::lsed + s * 1024);
              const int row = (bh * n1 + p) * kBlock;
              tma_load_2d(st + lane * kTileBytes, &tm_q, 0, row, bar);
              tma_load_2d(st + 8 * kTileBytes + lane * kTileBytes, &tm_do, 0, row, bar);
              bulk_load(smem_u32(ls + lane * kBlock), lse + row, kBlock * 4, bar);
              bulk_load(smem_u32(ls + 128 + lane * kBlock), ws + W.delta + row, kBlock * 4, bar);
            }
            issued_st[s] = gp;
            ++gp;
          }
        }
        mine = mine_next;
        ++x;
      }
      c_rs = n_rs;
      c_len = n_len;
    }
    // end of schedule: a terminal item completes the next stage phase without copies
    if (ok && gp >= 2) ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (kBarStFree + (gp & 1)), ((gp >> 1) - 1) & 1));
    if (ok && lane == 0) {
      ring[x % kTcRing].len = -1;
      mbar_arrive(bars + 8 * (kBarStFull + (gp & 1)));
    }
    if (!ok && lane == 0) {  // let the copies still in flight land before the CTA can exit
      for (int s = 0; s < 2; ++s)
        if (issued_st[s] >= 0) mbar_drain(bars + 8 * (kBarStFull + s), (issued_st[s] >> 1) & 1);
      for (int b = 0; b < 2; ++b)
        if (issued_kv[b] >= 0) mbar_drain(bars + 8 * (kBarKvFull + b), (issued_kv[b] >> 1) & 1);
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    // Two cursors walk the batch sequence: one issues the score products (S, dP) of a batch
    // once its tiles have landed, the other the gradient products (dV^T, dK^T) once the
    // compute warps have written its P and dS.  The thread polls both and issues whichever
    // is ready, so a batch's gradient products never wait for the next batch's copies.
    if (lane == 0) {
      constexpr uint32_t id_s = umma_idesc(128, 16, 0, 0);   // S, dP: A = Q_b / dO_b, B = K / V (K-major)
      constexpr uint32_t id_g = umma_idesc(64, 16, 1, 0);    // dV^T, dK^T: A = dO_b / Q_b (MN-major)
      struct Cursor {
        int x, b, nb, gm;  // item, batch within it (nb = 0: item not read yet), global batch
        __device__ void advance() {
          ++gm;
          if (++b == nb) {
            ++x;
            b = 0;
            nb = 0;
          }
        }
      };
      Cursor c12{0, 0, 0, 0}, c34{0, 0, 0, 0};
      bool live12 = true;
      long long t0 = clock64();
      unsigned idle = 0;
      uint32_t last_bar = 0, last_par = 0;  // the newest commit covers every product issued before it
      while (ok && (live12 || c34.gm < c12.gm)) {
        bool progressed = false;
        // score products of batch c12.gm: its S/dP columns were last read for batch gm-2,
        // whose gradient products the other cursor has already passed
        if (live12 && c12.gm <= c34.gm + 1) {
          const int s = c12.gm & 1, kvb = c12.x & 1;
          if (mbar_test(bars + 8 * (kBarStFull + s), (c12.gm >> 1) & 1)) {
            if (c12.nb == 0) {
              const int len = ring[c12.x % kTcRing].len;
              if (len < 0) live12 = false;
              else c12.nb = (len + kTcBatch - 1) / kTcBatch;
            }
            if (live12 && mbar_test(bars + 8 * (kBarKvFull + kvb), (c12.x >> 1) & 1)) {
              tc_fence_after();
              const uint32_t st = sb + TcMap::stage + s * TcMap::stage_bytes;
              const uint32_t kvt = sb + TcMap::kv + kvb * 2 * kTileBytes;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                umma_bf16(tmem + kColS + 16 * s, umma_desc(st + k * 32, 1024), umma_desc(kvt + k * 32, 1024), id_s,
                          k > 0);
                umma_bf16(tmem + kColDP + 16 * s, umma_desc(st + 8 * kTileBytes + k * 32, 1024),
                          umma_desc(kvt + kTileBytes + k * 32, 1024), id_s, k > 0);
              }
              umma_commit(bars + 8 * (kBarSReady + s));
              last_bar = bars + 8 * (kBarSReady + s);
              last_par = (c12.gm >> 1) & 1;
              if (c12.b == c12.nb - 1) umma_commit(bars + 8 * (kBarKvFree + kvb));
              c12.advance();
              progressed = true;
            }
          }
        }
        // gradient products of batch c34.gm; the first batch of an item also needs the
        // accumulators of item x-2 read out by the epilogue
        if (c34.gm < c12.gm) {
          if (c34.nb == 0) c34.nb = (ring[c34.x % kTcRing].len + kTcBatch - 1) / kTcBatch;
          const int s = c34.gm & 1, accb = c34.x & 1;
          const bool first = c34.b == 0, last = c34.b == c34.nb - 1;
          if ((!first || c34.x < 2 || mbar_test(bars + 8 * (kBarAccFree + accb), ((c34.x >> 1) - 1) & 1)) &&
              mbar_test(bars + 8 * (kBarPdsReady + s), (c34.gm >> 1) & 1)) {
            tc_fence_after();
            const uint32_t st = sb + TcMap::stage + s * TcMap::stage_bytes;
            const uint32_t pd = sb + TcMap::pds + s * TcMap::pds_bytes;
#pragma unroll
            for (int i = 0; i < kTcBatch; ++i) {
              const uint32_t acc = (first && i == 0) ? 0u : 1u;
              const uint32_t bo = (i >> 2) * kTileBytes + (i & 3) * 32;
              umma_bf16(tmem + kColDV + 16 * accb, umma_desc(st + 8 * kTileBytes + i * kTileBytes, 1024),
                        umma_desc(pd + bo, 1024), id_g, acc);
              umma_bf16(tmem + kColDK + 16 * accb, umma_desc(st + i * kTileBytes, 1024),
                        umma_desc(pd + 4096 + bo, 1024), id_g, acc);
            }
            umma_commit(bars + 8 * (kBarStFree + s));
            last_bar = bars + 8 * (kBarStFree + s);
            last_par = (c34.gm >> 1) & 1;
            if (last) umma_commit(bars + 8 * (kBarAccReady + accb));
            c34.advance();
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
          t0 = clock64();
        } else if ((++idle & 255u) == 0) {
          if (*reinterpret_cast<volatile int*>(&g_llsa_status) == LLSA_ERR_TIMEOUT) ok = false;
          if (clock64() - t0 > 4000000000LL) {
            record_error(LLSA_ERR_TIMEOUT);
            ok = false;
          }
        }
      }
      if (!ok && last_bar != 0) mbar_drain(last_bar, last_par);  // no product in flight at dealloc
    }
  } else {
    // ================================================================ compute warps 0-3
    // The epilogue of an item runs after the first batch of the next one, so its last
    // gradient products have completed by then (the accumulators are double-buffered in TMEM).
    // Lanes 0-15 of warp w hold channel d = 16 w + lane of dV^T/dK^T (M = 64 layout) and
    // store it for the 16 keys: one 32-byte sector per store instruction.
    const int t = threadIdx.x;  // query row of a batch, TMEM lane
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const int d = 16 * warp + (lane & 15);
    int gc = 0;
    // waits are voted across the warp: the TMEM loads below are warp-collective
    auto wait = [&](int bar, int parity) {
      ok = __all_sync(0xffffffffu, ok && mbar_wait(bars + 8 * bar, parity));
    };
    struct Pending {
      int valid, bh, j, x;
      float ak, av;
    } pend{0, 0, 0, 0, 0.f, 0.f};
    auto epilogue = [&]() {
      if (!pend.valid) return;
      const int accb = pend.x & 1;
      wait(kBarAccReady + accb, (pend.x >> 1) & 1);
      tc_fence_after();
      float a_v[16], a_k[16];
      tmem_ld16(tmem + lane_base + kColDV + 16 * accb, a_v);
      tmem_ld16(tmem + lane_base + kColDK + 16 * accb, a_k);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + 8 * (kBarAccFree + accb));
      if (ok && lane < 16) {
        const long long row0 = (long long)pend.bh * g.N + (long long)pend.j * kBlock;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          dk_out[(row0 + c) * kD + d] = __float2bfloat16_rn(a_k[c] * P.scale + pend.ak);
          dv_out[(row0 + c) * kD + d] = __float2bfloat16_rn(a_v[c] + pend.av);
        }
      }
      pend.valid = 0;
    };
    for (int x = 0; ok; ++x) {
      wait(kBarStFull + (gc & 1), (gc >> 1) & 1);
      if (!ok) break;
      const int len = ring[x % kTcRing].len;
      if (len < 0) break;
      const int bh = ring[x % kTcRing].bh, j = ring[x % kTcRing].j;
      // ancestors' coarse gradients of channel d (levels 2..L), summed after the first batch
      float rk[kMaxLevels], rv[kMaxLevels];
      {
        int span = 1, nl = n1;
        long long cg_level = 0;
#pragma unroll
        for (int lev = 2; lev <= kMaxLevels; ++lev) {
          rk[lev - 1] = rv[lev - 1] = 0.f;
          if (lev <= g.L) {
            span *= kBlock;
            nl /= kBlock;
            const long long r = cg_level + ((long long)bh * nl + j / span) * kD + d;
            rk[lev - 1] = __ldg(ws + W.cg_k + r);
            rv[lev - 1] = __ldg(ws + W.cg_v + r);
            cg_level += (long long)g.BH * nl * kD;
          }
        }
      }
      const int nb = (len + kTcBatch - 1) / kTcBatch;
      for (int b = 0; b < nb; ++b) {
        const int s = gc & 1;
        const int nq = min(kTcBatch, len - b * kTcBatch);
        if (b > 0) wait(kBarStFull + s, (gc >> 1) & 1);
        wait(kBarSReady + s, (gc >> 1) & 1);
        float sv[16], dpv[16];
        tc_fence_after();
        tmem_ld16(tmem + lane_base + kColS + 16 * s, sv);
        tmem_ld16(tmem + lane_base + kColDP + 16 * s, dpv);
        tmem_wait_ld();
        const float* ls = reinterpret_cast<const float*>(base + TcMap::lsed + s * 1024);
        const bool valid = ok && (t >> 4) < nq;
        const float l2 = valid ? ls[t] * kLog2e : 0.f;
        const float dl = valid ? ls[128 + t] : 0.f;
        // the P/dS buffer was last read by the gradient products of batch gc-2
        if (gc >= 2) wait(kBarStFree + s, ((gc >> 1) - 1) & 1);
        uint8_t* pd = base + TcMap::pds + s * TcMap::pds_bytes;
        const int blk = t >> 6, qq = t & 63;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p = valid ? ex2(fmaf(sv[c], P.scale_log2, -l2)) : 0.f;
          const float ds = valid ? p * (dpv[c] - dl) : 0.f;
          const uint32_t off = blk * kTileBytes + swz(c, qq >> 3) + (qq & 7) * 2;
          *reinterpret_cast<__nv_bfloat16*>(pd + off) = __float2bfloat16_rn(p);
          *reinterpret_cast<__nv_bfloat16*>(pd + 4096 + off) = __float2bfloat16_rn(ds);
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bars + 8 * (kBarPdsReady + s));
        ++gc;
        if (b == 0) epilogue();  // the previous item's
        if (!ok) break;
      }
      // mean-pool adjoint: weight 1/16^l for the level-l ancestor, the same for the 16 keys
      float ak = 0.f, av = 0.f, wgt = 1.0f / kBlock;
#pragma unroll
      for (int lev = 2; lev <= kMaxLevels; ++lev) {
        wgt *= 1.0f / kBlock;
        ak += wgt * rk[lev - 1];
        av += wgt * rv[lev - 1];
      }
      pend = Pending{1, bh, j, x, ak, av};
    }
    epilogue();
  }

  // ---- tear-down: every role has finished its schedule; free TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols));
  }
}

// dK, dV of fine key blocks that no query block selected: only the mean-pool adjoint of the
// ancestors' coarse gradients (the same value for the 16 tokens).  One warp per key block;
// rows with query blocks are left to the key-major kernel.
__global__ void __launch_bounds__(128) dkdv_empty_rows_kernel(AttnParams P, const int* __restrict__ row_ptr,
                                                               const float* __restrict__ ws,
                                                               __nv_bfloat16* __restrict__ dk_out,
                                                               __nv_bfloat16* __restrict__ dv_out) {
  pdl_enter();
  const Geometry& g = P.g;
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int lane = lane_id();
  const int n1 = g.n[1];
  const int kb = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (kb >= g.BH * n1) return;
  const int bh = kb >> g.log_n1;
  const int j = kb & (n1 - 1);
  const int* rp = row_ptr + g.rp_off[1] + (long long)bh * (n1 + 1);
  if (__ldg(rp + j + 1) != __ldg(rp + j)) return;
  float2 ak = make_float2(0.f, 0.f), av = make_float2(0.f, 0.f);  // channels 2 lane, 2 lane + 1
  int span = 1, nl = n1;
  float wgt = 1.0f / kBlock;
  long long cg_level = 0;
  for (int lev = 2; lev <= g.L; ++lev) {
    span *= kBlock;
    wgt *= 1.0f / kBlock;
    nl /= kBlock;
    const long long r = cg_level + ((long long)bh * nl + j / span) * kD + 2 * lane;
    const float2 xk = *reinterpret_cast<const float2*>(ws + W.cg_k + r);
    const float2 xv = *reinterpret_cast<const float2*>(ws + W.cg_v + r);
    ak.x += wgt * xk.x;
    ak.y += wgt * xk.y;
    av.x += wgt * xv.x;
    av.y += wgt * xv.y;
    cg_level += (long long)g.BH * nl * kD;
  }
  const uint32_t pk = pack_bf16(ak.x, ak.y), pv = pack_bf16(av.x, av.y);
  const long long row0 = (long long)bh * g.N + (long long)j * kBlock;
#pragma unroll
  for (int r = 0; r < kBlock; ++r) {
    reinterpret_cast<uint32_t*>(dk_out + (row0 + r) * kD)[lane] = pk;
    reinterpret_cast<uint32_t*>(dv_out + (row0 + r) * kD)[lane] = pv;
  }
}

}  // namespace llsa
