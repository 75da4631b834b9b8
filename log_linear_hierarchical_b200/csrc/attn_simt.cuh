// Steps 4a/4b for fp32 inputs: plain fp32 CUDA-core kernels with the same KV lists,
// workspace layout and coarse-gradient reduction as the bf16 tensor-core kernels.  fp32
// tensor-core modes round operands to 10 mantissa bits, which would not meet a 1e-4
// tolerance, so this path uses FMA units.  It is the small-problem / full-precision path;
// the bf16 kernels are the throughput path.
#pragma once

#include "attn_bwd.cuh"

namespace llsa {

constexpr int kSimtThreads = 128;

// KV list of a query block in these kernels: 16K fine tokens, then (level-1 variant) the K
// selected blocks' level-1 pyramid rows, then the C coarse pyramid rows.
__host__ __device__ inline int simt_coarse_start(const Geometry& g) { return kBlock * g.K + (g.pool1 ? g.K : 0); }
__host__ __device__ inline int simt_T(const Geometry& g) { return simt_coarse_start(g) + g.coarse; }

// Score bias of list entry e (scaled units): ln 16 for a level-1 pooled entry and the
// coarse entries' bias, both under the log-count variant only.
__device__ __forceinline__ float simt_entry_bias(const Geometry& g, int e) {
  if (e < kBlock * g.K) return 0.0f;
  const int c0 = simt_coarse_start(g);
  if (e < c0) return g.log_bias ? kLn16 : 0.0f;
  return coarse_log_bias(g, e - c0);
}

// Row pointers of block p's KV list (see simt_coarse_start), and whether each entry is a
// real token (a fine token at or past n_valid of a padded sequence is not; pooled entries,
// being selected, always are).
template <int D>
__device__ __forceinline__ void simt_kv_rows(const Geometry& g, int bh, int p, const float* __restrict__ k,
                                             const float* __restrict__ v, const float* __restrict__ k_pyr,
                                             const float* __restrict__ v_pyr, const int* __restrict__ idx,
                                             const float** krow, const float** vrow, int* real) {
  const int K = g.K;
  const int n1 = g.n[1];
  const int T = simt_T(g);
  const int c0 = simt_coarse_start(g);
  for (int e = threadIdx.x; e < T; e += blockDim.x) {
    long long r;
    const float* kb;
    const float* vb;
    int is_real = 1;
    if (e < kBlock * K) {
      const int j = checked_index(__ldg(idx + g.idx_off[1] + ((long long)bh * n1 + p) * K + e / kBlock), n1);
      const int t = j * kBlock + (e % kBlock);
      r = token_row(g, bh, t);
      is_real = t < g.nv;
      kb = k;
      vb = v;
    } else if (e < c0) {  // level-1 pooled token of selected block e - 16K
      const int j = checked_index(__ldg(idx + g.idx_off[1] + ((long long)bh * n1 + p) * K + (e - kBlock * K)), n1);
      r = (long long)bh * n1 + j;
      kb = k_pyr + g.pyr_off[1];
      vb = v_pyr + g.pyr_off[1];
    } else {
      int lev;
      const int jj = coarse_token(g, idx, bh, p, e - c0, lev);
      r = (long long)bh * g.n[lev] + jj;
      kb = k_pyr + g.pyr_off[lev];
      vb = v_pyr + g.pyr_off[lev];
    }
    krow[e] = kb + r * D;
    vrow[e] = vb + r * D;
    real[e] = is_real;
  }
}

template <int D>
__device__ __forceinline__ float dotD(const float* a, const float* b) {
  float s = 0.f;
#pragma unroll 16
  for (int d = 0; d < D; ++d) s = fmaf(a[d], b[d], s);
  return s;
}

// One CTA per query block.  smem: q[16][D], krow[T], vrow[T], S[16][T], real[T].  Padding
// queries of a padded sequence write O = 0 and LSE = 0; padding keys are left out.
template <int D>
__global__ void __launch_bounds__(kSimtThreads) attn_fwd_f32_kernel(Geometry g, float scale,
                                                                    const float* __restrict__ q,
                                                                    const float* __restrict__ k,
                                                                    const float* __restrict__ v,
                                                                    const float* __restrict__ k_pyr,
                                                                    const float* __restrict__ v_pyr,
                                                                    const int* __restrict__ idx, float* __restrict__ o,
                                                                    float* __restrict__ lse) {
  pdl_enter();
  extern __shared__ __align__(16) uint8_t simt_smem[];
  const int T = simt_T(g);
  const int gb = blockIdx.x;
  const int bh = gb / g.n[1];
  const int p = gb - bh * g.n[1];
  float* qs = reinterpret_cast<float*>(simt_smem);
  const float** krow = reinterpret_cast<const float**>(qs + kBlock * D);
  const float** vrow = krow + T;
  float* S = reinterpret_cast<float*>(vrow + T);
  int* real = reinterpret_cast<int*>(S + kBlock * T);
  const int qvalid = g.nv - p * kBlock;  // real queries of the block (>= 16 unless padded)
  for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x)
    qs[i] = i / D < qvalid ? q[token_row(g, bh, p * kBlock + i / D) * D + i % D] : 0.0f;
  simt_kv_rows<D>(g, bh, p, k, v, k_pyr, v_pyr, idx, krow, vrow, real);
  __syncthreads();
  for (int pr = threadIdx.x; pr < kBlock * T; pr += blockDim.x) {
    const int qi = pr / T;
    const int e = pr - qi * T;
    S[pr] = real[e] ? dotD<D>(qs + qi * D, krow[e]) * scale + simt_entry_bias(g, e) : -INFINITY;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int qi = warp; qi < kBlock; qi += blockDim.x >> 5) {
    float* row = S + qi * T;
    float m = -INFINITY;
    for (int e = lane; e < T; e += 32) m = fmaxf(m, row[e]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int e = lane; e < T; e += 32) {
      const float pe = expf(row[e] - m);
      row[e] = pe;
      l += pe;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = 1.0f / l;
    for (int e = lane; e < T; e += 32) row[e] *= inv;
    if (lane == 0) lse[token_row(g, bh, p * kBlock + qi)] = qi < qvalid ? m + logf(l) : 0.0f;
  }
  __syncthreads();
  for (int od = threadIdx.x; od < kBlock * D; od += blockDim.x) {
    const int qi = od / D;
    const int d = od - qi * D;
    const float* prow = S + qi * T;
    float acc = 0.f;
    for (int e = 0; e < T; ++e)
      if (real[e]) acc = fmaf(prow[e], vrow[e][d], acc);
    o[token_row(g, bh, p * kBlock + qi) * D + d] = qi < qvalid ? acc : 0.0f;
  }
}

template <int D>
inline size_t simt_fwd_smem(const Geometry& g) {
  const int T = simt_T(g);
  return sizeof(float) * kBlock * D + 2 * sizeof(void*) * T + sizeof(float) * kBlock * T + sizeof(int) * T;
}

// Query-major fp32 backward.  One CTA per level-2 group (16 query blocks) when L >= 2, so
// the coarse partials match the bf16 path's layout; one CTA per query block when L = 1.
// smem: q, dO [16][D]; krow, vrow [T]; P, dS [16][T]; cacc_k, cacc_v [C][D]; delta[16];
// real[T].  Padding queries and keys of a padded sequence take part in nothing (their rows
// are read as zeros and their P and dS are 0), and padding queries get dQ = 0.
template <int D>
__global__ void __launch_bounds__(kSimtThreads) attn_bwd_dq_f32_kernel(
    Geometry g, float scale, const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ o, const float* __restrict__ lse, const float* __restrict__ dO,
    const float* __restrict__ k_pyr, const float* __restrict__ v_pyr, const int* __restrict__ idx,
    float* __restrict__ dq_out, float* __restrict__ ws) {
  pdl_enter();
  extern __shared__ __align__(16) uint8_t simt_smem[];
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int T = simt_T(g);
  const int C = g.coarse;
  const int per_cta = g.L >= 2 ? kBlock : 1;
  float* qs = reinterpret_cast<float*>(simt_smem);
  float* ds_ = qs + kBlock * D;  // dO rows
  const float** krow = reinterpret_cast<const float**>(ds_ + kBlock * D);
  const float** vrow = krow + T;
  float* Pm = reinterpret_cast<float*>(vrow + T);
  float* dS = Pm + kBlock * T;
  float* cacc_k = dS + kBlock * T;
  float* cacc_v = cacc_k + C * D;
  float* delta = cacc_v + C * D;
  int* real = reinterpret_cast<int*>(delta + kBlock);
  for (int i = threadIdx.x; i < 2 * C * D; i += blockDim.x) cacc_k[i] = 0.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int bi = 0; bi < per_cta; ++bi) {
    const int gb = blockIdx.x * per_cta + bi;
    const int bh = gb / g.n[1];
    const int p = gb - bh * g.n[1];
    const long long rbase = (long long)gb * kBlock;
    const int qvalid = g.nv - p * kBlock;  // real queries of the block (>= 16 unless padded)
    __syncthreads();
    for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) {
      const bool rq = i / D < qvalid;
      const long long src = token_row(g, bh, p * kBlock + i / D) * D + i % D;
      qs[i] = rq ? q[src] : 0.0f;
      ds_[i] = rq ? dO[src] : 0.0f;
    }
    simt_kv_rows<D>(g, bh, p, k, v, k_pyr, v_pyr, idx, krow, vrow, real);
    __syncthreads();
    for (int qi = warp; qi < kBlock; qi += blockDim.x >> 5) {
      float s = 0.f;
      if (qi < qvalid)
        for (int d = lane; d < D; d += 32)
          s = fmaf(ds_[qi * D + d], o[token_row(g, bh, p * kBlock + qi) * D + d], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) {
        delta[qi] = s;
        ws[W.lsd + rbase + qi] = s;
      }
    }
    __syncthreads();
    for (int pr = threadIdx.x; pr < kBlock * T; pr += blockDim.x) {
      const int qi = pr / T;
      const int e = pr - qi * T;
      if (!real[e] || qi >= qvalid) {
        Pm[pr] = dS[pr] = 0.0f;
        continue;
      }
      const float bias = simt_entry_bias(g, e);
      const float pe = expf(dotD<D>(qs + qi * D, krow[e]) * scale + bias - lse[token_row(g, bh, p * kBlock + qi)]);
      const float dp = dotD<D>(ds_ + qi * D, vrow[e]);
      Pm[pr] = pe;
      dS[pr] = pe * (dp - delta[qi]);
    }
    __syncthreads();
    for (int od = threadIdx.x; od < kBlock * D; od += blockDim.x) {
      const int qi = od / D;
      const int d = od - qi * D;
      float acc = 0.f;
      for (int e = 0; e < T; ++e)
        if (real[e]) acc = fmaf(dS[qi * T + e], krow[e][d], acc);
      dq_out[token_row(g, bh, p * kBlock + qi) * D + d] = acc * scale;
    }
    for (int cd = threadIdx.x; cd < C * D; cd += blockDim.x) {
      const int c = cd / D;
      const int d = cd - c * D;
      const int e = simt_coarse_start(g) + c;
      float ak = 0.f, av = 0.f;
      for (int qi = 0; qi < kBlock; ++qi) {
        ak = fmaf(dS[qi * T + e], qs[qi * D + d], ak);
        av = fmaf(Pm[qi * T + e], ds_[qi * D + d], av);
      }
      cacc_k[cd] += ak;
      cacc_v[cd] += av;
    }
  }
  if (g.L < 2) return;
  __syncthreads();
  const int group = blockIdx.x;
  for (int cd = threadIdx.x; cd < C * D; cd += blockDim.x) {
    ws[W.part_k + (long long)group * C * D + cd] = cacc_k[cd];
    ws[W.part_v + (long long)group * C * D + cd] = cacc_v[cd];
  }
}

template <int D>
inline size_t simt_dq_smem(const Geometry& g) {
  const int T = simt_T(g);
  return sizeof(float) * 2 * kBlock * D + 2 * sizeof(void*) * T + sizeof(float) * 2 * kBlock * T +
         sizeof(float) * 2 * g.coarse * D + sizeof(float) * kBlock + sizeof(int) * T;
}

// Key-major fp32 backward: one CTA per fine key block; thread t owns D / 8 of the 16 x D dK
// and dV outputs.  Padding keys and queries of a padded sequence are read as zeros and
// masked out; padding positions get dK = dV = 0.  smem: K_j, V_j, Q_p, dO_p [16][64]; Pt, dSt [16][16]; lse, delta [16].
// Level-1 variant: the block's level-1 pyramid row (kbar, vbar) is in the list of every query
// block p of the row; its dK, dV reach the 16 rows with weight 1/16, which adds p / 16 to
// every Pt entry of query i and dS / 16 to every dSt entry.
template <int D>
__global__ void __launch_bounds__(kSimtThreads) attn_bwd_dkdv_f32_kernel(
    Geometry g, float scale, const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ k_pyr, const float* __restrict__ v_pyr, const float* __restrict__ lse,
    const float* __restrict__ dO, const int* __restrict__ row_ptr, const int* __restrict__ col,
    const float* __restrict__ ws, float* __restrict__ dk_out, float* __restrict__ dv_out) {
  pdl_enter();
  __shared__ float ks[kBlock * D], vs[kBlock * D], qs[kBlock * D], dos[kBlock * D];
  __shared__ float Pt[kBlock][kBlock + 1], dSt[kBlock][kBlock + 1];
  __shared__ float ls[kBlock], dl[kBlock];
  __shared__ float kbar[D], vbar[D], pool_p[kBlock], pool_ds[kBlock];
  const BwdWorkspace W = bwd_workspace_layout(g);
  const int n1 = g.n[1];
  const int kb = blockIdx.x;
  const int bh = kb / n1;
  const int j = kb - bh * n1;
  const int kvalid = g.nv - j * kBlock;  // real keys of the block (>= 16 unless padded)
  for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) {
    const bool rk = i / D < kvalid;
    const long long src = token_row(g, bh, j * kBlock + i / D) * D + i % D;
    ks[i] = rk ? k[src] : 0.0f;
    vs[i] = rk ? v[src] : 0.0f;
  }
  if (g.pool1)
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      kbar[d] = k_pyr[g.pyr_off[1] + (long long)kb * D + d];
      vbar[d] = v_pyr[g.pyr_off[1] + (long long)kb * D + d];
    }
  const int E = n1 * g.K;
  const int* rp = row_ptr + g.rp_off[1] + (long long)bh * (n1 + 1);
  int rs = rp[j], re = rp[j + 1];
  if (rs < 0 || re > E || rs > re) {
    if (threadIdx.x == 0) record_error(LLSA_ERR_INTERNAL);
    rs = re = 0;
  }
  const int* cl = col + g.idx_off[1] + (long long)bh * E;
  constexpr int PER = kBlock * D / kSimtThreads;  // outputs per thread
  float ak[PER], av[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) ak[i] = av[i] = 0.f;
  for (int e = rs; e < re; ++e) {
    const int p = checked_index(cl[e], n1);
    const long long qrow0 = (long long)bh * g.N + (long long)p * kBlock;
    const int qvalid = g.nv - p * kBlock;
    __syncthreads();
    for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) {
      const bool rq = i / D < qvalid;
      const long long src = token_row(g, bh, p * kBlock + i / D) * D + i % D;
      qs[i] = rq ? q[src] : 0.0f;
      dos[i] = rq ? dO[src] : 0.0f;
    }
    if (threadIdx.x < kBlock) {
      ls[threadIdx.x] = lse[token_row(g, bh, p * kBlock + threadIdx.x)];
      dl[threadIdx.x] = ws[W.lsd + qrow0 + threadIdx.x];
    }
    __syncthreads();
    if (g.pool1 && threadIdx.x < kBlock) {  // the level-1 entry's p / 16 and dS / 16 per query
      const int qi = threadIdx.x;
      const float pb = expf(dotD<D>(kbar, qs + qi * D) * scale + (g.log_bias ? kLn16 : 0.0f) - ls[qi]);
      pool_p[qi] = pb * (1.0f / kBlock);
      pool_ds[qi] = pb * (dotD<D>(vbar, dos + qi * D) - dl[qi]) * (1.0f / kBlock);
    }
    if (g.pool1) __syncthreads();
    for (int pr = threadIdx.x; pr < kBlock * kBlock; pr += blockDim.x) {
      const int kk = pr / kBlock;
      const int qi = pr - kk * kBlock;
      if (kk >= kvalid || qi >= qvalid) {  // padding of a padded sequence
        Pt[kk][qi] = dSt[kk][qi] = 0.0f;
        continue;
      }
      const float pe = expf(dotD<D>(ks + kk * D, qs + qi * D) * scale - ls[qi]);
      const float dp = dotD<D>(vs + kk * D, dos + qi * D);
      Pt[kk][qi] = g.pool1 ? pe + pool_p[qi] : pe;
      dSt[kk][qi] = g.pool1 ? fmaf(pe, dp - dl[qi], pool_ds[qi]) : pe * (dp - dl[qi]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int od = threadIdx.x + i * kSimtThreads;
      const int kk = od / D;
      const int d = od - kk * D;
      float a = 0.f, b = 0.f;
      for (int qi = 0; qi < kBlock; ++qi) {
        a = fmaf(dSt[kk][qi], qs[qi * D + d], a);
        b = fmaf(Pt[kk][qi], dos[qi * D + d], b);
      }
      ak[i] += a;
      av[i] += b;
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int od = threadIdx.x + i * kSimtThreads;
    const int kk = od / D;
    const int d = od - kk * D;
    float rk = ak[i] * scale, rv = av[i];
    int span = 1;
    for (int lev = 2; lev <= g.L; ++lev) {
      span *= kBlock;
      const float wgt = 1.0f / (float)pool_count(g, lev, j / span);  // 1 / 16^l unless padding cuts it
      const long long crow = W.cg_off[lev] + ((long long)bh * g.n[lev] + j / span) * D + d;
      rk += wgt * ws[W.cg_k + crow];
      rv += wgt * ws[W.cg_v + crow];
    }
    const long long dst = token_row(g, bh, j * kBlock + kk) * D + d;
    dk_out[dst] = kk < kvalid ? rk : 0.0f;
    dv_out[dst] = kk < kvalid ? rv : 0.0f;
  }
}

}  // namespace llsa
