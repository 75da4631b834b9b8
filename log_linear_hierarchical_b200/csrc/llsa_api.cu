// C ABI of the LLSA hot path (declarations and contracts in include/llsa.h).
// Single translation unit: every kernel header is included here, so the device status word
// is one module global per device.
#include <cudaTypedefs.h>

#include <mutex>
#include <new>

#include "attn_simt.cuh"
#include "probe.cuh"
#include "pyramid.cuh"
#include "pyramid_select.cuh"
#include "select.cuh"
#include "transpose.cuh"
#include "zorder.cuh"

using namespace llsa;

// Scratch of llsa_index_transpose_noalloc: one fixed array per device that loads the
// library.  Host code must not use this name as an address; it asks the runtime for the
// device address (cudaGetSymbolAddress) once per device.
static __device__ __align__(256) unsigned char g_llsa_noalloc_scratch[LLSA_NOALLOC_SCRATCH_BYTES];

namespace {

bool is_pow2(long long x) { return x > 0 && (x & (x - 1)) == 0; }

int ilog2(long long x) {
  int r = 0;
  while ((1LL << r) < x) ++r;
  return r;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

llsa_status validate(const llsa_shape* s) {
  if (!s) return LLSA_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->N < 1 || s->D < 1 || s->block < 1 || s->topk < 1 || s->levels < 1)
    return LLSA_ERR_INVALID_ARG;
  if (s->dtype != LLSA_BF16 && s->dtype != LLSA_F32) return LLSA_ERR_INVALID_ARG;
  if (s->flags & ~(LLSA_FLAG_LOG_BIAS | LLSA_FLAG_ALL_TOP | LLSA_FLAG_LEVEL1 | LLSA_FLAG_GRID_ORDER |
                   LLSA_FLAG_ONE_LAUNCH_SELECT | LLSA_FLAG_CAUSAL))
    return LLSA_ERR_INVALID_ARG;  // unknown flag bits
  if (s->n_valid < 0 || s->n_valid > s->N) return LLSA_ERR_INVALID_ARG;
  // N: any multiple of 16^L (the pages' implementation wants powers of two for N and topk;
  // the kernels here take any multiple and any topk)
  if (s->block != kBlock) return LLSA_ERR_UNSUPPORTED;
  if (s->D != 64 && s->D != 128) return LLSA_ERR_UNSUPPORTED;
  if (s->levels > kMaxLevels) return LLSA_ERR_UNSUPPORTED;
  if (s->N % (1LL << (4 * s->levels)) != 0) return LLSA_ERR_INVALID_ARG;  // n_L = N / 16^L whole
  const long long nL = (long long)s->N >> (4 * s->levels);
  if (s->topk > nL) return LLSA_ERR_INVALID_ARG;  // the coarsest level must hold K keys
  if (s->N > (1 << 20)) return LLSA_ERR_UNSUPPORTED;
  if (nL > 16384) return LLSA_ERR_UNSUPPORTED;
  if (s->topk > 64) return LLSA_ERR_UNSUPPORTED;
  if ((long long)(s->levels - 1) * s->topk > 32) return LLSA_ERR_UNSUPPORTED;
  if ((s->flags & LLSA_FLAG_ALL_TOP) && s->levels >= 2 && (long long)(s->levels - 2) * s->topk + nL > 96)
    return LLSA_ERR_UNSUPPORTED;  // the coarse entries of the all-coarsest variant
  if ((long long)s->B * s->H * s->N >= (1LL << 31)) return LLSA_ERR_UNSUPPORTED;
  if (s->n_valid != 0 && s->n_valid < s->N) {  // a padded sequence
    const long long span = 1LL << (4 * s->levels);
    if (s->topk > (s->n_valid + span - 1) / span) return LLSA_ERR_INVALID_ARG;  // K real coarsest tokens
    if (s->flags & ~LLSA_FLAG_ONE_LAUNCH_SELECT) return LLSA_ERR_UNSUPPORTED;  // default enrichment only
  }
  if (s->flags & LLSA_FLAG_CAUSAL) {  // bf16, the default enrichment, no padding, no grid order
    if (s->dtype != LLSA_BF16) return LLSA_ERR_UNSUPPORTED;
    if (s->flags & (LLSA_FLAG_LOG_BIAS | LLSA_FLAG_ALL_TOP | LLSA_FLAG_LEVEL1 | LLSA_FLAG_GRID_ORDER))
      return LLSA_ERR_UNSUPPORTED;
    if (s->n_valid != 0 && s->n_valid < s->N) return LLSA_ERR_UNSUPPORTED;
  }
  if (s->flags & LLSA_FLAG_GRID_ORDER) {  // a square grid of side 2^(log2 N / 2), 16 x 16 at least
    if (!is_pow2(s->N) || (ilog2(s->N) & 1)) return LLSA_ERR_INVALID_ARG;
    if (s->N < 256) return LLSA_ERR_UNSUPPORTED;
  }
  return LLSA_OK;
}

Geometry make_geometry(const llsa_shape* s) {
  Geometry g{};
  g.B = s->B;
  g.H = s->H;
  g.N = s->N;
  g.D = s->D;
  g.K = s->topk;
  g.L = s->levels;
  g.BH = s->B * s->H;
  for (int l = 0; l <= g.L; ++l) g.n[l] = s->N >> (4 * l);
  long long po = 0, io = 0, ro = 0;
  for (int l = 1; l <= g.L; ++l) {
    g.pyr_off[l] = po;
    g.idx_off[l] = io;
    g.rp_off[l] = ro;
    po += (long long)g.BH * g.n[l] * s->D;
    io += (long long)g.BH * g.n[l] * g.K;
    ro += (long long)g.BH * (g.n[l] + 1);
  }
  g.log_k = is_pow2(g.K) ? ilog2(g.K) : -1;
  g.log_n1 = is_pow2(g.n[1]) ? ilog2(g.n[1]) : -1;
  g.log_n = is_pow2(g.N) ? ilog2(g.N) : -1;
  const bool all_top = (s->flags & LLSA_FLAG_ALL_TOP) && g.L >= 2;
  g.coarse = all_top ? (g.L - 2) * g.K + g.n[g.L] : (g.L - 1) * g.K;
  g.coarse_pad = (g.coarse + kBlock - 1) / kBlock * kBlock;
  g.log_bias = (s->flags & LLSA_FLAG_LOG_BIAS) ? 1 : 0;
  g.top_first = all_top ? (g.L - 2) * g.K : g.coarse;
  g.pool1 = (s->flags & LLSA_FLAG_LEVEL1) ? 1 : 0;
  g.nv = (s->n_valid > 0 && s->n_valid < s->N) ? s->n_valid : s->N;
  g.grid = (s->flags & LLSA_FLAG_GRID_ORDER) ? 1 : 0;
  g.log_g = g.grid ? ilog2(s->N) / 2 : 0;
  g.causal = (s->flags & LLSA_FLAG_CAUSAL) ? 1 : 0;
  g.zcopy = (g.grid && s->dtype == LLSA_BF16) ? 1 : 0;
  for (int l = 0; l <= kMaxLevels; ++l) g.m[l] = l <= g.L ? (int)((g.nv + (1LL << (4 * l)) - 1) >> (4 * l)) : 0;
  return g;
}

TransposeGeo make_transpose_geo(const Geometry& g, long long* ent_total, long long* hist_total) {
  TransposeGeo t{};
  t.L = g.L;
  t.BH = g.BH;
  t.K = g.K;
  int cta_t = 0, cta_b = 0;
  long long hist = 0;
  for (int l = 1; l <= g.L; ++l) {
    TransposeLevel& L = t.lv[l - 1];
    L.n = g.n[l];
    L.E = g.n[l] * g.K;
    L.tiles = (L.E + kTrTile - 1) / kTrTile;
    int w = 1;  // keys per bucket: the smallest power of two giving at most kTrMaxBuckets buckets
    while ((L.n + w - 1) / w > kTrMaxBuckets) w <<= 1;
    L.nb = (L.n + w - 1) / w;
    L.wshift = ilog2(w);
    L.cta_tiles = cta_t;
    L.cta_buckets = cta_b;
    L.hstride = L.nb * L.tiles + 1;
    L.hist_off = hist;
    L.ent_off = g.idx_off[l];
    L.rp_off = g.rp_off[l];
    cta_t += g.BH * L.tiles;
    cta_b += g.BH * L.nb;
    hist += (long long)g.BH * L.hstride;
  }
  *ent_total = (long long)g.BH * g.K * [&] {
    long long s = 0;
    for (int l = 1; l <= g.L; ++l) s += g.n[l];
    return s;
  }();
  *hist_total = hist;
  return t;
}

size_t transpose_ws_bytes(const Geometry& g) {
  long long ent, hist;
  make_transpose_geo(g, &ent, &hist);
  return (size_t)(((ent + 63) & ~63LL) + hist) * 4;
}

// ---------------------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// q, k, v, dO as [B*H][n_valid][D] bf16 (row stride D, head stride N * D); box = 64
// channels (128 bytes, the swizzle span) x 16 rows x 1 head, so a 16-token tile is D / 64
// boxes at x = 0, 64.  Rows at or past n_valid (padding) are read as zeros.  Without
// padding the view is the flat [B*H*N][D] (box 64 x 16, row coordinate = flat token row).
// Under LLSA_FLAG_GRID_ORDER: [B*H*G][G][D] (pixel rows of every head's grid) with a
// 64-channel x 4 x 4 pixel box (one 16-token block of the quadtree order).
bool make_tile_map(CUtensorMap* m, const void* base, const Geometry& g, int lay) {
  auto fn = encode_fn();
  if (!fn) return false;
  // lay: the layout of the kernels that use the map; the rank here must match their
  // tma_load_tile<D, lay>
  if (lay == kGrid) {  // the heads' grids stacked: pixel rows of all heads, G pixels each
    const cuuint64_t G = 1ULL << g.log_g;
    cuuint64_t dims[3] = {(cuuint64_t)g.D, G, (cuuint64_t)g.BH * G};
    cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, G * g.D * 2};
    cuuint32_t box[3] = {64u, 4u, 4u};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  if (flat_tile_map(lay)) {  // no padding: one flat [B*H*N][D] view (cheaper per copy than 3-D)
    cuuint64_t dims[2] = {(cuuint64_t)g.D, (cuuint64_t)g.BH * g.N};
    cuuint64_t strides[1] = {(cuuint64_t)g.D * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)kBlock};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.nv, (cuuint64_t)g.BH};
  cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.N * g.D * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)kBlock, 1u};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The pyramid's view of a grid-order input: [B*H][G][G][D] (bf16 or fp32), box = one 16 x 16
// pixel patch of all D channels (a level-2 token), no swizzle.  A zeroed map when the input
// is in quadtree order (the pyramid then reads contiguous spans by bulk copy).
bool make_patch_map(CUtensorMap* m, const void* base, const Geometry& g, int dtype) {
  *m = CUtensorMap{};
  if (!g.grid) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t G = 1ULL << g.log_g;
  const cuuint64_t e = dtype == LLSA_BF16 ? 2 : 4;
  cuuint64_t dims[4] = {(cuuint64_t)g.D, G, G, (cuuint64_t)g.BH};
  cuuint64_t strides[3] = {(cuuint64_t)g.D * e, G * g.D * e, (cuuint64_t)g.N * g.D * e};
  cuuint32_t box[4] = {(cuuint32_t)g.D, 16u, 16u, 1u};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, dtype == LLSA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
            const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, 64] bf16 viewed as 2-D, box 64 x 16 with 128-byte swizzle (the gather probe).
bool make_probe_map(CUtensorMap* m, const void* base, long long rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {64u, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128u};
  cuuint32_t box[2] = {64u, (cuuint32_t)kBlock};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

llsa_status launch_status() { return cudaGetLastError() == cudaSuccess ? LLSA_OK : LLSA_ERR_CUDA; }

template <typename Kern>
bool allow_smem(Kern k, size_t bytes) {
  if (bytes <= 48 * 1024) return true;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess;
}

// Set while a public call whose first kernel reads data before its pdl_wait (the forward,
// and dQ in a build without the order phase) launches that kernel: the launch then goes
// without the attribute, so it starts only once everything ahead of it on the caller's
// stream has completed, whatever the caller launched there.  Inside a step the kernels
// ahead are this library's own and the pdl_wait ordering rule covers the early reads.
thread_local bool g_serial_next = false;

struct SerialFirstLaunch {
  SerialFirstLaunch() { g_serial_next = true; }
  ~SerialFirstLaunch() { g_serial_next = false; }
};

// Launch with programmatic stream serialization (see pdl_wait): the kernel may be scheduled
// while the one ahead of it on the stream drains; it waits for it on the device.  A failed
// launch is reported by cudaGetLastError, as for a triple-chevron launch.
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t cs, Args&&... args) {
  const bool serial = g_serial_next;
  g_serial_next = false;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = cs;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = serial ? 0 : 1;
  cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------- launch trace
enum KernelId {
  kKPyramidL12 = 1,
  kKPyramidUp,
  kKSelect,
  kKTransposeHist,
  kKTransposeScatter,
  kKTransposeBucket,
  kKFwdBf16,
  kKBwdDqBf16,
  kKBwdCoarseReduce,
  kKBwdDkdvBf16,
  kKFwdF32,
  kKBwdDqF32,
  kKBwdDkdvF32,
  kKBwdCoarseBf16,
  kKDkdvOrderCount,
  kKDkdvOrderScatter,
  kKZOrder,
  kKTransposeScan,
  kKWaitCheck,
  kKGatherProbe,
  kKPyramidSelect,
  kKNumKernels
};

const char* const kKernelNames[kKNumKernels] = {
    "unknown",           "pyramid_l12",        "pyramid_up",       "select",
    "transpose_hist",    "transpose_scatter",  "transpose_bucket", "attn_fwd_bf16",
    "attn_bwd_dq_bf16",  "coarse_grad_reduce", "attn_bwd_dkdv_bf16", "attn_fwd_f32",
    "attn_bwd_dq_f32",   "attn_bwd_dkdv_f32",  "attn_bwd_coarse_bf16", "dkdv_order_count",
    "dkdv_order_scatter", "zorder_permute",    "transpose_scan",   "bounded_wait_check",
    "gather_probe",      "pyramid_select"};

struct TraceState {
  cudaEvent_t* ev = nullptr;
  int32_t* ids = nullptr;
  int cap = 0;
  int used = 0;
};
thread_local TraceState g_trace;

// Launches through `f`, checks the launch, and records the trace events if tracing is on.
// Under stream capture the events become event-record nodes of the graph (external
// records), so a captured plan is traced each time it is launched.
void trace_record(cudaEvent_t e, cudaStream_t cs) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(cs, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, cs, cudaEventRecordExternal);
  else
    cudaEventRecord(e, cs);
}

template <class F>
llsa_status launch(int id, cudaStream_t cs, F&& f) {
  const bool tr = g_trace.ev != nullptr && g_trace.used < g_trace.cap;
  if (tr) trace_record(g_trace.ev[2 * g_trace.used], cs);
  f();
  const llsa_status st = launch_status();
  if (tr) {
    trace_record(g_trace.ev[2 * g_trace.used + 1], cs);
    g_trace.ids[g_trace.used] = id;
    ++g_trace.used;
  }
  return st;
}

constexpr int kFwdStages = LLSA_FWD_STAGES;
constexpr int kDqStages = LLSA_DQ_STAGES;
constexpr int kDkvStages = LLSA_KV_STAGES;
constexpr int kAttnWarps = 4;

template <int D>
llsa_status launch_coarse_reduce(const Geometry& g, float scale, const int32_t* idx, const int32_t* row_ptr,
                                 const int32_t* col, float* ws, cudaStream_t cs) {
  if (g.L < 2) return LLSA_OK;
  long long tokens = 0;
  for (int l = 2; l <= g.L; ++l) tokens += (long long)g.BH * g.n[l];
  return launch(kKBwdCoarseReduce, cs, [&] {
    launch_pdl(coarse_grad_reduce_kernel<D>, dim3((unsigned)tokens), dim3(kReduceWarps * 32), 0, cs, g, scale, idx, row_ptr, col, ws);
  });
}

// Device address of g_llsa_noalloc_scratch on the current device, looked up on the first
// call per device (with that device current) and remembered.
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

llsa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LLSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LLSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_llsa_noalloc_scratch) != cudaSuccess || p == nullptr) return LLSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return LLSA_OK;
}

}  // namespace

namespace {

// The backward in two phases.  The query side (dQ, Delta and the coarse-token partials)
// reads only the query-major selection; the key side (coarse-token gradients reduced
// through the level-l CSRs, then dK/dV through the level-1 CSR) needs the transpose, so a
// step can run the transpose concurrently with the forward and the query side.
// A third phase, the longest-first order of the fine key blocks for dK/dV, reads only the
// level-1 CSR and can run beside the query side too.
constexpr unsigned kQuerySide = 1, kKeySide = 2, kOrder = 4;

// The one-call step's quadtree-ordered copies of q, k, v, dO and LSE under grid order (in
// its backward workspace, made by the pyramid launch and the forward); the attention kernels
// then load only from these (layout kZStore).  Null: the separate calls, which read the
// row-major grid tensors themselves (layout kGrid).
struct ZCopies {
  const void* q;
  const void* k;
  const void* v;
  const void* dO;
  float* lse;
};

ZCopies step_zcopies(const Geometry& g, void* workspace) {
  float* z = static_cast<float*>(workspace) + bwd_workspace_layout(g).total;  // see bwd_workspace_floats
  const long long zt = (long long)g.BH * g.N * g.D / 2;
  return ZCopies{z, z + zt, z + 2 * zt, z + 3 * zt, z + 4 * zt};
}

// The instantiation of each bf16 attention kernel for a geometry and layout (layout_of(g),
// or kZStore for the step under grid order), and the level-1 variant (POOL), which padding
// does not combine with.
template <int D>
auto pick_fwd(const Geometry& g, int lay) {
  constexpr int S = kFwdStages;
  if (lay == kZStore)
    return g.pool1 ? attn_fwd_bf16_kernel<D, S, true, kZStore> : attn_fwd_bf16_kernel<D, S, false, kZStore>;
  if (lay == kPadded) return attn_fwd_bf16_kernel<D, S, false, kPadded>;
  if (lay == kCausal) return attn_fwd_bf16_kernel<D, S, false, kCausal>;
  if (lay == kGrid) return g.pool1 ? attn_fwd_bf16_kernel<D, S, true, kGrid> : attn_fwd_bf16_kernel<D, S, false, kGrid>;
  return g.pool1 ? attn_fwd_bf16_kernel<D, S, true, kFlat> : attn_fwd_bf16_kernel<D, S, false, kFlat>;
}
template <int D>
auto pick_dq(const Geometry& g, int lay) {
  constexpr int S = kDqStages;
  if (lay == kZStore)
    return g.pool1 ? attn_bwd_dq_bf16_kernel<D, S, true, kZStore> : attn_bwd_dq_bf16_kernel<D, S, false, kZStore>;
  if (lay == kPadded) return attn_bwd_dq_bf16_kernel<D, S, false, kPadded>;
  if (lay == kCausal) return attn_bwd_dq_bf16_kernel<D, S, false, kCausal>;
  if (lay == kGrid)
    return g.pool1 ? attn_bwd_dq_bf16_kernel<D, S, true, kGrid> : attn_bwd_dq_bf16_kernel<D, S, false, kGrid>;
  return g.pool1 ? attn_bwd_dq_bf16_kernel<D, S, true, kFlat> : attn_bwd_dq_bf16_kernel<D, S, false, kFlat>;
}
template <int D>
auto pick_dkdv(const Geometry& g, int lay) {
  constexpr int S = kDkvStages;
  if (lay == kZStore)
    return g.pool1 ? attn_bwd_dkdv_bf16_kernel<D, S, true, kZStore> : attn_bwd_dkdv_bf16_kernel<D, S, false, kZStore>;
  if (lay == kPadded) return attn_bwd_dkdv_bf16_kernel<D, S, false, kPadded>;
  if (lay == kCausal) return attn_bwd_dkdv_bf16_kernel<D, S, false, kCausal>;
  if (lay == kGrid)
    return g.pool1 ? attn_bwd_dkdv_bf16_kernel<D, S, true, kGrid> : attn_bwd_dkdv_bf16_kernel<D, S, false, kGrid>;
  return g.pool1 ? attn_bwd_dkdv_bf16_kernel<D, S, true, kFlat> : attn_bwd_dkdv_bf16_kernel<D, S, false, kFlat>;
}
template <int D>
auto pick_coarse(const Geometry& g, int lay) {
  if (lay == kZStore) return attn_bwd_coarse_bf16_kernel<D, kDkvStages, kZStore>;
  if (lay == kPadded) return attn_bwd_coarse_bf16_kernel<D, kDkvStages, kPadded>;
  if (lay == kGrid) return attn_bwd_coarse_bf16_kernel<D, kDkvStages, kGrid>;
  if (lay == kCausal) return attn_bwd_coarse_bf16_kernel<D, kDkvStages, kCausal>;
  return attn_bwd_coarse_bf16_kernel<D, kDkvStages, kFlat>;
}

template <int D>
llsa_status backward_phases_d(const llsa_shape* s, const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dO, const float* k_pyr, const float* v_pyr,
                              const int32_t* idx, const int32_t* row_ptr, const int32_t* col, void* dq, void* dk,
                              void* dv, void* workspace, unsigned phases, cudaStream_t cs,
                              const ZCopies* z) {
  llsa_status st = LLSA_OK;
  const Geometry g = make_geometry(s);
  float* ws = static_cast<float*>(workspace);
  const float scale = 1.0f / sqrtf((float)D);
  const int total_blocks = g.BH * g.n[1];
  if ((phases & kOrder) && s->dtype == LLSA_BF16) {
    const int tiles = order_tiles(g);
    st = launch(kKDkdvOrderCount, cs,
                [&] { launch_pdl(dkdv_order_count_kernel, dim3(tiles), dim3(kOrdThreads), 0, cs, g, row_ptr, ws); });
    if (st != LLSA_OK) return st;
    st = launch(kKDkdvOrderScatter, cs,
                [&] { launch_pdl(dkdv_order_scatter_kernel, dim3(tiles), dim3(kOrdThreads), 0, cs, g, row_ptr, ws); });
    if (st != LLSA_OK) return st;
  }
  if (s->dtype == LLSA_BF16) {
    const int lay = z ? kZStore : layout_of(g);
    CUtensorMap tq, tk, tv, tdo;
    if (!make_tile_map(&tq, z ? z->q : q, g, lay) || !make_tile_map(&tk, z ? z->k : k, g, lay) ||
        !make_tile_map(&tv, z ? z->v : v, g, lay) || !make_tile_map(&tdo, z ? z->dO : dO, g, lay))
      return LLSA_ERR_CUDA;
    const float* lse_in = z ? z->lse : lse;  // dQ's LSE tiles: the quadtree-ordered copy in the step
    AttnParams P{g, scale * kLog2e, scale};
    const size_t kv_bytes = (size_t)kv_smem<D, kDkvStages>(1).total();
    if (phases & kQuerySide) {
      const size_t smem = (size_t)dq_smem<D, kDqStages>(g, kAttnWarps).total();
      auto kern = pick_dq<D>(g, lay);
      if (!allow_smem(kern, smem)) return LLSA_ERR_CUDA;
      const int per_cta = kAttnWarps * kUnitBlocks;
      st = launch(kKBwdDqBf16, cs, [&] {
        launch_pdl(kern, dim3((total_blocks + per_cta - 1) / per_cta), dim3(32 * kAttnWarps), smem, cs, 
            tq, tk, tv, tdo, P, k_pyr, v_pyr, idx, static_cast<const __nv_bfloat16*>(o), lse_in,
            static_cast<__nv_bfloat16*>(dq), ws);
      });
      if (st != LLSA_OK) return st;
      if (g.L >= 2) {
        auto ckern = pick_coarse<D>(g, lay);
        if (!allow_smem(ckern, kv_bytes)) return LLSA_ERR_CUDA;
        const int ctas = g.BH * g.n[2] * (g.coarse_pad / kBlock);
        st = launch(kKBwdCoarseBf16, cs, [&] {
          launch_pdl(ckern, dim3(ctas), dim3(32), kv_bytes, cs, tq, tdo, P, k_pyr, v_pyr, idx, ws);
        });
        if (st != LLSA_OK) return st;
      }
    }
    if (!(phases & kKeySide)) return LLSA_OK;
    if ((st = launch_coarse_reduce<D>(g, scale, idx, row_ptr, col, ws, cs)) != LLSA_OK) return st;
    auto kern = pick_dkdv<D>(g, lay);
    if (!allow_smem(kern, kv_bytes)) return LLSA_ERR_CUDA;
    return launch(kKBwdDkdvBf16, cs, [&] {
      launch_pdl(kern, dim3(total_blocks), dim3(32), kv_bytes, cs, tq, tk, tv, tdo, P, row_ptr, col, ws,
                 static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), g.L >= 2 ? 1 : 0);
    });
  }
  if (phases & kQuerySide) {
    const size_t smem = simt_dq_smem<D>(g);
    if (!allow_smem(attn_bwd_dq_f32_kernel<D>, smem)) return LLSA_ERR_CUDA;
    const int per_cta = g.L >= 2 ? kBlock : 1;
    st = launch(kKBwdDqF32, cs, [&] {
      launch_pdl(attn_bwd_dq_f32_kernel<D>, dim3(total_blocks / per_cta), dim3(kSimtThreads), smem, cs, 
          g, scale, static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
          static_cast<const float*>(o), lse, static_cast<const float*>(dO), k_pyr, v_pyr, idx,
          static_cast<float*>(dq), ws);
    });
    if (st != LLSA_OK) return st;
  }
  if (!(phases & kKeySide)) return LLSA_OK;
  if ((st = launch_coarse_reduce<D>(g, scale, idx, row_ptr, col, ws, cs)) != LLSA_OK) return st;
  return launch(kKBwdDkdvF32, cs, [&] {
    launch_pdl(attn_bwd_dkdv_f32_kernel<D>, dim3(total_blocks), dim3(kSimtThreads), 0, cs, 
        g, scale, static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), k_pyr,
        v_pyr, lse, static_cast<const float*>(dO), row_ptr, col, ws, static_cast<float*>(dk),
        static_cast<float*>(dv));
  });
}

llsa_status backward_phases(const llsa_shape* s, const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, const float* k_pyr, const float* v_pyr,
                            const int32_t* idx, const int32_t* row_ptr, const int32_t* col, void* dq, void* dk,
                            void* dv, void* workspace, unsigned phases, cudaStream_t cs,
                            const ZCopies* z = nullptr) {
  auto f = s->D == 128 ? backward_phases_d<128> : backward_phases_d<64>;
  return f(s, q, k, v, o, lse, dO, k_pyr, v_pyr, idx, row_ptr, col, dq, dk, dv, workspace, phases, cs, z);
}

// ---------------------------------------------------------------------------- pyramid, select
// Levels 1-2 of the pyramid, and levels 3..L too when `upper`.
// With `z` (the step under grid order) the launch also writes the quadtree-ordered copies of
// q, k, v and, in a fourth slice of CTAs, of dO.
template <typename T, int D>
llsa_status pyramid_l12_launch(const Geometry& g, const void* q, const void* k, const void* v, float* q_pyr,
                               float* k_pyr, float* v_pyr, cudaStream_t cs, const ZCopies* z, const void* dO) {
  using C = PyrCfg<T, D>;
  dim3 grid(g.BH * ((g.n[1] + C::ROWS - 1) / C::ROWS), z ? 4 : 3);
  if (!allow_smem(pyramid_l12_kernel<T, D>, C::SPAN)) return LLSA_ERR_CUDA;
  const int dtype = sizeof(T) == 2 ? LLSA_BF16 : LLSA_F32;
  CUtensorMap pq, pk, pv, pd;
  if (!make_patch_map(&pq, q, g, dtype) || !make_patch_map(&pk, k, g, dtype) || !make_patch_map(&pv, v, g, dtype) ||
      !make_patch_map(&pd, z ? dO : q, g, dtype))
    return LLSA_ERR_CUDA;
  ZOut<T> zo{{nullptr, nullptr, nullptr, nullptr}, nullptr};
  if (z) {
    auto w = [](const void* p) { return static_cast<T*>(const_cast<void*>(p)); };
    zo = ZOut<T>{{w(z->q), w(z->k), w(z->v), w(z->dO)}, static_cast<const T*>(dO)};
  }
  return launch(kKPyramidL12, cs, [&] {
    launch_pdl(pyramid_l12_kernel<T, D>, dim3(grid), dim3(C::THREADS), C::SPAN, cs, g, static_cast<const T*>(q),
               static_cast<const T*>(k), static_cast<const T*>(v), q_pyr, k_pyr, v_pyr, pq, pk, pv, pd, zo);
  });
}

template <int D>
llsa_status pyramid_launch_d(const Geometry& g, int dtype, const void* q, const void* k, const void* v, float* q_pyr,
                             float* k_pyr, float* v_pyr, bool upper, cudaStream_t cs, const ZCopies* z,
                             const void* dO) {
  llsa_status st = dtype == LLSA_BF16
                       ? pyramid_l12_launch<__nv_bfloat16, D>(g, q, k, v, q_pyr, k_pyr, v_pyr, cs, z, dO)
                       : pyramid_l12_launch<float, D>(g, q, k, v, q_pyr, k_pyr, v_pyr, cs, nullptr, nullptr);
  if (st != LLSA_OK || !upper) return st;
  for (int l = 3; l <= g.L; ++l) {
    const long long total = (long long)g.BH * g.n[l] * D;
    dim3 grid((unsigned)((total + kPyrThreads - 1) / kPyrThreads), 3);
    st = launch(kKPyramidUp, cs,
                [&] { launch_pdl(pyramid_up_kernel<D>, dim3(grid), dim3(kPyrThreads), 0, cs, g, l, q_pyr, k_pyr, v_pyr); });
    if (st != LLSA_OK) return st;
  }
  return LLSA_OK;
}

llsa_status pyramid_launch(const Geometry& g, int dtype, const void* q, const void* k, const void* v, float* q_pyr,
                           float* k_pyr, float* v_pyr, bool upper, cudaStream_t cs, const ZCopies* z = nullptr,
                           const void* dO = nullptr) {
  auto f = g.D == 128 ? pyramid_launch_d<128> : pyramid_launch_d<64>;
  return f(g, dtype, q, k, v, q_pyr, k_pyr, v_pyr, upper, cs, z, dO);
}

// The pooled levels 3..L and the coarsest selection fit one small kernel per (b, h).
bool small_top(const Geometry& g) { return g.n[g.L] <= kTopMaxN && g.K <= 32 && (g.L < 3 || g.n[3] <= kTopMaxN); }

// Selection of every level, coarsest first.  With `pool_top` (only when small_top), the
// coarsest launch also pools levels 3..L (pyramid_launch was made with upper = false);
// v_pyr is needed only then.
template <int D>
llsa_status select_launch_d(const Geometry& g, float* q_pyr, float* k_pyr, float* v_pyr, int32_t* idx, bool pool_top,
                            cudaStream_t cs) {
  llsa_status st;
  for (int l = g.L; l >= 1; --l) {
    const bool sparse = l < g.L;
    const int n = g.n[l];
    if (!sparse && small_top(g)) {
      auto kern = pool_top ? coarsest_small_kernel<D, true> : coarsest_small_kernel<D, false>;
      constexpr int smem = coarsest_small_smem<D>();
      if (!allow_smem(kern, smem)) return LLSA_ERR_CUDA;
      st = launch(kKSelect, cs, [&] {
        launch_pdl(kern, dim3(g.BH), dim3(kTopThreads), smem, cs, g, q_pyr, k_pyr, v_pyr, idx);
      });
      if (st != LLSA_OK) return st;
      continue;
    }
    int gq, nc;
    if (sparse) {
      gq = kBlock;
      nc = kBlock * g.K;
    } else {
      nc = n;
      gq = kBlock;
      while (gq > 1 && (gq > n || (long long)gq * n > 16384)) gq >>= 1;
    }
    if (sparse && (g.K == 2 || g.K == 4 || g.K == 8 || g.K == 16)) {
      // children of the parent's K keys scored in registers (select_children_kernel)
      const size_t smem = select_children_smem_bytes<D>(nc);
      const float* qpl = q_pyr + g.pyr_off[l];
      const float* kpl = k_pyr + g.pyr_off[l];
      const int* par = idx + g.idx_off[l + 1];
      int* out = idx + g.idx_off[l];
      const unsigned grid = (unsigned)(g.BH * (n / kBlock));
      auto run = [&](auto kern) -> llsa_status {
        if (!allow_smem(kern, smem)) return LLSA_ERR_CUDA;
        return launch(kKSelect, cs, [&] { launch_pdl(kern, dim3(grid), dim3(kSelThreads), smem, cs, g, l, qpl, kpl, par, out); });
      };
      switch (g.K) {
        case 2: st = run(select_children_kernel<D, 1>); break;
        case 4: st = run(select_children_kernel<D, 2>); break;
        case 8: st = run(select_children_kernel<D, 4>); break;
        default: st = run(select_children_kernel<D, 8>); break;
      }
      if (st != LLSA_OK) return st;
      continue;
    }
    const size_t smem = select_smem_bytes<D>(gq, nc, g.K, sparse);
    if (!allow_smem(select_kernel<D>, smem)) return LLSA_ERR_CUDA;
    const int groups = (n + gq - 1) / gq;
    st = launch(kKSelect, cs, [&] {
      launch_pdl(select_kernel<D>, dim3(g.BH * groups), dim3(kSelThreads), smem, cs, g, l, gq, q_pyr + g.pyr_off[l],
                 k_pyr + g.pyr_off[l], sparse ? idx + g.idx_off[l + 1] : nullptr, idx + g.idx_off[l]);
    });
    if (st != LLSA_OK) return st;
  }
  return LLSA_OK;
}

llsa_status select_launch(const Geometry& g, float* q_pyr, float* k_pyr, float* v_pyr, int32_t* idx, bool pool_top,
                          cudaStream_t cs) {
  auto f = g.D == 128 ? select_launch_d<128> : select_launch_d<64>;
  return f(g, q_pyr, k_pyr, v_pyr, idx, pool_top, cs);
}

// The pyramid and every selection level in one cooperative launch (pyramid_select_kernel):
// bf16, L >= 2, a small coarsest level and K in {2, 4, 8, 16} (the register-resident
// children selection).
// Requested by LLSA_FLAG_ONE_LAUNCH_SELECT.
bool fused_pyramid_select(const Geometry& g, const llsa_shape* s) {
  return (s->flags & LLSA_FLAG_ONE_LAUNCH_SELECT) && !g.causal && !g.grid && s->dtype == LLSA_BF16 && g.L >= 2 &&
         small_top(g) &&
         (g.K == 2 || g.K == 4 || g.K == 8 || g.K == 16);
}

template <int D, int CPT>
llsa_status pyramid_select_launch_k(const Geometry& g, const void* q, const void* k, const void* v, float* q_pyr,
                                    float* k_pyr, float* v_pyr, int32_t* idx, unsigned* barrier, cudaStream_t cs) {
  auto kern = pyramid_select_kernel<D, CPT>;
  constexpr int smem = pyramid_select_smem<D, CPT>();
  if (!allow_smem(kern, smem)) return LLSA_ERR_CUDA;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSelThreads, smem) != cudaSuccess || per_sm < 1)
    return LLSA_ERR_CUDA;
  // no more CTAs than the largest phase has units
  long long units = 3LL * g.BH * ((g.n[1] + PyrCfg<__nv_bfloat16, D>::ROWS - 1) / PyrCfg<__nv_bfloat16, D>::ROWS);
  for (int l = 1; l < g.L; ++l) units = units > (long long)g.BH * (g.n[l] / kBlock) ? units : (long long)g.BH * (g.n[l] / kBlock);
  const int grid = (int)((long long)sms * per_sm < units ? (long long)sms * per_sm : units);
  CUtensorMap pq, pk, pv;
  if (!make_patch_map(&pq, q, g, LLSA_BF16) || !make_patch_map(&pk, k, g, LLSA_BF16) ||
      !make_patch_map(&pv, v, g, LLSA_BF16))
    return LLSA_ERR_CUDA;
  if (cudaMemsetAsync(barrier, 0, 16 * sizeof(unsigned), cs) != cudaSuccess) return LLSA_ERR_CUDA;
  return launch(kKPyramidSelect, cs, [&] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = cs;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barriers complete
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, g, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                       static_cast<const __nv_bfloat16*>(v), q_pyr, k_pyr, v_pyr, idx, barrier, pq, pk, pv);
  });
}

template <int D>
llsa_status pyramid_select_launch_d(const Geometry& g, const void* q, const void* k, const void* v, float* q_pyr,
                                    float* k_pyr, float* v_pyr, int32_t* idx, unsigned* barrier, cudaStream_t cs) {
  switch (g.K) {
    case 2: return pyramid_select_launch_k<D, 1>(g, q, k, v, q_pyr, k_pyr, v_pyr, idx, barrier, cs);
    case 4: return pyramid_select_launch_k<D, 2>(g, q, k, v, q_pyr, k_pyr, v_pyr, idx, barrier, cs);
    case 8: return pyramid_select_launch_k<D, 4>(g, q, k, v, q_pyr, k_pyr, v_pyr, idx, barrier, cs);
    default: return pyramid_select_launch_k<D, 8>(g, q, k, v, q_pyr, k_pyr, v_pyr, idx, barrier, cs);
  }
}

// ---------------------------------------------------------------------------- one step
// Host-side checks of a step's buffers (the per-call checks, done up front so that a
// rejected step launches nothing).
llsa_status validate_step(const llsa_shape* s, const llsa_step_buffers* b) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  if (!b) return LLSA_ERR_INVALID_ARG;
  const void* ptrs[17] = {b->q,   b->k,   b->v,  b->dO, b->q_pyr, b->k_pyr,
                          b->v_pyr, b->idx, b->row_ptr, b->col, b->o, b->lse,
                          b->dq,  b->dk,  b->dv, b->transpose_workspace, b->backward_workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LLSA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(s);
  if (b->transpose_workspace_bytes < transpose_ws_bytes(g)) return LLSA_ERR_WORKSPACE;
  if (b->backward_workspace_bytes < (size_t)bwd_workspace_floats(g) * sizeof(float)) return LLSA_ERR_WORKSPACE;
  return LLSA_OK;
}

// pyramid -> selection -> forward -> backward query side on `cs`; the transpose on `side`
// (forked after the selection, joined before the backward key side), or on `cs` if side
// is null.  The join is made on every path once the fork was made, so a capture that
// fails part-way still ends with both streams joined.
template <int D>
llsa_status forward_launch(const Geometry& g, int dtype, const void* q, const void* k, const void* v,
                           const float* k_pyr, const float* v_pyr, const int32_t* idx, void* o, float* lse,
                           cudaStream_t cs, const ZCopies* z) {
  const float scale = 1.0f / sqrtf((float)D);
  const int total_blocks = g.BH * g.n[1];
  if (dtype == LLSA_BF16) {
    const int lay = z ? kZStore : layout_of(g);
    CUtensorMap tq, tk, tv;
    if (!make_tile_map(&tq, z ? z->q : q, g, lay) || !make_tile_map(&tk, z ? z->k : k, g, lay) ||
        !make_tile_map(&tv, z ? z->v : v, g, lay))
      return LLSA_ERR_CUDA;
    AttnParams P{g, scale * kLog2e, scale};
    const size_t smem = (size_t)fwd_smem<D, kFwdStages>(g, kAttnWarps).total();
    auto kern = pick_fwd<D>(g, lay);
    if (!allow_smem(kern, smem)) return LLSA_ERR_CUDA;
    const int per_cta = kAttnWarps * kUnitBlocks;
    return launch(kKFwdBf16, cs, [&] {
      launch_pdl(kern, dim3((total_blocks + per_cta - 1) / per_cta), dim3(32 * kAttnWarps), smem, cs, tq, tk, tv, P,
                 k_pyr, v_pyr, idx, static_cast<__nv_bfloat16*>(o), lse, z ? z->lse : nullptr);
    });
  }
  const size_t smem = simt_fwd_smem<D>(g);
  if (!allow_smem(attn_fwd_f32_kernel<D>, smem)) return LLSA_ERR_CUDA;
  return launch(kKFwdF32, cs, [&] {
    launch_pdl(attn_fwd_f32_kernel<D>, dim3(total_blocks), dim3(kSimtThreads), smem, cs, g, scale,
               static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), k_pyr,
               v_pyr, idx, static_cast<float*>(o), lse);
  });
}

// The forward launch shared by llsa_forward and the step.
llsa_status forward_impl(const llsa_shape* s, const void* q, const void* k, const void* v, const float* k_pyr,
                         const float* v_pyr, const int32_t* idx, void* o, float* lse, llsa_stream_t stream,
                         const ZCopies* z = nullptr) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  const void* ptrs[8] = {q, k, v, k_pyr, v_pyr, idx, o, lse};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LLSA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(s);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  auto f = g.D == 128 ? forward_launch<128> : forward_launch<64>;
  return f(g, s->dtype, q, k, v, k_pyr, v_pyr, idx, o, lse, cs, z);
}

llsa_status step_impl(const llsa_shape* s, const llsa_step_buffers* b, cudaStream_t cs, cudaStream_t side) {
  const Geometry g = make_geometry(s);
  llsa_status st;
  // under grid order (bf16) the pyramid launch also writes quadtree-ordered copies of q, k,
  // v, dO into the workspace, and every attention kernel reads those instead of the grid
  const ZCopies zc = g.zcopy ? step_zcopies(g, b->backward_workspace) : ZCopies{};
  const ZCopies* z = g.zcopy ? &zc : nullptr;
  const bool fused = fused_pyramid_select(g, s);
  if (fused) {  // pyramid and selection in one cooperative launch
    unsigned* barrier =
        reinterpret_cast<unsigned*>(static_cast<float*>(b->backward_workspace) + bwd_workspace_layout(g).barrier);
    auto f = g.D == 128 ? pyramid_select_launch_d<128> : pyramid_select_launch_d<64>;
    st = f(g, b->q, b->k, b->v, b->q_pyr, b->k_pyr, b->v_pyr, b->idx, barrier, cs);
  } else {
    // pooled levels >= 3 are made by the coarsest-selection launch when they are small
    const bool fuse_top = g.L >= 3 && small_top(g);
    st = pyramid_launch(g, s->dtype, b->q, b->k, b->v, b->q_pyr, b->k_pyr, b->v_pyr, !fuse_top, cs, z, b->dO);
    if (st == LLSA_OK) st = select_launch(g, b->q_pyr, b->k_pyr, b->v_pyr, b->idx, fuse_top, cs);
  }
  if (st != LLSA_OK) return st;
  cudaEvent_t fork = nullptr, join = nullptr;
  if (side) {
    if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess) return LLSA_ERR_CUDA;
    if (cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
      cudaEventDestroy(fork);
      return LLSA_ERR_CUDA;
    }
    if (cudaEventRecord(fork, cs) != cudaSuccess || cudaStreamWaitEvent(side, fork, 0) != cudaSuccess)
      st = LLSA_ERR_CUDA;
    if (st == LLSA_OK)
      st = llsa_index_transpose(s, b->idx, b->row_ptr, b->col, b->transpose_workspace, b->transpose_workspace_bytes,
                                side);
    if (st == LLSA_OK)
      st = backward_phases(s, b->q, b->k, b->v, b->o, b->lse, b->dO, b->k_pyr, b->v_pyr, b->idx, b->row_ptr, b->col,
                           b->dq, b->dk, b->dv, b->backward_workspace, kOrder, side, z);
    if (cudaEventRecord(join, side) != cudaSuccess && st == LLSA_OK) st = LLSA_ERR_CUDA;
  }
  if (st == LLSA_OK) {
    // after the fused launch the forward's early reads (coarse rows and selections) would
    // be of the kernel right ahead of it, so it starts only once that kernel is complete
    if (fused) g_serial_next = true;
    st = forward_impl(s, b->q, b->k, b->v, b->k_pyr, b->v_pyr, b->idx, b->o, b->lse, cs, z);
  }
  if (st == LLSA_OK)
    st = backward_phases(s, b->q, b->k, b->v, b->o, b->lse, b->dO, b->k_pyr, b->v_pyr, b->idx, b->row_ptr, b->col,
                         b->dq, b->dk, b->dv, b->backward_workspace, kQuerySide, cs, z);
  if (side) {
    if (cudaStreamWaitEvent(cs, join, 0) != cudaSuccess && st == LLSA_OK) st = LLSA_ERR_CUDA;
    cudaEventDestroy(fork);
    cudaEventDestroy(join);
  } else if (st == LLSA_OK) {
    st = llsa_index_transpose(s, b->idx, b->row_ptr, b->col, b->transpose_workspace, b->transpose_workspace_bytes, cs);
    if (st == LLSA_OK)
      st = backward_phases(s, b->q, b->k, b->v, b->o, b->lse, b->dO, b->k_pyr, b->v_pyr, b->idx, b->row_ptr, b->col,
                           b->dq, b->dk, b->dv, b->backward_workspace, kOrder, cs, z);
  }
  if (st == LLSA_OK)
    st = backward_phases(s, b->q, b->k, b->v, b->o, b->lse, b->dO, b->k_pyr, b->v_pyr, b->idx, b->row_ptr, b->col,
                         b->dq, b->dk, b->dv, b->backward_workspace, kKeySide, cs, z);
  return st;
}

}  // namespace

struct llsa_plan {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

extern "C" {

const char* llsa_status_string(llsa_status s) {
  switch (s) {
    case LLSA_OK: return "ok";
    case LLSA_ERR_INVALID_ARG: return "invalid argument";
    case LLSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LLSA_ERR_WORKSPACE: return "workspace too small";
    case LLSA_ERR_CUDA: return "CUDA launch or runtime error";
    case LLSA_ERR_INTERNAL: return "out-of-range index seen on the device";
    case LLSA_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

llsa_status llsa_validate_shape(const llsa_shape* shape) { return validate(shape); }

size_t llsa_pyramid_elems(const llsa_shape* s) {
  if (validate(s) != LLSA_OK) return 0;
  const Geometry g = make_geometry(s);
  return (size_t)(g.pyr_off[g.L] + (long long)g.BH * g.n[g.L] * g.D);
}

size_t llsa_index_elems(const llsa_shape* s) {
  if (validate(s) != LLSA_OK) return 0;
  const Geometry g = make_geometry(s);
  return (size_t)(g.idx_off[g.L] + (long long)g.BH * g.n[g.L] * g.K);
}

size_t llsa_row_ptr_elems(const llsa_shape* s) {
  if (validate(s) != LLSA_OK) return 0;
  const Geometry g = make_geometry(s);
  return (size_t)(g.rp_off[g.L] + (long long)g.BH * (g.n[g.L] + 1));
}

size_t llsa_transpose_workspace_bytes(const llsa_shape* s) {
  if (validate(s) != LLSA_OK) return 0;
  return transpose_ws_bytes(make_geometry(s));
}

size_t llsa_backward_workspace_bytes(const llsa_shape* s) {
  if (validate(s) != LLSA_OK) return 0;
  return (size_t)bwd_workspace_floats(make_geometry(s)) * sizeof(float);
}

llsa_status llsa_build_pyramid(const llsa_shape* s, const void* q, const void* k, const void* v, float* q_pyr,
                               float* k_pyr, float* v_pyr, llsa_stream_t stream) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  const void* ptrs[6] = {q, k, v, q_pyr, k_pyr, v_pyr};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LLSA_ERR_INVALID_ARG;
  return pyramid_launch(make_geometry(s), s->dtype, q, k, v, q_pyr, k_pyr, v_pyr, true,
                        reinterpret_cast<cudaStream_t>(stream));
}

llsa_status llsa_select(const llsa_shape* s, const float* q_pyr, const float* k_pyr, int32_t* idx,
                        llsa_stream_t stream) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  if (!q_pyr || !k_pyr || !idx || !aligned16(q_pyr) || !aligned16(k_pyr) || !aligned16(idx))
    return LLSA_ERR_INVALID_ARG;
  return select_launch(make_geometry(s), const_cast<float*>(q_pyr), const_cast<float*>(k_pyr), nullptr, idx, false,
                       reinterpret_cast<cudaStream_t>(stream));
}

llsa_status llsa_index_transpose(const llsa_shape* s, const int32_t* idx, int32_t* row_ptr, int32_t* col,
                                 void* workspace, size_t workspace_bytes, llsa_stream_t stream) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  if (!idx || !row_ptr || !col || !workspace || !aligned16(idx) || !aligned16(row_ptr) || !aligned16(col) ||
      !aligned16(workspace))
    return LLSA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(s);
  if (workspace_bytes < transpose_ws_bytes(g)) return LLSA_ERR_WORKSPACE;
  long long ent_total, hist_total;
  const TransposeGeo tg = make_transpose_geo(g, &ent_total, &hist_total);
  uint32_t* ws_ent = static_cast<uint32_t*>(workspace);
  int* ws_hist = reinterpret_cast<int*>(ws_ent + ((ent_total + 63) & ~63LL));
  const TransposeLevel& last = tg.lv[g.L - 1];
  const int tile_ctas = last.cta_tiles + g.BH * last.tiles;
  const int bucket_ctas = last.cta_buckets + g.BH * last.nb;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  st = launch(kKTransposeHist, cs,
              [&] { launch_pdl(transpose_hist_kernel, dim3(tile_ctas), dim3(kTrThreads), 0, cs, tg, idx, ws_hist); });
  if (st != LLSA_OK) return st;
  int max_tiles = 0;
  for (int l = 0; l < g.L; ++l) max_tiles = tg.lv[l].tiles > max_tiles ? tg.lv[l].tiles : max_tiles;
  const bool scanned = max_tiles > kTrScanTiles;
  if (scanned) {
    st = launch(kKTransposeScan, cs,
                [&] { launch_pdl(transpose_scan_kernel, dim3(g.L * g.BH), dim3(kTrThreads), 0, cs, tg, ws_hist); });
    if (st != LLSA_OK) return st;
  }
  auto scatter = scanned ? transpose_scatter_kernel<true> : transpose_scatter_kernel<false>;
  auto bucket = scanned ? transpose_bucket_kernel<true> : transpose_bucket_kernel<false>;
  st = launch(kKTransposeScatter, cs,
              [&] { launch_pdl(scatter, dim3(tile_ctas), dim3(kTrThreads), 0, cs, tg, idx, ws_hist, ws_ent); });
  if (st != LLSA_OK) return st;
  return launch(kKTransposeBucket, cs, [&] {
    launch_pdl(bucket, dim3(bucket_ctas), dim3(kTrThreads), 0, cs, tg, ws_ent, ws_hist, row_ptr, col);
  });
}

llsa_status llsa_index_transpose_noalloc(const llsa_shape* s, const int32_t* idx, int32_t* row_ptr, int32_t* col,
                                         llsa_stream_t stream) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  if (!idx || !row_ptr || !col || !aligned16(idx) || !aligned16(row_ptr) || !aligned16(col))
    return LLSA_ERR_INVALID_ARG;
  if (transpose_ws_bytes(make_geometry(s)) > LLSA_NOALLOC_SCRATCH_BYTES) return LLSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != LLSA_OK) return st;
  return llsa_index_transpose(s, idx, row_ptr, col, scratch, LLSA_NOALLOC_SCRATCH_BYTES, stream);
}

llsa_status llsa_forward(const llsa_shape* s, const void* q, const void* k, const void* v, const float* k_pyr,
                         const float* v_pyr, const int32_t* idx, void* o, float* lse, llsa_stream_t stream) {
  SerialFirstLaunch serial;
  return forward_impl(s, q, k, v, k_pyr, v_pyr, idx, o, lse, stream);
}


llsa_status llsa_backward(const llsa_shape* s, const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dO, const float* k_pyr, const float* v_pyr,
                          const int32_t* idx, const int32_t* row_ptr, const int32_t* col, void* dq, void* dk,
                          void* dv, void* workspace, size_t workspace_bytes, llsa_stream_t stream) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  const void* ptrs[16] = {q, k, v, o, lse, dO, k_pyr, v_pyr, idx, row_ptr, col, dq, dk, dv, workspace, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LLSA_ERR_INVALID_ARG;
  if (workspace_bytes < (size_t)bwd_workspace_floats(make_geometry(s)) * sizeof(float)) return LLSA_ERR_WORKSPACE;
  SerialFirstLaunch serial;
  return backward_phases(s, q, k, v, o, lse, dO, k_pyr, v_pyr, idx, row_ptr, col, dq, dk, dv, workspace,
                         kOrder | kQuerySide | kKeySide, reinterpret_cast<cudaStream_t>(stream));
}

llsa_status llsa_train_step(const llsa_shape* s, const llsa_step_buffers* b, llsa_stream_t stream,
                            llsa_stream_t side_stream) {
  const llsa_status st = validate_step(s, b);
  if (st != LLSA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t side = reinterpret_cast<cudaStream_t>(side_stream);
  return step_impl(s, b, cs, side == cs ? nullptr : side);
}

llsa_status llsa_plan_create(const llsa_shape* s, const llsa_step_buffers* b, int32_t repeat, llsa_plan** plan_out) {
  if (!plan_out) return LLSA_ERR_INVALID_ARG;
  *plan_out = nullptr;
  if (repeat < 1 || repeat > 4096) return LLSA_ERR_INVALID_ARG;
  llsa_status st = validate_step(s, b);
  if (st != LLSA_OK) return st;
  cudaStream_t cs = nullptr, side = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return LLSA_ERR_CUDA;
  if (cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return LLSA_ERR_CUDA;
  }
  llsa_plan* plan = new (std::nothrow) llsa_plan();
  if (!plan) st = LLSA_ERR_CUDA;
  if (st == LLSA_OK && cudaStreamBeginCapture(cs, cudaStreamCaptureModeRelaxed) != cudaSuccess) st = LLSA_ERR_CUDA;
  if (st == LLSA_OK) {
    for (int r = 0; r < repeat && st == LLSA_OK; ++r) st = step_impl(s, b, cs, side);
    cudaGraph_t graph = nullptr;
    if (cudaStreamEndCapture(cs, &graph) != cudaSuccess && st == LLSA_OK) st = LLSA_ERR_CUDA;
    plan->graph = graph;
    if (st == LLSA_OK && cudaGraphInstantiate(&plan->exec, graph, 0) != cudaSuccess) st = LLSA_ERR_CUDA;
  }
  cudaStreamDestroy(side);
  cudaStreamDestroy(cs);
  cudaGetLastError();  // clears the error a failed capture leaves behind; `st` reports it
  if (st != LLSA_OK) {
    llsa_plan_destroy(plan);
    return st;
  }
  *plan_out = plan;
  return LLSA_OK;
}

llsa_status llsa_plan_launch(const llsa_plan* plan, llsa_stream_t stream) {
  if (!plan || !plan->exec) return LLSA_ERR_INVALID_ARG;
  return cudaGraphLaunch(plan->exec, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? LLSA_OK : LLSA_ERR_CUDA;
}

void llsa_plan_destroy(llsa_plan* plan) {
  if (!plan) return;
  if (plan->exec) cudaGraphExecDestroy(plan->exec);
  if (plan->graph) cudaGraphDestroy(plan->graph);
  delete plan;
}

llsa_status llsa_token_permute(const llsa_shape* s, const void* src, void* dst, int32_t to_z_order,
                               llsa_stream_t stream) {
  llsa_status st = validate(s);
  if (st != LLSA_OK) return st;
  if (!src || !dst || !aligned16(src) || !aligned16(dst) || src == dst) return LLSA_ERR_INVALID_ARG;
  if (!is_pow2(s->N)) return LLSA_ERR_INVALID_ARG;
  const int lg = ilog2(s->N);
  if (lg & 1) return LLSA_ERR_INVALID_ARG;  // N must be a square grid: side = 2^(lg/2)
  const long long rows = (long long)s->B * s->H * s->N;
  const int row_bytes = s->D * (s->dtype == LLSA_BF16 ? 2 : 4);
  const int pieces = row_bytes / 16;
  const long long threads = rows * pieces;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  return launch(kKZOrder, cs, [&] {
    launch_pdl(zorder_permute_kernel, dim3((unsigned)((threads + kZThreads - 1) / kZThreads)), dim3(kZThreads), 0,
               cs, static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, s->N, lg / 2, pieces,
               to_z_order ? 1 : 0);
  });
}

llsa_status llsa_device_status(int32_t* code_out, llsa_stream_t stream) {
  if (!code_out) return LLSA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return LLSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_llsa_status, sizeof(int)) != cudaSuccess) return LLSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_llsa_status, &zero, sizeof(int)) != cudaSuccess) return LLSA_ERR_CUDA;
  *code_out = v;
  return LLSA_OK;
}

llsa_status llsa_check_bounded_wait(int64_t limit_cycles, llsa_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > kWaitLimitCycles) return LLSA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  return launch(kKWaitCheck, cs, [&] { bounded_wait_check_kernel<<<1, 32, 0, cs>>>((long long)limit_cycles); });
}

llsa_status llsa_gather_probe(const void* src, int64_t rows, const int32_t* tile_rows, int32_t ntiles,
                              int32_t stages, int32_t ctas, llsa_stream_t stream) {
  if (!src || !tile_rows || !aligned16(src) || !aligned16(tile_rows)) return LLSA_ERR_INVALID_ARG;
  if (rows < kBlock || rows % kBlock != 0 || rows >= (1LL << 31) || ntiles < 1 || ctas < 1 || ctas > 65535)
    return LLSA_ERR_INVALID_ARG;
  if (stages != 2 && stages != 4 && stages != 8) return LLSA_ERR_INVALID_ARG;
  CUtensorMap tm;
  if (!make_probe_map(&tm, src, rows)) return LLSA_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  auto run = [&](auto kern, int smem) -> llsa_status {
    if (!allow_smem(kern, smem)) return LLSA_ERR_CUDA;
    return launch(kKGatherProbe, cs, [&] {
      kern<<<ctas, kProbeWarps * 32, smem, cs>>>(tm, tile_rows, ntiles, (int)rows);
    });
  };
  if (stages == 2) return run(gather_probe_kernel<2>, gather_probe_smem<2>());
  if (stages == 4) return run(gather_probe_kernel<4>, gather_probe_smem<4>());
  return run(gather_probe_kernel<8>, gather_probe_smem<8>());
}

llsa_status llsa_trace_begin(void** events, int32_t* kernel_ids, int32_t capacity) {
  if (!events || !kernel_ids || capacity < 0) return LLSA_ERR_INVALID_ARG;
  g_trace.ev = reinterpret_cast<cudaEvent_t*>(events);
  g_trace.ids = kernel_ids;
  g_trace.cap = capacity;
  g_trace.used = 0;
  return LLSA_OK;
}

llsa_status llsa_trace_end(int32_t* launches_out) {
  if (launches_out) *launches_out = g_trace.used;
  g_trace = TraceState{};
  return LLSA_OK;
}

const char* llsa_kernel_name(int32_t kernel_id) {
  return (kernel_id > 0 && kernel_id < kKNumKernels) ? kKernelNames[kernel_id] : kKernelNames[0];
}

}  // extern "C"
