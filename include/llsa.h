/*
 * llsa.h -- C ABI of the B200 (sm_100a) Log-linear Sparse Attention hot path.
 *
 * Log-linear Sparse Attention (LLSA) is non-causal multi-head attention in which each
 * block of 16 queries attends to K selected blocks of 16 keys plus K coarse (mean-pooled)
 * key tokens from each coarser level of a 16x pyramid ("Trainable Log-linear Sparse
 * Attention for Efficient Diffusion Transformers", abstract; skill page "Log Linear
 * Sparse Attention", Core Technique 1-3).  The LLSA GitHub README's usage section makes
 * it a drop-in for scaled_dot_product_attention(q, k, v, dropout_p=0, is_causal=False)
 * with block_size=16, and states that only non-causal attention is supported and that
 * the token length and topk must be powers of two.  This library lifts the second limit:
 * any topk, and any N that the 16x pyramid divides (a multiple of 16^L).
 *
 * The path is split into five calls, in this order for one training step:
 *   llsa_build_pyramid -> llsa_select -> llsa_forward            (forward)
 *   llsa_index_transpose -> llsa_backward                        (backward)
 * llsa_train_step makes all five (the transpose on a second stream), and a plan replays
 * a captured sequence of steps as one CUDA graph.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Shapes: B batches, H heads, N tokens, D channels per head, block = 16, topk = K,
 *    levels = L.  Level l (1..L) has n_l = N / 16^l tokens; level 0 is the input.
 *  - q, k, v, o, dO, dq, dk, dv: [B, H, N, D] contiguous row-major, element type
 *    `dtype` (bf16 or fp32): the scaled_dot_product_attention layout.
 *  - Pyramids q_pyr/k_pyr/v_pyr: fp32, levels 1..L concatenated level-major:
 *    [L][B, H, n_l, D]; llsa_pyramid_elems() gives the element count per tensor.
 *  - idx: int32 level-major [L][B, H, n_l, K]; row (l, b, h, a) holds the K level-l key
 *    indices selected for level-l query token a, strictly ascending.  Level-1 rows are
 *    the selected fine blocks of query block a (tokens 16a..16a+15).
 *  - row_ptr: int32 level-major [L][B, H, n_l + 1]; col: int32 level-major
 *    [L][B, H, n_l * K].  Row j of (l, b, h) lists, ascending, every level-l query a whose
 *    idx row contains key j (a CSR matrix; row_ptr offsets are local to (l, b, h)).
 *  - lse: fp32 [B, H, N], natural-log log-sum-exp of each query's scaled scores.
 *  - Every pointer is device memory owned by the caller, 16-byte aligned (256-byte
 *    alignment recommended).  The library allocates no device memory, keeps no state
 *    between calls (a plan, below, is state its handle owns) and is reentrant; calls on
 *    different streams must not share output buffers.
 *  - Every call is asynchronous on `stream` (NULL = legacy default stream) and never
 *    synchronises the host, except llsa_device_status.
 *  - Arguments are checked on the host before any launch.  A rejected call launches
 *    nothing and returns LLSA_ERR_INVALID_ARG (bad value, null pointer, misalignment,
 *    shape rules below) or LLSA_ERR_UNSUPPORTED (a legal value this library does not
 *    implement).  A launch failure returns LLSA_ERR_CUDA.  No exception crosses the ABI.
 *  - Shape rules: B, H >= 1; N a multiple of 16^L (so every n_l = N / 16^l is whole
 *    and n_L >= 1; N need not be a power of two; a shorter sequence is padded up to such an N
 *    and n_valid says where its padding starts); 1 <= topk <= n_L, any integer;
 *    block == 16; 1 <= levels <= 4; D == 64 or 128; N <= 2^20; n_L <= 16384; topk <= 64; (levels - 1) * topk <= 32;
 *    B * H * N < 2^31; with LLSA_FLAG_ALL_TOP also (levels - 2) * topk + n_L <= 96.
 *  - Device-side checks: every gathered index (idx entries, CSR entries) is range
 *    checked on the device; an out-of-range value is not dereferenced, and the call
 *    records LLSA_ERR_INTERNAL in a device status word that llsa_device_status reads.
 *    Bounded waits inside kernels that time out record LLSA_ERR_TIMEOUT the same way.
 */
#ifndef LLSA_H_
#define LLSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a pointer to the opaque CUstream_st). */
struct CUstream_st;
typedef struct CUstream_st* llsa_stream_t;

typedef enum {
  LLSA_OK = 0,
  LLSA_ERR_INVALID_ARG = 1,
  LLSA_ERR_UNSUPPORTED = 2,
  LLSA_ERR_WORKSPACE = 3,
  LLSA_ERR_CUDA = 4,
  LLSA_ERR_INTERNAL = 5,
  LLSA_ERR_TIMEOUT = 6
} llsa_status;

typedef enum { LLSA_BF16 = 0, LLSA_F32 = 1 } llsa_dtype;

/*
 * Enrichment variant (no counterpart on the pages, which give no weighting for the coarse
 * tokens): with LLSA_FLAG_LOG_BIAS the scaled score of every level-l coarse KV entry gets
 * + ln(16^l), the log of the number of input tokens the pooled token averages, so that it
 * carries their softmax mass when they are all equal.  Default 0: unit-weight entries.
 */
#define LLSA_FLAG_LOG_BIAS 1
/*
 * Enrichment variant: with LLSA_FLAG_ALL_TOP (and levels >= 2) the level-L part of every
 * query block's KV list is all n_L coarsest tokens, in index order, instead of the K that
 * the block's level-L ancestor selected; levels 2..L-1 and the selection are unchanged.
 * The list then has C = (L-2) K + n_L coarse entries; C > 96 -> LLSA_ERR_UNSUPPORTED.  It
 * combines with LLSA_FLAG_LOG_BIAS.  The level-L rows of the index transpose are still
 * produced (the backward does not need them).
 */
#define LLSA_FLAG_ALL_TOP 2
/*
 * Enrichment variant: with LLSA_FLAG_LEVEL1 the list also holds the level-1 pooled token
 * (the mean K and V of the 16 tokens) of each of the K selected fine blocks, so T grows by
 * K; with LLSA_FLAG_LOG_BIAS those entries get + ln 16.  Their gradient reaches the block's
 * 16 tokens through the mean-pool adjoint.  Combines with the other flags, at any levels.
 */
#define LLSA_FLAG_LEVEL1 4
/*
 * Token order (LLSA GitHub README, token reordering example: image tokens should be in the
 * quadtree order, so that every 16-token block is a 4 x 4 patch and every level-l pooled
 * token a 4^l x 4^l patch).  With LLSA_FLAG_GRID_ORDER, q, k, v, dO, o, dq, dk, dv and lse
 * are in the row-major order of a square G x G token grid (N = G * G, G a power of two,
 * N >= 256); the kernels read and write them in place through that order, so no separate
 * permutation pass is needed.  The pyramid, idx and the CSR refer to quadtree positions:
 * the results equal those of the same call on inputs permuted by llsa_token_permute, with
 * its outputs permuted back.  Not combined with padding (n_valid).
 */
#define LLSA_FLAG_GRID_ORDER 8
/*
 * Launch shape only; results are bit-identical with and without it.  With
 * LLSA_FLAG_ONE_LAUNCH_SELECT, llsa_train_step and plans run the pyramid and every selection
 * level as one cooperative persistent kernel whose phases are separated by grid-wide barriers,
 * instead of one launch per stage chained by programmatic dependent launch.  It applies to
 * bf16 inputs with levels >= 2, n_L <= 64 and topk in {2, 4, 8, 16}, without grid order or
 * the causal mask; elsewhere, and in the separate calls, the flag changes nothing.  Off by default: on one B200 the chained launches
 * are faster (the forward can start its set-up while they drain, but not while a cooperative
 * kernel does).
 */
#define LLSA_FLAG_ONE_LAUNCH_SELECT 16
/*
 * Causal attention (LLSA GitHub README, usage section: the released kernels are non-causal
 * only, to be addressed later; the pages define no causal variant, so this is a reading
 * that keeps SDPA's is_causal=True meaning -- query position i sees key positions t <= i --
 * and changes as little else as possible):
 *  - selection: a level-l query token a picks only among key tokens j <= a (the non-causal
 *    candidates with index <= a); a list with fewer than K such candidates ends in
 *    LLSA_NO_PICK entries (lists stay ascending).  Scores and pooled queries are the
 *    non-causal ones, so the choice of keys may depend on later queries of a coarse span;
 *  - attention: a picked block j < p is seen whole by query block p, the block's own block
 *    (j = p) with key t visible to query i only when t <= i, and a coarse level-l token j
 *    only when j is below p's level-l ancestor (the token lies wholly before the block);
 *  - index transpose: LLSA_NO_PICK entries are dropped (row_ptr[n_l] = number of picks).
 * bf16 only (fp32 -> LLSA_ERR_UNSUPPORTED); combines with no other flag except
 * LLSA_FLAG_ONE_LAUNCH_SELECT (ignored) and with no padding.
 */
#define LLSA_FLAG_CAUSAL 32
#define LLSA_NO_PICK 0x7fffffff

typedef struct {
  int32_t B, H, N, D;
  int32_t block;   /* must be 16 (README usage section: block_size=16) */
  int32_t topk;    /* K, 1 <= K <= n_L */
  int32_t levels;  /* L, number of pooled levels; llsa_l1 <-> 1, llsa_l2 <-> 2 */
  int32_t dtype;   /* llsa_dtype of q, k, v, o, dO, dq, dk, dv */
  int32_t flags;   /* LLSA_FLAG_* bits (0: the default enrichment); others -> INVALID_ARG */
  int32_t n_valid; /* real tokens per sequence: 0 (or N) = no padding; see "Padded sequences" */
} llsa_shape;

/*
 * Padded sequences (no counterpart on the pages, whose kernels need the token length to be a
 * power of two; the README's usage section says a later update will lift that).  With
 * 0 < n_valid < N, positions n_valid..N-1 of every (b, h) sequence are padding and take no
 * part in the result, whatever they hold:
 *  - a pooled token averages only the real tokens of its span (c of them, 0 <= c <= 16^l):
 *    level 1 adds its real tokens in index order and divides by c; level l >= 2 adds each
 *    child's count times its stored mean in index order and divides by c; a token with c = 0
 *    is 0.  Full tokens come out exactly as without padding;
 *  - empty tokens are never selected: the candidates of level l are the real tokens
 *    [0, ceil(n_valid / 16^l)); topk must not exceed ceil(n_valid / 16^L);
 *  - padding keys are masked out of every softmax; padding queries get O = 0, LSE = 0 and
 *    dQ = 0 and send no gradient; padding positions get dK = dV = 0;
 *  - a pooled token's gradient reaches each of its c real tokens with weight 1 / c.
 * Selection rows of padding query tokens are still written (scores of a zero mean).
 * Padding combines with no enrichment flag (flags != 0 -> LLSA_ERR_UNSUPPORTED).
 */

/* Static text for a status code. */
const char* llsa_status_string(llsa_status status);

/* Host-only check of a shape against the rules above. */
llsa_status llsa_validate_shape(const llsa_shape* shape);

/* Element counts of the caller-allocated buffers (0 for an invalid shape). */
size_t llsa_pyramid_elems(const llsa_shape* shape);   /* fp32 elements per pyramid tensor */
size_t llsa_index_elems(const llsa_shape* shape);     /* int32 elements of idx and of col */
size_t llsa_row_ptr_elems(const llsa_shape* shape);   /* int32 elements of row_ptr */

/*
 * Scratch bytes llsa_index_transpose / llsa_backward need in `workspace`.  For bf16 under
 * LLSA_FLAG_GRID_ORDER the backward workspace also has room for the quadtree-ordered copies
 * of q, k, v, dO (4 * B*H*N*D * 2 bytes) and of LSE (B*H*N * 4 bytes) that llsa_train_step
 * and plans make in it: there the pyramid launch writes those copies while it pools, and the
 * attention kernels gather whole 2 KB tiles from them instead of 4 x 4-pixel boxes from the
 * grid (the separate calls still read the grid tensors directly).
 */
size_t llsa_transpose_workspace_bytes(const llsa_shape* shape);
size_t llsa_backward_workspace_bytes(const llsa_shape* shape);

/*
 * Step 1 -- the mean-pooled Q/K/V pyramid (abstract: block-wise compression; skill page,
 * Core Technique 1: hierarchical compression).  For l = 1..L and every token j < n_l,
 * X_l[j] = (((0 + X_{l-1}[16j]) + X_{l-1}[16j+1]) + ... + X_{l-1}[16j+15]) * (1/16),
 * every addition rounded to fp32 in this order (X_0 = the input, widened exactly).
 * q, k, v: [B,H,N,D] `dtype`; q_pyr, k_pyr, v_pyr: [L][B,H,n_l,D] fp32 outputs.
 */
llsa_status llsa_build_pyramid(const llsa_shape* shape, const void* q, const void* k, const void* v,
                               float* q_pyr, float* k_pyr, float* v_pyr, llsa_stream_t stream);

/*
 * Step 2 -- hierarchical Top-K (skill page, Core Technique 1: sparse Top-K at each level
 * over the indices found at the previous level).  At level L every query token scores all
 * n_L key tokens; at level l < L query a scores only the 16K children 16c+r (r < 16) of
 * the K level-(l+1) keys c selected for its parent a/16.  Score = fp32 dot product of the
 * pooled q and k rows; the K largest are kept, the lower key index winning equal scores,
 * and written ascending.  q_pyr, k_pyr: pyramids from step 1; idx: output [L][B,H,n_l,K].
 */
llsa_status llsa_select(const llsa_shape* shape, const float* q_pyr, const float* k_pyr, int32_t* idx,
                        llsa_stream_t stream);

/*
 * Step 5 -- the sparse index transpose (skill page, Core Technique 3: a transpose that
 * works on the sparse indices and builds no dense mask).  For every level, batch and head
 * it turns the query -> key lists `idx` into key -> query CSR lists (row_ptr, col),
 * queries ascending within each row.  It is a stable counting sort by key bucket then by
 * key (histogram, scan, scatter), with no atomics, so the output is deterministic.
 * workspace: device scratch of at least llsa_transpose_workspace_bytes(shape) bytes,
 * 256-byte aligned; its contents are not read before being written.
 */
llsa_status llsa_index_transpose(const llsa_shape* shape, const int32_t* idx, int32_t* row_ptr,
                                 int32_t* col, void* workspace, size_t workspace_bytes,
                                 llsa_stream_t stream);

/*
 * Step 4a -- block-sparse attention forward with hierarchical KV enrichment (skill page,
 * Core Technique 2).  Query block p (tokens 16p..16p+15) attends to the KV list: the 16
 * tokens of each selected level-1 block j in idx[1][p], then for l = 2..L the K pooled
 * level-l tokens idx[l][p / 16^(l-1)] (k_pyr/v_pyr rows, each one ordinary KV entry).
 * O_i = softmax(q_i . k_e / sqrt(D)) over that list applied to v_e; lse_i = natural-log
 * log-sum-exp of the scaled scores.  Arithmetic: bf16 inputs use bf16 tensor-core
 * products (coarse fp32 rows rounded to bf16) with fp32 accumulation and fp32 softmax;
 * fp32 inputs use fp32 throughout.  o: [B,H,N,D] `dtype`; lse: [B,H,N] fp32.
 */
llsa_status llsa_forward(const llsa_shape* shape, const void* q, const void* k, const void* v,
                         const float* k_pyr, const float* v_pyr, const int32_t* idx, void* o, float* lse,
                         llsa_stream_t stream);

/*
 * Step 4b -- gradient of step 4a with the selection held fixed (the pages train LLSA
 * end to end: "trainable" in the title; skill page, Practical Results: training speedup).
 * With P the softmax over each query's list, Delta_i = sum_d dO_id * O_id and
 * dS = P * (dO v^T - Delta): dq_i = sum_e dS_ie k_e / sqrt(D); dk_e += dS_ie q_i / sqrt(D);
 * dv_e += P_ie dO_i.  Gradients of pooled level-l tokens are spread over their 16^l input
 * tokens with weight 1/16^l (the mean-pool adjoint); pooled queries get no gradient.
 * Fine-token dk/dv are gathered through the level-1 CSR (row_ptr, col from step 5) and
 * coarse-token gradients through the level-l CSRs, so no atomics are used.
 * o, lse: outputs of llsa_forward; dO: [B,H,N,D] `dtype`; dq, dk, dv: [B,H,N,D] `dtype`.
 * workspace: at least llsa_backward_workspace_bytes(shape) bytes, 256-byte aligned.
 */
llsa_status llsa_backward(const llsa_shape* shape, const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dO, const float* k_pyr,
                          const float* v_pyr, const int32_t* idx, const int32_t* row_ptr,
                          const int32_t* col, void* dq, void* dk, void* dv, void* workspace,
                          size_t workspace_bytes, llsa_stream_t stream);

/*
 * One training step (steps 1, 2, 4a, 5, 4b of this header) over caller-owned buffers
 * (no counterpart on the pages: an interface addition of this library).
 *
 * Device buffers of one step, each as described for the single calls above; the two
 * workspaces are those of llsa_index_transpose and llsa_backward and must not be shared
 * with concurrent work.
 */
typedef struct {
  const void* q; const void* k; const void* v; const void* dO;  /* inputs [B,H,N,D] `dtype` */
  float* q_pyr; float* k_pyr; float* v_pyr;                      /* [L][B,H,n_l,D] fp32 */
  int32_t* idx; int32_t* row_ptr; int32_t* col;                  /* selection and its CSR */
  void* o; float* lse;                                           /* forward outputs */
  void* dq; void* dk; void* dv;                                  /* gradients [B,H,N,D] `dtype` */
  void* transpose_workspace; size_t transpose_workspace_bytes;
  void* backward_workspace; size_t backward_workspace_bytes;
} llsa_step_buffers;

/*
 * llsa_build_pyramid -> llsa_select -> llsa_forward -> llsa_backward on `stream`, with
 * llsa_index_transpose on `side_stream`: the transpose is forked after the selection and
 * joined before the part of the backward that reads the CSR (the coarse-token reduction and
 * dK/dV), so it runs concurrently with the forward and dQ.  side_stream NULL or equal to
 * `stream` runs the transpose on `stream`.  Results are those of the five calls in order.
 * All checks are made before the first launch; a rejected step launches nothing.  Two
 * CUDA events are created and released per call (no device memory is allocated).
 */
llsa_status llsa_train_step(const llsa_shape* shape, const llsa_step_buffers* buffers, llsa_stream_t stream,
                            llsa_stream_t side_stream);

/*
 * A plan is `repeat` consecutive llsa_train_step calls on a fixed set of buffers, captured
 * once into a CUDA graph (two internal streams; the transpose on the second) and
 * instantiated; llsa_plan_launch replays it on `stream` with no per-kernel launch cost.
 * The graph holds the buffer addresses and the shape: the buffers must stay allocated and
 * unchanged in size while the plan exists, and their contents are read at launch time.
 * Kernel launches made while the calling thread traces (llsa_trace_begin) are captured
 * with their trace events, which the graph then records at every launch.
 * llsa_plan_create: repeat in [1, 4096]; *plan_out is NULL on failure.  The plan owns the
 * graph; llsa_plan_destroy releases it (NULL is ignored) and must not race a launch that
 * has not been ordered before it on the host.
 */
typedef struct llsa_plan llsa_plan;
llsa_status llsa_plan_create(const llsa_shape* shape, const llsa_step_buffers* buffers, int32_t repeat,
                             llsa_plan** plan_out);
llsa_status llsa_plan_launch(const llsa_plan* plan, llsa_stream_t stream);
void llsa_plan_destroy(llsa_plan* plan);

/*
 * Quadtree (Z) token order of a square token grid (LLSA GitHub README, token reordering
 * example: for images, reorder tokens so that nearby, similar tokens get adjacent indices;
 * each 16-token block is then a 4 x 4 square and each level-l pooled token a
 * 4^l x 4^l square).  N must be a power of four (side = sqrt(N)); grid position (r, c),
 * row-major index r * side + c, has Z index z = sum_b (2 r_b + c_b) 4^b.
 * to_z_order != 0: dst[b, h, z(p)] = src[b, h, p]; 0: the inverse, dst[b, h, p] =
 * src[b, h, z(p)].  src, dst: [B, H, N, D] `dtype`, distinct (not in place), 16-byte
 * aligned.  Non-square N or src == dst -> LLSA_ERR_INVALID_ARG.
 */
llsa_status llsa_token_permute(const llsa_shape* shape, const void* src, void* dst, int32_t to_z_order,
                               llsa_stream_t stream);

/*
 * Reads and clears the device status word that kernels set on an out-of-range index
 * (LLSA_ERR_INTERNAL) or a bounded wait that timed out (LLSA_ERR_TIMEOUT).  Synchronises
 * `stream` first.  *code_out receives LLSA_OK or the first error recorded since the last
 * call.  Returns LLSA_ERR_CUDA if the device cannot be queried.
 */
llsa_status llsa_device_status(int32_t* code_out, llsa_stream_t stream);

/*
 * Check of the bounded-wait failure path (no counterpart on the pages: a failure-detection
 * aid of this library).  Every wait of the kernels on an asynchronous copy gives up after a
 * cycle limit (about two seconds at the maximum SM clock), records LLSA_ERR_TIMEOUT in the
 * device status word and lets the kernel return, so a copy that never lands cannot hang the
 * GPU.  This call runs that same wait in a one-thread kernel on an mbarrier armed for 16
 * bytes that no copy will ever deliver (none is issued, so nothing is left in flight), with
 * a limit of `limit_cycles` SM cycles: the wait gives up, and the next llsa_device_status
 * returns LLSA_ERR_TIMEOUT.  limit_cycles outside [1, 4e9] -> LLSA_ERR_INVALID_ARG.
 * While the recorded timeout has not been read and cleared, the waits of other kernels give
 * up at their next check, so call it only when no other work of the library is in flight.
 */
llsa_status llsa_check_bounded_wait(int64_t limit_cycles, llsa_stream_t stream);

/*
 * L2 -> SM gather probe (a measurement aid; no counterpart on the pages).  The attention
 * kernels gather 16-row x 64-channel bf16 tiles by index with 2-D TMA copies (128-byte
 * swizzle); when the gathered K, V, Q and dO fit in L2 those copies are served from L2 and
 * HBM bandwidth does not bound them.  This call runs only that gather: `ctas` CTAs of 4 warps,
 * every warp streaming its share of the tiles through a ring of `stages` mbarrier stages and
 * doing nothing else with them.  Timing it on a buffer kept resident in L2 gives the gather
 * ceiling the attention kernels are compared with.
 * src: [rows, 64] bf16, rows a multiple of 16 and < 2^31, 16-byte aligned; tile_rows:
 * int32 [ntiles] first rows of the tiles (device-checked against rows; out-of-range values
 * read row 0 and record LLSA_ERR_INTERNAL); stages in {2, 4, 8}; 1 <= ctas <= 65535.
 * Writes nothing in global memory.
 */
llsa_status llsa_gather_probe(const void* src, int64_t rows, const int32_t* tile_rows, int32_t ntiles,
                              int32_t stages, int32_t ctas, llsa_stream_t stream);

/*
 * Index transpose for callers that cannot hand the library any device memory
 * (no counterpart on the pages: an interface addition of this library).
 *
 * llsa_index_transpose needs scratch that its caller allocates.  Some callers cannot do
 * that: a plugin host that passes kernels only their inputs and outputs, or a runtime whose
 * device memory is planned once at start-up and may not grow or be requested per call.
 * This entry point takes no workspace and allocates nothing (no cudaMalloc, no allocating
 * library routine).  Its scratch is a fixed array inside libllsa.so of
 * LLSA_NOALLOC_SCRATCH_BYTES (8 MiB), which every GPU that loads the library holds until the
 * process exits.
 *
 *  - Shapes whose llsa_transpose_workspace_bytes() exceeds LLSA_NOALLOC_SCRATCH_BYTES are
 *    rejected with LLSA_ERR_WORKSPACE before anything is launched (the headline shape
 *    B=1, H=6, N=65536, L=3, K=8 needs about 0.9 MB; N=262144, K=16 about 6.8 MB).
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *    with that device current; make that first call before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents.  The transpose
 *    writes every scratch word before it reads it, so nothing needs clearing, but calls
 *    whose kernels can overlap on the GPU (different streams, or different host threads
 *    without ordering) race on the array: order them, e.g. on one stream.
 *  - Arguments, outputs, validation and results are those of llsa_index_transpose.
 */
#define LLSA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
llsa_status llsa_index_transpose_noalloc(const llsa_shape* shape, const int32_t* idx, int32_t* row_ptr,
                                         int32_t* col, llsa_stream_t stream);

/*
 * Per-launch trace (instrumentation; no counterpart on the pages).  Between
 * llsa_trace_begin and llsa_trace_end, every kernel launch made by the calling host thread
 * through the calls above is bracketed by two cudaEventRecord calls on that call's stream:
 * launch i records events[2i] just before and events[2i+1] just after, and stores its kernel
 * id (llsa_kernel_name gives the name) in kernel_ids[i].  `events` holds 2 * capacity
 * cudaEvent_t handles created by the caller (timing enabled); launches beyond `capacity`
 * are not traced.  llsa_trace_end stops tracing and reports the number of launches traced.
 */
llsa_status llsa_trace_begin(void** events, int32_t* kernel_ids, int32_t capacity);
llsa_status llsa_trace_end(int32_t* launches_out);
const char* llsa_kernel_name(int32_t kernel_id);

#ifdef __cplusplus
}
#endif

#endif /* LLSA_H_ */
