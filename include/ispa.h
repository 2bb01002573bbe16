/*
 * ispa.h -- C ABI of the ISPA hot path for NVIDIA B200 (sm_100a).
 *
 * Method: "Towards Memory-Efficient Autoregressive Video Generation via
 * Instance-Specific Parametric Absorption" (ISPA).  Citations below name the
 * page and its section:
 *   [gist §2.1] gist.science technical summary, section 2, stage 1
 *               "Dual-Stream Warmup": A_full over sink + history + current,
 *               A_loc over sink + current, obtained from one Decomposable
 *               Attention pass (a local and a historical branch, each with its
 *               log-sum-exp state, fused post hoc).
 *   [gist §2.2] stage 2 "Layer Absorb": the ridge objective
 *               ||A_loc (W + dW) - A_full W||^2 + lambda ||dW||^2 and its
 *               closed-form minimiser dW = (A_loc^T A_loc + lambda I)^-1
 *               A_loc^T (A_full - A_loc) W.
 *   [gist §2.3] stage 3 "Memory-Efficient Inference": the selected layers evict
 *               K_hist, V_hist and run local attention with W_new = W + dW.
 *   [gist §3]   "Key Contributions" item 2: decomposition grounded in online
 *               softmax.
 *   [gist sel]  "Dynamic Layer Selection": every layer is ranked by its
 *               reconstruction error after the warm-up.
 *   [gist §4]   "Experimental Results", item "Speedup": ISPA combined with
 *               post-training W8A8 quantisation.
 *
 * Conventions shared by every entry point
 *   - Layout: token-major row-major matrices [n, D] with the heads interleaved,
 *     i.e. element (token t, head h, channel c) at t * row_stride + h * head_dim + c.
 *     D = n_heads * head_dim.  W is [D_in, D_out] row-major and y = A @ W.
 *   - Pointers are DEVICE pointers owned by the caller unless stated otherwise.
 *     The library never allocates, frees or synchronises; every call is
 *     asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream).  Device pointers must be 16-byte aligned and row strides
 *     multiples of 16 bytes.
 *   - A host-detectable problem (null required pointer, unsupported shape or
 *     dtype, misalignment) returns an error code synchronously and launches
 *     nothing; ispa_last_error() then describes it (thread-local string).
 *   - Device-detected problems are written to *dev_status (int32 in device
 *     memory; the caller zeroes it and reads it after synchronising): the first
 *     error wins.  ISPA_ERR_NOT_SPD carries the failing pivot row in
 *     dev_status[1] when the buffer holds two int32.
 *   - A launch failure returns ISPA_ERR_CUDA.
 *   - dtype ISPA_DT_BF16: activations are bf16, tensor-core (tcgen05) path,
 *     fp32 accumulation.  ISPA_DT_F32: activations are fp32, computed on the
 *     CUDA cores in fp32.
 */
#ifndef ISPA_H_
#define ISPA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ISPA_API __attribute__((visibility("default")))
#else
#define ISPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ISPA_OK = 0,
  ISPA_ERR_INVALID_ARG = 1,
  ISPA_ERR_UNSUPPORTED = 2,
  ISPA_ERR_CUDA = 3,
  ISPA_ERR_NOT_SPD = 4,
  ISPA_ERR_TIMEOUT = 5,
  ISPA_ERR_WORKSPACE = 6
} ispa_status_t;

typedef enum { ISPA_DT_BF16 = 0, ISPA_DT_F32 = 1 } ispa_dtype_t;

/* Maximum number of KV segments of one attention call, both branches together. */
#define ISPA_MAX_SEGMENTS 8

/* One contiguous run of cached keys and values (e.g. the sink frame, the
 * history, the current chunk).  k and v are [n_tokens, D] device matrices with
 * row stride `row_stride` ELEMENTS.  n_tokens may be 0 (the segment is then
 * ignored and k, v may be NULL). */
typedef struct {
  const void* k;
  const void* v;
  int64_t n_tokens;
  int64_t row_stride;
} ispa_kv_segment_t;

/*
 * ispa_dual_attention -- Decomposable Attention of one chunk [gist §2.1, §3].
 *
 * q        [n_q, D], row stride q_stride elements, post-positional-encoding.
 * local    n_local segments forming the local context (sink + current chunk).
 * hist     n_hist segments forming the evicted-history context; their total
 *          may be 0 tokens.
 * softmax_scale   multiplies q.k; 0 selects 1/sqrt(head_dim).
 *
 * Dual mode (a_loc != NULL): the local branch gives A_loc and LSE_loc, the
 *   historical branch gives (O_hist, LSE_hist); they are fused in the epilogue:
 *   LSE_full = logaddexp(LSE_loc, LSE_hist), w = exp(LSE_hist - LSE_full),
 *   A_full = A_loc + w (O_hist - A_loc), a_delta = A_full - A_loc.
 *   An empty history gives A_full = A_loc and a_delta = 0.
 * Single-pass mode (a_loc == NULL): one online-softmax pass over local + hist
 *   writes a_full and lse_full only (the F-layer after the transition, or
 *   attention over any key set).
 *
 * Outputs (device, caller-owned): a_loc, a_full, a_delta [n_q, D] with row
 * stride D, dtype dt (a_delta nullable); lse_loc, lse_full [n_heads, n_q] fp32
 * natural-log LSE (nullable).  head_dim must be 64 or 128; n_q >= 1; at least
 * one key overall, and at least one local key in dual mode.
 */
ISPA_API ispa_status_t ispa_dual_attention(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim,
                                  ispa_dtype_t dt, float softmax_scale, const ispa_kv_segment_t* local,
                                  int32_t n_local, const ispa_kv_segment_t* hist, int32_t n_hist, void* a_loc,
                                  void* a_full, void* a_delta, float* lse_loc, float* lse_full, int32_t* dev_status,
                                  void* stream);

/*
 * ispa_lse_merge -- standalone post-hoc fusion of two attention branches
 * through their LSE states [gist §2.1].  o_loc, o_hist [n_q, D] (dtype dt, row
 * stride D); lse_loc, lse_hist [n_heads, n_q] fp32 (lse_hist = -inf marks an
 * empty branch).  Writes a_full = exp(L_loc - L) o_loc + exp(L_hist - L) o_hist,
 * a_delta = a_full - o_loc (nullable) and lse_full = L (nullable), with
 * L = logaddexp(L_loc, L_hist).  A (row, head) pair whose two LSEs are both
 * -inf (both branches empty) gets both weights 0: a_full = 0 and L = -inf, as
 * attention over the empty union of the key sets.  Outputs may not alias inputs.
 */
ISPA_API ispa_status_t ispa_lse_merge(const void* o_loc, const float* lse_loc, const void* o_hist, const float* lse_hist,
                             int64_t n_q, int32_t n_heads, int32_t head_dim, ispa_dtype_t dt, void* a_full,
                             void* a_delta, float* lse_full, void* stream);

/*
 * ispa_gram_accumulate -- sufficient statistics of the Layer-Absorb ridge
 * problem [gist §2.2]: G += A_loc^T A_loc and R += A_loc^T (A_full - A_loc),
 * summed over the n_rows rows of one call (the warm-up rows, [gist §2.1]).
 * a_loc, a_delta [n_rows, d_model], dtype dt, row stride row_stride elements.
 * G, R [d_model, d_model] fp32 row-major, accumulated in place; zero_first != 0
 * overwrites them instead.  G is symmetric: only its lower triangle (row >= col)
 * is guaranteed; entries above the diagonal are unspecified (ispa_absorb_solve
 * reads the lower triangle only).  d_model must be a multiple of 128 (bf16) or 4
 * (fp32).  n_rows == 0 is a no-op (or a zero fill when zero_first != 0).
 */
ISPA_API ispa_status_t ispa_gram_accumulate(const void* a_loc, const void* a_delta, int64_t n_rows, int64_t d_model,
                                   int64_t row_stride, ispa_dtype_t dt, float* G, float* R, int32_t zero_first,
                                   void* stream);

/*
 * ispa_sym_gram_accumulate -- E += x^T x for the instance-specific layer
 * selection ("Dynamic Layer Selection" of the gist.science technical summary):
 * with x = A_full - A_loc over the warm-up rows, E completes, together with
 * G and R of ispa_gram_accumulate, the statistics from which a layer's
 * reconstruction error follows without storing its activations.
 * x [n_rows, d_model], dtype dt, row stride row_stride elements; E
 * [d_model, d_model] fp32 row-major, accumulated in place (zero_first != 0
 * overwrites).  Only the lower triangle of E (row >= col) is guaranteed.
 * d_model must be a multiple of 128 (bf16) or 4 (fp32).  n_rows == 0 is a
 * no-op (or a zero fill when zero_first != 0).
 */
ISPA_API ispa_status_t ispa_sym_gram_accumulate(const void* x, int64_t n_rows, int64_t d_model, int64_t row_stride,
                                                ispa_dtype_t dt, float* E, int32_t zero_first, void* stream);

/* Bytes of device workspace ispa_layer_error needs for d_model (32 d^2). */
ISPA_API size_t ispa_layer_error_workspace_bytes(int64_t d_model);

/*
 * ispa_layer_error -- reconstruction error of one layer after the warm-up
 * ("Dynamic Layer Selection": all layers are ranked by it and the lowest are
 * converted to L-layers).  The error is read as the relative squared
 * Frobenius error of the absorbed local stream over the warm-up rows,
 *   eps = ||A_loc (W + dW) - A_full W||^2 / ||A_full W||^2,
 * evaluated from the statistics: with dA = A_full - A_loc, G = A_loc^T A_loc,
 * R = A_loc^T dA, E = dA^T dA (lower triangles of G and E are read),
 *   num_den[0] = <dW, G dW> - 2 <dW, R W> + <W, E W>,
 *   num_den[1] = <W, G W> + 2 <W, R W> + <W, E W>,
 * and eps = num_den[0] / num_den[1].  G, R, E, delta_w fp32 [D, D]; W [D, D]
 * in w_dt; num_den: two device doubles (8-byte aligned), overwritten.  The
 * products: with a bf16 W and D % 128 == 0, D >= 256, split-precision
 * tensor-core products (each fp32 operand as a bf16 hi/lo pair, about 2^-17
 * relative; W is exact), otherwise fp32 products on the CUDA cores; sums in
 * fp64.  workspace: at least ispa_layer_error_workspace_bytes bytes, 16-byte
 * aligned.  Asynchronous on `stream`.
 */
ISPA_API ispa_status_t ispa_layer_error(const float* G, const float* R, const float* E, const void* W,
                                        ispa_dtype_t w_dt, const float* delta_w, int64_t d_model, void* workspace,
                                        size_t workspace_bytes, double* num_den, void* stream);

/*
 * ispa_select_layers -- host bookkeeping of the layer selection: selected[l]
 * = 1 for the k layers with the smallest eps[l] (host array of n_layers
 * doubles), ties to the lower layer index, NaN ranked after every number;
 * 0 elsewhere.  0 <= k <= n_layers <= 4096.
 */
ISPA_API ispa_status_t ispa_select_layers(const double* eps, int32_t n_layers, int32_t k, uint8_t* selected);

/* Bytes of device workspace ispa_absorb_solve needs for d_model. */
ISPA_API size_t ispa_absorb_workspace_bytes(int64_t d_model);

/*
 * ispa_absorb_solve -- closed-form weight modulation [gist §2.2, §2.3].
 * lambda = lambda_abs + lambda_rel * trace(G) / d_model (computed on the device);
 * delta_w = (G + lambda I)^-1 R W by a blocked Cholesky factorisation and
 * triangular solves; w_new = W + delta_w rounded to w_dt (nullable).  With a
 * bf16 W and d_model a multiple of 128 (>= 256) the products run on the tensor
 * cores in split precision (bf16 hi/lo pairs, about 2^-17 relative per
 * product) and the solves are carried through the factorisation; otherwise
 * (fp32 W, other sizes) the updates run on the CUDA cores in fp32.  The
 * tensor-core form runs its chain of diagonal factorisations on an internal
 * stream beside the panel applications and update products (joined by events
 * recorded on `stream`, so the call stays asynchronous and graph capture sees
 * one exchange of events per panel; each diagonal step is launched with
 * programmatic stream serialisation behind the one before it);
 * that stream and its two events are created on the first such call in a host
 * thread and CUDA context -- make that call before any stream capture -- and
 * live until the process exits.
 * G, R fp32 [D, D] (G symmetric; only its lower triangle is read), W and w_new
 * [D, D] in w_dt, delta_w fp32 [D, D].  workspace: device buffer of at least
 * ispa_absorb_workspace_bytes(d_model) bytes, 256-byte aligned.  dev_status
 * receives ISPA_ERR_NOT_SPD (and the pivot row in dev_status[1]) when
 * G + lambda I is not numerically positive definite; the outputs are then
 * undefined.  d_model must be a multiple of 64.
 */
ISPA_API ispa_status_t ispa_absorb_solve(const float* G, const float* R, const void* W, ispa_dtype_t w_dt, int64_t d_model,
                                double lambda_abs, double lambda_rel, float* delta_w, void* w_new, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * ispa_absorb_solve_noalloc -- the same solve as ispa_absorb_solve, for callers
 * that cannot allocate device memory.  The ISPA method has no counterpart of
 * this call; it exists for deployment: code running inside a host callback or
 * an allocator hook, a plugin that receives device pointers but no allocator,
 * or a serving process whose device memory is fixed before it starts cannot
 * call cudaMalloc, so it cannot provide the workspace ispa_absorb_solve needs.
 * Here the working matrices live in a device array owned by the library
 * (4 d^2 + 256 d + 256 bytes for d = 2048, about 17.3 MB), which every GPU that
 * loads libispa holds until the process exits.  The caller still passes G, R,
 * W and the outputs, exactly as for ispa_absorb_solve.  To keep the array that
 * small it always runs the compact form of the solve (fp32 CUDA-core updates),
 * whose dW agrees with ispa_absorb_solve's within the solve's accuracy.
 *   - d_model must be a multiple of 64 and at most 2048; larger sizes return
 *     ISPA_ERR_UNSUPPORTED without launching.
 *   - No allocation of any kind happens, and nothing needs clearing: each call
 *     writes every working value before reading it.
 *   - The first call in a CUDA context (normally one per device; a new one
 *     after cudaDeviceReset) looks up the array's device address in that
 *     context (cudaGetSymbolAddress) and caches it under the context's unique
 *     id; make that first call before any stream capture.
 *   - All calls on a device share the one array: calls whose executions overlap
 *     on the GPU (different streams without ordering between them) race and
 *     give undefined results.  Calls on one stream are safe.
 */
ISPA_API ispa_status_t ispa_absorb_solve_noalloc(const float* G, const float* R, const void* W, ispa_dtype_t w_dt,
                                                 int64_t d_model, double lambda_abs, double lambda_rel,
                                                 float* delta_w, void* w_new, int32_t* dev_status, void* stream);

/*
 * ispa_project -- y = a @ w for one layer's output projection (the warm-up and
 * F-layer output, and the second half of ispa_local_attention_project).
 * a [n_rows, d_in] (row stride a_stride elements), w [d_in, d_out] row-major,
 * y [n_rows, d_out] row-major; all dtype dt; fp32 accumulation.  bf16 needs
 * d_in and d_out multiples of 64.
 */
ISPA_API ispa_status_t ispa_project(const void* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                           ispa_dtype_t dt, const void* w, void* y, void* stream);

/*
 * ispa_local_attention_project -- post-transition L-layer [gist §2.3]:
 * A_loc = attention over the local segments only (the history was evicted),
 * then y = A_loc @ W_new.  a_loc_out [n_q, D] receives A_loc and is required
 * (it carries A_loc from the attention kernel to the projection kernel).
 * Arguments otherwise as ispa_dual_attention and ispa_project.
 */
ISPA_API ispa_status_t ispa_local_attention_project(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads,
                                           int32_t head_dim, ispa_dtype_t dt, float softmax_scale,
                                           const ispa_kv_segment_t* local, int32_t n_local, const void* w_new,
                                           void* y, void* a_loc_out, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- W8A8 --
 * Source: post-training W8A8 quantisation of the projection, which ISPA is
 * run with in "Instance-Specific Parametric Absorption" (gist.science
 * technical summary, section 4 "Experimental Results", item "Speedup").  The
 * page fixes no scheme.  This library's reading:
 *   - the 8-bit format is e4m3 (bias 7, 3 mantissa bits, largest finite 448,
 *     no infinity);
 *   - activations get one fp32 scale per token row, and the weight W
 *     [d_in, d_out] one per output channel (column): s = amax / 448, or 1 for
 *     an all-zero row or column;
 *   - code = e4m3(x / s), round to nearest even, saturating at +-448, with
 *     amax / 448 and x / s computed as IEEE fp32 divisions;
 *   - y[i, j] = s_a[i] * s_w[j] * sum_k dec(qa[i, k]) * dec(qw[k, j]), fp32
 *     accumulation on the tensor cores, bf16 output;
 *   - the weight is quantised after the absorb, that is W_new = W + dW.
 * All pointers are device pointers owned by the caller.  Nothing allocates;
 * everything runs asynchronously on `stream`.
 *
 * ispa_quantize_e4m3_rows:
 *   - x [n_rows, k] bf16, row_stride elements apart;
 *   - codes [n_rows, k] bytes, dense;
 *   - scales [n_rows] fp32;
 *   - k must be a multiple of 16; x, its rows and codes 16-byte aligned.
 * ispa_quantize_e4m3_weight:
 *   - w [d_in, d_out] bf16, row-major;
 *   - codes_t [d_out, d_in] bytes: the codes TRANSPOSED, one row per output
 *     channel;
 *   - scales [d_out] fp32;
 *   - d_in and d_out must be multiples of 16.
 * ispa_project_w8a8:
 *   - y [n_rows, d_out] bf16 from a_codes [n_rows, d_in], a_scales [n_rows],
 *     w_codes_t [d_out, d_in] and w_scales [d_out];
 *   - d_in % 16 == 0 and d_out % 128 == 0;
 *   - codes, w_scales and y must be 16-byte aligned.
 * ispa_local_attention_project_w8a8: the L-layer of ispa_local_attention_project
 * with the W8A8 projection.  It runs the bf16 local attention into a_loc_out,
 * quantises A_loc into a_codes [n_q, D] / a_scales [n_q], then projects with the
 * quantised W_new.
 * Errors:
 *   - ISPA_ERR_INVALID_ARG for a NULL or misaligned pointer or a non-positive
 *     size;
 *   - ISPA_ERR_UNSUPPORTED for another dtype or sizes off the multiples above;
 *   - nothing is launched in either case.
 */
ISPA_API ispa_status_t ispa_quantize_e4m3_rows(const void* x, int64_t n_rows, int64_t k, int64_t row_stride,
                                               ispa_dtype_t dt, uint8_t* codes, float* scales, void* stream);
ISPA_API ispa_status_t ispa_quantize_e4m3_weight(const void* w, int64_t d_in, int64_t d_out, ispa_dtype_t dt,
                                                 uint8_t* codes_t, float* scales, void* stream);
ISPA_API ispa_status_t ispa_project_w8a8(const uint8_t* a_codes, const float* a_scales, int64_t n_rows, int64_t d_in,
                                         const uint8_t* w_codes_t, const float* w_scales, int64_t d_out, void* y,
                                         void* stream);
ISPA_API ispa_status_t ispa_local_attention_project_w8a8(const void* q, int64_t n_q, int64_t q_stride,
                                                         int32_t n_heads, int32_t head_dim, ispa_dtype_t dt,
                                                         float softmax_scale, const ispa_kv_segment_t* local,
                                                         int32_t n_local, const uint8_t* w_codes_t,
                                                         const float* w_scales, void* y, void* a_loc_out,
                                                         uint8_t* a_codes, float* a_scales, int32_t* dev_status,
                                                         void* stream);

/* ------------------------------------------------------- W8A8, MX form --
 * The same W8A8 projection with block-scaled (MX) activation codes, which
 * the attention epilogue can write itself: a CTA there holds one head's
 * channels of a row, so it can scale blocks of 32 consecutive channels but not
 * a whole row.  Source as above (section 4, "Speedup"); this library's
 * reading of the MX form:
 *   - each block of 32 consecutive elements of an activation row has one
 *     power-of-two scale 2^e, e the smallest integer with amax * 2^-e <= 448
 *     (0 for an all-zero block, at least -127), stored as the ue8m0 byte
 *     e + 127;
 *   - code = e4m3(x * 2^-e), round to nearest even (the scaling is exact);
 *     the activations quantised are the bf16 values;
 *   - the weight keeps the per-output-channel codes and fp32 scales of
 *     ispa_quantize_e4m3_weight;
 *   - y[i, j] = s_w[j] * sum over blocks b of 2^(e[i, b])
 *     * sum over k in b of dec(qa[i, k]) * dec(qw[k, j]), fp32 accumulation
 *     (kind::mxf8f6f4 block-scaled tensor-core MMAs), bf16 output.
 * All pointers are device pointers owned by the caller.  Nothing allocates;
 * everything runs asynchronously on `stream`.
 *
 * ispa_mx_quantize_e4m3_rows:
 *   - x [n_rows, k] bf16, row_stride elements apart;
 *   - codes [n_rows, k] bytes, dense; exps [n_rows, k / 32] bytes, dense;
 *   - k must be a multiple of 32; x, its rows and codes 16-byte aligned.
 * ispa_project_mx:
 *   - y [n_rows, d_out] bf16 from a_codes [n_rows, d_in], a_exps
 *     [n_rows, d_in / 32], w_codes_t [d_out, d_in] and w_scales [d_out];
 *   - d_in a multiple of 128 and at most 3584 (the scales of a 128-row tile
 *     live in tensor memory beside its accumulators), d_out % 128 == 0;
 *   - codes, w_scales and y 16-byte aligned, a_exps 4-byte aligned.
 * ispa_local_attention_project_mx: the L-layer of ispa_local_attention_project
 * with the MX projection.  The single-pass local attention writes the MX codes
 * and exponents of A_loc (a_codes [n_q, D], a_exps [n_q, D / 32]) from its
 * epilogue instead of bf16 A_loc, then the block-scaled product with the
 * quantised W_new runs.  D = n_heads * head_dim as in ispa_project_mx.
 * Errors as for the W8A8 calls above; nothing is launched on an error.
 */
ISPA_API ispa_status_t ispa_mx_quantize_e4m3_rows(const void* x, int64_t n_rows, int64_t k, int64_t row_stride,
                                                  ispa_dtype_t dt, uint8_t* codes, uint8_t* exps, void* stream);
ISPA_API ispa_status_t ispa_project_mx(const uint8_t* a_codes, const uint8_t* a_exps, int64_t n_rows, int64_t d_in,
                                       const uint8_t* w_codes_t, const float* w_scales, int64_t d_out, void* y,
                                       void* stream);
ISPA_API ispa_status_t ispa_local_attention_project_mx(const void* q, int64_t n_q, int64_t q_stride,
                                                       int32_t n_heads, int32_t head_dim, ispa_dtype_t dt,
                                                       float softmax_scale, const ispa_kv_segment_t* local,
                                                       int32_t n_local, const uint8_t* w_codes_t,
                                                       const float* w_scales, void* y, uint8_t* a_codes,
                                                       uint8_t* a_exps, int32_t* dev_status, void* stream);

/* ------------------------------------------------------ host bookkeeping --
 * Streaming bookkeeping of [gist §2.1, §2.3], host-only and exact (integers).
 *
 * ispa_chunk_token_ranges: half-open token ranges [begin, end) of the sink,
 * history and current segments seen by rollout chunk `chunk` (0-based), written
 * to out[0..5] = {sink_b, sink_e, hist_b, hist_e, cur_b, cur_e}.  Chunk 0 holds
 * the sink frame inside its own current chunk: no separate sink, no history.
 * Chunk c >= 1: sink = first sink_frames frames, history = the frames between
 * the sink and the current chunk, current = frames [c*chunk_frames,
 * (c+1)*chunk_frames).  Returns ISPA_ERR_INVALID_ARG on negative sizes and,
 * for chunk >= 1, when the sink does not end before the current chunk starts
 * (sink_frames > chunk * chunk_frames): the ranges would overlap.
 */
ISPA_API ispa_status_t ispa_chunk_token_ranges(int64_t chunk, int64_t frame_tokens, int64_t chunk_frames,
                                      int64_t sink_frames, int64_t* out);

/* KV bytes held by n_layers layers at chunk `chunk`: bit l of l_layer_mask marks
 * an L-layer; once `transitioned` is non-zero an L-layer keeps only the sink and
 * current tokens, an F-layer keeps every frame up to the current chunk.
 * Returns -1 on invalid arguments (those ispa_chunk_token_ranges rejects
 * included). */
ISPA_API int64_t ispa_kv_bytes(int64_t chunk, int32_t n_layers, uint64_t l_layer_mask, int32_t transitioned,
                      int64_t frame_tokens, int64_t chunk_frames, int64_t d_model, int32_t elem_bytes,
                      int64_t sink_frames);

/* --------------------------------------------------------- diagnostics -- */
/* Runs one block that waits on a barrier nobody arrives at, with a limit of
 * timeout_us microseconds, then writes ISPA_ERR_TIMEOUT to *dev_status and
 * returns.  Exercises the bounded-wait path without faulting the GPU. */
ISPA_API ispa_status_t ispa_selftest_wait_timeout(uint32_t timeout_us, int32_t* dev_status, void* stream);

ISPA_API const char* ispa_status_string(ispa_status_t s);
ISPA_API const char* ispa_last_error(void);
ISPA_API int32_t ispa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ISPA_H_ */
