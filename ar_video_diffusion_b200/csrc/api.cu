// C ABI of libispa: argument validation and dispatch to the kernels.  Nothing
// here allocates, frees or synchronises; every launch goes to the caller's
// stream.  Host bookkeeping of the streaming KV cache lives here too.
#include <climits>
#include <cmath>
#include <cstring>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
ispa_status_t dual_attention_bf16_db(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim,
                                     float scale, const ispa_kv_segment_t* segs, int n_local_seg, int n_hist_seg,
                                     void* a_loc, void* a_full, void* a_delta, float* lse_loc, float* lse_full,
                                     int32_t* status, cudaStream_t stream, uint8_t* mx_codes = nullptr,
                                     uint8_t* mx_exps = nullptr);
ispa_status_t dual_attention_f32(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim,
                                 float scale, const ispa_kv_segment_t* segs, int n_local_seg, int n_hist_seg,
                                 void* a_loc, void* a_full, void* a_delta, float* lse_loc, float* lse_full,
                                 cudaStream_t stream);
ispa_status_t lse_merge_launch(const void* o_loc, const float* lse_loc, const void* o_hist, const float* lse_hist,
                               int64_t n_q, int32_t n_heads, int32_t head_dim, ispa_dtype_t dt, void* a_full,
                               void* a_delta, float* lse_full, cudaStream_t stream);
ispa_status_t gram_bf16(const void* a_loc, const void* a_delta, int64_t n_rows, int64_t D, int64_t row_stride,
                        float* G, float* R, bool overwrite, cudaStream_t stream);
ispa_status_t gram_f32(const float* a_loc, const float* a_delta, int64_t n_rows, int64_t D, int64_t row_stride,
                       float* G, float* R, bool overwrite, cudaStream_t st);
ispa_status_t project_bf16(const void* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                           const void* w, void* y, cudaStream_t stream);
ispa_status_t project_f32(const float* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                          const float* w, float* y, cudaStream_t st);
ispa_status_t sym_gram_bf16(const void* x, int64_t n_rows, int64_t D, int64_t row_stride, float* E, bool overwrite,
                            cudaStream_t stream);
ispa_status_t sym_gram_f32(const float* x, int64_t n_rows, int64_t D, int64_t row_stride, float* E, bool overwrite,
                           cudaStream_t st);
size_t layer_error_workspace_bytes(int64_t D);
ispa_status_t layer_error_launch(const float* G, const float* R, const float* E, const void* W, ispa_dtype_t w_dt,
                                 const float* dW, int64_t D, void* workspace, double* num_den, cudaStream_t st);
size_t absorb_workspace_bytes(int64_t D);
ispa_status_t absorb_solve_launch(const float* G, const float* R, const void* W, ispa_dtype_t w_dt, int64_t D,
                                  double lam_abs, double lam_rel, float* dW, void* w_new, void* workspace,
                                  int32_t* status, cudaStream_t st);

ispa_status_t quantize_rows_e4m3(const void* x, int64_t n_rows, int64_t K, int64_t stride, uint8_t* q, float* scale,
                                 cudaStream_t stream);
ispa_status_t quantize_weight_e4m3(const void* w, int64_t K, int64_t N, uint8_t* qt, float* scale,
                                   cudaStream_t stream);
ispa_status_t project_e4m3(const uint8_t* qa, const float* a_scale, int64_t n_rows, int64_t d_in,
                           const uint8_t* qw_t, const float* w_scale, int64_t d_out, void* y, cudaStream_t stream);
ispa_status_t mx_quantize_rows_e4m3(const void* x, int64_t n_rows, int64_t K, int64_t stride, uint8_t* q, uint8_t* e,
                                    cudaStream_t stream);
ispa_status_t project_mx(const uint8_t* qa, const uint8_t* ea, int64_t n_rows, int64_t d_in, const uint8_t* qw_t,
                         const float* w_scale, int64_t d_out, void* y, cudaStream_t stream);

static bool valid_dtype(ispa_dtype_t dt) { return dt == ISPA_DT_BF16 || dt == ISPA_DT_F32; }
static int64_t elem_bytes(ispa_dtype_t dt) { return dt == ISPA_DT_BF16 ? 2 : 4; }

// Validates the segment lists of an attention call and packs the non-empty
// segments (local first).  Returns ISPA_OK or an error with the reason set.
static ispa_status_t collect_segments(const ispa_kv_segment_t* local, int32_t n_local, const ispa_kv_segment_t* hist,
                                      int32_t n_hist, int64_t D, ispa_dtype_t dt, ispa_kv_segment_t* out,
                                      int* n_local_out, int* n_hist_out, int64_t* local_tokens,
                                      int64_t* hist_tokens) {
  if (n_local < 0 || n_hist < 0) return invalid("negative segment count");
  if ((n_local > 0 && !local) || (n_hist > 0 && !hist)) return invalid("segment list pointer is NULL");
  int k = 0;
  *local_tokens = *hist_tokens = 0;
  for (int b = 0; b < 2; ++b) {
    const ispa_kv_segment_t* list = b == 0 ? local : hist;
    const int n = b == 0 ? n_local : n_hist;
    int kept = 0;
    for (int i = 0; i < n; ++i) {
      const ispa_kv_segment_t& s = list[i];
      if (s.n_tokens < 0) return invalid("segment %d of branch %d has negative n_tokens", i, b);
      if (s.n_tokens == 0) continue;
      if (!s.k || !s.v) return invalid("segment %d of branch %d has a NULL k or v", i, b);
      if (s.row_stride < D) return invalid("segment row_stride %lld < D %lld", (long long)s.row_stride, (long long)D);
      if (!aligned16(s.k) || !aligned16(s.v) || (s.row_stride * elem_bytes(dt)) % 16)
        return invalid("segment k/v must be 16-byte aligned with 16-byte-multiple row strides");
      if (s.n_tokens > INT32_MAX / 2) return unsupported("segment longer than 2^30 tokens");
      if (k >= ISPA_MAX_SEGMENTS) return unsupported("more than %d non-empty KV segments", ISPA_MAX_SEGMENTS);
      out[k++] = s;
      ++kept;
      (b == 0 ? *local_tokens : *hist_tokens) += s.n_tokens;
    }
    (b == 0 ? *n_local_out : *n_hist_out) = kept;
  }
  return ISPA_OK;
}

static ispa_status_t check_attention_common(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads,
                                            int32_t head_dim, ispa_dtype_t dt, float scale) {
  if (!valid_dtype(dt)) return unsupported("unknown dtype %d", (int)dt);
  if (!q) return invalid("q is NULL");
  if (n_q <= 0) return invalid("n_q must be positive");
  if (n_q > INT32_MAX / 2) return unsupported("n_q too large");
  if (n_heads <= 0) return invalid("n_heads must be positive");
  if (head_dim != 64 && head_dim != 128) return unsupported("head_dim must be 64 or 128 (got %d)", head_dim);
  const int64_t D = (int64_t)n_heads * head_dim;
  if (q_stride < D) return invalid("q_stride %lld < D %lld", (long long)q_stride, (long long)D);
  if (!aligned16(q) || (q_stride * elem_bytes(dt)) % 16) return invalid("q must be 16-byte aligned");
  if (!(scale >= 0.f) || !std::isfinite(scale)) return invalid("softmax_scale must be finite and >= 0");
  return ISPA_OK;
}

}  // namespace ispa

using namespace ispa;

extern "C" ispa_status_t ispa_dual_attention(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads,
                                             int32_t head_dim, ispa_dtype_t dt, float softmax_scale,
                                             const ispa_kv_segment_t* local, int32_t n_local,
                                             const ispa_kv_segment_t* hist, int32_t n_hist, void* a_loc,
                                             void* a_full, void* a_delta, float* lse_loc, float* lse_full,
                                             int32_t* dev_status, void* stream) {
  ispa_status_t st = check_attention_common(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale);
  if (st != ISPA_OK) return st;
  const int64_t D = (int64_t)n_heads * head_dim;
  if (!a_full) return invalid("a_full is required");
  for (const void* o : {(const void*)a_loc, (const void*)a_full, (const void*)a_delta, (const void*)lse_loc,
                        (const void*)lse_full})
    if (o && !aligned16(o)) return invalid("outputs must be 16-byte aligned");
  ispa_kv_segment_t segs[ISPA_MAX_SEGMENTS];
  int nl = 0, nh = 0;
  int64_t lt = 0, ht = 0;
  st = collect_segments(local, n_local, hist, n_hist, D, dt, segs, &nl, &nh, &lt, &ht);
  if (st != ISPA_OK) return st;
  if (lt + ht == 0) return invalid("attention over an empty key set");
  if (a_loc && lt == 0) return invalid("dual mode needs at least one local key");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)head_dim);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dt == ISPA_DT_BF16)
    return dual_attention_bf16_db(q, n_q, q_stride, n_heads, head_dim, scale, segs, nl, nh, a_loc, a_full, a_delta,
                               lse_loc, lse_full, dev_status, s);
  return dual_attention_f32(q, n_q, q_stride, n_heads, head_dim, scale, segs, nl, nh, a_loc, a_full, a_delta,
                            lse_loc, lse_full, s);
}

extern "C" ispa_status_t ispa_lse_merge(const void* o_loc, const float* lse_loc, const void* o_hist,
                                        const float* lse_hist, int64_t n_q, int32_t n_heads, int32_t head_dim,
                                        ispa_dtype_t dt, void* a_full, void* a_delta, float* lse_full,
                                        void* stream) {
  if (!valid_dtype(dt)) return unsupported("unknown dtype %d", (int)dt);
  if (!o_loc || !lse_loc || !o_hist || !lse_hist || !a_full) return invalid("required pointer is NULL");
  if (n_q <= 0 || n_heads <= 0) return invalid("n_q and n_heads must be positive");
  if (head_dim <= 0 || head_dim % 8) return unsupported("head_dim must be a positive multiple of 8");
  if (n_heads > 64) return unsupported("at most 64 heads");
  for (const void* p : {o_loc, o_hist, (const void*)a_full, (const void*)a_delta})
    if (p && !aligned16(p)) return invalid("matrices must be 16-byte aligned");
  return lse_merge_launch(o_loc, lse_loc, o_hist, lse_hist, n_q, n_heads, head_dim, dt, a_full, a_delta, lse_full,
                          static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_gram_accumulate(const void* a_loc, const void* a_delta, int64_t n_rows, int64_t d_model,
                                              int64_t row_stride, ispa_dtype_t dt, float* G, float* R,
                                              int32_t zero_first, void* stream) {
  if (!valid_dtype(dt)) return unsupported("unknown dtype %d", (int)dt);
  if (!G || !R) return invalid("G and R are required");
  if (n_rows < 0 || d_model <= 0) return invalid("n_rows must be >= 0 and d_model > 0");
  if (row_stride < d_model) return invalid("row_stride < d_model");
  if (dt == ISPA_DT_BF16 && d_model % 128) return unsupported("bf16 statistics need d_model % 128 == 0");
  if (dt == ISPA_DT_F32 && d_model % 4) return unsupported("fp32 statistics need d_model % 4 == 0");
  if (d_model > 16384 || n_rows > INT32_MAX / 2) return unsupported("problem too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_rows == 0) {
    if (!zero_first) return ISPA_OK;
    cudaMemsetAsync(G, 0, (size_t)d_model * d_model * 4, s);
    cudaMemsetAsync(R, 0, (size_t)d_model * d_model * 4, s);
    return check_launch("memset");
  }
  if (!a_loc || !a_delta) return invalid("a_loc and a_delta are required");
  if (!aligned16(a_loc) || !aligned16(a_delta) || !aligned16(G) || !aligned16(R) ||
      (row_stride * elem_bytes(dt)) % 16)
    return invalid("pointers must be 16-byte aligned");
  if (dt == ISPA_DT_BF16) return gram_bf16(a_loc, a_delta, n_rows, d_model, row_stride, G, R, zero_first != 0, s);
  return gram_f32(static_cast<const float*>(a_loc), static_cast<const float*>(a_delta), n_rows, d_model, row_stride,
                  G, R, zero_first != 0, s);
}

extern "C" ispa_status_t ispa_sym_gram_accumulate(const void* x, int64_t n_rows, int64_t d_model, int64_t row_stride,
                                                  ispa_dtype_t dt, float* E, int32_t zero_first, void* stream) {
  if (!valid_dtype(dt)) return unsupported("unknown dtype %d", (int)dt);
  if (!E) return invalid("E is required");
  if (n_rows < 0 || d_model <= 0) return invalid("n_rows must be >= 0 and d_model > 0");
  if (row_stride < d_model) return invalid("row_stride < d_model");
  if (dt == ISPA_DT_BF16 && d_model % 128) return unsupported("bf16 statistics need d_model % 128 == 0");
  if (dt == ISPA_DT_F32 && d_model % 4) return unsupported("fp32 statistics need d_model % 4 == 0");
  if (d_model > 16384 || n_rows > INT32_MAX / 2) return unsupported("problem too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_rows == 0) {
    if (!zero_first) return ISPA_OK;
    cudaMemsetAsync(E, 0, (size_t)d_model * d_model * 4, s);
    return check_launch("memset");
  }
  if (!x) return invalid("x is required");
  if (!aligned16(x) || !aligned16(E) || (row_stride * elem_bytes(dt)) % 16)
    return invalid("pointers must be 16-byte aligned");
  if (dt == ISPA_DT_BF16) return sym_gram_bf16(x, n_rows, d_model, row_stride, E, zero_first != 0, s);
  return sym_gram_f32(static_cast<const float*>(x), n_rows, d_model, row_stride, E, zero_first != 0, s);
}

extern "C" size_t ispa_layer_error_workspace_bytes(int64_t d_model) {
  return d_model > 0 ? layer_error_workspace_bytes(d_model) : 0;
}

extern "C" ispa_status_t ispa_layer_error(const float* G, const float* R, const float* E, const void* W,
                                          ispa_dtype_t w_dt, const float* delta_w, int64_t d_model, void* workspace,
                                          size_t workspace_bytes, double* num_den, void* stream) {
  if (!valid_dtype(w_dt)) return unsupported("unknown dtype %d", (int)w_dt);
  if (!G || !R || !E || !W || !delta_w || !workspace || !num_den) return invalid("required pointer is NULL");
  if (d_model <= 0 || d_model > 16384) return unsupported("d_model must lie in [1, 16384]");
  if (workspace_bytes < layer_error_workspace_bytes(d_model)) {
    set_last_error("workspace holds %zu bytes, %zu needed", workspace_bytes, layer_error_workspace_bytes(d_model));
    return ISPA_ERR_WORKSPACE;
  }
  if ((reinterpret_cast<uintptr_t>(num_den) & 7u) != 0) return invalid("num_den must be 8-byte aligned");
  for (const void* p : {(const void*)G, (const void*)R, (const void*)E, W, (const void*)delta_w,
                        (const void*)workspace})
    if (!aligned16(p)) return invalid("matrices must be 16-byte aligned");
  return layer_error_launch(G, R, E, W, w_dt, delta_w, d_model, workspace, num_den, static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_select_layers(const double* eps, int32_t n_layers, int32_t k, uint8_t* selected) {
  if (n_layers < 0 || n_layers > 4096) return invalid("n_layers must lie in [0, 4096]");
  if (k < 0 || k > n_layers) return invalid("k must lie in [0, n_layers]");
  if (n_layers > 0 && (!eps || !selected)) return invalid("eps and selected are required");
  // rank: numbers before NaN, increasing value, then increasing layer index
  int32_t order[4096];
  for (int32_t l = 0; l < n_layers; ++l) order[l] = l;
  auto before = [&](int32_t a, int32_t b) {
    const bool na = std::isnan(eps[a]), nb = std::isnan(eps[b]);
    if (na != nb) return nb;
    if (!na && eps[a] != eps[b]) return eps[a] < eps[b];
    return a < b;
  };
  for (int32_t i = 1; i < n_layers; ++i) {  // insertion sort: stable, n_layers is small
    const int32_t v = order[i];
    int32_t j = i;
    for (; j > 0 && before(v, order[j - 1]); --j) order[j] = order[j - 1];
    order[j] = v;
  }
  for (int32_t l = 0; l < n_layers; ++l) selected[l] = 0;
  for (int32_t i = 0; i < k; ++i) selected[order[i]] = 1;
  return ISPA_OK;
}

extern "C" size_t ispa_absorb_workspace_bytes(int64_t d_model) {
  return d_model > 0 ? absorb_workspace_bytes(d_model) : 0;
}

extern "C" ispa_status_t ispa_absorb_solve(const float* G, const float* R, const void* W, ispa_dtype_t w_dt,
                                           int64_t d_model, double lambda_abs, double lambda_rel, float* delta_w,
                                           void* w_new, void* workspace, size_t workspace_bytes,
                                           int32_t* dev_status, void* stream) {
  if (!valid_dtype(w_dt)) return unsupported("unknown dtype %d", (int)w_dt);
  if (!G || !R || !W || !delta_w || !workspace) return invalid("required pointer is NULL");
  if (d_model <= 0 || d_model % 64) return unsupported("d_model must be a positive multiple of 64");
  if (d_model > 16384) return unsupported("d_model too large");
  if (!(lambda_abs >= 0.0) || !(lambda_rel >= 0.0) || !std::isfinite(lambda_abs) || !std::isfinite(lambda_rel))
    return invalid("lambda_abs and lambda_rel must be finite and >= 0");
  if (workspace_bytes < absorb_workspace_bytes(d_model)) {
    set_last_error("workspace holds %zu bytes, %zu needed", workspace_bytes, absorb_workspace_bytes(d_model));
    return ISPA_ERR_WORKSPACE;
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return invalid("workspace must be 256-byte aligned");
  for (const void* p : {(const void*)G, (const void*)R, W, (const void*)delta_w, (const void*)w_new})
    if (p && !aligned16(p)) return invalid("matrices must be 16-byte aligned");
  return absorb_solve_launch(G, R, W, w_dt, d_model, lambda_abs, lambda_rel, delta_w, w_new, workspace, dev_status,
                             static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_project(const void* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                                      ispa_dtype_t dt, const void* w, void* y, void* stream) {
  if (!valid_dtype(dt)) return unsupported("unknown dtype %d", (int)dt);
  if (!a || !w || !y) return invalid("required pointer is NULL");
  if (n_rows <= 0 || d_in <= 0 || d_out <= 0) return invalid("sizes must be positive");
  if (a_stride < d_in) return invalid("a_stride < d_in");
  if (!aligned16(a) || !aligned16(w) || !aligned16(y) || (a_stride * elem_bytes(dt)) % 16)
    return invalid("pointers must be 16-byte aligned");
  if (n_rows > INT32_MAX / 2 || d_in > 65536 || d_out > 65536) return unsupported("problem too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dt == ISPA_DT_BF16) {
    if (d_in % 64 || d_out % 128) return unsupported("bf16 projection needs d_in % 64 == 0 and d_out % 128 == 0");
    return project_bf16(a, n_rows, d_in, d_out, a_stride, w, y, s);
  }
  return project_f32(static_cast<const float*>(a), n_rows, d_in, d_out, a_stride, static_cast<const float*>(w),
                     static_cast<float*>(y), s);
}

extern "C" ispa_status_t ispa_local_attention_project(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads,
                                                      int32_t head_dim, ispa_dtype_t dt, float softmax_scale,
                                                      const ispa_kv_segment_t* local, int32_t n_local,
                                                      const void* w_new, void* y, void* a_loc_out,
                                                      int32_t* dev_status, void* stream) {
  if (!w_new || !y || !a_loc_out) return invalid("w_new, y and a_loc_out are required");
  const int64_t D = (int64_t)n_heads * head_dim;
  if (dt == ISPA_DT_BF16 && D % 128) return unsupported("bf16 L-layer projection needs D % 128 == 0");
  ispa_status_t st = ispa_dual_attention(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local,
                                         nullptr, 0, nullptr, a_loc_out, nullptr, nullptr, nullptr, dev_status,
                                         stream);
  if (st != ISPA_OK) return st;
  return ispa_project(a_loc_out, n_q, D, D, D, dt, w_new, y, stream);
}

// ------------------------------------------------------------------ W8A8
static inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

extern "C" ispa_status_t ispa_quantize_e4m3_rows(const void* x, int64_t n_rows, int64_t k, int64_t row_stride,
                                                 ispa_dtype_t dt, uint8_t* codes, float* scales, void* stream) {
  if (dt != ISPA_DT_BF16) return unsupported("e4m3 quantisation takes bf16 activations");
  if (!x || !codes || !scales) return invalid("required pointer is NULL");
  if (n_rows <= 0 || k <= 0) return invalid("sizes must be positive");
  if (k % 16) return unsupported("e4m3 quantisation needs k %% 16 == 0 (got %lld)", (long long)k);
  if (row_stride < k) return invalid("row_stride < k");
  if (!aligned16(x) || !aligned16(codes) || !aligned4(scales) || (row_stride * 2) % 16)
    return invalid("x and codes must be 16-byte aligned (rows too), scales 4-byte aligned");
  if (n_rows > INT32_MAX / 2 || k > 65536) return unsupported("problem too large");
  return quantize_rows_e4m3(x, n_rows, k, row_stride, codes, scales, static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_quantize_e4m3_weight(const void* w, int64_t d_in, int64_t d_out, ispa_dtype_t dt,
                                                   uint8_t* codes_t, float* scales, void* stream) {
  if (dt != ISPA_DT_BF16) return unsupported("e4m3 quantisation takes a bf16 weight");
  if (!w || !codes_t || !scales) return invalid("required pointer is NULL");
  if (d_in <= 0 || d_out <= 0) return invalid("sizes must be positive");
  if (d_in % 16 || d_out % 16) return unsupported("e4m3 weight quantisation needs d_in, d_out multiples of 16");
  if (!aligned16(w) || !aligned16(codes_t) || !aligned4(scales)) return invalid("pointers are misaligned");
  if (d_in > 65536 || d_out > 65536) return unsupported("problem too large");
  return quantize_weight_e4m3(w, d_in, d_out, codes_t, scales, static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_project_w8a8(const uint8_t* a_codes, const float* a_scales, int64_t n_rows,
                                           int64_t d_in, const uint8_t* w_codes_t, const float* w_scales,
                                           int64_t d_out, void* y, void* stream) {
  if (!a_codes || !a_scales || !w_codes_t || !w_scales || !y) return invalid("required pointer is NULL");
  if (n_rows <= 0 || d_in <= 0 || d_out <= 0) return invalid("sizes must be positive");
  if (d_in % 16 || d_out % 128)
    return unsupported("W8A8 projection needs d_in %% 16 == 0 and d_out %% 128 == 0 (got %lld, %lld)",
                       (long long)d_in, (long long)d_out);
  if (!aligned16(a_codes) || !aligned16(w_codes_t) || !aligned16(w_scales) || !aligned4(a_scales) || !aligned16(y))
    return invalid("codes, w_scales and y must be 16-byte aligned, a_scales 4-byte aligned");
  if (n_rows > INT32_MAX / 2 || d_in > 65536 || d_out > 65536) return unsupported("problem too large");
  return project_e4m3(a_codes, a_scales, n_rows, d_in, w_codes_t, w_scales, d_out, y,
                      static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_local_attention_project_w8a8(
    const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim, ispa_dtype_t dt,
    float softmax_scale, const ispa_kv_segment_t* local, int32_t n_local, const uint8_t* w_codes_t,
    const float* w_scales, void* y, void* a_loc_out, uint8_t* a_codes, float* a_scales, int32_t* dev_status,
    void* stream) {
  if (dt != ISPA_DT_BF16) return unsupported("the W8A8 L-layer path takes bf16 activations");
  if (!w_codes_t || !w_scales || !y || !a_loc_out || !a_codes || !a_scales)
    return invalid("w_codes_t, w_scales, y, a_loc_out, a_codes and a_scales are required");
  const int64_t D = (int64_t)n_heads * head_dim;
  if (D % 128) return unsupported("W8A8 L-layer projection needs D %% 128 == 0");
  ispa_status_t st = ispa_dual_attention(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale, local, n_local,
                                         nullptr, 0, nullptr, a_loc_out, nullptr, nullptr, nullptr, dev_status,
                                         stream);
  if (st != ISPA_OK) return st;
  st = ispa_quantize_e4m3_rows(a_loc_out, n_q, D, D, dt, a_codes, a_scales, stream);
  if (st != ISPA_OK) return st;
  return ispa_project_w8a8(a_codes, a_scales, n_q, D, w_codes_t, w_scales, D, y, stream);
}

extern "C" ispa_status_t ispa_mx_quantize_e4m3_rows(const void* x, int64_t n_rows, int64_t k, int64_t row_stride,
                                                    ispa_dtype_t dt, uint8_t* codes, uint8_t* exps, void* stream) {
  if (dt != ISPA_DT_BF16) return unsupported("MX quantisation takes bf16 activations");
  if (!x || !codes || !exps) return invalid("required pointer is NULL");
  if (n_rows <= 0 || k <= 0) return invalid("sizes must be positive");
  if (k % 32) return unsupported("MX quantisation needs k %% 32 == 0 (got %lld)", (long long)k);
  if (row_stride < k) return invalid("row_stride < k");
  if (!aligned16(x) || !aligned16(codes) || (row_stride * 2) % 16)
    return invalid("x and codes must be 16-byte aligned (rows too)");
  if (n_rows > INT32_MAX / 2 || k > 65536) return unsupported("problem too large");
  return mx_quantize_rows_e4m3(x, n_rows, k, row_stride, codes, exps, static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_project_mx(const uint8_t* a_codes, const uint8_t* a_exps, int64_t n_rows, int64_t d_in,
                                         const uint8_t* w_codes_t, const float* w_scales, int64_t d_out, void* y,
                                         void* stream) {
  if (!a_codes || !a_exps || !w_codes_t || !w_scales || !y) return invalid("required pointer is NULL");
  if (n_rows <= 0 || d_in <= 0 || d_out <= 0) return invalid("sizes must be positive");
  if (!aligned16(a_codes) || !aligned4(a_exps) || !aligned16(w_codes_t) || !aligned16(w_scales) || !aligned16(y))
    return invalid("codes, w_scales and y must be 16-byte aligned, a_exps 4-byte aligned");
  if (n_rows > INT32_MAX / 2 || d_out > 65536) return unsupported("problem too large");
  return project_mx(a_codes, a_exps, n_rows, d_in, w_codes_t, w_scales, d_out, y, static_cast<cudaStream_t>(stream));
}

extern "C" ispa_status_t ispa_local_attention_project_mx(
    const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim, ispa_dtype_t dt,
    float softmax_scale, const ispa_kv_segment_t* local, int32_t n_local, const uint8_t* w_codes_t,
    const float* w_scales, void* y, uint8_t* a_codes, uint8_t* a_exps, int32_t* dev_status, void* stream) {
  if (dt != ISPA_DT_BF16) return unsupported("the MX L-layer path takes bf16 activations");
  ispa_status_t st = check_attention_common(q, n_q, q_stride, n_heads, head_dim, dt, softmax_scale);
  if (st != ISPA_OK) return st;
  if (!w_codes_t || !w_scales || !y || !a_codes || !a_exps)
    return invalid("w_codes_t, w_scales, y, a_codes and a_exps are required");
  if (!aligned16(a_codes) || !aligned4(a_exps)) return invalid("a_codes must be 16-byte aligned, a_exps 4-byte");
  const int64_t D = (int64_t)n_heads * head_dim;
  if (D % 128) return unsupported("MX L-layer projection needs D %% 128 == 0");
  ispa_kv_segment_t segs[ISPA_MAX_SEGMENTS];
  int nl = 0, nh = 0;
  int64_t lt = 0, ht = 0;
  st = collect_segments(local, n_local, nullptr, 0, D, dt, segs, &nl, &nh, &lt, &ht);
  if (st != ISPA_OK) return st;
  if (lt == 0) return invalid("attention over an empty key set");
  // the projection's limits are checked before anything is launched
  if (D / 128 > 28) return unsupported("block-scaled projection needs D <= 3584 (got %lld)", (long long)D);
  if (!aligned16(w_codes_t) || !aligned16(w_scales) || !aligned16(y))
    return invalid("w_codes_t, w_scales and y must be 16-byte aligned");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)head_dim);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = dual_attention_bf16_db(q, n_q, q_stride, n_heads, head_dim, scale, segs, nl, 0, nullptr, nullptr, nullptr,
                              nullptr, nullptr, dev_status, s, a_codes, a_exps);
  if (st != ISPA_OK) return st;
  return project_mx(a_codes, a_exps, n_q, D, w_codes_t, w_scales, D, y, s);
}

// ------------------------------------------------------------ bookkeeping
extern "C" ispa_status_t ispa_chunk_token_ranges(int64_t chunk, int64_t frame_tokens, int64_t chunk_frames,
                                                 int64_t sink_frames, int64_t* out) {
  if (!out) return invalid("out is NULL");
  if (chunk < 0 || frame_tokens < 0 || chunk_frames < 0 || sink_frames < 0)
    return invalid("sizes must be non-negative");
  if (chunk > 0 && sink_frames > chunk * chunk_frames)
    return invalid("the sink (%lld frames) must end before chunk %lld starts (frame %lld)", (long long)sink_frames,
                   (long long)chunk, (long long)(chunk * chunk_frames));
  const int64_t F = frame_tokens, cf = chunk_frames;
  out[4] = chunk * cf * F;
  out[5] = (chunk + 1) * cf * F;
  if (chunk == 0) {
    out[0] = out[1] = out[2] = out[3] = 0;
  } else {
    out[0] = 0;
    out[1] = sink_frames * F;
    out[2] = sink_frames * F;
    out[3] = chunk * cf * F;
  }
  return ISPA_OK;
}

extern "C" int64_t ispa_kv_bytes(int64_t chunk, int32_t n_layers, uint64_t l_layer_mask, int32_t transitioned,
                                 int64_t frame_tokens, int64_t chunk_frames, int64_t d_model, int32_t elem_bytes,
                                 int64_t sink_frames) {
  if (chunk < 0 || n_layers < 0 || n_layers > 64 || frame_tokens < 0 || chunk_frames < 0 || d_model < 0 ||
      elem_bytes <= 0 || sink_frames < 0)
    return -1;
  int64_t r[6];
  if (ispa_chunk_token_ranges(chunk, frame_tokens, chunk_frames, sink_frames, r) != ISPA_OK) return -1;
  int64_t total = 0;
  for (int l = 0; l < n_layers; ++l) {
    const bool is_l = (l_layer_mask >> l) & 1u;
    const int64_t toks = (is_l && transitioned) ? (r[1] - r[0]) + (r[5] - r[4]) : r[5];
    total += toks * 2 * d_model * elem_bytes;
  }
  return total;
}

// --------------------------------------------------------------- selftest
namespace ispa {
__global__ void wait_timeout_kernel(uint64_t limit_ns, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the bounded wait must give up
    if (!mbar_wait_drain(&bar, 0, limit_ns)) report_status(status, ISPA_ERR_TIMEOUT);
  }
}
}  // namespace ispa

extern "C" ispa_status_t ispa_selftest_wait_timeout(uint32_t timeout_us, int32_t* dev_status, void* stream) {
  if (!dev_status) return invalid("dev_status is NULL");
  if (timeout_us == 0 || timeout_us > 10000000u) return invalid("timeout_us must be in (0, 10 s]");
  ispa::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)timeout_us * 1000ull,
                                                                              dev_status);
  return check_launch("wait_timeout_kernel");
}
