// fp32 Decomposable Attention on the CUDA cores (activations stored as fp32).
//
// Same outputs as the tensor-core kernel: a local branch and a historical
// branch, each an online softmax that keeps its log-sum-exp, fused post hoc
// ("Instance-Specific Parametric Absorption", gist.science technical summary,
// section 2 stage 1 and section 3 item 2).  One warp owns one (query row,
// head); lanes split the head dimension, scores are reduced with warp
// shuffles.  Meant for fp32 workloads, where rounding the operands to bf16
// would cost about 1e-3 of log-sum-exp accuracy.
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace attn32 {

constexpr int kMaxSeg = ISPA_MAX_SEGMENTS;
constexpr int kWarps = 4;

struct Seg {
  const float* k;
  const float* v;
  int64_t n;
  int64_t stride;
};

struct Params {
  Seg seg[kMaxSeg];
  int n_local_seg, n_seg;
  const float* q;
  int64_t q_stride, n_q;
  int n_heads;
  float scale;
  float* a_loc;
  float* a_full;
  float* a_delta;
  float* lse_loc;
  float* lse_full;
  int64_t out_stride;
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Online softmax of one row over segments [s0, s1).  o holds HD/32 channels per
// lane (channel lane + 32 j).  Returns through m (running max of the scaled
// scores) and l (sum of exp(s - m)); o is left unnormalised.
template <int HD>
__device__ void branch(const Params& p, int s0, int s1, const float (&q)[HD / 32], int head, float& m, float& l,
                       float (&o)[HD / 32]) {
  const int lane = threadIdx.x & 31;
  m = -INFINITY;
  l = 0.f;
#pragma unroll
  for (int j = 0; j < HD / 32; ++j) o[j] = 0.f;
  for (int s = s0; s < s1; ++s) {
    const Seg sg = p.seg[s];
    for (int64_t t = 0; t < sg.n; ++t) {
      const float* kr = sg.k + t * sg.stride + head * HD;
      float part = 0.f;
#pragma unroll
      for (int j = 0; j < HD / 32; ++j) part = fmaf(q[j], kr[lane + 32 * j], part);
      const float sc = warp_sum(part) * p.scale;
      const float m_new = fmaxf(m, sc);
      const float f = expf(m - m_new);
      const float e = expf(sc - m_new);
      l = l * f + e;
      const float* vr = sg.v + t * sg.stride + head * HD;
#pragma unroll
      for (int j = 0; j < HD / 32; ++j) o[j] = fmaf(e, vr[lane + 32 * j], o[j] * f);
      m = m_new;
    }
  }
}

template <int HD>
__global__ void __launch_bounds__(32 * kWarps) attention_f32_kernel(const Params p) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (item >= p.n_q * p.n_heads) return;
  const int head = (int)(item % p.n_heads);
  const int64_t row = item / p.n_heads;
  float q[HD / 32];
#pragma unroll
  for (int j = 0; j < HD / 32; ++j) q[j] = p.q[row * p.q_stride + head * HD + lane + 32 * j];
  const int64_t ob = row * p.out_stride + head * HD;
  const int64_t li = (int64_t)head * p.n_q + row;
  if (p.a_loc) {  // dual mode
    float mL, lL, oL[HD / 32], mH, lH, oH[HD / 32];
    branch<HD>(p, 0, p.n_local_seg, q, head, mL, lL, oL);
    branch<HD>(p, p.n_local_seg, p.n_seg, q, head, mH, lH, oH);
    const float lse_l = mL + logf(lL);
    float w = 0.f, lse_f = lse_l;
    if (lH > 0.f) {
      const float lse_h = mH + logf(lH);
      const float mm = fmaxf(lse_l, lse_h);
      lse_f = mm + logf(expf(lse_l - mm) + expf(lse_h - mm));
      w = expf(lse_h - lse_f);
    }
#pragma unroll
    for (int j = 0; j < HD / 32; ++j) {
      const float a = oL[j] / lL;
      const float d = lH > 0.f ? w * (oH[j] / lH - a) : 0.f;
      p.a_loc[ob + lane + 32 * j] = a;
      p.a_full[ob + lane + 32 * j] = a + d;
      if (p.a_delta) p.a_delta[ob + lane + 32 * j] = d;
    }
    if (lane == 0) {
      if (p.lse_loc) p.lse_loc[li] = lse_l;
      if (p.lse_full) p.lse_full[li] = lse_f;
    }
  } else {
    float m, l, o[HD / 32];
    branch<HD>(p, 0, p.n_seg, q, head, m, l, o);
#pragma unroll
    for (int j = 0; j < HD / 32; ++j) p.a_full[ob + lane + 32 * j] = o[j] / l;
    if (lane == 0 && p.lse_full) p.lse_full[li] = m + logf(l);
  }
}

}  // namespace attn32

ispa_status_t dual_attention_f32(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim,
                                 float scale, const ispa_kv_segment_t* segs, int n_local_seg, int n_hist_seg,
                                 void* a_loc, void* a_full, void* a_delta, float* lse_loc, float* lse_full,
                                 cudaStream_t stream) {
  using namespace attn32;
  Params p{};
  p.n_local_seg = n_local_seg;
  p.n_seg = n_local_seg + n_hist_seg;
  for (int i = 0; i < p.n_seg; ++i)
    p.seg[i] = Seg{static_cast<const float*>(segs[i].k), static_cast<const float*>(segs[i].v), segs[i].n_tokens,
                   segs[i].row_stride};
  p.q = static_cast<const float*>(q);
  p.q_stride = q_stride;
  p.n_q = n_q;
  p.n_heads = n_heads;
  p.scale = scale;
  p.a_loc = static_cast<float*>(a_loc);
  p.a_full = static_cast<float*>(a_full);
  p.a_delta = static_cast<float*>(a_delta);
  p.lse_loc = lse_loc;
  p.lse_full = lse_full;
  p.out_stride = (int64_t)n_heads * head_dim;
  const int64_t items = n_q * n_heads;
  const unsigned blocks = (unsigned)((items + kWarps - 1) / kWarps);
  if (head_dim == 128)
    attention_f32_kernel<128><<<blocks, 32 * kWarps, 0, stream>>>(p);
  else
    attention_f32_kernel<64><<<blocks, 32 * kWarps, 0, stream>>>(p);
  return check_launch("attention_f32_kernel");
}

}  // namespace ispa
