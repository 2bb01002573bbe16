// Standalone post-hoc fusion of two attention branches through their
// log-sum-exp states ("Instance-Specific Parametric Absorption", gist.science
// technical summary, section 2 stage 1 "Decomposable Attention").
//
//   L = logaddexp(L_loc, L_hist),  A_full = e^(L_loc-L) O_loc + e^(L_hist-L) O_hist,
//   delta = A_full - O_loc.
//
// Pure streaming work (HBM-bound): blocks of whole rows, 16-byte vectors of
// both branch outputs, the per-(row, head) weights computed once per block.
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace merge {

template <typename T>
struct Vec;  // 16 bytes of T
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
};
template <>
struct Vec<float> {
  static constexpr int kN = 4;
};

__device__ __forceinline__ void unpack(const uint4& u, float (&x)[8], __nv_bfloat16*) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = __uint_as_float(w[e] << 16);
    x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack(const float (&x)[8], __nv_bfloat16*) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}
__device__ __forceinline__ void unpack(const uint4& u, float (&x)[4], float*) {
  x[0] = __uint_as_float(u.x);
  x[1] = __uint_as_float(u.y);
  x[2] = __uint_as_float(u.z);
  x[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ uint4 pack(const float (&x)[4], float*) {
  return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

constexpr int kRowsPerBlock = 4;
constexpr int kMaxHeads = 64;

// One block fuses kRowsPerBlock whole rows.  The per-(row, head) weights
// e^(L_loc - L), e^(L_hist - L) and L are computed once into shared memory
// (and L written out); the block then streams the rows' 16-byte vectors with
// packed fp32 math, so the per-vector work stays within the instruction
// budget of an HBM-bound stream.
template <typename T>
__global__ void __launch_bounds__(256) lse_merge_kernel(const uint4* __restrict__ o_loc,
                                                        const float* __restrict__ lse_loc,
                                                        const uint4* __restrict__ o_hist,
                                                        const float* __restrict__ lse_hist, int64_t n_q, int D,
                                                        int head_dim, int n_heads, uint4* __restrict__ a_full,
                                                        uint4* __restrict__ a_delta, float* __restrict__ lse_full) {
  constexpr int N = Vec<T>::kN;
  __shared__ float2 wts[kRowsPerBlock][kMaxHeads];
  const int vec_per_row = D / N;
  const int vec_per_head = head_dim / N;
  for (int64_t r0 = (int64_t)blockIdx.x * kRowsPerBlock; r0 < n_q; r0 += (int64_t)gridDim.x * kRowsPerBlock) {
    const int rows = n_q - r0 < kRowsPerBlock ? (int)(n_q - r0) : kRowsPerBlock;
    for (int t = threadIdx.x; t < rows * n_heads; t += blockDim.x) {
      const int rr = t / n_heads, h = t - rr * n_heads;
      const int64_t li = (int64_t)h * n_q + r0 + rr;
      const float ll = __ldg(lse_loc + li), lh = __ldg(lse_hist + li);
      const float mx = fmaxf(ll, lh);
      // both branches empty: the union is empty too, so A_full = 0 and
      // L = -inf (attention over no keys), with both weights 0
      const bool none = mx == -INFINITY;
      const float L = none ? -INFINITY : mx + logf(expf(ll - mx) + expf(lh - mx));
      wts[rr][h] = none ? make_float2(0.f, 0.f) : make_float2(expf(ll - L), expf(lh - L));
      if (lse_full) lse_full[li] = L;
    }
    __syncthreads();
    const int nvec = rows * vec_per_row;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      const int rr = v / vec_per_row;
      const int h = (v - rr * vec_per_row) / vec_per_head;
      const int64_t e = (r0 + rr) * vec_per_row + (v - rr * vec_per_row);
      const uint4 ua = ld_stream(o_loc + e), ub = ld_stream(o_hist + e);
      const float2 w = wts[rr][h];
      float a[N], b[N], f[N], d[N];
      unpack(ua, a, (T*)nullptr);
      unpack(ub, b, (T*)nullptr);
#pragma unroll
      for (int j = 0; j < N; j += 2) {
        const float2 fa = ffma2(make_float2(a[j], a[j + 1]), make_float2(w.x, w.x),
                                make_float2(b[j] * w.y, b[j + 1] * w.y));
        const float2 da = fadd2(fa, make_float2(-a[j], -a[j + 1]));
        f[j] = fa.x;
        f[j + 1] = fa.y;
        d[j] = da.x;
        d[j + 1] = da.y;
      }
      st_stream(a_full + e, pack(f, (T*)nullptr));
      if (a_delta) st_stream(a_delta + e, pack(d, (T*)nullptr));
    }
    __syncthreads();
  }
}

}  // namespace merge

ispa_status_t lse_merge_launch(const void* o_loc, const float* lse_loc, const void* o_hist, const float* lse_hist,
                               int64_t n_q, int32_t n_heads, int32_t head_dim, ispa_dtype_t dt, void* a_full,
                               void* a_delta, float* lse_full, cudaStream_t stream) {
  const int D = n_heads * head_dim;
  const int64_t row_blocks = (n_q + merge::kRowsPerBlock - 1) / merge::kRowsPerBlock;
  const int64_t cap = (int64_t)num_sms() * 8;
  const int blocks = (int)(row_blocks < cap ? row_blocks : cap);
  if (dt == ISPA_DT_BF16)
    merge::lse_merge_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
        (const uint4*)o_loc, lse_loc, (const uint4*)o_hist, lse_hist, n_q, D, head_dim, n_heads, (uint4*)a_full,
        (uint4*)a_delta, lse_full);
  else
    merge::lse_merge_kernel<float><<<blocks, 256, 0, stream>>>((const uint4*)o_loc, lse_loc, (const uint4*)o_hist,
                                                               lse_hist, n_q, D, head_dim, n_heads, (uint4*)a_full,
                                                               (uint4*)a_delta, lse_full);
  return check_launch("lse_merge_kernel");
}

}  // namespace ispa
