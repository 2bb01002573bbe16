// Standalone post-hoc fusion of two attention branches through their
// log-sum-exp states ("Instance-Specific Parametric Absorption", gist.science
// technical summary, section 2 stage 1 "Decomposable Attention").
//
//   L = logaddexp(L_loc, L_hist),  A_full = e^(L_loc-L) O_loc + e^(L_hist-L) O_hist,
//   delta = A_full - O_loc.
//
// Pure streaming work (HBM-bound): every thread moves 16-byte vectors of both
// branch outputs, grid-stride over the [n_q, D] matrices; the per-(head,row)
// weights come from the two LSE arrays, which stay in L1/L2.
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

// Each thread handles kUnroll independent 16-byte vectors per pass so that
// enough loads are in flight to cover HBM latency.
template <typename T>
__global__ void __launch_bounds__(256) lse_merge_kernel(const uint4* __restrict__ o_loc,
                                                        const float* __restrict__ lse_loc,
                                                        const uint4* __restrict__ o_hist,
                                                        const float* __restrict__ lse_hist, int64_t n_q, int D,
                                                        int head_dim, uint4* __restrict__ a_full,
                                                        uint4* __restrict__ a_delta, float* __restrict__ lse_full) {
  constexpr int N = Vec<T>::kN;
  constexpr int kUnroll = 2;
  const int vec_per_row = D / N;
  const int64_t total = n_q * vec_per_row;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e0 < total; e0 += stride * kUnroll) {
    uint4 ua[kUnroll], ub[kUnroll];
    float wl[kUnroll], wh[kUnroll], Ls[kUnroll];
    bool act[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t e = e0 + u * stride;
      act[u] = e < total;
      if (!act[u]) continue;
      ua[u] = ld_stream(o_loc + e);
      ub[u] = ld_stream(o_hist + e);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!act[u]) continue;
      const int64_t e = e0 + u * stride;
      const int64_t row = e / vec_per_row;
      const int head = (int)(e - row * vec_per_row) * N / head_dim;
      const float ll = __ldg(lse_loc + (int64_t)head * n_q + row);
      const float lh = __ldg(lse_hist + (int64_t)head * n_q + row);
      const float mx = fmaxf(ll, lh);
      Ls[u] = mx + logf(expf(ll - mx) + expf(lh - mx));
      wl[u] = expf(ll - Ls[u]);
      wh[u] = expf(lh - Ls[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!act[u]) continue;
      const int64_t e = e0 + u * stride;
      float a[N], b[N], f[N], d[N];
      unpack(ua[u], a, (T*)nullptr);
      unpack(ub[u], b, (T*)nullptr);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        f[j] = wl[u] * a[j] + wh[u] * b[j];
        d[j] = f[j] - a[j];
      }
      st_stream(a_full + e, pack(f, (T*)nullptr));
      if (a_delta) st_stream(a_delta + e, pack(d, (T*)nullptr));
      const int64_t row = e / vec_per_row;
      const int col = (int)(e - row * vec_per_row) * N;
      if (lse_full && col % head_dim == 0) lse_full[(int64_t)(col / head_dim) * n_q + row] = Ls[u];
    }
  }
}

}  // namespace merge

ispa_status_t lse_merge_launch(const void* o_loc, const float* lse_loc, const void* o_hist, const float* lse_hist,
                               int64_t n_q, int32_t n_heads, int32_t head_dim, ispa_dtype_t dt, void* a_full,
                               void* a_delta, float* lse_full, cudaStream_t stream) {
  const int D = n_heads * head_dim;
  const int N = dt == ISPA_DT_BF16 ? 8 : 4;
  const int64_t total = n_q * (D / N);
  const int64_t want = (total + 511) / 512;  // two vectors per thread
  const int cap = num_sms() * 8;
  const int blocks = (int)(want < cap ? want : cap);
  if (dt == ISPA_DT_BF16)
    merge::lse_merge_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
        (const uint4*)o_loc, lse_loc, (const uint4*)o_hist, lse_hist, n_q, D, head_dim, (uint4*)a_full,
        (uint4*)a_delta, lse_full);
  else
    merge::lse_merge_kernel<float><<<blocks, 256, 0, stream>>>((const uint4*)o_loc, lse_loc, (const uint4*)o_hist,
                                                               lse_hist, n_q, D, head_dim, (uint4*)a_full,
                                                               (uint4*)a_delta, lse_full);
  return check_launch("lse_merge_kernel");
}

}  // namespace ispa
