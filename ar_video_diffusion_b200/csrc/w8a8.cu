// e4m3 quantisation of activations and weights for the W8A8 output
// projection.  Source: "Instance-Specific Parametric Absorption", gist.science
// technical summary, section 4 "Experimental Results", item "Speedup".  ISPA
// runs with post-training W8A8 quantisation there; the page fixes no scheme.
//
// Scheme:
//   * a row of activations, or a column of W [D_in, D_out] (one output
//     channel), has scale s = amax / 448, or 1 when it is all zero;
//   * each element's code is e4m3(x / s), round to nearest even, saturating at
//     +-448;
//   * both divisions are IEEE fp32;
//   * the weight codes are written transposed, [D_out, D_in], so both operands
//     of the tensor-core product are K-major.
// Block-scaled (MX) activation codes: one power-of-two scale per 32
// consecutive elements of a row (see mx_quantize32), for the block-scaled
// tensor-core product.
// Both kernels are HBM-bound streams with 16-byte loads and stores.
#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace w8a8 {

constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f; }

__device__ __forceinline__ void bf16x8(const uint4& u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = __uint_as_float(w[e] << 16);
    x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint2 codes8(const float (&x)[8], float s) {
  uint32_t c[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) c[e] = cvt_e4m3x2(__fdiv_rn(x[2 * e], s), __fdiv_rn(x[2 * e + 1], s));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// One warp per row.  Rows of up to 2048 elements stay in registers (8
// 16-byte vectors per lane) between the amax and the codes, so each byte of x
// is read once; longer rows are read twice (the second read hits L1/L2).
// Codes go out as 8-byte pieces, consecutive lanes contiguous.
constexpr int kRegVecs = 8;

__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t n_rows,
                                                            int K, int64_t stride, uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = K / 8;
  for (int64_t row = (int64_t)blockIdx.x * 8 + warp; row < n_rows; row += (int64_t)gridDim.x * 8) {
    const uint4* src = reinterpret_cast<const uint4*>(x + row * stride);
    uint2* dst = reinterpret_cast<uint2*>(q + row * K);
    float amax = 0.f;
    if (nv <= 32 * kRegVecs) {
      uint4 buf[kRegVecs];
#pragma unroll
      for (int i = 0; i < kRegVecs; ++i) {
        const int v = lane + 32 * i;
        buf[i] = v < nv ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
        float f[8];
        bf16x8(buf[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s = scale_of(amax);
      if (lane == 0) scale[row] = s;
#pragma unroll
      for (int i = 0; i < kRegVecs; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) {
          float f[8];
          bf16x8(buf[i], f);
          dst[v] = codes8(f, s);
        }
      }
    } else {
      for (int v = lane; v < nv; v += 32) {
        float f[8];
        bf16x8(__ldg(src + v), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s = scale_of(amax);
      if (lane == 0) scale[row] = s;
      for (int v = lane; v < nv; v += 32) {
        float f[8];
        bf16x8(__ldg(src + v), f);
        dst[v] = codes8(f, s);
      }
    }
  }
}

// Column amax of W [K, N]: block = 32 columns x 8 row-slices; warp w, lane l
// walks rows w, w + 8, ... of column c0 + l, then the 8 partial maxima meet in
// shared memory.
__global__ void __launch_bounds__(256) weight_scale_kernel(const __nv_bfloat16* __restrict__ w, int K, int N,
                                                           float* __restrict__ scale) {
  __shared__ float part[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * 32 + lane;
  float amax = 0.f;
  if (col < N)
    for (int k = warp; k < K; k += 8) amax = fmaxf(amax, fabsf(__bfloat162float(w[(int64_t)k * N + col])));
  part[warp][lane] = amax;
  __syncthreads();
  if (warp == 0) {
    float m = part[0][lane];
#pragma unroll
    for (int i = 1; i < 8; ++i) m = fmaxf(m, part[i][lane]);
    if (col < N) scale[col] = scale_of(m);
  }
}

// Codes of W, transposed: a 64 (k) x 64 (n) tile is read as 16-byte row
// pieces, quantised with its column's scale, and written as qt[n, k..k+15]
// (16 bytes per thread) through a shared-memory transpose.
__global__ void __launch_bounds__(256) weight_codes_t_kernel(const __nv_bfloat16* __restrict__ w, int K, int N,
                                                             const float* __restrict__ scale,
                                                             uint8_t* __restrict__ qt) {
  __shared__ uint8_t tile[64][64 + 16];  // [n][k]
  const int k0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int t = threadIdx.x;
  // load: 64 rows (k) x 8 vectors of 8 columns
  for (int i = t; i < 64 * 8; i += 256) {
    const int kr = i >> 3, nv = i & 7;
    const int k = k0 + kr, n = n0 + nv * 8;
    uint8_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (k < K && n < N) {  // N % 16 == 0, so a vector is either wholly inside or wholly outside
      float f[8];
      bf16x8(__ldg(reinterpret_cast<const uint4*>(w + (int64_t)k * N + n)), f);
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const uint16_t p = cvt_e4m3x2(__fdiv_rn(f[e], __ldg(scale + n + e)),
                                      __fdiv_rn(f[e + 1], __ldg(scale + n + e + 1)));
        c[e] = (uint8_t)(p & 0xFF);
        c[e + 1] = (uint8_t)(p >> 8);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[nv * 8 + e][kr] = c[e];
  }
  __syncthreads();
  // store: 64 rows (n) x 4 pieces of 16 codes (k)
  const int nr = t >> 2, kp = (t & 3) * 16;
  const int n = n0 + nr, k = k0 + kp;
  if (n < N && k < K) {  // K % 16 == 0
    uint4 u;
    u.x = *reinterpret_cast<const uint32_t*>(&tile[nr][kp]);
    u.y = *reinterpret_cast<const uint32_t*>(&tile[nr][kp + 4]);
    u.z = *reinterpret_cast<const uint32_t*>(&tile[nr][kp + 8]);
    u.w = *reinterpret_cast<const uint32_t*>(&tile[nr][kp + 12]);
    *reinterpret_cast<uint4*>(qt + (int64_t)n * K + k) = u;
  }
}

// MX codes of activation rows: one thread per block of 32 consecutive
// elements of a row (64 bytes read as four 16-byte vectors, 32 code bytes
// written as two, one exponent byte), consecutive threads on consecutive
// blocks of a row, so every access of a warp is contiguous.
__global__ void __launch_bounds__(256) mx_quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t n_rows,
                                                               int K, int64_t stride, uint8_t* __restrict__ q,
                                                               uint8_t* __restrict__ e) {
  const int nb = K / 32;
  const int64_t total = n_rows * nb;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / nb;
    const int b = (int)(i - row * nb);
    const uint4* src = reinterpret_cast<const uint4*>(x + row * stride + 32 * b);
    float f[32];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      float g[8];
      bf16x8(__ldg(src + v), g);
#pragma unroll
      for (int j = 0; j < 8; ++j) f[8 * v + j] = g[j];
    }
    uint32_t c[8];
    e[i] = (uint8_t)mx_quantize32(f, c);
    uint4* dst = reinterpret_cast<uint4*>(q + row * K + 32 * b);
    dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
    dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
  }
}

}  // namespace w8a8

ispa_status_t mx_quantize_rows_e4m3(const void* x, int64_t n_rows, int64_t K, int64_t stride, uint8_t* q, uint8_t* e,
                                    cudaStream_t stream) {
  const int64_t want = (n_rows * (K / 32) + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  const int blocks = (int)(want < cap ? want : cap);
  if (blocks == 0) return ISPA_OK;
  w8a8::mx_quantize_rows_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), n_rows, (int)K,
                                                            stride, q, e);
  return check_launch("mx_quantize_rows_kernel");
}

ispa_status_t quantize_rows_e4m3(const void* x, int64_t n_rows, int64_t K, int64_t stride, uint8_t* q, float* scale,
                                 cudaStream_t stream) {
  const int64_t want = (n_rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 16;
  const int blocks = (int)(want < cap ? want : cap);
  w8a8::quantize_rows_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), n_rows, (int)K,
                                                         stride, q, scale);
  return check_launch("quantize_rows_kernel");
}

ispa_status_t quantize_weight_e4m3(const void* w, int64_t K, int64_t N, uint8_t* qt, float* scale,
                                   cudaStream_t stream) {
  const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(w);
  w8a8::weight_scale_kernel<<<(unsigned)((N + 31) / 32), 256, 0, stream>>>(wb, (int)K, (int)N, scale);
  ispa_status_t st = check_launch("weight_scale_kernel");
  if (st != ISPA_OK) return st;
  dim3 grid((unsigned)((N + 63) / 64), (unsigned)((K + 63) / 64));
  w8a8::weight_codes_t_kernel<<<grid, 256, 0, stream>>>(wb, (int)K, (int)N, scale, qt);
  return check_launch("weight_codes_t_kernel");
}

}  // namespace ispa
