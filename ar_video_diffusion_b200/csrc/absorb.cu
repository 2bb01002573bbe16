// Layer Absorb: the closed-form ridge solve
//   dW = (G + lambda I)^-1 R W,   lambda = lambda_abs + lambda_rel tr(G) / D,
// ("Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", gist.science technical summary,
// section 2 stage 2 "Layer Absorb"), then W_new = W + dW (stage 3).
//
// All on the device, stream ordered, in two forms.
// Tensor-core form (bf16 W, D a multiple of 128, D >= 256):
//   1. S = R W on the tensor cores as hi(R) W + lo(R) W (W is exactly bf16);
//   2. trace(G) -> lambda (one block, fp64 sum);  M = G + lambda I;
//   3. right-looking blocked Cholesky M = L L^T with 64-wide panels, the
//      right-hand sides [S | I] carried along: per panel the diagonal block
//      is factored (and its factor inverted) by one CTA, the panel below and
//      the panel's rows of the right-hand sides are multiplied by that
//      inverse, and one split-precision tensor-core product updates the
//      trailing lower triangle from the second column block on and the
//      remaining right-hand-side rows; the first trailing column block is
//      updated by the next diagonal step itself, so the chain of diagonal
//      steps runs on a second stream beside the panels and products;
//   4. dW = (L^-1)^T (L^-1 S), one split-precision tensor-core product;
//   5. W_new = W + dW, rounded to W's dtype.
// Compact form (every other case, and the no-allocation entry point): the
// same factorisation with fp32 CUDA-core updates and blocked triangular
// solves L Y = S, L^T X = Y.  Its fp32 GEMM (also the fp32 activation path of
// the statistics and the projection) is a 64 x 64-tile CUDA-core kernel with
// arbitrary strides, so transposed operands are read in place.
#include <cudaTypedefs.h>

#include <cstring>
#include <vector>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace simt {

constexpr int kT = 64;   // tile edge
constexpr int kTK = 16;  // K slice per shared-memory stage

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// C[m, n] = beta * C[m, n] + alpha * sum_k A(m, k) B(k, n) with
// A(m, k) = A[m * a_rs + k * a_cs], B(k, n) = B[k * b_rs + n * b_cs].
// lower_only: tiles strictly above the block diagonal are skipped.
template <typename TA, typename TB>
__global__ void __launch_bounds__(256) gemm_f32_kernel(int M, int N, int K, float alpha, const TA* __restrict__ A,
                                                       int64_t a_rs, int64_t a_cs, const TB* __restrict__ B,
                                                       int64_t b_rs, int64_t b_cs, float beta, float* C,
                                                       int64_t ldc, int lower_only) {
  const int tm = blockIdx.y, tn = blockIdx.x;
  if (lower_only && tn > tm) return;
  __shared__ float As[kTK][kT + 4];
  __shared__ float Bs[kTK][kT + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = tm * kT, n0 = tn * kT;
  float acc[4][4] = {};
  const bool a_k_fast = a_cs == 1;
  const bool b_n_fast = b_cs == 1;
  for (int k0 = 0; k0 < K; k0 += kTK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i;
      int mm, kk;
      if (a_k_fast) {
        kk = idx % kTK;
        mm = idx / kTK;
      } else {
        mm = idx % kT;
        kk = idx / kT;
      }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? to_f32(A[gm * a_rs + gk * a_cs]) : 0.f;
      int nn, kb;
      if (b_n_fast) {
        nn = idx % kT;
        kb = idx / kT;
      } else {
        kb = idx % kTK;
        nn = idx / kTK;
      }
      const int gn = n0 + nn, gkb = k0 + kb;
      Bs[kb][nn] = (gn < N && gkb < K) ? to_f32(B[gkb * b_rs + gn * b_cs]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      float* c = C + gm * ldc + gn;
      *c = (beta == 0.f ? 0.f : beta * *c) + alpha * acc[i][j];
    }
  }
}

template <typename TA, typename TB>
void gemm_f32(cudaStream_t st, int M, int N, int K, float alpha, const TA* A, int64_t a_rs, int64_t a_cs, const TB* B,
              int64_t b_rs, int64_t b_cs, float beta, float* C, int64_t ldc, bool lower_only = false) {
  if (M <= 0 || N <= 0) return;
  dim3 grid((N + kT - 1) / kT, (M + kT - 1) / kT);
  gemm_f32_kernel<TA, TB><<<grid, 256, 0, st>>>(M, N, K, alpha, A, a_rs, a_cs, B, b_rs, b_cs, beta, C, ldc,
                                                lower_only ? 1 : 0);
}

// ---------------------------------------------------------------- absorb
__global__ void trace_lambda_kernel(const float* __restrict__ G, int D, double lam_abs, double lam_rel,
                                    double* __restrict__ lam_out) {
  __shared__ double part[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < D; i += blockDim.x) s += (double)G[(int64_t)i * D + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *lam_out = lam_abs + lam_rel * part[0] / D;
}

__global__ void shift_kernel(const float* __restrict__ G, float* __restrict__ M, int D,
                             const double* __restrict__ lam) {
  const float l = (float)*lam;
  const int64_t total = (int64_t)D * D / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    float4 g = reinterpret_cast<const float4*>(G)[e];
    const int64_t i = (e * 4) / D, j0 = (e * 4) % D;
    const int64_t off = i - j0;  // position of the diagonal inside this float4, if any
    g.x += off == 0 ? l : 0.f;
    g.y += off == 1 ? l : 0.f;
    g.z += off == 2 ? l : 0.f;
    g.w += off == 3 ? l : 0.f;
    reinterpret_cast<float4*>(M)[e] = g;
  }
}

// Factor the 64 x 64 diagonal block k of M in place (lower triangle) and
// write the inverse of its Cholesky factor to Linv (64 x 64, row-major).
// Blocked by 16: each 16 x 16 diagonal block is factored by one warp in
// registers (a row per lane, pivots and columns exchanged with shuffles) and
// inverted column by column by the same warp; the CTA then forms the 16-column
// panel below, L_ik = A_ik L_kk^-T, and the rank-16 update of the trailing
// lower triangle from shared memory.  The off-diagonal blocks of L^-1 follow
// from X_ik = -X_ii sum_{j=k}^{i-1} L_ij X_jk, one block diagonal at a time.
// A pivot <= 0 or non-finite records ISPA_ERR_NOT_SPD and its row; the
// factorisation then continues with the pivot replaced by 1.
constexpr int kSub = 16;

__global__ void __launch_bounds__(256) potrf_diag_kernel(float* M, int D, int k, float* Linv, int32_t* status) {
  __shared__ float A[kT][kT + 1];  // the block, then L (lower triangle)
  __shared__ float X[kT][kT + 1];  // L^-1 (lower triangle, zero above)
  __shared__ float T[3][kSub][kSub + 1];
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* blk = M + (int64_t)k * kT * D + (int64_t)k * kT;
  for (int e = tid; e < kT * kT; e += 256) {
    const int i = e >> 6, j = e & 63;
    A[i][j] = blk[(int64_t)i * D + j];
    X[i][j] = 0.f;
  }
  if (tid == 0) bad = -1;
  __syncthreads();
#pragma unroll 1
  for (int kb = 0; kb < kT / kSub; ++kb) {
    const int o = kSub * kb;
    if (warp == 0) {
      // (a) factor the diagonal block: lane r (and r + 16, a duplicate) holds row r
      const int r = lane & (kSub - 1);
      float a[kSub];
#pragma unroll
      for (int c = 0; c < kSub; ++c) a[c] = (c <= r) ? A[o + r][o + c] : 0.f;
#pragma unroll
      for (int j = 0; j < kSub; ++j) {
        float d = __shfl_sync(0xffffffffu, a[j], j);
        if (!(d > 0.f) || !isfinite(d)) {
          if (lane == 0 && bad < 0) bad = o + j;
          d = 1.f;
        }
        const float ljj = sqrtf(d);
        const float inv = 1.0f / ljj;
        a[j] = (r == j) ? ljj : (r > j ? a[j] * inv : 0.f);
#pragma unroll
        for (int c = 1; c < kSub; ++c) {  // constant trip count: every index stays static
          if (c > j) {
            const float lcj = __shfl_sync(0xffffffffu, a[j], c);  // L[c][j], held by lane c
            if (r >= c) a[c] -= a[j] * lcj;
          }
        }
      }
      if (lane < kSub) {
#pragma unroll
        for (int c = 0; c < kSub; ++c)
          if (c <= r) A[o + r][o + c] = a[c];
      }
      __syncwarp();
      // its inverse: lane c solves L x = e_c by forward substitution
      if (lane < kSub) {
        const int c = lane;
        float x[kSub];
#pragma unroll
        for (int rr = 0; rr < kSub; ++rr) {
          float acc = (rr == c) ? 1.f : 0.f;
#pragma unroll
          for (int m = 0; m < rr; ++m) acc -= A[o + rr][o + m] * x[m];
          x[rr] = (rr < c) ? 0.f : acc / A[o + rr][o + rr];
        }
#pragma unroll
        for (int rr = 0; rr < kSub; ++rr)
          if (rr >= c) X[o + rr][o + c] = x[rr];
      }
    }
    __syncthreads();
    // (b) panel: L[i][o + c] = sum_{m <= c} A[i][o + m] X[o + c][o + m] for rows i below the block
    const int rows = kT - o - kSub;
    float pv[3];  // at most 48 x 16 panel entries over 256 threads
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int e = tid + 256 * q;
      pv[q] = 0.f;
      if (e < rows * kSub) {
        const int i = o + kSub + e / kSub, c = e % kSub;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < kSub; ++m)
          if (m <= c) acc += A[i][o + m] * X[o + c][o + m];
        pv[q] = acc;
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int e = tid + 256 * q;
      if (e < rows * kSub) A[o + kSub + e / kSub][o + e % kSub] = pv[q];
    }
    __syncthreads();
    // (c) trailing lower triangle: A[i][j] -= sum_c L[i][o + c] L[j][o + c], o + 16 <= j <= i
    for (int e = tid; e < rows * rows; e += 256) {
      const int i = o + kSub + e / rows, j = o + kSub + e % rows;
      if (j > i) continue;
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < kSub; ++c) acc += A[i][o + c] * A[j][o + c];
      A[i][j] -= acc;
    }
    __syncthreads();
  }
  // (d) off-diagonal blocks of X = L^-1, by block distance dd = ib - jb
#pragma unroll 1
  for (int dd = 1; dd < kT / kSub; ++dd) {
    const int nblk = kT / kSub - dd;
    // T_b = sum_{jb <= m < ib} L[ib][m] X[m][jb]  (16 x 16 each, blocks b = 0..nblk-1)
    for (int e = tid; e < nblk * kSub * kSub; e += 256) {
      const int b = e / (kSub * kSub), rr = (e / kSub) % kSub, cc = e % kSub;
      const int ib = b + dd, jb = b;
      float acc = 0.f;
      for (int m = kSub * jb; m < kSub * ib; ++m) acc += A[kSub * ib + rr][m] * X[m][kSub * jb + cc];
      T[b][rr][cc] = acc;
    }
    __syncthreads();
    // X[ib][jb] = -X[ib][ib] T_b
    for (int e = tid; e < nblk * kSub * kSub; e += 256) {
      const int b = e / (kSub * kSub), rr = (e / kSub) % kSub, cc = e % kSub;
      const int ib = b + dd, jb = b;
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < kSub; ++m)
        if (m <= rr) acc += X[kSub * ib + rr][kSub * ib + m] * T[b][m][cc];
      X[kSub * ib + rr][kSub * jb + cc] = -acc;
    }
    __syncthreads();
  }
  if (tid == 0 && bad >= 0 && status) {
    if (atomicCAS(status, 0, (int32_t)ISPA_ERR_NOT_SPD) == 0) status[1] = k * kT + bad;
  }
  for (int e = tid; e < kT * kT; e += 256) {
    const int i = e >> 6, j = e & 63;
    if (j <= i) blk[(int64_t)i * D + j] = A[i][j];
    Linv[i * kT + j] = X[i][j];
  }
}

// 64 x 64 x 64 product out = P Q (with P or Q read transposed), register
// tiled: thread (ty, tx) of 16 x 16 owns rows ty + 16 a, columns tx + 16 b.
// pt: P is given transposed (P(i, t) = Ps[t][i]); qt: Q(t, c) = Qs[c][t].
__device__ __forceinline__ void mm64(const float (*Ps)[kT + 1], const float (*Qs)[kT + 1], bool pt, bool qt,
                                     float (&acc)[4][4]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
  for (int t = 0; t < kT; ++t) {
    float pa[4], qb[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) pa[a] = pt ? Ps[t][ty + 16 * a] : Ps[ty + 16 * a][t];
#pragma unroll
    for (int b = 0; b < 4; ++b) qb[b] = qt ? Qs[tx + 16 * b][t] : Qs[t][tx + 16 * b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(pa[a], qb[b], acc[a][b]);
  }
}

// 64 x 64 operands stored with the contraction index first (row stride
// kLdv, rows 16-byte aligned): acc[a][b] = sum_t P[t][4 ty + a] Q[t][4 tx + b].
// Per t a warp reads one 16-byte vector of P (two addresses, one wavefront)
// and sixteen of Q (256 contiguous bytes, two wavefronts), against eight
// scalar wavefronts in mm64.
constexpr int kLdv = kT + 4;
__device__ __forceinline__ void mm64v(const float (*P)[kLdv], const float (*Q)[kLdv], float (&acc)[4][4]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
  for (int t = 0; t < kT; ++t) {
    const float4 pv = *reinterpret_cast<const float4*>(&P[t][4 * ty]);
    const float4 qv = *reinterpret_cast<const float4*>(&Q[t][4 * tx]);
    const float pa[4] = {pv.x, pv.y, pv.z, pv.w}, qb[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(pa[a], qb[b], acc[a][b]);
  }
}

// 64 x 64 block of a row-major fp32 matrix (row stride ld, 16-byte aligned
// rows) into shared memory as it is (S[i][j] = G[i][j]) or transposed
// (S[j][i] = G[i][j]; consecutive threads take consecutive rows, so the
// scalar stores hit distinct banks)
__device__ __forceinline__ void load_n64(float (*S)[kLdv], const float* __restrict__ G, int64_t ld) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = threadIdx.x + 256 * q, i = e >> 4, j = (e & 15) * 4;
    *reinterpret_cast<float4*>(&S[i][j]) = *reinterpret_cast<const float4*>(G + (int64_t)i * ld + j);
  }
}
__device__ __forceinline__ void load_t64(float (*S)[kLdv], const float* __restrict__ G, int64_t ld) {
  float4 v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = threadIdx.x + 256 * q, i = e & 63, j = (e >> 6) * 4;
    v[q] = *reinterpret_cast<const float4*>(G + (int64_t)i * ld + j);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = threadIdx.x + 256 * q, i = e & 63, j = (e >> 6) * 4;
    S[j][i] = v[q].x, S[j + 1][i] = v[q].y, S[j + 2][i] = v[q].z, S[j + 3][i] = v[q].w;
  }
}

// Panel below diagonal block k: M[r, k] <- M[r, k] Linv_k^T, one 64-row block per CTA.
__global__ void __launch_bounds__(256) panel_kernel(float* M, int D, int k, const float* __restrict__ Linv) {
  __shared__ float Li[kT][kT + 1];
  __shared__ float P[kT][kT + 1];
  const int r = k + 1 + blockIdx.x;
  float* blk = M + (int64_t)r * kT * D + (int64_t)k * kT;
  for (int e = threadIdx.x; e < kT * kT; e += 256) {
    Li[e / kT][e % kT] = Linv[e];
    P[e / kT][e % kT] = blk[(int64_t)(e / kT) * D + e % kT];
  }
  __syncthreads();
  float acc[4][4];
  mm64(P, Li, false, true, acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) blk[(int64_t)(ty + 16 * a) * D + tx + 16 * b] = acc[a][b];
}

// X[k-block rows, :] <- Linv_k X  (transpose_l = 0) or Linv_k^T X (1), in place;
// one 64-column slab per CTA.
__global__ void __launch_bounds__(256) diag_apply_kernel(float* X, int D, int k, const float* __restrict__ Linv,
                                                         int transpose_l) {
  __shared__ float Li[kT][kT + 1];
  __shared__ float T[kT][kT + 1];
  float* blk = X + (int64_t)k * kT * D + (int64_t)blockIdx.x * kT;
  for (int e = threadIdx.x; e < kT * kT; e += 256) {
    Li[e / kT][e % kT] = Linv[e];
    T[e / kT][e % kT] = blk[(int64_t)(e / kT) * D + e % kT];
  }
  __syncthreads();
  float acc[4][4];
  mm64(Li, T, transpose_l != 0, false, acc);
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) blk[(int64_t)(ty + 16 * a) * D + tx + 16 * b] = acc[a][b];
}

// R (fp32) -> hi = bf16(R), lo = bf16(R - hi): R = hi + lo to about 2^-16 relative.
__global__ void split_bf16_kernel(const float* __restrict__ R, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float v = R[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

template <typename TW>
__global__ void wnew_kernel(const TW* __restrict__ W, const float* __restrict__ dW, TW* __restrict__ Wn, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float v = to_f32(W[e]) + dW[e];
    if constexpr (sizeof(TW) == 2)
      Wn[e] = __float2bfloat16_rn(v);
    else
      Wn[e] = v;
  }
}

}  // namespace simt

// ------------------------------------------- tensor-core form of the solve
// For bf16 W and D a multiple of 128 (D >= 256) the solve runs its products on
// the tensor cores in split precision (hi/lo bf16 pairs, about 2^-17 relative
// per product), with the right-hand sides carried through the factorisation:
//   RHS = [S | I] (D x 2D) with S = R W;
//   for each 64-wide panel k (right-looking):
//     factor the diagonal block and invert its factor (one CTA), after
//     applying panel k - 1 to column block k (the other CTAs of that step);
//     L21 = A21 L_kk^-T for the rows below, and Y_k = L_kk^-1 RHS_k for the
//     panel's rows of the right-hand sides (final rows of L^-1 S and L^-1);
//     one tensor-core update [M22 | RHS_2] -= L21 [L21^T | Y_k], without
//     M22's first column block;
//   after the last panel RHS = [L^-1 S | L^-1], and
//   dW = (L^-1)^T (L^-1 S) = (G + lambda I)^-1 S is one tensor-core product
//   whose A operand (L^-1)^T is upper triangular.
namespace simt {

// 32 x 32 Cholesky factor of a lower triangle in shared memory (row stride
// ld), by one warp.  Lane r holds row r in registers with the columns rotated
// (a[0] is the current column), so the loop body is short and its register
// indices static, and the loop stays rolled (an unrolled factorisation run
// once by one warp is bound by instruction fetch).  Column j of L goes to the
// lower triangle of A and, shifted, to row j of Ls (Ls[j][c] = L[j + c][j],
// zero beyond the matrix), read back as eight 16-byte vectors for the update
// of the remaining columns.  The next pivot does not wait for that round
// trip: lane j + 1 updates its own diagonal entry with its own l and passes it
// on with one shuffle, so the chain per column is shuffle, reciprocal square
// root, two multiply-adds.  rinv[j] = 1 / L[j][j].  A pivot <= 0 or
// non-finite is replaced by 1 and its index (first only) recorded.
__device__ __forceinline__ void chol32_rot(float* A, int ld, float (*Ls)[32], float* rinv, int lane, int base,
                                           int* bad) {
  float a[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) a[c] = c <= lane ? A[lane * ld + c] : 0.f;
  float d = __shfl_sync(0xffffffffu, a[0], 0);
#pragma unroll 1
  for (int j = 0; j < 32; ++j) {
    if (!(d > 0.f) || !isfinite(d)) {
      if (lane == 0 && *bad < 0) *bad = base + j;
      d = 1.f;
    }
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));  // d > 0 and finite here
    const float l = lane == j ? d * r : (lane > j ? a[0] * r : 0.f);
    // the next pivot: lane j + 1's entry (j + 1, j + 1) less its own l squared
    const float dn = __shfl_sync(0xffffffffu, a[1] - l * l, (j + 1) & 31);
    if (lane >= j) A[lane * ld + j] = l;
    if (lane == 0) rinv[j] = r;
    Ls[j][(lane - j) & 31] = lane >= j ? l : 0.f;  // lanes < j zero the tail
    __syncwarp();
    const float4* col = reinterpret_cast<const float4*>(Ls[j]);
    float lk[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v = col[q];
      lk[4 * q] = v.x, lk[4 * q + 1] = v.y, lk[4 * q + 2] = v.z, lk[4 * q + 3] = v.w;
    }
    // a[c] holds column j + c: subtract l * L[j + c][j]
#pragma unroll
    for (int c = 1; c < 32; ++c) a[c - 1] = a[c] - l * lk[c];
    a[31] = 0.f;
    d = dn;
  }
}

// Forward elimination x = L^-1 b for the 32 x 32 lower-triangular L whose
// columns chol32_rot left shifted in Ls (rinv: reciprocals of its diagonal),
// by one warp with one right-hand side per lane, rotated in registers
// (b[0] is the current row); x[m] goes to out[m * s_m + lane * s_l].  The
// column for step m + 1 is loaded while step m runs, so a step's chain is
// one multiply and one multiply-add.
__device__ __forceinline__ void trsv32_rot(const float (*Ls)[32], const float* rinv, float (&b)[32], float* out,
                                           int s_m, int s_l, int lane, float* out_t = nullptr, int t_ld = 0) {
  float4 nx[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) nx[q] = reinterpret_cast<const float4*>(Ls[0])[q];
  float rn = rinv[0];
#pragma unroll 1
  for (int m = 0; m < 32; ++m) {
    float lr[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) lr[4 * q] = nx[q].x, lr[4 * q + 1] = nx[q].y, lr[4 * q + 2] = nx[q].z, lr[4 * q + 3] = nx[q].w;
    const float rm = rn;
    const float4* nxt = reinterpret_cast<const float4*>(Ls[(m + 1) & 31]);  // wraps harmlessly after the last
#pragma unroll
    for (int q = 0; q < 8; ++q) nx[q] = nxt[q];
    rn = rinv[(m + 1) & 31];
    const float x = b[0] * rm;
    out[m * s_m + lane * s_l] = x;
    if (out_t) out_t[m * t_ld + lane] = x;  // the same value, x[m] of lane at [m][lane]
#pragma unroll
    for (int c = 1; c < 32; ++c) b[c - 1] = b[c] - lr[c] * x;
    b[31] = 0.f;
  }
}

// Cholesky factor of the 64 x 64 block in A (shared, row stride 65; lower
// triangle used) and the inverse X of that factor (shared, row stride 65),
// by the 256 threads of a CTA:
//   L11 = chol(A11) by warp 0;
//   then at once X11 = L11^-1 (warp 0) and L21 = A21 L11^-T (warp 1, a row
//   of A21 per lane, solved in place and also stored transposed in Lt);
//   A22 - L21 L21^T (all, from Lt);
//   then at once L22 = chol(.) (warp 0) and T = L21 X11 (warps 1, 2, 3 and
//   5, which leave warp 0's scheduler to it);
//   X22 = L22^-1 (warp 0); X21 = -X22 T (all).
// The 32 x 32 products read two-element vectors of an operand stored with
// the contraction index first.  T, Lt: 32 x 36 scratch (8-byte aligned
// rows); Ls: 32 x 32, 16-byte aligned; rinv: 32 floats.
__device__ void factor_diag64(float (*A)[65], float (*X)[65], float (*T)[36], float (*Lt)[36], float (*Ls)[32],
                              float* rinv, int* bad, int base) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ti = tid >> 4, tj = tid & 15;  // a 2 x 2 block of a 32 x 32 product
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // the upper right quarter of X is zero
    const int e = tid + 256 * q;
    X[e >> 5][32 + (e & 31)] = 0.f;
  }
  if (warp == 0) chol32_rot(&A[0][0], 65, Ls, rinv, lane, base, bad);
  __syncthreads();
  if (warp < 2) {
    float b[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) b[c] = warp == 0 ? (c == lane ? 1.f : 0.f) : A[32 + lane][c];
    if (warp == 0)
      trsv32_rot(Ls, rinv, b, &X[0][0], 65, 1, lane);  // column `lane` of X11
    else
      trsv32_rot(Ls, rinv, b, &A[32][0], 1, 65, lane, &Lt[0][0], 36);  // row `lane` of L21
  }
  __syncthreads();
  {  // A22 -= L21 L21^T: rows 2 ti + a, columns 2 tj + c
    float v[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
      const float2 p = *reinterpret_cast<const float2*>(&Lt[m][2 * ti]);
      const float2 q = *reinterpret_cast<const float2*>(&Lt[m][2 * tj]);
      v[0][0] = fmaf(p.x, q.x, v[0][0]), v[0][1] = fmaf(p.x, q.y, v[0][1]);
      v[1][0] = fmaf(p.y, q.x, v[1][0]), v[1][1] = fmaf(p.y, q.y, v[1][1]);
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 2; ++c) A[32 + 2 * ti + a][32 + 2 * tj + c] -= v[a][c];
  }
  __syncthreads();
  if (warp == 0) {
    chol32_rot(&A[32][32], 65, Ls, rinv, lane, base + 32, bad);
    __syncwarp();
    float b[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) b[c] = c == lane ? 1.f : 0.f;
    trsv32_rot(Ls, rinv, b, &X[32][32], 65, 1, lane);
  } else if (warp <= 3 || warp == 5) {  // T = L21 X11: 128 threads, rows 2 ui + a, columns uj + 4 c
    const int u = (warp <= 3 ? warp - 1 : 3) * 32 + lane;
    const int ui = u >> 3, uj = u & 7;  // ui < 16
    float v[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int m = 0; m < 32; ++m) {
      const float2 p = *reinterpret_cast<const float2*>(&Lt[m][2 * ui]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float x = X[m][uj + 8 * c];
        v[0][c] = fmaf(p.x, x, v[0][c]);
        v[1][c] = fmaf(p.y, x, v[1][c]);
      }
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) T[2 * ui + a][uj + 8 * c] = v[a][c];
  }
  __syncthreads();
  {  // X21 = -X22 T: rows ti and ti + 16, columns 2 tj + c
    float v[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
      const float x0 = X[32 + ti][32 + m], x1 = X[48 + ti][32 + m];
      const float2 t = *reinterpret_cast<const float2*>(&T[m][2 * tj]);
      v[0][0] = fmaf(x0, t.x, v[0][0]), v[0][1] = fmaf(x0, t.y, v[0][1]);
      v[1][0] = fmaf(x1, t.x, v[1][0]), v[1][1] = fmaf(x1, t.y, v[1][1]);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      X[32 + ti][2 * tj + c] = -v[0][c];
      X[48 + ti][2 * tj + c] = -v[1][c];
    }
  }
  __syncthreads();
}

// 16 consecutive values (times `sign`) as bf16 hi and lo halves, two 16-byte
// stores each (hi and lo 32-byte aligned)
__device__ __forceinline__ void split_store16(const float (&v)[16], float sign, __nv_bfloat16* hi,
                                              __nv_bfloat16* lo) {
  uint32_t h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float a = sign * v[2 * e], b = sign * v[2 * e + 1];
    const __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(a - __low2float(hh), b - __high2float(hh));
    h[e] = *reinterpret_cast<const uint32_t*>(&hh);
    l[e] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  uint4* h4 = reinterpret_cast<uint4*>(hi);
  uint4* l4 = reinterpret_cast<uint4*>(lo);
  h4[0] = make_uint4(h[0], h[1], h[2], h[3]);
  h4[1] = make_uint4(h[4], h[5], h[6], h[7]);
  l4[0] = make_uint4(l[0], l[1], l[2], l[3]);
  l4[1] = make_uint4(l[4], l[5], l[6], l[7]);
}

// 64 x 64 block of a row-major fp32 matrix (row stride ld) into shared memory
__device__ __forceinline__ void load_block64(float (*S)[kT + 1], const float* __restrict__ src, int64_t ld) {
  float v[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int e = threadIdx.x + 256 * q;
    v[q] = src[(int64_t)(e >> 6) * ld + (e & 63)];
  }
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int e = threadIdx.x + 256 * q;
    S[e >> 6][e & 63] = v[q];
  }
}

// Step k of the chain of diagonal blocks (grid nb - k CTAs; k = 0: one CTA).
// It finishes the update of column block k by panel k - 1 and factors the
// diagonal block, reading only column blocks k - 1 and k of M, which the
// update products of panels <= k - 2 and step k - 1 have completed:
//   every CTA forms L_{k,k-1} = A_{k,k-1} L_{k-1}^-T (L_{k-1}^-1 from step k - 1);
//   CTA r > 0 forms L_{k+r,k-1} = A_{k+r,k-1} L_{k-1}^-T and writes
//     A_{k+r,k} - L_{k+r,k-1} L_{k,k-1}^T back to M;
//   CTA 0 factors A_kk - L_{k,k-1} L_{k,k-1}^T and writes the inverse of its
//     Cholesky factor to Linv_k (64 x 64 row-major, at Linv + 64 * 64 k).
// The tensor-core update of panel k - 1 leaves column block k alone, so this
// runs beside that panel's own kernels and product.  A bad pivot records
// ISPA_ERR_NOT_SPD and its row.
__global__ void __launch_bounds__(256) diag_step_kernel(float* M, int D, int k, float* __restrict__ Linv,
                                                        int32_t* status) {
  // the products' operands, contraction index first; then the block to
  // factor (A) and its inverse factor (X), row stride 65, in the same storage
  __shared__ __align__(16) float U[kT][kLdv];
  __shared__ __align__(16) float V[kT][kLdv];
  __shared__ __align__(16) float T[32][36];
  __shared__ __align__(16) float Lt[32][36];
  __shared__ __align__(16) float Ls[32][32];
  __shared__ float rinv[32];
  __shared__ int bad;
  auto A = reinterpret_cast<float (*)[kT + 1]>(&U[0][0]);
  auto X = reinterpret_cast<float (*)[kT + 1]>(&V[0][0]);
  // the next step may be resident early: it waits below for this grid's end
  asm volatile("griddepcontrol.launch_dependents;");
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int r = blockIdx.x;
  const int64_t ld = D;
  auto block = [&](int bi, int bj) { return M + (int64_t)bi * kT * ld + (int64_t)bj * kT; };
  if (tid == 0) bad = -1;
  // every read of M and Linv follows the completion of the previous step
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (k == 0) {
    load_block64(A, block(0, 0), ld);
    __syncthreads();
  } else {
    load_t64(U, block(k, k - 1), ld);                   // U[t][i] = A_{k,k-1}[i][t]
    load_t64(V, Linv + (int64_t)(k - 1) * kT * kT, kT);  // V[t][j] = L_{k-1}^-1[j][t]
    __syncthreads();
    float lk[4][4], lr[4][4];
    mm64v(U, V, lk);  // L_{k,k-1}
    if (r > 0) {
      __syncthreads();
      load_t64(U, block(k + r, k - 1), ld);
      __syncthreads();
      mm64v(U, V, lr);  // L_{k+r,k-1}
    }
    float* tgt = block(k + r, k);
    float4 tv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) tv[a] = *reinterpret_cast<const float4*>(tgt + (int64_t)(4 * ty + a) * ld + 4 * tx);
    __syncthreads();
    // U[t][i] = L_{k+r,k-1}[i][t], V[t][j] = L_{k,k-1}[j][t]
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float(&w)[4][4] = r > 0 ? lr : lk;
      *reinterpret_cast<float4*>(&U[4 * tx + b][4 * ty]) = make_float4(w[0][b], w[1][b], w[2][b], w[3][b]);
      *reinterpret_cast<float4*>(&V[4 * tx + b][4 * ty]) = make_float4(lk[0][b], lk[1][b], lk[2][b], lk[3][b]);
    }
    __syncthreads();
    float acc[4][4];
    mm64v(U, V, acc);  // L_{k+r,k-1} L_{k,k-1}^T
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      tv[a].x -= acc[a][0], tv[a].y -= acc[a][1], tv[a].z -= acc[a][2], tv[a].w -= acc[a][3];
    }
    if (r > 0) {
#pragma unroll
      for (int a = 0; a < 4; ++a) *reinterpret_cast<float4*>(tgt + (int64_t)(4 * ty + a) * ld + 4 * tx) = tv[a];
      return;
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float* row = &A[4 * ty + a][4 * tx];
      row[0] = tv[a].x, row[1] = tv[a].y, row[2] = tv[a].z, row[3] = tv[a].w;
    }
    __syncthreads();
  }
  factor_diag64(A, X, T, Lt, Ls, rinv, &bad, k * kT);
  if (tid == 0 && bad >= 0 && status) {
    if (atomicCAS(status, 0, (int32_t)ISPA_ERR_NOT_SPD) == 0) status[1] = bad;
  }
  float* out = Linv + (int64_t)k * kT * kT;
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int e = tid + 256 * q;
    out[e] = X[e >> 6][e & 63];
  }
}

// Panel k with L_kk^-1 given (Linv, from diag_step_kernel):
//   blocks [0, rest): one 64-row block r below the diagonal,
//     L_rk = A_rk L_kk^-T as split operands only: -hi/-lo as K-major
//     [rows, 64] (a_hi, a_lo, local row index) and hi/lo transposed as
//     [64, ld_t] (lt_hi, lt_lo); M is only read (step k + 1 of the diagonal
//     chain reads the same A_rk beside this kernel);
//   blocks [rest, rest + ncb): one 64-column block of the panel's
//     right-hand-side rows, Y = L_kk^-1 RHS_k, written back to RHS, plus hi/lo
//     [64, ld_y] (y_hi, y_lo).
__global__ void __launch_bounds__(256) panel_apply_kernel(const float* M, int D, int k, int rest,
                                                          const float* __restrict__ Linv, float* RHS, int64_t rhs_ld,
                                                          int rhs_cols, __nv_bfloat16* a_hi, __nv_bfloat16* a_lo,
                                                          __nv_bfloat16* lt_hi, __nv_bfloat16* lt_lo, int64_t ld_t,
                                                          __nv_bfloat16* y_hi, __nv_bfloat16* y_lo, int64_t ld_y) {
  // operands with the contraction index first; the result then goes through
  // the storage of the first, row stride 65
  __shared__ __align__(16) float U[kT][kLdv];  // this CTA's block
  __shared__ __align__(16) float V[kT][kLdv];  // V[t][j] = L_kk^-1[j][t]
  auto A = reinterpret_cast<float (*)[kT + 1]>(&U[0][0]);
  const int tid = threadIdx.x;
  const bool row_block = (int)blockIdx.x < rest;
  const int c0 = row_block ? 0 : ((int)blockIdx.x - rest) * kT;
  const float* own = row_block ? M + (int64_t)(k + 1 + blockIdx.x) * kT * D + (int64_t)k * kT
                               : RHS + (int64_t)k * kT * rhs_ld + c0;
  load_t64(V, Linv, kT);
  if (row_block)
    load_t64(U, own, D);  // U[t][i] = A_rk[i][t]
  else
    load_n64(U, own, rhs_ld);  // U[t][j] = RHS_k[t][j]
  __syncthreads();
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4];
  if (row_block)
    mm64v(U, V, acc);  // A_rk L_kk^-T
  else
    mm64v(V, U, acc);  // L_kk^-1 RHS_k
  __syncthreads();
  // the 64 x 64 result through shared memory, so that every global store
  // below is a 16-byte vector of one row
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) A[4 * ty + a][4 * tx + b] = acc[a][b];
  __syncthreads();
  const int ri = tid >> 2, c16 = (tid & 3) * 16;  // this thread: row (or column) ri, 16 values from c16
  float v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = A[ri][c16 + e];
  if (row_block) {
    const int64_t row0 = (int64_t)blockIdx.x * kT;  // local row of the trailing block
    split_store16(v, -1.f, a_hi + (row0 + ri) * 64 + c16, a_lo + (row0 + ri) * 64 + c16);
    // L21^T: row ri of the transpose is column ri of the block
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = A[c16 + e][ri];
    split_store16(v, 1.f, lt_hi + (int64_t)ri * ld_t + row0 + c16, lt_lo + (int64_t)ri * ld_t + row0 + c16);
  } else {
    // rhs_cols and c0 are multiples of 64: the block lies wholly inside
    float4* dst = reinterpret_cast<float4*>(RHS + (int64_t)k * kT * rhs_ld + (int64_t)ri * rhs_ld + c0 + c16);
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    split_store16(v, 1.f, y_hi + (int64_t)ri * ld_y + c0 + c16, y_lo + (int64_t)ri * ld_y + c0 + c16);
  }
}

// RHS = [0 | I] (D x 2D fp32, 16-byte vectors)
__global__ void init_rhs_kernel(float* __restrict__ RHS, int D) {
  const int64_t n4 = (int64_t)D * 2 * D / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = (e * 4) / (2 * D), j0 = (e * 4) % (2 * D) - D;  // column within the identity part
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t off = i - j0;
    v.x = off == 0 ? 1.f : 0.f;
    v.y = off == 1 ? 1.f : 0.f;
    v.z = off == 2 ? 1.f : 0.f;
    v.w = off == 3 ? 1.f : 0.f;
    reinterpret_cast<float4*>(RHS)[e] = v;
  }
}

// [Y | X] (D x 2D fp32) -> hi/lo of Y and of X, each D x D bf16; four
// elements per thread and step (16-byte loads, 8-byte stores)
__global__ void split_rhs_kernel(const float* __restrict__ RHS, int D, __nv_bfloat16* __restrict__ yh,
                                 __nv_bfloat16* __restrict__ yl, __nv_bfloat16* __restrict__ xh,
                                 __nv_bfloat16* __restrict__ xl) {
  const int64_t n4 = (int64_t)D * 2 * D / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(RHS)[e];
    const int64_t i = (e * 4) / (2 * D), j = (e * 4) % (2 * D);  // j multiple of 4: never straddles D
    __nv_bfloat16* hi = j < D ? yh + i * D + j : xh + i * D + j - D;
    __nv_bfloat16* lo = j < D ? yl + i * D + j : xl + i * D + j - D;
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v.x, v.y), h1 = __floats2bfloat162_rn(v.z, v.w);
    const __nv_bfloat162 l0 = __floats2bfloat162_rn(v.x - __low2float(h0), v.y - __high2float(h0));
    const __nv_bfloat162 l1 = __floats2bfloat162_rn(v.z - __low2float(h1), v.w - __high2float(h1));
    *reinterpret_cast<uint2*>(hi) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
    *reinterpret_cast<uint2*>(lo) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&l0), *reinterpret_cast<const uint32_t*>(&l1));
  }
}

}  // namespace simt

// workspace of the tensor-core form: M (4 D^2) | RHS (8 D^2) | split area (4 D^2) |
// Linv (256 D) | A hi/lo (256 D) | L21^T hi/lo (256 D) | Y_k hi/lo (512 D) | lambda (256)
static bool tc_eligible(ispa_dtype_t w_dt, int64_t D) { return w_dt == ISPA_DT_BF16 && D % 128 == 0 && D >= 256; }
static size_t tc_workspace_bytes(int64_t D) { return (size_t)(16 * D * D + 1280 * D + 256); }
static size_t compact_workspace_bytes(int64_t D) { return (size_t)(4 * D * D + 256 * D + 256); }

size_t absorb_workspace_bytes(int64_t D) { return D % 128 == 0 && D >= 256 ? tc_workspace_bytes(D) : compact_workspace_bytes(D); }
size_t absorb_compact_workspace_bytes(int64_t D) { return compact_workspace_bytes(D); }

ispa_status_t absorb_step_update(int64_t rows, int64_t m_col0, const void* a_hi, const void* a_lo,
                                 const void* lt_hi, const void* lt_lo, int64_t lt_ld, const void* y_hi,
                                 const void* y_lo, int64_t y_ld, int64_t rhs_cols, float* m_sub, int64_t m_ld,
                                 float* rhs_sub, int64_t rhs_ld, cudaStream_t stream);
ispa_status_t gemm_split3_xt_y(int64_t D, int64_t N, const void* x_hi, const void* x_lo, int64_t x_ld,
                               const void* y_hi, const void* y_lo, int64_t y_ld, float* c, int64_t ldc,
                               cudaStream_t stream);
ispa_status_t gemm_hilo_w(int64_t M, int64_t K, const void* a_hi, const void* a_lo, const void* w, int64_t N,
                          float* c, int64_t ldc, cudaStream_t stream);
ispa_status_t gemm_split3(int64_t M, int64_t N, int64_t K, const void* a_hi, const void* a_lo, int64_t lda,
                          const void* b_hi, const void* b_lo, int64_t ldb, float* c, int64_t ldc,
                          cudaStream_t stream);

// One side stream and two events per host thread and CUDA context, created on
// the first tensor-core solve there (make that first call before any stream
// capture) and kept until the process exits.
namespace {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}
struct SideStream {
  unsigned long long ctx;
  cudaStream_t stream;
  cudaEvent_t fork, join;
};
thread_local std::vector<SideStream> t_side;
}  // namespace

static ispa_status_t side_stream_for_current_context(cudaStream_t* s, cudaEvent_t* fork, cudaEvent_t* join) {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) {
    set_last_error("no current CUDA context for the absorb solve's side stream");
    return ISPA_ERR_CUDA;
  }
  for (const auto& e : t_side)
    if (e.ctx == id) {
      *s = e.stream, *fork = e.fork, *join = e.join;
      return ISPA_OK;
    }
  SideStream e{id, nullptr, nullptr, nullptr};
  if (cudaStreamCreateWithFlags(&e.stream, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&e.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&e.join, cudaEventDisableTiming) != cudaSuccess)
    return check_launch("creating the absorb solve's side stream");
  t_side.push_back(e);
  *s = e.stream, *fork = e.fork, *join = e.join;
  return ISPA_OK;
}

static ispa_status_t absorb_solve_tc(const float* G, const float* R, const __nv_bfloat16* W, int64_t D64,
                                    double lam_abs, double lam_rel, float* dW, __nv_bfloat16* w_new, void* workspace,
                                    int32_t* status, cudaStream_t st) {
  using namespace simt;
  const int D = (int)D64;
  const int nb = D / kT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* M = reinterpret_cast<float*>(ws);
  float* RHS = reinterpret_cast<float*>(ws + 4 * D64 * D64);
  uint8_t* split = ws + 12 * D64 * D64;
  __nv_bfloat16* a_hi = reinterpret_cast<__nv_bfloat16*>(ws + 16 * D64 * D64 + 256 * D64);
  __nv_bfloat16* a_lo = a_hi + 64 * D64;
  __nv_bfloat16* lt_hi = a_lo + 64 * D64;
  __nv_bfloat16* lt_lo = lt_hi + 64 * D64;
  __nv_bfloat16* y_hi = lt_lo + 64 * D64;
  __nv_bfloat16* y_lo = y_hi + 128 * D64;
  double* lam = reinterpret_cast<double*>(ws + 16 * D64 * D64 + 1280 * D64);
  float* Linv = reinterpret_cast<float*>(ws + 16 * D64 * D64);
  const int sms = num_sms();
  const int64_t rhs_ld = 2 * D64;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  ispa_status_t s0 = side_stream_for_current_context(&side, &ev_fork, &ev_join);
  if (s0 != ISPA_OK) return s0;

  // S = R W into RHS[:, :D], RHS[:, D:] = I
  __nv_bfloat16* r_hi = reinterpret_cast<__nv_bfloat16*>(split);
  __nv_bfloat16* r_lo = r_hi + D64 * D64;
  split_bf16_kernel<<<sms * 4, 256, 0, st>>>(R, r_hi, r_lo, D64 * D64);
  init_rhs_kernel<<<sms * 4, 256, 0, st>>>(RHS, D);
  ispa_status_t s1 = gemm_hilo_w(D, D, r_hi, r_lo, W, D, RHS, rhs_ld, st);
  if (s1 != ISPA_OK) return s1;
  trace_lambda_kernel<<<1, 256, 0, st>>>(G, D, lam_abs, lam_rel, lam);
  shift_kernel<<<sms * 4, 256, 0, st>>>(G, M, D, lam);
  // The chain of diagonal steps runs on the side stream: step k + 1 needs
  // step k and the update product of panel k - 1 only, so it runs beside
  // panel k's kernel and product on the main stream, which need step k (and
  // the product of panel k - 1, earlier on the same stream).  Host order
  // keeps one event per direction: ev_join marks the latest diagonal step,
  // ev_fork the latest update product, each waited on before it is recorded
  // again.
  diag_step_kernel<<<1, 256, 0, st>>>(M, D, 0, Linv, status);
  if (nb > 1 && (cudaEventRecord(ev_fork, st) != cudaSuccess || cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess))
    return check_launch("absorb fork");
  for (int k = 0; k < nb; ++k) {
    const int rest = nb - k - 1;
    const int off = (k + 1) * kT;
    const int rhs_cols = D + off;  // nonzero columns of the panel's rows of [L^-1 S | L^-1]
    if (k > 0 && cudaStreamWaitEvent(st, ev_join, 0) != cudaSuccess) return check_launch("absorb join");
    panel_apply_kernel<<<rest + (rhs_cols + kT - 1) / kT, 256, 0, st>>>(
        M, D, k, rest, Linv + (int64_t)k * kT * kT, RHS, rhs_ld, rhs_cols, a_hi, a_lo, lt_hi, lt_lo, D64, y_hi,
        y_lo, rhs_ld);
    if (rest > 0) {
      // programmatic launch: the step's CTAs may become resident while the
      // previous step runs (the kernel waits for its end before any read)
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)rest);
      cfg.blockDim = dim3(256);
      cfg.stream = side;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, diag_step_kernel, M, D, k + 1, Linv, status) != cudaSuccess)
        return check_launch("absorb diagonal step");
      if (cudaEventRecord(ev_join, side) != cudaSuccess) return check_launch("absorb join");
      // trailing columns from block k + 2: step k + 1 updates block k + 1
      s1 = absorb_step_update(D - off, kT, a_hi, a_lo, lt_hi, lt_lo, D64, y_hi, y_lo, rhs_ld, rhs_cols,
                              M + (int64_t)off * D + off, D64, RHS + (int64_t)off * rhs_ld, rhs_ld, st);
      if (s1 != ISPA_OK) return s1;
      if (rest > 1 &&
          (cudaEventRecord(ev_fork, st) != cudaSuccess || cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess))
        return check_launch("absorb fork");
    }
  }
  // dW = (L^-1)^T (L^-1 S): hi/lo of L^-1 S into M's storage, of L^-1 into the split area
  __nv_bfloat16* yh = reinterpret_cast<__nv_bfloat16*>(M);
  __nv_bfloat16* yl = yh + D64 * D64;
  __nv_bfloat16* xh = reinterpret_cast<__nv_bfloat16*>(split);
  __nv_bfloat16* xl = xh + D64 * D64;
  split_rhs_kernel<<<sms * 4, 256, 0, st>>>(RHS, D, yh, yl, xh, xl);
  if (cudaMemsetAsync(dW, 0, (size_t)D64 * D64 * 4, st) != cudaSuccess) return check_launch("cudaMemsetAsync of dW");
  s1 = gemm_split3_xt_y(D, D, xh, xl, D64, yh, yl, D64, dW, D64, st);
  if (s1 != ISPA_OK) return s1;
  if (w_new) wnew_kernel<<<sms * 4, 256, 0, st>>>(W, dW, w_new, D64 * D64);
  return check_launch("absorb_solve");
}

// C[M, N] (= | +=) A[M, K] W[K, N] on the tensor cores (bf16 operands, fp32 C).
ispa_status_t gemm_rm_bf16_f32(const void* a, int64_t M, int64_t K, int64_t a_stride, const void* w, int64_t N,
                               float* c, int64_t ldc, bool accumulate, cudaStream_t stream);

// Compact form of the solve (workspace 4 D^2 + 256 D + 256 bytes): the same
// factorisation with its updates and triangular solves on the CUDA cores in
// fp32.  Used for fp32 W (whose 1e-3 accuracy the split-precision products do
// not keep for ill-conditioned statistics), for D that the tensor-core form
// does not tile, and by the no-allocation entry point.
ispa_status_t absorb_solve_compact(const float* G, const float* R, const void* W, ispa_dtype_t w_dt, int64_t D64,
                                   double lam_abs, double lam_rel, float* dW, void* w_new, void* workspace,
                                   int32_t* status, cudaStream_t st) {
  using namespace simt;
  const int D = (int)D64;
  const int nb = D / kT;
  float* M = static_cast<float*>(workspace);
  float* Linv = M + (int64_t)D * D;
  double* lam = reinterpret_cast<double*>(Linv + (int64_t)D * kT);

  const int sms = num_sms();
  // S = R W, written into dW.  With bf16 W the product runs on the tensor
  // cores as hi(R) W + lo(R) W, the two bf16 halves of R staged in M's storage
  // before M is formed.
  if (w_dt == ISPA_DT_BF16 && D % 128 == 0) {
    __nv_bfloat16* Rh = reinterpret_cast<__nv_bfloat16*>(M);
    __nv_bfloat16* Rl = Rh + (int64_t)D * D;
    split_bf16_kernel<<<sms * 4, 256, 0, st>>>(R, Rh, Rl, (int64_t)D * D);
    ispa_status_t s1 = gemm_rm_bf16_f32(Rh, D, D, D, W, D, dW, D, false, st);
    if (s1 != ISPA_OK) return s1;
    s1 = gemm_rm_bf16_f32(Rl, D, D, D, W, D, dW, D, true, st);
    if (s1 != ISPA_OK) return s1;
  } else if (w_dt == ISPA_DT_BF16) {
    gemm_f32(st, D, D, D, 1.f, R, D, 1, static_cast<const __nv_bfloat16*>(W), D, 1, 0.f, dW, D);
  } else {
    gemm_f32(st, D, D, D, 1.f, R, D, 1, static_cast<const float*>(W), D, 1, 0.f, dW, D);
  }
  trace_lambda_kernel<<<1, 256, 0, st>>>(G, D, lam_abs, lam_rel, lam);
  shift_kernel<<<sms * 4, 256, 0, st>>>(G, M, D, lam);
  // Cholesky
  for (int k = 0; k < nb; ++k) {
    float* Lk = Linv + (int64_t)k * kT * kT;
    potrf_diag_kernel<<<1, 256, 0, st>>>(M, D, k, Lk, status);
    const int rest = nb - k - 1;
    if (rest > 0) {
      panel_kernel<<<rest, 256, 0, st>>>(M, D, k, Lk);
      const int off = (k + 1) * kT;
      const float* P = M + (int64_t)off * D + (int64_t)k * kT;
      gemm_f32(st, D - off, D - off, kT, -1.f, P, D, 1, P, 1, D, 1.f, M + (int64_t)off * D + off, D, true);
    }
  }
  // forward: L Y = S
  for (int k = 0; k < nb; ++k) {
    diag_apply_kernel<<<nb, 256, 0, st>>>(dW, D, k, Linv + (int64_t)k * kT * kT, 0);
    const int off = (k + 1) * kT;
    if (off < D)
      gemm_f32(st, D - off, D, kT, -1.f, M + (int64_t)off * D + (int64_t)k * kT, D, 1, dW + (int64_t)k * kT * D, D,
               1, 1.f, dW + (int64_t)off * D, D);
  }
  // backward: L^T X = Y
  for (int k = nb - 1; k >= 0; --k) {
    diag_apply_kernel<<<nb, 256, 0, st>>>(dW, D, k, Linv + (int64_t)k * kT * kT, 1);
    const int rows = k * kT;
    if (rows > 0)
      gemm_f32(st, rows, D, kT, -1.f, M + (int64_t)k * kT * D, 1, D, dW + (int64_t)k * kT * D, D, 1, 1.f, dW, D);
  }
  if (w_new) {
    const int64_t n = (int64_t)D * D;
    if (w_dt == ISPA_DT_BF16)
      wnew_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), dW,
                                           static_cast<__nv_bfloat16*>(w_new), n);
    else
      wnew_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const float*>(W), dW, static_cast<float*>(w_new), n);
  }
  return check_launch("absorb_solve");
}

ispa_status_t absorb_solve_launch(const float* G, const float* R, const void* W, ispa_dtype_t w_dt, int64_t D,
                                  double lam_abs, double lam_rel, float* dW, void* w_new, void* workspace,
                                  int32_t* status, cudaStream_t st) {
  if (tc_eligible(w_dt, D))
    return absorb_solve_tc(G, R, static_cast<const __nv_bfloat16*>(W), D, lam_abs, lam_rel, dW,
                           static_cast<__nv_bfloat16*>(w_new), workspace, status, st);
  return absorb_solve_compact(G, R, W, w_dt, D, lam_abs, lam_rel, dW, w_new, workspace, status, st);
}

// ------------------------------------------------------- layer selection
// Reconstruction error of one layer after the warm-up ("Instance-Specific
// Parametric Absorption", gist.science technical summary, "Dynamic Layer
// Selection"), ||A_loc (W + dW) - A_full W||^2 / ||A_full W||^2, from the
// warm-up statistics alone: with dA = A_full - A_loc, G = A_loc^T A_loc,
// R = A_loc^T dA, E = dA^T dA,
//   num = <dW, G dW> - 2 <dW, R W> + <W, E W>,
//   den = <W, G W> + 2 <W, R W> + <W, E W>,
// <X, Y> the Frobenius inner product.  Products in fp32, sums in fp64.
namespace simt {

// out = the symmetric matrix whose lower triangle (row >= col) is that of in
__global__ void symmetrize_kernel(const float* __restrict__ in, float* __restrict__ out, int D) {
  const int64_t n = (int64_t)D * D;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / D), j = (int)(e - (int64_t)i * D);
    out[e] = i >= j ? in[e] : in[(int64_t)j * D + i];
  }
}

// *out += coef * <x, y> (fp64 accumulation)
template <typename TX>
__global__ void frob_dot_kernel(const TX* __restrict__ x, const float* __restrict__ y, int64_t n, double coef,
                                double* __restrict__ out) {
  __shared__ double part[8];
  double acc = 0.0;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    acc += (double)to_f32(x[e]) * (double)y[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
    atomicAdd(out, coef * t);
  }
}

}  // namespace simt

// Tensor-core form (bf16 W, D % 128 == 0, D >= 256): the four products as
// split-precision tcgen05 products, [P_R; P_E; P_G] = [R; sym(E); sym(G)] W
// in one launch (W is exactly bf16: two operand pairs) and P_1 = sym(G) dW
// (three pairs), then all six inner products in one pass.  Workspace:
// P_R, P_E, P_G, P_1 (4 D^2 fp32), the bf16 hi / lo halves of the stacked
// [R; sym(E); sym(G)] (2 x 3 D^2) and of dW (2 x D^2): 32 D^2 bytes.
size_t layer_error_workspace_bytes(int64_t D) { return (size_t)32 * D * D; }

// hi / lo bf16 halves of the rows of [R; sym(E); sym(G)] (3D x D): one 32 x 32
// output tile per block, read through shared memory both as itself and
// transposed, so the mirrored upper triangles are read with coalesced rows.
__global__ void __launch_bounds__(256) split_stack_kernel(const float* __restrict__ R, const float* __restrict__ E,
                                                          const float* __restrict__ G, int D,
                                                          __nv_bfloat16* __restrict__ hi,
                                                          __nv_bfloat16* __restrict__ lo) {
  __shared__ float t[32][33], u[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;  // rows of the stack, columns
  const int part = r0 / D, i0 = r0 - part * D;  // D % 32 == 0: a tile never straddles two parts
  const float* M = part == 0 ? R : part == 1 ? E : G;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const bool need_t = part == 0 || i0 + 31 >= c0;  // some element on or below the diagonal
  const bool need_u = part > 0 && i0 < c0 + 31;    // some element above it: read mirrored
  for (int y = ty; y < 32; y += 8) {
    if (need_t) t[y][tx] = M[(int64_t)(i0 + y) * D + c0 + tx];
    if (need_u) u[y][tx] = M[(int64_t)(c0 + y) * D + i0 + tx];  // the mirrored tile, row by row
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int i = i0 + y, j = c0 + tx;
    const float v = (part == 0 || i >= j) ? t[y][tx] : u[tx][y];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const int64_t e = (int64_t)(r0 + y) * D + j;
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// num += <dW, P_1> - 2 <dW, P_R> + <W, P_E>, den += <W, P_G> + 2 <W, P_R> + <W, P_E>
// (fp64 accumulation, one pass over the six matrices)
__global__ void __launch_bounds__(256) error_terms_kernel(const float* __restrict__ dW,
                                                          const __nv_bfloat16* __restrict__ W,
                                                          const float* __restrict__ P, int64_t n,
                                                          double* __restrict__ num_den) {
  __shared__ double part[2][8];
  const float* PR = P;
  const float* PE = P + n;
  const float* PG = P + 2 * n;
  const float* P1 = P + 3 * n;
  double a_num = 0.0, a_den = 0.0;
  // four consecutive elements per step (n % 4 == 0): 16-byte loads, 8 bytes of W
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n / 4; v += (int64_t)gridDim.x * blockDim.x) {
    const float4 d4 = __ldg(reinterpret_cast<const float4*>(dW) + v);
    const float4 p1 = __ldg(reinterpret_cast<const float4*>(P1) + v);
    const float4 pr = __ldg(reinterpret_cast<const float4*>(PR) + v);
    const float4 pe = __ldg(reinterpret_cast<const float4*>(PE) + v);
    const float4 pg = __ldg(reinterpret_cast<const float4*>(PG) + v);
    const uint2 wb = __ldg(reinterpret_cast<const uint2*>(W) + v);
    const float d[4] = {d4.x, d4.y, d4.z, d4.w}, q1[4] = {p1.x, p1.y, p1.z, p1.w};
    const float qr[4] = {pr.x, pr.y, pr.z, pr.w}, qe[4] = {pe.x, pe.y, pe.z, pe.w}, qg[4] = {pg.x, pg.y, pg.z, pg.w};
    const float w[4] = {__uint_as_float(wb.x << 16), __uint_as_float(wb.x & 0xFFFF0000u), __uint_as_float(wb.y << 16),
                        __uint_as_float(wb.y & 0xFFFF0000u)};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double dj = d[j], wj = w[j], rj = qr[j], ej = qe[j];
      a_num += dj * (double)q1[j] - 2.0 * dj * rj + wj * ej;
      a_den += wj * (double)qg[j] + 2.0 * wj * rj + wj * ej;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a_num += __shfl_xor_sync(0xffffffffu, a_num, o);
    a_den += __shfl_xor_sync(0xffffffffu, a_den, o);
  }
  if ((threadIdx.x & 31) == 0) {
    part[0][threadIdx.x >> 5] = a_num;
    part[1][threadIdx.x >> 5] = a_den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double x = 0.0, y = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) x += part[0][w], y += part[1][w];
    atomicAdd(num_den, x);
    atomicAdd(num_den + 1, y);
  }
}

static ispa_status_t layer_error_tc(const float* G, const float* R, const float* E, const __nv_bfloat16* W,
                                    const float* dW, int64_t D, uint8_t* ws, double* num_den, cudaStream_t st) {
  const int64_t n = D * D;
  float* P = reinterpret_cast<float*>(ws);  // P_R, P_E, P_G, P_1
  __nv_bfloat16* s_hi = reinterpret_cast<__nv_bfloat16*>(ws + 16 * n);
  __nv_bfloat16* s_lo = s_hi + 3 * n;
  __nv_bfloat16* d_hi = s_lo + 3 * n;
  __nv_bfloat16* d_lo = d_hi + n;
  const int sms = num_sms();
  if (cudaMemsetAsync(P, 0, 16 * (size_t)n, st) != cudaSuccess ||
      cudaMemsetAsync(num_den, 0, 2 * sizeof(double), st) != cudaSuccess)
    return check_launch("cudaMemsetAsync of the layer-error products");
  split_stack_kernel<<<dim3((unsigned)(D / 32), (unsigned)(3 * D / 32)), 256, 0, st>>>(R, E, G, (int)D, s_hi, s_lo);
  simt::split_bf16_kernel<<<sms * 4, 256, 0, st>>>(dW, d_hi, d_lo, n);
  ispa_status_t s1 = check_launch("split_stack_kernel / split_bf16_kernel");
  if (s1 != ISPA_OK) return s1;
  s1 = gemm_hilo_w(3 * D, D, s_hi, s_lo, W, D, P, D, st);  // [R; E; G] W
  if (s1 != ISPA_OK) return s1;
  s1 = gemm_split3(D, D, D, s_hi + 2 * n, s_lo + 2 * n, D, d_hi, d_lo, D, P + 3 * n, D, st);  // G dW
  if (s1 != ISPA_OK) return s1;
  error_terms_kernel<<<sms * 8, 256, 0, st>>>(dW, W, P, n, num_den);
  return check_launch("error_terms_kernel");
}

template <typename TW>
static void layer_error_impl(const float* G, const float* R, const float* E, const TW* W, const float* dW, int D,
                             float* ws, double* num_den, cudaStream_t st) {
  using namespace simt;
  const int64_t n = (int64_t)D * D;
  float* Gs = ws;
  float* Es = ws + n;
  float* P = ws + 2 * n;
  const int sms = num_sms();
  symmetrize_kernel<<<sms * 4, 256, 0, st>>>(G, Gs, D);
  symmetrize_kernel<<<sms * 4, 256, 0, st>>>(E, Es, D);
  // on failure nothing more is launched; the caller's check_launch reports the error
  if (cudaMemsetAsync(num_den, 0, 2 * sizeof(double), st) != cudaSuccess) return;
  double* num = num_den;
  double* den = num_den + 1;
  gemm_f32(st, D, D, D, 1.f, Gs, D, 1, dW, D, 1, 0.f, P, D);  // G dW
  frob_dot_kernel<float><<<sms * 2, 256, 0, st>>>(dW, P, n, 1.0, num);
  gemm_f32(st, D, D, D, 1.f, R, D, 1, W, D, 1, 0.f, P, D);  // R W
  frob_dot_kernel<float><<<sms * 2, 256, 0, st>>>(dW, P, n, -2.0, num);
  frob_dot_kernel<TW><<<sms * 2, 256, 0, st>>>(W, P, n, 2.0, den);
  gemm_f32(st, D, D, D, 1.f, Es, D, 1, W, D, 1, 0.f, P, D);  // E W
  frob_dot_kernel<TW><<<sms * 2, 256, 0, st>>>(W, P, n, 1.0, num);
  frob_dot_kernel<TW><<<sms * 2, 256, 0, st>>>(W, P, n, 1.0, den);
  gemm_f32(st, D, D, D, 1.f, Gs, D, 1, W, D, 1, 0.f, P, D);  // G W
  frob_dot_kernel<TW><<<sms * 2, 256, 0, st>>>(W, P, n, 1.0, den);
}

ispa_status_t layer_error_launch(const float* G, const float* R, const float* E, const void* W, ispa_dtype_t w_dt,
                                 const float* dW, int64_t D, void* workspace, double* num_den, cudaStream_t st) {
  // the tensor-core form reads W and dW through TMA and 16-byte vectors
  if (tc_eligible(w_dt, D) && aligned16(W) && aligned16(dW) && aligned16(G) && aligned16(R) && aligned16(E))
    return layer_error_tc(G, R, E, static_cast<const __nv_bfloat16*>(W), dW, D, static_cast<uint8_t*>(workspace),
                          num_den, st);
  float* ws = static_cast<float*>(workspace);
  if (w_dt == ISPA_DT_BF16)
    layer_error_impl(G, R, E, static_cast<const __nv_bfloat16*>(W), dW, (int)D, ws, num_den, st);
  else
    layer_error_impl(G, R, E, static_cast<const float*>(W), dW, (int)D, ws, num_den, st);
  return check_launch("layer_error");
}

// fp32 path of the symmetric statistics: E (+)= X^T X (every entry written).
ispa_status_t sym_gram_f32(const float* x, int64_t n_rows, int64_t D, int64_t row_stride, float* E, bool overwrite,
                           cudaStream_t st) {
  simt::gemm_f32(st, (int)D, (int)D, (int)n_rows, 1.f, x, 1, row_stride, x, row_stride, 1, overwrite ? 0.f : 1.f, E, D);
  return check_launch("sym_gram_f32");
}

// fp32 activation path of the statistics: [G | R] (+)= A_loc^T [A_loc | delta].
ispa_status_t gram_f32(const float* a_loc, const float* a_delta, int64_t n_rows, int64_t D, int64_t row_stride,
                       float* G, float* R, bool overwrite, cudaStream_t st) {
  using namespace simt;
  const float beta = overwrite ? 0.f : 1.f;
  gemm_f32(st, (int)D, (int)D, (int)n_rows, 1.f, a_loc, 1, row_stride, a_loc, row_stride, 1, beta, G, D);
  gemm_f32(st, (int)D, (int)D, (int)n_rows, 1.f, a_loc, 1, row_stride, a_delta, row_stride, 1, beta, R, D);
  return check_launch("gram_f32");
}

// fp32 activation path of the projection: y = a w.
ispa_status_t project_f32(const float* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                          const float* w, float* y, cudaStream_t st) {
  simt::gemm_f32(st, (int)n_rows, (int)d_out, (int)d_in, 1.f, a, a_stride, 1, w, d_out, 1, 0.f, y, d_out);
  return check_launch("project_f32");
}

}  // namespace ispa
