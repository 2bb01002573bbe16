// bf16 GEMM on sm_100a tensor cores: C[M, N] (=|+=) A[M, K] * B[K, N], fp32
// accumulation in tensor memory, operands staged by TMA.
//
// Serves two steps of the ISPA hot path:
//  * the Layer-Absorb statistics [G | R] += A_loc^T [A_loc | A_full - A_loc]
//    ("Instance-Specific Parametric Absorption", gist.science technical
//    summary, section 2 stage 2): both operands are the token-major activation
//    matrices read "MN-major" (the contraction runs over tokens, which is the
//    row index of A_loc), so no transpose is ever materialised;
//  * the output projection y = A W (stage 1 and stage 3 of the same section):
//    A is K-major (token rows), W [D_in, D_out] is MN-major.
// One CTA computes one 128 x BN tile: warp 0 issues TMA loads into an
// NST-deep ring, warp 1 issues tcgen05.mma (M=128, N=BN, K=16), warp 2 owns
// the tensor memory, warps 4-7 drain the accumulator (one row per thread).
#include <cstring>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace gemm {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 256;

enum Mode : int { kStoreBf16 = 0, kStoreF32 = 1, kAccumF32 = 2 };

struct Params {
  CUtensorMap a_map;
  CUtensorMap b_map[2];
  int32_t M, N, K;
  int32_t n_split;  // columns [0, n_split) come from b_map[0] / c[0], the rest from b_map[1] / c[1]
  void* c[2];
  int64_t ldc;
  int32_t mode;
  int32_t* status;
};

template <int BN, int NST>
struct Layout {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kBars = NST * kStage;
  static constexpr int kNumBars = 2 * NST + 2;  // full[NST], empty[NST], acc_full, teardown
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

template <bool A_MN, bool B_MN, int BN, int NST>
__global__ void __launch_bounds__(kThreads, 1) gemm_bf16_kernel(const __grid_constant__ Params p) {
  using L = Layout<BN, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* empty = full + NST;
  uint64_t* acc_full = empty + NST;
  uint64_t* teardown = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0g = blockIdx.x * BN, m0 = blockIdx.y * kBM;
  const int half = n0g >= p.n_split ? 1 : 0;
  const int n0 = n0g - half * p.n_split;
  const int nk = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    const CUtensorMap* bm = &p.b_map[half];
    tma_prefetch_desc(&p.a_map);
    tma_prefetch_desc(bm);
    int kb = 0;
    for (; kb < nk; ++kb) {
      const int stage = kb % NST;
      if (kb >= NST && !mbar_wait(&empty[stage], ((kb / NST) - 1) & 1, abort_flag)) break;
      uint8_t* sa = smem + stage * L::kStage;
      uint8_t* sb = sa + L::kABytes;
      const int k0 = kb * kBK;
      mbar_arrive_expect_tx(&full[stage], L::kStage);
      if (A_MN) {
        tma_load_2d(sa, &p.a_map, &full[stage], m0, k0);
        tma_load_2d(sa + 8192, &p.a_map, &full[stage], m0 + 64, k0);
      } else {
        tma_load_2d(sa, &p.a_map, &full[stage], k0, m0);
      }
      if (B_MN) {
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * 8192, bm, &full[stage], n0 + 64 * c, k0);
      } else {
        tma_load_2d(sb, bm, &full[stage], k0, n0);
      }
    }
    if (kb < nk) {  // unwinding after a timeout
      for (int j = kb > NST ? kb - NST : 0; j < kb; ++j)
        mbar_wait_drain(&full[j % NST], (j / NST) & 1, 100000000ull);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, BN, A_MN, B_MN);
    const uint32_t base = smem_u32(smem);
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      const int stage = kb % NST;
      if (!mbar_wait(&full[stage], (kb / NST) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = base + stage * L::kStage;
      const uint32_t sb = sa + L::kABytes;
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        const uint64_t da = A_MN ? sdesc_sw128(sa + kk * 2048, 8192, 1024) : sdesc_sw128(sa + kk * 32, 16, 1024);
        const uint64_t db = B_MN ? sdesc_sw128(sb + kk * 2048, 8192, 1024) : sdesc_sw128(sb + kk * 32, 16, 1024);
        umma_ss(tmem, da, db, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&empty[stage]);
    }
    if (ok) umma_commit(acc_full);
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, 100000000ull);
  } else if (warp >= 4) {
    // ----------------------------------------------------------- epilogue
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int gm = m0 + row;
    bool ok = __all_sync(0xffffffffu, nk == 0 ? true : mbar_wait(acc_full, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16);
      const int n_cols = p.n_split < p.N ? (half ? p.N - p.n_split : p.n_split) : p.N;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * c, r);
        tmem_wait_ld();
        const int gn = n0 + 32 * c;
        if (gm >= p.M || gn >= n_cols) continue;
        if (p.mode == kStoreBf16) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c[half]) + (int64_t)gm * p.ldc + gn);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
            u.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
            u.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
            u.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
            dst[v] = u;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c[half]) + (int64_t)gm * p.ldc + gn);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            float4 x = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                   __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            if (p.mode == kAccumF32) {
              const float4 o = dst[v];
              x.x += o.x;
              x.y += o.y;
              x.z += o.z;
              x.w += o.w;
            }
            dst[v] = x;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, BN);
  if (threadIdx.x == 0 && *abort_flag) report_status(p.status, ISPA_ERR_TIMEOUT);
}

template <bool A_MN, bool B_MN, int BN, int NST>
static ispa_status_t launch(const Params& p, cudaStream_t stream) {
  using L = Layout<BN, NST>;
  auto kern = gemm_bf16_kernel<A_MN, B_MN, BN, NST>;
  ispa_status_t st = set_smem(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (st != ISPA_OK) return st;
  dim3 grid(p.N / BN, (p.M + kBM - 1) / kBM);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p);
  return check_launch("gemm_bf16_kernel");
}

}  // namespace gemm

// [G | R] (+)= A_loc^T [A_loc | delta]  (bf16 inputs, fp32 outputs).
ispa_status_t gram_bf16(const void* a_loc, const void* a_delta, int64_t n_rows, int64_t D, int64_t row_stride,
                        float* G, float* R, bool overwrite, cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  // A operand: element (i, n) = A_loc[n, i]  -> [K = n_rows rows, M = D contiguous]
  if (!encode_map_bf16_2d(&p.a_map, a_loc, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[0], a_loc, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[1], a_delta, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  p.M = (int32_t)D;
  p.N = (int32_t)(2 * D);
  p.K = (int32_t)n_rows;
  p.n_split = (int32_t)D;
  p.c[0] = G;
  p.c[1] = R;
  p.ldc = D;
  p.mode = overwrite ? kStoreF32 : kAccumF32;
  if (D % 256 == 0) return launch<true, true, 256, 4>(p, stream);
  return launch<true, true, 128, 6>(p, stream);
}

// y[n_rows, d_out] = a[n_rows, d_in] * w[d_in, d_out]  (bf16 in/out).
ispa_status_t project_bf16(const void* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                           const void* w, void* y, cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  if (!encode_map_bf16_2d(&p.a_map, a, d_in, n_rows, a_stride * 2, 64, kBM)) return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[0], w, d_out, d_in, d_out * 2, 64, 64)) return ISPA_ERR_CUDA;
  p.b_map[1] = p.b_map[0];
  p.M = (int32_t)n_rows;
  p.N = (int32_t)d_out;
  p.K = (int32_t)d_in;
  p.n_split = (int32_t)d_out;
  p.c[0] = y;
  p.c[1] = y;
  p.ldc = d_out;
  p.mode = kStoreBf16;
  if (d_out % 128 == 0) return launch<false, true, 128, 6>(p, stream);
  return unsupported("bf16 projection needs d_out to be a multiple of 128 (got %lld)", (long long)d_out);
}

}  // namespace ispa
