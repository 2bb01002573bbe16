// bf16 GEMM on sm_100a tensor cores: C[M, N] (=|+=) A[M, K] * B[K, N], fp32
// accumulation in tensor memory, operands staged by TMA.
//
// Serves two steps of the ISPA hot path:
//  * the Layer-Absorb statistics [G | R] += A_loc^T [A_loc | A_full - A_loc]
//    ("Instance-Specific Parametric Absorption", gist.science technical
//    summary, section 2 stage 2): both operands are the token-major activation
//    matrices read "MN-major" (the contraction runs over tokens, the row index
//    of A_loc), so no transpose is ever materialised; only the tiles of G that
//    touch its lower triangle are computed (G is symmetric and the solve reads
//    its lower triangle), and the token range is split across CTAs whose
//    partial sums are added into G, R with vector reductions in L2;
//  * the output projection y = A W (stages 1 and 3 of the same section): A is
//    K-major (token rows), W [D_in, D_out] is MN-major.
// One CTA computes either a 256 x BN tile as two 128-row halves that share
// every B tile, or (the "wide" form) a 128 x 2BN tile as two BN-column halves
// that share every A tile: two M=128 MMAs per K step either way, which halves
// the operand traffic per FLOP against a single 128 x BN product.  The wide
// form lets a 4680 x 1536 output be cut into exactly 148 tiles (128 x 384).
// Warp 0 issues TMA loads into an NST-deep ring, warp 1 issues tcgen05.mma,
// warp 2 owns the tensor-memory columns (two BN-column accumulators) and
// warps 4-11 drain them (one row per thread, one accumulator per warpgroup).
#include <cstring>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace gemm {

constexpr int kBM = 256;  // two tensor-core M=128 halves
constexpr int kBK = 64;    // K elements per stage for bf16 (128 bytes of a row)
constexpr int kBK8 = 128;  // K elements per stage for e4m3 (the same 128 bytes)
constexpr int kThreads = 384;

enum Mode : int { kStoreBf16 = 0, kStoreF32 = 1, kReduceF32 = 2 };

constexpr int kMaxPairs = 3;  // operand pairs summed into one accumulator

struct Params {
  // C = sum_{q < n_pairs} A_q B_q: the K loop runs over the pairs, q-major, so
  // every pair lands in the same tensor-memory accumulator (split-precision
  // products: hi(A) hi(B) + hi(A) lo(B) + lo(A) hi(B))
  CUtensorMap a_map[kMaxPairs];
  CUtensorMap b_map[2][kMaxPairs];  // [column range][pair]
  CUtensorMap c_map[2];  // output maps (32 x 32 boxes) for the TMA epilogue, when c_tma
  int32_t c_tma;
  int32_t M, N, K;
  int32_t n_split;      // columns [0, n_split) come from b_map[0] / c[0], the rest from b_map[1] / c[1]
  int32_t n_cols[2];    // valid columns of each range (outputs beyond are not written)
  int32_t n_pairs;
  int32_t lower_only0;  // skip tiles of the first column range that lie strictly above the diagonal
  int32_t a_upper;      // A(m, k) = 0 for k < m: a row block skips the K steps before it
  int32_t k_per_split;  // K rows per blockIdx.z, a multiple of kBK
  void* c[2];
  int64_t ldc;
  int32_t mode;
  int32_t* status;
  const float* row_scale;  // e4m3 inputs: y[i, j] = acc[i, j] * row_scale[i] * col_scale[j] (no row_scale: 1)
  const float* col_scale;
  const uint8_t* a_exps;  // block-scaled A: ue8m0 exponent bytes [M, K / 32], exps_ld bytes per row
  int32_t exps_ld;
};

template <int BN, int NST, bool WIDE = false>
struct Layout {
  static constexpr int kRows = WIDE ? 128 : kBM;  // output rows of a tile
  static constexpr int kCols = WIDE ? 2 * BN : BN;  // output columns of a tile
  static constexpr int kABytes = kRows * kBK * 2;
  // B is loaded in 64-column boxes (MN-major) or kCols-row boxes (K-major):
  // a tile width that is not a multiple of 64 still lands whole boxes
  static constexpr int kBBytes = (kCols + 63) / 64 * 64 * kBK * 2;
  static constexpr int kTmemCols = 2 * BN <= 256 ? 256 : 512;  // a power of two
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kBars = NST * kStage;
  static constexpr int kNumBars = 2 * NST + 3;  // full[NST], empty[NST], acc_full, teardown, sf_ready
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Tensor-memory columns of the block-scaled form (wide tile, BN = 192: the
// accumulators take columns 0-383): unit B scales in 16 columns, then the A
// scales, 4 columns per 128-element K stage.
constexpr uint32_t kSfbCol = 384;
constexpr uint32_t kSfaCol = 400;
constexpr int kMxMaxStages = (512 - (int)kSfaCol) / 4;  // K <= 28 * 128 = 3584

// The body shared by the bf16 kernels and the e4m3 kernels (F8: both operands
// K-major e4m3, kind::f8f6f4 MMAs with K = 32, the same 128-byte rows and
// swizzle per stage as bf16, and a scaled bf16 epilogue through TMA).
//
// MX (block-scaled A, wide tile only): the MMAs are kind::mxf8f6f4 with one
// ue8m0 scale per 32 K-elements of each row of A and unit scales for B (the
// per-column weight scale stays in the epilogue).  Before the first MMA,
// warps 4-11 write every scale of the tile's 128 rows into tensor memory in
// the layout the instruction reads for M = 128: the scale of row 32c + l for
// the K block 4j + b sits in byte b of column kSfaCol + 4j + c, lane l, and is
// repeated in the lanes l + 32, l + 64, l + 96 of the other three
// sub-partitions.
template <bool A_MN, bool B_MN, int BN, int NST, bool F8, bool WIDE, bool MX = false>
__device__ __forceinline__ void gemm_body(const Params& p) {
  using L = Layout<BN, NST, WIDE>;
  static_assert(!F8 || (!A_MN && !B_MN), "e4m3 operands are K-major");
  static_assert(!MX || (F8 && WIDE && BN == 192), "the block-scaled form uses the wide e4m3 tile");
  constexpr int BK = F8 ? kBK8 : kBK;
  const int n0g = blockIdx.x * L::kCols, m0 = blockIdx.y * L::kRows;
  const int half_n = n0g >= p.n_split ? 1 : 0;
  const int n0 = n0g - half_n * p.n_split;
  // whole-CTA early exit (before any barrier or tensor-memory use): a tile of
  // a lower-triangular output that lies strictly above the diagonal
  if (half_n == 0 && p.lower_only0 && n0 > m0 + L::kRows - 1) return;
  int k_begin = blockIdx.z * p.k_per_split;
  const int k_end = min(p.K, k_begin + p.k_per_split);
  if (p.a_upper) k_begin = max(k_begin, (m0 / BK) * BK);
  if (k_begin >= k_end) return;
  const int nk = (k_end - k_begin + BK - 1) / BK;
  const int steps = p.n_pairs * nk;  // K steps over every pair

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* empty = full + NST;
  uint64_t* acc_full = empty + NST;
  uint64_t* teardown = acc_full + 1;
  uint64_t* sf_ready = teardown + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(teardown, 1);
    mbar_init(sf_ready, 256);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (MX && warp >= 4) {
    // ------------------------------------------------- block scales (MX)
    // both epilogue warpgroups take turns over the 16-column groups (a warp
    // reaches the lanes of its own sub-partition, warp mod 4)
    const int wg = (warp - 4) >> 2;
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t r[16];
    if (wg == 0) {
#pragma unroll
      for (int j = 0; j < 16; ++j) r[j] = 0x7F7F7F7Fu;  // 2^0 in every byte
      tmem_st16(tmem + lanes + kSfbCol, r);
    }
#pragma unroll 1
    for (int g = wg; g < (nk + 3) / 4; g += 2) {  // 16 columns: 4 K stages x 4 row groups
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int j = 4 * g + t;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int row = m0 + 32 * c + lane;
          r[4 * t + c] = (j < nk && row < p.M)
                             ? __ldg(reinterpret_cast<const uint32_t*>(p.a_exps + (int64_t)row * p.exps_ld + 4 * j))
                             : 0x7F7F7F7Fu;
        }
      }
      tmem_st16(tmem + lanes + kSfaCol + 16 * g, r);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(sf_ready);
  }

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    for (int q = 0; q < p.n_pairs; ++q) {
      tma_prefetch_desc(&p.a_map[q]);
      tma_prefetch_desc(&p.b_map[half_n][q]);
    }
    int kb = 0;
    for (; kb < steps; ++kb) {
      const int stage = kb % NST;
      if (kb >= NST && !mbar_wait(&empty[stage], ((kb / NST) - 1) & 1, abort_flag)) break;
      uint8_t* sa = smem + stage * L::kStage;
      uint8_t* sb = sa + L::kABytes;
      const int q = kb / nk;
      const int k0 = k_begin + (kb - q * nk) * BK;
      const CUtensorMap* am = &p.a_map[q];
      const CUtensorMap* bm = &p.b_map[half_n][q];
      mbar_arrive_expect_tx(&full[stage], L::kStage);
      if (A_MN) {
#pragma unroll
        for (int c = 0; c < L::kRows / 64; ++c) tma_load_2d(sa + c * 8192, am, &full[stage], m0 + 64 * c, k0);
      } else {
        tma_load_2d(sa, am, &full[stage], k0, m0);  // one box of kRows rows
      }
      if (B_MN) {
#pragma unroll
        for (int c = 0; c < (L::kCols + 63) / 64; ++c) tma_load_2d(sb + c * 8192, bm, &full[stage], n0 + 64 * c, k0);
      } else {
#pragma unroll
        for (int h = 0; h < L::kCols / BN; ++h)  // boxes of BN rows (a box is at most 256 rows)
          tma_load_2d(sb + h * BN * 128, bm, &full[stage], k0, n0 + h * BN);
      }
    }
    if (kb < steps) {  // unwinding after a timeout
      for (int j = kb > NST ? kb - NST : 0; j < kb; ++j)
        mbar_wait_drain(&full[j % NST], (j / NST) & 1, 100000000ull);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t kIdesc =
        MX ? idesc_mxf8_f32(128, BN) : F8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN, A_MN, B_MN);
    const uint32_t base = smem_u32(smem);
    bool ok = true;
    if (MX) {
      ok = mbar_wait(sf_ready, 0, abort_flag);
      tc_fence_after();
    }
    for (int kb = 0; ok && kb < steps; ++kb) {
      const int stage = kb % NST;
      if (!mbar_wait(&full[stage], (kb / NST) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = base + stage * L::kStage;
      const uint32_t sb = sa + L::kABytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // 4 MMAs of 32 bytes of K (16 bf16 or 32 e4m3)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // tall tile: rows 128h..128h+127 of the A tile (MN-major blocks 2h,
          // 2h+1 / K-major rows) against the whole B tile; wide tile: the
          // whole A tile against columns BN h .. BN h + BN - 1 of the B tile
          const int ah = WIDE ? 0 : h, bh = WIDE ? h : 0;
          const uint64_t da = A_MN ? sdesc_sw128(sa + ah * 16384 + kk * 2048, 8192, 1024)
                                   : sdesc_sw128(sa + ah * 16384 + kk * 32, 16, 1024);
          const uint64_t db = B_MN ? sdesc_sw128(sb + bh * (BN / 64) * 8192 + kk * 2048, 8192, 1024)
                                   : sdesc_sw128(sb + bh * BN * 128 + kk * 32, 16, 1024);
          if (MX)  // A scales of K stage kb, byte kk (k_begin is 0: the block-scaled form has no K split)
            umma_mx(tmem + h * BN, da, db, kIdesc | ((uint32_t)kk << 29),
                    (tmem + kSfaCol + 4 * kb) | ((uint32_t)kk << 30), tmem + kSfbCol, (kb > 0 || kk > 0) ? 1u : 0u);
          else if (F8)
            umma_ss_f8(tmem + h * BN, da, db, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          else
            umma_ss(tmem + h * BN, da, db, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
        }
      }
      umma_commit(&empty[stage]);
    }
    if (ok) umma_commit(acc_full);
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, 100000000ull);
  } else if (warp >= 4) {
    // ----------------------------------------------------------- epilogue
    const int h = (warp - 4) >> 2;  // accumulator: row half (tall tile) or column half (wide tile)
    const int wq = warp & 3;
    const int row0 = m0 + (WIDE ? 0 : h * 128) + wq * 32;
    const int col0 = n0 + (WIDE ? h * BN : 0);
    const int gm = row0 + lane;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag));
    if (ok && p.c_tma) {
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + h * BN;
      const int n_cols = p.n_cols[half_n];
      // The operand ring is idle once acc_full has fired (every MMA that read
      // it has completed).  Each warp stages its 32 rows in 32 x 32 blocks
      // there, double-buffered (2 x 4 KB per warp), in the swizzled layout of
      // the output map, and one lane hands each block to a TMA store or
      // reduction: whole 128-byte lines reach L2 instead of one 16-byte
      // piece of 32 different rows per warp instruction.
      uint8_t* stage_base = smem + (warp - 4) * 8192;
      const CUtensorMap* cm = &p.c_map[half_n];
      const bool rows_in = row0 < p.M;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * c, r);
        tmem_wait_ld();
        if (F8) {
          // per-row and per-column dequantisation scales
          const float sa = !p.row_scale ? 1.f : gm < p.M ? __ldg(p.row_scale + gm) : 0.f;
          const float4* sw4 = reinterpret_cast<const float4*>(p.col_scale + col0 + 32 * c);
          const bool cols_in = col0 + 32 * c < p.n_cols[half_n];  // a ragged last tile reads no scale past N
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 w4 = cols_in ? __ldg(sw4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            r[4 * j + 0] = __float_as_uint(__uint_as_float(r[4 * j + 0]) * (sa * w4.x));
            r[4 * j + 1] = __float_as_uint(__uint_as_float(r[4 * j + 1]) * (sa * w4.y));
            r[4 * j + 2] = __float_as_uint(__uint_as_float(r[4 * j + 2]) * (sa * w4.z));
            r[4 * j + 3] = __float_as_uint(__uint_as_float(r[4 * j + 3]) * (sa * w4.w));
          }
        }
        uint8_t* buf = stage_base + (c & 1) * 4096;
        if (c >= 2) {
          if (lane == 0) bulk_wait_read<1>();  // the block staged two steps ago has been read
          __syncwarp();
        }
        if (p.mode == kStoreBf16) {
          // 64-byte rows, 64-byte swizzle: 16-byte chunk j of row `lane` sits at j ^ ((lane >> 1) & 3)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
            u.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
            u.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
            u.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = u;
          }
        } else {
          // 128-byte rows, 128-byte swizzle: chunk j of row `lane` sits at j ^ (lane & 7)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int gn = col0 + 32 * c;
          if (rows_in && gn < n_cols) {  // boxes are clipped at the matrix edge; skip wholly outside ones
            if (p.mode == kReduceF32)
              tma_reduce_add_2d(cm, buf, gn, row0);
            else
              tma_store_2d(cm, buf, gn, row0);
          }
          bulk_commit();
        }
      }
      if (lane == 0) bulk_wait<0>();
      __syncwarp();
    } else if (ok && !F8) {  // outputs the TMA epilogue cannot address (e4m3 callers always use TMA)
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + h * BN;
      const int n_cols = p.n_cols[half_n];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * c, r);
        tmem_wait_ld();
        const int gn = col0 + 32 * c;
        if (gm >= p.M || gn >= n_cols) continue;
        if (p.mode == kStoreBf16) {
          uint4* dst =
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c[half_n]) + (int64_t)gm * p.ldc + gn);
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
          float* dst = static_cast<float*>(p.c[half_n]) + (int64_t)gm * p.ldc + gn;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float a = __uint_as_float(r[4 * v]), b = __uint_as_float(r[4 * v + 1]);
            const float c2 = __uint_as_float(r[4 * v + 2]), d = __uint_as_float(r[4 * v + 3]);
            if (p.mode == kReduceF32)
              red_add_v4(dst + 4 * v, a, b, c2, d);
            else
              reinterpret_cast<float4*>(dst)[v] = make_float4(a, b, c2, d);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, L::kTmemCols);
  if (threadIdx.x == 0 && *abort_flag) report_status(p.status, ISPA_ERR_TIMEOUT);
}

template <bool A_MN, bool B_MN, int BN, int NST, bool WIDE = false>
__global__ void __launch_bounds__(kThreads, 1) gemm_bf16_kernel(const __grid_constant__ Params p) {
  gemm_body<A_MN, B_MN, BN, NST, false, WIDE>(p);
}

template <int BN, int NST, bool WIDE = false, bool MX = false>
__global__ void __launch_bounds__(kThreads, 1) gemm_e4m3_kernel(const __grid_constant__ Params p) {
  gemm_body<false, false, BN, NST, true, WIDE, MX>(p);
}

// Output maps for the TMA epilogue: c[0] has inner0 columns, c[1] inner1, both
// `rows` rows `ld` elements apart.  Outputs whose base or row pitch is not
// 16-byte aligned keep the per-thread epilogue (c_tma = 0).
static bool set_out_maps(Params& p, bool f32, int64_t rows, int64_t ld, int64_t inner0, int64_t inner1) {
  const int64_t eb = f32 ? 4 : 2;
  p.c_tma = 0;
  if (!aligned16(p.c[0]) || !aligned16(p.c[1]) || (ld * eb) % 16 != 0) return true;
  if (!encode_map_out_2d(&p.c_map[0], p.c[0], f32, inner0, rows, ld * eb)) return false;
  if (!encode_map_out_2d(&p.c_map[1], p.c[1], f32, inner1, rows, ld * eb)) return false;
  p.c_tma = 1;
  return true;
}

template <int BN, int NST, bool WIDE = false, bool MX = false>
static ispa_status_t launch_e4m3(const Params& p, cudaStream_t stream) {
  using L = Layout<BN, NST, WIDE>;
  auto kern = gemm_e4m3_kernel<BN, NST, WIDE, MX>;
  if (p.n_split < p.N && p.n_split % L::kCols) return unsupported("GEMM column ranges must start on a tile");
  ispa_status_t st = set_smem(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (st != ISPA_OK) return st;
  dim3 grid((p.N + L::kCols - 1) / L::kCols, (p.M + L::kRows - 1) / L::kRows, 1);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p);
  return check_launch("gemm_e4m3_kernel");
}

template <bool A_MN, bool B_MN, int BN, int NST, bool WIDE = false>
static ispa_status_t launch(const Params& p, int k_splits, cudaStream_t stream) {
  using L = Layout<BN, NST, WIDE>;
  auto kern = gemm_bf16_kernel<A_MN, B_MN, BN, NST, WIDE>;
  if (p.n_split < p.N && p.n_split % L::kCols) return unsupported("GEMM column ranges must start on a tile");
  ispa_status_t st = set_smem(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (st != ISPA_OK) return st;
  dim3 grid((p.N + L::kCols - 1) / L::kCols, (p.M + L::kRows - 1) / L::kRows, k_splits);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p);
  return check_launch("gemm_bf16_kernel");
}

// Output tile of a projection [M, N] (N a multiple of 128): 256 x 256,
// 256 x 128 or the wide 128 x 384.  Each CTA holds one tile and one CTA fits
// an SM, so the launch takes ceil(tiles / SMs) waves, each as long as one
// tile; the shape with the least wave time (tile area over a relative
// efficiency, measured on B200 at 4680 x 1536 and 4680 x 5120) wins.  A
// wide tile may overhang the last columns (its loads read zeros there and its
// stores are clipped).
enum class ProjTile : int { kTall256, kTall128, kWide192 };

static ProjTile projection_tile(int64_t M, int64_t N) {
  struct Cand {
    ProjTile t;
    int64_t rows, cols;
    double eff;
  };
  // time per tile area relative to 256 x 256, from B200 runs of one to
  // six waves: the narrower tiles re-read more operand bytes per FLOP
  const Cand cands[3] = {{ProjTile::kTall256, 256, 256, 1.0},
                         {ProjTile::kWide192, 128, 384, 0.87},
                         {ProjTile::kTall128, 256, 128, 0.75}};
  const int64_t sms = num_sms();
  ProjTile best = ProjTile::kTall128;
  double best_cost = 0.0;
  for (const Cand& c : cands) {
    if (c.t == ProjTile::kTall256 && N % 256) continue;
    const int64_t tiles = ((M + c.rows - 1) / c.rows) * ((N + c.cols - 1) / c.cols);
    const double cost = (double)((tiles + sms - 1) / sms) * (double)(c.rows * c.cols) / c.eff;
    if (best_cost == 0.0 || cost < best_cost) best = c.t, best_cost = cost;
  }
  return best;
}

}  // namespace gemm

namespace gemm {

// Tile width and token split of the statistics [G | R] (with_r) or E.  The
// row tile is 256 (two M=128 halves); the column tile BN is 256, 224 or 128
// (D % 128 == 0 is required).  Tiles: those of G that touch its lower
// triangle, plus all of R.  The token range of every tile is split in
// `splits` parts so that the launch fills one wave of SMs where it can
// (at least 8 K steps per part), and the plan with the least time per SM --
// waves x tile width x K steps per part -- wins.  The 224-wide tile (69
// tiles x 2 parts = 138 CTAs at D = 1536 instead of 57 x 2 = 114) is taken
// only for short parts (at most 64 K steps): measured on B200, it saves 10 %
// over 4680 rows, but over long token ranges, where the wave streams its
// operands from L2 at 11-13 TB/s, its more numerous CTAs and the unused
// quarter of its last B box cost more than the narrower tile saves (93600
// rows: 511 against 490 us).
// G's column range is padded to whole tiles (g_cols) so that R's starts on a
// tile; the padding columns are clipped by the output maps.
struct StatPlan {
  int BN;
  int64_t g_cols;
  int32_t k_per_split;
  int splits;
};

static StatPlan statistics_plan(int64_t D, int64_t n_rows, bool with_r) {
  const int64_t sms = num_sms();
  const int64_t k_blocks = (n_rows + kBK - 1) / kBK;
  const int widths[3] = {256, 224, 128};
  const double eff[3] = {1.0, 1.0, 0.9};  // per-area rate of each width, relative to 256
  StatPlan best{128, 0, 0, 1};
  double best_cost = -1.0;
  for (int w = 0; w < 3; ++w) {
    const int BN = widths[w];
    if (BN == 256 && D % 256) continue;
    const int64_t m_tiles = (D + kBM - 1) / kBM, n_tiles = (D + BN - 1) / BN;
    int64_t tiles = with_r ? m_tiles * n_tiles : 0;
    for (int64_t i = 0; i < m_tiles; ++i)
      for (int64_t j = 0; j < n_tiles; ++j) tiles += (j * BN <= i * kBM + kBM - 1) ? 1 : 0;
    int64_t splits = sms / tiles;
    if (splits > k_blocks / 8) splits = k_blocks / 8;
    if (splits < 1) splits = 1;
    const int64_t per = (k_blocks + splits - 1) / splits;
    if (BN == 224 && per > 64) continue;
    splits = (k_blocks + per - 1) / per;
    const int64_t waves = (tiles * splits + sms - 1) / sms;
    const double cost = (double)waves * BN * per / eff[w];
    if (best_cost < 0.0 || cost < best_cost) {
      best = {BN, n_tiles * BN, (int32_t)(per * kBK), (int)splits};
      best_cost = cost;
    }
  }
  return best;
}

static ispa_status_t launch_statistics(const Params& p, const StatPlan& sp, cudaStream_t stream) {
  if (sp.BN == 256) return launch<true, true, 256, 3>(p, sp.splits, stream);
  if (sp.BN == 224) return launch<true, true, 224, 3>(p, sp.splits, stream);
  return launch<true, true, 128, 4>(p, sp.splits, stream);
}

}  // namespace gemm

// [G | R] (+)= A_loc^T [A_loc | delta]  (bf16 inputs, fp32 outputs).  Only the
// lower triangle of G (and all of R) is produced; the K range (rows) is split
// across CTAs so that the launch fills the GPU, and the partial products are
// added into G, R in L2 (they are zeroed first when `overwrite`).
ispa_status_t gram_bf16(const void* a_loc, const void* a_delta, int64_t n_rows, int64_t D, int64_t row_stride,
                        float* G, float* R, bool overwrite, cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  // A operand: element (i, n) = A_loc[n, i]  -> [K = n_rows rows, M = D contiguous]
  if (!encode_map_bf16_2d(&p.a_map[0], a_loc, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[0][0], a_loc, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[1][0], a_delta, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  if (overwrite && (cudaMemsetAsync(G, 0, (size_t)D * D * 4, stream) != cudaSuccess ||
                    cudaMemsetAsync(R, 0, (size_t)D * D * 4, stream) != cudaSuccess))
    return check_launch("cudaMemsetAsync of G, R");
  p.M = (int32_t)D;
  p.N = (int32_t)(2 * D);
  p.K = (int32_t)n_rows;
  p.n_split = (int32_t)D;
  p.n_pairs = 1;
  p.n_cols[0] = (int32_t)(D);
  p.n_cols[1] = p.N - p.n_cols[0];
  p.lower_only0 = 1;
  p.c[0] = G;
  p.c[1] = R;
  p.ldc = D;
  p.mode = kReduceF32;
  if (!set_out_maps(p, true, D, D, D, D)) return ISPA_ERR_CUDA;
  const StatPlan sp = statistics_plan(D, n_rows, true);
  p.n_split = (int32_t)sp.g_cols;  // the R range starts on a whole tile
  p.N = p.n_split + (int32_t)D;
  p.k_per_split = sp.k_per_split;
  return launch_statistics(p, sp, stream);
}

// E (+)= X^T X (bf16 input, fp32 output): the lower triangle of a symmetric
// Gram matrix, with the same kernel, tiling and one-wave K split as gram_bf16
// but a single column range.
ispa_status_t sym_gram_bf16(const void* x, int64_t n_rows, int64_t D, int64_t row_stride, float* E, bool overwrite,
                            cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  if (!encode_map_bf16_2d(&p.a_map[0], x, D, n_rows, row_stride * 2, 64, 64)) return ISPA_ERR_CUDA;
  p.b_map[0][0] = p.a_map[0];
  p.b_map[1][0] = p.a_map[0];
  if (overwrite && cudaMemsetAsync(E, 0, (size_t)D * D * 4, stream) != cudaSuccess)
    return check_launch("cudaMemsetAsync of E");
  p.M = (int32_t)D;
  p.N = (int32_t)D;
  p.K = (int32_t)n_rows;
  p.n_split = (int32_t)D;
  p.n_pairs = 1;
  p.n_cols[0] = (int32_t)(D);
  p.n_cols[1] = p.N - p.n_cols[0];
  p.lower_only0 = 1;
  p.c[0] = E;
  p.c[1] = E;
  p.ldc = D;
  p.mode = kReduceF32;
  if (!set_out_maps(p, true, D, D, D, D)) return ISPA_ERR_CUDA;
  const StatPlan sp = statistics_plan(D, n_rows, false);
  p.n_split = (int32_t)sp.g_cols;
  p.N = (int32_t)sp.g_cols;
  p.k_per_split = sp.k_per_split;
  return launch_statistics(p, sp, stream);
}

// C[M, N] (= | +=) A[M, K] W[K, N]: bf16 row-major A and W, fp32 C (ldc).
ispa_status_t gemm_rm_bf16_f32(const void* a, int64_t M, int64_t K, int64_t a_stride, const void* w, int64_t N,
                               float* c, int64_t ldc, bool accumulate, cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  if (!encode_map_bf16_2d(&p.a_map[0], a, K, M, a_stride * 2, 64, kBM)) return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[0][0], w, N, K, N * 2, 64, 64)) return ISPA_ERR_CUDA;
  p.b_map[1][0] = p.b_map[0][0];
  p.M = (int32_t)M;
  p.N = (int32_t)N;
  p.K = (int32_t)K;
  p.n_split = (int32_t)N;
  p.n_pairs = 1;
  p.n_cols[0] = (int32_t)(N);
  p.n_cols[1] = p.N - p.n_cols[0];
  p.k_per_split = (int32_t)(((K + kBK - 1) / kBK) * kBK);
  p.c[0] = c;
  p.c[1] = c;
  p.ldc = ldc;
  p.mode = accumulate ? kReduceF32 : kStoreF32;
  if (!set_out_maps(p, true, M, ldc, N, N)) return ISPA_ERR_CUDA;
  if (N % 128) return unsupported("tensor-core GEMM needs N %% 128 == 0");
  return launch<false, true, 128, 4>(p, 1, stream);
}

// y[n_rows, d_out] = a[n_rows, d_in] * w[d_in, d_out]  (bf16 in/out).
ispa_status_t project_bf16(const void* a, int64_t n_rows, int64_t d_in, int64_t d_out, int64_t a_stride,
                           const void* w, void* y, cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  if (d_out % 128) return unsupported("bf16 projection needs d_out to be a multiple of 128 (got %lld)", (long long)d_out);
  const ProjTile t = projection_tile(n_rows, d_out);
  if (!encode_map_bf16_2d(&p.a_map[0], a, d_in, n_rows, a_stride * 2, 64, t == ProjTile::kWide192 ? 128 : kBM))
    return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&p.b_map[0][0], w, d_out, d_in, d_out * 2, 64, 64)) return ISPA_ERR_CUDA;
  p.b_map[1][0] = p.b_map[0][0];
  p.M = (int32_t)n_rows;
  p.N = (int32_t)d_out;
  p.K = (int32_t)d_in;
  p.n_split = (int32_t)d_out;
  p.n_pairs = 1;
  p.n_cols[0] = (int32_t)(d_out);
  p.n_cols[1] = p.N - p.n_cols[0];
  p.k_per_split = (int32_t)(((d_in + kBK - 1) / kBK) * kBK);
  p.c[0] = y;
  p.c[1] = y;
  p.ldc = d_out;
  p.mode = kStoreBf16;
  if (!set_out_maps(p, false, n_rows, d_out, d_out, d_out)) return ISPA_ERR_CUDA;
  switch (t) {
    case ProjTile::kWide192: return launch<false, true, 192, 3, true>(p, 1, stream);
    case ProjTile::kTall256: return launch<false, true, 256, 3>(p, 1, stream);
    default: return launch<false, true, 128, 4>(p, 1, stream);
  }
}

// y[n_rows, d_out] (bf16) = diag(a_scale) qa[n_rows, d_in] qw_t[d_out, d_in]^T diag(w_scale):
// e4m3 codes of the activations (row-major, token rows) and of the weight
// stored transposed (one row per output channel), fp32 accumulation.
ispa_status_t project_e4m3(const uint8_t* qa, const float* a_scale, int64_t n_rows, int64_t d_in,
                           const uint8_t* qw_t, const float* w_scale, int64_t d_out, void* y, cudaStream_t stream) {
  using namespace gemm;
  Params p;
  memset(&p, 0, sizeof(p));
  if (d_out % 128) return unsupported("e4m3 projection needs d_out to be a multiple of 128 (got %lld)", (long long)d_out);
  const ProjTile t = projection_tile(n_rows, d_out);
  const int BN = t == ProjTile::kWide192 ? 192 : t == ProjTile::kTall256 ? 256 : 128;
  if (!encode_map_u8_2d(&p.a_map[0], qa, d_in, n_rows, d_in, kBK8, t == ProjTile::kWide192 ? 128 : kBM))
    return ISPA_ERR_CUDA;
  if (!encode_map_u8_2d(&p.b_map[0][0], qw_t, d_in, d_out, d_in, kBK8, BN)) return ISPA_ERR_CUDA;
  p.b_map[1][0] = p.b_map[0][0];
  p.M = (int32_t)n_rows;
  p.N = (int32_t)d_out;
  p.K = (int32_t)d_in;
  p.n_split = (int32_t)d_out;
  p.n_pairs = 1;
  p.n_cols[0] = (int32_t)(d_out);
  p.n_cols[1] = p.N - p.n_cols[0];
  p.k_per_split = (int32_t)(((d_in + kBK8 - 1) / kBK8) * kBK8);
  p.c[0] = y;
  p.c[1] = y;
  p.ldc = d_out;
  p.mode = kStoreBf16;
  p.row_scale = a_scale;
  p.col_scale = w_scale;
  if (!set_out_maps(p, false, n_rows, d_out, d_out, d_out)) return ISPA_ERR_CUDA;
  if (!p.c_tma) return unsupported("e4m3 projection needs a 16-byte aligned output");
  switch (t) {
    case ProjTile::kWide192: return launch_e4m3<192, 3, true>(p, stream);
    case ProjTile::kTall256: return launch_e4m3<256, 3>(p, stream);
    default: return launch_e4m3<128, 4>(p, stream);
  }
}

// y[n_rows, d_out] (bf16) = block-scaled product of MX activation codes
// qa [n_rows, d_in] with exponent bytes ea [n_rows, d_in / 32] (ue8m0) and the
// per-channel weight codes qw_t [d_out, d_in] with w_scale [d_out]:
// y[i, j] = w_scale[j] * sum_b 2^(ea[i, b] - 127) sum_{k in b} qa[i, k] qw[k, j].
ispa_status_t project_mx(const uint8_t* qa, const uint8_t* ea, int64_t n_rows, int64_t d_in, const uint8_t* qw_t,
                         const float* w_scale, int64_t d_out, void* y, cudaStream_t stream) {
  using namespace gemm;
  if (d_in % kBK8 || d_in / kBK8 > kMxMaxStages)
    return unsupported("block-scaled projection needs d_in to be a multiple of 128 up to %d (got %lld)",
                       kMxMaxStages * kBK8, (long long)d_in);
  if (d_out % 128) return unsupported("block-scaled projection needs d_out %% 128 == 0 (got %lld)", (long long)d_out);
  Params p;
  memset(&p, 0, sizeof(p));
  if (!encode_map_u8_2d(&p.a_map[0], qa, d_in, n_rows, d_in, kBK8, 128)) return ISPA_ERR_CUDA;
  if (!encode_map_u8_2d(&p.b_map[0][0], qw_t, d_in, d_out, d_in, kBK8, 192)) return ISPA_ERR_CUDA;
  p.b_map[1][0] = p.b_map[0][0];
  p.M = (int32_t)n_rows;
  p.N = (int32_t)d_out;
  p.K = (int32_t)d_in;
  p.n_split = (int32_t)d_out;
  p.n_pairs = 1;
  p.n_cols[0] = (int32_t)d_out;
  p.k_per_split = (int32_t)d_in;
  p.c[0] = y;
  p.c[1] = y;
  p.ldc = d_out;
  p.mode = kStoreBf16;
  p.row_scale = nullptr;
  p.col_scale = w_scale;
  p.a_exps = ea;
  p.exps_ld = (int32_t)(d_in / 32);
  if (!set_out_maps(p, false, n_rows, d_out, d_out, d_out)) return ISPA_ERR_CUDA;
  if (!p.c_tma) return unsupported("block-scaled projection needs a 16-byte aligned output");
  return launch_e4m3<192, 3, true, true>(p, stream);
}

}  // namespace ispa

// ------------------------------------------------------- absorb products
// Split-precision products of the absorb solve.  An fp32 operand x is held as
// two bf16 matrices hi = bf16(x), lo = bf16(x - hi); a product of two such
// operands is summed in one accumulator as hi(A) hi(B) + hi(A) lo(B) +
// lo(A) hi(B) (the dropped lo(A) lo(B) and the representation error are about
// 2^-17 of |A| |B|).
namespace ispa {

// One trailing update of the blocked Cholesky with its right-hand sides
// (panel width 64, rows and columns from `off`):
//   M[off:, off + m_col0:] (lower tiles) += A  [L^T](:, m_col0:)   A = -L21 (rows x 64),
//   RHS[off:, :rhs_cols]                 += A  Y_k                 Y_k (64 x rhs_cols),
// A given as K-major hi/lo [rows, 64]; L21^T as MN-major hi/lo [64, rows]
// with row stride lt_ld; Y_k as MN-major hi/lo [64, rhs_cols] with row stride
// y_ld.  M has row stride D, RHS row stride rhs_ld (fp32, reduced in L2).
// m_col0 (a multiple of 64) leaves the first trailing columns to the caller.
ispa_status_t absorb_step_update(int64_t rows, int64_t m_col0, const void* a_hi, const void* a_lo,
                                 const void* lt_hi, const void* lt_lo, int64_t lt_ld, const void* y_hi,
                                 const void* y_lo, int64_t y_ld, int64_t rhs_cols, float* m_sub, int64_t m_ld,
                                 float* rhs_sub, int64_t rhs_ld, cudaStream_t stream) {
  using namespace gemm;
  constexpr int BN = 128;
  if (m_col0 < 0 || m_col0 > rows || m_col0 % 64) return unsupported("absorb update: first trailing column");
  const int64_t m_cols = rows - m_col0;  // trailing columns this product updates
  Params p;
  memset(&p, 0, sizeof(p));
  CUtensorMap ah, al, bh0, bl0, bh1, bl1;
  if (!encode_map_bf16_2d(&ah, a_hi, 64, rows, 128, 64, kBM) || !encode_map_bf16_2d(&al, a_lo, 64, rows, 128, 64, kBM))
    return ISPA_ERR_CUDA;
  // with no trailing column left the first range is empty and its maps are
  // never read: they are encoded over the whole block so that they are valid
  const int64_t b0 = m_cols > 0 ? m_col0 : 0, nb0 = m_cols > 0 ? m_cols : rows;
  if (!encode_map_bf16_2d(&bh0, static_cast<const __nv_bfloat16*>(lt_hi) + b0, nb0, 64, lt_ld * 2, 64, 64) ||
      !encode_map_bf16_2d(&bl0, static_cast<const __nv_bfloat16*>(lt_lo) + b0, nb0, 64, lt_ld * 2, 64, 64))
    return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&bh1, y_hi, rhs_cols, 64, y_ld * 2, 64, 64) ||
      !encode_map_bf16_2d(&bl1, y_lo, rhs_cols, 64, y_ld * 2, 64, 64))
    return ISPA_ERR_CUDA;
  p.a_map[0] = ah, p.a_map[1] = ah, p.a_map[2] = al;
  p.b_map[0][0] = bh0, p.b_map[0][1] = bl0, p.b_map[0][2] = bh0;
  p.b_map[1][0] = bh1, p.b_map[1][1] = bl1, p.b_map[1][2] = bh1;
  p.n_pairs = 3;
  if (!encode_map_out_2d(&p.c_map[0], m_sub + b0, true, nb0, rows, m_ld * 4) ||
      !encode_map_out_2d(&p.c_map[1], rhs_sub, true, rhs_cols, rows, rhs_ld * 4))
    return ISPA_ERR_CUDA;
  p.c_tma = 1;
  p.c[0] = m_sub + b0;
  p.c[1] = rhs_sub;
  p.M = (int32_t)rows;
  p.K = 64;
  p.k_per_split = 64;
  p.n_split = (int32_t)((m_cols + BN - 1) / BN * BN);  // range 0 padded to whole tiles
  p.N = p.n_split + (int32_t)rhs_cols;
  p.n_cols[0] = (int32_t)m_cols;
  p.n_cols[1] = (int32_t)rhs_cols;
  // tiles wholly above the diagonal are skipped; the column shift only makes
  // the test keep a few more tiles than the triangle needs
  p.lower_only0 = 1;
  p.mode = kReduceF32;
  return launch<false, true, BN, 4>(p, 1, stream);
}

// C[D, N] += sum of split-precision pairs of A^T B, A = X [K, D] lower
// triangular (so A^T is upper: a row block of C skips the K rows above it),
// B [K, N]; hi/lo bf16 row-major with row strides x_ld, y_ld; C fp32 (ldc),
// which the caller zeroes (the K range is split across CTAs, reduced in L2).
ispa_status_t gemm_split3_xt_y(int64_t D, int64_t N, const void* x_hi, const void* x_lo, int64_t x_ld,
                               const void* y_hi, const void* y_lo, int64_t y_ld, float* c, int64_t ldc,
                               cudaStream_t stream) {
  using namespace gemm;
  constexpr int BN = 128;
  Params p;
  memset(&p, 0, sizeof(p));
  CUtensorMap xh, xl, yh, yl;
  if (!encode_map_bf16_2d(&xh, x_hi, D, D, x_ld * 2, 64, 64) || !encode_map_bf16_2d(&xl, x_lo, D, D, x_ld * 2, 64, 64))
    return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&yh, y_hi, N, D, y_ld * 2, 64, 64) || !encode_map_bf16_2d(&yl, y_lo, N, D, y_ld * 2, 64, 64))
    return ISPA_ERR_CUDA;
  p.a_map[0] = xh, p.a_map[1] = xh, p.a_map[2] = xl;
  p.b_map[0][0] = yh, p.b_map[0][1] = yl, p.b_map[0][2] = yh;
  for (int q = 0; q < 3; ++q) p.b_map[1][q] = p.b_map[0][q];
  p.n_pairs = 3;
  p.a_upper = 1;
  p.c[0] = c;
  p.c[1] = c;
  p.ldc = ldc;
  p.M = (int32_t)D;
  p.N = (int32_t)N;
  p.K = (int32_t)D;
  p.n_split = (int32_t)N;
  p.n_cols[0] = (int32_t)N;
  p.mode = kReduceF32;
  if (!encode_map_out_2d(&p.c_map[0], c, true, N, D, ldc * 4)) return ISPA_ERR_CUDA;
  p.c_map[1] = p.c_map[0];
  p.c_tma = 1;
  // two K halves per tile: the 6 x 12 tiles of D = 1536 then fill the GPU
  const int64_t k_blocks = (D + kBK - 1) / kBK;
  const int64_t per = (k_blocks + 1) / 2;
  p.k_per_split = (int32_t)(per * kBK);
  return launch<true, true, BN, 4>(p, (int)((k_blocks + per - 1) / per), stream);
}

// C[M, N] += A B for two fp32 matrices held as bf16 hi/lo pairs (A [M, K]
// row-major with row stride lda, B [K, N] row-major with row stride ldb),
// summed as hi(A) hi(B) + hi(A) lo(B) + lo(A) hi(B) in one accumulator; C fp32
// (ldc), zeroed by the caller.  Two K halves per tile, reduced in L2.
ispa_status_t gemm_split3(int64_t M, int64_t N, int64_t K, const void* a_hi, const void* a_lo, int64_t lda,
                          const void* b_hi, const void* b_lo, int64_t ldb, float* c, int64_t ldc,
                          cudaStream_t stream) {
  using namespace gemm;
  constexpr int BN = 128;
  if (N % BN) return unsupported("split-precision product needs N %% 128 == 0");
  Params p;
  memset(&p, 0, sizeof(p));
  CUtensorMap ah, al, bh, bl;
  if (!encode_map_bf16_2d(&ah, a_hi, K, M, lda * 2, 64, kBM) || !encode_map_bf16_2d(&al, a_lo, K, M, lda * 2, 64, kBM))
    return ISPA_ERR_CUDA;
  if (!encode_map_bf16_2d(&bh, b_hi, N, K, ldb * 2, 64, 64) || !encode_map_bf16_2d(&bl, b_lo, N, K, ldb * 2, 64, 64))
    return ISPA_ERR_CUDA;
  p.a_map[0] = ah, p.a_map[1] = ah, p.a_map[2] = al;
  p.b_map[0][0] = bh, p.b_map[0][1] = bl, p.b_map[0][2] = bh;
  for (int q = 0; q < 3; ++q) p.b_map[1][q] = p.b_map[0][q];
  p.n_pairs = 3;
  p.c[0] = c;
  p.c[1] = c;
  p.ldc = ldc;
  p.M = (int32_t)M;
  p.N = (int32_t)N;
  p.K = (int32_t)K;
  p.n_split = (int32_t)N;
  p.n_cols[0] = (int32_t)N;
  p.mode = kReduceF32;
  if (!encode_map_out_2d(&p.c_map[0], c, true, N, M, ldc * 4)) return ISPA_ERR_CUDA;
  p.c_map[1] = p.c_map[0];
  p.c_tma = 1;
  const int64_t k_blocks = (K + kBK - 1) / kBK;
  const int64_t per = (k_blocks + 1) / 2;
  p.k_per_split = (int32_t)(per * kBK);
  return launch<false, true, BN, 4>(p, (int)((k_blocks + per - 1) / per), stream);
}

// C[M, N] += (a_hi + a_lo) W, W exactly bf16 [K, N] row-major; a_hi / a_lo
// bf16 [M, K] row-major; C fp32 (ldc), zeroed by the caller.  Two K halves
// per tile, reduced in L2.
ispa_status_t gemm_hilo_w(int64_t M, int64_t K, const void* a_hi, const void* a_lo, const void* w, int64_t N,
                          float* c, int64_t ldc, cudaStream_t stream) {
  using namespace gemm;
  constexpr int BN = 128;
  Params p;
  memset(&p, 0, sizeof(p));
  if (!encode_map_bf16_2d(&p.a_map[0], a_hi, K, M, K * 2, 64, kBM) ||
      !encode_map_bf16_2d(&p.a_map[1], a_lo, K, M, K * 2, 64, kBM) ||
      !encode_map_bf16_2d(&p.b_map[0][0], w, N, K, N * 2, 64, 64))
    return ISPA_ERR_CUDA;
  p.b_map[0][1] = p.b_map[0][0];
  p.b_map[1][0] = p.b_map[1][1] = p.b_map[0][0];
  p.n_pairs = 2;
  p.c[0] = c;
  p.c[1] = c;
  p.ldc = ldc;
  p.M = (int32_t)M;
  p.N = (int32_t)N;
  p.K = (int32_t)K;
  p.n_split = (int32_t)N;
  p.n_cols[0] = (int32_t)N;
  p.mode = kReduceF32;
  if (!encode_map_out_2d(&p.c_map[0], c, true, N, M, ldc * 4)) return ISPA_ERR_CUDA;
  p.c_map[1] = p.c_map[0];
  p.c_tma = 1;
  const int64_t k_blocks = (K + kBK - 1) / kBK;
  const int64_t per = (k_blocks + 1) / 2;
  p.k_per_split = (int32_t)(per * kBK);
  return launch<false, true, BN, 4>(p, (int)((k_blocks + per - 1) / per), stream);
}

}  // namespace ispa
