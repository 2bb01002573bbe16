// Decomposable (dual-stream) attention on sm_100a tensor cores.
//
// Computes, for one chunk of queries, attention over a local key set (sink +
// current chunk) and over the evicted history as two online-softmax branches
// that each keep their log-sum-exp state, then fuses them in the epilogue
// ("Towards Memory-Efficient Autoregressive Video Generation via
// Instance-Specific Parametric Absorption", gist.science technical summary,
// section 2 stage 1 "Dual-Stream Warmup", and section 3 item 2).
//
// One CTA owns 128 query rows of one head.  Its 12 warps:
//   warp 0      TMA producer: Q once, then K/V tiles of 128 keys into a ring
//               of NST shared-memory stages;
//   warp 1      tcgen05 issuer: S = Q K^T (both operands K-major in shared
//               memory) and O += P V (P from tensor memory, V MN-major);
//   warp 2      allocates / frees the 512 tensor-memory columns;
//   warps 4-7   softmax "slot A", warps 8-11 softmax "slot B".  Each slot owns
//               a 128-column S buffer (P aliased into it as bf16) and a
//               head_dim-column O accumulator in tensor memory; the two slots
//               work on disjoint tile ranges so the tensor core alternates
//               between them while the other slot runs its softmax.
// Tile schedule: the local tiles come first, then the history tiles.  Slot A
// takes [0, cut), slot B takes [cut, T).  In dual mode slot A always finishes
// the local branch first; when it continues into history tiles it writes
// A_loc and LSE_loc to global memory at the branch boundary and restarts its
// accumulator; the epilogue merges the history partials of both slots and
// then fuses the merged history with A_loc.
// Online softmax works in the log2 domain with a lazily updated row maximum:
// O is rescaled only when the running maximum grows by more than 2^8.
#include <cstring>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace attn {

constexpr int kBM = 128;       // query rows per CTA (= tensor-memory lanes)
constexpr int kBN = 128;       // keys per tile
constexpr int kThreads = 384;  // 12 warps
constexpr int kMaxSeg = ISPA_MAX_SEGMENTS;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;
// bit j set: column pair j (mod 8) of a score row takes 2^x from exp2_fma2
constexpr uint32_t kEmuPairs = 0x00u;

struct Params {
  CUtensorMap q_map;
  CUtensorMap k_map[kMaxSeg];
  CUtensorMap v_map[kMaxSeg];
  int32_t seg_tokens[kMaxSeg];
  int32_t seg_first_tile[kMaxSeg + 1];
  int32_t n_seg;
  int32_t n_local_tiles;
  int32_t n_tiles;
  int32_t cut;
  int32_t dual;
  int32_t n_q;
  float scale_log2;
  __nv_bfloat16* a_loc;
  __nv_bfloat16* a_full;
  __nv_bfloat16* a_delta;
  float* lse_loc;
  float* lse_full;
  int64_t out_stride;
  int32_t* status;
};

template <int HD, int NST>
struct Layout {
  static constexpr int kTileBytes = kBN * HD * 2;  // one K, V or Q tile
  static constexpr int kBoxBytes = kBN * 128;      // 128 rows x 64 bf16 (one 128-byte swizzle column block)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + NST * kTileBytes;
  static constexpr int kXch = kV + NST * kTileBytes;  // slot-B row statistics: 2 x 128 floats
  static constexpr int kBars = kXch + 2 * kBM * 4;
  // q_full, kv_full[NST], kv_empty[NST], s_full[2], p_full[2], o_done[2], x_ready, teardown
  static constexpr int kNumBars = 1 + 2 * NST + 2 + 2 + 2 + 1 + 1;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 bytes
  static_assert(kAlloc <= 232448, "shared memory budget");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tile_info(const Params& p, int t, int& seg, int& tok0, int& valid) {
  seg = 0;
#pragma unroll 1
  while (seg + 1 < p.n_seg && t >= p.seg_first_tile[seg + 1]) ++seg;
  tok0 = (t - p.seg_first_tile[seg]) * kBN;
  valid = min(kBN, p.seg_tokens[seg] - tok0);
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&x)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 u = s4[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[v * 8 + 2 * e] = __uint_as_float(w[e] << 16);
      x[v * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&x)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 u;
    u.x = pack_bf16x2(x[v * 8 + 0], x[v * 8 + 1]);
    u.y = pack_bf16x2(x[v * 8 + 2], x[v * 8 + 3]);
    u.z = pack_bf16x2(x[v * 8 + 4], x[v * 8 + 5]);
    u.w = pack_bf16x2(x[v * 8 + 6], x[v * 8 + 7]);
    d4[v] = u;
  }
}

// ------------------------------------------------------------------ producer
template <int HD, int NST>
__device__ void producer(const Params& p, uint8_t* smem, uint64_t* q_full, uint64_t* kv_full, uint64_t* kv_empty,
                         volatile int* abort_flag, int q0, int head, int nA, int nB) {
  using L = Layout<HD, NST>;
  tma_prefetch_desc(&p.q_map);
  mbar_arrive_expect_tx(q_full, L::kTileBytes);
#pragma unroll
  for (int c = 0; c < HD / 64; ++c)
    tma_load_2d(smem + L::kQ + c * L::kBoxBytes, &p.q_map, q_full, head * HD + 64 * c, q0);
  int n = 0, ia = 0, ib = 0;
  bool ok = true;
  while (ok && (ia < nA || ib < nB)) {
#pragma unroll 1
    for (int s = 0; s < 2; ++s) {
      int t;
      if (s == 0) {
        if (ia >= nA) continue;
        t = ia++;
      } else {
        if (ib >= nB) continue;
        t = nA + ib++;
      }
      const int stage = n % NST;
      if (n >= NST && !mbar_wait(&kv_empty[stage], ((n / NST) - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      int seg, tok0, valid;
      tile_info(p, t, seg, tok0, valid);
      mbar_arrive_expect_tx(&kv_full[stage], 2 * L::kTileBytes);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) {
        tma_load_2d(smem + L::kK + stage * L::kTileBytes + c * L::kBoxBytes, &p.k_map[seg], &kv_full[stage],
                    head * HD + 64 * c, tok0);
        tma_load_2d(smem + L::kV + stage * L::kTileBytes + c * L::kBoxBytes, &p.v_map[seg], &kv_full[stage],
                    head * HD + 64 * c, tok0);
      }
      ++n;
    }
  }
  if (!ok) {
    // unwinding: wait (bounded) for every copy still in flight before exit
    mbar_wait_drain(q_full, 0, 100000000ull);
    for (int j = n > NST ? n - NST : 0; j < n; ++j) mbar_wait_drain(&kv_full[j % NST], (j / NST) & 1, 100000000ull);
  }
}

// ------------------------------------------------------------- MMA issuer
template <int HD, int NST>
__device__ void mma_issuer(const Params& p, uint8_t* smem, uint64_t* q_full, uint64_t* kv_full, uint64_t* kv_empty,
                           uint64_t* s_full, uint64_t* p_full, uint64_t* o_done, uint64_t* teardown,
                           volatile int* abort_flag, uint32_t tmem, int nA, int nB) {
  using L = Layout<HD, NST>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, false, true);
  const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
  const int n_loc = p.n_local_tiles;
  int n_s = 0;
  int stage_of[2] = {0, 0};

  auto issue_s = [&](int s) -> bool {
    const int stage = n_s % NST;
    if (!mbar_wait(&kv_full[stage], (n_s / NST) & 1, abort_flag)) return false;
    tc_fence_after();
    const uint32_t kb = sK + stage * L::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
      umma_ss(tmem + s * 128, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), kIdescQK,
              kk > 0 ? 1u : 0u);
    }
    umma_commit(&s_full[s]);
    stage_of[s] = stage;
    ++n_s;
    return true;
  };
  auto issue_pv = [&](int s, int i, bool last) -> bool {
    if (!mbar_wait(&p_full[s], i & 1, abort_flag)) return false;
    tc_fence_after();
    const bool fresh = (i == 0) || (p.dual && s == 0 && i == n_loc);
    const uint32_t vb = sV + stage_of[s] * L::kTileBytes;
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
      umma_ts(tmem + 256 + s * 128, tmem + s * 128 + 32 + kk * 8, sdesc_sw128(vb + kk * 2048, L::kBoxBytes, 1024),
              kIdescPV, (kk > 0 || !fresh) ? 1u : 0u);
    }
    umma_commit(&kv_empty[stage_of[s]]);
    if (last) umma_commit(&o_done[s]);
    return true;
  };

  bool ok = mbar_wait(q_full, 0, abort_flag);
  tc_fence_after();
  if (ok && nA > 0) ok = issue_s(0);
  if (ok && nB > 0) ok = issue_s(1);
  int pa = 0, pb = 0;
  while (ok && (pa < nA || pb < nB)) {
    if (pa < nA) {
      ok = issue_pv(0, pa, pa + 1 == nA);
      ++pa;
      if (ok && pa < nA) ok = issue_s(0);
    }
    if (ok && pb < nB) {
      ok = issue_pv(1, pb, pb + 1 == nB);
      ++pb;
      if (ok && pb < nB) ok = issue_s(1);
    }
  }
  // every MMA must have completed before tensor memory is released
  umma_commit(teardown);
  mbar_wait_drain(teardown, 0, 100000000ull);
}

// ------------------------------------------------------------------ softmax
// Normalises the slot-A accumulator into A_loc (bf16, global) and LSE_loc.
// Returns LSE_loc in log2 units.
template <int HD>
__device__ float write_local(const Params& p, uint32_t o_addr, float m, float l, int grow, int head, bool row_ok) {
  const float inv = 1.0f / l;
  __nv_bfloat16* dst = p.a_loc + (int64_t)grow * p.out_stride + head * HD;
#pragma unroll 1
  for (int c = 0; c < HD / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(o_addr + 32 * c, r);
    tmem_wait_ld();
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(r[j]) * inv;
    if (row_ok) store_bf16x32(dst + 32 * c, x);
  }
  const float lse2 = m + log2f(l);
  if (row_ok && p.lse_loc) p.lse_loc[(int64_t)head * p.n_q + grow] = lse2 * kLn2;
  return lse2;
}

template <int HD, int NST>
__device__ void softmax_slot(const Params& p, uint8_t* smem, int s, uint32_t tmem, uint64_t* s_full,
                             uint64_t* p_full, uint64_t* o_done, uint64_t* x_ready, volatile int* abort_flag, int q0,
                             int head, int nA, int nB) {
  using L = Layout<HD, NST>;
  float* xch = reinterpret_cast<float*>(smem + L::kXch);
  const int wq = (threadIdx.x >> 5) & 3;  // tensor-memory lane quadrant of this warp
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;
  const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t s_addr = lane_base + s * 128;
  const uint32_t p_addr = s_addr + 32;
  const uint32_t oA = lane_base + 256, oB = lane_base + 384;
  const uint32_t o_addr = s == 0 ? oA : oB;
  const int n_my = s == 0 ? nA : nB;
  const int t_begin = s == 0 ? 0 : nA;
  const int n_loc = p.n_local_tiles;
  const bool dual = p.dual != 0;
  const int grow = q0 + row;
  const bool row_ok = grow < p.n_q;
  const float sl2 = p.scale_log2;

  float m_used = -INFINITY, l = 0.f;
  float lse_loc2 = 0.f;
  bool ok = true;

#pragma unroll 1
  for (int i = 0; i < n_my; ++i) {
    ok = __all_sync(0xffffffffu, mbar_wait(&s_full[s], i & 1, abort_flag));
    if (!ok) break;
    tc_fence_after();
    const bool boundary = dual && s == 0 && i == n_loc && i > 0;
    if (boundary) {
      lse_loc2 = write_local<HD>(p, oA, m_used, l, grow, head, row_ok);
      m_used = -INFINITY;
      l = 0.f;
    }
    const bool fresh = (i == 0) || boundary;
    int seg, tok0, valid;
    tile_info(p, t_begin + i, seg, tok0, valid);

    uint32_t r[4][32];
    tmem_ld32(s_addr, r[0]);
    tmem_ld32(s_addr + 32, r[1]);
    tmem_ld32(s_addr + 64, r[2]);
    tmem_ld32(s_addr + 96, r[3]);
    tmem_wait_ld();
    if (valid < kBN) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j >= valid) r[c][j] = __float_as_uint(-INFINITY);
    }
    // row maximum: four independent three-input chains, then combined
    float mc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mc[c] = fmaxf(__uint_as_float(r[c][0]), __uint_as_float(r[c][1]));
#pragma unroll
      for (int j = 1; j < 16; ++j) mc[c] = fmax3(mc[c], __uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1]));
    }
    const float m_tile = fmax3(mc[0], mc[1], fmaxf(mc[2], mc[3])) * sl2;
    if (fresh) {
      m_used = m_tile;
    } else if (__any_sync(0xffffffffu, m_tile > m_used + kRescaleLog2)) {
      const float m_new = fmaxf(m_used, m_tile);
      const float f = fast_exp2(m_used - m_new);
      l *= f;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_addr + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
        tmem_st32(o_addr + 32 * c, o);
      }
      tmem_wait_st();
      m_used = m_new;
    }
    // P = 2^(s * scale_log2 - m): pairs of columns with packed fp32 math; a
    // fixed quarter of the pairs evaluate 2^x on the FMA pipe (kEmuPairs) to
    // relieve the MUFU pipe, the rest use ex2.approx.
    const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_used, -m_used);
    float2 sum2[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      sum2[c] = make_float2(0.f, 0.f);
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 x = ffma2(make_float2(__uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1])), sc2, nm2);
        float2 pv;
        if (kEmuPairs & (1u << (j & 7))) {
          pv = exp2_fma2(x);
        } else {
          pv.x = fast_exp2(x.x);
          pv.y = fast_exp2(x.y);
        }
        sum2[c] = fadd2(sum2[c], pv);
        pk[j] = pack_bf16x2(pv.x, pv.y);
      }
      tmem_st16(p_addr + 16 * c, pk);
    }
    const float2 s01 = fadd2(sum2[0], sum2[1]), s23 = fadd2(sum2[2], sum2[3]);
    const float sum = (s01.x + s01.y) + (s23.x + s23.y);
    tmem_wait_st();
    l += sum;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&p_full[s]);
  }
  if (ok && n_my > 0) {
    ok = __all_sync(0xffffffffu, mbar_wait(&o_done[s], 0, abort_flag));
    tc_fence_after();
  }

  if (s == 1) {  // publish this slot's row statistics for the epilogue
    xch[row] = m_used;
    xch[kBM + row] = l;
    mbar_arrive(x_ready);
    return;
  }
  if (!ok) return;
  ok = __all_sync(0xffffffffu, mbar_wait(x_ready, 0, abort_flag));
  if (ok && nB > 0) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[1], 0, abort_flag));
  if (!ok || *abort_flag) return;
  tc_fence_after();
  const float mB = xch[row], lB = xch[kBM + row];

  if (dual) {
    bool hasA = true;  // slot A holds history tiles
    if (nA == n_loc) {
      lse_loc2 = write_local<HD>(p, oA, m_used, l, grow, head, row_ok);
      hasA = false;
    }
    const bool hasB = nB > 0;
    const float mA = hasA ? m_used : -INFINITY;
    const float lA = hasA ? l : 0.f;
    const bool any_hist = hasA || hasB;
    const float mh = fmaxf(mA, mB);
    const float fA = hasA ? fast_exp2(mA - mh) : 0.f;
    const float fB = hasB ? fast_exp2(mB - mh) : 0.f;
    const float lh = lA * fA + lB * fB;
    float w = 0.f, inv_lh = 0.f, lse_full2 = lse_loc2;
    if (any_hist) {
      const float lse_h2 = mh + log2f(lh);
      const float mm = fmaxf(lse_loc2, lse_h2);
      lse_full2 = mm + log2f(exp2f(lse_loc2 - mm) + exp2f(lse_h2 - mm));
      w = exp2f(lse_h2 - lse_full2);
      inv_lh = 1.0f / lh;
    }
    const __nv_bfloat16* aloc = p.a_loc + (int64_t)grow * p.out_stride + head * HD;
    __nv_bfloat16* afull = p.a_full + (int64_t)grow * p.out_stride + head * HD;
    __nv_bfloat16* adelta = p.a_delta ? p.a_delta + (int64_t)grow * p.out_stride + head * HD : nullptr;
#pragma unroll 1
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t ra[32], rb[32];
      if (hasA) tmem_ld32(oA + 32 * c, ra);
      if (hasB) tmem_ld32(oB + 32 * c, rb);
      tmem_wait_ld();
      if (!row_ok) continue;
      float a[32], full[32], dl[32];
      load_bf16x32(aloc + 32 * c, a);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float oh = 0.f;
        if (hasA) oh += __uint_as_float(ra[j]) * fA;
        if (hasB) oh += __uint_as_float(rb[j]) * fB;
        oh *= inv_lh;
        dl[j] = any_hist ? w * (oh - a[j]) : 0.f;
        full[j] = a[j] + dl[j];
      }
      store_bf16x32(afull + 32 * c, full);
      if (adelta) store_bf16x32(adelta + 32 * c, dl);
    }
    if (row_ok && p.lse_full) p.lse_full[(int64_t)head * p.n_q + grow] = lse_full2 * kLn2;
  } else {
    const bool hasA = nA > 0, hasB = nB > 0;
    const float mA = hasA ? m_used : -INFINITY;
    const float lA = hasA ? l : 0.f;
    const float mm = fmaxf(mA, mB);
    const float fA = hasA ? fast_exp2(mA - mm) : 0.f;
    const float fB = hasB ? fast_exp2(mB - mm) : 0.f;
    const float lt = lA * fA + lB * fB;
    const float inv = 1.0f / lt;
    __nv_bfloat16* afull = p.a_full + (int64_t)grow * p.out_stride + head * HD;
#pragma unroll 1
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t ra[32], rb[32];
      if (hasA) tmem_ld32(oA + 32 * c, ra);
      if (hasB) tmem_ld32(oB + 32 * c, rb);
      tmem_wait_ld();
      if (!row_ok) continue;
      float o[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float v = 0.f;
        if (hasA) v += __uint_as_float(ra[j]) * fA;
        if (hasB) v += __uint_as_float(rb[j]) * fB;
        o[j] = v * inv;
      }
      store_bf16x32(afull + 32 * c, o);
    }
    if (row_ok && p.lse_full) p.lse_full[(int64_t)head * p.n_q + grow] = (mm + log2f(lt)) * kLn2;
  }
}

// ------------------------------------------------------------------- kernel
template <int HD, int NST>
__global__ void __launch_bounds__(kThreads, 1) dual_attention_kernel(const __grid_constant__ Params p) {
  using L = Layout<HD, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* s_full = kv_empty + NST;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* x_ready = o_done + 2;
  uint64_t* teardown = x_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kBM, head = blockIdx.y;
  const int nA = p.cut, nB = p.n_tiles - p.cut;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);
      mbar_init(&o_done[s], 1);
    }
    mbar_init(x_ready, 128);
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer<HD, NST>(p, smem, q_full, kv_full, kv_empty, abort_flag, q0, head, nA, nB);
  } else if (warp == 1) {
    if (lane == 0)
      mma_issuer<HD, NST>(p, smem, q_full, kv_full, kv_empty, s_full, p_full, o_done, teardown, abort_flag, tmem, nA,
                          nB);
  } else if (warp >= 4) {
    softmax_slot<HD, NST>(p, smem, (warp - 4) >> 2, tmem, s_full, p_full, o_done, x_ready, abort_flag, q0, head, nA,
                          nB);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
  if (threadIdx.x == 0 && *abort_flag) report_status(p.status, ISPA_ERR_TIMEOUT);
}

template <int HD, int NST>
static ispa_status_t launch(Params& p, int n_heads, cudaStream_t stream) {
  using L = Layout<HD, NST>;
  auto kern = dual_attention_kernel<HD, NST>;
  ispa_status_t st = set_smem(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (st != ISPA_OK) return st;
  dim3 grid((p.n_q + kBM - 1) / kBM, n_heads);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p);
  return check_launch("dual_attention_kernel");
}

}  // namespace attn

// Host entry used by the C ABI for bf16 activations.  Segments with zero
// tokens must already be removed; local segments come first.
ispa_status_t dual_attention_bf16(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim,
                                  float scale, const ispa_kv_segment_t* segs, int n_local_seg, int n_hist_seg,
                                  void* a_loc, void* a_full, void* a_delta, float* lse_loc, float* lse_full,
                                  int32_t* status, cudaStream_t stream) {
  using namespace attn;
  static_assert(sizeof(Params) <= 32764, "kernel parameter space");
  Params p;
  memset(&p, 0, sizeof(p));
  const int64_t D = (int64_t)n_heads * head_dim;
  if (!encode_map_bf16_2d(&p.q_map, q, D, n_q, q_stride * 2, 64, kBM)) return ISPA_ERR_CUDA;
  const int n_seg = n_local_seg + n_hist_seg;
  int tiles = 0, local_tiles = 0;
  for (int i = 0; i < n_seg; ++i) {
    if (!encode_map_bf16_2d(&p.k_map[i], segs[i].k, D, segs[i].n_tokens, segs[i].row_stride * 2, 64, kBN))
      return ISPA_ERR_CUDA;
    if (!encode_map_bf16_2d(&p.v_map[i], segs[i].v, D, segs[i].n_tokens, segs[i].row_stride * 2, 64, kBN))
      return ISPA_ERR_CUDA;
    p.seg_tokens[i] = (int32_t)segs[i].n_tokens;
    p.seg_first_tile[i] = tiles;
    tiles += (int)((segs[i].n_tokens + kBN - 1) / kBN);
    if (i + 1 == n_local_seg) local_tiles = tiles;
  }
  p.seg_first_tile[n_seg] = tiles;
  p.n_seg = n_seg;
  p.n_tiles = tiles;
  p.n_local_tiles = local_tiles;
  p.dual = a_loc != nullptr;
  if (p.dual) {
    const int hist_tiles = tiles - local_tiles;
    p.cut = hist_tiles > local_tiles ? local_tiles + (hist_tiles - local_tiles) / 2 : local_tiles;
  } else {
    p.cut = (tiles + 1) / 2;
  }
  p.n_q = (int32_t)n_q;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.a_loc = static_cast<__nv_bfloat16*>(a_loc);
  p.a_full = static_cast<__nv_bfloat16*>(a_full);
  p.a_delta = static_cast<__nv_bfloat16*>(a_delta);
  p.lse_loc = lse_loc;
  p.lse_full = lse_full;
  p.out_stride = D;
  p.status = status;
  if (head_dim == 128) return launch<128, 3>(p, n_heads, stream);
  return launch<64, 6>(p, n_heads, stream);
}

}  // namespace ispa
