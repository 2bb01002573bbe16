// Decomposable (dual-stream) attention on sm_100a tensor cores.
//
// For one chunk of queries: attention over a local key set (sink + current
// chunk) and over the evicted history, each an online softmax that keeps its
// log-sum-exp, fused post hoc in the epilogue ("Towards Memory-Efficient
// Autoregressive Video Generation via Instance-Specific Parametric
// Absorption", gist.science technical summary, section 2 stage 1
// "Dual-Stream Warmup", and section 3 item 2).
//
// One CTA owns 128 query rows of one head and walks the key tiles (128 keys)
// of the local segments first, then of the history segments.
//   warps 0, 3  TMA producers: Q and the K tiles (warp 0), the V tiles
//               (warp 3), each into its own NST-stage ring (a K tile is
//               released once S(j) is done, a V tile after PV(j));
//   warp 1      tcgen05 issuer, the whole warp converged, one elected lane
//               issuing: S(j) = Q K(j)^T (both operands K-major in shared
//               memory) and O_w += P(j) V(j) (P from tensor memory, V
//               MN-major in shared memory);
//   warp 2      allocates / frees the 512 tensor-memory columns;
//   warps 4-11  softmax: two warpgroups; warpgroup w owns the key tiles
//               j = w mod 2; thread = query row = TMEM lane.
// Tensor memory: one S buffer and one O accumulator per warpgroup
// (2 x 128 + 2 x head_dim columns).  Each warpgroup runs its own online
// softmax (running maximum and sum) over its tiles; the two are merged once,
// when a result is normalised.  The issue order S(0), S(1), PV(0), S(2),
// PV(1), ... lets one warpgroup exponentiate while the other's products run.
// A softmax thread holds the whole 128-key row of S in registers (the
// warpgroups' register budget is raised with setmaxnreg) and writes the bf16
// P into the first 64 columns of its S buffer.  Online softmax in the log2
// domain with a lazily updated maximum: O_w is rescaled only when the
// running maximum grows by more than 2^16 (P <= 2^16 is exact-range in bf16
// and keeps the fp32 sums far from overflow; relative precision does not
// depend on the scale).
// Dual mode: before its first history tile each warpgroup takes a local
// checkpoint; warpgroup 0 merges both accumulators and writes A_loc, LSE_loc,
// and both restart; the epilogue fuses the history result with A_loc
// (logaddexp of the two LSEs).  Single-pass mode runs one softmax over every
// tile.
#include <cstring>

#include "internal.h"
#include "sm100.cuh"

namespace ispa {
namespace attn2 {

constexpr int kBM = 128;       // query rows per CTA (= tensor-memory lanes)
constexpr int kBN = 128;       // keys per tile
constexpr int kThreads = 384;  // 12 warps
constexpr int kMaxSeg = ISPA_MAX_SEGMENTS;
constexpr float kRescaleLog2 = 16.0f;  // lazy rescale threshold (log2)
constexpr float kLn2 = 0.69314718055994530942f;
// tensor-memory column map
constexpr uint32_t kTmS = 0;    // S buffers: warpgroup w at kTmS + 128 w
constexpr uint32_t kTmO = 256;  // O accumulators: warpgroup w at kTmO + w * head_dim
// bit j set: column pair j (mod 8) of a score row takes 2^x from the FMA-pipe
// polynomial (exp2_fma2) instead of the special-function unit
constexpr uint32_t kEmuPairs = 0x00u;

struct Params {
  CUtensorMap q_map;
  CUtensorMap k_map[kMaxSeg];
  CUtensorMap v_map[kMaxSeg];
  int32_t seg_tokens[kMaxSeg];
  int32_t seg_first_tile[kMaxSeg + 1];
  int32_t seg_last_tile[kMaxSeg];   // last (possibly partial) tile of each segment, -1 if unused
  int32_t seg_last_valid[kMaxSeg];  // valid keys in that tile
  int32_t n_seg;
  int32_t n_local_tiles;
  int32_t n_tiles;
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
  static constexpr int kTileBytes = kBN * HD * 2;  // one K or V tile
  static constexpr int kBoxBytes = kBN * 128;      // 128 rows x 64 bf16 (one swizzle column block)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + NST * kTileBytes;
  static constexpr int kXs = kV + NST * kTileBytes;  // warpgroup 1's (m, l) per row at the local checkpoint
  static constexpr int kBars = kXs + 2 * kBM * 4;
  // kv_full[NST], kv_empty[NST], q_full, s_full[2], p_full[2], pv_done[2], ck_done, xsum[2], teardown
  static constexpr int kNumBars = 4 * NST + 1 + 2 + 2 + 2 + 1 + 2 + 1;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

__device__ __forceinline__ float ex2(float x) {
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

__device__ __forceinline__ void unpack_bf16x32(const uint4* s4, float (&x)[32]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 u = s4[v];
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
// One producer thread per operand: a K tile is released once S(j) is done,
// a V tile only after PV(j).
template <int HD, int NST>
__device__ void producer(const Params& p, uint8_t* smem, bool v_side, uint64_t* q_full, uint64_t* full,
                         uint64_t* empty, volatile int* abort_flag, int q0, int head) {
  using L = Layout<HD, NST>;
  if (!v_side) {
    tma_prefetch_desc(&p.q_map);
    mbar_arrive_expect_tx(q_full, L::kTileBytes);
#pragma unroll
    for (int c = 0; c < HD / 64; ++c)
      tma_load_2d(smem + L::kQ + c * L::kBoxBytes, &p.q_map, q_full, head * HD + 64 * c, q0);
  }
  uint8_t* ring = smem + (v_side ? L::kV : L::kK);
  const CUtensorMap* maps = v_side ? p.v_map : p.k_map;
  int n = 0;
  bool ok = true;
  for (; n < p.n_tiles; ++n) {
    const int stage = n % NST;
    if (n >= NST && !mbar_wait(&empty[stage], ((n / NST) - 1) & 1, abort_flag)) {
      ok = false;
      break;
    }
    int seg, tok0, valid;
    tile_info(p, n, seg, tok0, valid);
    if (n < p.n_seg) tma_prefetch_desc(&maps[n]);
    mbar_arrive_expect_tx(&full[stage], L::kTileBytes);
#pragma unroll
    for (int c = 0; c < HD / 64; ++c)
      tma_load_2d(ring + stage * L::kTileBytes + c * L::kBoxBytes, &maps[seg], &full[stage], head * HD + 64 * c, tok0);
  }
  if (!ok) {
    if (!v_side) mbar_wait_drain(q_full, 0, 100000000ull);
    for (int j = n > NST ? n - NST : 0; j < n; ++j) mbar_wait_drain(&full[j % NST], (j / NST) & 1, 100000000ull);
  }
}

// ------------------------------------------------------------- MMA issuer
// The whole warp runs the loop; one elected lane issues.  Key tile i belongs to softmax
// warpgroup i & 1, whose S buffer and O accumulator it uses.
template <int HD, int NST>
__device__ void mma_issuer(const Params& p, uint8_t* smem, uint64_t* q_full, uint64_t* kv_full, uint64_t* kv_empty,
                           uint64_t* v_full, uint64_t* v_empty, uint64_t* s_full, uint64_t* p_full, uint64_t* pv_done, uint64_t* ck_done,
                           uint64_t* teardown, volatile int* abort_flag, uint32_t tmem) {
  using L = Layout<HD, NST>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, false, true);
  const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
  const int T = p.n_tiles, n_loc = p.n_local_tiles;
  const bool ck = p.dual && n_loc > 0 && n_loc < T;  // a local result is taken between the tiles

  // the whole warp runs the loop and every wait; the elected lane issues
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
  };
  auto issue_s = [&](int j) -> bool {
    const int stage = j % NST;
    if (!wait(&kv_full[stage], (j / NST) & 1)) return false;
    tc_fence_after();
    const uint32_t kb = sK + stage * L::kTileBytes;
    const uint32_t d = tmem + kTmS + (j & 1) * 128;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
      umma_ss_warp(d, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), kIdescQK,
                   kk > 0 ? 1u : 0u);
    }
    umma_commit_warp(&s_full[j & 1]);
    umma_commit_warp(&kv_empty[stage]);
    return true;
  };

  bool ok = wait(q_full, 0);
  tc_fence_after();
  if (ok && T > 0) ok = issue_s(0);
  if (ok && T > 1) ok = issue_s(1);
  bool ck_seen = false;
  for (int i = 0; ok && i < T; ++i) {
    const int w = i & 1;
    const bool first_hist = ck && i >= n_loc && i - 2 < n_loc;
    const bool fresh = i < 2 || first_hist;
    if (first_hist && !ck_seen) {
      // the first history products overwrite the accumulators; the local
      // result must have been read out of them first
      if (!wait(ck_done, 0)) break;
      ck_seen = true;
    }
    const int stage = i % NST;
    const uint32_t vb = sV + stage * L::kTileBytes;
    const uint32_t pb = tmem + kTmS + w * 128;
    // p_full[w] completes once per tile of warpgroup w; its next phase needs
    // S(i + 2), issued below, so the parity is unambiguous
    if (!wait(&v_full[stage], (i / NST) & 1)) break;
    if (!wait(&p_full[w], (i >> 1) & 1)) break;
    tc_fence_after();
    // O_w += P V: P (bf16, 128 keys) in the first 64 columns of the S buffer
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      umma_ts_warp(tmem + kTmO + w * HD, pb + kk * 8, sdesc_sw128(vb + kk * 2048, L::kBoxBytes, 1024), kIdescPV,
                   (kk > 0 || !fresh) ? 1u : 0u);
    umma_commit_warp(&v_empty[stage]);
    umma_commit_warp(&pv_done[w]);
    if (i + 2 < T) ok = issue_s(i + 2);
  }
  // every MMA must have completed before tensor memory is released
  umma_commit_warp(teardown);
  mbar_wait_drain(teardown, 0, 100000000ull);
  __syncwarp();
}

// ------------------------------------------------------------------ softmax
// bf16 pair from two non-negative floats, rounded to nearest (ties away from
// zero) with integer ALU operations, so the conversion does not compete with
// the exponentials for the special-function pipe.
__device__ __forceinline__ uint32_t pack_p_bf16x2(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

struct Row {
  int wg, lane, row, grow;
  bool row_ok;
  uint32_t lane_base;
};

// Merged, normalised accumulator for channels [32 cc, 32 cc + 32) of this
// row: (O_0 w0 + O_1 w1) / lt.  A weight of 0 means that accumulator holds
// nothing of this result (it may hold stale data) and is not read.
template <int HD>
__device__ __forceinline__ void load_merged(const Row& r, int cc, float w0, float w1, float inv, float (&x)[32]) {
  uint32_t a[32], b[32];
  tmem_ld32(r.lane_base + kTmO + 32 * cc, a);
  tmem_ld32(r.lane_base + kTmO + HD + 32 * cc, b);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float u = w0 != 0.f ? __uint_as_float(a[j]) * w0 : 0.f;
    const float v = w1 != 0.f ? __uint_as_float(b[j]) * w1 : 0.f;
    x[j] = (u + v) * inv;
  }
}

// Waits (all lanes) for the product of warpgroup w's tile number k (counted
// per warpgroup) to have completed.
__device__ __forceinline__ bool wait_pv(uint64_t* pv_done, int w, int k, volatile int* abort_flag) {
  if (k < 0) return true;
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[w], k & 1, abort_flag));
  tc_fence_after();
  return ok;
}

template <int HD, int NST>
__device__ void softmax(const Params& p, uint8_t* smem, uint32_t tmem, uint64_t* s_full, uint64_t* p_full,
                        uint64_t* pv_done, uint64_t* ck_done, uint64_t* xsum, volatile int* abort_flag, int q0,
                        int head) {
  using L = Layout<HD, NST>;
  float* xck = reinterpret_cast<float*>(smem + L::kXs);  // checkpoint: warpgroup 1's (m, l) per row
  float* xfin = reinterpret_cast<float*>(smem + L::kQ);  // final: [wg][m, l, lse_loc][row]; Q is dead by then
  Row r;
  const int warp = threadIdx.x >> 5;
  r.wg = (warp - 4) >> 2;
  r.lane = threadIdx.x & 31;
  r.row = (warp & 3) * 32 + r.lane;
  r.grow = q0 + r.row;
  r.row_ok = r.grow < p.n_q;
  r.lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const int w = r.wg;
  const uint32_t o_own = r.lane_base + kTmO + w * HD;
  const uint32_t sbuf = r.lane_base + kTmS + w * 128;
  const float sl2 = p.scale_log2;
  const int T = p.n_tiles, n_loc = p.n_local_tiles;
  const bool dual = p.dual != 0;
  const bool ck = dual && n_loc > 0 && n_loc < T;
  bool ck_pending = ck;
  bool ok = true;

  float m_used = -INFINITY, l = 0.f, lse_loc2 = 0.f;
  bool o_live = false;  // O_w holds products of the current accumulation

  // local result: the two warpgroups' accumulators are merged, normalised and
  // written (A_loc, LSE_loc) by warpgroup 0; then both restart
  auto checkpoint = [&](int k_next) -> bool {
    if (!wait_pv(pv_done, w, k_next - 1, abort_flag)) return false;  // own last local product
    if (w == 1) {
      xck[r.row] = m_used;
      xck[kBM + r.row] = l;
      mbar_arrive(&xsum[0]);
    } else {
      if (!wait_pv(pv_done, 1, (n_loc >> 1) - 1, abort_flag)) return false;  // warpgroup 1's last local product
      if (!__all_sync(0xffffffffu, mbar_wait(&xsum[0], 0, abort_flag))) return false;
      const float m1 = xck[r.row], l1 = xck[kBM + r.row];
      const float mm = fmaxf(m_used, m1);
      const float w0 = l > 0.f ? ex2(m_used - mm) : 0.f, w1 = l1 > 0.f ? ex2(m1 - mm) : 0.f;
      const float lt = l * w0 + l1 * w1;
      const float inv = 1.0f / lt;
      __nv_bfloat16* dst = p.a_loc + (int64_t)r.grow * p.out_stride + head * HD;
#pragma unroll 1
      for (int cc = 0; cc < HD / 32; ++cc) {
        float x[32];
        load_merged<HD>(r, cc, w0, w1, inv, x);
        if (r.row_ok) store_bf16x32(dst + 32 * cc, x);
      }
      lse_loc2 = mm + log2f(lt);
      if (r.row_ok && p.lse_loc) p.lse_loc[(int64_t)head * p.n_q + r.grow] = lse_loc2 * kLn2;
      tc_fence_before();
      __syncwarp();
      if (r.lane == 0) mbar_arrive(ck_done);
    }
    m_used = -INFINITY;
    l = 0.f;
    o_live = false;
    return true;
  };

#pragma unroll 1
  for (int i = w; i < T; i += 2) {
    const int k = i >> 1;  // this warpgroup's tile count
    if (ck_pending && i >= n_loc) {
      ck_pending = false;
      if (!(ok = checkpoint(k))) break;
    }
    ok = __all_sync(0xffffffffu, mbar_wait(&s_full[w], k & 1, abort_flag));
    if (!ok) break;
    tc_fence_after();
    int valid = kBN;
#pragma unroll
    for (int q = 0; q < kMaxSeg; ++q)
      if (i == p.seg_last_tile[q]) valid = p.seg_last_valid[q];

    // the whole 128-key row of S in registers
    uint32_t s[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(sbuf + 32 * c, s[c]);
    tmem_wait_ld();
    if (valid < kBN) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j >= valid) s[c][j] = __float_as_uint(-INFINITY);
    }
    // P = 2^(s * scale_log2 - m) as bf16 into the first 64 columns of the S
    // buffer (whose values are all in registers by now); returns the sum of P
    auto exponentiate = [&](float m) -> float {
      const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m, -m);
      float2 sum2[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sum2[c] = make_float2(0.f, 0.f);
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 x =
              ffma2(make_float2(__uint_as_float(s[c][2 * j]), __uint_as_float(s[c][2 * j + 1])), sc2, nm2);
          const float2 pv = (kEmuPairs & (1u << (j & 7))) ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
          sum2[c] = fadd2(sum2[c], pv);
          pk[j] = pack_p_bf16x2(pv.x, pv.y);
        }
        tmem_st16(sbuf + 16 * c, pk);
      }
      const float2 st2 = fadd2(fadd2(sum2[0], sum2[1]), fadd2(sum2[2], sum2[3]));
      return st2.x + st2.y;
    };
    auto tile_max = [&]() -> float {
      float mc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t* v = &s[q >> 1][(q & 1) * 16];
        mc[q] = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
        for (int j = 1; j < 8; ++j) mc[q] = fmax3(mc[q], __uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
      }
      const float a = fmax3(mc[0], mc[1], mc[2]), b = fmax3(mc[3], mc[4], mc[5]), c = fmaxf(mc[6], mc[7]);
      return fmax3(a, b, c) * sl2;  // -inf if all masked
    };
    // exponentials with the running maximum straight away, the tile maximum
    // alongside; a growth beyond 2^16 (rare, and always at the start of an
    // accumulation) rescales what was accumulated and redoes the tile.  O_w
    // is quiescent here: S(i) was issued after this warpgroup's previous
    // product, and its completion implies that product's.
    const bool first = __any_sync(0xffffffffu, m_used == -INFINITY);
    float psum = first ? 0.f : exponentiate(m_used);
    const float m_tile = tile_max();
    if (first || __any_sync(0xffffffffu, m_tile > m_used + kRescaleLog2)) {
      const float m_new = fmaxf(m_used, m_tile);
      // rows whose keys are all masked so far keep m = -inf: their P is exactly 0
      const float f = (m_used == -INFINITY || m_new == -INFINITY) ? 0.f : ex2(m_used - m_new);
      if (o_live) {
#pragma unroll 1
        for (int cc = 0; cc < HD / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(o_own + 32 * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tmem_st32(o_own + 32 * cc, o);
        }
      }
      tmem_wait_st();  // the first pass's P stores complete before they are overwritten
      l *= f;
      m_used = m_new;
      psum = exponentiate(m_used == -INFINITY ? 0.f : m_used);
    }
    l += psum;
    if (!ok) break;
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (r.lane == 0) mbar_arrive(&p_full[w]);
    o_live = true;
  }
  if (!ok || *abort_flag) return;
  if (ck_pending) {  // no history tile fell to this warpgroup
    if (!checkpoint((T - w + 1) >> 1)) return;
  }
  // both accumulators final (own first, so the other is at most one phase behind)
  const int n_own = (T - w + 1) >> 1, n_other = (T - (1 - w) + 1) >> 1;
  if (!wait_pv(pv_done, w, n_own - 1, abort_flag)) return;
  if (!wait_pv(pv_done, 1 - w, n_other - 1, abort_flag)) return;
  // final merge of the two warpgroups' statistics (the Q tile is no longer read)
  xfin[(w * 3 + 0) * kBM + r.row] = m_used;
  xfin[(w * 3 + 1) * kBM + r.row] = l;
  xfin[(w * 3 + 2) * kBM + r.row] = lse_loc2;
  mbar_arrive(&xsum[1]);
  if (!__all_sync(0xffffffffu, mbar_wait(&xsum[1], 0, abort_flag))) return;
  const float m0 = xfin[r.row], l0 = xfin[kBM + r.row];
  const float m1 = xfin[3 * kBM + r.row], l1 = xfin[4 * kBM + r.row];
  lse_loc2 = xfin[2 * kBM + r.row];  // computed by warpgroup 0 at the checkpoint
  const float mm = fmaxf(m0, m1);
  const float w0 = l0 > 0.f ? ex2(m0 - mm) : 0.f, w1 = l1 > 0.f ? ex2(m1 - mm) : 0.f;
  const float lt = l0 * w0 + l1 * w1;
  const float inv = 1.0f / lt;
  const float lse2 = mm + log2f(lt);
  const int64_t li = (int64_t)head * p.n_q + r.grow;
  const int64_t base = (int64_t)r.grow * p.out_stride + head * HD + w * (HD / 2);
  const int c_first = w * (HD / 64);  // this warpgroup's 32-channel blocks

  if (!dual || T == n_loc) {  // single pass, or dual with no history (A_full = A_loc, delta = 0)
#pragma unroll 1
    for (int kc = 0; kc < HD / 64; ++kc) {
      float x[32];
      load_merged<HD>(r, c_first + kc, w0, w1, inv, x);
      if (!r.row_ok) continue;
      store_bf16x32(p.a_full + base + 32 * kc, x);
      if (dual) {
        store_bf16x32(p.a_loc + base + 32 * kc, x);
        if (p.a_delta) {
          float z[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) z[j] = 0.f;
          store_bf16x32(p.a_delta + base + 32 * kc, z);
        }
      }
    }
    if (w == 0 && r.row_ok) {
      if (p.lse_full) p.lse_full[li] = lse2 * kLn2;
      if (dual && p.lse_loc) p.lse_loc[li] = lse2 * kLn2;
    }
    return;
  }
  // fuse the history result with the checkpointed local result
  const float mx = fmaxf(lse_loc2, lse2);
  const float lse_full2 = mx + log2f(exp2f(lse_loc2 - mx) + exp2f(lse2 - mx));
  const float wgt = exp2f(lse2 - lse_full2);
#pragma unroll 1
  for (int kc = 0; kc < HD / 64; ++kc) {
    float oh[32];
    load_merged<HD>(r, c_first + kc, w0, w1, inv, oh);
    if (!r.row_ok) continue;
    float a[32], full[32], dl[32];
    unpack_bf16x32(reinterpret_cast<const uint4*>(p.a_loc + base + 32 * kc), a);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      dl[j] = wgt * (oh[j] - a[j]);
      full[j] = a[j] + dl[j];
    }
    store_bf16x32(p.a_full + base + 32 * kc, full);
    if (p.a_delta) store_bf16x32(p.a_delta + base + 32 * kc, dl);
  }
  if (w == 0 && r.row_ok && p.lse_full) p.lse_full[li] = lse_full2 * kLn2;
}

// ------------------------------------------------------------------- kernel
template <int HD, int NST>
__global__ void __launch_bounds__(kThreads, 1) attention_kernel(const __grid_constant__ Params p) {
  using L = Layout<HD, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* v_full = kv_empty + NST;
  uint64_t* v_empty = v_full + NST;
  uint64_t* q_full = v_empty + NST;
  uint64_t* s_full = q_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* ck_done = pv_done + 2;
  uint64_t* xsum = ck_done + 1;
  uint64_t* teardown = xsum + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kBM, head = blockIdx.y;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(ck_done, 4);
    mbar_init(&xsum[0], 128);
    mbar_init(&xsum[1], 256);
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

  // registers: the control warpgroup (producer, MMA issuer, tensor-memory
  // owner) needs few, the softmax warpgroups hold a whole row of S:
  // 128 x 88 + 256 x 208 = 384 x 168, the launch budget
  if (warp >= 4) {
    regs_inc<208>();
    softmax<HD, NST>(p, smem, tmem, s_full, p_full, pv_done, ck_done, xsum, abort_flag, q0, head);
  } else {
    regs_dec<88>();
    if (warp == 0) {
      if (lane == 0) producer<HD, NST>(p, smem, false, q_full, kv_full, kv_empty, abort_flag, q0, head);
    } else if (warp == 1) {
      mma_issuer<HD, NST>(p, smem, q_full, kv_full, kv_empty, v_full, v_empty, s_full, p_full, pv_done, ck_done, teardown, abort_flag,
                          tmem);
    } else if (warp == 3) {
      if (lane == 0) producer<HD, NST>(p, smem, true, nullptr, v_full, v_empty, abort_flag, q0, head);
    }
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
  auto kern = attention_kernel<HD, NST>;
  ispa_status_t st = set_smem(reinterpret_cast<const void*>(kern), L::kAlloc);
  if (st != ISPA_OK) return st;
  dim3 grid((p.n_q + kBM - 1) / kBM, n_heads);
  kern<<<grid, kThreads, L::kAlloc, stream>>>(p);
  return check_launch("attention_kernel");
}

}  // namespace attn2

// Host entry for bf16 activations.  Segments with zero tokens must already be
// removed; local segments come first.
ispa_status_t dual_attention_bf16_db(const void* q, int64_t n_q, int64_t q_stride, int32_t n_heads, int32_t head_dim,
                                     float scale, const ispa_kv_segment_t* segs, int n_local_seg, int n_hist_seg,
                                     void* a_loc, void* a_full, void* a_delta, float* lse_loc, float* lse_full,
                                     int32_t* status, cudaStream_t stream) {
  using namespace attn2;
  static_assert(sizeof(Params) <= 4096, "kernel parameter space");
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
  for (int i = 0; i < kMaxSeg; ++i) {
    p.seg_last_tile[i] = i < n_seg ? p.seg_first_tile[i + 1] - 1 : -1;
    p.seg_last_valid[i] = i < n_seg ? (int32_t)(segs[i].n_tokens - (int64_t)(p.seg_first_tile[i + 1] - 1 - p.seg_first_tile[i]) * kBN) : kBN;
  }
  p.n_seg = n_seg;
  p.n_tiles = tiles;
  p.n_local_tiles = local_tiles;
  p.dual = a_loc != nullptr;
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
