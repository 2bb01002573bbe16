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
//   warps 1, 2  tcgen05 issuers, each converged with one elected lane
//               issuing: warp 2 S(j) = Q K(j)^T (both operands K-major in
//               shared memory), warp 1 O += P(j) V(j) (P from tensor memory,
//               V MN-major in shared memory); warp 2 also allocates and frees
//               the 512 tensor-memory columns;
//   warps 4-11  softmax: two warpgroups; warpgroup w takes the key tiles
//               j = w mod 2; thread = query row = TMEM lane.
// Tensor memory: three S buffers (tile j uses buffer j mod 3) and ONE O
// accumulator (head_dim columns) that both warpgroups' products add into.
// With three S buffers, S(j+3) is issued as soon as PV(j) (the product that
// reads P(j) out of the same columns) has completed, so a warpgroup's next S
// is computed while it is still exponentiating, and the two issuers keep the
// tensor core fed independently.
// Online softmax in the log2 domain with one running maximum per row shared
// by the two warpgroups: the warpgroup of tile j reads the maximum m(j-1)
// that tile j-1 used (a per-row value in shared memory, published through one
// mbarrier per warp quarter), decides m(j), publishes it before its
// exponentials, and computes P(j) = 2^(s scale log2e - m(j)).  The maximum is
// raised lazily: only when a tile's maximum exceeds m(j-1) by more than 2^16
// (P <= 2^16 is exact-range in bf16 and keeps the fp32 sums far from
// overflow), and then O -- holding sum_{i<j} P(i) V(i) -- is rescaled by the
// warpgroup of tile j once PV(j-1) has completed and before it hands P(j)
// over, so every product lands on the right scale.  Each warpgroup keeps its
// own partial row sum, brought to the current maximum when it next uses it.
// Dual mode: once PV of the last local tile has completed, the warpgroup that
// does not own the first history tile normalises O into A_loc and writes
// LSE_loc while the other goes on with that tile; the first history product
// then restarts O and the maximum chain restarts.  The epilogue fuses the history result with A_loc (logaddexp of
// the two LSEs).  Single-pass mode runs one softmax over every tile.
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
constexpr int kNS = 3;          // S buffers: tile j uses buffer j mod kNS at kTmS + kBN (j mod kNS)
constexpr uint32_t kTmS = 0;
constexpr uint32_t kTmO = kNS * kBN;  // the O accumulator (head_dim columns)
static_assert(kTmO + 128 <= 512, "tensor-memory budget");
static_assert(kBN % 32 == 0 && kBN <= 128, "key tile");
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
  // single pass only: MX e4m3 codes [n_q, D] and exponent bytes [n_q, D / 32]
  // of the bf16-rounded output (a_full may then be NULL)
  uint8_t* mx_codes;
  uint8_t* mx_exps;
};

template <int HD, int NST>
struct Layout {
  static constexpr int kQBytes = kBM * HD * 2;     // the Q tile
  static constexpr int kQBox = kBM * 128;          // kBM rows x 64 bf16 (one swizzle column block)
  static constexpr int kTileBytes = kBN * HD * 2;  // one K or V tile
  static constexpr int kBoxBytes = kBN * 128;      // kBN rows x 64 bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + NST * kTileBytes;
  static constexpr int kXs = kV + NST * kTileBytes;  // local checkpoint exchange: (m, l) per row
  static constexpr int kMref = kXs + 2 * kBM * 4;     // the shared running maximum, one float per row
  static constexpr int kBars = kMref + kBM * 4;
  // kv_full, kv_empty, v_full, v_empty [NST]; q_full; s_full, p_full, pv_done [kNS]; mref_full[4];
  // ck_ready, ck_done, fin_ready; xsum[3]; teardown[2]
  static constexpr int kNumBars = 4 * NST + 1 + 3 * kNS + 4 + 3 + 3 + 2;
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
    mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
    for (int c = 0; c < HD / 64; ++c)
      tma_load_2d(smem + L::kQ + c * L::kQBox, &p.q_map, q_full, head * HD + 64 * c, q0);
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
// The whole warp runs the loop; one elected lane issues.  Tile j's S goes to
// S buffer j mod 3 and its P is read from there by PV(j); every PV adds into
// the one O accumulator.  Issue order: S(0), S(1), S(2), then per tile j:
// PV(j), S(j + 3) (into the buffer PV(j) has just read: tcgen05 MMAs of one
// thread execute in issue order).
// The CTA's mbarriers, at fixed offsets from one base (so that an address
// costs one add, not a live register).
template <int NST>
struct Bars {
  uint64_t* base;
  __device__ __forceinline__ uint64_t* kv_full(int i) const { return base + i; }
  __device__ __forceinline__ uint64_t* kv_empty(int i) const { return base + NST + i; }
  __device__ __forceinline__ uint64_t* v_full(int i) const { return base + 2 * NST + i; }
  __device__ __forceinline__ uint64_t* v_empty(int i) const { return base + 3 * NST + i; }
  __device__ __forceinline__ uint64_t* q_full() const { return base + 4 * NST; }
  static constexpr int kS = 4 * NST + 1;  // the per-S-buffer barriers start here
  static constexpr int kR = kS + 3 * kNS;  // and the rest here
  __device__ __forceinline__ uint64_t* s_full(int b) const { return base + kS + b; }  // per S buffer
  __device__ __forceinline__ uint64_t* p_full(int b) const { return base + kS + kNS + b; }
  __device__ __forceinline__ uint64_t* pv_done(int b) const { return base + kS + 2 * kNS + b; }
  __device__ __forceinline__ uint64_t* mref_full(int q) const { return base + kR + q; }  // per warp quarter
  __device__ __forceinline__ uint64_t* ck_ready() const { return base + kR + 4; }
  __device__ __forceinline__ uint64_t* ck_done() const { return base + kR + 5; }
  __device__ __forceinline__ uint64_t* fin_ready() const { return base + kR + 6; }
  __device__ __forceinline__ uint64_t* xsum(int k) const { return base + kR + 7 + k; }
  __device__ __forceinline__ uint64_t* teardown(int w) const { return base + kR + 10 + w; }  // per issuer
  static constexpr int kCount = kR + 12;
};

// Two issuing warps, each converged with one elected lane issuing:
//   warp 2 issues S(j) = Q K(j)^T into S buffer j mod 3 once K(j) has arrived
//   and PV(j - 3) -- the product that reads P(j - 3) out of that buffer -- has
//   completed;
//   warp 1 issues O += P(i) V(i) in tile order once P(i) and V(i) are there.
// Each waits only for its own operands, so the tensor core is fed from one
// while the other waits (a single issuer interleaving both spent a third of
// every tile period in waits while the MMA queue ran dry).
template <int HD, int NST>
__device__ void s_issuer(const Params& p, uint8_t* smem, const Bars<NST>& B, volatile int* abort_flag, uint32_t tmem) {
  using L = Layout<HD, NST>;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false, false);
  const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK);
  const int T = p.n_tiles;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
  };
  bool ok = wait(B.q_full(), 0);
  for (int j = 0; ok && j < T; ++j) {
    const int stage = j % NST, b = j % kNS;
    // buffer b still holds P(j - 3) until PV(j - 3) has completed
    if (j >= kNS && !(ok = wait(B.pv_done(b), ((j - kNS) / kNS) & 1))) break;
    if (!(ok = wait(B.kv_full(stage), (j / NST) & 1))) break;
    tc_fence_after();
    const uint32_t kb = sK + stage * L::kTileBytes;
    const uint32_t d = tmem + kTmS + b * kBN;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      // 16 head-dim elements (32 bytes) of every row, in the column block kk / 4
      const uint32_t offq = (kk >> 2) * L::kQBox + (kk & 3) * 32;
      const uint32_t offk = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
      umma_ss_warp(d, sdesc_sw128(sQ + offq, 16, 1024), sdesc_sw128(kb + offk, 16, 1024), kIdescQK,
                   kk > 0 ? 1u : 0u);
    }
    umma_commit_warp(B.s_full(b));
    umma_commit_warp(B.kv_empty(stage));
  }
  // every MMA must have completed before tensor memory is released
  umma_commit_warp(B.teardown(1));
  mbar_wait_drain(B.teardown(1), 0, 100000000ull);
  __syncwarp();
}

template <int HD, int NST>
__device__ void pv_issuer(const Params& p, uint8_t* smem, const Bars<NST>& B, volatile int* abort_flag,
                          uint32_t tmem) {
  using L = Layout<HD, NST>;
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, false, true);
  const uint32_t sV = smem_u32(smem + L::kV);
  const int T = p.n_tiles, n_loc = p.n_local_tiles;
  const bool ck = p.dual && n_loc > 0 && n_loc < T;  // a local result is taken between the tiles
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
  };
  for (int i = 0; i < T; ++i) {
    const int b = i % kNS;
    const bool first_hist = ck && i == n_loc;
    const bool fresh = i == 0 || first_hist;
    // the first history product overwrites O: the local result must have
    // been read out of it first
    if (first_hist && !wait(B.ck_done(), 0)) break;
    const int stage = i % NST;
    const uint32_t vb = sV + stage * L::kTileBytes;
    const uint32_t pb = tmem + kTmS + b * kBN;
    if (!wait(B.v_full(stage), (i / NST) & 1)) break;
    // p_full[b] completes once per use of buffer b; its next phase needs
    // S(i + 3), which waits for PV(i), so the parity is unambiguous
    if (!wait(B.p_full(b), (i / kNS) & 1)) break;
    tc_fence_after();
    // O += P V: P (bf16, kBN keys) in the first kBN / 2 columns of S buffer b
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk)
      umma_ts_warp(tmem + kTmO, pb + kk * 8, sdesc_sw128(vb + kk * 2048, L::kBoxBytes, 1024), kIdescPV,
                   (kk > 0 || !fresh) ? 1u : 0u);
    umma_commit_warp(B.v_empty(stage));
    umma_commit_warp(B.pv_done(b));
    if (ck && i == n_loc - 1) umma_commit_warp(B.ck_ready());
    if (i == T - 1) umma_commit_warp(B.fin_ready());
  }
  // every MMA must have completed before tensor memory is released
  umma_commit_warp(B.teardown(0));
  mbar_wait_drain(B.teardown(0), 0, 100000000ull);
  __syncwarp();
}

// ------------------------------------------------------------------ softmax

struct Row {
  int wg, lane, row, grow, quarter;
  bool row_ok;
  uint32_t lane_base;
};

// Normalised accumulator for channels [32 cc, 32 cc + 32) of this row: O / l.
__device__ __forceinline__ void load_o(const Row& r, int cc, float inv, float (&x)[32]) {
  uint32_t a[32];
  tmem_ld32(r.lane_base + kTmO + 32 * cc, a);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(a[j]) * inv;
}

// Combined row sum of the two warpgroups, each (m, l) relative to its own
// maximum: returns (m, l) relative to the larger one.
__device__ __forceinline__ float2 combine(float m0, float l0, float m1, float l1) {
  const float mm = fmaxf(m0, m1);
  const float a = l0 > 0.f ? l0 * ex2(m0 - mm) : 0.f;
  const float b = l1 > 0.f ? l1 * ex2(m1 - mm) : 0.f;
  return make_float2(mm, a + b);
}

template <int HD, int NST>
__device__ void softmax(const Params& p, uint8_t* smem, uint32_t tmem, const Bars<NST>& B, volatile int* abort_flag,
                        int q0, int head) {
  using L = Layout<HD, NST>;
  float* xck = reinterpret_cast<float*>(smem + L::kXs);  // checkpoint exchange [m | l][row]
  float* mref = reinterpret_cast<float*>(smem + L::kMref);
  float* xfin = reinterpret_cast<float*>(smem + L::kQ);  // final: [wg][m, l][row]; Q is dead by then
  Row r;
  const int warp = threadIdx.x >> 5;
  r.wg = (warp - 4) >> 2;
  r.quarter = warp & 3;
  r.lane = threadIdx.x & 31;
  r.row = r.quarter * 32 + r.lane;
  r.grow = q0 + r.row;
  r.row_ok = r.grow < p.n_q;
  r.lane_base = tmem + ((uint32_t)(r.quarter * 32) << 16);
  const int w = r.wg;
  const uint32_t o_row = r.lane_base + kTmO;
  const float sl2 = p.scale_log2;
  const int T = p.n_tiles, n_loc = p.n_local_tiles;
  const bool dual = p.dual != 0;
  const bool ck = dual && n_loc > 0 && n_loc < T;
  bool ck_pending = ck;
  bool ok = true;
  auto all = [&](bool v) { return __all_sync(0xffffffffu, v); };

  // this warpgroup's partial row sum l, relative to the maximum m_l it last used
  float m_l = -INFINITY, l = 0.f, lse_loc2 = 0.f;

  // local result: O / l written as A_loc and LSE_loc, then a fresh
  // accumulation.  One warpgroup does it: the one that does not own tile
  // n_loc (the first history tile), so that the other hands over its partial
  // sums and goes straight on to that tile's scores while the local result is
  // read out; the product of tile n_loc waits for the checkpoint (ck_done).
  const int ck_wg = (n_loc + 1) & 1;
  auto checkpoint = [&]() -> bool {
    if (w != ck_wg) {
      xck[r.row] = m_l;
      xck[kBM + r.row] = l;
      mbar_arrive(B.xsum(0));
      m_l = -INFINITY;
      l = 0.f;
      return true;
    }
    if (!all(mbar_wait(B.ck_ready(), 0, abort_flag))) return false;  // PV of the last local tile complete
    tc_fence_after();
    if (!all(mbar_wait(B.xsum(0), 0, abort_flag))) return false;
    const float2 c = combine(m_l, l, xck[r.row], xck[kBM + r.row]);
    const float inv = 1.0f / c.y;
    __nv_bfloat16* dst = p.a_loc + (int64_t)r.grow * p.out_stride + head * HD;
#pragma unroll 1
    for (int kc = 0; kc < HD / 32; ++kc) {
      float x[32];
      load_o(r, kc, inv, x);
      if (r.row_ok) store_bf16x32(dst + 32 * kc, x);
    }
    lse_loc2 = c.x + log2f(c.y);
    xck[r.row] = lse_loc2;  // for the other warpgroup's final fusion (read after xsum(2))
    if (r.row_ok && p.lse_loc) p.lse_loc[(int64_t)head * p.n_q + r.grow] = lse_loc2 * kLn2;
    tc_fence_before();
    __syncwarp();
    if (r.lane == 0) mbar_arrive(B.ck_done());
    m_l = -INFINITY;
    l = 0.f;
    return true;
  };

#pragma unroll 1
  for (int i = w; i < T; i += 2) {
    const int b = i % kNS;
    if (ck_pending && i >= n_loc) {
      ck_pending = false;
      if (!(ok = checkpoint())) break;
    }
    // the maximum tile i - 1 used (none at the start of an accumulation),
    // read before the scores occupy the registers.  Every tile's publication
    // is one phase of mref_full, in tile order, so even the first history
    // tile, which does not use it, waits for tile i - 1's publication before
    // making its own (it would otherwise complete that phase in its place and
    // leave a stale maximum in mref for the tile after it)
    const bool first_acc = i == 0 || (ck && i == n_loc);
    float m_prev = -INFINITY;
    if (i > 0) {
      if (!(ok = all(mbar_wait(B.mref_full(r.quarter), (i - 1) & 1, abort_flag)))) break;
      if (!first_acc) m_prev = mref[r.row];
    }
    if (!(ok = all(mbar_wait(B.s_full(b), (i / kNS) & 1, abort_flag)))) break;
    tc_fence_after();
    int valid = kBN;
#pragma unroll
    for (int q = 0; q < kMaxSeg; ++q)
      if (i == p.seg_last_tile[q]) valid = p.seg_last_valid[q];

    // the whole kBN-key row of S in registers
    constexpr int NC = kBN / 32;
    const uint32_t sbuf = r.lane_base + kTmS + b * kBN;
    uint32_t s[NC][32];
#pragma unroll
    for (int c = 0; c < NC; ++c) tmem_ld32(sbuf + 32 * c, s[c]);
    tmem_wait_ld();
    if (valid < kBN) {
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j >= valid) s[c][j] = __float_as_uint(-INFINITY);
    }
    // tile maximum (scaled, log2 domain; -inf if every key is masked)
    float m_tile;
    {
      constexpr int NG = kBN / 16;  // groups of 16 scores, reduced independently
      float mc[NG];
#pragma unroll
      for (int q = 0; q < NG; ++q) {
        const uint32_t* v = &s[q >> 1][(q & 1) * 16];
        mc[q] = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
        for (int j = 1; j < 8; ++j) mc[q] = fmax3(mc[q], __uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
      }
      float m = mc[0];
#pragma unroll
      for (int q = 1; q + 1 < NG; q += 2) m = fmax3(m, mc[q], mc[q + 1]);
      if (NG % 2 == 0) m = fmaxf(m, mc[NG - 1]);
      m_tile = m * sl2;
    }
    const bool fin_prev = m_prev != -INFINITY;
    const bool grow = __any_sync(0xffffffffu, fin_prev && m_tile > m_prev + kRescaleLog2);
    const float m_i = !fin_prev ? m_tile : (grow ? fmaxf(m_prev, m_tile) : m_prev);
    mref[r.row] = m_i;
    mbar_arrive(B.mref_full(r.quarter));

    // P = 2^(s * scale_log2 - m) as bf16 into the first kBN / 2 columns of
    // the S buffer (whose values are all in registers by now); the sum of P
    float psum;
    {
      const float m = m_i == -INFINITY ? 0.f : m_i;
      const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m, -m);
      float2 sum2[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        sum2[c] = make_float2(0.f, 0.f);
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 x =
              ffma2(make_float2(__uint_as_float(s[c][2 * j]), __uint_as_float(s[c][2 * j + 1])), sc2, nm2);
          const float2 pv = (kEmuPairs & (1u << (j & 7))) ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
          sum2[c] = fadd2(sum2[c], pv);
          pk[j] = pack_bf16x2(pv.x, pv.y);  // one packed round-to-nearest-even conversion
        }
        tmem_st16(sbuf + 16 * c, pk);
      }
      float2 st2 = sum2[0];
#pragma unroll
      for (int c = 1; c < NC; ++c) st2 = fadd2(st2, sum2[c]);
      psum = st2.x + st2.y;
    }
    if (l > 0.f && m_i != m_l) l *= ex2(m_l - m_i);
    l += psum;
    if (m_i != -INFINITY) m_l = m_i;

    // a raised maximum: O (every product before tile i) moves to the new
    // scale once PV(i - 1) has completed; PV(i) waits for p_full below
    const bool rescale_row = fin_prev && m_i > m_prev;
    if (__any_sync(0xffffffffu, rescale_row)) {
      if (!(ok = all(mbar_wait(B.pv_done((i - 1) % kNS), ((i - 1) / kNS) & 1, abort_flag)))) break;
      tc_fence_after();
      const float f = rescale_row ? ex2(m_prev - m_i) : 1.f;
#pragma unroll 1
      for (int cc = 0; cc < HD / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(o_row + 32 * cc, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
        tmem_st32(o_row + 32 * cc, o);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (r.lane == 0) mbar_arrive(B.p_full(b));
  }
  if (!ok || *abort_flag) return;
  if (ck_pending && !checkpoint()) return;  // no history tile fell to this warpgroup
  // the last product complete: O final
  if (!all(mbar_wait(B.fin_ready(), 0, abort_flag))) return;
  tc_fence_after();
  // final row sums of the two warpgroups (the Q tile is no longer read)
  xfin[(w * 2 + 0) * kBM + r.row] = m_l;
  xfin[(w * 2 + 1) * kBM + r.row] = l;
  mbar_arrive(B.xsum(2));
  if (!all(mbar_wait(B.xsum(2), 0, abort_flag))) return;
  const float2 cmb = combine(xfin[r.row], xfin[kBM + r.row], xfin[2 * kBM + r.row], xfin[3 * kBM + r.row]);
  if (ck && w != ck_wg) lse_loc2 = xck[r.row];  // published by the checkpoint warpgroup
  const float inv = 1.0f / cmb.y;
  const float lse2 = cmb.x + log2f(cmb.y);
  const int64_t li = (int64_t)head * p.n_q + r.grow;
  const int64_t base = (int64_t)r.grow * p.out_stride + head * HD + w * (HD / 2);
  const int c_first = w * (HD / 64);  // this warpgroup's 32-channel blocks

  if (!dual || T == n_loc) {  // single pass, or dual with no history (A_full = A_loc, delta = 0)
#pragma unroll 1
    for (int kc = 0; kc < HD / 64; ++kc) {
      float x[32];
      load_o(r, c_first + kc, inv, x);
      if (!r.row_ok) continue;
      if (p.a_full) store_bf16x32(p.a_full + base + 32 * kc, x);
      if (p.mx_codes) {
        // the block of the bf16 output, quantised with its own power-of-two scale
        float xb[32];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const uint32_t u = pack_bf16x2(x[j], x[j + 1]);
          xb[j] = __uint_as_float(u << 16);
          xb[j + 1] = __uint_as_float(u & 0xFFFF0000u);
        }
        uint32_t c[8];
        const uint32_t ebyte = mx_quantize32(xb, c);
        const int64_t ch = (int64_t)head * HD + w * (HD / 2) + 32 * kc;  // first channel of the block
        uint4* dst = reinterpret_cast<uint4*>(p.mx_codes + (int64_t)r.grow * p.out_stride + ch);
        dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
        dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
        p.mx_exps[(int64_t)r.grow * (p.out_stride / 32) + ch / 32] = (uint8_t)ebyte;
      }
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
  // fuse the history result with the checkpointed local result (A_loc was
  // written by the checkpoint warpgroup before its xsum(2) arrival)
  const float mx = fmaxf(lse_loc2, lse2);
  const float lse_full2 = mx + log2f(exp2f(lse_loc2 - mx) + exp2f(lse2 - mx));
  const float wgt = exp2f(lse2 - lse_full2);
#pragma unroll 1
  for (int kc = 0; kc < HD / 64; ++kc) {
    float oh[32];
    load_o(r, c_first + kc, inv, oh);
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
  Bars<NST> B{bars};
  static_assert(Bars<NST>::kCount == L::kNumBars, "barrier count");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kBM, head = blockIdx.y;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(B.kv_full(i), 1);
      mbar_init(B.kv_empty(i), 1);
      mbar_init(B.v_full(i), 1);
      mbar_init(B.v_empty(i), 1);
    }
    mbar_init(B.q_full(), 1);
    for (int i = 0; i < kNS; ++i) {
      mbar_init(B.s_full(i), 1);
      mbar_init(B.p_full(i), 4);  // the four warps of the tile's warpgroup
      mbar_init(B.pv_done(i), 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(B.mref_full(i), 32);  // the 32 rows of one warp
    mbar_init(B.ck_ready(), 1);
    mbar_init(B.ck_done(), 4);  // the four warps of the checkpoint warpgroup
    mbar_init(B.fin_ready(), 1);
    mbar_init(B.xsum(0), 128);  // the partial sums handed to the checkpoint warpgroup
    mbar_init(B.xsum(2), 256);  // the final (m, l) exchange; xsum(1) is unused
    mbar_init(B.teardown(0), 1);
    mbar_init(B.teardown(1), 1);
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
    softmax<HD, NST>(p, smem, tmem, B, abort_flag, q0, head);
  } else {
    regs_dec<88>();
    if (warp == 0) {
      if (lane == 0) producer<HD, NST>(p, smem, false, B.q_full(), B.kv_full(0), B.kv_empty(0), abort_flag, q0, head);
    } else if (warp == 1) {
      pv_issuer<HD, NST>(p, smem, B, abort_flag, tmem);
    } else if (warp == 2) {
      s_issuer<HD, NST>(p, smem, B, abort_flag, tmem);
    } else if (warp == 3) {
      if (lane == 0) producer<HD, NST>(p, smem, true, nullptr, B.v_full(0), B.v_empty(0), abort_flag, q0, head);
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
                                     int32_t* status, cudaStream_t stream, uint8_t* mx_codes, uint8_t* mx_exps) {
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
  p.mx_codes = mx_codes;
  p.mx_exps = mx_exps;
  if (head_dim == 128) return launch<128, 3>(p, n_heads, stream);
  return launch<64, 6>(p, n_heads, stream);
}

}  // namespace ispa
