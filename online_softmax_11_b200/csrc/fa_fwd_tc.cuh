// fa_fwd_tc.cuh -- bf16 attention forward on the Blackwell tensor cores (sm_100a).
//
// A work tile is two 128-row query tiles (Q0, Q1) of one (batch, query head).  For each
// 128-key K/V tile j the work tile needs, and each query tile i, the CTA computes
// ("Module 16: Efficient and Long Attention", 16.1 and 16.2):
//   S_i   = Q_i K_j^T                          tcgen05.mma, A and B from shared memory,
//                                              fp32 accumulator in tensor memory (TMEM)
//   s    <- scale * s, soft-cap, mask          (16.5 soft-cap; 16.2 "Measured": the mask
//                                              uses positions in the full sequence)
//   m_new = max(m, rowmax s)                   one query row per thread: row max and sum
//   P     = exp(s - m), l = alpha l + sum P    are thread-local; P rounded to bf16 and
//                                              stored to shared memory
//   O_i   = alpha O_i + P V_j                  tcgen05.mma, A = P and B = V (MN-major, no
//                                              transpose) from shared memory
// and finally O_i / l (bf16) and LSE = m + ln l (fp32), each written to HBM once.  The
// score matrix never leaves the SM.
//
// Pipeline.  The softmax reads its whole 128-score row of S from TMEM (two 64-column
// loads, one wait) and says so at once; S of the next key tile can then be computed into
// the same TMEM columns while the softmax is still exponentiating, so per query tile the
// tensor core runs S_{j+1} in the shadow of softmax_j and P_j V_j right after it (P lives
// in shared memory, one 32 KB buffer per query tile, in two 64-key slabs with their own
// barriers so each half's P.V starts as soon as that half is stored).  The two query tiles run the
// same chain independently and share the tensor core and the K/V ring.  The ring streams
// K one tile ahead of V (K_0, K_1, V_0, K_2, V_1, ...), the order the MMAs consume them.
//
// Persistent CTAs, one per SM.  The work tiles are grouped in units of two query-tile
// pairs of one head, {q-pair n-1-p, q-pair p}; under a causal mask the two halves of a
// unit cost (2(n-1-p)+1.5) + (2p+1.5) key tiles, the same for every unit, so a static
// round-robin of units over the CTAs is balanced.  Units are numbered head-major, so the
// CTAs running at the same time share the K/V of a few heads in L2.
//
// Roles (384 threads = 3 warpgroups):
//   warpgroup 0  softmax for Q0 (thread t owns TMEM lane t = query row t), the lazy
//                rescale of its row of O, and the epilogue of Q0
//   warpgroup 1  the same for Q1
//   warpgroup 2  warp 8: TMA producer (Q0/Q1 per work tile, then K and V tiles into a ring
//                of shared-memory slots); warps 9 and 10: one MMA-issuing thread per query
//                tile (warp 9 also owns the TMEM allocation); warp 11 idle.
// With 12 warps, at most 3 share an SM sub-partition, so each thread gets up to 168
// registers: enough for a softmax thread to hold its whole 128-score row.  There is no
// separate correction warpgroup: with lazy rescaling (below) O is rescaled rarely, so the
// softmax warps do it themselves.  A fourth warpgroup taking over the epilogue (512
// threads, softmax re-sized to 192 registers with setmaxnreg) measured slower: it made
// every key tile's softmax about 6% longer, more than the epilogue it removed.
// Per key tile a softmax warp waits on two barriers (S ready, both halves of the previous
// P read); each wait tests the phase without blocking first, since it has nearly always
// completed already and every mbarrier test costs a shared-memory round trip.
// Epilogue: O / l is written as bf16 into the query tile's P buffer (free once the last
// P.V has completed) in the 128-byte-swizzled layout of the O tensor map, and each warp
// stores its own 32 rows with TMA (boxes of 32 rows x 64 columns), waiting for the store
// to have read them only when it next writes P there.
//
// Online-softmax details:
//   * Scores are handled in log2 units, u = s * scale * log2(e), so P = exp2(u - m) is one
//     FFMA plus one ex2 per score.
//   * Lazy rescaling: the running maximum used for P only moves when the row maximum
//     grows by more than kRescaleLog2 (2^8); P then stays <= 256, and O and l always share
//     the same (possibly stale) reference, so the result is still exact up to rounding
//     (Module 16, 16.2: the max subtraction is about range, not correctness).  When it
//     moves, the row of O in TMEM is multiplied by alpha = exp2(m_old - m_new) once the
//     previous tile's P.V has landed and before this tile's P.V is released.
//   * A row whose maximum is still -inf uses 0 as its reference, so masked scores give
//     P = 0 and never NaN; alpha is 0 in that case (the guard of oxios'
//     FlashAttention::attention for the first rescale).
//
// Every wait is bounded (see mbar_wait): a lost phase turns into FA_ERR_TIMEOUT in the
// device status word and an orderly exit, never a hang.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {
namespace tc {

constexpr int BM = 128;                       // query rows per Q tile (= TMEM lanes)
constexpr int BN = 128;                       // keys per K/V tile
constexpr int NQ = 2;                         // Q tiles per work tile
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 384;                 // 3 warpgroups
constexpr int kTmemCols = 512;                // S0 | S1 | O0 | O1, 128 columns each
constexpr float kRescaleLog2 = 8.0f;          // lazy-rescale threshold (log2 units)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kLaunchRegs = 168;  // 384 threads, one CTA per SM

template <int D>
struct Layout {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static constexpr int kHalves = D / 64;               // 64-column (128-byte) slabs per row
  static constexpr int kHalfBytes = 128 * 128;         // one slab of a 128-row tile
  static constexpr int kTileBytes = 128 * D * 2;       // a Q, K or V tile
  static constexpr int kStages = D == 128 ? 3 : 8;     // K/V ring slots
  static constexpr int kPBytes = 128 * BN * 2;         // P of one query tile (bf16, 128 x 128)
  static constexpr int kQOff = 0;
  static constexpr int kPOff = kQOff + NQ * kTileBytes;
  static constexpr int kRingOff = kPOff + NQ * kPBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // barriers
  static constexpr int kBarQFull = 0;                     // [NQ]
  static constexpr int kBarQEmpty = kBarQFull + NQ;       // [NQ]
  static constexpr int kBarKvFull = kBarQEmpty + NQ;      // [kStages]
  static constexpr int kBarKvEmpty = kBarKvFull + kStages;
  static constexpr int kBarSFull = kBarKvEmpty + kStages; // [NQ]: S computed
  static constexpr int kBarSFree = kBarSFull + NQ;        // [NQ]: S read into registers
  static constexpr int kBarPFull = kBarSFree + NQ;        // [NQ][2]: P of key half 0 / 1 stored
  static constexpr int kBarPFree = kBarPFull + 2 * NQ;    // [NQ][2]: ... and read by its P.V
  static constexpr int kBarOFull = kBarPFree + 2 * NQ;    // [NQ]
  static constexpr int kBarDrain = kBarOFull + NQ;
  static constexpr int kNumBars = kBarDrain + NQ;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // u32 tmem base, int abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;         // slack for 1024-byte alignment
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
  // TMEM columns: S_i at 128 i, O_i at 256 + 128 i
  __device__ static constexpr uint32_t col_s(int i) { return static_cast<uint32_t>(i) * 128u; }
  __device__ static constexpr uint32_t col_o(int i) { return 256u + static_cast<uint32_t>(i) * 128u; }
  // The d = 64 variant must not share an SM with a second CTA (TMEM is fully allocated).
  static constexpr int kSmemLaunch = kSmemAlloc > 120 * 1024 ? kSmemAlloc : 120 * 1024;
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int Hq, Hkv;
  int Nq, Nk;          // query rows and key rows per head
  int pos_off;         // Nk - Nq: query row i sits at position i + pos_off of the keys
  int n_sink;          // keys [0, n_sink) are exempt from the window (0: none)
  int n_bh;            // B * Hq
  int n_qp;            // ceil(Nq / 256): query-tile pairs per head
  int units_per_head;  // ceil(n_qp / 2)
  int n_units;         // n_bh * units_per_head
  int causal;
  int window;          // <= 0: off
  float scale_log2;    // scale * log2(e)
  int use_softcap;
  float cap_inner;     // scale / softcap
  float cap_outer;     // softcap * log2(e)
  unsigned long long timeout_ns;
  // split-KV: the key tiles of every query-tile pair are cut into num_splits contiguous
  // chunks, each chunk a work tile of its own, writing a partial O (fp32, normalised
  // within the chunk) and a partial LSE for a merge pass (fa_merge.cuh)
  int num_splits;      // 1: plain forward, outputs o / lse
  float* o_part;       // [num_splits][B*Hq][Nq][d]
  float* lse_part;     // [num_splits][B*Hq][Nq]
};

// Accurate tanh for the soft-cap: Taylor series about 0 through x^11 for |x| < 0.3
// (truncation error below 1e-9), otherwise 1 - 2 / (exp(2|x|) + 1) with the sign of x.
// The coefficients are the series of tanh: 1, -1/3, 2/15, -17/315, 62/2835, -1382/155925.
__device__ __forceinline__ float tanh_cap(float x) {
  const float ax = fabsf(x);
  if (ax < 0.3f) {
    const float x2 = x * x;
    float p = -1382.0f / 155925.0f;
    p = fmaf(p, x2, 62.0f / 2835.0f);
    p = fmaf(p, x2, -17.0f / 315.0f);
    p = fmaf(p, x2, 2.0f / 15.0f);
    p = fmaf(p, x2, -1.0f / 3.0f);
    return fmaf(p * x2, x, x);
  }
  const float e = ex2_approx(2.0f * kLog2e * ax);
  const float t = 1.0f - __fdividef(2.0f, e + 1.0f);
  return copysignf(t, x);
}

__device__ __forceinline__ float2 ex2_pair(float2 x) { return make_float2(ex2_approx(x.x), ex2_approx(x.y)); }

// u = co tanh(x) - m for a pair with |x| < 0.3: the Taylor series of tanh through x^11, or
// through x^7 when kShort and |x| < 0.12 (the next term is below 1e-10 there), with the
// outer scale co folded into its coefficients: co tanh(x) = x (co + x^2 (b1 + x^2 (b2 +
// ...))), b_k = co c_k, c_k = -1/3, 2/15, -17/315, 62/2835, -1382/155925.  b holds b1 ..
// b5 (kShort reads b1 .. b3).
template <bool kShort>
__device__ __forceinline__ float2 cap_u_pair(float2 x, const float* b, float co, float2 negm) {
  const float2 x2 = __fmul2_rn(x, x);
  float2 r;
  if (kShort) {
    r = __ffma2_rn(make_float2(b[2], b[2]), x2, make_float2(b[1], b[1]));
  } else {
    r = __ffma2_rn(make_float2(b[4], b[4]), x2, make_float2(b[3], b[3]));
    r = __ffma2_rn(r, x2, make_float2(b[2], b[2]));
    r = __ffma2_rn(r, x2, make_float2(b[1], b[1]));
  }
  r = __ffma2_rn(r, x2, make_float2(b[0], b[0]));
  const float2 w = __ffma2_rn(r, x2, make_float2(co, co));
  return __ffma2_rn(w, x, negm);
}

// How P is produced from the scores of one tile (chosen per tile, warp-uniformly).
enum class PMode {
  kPlain,        // no soft-cap: ex2 on the exponential unit for every score (masked keys,
                 // -inf, give exactly 0); one code path for masked and unmasked tiles
                 // keeps the loop small
  kCapShort,     // soft-cap, every |s * scale / cap| < 0.12
  kCapLong,      // soft-cap, every |s * scale / cap| < 0.3
  kCapGeneral,   // soft-cap, anything else (including masked keys)
};

constexpr int kHalf = BN / 2;  // the softmax works on 64-score halves of a row

// P = exp2(u - m) for 64 scores of this thread's row (s[0 .. 63]), rounded to bf16 and
// stored to this row of a 64-key slab of P in shared memory: 8 chunks of 8 keys (16 B),
// chunk c at 16 (c ^ (row & 7)) -- the 128-byte swizzle the tensor core reads K-major
// operands in.  Returns the fp32 sum of these P.
template <PMode kMode>
__device__ __forceinline__ float make_p(const float* s, uint8_t* prow, int rsw, float scale_log2, float cap_inner,
                                        float cap_outer, float m_use, const float* cap_b = nullptr) {
  const float2 negm = make_float2(-m_use, -m_use);
  float2 lsum0 = make_float2(0.f, 0.f), lsum1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < kHalf / 8; ++c) {
    uint32_t packed[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float2 sv = make_float2(s[c * 8 + 2 * x], s[c * 8 + 2 * x + 1]);
      float2 e;
      if constexpr (kMode == PMode::kPlain) {
        e = ex2_pair(__ffma2_rn(sv, make_float2(scale_log2, scale_log2), negm));
      } else if constexpr (kMode == PMode::kCapShort || kMode == PMode::kCapLong) {
        e = ex2_pair(cap_u_pair<kMode == PMode::kCapShort>(__fmul2_rn(sv, make_float2(cap_inner, cap_inner)),
                                                           cap_b, cap_outer, negm));
      } else {
        e.x = ex2_approx(fmaf(tanh_cap(sv.x * cap_inner), cap_outer, -m_use));
        e.y = ex2_approx(fmaf(tanh_cap(sv.y * cap_inner), cap_outer, -m_use));
        e.x = (sv.x == -CUDART_INF_F) ? 0.f : e.x;
        e.y = (sv.y == -CUDART_INF_F) ? 0.f : e.y;
      }
      if (x & 1)
        lsum1 = __fadd2_rn(lsum1, e);
      else
        lsum0 = __fadd2_rn(lsum0, e);
      packed[x] = pack_bf16x2(e.x, e.y);
    }
    *reinterpret_cast<uint4*>(prow + ((c ^ rsw) << 4)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
  const float2 lsum = __fadd2_rn(lsum0, lsum1);
  return lsum.x + lsum.y;
}

// The 128 scores of the row for one key tile from TMEM (two loads, one wait), masked when
// the tile needs a mask: -inf above column c_hi and in the hole [h_lo, h_hi) of columns
// below the window that are not attention sinks.  sink_cols (uniform over the tile) says
// whether the tile holds sink columns at all; without them the hole starts at column 0.
// kSinks = false (no sinks in the launch) compiles only that second form.
template <bool kSinks>
__device__ __forceinline__ void load_row(uint32_t taddr, bool need_mask, bool sink_cols, int h_lo, int h_hi,
                                         int c_hi, float (&s)[BN]) {
  uint32_t r[BN];
  tmem_ld64x2_wait(taddr, r);
#pragma unroll
  for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(r[c]);
  if (need_mask) {
    if (kSinks && sink_cols) {
      const uint32_t hole = static_cast<uint32_t>(h_hi - h_lo);
#pragma unroll
      for (int c = 0; c < BN; ++c)
        s[c] = (static_cast<uint32_t>(c - h_lo) < hole || c > c_hi) ? -CUDART_INF_F : s[c];
    } else {
#pragma unroll
      for (int c = 0; c < BN; ++c) s[c] = (c < h_hi || c > c_hi) ? -CUDART_INF_F : s[c];
    }
  }
}

// A set of 128-key tiles as two ascending runs, [a0, a1) then [b0, b1) with a1 <= b0.
// The first run holds attention-sink tiles when they are apart from the window's tiles;
// otherwise it is empty and everything is in the second run.  Empty runs are (0, 0).
struct TileSet {
  int a0, a1, b0, b1;
  __device__ int count() const { return (a1 - a0) + (b1 - b0); }
  __device__ int at(int n) const { return n < a1 - a0 ? a0 + n : b0 + (n - (a1 - a0)); }
};

__device__ __forceinline__ void run_and(int x0, int x1, int y0, int y1, int& r0, int& r1) {
  r0 = max(x0, y0);
  r1 = min(x1, y1);
  if (r1 <= r0) r0 = r1 = 0;
}

// Key tiles of one query tile: rows r0 .. r1 (r1 < Nq) at positions r + pos_off.
struct TileRange {
  int r0, r1;   // first / last query row
  TileSet ks;   // key tiles this work tile streams for it
  bool active;  // the tile has rows below Nq
  bool part;    // ... and key tiles to process in this work tile
};

__device__ __forceinline__ TileRange tile_range(const Params& p, int r0, int nkv) {
  TileRange t;
  t.r0 = r0;
  t.active = r0 < p.Nq;
  t.r1 = min(p.Nq, r0 + BM) - 1;
  const int pr0 = r0 + p.pos_off, pr1 = t.r1 + p.pos_off;
  int lo = 0, hi = nkv;
  if (p.causal) hi = pr1 < 0 ? 0 : min(nkv, pr1 / BN + 1);
  if (p.window > 0) lo = min(hi, max(0, pr0 - p.window + 1) / BN);
  t.ks = TileSet{0, 0, lo, hi};
  if (p.window > 0 && p.n_sink > 0) {
    const int sink_tiles = min(hi, (p.n_sink + BN - 1) / BN);
    if (lo <= sink_tiles) t.ks.b0 = 0;  // sinks and window join up: one run from key 0
    else t.ks.a1 = sink_tiles;
  }
  if (!t.active || t.ks.count() <= 0) t.ks = TileSet{0, 0, 0, 0};
  t.part = t.ks.count() > 0;
  return t;
}

// One work tile: (batch*head, query-tile pair, key chunk) and the key tiles it streams.
struct WorkTile {
  int bh, kvh;
  int split;   // key chunk (0 without split-KV)
  TileRange tr0, tr1;
  TileSet ks;  // key tiles streamed: the union of both query tiles' sets (or a chunk of it)
  __device__ const TileRange& tr(int i) const { return i == 0 ? tr0 : tr1; }
};

// Keep the part of t's tiles inside chunk c.  Each run of t meets at most one run of c
// (sink tiles lie below every window tile of the pair when the union keeps them apart).
__device__ __forceinline__ void clip(TileRange& t, const TileSet& c) {
  int x0, x1, y0, y1;
  TileSet k;
  run_and(t.ks.a0, t.ks.a1, c.a0, c.a1, x0, x1);
  run_and(t.ks.a0, t.ks.a1, c.b0, c.b1, y0, y1);
  k.a0 = x1 > x0 ? x0 : y0;
  k.a1 = x1 > x0 ? x1 : y1;
  run_and(t.ks.b0, t.ks.b1, c.a0, c.a1, x0, x1);
  run_and(t.ks.b0, t.ks.b1, c.b0, c.b1, y0, y1);
  k.b0 = x1 > x0 ? x0 : y0;
  k.b1 = x1 > x0 ? x1 : y1;
  t.ks = k;
  t.part = t.active && k.count() > 0;
  if (!t.part) t.ks = TileSet{0, 0, 0, 0};
}

__device__ __forceinline__ WorkTile make_work_tile(const Params& p, int bh, int qp, int split) {
  WorkTile w;
  w.bh = bh;
  w.split = split;
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  w.kvh = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const int nkv = (p.Nk + BN - 1) / BN;
  w.tr0 = tile_range(p, qp * NQ * BM, nkv);
  w.tr1 = tile_range(p, qp * NQ * BM + BM, nkv);
  // union: sink runs start at tile 0; the window runs of the two query tiles overlap or
  // touch (the second starts at most one tile past the first's end), so the union is
  // again two runs, joined when the sink run reaches the window run
  const TileSet& s0 = w.tr0.ks;
  const TileSet& s1 = w.tr1.ks;
  TileSet u{0, max(s0.a1, s1.a1), 0, 0};
  if (s0.b1 > s0.b0 && s1.b1 > s1.b0) {
    u.b0 = min(s0.b0, s1.b0);
    u.b1 = max(s0.b1, s1.b1);
  } else if (s0.b1 > s0.b0) {
    u.b0 = s0.b0;
    u.b1 = s0.b1;
  } else {
    u.b0 = s1.b0;
    u.b1 = s1.b1;
  }
  if (u.a1 > 0 && u.a1 >= u.b0) u = TileSet{0, 0, 0, max(u.a1, u.b1)};
  w.ks = u;
  if (p.num_splits > 1) {  // this work tile keeps chunk `split` of the pair's key tiles
    const int T = u.count();
    const int c0 = (split * T) / p.num_splits;
    const int c1 = ((split + 1) * T) / p.num_splits;
    const int na = u.a1 - u.a0;
    TileSet c;
    c.a0 = u.a0 + min(c0, na);
    c.a1 = u.a0 + min(c1, na);
    c.b0 = u.b0 + max(c0 - na, 0);
    c.b1 = u.b0 + max(c1 - na, 0);
    if (c.a1 <= c.a0) c.a0 = c.a1 = 0;
    if (c.b1 <= c.b0) c.b0 = c.b1 = 0;
    clip(w.tr0, c);
    clip(w.tr1, c);
    w.ks = c;
  }
  return w;
}

// The static schedule: CTA c takes units c, c + G, ....  Without split-KV, unit u is head
// u / U, pair index p = u % U, and covers q-pairs n_qp-1-p (longer under causal) and p
// (when distinct).  With split-KV, unit u is (head, q-pair from the longest, key chunk).
// Every role walks the same sequence; the callback returns false to stop (abort).
template <typename F>
__device__ __forceinline__ void for_each_tile(const Params& p, F&& f) {
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    if (p.num_splits > 1) {
      const int per_head = p.n_qp * p.num_splits;
      const int bh = u / per_head;
      if (bh >= p.n_bh) return;  // never past the last head, whatever n_units says
      const int rem = u - bh * per_head;
      const int qp = p.n_qp - 1 - rem / p.num_splits;
      if (!f(make_work_tile(p, bh, qp, rem % p.num_splits))) return;
      continue;
    }
    const int bh = u / p.units_per_head;
    if (bh >= p.n_bh) return;
    const int pi = u - bh * p.units_per_head;
    const int qa = p.n_qp - 1 - pi;
    for (int half = 0; half < (pi != qa ? 2 : 1); ++half) {  // one call site: f inlines once
      if (!f(make_work_tile(p, bh, half == 0 ? qa : pi, 0))) return;
    }
  }
}

// kSplit: write fp32 partials for the split-KV merge instead of O and LSE.
// kSinks: the launch has attention sinks (a separate run of sink tiles may precede the
// window's tiles); without them every key-tile set is one run and the loops are the
// plain ranges.
// kCap: logit soft-cap on; without it the soft-cap code is not compiled in (fewer live
// registers in the softmax).
template <int D, bool kSplit, bool kSinks, bool kCap>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  // ---- set-up: barriers, abort flag, TMEM
  if (threadIdx.x == 0) {
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&bars[L::kBarQFull + i], 1);
      mbar_init(&bars[L::kBarQEmpty + i], 1);
      mbar_init(&bars[L::kBarSFull + i], 1);
      mbar_init(&bars[L::kBarSFree + i], BM);
      for (int h = 0; h < 2; ++h) {
        mbar_init(&bars[L::kBarPFull + 2 * i + h], BM);
        mbar_init(&bars[L::kBarPFree + 2 * i + h], 1);
      }
      mbar_init(&bars[L::kBarOFull + i], 1);
    }
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bars[L::kBarKvFull + s], 1);
      mbar_init(&bars[L::kBarKvEmpty + s], NQ);  // released by both MMA issuers
    }
    for (int i = 0; i < NQ; ++i) mbar_init(&bars[L::kBarDrain + i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const WaitCtl ctl{abort_flag, p.timeout_ns};
  constexpr unsigned long long kDrainNs = 50ull * 1000 * 1000;

  if (wg == 2) {
    if (warp == kLoadWarp && lane == 0) {
      // =========================== TMA producer ===========================
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint8_t* sQ = smem + L::kQOff;
      uint32_t q_cnt[NQ] = {0, 0};
      int issued = 0;  // loads issued into the ring (K and V alternate)
      for_each_tile(p, [&](const WorkTile& w) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
          const TileRange& t = w.tr(i);
          if (!t.part) continue;
          if (!mbar_wait(&bars[L::kBarQEmpty + i], (q_cnt[i] & 1u) ^ 1u, ctl)) return false;
          mbar_arrive_expect_tx(&bars[L::kBarQFull + i], L::kTileBytes);
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(sQ + i * L::kTileBytes + h * L::kHalfBytes, &tmQ, &bars[L::kBarQFull + i], h * 64, t.r0,
                        w.bh);
          ++q_cnt[i];
        }
        // ring order K_0, then (K_{n+1}, V_n) per position, V_{T-1} last: each key tile's
        // S is issued one tile ahead of its neighbour's P.V
        const int T = w.ks.count();
        for (int x = 0; x < 2 * T; ++x) {
          const bool is_v = x > 0 && (x == 2 * T - 1 || (x & 1) == 0);
          const int n = is_v ? (x == 2 * T - 1 ? T - 1 : (x - 2) / 2) : (x == 0 ? 0 : (x + 1) / 2);
          const int j = w.ks.at(n);
          const int s = issued % L::kStages;
          const uint32_t fill = issued / L::kStages;
          if (!mbar_wait(&bars[L::kBarKvEmpty + s], (fill & 1u) ^ 1u, ctl)) return false;
          uint8_t* dst = smem + L::kRingOff + s * L::kTileBytes;
          mbar_arrive_expect_tx(&bars[L::kBarKvFull + s], L::kTileBytes);
          for (int h = 0; h < L::kHalves; ++h)
            tma_load_3d(dst + h * L::kHalfBytes, is_v ? &tmV : &tmK, &bars[L::kBarKvFull + s], h * 64, j * BN,
                        w.kvh);
          ++issued;
        }
        return true;
      });
      if (*abort_flag) {
        // let the copies already in flight land before the CTA's shared memory goes away
        int no_abort = 0;
        const WaitCtl c{&no_abort, kDrainNs};
        for (int i = 0; i < NQ; ++i)
          if (q_cnt[i] > 0) mbar_wait(&bars[L::kBarQFull + i], (q_cnt[i] - 1) & 1u, c);
        for (int k = issued - 1; k >= 0 && k >= issued - L::kStages; --k)
          mbar_wait(&bars[L::kBarKvFull + (k % L::kStages)], (k / L::kStages) & 1u, c);
      }
    } else if ((warp == kMmaWarp || warp == kMmaWarp + 1) && lane == 0) {
      // =========================== MMA issuers ===========================
      // One issuing thread per query tile (warp 9: Q0, warp 10: Q1).  P lives in shared
      // memory, so S of the next key tile only has to wait until the softmax has read the
      // current S into registers: per position n the thread issues S_n (once S_{n-1} is
      // read), then P_{n-1} V_{n-1} in two 64-key halves (as each half of P is stored).
      // Every K/V slot is released by both issuers (count 2): with a commit after the MMAs
      // that read it, or a plain arrive when its query tile does not use that key tile
      // (after the fill has landed, so a thread can never arrive ahead into the slot's
      // next phase).
      const int i = warp - kMmaWarp;
      constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, 0, 0);   // Q (K-major) x K (K-major)
      constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, D, 0, 1);   // P (K-major) x V (MN-major)
      // Descriptor of the first 16-column K step of each operand tile; later steps add
      // their byte offset / 16 to the start-address field (no carry: addresses < 256 KB).
      const uint64_t dq = smem_desc_sw128(smem_addr(smem + L::kQOff + i * L::kTileBytes), 16, 1024);
      const uint64_t dpv = smem_desc_sw128(smem_addr(smem + L::kPOff + i * L::kPBytes), 16, 1024);
      const uint64_t dring = smem_desc_sw128(smem_addr(smem + L::kRingOff), 16, 1024);
      const uint64_t dvring = smem_desc_sw128(smem_addr(smem + L::kRingOff), L::kHalfBytes, 1024);
      const uint32_t d_s = tmem + L::col_s(i);
      const uint32_t d_o = tmem + L::col_o(i);
      uint32_t q_cnt = 0, g_s = 0, g_p = 0;
      int used = 0;  // ring loads consumed before the current work tile

      for_each_tile(p, [&](const WorkTile& w) {
        const TileRange& t = w.tr(i);
        const int T = w.ks.count();
        // this query tile's key tiles as positions in the work tile's sequence: each of
        // its runs lies inside one run of the sequence, so it is a run of positions too
        int sa0 = 0, sa1 = 0, sb0 = 0, sb1 = 0;
        if constexpr (kSinks) {
          const int na = w.ks.a1 - w.ks.a0;
          if (t.ks.a1 > t.ks.a0) {
            sa0 = (t.ks.a0 >= w.ks.a0 && t.ks.a0 < w.ks.a1) ? t.ks.a0 - w.ks.a0 : na + (t.ks.a0 - w.ks.b0);
            sa1 = sa0 + (t.ks.a1 - t.ks.a0);
          }
          if (t.ks.b1 > t.ks.b0) {
            sb0 = (t.ks.b0 >= w.ks.a0 && t.ks.b0 < w.ks.a1) ? t.ks.b0 - w.ks.a0 : na + (t.ks.b0 - w.ks.b0);
            sb1 = sb0 + (t.ks.b1 - t.ks.b0);
          }
        } else if (t.ks.b1 > t.ks.b0) {  // one run each
          sb0 = t.ks.b0 - w.ks.b0;
          sb1 = t.ks.b1 - w.ks.b0;
        }
        const int n_first = sa1 > sa0 ? sa0 : sb0;
        const int n_last = sb1 > sb0 ? sb1 - 1 : sa1 - 1;
        auto uses = [&](int n) { return (kSinks && n >= sa0 && n < sa1) || (n >= sb0 && n < sb1); };
        uint32_t o_acc = 0;
        // V_n: O_i (+)= P_i V_n in two halves of 64 keys, or release
        auto pv = [&](int n) -> bool {
          const int vidx = used + (n == T - 1 ? 2 * T - 1 : 2 * n + 2);
          const int vslot = vidx % L::kStages;
          if (!mbar_wait(&bars[L::kBarKvFull + vslot], (vidx / L::kStages) & 1u, ctl)) return false;
          if (!uses(n)) {
            mbar_arrive(&bars[L::kBarKvEmpty + vslot]);
            return true;
          }
          const uint64_t dv = dvring + ((vslot * L::kTileBytes) >> 4);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // P half h stored (by the softmax warps' generic-proxy stores, fenced for the
            // async proxy) and, for half 0, O rescaled in TMEM
            if (!mbar_wait(&bars[L::kBarPFull + 2 * i + h], g_p & 1u, ctl)) return false;
            tc_fence_after();
            // A = 16 keys of P (32 B of each 128-byte swizzled row; the halves are one
            // 16 KB slab each); B = 16 key rows of V (128 B each; half 1 starts 64 rows in)
            mma_ss_pv4(d_o, dpv + h * (L::kHalfBytes >> 4), dv + h * 512, kIdescPV, (o_acc | h) != 0u);
            mma_commit(&bars[L::kBarPFree + 2 * i + h]);
          }
          o_acc = 1;
          if (n == n_last) mma_commit(&bars[L::kBarOFull + i]);  // O_i is final
          mma_commit(&bars[L::kBarKvEmpty + vslot]);
          ++g_p;
          return true;
        };
        for (int n = 0; n < T; ++n) {
          const int kidx = used + (n == 0 ? 0 : 2 * n - 1);
          const int kslot = kidx % L::kStages;
          if (!mbar_wait(&bars[L::kBarKvFull + kslot], (kidx / L::kStages) & 1u, ctl)) return false;
          if (uses(n)) {
            if (n == n_first) {  // first use of this work tile's Q_i
              if (!mbar_wait(&bars[L::kBarQFull + i], q_cnt & 1u, ctl)) return false;
              ++q_cnt;
            }
            if (g_s > 0) {  // the softmax has the previous S of this query tile in registers
              if (!mbar_wait(&bars[L::kBarSFree + i], (g_s - 1) & 1u, ctl)) return false;
              tc_fence_after();
            }
            mma_ss_kloop<D / 16>(d_s, dq, dring + ((kslot * L::kTileBytes) >> 4), kIdescS);
            mma_commit(&bars[L::kBarSFull + i]);
            if (n == n_last) mma_commit(&bars[L::kBarQEmpty + i]);  // Q_i no longer read
            mma_commit(&bars[L::kBarKvEmpty + kslot]);
            ++g_s;
          } else {
            mbar_arrive(&bars[L::kBarKvEmpty + kslot]);
          }
          if (n > 0 && !pv(n - 1)) return false;
        }
        if (T > 0 && !pv(T - 1)) return false;
        used += 2 * T;
        return true;
      });
      // make sure nothing this thread issued is still running before TMEM is released
      mma_commit(&bars[L::kBarDrain + i]);
      int no_abort = 0;
      mbar_wait(&bars[L::kBarDrain + i], 0, WaitCtl{&no_abort, kDrainNs});
    }
  } else {
    // =========================== softmax warpgroups ===========================
    const int i = wg;               // which Q tile
    const int wq = warp & 3;        // TMEM lane quarter of this warp
    const int trow = wq * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t colS = L::col_s(i);
    const uint32_t colO = L::col_o(i);
    uint8_t* prow = smem + L::kPOff + i * L::kPBytes + trow * 128;  // this row of P (slab 0)
    const int rsw = trow & 7;
    uint32_t s_phase = 0, o_phase = 0, g = 0;
    bool stg_pending = false;  // this warp's last O store may still be reading its rows of P
    // soft-cap series coefficients with the outer scale folded in (tanh's Taylor terms)
    const float cap_b[5] = {p.cap_outer * (-1.0f / 3.0f), p.cap_outer * (2.0f / 15.0f), p.cap_outer * (-17.0f / 315.0f),
                            p.cap_outer * (62.0f / 2835.0f), p.cap_outer * (-1382.0f / 155925.0f)};

    for_each_tile(p, [&](const WorkTile& w) {
      const TileRange& t = w.tr(i);
      if (!t.active) return true;  // rows past Nq: nothing to write
      const int row = t.r0 + trow;
      const int pos = row + p.pos_off;  // the row's position in the key sequence
      const int pr0 = t.r0 + p.pos_off, pr1 = t.r1 + p.pos_off;
      float m = -CUDART_INF_F;  // running reference maximum (log2 units)
      float l = 0.f;            // running sum of P (fp32) relative to m
      float lr = 0.f;           // normaliser of O (l with each tile maximum's P as rounded)
      bool o_valid = false;

      // the query tile's key tiles: the sink run, then the window run
      for (int run = kSinks ? 0 : 1; run < 2; ++run)
      for (int j = run == 0 ? t.ks.a0 : t.ks.b0, j_end = run == 0 ? t.ks.a1 : t.ks.b1; j < j_end; ++j) {
        // tcgen05.ld/st are warp-collective: the whole warp leaves together or not at all
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[L::kBarSFull + i], s_phase, ctl))) return false;
        s_phase ^= 1u;
        tc_fence_after();

        const int k0 = j * BN;
        const bool need_mask = (k0 + BN > p.Nk) || (p.causal && k0 + BN - 1 > pr0) ||
                               (p.window > 0 && pr1 - k0 >= p.window && k0 + BN > p.n_sink);
        // valid keys of this row: columns up to c_hi (keys below Nk, at most the query's
        // own position when causal), minus the hole [h_lo, h_hi) of keys that are below
        // the window and are not attention sinks
        int c_hi = min(BN - 1, p.Nk - 1 - k0);
        if (p.causal) c_hi = min(c_hi, pos - k0);
        const int w_lo = p.window > 0 ? max(0, pos - p.window + 1 - k0) : 0;  // window's first column
        const bool sink_cols = kSinks && p.n_sink > k0;
        const int h_lo = min(max(0, p.n_sink - k0), w_lo);
        const int h_hi = w_lo;

        // The whole row of S in registers with one TMEM round trip, then the row maximum (and
        // minimum, for the soft-cap range check) with three-input max in four independent
        // chains.
        float s[BN];
        load_row<kSinks>(lane_base + colS, need_mask, sink_cols, h_lo, h_hi, c_hi, s);
        // S is in registers: the next key tile's S may overwrite it
        tc_fence_before();
        mbar_arrive(&bars[L::kBarSFree + i]);
        float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F, mx2 = -CUDART_INF_F, mx3 = -CUDART_INF_F;
        float mn0 = CUDART_INF_F, mn1 = CUDART_INF_F;
#pragma unroll
        for (int c = 0; c < BN; c += 8) {
          mx0 = fmax3(mx0, s[c], s[c + 1]);
          mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
          mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
          mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
        }
        if constexpr (kCap) {
#pragma unroll
          for (int c = 0; c < BN; c += 4) {
            mn0 = fmin3(mn0, s[c], s[c + 1]);
            mn1 = fmin3(mn1, s[c + 2], s[c + 3]);
          }
        }
        const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
        const float mn = fminf(mn0, mn1);
        float m_tile;
        if constexpr (kCap)
          m_tile = (mx == -CUDART_INF_F) ? -CUDART_INF_F : p.cap_outer * tanh_cap(mx * p.cap_inner);
        else
          m_tile = mx * p.scale_log2;
        const float m_new = fmaxf(m, m_tile);

        // alpha: the factor O is rescaled by (when the warp has a row that moved its
        // reference); applied below, after the first half of P, when half of the scores
        // no longer occupy registers, and after the previous tile's P.V has landed.
        float alpha = 1.0f;
        bool rescale = false;
        if (!o_valid) {
          m = m_new;  // nothing accumulated yet: adopt the maximum as is
        } else {
          const bool need = m_new > m + kRescaleLog2;
          rescale = __any_sync(0xffffffffu, need);
          if (need) {
            alpha = ex2_approx(m - m_new);
            l *= alpha;
            lr *= alpha;
            m = m_new;
          }
        }
        const float m_use = (m == -CUDART_INF_F) ? 0.f : m;

        // P = exp2(u - m) per 64-key half into its shared-memory slab, once the previous
        // tile's P.V has read the slabs.  lt: fp32 sum of this tile's P; pmax: the P of
        // the tile maximum, recomputed with the same instructions as in make_p (so it is
        // bit-identical to the value packed).
        float lt = 0.f, pmax;
        int wtier = 0;
        if constexpr (kCap) {
          const float amax = fmaxf(fabsf(mx), fabsf(mn)) * p.cap_inner;  // max |x| of the row
          const int tier = need_mask ? 2 : (amax < 0.12f ? 0 : (amax < 0.3f ? 1 : 2));
          wtier = __reduce_max_sync(0xffffffffu, tier);
        }
        if constexpr (!kCap) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float* sh = s + h * kHalf;
            uint8_t* ph = prow + h * L::kHalfBytes;
            // the previous tile's P.V has read both slabs: one wait, on the second half's
            // release, covers both, since the MMAs of one thread complete in the order they
            // were issued (the first wait of a fresh barrier passes: there is no previous
            // tile).  It has nearly always come by now, and every mbarrier test costs a
            // shared-memory round trip, so the first half's release is not waited for.
            if (h == 0 && !__all_sync(0xffffffffu, mbar_wait(&bars[L::kBarPFree + 2 * i + 1], (g & 1u) ^ 1u, ctl)))
              return false;
            if (h == 0 && stg_pending) {  // these rows of P held O for the warp's last TMA store
              if (lane == 0) bulk_wait_group_read0();
              __syncwarp();
              stg_pending = false;
            }
            lt += make_p<PMode::kPlain>(sh, ph, rsw, p.scale_log2, 0.f, 0.f, m_use);
            fence_proxy_async_smem();  // the tensor core reads P through the async proxy
            if (h == 0 && rescale) {
              // O must hold the previous tile's whole P.V: its second half has landed, as the
              // wait above has shown
              tc_fence_after();
#pragma unroll 1
              for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32_wait(lane_base + colO + c * 32, r);
#pragma unroll
                for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
                tmem_st32(lane_base + colO + c * 32, r);
              }
              tmem_wait_st();
            }
            // this half of P is stored (and O rescaled): its P.V can start
            tc_fence_before();
            mbar_arrive(&bars[L::kBarPFull + 2 * i + h]);
          }
        } else {
          // Soft-capped launches run both halves through one loop body: their three P tiers
          // are long code, and the smaller loop measured faster (+8 % on the window +
          // soft-cap workloads); the plain launch keeps the unrolled form.
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            const float* sh = s;  // the half being converted is always in s[0 .. 63]
            uint8_t* ph = prow + h * L::kHalfBytes;
            // as above: one wait for both slabs of the previous tile's P
            if (h == 0 && !__all_sync(0xffffffffu, mbar_wait(&bars[L::kBarPFree + 2 * i + 1], (g & 1u) ^ 1u, ctl)))
              return false;
            if (h == 0 && stg_pending) {  // these rows of P held O for the warp's last TMA store
              if (lane == 0) bulk_wait_group_read0();
              __syncwarp();
              stg_pending = false;
            }
            if (wtier == 0) {
              lt += make_p<PMode::kCapShort>(sh, ph, rsw, 0.f, p.cap_inner, p.cap_outer, m_use, cap_b);
            } else if (wtier == 1) {
              lt += make_p<PMode::kCapLong>(sh, ph, rsw, 0.f, p.cap_inner, p.cap_outer, m_use, cap_b);
            } else {
              lt += make_p<PMode::kCapGeneral>(sh, ph, rsw, 0.f, p.cap_inner, p.cap_outer, m_use);
            }
            fence_proxy_async_smem();  // the tensor core reads P through the async proxy
            if (h == 0 && rescale) {
              // O must hold the previous tile's whole P.V: its second half has landed, as the
              // wait above has shown
              tc_fence_after();
#pragma unroll 1
              for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32_wait(lane_base + colO + c * 32, r);
#pragma unroll
                for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
                tmem_st32(lane_base + colO + c * 32, r);
              }
              tmem_wait_st();
            }
            // this half of P is stored (and O rescaled): its P.V can start
            tc_fence_before();
            mbar_arrive(&bars[L::kBarPFull + 2 * i + h]);
#pragma unroll
            for (int c = 0; c < kHalf; ++c) s[c] = s[c + kHalf];  // the second half moves down
          }
        }
        ++g;
        if constexpr (!kCap) {
          const float u = fmaf(mx, p.scale_log2, -m_use);
          pmax = ex2_approx(u);
        } else {
          const float xm = mx * p.cap_inner;
          if (wtier == 0)
            pmax = ex2_approx(cap_u_pair<true>(make_float2(xm, xm), cap_b, p.cap_outer, make_float2(-m_use, -m_use)).x);
          else if (wtier == 1)
            pmax = ex2_approx(cap_u_pair<false>(make_float2(xm, xm), cap_b, p.cap_outer, make_float2(-m_use, -m_use)).x);
          else
            pmax = ex2_approx(fmaf(tanh_cap(xm), p.cap_outer, -m_use));
        }
        if (mx == -CUDART_INF_F) pmax = 0.f;
        // The normaliser of O is the fp32 sum with the tile maximum's term replaced by its
        // bf16-rounded value, the weight the tensor core actually multiplied V with.  With
        // a stale reference the largest P of a row can be up to 256 and is not exact in
        // bf16; that one term dominates peaked rows, the other roundings average out.
        l += lt;
        lr += lt + (__bfloat162float(__float2bfloat16_rn(pmax)) - pmax);
        o_valid = true;
      }

      // ---- epilogue: O / lr -> bf16, LSE = (m + log2 l) ln 2 (split-KV: fp32 partials;
      // a query tile with no key tile in this chunk writes O = 0 and LSE = -inf)
      if (t.part) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[L::kBarOFull + i], o_phase, ctl))) return false;
        o_phase ^= 1u;
        tc_fence_after();
      }
      const float inv = lr > 0.f ? 1.0f / lr : 0.f;
      if constexpr (kSplit) {
        const int64_t prow = (static_cast<int64_t>(w.split) * p.n_bh + w.bh) * p.Nq + row;
        float* orow = p.o_part + prow * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          if (t.part) {
            tmem_ld32_wait(lane_base + colO + c * 32, r);
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) r[x] = 0u;
          }
          if (row < p.Nq) {
            float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              dst[x] = make_float4(__uint_as_float(r[4 * x]) * inv, __uint_as_float(r[4 * x + 1]) * inv,
                                   __uint_as_float(r[4 * x + 2]) * inv, __uint_as_float(r[4 * x + 3]) * inv);
          }
        }
        if (row < p.Nq) p.lse_part[prow] = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
        return true;
      }
      // O / lr as bf16 into this query tile's P buffer (free: the last P.V, which read
      // it, has completed) in the 128-byte-swizzled layout of the O tensor map, then lane 0
      // of each warp stores the warp's 32 rows with TMA, one 64-column slab per store, with
      // no barrier across warps.  The warp waits for its stores to have read the rows only
      // when it next writes P there (the first tile of the next work tile).
      uint32_t r[D];
      if (t.part) {
        if constexpr (D == 128)
          tmem_ld64x2_wait(lane_base + colO, r);
        else
          tmem_ld64_wait(lane_base + colO, r);
      } else {  // no key at all for this query tile (fewer keys than queries, causal)
#pragma unroll
        for (int x = 0; x < D; ++x) r[x] = 0u;
      }
      uint8_t* stg = smem + L::kPOff + i * L::kPBytes + trow * 128;
      const float2 inv2 = make_float2(inv, inv);
      auto scaled = [&](const uint32_t* rq) {  // two columns of O / lr, packed to bf16
        const float2 v = __fmul2_rn(make_float2(__uint_as_float(rq[0]), __uint_as_float(rq[1])), inv2);
        return pack_bf16x2(v.x, v.y);
      };
#pragma unroll
      for (int q = 0; q < D / 8; ++q) {  // 16-byte chunk q of the row: slab q / 8, chunk q % 8
        const uint32_t* rq = r + 8 * q;
        *reinterpret_cast<uint4*>(stg + (q >> 3) * L::kHalfBytes + (((q & 7) ^ rsw) << 4)) =
            make_uint4(scaled(rq), scaled(rq + 2), scaled(rq + 4), scaled(rq + 6));
      }
      fence_proxy_async_smem();
      __syncwarp();  // the warp's rows are staged
      // each warp stores its own 32 rows (a 32-row box per 64-column slab); a box that
      // starts past Nq has nothing to write, one that ends past it is clipped
      const int wrow = t.r0 + wq * 32;
      if (lane == 0 && wrow < p.Nq) {
        uint8_t* base = smem + L::kPOff + i * L::kPBytes + wq * 32 * 128;
        for (int h = 0; h < L::kHalves; ++h) tma_store_3d(&tmO, base + h * L::kHalfBytes, h * 64, wrow, w.bh);
        bulk_commit_group();
      }
      stg_pending = true;
      if (p.lse != nullptr && row < p.Nq)
        p.lse[static_cast<int64_t>(w.bh) * p.Nq + row] = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
      return true;
    });
    if (lane == 0) bulk_wait_group0();  // the last O stores have completed
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace fa
