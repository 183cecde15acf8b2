// fa_decode.cuh -- attention for few query rows per key/value head (decoding against a
// KV cache, or short cross-attention): g = Hq / Hkv query heads x Nq rows <= 16.
//
// The tensor-core kernel gives every query tile 128 rows; with one query row per head
// nearly all of that work is padding and the per-tile chain S -> softmax -> P -> P.V sets
// the pace, far below the HBM bandwidth that bounds this case (each key/value row is used
// by at most 16 query rows).  Here the query rows of one key/value head -- all g heads of
// the group, so K and V cross HBM once for the group -- form one 16-row block, and the
// online softmax of the pages runs per warp:
//
//  * a block of 4 warps owns one (batch, key/value head, key chunk); warp w streams key
//    tiles w, w + 4, ... of the chunk (32 keys each) through its own 3-stage ring of TMA
//    loads (K and V tiles, 128-byte swizzle, rows past Nk read as zero);
//  * per tile: S = Q K^T (16 x 32) and O += P V (16 x d) with warp-level bf16 MMAs
//    (m16n8k16, fp32 accumulators in registers; P goes from the S accumulators to the A
//    operand in registers), the running maximum / sum / rescale of the online softmax
//    in between ("Module 16: Efficient and Long Attention", section 16.2);
//  * the four warps' (m, l, O) are merged with the section's two-block identities, then
//    O / l and LSE are written (or, with split-KV, fp32 partials for the merge kernel).
//
// Masks are those of the tensor-core kernel: query row i at key position i + Nk - Nq,
// causal, window, attention sinks, soft-cap.  Waits are bounded like everywhere else.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa {
namespace dec {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kRows = 16;       // query rows per block (the MMA's M)
constexpr int kKeys = 32;       // keys per tile
constexpr int kStages = 3;      // ring depth per warp
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct Smem {
  static constexpr int kSlabBytes = kKeys * 128;            // 32 rows x 64 bf16
  static constexpr int kTileBytes = (D / 64) * kSlabBytes;  // K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;        // K then V
  static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
  static constexpr int kMergeBytes = kWarps * kRows * (D + 2) * 4;  // O, m, l per warp
  static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  static constexpr int kBarOff = kDataBytes;
  static constexpr int kBytes = kBarOff + kWarps * kStages * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

struct Params {
  const __nv_bfloat16* q;  // [B, Hq, Nq, d]
  __nv_bfloat16* o;        // [B, Hq, Nq, d]
  float* lse;              // [B, Hq, Nq] or null
  int Hq, Hkv, Nq, Nk, group;
  int n_bh;                // B * Hq
  int causal, window, n_sink;
  float scale_log2;        // scale * log2(e)
  int use_softcap;
  float cap_inner, cap_outer;  // scale / softcap, softcap * log2(e)
  int num_splits;          // 1: plain outputs; > 1: partials
  float* o_part;           // [num_splits][B*Hq][Nq][d]
  float* lse_part;         // [num_splits][B*Hq][Nq]
  unsigned long long timeout_ns;
};

// Byte offset of (row, column c in 0..63) in a 32 x 64 bf16 slab written by TMA with
// 128-byte swizzle: the 16-byte chunk index is XORed with the row modulo 8.
__device__ __forceinline__ uint32_t swz(int row, int c) {
  return static_cast<uint32_t>(row * 128 + ((((c >> 3) ^ row) & 7) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Soft-cap in log2 units: softcap * tanh(s * scale / softcap) * log2(e).
__device__ __forceinline__ float capped(float s, const Params& p) {
  return p.use_softcap ? p.cap_outer * tanhf(s * p.cap_inner) : s * p.scale_log2;
}

// Key tiles of a block: a run of sink tiles [a0, a1) and the window's run [b0, b1).
struct Runs {
  int a0, a1, b0, b1;
  __device__ int count() const { return (a1 - a0) + (b1 - b0); }
  __device__ int at(int n) const { return n < a1 - a0 ? a0 + n : b0 + (n - (a1 - a0)); }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const Params p) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  int* abort_flag = reinterpret_cast<int*>(smem + S::kBarOff + kWarps * kStages * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const int split = blockIdx.x % p.num_splits;
  const int kvh = blockIdx.x / p.num_splits;  // b * Hkv + key/value head
  const int b = kvh / p.Hkv;
  const int R = p.group * p.Nq;  // valid rows: row r = head-in-group (r / Nq), query (r % Nq)

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWarps * kStages; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl ctl{abort_flag, p.timeout_ns};

  // ---- key tiles of this block: the tiles any valid row needs, then this chunk of them
  const int pos_off = p.Nk - p.Nq;
  const int p_min = pos_off, p_max = p.Nq - 1 + pos_off;  // positions of the first / last query
  const int ntiles = (p.Nk + kKeys - 1) / kKeys;
  int hi = ntiles, lo = 0;
  if (p.causal) hi = p_max < 0 ? 0 : min(ntiles, p_max / kKeys + 1);
  if (p.window > 0) lo = min(hi, max(0, p_min - p.window + 1) / kKeys);
  Runs all{0, 0, lo, hi};
  if (p.window > 0 && p.n_sink > 0) {
    const int st = min(hi, (p.n_sink + kKeys - 1) / kKeys);
    if (lo <= st) all.b0 = 0;
    else all.a1 = st;
  }
  const int T = all.count();
  const int c0 = (split * T) / p.num_splits, c1 = ((split + 1) * T) / p.num_splits;
  const int nmine = c1 - c0;  // tiles of this chunk; warp w takes positions w, w + 4, ...

  // ---- Q as the MMA's A operand, kept in registers: rows g and g + 8, columns of k-step ks
  uint32_t qa[D / 16][4];
  {
    auto qrow = [&](int r) -> const __nv_bfloat16* {
      const int h = r / p.Nq, i = r - h * p.Nq;
      const int hq = (kvh - b * p.Hkv) * p.group + h;
      return p.q + ((static_cast<int64_t>(b) * p.Hq + hq) * p.Nq + i) * D;
    };
    const __nv_bfloat16* r0 = g < R ? qrow(g) : nullptr;
    const __nv_bfloat16* r1 = g + 8 < R ? qrow(g + 8) : nullptr;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int c = ks * 16 + 2 * t;
      qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t*>(r0 + c) : 0u;
      qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t*>(r1 + c) : 0u;
      qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t*>(r0 + c + 8) : 0u;
      qa[ks][3] = r1 ? *reinterpret_cast<const uint32_t*>(r1 + c + 8) : 0u;
    }
  }
  // query positions of this thread's two rows (padding rows see no key)
  const int pos0 = g < R ? (g % p.Nq) + pos_off : -0x40000000;
  const int pos1 = g + 8 < R ? ((g + 8) % p.Nq) + pos_off : -0x40000000;

  // ---- this warp's ring
  uint8_t* ring = smem + warp * kStages * S::kStageBytes;
  uint64_t* wbar = bars + warp * kStages;
  int issued = 0;  // tiles whose loads this warp has issued
  auto issue = [&](int k) {  // k-th tile of this warp (chunk position warp + 4 k)
    const int j = all.at(c0 + warp + kWarps * k);
    const int s = k % kStages;
    uint8_t* dst = ring + s * S::kStageBytes;
    mbar_arrive_expect_tx(&wbar[s], S::kStageBytes);
#pragma unroll
    for (int sl = 0; sl < D / 64; ++sl) {
      tma_load_3d(dst + sl * S::kSlabBytes, &tmK, &wbar[s], sl * 64, j * kKeys, kvh);
      tma_load_3d(dst + S::kTileBytes + sl * S::kSlabBytes, &tmV, &wbar[s], sl * 64, j * kKeys, kvh);
    }
  };
  const int my_tiles = nmine > warp ? (nmine - warp + kWarps - 1) / kWarps : 0;
  if (lane == 0) {
    if (warp == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    for (int k = 0; k < my_tiles && k < kStages; ++k) issue(k);
  }
  issued = my_tiles < kStages ? my_tiles : kStages;

  float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F;  // running maxima (log2 units), rows g, g + 8
  float l0 = 0.f, l1 = 0.f;                      // this thread's part of the running sums
  float oacc[D / 8][4];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.f;

  bool ok = true;
  int done = 0;  // tiles consumed
  for (int k = 0; k < my_tiles; ++k) {
    const int s = k % kStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&wbar[s], (k / kStages) & 1u, ctl))) {
      ok = false;
      break;
    }
    const int j = all.at(c0 + warp + kWarps * k);
    const int k0 = j * kKeys;
    const uint32_t kbase = smem_addr(ring + s * S::kStageBytes);
    const uint32_t vbase = kbase + S::kTileBytes;

    // S = Q K^T: 4 n-blocks of 8 keys; B fragments by ldmatrix (keys are rows)
    float sc[4][4];
#pragma unroll
    for (int nb = 0; nb < 4; ++nb) sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int nbp = 0; nbp < 2; ++nbp) {
        const int mi = lane >> 3;
        const int key = (2 * nbp + (mi >> 1)) * 8 + (lane & 7);
        const int col = ks * 16 + (mi & 1) * 8;
        uint32_t b00, b01, b10, b11;
        ldsm_x4(kbase + (col >> 6) * S::kSlabBytes + swz(key, col & 63), b00, b01, b10, b11);
        mma_bf16_16816(sc[2 * nbp], qa[ks], b00, b01);
        mma_bf16_16816(sc[2 * nbp + 1], qa[ks], b10, b11);
      }
    }

    // scores in log2 units, masked where the tile crosses a boundary of some row
    // (padding rows r >= R have Q = 0: finite scores, never written)
    const bool full = (k0 + kKeys <= p.Nk) && (!p.causal || k0 + kKeys - 1 <= p_min) &&
                      (p.window <= 0 || p_max - k0 < p.window || k0 + kKeys <= p.n_sink);
    float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
    for (int nb = 0; nb < 4; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = capped(sc[nb][e], p);
        if (!full) {
          const int key = k0 + nb * 8 + 2 * t + (e & 1);
          const int pos = e < 2 ? pos0 : pos1;
          const bool valid = key < p.Nk && (!p.causal || key <= pos) &&
                             (p.window <= 0 || pos - key < p.window || key < p.n_sink) && pos > -0x40000000;
          v = valid ? v : -CUDART_INF_F;
        }
        sc[nb][e] = v;
      }
      mx0 = fmaxf(mx0, fmaxf(sc[nb][0], sc[nb][1]));
      mx1 = fmaxf(mx1, fmaxf(sc[nb][2], sc[nb][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float a0 = m0 == -CUDART_INF_F ? 0.f : ex2_approx(m0 - n0);  // -inf guard
    const float a1 = m1 == -CUDART_INF_F ? 0.f : ex2_approx(m1 - n1);
    m0 = n0;
    m1 = n1;
    const float u0 = m0 == -CUDART_INF_F ? 0.f : m0, u1 = m1 == -CUDART_INF_F ? 0.f : m1;
    l0 *= a0;
    l1 *= a1;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      oacc[nd][0] *= a0;
      oacc[nd][1] *= a0;
      oacc[nd][2] *= a1;
      oacc[nd][3] *= a1;
    }
    // P = exp2(s - m) as the A operand of P V (k-step kk covers n-blocks 2kk, 2kk + 1)
    uint32_t pa[2][4];
#pragma unroll
    for (int nb = 0; nb < 4; ++nb) {
      const float p0 = ex2_approx(sc[nb][0] - u0), p1 = ex2_approx(sc[nb][1] - u0);
      const float p2 = ex2_approx(sc[nb][2] - u1), p3 = ex2_approx(sc[nb][3] - u1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      pa[nb >> 1][(nb & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[nb >> 1][(nb & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    // O += P V: k-steps of 16 keys, d in pairs of 8-column n-blocks; B by ldmatrix.trans
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int mi = lane >> 3;
        const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
        const int col = dp * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + (col >> 6) * S::kSlabBytes + swz(key, col & 63), b0, b1, b2, b3);
        mma_bf16_16816(oacc[2 * dp], pa[kk], b0, b1);
        mma_bf16_16816(oacc[2 * dp + 1], pa[kk], b2, b3);
      }
    }
    // the stage is consumed: refill it with this warp's tile k + kStages
    __syncwarp();
    if (issued < my_tiles && lane == 0) {
      fence_proxy_async_smem();  // our generic reads of the stage before the async writes
      issue(issued);
    }
    issued = issued < my_tiles ? issued + 1 : issued;
    ++done;
  }
  if (!ok) {
    // let the copies already in flight land before the block's shared memory goes away
    int no_abort = 0;
    const WaitCtl c{&no_abort, 50ull * 1000 * 1000};
    for (int k = done; k < issued; ++k) mbar_wait(&wbar[k % kStages], (k / kStages) & 1u, c);
  }
  const bool all_ok = __syncthreads_and(ok);
  if (!all_ok) return;

  // ---- merge the four warps (section 16.2's identities) and write
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* mo = reinterpret_cast<float*>(smem);             // [warp][row][D]
  float* mm = mo + kWarps * kRows * D;                    // [warp][row]
  float* ml = mm + kWarps * kRows;                        // [warp][row]
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) {
    const int c = nd * 8 + 2 * t;
    mo[(warp * kRows + g) * D + c] = oacc[nd][0];
    mo[(warp * kRows + g) * D + c + 1] = oacc[nd][1];
    mo[(warp * kRows + g + 8) * D + c] = oacc[nd][2];
    mo[(warp * kRows + g + 8) * D + c + 1] = oacc[nd][3];
  }
  if (t == 0) {
    mm[warp * kRows + g] = m0;
    mm[warp * kRows + g + 8] = m1;
    ml[warp * kRows + g] = l0;
    ml[warp * kRows + g + 8] = l1;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < R * D; e += kThreads) {
    const int r = e / D, c = e - r * D;
    float mstar = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mstar = fmaxf(mstar, mm[w * kRows + r]);
    float L = 0.f, acc = 0.f;
    if (mstar != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = ex2_approx(mm[w * kRows + r] - mstar);  // exp2(-inf) = 0 for empty warps
        L += f * ml[w * kRows + r];
        acc += f * mo[(w * kRows + r) * D + c];
      }
    }
    const int h = r / p.Nq, i = r - h * p.Nq;
    const int64_t bh = static_cast<int64_t>(b) * p.Hq + (kvh - b * p.Hkv) * p.group + h;
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    const float lse = L > 0.f ? (mstar + log2f(L)) * kLn2 : -CUDART_INF_F;
    if (p.num_splits > 1) {
      const int64_t prow = (static_cast<int64_t>(split) * p.n_bh + bh) * p.Nq + i;
      p.o_part[prow * D + c] = acc * inv;
      if (c == 0) p.lse_part[prow] = lse;
    } else {
      p.o[(bh * p.Nq + i) * D + c] = __float2bfloat16_rn(acc * inv);
      if (c == 0 && p.lse != nullptr) p.lse[bh * p.Nq + i] = lse;
    }
  }
}

}  // namespace dec
}  // namespace fa
