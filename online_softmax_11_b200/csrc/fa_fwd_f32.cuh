// fa_fwd_f32.cuh -- fp32 attention forward on the CUDA cores (no tensor cores, no TF32).
//
// The same tile-by-tile online softmax as the tensor-core path, in fp32 throughout,
// for head dimensions 1..128.  It was built for the n = 64, d = 32 f32 workload of
// nx_flashattn_scale.nx, where the streaming loop is checked against a direct softmax
// in f32; accuracy, not throughput, is its job (max-abs error ~1e-7 against fp64).
//
// Work split: one CTA of 8 warps takes 32 query rows of one (batch, query head); each
// warp owns 4 of those rows.  Keys stream through shared memory 32 at a time.  For a
// key tile, lane l computes the scores of key l against the warp's 4 rows (fp32 FMAs
// over d), the warp reduces max / sum with shuffles, and lane l then accumulates
// output columns l, l+32, l+64, l+96 with the tile's probabilities broadcast by shuffle.
// The recurrence per row and tile ("Online Softmax Without the Attention Matrix",
// streaming function; "Module 16", 16.2): m_new = max(m, tile max); the running sum and
// output are multiplied by exp(m - m_new) (0 while m is still -inf, the oxios guard);
// p = exp(s - m_new) is added.  expf is the accurate library exponential.
#pragma once

#include <cstdint>
#include <math_constants.h>

namespace fa {

namespace f32path {
constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 4;
constexpr int kRows = kWarps * kRowsPerWarp;  // 32 query rows per CTA
constexpr int kKeys = 32;                      // keys per tile (one per lane)
constexpr int kMaxD = 128;
constexpr int kThreads = kWarps * 32;
}  // namespace f32path

// Accurate soft-cap kappa * tanh(x / kappa) for the fp32 path: library tanhf.
__device__ __forceinline__ float softcap_f32(float s, float kappa) { return kappa * tanhf(s / kappa); }

template <int DPL>  // output columns per lane: ceil(d / 32)
__global__ void __launch_bounds__(f32path::kThreads)
    fa_fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                      float* __restrict__ o, float* __restrict__ lse, int Hq, int Hkv, int N, int d, float scale,
                      int causal, int window, float softcap, int q_blocks) {
  using namespace f32path;
  extern __shared__ float smem_f32[];
  float* sQ = smem_f32;                   // [kRows][d]
  float* sK = sQ + kRows * d;             // [kKeys][d + 1]  (padded: lane-major reads)
  float* sV = sK + kKeys * (d + 1);       // [kKeys][d]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qb = blockIdx.x % q_blocks;
  const int bh = blockIdx.x / q_blocks;  // b * Hq + hq
  const int b = bh / Hq;
  const int hq = bh - b * Hq;
  const int kvh = b * Hkv + hq / (Hq / Hkv);
  const int row0 = qb * kRows;

  const float* qh = q + (static_cast<int64_t>(bh) * N) * d;
  const float* kh = k + (static_cast<int64_t>(kvh) * N) * d;
  const float* vh = v + (static_cast<int64_t>(kvh) * N) * d;

  for (int idx = tid; idx < kRows * d; idx += kThreads) {
    const int r = idx / d, c = idx - r * d;
    const int row = row0 + r;
    sQ[idx] = row < N ? qh[static_cast<int64_t>(row) * d + c] : 0.f;
  }

  // key range this CTA needs
  const int row_last = min(N, row0 + kRows) - 1;
  int kv_lo = 0, kv_hi = N;
  if (causal) kv_hi = row_last + 1;
  if (window > 0) kv_lo = max(0, row0 - window + 1);

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][DPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -CUDART_INF_F;
    l[r] = 0.f;
#pragma unroll
    for (int t = 0; t < DPL; ++t) acc[r][t] = 0.f;
  }

  for (int key0 = (kv_lo / kKeys) * kKeys; key0 < kv_hi; key0 += kKeys) {
    __syncthreads();  // previous tile fully consumed (and sQ written, first time)
    for (int idx = tid; idx < kKeys * d; idx += kThreads) {
      const int j = idx / d, c = idx - j * d;
      const int key = key0 + j;
      const bool in = key < N;
      sK[j * (d + 1) + c] = in ? kh[static_cast<int64_t>(key) * d + c] : 0.f;
      sV[j * d + c] = in ? vh[static_cast<int64_t>(key) * d + c] : 0.f;
    }
    __syncthreads();

    // scores of key (key0 + lane) against this warp's rows
    float s[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) s[r] = 0.f;
    const float* krow = sK + lane * (d + 1);
    for (int c = 0; c < d; ++c) {
      const float kc = krow[c];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) s[r] = fmaf(sQ[(warp * kRowsPerWarp + r) * d + c], kc, s[r]);
    }

    const int key = key0 + lane;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int row = row0 + warp * kRowsPerWarp + r;
      float sr = s[r] * scale;
      if (softcap > 0.f) sr = softcap_f32(sr, softcap);
      bool valid = key < N && key >= kv_lo;
      if (causal && key > row) valid = false;
      if (window > 0 && row - key >= window) valid = false;
      sr = valid ? sr : -CUDART_INF_F;

      float tmax = sr;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      const float m_new = fmaxf(m[r], tmax);
      // rows with nothing valid yet keep m = -inf; exp(-inf - m_use) = 0 for them
      const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
      const float corr = (m[r] == -CUDART_INF_F) ? 0.f : expf(m[r] - m_use);
      const float p = valid ? expf(sr - m_use) : 0.f;
      float psum = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      l[r] = l[r] * corr + psum;
#pragma unroll
      for (int t = 0; t < DPL; ++t) acc[r][t] *= corr;
      for (int j = 0; j < kKeys; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
        for (int t = 0; t < DPL; ++t) {
          const int c = lane + 32 * t;
          if (c < d) acc[r][t] = fmaf(pj, sV[j * d + c], acc[r][t]);
        }
      }
      m[r] = m_new;
    }
  }

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = row0 + warp * kRowsPerWarp + r;
    if (row >= N) continue;
    const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
    float* orow = o + (static_cast<int64_t>(bh) * N + row) * d;
#pragma unroll
    for (int t = 0; t < DPL; ++t) {
      const int c = lane + 32 * t;
      if (c < d) orow[c] = acc[r][t] * inv;
    }
    if (lse != nullptr && lane == 0)
      lse[static_cast<int64_t>(bh) * N + row] = l[r] > 0.f ? m[r] + logf(l[r]) : -CUDART_INF_F;
  }
}

}  // namespace fa
