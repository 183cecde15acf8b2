// fa_merge.cuh -- combine split-KV partial results into O and LSE.
//
// Split-KV cuts the keys of every query row into contiguous chunks; chunk s yields its own
// normalised output O_s and log-sum-exp LSE_s = m_s + ln l_s.  "Module 16: Efficient and
// Long Attention", section 16.2, gives the merge of two blocks, repeated for more blocks:
// with the common reference m, l = sum_s e^(m_s - m) l_s and O = sum_s (e^(m_s - m) l_s / l) O_s.
// Taking m = max_s LSE_s, the weight e^(m_s - m) l_s of chunk s is e^(LSE_s - m), so each
// row needs only its LSE_s: w_s = exp(LSE_s - m), l = sum w_s, O = sum w_s O_s / l,
// LSE = m + ln l.  A chunk with no valid key has LSE_s = -inf and weight 0.
//
// One warp per query row; lane c owns D/32 consecutive columns (vector loads).  The pass
// reads num_splits x (D + 1) floats and writes D bf16 + one float per row: bound by HBM.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include <cstdint>

namespace fa {

constexpr int kMergeRowsPerBlock = 8;

template <int D>
__global__ void __launch_bounds__(32 * kMergeRowsPerBlock)
    fa_merge_splits_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                           __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int64_t rows, int num_splits) {
  constexpr int kPer = D / 32;  // columns per lane: 4 (d = 128) or 2 (d = 64)
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;

  float m = -CUDART_INF_F;
  for (int s = 0; s < num_splits; ++s) m = fmaxf(m, lse_part[s * rows + row]);

  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
  float l = 0.f;
  if (m != -CUDART_INF_F) {
    for (int s = 0; s < num_splits; ++s) {
      const float ls = lse_part[s * rows + row];
      const float w = (ls == -CUDART_INF_F) ? 0.f : expf(ls - m);
      l += w;
      const float* src = o_part + (s * rows + row) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
      }
    }
  }
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  __nv_bfloat16* dst = o + row * D + lane * kPer;
#pragma unroll
  for (int c = 0; c < kPer; c += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + c) = __floats2bfloat162_rn(acc[c] * inv, acc[c + 1] * inv);
  if (lane == 0 && lse != nullptr) lse[row] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
}

}  // namespace fa
