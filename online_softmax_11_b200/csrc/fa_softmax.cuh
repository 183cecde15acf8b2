// fa_softmax.cuh -- stand-alone softmax with the online normaliser, and softmax fused
// with top-K ("Online normalizer calculation for softmax", Milakov and Gimelshein).
//
// The classical softmax y_i = exp(x_i - m) / d with m = max_i x_i and d = sum_i exp(x_i - m)
// needs the maximum before the normaliser: one pass for m, one for d, one to write y.  The
// online normaliser keeps both in one pass: a running maximum m and a normaliser d that is
// multiplied by exp(m_old - m_new) whenever the maximum grows.  Two (m, d) pairs over
// disjoint parts of a row merge the same way, so every thread keeps its own pair and the
// block combines them in a tree.  Softmax then reads the row twice (the second read is
// served by L2: see below) and writes it once; softmax + top-K reads it once and writes
// only K probabilities and K indices.
//
// Both kernels are bound by HBM bandwidth, not by arithmetic: one block per row, float4
// loads (16-byte aligned rows, scalar head and tail otherwise), exponentials as exp2 on
// the MUFU pipe of (x - m) log2(e): the maximum stays in the inputs' units, so x - m is
// exact for inputs near the maximum and the product's rounding is relative to |x - m|,
// not to |x| (inputs of 1000 keep full fp32 accuracy).  The softmax block is 1024 threads and two blocks share an
// SM, so about 300 rows are in flight: at 32 K floats a row that is 38 MB, well inside the
// 126 MB L2, which keeps the second read of a row on chip for rows up to a few hundred
// thousand bytes.  Stores and the second read are marked streaming (evict-first).
#pragma once

#include <cuda_runtime.h>
#include <math_constants.h>

#include <cstdint>

namespace fa {
namespace smx {

constexpr int kSoftmaxThreads = 1024;
// top-K blocks: 512 threads (four blocks, four rows in flight per SM) up to rows of 128 K
// floats, 1024 threads (two per SM) for longer rows, where fewer, larger blocks measured
// faster
constexpr int kTopkThreadsShort = 512;
constexpr int kTopkThreadsLong = 1024;
constexpr int kMaxTopK = 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Running maximum and normaliser of a set of inputs: d = sum exp(x - m).
struct MD {
  float m;
  float d;
};

// Merge of two disjoint sets (the block-merge identity): both normalisers move to the
// larger maximum.  A set with no element has m = -inf, d = 0.
__device__ __forceinline__ MD md_merge(MD a, MD b) {
  const float m = fmaxf(a.m, b.m);
  if (m == -CUDART_INF_F) return MD{m, 0.f};
  return MD{m, a.d * ex2((a.m - m) * kLog2e) + b.d * ex2((b.m - m) * kLog2e)};
}

// exp(x - m) as exp2((x - m) log2 e).
__device__ __forceinline__ float exp_rel(float x, float m) { return ex2((x - m) * kLog2e); }

// Add four inputs to a running pair: raise the maximum first, then add the four terms
// relative to it.  While every input so far is -inf the maximum stays -inf and the terms
// are exp(-inf - 0) = 0 (never -inf - -inf).
__device__ __forceinline__ void md_add4(MD& s, float x0, float x1, float x2, float x3) {
  const float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
  if (mx > s.m) {
    s.d = (s.m == -CUDART_INF_F) ? 0.f : s.d * exp_rel(s.m, mx);
    s.m = mx;
  }
  const float m = s.m == -CUDART_INF_F ? 0.f : s.m;
  s.d += (exp_rel(x0, m) + exp_rel(x1, m)) + (exp_rel(x2, m) + exp_rel(x3, m));
}

__device__ __forceinline__ void md_add1(MD& s, float x) {
  if (x > s.m) {
    s.d = (s.m == -CUDART_INF_F) ? 0.f : s.d * exp_rel(s.m, x);
    s.m = x;
  }
  s.d += exp_rel(x, s.m == -CUDART_INF_F ? 0.f : s.m);
}

// (m, d) of the whole block, returned to every thread.  `red` holds 32 pairs.
__device__ __forceinline__ MD block_md(MD s, MD* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    MD t{__shfl_xor_sync(0xffffffffu, s.m, o), __shfl_xor_sync(0xffffffffu, s.d, o)};
    s = md_merge(s, t);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  if (lane == 0) red[warp] = s;
  __syncthreads();
  if (warp == 0) {
    MD t = lane < nwarps ? red[lane] : MD{-CUDART_INF_F, 0.f};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      MD u{__shfl_xor_sync(0xffffffffu, t.m, o), __shfl_xor_sync(0xffffffffu, t.d, o)};
      t = md_merge(t, u);
    }
    if (lane == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// A row split into a scalar head (up to 3 elements, until the 16-byte boundary), a body
// of float4 and a scalar tail.
struct RowSplit {
  int head, n4, tail;
};

__device__ __forceinline__ RowSplit split_row(const float* row, int V) {
  RowSplit r;
  const int mis = static_cast<int>((reinterpret_cast<uintptr_t>(row) >> 2) & 3u);
  r.head = min(V, (4 - mis) & 3);
  r.n4 = (V - r.head) >> 2;
  r.tail = V - r.head - 4 * r.n4;
  return r;
}

// One block per row: pass 1 reads the row and builds (m, d); pass 2 reads it again and
// writes y = exp(x - m) / d.  lse (optional) = m + ln d.
__global__ void __launch_bounds__(kSoftmaxThreads, 2)
    softmax_online_kernel(const float* __restrict__ x, float* __restrict__ y, float* __restrict__ lse, int V) {
  __shared__ MD red[32];
  const int64_t r = blockIdx.x;
  const float* xr = x + r * V;
  float* yr = y + r * V;
  const RowSplit sp = split_row(xr, V);
  const float4* x4 = reinterpret_cast<const float4*>(xr + sp.head);
  const int tid = threadIdx.x, nt = blockDim.x;

  MD s{-CUDART_INF_F, 0.f};
  if (tid < sp.head) md_add1(s, xr[tid]);
  if (tid < sp.tail) md_add1(s, xr[sp.head + 4 * sp.n4 + tid]);
  for (int i = tid; i < sp.n4; i += nt) {
    const float4 v = __ldg(x4 + i);
    md_add4(s, v.x, v.y, v.z, v.w);
  }
  const MD t = block_md(s, red);
  const float m = t.m == -CUDART_INF_F ? 0.f : t.m;
  const float inv = 1.0f / t.d;

  float4* y4 = reinterpret_cast<float4*>(yr + sp.head);
  if (tid < sp.head) yr[tid] = exp_rel(xr[tid], m) * inv;
  if (tid < sp.tail) {
    const int c = sp.head + 4 * sp.n4 + tid;
    yr[c] = exp_rel(xr[c], m) * inv;
  }
  for (int i = tid; i < sp.n4; i += nt) {
    const float4 v = __ldcs(x4 + i);  // last use of the row
    float4 o;
    o.x = exp_rel(v.x, m) * inv;
    o.y = exp_rel(v.y, m) * inv;
    o.z = exp_rel(v.z, m) * inv;
    o.w = exp_rel(v.w, m) * inv;
    __stcs(y4 + i, o);
  }
  if (lse != nullptr && tid == 0) lse[r] = t.m + __log2f(t.d) * kLn2;
}

// ---------------------------------------------------------------------------------
// softmax + top-K
// ---------------------------------------------------------------------------------

// Order of the top-K list: larger value first, equal values by lower index.
__device__ __forceinline__ bool before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// A thread's list of its KMAX best (value, index), best first, in the order of `before`.
// Empty slots hold (-inf, INT_MAX), so a real -inf input still enters an empty slot; a
// thread visits its indices in increasing order, so a later equal value never displaces
// an earlier one.
template <int KMAX>
struct TopList {
  float v[KMAX];
  int i[KMAX];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      v[k] = -CUDART_INF_F;
      i[k] = 0x7fffffff;
    }
  }
  __device__ __forceinline__ void insert(float val, int idx) {
    if (!before(val, idx, v[KMAX - 1], i[KMAX - 1])) return;
    v[KMAX - 1] = val;
    i[KMAX - 1] = idx;
#pragma unroll
    for (int k = KMAX - 1; k > 0; --k) {
      if (before(v[k], i[k], v[k - 1], i[k - 1])) {
        const float tv = v[k];
        v[k] = v[k - 1];
        v[k - 1] = tv;
        const int ti = i[k];
        i[k] = i[k - 1];
        i[k - 1] = ti;
      }
    }
  }
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int k = 0; k < KMAX - 1; ++k) {
      v[k] = v[k + 1];
      i[k] = i[k + 1];
    }
    v[KMAX - 1] = -CUDART_INF_F;
    i[KMAX - 1] = 0x7fffffff;
  }
};

// float <-> int with the same order, for the warp's integer max reduction.
__device__ __forceinline__ int float_key(float f) {
  const int b = __float_as_int(f);
  return b ^ ((b >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float key_float(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7fffffff)); }

// K rounds over the 32 lanes' lists: each round the best head of the warp is taken and
// its lane pops it.  Round k's winner is returned in (out_v[k], out_i[k]) on every lane.
template <int KMAX>
__device__ __forceinline__ void warp_topk(TopList<KMAX>& L, int K, float* out_v, int* out_i) {
  for (int k = 0; k < K; ++k) {
    float bv = L.v[0];
    int bi = L.i[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (before(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (L.i[0] == bi && L.v[0] == bv) L.pop();
    if ((threadIdx.x & 31) == 0) {
      out_v[k] = bv;
      out_i[k] = bi;
    }
  }
}

// The K-th largest of the block's per-thread values `lm` (with multiplicity), or a value
// below it: each warp takes its own K-th largest (K rounds of the warp maximum, removing
// every lane that holds it), the block the largest of those.  Any of them is at most the
// block's K-th largest, which is what the filter below needs.
__device__ __forceinline__ float block_kth_bound(float lm, int K, float* red_f) {
  int key = float_key(lm);
  int taken = 0;
  float kth = -CUDART_INF_F;
  for (int k = 0; k < K && taken < K; ++k) {
    const int mx = __reduce_max_sync(0xffffffffu, key);
    const unsigned hit = __ballot_sync(0xffffffffu, key == mx);
    taken += __popc(hit);
    kth = key_float(mx);
    if (key == mx) key = float_key(-CUDART_INF_F) - 1;  // below every float key
  }
  if (taken < K) kth = -CUDART_INF_F;  // the warp holds fewer than K values
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red_f[warp] = kth;
  __syncthreads();
  float b = -CUDART_INF_F;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = fmaxf(b, red_f[w]);
  return b;
}

// One block per row, three steps:
//  1. one read of the row from HBM: the online (m, d) and each thread's largest input;
//  2. tau = a lower bound on the row's K-th largest input (block_kth_bound of the
//     threads' maxima: the K largest of them are K distinct inputs);
//  3. a second read -- from L2: two 1024-thread blocks per SM keep about 300 rows in
//     flight, 38 MB at 32 K floats a row -- collects the inputs >= tau into shared
//     memory (typically a handful), and one warp picks the top K of them.
// If more than kCand inputs are >= tau (rows of equal values), step 3 instead scans the
// row with a per-thread list of the KMAX best.
constexpr int kCand = 1024;

template <int KMAX, int kTopkThreads>
__global__ void __launch_bounds__(kTopkThreads, 2048 / kTopkThreads)
    softmax_topk_kernel(const float* __restrict__ x, float* __restrict__ probs, int* __restrict__ idx,
                        float* __restrict__ lse, int V, int K) {
  __shared__ MD red[32];
  __shared__ float red_f[32];
  __shared__ float cand_v[kCand];
  __shared__ int cand_i[kCand];
  __shared__ int n_cand;
  const int64_t r = blockIdx.x;
  const float* xr = x + r * V;
  const RowSplit sp = split_row(xr, V);
  const float4* x4 = reinterpret_cast<const float4*>(xr + sp.head);
  const int tid = threadIdx.x, nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int tail0 = sp.head + 4 * sp.n4;

  if (tid == 0) n_cand = 0;
  MD s{-CUDART_INF_F, 0.f};
  float lm = -CUDART_INF_F;
  if (tid < sp.head) {
    md_add1(s, xr[tid]);
    lm = xr[tid];
  }
  if (tid < sp.tail) {
    md_add1(s, xr[tail0 + tid]);
    lm = fmaxf(lm, xr[tail0 + tid]);
  }
  int i = tid;
  for (; i + 3 * nt < sp.n4; i += 4 * nt) {  // four loads in flight per thread
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(x4 + i + u * nt);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      md_add4(s, v[u].x, v[u].y, v[u].z, v[u].w);
      lm = fmaxf(lm, fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w)));
    }
  }
  for (; i < sp.n4; i += nt) {
    const float4 v = __ldg(x4 + i);
    md_add4(s, v.x, v.y, v.z, v.w);
    lm = fmaxf(lm, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
  }
  const MD t = block_md(s, red);  // its barriers also order n_cand = 0 before the appends
  const float tau = block_kth_bound(lm, K, red_f);

  auto keep = [&](float val, int c) {
    if (val >= tau) {
      const int slot = atomicAdd(&n_cand, 1);
      if (slot < kCand) {
        cand_v[slot] = val;
        cand_i[slot] = c;
      }
    }
  };
  if (tid < sp.head) keep(xr[tid], tid);
  if (tid < sp.tail) keep(xr[tail0 + tid], tail0 + tid);
  int j = tid;
  for (; j + 3 * nt < sp.n4; j += 4 * nt) {  // four loads in flight per thread
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(x4 + j + u * nt);  // last use of the row
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w)) >= tau) {
        const int c = sp.head + 4 * (j + u * nt);
        keep(v[u].x, c);
        keep(v[u].y, c + 1);
        keep(v[u].z, c + 2);
        keep(v[u].w, c + 3);
      }
    }
  }
  for (int i = j; i < sp.n4; i += nt) {
    const float4 v = __ldcs(x4 + i);  // last use of the row
    if (fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)) >= tau) {
      const int c = sp.head + 4 * i;
      keep(v.x, c);
      keep(v.y, c + 1);
      keep(v.z, c + 2);
      keep(v.w, c + 3);
    }
  }
  __syncthreads();
  const int nc = n_cand;
  if (nc > kCand) {
    // many ties at the bound: every thread keeps its KMAX best of the row, the warps
    // merge them, and warp 0 merges the warps' lists (cand_* are reused for them)
    TopList<KMAX> L;
    L.init();
    if (tid < sp.head) L.insert(xr[tid], tid);
    for (int i = tid; i < sp.n4; i += nt) {
      const float4 v = __ldcs(x4 + i);
      const int c = sp.head + 4 * i;
      L.insert(v.x, c);
      L.insert(v.y, c + 1);
      L.insert(v.z, c + 2);
      L.insert(v.w, c + 3);
    }
    if (tid < sp.tail) L.insert(xr[tail0 + tid], tail0 + tid);
    __syncthreads();  // everyone has read n_cand
    warp_topk<KMAX>(L, K, cand_v + warp * KMAX, cand_i + warp * KMAX);
    __syncthreads();
  }
  if (warp == 0) {
    // warp 0: lane l holds candidates l, l + 32, ... (or warp l's list after the scan)
    TopList<KMAX> W;
    W.init();
    if (nc <= kCand) {
      for (int c = lane; c < nc; c += 32) W.insert(cand_v[c], cand_i[c]);
    } else if (lane < (nt >> 5)) {
      for (int k = 0; k < K; ++k) W.insert(cand_v[lane * KMAX + k], cand_i[lane * KMAX + k]);
    }
    __syncwarp();
    warp_topk<KMAX>(W, K, cand_v, cand_i);  // winners over cand_[0..K): already read
    __syncwarp();
    const float m = t.m == -CUDART_INF_F ? 0.f : t.m;
    const float inv = 1.0f / t.d;
    for (int k = lane; k < K; k += 32) {
      probs[r * K + k] = exp_rel(cand_v[k], m) * inv;
      idx[r * K + k] = cand_i[k];
    }
    if (lse != nullptr && lane == 0) lse[r] = t.m + __log2f(t.d) * kLn2;
  }
}

}  // namespace smx
}  // namespace fa
