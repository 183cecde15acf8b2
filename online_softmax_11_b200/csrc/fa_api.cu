// fa_api.cu -- host side of the C ABI declared in include/fa.h: argument checks, TMA
// descriptors, kernel selection and launch.  Everything here is plain pointers and sizes;
// no framework types cross the boundary.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa.h"
#include "fa_decode.cuh"
#include "fa_fwd_f32.cuh"
#include "fa_fwd_tc.cuh"
#include "fa_merge.cuh"
#include "fa_softmax.cuh"
#include "host_once.h"

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

// Default limit of one device-side wait.  A healthy wait ends in microseconds; the
// limit only has to separate "slow" from "never".
constexpr unsigned long long kWaitLimitNs = 2ull * 1000 * 1000 * 1000;

constexpr int kMaxDevices = 64;

// Per-device facts checked once: compute capability and kernel attributes (a failed
// check is retried by the next call, see host_once.h).
struct DeviceState {
  fa::OnceOnSuccess once;
  int num_sms = 0;
  bool tc_ok = false;  // the tensor-core kernels were built with the launch register count they assume
};
DeviceState g_dev[kMaxDevices];

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (*dev < 0 || *dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Shared-memory size, and a check of the launch register count: one CTA of kThreads
// threads must fit an SM's register file at kLaunchRegs registers each.  A build that
// uses more (or allows fewer threads per block) could not launch, so such a kernel is
// refused here instead.
template <typename K>
cudaError_t prepare_tc_kernel(K kernel, int smem_bytes, bool* regs_ok) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes a;
  e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return e;
  if (a.numRegs > static_cast<int>(fa::tc::kLaunchRegs) || a.maxThreadsPerBlock < fa::tc::kThreads) *regs_ok = false;
  return cudaSuccess;
}

template <int D, bool kSplit, bool kSinks>
cudaError_t set_tc_attributes(bool* regs_ok) {
  constexpr int kSmem = fa::tc::Layout<D>::kSmemLaunch;
  cudaError_t e = prepare_tc_kernel(fa::tc::fa_fwd_tc_kernel<D, kSplit, kSinks, false>, kSmem, regs_ok);
  if (e == cudaSuccess) e = prepare_tc_kernel(fa::tc::fa_fwd_tc_kernel<D, kSplit, kSinks, true>, kSmem, regs_ok);
  return e;
}

struct TcMaps {
  CUtensorMap q, k, v, o;
};

template <int D, bool kSplit, bool kSinks>
void launch_tc_kernel(bool cap, unsigned grid, const TcMaps& m, const fa::tc::Params& p, cudaStream_t s) {
  constexpr int kSmem = fa::tc::Layout<D>::kSmemLaunch;
  if (cap)
    fa::tc::fa_fwd_tc_kernel<D, kSplit, kSinks, true><<<grid, fa::tc::kThreads, kSmem, s>>>(m.q, m.k, m.v, m.o, p);
  else
    fa::tc::fa_fwd_tc_kernel<D, kSplit, kSinks, false><<<grid, fa::tc::kThreads, kSmem, s>>>(m.q, m.k, m.v, m.o, p);
}

template <int D>
void launch_tc_variant(bool split, bool sinks, bool cap, unsigned grid, const TcMaps& m, const fa::tc::Params& p,
                       cudaStream_t s) {
  if (split) {
    if (sinks) launch_tc_kernel<D, true, true>(cap, grid, m, p, s);
    else launch_tc_kernel<D, true, false>(cap, grid, m, p, s);
  } else {
    if (sinks) launch_tc_kernel<D, false, true>(cap, grid, m, p, s);
    else launch_tc_kernel<D, false, false>(cap, grid, m, p, s);
  }
}

int prepare_device(int dev, int* num_sms = nullptr, bool* tc_ok = nullptr) {
  DeviceState& st = g_dev[dev];
  const int status = st.once.run([&]() -> int {
    cudaDeviceProp prop;
    cudaError_t e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (prop.major != 10 || prop.minor != 0) return FA_ERR_UNSUPPORTED;  // built for sm_100a only

    e = cudaFuncSetAttribute(fa::dec::fa_decode_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::dec::Smem<128>::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::dec::fa_decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::dec::Smem<64>::kAlloc);
    bool regs_ok = true;
    if (e == cudaSuccess) e = set_tc_attributes<128, false, false>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<128, true, false>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<128, false, true>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<128, true, true>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<64, false, false>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<64, true, false>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<64, false, true>(&regs_ok);
    if (e == cudaSuccess) e = set_tc_attributes<64, true, true>(&regs_ok);
    st.tc_ok = regs_ok;
    if (e == cudaSuccess)  // two 1024-thread softmax blocks per SM: keep L1 small, shared memory is tiny
      e = cudaFuncSetAttribute(fa::smx::softmax_online_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 10);
    // the fp32 path needs up to 4 * (32 d + 32 (d + 1) + 32 d) bytes = 49280 at d = 128
    const int f32_smem = 64 * 1024;
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_fwd_f32_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, f32_smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_fwd_f32_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, f32_smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_fwd_f32_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, f32_smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_fwd_f32_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, f32_smem);
    if (e != cudaSuccess) return cuda_fail(e);
    st.num_sms = prop.multiProcessorCount;
    return FA_OK;
  });
  if (num_sms) *num_sms = st.num_sms;
  if (tc_ok) *tc_ok = st.tc_ok;
  return status;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [heads, N, d] bf16 tensor viewed as 3-D (d, N, heads) with boxes of 64 columns x
// box_rows rows and 128-byte swizzle, which is the canonical K-major (Q, K) and MN-major
// (V) operand layout of tcgen05.mma and the kernel's O staging layout.  Loads read rows
// past N as zero; stores do not write them.
int make_map(CUtensorMap* map, const void* base, int heads, int N, int d, unsigned box_rows = 128,
             unsigned box_cols = 64, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {box_cols, box_rows, 1};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, elem_strides,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Checks shared by every entry point.  Returns FA_OK, an error, or 1 for "empty problem"
// (no query rows).  With query rows but no keys (Nk == 0) k and v may be NULL.
int check_common(const void* q, const void* k, const void* v, const void* o, int B, int Hq, int Hkv, int Nq, int Nk,
                 int d, float scale, int causal, int window, int n_sink, float softcap) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0 || d < 0) return FA_ERR_BAD_SHAPE;
  if (Hkv == 0 || (Hq % Hkv) != 0) return FA_ERR_BAD_SHAPE;
  if (!std::isfinite(scale) || !(scale > 0.f) || !std::isfinite(softcap) || n_sink < 0) return FA_ERR_BAD_ARG;
  if (window > 0 && !causal) return FA_ERR_UNSUPPORTED;
  // element counts must fit the kernels' index arithmetic
  const long long rows = static_cast<long long>(B) * Hq * Nq;
  const long long kv_rows = static_cast<long long>(B) * Hkv * Nk;
  if (rows > (1ll << 31) - 1 || kv_rows > (1ll << 31) - 1 || static_cast<long long>(B) * Hq > (1ll << 31) - 1)
    return FA_ERR_BAD_SHAPE;
  if (B == 0 || Hq == 0 || Nq == 0) return 1;
  if (d == 0) return FA_ERR_UNSUPPORTED;
  if (!q || !o || (Nk > 0 && (!k || !v))) return FA_ERR_NULL_PTR;
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

int fa_last_cuda_error(void) { return g_last_cuda_error; }

const char* fa_strerror(int code) {
  switch (code) {
    case FA_OK: return "ok";
    case FA_ERR_NULL_PTR: return "a required pointer is NULL";
    case FA_ERR_BAD_SHAPE: return "bad shape (negative size, Hkv == 0, Hq % Hkv != 0 or size overflow)";
    case FA_ERR_UNSUPPORTED: return "unsupported head dimension, mask combination or device";
    case FA_ERR_ALIGN: return "pointer not aligned as required";
    case FA_ERR_BAD_ARG: return "scale must be finite and > 0, softcap finite";
    case FA_ERR_CUDA: return "CUDA call failed (see fa_last_cuda_error)";
    case FA_ERR_TIMEOUT: return "a device-side wait exceeded its limit";
    case FA_ERR_WORKSPACE: return "workspace missing, misaligned or smaller than fa_fwd_splitkv_workspace()";
    case FA_ERR_SCRATCH_LIMIT:
      return "problem needs more split-KV scratch than fa_fwd_splitkv_static's fixed array (FA_STATIC_SCRATCH_BYTES)";
    default: return "unknown error code";
  }
}

}  // extern "C"

namespace {

// O = 0 and LSE = -inf for every row: the merge of zero chunks (query rows, no keys).
int launch_no_keys(void* o, float* lse, long long rows, int d, cudaStream_t s) {
  const unsigned mgrid = static_cast<unsigned>((rows + fa::kMergeRowsPerBlock - 1) / fa::kMergeRowsPerBlock);
  if (d == 128)
    fa::fa_merge_splits_kernel<128><<<mgrid, 32 * fa::kMergeRowsPerBlock, 0, s>>>(
        nullptr, nullptr, static_cast<__nv_bfloat16*>(o), lse, rows, 0);
  else
    fa::fa_merge_splits_kernel<64><<<mgrid, 32 * fa::kMergeRowsPerBlock, 0, s>>>(
        nullptr, nullptr, static_cast<__nv_bfloat16*>(o), lse, rows, 0);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

// Few query rows per key/value head (the whole group's rows fit one 16-row block): the
// decode kernel, one block per (batch, key/value head, key chunk).
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                  int Nk, int d, float scale, int causal, int window, int n_sink, float softcap, int num_splits,
                  float* o_part, float* lse_part, cudaStream_t s) {
  int rc;
  CUtensorMap mk, mv;
  if ((rc = make_map(&mk, k, B * Hkv, Nk, d, fa::dec::kKeys)) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * Hkv, Nk, d, fa::dec::kKeys)) != FA_OK) return rc;
  fa::dec::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.group = Hq / Hkv;
  p.n_bh = B * Hq;
  p.causal = causal ? 1 : 0;
  p.window = window > 0 ? window : 0;
  p.n_sink = window > 0 ? n_sink : 0;
  p.scale_log2 = scale * fa::dec::kLog2e;
  p.use_softcap = softcap > 0.f ? 1 : 0;
  p.cap_inner = softcap > 0.f ? scale / softcap : 0.f;
  p.cap_outer = softcap > 0.f ? softcap * fa::dec::kLog2e : 0.f;
  const bool split = num_splits >= 1;
  p.num_splits = split ? num_splits : 1;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.timeout_ns = kWaitLimitNs;
  const long long blocks = static_cast<long long>(B) * Hkv * p.num_splits;
  if (blocks > 0x7fffffffll) return FA_ERR_BAD_SHAPE;
  // with one chunk the kernel writes bf16 O / LSE itself; with more, fp32 partials
  if (p.num_splits == 1) {
    p.o_part = nullptr;
    p.lse_part = nullptr;
  }
  const unsigned grid = static_cast<unsigned>(blocks);
  if (d == 128)
    fa::dec::fa_decode_kernel<128><<<grid, fa::dec::kThreads, fa::dec::Smem<128>::kAlloc, s>>>(mk, mv, p);
  else
    fa::dec::fa_decode_kernel<64><<<grid, fa::dec::kThreads, fa::dec::Smem<64>::kAlloc, s>>>(mk, mv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  if (p.num_splits > 1) {
    const long long rows = static_cast<long long>(B) * Hq * Nq;
    const unsigned mgrid = static_cast<unsigned>((rows + fa::kMergeRowsPerBlock - 1) / fa::kMergeRowsPerBlock);
    if (d == 128)
      fa::fa_merge_splits_kernel<128><<<mgrid, 32 * fa::kMergeRowsPerBlock, 0, s>>>(
          o_part, lse_part, static_cast<__nv_bfloat16*>(o), lse, rows, num_splits);
    else
      fa::fa_merge_splits_kernel<64><<<mgrid, 32 * fa::kMergeRowsPerBlock, 0, s>>>(
          o_part, lse_part, static_cast<__nv_bfloat16*>(o), lse, rows, num_splits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FA_OK;
}

// Launch the tensor-core kernel: plain (num_splits == 0: bf16 O and fp32 LSE) or split-KV
// (num_splits >= 1: fp32 partials into o_part / lse_part, then the merge kernel).
int launch_tc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
              int Nk, int d, float scale, int causal, int window, int n_sink, float softcap, int num_splits,
              float* o_part, float* lse_part, cudaStream_t s) {
  int rc;
  int dev, num_sms = 0;
  bool tc_ok = false;
  if ((rc = current_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_device(dev, &num_sms, &tc_ok)) != FA_OK) return rc;
  if (Nk == 0) return launch_no_keys(o, lse, static_cast<long long>(B) * Hq * Nq, d, s);
  if ((Hq / Hkv) * static_cast<long long>(Nq) <= fa::dec::kRows)
    return launch_decode(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, n_sink, softcap, num_splits,
                         o_part, lse_part, s);

  if (!tc_ok) return FA_ERR_UNSUPPORTED;  // never launch a kernel whose register split cannot be met
  namespace tc = fa::tc;
  const bool split = num_splits >= 1;
  TcMaps maps;
  if ((rc = make_map(&maps.q, q, B * Hq, Nq, d, tc::BM)) != FA_OK) return rc;
  if ((rc = make_map(&maps.k, k, B * Hkv, Nk, d, tc::BN)) != FA_OK) return rc;
  if ((rc = make_map(&maps.v, v, B * Hkv, Nk, d, tc::BN)) != FA_OK) return rc;
  if (split)
    maps.o = maps.q;  // the split-KV epilogue writes fp32 partials without TMA
  else if ((rc = make_map(&maps.o, o, B * Hq, Nq, d, 32)) != FA_OK)  // one box per warp's 32 rows
    return rc;
  tc::Params p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.pos_off = Nk - Nq;
  p.n_sink = window > 0 ? n_sink : 0;  // sinks only matter beside a window
  p.n_bh = B * Hq;
  p.n_qp = (Nq + tc::NQ * tc::BM - 1) / (tc::NQ * tc::BM);
  p.units_per_head = (p.n_qp + 1) / 2;
  p.causal = causal ? 1 : 0;
  p.window = window > 0 ? window : 0;
  p.scale_log2 = scale * tc::kLog2e;
  p.use_softcap = softcap > 0.f ? 1 : 0;
  p.cap_inner = softcap > 0.f ? scale / softcap : 0.f;
  p.cap_outer = softcap > 0.f ? softcap * tc::kLog2e : 0.f;
  p.timeout_ns = kWaitLimitNs;
  p.num_splits = split ? num_splits : 1;
  p.o_part = o_part;
  p.lse_part = lse_part;

  // the kernel walks split units (head, q-pair, chunk) only for more than one chunk; a
  // single chunk keeps the paired schedule of the plain forward (for_each_tile)
  const long long units = p.num_splits > 1 ? static_cast<long long>(B) * Hq * p.n_qp * p.num_splits
                                           : static_cast<long long>(B) * Hq * p.units_per_head;
  if (units > 0x7fffffffll) return FA_ERR_BAD_SHAPE;
  p.n_units = static_cast<int>(units);
  // persistent: one CTA per SM (never more CTAs than units)
  const unsigned grid = static_cast<unsigned>(units < num_sms ? units : num_sms);
  const bool sinks = p.n_sink > 0;
  const bool cap = p.use_softcap != 0;
  if (d == 128)
    launch_tc_variant<128>(split, sinks, cap, grid, maps, p, s);
  else
    launch_tc_variant<64>(split, sinks, cap, grid, maps, p, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  if (split) {
    const long long rows = static_cast<long long>(B) * Hq * Nq;
    const unsigned mgrid = static_cast<unsigned>((rows + fa::kMergeRowsPerBlock - 1) / fa::kMergeRowsPerBlock);
    if (d == 128)
      fa::fa_merge_splits_kernel<128><<<mgrid, 32 * fa::kMergeRowsPerBlock, 0, s>>>(
          o_part, lse_part, static_cast<__nv_bfloat16*>(o), lse, rows, num_splits);
    else
      fa::fa_merge_splits_kernel<64><<<mgrid, 32 * fa::kMergeRowsPerBlock, 0, s>>>(
          o_part, lse_part, static_cast<__nv_bfloat16*>(o), lse, rows, num_splits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FA_OK;
}

int check_bf16(const void* q, const void* k, const void* v, const void* o, const float* lse, int B, int Hq, int Hkv,
               int Nq, int Nk, int d, float scale, int causal, int window, int n_sink, float softcap) {
  int rc = check_common(q, k, v, o, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, n_sink, softcap);
  if (rc != FA_OK) return rc;  // 1 = empty problem
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || (lse && !aligned(lse, 4)))
    return FA_ERR_ALIGN;
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N, int d,
           float scale, int causal, int window, float softcap, void* stream) {
  int rc = check_bf16(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  return launch_tc(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap, 0, nullptr, nullptr,
                   static_cast<cudaStream_t>(stream));
}

size_t fa_fwd_splitkv_workspace(int B, int Hq, int N, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || N <= 0 || d <= 0 || num_splits < 1) return 0;
  const size_t rows = static_cast<size_t>(B) * Hq * N;
  return static_cast<size_t>(num_splits) * rows * (static_cast<size_t>(d) + 1) * sizeof(float);
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                   int d, float scale, int causal, int window, float softcap, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream) {
  const int rc = check_bf16(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (num_splits < 1 || num_splits > FA_MAX_SPLITS) return FA_ERR_BAD_ARG;  // 0 means "no split" only in fa_fwd_ext
  return fa_fwd_ext(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap, num_splits, workspace,
                    workspace_bytes, stream);
}

int fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
               int Nk, int d, float scale, int causal, int window, int n_sink, float softcap, int num_splits,
               void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_bf16(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, n_sink, softcap);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (num_splits < 0 || num_splits > FA_MAX_SPLITS) return FA_ERR_BAD_ARG;
  if (num_splits == 0)
    return launch_tc(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, n_sink, softcap, 0, nullptr,
                     nullptr, static_cast<cudaStream_t>(stream));
  const size_t need = fa_fwd_splitkv_workspace(B, Hq, Nq, d, num_splits);
  if (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  const size_t rows = static_cast<size_t>(B) * Hq * Nq;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = o_part + static_cast<size_t>(num_splits) * rows * d;
  return launch_tc(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, n_sink, softcap, num_splits, o_part,
                   lse_part, static_cast<cudaStream_t>(stream));
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int Hq, int Hkv, int N,
               int d, float scale, int causal, int window, float softcap, void* stream) {
  int rc = check_common(q, k, v, o, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (d < 1 || d > fa::f32path::kMaxD) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 4) || !aligned(k, 4) || !aligned(v, 4) || !aligned(o, 4) || (lse && !aligned(lse, 4)))
    return FA_ERR_ALIGN;
  int dev;
  if ((rc = current_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_device(dev)) != FA_OK) return rc;

  namespace f = fa::f32path;
  const int q_blocks = (N + f::kRows - 1) / f::kRows;
  const long long grid = static_cast<long long>(B) * Hq * q_blocks;
  if (grid > 0x7fffffffll) return FA_ERR_BAD_SHAPE;
  const size_t smem = sizeof(float) * (static_cast<size_t>(f::kRows) * d + static_cast<size_t>(f::kKeys) * (d + 1) +
                                       static_cast<size_t>(f::kKeys) * d);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float cap = softcap > 0.f ? softcap : 0.f;
  const int win = window > 0 ? window : 0;
  const int dpl = (d + 31) / 32;
  const unsigned g = static_cast<unsigned>(grid);
  switch (dpl) {
    case 1: fa::fa_fwd_f32_kernel<1><<<g, f::kThreads, smem, s>>>(q, k, v, o, lse, Hq, Hkv, N, d, scale, causal, win, cap, q_blocks); break;
    case 2: fa::fa_fwd_f32_kernel<2><<<g, f::kThreads, smem, s>>>(q, k, v, o, lse, Hq, Hkv, N, d, scale, causal, win, cap, q_blocks); break;
    case 3: fa::fa_fwd_f32_kernel<3><<<g, f::kThreads, smem, s>>>(q, k, v, o, lse, Hq, Hkv, N, d, scale, causal, win, cap, q_blocks); break;
    default: fa::fa_fwd_f32_kernel<4><<<g, f::kThreads, smem, s>>>(q, k, v, o, lse, Hq, Hkv, N, d, scale, causal, win, cap, q_blocks); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// split-KV without a caller workspace
// ---------------------------------------------------------------------------------
namespace {

// Scratch of fa_fwd_splitkv_static: a fixed array in this library's device image.  Every
// GPU the library is loaded on holds it until the process exits.  In host code its name
// only stands in for the symbol; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_splitkv_scratch[FA_STATIC_SCRATCH_BYTES];

struct ScratchState {
  fa::OnceOnSuccess once;
  void* ptr = nullptr;
};
ScratchState g_scratch[kMaxDevices];

// Device address of the scratch array on device `dev` (the current device): looked up
// on the first call made with that device current, and again on later calls until a
// lookup succeeds (a failed first lookup does not disable the device for good).
int scratch_address(int dev, void** out) {
  ScratchState& st = g_scratch[dev];
  const int status = st.once.run([&]() -> int {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_splitkv_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    st.ptr = ptr;
    return FA_OK;
  });
  *out = st.ptr;
  return status;
}

}  // namespace

extern "C" {

int fa_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int N, int d, float scale, int causal, int window, float softcap, int num_splits,
                          void* stream) {
  int rc = check_bf16(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (num_splits < 1 || num_splits > FA_MAX_SPLITS) return FA_ERR_BAD_ARG;
  const size_t need = fa_fwd_splitkv_workspace(B, Hq, N, d, num_splits);
  if (need > static_cast<size_t>(FA_STATIC_SCRATCH_BYTES)) return FA_ERR_SCRATCH_LIMIT;
  int dev;
  if ((rc = current_device(&dev)) != FA_OK) return rc;
  void* scratch = nullptr;
  if ((rc = scratch_address(dev, &scratch)) != FA_OK) return rc;
  // Every partial the merge reads is written earlier in the same call (each chunk writes
  // O and LSE for every row, -inf / 0 where it has no keys), so nothing has to be cleared.
  const size_t rows = static_cast<size_t>(B) * Hq * N;
  float* o_part = static_cast<float*>(scratch);
  float* lse_part = o_part + static_cast<size_t>(num_splits) * rows * d;
  return launch_tc(q, k, v, o, lse, B, Hq, Hkv, N, N, d, scale, causal, window, 0, softcap, num_splits, o_part,
                   lse_part, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// status word and the failure-detection self-test
// ---------------------------------------------------------------------------------
namespace {

__global__ void fa_wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar, 1);
    abort_flag = 0;
    fa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the bounded wait must give up by itself
    fa::mbar_wait(&bar, 0, fa::WaitCtl{&abort_flag, limit_ns});
  }
  __syncthreads();
}

}  // namespace

extern "C" {

int fa_check_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int st = 0;
  e = cudaMemcpyFromSymbol(&st, fa::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  if (st != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    return st;
  }
  return FA_OK;
}

int fa_selftest_wait_timeout(unsigned timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return FA_ERR_BAD_ARG;
  int dev, rc;
  if ((rc = current_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_device(dev)) != FA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fa_wait_selftest_kernel<<<1, 32, 0, s>>>(static_cast<unsigned long long>(timeout_us) * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return fa_check_status(stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// stand-alone softmax (online normaliser) and softmax + top-K
// ---------------------------------------------------------------------------------
extern "C" {

int fa_softmax(const float* x, float* y, float* lse, int rows, int V, void* stream) {
  if (rows < 0 || V < 0) return FA_ERR_BAD_SHAPE;
  if (rows == 0) return FA_OK;
  if (V > 0 && (!x || !y)) return FA_ERR_NULL_PTR;  // V == 0: nothing is read, only lse is written
  if (!aligned(x, 16) || !aligned(y, 16) || (lse && !aligned(lse, 4))) return FA_ERR_ALIGN;
  int dev, rc;
  if ((rc = current_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_device(dev)) != FA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1024 threads for long rows; short rows do not need that many
  const int threads = V >= 16384 ? fa::smx::kSoftmaxThreads : 256;
  fa::smx::softmax_online_kernel<<<static_cast<unsigned>(rows), threads, 0, s>>>(x, y, lse, V);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

}  // extern "C"

namespace {

template <int T>
void launch_topk(unsigned g, const float* x, float* probs, int* idx, float* lse, int V, int K, cudaStream_t s) {
  if (K <= 4)
    fa::smx::softmax_topk_kernel<4, T><<<g, T, 0, s>>>(x, probs, idx, lse, V, K);
  else if (K <= 8)
    fa::smx::softmax_topk_kernel<8, T><<<g, T, 0, s>>>(x, probs, idx, lse, V, K);
  else if (K <= 16)
    fa::smx::softmax_topk_kernel<16, T><<<g, T, 0, s>>>(x, probs, idx, lse, V, K);
  else
    fa::smx::softmax_topk_kernel<32, T><<<g, T, 0, s>>>(x, probs, idx, lse, V, K);
}

}  // namespace

extern "C" {

int fa_softmax_topk(const float* x, float* probs, int* idx, float* lse, int rows, int V, int K, void* stream) {
  if (rows < 0 || V < 0) return FA_ERR_BAD_SHAPE;
  if (K < 1 || K > fa::smx::kMaxTopK || (rows > 0 && K > V)) return FA_ERR_BAD_ARG;
  if (rows == 0) return FA_OK;
  if (!x || !probs || !idx) return FA_ERR_NULL_PTR;
  if (!aligned(x, 16) || !aligned(probs, 4) || !aligned(idx, 4) || (lse && !aligned(lse, 4))) return FA_ERR_ALIGN;
  int dev, rc;
  if ((rc = current_device(&dev)) != FA_OK) return rc;
  if ((rc = prepare_device(dev)) != FA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned g = static_cast<unsigned>(rows);
  if (V <= 131072)
    launch_topk<fa::smx::kTopkThreadsShort>(g, x, probs, idx, lse, V, K, s);
  else
    launch_topk<fa::smx::kTopkThreadsLong>(g, x, probs, idx, lse, V, K, s);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

}  // extern "C"
