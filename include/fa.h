/*
 * fa.h -- C ABI of the B200 (sm_100a) FlashAttention forward library (libfa_sm100.so).
 *
 * What is computed
 * ----------------
 * Exact scaled dot-product attention, one tile of keys at a time, with the online
 * softmax: per query row a running maximum m and sum l are kept, and the output
 * accumulator is rescaled by exp(m_old - m_new) whenever the maximum grows, so the
 * N x N score matrix never reaches device memory.  Sources:
 *   - "Module 16: Efficient and Long Attention" (transformers-and-math), section 16.2,
 *     the online softmax and the two-block merge identities; "the result is exactly
 *     standard attention, up to rounding";
 *   - "Online Softmax Without the Attention Matrix" (notebook): the tile recurrence
 *     new max -> correction exp(old - new) -> rescaled sums;
 *   - oxios flash_attention.rs, FlashAttention::attention: queries / keys / values ->
 *     output, scale 1/(temperature * sqrt(d)), the -inf guard on the first rescale.
 *
 * For every batch b, query head hq and query row i (0 <= i < N), with the key/value
 * head kv = hq / (Hq / Hkv) (contiguous groups for grouped-query attention):
 *   s_j   = scale * <q[b,hq,i,:], k[b,kv,j,:]>                       0 <= j < N
 *   s_j   = softcap * tanh(s_j / softcap)        if softcap > 0     (Module 16, 16.5)
 *   s_j   = -inf   if causal and j > i                              (Module 16, 16.2)
 *   s_j   = -inf   if window > 0 and i - j >= window                (Module 16, 16.3:
 *                                                                    the W most recent
 *                                                                    tokens, self included)
 *   o[b,hq,i,:] = sum_j softmax(s)_j * v[b,kv,j,:]
 *   lse[b,hq,i] = ln sum_j exp(s_j)        (natural log of the final, masked scores)
 *
 * Layout and ownership
 * --------------------
 *   q, o : [B, Hq,  N, d] row-major, contiguous;  k, v : [B, Hkv, N, d];  lse : [B, Hq, N].
 *   All pointers are DEVICE pointers owned by the caller.  q, k, v and o must be 16-byte
 *   aligned, lse 4-byte aligned.  The library allocates no device memory, keeps no
 *   per-call state and does not synchronise: work is queued on `stream` (a
 *   cudaStream_t; NULL is the legacy default stream) and the outputs are valid once
 *   that stream has been synchronised.  Calls are asynchronous, so launch errors that
 *   only show later (and device-side wait timeouts) are reported by fa_check_status().
 *
 * Errors
 * ------
 * Every entry point returns FA_OK (0) or one of the negative codes below and writes
 * nothing when it rejects its arguments.  B == 0 or N == 0 (or Hq == 0) is a valid
 * empty problem: it returns FA_OK and touches no memory (oxios returns an empty result
 * for empty input).  lse == NULL skips the log-sum-exp output.
 */
#ifndef FA_SM100_H_
#define FA_SM100_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA_OK 0
#define FA_ERR_NULL_PTR (-1)    /* q, k, v or o is NULL (and the problem is not empty)   */
#define FA_ERR_BAD_SHAPE (-2)   /* a size < 0, Hkv == 0 or Hq % Hkv != 0, size overflow  */
#define FA_ERR_UNSUPPORTED (-3) /* head dim / mask combination this path does not cover,
                                   or the current device is not sm_100                  */
#define FA_ERR_ALIGN (-4)       /* a pointer breaks the alignment rule above             */
#define FA_ERR_BAD_ARG (-5)     /* scale not finite or <= 0, softcap not finite, n_sink < 0,
                                   num_splits out of range                               */
#define FA_ERR_CUDA (-6)        /* a CUDA runtime/driver call failed: fa_last_cuda_error */
#define FA_ERR_TIMEOUT (-7)     /* a device-side wait exceeded its limit (see below)     */
#define FA_ERR_WORKSPACE (-8)   /* split-KV workspace NULL, not 16-byte aligned or too small */

#define FA_ERR_SCRATCH_LIMIT (-9) /* fa_fwd_splitkv_static: problem too large for the fixed
                                     scratch array (see FA_STATIC_SCRATCH_BYTES)           */

#define FA_MAX_SPLITS 64        /* largest num_splits accepted by fa_fwd_splitkv          */
#define FA_STATIC_SCRATCH_BYTES (32u << 20) /* scratch array of fa_fwd_splitkv_static     */

/*
 * fa_fwd -- bf16 attention forward on the tensor cores (tcgen05 + TMA + TMEM).
 *   q, k, v, o : __nv_bfloat16 device arrays (layout above); lse : float or NULL.
 *   B, Hq, Hkv, N : batch, query heads, key/value heads, sequence length (queries and
 *                   keys share N: self-attention).
 *   d        : head dimension, 64 or 128.
 *   scale    : multiplier of q.k (e.g. 1/sqrt(d); a softmax temperature T folds in as
 *              1/(T sqrt(d))), finite and > 0.
 *   causal   : non-zero masks keys j > i.
 *   window   : > 0 keeps only keys with i - j < window (requires causal); <= 0 is off.
 *   softcap  : > 0 applies softcap * tanh(s / softcap) after the scale; <= 0 is off.
 *   stream   : cudaStream_t (NULL = legacy default stream).
 * Precision: bf16 operands, fp32 accumulation of Q.K^T and P.V, probabilities P
 * rounded to bf16 (round-to-nearest-even) for the P.V product, running sum l in fp32,
 * output rounded to bf16 (RNE), lse in fp32.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
           int N, int d, float scale, int causal, int window, float softcap, void* stream);

/*
 * fa_fwd_splitkv -- the same operation as fa_fwd with the keys of every query row cut
 * into num_splits contiguous chunks processed as separate work items (more parallelism
 * for short sequences and few heads), then merged.  Chunk s yields a partial output O_s
 * (normalised within the chunk) and LSE_s; the merge applies the two-block merge
 * identities of "Module 16: Efficient and Long Attention", section 16.2, repeated over
 * the chunks: with m = max_s LSE_s, weights w_s = exp(LSE_s - m), O = sum w_s O_s / sum w_s,
 * LSE = m + ln sum w_s.  Same result as fa_fwd up to rounding.
 *   num_splits : 1 .. FA_MAX_SPLITS.
 *   workspace  : caller-owned DEVICE buffer of at least
 *                fa_fwd_splitkv_workspace(B, Hq, N, d, num_splits) bytes, 16-byte aligned:
 *                fp32 partial outputs [num_splits][B*Hq][N][d] followed by fp32 partial
 *                LSE [num_splits][B*Hq][N].  Overwritten; no state kept between calls.
 *                Calls that share one workspace must not overlap on the GPU.
 *   Other arguments as fa_fwd.  FA_ERR_WORKSPACE if the workspace is missing, misaligned
 *   or too small; FA_ERR_BAD_ARG for num_splits outside 1 .. FA_MAX_SPLITS.
 */
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                   int N, int d, float scale, int causal, int window, float softcap, int num_splits,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_fwd_ext -- the general form: queries and keys of different lengths (cross-attention,
 * decoding against a key/value cache), attention sinks, and optional split-KV.
 *   q, o : [B, Hq, Nq, d];  k, v : [B, Hkv, Nk, d];  lse : [B, Hq, Nq].
 *   Nq, Nk : query rows and key rows per head (>= 0).  Query row i sits at position
 *            p = i + (Nk - Nq) of the key sequence: the queries are the last Nq
 *            positions (with Nq == Nk this is self-attention, p = i).  The causal and
 *            window masks use p: keys j > p are masked (causal), and keys with
 *            p - j >= window (window > 0).  A row with no valid key (Nq > Nk, causal,
 *            rows i < Nq - Nk; or Nk == 0) gets O = 0 and LSE = -inf.
 *            Cross-attention: oxios flash_attention.rs, FlashAttention::cross_attention
 *            (queries from one sequence, keys and values from another).
 *   n_sink : >= 0.  With a window, keys 0 .. n_sink-1 (the attention sinks) are exempt
 *            from the window; they stay under the causal mask.  "Module 16: Efficient and
 *            Long Attention", section 16.6, keeps the first 4 tokens beside the sliding
 *            window.  Without a window every key is kept anyway and n_sink has no effect.
 *   num_splits : 0 runs the plain forward (workspace may be NULL); 1 .. FA_MAX_SPLITS runs
 *            split-KV as fa_fwd_splitkv with a workspace of at least
 *            fa_fwd_splitkv_workspace(B, Hq, Nq, d, num_splits) bytes.
 *   Other arguments, precision and errors as fa_fwd and fa_fwd_splitkv; k and v may be
 *   NULL when Nk == 0.  FA_ERR_BAD_ARG for n_sink < 0 or num_splits out of range.
 */
int fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
               int Nk, int d, float scale, int causal, int window, int n_sink, float softcap, int num_splits,
               void* workspace, size_t workspace_bytes, void* stream);

/* fa_fwd_splitkv_workspace -- bytes of workspace fa_fwd_splitkv needs (0 for an empty or
 * invalid problem): num_splits * B * Hq * N * (d + 1) * 4. */
size_t fa_fwd_splitkv_workspace(int B, int Hq, int N, int d, int num_splits);

/*
 * fa_fwd_splitkv_static -- fa_fwd_splitkv for callers that cannot allocate device memory.
 * The reference pages have no counterpart to this entry point; it is a deployment
 * convenience of this library.
 *
 * Some callers have no way to obtain a workspace: a host program that runs under a fixed
 * device-memory plan where nothing may call cudaMalloc after start-up (cudaMalloc and
 * cudaFree can also synchronise the device, which latency-bound callers avoid), or a
 * plug-in inside a framework that owns all device memory through its own allocator and
 * offers no scratch to plug-ins.  This entry point takes no workspace and allocates
 * nothing (no cudaMalloc, no cudaFree, no allocating library call): its scratch is a
 * fixed array of FA_STATIC_SCRATCH_BYTES (32 MiB) compiled into the library, which every
 * GPU the library is loaded on holds until the process exits.
 *   Arguments: as fa_fwd_splitkv without workspace / workspace_bytes.  The caller still
 *   owns q, k, v, o and lse.
 *   Limit: problems whose fa_fwd_splitkv_workspace(B, Hq, N, d, num_splits) exceeds
 *   FA_STATIC_SCRATCH_BYTES are rejected with FA_ERR_SCRATCH_LIMIT (nothing is written).
 *   Set-up: the first call on a device, with that device current, looks up the array's
 *   device address (cudaGetSymbolAddress) once; make that first call before any stream
 *   capture is begun on the device.
 *   Sharing: every call on a device uses the same array, and the array keeps the last
 *   call's partial results.  Nothing in it has to start at zero (each call writes every
 *   partial it reads), but calls that overlap on the GPU (on different streams, or from
 *   different host threads) race on the array: serialise them.
 */
int fa_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                          int Hkv, int N, int d, float scale, int causal, int window, float softcap,
                          int num_splits, void* stream);

/*
 * fa_fwd_f32 -- the same operation in fp32 on the CUDA cores (FFMA, no TF32), for
 * small head dimensions: 1 <= d <= 128.  Same arguments as fa_fwd with float q, k, v,
 * o.  Pointers need 4-byte alignment.  Scores, the online-softmax state and the
 * accumulator are fp32; exponentials use the accurate expf.
 * Source of the workload it was built for: nx_flashattn_scale.nx (n = 64, d = 32,
 * f32 streaming attention checked against a direct softmax).
 */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int Hq,
               int Hkv, int N, int d, float scale, int causal, int window, float softcap, void* stream);

/*
 * fa_softmax -- stand-alone softmax of every row with the online normaliser.
 * Source: "Online normalizer calculation for softmax" (Milakov and Gimelshein): the
 * classical softmax, computed with fewer memory accesses by keeping the running maximum
 * and the normaliser together in one pass (the normaliser is rescaled by
 * exp(m_old - m_new) when the maximum grows); a second pass writes the outputs.
 *   x, y : float device arrays [rows, V], row-major, 16-byte aligned, not overlapping.
 *          y[r, i] = exp(x[r, i] - m_r) / d_r, m_r = max_i x[r, i],
 *          d_r = sum_i exp(x[r, i] - m_r).
 *   lse  : float [rows] or NULL: m_r + ln d_r (-inf for V == 0).
 *   rows, V >= 0.  A row whose inputs are all -inf is undefined (0 / 0).
 * Precision: fp32 in and out; exponentials as exp2 of x log2(e) (approximate exp2,
 * relative error about 2^-22), normaliser summed in fp32.
 * Errors: FA_ERR_BAD_SHAPE (rows or V < 0), FA_ERR_NULL_PTR, FA_ERR_ALIGN, FA_ERR_CUDA.
 */
int fa_softmax(const float* x, float* y, float* lse, int rows, int V, void* stream);

/*
 * fa_softmax_topk -- softmax fused with top-K: one read of each row gives the row's
 * maximum and normaliser and its K largest inputs (the fused Softmax+TopK of "Online
 * normalizer calculation for softmax").  Nothing of size V is written.
 *   x     : float [rows, V], 16-byte aligned.
 *   probs : float [rows, K]: softmax probabilities exp(x_k - m) / d of the K largest
 *           inputs, largest first.
 *   idx   : int [rows, K]: their column indices.  Equal inputs are ordered by lower
 *           index first (the page does not say; this is the library's rule).
 *   lse   : float [rows] or NULL, as fa_softmax.
 *   1 <= K <= 32 and K <= V (FA_ERR_BAD_ARG otherwise).  Other errors as fa_softmax.
 */
int fa_softmax_topk(const float* x, float* probs, int* idx, float* lse, int rows, int V, int K, void* stream);

/*
 * fa_check_status -- synchronise `stream`, then report (and clear) the device status
 * word that kernels of this library set when one of their bounded waits ran out
 * (FA_ERR_TIMEOUT) on the current device, or a pending CUDA error (FA_ERR_CUDA).
 * Returns FA_OK when neither happened.
 * The status word is ONE word per device, shared by every stream and every caller of
 * the library on that device: a timeout raised by a kernel on another stream is
 * reported (and cleared) by whichever fa_check_status call reads the word first, and a
 * kernel on another stream that is still running when this call returns may set it
 * afterwards.  Callers that issue work from several streams and need to know which of
 * them timed out should synchronise all of them (or the device) before checking.
 */
int fa_check_status(void* stream);

/*
 * fa_selftest_wait_timeout -- failure-detection self-test: launches one tiny kernel
 * whose single wait (the same bounded mbarrier wait the attention kernels use) is on a
 * barrier that nothing ever arrives at, with a limit of `timeout_us` microseconds
 * (1..1000000).  The wait gives up, the kernel records FA_ERR_TIMEOUT and exits.
 * Synchronises `stream` and returns what fa_check_status() reports (FA_ERR_TIMEOUT
 * when the mechanism works); the device stays usable.
 */
int fa_selftest_wait_timeout(unsigned timeout_us, void* stream);

/* fa_strerror -- static description of an FA_* code. */
const char* fa_strerror(int code);

/* fa_last_cuda_error -- the cudaError_t of the last failed CUDA call on this thread. */
int fa_last_cuda_error(void);

/* fa_version -- library ABI version (major * 100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H_ */
