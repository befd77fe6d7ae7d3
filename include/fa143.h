/*
 * fa143.h -- C ABI of the B200 (sm_100a) exact-attention library libfa143.so.
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(Q K^T * softmax_scale + mask) V
 *
 * ("optimizing-attention-flash", Workflow 1 Step 2: the standard-attention
 * form softmax(q k^T / sqrt(d_k)) v that the fused kernel replaces) tile by
 * tile, so the N x N score matrix never reaches HBM ("Что такое
 * FlashAttention…", section "Основной механизм простыми словами": blocks of
 * Q, K, V are brought from HBM into on-chip memory, attention is computed per
 * block and the output is updated incrementally; the result is exact, without
 * approximation).  The backward pass rebuilds the probabilities from the
 * per-row log-sum-exp saved by the forward ("tiling and recomputation",
 * "optimizing-attention-flash", Quick start).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors use the [batch, seqlen, heads, head_dim] layout of
 *    flash_attn_func ("optimizing-attention-flash", Workflow 2 Step 2).
 *    Each tensor is described by a device pointer plus three strides, in
 *    ELEMENTS, for (batch, seq, head); head_dim is contiguous (stride 1).
 *    Pointers must be 16-byte aligned and the three strides must be
 *    multiples of 8 elements (16 bytes), as the tensor-memory-accelerator
 *    copies require; otherwise FA_ERR_ALIGNMENT.
 *  - dtype is FA_F16 or FA_BF16 for every tensor of one call; fp32 inputs
 *    are not supported (the pages' troubleshooting section: fp16/bf16 only).
 *  - head_dim d is 64 or 128; the forward calls (fa_fwd, fa_fwd_varlen) also
 *    take 256 (head dims up to 256, with the backward limited above 192:
 *    "Что такое FlashAttention…", section on versions and hardware).  The
 *    backward calls return FA_ERR_UNSUPPORTED for d = 256.
 *  - Hq query heads, Hkv key/value heads, Hq % Hkv == 0: query head h reads
 *    kv head h / (Hq / Hkv) (MQA/GQA, Workflow 2 Step 3).
 *  - causal != 0 hides key j from query i when j > i + (Nk - Nq) (masks are
 *    aligned to the bottom-right corner when Nq != Nk).  window_left /
 *    window_right >= 0 keep only keys with
 *        i + (Nk - Nq) - window_left <= j <= i + (Nk - Nq) + window_right
 *    (bounds inclusive); -1 means unbounded on that side (Workflow 2
 *    Step 3's window_size=(left, right), (-1, -1) = no window).  causal and
 *    a window combine as the intersection.
 *  - A query row that sees no key gets O = 0 and LSE = -inf, and zero dQ.
 *  - softmax_scale is passed explicitly and must be finite (the Python
 *    binding maps "None" to 1/sqrt(head_dim), Workflow 2 Step 2).
 *  - LSE is float32, contiguous [batch, Hq, Nq], natural logarithm of
 *    sum_j exp(softmax_scale * q_i . k_j) over the visible keys.
 *  - Everything is asynchronous on `stream` (a cudaStream_t passed as a void
 *    pointer; NULL = legacy default stream).  Errors are returned as status
 *    codes, never thrown; argument errors are detected on the host before any
 *    launch.  The caller owns every buffer; outputs must not alias inputs.
 *  - Device-side waits are bounded: a kernel whose pipeline stalls past the
 *    limit records FA_ERR_DEVICE_TIMEOUT in a device error word and returns;
 *    read it with fa_get_device_error().
 */
#ifndef FA143_H
#define FA143_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FA_F16 = 0, FA_BF16 = 1 } fa_dtype;

enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad window, Hq % Hkv != 0, aliasing */
    FA_ERR_UNSUPPORTED = 2,    /* dtype or head_dim outside what the kernels implement */
    FA_ERR_ALIGNMENT = 3,      /* pointer or stride violates the 16-byte rules above */
    FA_ERR_WORKSPACE = 4,      /* backward workspace missing or too small */
    FA_ERR_CUDA = 5,           /* a CUDA runtime/driver call or a launch failed */
    FA_ERR_DEVICE_TIMEOUT = 6  /* a bounded device-side wait ran out (see fa_get_device_error) */
};

/* Human-readable text of a status code (static storage, never NULL). */
const char* fa_status_string(int status);

/*
 * Forward pass: O and the per-row LSE.
 *   q      [B, Nq, Hq, d]   read-only     strides q_stride = {batch, seq, head}
 *   k, v   [B, Nk, Hkv, d]  read-only     strides k_stride, v_stride
 *   o      [B, Nq, Hq, d]   written       strides o_stride
 *   lse    [B, Hq, Nq] fp32 written       contiguous
 * One kernel launch on `stream`.  Returns FA_OK or an error status.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int Nq, int Nk, int Hq, int Hkv, int d,
           const int64_t q_stride[3], const int64_t k_stride[3],
           const int64_t v_stride[3], const int64_t o_stride[3],
           int dtype, float softmax_scale, int causal, int window_left,
           int window_right, void* stream);

/*
 * Forward pass over a variable-length packed batch (no padding): sequence b
 * owns query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) of q and o and key rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]) of k and v.  The pages name native
 * dynamic sequence lengths without padding inputs to a fixed length
 * ("FlashAttention V3原理与训练推理加速实战指南", section "一、FlashAttention V3
 * 核心原理革新") and variable sequence lengths among the backend features
 * ("Что такое FlashAttention…", section "Версии, оборудование и
 * первоисточники").
 *   q, o       [total_q, Hq, d]    strides {token, head} in elements
 *   k, v       [total_k, Hkv, d]   strides {token, head}
 *   lse        [Hq, total_q] fp32  contiguous, written
 *   cu_seqlens_q, cu_seqlens_k: device int32 [B + 1], non-decreasing,
 *              starting at 0 and ending at total_q / total_k
 *   max_seqlen_q / max_seqlen_k: bounds on the sequence lengths (they size the
 *              grid).  Masks (causal, window) apply within each sequence, with
 *              the same bottom-right alignment as fa_fwd.
 * The offsets are read on the device: lengths are clamped to the max_seqlen
 * bounds and rows to the totals, so malformed offsets give wrong results but
 * never an access outside the tensors.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                  int Hq, int Hkv, int d,
                  const int64_t q_stride[2], const int64_t k_stride[2],
                  const int64_t v_stride[2], const int64_t o_stride[2],
                  int dtype, float softmax_scale, int causal, int window_left,
                  int window_right, void* stream);

/*
 * Forward and backward with dropout on the attention probabilities
 * ("optimizing-attention-flash", the dropout_p argument of flash_attn_func).
 * P_ij is multiplied by (256 / T) M_ij before P V, T = round(256 (1 - p)),
 * where the keep bit M_ij of element (i, j) of (batch b, query head h) is
 * byte (j mod 4) of output word (i mod 4) of Philox4x32-10 (Salmon et al.,
 * SC 2011) at counter (j / 4, i / 4, b Hq + h, offset) with key = seed (low
 * word first), kept iff the byte is below T; LSE is that of the undropped
 * probabilities.  The backward must get the same seed and offset.  The
 * arguments are those of fa_fwd / fa_bwd plus dropout_p in [0, 1), seed
 * and offset; T = 256 (p < 1/512) runs the plain kernels, and p so close to
 * 1 that T = 0 is FA_ERR_INVALID_ARG.  d is 64 or 128.  The _varlen forms take
 * the arguments of fa_fwd_varlen / fa_bwd_varlen plus the same three; there b
 * in the counter is the sequence index and i, j are positions within the
 * sequence.
 */
int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int Nq, int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3],
                   const int64_t k_stride[3], const int64_t v_stride[3],
                   const int64_t o_stride[3], int dtype, float softmax_scale, int causal,
                   int window_left, int window_right, float dropout_p, uint64_t seed,
                   uint32_t offset, void* stream);
int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                   const int64_t q_stride[3], const int64_t k_stride[3],
                   const int64_t v_stride[3], const int64_t o_stride[3],
                   const int64_t do_stride[3], const int64_t dq_stride[3],
                   const int64_t dk_stride[3], const int64_t dv_stride[3], int dtype,
                   float softmax_scale, int causal, int window_left, int window_right,
                   float dropout_p, uint64_t seed, uint32_t offset, void* stream);
int fa_fwd_varlen_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                          int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq,
                          int Hkv, int d, const int64_t q_stride[2], const int64_t k_stride[2],
                          const int64_t v_stride[2], const int64_t o_stride[2], int dtype,
                          float softmax_scale, int causal, int window_left, int window_right,
                          float dropout_p, uint64_t seed, uint32_t offset, void* stream);
int fa_bwd_varlen_dropout(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, const int* cu_seqlens_q,
                          const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k,
                          int total_q, int total_k, int Hq, int Hkv, int d,
                          const int64_t q_stride[2], const int64_t k_stride[2],
                          const int64_t v_stride[2], const int64_t o_stride[2],
                          const int64_t do_stride[2], const int64_t dq_stride[2],
                          const int64_t dk_stride[2], const int64_t dv_stride[2], int dtype,
                          float softmax_scale, int causal, int window_left, int window_right,
                          float dropout_p, uint64_t seed, uint32_t offset, void* stream);

/*
 * Forward on FP8 inputs: q, k, v hold float8_e4m3fn values (one byte each;
 * "optimizing-attention-flash", Workflow 3: inputs cast to float8_e4m3fn and
 * passed to the same attention call), o is bf16, lse fp32 [B, Hq, Nq].
 * The result is exact attention of (descale_q q, descale_k k, descale_v v)
 * with the masks and GQA mapping of fa_fwd.  S = Q K^T is exact in fp32; for
 * P V the probabilities are rounded to e4m3 (held as 2^6 exp(s - m), at most
 * 256), so each term of O carries a relative error of at most 2^-4, or an
 * absolute error of at most 2^-16 where P < 2^-12.  Strides are in elements;
 * q, k and v strides must be multiples of 16 (16 bytes), o strides multiples
 * of 8.  d is 64 or 128.  Returns as fa_fwd.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
               int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3],
               const int64_t k_stride[3], const int64_t v_stride[3], const int64_t o_stride[3],
               float descale_q, float descale_k, float descale_v, float softmax_scale,
               int causal, int window_left, int window_right, void* stream);

/*
 * Decode against a paged KV cache.
 *
 * Sequence b holds cache_seqlens[b] keys; key j of it is row j % page_size of
 * page block_table[b * block_table_stride + j / page_size] of k_cache and
 * v_cache ("optimizing-attention-flash", the list of advanced features, which
 * names a paged KV cache; "FlashAttention V3 原理与…实战指南", section 四 on
 * inference: the KV cache kept in pages of 16 tokens in its vLLM example).
 * The Nq queries of sequence b attend to those keys exactly as in fa_fwd, the
 * masks aligned bottom-right against cache_seqlens[b]: query i is position
 * cache_seqlens[b] - Nq + i (so with Nq = 1 and causal it sees every key).
 *   q, o            [B, Nq, Hq, d]            strides {batch, seq, head}
 *   k_cache, v_cache [num_pages, page_size, Hkv, d] strides {page, token, head}
 *   block_table     device int32, row b at b * block_table_stride, first
 *                   ceil(cache_seqlens[b] / page_size) entries used
 *   cache_seqlens   device int32 [B]
 *   lse             [B, Hq, Nq] fp32, natural log, contiguous, written
 *   page_size       a power of two, 8 or more
 *   num_splits      0 = chosen by the library; k > 0 = the key tiles of each
 *                   (sequence, kv head) are cut into at most k parts
 *   workspace       device memory of fa_fwd_paged_workspace_size() bytes,
 *                   256-byte aligned (may be NULL when that size is 0)
 * (Hq / Hkv) * Nq must be at most 128.  Lengths are clamped to
 * [0, max_pages_per_seq * page_size] on the device, and a page id outside
 * [0, num_pages) reads zeros, so a malformed table gives wrong results but no
 * access outside the caches.  A sequence with no visible key gets O = 0 and
 * LSE = -inf.  Inputs are read only; o and lse must not overlap them.
 * Returns FA_OK once queued, FA_ERR_WORKSPACE if the workspace is missing or
 * too small, FA_ERR_UNSUPPORTED for dtype, head_dim or a query tile over 128
 * rows, FA_ERR_ALIGNMENT or FA_ERR_INVALID_ARG as for fa_fwd.
 */
size_t fa_fwd_paged_workspace_size(int B, int Nq, int Hq, int Hkv, int d, int page_size,
                                   int max_pages_per_seq, int num_splits);
int fa_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* block_table, const int32_t* cache_seqlens, void* o, float* lse,
                 int B, int Nq, int Hq, int Hkv, int d, int page_size, int num_pages,
                 int max_pages_per_seq, int64_t block_table_stride,
                 const int64_t q_stride[3], const int64_t kcache_stride[3],
                 const int64_t vcache_stride[3], const int64_t o_stride[3], int dtype,
                 float softmax_scale, int causal, int window_left, int window_right,
                 int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: an fp32 dQ
 * accumulator [B, Nq, Hq, d] and the fp32 row terms D and LSE*log2(e)
 * [B, Hq, Nq].  The caller allocates it (256-byte aligned); its contents
 * on entry do not matter.
 */
size_t fa_bwd_workspace_size(int B, int Nq, int Hq, int d);

/*
 * Backward pass: dQ, dK, dV of L = sum(dout * O), recomputing the
 * probabilities from the forward's LSE (the textbook gradient of the
 * definition above: dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
 * dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q; the query heads of
 * one GQA group are summed into their shared kv head).
 *   q, o, dout [B, Nq, Hq, d]  read-only   (o and lse from fa_fwd with the
 *   k, v       [B, Nk, Hkv, d] read-only    same arguments)
 *   lse        [B, Hq, Nq] fp32 read-only
 *   dq         [B, Nq, Hq, d]  written
 *   dk, dv     [B, Nk, Hkv, d] written
 *   workspace  >= fa_bwd_workspace_size(B, Nq, Hq, d) bytes, device memory
 * Launches a short sequence of kernels on `stream`.  The partial dQ of the
 * key tiles are added into the fp32 accumulator with bulk tensor reduce-adds
 * in an order that varies from run to run, so dQ's last bits may differ
 * between runs; dK and dV are summed without atomics and are reproducible.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, void* workspace,
           size_t workspace_bytes,
           int B, int Nq, int Nk, int Hq, int Hkv, int d,
           const int64_t q_stride[3], const int64_t k_stride[3],
           const int64_t v_stride[3], const int64_t o_stride[3],
           const int64_t do_stride[3], const int64_t dq_stride[3],
           const int64_t dk_stride[3], const int64_t dv_stride[3],
           int dtype, float softmax_scale, int causal, int window_left,
           int window_right, void* stream);

/*
 * Backward pass for callers that cannot allocate device memory.
 *
 * Some callers of this library cannot call cudaMalloc: for example a plugin
 * running inside a host framework that owns all device memory and gives
 * its operators no workspace, or a latency-critical loop where an
 * allocation's implicit device synchronisation is not allowed.  This entry
 * point takes the same arguments as fa_bwd minus the workspace, and uses a
 * scratch buffer built into the library instead: a static device array of
 * FA_BWD_NOALLOC_SCRATCH_BYTES bytes that every GPU loading the library
 * holds until the process exits.  It allocates nothing itself.
 *
 *  - Sizes whose fa_bwd_workspace_size() exceeds FA_BWD_NOALLOC_SCRATCH_BYTES
 *    are rejected with FA_ERR_WORKSPACE before anything is launched.
 *  - Each call looks up the buffer's device address on the current device
 *    (cudaGetSymbolAddress).  The first call on a device is also where the
 *    runtime loads the library's device code there; make that first call
 *    before any stream capture.
 *  - All calls share the one buffer, which keeps the previous call's
 *    contents (the kernels re-initialise what must start at zero).  Calls
 *    that overlap on the GPU (for example on two streams at once) race on it.
 * Results equal fa_bwd's (dQ up to the order of its fp32 reduce-adds).
 * The pages describe no such variant; it has no counterpart there.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* The size of that built-in scratch buffer in bytes
 * (FA_BWD_NOALLOC_SCRATCH_BYTES as the library was built), so a caller can
 * check fa_bwd_workspace_size() against the library it actually loaded.
 * Host only; never fails. */
size_t fa_bwd_noalloc_scratch_bytes(void);

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv,
                   int B, int Nq, int Nk, int Hq, int Hkv, int d,
                   const int64_t q_stride[3], const int64_t k_stride[3],
                   const int64_t v_stride[3], const int64_t o_stride[3],
                   const int64_t do_stride[3], const int64_t dq_stride[3],
                   const int64_t dk_stride[3], const int64_t dv_stride[3],
                   int dtype, float softmax_scale, int causal, int window_left,
                   int window_right, void* stream);

/*
 * Backward pass over a variable-length packed batch (layouts and offsets as in
 * fa_fwd_varlen; dq like q, dk and dv like k; lse [Hq, total_q] from
 * fa_fwd_varlen).  workspace >= fa_bwd_workspace_size(B, max_seqlen_q, Hq, d)
 * bytes.  Same gradient, accumulation and error behaviour as fa_bwd.
 */
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                  const void* dout, const float* lse, void* dq, void* dk, void* dv,
                  void* workspace, size_t workspace_bytes,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                  int Hq, int Hkv, int d,
                  const int64_t q_stride[2], const int64_t k_stride[2],
                  const int64_t v_stride[2], const int64_t o_stride[2],
                  const int64_t do_stride[2], const int64_t dq_stride[2],
                  const int64_t dk_stride[2], const int64_t dv_stride[2],
                  int dtype, float softmax_scale, int causal, int window_left,
                  int window_right, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device error word of
 * the current device: FA_OK, or FA_ERR_DEVICE_TIMEOUT if a kernel gave up
 * on a bounded wait since the last call (FA_ERR_CUDA if the query failed).
 */
int fa_get_device_error(void* stream);

/*
 * Optional instrumentation.  When ev_start and ev_stop are cudaEvent_t
 * handles (passed as void pointers), every later fa_bwd call records
 * ev_start on its stream right before it launches its main kernel and
 * ev_stop right after, so the caller can time that kernel alone with
 * cudaEventElapsedTime.  NULL, NULL turns it off.  The caller owns the
 * events; the setting is process-wide.  Returns FA_OK.
 */
int fa_set_bwd_main_events(void* ev_start, void* ev_stop);

/*
 * Self-test of the bounded device-side waits.  Launches one small kernel on
 * `stream` whose thread waits, through the same bounded wait the attention
 * kernels use, on a shared-memory barrier that nothing ever completes.  After
 * limit_ns the wait gives up, records FA_ERR_DEVICE_TIMEOUT in the device
 * error word and the kernel returns; no copy or tensor-core operation is in
 * flight, so the context stays usable.  Read the outcome with
 * fa_get_device_error().  Returns FA_OK once launched, FA_ERR_INVALID_ARG if
 * limit_ns is 0 or above 10 s.
 */
int fa_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * Self-test of the FMA-pipe 2^x that the softmax uses for part of its
 * exponentials (a degree-3 minimax polynomial for 2^f on [-1/2, 1/2] times
 * 2^n built in the exponent bits; x is clamped at -127, where the result is
 * +0).  Writes y[i] = that 2^x[i] for i < n (x, y: device fp32, 4-byte
 * aligned); bf16 != 0 selects the instantiation the bf16 kernels use.  One
 * launch on `stream`.  Returns FA_ERR_INVALID_ARG for null pointers or n < 1,
 * FA_ERR_ALIGNMENT for misaligned pointers.  The pages have no counterpart:
 * it exists so the approximation can be checked against the exact function.
 */
int fa_selftest_exp2(const float* x, float* y, int n, int bf16, void* stream);

/*
 * Sets the per-wait limit of device-side waits, in nanoseconds (default
 * 2e9).  Returns the previous value.  For tests of the timeout path only.
 */
uint64_t fa_set_wait_limit_ns(uint64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* FA143_H */
