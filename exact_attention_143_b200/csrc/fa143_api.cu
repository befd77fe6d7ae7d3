// fa143_api.cu -- the C ABI of libfa143.so (declared in include/fa143.h):
// argument validation, tensor-map (TMA descriptor) construction and kernel
// launches.  No device memory is allocated here beyond the process-lifetime
// error word below; the caller owns every tensor and the workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "fa143.h"
#include "fa_bwd.cuh"
#include "fa_bwd_aux.cuh"
#include "fa_bwd256.cuh"
#include "fa_decode.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd256.cuh"
#include "fa_fwd_fp8.cuh"

namespace {

int sm_count();  // streaming multiprocessors of the current device (cached per device)

__device__ unsigned int g_device_error = 0u;

// read by every launch, set by fa_set_wait_limit_ns from any host thread
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

// One-time set-up per device (per kernel instantiation): kernel attributes
// such as the dynamic shared-memory opt-in apply to the current device only,
// so a process that drives several devices needs them once on each.
constexpr int kMaxDevices = 64;
struct DeviceOnce {
  std::atomic<uint8_t> done[kMaxDevices];  // static storage: starts at zero
};
template <typename F>
int once_per_device(DeviceOnce& once, F&& setup) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (once.done[dev].load(std::memory_order_acquire)) return FA_OK;
  const int rc = setup();  // idempotent: two threads may both run it
  if (rc == FA_OK) once.done[dev].store(1, std::memory_order_release);
  return rc;
}
cudaEvent_t g_bwd_ev_start = nullptr, g_bwd_ev_stop = nullptr;

// ------------------------------------------------------------------ driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// ------------------------------------------------------------------ validation helpers
struct TensorDesc {
  const void* ptr;
  int64_t sb, ss, sh;  // element strides: batch, seq, head
  int B, N, H, d;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_tensor(const TensorDesc& t) {
  if (t.ptr == nullptr) return FA_ERR_INVALID_ARG;
  if (t.sb < 0 || t.ss < 0 || t.sh < 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return FA_ERR_ALIGNMENT;
  // a stride only matters when its dimension has more than one index
  if ((t.B > 1 && t.sb % 8) || (t.N > 1 && t.ss % 8) || (t.H > 1 && t.sh % 8))
    return FA_ERR_ALIGNMENT;
  return FA_OK;
}

// byte interval [lo, hi) touched by a tensor
void tensor_extent(const TensorDesc& t, uintptr_t& lo, uintptr_t& hi) {
  const int64_t last = int64_t(t.B - 1) * t.sb + int64_t(t.N - 1) * t.ss +
                       int64_t(t.H - 1) * t.sh + t.d;
  lo = reinterpret_cast<uintptr_t>(t.ptr);
  hi = lo + uintptr_t(last) * 2u;
}

bool overlaps(uintptr_t a0, uintptr_t a1, uintptr_t b0, uintptr_t b1) {
  return a0 < b1 && b0 < a1;
}

bool overlaps_t(const TensorDesc& a, const TensorDesc& b) {
  uintptr_t a0, a1, b0, b1;
  tensor_extent(a, a0, a1);
  tensor_extent(b, b0, b1);
  return overlaps(a0, a1, b0, b1);
}

bool overlaps_span(const TensorDesc& a, const void* p, size_t bytes) {
  uintptr_t a0, a1;
  tensor_extent(a, a0, a1);
  const uintptr_t b0 = reinterpret_cast<uintptr_t>(p);
  return overlaps(a0, a1, b0, b0 + bytes);
}

int check_common(int B, int Nq, int Nk, int Hq, int Hkv, int d, int dtype, float scale,
                 int window_left, int window_right, bool allow_d256 = false) {
  if (B < 1 || Nq < 1 || Nk < 1 || Hq < 1 || Hkv < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (window_left < -1 || window_right < -1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128 && !(allow_d256 && d == 256)) return FA_ERR_UNSUPPORTED;
  if (d == 256 && (Nq + 127) / 128 > 65535) return FA_ERR_INVALID_ARG;
  // grid and TMA coordinate limits
  if (Nq > (1 << 24) || Nk > (1 << 24) || int64_t(B) * Hq > (int64_t(1) << 30) ||
      (Nq + 255) / 256 > 65535 || (Nk + 127) / 128 > 65535)
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// 4-D tensor map over [B, N, H, d] (innermost first: d, N, H, B), box of
// 64 columns x 128 rows, 128-byte swizzle, zero fill outside the tensor.
int make_map(CUtensorMap* map, const TensorDesc& t, int dtype, int box_rows = 128) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  // strides of size-1 dimensions are never used; give them a legal value
  const int64_t ss = t.N > 1 ? t.ss : 8;
  const int64_t sh = t.H > 1 ? t.sh : 8;
  const int64_t sb = t.B > 1 ? t.sb : 8;
  cuuint64_t dims[4] = {cuuint64_t(t.d), cuuint64_t(t.N), cuuint64_t(t.H), cuuint64_t(t.B)};
  cuuint64_t strides[3] = {cuuint64_t(ss) * 2, cuuint64_t(sh) * 2, cuuint64_t(sb) * 2};
  cuuint32_t box[4] = {64, cuuint32_t(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map,
                   dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   4, const_cast<void*>(t.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_ALIGNMENT;
}

unsigned int* device_error_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

// |scale| * log2(e); zero is replaced by a value too small to change any fp32
// product of a finite score, so masked (-inf) scores still map to -inf.
float scale_log2_of(float scale) {
  const float a = std::fabs(scale) * 1.4426950408889634f;
  return a > 0.f ? a : 1e-30f;
}

// A wait on a barrier nothing completes: exercises the timeout path of the
// bounded waits (error word set, kernel returns) without any copy in flight.
__global__ void fa_selftest_wait_kernel(unsigned int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    fa::mbar_init(fa::smem_u32(&bar), 1);
    abort_flag = 0;
    fa::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    fa::WaitCtx wc{&abort_flag, err, limit_ns};
    fa::mbar_wait(fa::smem_u32(&bar), 0, wc);
  }
}

// 2^x by the FMA-pipe polynomial the softmax uses for part of its column
// pairs, one pair per thread, so it can be tested against the exact function.
__global__ void fa_selftest_exp2_kernel(const float* x, float* y, int n, int bf16) {
  const int i = 2 * int(blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 r = bf16 ? fa::exp2_fma_pair<true>(in) : fa::exp2_fma_pair<false>(in);
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

template <int D, bool BF16, bool DROP = false>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const fa::FwdParams& prm, cudaStream_t st) {
  // work tiles: (batch, query head or head pair) x query blocks
  using Cfg = fa::FwdCfg<D>;
  auto kern = fa::fa_fwd_kernel<D, BF16, DROP>;
  static DeviceOnce once;  // per instantiation: attributes set on each device used
  {
    const int rc_once = once_per_device(once, [&]() -> int {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes) != cudaSuccess)
        return int(FA_ERR_CUDA);
      // the kernel moves registers between warpgroups (setmaxnreg); that is only
      // sound when it is launched with exactly the planned count per thread
      cudaFuncAttributes fattr{};
      if (cudaFuncGetAttributes(&fattr, kern) != cudaSuccess || fattr.numRegs != Cfg::kRegsLaunch)
        return int(FA_ERR_CUDA);
      return int(FA_OK);
    });
    if (rc_once) return rc_once;
  }
  dim3 grid(unsigned(prm.B * (prm.Hq >> prm.pair)), unsigned(prm.n_mblocks));
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool BF16>
int launch_fwd256(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const fa::FwdParams& prm, cudaStream_t st) {
  using Cfg = fa::Fwd256Cfg;
  auto kern = fa::fa_fwd256_kernel<BF16>;
  static DeviceOnce once;  // per instantiation: attributes set on each device used
  {
    const int rc_once = once_per_device(once, [&]() -> int {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes) != cudaSuccess)
        return int(FA_ERR_CUDA);
      return int(FA_OK);
    });
    if (rc_once) return rc_once;
  }
  dim3 grid(unsigned(prm.B * prm.Hq), unsigned(prm.n_mblocks));
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// 3-D fp32 tensor map over the dQ accumulator [B*Hq, Nq, d] for the bulk
// reduce-adds: box of 32 columns (128 B, 128-byte swizzle) x rows_per_box rows.
int make_dq_acc_map(CUtensorMap* map, float* dq_acc, int B, int Nq, int Hq, int d,
                    int rows_per_box, bool swizzle128 = true) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(Nq), cuuint64_t(B) * cuuint64_t(Hq)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 4, cuuint64_t(Nq) * cuuint64_t(d) * 4};
  cuuint32_t box[3] = {32, cuuint32_t(rows_per_box), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dq_acc, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16, bool DROP = false>
int launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mdo, const fa::BwdParams& prm, cudaStream_t st) {
  CUtensorMap mdq;
  int rc = make_dq_acc_map(&mdq, prm.dq_acc, prm.B, prm.Nq, prm.Hq, D, 128);
  if (rc) return rc;
  using Cfg = fa::BwdCfg<D>;
  auto kern = fa::fa_bwd_main_kernel<D, BF16, DROP>;
  static DeviceOnce once;  // per instantiation: attributes set on each device used
  {
    const int rc_once = once_per_device(once, [&]() -> int {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes) != cudaSuccess)
        return int(FA_ERR_CUDA);
      // the kernel moves registers between warpgroups (setmaxnreg); that is only
      // sound when it is launched with exactly the planned count per thread
      cudaFuncAttributes fattr{};
      if (cudaFuncGetAttributes(&fattr, kern) != cudaSuccess || fattr.numRegs != Cfg::kRegsLaunch)
        return int(FA_ERR_CUDA);
      return int(FA_OK);
    });
    if (rc_once) return rc_once;
  }
  dim3 grid(unsigned(prm.B * prm.Hkv), unsigned(prm.n_ntiles));
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool BF16>
int launch_bwd256(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const CUtensorMap& mdo, const fa::BwdParams& prm, cudaStream_t st) {
  using Cfg = fa::Bwd256Cfg;
  CUtensorMap mdq;  // fp32 dQ accumulator, blocks of 32 columns x 32 rows, unswizzled
  int rc = make_dq_acc_map(&mdq, prm.dq_acc, prm.B, prm.Nq, prm.Hq, Cfg::D, Cfg::kQ, false);
  if (rc) return rc;
  auto kern = fa::fa_bwd256_main_kernel<BF16>;
  static DeviceOnce once;  // per instantiation: attributes set on each device used
  {
    const int rc_once = once_per_device(once, [&]() -> int {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes) != cudaSuccess)
        return int(FA_ERR_CUDA);
      return int(FA_OK);
    });
    if (rc_once) return rc_once;
  }
  dim3 grid(unsigned(prm.B * prm.Hkv), unsigned(prm.n_ntiles), 2u);  // z: half of d
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported dtype or head_dim";
    case FA_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "backward workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case FA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int fa_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return FA_ERR_INVALID_ARG;
  unsigned int* err = device_error_ptr();
  if (!err) return FA_ERR_CUDA;
  fa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_selftest_exp2(const float* x, float* y, int n, int bf16, void* stream) {
  if (x == nullptr || y == nullptr || n < 1) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u))
    return FA_ERR_ALIGNMENT;
  const int pairs = (n + 1) / 2;
  fa_selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y, n, bf16);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_set_bwd_main_events(void* ev_start, void* ev_stop) {
  g_bwd_ev_start = static_cast<cudaEvent_t>(ev_start);
  g_bwd_ev_stop = static_cast<cudaEvent_t>(ev_stop);
  return FA_OK;
}

uint64_t fa_set_wait_limit_ns(uint64_t limit_ns) {
  return g_wait_limit_ns.exchange(limit_ns, std::memory_order_relaxed);
}

}  // extern "C"

namespace {

// Shared body of fa_fwd and fa_fwd_varlen.  Dense: tq/tk/tv/to span [B, N, H, d],
// cu_q == cu_k == nullptr.  Varlen: the descriptors span [1, total, H, d] and
// B counts the sequences; Nq / Nk are the longest sequence lengths.
int fwd_impl(const TensorDesc& tq, const TensorDesc& tk, const TensorDesc& tv,
             const TensorDesc& to, float* lse, size_t lse_bytes, int B, int Nq, int Nk, int Hq,
             int Hkv, int d, const int* cu_q, const int* cu_k, int total_q, int total_k,
             int dtype, float softmax_scale, int causal, int window_left, int window_right,
             void* stream, const fa::DropoutParams* drop = nullptr) {
  int rc;
  for (const TensorDesc* t : {&tq, &tk, &tv, &to})
    if ((rc = check_tensor(*t))) return rc;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_ALIGNMENT;
  if (overlaps_t(to, tq) || overlaps_t(to, tk) || overlaps_t(to, tv) ||
      overlaps_span(tq, lse, lse_bytes) || overlaps_span(tk, lse, lse_bytes) ||
      overlaps_span(tv, lse, lse_bytes) || overlaps_span(to, lse, lse_bytes))
    return FA_ERR_INVALID_ARG;

  // d = 256 streams K and V in tiles of 64 keys
  const int kv_rows = d == 256 ? 64 : 128;
  CUtensorMap mq, mk, mv;
  if ((rc = make_map(&mq, tq, dtype)) || (rc = make_map(&mk, tk, dtype, kv_rows)) ||
      (rc = make_map(&mv, tv, dtype, kv_rows)))
    return rc;
  fa::FwdParams prm{};
  prm.o = const_cast<void*>(to.ptr);
  prm.lse = lse;
  prm.o_sb = to.sb;
  prm.o_ss = to.ss;
  prm.o_sh = to.sh;
  prm.B = B;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  // 256 query rows per CTA; a causal problem that would not fill the SMs runs
  // one 128-row tile per CTA, which halves the longest CTA (the last query
  // block sees the most keys).  The d = 256 kernel always takes 128 rows.
  prm.mrows = 256;
  if (d == 256 || (causal && int64_t(B) * Hq * ((Nq + 255) / 256) < sm_count())) prm.mrows = 128;
  // Short key ranges (a 128-row tile sees at most 4 K tiles): a work tile
  // takes two query heads of one GQA group over the same 128 rows, so both
  // query tiles walk the same few K tiles side by side and share each load.
  {
    const int right = causal ? 0 : window_right;
    if (d != 256 && (Hq / Hkv) % 2 == 0 && window_left >= 0 && right >= 0 &&
        int64_t(window_left) + right <= 384) {
      prm.pair = 1;
      prm.mrows = 128;
    }
  }
  prm.n_mblocks = (Nq + prm.mrows - 1) / prm.mrows;
  prm.scale_log2 = scale_log2_of(softmax_scale);
  prm.qk_negate = softmax_scale < 0.f ? 1u : 0u;
  prm.causal = causal ? 1 : 0;
  prm.wl = window_left;
  prm.wr = window_right;
  prm.err = device_error_ptr();
  prm.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  prm.cu_q = cu_q;
  prm.cu_k = cu_k;
  prm.total_q = total_q;
  prm.total_k = total_k;
  if (drop) prm.drop = *drop;
  if (!prm.err) return FA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (drop) {
    if (d == 256) return FA_ERR_UNSUPPORTED;
    if (dtype == FA_BF16)
      return d == 64 ? launch_fwd<64, true, true>(mq, mk, mv, prm, st)
                     : launch_fwd<128, true, true>(mq, mk, mv, prm, st);
    return d == 64 ? launch_fwd<64, false, true>(mq, mk, mv, prm, st)
                   : launch_fwd<128, false, true>(mq, mk, mv, prm, st);
  }
  if (d == 256)
    return dtype == FA_BF16 ? launch_fwd256<true>(mq, mk, mv, prm, st)
                            : launch_fwd256<false>(mq, mk, mv, prm, st);
  if (dtype == FA_BF16)
    return d == 64 ? launch_fwd<64, true>(mq, mk, mv, prm, st)
                   : launch_fwd<128, true>(mq, mk, mv, prm, st);
  return d == 64 ? launch_fwd<64, false>(mq, mk, mv, prm, st)
                 : launch_fwd<128, false>(mq, mk, mv, prm, st);
}

int check_varlen(const int* cu_q, const int* cu_k, int B, int max_q, int max_k, int total_q,
                 int total_k) {
  if (!cu_q || !cu_k) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u))
    return FA_ERR_ALIGNMENT;
  if (B < 1 || max_q < 1 || max_k < 1 || total_q < 1 || total_k < 1) return FA_ERR_INVALID_ARG;
  if (max_q > total_q || max_k > total_k) return FA_ERR_INVALID_ARG;
  return FA_OK;
}


// The dense and packed-batch forward entry points, with or without dropout
// (dp = nullptr: none; head_dim 256 only without).
int fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
              int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3],
              const int64_t k_stride[3], const int64_t v_stride[3], const int64_t o_stride[3],
              int dtype, float softmax_scale, int causal, int window_left, int window_right,
              void* stream, const fa::DropoutParams* dp) {
  int rc = check_common(B, Nq, Nk, Hq, Hkv, d, dtype, softmax_scale, window_left, window_right,
                        dp == nullptr);
  if (rc) return rc;
  if (!q_stride || !k_stride || !v_stride || !o_stride || !lse) return FA_ERR_INVALID_ARG;
  const TensorDesc tq{q, q_stride[0], q_stride[1], q_stride[2], B, Nq, Hq, d};
  const TensorDesc tk{k, k_stride[0], k_stride[1], k_stride[2], B, Nk, Hkv, d};
  const TensorDesc tv{v, v_stride[0], v_stride[1], v_stride[2], B, Nk, Hkv, d};
  const TensorDesc to{o, o_stride[0], o_stride[1], o_stride[2], B, Nq, Hq, d};
  return fwd_impl(tq, tk, tv, to, lse, size_t(B) * Hq * Nq * sizeof(float), B, Nq, Nk, Hq, Hkv,
                  d, nullptr, nullptr, 0, 0, dtype, softmax_scale, causal, window_left,
                  window_right, stream, dp);
}

int fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
               const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
               int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d,
               const int64_t q_stride[2], const int64_t k_stride[2], const int64_t v_stride[2],
               const int64_t o_stride[2], int dtype, float softmax_scale, int causal,
               int window_left, int window_right, void* stream, const fa::DropoutParams* dp) {
  int rc = check_common(B, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, dtype, softmax_scale,
                        window_left, window_right, dp == nullptr);
  if (rc) return rc;
  if ((rc = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q,
                         total_k)))
    return rc;
  if (total_q > (1 << 28) || total_k > (1 << 28)) return FA_ERR_INVALID_ARG;
  if (!q_stride || !k_stride || !v_stride || !o_stride || !lse) return FA_ERR_INVALID_ARG;
  const TensorDesc tq{q, 0, q_stride[0], q_stride[1], 1, total_q, Hq, d};
  const TensorDesc tk{k, 0, k_stride[0], k_stride[1], 1, total_k, Hkv, d};
  const TensorDesc tv{v, 0, v_stride[0], v_stride[1], 1, total_k, Hkv, d};
  const TensorDesc to{o, 0, o_stride[0], o_stride[1], 1, total_q, Hq, d};
  return fwd_impl(tq, tk, tv, to, lse, size_t(Hq) * total_q * sizeof(float), B, max_seqlen_q,
                  max_seqlen_k, Hq, Hkv, d, cu_seqlens_q, cu_seqlens_k, total_q, total_k, dtype,
                  softmax_scale, causal, window_left, window_right, stream, dp);
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
           int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3], const int64_t k_stride[3],
           const int64_t v_stride[3], const int64_t o_stride[3], int dtype, float softmax_scale,
           int causal, int window_left, int window_right, void* stream) {
  return fwd_dense(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride,
                   dtype, softmax_scale, causal, window_left, window_right, stream, nullptr);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d,
                  const int64_t q_stride[2], const int64_t k_stride[2],
                  const int64_t v_stride[2], const int64_t o_stride[2], int dtype,
                  float softmax_scale, int causal, int window_left, int window_right,
                  void* stream) {
  return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                    total_q, total_k, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride, dtype,
                    softmax_scale, causal, window_left, window_right, stream, nullptr);
}

size_t fa_bwd_workspace_size(int B, int Nq, int Hq, int d) {
  if (B < 1 || Nq < 1 || Hq < 1 || d < 1) return 0;
  const size_t nq_pad = (size_t(Nq) + 127) / 128 * 128;
  return (size_t(B) * Hq * Nq * d + 2 * size_t(B) * Hq * nq_pad) * sizeof(float);
}

}  // extern "C"

namespace {

// Shared body of fa_bwd and fa_bwd_varlen (see fwd_impl for the conventions).
int bwd_impl(const TensorDesc& tq, const TensorDesc& tk, const TensorDesc& tv,
             const TensorDesc& to, const TensorDesc& tdo, const TensorDesc& tdq,
             const TensorDesc& tdk, const TensorDesc& tdv, const float* lse, size_t lse_bytes,
             void* workspace, size_t workspace_bytes, int B, int Nq, int Nk, int Hq, int Hkv,
             int d, const int* cu_q, const int* cu_k, int total_q, int total_k, int dtype,
             float softmax_scale, int causal, int window_left, int window_right, void* stream,
             const fa::DropoutParams* drop = nullptr) {
  int rc;
  for (const TensorDesc* t : {&tq, &tk, &tv, &to, &tdo, &tdq, &tdk, &tdv})
    if ((rc = check_tensor(*t))) return rc;
  if (!lse) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_ALIGNMENT;
  const size_t need = fa_bwd_workspace_size(B, Nq, Hq, d);
  if (workspace == nullptr || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_ALIGNMENT;
  // outputs (dq, dk, dv, workspace) must not overlap each other or any input
  const TensorDesc* ins[] = {&tq, &tk, &tv, &to, &tdo};
  const TensorDesc* outs[] = {&tdq, &tdk, &tdv};
  for (const TensorDesc* ot : outs) {
    for (const TensorDesc* it : ins)
      if (overlaps_t(*ot, *it)) return FA_ERR_INVALID_ARG;
    if (overlaps_span(*ot, lse, lse_bytes) || overlaps_span(*ot, workspace, need))
      return FA_ERR_INVALID_ARG;
  }
  if (overlaps_t(tdq, tdk) || overlaps_t(tdq, tdv) || overlaps_t(tdk, tdv))
    return FA_ERR_INVALID_ARG;
  for (const TensorDesc* it : ins)
    if (overlaps_span(*it, workspace, need)) return FA_ERR_INVALID_ARG;
  {
    const uintptr_t w0 = reinterpret_cast<uintptr_t>(workspace);
    const uintptr_t l0 = reinterpret_cast<uintptr_t>(lse);
    if (overlaps(w0, w0 + need, l0, l0 + lse_bytes)) return FA_ERR_INVALID_ARG;
  }

  if (drop && d == 256) return FA_ERR_UNSUPPORTED;
  // d = 256 streams Q and dO in steps of 32 query rows
  const int q_rows = d == 256 ? fa::Bwd256Cfg::kQ : 128;
  CUtensorMap mq, mk, mv, mdo;
  if ((rc = make_map(&mq, tq, dtype, q_rows)) || (rc = make_map(&mk, tk, dtype)) ||
      (rc = make_map(&mv, tv, dtype)) || (rc = make_map(&mdo, tdo, dtype, q_rows)))
    return rc;
  unsigned int* err = device_error_ptr();
  if (!err) return FA_ERR_CUDA;
  const int nq_pad = (Nq + 127) / 128 * 128;
  float* dq_acc = static_cast<float*>(workspace);
  float* lse2 = dq_acc + size_t(B) * Hq * Nq * d;
  float* Dvec = lse2 + size_t(B) * Hq * nq_pad;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == FA_BF16;

  fa::BwdPrepParams pp{};
  pp.o = to.ptr;
  pp.dout = tdo.ptr;
  pp.lse = lse;
  pp.lse2 = lse2;
  pp.Dvec = Dvec;
  pp.dq_acc = reinterpret_cast<float4*>(dq_acc);
  pp.o_sb = to.sb;
  pp.o_ss = to.ss;
  pp.o_sh = to.sh;
  pp.do_sb = tdo.sb;
  pp.do_ss = tdo.ss;
  pp.do_sh = tdo.sh;
  pp.B = B;
  pp.Nq = Nq;
  pp.Nq_pad = nq_pad;
  pp.Hq = Hq;
  pp.d = d;
  pp.dq_acc_vec4 = int64_t(B) * Hq * Nq * d / 4;
  pp.cu_q = cu_q;
  pp.total_q = total_q;
  {
    const int64_t rows = int64_t(B) * Hq * nq_pad;
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, 148 * 16);
    if (bf16)
      fa::fa_bwd_prep_kernel<true><<<unsigned(blocks), 256, 0, st>>>(pp);
    else
      fa::fa_bwd_prep_kernel<false><<<unsigned(blocks), 256, 0, st>>>(pp);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }

  fa::BwdParams bp{};
  bp.lse2 = lse2;
  bp.Dvec = Dvec;
  bp.dq_acc = dq_acc;
  bp.dk = const_cast<void*>(tdk.ptr);
  bp.dv = const_cast<void*>(tdv.ptr);
  bp.dk_sb = tdk.sb;
  bp.dk_ss = tdk.ss;
  bp.dk_sh = tdk.sh;
  bp.dv_sb = tdv.sb;
  bp.dv_ss = tdv.ss;
  bp.dv_sh = tdv.sh;
  bp.B = B;
  bp.Nq = Nq;
  bp.Nq_pad = nq_pad;
  bp.Nk = Nk;
  bp.Hq = Hq;
  bp.Hkv = Hkv;
  bp.n_ntiles = (Nk + 127) / 128;
  bp.scale = softmax_scale;
  bp.scale_log2 = softmax_scale * 1.4426950408889634f;
  bp.causal = causal ? 1 : 0;
  bp.wl = window_left;
  bp.wr = window_right;
  bp.err = err;
  bp.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  bp.cu_q = cu_q;
  bp.cu_k = cu_k;
  bp.total_q = total_q;
  bp.total_k = total_k;
  if (drop) bp.drop = *drop;
  if (g_bwd_ev_start && cudaEventRecord(g_bwd_ev_start, st) != cudaSuccess) return FA_ERR_CUDA;
  if (d == 256) {
    rc = bf16 ? launch_bwd256<true>(mq, mk, mv, mdo, bp, st)
              : launch_bwd256<false>(mq, mk, mv, mdo, bp, st);
  } else if (drop) {
    if (bf16)
      rc = d == 64 ? launch_bwd<64, true, true>(mq, mk, mv, mdo, bp, st)
                   : launch_bwd<128, true, true>(mq, mk, mv, mdo, bp, st);
    else
      rc = d == 64 ? launch_bwd<64, false, true>(mq, mk, mv, mdo, bp, st)
                   : launch_bwd<128, false, true>(mq, mk, mv, mdo, bp, st);
  } else if (bf16) {
    rc = d == 64 ? launch_bwd<64, true>(mq, mk, mv, mdo, bp, st)
                 : launch_bwd<128, true>(mq, mk, mv, mdo, bp, st);
  } else {
    rc = d == 64 ? launch_bwd<64, false>(mq, mk, mv, mdo, bp, st)
                 : launch_bwd<128, false>(mq, mk, mv, mdo, bp, st);
  }
  if (rc) return rc;
  if (g_bwd_ev_stop && cudaEventRecord(g_bwd_ev_stop, st) != cudaSuccess) return FA_ERR_CUDA;

  fa::BwdConvertParams cp{};
  cp.dq_acc = dq_acc;
  cp.dq = const_cast<void*>(tdq.ptr);
  cp.dq_sb = tdq.sb;
  cp.dq_ss = tdq.ss;
  cp.dq_sh = tdq.sh;
  cp.B = B;
  cp.Nq = Nq;
  cp.Hq = Hq;
  cp.d = d;
  cp.cu_q = cu_q;
  cp.total_q = total_q;
  {
    const int64_t n = int64_t(B) * Hq * Nq * (d / 8);
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 32);
    if (bf16)
      fa::fa_bwd_dq_convert_kernel<true><<<unsigned(blocks), 256, 0, st>>>(cp);
    else
      fa::fa_bwd_dq_convert_kernel<false><<<unsigned(blocks), 256, 0, st>>>(cp);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}


// The dense and packed-batch backward entry points, with or without dropout
// (dp = nullptr: none; head_dim 256 only without).
int bwd_dense(const void* q, const void* k, const void* v, const void* o, const void* dout,
              const float* lse, void* dq, void* dk, void* dv, void* workspace,
              size_t workspace_bytes, int B, int Nq, int Nk, int Hq, int Hkv, int d,
              const int64_t q_stride[3], const int64_t k_stride[3], const int64_t v_stride[3],
              const int64_t o_stride[3], const int64_t do_stride[3],
              const int64_t dq_stride[3], const int64_t dk_stride[3],
              const int64_t dv_stride[3], int dtype, float softmax_scale, int causal,
              int window_left, int window_right, void* stream, const fa::DropoutParams* dp) {
  int rc = check_common(B, Nq, Nk, Hq, Hkv, d, dtype, softmax_scale, window_left, window_right,
                        dp == nullptr);
  if (rc) return rc;
  if (!q_stride || !k_stride || !v_stride || !o_stride || !do_stride || !dq_stride ||
      !dk_stride || !dv_stride)
    return FA_ERR_INVALID_ARG;
  const TensorDesc tq{q, q_stride[0], q_stride[1], q_stride[2], B, Nq, Hq, d};
  const TensorDesc tk{k, k_stride[0], k_stride[1], k_stride[2], B, Nk, Hkv, d};
  const TensorDesc tv{v, v_stride[0], v_stride[1], v_stride[2], B, Nk, Hkv, d};
  const TensorDesc to{o, o_stride[0], o_stride[1], o_stride[2], B, Nq, Hq, d};
  const TensorDesc tdo{dout, do_stride[0], do_stride[1], do_stride[2], B, Nq, Hq, d};
  const TensorDesc tdq{dq, dq_stride[0], dq_stride[1], dq_stride[2], B, Nq, Hq, d};
  const TensorDesc tdk{dk, dk_stride[0], dk_stride[1], dk_stride[2], B, Nk, Hkv, d};
  const TensorDesc tdv{dv, dv_stride[0], dv_stride[1], dv_stride[2], B, Nk, Hkv, d};
  return bwd_impl(tq, tk, tv, to, tdo, tdq, tdk, tdv, lse, size_t(B) * Hq * Nq * sizeof(float),
                  workspace, workspace_bytes, B, Nq, Nk, Hq, Hkv, d, nullptr, nullptr, 0, 0,
                  dtype, softmax_scale, causal, window_left, window_right, stream, dp);
}

int bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, void* workspace,
               size_t workspace_bytes, const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
               int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv,
               int d, const int64_t q_stride[2], const int64_t k_stride[2],
               const int64_t v_stride[2], const int64_t o_stride[2], const int64_t do_stride[2],
               const int64_t dq_stride[2], const int64_t dk_stride[2],
               const int64_t dv_stride[2], int dtype, float softmax_scale, int causal,
               int window_left, int window_right, void* stream, const fa::DropoutParams* dp) {
  int rc = check_common(B, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, dtype, softmax_scale,
                        window_left, window_right, dp == nullptr);
  if (rc) return rc;
  if ((rc = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q,
                         total_k)))
    return rc;
  if (total_q > (1 << 28) || total_k > (1 << 28)) return FA_ERR_INVALID_ARG;
  if (!q_stride || !k_stride || !v_stride || !o_stride || !do_stride || !dq_stride ||
      !dk_stride || !dv_stride)
    return FA_ERR_INVALID_ARG;
  const TensorDesc tq{q, 0, q_stride[0], q_stride[1], 1, total_q, Hq, d};
  const TensorDesc tk{k, 0, k_stride[0], k_stride[1], 1, total_k, Hkv, d};
  const TensorDesc tv{v, 0, v_stride[0], v_stride[1], 1, total_k, Hkv, d};
  const TensorDesc to{o, 0, o_stride[0], o_stride[1], 1, total_q, Hq, d};
  const TensorDesc tdo{dout, 0, do_stride[0], do_stride[1], 1, total_q, Hq, d};
  const TensorDesc tdq{dq, 0, dq_stride[0], dq_stride[1], 1, total_q, Hq, d};
  const TensorDesc tdk{dk, 0, dk_stride[0], dk_stride[1], 1, total_k, Hkv, d};
  const TensorDesc tdv{dv, 0, dv_stride[0], dv_stride[1], 1, total_k, Hkv, d};
  return bwd_impl(tq, tk, tv, to, tdo, tdq, tdk, tdv, lse, size_t(Hq) * total_q * sizeof(float),
                  workspace, workspace_bytes, B, max_seqlen_q, max_seqlen_k, Hq, Hkv, d,
                  cu_seqlens_q, cu_seqlens_k, total_q, total_k, dtype, softmax_scale, causal,
                  window_left, window_right, stream, dp);
}

}  // namespace

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, void* workspace,
           size_t workspace_bytes, int B, int Nq, int Nk, int Hq, int Hkv, int d,
           const int64_t q_stride[3], const int64_t k_stride[3], const int64_t v_stride[3],
           const int64_t o_stride[3], const int64_t do_stride[3], const int64_t dq_stride[3],
           const int64_t dk_stride[3], const int64_t dv_stride[3], int dtype,
           float softmax_scale, int causal, int window_left, int window_right, void* stream) {
  return bwd_dense(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, Nq, Nk, Hq,
                   Hkv, d, q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride, dk_stride,
                   dv_stride, dtype, softmax_scale, causal, window_left, window_right, stream,
                   nullptr);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, void* workspace,
                  size_t workspace_bytes, const int* cu_seqlens_q, const int* cu_seqlens_k,
                  int B, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq,
                  int Hkv, int d, const int64_t q_stride[2], const int64_t k_stride[2],
                  const int64_t v_stride[2], const int64_t o_stride[2],
                  const int64_t do_stride[2], const int64_t dq_stride[2],
                  const int64_t dk_stride[2], const int64_t dv_stride[2], int dtype,
                  float softmax_scale, int causal, int window_left, int window_right,
                  void* stream) {
  return bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, cu_seqlens_q,
                    cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d,
                    q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride, dk_stride,
                    dv_stride, dtype, softmax_scale, causal, window_left, window_right, stream,
                    nullptr);
}

int fa_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int v = 0u, zero = 0u;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_CUDA;
  return (v & fa::kDevErrTimeout) ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation backward
// fa_bwd_noalloc: the backward for callers that cannot call cudaMalloc.  Its
// scratch is this file-scope device array; host code must not pass the
// array's name to a kernel (in host code it is only a stand-in), so the
// device address is looked up once per device with cudaGetSymbolAddress.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device, or nullptr on
// failure.  It is looked up on every call (cheap once the module is loaded on
// the device), so a context that was torn down and created again is never
// handed a stale address.
void* noalloc_scratch_address() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" size_t fa_bwd_noalloc_scratch_bytes(void) { return FA_BWD_NOALLOC_SCRATCH_BYTES; }

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int B, int Nq, int Nk, int Hq, int Hkv, int d,
                              const int64_t q_stride[3], const int64_t k_stride[3],
                              const int64_t v_stride[3], const int64_t o_stride[3],
                              const int64_t do_stride[3], const int64_t dq_stride[3],
                              const int64_t dk_stride[3], const int64_t dv_stride[3], int dtype,
                              float softmax_scale, int causal, int window_left,
                              int window_right, void* stream) {
  const size_t need = fa_bwd_workspace_size(B, Nq, Hq, d);
  if (need > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;  // larger than the array
  void* scratch = noalloc_scratch_address();
  if (scratch == nullptr) return FA_ERR_CUDA;
  // fa_bwd zeroes the dQ accumulator and rewrites the row terms on every call,
  // so the previous call's contents of the shared array do not matter.
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, B, Nq,
                Nk, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride,
                dk_stride, dv_stride, dtype, softmax_scale, causal, window_left, window_right,
                stream);
}

// ------------------------------------------------------------------ paged KV cache (decode)
namespace {

int sm_count() {
  static std::atomic<int> cached[kMaxDevices];  // 0 = not yet read
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < kMaxDevices && (v = cached[dev].load(std::memory_order_relaxed)) > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    return 148;
  if (dev < kMaxDevices) cached[dev].store(v, std::memory_order_relaxed);
  return v;
}

// Splits of the key tiles of every (sequence, kv head): enough CTAs for about
// four per SM (two run at a time) when the batch alone does not provide them,
// and no split longer than 32 tiles, so that long sequences do not leave a
// tail of lone CTAs; at least one tile each.
int decode_splits(int B, int Hkv, int max_tiles, int requested, int& tiles_per_split) {
  int splits;
  if (requested > 0) {
    splits = requested;
  } else {
    const int64_t units = int64_t(B) * Hkv;
    const int64_t want = 4 * int64_t(sm_count());
    const int by_fill = units >= want ? 1 : int((want + units - 1) / units);
    const int by_length = (max_tiles + 31) / 32;
    splits = std::max(by_fill, by_length);
  }
  splits = std::max(1, std::min(splits, max_tiles));
  tiles_per_split = (max_tiles + splits - 1) / splits;
  return (max_tiles + tiles_per_split - 1) / tiles_per_split;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int check_paged_shape(int B, int Nq, int Hq, int Hkv, int d, int page_size, int num_pages,
                      int max_pages, int dtype, float scale, int window_left, int window_right) {
  if (B < 1 || Nq < 1 || Hq < 1 || Hkv < 1 || num_pages < 1 || max_pages < 1)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (window_left < -1 || window_right < -1 || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * Nq > 128) return FA_ERR_UNSUPPORTED;  // one 128-row query tile per kv head
  if (!is_pow2(page_size) || page_size < 8 || page_size > (1 << 20)) return FA_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535 || num_pages > (1 << 30) ||
      int64_t(max_pages) * page_size > (int64_t(1) << 30))
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// 4-D map over a paged cache [num_pages, P, Hkv, d] (innermost first: d, Hkv,
// P, pages), box of 64 columns x 1 head x min(P, 64) rows x 1 page.
int make_cache_map(CUtensorMap* map, const void* ptr, const int64_t st[3], int num_pages, int P,
                   int Hkv, int d, int dtype) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const int64_t sp = num_pages > 1 ? st[0] : 8;
  const int64_t stok = P > 1 ? st[1] : 8;
  const int64_t sh = Hkv > 1 ? st[2] : 8;
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(Hkv), cuuint64_t(P), cuuint64_t(num_pages)};
  cuuint64_t strides[3] = {cuuint64_t(sh) * 2, cuuint64_t(stok) * 2, cuuint64_t(sp) * 2};
  cuuint32_t box[4] = {64, 1, cuuint32_t(std::min(P, 64)), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map,
                   dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_ALIGNMENT;
}

// 4-D map over q [B, Nq, Hq, d] whose box is the whole query tile of one kv
// head: 64 columns x Nq queries x G heads x 1 sequence (rows h' * Nq + i).
int make_group_q_map(CUtensorMap* map, const TensorDesc& t, int G, int dtype) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const int64_t ss = t.N > 1 ? t.ss : 8;
  const int64_t sh = t.H > 1 ? t.sh : 8;
  const int64_t sb = t.B > 1 ? t.sb : 8;
  cuuint64_t dims[4] = {cuuint64_t(t.d), cuuint64_t(t.N), cuuint64_t(t.H), cuuint64_t(t.B)};
  cuuint64_t strides[3] = {cuuint64_t(ss) * 2, cuuint64_t(sh) * 2, cuuint64_t(sb) * 2};
  cuuint32_t box[4] = {64, cuuint32_t(t.N), cuuint32_t(G), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map,
                   dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   4, const_cast<void*>(t.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_ALIGNMENT;
}

size_t paged_workspace_bytes(int B, int Hkv, int R, int d, int splits) {
  if (splits <= 1) return 0;
  const size_t rows = size_t(B) * Hkv * splits * R;
  const size_t o_bytes = (rows * d * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + rows * sizeof(float);
}

template <int D, bool BF16>
int launch_decode(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const fa::DecodeParams& prm, cudaStream_t st) {
  using Cfg = fa::DecCfg<D>;
  auto kern = fa::fa_decode_kernel<D, BF16>;
  static DeviceOnce once;  // per instantiation: attributes set on each device used
  {
    const int rc_once = once_per_device(once, [&]() -> int {  // room for the largest query tile (128 rows)
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::smem_bytes(128)) != cudaSuccess)
        return int(FA_ERR_CUDA);
      return int(FA_OK);
    });
    if (rc_once) return rc_once;
  }
  const int smem = Cfg::smem_bytes((prm.R + 7) & ~7);
  dim3 grid(unsigned(prm.n_splits), unsigned(prm.Hkv), unsigned(prm.B));
  kern<<<grid, Cfg::kThreads, smem, st>>>(mq, mk, mv, prm);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (prm.n_splits > 1) {
    const int64_t rows = int64_t(prm.B) * prm.Hq * prm.Nq;
    fa::fa_decode_combine_kernel<D, BF16><<<unsigned((rows + 3) / 4), 128, 0, st>>>(prm);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

}  // namespace

extern "C" {

size_t fa_fwd_paged_workspace_size(int B, int Nq, int Hq, int Hkv, int d, int page_size,
                                   int max_pages_per_seq, int num_splits) {
  if (check_paged_shape(B, Nq, Hq, Hkv, d, page_size, 1, max_pages_per_seq, FA_BF16, 1.f, -1,
                        -1))
    return 0;
  const int max_tiles =
      int((int64_t(max_pages_per_seq) * page_size + fa::DecCfg<128>::kKeys - 1) /
          fa::DecCfg<128>::kKeys);
  int tps = 0;
  const int splits = decode_splits(B, Hkv, max_tiles, num_splits, tps);
  return paged_workspace_bytes(B, Hkv, (Hq / Hkv) * Nq, d, splits);
}

int fa_fwd_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                 const int* cache_seqlens, void* o, float* lse, int B, int Nq, int Hq, int Hkv,
                 int d, int page_size, int num_pages, int max_pages_per_seq,
                 int64_t block_table_stride, const int64_t q_stride[3],
                 const int64_t kcache_stride[3], const int64_t vcache_stride[3],
                 const int64_t o_stride[3], int dtype, float softmax_scale, int causal,
                 int window_left, int window_right, int num_splits, void* workspace,
                 size_t workspace_bytes, void* stream) {
  int rc = check_paged_shape(B, Nq, Hq, Hkv, d, page_size, num_pages, max_pages_per_seq, dtype,
                             softmax_scale, window_left, window_right);
  if (rc) return rc;
  if (!q_stride || !kcache_stride || !vcache_stride || !o_stride || !lse || !block_table ||
      !cache_seqlens || num_splits < 0)
    return FA_ERR_INVALID_ARG;
  if (block_table_stride < max_pages_per_seq) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGNMENT;
  const int G = Hq / Hkv;
  const TensorDesc tq{q, q_stride[0], q_stride[1], q_stride[2], B, Nq, Hq, d};
  const TensorDesc to{o, o_stride[0], o_stride[1], o_stride[2], B, Nq, Hq, d};
  // the caches as [pages, page_size, Hkv, d] descriptors (batch = page)
  const TensorDesc tk{k_cache, kcache_stride[0], kcache_stride[1], kcache_stride[2], num_pages,
                      page_size, Hkv, d};
  const TensorDesc tv{v_cache, vcache_stride[0], vcache_stride[1], vcache_stride[2], num_pages,
                      page_size, Hkv, d};
  for (const TensorDesc* t : {&tq, &to, &tk, &tv})
    if ((rc = check_tensor(*t))) return rc;
  const size_t lse_bytes = size_t(B) * Hq * Nq * sizeof(float);
  if (overlaps_t(to, tq) || overlaps_t(to, tk) || overlaps_t(to, tv) ||
      overlaps_span(tq, lse, lse_bytes) || overlaps_span(tk, lse, lse_bytes) ||
      overlaps_span(tv, lse, lse_bytes) || overlaps_span(to, lse, lse_bytes))
    return FA_ERR_INVALID_ARG;

  const int max_tiles = int((int64_t(max_pages_per_seq) * page_size + fa::DecCfg<128>::kKeys - 1) /
                            fa::DecCfg<128>::kKeys);
  int tps = 0;
  const int splits = decode_splits(B, Hkv, max_tiles, num_splits, tps);
  const size_t need = paged_workspace_bytes(B, Hkv, G * Nq, d, splits);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_ALIGNMENT;
    if (overlaps_span(to, workspace, need) || overlaps_span(tq, workspace, need) ||
        overlaps(reinterpret_cast<uintptr_t>(lse), reinterpret_cast<uintptr_t>(lse) + lse_bytes,
                 reinterpret_cast<uintptr_t>(workspace),
                 reinterpret_cast<uintptr_t>(workspace) + need))
      return FA_ERR_INVALID_ARG;
  }

  CUtensorMap mq, mk, mv;
  if ((rc = make_group_q_map(&mq, tq, G, dtype)) ||
      (rc = make_cache_map(&mk, k_cache, kcache_stride, num_pages, page_size, Hkv, d, dtype)) ||
      (rc = make_cache_map(&mv, v_cache, vcache_stride, num_pages, page_size, Hkv, d, dtype)))
    return rc;
  fa::DecodeParams prm{};
  prm.block_table = block_table;
  prm.cache_seqlens = cache_seqlens;
  prm.bt_stride = block_table_stride;
  prm.B = B;
  prm.Nq = Nq;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = G;
  prm.R = G * Nq;
  prm.P = page_size;
  prm.num_pages = num_pages;
  prm.max_pages = max_pages_per_seq;
  prm.n_splits = splits;
  prm.tiles_per_split = tps;
  prm.scale_log2 = scale_log2_of(softmax_scale);
  prm.qk_negate = softmax_scale < 0.f ? 1u : 0u;
  prm.causal = causal ? 1 : 0;
  prm.wl = window_left;
  prm.wr = window_right;
  prm.o = o;
  prm.o_sb = to.sb;
  prm.o_ss = to.ss;
  prm.o_sh = to.sh;
  prm.lse = lse;
  if (need > 0) {
    const size_t rows = size_t(B) * Hkv * splits * G * Nq;
    prm.part_o = static_cast<float*>(workspace);
    prm.part_lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                             ((rows * d * sizeof(float) + 255) & ~size_t(255)));
  }
  prm.err = device_error_ptr();
  prm.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  if (!prm.err) return FA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? launch_decode<64, true>(mq, mk, mv, prm, st)
                   : launch_decode<128, true>(mq, mk, mv, prm, st);
  return d == 64 ? launch_decode<64, false>(mq, mk, mv, prm, st)
                 : launch_decode<128, false>(mq, mk, mv, prm, st);
}

}  // extern "C"

// ------------------------------------------------------------------ FP8 (e4m3) forward
namespace {

// An e4m3 tensor [B, N, H, d]: one byte per element, so strides (in
// elements) must be multiples of 16 for the 16-byte TMA rule.
int check_tensor_fp8(const TensorDesc& t) {
  if (t.ptr == nullptr) return FA_ERR_INVALID_ARG;
  if (t.sb < 0 || t.ss < 0 || t.sh < 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return FA_ERR_ALIGNMENT;
  if ((t.B > 1 && t.sb % 16) || (t.N > 1 && t.ss % 16) || (t.H > 1 && t.sh % 16))
    return FA_ERR_ALIGNMENT;
  return FA_OK;
}

void tensor_extent_bytes(const TensorDesc& t, int elem, uintptr_t& lo, uintptr_t& hi) {
  const int64_t last = int64_t(t.B - 1) * t.sb + int64_t(t.N - 1) * t.ss +
                       int64_t(t.H - 1) * t.sh + t.d;
  lo = reinterpret_cast<uintptr_t>(t.ptr);
  hi = lo + uintptr_t(last) * uintptr_t(elem);
}

// 4-D map over an e4m3 [B, N, H, d] tensor, box of d columns x 128 rows, with
// the 128-byte (d = 128) or 64-byte (d = 64) swizzle of one row.
int make_map_fp8(CUtensorMap* map, const TensorDesc& t) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const int64_t ss = t.N > 1 ? t.ss : 16;
  const int64_t sh = t.H > 1 ? t.sh : 16;
  const int64_t sb = t.B > 1 ? t.sb : 16;
  cuuint64_t dims[4] = {cuuint64_t(t.d), cuuint64_t(t.N), cuuint64_t(t.H), cuuint64_t(t.B)};
  cuuint64_t strides[3] = {cuuint64_t(ss), cuuint64_t(sh), cuuint64_t(sb)};
  cuuint32_t box[4] = {cuuint32_t(t.d), 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(t.ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   t.d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_ALIGNMENT;
}

template <int D>
int launch_fwd_fp8(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const fa::Fp8Params& prm, cudaStream_t st) {
  using Cfg = fa::Fp8Cfg<D>;
  auto kern = fa::fa_fwd_fp8_kernel<D>;
  static DeviceOnce once;  // per instantiation: attributes set on each device used
  {
    const int rc_once = once_per_device(once, [&]() -> int {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::kSmemBytes) != cudaSuccess)
        return int(FA_ERR_CUDA);
      return int(FA_OK);
    });
    if (rc_once) return rc_once;
  }
  dim3 grid(unsigned(prm.B * prm.Hq), unsigned(prm.n_mblocks));
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
               int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3],
               const int64_t k_stride[3], const int64_t v_stride[3], const int64_t o_stride[3],
               float descale_q, float descale_k, float descale_v, float softmax_scale,
               int causal, int window_left, int window_right, void* stream) {
  // dtype argument of the 16-bit checks: the output is bf16
  int rc = check_common(B, Nq, Nk, Hq, Hkv, d, FA_BF16, softmax_scale, window_left,
                        window_right);
  if (rc) return rc;
  if (!q_stride || !k_stride || !v_stride || !o_stride || !lse) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(descale_q) || !std::isfinite(descale_k) || !std::isfinite(descale_v))
    return FA_ERR_INVALID_ARG;
  const TensorDesc tq{q, q_stride[0], q_stride[1], q_stride[2], B, Nq, Hq, d};
  const TensorDesc tk{k, k_stride[0], k_stride[1], k_stride[2], B, Nk, Hkv, d};
  const TensorDesc tv{v, v_stride[0], v_stride[1], v_stride[2], B, Nk, Hkv, d};
  const TensorDesc to{o, o_stride[0], o_stride[1], o_stride[2], B, Nq, Hq, d};
  for (const TensorDesc* t : {&tq, &tk, &tv})
    if ((rc = check_tensor_fp8(*t))) return rc;
  if ((rc = check_tensor(to))) return rc;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_ALIGNMENT;
  const size_t lse_bytes = size_t(B) * Hq * Nq * sizeof(float);
  uintptr_t o0, o1, l0 = reinterpret_cast<uintptr_t>(lse), l1 = l0 + lse_bytes;
  tensor_extent(to, o0, o1);
  for (const TensorDesc* t : {&tq, &tk, &tv}) {
    uintptr_t a0, a1;
    tensor_extent_bytes(*t, 1, a0, a1);
    if (overlaps(a0, a1, o0, o1) || overlaps(a0, a1, l0, l1)) return FA_ERR_INVALID_ARG;
  }
  if (overlaps(o0, o1, l0, l1)) return FA_ERR_INVALID_ARG;

  CUtensorMap mq, mk, mv;
  if ((rc = make_map_fp8(&mq, tq)) || (rc = make_map_fp8(&mk, tk)) ||
      (rc = make_map_fp8(&mv, tv)))
    return rc;
  fa::Fp8Params prm{};
  prm.o = o;
  prm.lse = lse;
  prm.o_sb = to.sb;
  prm.o_ss = to.ss;
  prm.o_sh = to.sh;
  prm.B = B;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.n_mblocks = (Nq + 255) / 256;
  // the dequantisation factors of Q and K scale every score; a negative
  // product flips the sign of Q K^T like a negative softmax scale
  const float qk = softmax_scale * descale_q * descale_k;
  prm.scale_log2 = scale_log2_of(qk);
  prm.qk_negate = qk < 0.f ? 1u : 0u;
  prm.out_scale = descale_v;
  prm.causal = causal ? 1 : 0;
  prm.wl = window_left;
  prm.wr = window_right;
  prm.err = device_error_ptr();
  prm.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  if (!prm.err) return FA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_fwd_fp8<64>(mq, mk, mv, prm, st)
                 : launch_fwd_fp8<128>(mq, mk, mv, prm, st);
}

}  // extern "C"

// ------------------------------------------------------------------ dropout
namespace {

// Keep threshold of dropout probability p: T = round(256 (1 - p)).  Returns
// FA_OK with *T in [1, 256] (256: nothing is dropped), or INVALID_ARG.
int dropout_threshold(float p, int* T) {
  if (!std::isfinite(p) || p < 0.f || p >= 1.f) return FA_ERR_INVALID_ARG;
  const int t = int(std::lround(256.0 * (1.0 - double(p))));
  if (t < 1) return FA_ERR_INVALID_ARG;
  *T = std::min(t, 256);
  return FA_OK;
}

fa::DropoutParams make_dropout(int T, uint64_t seed, uint32_t offset) {
  fa::DropoutParams dp{};
  dp.T = uint32_t(T);
  dp.seed_lo = uint32_t(seed);
  dp.seed_hi = uint32_t(seed >> 32);
  dp.offset = offset;
  dp.scale = 256.f / float(T);
  return dp;
}

}  // namespace

extern "C" {

int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int Nq, int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3],
                   const int64_t k_stride[3], const int64_t v_stride[3],
                   const int64_t o_stride[3], int dtype, float softmax_scale, int causal,
                   int window_left, int window_right, float dropout_p, uint64_t seed,
                   uint32_t offset, void* stream) {
  int T = 0;
  const int rc = dropout_threshold(dropout_p, &T);
  if (rc) return rc;
  if (T >= 256)  // nothing is dropped
    return fwd_dense(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride,
                     dtype, softmax_scale, causal, window_left, window_right, stream, nullptr);
  const fa::DropoutParams dp = make_dropout(T, seed, offset);
  return fwd_dense(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride,
                   dtype, softmax_scale, causal, window_left, window_right, stream, &dp);
}

int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                   const int64_t q_stride[3], const int64_t k_stride[3],
                   const int64_t v_stride[3], const int64_t o_stride[3],
                   const int64_t do_stride[3], const int64_t dq_stride[3],
                   const int64_t dk_stride[3], const int64_t dv_stride[3], int dtype,
                   float softmax_scale, int causal, int window_left, int window_right,
                   float dropout_p, uint64_t seed, uint32_t offset, void* stream) {
  int T = 0;
  const int rc = dropout_threshold(dropout_p, &T);
  if (rc) return rc;
  if (T >= 256)  // nothing is dropped
    return bwd_dense(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, Nq, Nk, Hq,
                     Hkv, d, q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride,
                     dk_stride, dv_stride, dtype, softmax_scale, causal, window_left, window_right,
                     stream, nullptr);
  const fa::DropoutParams dp = make_dropout(T, seed, offset);
  return bwd_dense(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, Nq, Nk, Hq,
                   Hkv, d, q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride, dk_stride,
                   dv_stride, dtype, softmax_scale, causal, window_left, window_right, stream, &dp);
}

int fa_fwd_varlen_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                          int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq,
                          int Hkv, int d, const int64_t q_stride[2], const int64_t k_stride[2],
                          const int64_t v_stride[2], const int64_t o_stride[2], int dtype,
                          float softmax_scale, int causal, int window_left, int window_right,
                          float dropout_p, uint64_t seed, uint32_t offset, void* stream) {
  int T = 0;
  const int rc = dropout_threshold(dropout_p, &T);
  if (rc) return rc;
  if (T >= 256)  // nothing is dropped
    return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                      total_q, total_k, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride, dtype,
                      softmax_scale, causal, window_left, window_right, stream, nullptr);
  const fa::DropoutParams dp = make_dropout(T, seed, offset);
  return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                    total_q, total_k, Hq, Hkv, d, q_stride, k_stride, v_stride, o_stride, dtype,
                    softmax_scale, causal, window_left, window_right, stream, &dp);
}

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
                          float dropout_p, uint64_t seed, uint32_t offset, void* stream) {
  int T = 0;
  const int rc = dropout_threshold(dropout_p, &T);
  if (rc) return rc;
  if (T >= 256)  // nothing is dropped
    return bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, cu_seqlens_q,
                      cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d,
                      q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride, dk_stride,
                      dv_stride, dtype, softmax_scale, causal, window_left, window_right, stream,
                      nullptr);
  const fa::DropoutParams dp = make_dropout(T, seed, offset);
  return bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, cu_seqlens_q,
                    cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d,
                    q_stride, k_stride, v_stride, o_stride, do_stride, dq_stride, dk_stride,
                    dv_stride, dtype, softmax_scale, causal, window_left, window_right, stream,
                    &dp);
}

}  // extern "C"
