// fa143_api.cu -- the C ABI of libfa143.so (declared in include/fa143.h):
// argument validation, tensor-map (TMA descriptor) construction and kernel
// launches.  No device memory is allocated here beyond the process-lifetime
// error word below; the caller owns every tensor and the workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa143.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"

namespace {

__device__ unsigned int g_device_error = 0u;

uint64_t g_wait_limit_ns = 2000000000ull;

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
                 int window_left, int window_right) {
  if (B < 1 || Nq < 1 || Nk < 1 || Hq < 1 || Hkv < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (window_left < -1 || window_right < -1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // grid and TMA coordinate limits
  if (Nq > (1 << 24) || Nk > (1 << 24) || int64_t(B) * Hq > (int64_t(1) << 30))
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// 4-D tensor map over [B, N, H, d] (innermost first: d, N, H, B), box of
// 64 columns x 128 rows, 128-byte swizzle, zero fill outside the tensor.
int make_map(CUtensorMap* map, const TensorDesc& t, int dtype) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  // strides of size-1 dimensions are never used; give them a legal value
  const int64_t ss = t.N > 1 ? t.ss : 8;
  const int64_t sh = t.H > 1 ? t.sh : 8;
  const int64_t sb = t.B > 1 ? t.sb : 8;
  cuuint64_t dims[4] = {cuuint64_t(t.d), cuuint64_t(t.N), cuuint64_t(t.H), cuuint64_t(t.B)};
  cuuint64_t strides[3] = {cuuint64_t(ss) * 2, cuuint64_t(sh) * 2, cuuint64_t(sb) * 2};
  cuuint32_t box[4] = {64, 128, 1, 1};
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

template <int D, bool BF16>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const fa::FwdParams& prm, cudaStream_t st) {
  using Cfg = fa::FwdCfg<D>;
  auto kern = fa::fa_fwd_kernel<D, BF16>;
  static bool attr_done = false;  // per instantiation and process
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmemBytes) != cudaSuccess)
      return FA_ERR_CUDA;
    attr_done = true;
  }
  dim3 grid(unsigned(prm.B * prm.Hq), unsigned(prm.n_mblocks));
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mq, mk, mv, prm);
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

uint64_t fa_set_wait_limit_ns(uint64_t limit_ns) {
  const uint64_t old = g_wait_limit_ns;
  g_wait_limit_ns = limit_ns;
  return old;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
           int Nk, int Hq, int Hkv, int d, const int64_t q_stride[3], const int64_t k_stride[3],
           const int64_t v_stride[3], const int64_t o_stride[3], int dtype, float softmax_scale,
           int causal, int window_left, int window_right, void* stream) {
  int rc = check_common(B, Nq, Nk, Hq, Hkv, d, dtype, softmax_scale, window_left, window_right);
  if (rc) return rc;
  if (!q_stride || !k_stride || !v_stride || !o_stride || !lse) return FA_ERR_INVALID_ARG;
  const TensorDesc tq{q, q_stride[0], q_stride[1], q_stride[2], B, Nq, Hq, d};
  const TensorDesc tk{k, k_stride[0], k_stride[1], k_stride[2], B, Nk, Hkv, d};
  const TensorDesc tv{v, v_stride[0], v_stride[1], v_stride[2], B, Nk, Hkv, d};
  const TensorDesc to{o, o_stride[0], o_stride[1], o_stride[2], B, Nq, Hq, d};
  for (const TensorDesc* t : {&tq, &tk, &tv, &to})
    if ((rc = check_tensor(*t))) return rc;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_ALIGNMENT;
  const size_t lse_bytes = size_t(B) * Hq * Nq * sizeof(float);
  if (overlaps_t(to, tq) || overlaps_t(to, tk) || overlaps_t(to, tv) ||
      overlaps_span(tq, lse, lse_bytes) || overlaps_span(tk, lse, lse_bytes) ||
      overlaps_span(tv, lse, lse_bytes) || overlaps_span(to, lse, lse_bytes))
    return FA_ERR_INVALID_ARG;

  CUtensorMap mq, mk, mv;
  if ((rc = make_map(&mq, tq, dtype)) || (rc = make_map(&mk, tk, dtype)) ||
      (rc = make_map(&mv, tv, dtype)))
    return rc;
  fa::FwdParams prm{};
  prm.o = o;
  prm.lse = lse;
  prm.o_sb = o_stride[0];
  prm.o_ss = o_stride[1];
  prm.o_sh = o_stride[2];
  prm.B = B;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.n_mblocks = (Nq + 255) / 256;
  prm.scale_log2 = scale_log2_of(softmax_scale);
  prm.qk_negate = softmax_scale < 0.f ? 1u : 0u;
  prm.causal = causal ? 1 : 0;
  prm.wl = window_left;
  prm.wr = window_right;
  prm.err = device_error_ptr();
  prm.wait_limit_ns = g_wait_limit_ns;
  if (!prm.err) return FA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16)
    return d == 64 ? launch_fwd<64, true>(mq, mk, mv, prm, st)
                   : launch_fwd<128, true>(mq, mk, mv, prm, st);
  return d == 64 ? launch_fwd<64, false>(mq, mk, mv, prm, st)
                 : launch_fwd<128, false>(mq, mk, mv, prm, st);
}

size_t fa_bwd_workspace_size(int B, int Nq, int Hq, int d) {
  if (B < 1 || Nq < 1 || Hq < 1 || d < 1) return 0;
  return size_t(B) * Nq * Hq * d * sizeof(float) + 2 * size_t(B) * Hq * Nq * sizeof(float) + 256;
}

int fa_bwd(const void*, const void*, const void*, const void*, const void*, const float*, void*,
           void*, void*, void*, size_t, int, int, int, int, int, int, const int64_t*,
           const int64_t*, const int64_t*, const int64_t*, const int64_t*, const int64_t*,
           const int64_t*, const int64_t*, int, float, int, int, int, void*) {
  return FA_ERR_UNSUPPORTED;
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
