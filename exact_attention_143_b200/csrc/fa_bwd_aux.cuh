// fa_bwd_aux.cuh -- the two small launches around the backward main kernel
// (fa_bwd.cuh describes the whole backward):
//   1. fa_bwd_prep_kernel: D_i = sum_c dO_ic O_ic and LSE2_i = LSE_i * log2(e)
//      per query row (fp32, padded to a multiple of 128 rows), and zeroes the
//      fp32 dQ accumulator.
//   3. fa_bwd_dq_convert_kernel: the fp32 dQ accumulator -> dQ in the input
//      dtype.
#pragma once

#include <cuda_fp16.h>

#include "fa_bwd.cuh"
#include "fa_ptx.cuh"

namespace fa {

// ------------------------------------------------------------------ kernel 1
struct BwdPrepParams {
  const void* o;
  const void* dout;
  const float* lse;
  float* lse2;     // [B, Hq, Nq_pad]
  float* Dvec;     // [B, Hq, Nq_pad]
  float4* dq_acc;  // [B, Hq, Nq, d] fp32, zeroed here
  int64_t o_sb, o_ss, o_sh, do_sb, do_ss, do_sh;
  int B, Nq, Nq_pad, Hq, d;
  int64_t dq_acc_vec4;  // number of float4 in dq_acc
  const int* cu_q;      // variable-length batches: token offsets [B + 1] (else nullptr)
  int total_q;
};

// Dot product of four 16-bit values packed in two words with four others.
template <bool BF16>
__device__ __forceinline__ float dot4_16(uint2 a, uint2 b) {
  float2 a0, a1, b0, b1;
  if constexpr (BF16) {
    a0 = make_float2(__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xFFFF0000u));
    a1 = make_float2(__uint_as_float(a.y << 16), __uint_as_float(a.y & 0xFFFF0000u));
    b0 = make_float2(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u));
    b1 = make_float2(__uint_as_float(b.y << 16), __uint_as_float(b.y & 0xFFFF0000u));
  } else {
    a0 = __half22float2(*reinterpret_cast<const __half2*>(&a.x));
    a1 = __half22float2(*reinterpret_cast<const __half2*>(&a.y));
    b0 = __half22float2(*reinterpret_cast<const __half2*>(&b.x));
    b1 = __half22float2(*reinterpret_cast<const __half2*>(&b.y));
  }
  return fmaf(a0.x, b0.x, fmaf(a0.y, b0.y, fmaf(a1.x, b1.x, a1.y * b1.y)));
}

// Each lane reads 4 consecutive elements (8 bytes) of a row of O and of dO;
// min(32, d / 4) lanes share a row, so a warp covers 32 / that many rows per
// pass (2 at d = 64, 1 at d = 128 and 256).
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const BwdPrepParams p) {
  const int64_t nrows = int64_t(p.B) * p.Hq * p.Nq_pad;
  const int lpr = min(32, p.d / 4);  // lanes per row
  const int rpw = 32 / lpr;          // rows per warp pass
  const int lane = threadIdx.x & 31;
  const int sub = lane / lpr, sl = lane % lpr;
  const int64_t warp_id = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r0 = warp_id * rpw; r0 < nrows; r0 += nwarps * rpw) {
    const int64_t r = r0 + sub;
    float acc = 0.f, lse2 = INFINITY;
    if (r < nrows) {
      const int i = int(r % p.Nq_pad);
      const int64_t bh = r / p.Nq_pad;
      const int h = int(bh % p.Hq), b = int(bh / p.Hq);
      int len, start;
      seq_rows(p.cu_q, b, p.total_q, p.Nq, len, start);
      const int bc = p.cu_q ? 0 : b;
      if (i < len) {
        const uint16_t* orow = static_cast<const uint16_t*>(p.o) + bc * p.o_sb +
                               int64_t(start + i) * p.o_ss + int64_t(h) * p.o_sh;
        const uint16_t* drow = static_cast<const uint16_t*>(p.dout) + bc * p.do_sb +
                               int64_t(start + i) * p.do_ss + int64_t(h) * p.do_sh;
        for (int c = 4 * sl; c < p.d; c += 4 * lpr)
          acc += dot4_16<BF16>(*reinterpret_cast<const uint2*>(orow + c),
                               *reinterpret_cast<const uint2*>(drow + c));
        const float l = p.cu_q ? p.lse[int64_t(h) * p.total_q + start + i]
                               : p.lse[(int64_t(b) * p.Hq + h) * p.Nq + i];
        lse2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
      }
    }
    // sum over the lanes of the row (an aligned group of lpr lanes)
    for (int o = lpr / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (sl == 0 && r < nrows) {
      p.Dvec[r] = acc;
      p.lse2[r] = lse2;
    }
  }
  // zero the dQ accumulator
  const int64_t tid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthr = int64_t(gridDim.x) * blockDim.x;
  for (int64_t x = tid; x < p.dq_acc_vec4; x += nthr) p.dq_acc[x] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------ kernel 3
struct BwdConvertParams {
  const float* dq_acc;  // [B, Hq, Nq, d]
  void* dq;
  int64_t dq_sb, dq_ss, dq_sh;
  int B, Nq, Hq, d;
  const int* cu_q;  // variable-length batches (else nullptr)
  int total_q;
};

// One thread per 8 consecutive elements of one row (16-byte store).
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const BwdConvertParams p) {
  const int per_row = p.d / 8;
  const int64_t n = int64_t(p.B) * p.Hq * p.Nq * per_row;
  for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < n;
       x += int64_t(gridDim.x) * blockDim.x) {
    const int c8 = int(x % per_row);
    const int64_t row = x / per_row;  // (b, h, i)
    const int i = int(row % p.Nq);
    const int64_t bh = row / p.Nq;
    const int h = int(bh % p.Hq), b = int(bh / p.Hq);
    int len, start;
    seq_rows(p.cu_q, b, p.total_q, p.Nq, len, start);
    if (i >= len) continue;
    const int bc = p.cu_q ? 0 : b;
    const float4* src = reinterpret_cast<const float4*>(p.dq_acc + row * p.d + c8 * 8);
    const float4 a = src[0], c = src[1];
    uint4 out;
    out.x = pack2<BF16>(a.x, a.y);
    out.y = pack2<BF16>(a.z, a.w);
    out.z = pack2<BF16>(c.x, c.y);
    out.w = pack2<BF16>(c.z, c.w);
    uint16_t* dst = static_cast<uint16_t*>(p.dq) + bc * p.dq_sb + int64_t(start + i) * p.dq_ss +
                    int64_t(h) * p.dq_sh + c8 * 8;
    *reinterpret_cast<uint4*>(dst) = out;
  }
}

}  // namespace fa
