// fa_fwd_fp8.cuh -- sm_100a forward of exact attention on FP8 (e4m3) inputs.
//
// Q, K and V arrive as float8_e4m3fn ("optimizing-attention-flash", Workflow
// 3, Steps 3 and 4: inputs cast to float8_e4m3fn and passed to the same
// attention call; "Что такое FlashAttention…", section on versions and
// hardware: FP8 runs at about twice the FP16 tensor rate), optionally with
// per-tensor dequantisation factors: the kernel computes attention of
// descale_q Q, descale_k K and descale_v V, with the output in bf16 and the
// LSE in fp32, like the 16-bit forward.
//
// Both products run on the tensor cores in kind::f8f6f4 (e4m3 x e4m3, fp32
// accumulation).  S = Q K^T is exact up to fp32 accumulation.  For O += P V,
// P is rounded to e4m3, scaled first by 2^6 so that the probabilities that
// matter stay in e4m3's normal range: with the lazy rescale threshold of 2^2
// used here P' = 2^6 exp2(s - m) never exceeds 2^8 = 256 (e4m3 saturates at
// 448).  The row sum l is accumulated from the unrounded fp32 P', so the 2^6
// cancels in O / l and is taken out of the LSE.
//
// B200 mapping (one CTA = 256 query rows of one (batch, head)):
//   warp 9       TMA producer: Q tiles once, then a ring of K and V tiles of
//                128 rows, 128- (d = 128) or 64-byte (d = 64) swizzled.
//   warp 8       tcgen05 issuer, in order: P_t V_j, then S_t(j+1) into the same
//                tensor-memory region (P overlays the first 32 columns of S).
//   warps 0-7    softmax of query tiles 0 and 1, thread r = row r; epilogue.
// Tensor memory: S_0, S_1 at columns 0 and 128, O_0, O_1 at 256 and 256 + d.
#pragma once

#include <cuda_fp16.h>

#include "fa_exp2.cuh"
#include "fa_fwd.cuh"  // row_key_range, fmax3
#include "fa_ptx.cuh"

namespace fa {

struct Fp8Params {
  void* o;  // bf16 [B, Nq, Hq, d]
  float* lse;
  int64_t o_sb, o_ss, o_sh;
  int B, Nq, Nk, Hq, Hkv;
  int n_mblocks;
  float scale_log2;  // |softmax_scale| * descale_q * descale_k * log2(e)
  float out_scale;   // descale_v
  uint32_t qk_negate;
  int causal, wl, wr;
  unsigned int* err;
  uint64_t wait_limit_ns;
};

template <int D>
struct Fp8Cfg {
  static constexpr int kTileBytes = 128 * D;  // 128 rows of d one-byte elements
  static constexpr int kStages = D == 64 ? 8 : 4;
  static constexpr int kThreads = 320;
  static constexpr int kSmemQ = 1024;
  static constexpr int kSmemK = kSmemQ + 2 * kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBytes = kSmemV + kStages * kTileBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
  // shared-memory descriptor layout type: 2 = 128-byte swizzle, 4 = 64-byte
  static constexpr uint64_t kLayout = D == 128 ? 2 : 4;
  static constexpr int kEmuPairsPer8 = D == 64 ? 3 : 2;
  static constexpr float kPShift = 6.f;  // P is held as 2^6 exp2(s - m)
  static constexpr float kLazy = 2.f;    // rescale once the row max grows by more than 2^2
};

// Constant part of a shared-memory descriptor with the given swizzle layout
// type (PTX ISA, "Shared memory descriptor": LBO >> 4 at [16,30), SBO >> 4 at
// [32,46), version 1 at 46, layout type at [61,64)).
__host__ __device__ constexpr uint64_t sdesc_const_layout(uint32_t lbo, uint32_t sbo,
                                                          uint64_t layout) {
  return (uint64_t((lbo >> 4) & 0x3FFFu) << 16) | (uint64_t((sbo >> 4) & 0x3FFFu) << 32) |
         (uint64_t(1) << 46) | (layout << 61);
}

// Instruction descriptor of kind::f8f6f4 with e4m3 A and B (format code 0)
// and fp32 accumulation; same field positions as kind::f16.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int M, int N, bool a_mn_major,
                                                       bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Four fp32 values as four e4m3 bytes of one 32-bit word, x0 in the lowest
// byte (round to nearest even, saturating at the largest finite value).
__device__ __forceinline__ uint32_t pack4_e4m3(float x0, float x1, float x2, float x3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
  return uint32_t(lo) | (uint32_t(hi) << 16);
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Fp8Params p) {
  using Cfg = Fp8Cfg<D>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  const uint32_t bar_q = smem_u32(&bars[0]);
  auto bar_kvfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bar_kvempty = [&](int s) { return smem_u32(&bars[1 + S + s]); };
  auto bar_sfull = [&](int t) { return smem_u32(&bars[1 + 2 * S + t]); };
  auto bar_pfull = [&](int t) { return smem_u32(&bars[3 + 2 * S + t]); };
  auto bar_odone = [&](int t) { return smem_u32(&bars[5 + 2 * S + t]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int mblock = p.n_mblocks - 1 - int(blockIdx.y);  // heaviest causal blocks first
  const int Nq = p.Nq, Nk = p.Nk;

  // K-tile range [jlo_t, jhi_t) of query tile t
  auto tile_range = [&](int t, int& lo_j, int& hi_j) {
    const int r0 = mblock * 256 + t * 128;
    lo_j = 0;
    hi_j = 0;
    if (r0 < Nq) {
      const int r1 = min(r0 + 127, Nq - 1);
      int lo0, hi0, lo1, hi1;
      row_key_range(r0, Nq, Nk, p.causal, p.wl, p.wr, lo0, hi0);
      row_key_range(r1, Nq, Nk, p.causal, p.wl, p.wr, lo1, hi1);
      if (lo0 <= hi1) {
        lo_j = lo0 / 128;
        hi_j = hi1 / 128 + 1;
      }
    }
  };
  int jlo0, jhi0, jlo1, jhi1;
  tile_range(0, jlo0, jhi0);
  tile_range(1, jlo1, jhi1);
  const bool any0 = jhi0 > jlo0, any1 = jhi1 > jlo1;
  const int JLO = any0 ? (any1 ? min(jlo0, jlo1) : jlo0) : jlo1;
  const int JHI = any0 ? (any1 ? max(jhi0, jhi1) : jhi0) : jhi1;

  WaitCtx wc{abort_flag, p.err, p.wait_limit_ns};
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_kvfull(s), 1);
      mbar_init(bar_kvempty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 128);
      mbar_init(bar_odone(t), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && JHI > JLO) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar_q, 2 * Cfg::kTileBytes);
      for (int t = 0; t < 2; ++t)
        tma_load_4d(sbase + Cfg::kSmemQ + t * Cfg::kTileBytes, &tmQ, bar_q, 0,
                    mblock * 256 + t * 128, h, b);
      bool ok = true;
      for (int j = JLO; j < JHI && ok; ++j) {
        const int idx = j - JLO, s = idx % S, u = idx / S;
        if (u > 0 && !(ok = mbar_wait(bar_kvempty(s), (u - 1) & 1, wc))) break;
        mbar_arrive_expect_tx(bar_kvfull(s), 2 * Cfg::kTileBytes);
        tma_load_4d(sbase + Cfg::kSmemK + s * Cfg::kTileBytes, &tmK, bar_kvfull(s), 0, j * 128, g,
                    b);
        tma_load_4d(sbase + Cfg::kSmemV + s * Cfg::kTileBytes, &tmV, bar_kvfull(s), 0, j * 128, g,
                    b);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (JHI > JLO) {
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
      };
      auto in_range = [&](int t, int j) {
        return t ? (j >= jlo1 && j < jhi1) : (j >= jlo0 && j < jhi0);
      };
      // K-major Q and K rows of d bytes: 8-row groups d * 8 bytes apart, a K
      // step of 32 elements adds 32 bytes.  V is read MN-major (d along N, one
      // swizzle atom wide): 8-key groups d * 8 bytes apart, a K step of 32
      // keys adds 32 * d bytes.
      constexpr uint64_t kDescK = sdesc_const_layout(16, 8 * D, Cfg::kLayout);
      constexpr uint64_t kDescV = sdesc_const_layout(8 * D, 8 * D, Cfg::kLayout);
      const uint32_t idesc_qk = make_idesc_e4m3(128, 128, false, false) | (p.qk_negate << 13);
      const uint32_t idesc_pv = make_idesc_e4m3(128, D, false, true);
      const uint64_t dQ0 = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
      const uint64_t dK0 = sdesc_at(kDescK, sbase + Cfg::kSmemK);
      const uint64_t dV0 = sdesc_at(kDescV, sbase + Cfg::kSmemV);
      auto issue_s = [&](int t, int j) {
        const int s = (j - JLO) % S;
        const uint64_t qa = dQ0 + uint64_t((t * Cfg::kTileBytes) >> 4);
        const uint64_t kb = dK0 + uint64_t((s * Cfg::kTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_ss_f8(tmem + t * 128, qa + uint64_t(kk * 2), kb + uint64_t(kk * 2), idesc_qk,
                      kk > 0 ? 1u : 0u);
          mma_commit(bar_sfull(t));
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int j) {
        const int s = (j - JLO) % S;
        const int jlo_t = t ? jlo1 : jlo0;
        const uint64_t vb = dV0 + uint64_t((s * Cfg::kTileBytes) >> 4);
        const uint32_t acc0 = j > jlo_t ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 128 / 32; ++kk)  // P: 32 keys of e4m3 = 8 tensor-memory columns
            mma_ts_f8(tmem + Cfg::kColO + t * D, tmem + t * 128 + kk * 8,
                      vb + uint64_t((kk * 32 * D) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
          mma_commit(bar_odone(t));
        }
        __syncwarp();
      };
      bool ok = wait_all(bar_q, 0);
      if (ok) ok = wait_all(bar_kvfull(0), 0);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (in_range(t, JLO)) issue_s(t, JLO);
      }
      for (int j = JLO; j < JHI && ok; ++j) {
        const int idx = j - JLO, s = idx % S;
        const int s1 = (idx + 1) % S, u1 = (idx + 1) / S;
        bool next_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (in_range(t, j)) {
            const int jlo_t = t ? jlo1 : jlo0;
            if (!(ok = wait_all(bar_pfull(t), (j - jlo_t) & 1))) break;
            tc_fence_after();
            issue_pv(t, j);
          }
          if (in_range(t, j + 1)) {
            if (!next_ready) {
              if (!(ok = wait_all(bar_kvfull(s1), u1 & 1))) break;
              next_ready = true;
            }
            tc_fence_after();
            issue_s(t, j + 1);
          }
        }
        if (!ok) break;
        if (elect_one()) mma_commit(bar_kvempty(s));
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const int row = mblock * 256 + t * 128 + r;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + Cfg::kColO + t * D;
    int lo_i, hi_i;
    row_key_range(row, Nq, Nk, p.causal, p.wl, p.wr, lo_i, hi_i);
    const float sc = p.scale_log2;
    float m_use = -INFINITY;
    float l = 0.f;
    const int my_jlo = t ? jlo1 : jlo0;
    const int n = (t ? jhi1 : jhi0) - my_jlo;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const int j = my_jlo + jj;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(t), jj & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr0[32], sr1[32], sr2[32], sr3[32];
      tmem_ld32(tS + 0, sr0);
      tmem_ld32(tS + 32, sr1);
      tmem_ld32(tS + 64, sr2);
      tmem_ld32(tS + 96, sr3);
      tmem_wait_ld();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        sv[c] = __uint_as_float(sr0[c]);
        sv[32 + c] = __uint_as_float(sr1[c]);
        sv[64 + c] = __uint_as_float(sr2[c]);
        sv[96 + c] = __uint_as_float(sr3[c]);
      }
      const int key0 = j * 128;
      const bool need_mask = (lo_i > key0) || (hi_i < key0 + 127);
      if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          sv[c] = (key0 + c >= lo_i && key0 + c <= hi_i) ? sv[c] : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmax3(sv[e], sv[e + 8], sv[e + 16]);
#pragma unroll
      for (int c = 24; c < 120; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], sv[c + e], sv[c + 8 + e]);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], sv[120 + e]);
      const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                             fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
      const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sc;
      const float m_new = fmaxf(m_use, m_tile);
      const bool grow = m_new > m_use + Cfg::kLazy || (m_use == -INFINITY && m_new != -INFINITY);
      float alpha = 1.f;
      if (grow) {
        alpha = (m_use == -INFINITY) ? 0.f : fast_exp2(m_use - m_new);
        m_use = m_new;
        l *= alpha;
      }
      // P' = 2^6 exp2(s * scale - m) <= 2^8, rounded to e4m3 four to a word
      const float base = (m_use == -INFINITY) ? 0.f : m_use - Cfg::kPShift;
      const float2 sc2 = make_float2(sc, sc);
      const float2 nb2 = make_float2(-base, -base);
      float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {  // keys 4c .. 4c + 3
        float2 pv[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int cc = 2 * c + hh;  // key pair
          const float2 x = __ffma2_rn(make_float2(sv[2 * cc], sv[2 * cc + 1]), sc2, nb2);
          if ((cc & 7) < Cfg::kEmuPairsPer8) {
            pv[hh] = exp2_fma_pair<true>(x);
          } else {
            pv[hh] = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          }
          lsum[cc & 3] = __fadd2_rn(lsum[cc & 3], pv[hh]);
        }
        pk[c] = pack4_e4m3(pv[0].x, pv[0].y, pv[1].x, pv[1].y);
      }
      // P goes over the first 32 columns of S (already read) once P V_{j-1},
      // the last reader of P, is done; awaited on its own barrier, since the
      // completion of S(j), issued after it, does not imply it
      if (jj > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (jj - 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st32(tS, pk);
      const float2 ls2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
      l += ls2.x + ls2.y;
      if (jj > 0 && __any_sync(0xffffffffu, grow)) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (jj - 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(tO + c0, orr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(tO + c0, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pfull(t));
    }
    // epilogue: O = descale_v * acc / l in bf16, LSE = ln 2 (m + log2 l - 6)
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (n - 1) & 1, wc));
    if (ok) {
      tc_fence_after();
      const bool has = (n > 0) && (l > 0.f);
      const float mul = has ? p.out_scale / l : 0.f;
      const float lse = has ? (m_use + __log2f(l) - Cfg::kPShift) * 0.69314718055994531f : -INFINITY;
      const bool store = row < Nq;
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + b * p.o_sb + int64_t(row) * p.o_ss +
                       int64_t(h) * p.o_sh;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t orr[32];
        if (n > 0) {
          tmem_ld32(tO + c0, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = 0u;
        }
        uint32_t pkd[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pkd[c] = pack2<true>(__uint_as_float(orr[2 * c]) * mul,
                               __uint_as_float(orr[2 * c + 1]) * mul);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_uint4(pkd[4 * q4], pkd[4 * q4 + 1], pkd[4 * q4 + 2], pkd[4 * q4 + 3]);
        }
      }
      if (store) p.lse[(int64_t(b) * p.Hq + h) * p.Nq + row] = lse;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
