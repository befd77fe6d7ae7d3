// fa_fwd256.cuh -- sm_100a forward of exact attention for head_dim 256.
//
// Head dimensions up to 256 are supported by the method; above 192 the
// backward is limited ("Что такое FlashAttention…", section on versions and
// hardware).  This kernel is the forward for d = 256; it computes the same
// O and LSE as the d = 64 / 128 forward.
//
// With d = 256 one 128-row query tile already needs 384 tensor-memory
// columns (S 128 + O 256) and 64 KB of shared memory for Q, so the layout
// differs from the smaller head dims:
//   one query tile of 128 rows per CTA; K and V tiles of 64 keys (32 KB
//   each), two stages of each;
//   warp 4   TMA: Q once (4 column chunks of 64), then the K and V rings;
//   warp 5   tcgen05 issuer: S(j) = Q K_j^T (M 128, N 64, K 256) into one of
//            two 64-column regions, O += P(j) V_j (N 256) with P(j) in one of
//            two regions of its own; S(j+2) is issued right after P V(j), and
//            P never shares columns with an S the pipe may be writing while
//            P V still reads it;
//   warps 0-3 softmax, thread r = row r, and the epilogue.
// Tensor memory: S regions at columns 0 and 64, O at 128..383, P regions at
// 384 and 416.
#pragma once

#include <climits>

#include "fa_exp2.cuh"
#include "fa_fwd.cuh"  // FwdParams, row_key_range, fmax3
#include "fa_ptx.cuh"

namespace fa {

struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int kQChunk = 128 * 64 * 2;  // 128 rows x 64 columns
  static constexpr int kKVChunk = 64 * 64 * 2;  // 64 rows x 64 columns
  static constexpr int kQBytes = 4 * kQChunk;
  static constexpr int kKVBytes = 4 * kKVChunk;  // a 64-key tile
  static constexpr int kStages = 2;
  static constexpr int kThreads = 192;
  static constexpr int kSmemQ = 1024;
  static constexpr int kSmemK = kSmemQ + kQBytes;
  static constexpr int kSmemV = kSmemK + kStages * kKVBytes;
  static constexpr int kSmemBytes = kSmemV + kStages * kKVBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 128;
  static constexpr uint32_t kColP = 384;  // P(j) at 384 + 32 (j % 2)
  static constexpr int kEmuPairsPer8 = 0;
};

template <bool BF16>
__global__ void __launch_bounds__(192, 1)
    fa_fwd256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Cfg = Fwd256Cfg;
  constexpr int D = Cfg::D;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  const uint32_t bar_q = smem_u32(&bars[0]);
  auto bar_kfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bar_kempty = [&](int s) { return smem_u32(&bars[1 + S + s]); };
  auto bar_vfull = [&](int s) { return smem_u32(&bars[1 + 2 * S + s]); };
  auto bar_vempty = [&](int s) { return smem_u32(&bars[1 + 3 * S + s]); };
  auto bar_sfull = [&](int r) { return smem_u32(&bars[1 + 4 * S + r]); };
  auto bar_pfull = [&](int r) { return smem_u32(&bars[3 + 4 * S + r]); };
  // P V(j) done, one barrier per P region (r = j % 2): every wait names the
  // MMA it depends on, so no phase is ever ambiguous and no wait relies on a
  // later commit covering an earlier MMA
  auto bar_odone = [&](int r) { return smem_u32(&bars[5 + 4 * S + r]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int mblock = p.n_mblocks - 1 - int(blockIdx.y);  // heaviest causal blocks first
  int Nq = p.Nq, Nk = p.Nk, qstart = 0, kstart = 0, bc = b;
  if (p.cu_q != nullptr) {
    const int q0 = min(max(p.cu_q[b], 0), p.total_q), q1 = min(max(p.cu_q[b + 1], q0), p.total_q);
    const int k0 = min(max(p.cu_k[b], 0), p.total_k), k1 = min(max(p.cu_k[b + 1], k0), p.total_k);
    Nq = min(q1 - q0, p.Nq);
    Nk = min(k1 - k0, p.Nk);
    qstart = q0;
    kstart = k0;
    bc = 0;
  }
  if (mblock * 128 >= Nq) return;  // no query row of this sequence here (CTA-uniform)

  // 64-key tiles [JLO, JHI) seen by some row of the tile
  int JLO = 0, JHI = 0;
  {
    const int r0 = mblock * 128, r1 = min(r0 + 127, Nq - 1);
    int lo0, hi0, lo1, hi1;
    row_key_range(r0, Nq, Nk, p.causal, p.wl, p.wr, lo0, hi0);
    row_key_range(r1, Nq, Nk, p.causal, p.wl, p.wr, lo1, hi1);
    if (lo0 <= hi1) {
      JLO = lo0 / 64;
      JHI = hi1 / 64 + 1;
    }
  }
  const int n = JHI - JLO;

  WaitCtx wc{abort_flag, p.err, p.wait_limit_ns};
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(bar_sfull(r), 1);
      mbar_init(bar_pfull(r), 128);
      mbar_init(bar_odone(r), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar_q, Cfg::kQBytes);
      for (int c = 0; c < 4; ++c)
        tma_load_4d(sbase + Cfg::kSmemQ + c * Cfg::kQChunk, &tmQ, bar_q, c * 64,
                    qstart + mblock * 128, h, bc);
      bool ok = true;
      // K runs ahead of V: K_j is needed by S(j), V_j only by P V(j)
      for (int jj = 0; jj < n && ok; ++jj) {
        const int s = jj % S, u = jj / S;
        const int key = kstart + (JLO + jj) * 64;
        if (u > 0 && !(ok = mbar_wait(bar_kempty(s), (u - 1) & 1, wc))) break;
        mbar_arrive_expect_tx(bar_kfull(s), Cfg::kKVBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sbase + Cfg::kSmemK + s * Cfg::kKVBytes + c * Cfg::kKVChunk, &tmK,
                      bar_kfull(s), c * 64, key, g, bc);
        if (u > 0 && !(ok = mbar_wait(bar_vempty(s), (u - 1) & 1, wc))) break;
        mbar_arrive_expect_tx(bar_vfull(s), Cfg::kKVBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sbase + Cfg::kSmemV + s * Cfg::kKVBytes + c * Cfg::kKVChunk, &tmV,
                      bar_vfull(s), c * 64, key, g, bc);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (n > 0) {
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
      };
      constexpr uint64_t kDescK = sdesc_sw128_const(16, 1024);                 // Q, K: K-major
      constexpr uint64_t kDescV = sdesc_sw128_const(Cfg::kKVChunk, 1024);       // V: MN-major
      const uint32_t idesc_qk = make_idesc_f16(BF16, 128, 64, false, false) | (p.qk_negate << 13);
      const uint32_t idesc_pv = make_idesc_f16(BF16, 128, D, false, true);
      const uint64_t dQ = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
      const uint64_t dK0 = sdesc_at(kDescK, sbase + Cfg::kSmemK);
      const uint64_t dV0 = sdesc_at(kDescV, sbase + Cfg::kSmemV);
      auto issue_s = [&](int jj) {
        const int s = jj % S;
        const uint64_t kb = dK0 + uint64_t((s * Cfg::kKVBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t qo = uint64_t(((kk >> 2) * Cfg::kQChunk + (kk & 3) * 32) >> 4);
            const uint64_t ko = uint64_t(((kk >> 2) * Cfg::kKVChunk + (kk & 3) * 32) >> 4);
            mma_ss(tmem + (jj & 1) * 64, dQ + qo, kb + ko, idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sfull(jj & 1));
          mma_commit(bar_kempty(s));
        }
        __syncwarp();
      };
      bool ok = wait_all(bar_q, 0);
      for (int jj = 0; jj < 2 && jj < n && ok; ++jj) {
        if (!(ok = wait_all(bar_kfull(jj % S), (jj / S) & 1))) break;
        tc_fence_after();
        issue_s(jj);
      }
      for (int jj = 0; jj < n && ok; ++jj) {
        const int s = jj % S;
        if (!(ok = wait_all(bar_vfull(s), (jj / S) & 1))) break;
        if (!(ok = wait_all(bar_pfull(jj & 1), (jj >> 1) & 1))) break;
        tc_fence_after();
        const uint64_t vb = dV0 + uint64_t((s * Cfg::kKVBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 64 / 16; ++kk)  // P: 16 keys of 16-bit values = 8 columns
            mma_ts(tmem + Cfg::kColO, tmem + Cfg::kColP + (jj & 1) * 32 + kk * 8,
                   vb + uint64_t((kk * 16 * 128) >> 4), idesc_pv, (kk > 0 || jj > 0) ? 1u : 0u);
          mma_commit(bar_odone(jj & 1));
          mma_commit(bar_vempty(s));
        }
        __syncwarp();
        if (jj + 2 < n) {
          if (!(ok = wait_all(bar_kfull((jj + 2) % S), ((jj + 2) / S) & 1))) break;
          tc_fence_after();
          issue_s(jj + 2);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = threadIdx.x;  // row == tensor-memory lane (warps 0-3)
    const int row = mblock * 128 + r;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + Cfg::kColO;
    int lo_i, hi_i;
    row_key_range(row, Nq, Nk, p.causal, p.wl, p.wr, lo_i, hi_i);
    const float sc = p.scale_log2;
    float m_use = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const uint32_t tS = tmem + lane_base + (jj & 1) * 64;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(jj & 1), (jj >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr0[32], sr1[32];
      tmem_ld32(tS + 0, sr0);
      tmem_ld32(tS + 32, sr1);
      tmem_wait_ld();
      float sv[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        sv[c] = __uint_as_float(sr0[c]);
        sv[32 + c] = __uint_as_float(sr1[c]);
      }
      const int key0 = (JLO + jj) * 64;
      const bool need_mask = (lo_i > key0) || (hi_i < key0 + 63);
      if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          sv[c] = (key0 + c >= lo_i && key0 + c <= hi_i) ? sv[c] : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmax3(sv[e], sv[e + 8], sv[e + 16]);
#pragma unroll
      for (int c = 24; c < 56; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], sv[c + e], sv[c + 8 + e]);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], sv[56 + e]);
      const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                             fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
      const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sc;
      const float m_new = fmaxf(m_use, m_tile);
      const bool grow = m_new > m_use + 8.0f || (m_use == -INFINITY && m_new != -INFINITY);
      float alpha = 1.f;
      if (grow) {
        alpha = (m_use == -INFINITY) ? 0.f : fast_exp2(m_use - m_new);
        m_use = m_new;
        l *= alpha;
      }
      const float base = (m_use == -INFINITY) ? 0.f : m_use;
      const float2 sc2 = make_float2(sc, sc);
      const float2 nb2 = make_float2(-base, -base);
      float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {  // key pair
        const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nb2);
        float2 pv;
        if ((c & 7) < Cfg::kEmuPairsPer8) {
          pv = exp2_fma_pair<BF16>(x);
        } else {
          pv = make_float2(fast_exp2(x.x), fast_exp2(x.y));
        }
        lsum[c & 3] = __fadd2_rn(lsum[c & 3], pv);
        pk[c] = pack2<BF16>(pv.x, pv.y);
      }
      // P(j) goes to its own region once P V(j-2), its last reader, is done
      if (jj >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(jj & 1), ((jj >> 1) + 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st32(tmem + lane_base + Cfg::kColP + (jj & 1) * 32, pk);
      const float2 ls2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
      l += ls2.x + ls2.y;
      if (jj > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds P V(j-1) once that MMA is done
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar_odone((jj - 1) & 1), ((jj - 1) >> 1) & 1, wc));
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
      mbar_arrive(bar_pfull(jj & 1));
    }
    // every P V done: the last two, one per region (earlier ones were awaited)
    for (int jl = max(0, n - 2); jl < n && ok; ++jl)
      ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(jl & 1), (jl >> 1) & 1, wc));
    if (ok) {
      tc_fence_after();
      const bool has = (n > 0) && (l > 0.f);
      const float inv_l = has ? 1.f / l : 0.f;
      const float lse = has ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const bool store = row < Nq;
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + bc * p.o_sb +
                       int64_t(qstart + row) * p.o_ss + int64_t(h) * p.o_sh;
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
          pkd[c] = pack2<BF16>(__uint_as_float(orr[2 * c]) * inv_l,
                               __uint_as_float(orr[2 * c + 1]) * inv_l);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_uint4(pkd[4 * q4], pkd[4 * q4 + 1], pkd[4 * q4 + 2], pkd[4 * q4 + 3]);
        }
      }
      if (store) {
        if (p.cu_q != nullptr)
          p.lse[int64_t(h) * p.total_q + qstart + row] = lse;
        else
          p.lse[(int64_t(b) * p.Hq + h) * p.Nq + row] = lse;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
