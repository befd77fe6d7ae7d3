// fa_fwd.cuh -- sm_100a forward kernel of exact attention.
//
// Computes O = softmax(Q K^T * scale + mask) V and the per-row LSE tile by
// tile with a running max / running sum, so the score matrix never leaves the
// SM ("Что такое FlashAttention…", section "Основной механизм простыми
// словами": blocks of Q, K, V move from HBM into fast on-chip memory,
// attention is computed per block and the output is updated incrementally
// with correct normalisation; matmul -> softmax -> matmul fused in one kernel).
//
// B200 mapping (one CTA = 256 query rows of one (batch, head)):
//   warp 9       TMA producer: Q tiles once, then a ring of K and V tiles
//                (128 keys x d each, 128-byte swizzle) with mbarrier hand-off.
//   warp 8       tcgen05 issuer (one thread): S_t = Q_t K_j^T into tensor
//                memory (fp32), then O_t += P_t V_j with P_t read from tensor
//                memory.  Two query tiles t = 0, 1 alternate so the tensor
//                core works on one tile while the other tile's softmax runs.
//   warps 0-3/4-7 softmax warpgroup of tile 0/1: thread r owns row r of its
//                tile (tensor-memory lane r), so row max and row sum are
//                in-thread; it masks boundary tiles, keeps the running max m
//                and sum l, writes P (16-bit) back over S, rescales O in
//                tensor memory when m grows by more than 2^8 (exact: the
//                final O / l uses the same m), and runs the epilogue
//                (O / l to HBM, LSE = ln 2 * (m + log2 l)).
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 and O_1 at
// 256 and 256 + d.  K/V tiles that no row of a tile can see are skipped whole.
#pragma once

#include "fa_ptx.cuh"

namespace fa {

struct FwdParams {
  void* o;
  float* lse;
  int64_t o_sb, o_ss, o_sh;  // element strides of O: batch, seq, head
  int B, Nq, Nk, Hq, Hkv;
  int n_mblocks;             // ceil(Nq / 256)
  float scale_log2;          // |softmax_scale| * log2(e)
  int causal, wl, wr;        // wl / wr: -1 = unbounded
  uint32_t qk_negate;        // 1 if softmax_scale < 0 (negate A in Q K^T)
  unsigned int* err;
  uint64_t wait_limit_ns;
};

template <int D>
struct FwdCfg {
  static constexpr int kRows = 128;                 // rows per query tile (MMA M)
  static constexpr int kTiles = 2;                  // query tiles per CTA
  static constexpr int kKeys = 128;                 // keys per K/V tile (MMA N of Q K^T)
  static constexpr int kChunk = 128 * 64 * 2;       // one 128-row x 64-column swizzled chunk
  static constexpr int kTileBytes = 128 * D * 2;    // a 128-row tile
  static constexpr int kStages = D == 64 ? 4 : 2;   // K ring and V ring depth
  static constexpr int kThreads = 320;
  static constexpr int kSmemQ = 1024;
  static constexpr int kSmemK = kSmemQ + kTiles * kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBytes = kSmemV + kStages * kTileBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
};

// Visible key range of query row i, [lo, hi] inclusive; empty if lo > hi.
__device__ __forceinline__ void row_key_range(int i, int Nq, int Nk, int causal, int wl, int wr,
                                              int& lo, int& hi) {
  const int ip = i + (Nk - Nq);
  const int right = causal ? 0 : wr;
  lo = wl >= 0 ? max(0, ip - wl) : 0;
  hi = right >= 0 ? min(Nk - 1, ip + right) : Nk - 1;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(320, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  // barrier block at the head of shared memory
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  const uint32_t bar_q = smem_u32(&bars[0]);
  auto bar_kfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bar_vfull = [&](int s) { return smem_u32(&bars[1 + S + s]); };
  auto bar_kempty = [&](int s) { return smem_u32(&bars[1 + 2 * S + s]); };
  auto bar_vempty = [&](int s) { return smem_u32(&bars[1 + 3 * S + s]); };
  auto bar_sfull = [&](int t) { return smem_u32(&bars[1 + 4 * S + t]); };
  auto bar_pfull = [&](int t) { return smem_u32(&bars[3 + 4 * S + t]); };
  auto bar_odone = [&](int t) { return smem_u32(&bars[5 + 4 * S + t]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work unit: (batch, head) from blockIdx.x, heaviest query block first
  const int bh = blockIdx.x;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int mblock = p.n_mblocks - 1 - int(blockIdx.y);

  // K-tile range [jlo_t, jhi_t) of each query tile t (empty when jlo_t == jhi_t)
  auto tile_range = [&](int t, int& lo_j, int& hi_j) {
    const int r0 = mblock * 256 + t * 128;
    lo_j = 0;
    hi_j = 0;
    if (r0 < p.Nq) {
      const int r1 = min(r0 + 127, p.Nq - 1);
      int lo0, hi0, lo1, hi1;
      row_key_range(r0, p.Nq, p.Nk, p.causal, p.wl, p.wr, lo0, hi0);
      row_key_range(r1, p.Nq, p.Nk, p.causal, p.wl, p.wr, lo1, hi1);
      if (lo0 <= hi1) {  // both bounds grow with the row
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
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 128);
      mbar_init(bar_odone(t), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
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
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemQ + t * Cfg::kTileBytes + c * Cfg::kChunk, &tmQ, bar_q,
                      c * 64, mblock * 256 + t * 128, h, b);
      bool ok = true;
      for (int j = JLO; j < JHI && ok; ++j) {
        const int idx = j - JLO, s = idx % S, u = idx / S;
        if (u > 0) ok = mbar_wait(bar_kempty(s), (u - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kfull(s), Cfg::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemK + s * Cfg::kTileBytes + c * Cfg::kChunk, &tmK,
                      bar_kfull(s), c * 64, j * 128, g, b);
        if (u > 0) ok = mbar_wait(bar_vempty(s), (u - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar_vfull(s), Cfg::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemV + s * Cfg::kTileBytes + c * Cfg::kChunk, &tmV,
                      bar_vfull(s), c * 64, j * 128, g, b);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && JHI > JLO) {
      const uint32_t idesc_qk = make_idesc_f16(BF16, 128, 128, false, false) | (p.qk_negate << 13);
      const uint32_t idesc_pv = make_idesc_f16(BF16, 128, D, false, true);
      bool ok = mbar_wait(bar_q, 0, wc);
      auto in_range = [&](int t, int j) {
        return t ? (j >= jlo1 && j < jhi1) : (j >= jlo0 && j < jhi0);
      };
      auto issue_s = [&](int t, int j) -> bool {
        const int idx = j - JLO, s = idx % S, u = idx / S;
        if (!mbar_wait(bar_kfull(s), u & 1, wc)) return false;
        tc_fence_after();
        const uint32_t qa = sbase + Cfg::kSmemQ + t * Cfg::kTileBytes;
        const uint32_t kb = sbase + Cfg::kSmemK + s * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Cfg::kChunk + (kk & 3) * 32;
          mma_ss(tmem + t * 128, make_sdesc_sw128(qa + off, 16, 1024),
                 make_sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull(t));
        return true;
      };
      for (int t = 0; t < 2 && ok; ++t)
        if (in_range(t, JLO)) ok = issue_s(t, JLO);
      for (int j = JLO; j < JHI && ok; ++j) {
        const int idx = j - JLO, s = idx % S, u = idx / S;
        bool v_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (in_range(t, j)) {
            if (!v_ready) {
              ok = mbar_wait(bar_vfull(s), u & 1, wc);
              v_ready = true;
            }
            const int jlo_t = t ? jlo1 : jlo0;
            if (ok) ok = mbar_wait(bar_pfull(t), (j - jlo_t) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            const uint32_t vb = sbase + Cfg::kSmemV + s * Cfg::kTileBytes;
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk) {
              // P_t: 16 keys of 16-bit values = 8 tensor-memory columns per step
              mma_ts(tmem + Cfg::kColO + t * D, tmem + t * 128 + kk * 8,
                     make_sdesc_sw128(vb + kk * 16 * 128, Cfg::kChunk, 1024), idesc_pv,
                     (j > jlo_t || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar_odone(t));
          }
          if (ok && in_range(t, j + 1)) ok = issue_s(t, j + 1);
        }
        if (!ok) break;
        mma_commit(bar_kempty(s));
        mma_commit(bar_vempty(s));
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;          // query tile of this warpgroup
    const int r = threadIdx.x & 127;  // row within the tile == tensor-memory lane
    const int row = mblock * 256 + t * 128 + r;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + Cfg::kColO + t * D;
    int lo_i, hi_i;
    row_key_range(row, p.Nq, p.Nk, p.causal, p.wl, p.wr, lo_i, hi_i);
    const float sc = p.scale_log2;
    float m_use = -INFINITY;  // running max in scaled log2 units (reference for O and l)
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
      float s[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(sr0[c]);
        s[32 + c] = __uint_as_float(sr1[c]);
        s[64 + c] = __uint_as_float(sr2[c]);
        s[96 + c] = __uint_as_float(sr3[c]);
      }
      const int key0 = j * 128;
      const bool need_mask = (lo_i > key0) || (hi_i < key0 + 127);
      if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          s[c] = (key0 + c >= lo_i && key0 + c <= hi_i) ? s[c] : -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
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
      float l0 = 0.f, l1 = 0.f;
      uint32_t pk0[32], pk1[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = fast_exp2(fmaf(s[2 * c], sc, -base));
        const float p1 = fast_exp2(fmaf(s[2 * c + 1], sc, -base));
        const float p2 = fast_exp2(fmaf(s[64 + 2 * c], sc, -base));
        const float p3 = fast_exp2(fmaf(s[64 + 2 * c + 1], sc, -base));
        l0 += p0 + p1;
        l1 += p2 + p3;
        pk0[c] = pack2<BF16>(p0, p1);
        pk1[c] = pack2<BF16>(p2, p3);
      }
      l += l0 + l1;
      tmem_st32(tS + 0, pk0);
      tmem_st32(tS + 32, pk1);
      tmem_wait_st();
      if (jj > 0 && __any_sync(0xffffffffu, grow)) {
        // O_t must hold P_{j-1} V_{j-1} before it is rescaled (S is consumed by
        // now, which keeps register pressure low here)
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
    // epilogue
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (n - 1) & 1, wc));
    if (ok) {
      tc_fence_after();
      const bool has = (n > 0) && (l > 0.f);
      const float inv_l = has ? 1.f / l : 0.f;
      const float lse = has ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const bool store = row < p.Nq;
      using elem_t = uint16_t;
      elem_t* orow = reinterpret_cast<elem_t*>(p.o) + b * p.o_sb + int64_t(row) * p.o_ss +
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
          pkd[c] = pack2<BF16>(__uint_as_float(orr[2 * c]) * inv_l,
                               __uint_as_float(orr[2 * c + 1]) * inv_l);
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

  // teardown: every role is done; release tensor memory
  __syncwarp();  // lanes that skipped a single-thread role rejoin before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
