// fa_fwd.cuh -- sm_100a forward kernel of exact attention.
//
// Computes O = softmax(Q K^T * scale + mask) V and the per-row LSE tile by
// tile with a running max / running sum, so the score matrix never leaves the
// SM ("Что такое FlashAttention…", section "Основной механизм простыми
// словами": blocks of Q, K, V move from HBM into fast on-chip memory,
// attention is computed per block and the output is updated incrementally
// with correct normalisation; matmul -> softmax -> matmul fused in one kernel).
//
// B200 mapping (one CTA = 256 query rows of one (batch, head); 128 rows, tile 1
// idle, for causal problems too small to fill the SMs):
//   warp 10      TMA producer: Q tiles once, then a ring of K and V tiles
//                (128 keys x d each, 128-byte swizzle) with mbarrier hand-off.
//   warps 8, 9   tcgen05 issuers: warp 8 issues S_t = Q_t K_j^T into tensor
//                memory (fp32), warp 9 issues O_t += P_t V_j with P_t read from
//                tensor memory.  Two query tiles t = 0, 1 alternate so the
//                tensor core works on one tile while the other tile's softmax
//                runs.
//   warps 0-3/4-7 softmax warpgroup of tile 0/1: thread r owns row r of its
//                tile (tensor-memory lane r), so row max and row sum are
//                in-thread; it masks boundary tiles, keeps the running max m
//                and sum l, writes P (16-bit) to tensor memory, rescales O in
//                tensor memory when m grows by more than 2^8 (exact: the
//                final O / l uses the same m), and runs the epilogue
//                (O / l to HBM, LSE = ln 2 * (m + log2 l)).
//   warp 11      idle; it completes warpgroup 2, whose registers move to the
//                softmax warpgroups (setmaxnreg) after the prologue.
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 and O_1 at 256
// and 256 + d.  With d = 64 the 128 spare columns hold P_0 and P_1, so
// S_t(j+1) is computed while the softmax of S_t(j) is still running; with
// d = 128 P_t is written over S_t and S_t(j+1) waits for P_t V_j.
// The exponentials are split between the MUFU unit (ex2.approx) and a
// polynomial on the FMA pipe (fit by fit_exp2_poly.py), which keeps the
// special-function unit from bounding the kernel.  K/V tiles that no row of
// a tile can see are skipped whole.
#pragma once

#include "fa_dropout.cuh"
#include "fa_exp2.cuh"
#include "fa_ptx.cuh"

namespace fa {

struct FwdParams {
  void* o;
  float* lse;
  int64_t o_sb, o_ss, o_sh;  // element strides of O: batch, seq, head
  int B, Nq, Nk, Hq, Hkv;
  int n_mblocks;             // ceil(Nq / mrows)
  float scale_log2;          // |softmax_scale| * log2(e)
  int causal, wl, wr;        // wl / wr: -1 = unbounded
  uint32_t qk_negate;        // 1 if softmax_scale < 0 (negate A in Q K^T)
  unsigned int* err;
  uint64_t wait_limit_ns;
  // variable-length packed batches: sequence b owns token rows
  // [cu_q[b], cu_q[b+1]) of q/o and [cu_k[b], cu_k[b+1]) of k/v (nullptr for
  // the dense layout); Nq / Nk then hold the longest sequence lengths and LSE
  // is [Hq, total_q]
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  DropoutParams drop;  // used by the DROP instantiations only
  // query rows per CTA: 256 (two tiles), or 128 (tile 1 idle) where fewer
  // CTAs than SMs would otherwise run
  int mrows;
};

template <int D>
struct FwdCfg {
  static constexpr int kTiles = 2;                  // query tiles of 128 rows per CTA
  static constexpr int kChunk = 128 * 64 * 2;       // one 128-row x 64-column swizzled chunk
  static constexpr int kTileBytes = 128 * D * 2;    // a 128-row tile
  static constexpr int kStages = D == 64 ? 4 : 2;   // K ring and V ring depth
  static constexpr int kThreads = 384;               // 3 warpgroups, warp 11 idle
  // registers per thread: at launch, and after the split that moves them from
  // the control warpgroup (MMA issue, TMA) to the two softmax warpgroups;
  // 128 * (2 * kRegsSoftmax + kRegsCtl) must equal kThreads * kRegsLaunch
  static constexpr int kRegsLaunch = 168;
  static constexpr int kRegsSoftmax = 216;
  static constexpr int kRegsCtl = 72;
  static constexpr int kSmemQ = 1024;
  static constexpr int kSmemK = kSmemQ + kTiles * kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBytes = kSmemV + kStages * kTileBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
  static constexpr bool kSepP = D == 64;            // P in its own tensor-memory region
  static constexpr uint32_t kColP = 384;            // P_t at 384 + 64 t (d = 64 only)
  // of every 8 column pairs of a row, how many take the FMA-pipe exp2
#ifndef FA_FWD_EMU_PAIRS_D64  // tuning overrides (compile-time)
#define FA_FWD_EMU_PAIRS_D64 3
#endif
#ifndef FA_FWD_EMU_PAIRS_D128
#define FA_FWD_EMU_PAIRS_D128 0
#endif
  static constexpr int kEmuPairsPer8 = D == 64 ? FA_FWD_EMU_PAIRS_D64 : FA_FWD_EMU_PAIRS_D128;
};

// Visible key range of query row i, [lo, hi] inclusive; empty if lo > hi.
__device__ __forceinline__ void row_key_range(int i, int Nq, int Nk, int causal, int wl, int wr,
                                              int& lo, int& hi) {
  const int ip = i + (Nk - Nq);
  const int right = causal ? 0 : wr;
  lo = wl >= 0 ? max(0, ip - wl) : 0;
  hi = right >= 0 ? min(Nk - 1, ip + right) : Nk - 1;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D, bool BF16, bool DROP = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int S = Cfg::kStages;
  constexpr bool kSepP = Cfg::kSepP;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  // barrier block at the head of shared memory
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  const uint32_t bar_q = smem_u32(&bars[0]);
  auto bar_kvfull = [&](int s) { return smem_u32(&bars[1 + s]); };  // K_j and V_j landed
  auto bar_kempty = [&](int s) { return smem_u32(&bars[1 + 2 * S + s]); };
  auto bar_vempty = [&](int s) { return smem_u32(&bars[1 + 3 * S + s]); };
  auto bar_sfull = [&](int t) { return smem_u32(&bars[1 + 4 * S + t]); };
  auto bar_pfull = [&](int t) { return smem_u32(&bars[3 + 4 * S + t]); };
  auto bar_odone = [&](int t) { return smem_u32(&bars[5 + 4 * S + t]); };
  auto bar_sfree = [&](int t) { return smem_u32(&bars[7 + 4 * S + t]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work unit: (batch, head) from blockIdx.x, query block from blockIdx.y with
  // the heaviest (latest, under a causal mask) blocks launched first
  const int bh = blockIdx.x;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int mblock = p.n_mblocks - 1 - int(blockIdx.y);
  // this sequence's lengths and first rows (dense: the whole tensor, batch b)
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
  if (mblock * p.mrows >= Nq) return;  // no query row of this sequence here (CTA-uniform)

  // K-tile range [jlo_t, jhi_t) of each query tile t (empty when jlo_t == jhi_t)
  auto tile_range = [&](int t, int& lo_j, int& hi_j) {
    const int r0 = mblock * p.mrows + t * 128;
    lo_j = 0;
    hi_j = 0;
    if (t * 128 < p.mrows && r0 < Nq) {
      const int r1 = min(r0 + 127, Nq - 1);
      int lo0, hi0, lo1, hi1;
      row_key_range(r0, Nq, Nk, p.causal, p.wl, p.wr, lo0, hi0);
      row_key_range(r1, Nq, Nk, p.causal, p.wl, p.wr, lo1, hi1);
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
      mbar_init(bar_kvfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 128);
      mbar_init(bar_odone(t), 1);
      mbar_init(bar_sfree(t), 128);
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

  static_assert(128 * (2 * Cfg::kRegsSoftmax + Cfg::kRegsCtl) == Cfg::kThreads * Cfg::kRegsLaunch,
                "register split must add up to the launch budget");
  if (warp >= 8) {
   // warpgroup 2 (warp 11 idle) hands registers to the softmax warpgroups;
   // the instruction is executed by all four warps before they diverge
   regs_dec<Cfg::kRegsCtl>();
   if (warp == 10) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && JHI > JLO) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar_q, 2 * Cfg::kTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemQ + t * Cfg::kTileBytes + c * Cfg::kChunk, &tmQ, bar_q,
                      c * 64, qstart + mblock * p.mrows + t * 128, h, bc);
      bool ok = true;
      for (int j = JLO; j < JHI && ok; ++j) {
        const int idx = j - JLO, s = idx % S, u = idx / S;
        if (u > 0) {  // both readers of the stage are done: S(j - S) and P V(j - S)
          ok = mbar_wait(bar_kempty(s), (u - 1) & 1, wc);
          if (ok) ok = mbar_wait(bar_vempty(s), (u - 1) & 1, wc);
        }
        if (!ok) break;
        mbar_arrive_expect_tx(bar_kvfull(s), 2 * Cfg::kTileBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(sbase + Cfg::kSmemK + s * Cfg::kTileBytes + c * Cfg::kChunk, &tmK,
                      bar_kvfull(s), c * 64, kstart + j * 128, g, bc);
          tma_load_4d(sbase + Cfg::kSmemV + s * Cfg::kTileBytes + c * Cfg::kChunk, &tmV,
                      bar_kvfull(s), c * 64, kstart + j * 128, g, bc);
        }
      }
    }
  } else if (warp == 8 || warp == 9) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 8 issues S_t = Q_t K^T, warp 9 issues O_t += P_t V.  An MMA issue
    // blocks until the tensor pipe accepts it, so one issuing warp would leave
    // the pipe idle during each of its barrier waits; with two, one warp's
    // waits overlap the other warp's MMAs.  Each warp runs its loop converged
    // and one elected lane issues each batch and its commits (tcgen05.commit
    // covers the MMAs of the committing thread).
    if (JHI > JLO) {
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
      };
      auto in_range = [&](int t, int j) {
        return t ? (j >= jlo1 && j < jhi1) : (j >= jlo0 && j < jhi0);
      };
      // descriptors are built once; an MMA only adds a compile-time offset
      // (address >> 4) to them
      constexpr uint64_t kDescK = sdesc_sw128_const(16, 1024);            // K-major tiles
      constexpr uint64_t kDescMN = sdesc_sw128_const(Cfg::kChunk, 1024);  // V, MN-major
      bool ok = true;
      if constexpr (!kSepP) {
        // P_t overlays S_t (d = 128): one warp issues everything, so S_t(j+1)
        // follows P_t V_j in the in-order tensor pipe without waiting for it
        if (warp == 8) {
          const uint32_t idesc_qk =
              make_idesc_f16(BF16, 128, 128, false, false) | (p.qk_negate << 13);
          const uint32_t idesc_pv = make_idesc_f16(BF16, 128, D, false, true);
          const uint64_t dQ0 = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
          const uint64_t dK0 = sdesc_at(kDescK, sbase + Cfg::kSmemK);
          const uint64_t dV0 = sdesc_at(kDescMN, sbase + Cfg::kSmemV);
          auto issue_s = [&](int t, int j) {
            const int s = (j - JLO) % S;
            const uint64_t qa = dQ0 + uint64_t((t * Cfg::kTileBytes) >> 4);
            const uint64_t kb = dK0 + uint64_t((s * Cfg::kTileBytes) >> 4);
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = uint64_t(((kk >> 2) * Cfg::kChunk + (kk & 3) * 32) >> 4);
                mma_ss(tmem + t * 128, qa + off, kb + off, idesc_qk, kk > 0 ? 1u : 0u);
              }
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
              for (int kk = 0; kk < 128 / 16; ++kk)
                mma_ts(tmem + Cfg::kColO + t * D, tmem + t * 128 + kk * 8,
                       vb + uint64_t((kk * 16 * 128) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
              mma_commit(bar_odone(t));
            }
            __syncwarp();
          };
          ok = wait_all(bar_q, 0);
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
            if (elect_one()) {
              mma_commit(bar_kempty(s));
              mma_commit(bar_vempty(s));
            }
            __syncwarp();
          }
        }
      } else if (warp == 8) {
        const uint32_t idesc_qk =
            make_idesc_f16(BF16, 128, 128, false, false) | (p.qk_negate << 13);
        const uint64_t dQ0 = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
        const uint64_t dK0 = sdesc_at(kDescK, sbase + Cfg::kSmemK);
        ok = wait_all(bar_q, 0);
        for (int j = JLO; j < JHI && ok; ++j) {
          const int idx = j - JLO, s = idx % S, u = idx / S;
          bool kv_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (!in_range(t, j)) continue;
            if (j > (t ? jlo1 : jlo0)) {
              // the softmax must be done with S_t(j-1): read it (separate P) or
              // had P_t(j-1) V consumed (P over S)
              const int prev = j - 1 - (t ? jlo1 : jlo0);
              ok = kSepP ? wait_all(bar_sfree(t), prev & 1) : wait_all(bar_odone(t), prev & 1);
              if (!ok) break;
            }
            if (!kv_ready) {
              ok = wait_all(bar_kvfull(s), u & 1);
              kv_ready = true;
              if (!ok) break;
            }
            tc_fence_after();
            const uint64_t qa = dQ0 + uint64_t((t * Cfg::kTileBytes) >> 4);
            const uint64_t kb = dK0 + uint64_t((s * Cfg::kTileBytes) >> 4);
            const uint32_t dst = tmem + t * 128;
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = uint64_t(((kk >> 2) * Cfg::kChunk + (kk & 3) * 32) >> 4);
                mma_ss(dst, qa + off, kb + off, idesc_qk, kk > 0 ? 1u : 0u);
              }
              mma_commit(bar_sfull(t));
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) mma_commit(bar_kempty(s));  // K_j: both S_t(j) issued
          __syncwarp();
        }
      } else {
        const uint32_t idesc_pv = make_idesc_f16(BF16, 128, D, false, true);
        const uint64_t dV0 = sdesc_at(kDescMN, sbase + Cfg::kSmemV);
        for (int j = JLO; j < JHI && ok; ++j) {
          const int idx = j - JLO, s = idx % S, u = idx / S;
          bool kv_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (!in_range(t, j)) continue;
            const int jlo_t = t ? jlo1 : jlo0;
            if (!kv_ready) {
              ok = wait_all(bar_kvfull(s), u & 1);
              kv_ready = true;
              if (!ok) break;
            }
            if (!(ok = wait_all(bar_pfull(t), (j - jlo_t) & 1))) break;
            tc_fence_after();
            const uint32_t pbase = kSepP ? tmem + Cfg::kColP + t * 64 : tmem + t * 128;
            const uint32_t dst = tmem + Cfg::kColO + t * D;
            const uint64_t vb = dV0 + uint64_t((s * Cfg::kTileBytes) >> 4);
            const uint32_t acc0 = j > jlo_t ? 1u : 0u;
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < 128 / 16; ++kk) {
                // P_t: 16 keys of 16-bit values = 8 tensor-memory columns per step
                mma_ts(dst, pbase + kk * 8, vb + uint64_t((kk * 16 * 128) >> 4), idesc_pv,
                       kk > 0 ? 1u : acc0);
              }
              mma_commit(bar_odone(t));
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) mma_commit(bar_vempty(s));  // V_j: both P_t V_j issued
          __syncwarp();
        }
      }
    }
   }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    regs_inc<Cfg::kRegsSoftmax>();
    const int t = warp >> 2;          // query tile of this warpgroup
    const int r = threadIdx.x & 127;  // row within the tile == tensor-memory lane
    const int row = mblock * p.mrows + t * 128 + r;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tP = kSepP ? tmem + lane_base + Cfg::kColP + t * 64 : tS;
    const uint32_t tO = tmem + lane_base + Cfg::kColO + t * D;
    int lo_i, hi_i;
    row_key_range(row, Nq, Nk, p.causal, p.wl, p.wr, lo_i, hi_i);
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
      if constexpr (kSepP) {  // S_t is in registers: the next S_t may be computed
        tc_fence_before();
        mbar_arrive(bar_sfree(t));
      }
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
      // row max as a tree of 3-input maxima (no long dependent chain)
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmax3(s[e], s[e + 8], s[e + 16]);
#pragma unroll
      for (int c = 24; c < 120; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], s[c + e], s[c + 8 + e]);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], s[120 + e]);
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
      // P = exp2(S * scale * log2 e - m), packed to 16 bit; a fixed share of
      // the column pairs takes the FMA-pipe exp2, the rest the MUFU ex2
      const float base = (m_use == -INFINITY) ? 0.f : m_use;
      const float2 sc2 = make_float2(sc, sc);
      const float2 nb2 = make_float2(-base, -base);
      float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
        uint32_t kw4[4];  // dropout keep bytes of the current 16 keys
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          // with dropout, the keep bytes of keys 64 half + 16 (c / 8) .. + 15
          // (this row's word of four generator outputs) are drawn just before
          // the eight pairs that use them
          if constexpr (DROP) {
            if ((c & 7) == 0)
              dropout_row_words4(p.drop, uint32_t(b * p.Hq + h), row, key0 + 64 * half, c >> 3,
                                 kw4);
          }
          const int cc = 32 * half + c;  // column pair
          const float2 x = __ffma2_rn(make_float2(s[2 * cc], s[2 * cc + 1]), sc2, nb2);
          float2 pv;
          if ((cc & 7) < Cfg::kEmuPairsPer8) {
            pv = exp2_fma_pair<BF16>(x);
          } else {
            pv.x = fast_exp2(x.x);
            pv.y = fast_exp2(x.y);
          }
          lsum[cc & 3] = __fadd2_rn(lsum[cc & 3], pv);  // l keeps the undropped sum
          pk[c] = pack2<BF16>(pv.x, pv.y);
          if constexpr (DROP) {  // keys 2c, 2c + 1: bytes 2 (c & 1), + 1 of group c / 2
            const uint32_t kb = keep_bytes(kw4[(c >> 1) & 3], p.drop.T);
            pk[c] &= pair_mask(kb, (c & 1) * 2);
          }
        }
        // P_t V_{j-1}, the last reader of P_t, must be complete before P_t is
        // rewritten.  It is awaited on its own barrier: the completion of
        // S_t(j), issued after it, does not imply it.
        if (half == 0 && jj > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (jj - 1) & 1, wc));
          if (!ok) break;
          tc_fence_after();
        }
        tmem_st32(tP + 32 * half, pk);
      }
      if (!ok) break;
      const float2 ls2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
      l += ls2.x + ls2.y;
      if (jj > 0 && __any_sync(0xffffffffu, grow)) {
        if constexpr (!kSepP) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (jj - 1) & 1, wc));
          if (!ok) break;
          tc_fence_after();
        }
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
      const float inv_l = has ? (DROP ? p.drop.scale : 1.f) / l : 0.f;
      const float lse = has ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const bool store = row < Nq && t * 128 < p.mrows;  // tile 1 idles at 128 rows
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + bc * p.o_sb + int64_t(qstart + row) * p.o_ss +
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
      if (store) {
        if (p.cu_q != nullptr)
          p.lse[int64_t(h) * p.total_q + qstart + row] = lse;
        else
          p.lse[(int64_t(b) * p.Hq + h) * p.Nq + row] = lse;
      }
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
