// fa_bwd.cuh -- sm_100a backward kernels of exact attention.
//
// The backward recomputes the probabilities from the forward's per-row
// log-sum-exp instead of storing them ("tiling and recomputation",
// "optimizing-attention-flash", Quick start; "Что такое FlashAttention…",
// section "Основной механизм простыми словами": tiling and recomputation).
// With P = exp(scale * Q K^T - LSE) on visible keys, the gradient of
// L = sum(dO * O) is the textbook one:
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three launches (1 and 3 are in fa_bwd_aux.cuh):
//   1. fa_bwd_prep_kernel: D_i = sum_c dO_ic O_ic and LSE2_i = LSE_i * log2(e)
//      (fp32, padded to a multiple of 128 rows), and zeroes the fp32 dQ
//      accumulator.
//   2. fa_bwd_main_kernel: one CTA per (128-key tile, kv head, batch).  K and V
//      stay in shared memory; the CTA loops over every query tile that can see
//      its keys, for every query head of the GQA group, so dK and dV are summed
//      in tensor memory without atomics.  Per step (query tile i, head h):
//        S^T  = K Q_i^T        (tcgen05, A = K, B = Q_i, both from smem)
//        dP^T = V dO_i^T       (A = V, B = dO_i)
//        P^T  = exp2(S^T * scale * log2 e - LSE2)   (compute warps, written
//                                                    back as 16-bit over S^T)
//        dV  += P^T dO_i       (A = P^T from tensor memory)
//        dS^T = P^T * (dP^T - D)                     (to tensor memory and to
//                                                    smem as the dQ operand)
//        dK  += dS^T Q_i       (A = dS^T from tensor memory)
//        dQ_i = dS K           (A = dS from smem, MN-major)
//      and scale * dQ_i is added into the fp32 accumulator with TMA bulk
//      reduce-adds staged through shared memory.
//   3. fa_bwd_dq_convert_kernel: dQ accumulator -> dQ in the input dtype.
//
// Roles (512 threads): warps 0-7 compute (thread = key row = tensor-memory
// lane; warps 0-3 take queries 0-63 of a tile, warps 4-7 queries 64-127),
// warps 8-11 move dQ out of tensor memory into a staging buffer, warp 14
// reduces the staged rows into the fp32 accumulator (TMA bulk reduce-add),
// warp 13 issues TMA loads, and two warps issue MMAs (one elected lane of a
// converged warp each): warp 15 the S^T and dP^T products the compute warps
// wait for, warp 12 the dV, dK and dQ accumulations.  Warpgroup 3 (warps
// 12-15) runs on fewer registers so the dQ warpgroup can hold a whole dQ row.
// dO has one buffer, refilled as soon as dP^T and dV have read it; that frees
// the staging buffer so the compute warps never wait for dQ.
// Tensor memory: two 128-column regions R0/R1 swap roles every step.  The
// region of step s holds S^T(s), then P^T(s) and dS^T(s) packed side by side,
// then dQ(s), then dP^T(s+1); the other holds dP^T(s), then S^T(s+1).  dK sits
// at column 256, dV at 256 + d.  S^T(s+1) is computed as soon as the compute
// warps have read dP^T(s), during the dS phase of step s.
#pragma once

#include <climits>

#include <cuda_fp16.h>

#include "fa_ptx.cuh"
#include "fa_dropout.cuh"
#include "fa_exp2.cuh"

namespace fa {

// Length and first token row of sequence b (dense layout: Nq rows, batch b).
__device__ __forceinline__ void seq_rows(const int* cu, int b, int total, int maxlen, int& len,
                                         int& start) {
  if (cu == nullptr) {
    len = maxlen;
    start = 0;
    return;
  }
  const int a0 = min(max(cu[b], 0), total), a1 = min(max(cu[b + 1], a0), total);
  len = min(a1 - a0, maxlen);
  start = a0;
}

// ------------------------------------------------------------------ kernel 2
struct BwdParams {
  const float* lse2;  // [B, Hq, Nq_pad]
  const float* Dvec;  // [B, Hq, Nq_pad]
  float* dq_acc;      // [B, Hq, Nq, d]
  void* dk;
  void* dv;
  int64_t dk_sb, dk_ss, dk_sh, dv_sb, dv_ss, dv_sh;
  int B, Nq, Nq_pad, Nk, Hq, Hkv;
  int n_ntiles;     // ceil(Nk / 128)
  float scale;      // softmax_scale (signed)
  float scale_log2; // softmax_scale * log2(e) (signed)
  int causal, wl, wr;
  unsigned int* err;
  uint64_t wait_limit_ns;
  // variable-length batches: token offsets [B + 1] of q and k (else nullptr);
  // Nq / Nk then hold the longest sequence lengths
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  DropoutParams drop;  // used by the DROP instantiations only
};

template <int D>
struct BwdCfg {
  static constexpr int kChunk = 128 * 64 * 2;     // 128 rows x 64 columns, 16-bit, swizzled
  static constexpr int kTileBytes = 128 * D * 2;  // a 128-row tile
  static constexpr int kThreads = 512;
  // registers per thread: launched with 65536 / 512 = 128; warpgroup 3 (MMA,
  // TMA, reduce issuer, one idle warp) gives some to warpgroup 2 (dQ readout):
  // 128 * (128 + 128 + kRegsDq + kRegsCtl) must equal 512 * 128
  static constexpr int kRegsLaunch = 128;
  static constexpr int kRegsDq = 160;
  static constexpr int kRegsCtl = 96;
  static constexpr int kSmemK = 0;
  static constexpr int kSmemV = kSmemK + kTileBytes;
  static constexpr int kSmemQ = kSmemV + kTileBytes;        // 2 stages
  static constexpr int kSmemDO = kSmemQ + 2 * kTileBytes;   // 1 stage
  static constexpr int kSmemDS = kSmemDO + kTileBytes;      // 128 keys x 128 queries, 16-bit
  static constexpr int kSmemSTG = kSmemDS + 2 * kChunk;     // dQ staging: 128 rows x 64 fp32
  static constexpr int kSmemLSE = kSmemSTG + 32768;         // 2 stages x 128 fp32
  static constexpr int kSmemDv = kSmemLSE + 2 * 512;        // 2 stages x 128 fp32
  static constexpr int kSmemBar = kSmemDv + 2 * 512;
  static constexpr int kSmemBytes = kSmemBar + 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColDK = 256;
  static constexpr uint32_t kColDV = 256 + D;
  static constexpr int kDqRounds = D / 64;  // 64 dQ columns (2 boxes of 32) per reduce round
  // of every 8 query pairs of a row, how many take the FMA-pipe exp2
  static constexpr int kEmuPairsPer8 = 2;
};

__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <int D, bool BF16, bool DROP = false>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.err, kDevErrTimeout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kSmemBar);
  const uint32_t bar_kv = smem_u32(&bars[0]);
  auto bar_qfull = [&](int st) { return smem_u32(&bars[1 + st]); };   // Q, LSE2, D of a step
  auto bar_qempty = [&](int st) { return smem_u32(&bars[3 + st]); };
  const uint32_t bar_dofull = smem_u32(&bars[5]);     // dO of a step (one buffer)
  const uint32_t bar_doempty = smem_u32(&bars[6]);
  const uint32_t bar_s = smem_u32(&bars[7]);
  const uint32_t bar_dp = smem_u32(&bars[8]);
  const uint32_t bar_p = smem_u32(&bars[9]);
  const uint32_t bar_ds = smem_u32(&bars[10]);
  const uint32_t bar_dq = smem_u32(&bars[11]);
  const uint32_t bar_dqfree = smem_u32(&bars[12]);
  const uint32_t bar_staged = smem_u32(&bars[13]);     // a dQ round staged (128 arrivals)
  const uint32_t bar_roundfree = smem_u32(&bars[14]);  // staged round read by the TMA unit
  const uint32_t bar_dpfree = smem_u32(&bars[15]);     // dP^T read out of tensor memory (256)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kSmemBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kSmemBar + 200);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work unit: (batch, kv head) from blockIdx.x, key tile from blockIdx.y
  // (under a causal mask the first key tiles see the most queries and are
  // launched first)
  const int bg = blockIdx.x;
  const int g = bg % p.Hkv;
  const int b = bg / p.Hkv;
  const int ntile = int(blockIdx.y);
  const int G = p.Hq / p.Hkv;
  const int key0 = ntile * 128;
  // this sequence's lengths and first rows (dense: the whole tensor, batch b)
  int Nq, Nk, qstart, kstart;
  seq_rows(p.cu_q, b, p.total_q, p.Nq, Nq, qstart);
  seq_rows(p.cu_k, b, p.total_k, p.Nk, Nk, kstart);
  const int bc = p.cu_q ? 0 : b;
  if (key0 >= Nk) return;  // no key of this sequence here (CTA-uniform)

  // query rows that can see some key of this tile (bounds are monotone in the row)
  const int off = Nk - Nq;
  const int right = p.causal ? 0 : p.wr;
  const int key1 = min(key0 + 127, Nk - 1);
  int i_min = right >= 0 ? max(0, key0 - off - right) : 0;
  int i_max = p.wl >= 0 ? min(Nq - 1, key1 - off + p.wl) : Nq - 1;
  const int mlo = i_min / 128;
  const int nm = (i_min <= i_max) ? (i_max / 128 - mlo + 1) : 0;
  const int T = nm * G;  // steps: (query head, query tile)

  WaitCtx wc{abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar_qfull(st), 1);
      mbar_init(bar_qempty(st), 1);
    }
    mbar_init(bar_dofull, 1);
    mbar_init(bar_doempty, 2);  // one commit from each MMA issuer
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dqfree, 128);
    mbar_init(bar_staged, 128);
    mbar_init(bar_roundfree, 1);
    mbar_init(bar_dpfree, 256);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  __syncwarp();
  if (warp == 12) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto step_head = [&](int s) { return g * G + s / nm; };
  auto step_mtile = [&](int s) { return mlo + s % nm; };
  auto wait_all = [&](uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
  };
  static_assert(128 * (2 * Cfg::kRegsLaunch + Cfg::kRegsDq + Cfg::kRegsCtl) ==
                    Cfg::kThreads * Cfg::kRegsLaunch,
                "register split must add up to the launch budget");

  if (warp >= 12) {
   // warpgroup 3 hands registers to the dQ warpgroup (same instruction for all 4 warps)
   regs_dec<Cfg::kRegsCtl>();
   if (warp == 13) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && T > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * Cfg::kTileBytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(sbase + Cfg::kSmemK + c * Cfg::kChunk, &tmK, bar_kv, c * 64, kstart + key0, g,
                    bc);
        tma_load_4d(sbase + Cfg::kSmemV + c * Cfg::kChunk, &tmV, bar_kv, c * 64, kstart + key0, g,
                    bc);
      }
      for (int s = 0; s < T; ++s) {
        const int st = s & 1, u = s >> 1;
        const int h = step_head(s), m = step_mtile(s);
        // Q, LSE2 and D: two stages
        if (u > 0 && !mbar_wait(bar_qempty(st), (u - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(bar_qfull(st), Cfg::kTileBytes + 1024);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemQ + st * Cfg::kTileBytes + c * Cfg::kChunk, &tmQ,
                      bar_qfull(st), c * 64, qstart + m * 128, h, bc);
        const int64_t rowoff = (int64_t(b) * p.Hq + h) * p.Nq_pad + int64_t(m) * 128;
        bulk_load_1d(sbase + Cfg::kSmemLSE + st * 512, p.lse2 + rowoff, 512, bar_qfull(st));
        bulk_load_1d(sbase + Cfg::kSmemDv + st * 512, p.Dvec + rowoff, 512, bar_qfull(st));
        // dO: one buffer, refilled once dV(s-1) has read it
        if (s > 0 && !mbar_wait(bar_doempty, (s - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(bar_dofull, Cfg::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemDO + c * Cfg::kChunk, &tmDO, bar_dofull, c * 64,
                      qstart + m * 128, h, bc);
      }
    }
   } else if (warp == 14) {
    // ------------------------------------------------------------ dQ reduce issuer
    // Once a round of dQ rows is staged, one elected lane reduces it into the
    // fp32 accumulator (two bulk tensor reduce-adds of 32 columns x 128 rows)
    // and reports when the TMA unit has read the staging buffer.
    if (T > 0) {
      bool ok = true;
      for (int s = 0; s < T && ok; ++s) {
        const int h = step_head(s), m = step_mtile(s);
        for (int rd = 0; rd < Cfg::kDqRounds && ok; ++rd) {
          if (!(ok = wait_all(bar_staged, uint32_t(s * Cfg::kDqRounds + rd) & 1u))) break;
          if (elect_one()) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_reduce_add_3d(&tmDQ, sbase + Cfg::kSmemSTG + c * (128 * 128), rd * 64 + c * 32,
                                m * 128, b * p.Hq + h);
            bulk_commit();
            bulk_wait_read0();
            mbar_arrive(bar_roundfree);
          }
          __syncwarp();
        }
      }
      if (elect_one()) bulk_wait0();  // reduce-adds complete before the CTA exits
      __syncwarp();
    }
   } else {
    // ------------------------------------------------------------ MMA issuers
    // Two warps issue MMAs, each running its whole loop and waiting as a
    // converged warp while one elected lane issues a batch and its commits:
    //   warp 15: S^T(s) and dP^T(s), the products the compute warps wait for;
    //   warp 12: dV(s), dK(s), dQ(s), the accumulations.
    // A commit tracks only the committing thread's MMAs; dO is read by both
    // warps, so its buffer is released by one commit from each.
    if (T > 0) {
      const uint32_t idesc_ss = make_idesc_f16(BF16, 128, 128, false, false);   // S^T, dP^T
      const uint32_t idesc_acc = make_idesc_f16(BF16, 128, D, false, true);    // dV, dK
      const uint32_t idesc_dq = make_idesc_f16(BF16, 128, D, true, true);      // dQ
      constexpr uint64_t kDescK = sdesc_sw128_const(16, 1024);            // K-major tiles
      constexpr uint64_t kDescMN = sdesc_sw128_const(Cfg::kChunk, 1024);  // MN-major tiles
      bool ok = wait_all(bar_kv, 0);
      if (warp == 15) {
        uint64_t dK_k = sdesc_at(kDescK, sbase + Cfg::kSmemK);
        uint64_t dV_k = sdesc_at(kDescK, sbase + Cfg::kSmemV);
        uint64_t dQ_k0 = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
        uint64_t dDO_k = sdesc_at(kDescK, sbase + Cfg::kSmemDO);
        // on a reduced register budget: hide the bases from the optimiser once
        // per step so base + offset is formed where it is used
        auto opaque_bases = [&]() {
          asm volatile("" : "+l"(dK_k), "+l"(dV_k), "+l"(dQ_k0), "+l"(dDO_k));
        };
        // S^T(s) = K Q_s^T into region r (M = keys, N = queries, K-dim = d)
        auto issue_s = [&](int s, uint32_t r) {
          const uint64_t stoff = uint64_t(((s & 1) * Cfg::kTileBytes) >> 4);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t o = uint64_t(((kk >> 2) * Cfg::kChunk + (kk & 3) * 32) >> 4);
              mma_ss(r, dK_k + o, dQ_k0 + stoff + o, idesc_ss, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_s);
          }
          __syncwarp();
        };
        // dP^T(s) = V dO_s^T into region r; dO is then free as far as this warp goes
        auto issue_dp = [&](uint32_t r) {
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t o = uint64_t(((kk >> 2) * Cfg::kChunk + (kk & 3) * 32) >> 4);
              mma_ss(r, dV_k + o, dDO_k + o, idesc_ss, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_dp);
            mma_commit(bar_doempty);
          }
          __syncwarp();
        };
        if (ok) ok = wait_all(bar_qfull(0), 0);
        if (ok) {
          tc_fence_after();
          issue_s(0, tmem);
          ok = wait_all(bar_dofull, 0);
          if (ok) {
            tc_fence_after();
            issue_dp(tmem + 128);
          }
        }
        for (int s = 0; s + 1 < T && ok; ++s) {
          opaque_bases();
          const uint32_t Ra = tmem + (s & 1) * 128, Rb = tmem + ((s + 1) & 1) * 128;
          // S^T(s+1) into Rb once the compute warps hold dP^T(s) in registers
          if (!(ok = wait_all(bar_dpfree, s & 1))) break;
          if (!(ok = wait_all(bar_qfull((s + 1) & 1), ((s + 1) >> 1) & 1))) break;
          tc_fence_after();
          issue_s(s + 1, Rb);
          // dP^T(s+1) into Ra once dO(s+1) is in (normally long since) and dQ(s)
          // has been read out of Ra (the wait on the critical path comes last)
          if (!(ok = wait_all(bar_dofull, (s + 1) & 1))) break;
          if (!(ok = wait_all(bar_dqfree, s & 1))) break;
          tc_fence_after();
          issue_dp(Ra);
        }
      } else if (warp == 12) {
        uint64_t dK_mn = sdesc_at(kDescMN, sbase + Cfg::kSmemK);
        uint64_t dDS_mn = sdesc_at(kDescMN, sbase + Cfg::kSmemDS);
        uint64_t dQ_mn0 = sdesc_at(kDescMN, sbase + Cfg::kSmemQ);
        uint64_t dDO_mn = sdesc_at(kDescMN, sbase + Cfg::kSmemDO);
        auto opaque_bases = [&]() {
          asm volatile("" : "+l"(dK_mn), "+l"(dDS_mn), "+l"(dQ_mn0), "+l"(dDO_mn));
        };
        // P^T sits in columns [0, 32) (queries 0-63) and [64, 96) (queries
        // 64-127) of its region, dS^T 32 columns further: 16 queries per K
        // step = 8 columns
        auto acol = [](int kk) { return uint32_t(kk < 4 ? kk * 8 : 64 + (kk - 4) * 8); };
        for (int s = 0; s < T && ok; ++s) {
          opaque_bases();
          const int st = s & 1;
          const uint32_t Ra = tmem + (s & 1) * 128;
          const uint64_t stoff = uint64_t((st * Cfg::kTileBytes) >> 4);
          const uint32_t acc0 = s > 0 ? 1u : 0u;
          // dV += P^T dO (A = P^T from tensor memory, B = dO MN-major)
          if (!(ok = wait_all(bar_dofull, s & 1))) break;
          if (!(ok = wait_all(bar_p, s & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + Cfg::kColDV, Ra + acol(kk), dDO_mn + uint64_t((kk * 2048) >> 4),
                     idesc_acc, kk > 0 ? 1u : acc0);
            mma_commit(bar_doempty);
          }
          __syncwarp();
          // dK += dS^T Q (A = dS^T from tensor memory, beside P^T; B = Q MN-major)
          if (!(ok = wait_all(bar_qfull(st), (s >> 1) & 1))) break;
          if (!(ok = wait_all(bar_ds, s & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + Cfg::kColDK, Ra + 32 + acol(kk),
                     dQ_mn0 + stoff + uint64_t((kk * 2048) >> 4), idesc_acc, kk > 0 ? 1u : acc0);
            mma_commit(bar_qempty(st));  // Q_s, LSE_s, D_s are no longer read
          }
          __syncwarp();
          // dQ(s) = dS K into Ra (A = dS from smem, MN-major; B = K MN-major)
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(Ra, dDS_mn + uint64_t((kk * 2048) >> 4), dK_mn + uint64_t((kk * 2048) >> 4),
                     idesc_dq, kk > 0 ? 1u : 0u);
            mma_commit(bar_dq);
          }
          __syncwarp();
        }
      }
    }
   }
  } else if (warp >= 8) {
    regs_inc<Cfg::kRegsDq>();
    // ------------------------------------------------------------ dQ readout (warps 8-11)
    // dQ(s) leaves tensor memory (thread = query row r) 64 columns at a time;
    // scale * dQ is staged, 128-byte swizzled, in the staging buffer for the
    // reduce issuer.  The tensor-memory region is released right after the
    // last load, before the staging of the last round.
    const int r = threadIdx.x - 256;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    uint8_t* stage = smem + Cfg::kSmemSTG;
    constexpr int kR = Cfg::kDqRounds;
    bool ok = true;
    for (int s = 0; s < T && ok; ++s) {
      if (!(ok = wait_all(bar_dq, s & 1))) break;
      tc_fence_after();
      const uint32_t R = tmem + lane_base + (s & 1) * 128;
      // all of dQ(s) into registers, then the region is released at once
      uint32_t v[D];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32)
        tmem_ld32(R + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[c0]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_dqfree);
#pragma unroll
      for (int rd = 0; rd < kR; ++rd) {
        // the previous round's staging must have been read by the TMA unit
        // (no early exit here: the loop must unroll so v stays in registers)
        const int prev = s * kR + rd - 1;
        if (ok && prev >= 0) ok = wait_all(bar_roundfree, prev & 1);
        if (!ok) continue;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint8_t* chunk = stage + c * (128 * 128) + r * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float* x = reinterpret_cast<const float*>(&v[rd * 64 + c * 32 + u * 4]);
            *reinterpret_cast<float4*>(chunk + ((u ^ (r & 7)) * 16)) =
                make_float4(x[0] * p.scale, x[1] * p.scale, x[2] * p.scale, x[3] * p.scale);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_staged);
      }
    }
  } else {
    // ------------------------------------------------------------ compute (warps 0-7)
    const int half = warp >> 2;                 // query half of every tile
    const int j = (warp & 3) * 32 + lane;       // key row == tensor-memory lane
    const int key = key0 + j;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t colS = half * 64;            // S^T / dP^T columns of this half
    const uint32_t colP = half * 64;            // packed P^T / dS^T: [colP, colP + 32)
    // queries that see this key: [qlo, qhi]
    int qlo = right >= 0 ? key - off - right : INT_MIN;
    int qhi = p.wl >= 0 ? key - off + p.wl : INT_MAX;
    if (key >= Nk) {
      qlo = INT_MAX;
      qhi = INT_MIN;
    }
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int s = 0; s < T; ++s) {
      const int st = s & 1;
      const uint32_t Ra = tmem + lane_base + (s & 1) * 128;
      const uint32_t Rb = tmem + lane_base + ((s + 1) & 1) * 128;
      const float* lse2 = reinterpret_cast<const float*>(smem + Cfg::kSmemLSE + st * 512) + half * 64;
      const float* Dv = reinterpret_cast<const float*>(smem + Cfg::kSmemDv + st * 512) + half * 64;
      const int q0 = step_mtile(s) * 128 + half * 64;
      const bool need_mask = __any_sync(0xffffffffu, qlo > q0 || qhi < q0 + 63);
      if (!(ok = wait_all(bar_s, s & 1))) break;
      tc_fence_after();
      // P^T = exp2(S^T * scale * log2 e - LSE2), 32 queries at a time; a share
      // of the query pairs takes the FMA-pipe exp2.  With dropout the dV
      // operand Z^T = P^T o M^T goes to [colP, colP + 32) and the undropped
      // P^T, which dS needs, to [colP + 32, colP + 64) until dS^T replaces it;
      // all of S^T is read first since those columns still hold it.
      uint32_t srall[DROP ? 64 : 1];
      uint32_t kwd[DROP ? 16 : 1];
      if constexpr (DROP) {
        tmem_ld32(Ra + colS, *reinterpret_cast<uint32_t(*)[32]>(&srall[0]));
        tmem_ld32(Ra + colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&srall[32]));
        tmem_wait_ld();
        dropout_col_words(p.drop, uint32_t(b * p.Hq + step_head(s)), key, q0, kwd);
      }
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t sr_own[DROP ? 1 : 32];
        const uint32_t* sr = DROP ? &srall[c0] : sr_own;
        if constexpr (!DROP) {
          tmem_ld32(Ra + colS + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr_own[0]));
          tmem_wait_ld();
        }
        uint32_t pk[16], zk[DROP ? 16 : 1];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c0 + c);
          const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                        sc2, make_float2(-l4.x, -l4.y));
          const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])),
                                        sc2, make_float2(-l4.z, -l4.w));
          const int pair = (c0 + c) / 2;  // query pair index within this half
          float2 p01, p23;
          if ((pair & 7) < Cfg::kEmuPairsPer8) {
            p01 = exp2_fma_pair<BF16>(x01);
          } else {
            p01 = make_float2(fast_exp2(x01.x), fast_exp2(x01.y));
          }
          if (((pair + 1) & 7) < Cfg::kEmuPairsPer8) {
            p23 = exp2_fma_pair<BF16>(x23);
          } else {
            p23 = make_float2(fast_exp2(x23.x), fast_exp2(x23.y));
          }
          float pv[4] = {p01.x, p01.y, p23.x, p23.y};
          if (need_mask) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = q0 + c0 + c + e;
              pv[e] = (q >= qlo && q <= qhi) ? pv[e] : 0.f;
            }
          }
          pk[c / 2] = pack2<BF16>(pv[0], pv[1]);
          pk[c / 2 + 1] = pack2<BF16>(pv[2], pv[3]);
          if constexpr (DROP) {  // queries c0 + c .. + 3 form one group of four
            const uint32_t wd = kwd[(c0 + c) >> 2];
            zk[c / 2] = pack2<BF16>(pv[0] * keep_of(wd, 0, p.drop.T), pv[1] * keep_of(wd, 1, p.drop.T));
            zk[c / 2 + 1] =
                pack2<BF16>(pv[2] * keep_of(wd, 2, p.drop.T), pv[3] * keep_of(wd, 3, p.drop.T));
          }
        }
        if constexpr (DROP) {
          tmem_st16(Ra + colP + c0 / 2, zk);
          tmem_st16(Ra + colP + 32 + c0 / 2, pk);
        } else {
          // packed P^T written over S^T columns this thread has already read
          tmem_st16(Ra + colP + c0 / 2, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p);
      // dS^T = P^T * (dP^T - D), to tensor memory (beside P^T) and to smem (dQ
      // operand); the dQ(s-1) MMA, the last reader of the smem buffer,
      // completed before dP^T(s) was issued.  dP^T(s) is read out first so
      // that S^T(s+1) can be computed into its region during this phase.
      if (!(ok = wait_all(bar_dp, s & 1))) break;
      tc_fence_after();
      uint8_t* dsrow = smem + Cfg::kSmemDS + half * Cfg::kChunk + j * 128;
      uint32_t dpr[DROP ? 32 : 64];
      if constexpr (!DROP) {
        tmem_ld32(Rb + colS, *reinterpret_cast<uint32_t(*)[32]>(&dpr[0]));
        tmem_ld32(Rb + colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&dpr[32]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_dpfree);
      }
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t pr[16], dk[16], zr[DROP ? 16 : 1];
        const uint32_t* dpc = DROP ? dpr : &dpr[c0 % (DROP ? 32 : 64)];
        if constexpr (DROP) {
          // dP^T chunk, Z^T (whose zeros are the dropped pairs) and P^T
          tmem_ld32(Rb + colS + c0, *reinterpret_cast<uint32_t(*)[32]>(&dpr[0]));
          tmem_ld16(Ra + colP + c0 / 2, *reinterpret_cast<uint32_t(*)[16]>(&zr[0]));
          tmem_ld16(Ra + colP + 32 + c0 / 2, pr);
          tmem_wait_ld();
          if (c0 == 32) {  // all of dP^T(s) is in registers
            tc_fence_before();
            mbar_arrive(bar_dpfree);
          }
        } else {
          tmem_ld16(Ra + colP + c0 / 2, pr);
          tmem_wait_ld();
        }
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(Dv + c0 + c);
          const uint32_t pa = pr[c / 2], pb = pr[c / 2 + 1];
          float pf[4];
          if constexpr (BF16) {
            pf[0] = __uint_as_float(pa << 16);
            pf[1] = __uint_as_float(pa & 0xFFFF0000u);
            pf[2] = __uint_as_float(pb << 16);
            pf[3] = __uint_as_float(pb & 0xFFFF0000u);
          } else {
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&pa));
            const float2 bb = __half22float2(*reinterpret_cast<const __half2*>(&pb));
            pf[0] = a.x;
            pf[1] = a.y;
            pf[2] = bb.x;
            pf[3] = bb.y;
          }
          float dq4[4] = {__uint_as_float(dpc[c]), __uint_as_float(dpc[c + 1]),
                          __uint_as_float(dpc[c + 2]), __uint_as_float(dpc[c + 3])};
          if constexpr (DROP) {  // dP through the dropout multiplier
            const uint32_t za = zr[c / 2], zb = zr[c / 2 + 1];
            dq4[0] = (za & 0xFFFFu) ? dq4[0] * p.drop.scale : 0.f;
            dq4[1] = (za >> 16) ? dq4[1] * p.drop.scale : 0.f;
            dq4[2] = (zb & 0xFFFFu) ? dq4[2] * p.drop.scale : 0.f;
            dq4[3] = (zb >> 16) ? dq4[3] * p.drop.scale : 0.f;
          }
          const float2 d01 = __fmul2_rn(make_float2(pf[0], pf[1]),
                                        __fadd2_rn(make_float2(dq4[0], dq4[1]),
                                                   make_float2(-d4.x, -d4.y)));
          const float2 d23 = __fmul2_rn(make_float2(pf[2], pf[3]),
                                        __fadd2_rn(make_float2(dq4[2], dq4[3]),
                                                   make_float2(-d4.z, -d4.w)));
          dk[c / 2] = pack2<BF16>(d01.x, d01.y);
          dk[c / 2 + 1] = pack2<BF16>(d23.x, d23.y);
        }
        // columns of S^T(s) this thread has already read (with dropout: the
        // P^T chunk just loaded)
        tmem_st16(Ra + colP + 32 + c0 / 2, dk);
        // smem copy in the MN-major 128-byte-swizzled layout of the dQ A operand:
        // chunk `half` holds queries [64 half, 64 half + 64) of every key row;
        // the 16-byte unit u of row j sits at unit u ^ (j % 8).
        const int u0 = c0 >> 3;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int u = (u0 + uu) ^ (j & 7);
          *reinterpret_cast<uint4*>(dsrow + u * 16) =
              make_uint4(dk[4 * uu], dk[4 * uu + 1], dk[4 * uu + 2], dk[4 * uu + 3]);
        }
      }
      fence_proxy_async_smem();  // generic-proxy smem writes -> visible to the tensor core
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_ds);
    }
    if (ok && T > 0) ok = wait_all(bar_dq, (T - 1) & 1);  // every MMA of this CTA is done
    // epilogue: dK = scale * (sum of dS^T Q), dV = sum of P^T dO, in the input
    // dtype; this thread writes half of the columns of key row j
    if (ok) {
      tc_fence_after();
      const bool store = key < Nk;
      uint16_t* dkrow = static_cast<uint16_t*>(p.dk) + bc * p.dk_sb +
                        int64_t(kstart + key) * p.dk_ss + int64_t(g) * p.dk_sh + half * (D / 2);
      uint16_t* dvrow = static_cast<uint16_t*>(p.dv) + bc * p.dv_sb +
                        int64_t(kstart + key) * p.dv_ss + int64_t(g) * p.dv_sh + half * (D / 2);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = (which == 0 ? Cfg::kColDK : Cfg::kColDV) + half * (D / 2);
        const float mul = which == 0 ? p.scale : (DROP ? p.drop.scale : 1.f);
        uint16_t* dst_row = which == 0 ? dkrow : dvrow;
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          uint32_t r[32];
          if (T > 0) {
            tmem_ld32(tmem + lane_base + col + c0, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = 0u;
          }
          uint32_t pkd[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pkd[c] = pack2<BF16>(__uint_as_float(r[2 * c]) * mul,
                                 __uint_as_float(r[2 * c + 1]) * mul);
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              dst[q4] = make_uint4(pkd[4 * q4], pkd[4 * q4 + 1], pkd[4 * q4 + 2], pkd[4 * q4 + 3]);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
