// fa_bwd256.cuh -- sm_100a backward main kernel for head_dim 256.
//
// Same mathematics as fa_bwd.cuh (recomputation from the forward's LSE, the
// textbook gradient: dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
// dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q), for the head
// dimension up to which the pages list FlashAttention's support ("Что такое
// FlashAttention…", section "Версии, оборудование и первоисточники": head
// dimensions up to 256).  The prep and dQ-convert launches of fa_bwd_aux.cuh
// are shared.
//
// At d = 256 the d = 128 layout does not fit an SM: dK and dV alone would fill
// the 512 tensor-memory columns, and K, V, two Q stages and dO of 128 rows
// need 320 KB of shared memory.  So:
//   - each CTA owns one 128-key tile and one half (128 columns) of d: it
//     accumulates dK and dV for its half in tensor memory and adds dQ for its
//     half into the fp32 accumulator; the grid has a CTA per half;
//   - S^T = K Q^T and dP^T = V dO^T still contract over all of d, so K and V
//     are resident whole (128 KB) and both CTAs of a key tile compute them;
//   - a step covers 32 queries, so Q and dO (16 KB each) are double-buffered;
//   - dQ of a step leaves as dQ^T = K_half^T dS^T (M = 128 columns of d,
//     N = 32 queries), since an MMA needs M >= 64.
// Shared memory: K, V 64 KB each; Q, dO 2 x 16 KB each; dS^T 16 KB (128 key
// rows of 128 bytes, 32 queries used); dQ staging 16 KB; LSE2 and D 2 x 128 B.
// Tensor memory: dK [0,128), dV [128,256); per step parity st: S^T then P^T
// and dS^T at 256 + 32 st, dP^T at 320 + 32 st, dQ^T at 384 + 32 st.
//
// Roles (384 threads): warps 0-3 compute P^T and dS^T (thread = key row =
// tensor-memory lane); warps 4-7 read dQ^T (thread = column of d) and stage
// it; warp 8 issues TMA loads; warp 9 issues S^T and dP^T; warp 10 issues
// dV, dK and dQ^T; warp 11 adds each staged dQ block into the accumulator
// with bulk tensor reduce-adds.
#pragma once

#include <climits>

#include "fa_bwd.cuh"

namespace fa {

struct Bwd256Cfg {
  static constexpr int D = 256;
  static constexpr int kQ = 32;                  // queries per step
  static constexpr int kKChunk = 128 * 128;      // 128 rows x 64 columns, 16-bit, swizzled
  static constexpr int kQChunk = kQ * 128;       // 32 rows x 64 columns
  static constexpr int kKBytes = 4 * kKChunk;    // a 128 x 256 tile
  static constexpr int kQBytes = 4 * kQChunk;    // a 32 x 256 tile
  static constexpr int kThreads = 384;
  static constexpr int kSmemK = 0;
  static constexpr int kSmemV = kSmemK + kKBytes;
  static constexpr int kSmemQ = kSmemV + kKBytes;         // 2 stages
  static constexpr int kSmemDO = kSmemQ + 2 * kQBytes;    // 2 stages
  static constexpr int kSmemDS = kSmemDO + 2 * kQBytes;   // dS^T: 128 rows x 128 B
  static constexpr int kSmemSTG = kSmemDS + 128 * 128;    // 4 blocks of 32 queries x 32 fp32
  static constexpr int kSmemLSE = kSmemSTG + 4 * kQ * 128;  // 2 stages x 32 fp32
  static constexpr int kSmemDv = kSmemLSE + 2 * 128;        // 2 stages x 32 fp32
  static constexpr int kSmemBar = kSmemDv + 2 * 128;
  static constexpr int kSmemBytes = kSmemBar + 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColDK = 0, kColDV = 128, kColS = 256, kColDP = 320, kColDQ = 384;
  static constexpr int kEmuPairsPer8 = 2;  // of every 8 query pairs, FMA-pipe exp2
};
static_assert(Bwd256Cfg::kSmemBytes <= 227 * 1024, "shared memory of one CTA");

template <bool BF16>
__global__ void __launch_bounds__(384, 1)
    fa_bwd256_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using Cfg = Bwd256Cfg;
  constexpr int QN = Cfg::kQ;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.err, kDevErrTimeout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kSmemBar);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const uint32_t bar_kv = bar(0);
  auto bar_qfull = [&](int st) { return bar(1 + st); };     // Q, LSE2, D of a step landed
  auto bar_qempty = [&](int st) { return bar(3 + st); };    // S^T and dK read Q (2 commits)
  auto bar_dofull = [&](int st) { return bar(5 + st); };
  auto bar_doempty = [&](int st) { return bar(7 + st); };   // dP^T and dV read dO (2 commits)
  auto bar_sfull = [&](int st) { return bar(9 + st); };     // S^T in tensor memory
  auto bar_dpfull = [&](int st) { return bar(11 + st); };   // dP^T in tensor memory
  auto bar_pready = [&](int st) { return bar(13 + st); };   // P^T written (128 arrivals)
  auto bar_dsready = [&](int st) { return bar(15 + st); };  // dS^T written (128 arrivals)
  auto bar_sfree = [&](int st) { return bar(17 + st); };    // dV and dK read P^T / dS^T
  auto bar_dpread = [&](int st) { return bar(19 + st); };   // dP^T read out (128 arrivals)
  auto bar_dqfull = [&](int st) { return bar(21 + st); };   // dQ^T done (dS^T smem read)
  auto bar_dqfree = [&](int st) { return bar(23 + st); };   // dQ^T read out (128 arrivals)
  const uint32_t bar_staged = bar(25);                      // a dQ block staged (128)
  const uint32_t bar_roundfree = bar(26);                   // staging read by the TMA unit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kSmemBar + 224);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kSmemBar + 232);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work unit: (batch, kv head) from blockIdx.x, key tile from blockIdx.y (the
  // first key tiles see the most queries under a causal mask), half of d from
  // blockIdx.z
  const int bg = blockIdx.x;
  const int g = bg % p.Hkv;
  const int b = bg / p.Hkv;
  const int ntile = int(blockIdx.y);
  const int half = int(blockIdx.z);
  const int G = p.Hq / p.Hkv;
  const int key0 = ntile * 128;
  int Nq, Nk, qstart, kstart;
  seq_rows(p.cu_q, b, p.total_q, p.Nq, Nq, qstart);
  seq_rows(p.cu_k, b, p.total_k, p.Nk, Nk, kstart);
  const int bc = p.cu_q ? 0 : b;
  if (key0 >= Nk) return;  // no key of this sequence here (CTA-uniform)

  // query rows that can see some key of this tile (bounds are monotone in the row)
  const int off = Nk - Nq;
  const int right = p.causal ? 0 : p.wr;
  const int key1 = min(key0 + 127, Nk - 1);
  const int i_min = right >= 0 ? max(0, key0 - off - right) : 0;
  const int i_max = p.wl >= 0 ? min(Nq - 1, key1 - off + p.wl) : Nq - 1;
  const int mlo = i_min / QN;
  const int nm = (i_min <= i_max) ? (i_max / QN - mlo + 1) : 0;
  const int T = nm * G;  // steps: (query head, 32-query block)

  WaitCtx wc{abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar_qfull(st), 1);
      mbar_init(bar_qempty(st), 2);
      mbar_init(bar_dofull(st), 1);
      mbar_init(bar_doempty(st), 2);
      mbar_init(bar_sfull(st), 1);
      mbar_init(bar_dpfull(st), 1);
      mbar_init(bar_pready(st), 128);
      mbar_init(bar_dsready(st), 128);
      mbar_init(bar_sfree(st), 1);
      mbar_init(bar_dpread(st), 128);
      mbar_init(bar_dqfull(st), 1);
      mbar_init(bar_dqfree(st), 128);
    }
    mbar_init(bar_staged, 128);
    mbar_init(bar_roundfree, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  __syncwarp();
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto step_head = [&](int s) { return g * G + s / nm; };
  auto step_mblk = [&](int s) { return mlo + s % nm; };
  auto wait_all = [&](uint32_t bb, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bb, parity, wc));
  };

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && T > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar_kv, 2 * Cfg::kKBytes);
      for (int c = 0; c < 4; ++c) {
        tma_load_4d(sbase + Cfg::kSmemK + c * Cfg::kKChunk, &tmK, bar_kv, c * 64, kstart + key0, g,
                    bc);
        tma_load_4d(sbase + Cfg::kSmemV + c * Cfg::kKChunk, &tmV, bar_kv, c * 64, kstart + key0, g,
                    bc);
      }
      for (int s = 0; s < T; ++s) {
        const int st = s & 1, u = s >> 1;
        const int h = step_head(s), m = step_mblk(s);
        if (u > 0 && !mbar_wait(bar_qempty(st), (u - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(bar_qfull(st), Cfg::kQBytes + 256);
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sbase + Cfg::kSmemQ + st * Cfg::kQBytes + c * Cfg::kQChunk, &tmQ,
                      bar_qfull(st), c * 64, qstart + m * QN, h, bc);
        const int64_t rowoff = (int64_t(b) * p.Hq + h) * p.Nq_pad + int64_t(m) * QN;
        bulk_load_1d(sbase + Cfg::kSmemLSE + st * 128, p.lse2 + rowoff, 128, bar_qfull(st));
        bulk_load_1d(sbase + Cfg::kSmemDv + st * 128, p.Dvec + rowoff, 128, bar_qfull(st));
        if (u > 0 && !mbar_wait(bar_doempty(st), (u - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(bar_dofull(st), Cfg::kQBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sbase + Cfg::kSmemDO + st * Cfg::kQBytes + c * Cfg::kQChunk, &tmDO,
                      bar_dofull(st), c * 64, qstart + m * QN, h, bc);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // Each runs its loop as a converged warp; one elected lane issues a batch
    // of MMAs and its commits (a commit covers that thread's earlier MMAs).
    if (T > 0) {
      constexpr uint64_t kDescK = sdesc_sw128_const(16, 1024);              // K-major tiles
      constexpr uint64_t kDescMNq = sdesc_sw128_const(Cfg::kQChunk, 1024);  // Q, dO as MN-major
      constexpr uint64_t kDescMNk = sdesc_sw128_const(Cfg::kKChunk, 1024);  // K^T (d-major)
      constexpr uint64_t kDescDS = sdesc_sw128_const(16, 1024);             // dS^T, one chunk
      bool ok = wait_all(bar_kv, 0);
      if (warp == 9) {
        // S^T(s) = K Q_s^T and dP^T(s) = V dO_s^T: M = 128 keys, N = 32
        // queries, contracted over all 256 columns of d (16 K steps)
        const uint32_t idesc_s = make_idesc_f16(BF16, 128, QN, false, false);
        const uint64_t dK_k = sdesc_at(kDescK, sbase + Cfg::kSmemK);
        const uint64_t dV_k = sdesc_at(kDescK, sbase + Cfg::kSmemV);
        const uint64_t dQ_k = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
        const uint64_t dDO_k = sdesc_at(kDescK, sbase + Cfg::kSmemDO);
        for (int s = 0; s < T && ok; ++s) {
          const int st = s & 1, u = s >> 1;
          const uint64_t qoff = uint64_t((st * Cfg::kQBytes) >> 4);
          // S^T(s) into its region once dV and dK of step s - 2 have read it
          if (!(ok = wait_all(bar_qfull(st), u & 1))) break;
          if (u > 0 && !(ok = wait_all(bar_sfree(st), (u - 1) & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
              const uint64_t oa = uint64_t(((kk >> 2) * Cfg::kKChunk + (kk & 3) * 32) >> 4);
              const uint64_t ob = uint64_t(((kk >> 2) * Cfg::kQChunk + (kk & 3) * 32) >> 4);
              mma_ss(tmem + Cfg::kColS + 32 * st, dK_k + oa, dQ_k + qoff + ob, idesc_s,
                     kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_sfull(st));
            mma_commit(bar_qempty(st));
          }
          __syncwarp();
          // dP^T(s) once the compute warps have read dP^T(s - 2) out
          if (!(ok = wait_all(bar_dofull(st), u & 1))) break;
          if (u > 0 && !(ok = wait_all(bar_dpread(st), (u - 1) & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
              const uint64_t oa = uint64_t(((kk >> 2) * Cfg::kKChunk + (kk & 3) * 32) >> 4);
              const uint64_t ob = uint64_t(((kk >> 2) * Cfg::kQChunk + (kk & 3) * 32) >> 4);
              mma_ss(tmem + Cfg::kColDP + 32 * st, dV_k + oa, dDO_k + qoff + ob, idesc_s,
                     kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_dpfull(st));
            mma_commit(bar_doempty(st));
          }
          __syncwarp();
        }
      } else {
        // dV += P^T dO_half, dK += dS^T Q_half (M = 128 keys, N = 128
        // columns, K = 32 queries, A from tensor memory), then
        // dQ^T_half = K_half^T dS^T (M = 128 columns, N = 32 queries, K = 128
        // keys, both operands in shared memory)
        const uint32_t idesc_acc = make_idesc_f16(BF16, 128, 128, false, true);
        const uint32_t idesc_dq = make_idesc_f16(BF16, 128, QN, true, true);
        const uint64_t dQ_mn = sdesc_at(kDescMNq, sbase + Cfg::kSmemQ + half * 2 * Cfg::kQChunk);
        const uint64_t dDO_mn = sdesc_at(kDescMNq, sbase + Cfg::kSmemDO + half * 2 * Cfg::kQChunk);
        const uint64_t dKT = sdesc_at(kDescMNk, sbase + Cfg::kSmemK + half * 2 * Cfg::kKChunk);
        const uint64_t dDS = sdesc_at(kDescDS, sbase + Cfg::kSmemDS);
        for (int s = 0; s < T && ok; ++s) {
          const int st = s & 1, u = s >> 1;
          const uint64_t qoff = uint64_t((st * Cfg::kQBytes) >> 4);
          const uint32_t acc0 = s > 0 ? 1u : 0u;
          const uint32_t rS = tmem + Cfg::kColS + 32 * st;
          if (!(ok = wait_all(bar_dofull(st), u & 1))) break;
          if (!(ok = wait_all(bar_pready(st), u & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < QN / 16; ++kk)  // 16 queries = 8 tensor-memory columns
              mma_ts(tmem + Cfg::kColDV, rS + kk * 8, dDO_mn + qoff + uint64_t((kk * 2048) >> 4),
                     idesc_acc, kk > 0 ? 1u : acc0);
            mma_commit(bar_doempty(st));
          }
          __syncwarp();
          if (!(ok = wait_all(bar_qfull(st), u & 1))) break;
          if (!(ok = wait_all(bar_dsready(st), u & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < QN / 16; ++kk)
              mma_ts(tmem + Cfg::kColDK, rS + 16 + kk * 8, dQ_mn + qoff + uint64_t((kk * 2048) >> 4),
                     idesc_acc, kk > 0 ? 1u : acc0);
            mma_commit(bar_qempty(st));
            mma_commit(bar_sfree(st));
          }
          __syncwarp();
          // dQ^T(s) into its region once the readout has taken dQ^T(s - 2)
          if (u > 0 && !(ok = wait_all(bar_dqfree(st), (u - 1) & 1))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys per K step
              mma_ss(tmem + Cfg::kColDQ + 32 * st, dKT + uint64_t((kk * 2048) >> 4),
                     dDS + uint64_t((kk * 2048) >> 4), idesc_dq, kk > 0 ? 1u : 0u);
            mma_commit(bar_dqfull(st));
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------ dQ reduce issuer
    if (T > 0) {
      bool ok = true;
      for (int s = 0; s < T && ok; ++s) {
        const int h = step_head(s), m = step_mblk(s);
        if (!(ok = wait_all(bar_staged, uint32_t(s) & 1u))) break;
        if (elect_one()) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tma_reduce_add_3d(&tmDQ, sbase + Cfg::kSmemSTG + c * (QN * 128), half * 128 + c * 32,
                              m * QN, b * p.Hq + h);
          bulk_commit();
          bulk_wait_read0();
          mbar_arrive(bar_roundfree);
        }
        __syncwarp();
      }
      if (elect_one()) bulk_wait0();  // reduce-adds complete before the CTA exits
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dQ^T readout (warps 4-7)
    // Thread c holds column half * 128 + c of d; the 32 queries of a step go to
    // the staging buffer as four row-major blocks of 32 queries x 32 columns.
    const int c = threadIdx.x - 128;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + Cfg::kSmemSTG) + (c >> 5) * (QN * 32) + (c & 31);
    bool ok = true;
    for (int s = 0; s < T && ok; ++s) {
      const int st = s & 1, u = s >> 1;
      if (!(ok = wait_all(bar_dqfull(st), u & 1))) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + Cfg::kColDQ + 32 * st, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_dqfree(st));
      if (s > 0 && !(ok = wait_all(bar_roundfree, (s - 1) & 1))) break;
#pragma unroll
      for (int q = 0; q < QN; ++q) stage[q * 32] = __uint_as_float(v[q]) * p.scale;
      fence_proxy_async_smem();
      mbar_arrive(bar_staged);
    }
  } else {
    // ------------------------------------------------------------ compute (warps 0-3)
    const int j = threadIdx.x;  // key row == tensor-memory lane
    const int key = key0 + j;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    int qlo = right >= 0 ? key - off - right : INT_MIN;
    int qhi = p.wl >= 0 ? key - off + p.wl : INT_MAX;
    if (key >= Nk) {
      qlo = INT_MAX;
      qhi = INT_MIN;
    }
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    uint8_t* dsrow = smem + Cfg::kSmemDS + j * 128;
    bool ok = true;
    for (int s = 0; s < T; ++s) {
      const int st = s & 1, u = s >> 1;
      const uint32_t rS = tmem + lane_base + Cfg::kColS + 32 * st;
      const float* lse2 = reinterpret_cast<const float*>(smem + Cfg::kSmemLSE + st * 128);
      const float* Dv = reinterpret_cast<const float*>(smem + Cfg::kSmemDv + st * 128);
      const int q0 = step_mblk(s) * QN;
      const bool need_mask = __any_sync(0xffffffffu, qlo > q0 || qhi < q0 + QN - 1);
      if (!(ok = wait_all(bar_sfull(st), u & 1))) break;
      tc_fence_after();
      // P^T = exp2(S^T * scale * log2 e - LSE2) for 32 queries
      uint32_t sr[32];
      tmem_ld32(rS, sr);
      tmem_wait_ld();
      float pf[32];
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < QN; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
        const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                      sc2, make_float2(-l4.x, -l4.y));
        const float2 x23 = __ffma2_rn(
            make_float2(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sc2,
            make_float2(-l4.z, -l4.w));
        const int pair = c / 2;
        float2 p01, p23;
        if ((pair & 7) < Cfg::kEmuPairsPer8)
          p01 = exp2_fma_pair<BF16>(x01);
        else
          p01 = make_float2(fast_exp2(x01.x), fast_exp2(x01.y));
        if (((pair + 1) & 7) < Cfg::kEmuPairsPer8)
          p23 = exp2_fma_pair<BF16>(x23);
        else
          p23 = make_float2(fast_exp2(x23.x), fast_exp2(x23.y));
        pf[c] = p01.x;
        pf[c + 1] = p01.y;
        pf[c + 2] = p23.x;
        pf[c + 3] = p23.y;
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = q0 + c + e;
            pf[c + e] = (q >= qlo && q <= qhi) ? pf[c + e] : 0.f;
          }
        }
        pk[c / 2] = pack2<BF16>(pf[c], pf[c + 1]);
        pk[c / 2 + 1] = pack2<BF16>(pf[c + 2], pf[c + 3]);
      }
      // packed P^T over the S^T columns [0, 16) this thread has already read
      tmem_st16(rS, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pready(st));
      // dS^T = P^T * (dP^T - D), with P rounded to the input dtype as in dV
      if (!(ok = wait_all(bar_dpfull(st), u & 1))) break;
      tc_fence_after();
      uint32_t dp[32];
      tmem_ld32(tmem + lane_base + Cfg::kColDP + 32 * st, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_dpread(st));
      uint32_t dk[16];
#pragma unroll
      for (int c = 0; c < QN; c += 4) {
        const float4 d4 = *reinterpret_cast<const float4*>(Dv + c);
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const uint32_t w = pk[(c + e) / 2];
          if constexpr (BF16) {
            pr[e] = __uint_as_float(w << 16);
            pr[e + 1] = __uint_as_float(w & 0xFFFF0000u);
          } else {
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w));
            pr[e] = a.x;
            pr[e + 1] = a.y;
          }
        }
        const float2 d01 = __fmul2_rn(make_float2(pr[0], pr[1]),
                                      __fadd2_rn(make_float2(__uint_as_float(dp[c]),
                                                             __uint_as_float(dp[c + 1])),
                                                 make_float2(-d4.x, -d4.y)));
        const float2 d23 = __fmul2_rn(make_float2(pr[2], pr[3]),
                                      __fadd2_rn(make_float2(__uint_as_float(dp[c + 2]),
                                                             __uint_as_float(dp[c + 3])),
                                                 make_float2(-d4.z, -d4.w)));
        dk[c / 2] = pack2<BF16>(d01.x, d01.y);
        dk[c / 2 + 1] = pack2<BF16>(d23.x, d23.y);
      }
      tmem_st16(rS + 16, dk);
      // the smem copy is the B operand of dQ^T (MN-major, 128-byte swizzle:
      // the 16-byte unit u of row j sits at unit u ^ (j % 8)); dQ^T(s - 1),
      // its last reader, must be done
      if (s > 0 && !(ok = wait_all(bar_dqfull((s - 1) & 1), ((s - 1) >> 1) & 1))) break;
#pragma unroll
      for (int uu = 0; uu < 4; ++uu)
        *reinterpret_cast<uint4*>(dsrow + ((uu ^ (j & 7)) * 16)) =
            make_uint4(dk[4 * uu], dk[4 * uu + 1], dk[4 * uu + 2], dk[4 * uu + 3]);
      fence_proxy_async_smem();  // generic-proxy smem writes -> visible to the tensor core
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_dsready(st));
    }
    // every MMA of this CTA is done once the last dQ^T is
    if (ok && T > 0) ok = wait_all(bar_dqfull((T - 1) & 1), ((T - 1) >> 1) & 1);
    // epilogue: this CTA's half of dK = scale * (sum of dS^T Q) and of
    // dV = sum of P^T dO for key row j
    if (ok) {
      tc_fence_after();
      const bool store = key < Nk;
      uint16_t* dkrow = static_cast<uint16_t*>(p.dk) + bc * p.dk_sb +
                        int64_t(kstart + key) * p.dk_ss + int64_t(g) * p.dk_sh + half * 128;
      uint16_t* dvrow = static_cast<uint16_t*>(p.dv) + bc * p.dv_sb +
                        int64_t(kstart + key) * p.dv_ss + int64_t(g) * p.dv_sh + half * 128;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? Cfg::kColDK : Cfg::kColDV;
        const float mul = which == 0 ? p.scale : 1.f;
        uint16_t* dst_row = which == 0 ? dkrow : dvrow;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace fa
