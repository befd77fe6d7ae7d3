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
// Tensor memory (512 columns).  d = 128: S_0 [0,128), S_1 [128,256), O_0 and
// O_1 at 256 and 384; P_t is written over S_t and S_t(j+1) follows P_t V_j.
// d = 64: a ring of three 128-column regions [0,384) shared by both tiles, O_0
// and O_1 at 384 and 448.  The (tile, K tile) steps are numbered in issue
// order (K tile j, then tile 0 before tile 1); step k uses region k mod 3,
// where S(k) lands, the softmax writes P(k) over it in place and P(k) V reads
// it.  The softmax therefore never waits for a P V before writing P, and
// S(k+1), S(k+2) are computed while the softmax of step k runs; S(k) only
// waits for P V(k-3), the previous reader of its region.
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
  // 1: a work tile is the same 128 query rows of two query heads of one kv
  // head (query tile t = head 2i + t), which then see the same K tiles; used
  // for GQA groups with short key ranges (mrows is 128)
  int pair;
};

template <int D>
struct FwdCfg {
  static constexpr int kTiles = 2;                  // query tiles of 128 rows per CTA
  static constexpr int kChunk = 128 * 64 * 2;       // one 128-row x 64-column swizzled chunk
  static constexpr int kTileBytes = 128 * D * 2;    // a 128-row tile
  static constexpr int kStages = D == 64 ? 4 : 2;   // K ring and V ring depth
  static constexpr int kThreads = 384;               // 3 warpgroups
  // registers per thread: at launch, and after the split that moves them from
  // the control warpgroup (MMA issue, TMA) to the two softmax warpgroups;
  // 128 * (2 * kRegsSoftmax + kRegsCtl) must equal kThreads * kRegsLaunch
  static constexpr int kRegsLaunch = 168;
  static constexpr int kRegsSoftmax = D == 64 ? 216 : 200;
  static constexpr int kRegsCtl = D == 64 ? 72 : 104;  // d = 128: one warp issues every MMA
  // Q slots of one 128-row tile each, used in turn (work tile i takes slots
  // 2i and 2i + 1 modulo kQSlots) and released as soon as the last Q_t K^T of
  // their tile is done: at d = 128 the third slot lets the next work tile's
  // first Q tile land while both tiles of the current one are in use, and the
  // second follows once the current Q_0 is done
  static constexpr int kQSlots = D == 64 ? 4 : 3;
  static constexpr int kSmemQ = 1024;
  static constexpr int kSmemK = kSmemQ + kQSlots * kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBytes = kSmemV + kStages * kTileBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr bool kRing = D == 64;            // three S/P regions shared by both tiles
  static constexpr int kRegions = kRing ? 3 : 2;    // 128 columns each, from column 0
  static constexpr uint32_t kColO = kRegions * 128; // O_t at kColO + d t
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

// ---------------------------------------------------------------- work tiles
// Cluster launch control (PTX ISA, "clusterlaunchcontrol"): a running CTA asks
// for a CTA of its grid that has not been launched yet; if the request
// succeeds that CTA never starts and the asking CTA computes its tile.  The
// 16-byte response lands in shared memory and completes `bar` (transaction
// bytes).  Once a request has failed, no further request may be made.
__device__ __forceinline__ void clc_try_cancel(uint32_t resp_smem, uint32_t bar) {
  asm volatile(
      "clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 "
      "[%0], [%1];" ::"r"(resp_smem),
      "r"(bar)
      : "memory");
}
// true and the taken CTA's (x, y) block index if the request succeeded
__device__ __forceinline__ bool clc_query(uint32_t resp_smem, int& x, int& y) {
  uint32_t ok, cx = 0u, cy = 0u;
  asm volatile(
      "{\n\t.reg .b128 r;\n\t.reg .pred p;\n\t"
      "ld.shared.b128 r, [%3];\n\t"
      "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "@p clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %1, r;\n\t"
      "@p clusterlaunchcontrol.query_cancel.get_first_ctaid::y.b32.b128 %2, r;\n\t}"
      : "=r"(ok), "+r"(cx), "+r"(cy)
      : "r"(resp_smem)
      : "memory");
  x = int(cx);
  y = int(cy);
  return ok != 0u;
}

// One work tile: up to 256 query rows (two 128-row tiles) of one (batch,
// head), and the K-tile range each of its query tiles can see.
struct FwdTile {
  int b, h, g, mblock;     // batch, query head, kv head, query block
  int Nq, Nk, qstart, kstart, bc;  // this sequence's lengths and first rows
  int jlo0, jhi0, jlo1, jhi1;      // K-tile ranges [jlo_t, jhi_t) (empty if equal)
  int JLO, JHI;                    // their union
  bool rows;                       // the block holds query rows of the sequence
};

// Decode the tile of block index (x, y): (batch, head) from x, query block
// from y with the heaviest (latest, under a causal mask) blocks first.
__device__ __forceinline__ void fwd_tile(const FwdParams& p, int x, int y, FwdTile& w) {
  const int hunits = p.Hq >> p.pair;
  w.h = (x % hunits) << p.pair;
  w.b = x / hunits;
  w.g = w.h / (p.Hq / p.Hkv);
  w.mblock = p.n_mblocks - 1 - y;
  w.Nq = p.Nq;
  w.Nk = p.Nk;
  w.qstart = 0;
  w.kstart = 0;
  w.bc = w.b;
  if (p.cu_q != nullptr) {
    const int q0 = min(max(p.cu_q[w.b], 0), p.total_q), q1 = min(max(p.cu_q[w.b + 1], q0), p.total_q);
    const int k0 = min(max(p.cu_k[w.b], 0), p.total_k), k1 = min(max(p.cu_k[w.b + 1], k0), p.total_k);
    w.Nq = min(q1 - q0, p.Nq);
    w.Nk = min(k1 - k0, p.Nk);
    w.qstart = q0;
    w.kstart = k0;
    w.bc = 0;
  }
  w.rows = w.mblock * p.mrows < w.Nq;
  int lo[2] = {0, 0}, hi[2] = {0, 0};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r0 = w.mblock * p.mrows + (p.pair ? 0 : t * 128);
    if ((p.pair || t * 128 < p.mrows) && r0 < w.Nq) {
      const int r1 = min(r0 + 127, w.Nq - 1);
      int lo0, hi0, lo1, hi1;
      row_key_range(r0, w.Nq, w.Nk, p.causal, p.wl, p.wr, lo0, hi0);
      row_key_range(r1, w.Nq, w.Nk, p.causal, p.wl, p.wr, lo1, hi1);
      if (lo0 <= hi1) {  // both bounds grow with the row
        lo[t] = lo0 / 128;
        hi[t] = hi1 / 128 + 1;
      }
    }
  }
  w.jlo0 = lo[0];
  w.jhi0 = hi[0];
  w.jlo1 = lo[1];
  w.jhi1 = hi[1];
  const bool any0 = w.jhi0 > w.jlo0, any1 = w.jhi1 > w.jlo1;
  w.JLO = any0 ? (any1 ? min(w.jlo0, w.jlo1) : w.jlo0) : w.jlo1;
  w.JHI = any0 ? (any1 ? max(w.jhi0, w.jhi1) : w.jhi0) : w.jhi1;
}

// A decoded tile in a 64-byte shared-memory work queue entry; word 0: 0 = no
// more work, 1 = a tile with query rows, 2 = a tile without.  Entries are
// written before, and read after, an mbarrier hand-off (release / acquire).
constexpr int kTileInts = 16;
__device__ __forceinline__ void put_tile(int* en, const FwdTile& w) {
  int4* v = reinterpret_cast<int4*>(en);
  v[0] = make_int4(w.rows ? 1 : 2, w.b, w.h, w.g);
  v[1] = make_int4(w.mblock, w.Nq, w.Nk, w.qstart);
  v[2] = make_int4(w.kstart, w.bc, w.jlo0, w.jhi0);
  v[3] = make_int4(w.jlo1, w.jhi1, w.JLO, w.JHI);
}
// 1 = a tile (read into w), 0 = no more work
__device__ __forceinline__ int get_tile(const int* en, FwdTile& w) {
  const int4* v = reinterpret_cast<const int4*>(en);
  const int4 a = v[0], b = v[1], c = v[2], d = v[3];
  w.rows = a.x == 1;
  w.b = a.y;
  w.h = a.z;
  w.g = a.w;
  w.mblock = b.x;
  w.Nq = b.y;
  w.Nk = b.z;
  w.qstart = b.w;
  w.kstart = c.x;
  w.bc = c.y;
  w.jlo0 = c.z;
  w.jhi0 = c.w;
  w.jlo1 = d.x;
  w.jhi1 = d.y;
  w.JLO = d.z;
  w.JHI = d.w;
  return a.x == 0 ? 0 : 1;
}

// ---------------------------------------------------------------- kernel
// Persistent over work tiles: each CTA starts with its own block's tile and
// then keeps taking blocks that have not been launched yet (cluster launch
// control), in launch order, so the heaviest tiles still go first and the
// hardware still balances the SMs.  Every ring and barrier phase continues
// from one tile to the next, so the next tile's Q load, K/V loads and first
// Q K^T run while the current tile's last softmax steps and epilogue do.
template <int D, bool BF16, bool DROP = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int S = Cfg::kStages;
  constexpr int NQ = Cfg::kQSlots;
  constexpr bool kRing = Cfg::kRing;
  static_assert(S <= 4 && NQ <= 4, "barrier block layout");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);

  // barrier block at the head of shared memory
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto bar_qfull = [&](int q) { return bar(46 + q); };   // Q slot q landed
  auto bar_qempty = [&](int q) { return bar(50 + q); };  // its tile's Q K^T all done
  auto bar_wfull = [&](int e) { return bar(5 + e); };    // work queue entry e written
  auto bar_wempty = [&](int e) { return bar(7 + e); };   // entry e read by every role
  const uint32_t bar_clc = bar(9);                       // launch-control response
  auto bar_kvfull = [&](int s) { return bar(10 + s); };  // K_j and V_j landed
  auto bar_kempty = [&](int s) { return bar(14 + s); };
  auto bar_vempty = [&](int s) { return bar(18 + s); };
  // d = 128: per query tile
  auto bar_sfull = [&](int t) { return bar(22 + t); };
  auto bar_pfull = [&](int t) { return bar(24 + t); };
  auto bar_odone = [&](int t) { return bar(26 + t); };
  // ring (d = 64): P V of region r done; S_t landed in region r (one barrier
  // per tile and region, so each is awaited by one warpgroup only and its
  // phases stay exact); P_t(i) written / P_t(i) V done, one barrier per tile
  // and parity of the step i, so the softmax can trail the P V it awaits
  auto bar_rfree = [&](int r) { return bar(28 + r); };
  auto bar_rfull = [&](int t, int r) { return bar(31 + 3 * t + r); };
  auto bar_pfull2 = [&](int t, int x) { return bar(37 + 2 * t + x); };
  auto bar_odone2 = [&](int t, int x) { return bar(41 + 2 * t + x); };
  // the TMA producer has reached the last K/V load of the tile it is on: time
  // to ask for the next tile (late enough that SMs which finish first take the
  // tiles left, early enough to hide the request and the next Q load)
  const uint32_t bar_want = bar(45);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);
  const uint32_t clc_resp = sbase + 704;                           // 16-byte aligned
  int* wq = reinterpret_cast<int*>(smem + 768);  // 2 decoded work tiles of 64 bytes

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtx wc{abort_flag, p.err, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int q = 0; q < NQ; ++q) {
      mbar_init(bar_qfull(q), 1);
      mbar_init(bar_qempty(q), 1);
    }
    for (int e = 0; e < 2; ++e) {
      mbar_init(bar_wfull(e), 1);
      mbar_init(bar_wempty(e), 11);  // TMA, S, P V issuer warps and the 8 softmax warps
    }
    mbar_init(bar_clc, 1);
    mbar_init(bar_want, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_kvfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 128);
      mbar_init(bar_odone(t), 1);
      for (int r = 0; r < 3; ++r) mbar_init(bar_rfull(t, r), 1);
      for (int x = 0; x < 2; ++x) {
        mbar_init(bar_pfull2(t, x), 128);
        mbar_init(bar_odone2(t, x), 1);
      }
    }
    for (int r = 0; r < 3; ++r) mbar_init(bar_rfree(r), 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    // work queue entry 0: this block's own tile
    FwdTile w0;
    fwd_tile(p, int(blockIdx.x), int(blockIdx.y), w0);
    put_tile(wq, w0);
    mbar_arrive(bar_wfull(0));
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

  // Read work queue entry `e` (whole warp): 1 = a tile (in w), 0 = no more
  // work, -1 = a wait gave up.  Lane 0 then frees the entry for this warp.
  auto read_work = [&](int e, FwdTile& w) -> int {
    if (!__all_sync(0xffffffffu, mbar_wait(bar_wfull(e & 1), (e >> 1) & 1, wc))) return -1;
    const int st = get_tile(wq + kTileInts * (e & 1), w);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_wempty(e & 1));
    return st;
  };
  auto wait_all = [&](uint32_t b, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(b, parity, wc));
  };

  static_assert(128 * (2 * Cfg::kRegsSoftmax + Cfg::kRegsCtl) == Cfg::kThreads * Cfg::kRegsLaunch,
                "register split must add up to the launch budget");
  if (warp >= 8) {
   // warpgroup 2 hands registers to the softmax warpgroups; the instruction
   // is executed by all four warps before they diverge
   regs_dec<Cfg::kRegsCtl>();
   if (warp == 11) {
    // ------------------------------------------------------------ tile scheduler
    // Entry e is requested once the TMA producer is on the last K/V load of
    // entry e - 1 and every role has read entry e - 2 (whose slot it reuses).
    // The scheduler decodes each tile once for all roles.
    // Its waits sleep between polls: they are off the critical path, and the
    // sub-partition it runs on also runs two softmax warps.
    if (lane == 0) {
      for (int e = 1;; ++e) {
        if (!mbar_wait_sleepy(bar_want, (e - 1) & 1, wc)) break;
        if (e >= 2 && !mbar_wait_sleepy(bar_wempty(e & 1), ((e - 2) >> 1) & 1, wc)) break;
        fence_proxy_async_smem();  // the previous response was read before it is rewritten
        mbar_arrive_expect_tx(bar_clc, 16);
        clc_try_cancel(clc_resp, bar_clc);
        if (!mbar_wait_sleepy(bar_clc, (e - 1) & 1, wc)) break;
        int x = 0, y = 0;
        const bool got = clc_query(clc_resp, x, y);
        int* en = wq + kTileInts * (e & 1);
        if (got) {
          FwdTile w;
          fwd_tile(p, x, y, w);
          put_tile(en, w);
        } else {
          en[0] = 0;
        }
        mbar_arrive(bar_wfull(e & 1));
        if (!got) break;
      }
    }
   } else if (warp == 10) {
    // ------------------------------------------------------------ TMA producer
    // one thread: lane 0 (the other lanes wait at the final barrier)
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int iq = 0, gkv = 0;  // tiles with work so far; K/V tiles loaded so far
      bool ok = true;
      for (int e = 0; ok; ++e) {
        if (!(ok = mbar_wait(bar_wfull(e & 1), (e >> 1) & 1, wc))) break;
        FwdTile w;
        const int st = get_tile(wq + kTileInts * (e & 1), w);
        mbar_arrive(bar_wempty(e & 1));
        if (st == 0) break;
        if (!w.rows || w.JHI <= w.JLO) {
          mbar_arrive(bar_want);
          continue;
        }
        for (int t = 0; t < 2 && ok; ++t) {
          const int sl = (2 * iq + t) % NQ, u = (2 * iq + t) / NQ;
          if (u > 0 && !(ok = mbar_wait(bar_qempty(sl), (u - 1) & 1, wc))) break;
          mbar_arrive_expect_tx(bar_qfull(sl), Cfg::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sbase + Cfg::kSmemQ + sl * Cfg::kTileBytes + c * Cfg::kChunk, &tmQ,
                        bar_qfull(sl), c * 64,
                        w.qstart + w.mblock * p.mrows + (p.pair ? 0 : t * 128), w.h + p.pair * t,
                        w.bc);
        }
        if (!ok) break;
        for (int j = w.JLO; j < w.JHI; ++j, ++gkv) {
          if (j == w.JHI - 1) mbar_arrive(bar_want);
          const int s = gkv % S, u = gkv / S;
          if (u > 0) {  // both readers of the stage are done: Q K^T and P V of K/V tile gkv - S
            ok = mbar_wait(bar_kempty(s), (u - 1) & 1, wc);
            if (ok) ok = mbar_wait(bar_vempty(s), (u - 1) & 1, wc);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(bar_kvfull(s), 2 * Cfg::kTileBytes);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sbase + Cfg::kSmemK + s * Cfg::kTileBytes + c * Cfg::kChunk, &tmK,
                        bar_kvfull(s), c * 64, w.kstart + j * 128, w.g, w.bc);
            tma_load_4d(sbase + Cfg::kSmemV + s * Cfg::kTileBytes + c * Cfg::kChunk, &tmV,
                        bar_kvfull(s), c * 64, w.kstart + j * 128, w.g, w.bc);
          }
        }
        ++iq;
      }
    }
   } else {
    // ------------------------------------------------------------ MMA issuers
    // An MMA issue blocks until the tensor pipe accepts it.  Each issuing warp
    // runs its loop converged and one elected lane issues each batch and its
    // commits (tcgen05.commit covers the MMAs of the committing thread).
    // descriptors are built once; an MMA only adds a compile-time offset
    // (address >> 4) to them
    constexpr uint64_t kDescK = sdesc_sw128_const(16, 1024);            // K-major tiles
    constexpr uint64_t kDescMN = sdesc_sw128_const(Cfg::kChunk, 1024);  // V, MN-major
    const uint32_t idesc_qk = make_idesc_f16(BF16, 128, 128, false, false) | (p.qk_negate << 13);
    const uint32_t idesc_pv = make_idesc_f16(BF16, 128, D, false, true);
    const uint64_t dQ0 = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
    const uint64_t dK0 = sdesc_at(kDescK, sbase + Cfg::kSmemK);
    const uint64_t dV0 = sdesc_at(kDescMN, sbase + Cfg::kSmemV);
    // S = Q K^T of the Q tile in slot sl into tensor-memory column `col`, K/V stage s
    auto issue_s = [&](uint32_t col, int sl, int s, uint32_t done_bar) {
      const uint64_t qa = dQ0 + uint64_t((sl * Cfg::kTileBytes) >> 4);
      const uint64_t kb = dK0 + uint64_t((s * Cfg::kTileBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = uint64_t(((kk >> 2) * Cfg::kChunk + (kk & 3) * 32) >> 4);
          mma_ss(tmem + col, qa + off, kb + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(done_bar);
      }
      __syncwarp();
    };
    // O_t += P V_s with P (16-bit, 128 keys) read from tensor-memory column `pcol`
    auto issue_pv = [&](uint32_t pcol, int t, int s, uint32_t acc0) {
      const uint64_t vb = dV0 + uint64_t((s * Cfg::kTileBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)  // 16 keys = 8 tensor-memory columns per step
          mma_ts(tmem + Cfg::kColO + t * D, tmem + pcol + kk * 8,
                 vb + uint64_t((kk * 16 * 128) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
      }
    };
    bool ok = true;
    // Q slots of work tile iq: each query tile's slot is awaited before its
    // first Q K^T and released after its last (at once if it has none)
    auto q_slot = [&](int iq, int t) { return (2 * iq + t) % NQ; };
    auto q_wait = [&](int iq, int t) {
      return wait_all(bar_qfull(q_slot(iq, t)), ((2 * iq + t) / NQ) & 1);
    };
    auto q_release = [&](int iq, int t) {
      if (elect_one()) mma_commit(bar_qempty(q_slot(iq, t)));
      __syncwarp();
    };
    if constexpr (!kRing) {
      // d = 128, warp 8: P_t overlays S_t, so one warp issues everything and
      // S_t(j+1) follows P_t V_j in the in-order tensor pipe without waiting
      // for it.  Warp 9 only reads the work queue along.
      if (warp == 9) {
        for (int e = 0;; ++e) {
          FwdTile w;
          if (read_work(e, w) <= 0) break;
        }
      } else {
        int iq = 0, gkv = 0, gs0 = 0, gs1 = 0;  // tiles, K/V tiles, P V steps per query tile
        for (int e = 0; ok; ++e) {
          FwdTile w;
          if (read_work(e, w) <= 0) break;
          if (!w.rows || w.JHI <= w.JLO) continue;
          auto in_range = [&](int t, int j) {
            return t ? (j >= w.jlo1 && j < w.jhi1) : (j >= w.jlo0 && j < w.jhi0);
          };
          const int jhi[2] = {w.jhi0, w.jhi1};
          bool qready[2] = {false, false};
          for (int t = 0; t < 2 && ok; ++t)  // a query tile with no K tile: its slot at once
            if (jhi[t] <= (t ? w.jlo1 : w.jlo0)) {
              if (!(ok = q_wait(iq, t))) break;
              q_release(iq, t);
            }
          if (!ok) break;
          if (!(ok = wait_all(bar_kvfull(gkv % S), (gkv / S) & 1))) break;
          tc_fence_after();
          for (int t = 0; t < 2 && ok; ++t)
            if (in_range(t, w.JLO)) {
              if (!(ok = q_wait(iq, t))) break;
              qready[t] = true;
              tc_fence_after();
              issue_s(t * 128, q_slot(iq, t), gkv % S, bar_sfull(t));
              if (w.JLO == jhi[t] - 1) q_release(iq, t);
            }
          if (!ok) break;
          for (int j = w.JLO; j < w.JHI && ok; ++j, ++gkv) {
            const int s = gkv % S, s1 = (gkv + 1) % S, u1 = (gkv + 1) / S;
            bool next_ready = false;
            for (int t = 0; t < 2 && ok; ++t) {
              if (in_range(t, j)) {
                int& gs = t ? gs1 : gs0;
                if (!(ok = wait_all(bar_pfull(t), gs & 1))) break;
                ++gs;
                tc_fence_after();
                issue_pv(t * 128, t, s, j > (t ? w.jlo1 : w.jlo0) ? 1u : 0u);
                if (elect_one()) mma_commit(bar_odone(t));
                __syncwarp();
              }
              if (in_range(t, j + 1)) {
                if (!next_ready) {
                  if (!(ok = wait_all(bar_kvfull(s1), u1 & 1))) break;
                  next_ready = true;
                }
                if (!qready[t]) {
                  if (!(ok = q_wait(iq, t))) break;
                  qready[t] = true;
                }
                tc_fence_after();
                issue_s(t * 128, q_slot(iq, t), s1, bar_sfull(t));
                if (j + 1 == jhi[t] - 1) q_release(iq, t);
              }
            }
            if (!ok) break;
            if (elect_one()) {
              mma_commit(bar_kempty(s));
              mma_commit(bar_vempty(s));
            }
            __syncwarp();
          }
          if (!ok) break;
          ++iq;
        }
      }
    } else if (warp == 8) {
      // d = 64, S issuer: S(k) = Q_t K_j^T into region k mod 3 once P V(k - 3),
      // the previous reader of that region, is done.  k counts the steps of
      // all tiles of this CTA in issue order (K tile j, tile 0 before tile 1).
      int iq = 0, gkv = 0, r = 0, ur = 0;  // ur: earlier uses of region r
      for (int e = 0; ok; ++e) {
        FwdTile w;
        if (read_work(e, w) <= 0) break;
        if (!w.rows || w.JHI <= w.JLO) continue;
        // both Q tiles before the first Q K^T; both slots released once the
        // tile's Q K^T are all issued (at d = 64 the four slots double-buffer
        // whole work tiles)
        for (int t = 0; t < 2 && ok; ++t) ok = q_wait(iq, t);
        if (!ok) break;
        for (int j = w.JLO; j < w.JHI && ok; ++j, ++gkv) {
          const int s = gkv % S, u = gkv / S;
          bool kv_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (!(t ? (j >= w.jlo1 && j < w.jhi1) : (j >= w.jlo0 && j < w.jhi0))) continue;
            if (ur > 0 && !(ok = wait_all(bar_rfree(r), (ur - 1) & 1))) break;
            if (!kv_ready) {
              kv_ready = true;
              if (!(ok = wait_all(bar_kvfull(s), u & 1))) break;
            }
            tc_fence_after();
            issue_s(r * 128, q_slot(iq, t), s, bar_rfull(t, r));
            if (++r == 3) {
              r = 0;
              ++ur;
            }
          }
          if (!ok) break;
          if (elect_one()) mma_commit(bar_kempty(s));  // K_j: both S_t(j) issued
          __syncwarp();
        }
        if (!ok) break;
        q_release(iq, 0);
        q_release(iq, 1);
        ++iq;
      }
    } else {
      // d = 64, P V issuer: O_t += P(k) V_j with P(k) read from region k mod 3;
      // the commits free the region for S(k + 3) and tell the softmax that
      // O_t holds step i of tile t
      int gkv = 0, r = 0, gs0 = 0, gs1 = 0;
      for (int e = 0; ok; ++e) {
        FwdTile w;
        if (read_work(e, w) <= 0) break;
        if (!w.rows || w.JHI <= w.JLO) continue;
        for (int j = w.JLO; j < w.JHI && ok; ++j, ++gkv) {
          const int s = gkv % S, u = gkv / S;
          bool kv_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            const int jlo_t = t ? w.jlo1 : w.jlo0;
            if (!(j >= jlo_t && j < (t ? w.jhi1 : w.jhi0))) continue;
            if (!kv_ready) {
              kv_ready = true;
              if (!(ok = wait_all(bar_kvfull(s), u & 1))) break;
            }
            int& gs = t ? gs1 : gs0;
            if (!(ok = wait_all(bar_pfull2(t, gs & 1), (gs >> 1) & 1))) break;
            tc_fence_after();
            issue_pv(r * 128, t, s, j > jlo_t ? 1u : 0u);
            if (elect_one()) {
              mma_commit(bar_rfree(r));
              mma_commit(bar_odone2(t, gs & 1));
            }
            __syncwarp();
            ++gs;
            if (++r == 3) r = 0;
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
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_base + Cfg::kColO + t * D;
    const float sc = p.scale_log2;
    int gs = 0;              // steps of this query tile in all tiles so far
    int kbase = 0;           // ring: steps of both query tiles in all tiles so far
    uint32_t ring_par = 0u;  // ring: bit r is the parity of this tile's next wait on region r
    bool ok = true;
    for (int e = 0; ok; ++e) {
      FwdTile w;
      if (read_work(e, w) <= 0) break;
      if (!w.rows) continue;
      const int b = w.b, h = w.h + p.pair * t;
      const int row = w.mblock * p.mrows + (p.pair ? 0 : t * 128) + r;
      int lo_i, hi_i;
      row_key_range(row, w.Nq, w.Nk, p.causal, p.wl, p.wr, lo_i, hi_i);
      float m_use = -INFINITY;  // running max in scaled log2 units (reference for O and l)
      float l = 0.f;
      const int my_jlo = t ? w.jlo1 : w.jlo0;
      const int n = (t ? w.jhi1 : w.jhi0) - my_jlo;
      // ring: the other query tile's steps before step jj of this one are
      // clamp(jj + ring_c, 0, ring_n) (tile 0 issues first at each K tile, so
      // tile 1 counts K tile j)
      const int ring_c = t ? w.jlo1 - w.jlo0 + 1 : w.jlo0 - w.jlo1;
      const int ring_n = t ? w.jhi0 - w.jlo0 : w.jhi1 - w.jlo1;
      for (int jj = 0; jj < n; ++jj, ++gs) {
        const int j = my_jlo + jj;
        // S_t(j) and P_t(j): region t (d = 128), or region k mod 3 of the ring
        // (d = 64), where k = kbase + jj + the other tile's steps before it
        int region = t;
        if constexpr (kRing) region = (kbase + jj + min(max(jj + ring_c, 0), ring_n)) % 3;
        const uint32_t tS = tmem + lane_base + region * 128;
        const uint32_t tP = tS;  // P (16-bit) overlays the S columns already read
        if constexpr (kRing) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(bar_rfull(t, region), (ring_par >> region) & 1u, wc));
          ring_par ^= 1u << region;
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(t), gs & 1, wc));
        }
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
        // row max as a tree of 3-input maxima (no long dependent chain)
        float mx8[8];
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) mx8[e8] = fmax3(s[e8], s[e8 + 8], s[e8 + 16]);
#pragma unroll
        for (int c = 24; c < 120; c += 16)
#pragma unroll
          for (int e8 = 0; e8 < 8; ++e8) mx8[e8] = fmax3(mx8[e8], s[c + e8], s[c + 8 + e8]);
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) mx8[e8] = fmaxf(mx8[e8], s[120 + e8]);
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
            const float2 xv = __ffma2_rn(make_float2(s[2 * cc], s[2 * cc + 1]), sc2, nb2);
            float2 pv;
            if ((cc & 7) < Cfg::kEmuPairsPer8) {
              pv = exp2_fma_pair<BF16>(xv);
            } else {
              pv.x = fast_exp2(xv.x);
              pv.y = fast_exp2(xv.y);
            }
            lsum[cc & 3] = __fadd2_rn(lsum[cc & 3], pv);  // l keeps the undropped sum
            pk[c] = pack2<BF16>(pv.x, pv.y);
            if constexpr (DROP) {  // keys 2c, 2c + 1: bytes 2 (c & 1), + 1 of group c / 2
              const uint32_t kb = keep_bytes(kw4[(c >> 1) & 3], p.drop.T);
              pk[c] &= pair_mask(kb, (c & 1) * 2);
            }
          }
          // d = 128: P_t V of the previous step, the last reader of P_t, must
          // be complete before P_t is rewritten.  It is awaited on its own
          // barrier: the completion of S_t(j), issued after it, does not imply
          // it.  (The first step of a tile follows the epilogue's wait.  The
          // ring's region was last read by P V(k - 3), awaited before S(k).)
          if (!kRing && half == 0 && jj > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (gs - 1) & 1, wc));
            if (!ok) break;
            tc_fence_after();
          }
          tmem_st32(tP + 32 * half, pk);
        }
        if (!ok) break;
        const float2 ls2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
        l += ls2.x + ls2.y;
        // Ring: every step awaits P_t V two steps back (on the barrier of its
        // step parity), and the previous step's P_t V only when O_t is
        // rescaled.  A parity wait is exact while its barrier is at most one
        // phase ahead: each barrier serves every other step, and step i + 2
        // cannot complete before this thread has arrived for it.  The
        // trailing wait also keeps any thread from arriving for step i + 2
        // before all have for step i.
        if constexpr (kRing) {
          if (gs >= 2) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(bar_odone2(t, gs & 1), ((gs - 2) >> 1) & 1, wc));
            if (!ok) break;
          }
        }
        if (jj > 0 && __any_sync(0xffffffffu, grow)) {
          // O_t may be rescaled once the previous step's P_t V has accumulated
          if constexpr (kRing) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(bar_odone2(t, (gs - 1) & 1), ((gs - 1) >> 1) & 1, wc));
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
        if constexpr (kRing)
          mbar_arrive(bar_pfull2(t, gs & 1));
        else
          mbar_arrive(bar_pfull(t));
      }
      if (!ok) break;
      // epilogue: wait for the last P_t V (step gs - 1), then O / l and LSE
      if (n > 0) {
        if constexpr (kRing)
          ok = __all_sync(0xffffffffu,
                          mbar_wait(bar_odone2(t, (gs - 1) & 1), ((gs - 1) >> 1) & 1, wc));
        else
          ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(t), (gs - 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
      }
      const bool has = (n > 0) && (l > 0.f);
      const float inv_l = has ? (DROP ? p.drop.scale : 1.f) / l : 0.f;
      const float lse = has ? (m_use + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      // tile 1 idles at 128 rows unless it holds the second head
      const bool store = row < w.Nq && (p.pair || t * 128 < p.mrows);
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + w.bc * p.o_sb +
                       int64_t(w.qstart + row) * p.o_ss + int64_t(h) * p.o_sh;
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
          p.lse[int64_t(h) * p.total_q + w.qstart + row] = lse;
        else
          p.lse[(int64_t(b) * p.Hq + h) * p.Nq + row] = lse;
      }
      // the next tile's first P V overwrites O_t: the reads above are complete
      // (tcgen05.wait::ld) before this thread's next arrival on a P barrier
      kbase += (w.jhi0 - w.jlo0) + (w.jhi1 - w.jlo1);
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
