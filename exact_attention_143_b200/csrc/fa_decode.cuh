// fa_decode.cuh -- sm_100a attention of a few new queries against a paged KV
// cache (decode).
//
// The keys and values of sequence b are the first cache_seqlens[b] rows of a
// cache made of fixed-size pages: key j sits in row j % P of page
// block_table[b][j / P], and a page is laid out [P, Hkv, d]
// ("optimizing-attention-flash", the list of advanced features, which names a
// paged KV cache; "FlashAttention V3 原理与…实战指南", section 四 on
// inference: the KV cache kept in pages, 16 tokens per page in its vLLM
// example).  The result is exact attention over those keys, the mask aligned
// bottom-right against the sequence's own length, so the Nq new queries are
// the last Nq positions.
//
// Decode reads every cached key and value once and does little arithmetic per
// byte, so the kernel is bound by HBM; its design goal is to keep enough page
// loads in flight on every SM.
//
// B200 mapping (two CTAs per SM, so two independent load pipelines):
//   grid (split, kv head g, sequence b).  The visible key tiles of a sequence
//   are cut into splits of `tiles_per_split` 64-key tiles, so short batches
//   still fill the 148 SMs; a combine kernel merges the splits.
//   rows: the G query heads of kv head g times the Nq queries (r = h' Nq + i)
//   form the query tile, loaded by one TMA box per 64-column chunk; a chunk
//   holds R rounded up to 8 rows (the rest zero), which keeps shared memory
//   small enough for two CTAs per SM.
//   warp 4   TMA: the query tile once, then a ring of K and V tiles of 64
//            keys, each assembled from 64 / min(P, 64) page boxes issued by as
//            many lanes; a page past the sequence is fetched at an
//            out-of-range page coordinate, which TMA fills with zeros.
//   warp 5   tcgen05 issuer: S = Q K^T (N = 64) into one of two 64-column
//            regions, O += P V with P over S.
//   warps 0-3 softmax: thread r owns row r (tensor-memory lane r); masks,
//            running max / sum with the lazy O rescale.  P(j) is written once
//            P V(j-2), the last reader of its region, is done, and O is
//            rescaled once P V(j-1) is done, each awaited on the barrier
//            committed with that MMA.
//            Thread r < 64 also clears V row r of the tile when its key lies
//            past the cache length: a partly filled page holds whatever the
//            caller left there, and 0 * NaN would poison O.
// Tensor memory (256 columns): S regions at 0 and 64, O at 128.
#pragma once

#include <cuda_fp16.h>

#include "fa_exp2.cuh"
#include "fa_ptx.cuh"

namespace fa {

struct DecodeParams {
  const int* block_table;    // [B, bt_stride] page ids
  const int* cache_seqlens;  // [B] keys held by each sequence
  int64_t bt_stride;
  int B, Nq, Hq, Hkv, G, R;  // R = G * Nq rows per CTA
  int P, num_pages, max_pages;
  int n_splits, tiles_per_split;
  float scale_log2;     // |softmax_scale| * log2(e)
  uint32_t qk_negate;   // 1 if softmax_scale < 0
  int causal, wl, wr;
  // final outputs (written directly when n_splits == 1)
  void* o;
  int64_t o_sb, o_ss, o_sh;
  float* lse;  // [B, Hq, Nq], natural log
  // split partials: O / l in fp32 and the split's log2-sum-exp2 (base 2,
  // scaled units), [B, Hkv, n_splits, R, d] and [B, Hkv, n_splits, R]
  float* part_o;
  float* part_lse2;
  unsigned int* err;
  uint64_t wait_limit_ns;
};

template <int D>
struct DecCfg {
  static constexpr int kKeys = 64;                  // keys per K/V tile
  static constexpr int kKVChunk = kKeys * 128;      // 64 rows x 64 columns, 128-byte swizzled
  static constexpr int kTileBytes = kKeys * D * 2;  // one K or one V tile
  static constexpr int kStages = D == 64 ? 6 : 3;   // K+V ring depth
  static constexpr int kThreads = 192;
  static constexpr int kSmemQ = 1024;               // barriers and the tensor-memory slot below
  static constexpr uint32_t kTmemCols = 256;        // two CTAs share an SM's 512 columns
  static constexpr uint32_t kColO = 128;            // S regions at 0 and 64, O at 128
  // shared memory of a launch whose query tile has r_pad rows per column chunk:
  // Q, then the K ring and the V ring (each 1024-byte aligned), + alignment slack
  __host__ __device__ static constexpr int q_bytes(int r_pad) { return (D / 64) * r_pad * 128; }
  __host__ __device__ static constexpr int k_off(int r_pad) { return (kSmemQ + q_bytes(r_pad) + 1023) / 1024 * 1024; }
  __host__ __device__ static constexpr int v_off(int r_pad) { return k_off(r_pad) + kStages * kTileBytes; }
  __host__ __device__ static constexpr int smem_bytes(int r_pad) { return v_off(r_pad) + kStages * kTileBytes + 1024; }
};

// Visible key range [lo, hi] of query i of a sequence holding Nk keys.
__device__ __forceinline__ void decode_key_range(int i, int Nq, int Nk, int causal, int wl, int wr,
                                                 int& lo, int& hi) {
  const int ip = i + (Nk - Nq);
  const int right = causal ? 0 : wr;
  lo = wl >= 0 ? max(0, ip - wl) : 0;
  hi = right >= 0 ? min(Nk - 1, ip + right) : Nk - 1;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(192, 2)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using Cfg = DecCfg<D>;
  constexpr int S = Cfg::kStages;
  constexpr int KT = Cfg::kKeys;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  // the query tile holds r_pad rows per 64-column chunk (R rounded up to 8);
  // the MMA reads 128 rows from each chunk base, the rows past r_pad landing
  // in this CTA's K/V ring: they only feed output rows that are never stored
  const int r_pad = (p.R + 7) & ~7;
  const int q_chunk = r_pad * 128;
  const int off_k = Cfg::k_off(r_pad), off_v = Cfg::v_off(r_pad);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  const uint32_t bar_q = smem_u32(&bars[0]);
  auto bar_full = [&](int s) { return smem_u32(&bars[1 + s]); };       // K_j, V_j landed
  auto bar_empty = [&](int s) { return smem_u32(&bars[1 + S + s]); };  // S_j and P_j V_j done
  auto bar_sfull = [&](int r) { return smem_u32(&bars[1 + 2 * S + r]); };
  auto bar_pfull = [&](int r) { return smem_u32(&bars[3 + 2 * S + r]); };
  auto bar_odone = [&](int r) { return smem_u32(&bars[5 + 2 * S + r]); };  // P V(j), r = j % 2
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 520);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = int(blockIdx.x);
  const int g = int(blockIdx.y);
  const int b = int(blockIdx.z);
  const int Nq = p.Nq;
  const int Nk = min(max(p.cache_seqlens[b], 0), p.max_pages * p.P);

  // 64-key tiles any row can see ([lo, hi] grows with the query index), and
  // this split's share of them
  int lo0, hi0, lo1, hi1;
  decode_key_range(0, Nq, Nk, p.causal, p.wl, p.wr, lo0, hi0);
  decode_key_range(Nq - 1, Nq, Nk, p.causal, p.wl, p.wr, lo1, hi1);
  int JLO = 0, JHI = 0;
  if (lo0 <= hi1 && Nk > 0) {
    JLO = lo0 / KT;
    JHI = hi1 / KT + 1;
  }
  const int j0 = JLO + split * p.tiles_per_split;
  const int j1 = min(JHI, j0 + p.tiles_per_split);
  const int n = max(0, j1 - j0);

  WaitCtx wc{abort_flag, p.err, p.wait_limit_ns};
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(bar_sfull(r), 1);
      mbar_init(bar_pfull(r), 128);
      mbar_init(bar_odone(r), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // query rows R .. r_pad - 1 of each chunk are zero
  for (int idx = threadIdx.x; idx < (r_pad - p.R) * (D / 8); idx += blockDim.x) {
    const int row = p.R + idx / (D / 8), u = idx % (D / 8);  // 16-byte unit of the row
    *reinterpret_cast<uint4*>(smem + Cfg::kSmemQ + (u / 8) * q_chunk + row * 128 + (u % 8) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
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
    // The whole warp runs the loop.  Lane bx reads the page id of box bx of
    // the tile before the wait for the free stage and then issues that box's
    // copies, so the copies of one tile leave from up to 8 threads.
    if (n > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(bar_q, uint32_t(p.R * 128 * (D / 64)));
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sbase + Cfg::kSmemQ + c * q_chunk, &tmQ, bar_q, c * 64, 0, g * p.G, b);
      }
      const int rows_per_box = min(p.P, KT);
      const int boxes = KT / rows_per_box;  // at most 8 (pages of 8 or more rows)
      const int* bt = p.block_table + int64_t(b) * p.bt_stride;
      const int n_seq_pages = (Nk + p.P - 1) / p.P;
      bool ok = true;
      for (int jj = 0; jj < n && ok; ++jj) {
        const int s = jj % S, u = jj / S;
        const int key0 = (j0 + jj) * KT;
        // a page the sequence does not hold is read at an out-of-range page
        // coordinate: TMA delivers zeros for it
        int my_page = p.num_pages;
        if (lane < boxes) {
          const int pg = (key0 + lane * rows_per_box) / p.P;
          if (pg < n_seq_pages) my_page = bt[pg];
        }
        if (u > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_empty(s), (u - 1) & 1, wc));
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(bar_full(s), 2 * Cfg::kTileBytes);
        __syncwarp();
        if (lane < boxes) {
          const int tok = (key0 + lane * rows_per_box) % p.P;
          const uint32_t row_off = uint32_t(lane * rows_per_box * 128);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sbase + off_k + s * Cfg::kTileBytes + c * Cfg::kKVChunk + row_off, &tmK,
                        bar_full(s), c * 64, g, tok, my_page);
            tma_load_4d(sbase + off_v + s * Cfg::kTileBytes + c * Cfg::kKVChunk + row_off, &tmV,
                        bar_full(s), c * 64, g, tok, my_page);
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // S_j goes to region j % 2 and P_j over it; S_{j+2} is issued after
    // P_j V_j, so two S tiles run ahead of the softmax.
    if (n > 0) {
      auto wait_all = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc));
      };
      constexpr uint64_t kDescK = sdesc_sw128_const(16, 1024);              // K-major tiles
      constexpr uint64_t kDescMN = sdesc_sw128_const(Cfg::kKVChunk, 1024);  // V, MN-major
      const uint32_t idesc_qk = make_idesc_f16(BF16, 128, KT, false, false) | (p.qk_negate << 13);
      const uint32_t idesc_pv = make_idesc_f16(BF16, 128, D, false, true);
      const uint64_t dQ = sdesc_at(kDescK, sbase + Cfg::kSmemQ);
      const uint64_t dK0 = sdesc_at(kDescK, sbase + off_k);
      const uint64_t dV0 = sdesc_at(kDescMN, sbase + off_v);
      auto issue_s = [&](int jj) {
        const int s = jj % S;
        const uint64_t kb = dK0 + uint64_t((s * Cfg::kTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t qo = uint64_t(((kk >> 2) * q_chunk + (kk & 3) * 32) >> 4);
            const uint64_t ko = uint64_t(((kk >> 2) * Cfg::kKVChunk + (kk & 3) * 32) >> 4);
            mma_ss(tmem + (jj & 1) * 64, dQ + qo, kb + ko, idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sfull(jj & 1));
        }
        __syncwarp();
      };
      bool ok = wait_all(bar_q, 0);
      for (int jj = 0; jj < 2 && jj < n && ok; ++jj) {
        if (!(ok = wait_all(bar_full(jj % S), (jj / S) & 1))) break;
        tc_fence_after();
        issue_s(jj);
      }
      for (int jj = 0; jj < n && ok; ++jj) {
        const int s = jj % S;
        if (!(ok = wait_all(bar_pfull(jj & 1), (jj >> 1) & 1))) break;
        tc_fence_after();
        const uint64_t vb = dV0 + uint64_t((s * Cfg::kTileBytes) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk)  // P: 16 keys of 16-bit values = 8 columns
            mma_ts(tmem + Cfg::kColO, tmem + (jj & 1) * 64 + kk * 8,
                   vb + uint64_t((kk * 16 * 128) >> 4), idesc_pv, (kk > 0 || jj > 0) ? 1u : 0u);
          mma_commit(bar_odone(jj & 1));
          mma_commit(bar_empty(s));
        }
        __syncwarp();
        if (jj + 2 < n) {
          if (!(ok = wait_all(bar_full((jj + 2) % S), ((jj + 2) / S) & 1))) break;
          tc_fence_after();
          issue_s(jj + 2);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = threadIdx.x;  // row == tensor-memory lane (warps 0-3)
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const bool warp_has_rows = warp * 32 < p.R;
    const bool valid = r < p.R;
    const int hl = valid ? r / Nq : 0;  // head within the group
    const int i = valid ? r % Nq : 0;   // query
    const int h = g * p.G + hl;
    int lo_i = 1, hi_i = 0;
    if (valid) decode_key_range(i, Nq, Nk, p.causal, p.wl, p.wr, lo_i, hi_i);
    const float sc = p.scale_log2;
    float m_use = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const int s = jj % S;
      const int key0 = (j0 + jj) * KT;
      const uint32_t tS = tmem + lane_base + (jj & 1) * 64;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(jj & 1), (jj >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      // V row r of this tile holds key key0 + r: clear it when that key is past
      // the cache length (the S MMA has completed, so the tile has landed)
      if (r < KT && key0 + r >= Nk) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint4* vrow = reinterpret_cast<uint4*>(smem + off_v + s * Cfg::kTileBytes +
                                                 c * Cfg::kKVChunk + r * 128);
#pragma unroll
          for (int u = 0; u < 8; ++u) vrow[u] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      float alpha = 1.f;
      bool grow = false;
      if (warp_has_rows) {
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
        const bool need_mask = (lo_i > key0) || (hi_i < key0 + KT - 1);
        if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            sv[c] = (key0 + c >= lo_i && key0 + c <= hi_i) ? sv[c] : -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = sv[e];
#pragma unroll
        for (int c = 8; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * sc;
        const float m_new = fmaxf(m_use, m_tile);
        grow = m_new > m_use + 8.0f || (m_use == -INFINITY && m_new != -INFINITY);
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
          const float2 pv = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          lsum[c & 3] = __fadd2_rn(lsum[c & 3], pv);
          pk[c] = pack2<BF16>(pv.x, pv.y);
        }
        // P(j) goes over S(j) (already read) once P V(j-2), the last reader of
        // this region's P, is done
        if (jj >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_odone(jj & 1), ((jj >> 1) + 1) & 1, wc));
          if (!ok) break;
          tc_fence_after();
        }
        tmem_st32(tS, pk);
        const float2 ls2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
        l += ls2.x + ls2.y;
      }
      if (jj > 0 && __any_sync(0xffffffffu, grow)) {
        // P_{j-1} V_{j-1} must be in O before it is rescaled
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar_odone((jj - 1) & 1), ((jj - 1) >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tO = tmem + lane_base + Cfg::kColO;
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
    if (ok && warp_has_rows) {
      tc_fence_after();
      const bool has = (n > 0) && (l > 0.f);
      const float inv_l = has ? 1.f / l : 0.f;
      const float lse2 = has ? m_use + __log2f(l) : -INFINITY;
      const uint32_t tO = tmem + lane_base + Cfg::kColO;
      if (p.n_splits == 1) {
        uint16_t* orow = valid ? reinterpret_cast<uint16_t*>(p.o) + int64_t(b) * p.o_sb +
                                     int64_t(i) * p.o_ss + int64_t(h) * p.o_sh
                               : nullptr;
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
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              dst[q4] = make_uint4(pkd[4 * q4], pkd[4 * q4 + 1], pkd[4 * q4 + 2], pkd[4 * q4 + 3]);
          }
        }
        if (valid)
          p.lse[(int64_t(b) * p.Hq + h) * Nq + i] =
              has ? lse2 * 0.69314718055994531f : -INFINITY;
      } else {
        // tensor-memory loads are warp-collective: every lane loads, valid
        // rows store
        const int64_t prow = ((int64_t(b) * p.Hkv + g) * p.n_splits + split) * p.R + r;
        if (valid) p.part_lse2[prow] = lse2;
        float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
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
          if (valid) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[c0 / 4 + q4] = make_float4(__uint_as_float(orr[4 * q4]) * inv_l,
                                             __uint_as_float(orr[4 * q4 + 1]) * inv_l,
                                             __uint_as_float(orr[4 * q4 + 2]) * inv_l,
                                             __uint_as_float(orr[4 * q4 + 3]) * inv_l);
          }
        }
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

// Merge of the splits of one output row (b, h, i): one warp per row, lanes
// over the head dimension.  With L_s the base-2 log-sum-exp2 of split s and
// O_s its normalised output, O = sum_s 2^(L_s - L) O_s with L = log2 sum_s
// 2^L_s; LSE = L ln 2.  Splits that saw no key (L_s = -inf) do not count.
template <int D, bool BF16>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(const DecodeParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * 4 + warp;  // (b, h, i)
  const int64_t n_rows = int64_t(p.B) * p.Hq * p.Nq;
  if (row >= n_rows) return;
  const int i = int(row % p.Nq);
  const int h = int((row / p.Nq) % p.Hq);
  const int b = int(row / (int64_t(p.Nq) * p.Hq));
  const int g = h / p.G, hl = h % p.G;
  const int r = hl * p.Nq + i;
  const int64_t base = (int64_t(b) * p.Hkv + g) * p.n_splits;
  float m = -INFINITY;
  for (int s = lane; s < p.n_splits; s += 32) m = fmaxf(m, p.part_lse2[(base + s) * p.R + r]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  constexpr int kPer = D / 32;  // columns per lane
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < p.n_splits; ++s) {
      const float ls = p.part_lse2[(base + s) * p.R + r];
      if (ls == -INFINITY) continue;
      const float w = exp2f(ls - m);
      wsum += w;
      const float* src = p.part_o + ((base + s) * p.R + r) * D + lane * kPer;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] += w * src[e];
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + int64_t(b) * p.o_sb + int64_t(i) * p.o_ss +
                   int64_t(h) * p.o_sh + lane * kPer;
#pragma unroll
  for (int e = 0; e < kPer; e += 2) {
    const uint32_t v = pack2<BF16>(acc[e] * inv, acc[e + 1] * inv);
    *reinterpret_cast<uint32_t*>(orow + e) = v;
  }
  if (lane == 0)
    p.lse[(int64_t(b) * p.Hq + h) * p.Nq + i] =
        wsum > 0.f ? (m + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace fa
