// fa_dropout.cuh -- dropout keep bits of the attention probabilities.
//
// Dropout multiplies P_ij by (256 / T) M_ij before P V ("optimizing-
// attention-flash", the dropout_p argument of flash_attn_func; "Что такое
// FlashAttention…", versions section: dropout among the features).  The keep
// bit M_ij of element (i, j) of (batch b, query head h) is byte (j mod 4) of
// output word (i mod 4) of Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011) at counter
// (j / 4, i / 4, b Hq + h, offset) with the 64-bit seed as key: kept iff that
// byte is below T = round(256 (1 - p)).  One generator call covers a 4 x 4
// block of (query, key) pairs, so the forward (a thread per query row) and
// the backward (a thread per key row) draw the same bits.
#pragma once

#include <cstdint>

namespace fa {

struct DropoutParams {
  uint32_t T;        // keep threshold, 1..255; 0 = no dropout
  uint32_t seed_lo, seed_hi;
  uint32_t offset;
  float scale;       // 256 / T
};

// Ten rounds of two 32 x 32 -> 64-bit products (multipliers 0xD2511F53,
// 0xCD9E8D57); the key is bumped by the Weyl constants 0x9E3779B9,
// 0xBB67AE85 between rounds.  Each product is formed as separate high and low
// 32-bit halves (mul.hi, mul.lo), which runs about 24% faster on sm_100 than
// one 64-bit wide multiply and gives the same words.
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t y0 = hi1 ^ c1 ^ k0, y2 = hi0 ^ c3 ^ k1;
    c0 = y0;
    c1 = lo1;
    c2 = y2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// 4 x 4 transpose across the four lanes of a group (lanes 4t .. 4t + 3): lane
// q holds r[k] = v(q, k) on entry and v(k, q) on exit.  Two exchange rounds
// (lane distance 1, then 2) with predicated selects: no lane-dependent
// indexing, so no divergent branches.
__device__ __forceinline__ void transpose4_lanes(uint32_t (&r)[4], int q) {
  const bool o1 = (q & 1) != 0, o2 = (q & 2) != 0;
  // round 1: entries k with bit 0 of k != bit 0 of q come from lane q ^ 1
  uint32_t sa = o1 ? r[0] : r[1], sb = o1 ? r[2] : r[3];
  sa = __shfl_xor_sync(0xffffffffu, sa, 1);
  sb = __shfl_xor_sync(0xffffffffu, sb, 1);
  if (o1) {
    r[0] = sa;
    r[2] = sb;
  } else {
    r[1] = sa;
    r[3] = sb;
  }
  // round 2: entries k with bit 1 of k != bit 1 of q come from lane q ^ 2
  sa = o2 ? r[0] : r[2];
  sb = o2 ? r[1] : r[3];
  sa = __shfl_xor_sync(0xffffffffu, sa, 2);
  sb = __shfl_xor_sync(0xffffffffu, sb, 2);
  if (o2) {
    r[0] = sa;
    r[1] = sb;
  } else {
    r[2] = sa;
    r[3] = sb;
  }
}

// Forward, four key groups at a time: word (i mod 4) of the generator output
// of groups jg0/4 + 4k .. + 3 (keys jg0 + 16k .. + 15), out[m] for group 4k + m.
// The four lanes of a 4-row group (rows i with i mod 4 = lane mod 4) each make
// one of the four calls; a transpose across the group hands lane q word q of
// every call.
__device__ __forceinline__ void dropout_row_words4(const DropoutParams& dp, uint32_t bh, int i,
                                                   int jg0, int k, uint32_t (&out)[4]) {
  const int q = threadIdx.x & 3;
  const uint4 w = philox4x32_10(uint32_t((jg0 >> 2) + 4 * k + q), uint32_t(i >> 2), bh, dp.offset,
                                dp.seed_lo, dp.seed_hi);
  out[0] = w.x;
  out[1] = w.y;
  out[2] = w.z;
  out[3] = w.w;
  transpose4_lanes(out, q);
}

// 0xFF in each byte of `word` that is below T (T in 1..255), 0x00 elsewhere.
__device__ __forceinline__ uint32_t keep_bytes(uint32_t word, uint32_t T) {
  return __vcmpltu4(word, T * 0x01010101u);
}

// A mask for a packed pair of 16-bit values: the low half from byte b of
// `m`, the high half from byte b + 1 (b = 0 or 2).
__device__ __forceinline__ uint32_t pair_mask(uint32_t m, int b) {
  return __byte_perm(m, 0u, b == 0 ? 0x1100u : 0x3322u);
}

// Backward: the keep bytes of key row j for 16 query groups (64 queries)
// starting at query ig0 (a multiple of 4): out[g] holds, in byte k, the byte
// of query ig0 + 4g + k, i.e. byte (j mod 4) of word k of group g's output.
// Lanes 4t .. 4t + 3 (keys with the same j / 4, j mod 4 = lane mod 4) share
// the calls: lane q calls for query group 4k + q and packs, for each lane r
// of the group, byte r of the four words; the transpose then hands lane q
// the packs meant for it.
__device__ __forceinline__ void dropout_col_words(const DropoutParams& dp, uint32_t bh, int j,
                                                  int ig0, uint32_t (&out)[16]) {
  const int q = threadIdx.x & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 w = philox4x32_10(uint32_t(j >> 2), uint32_t((ig0 >> 2) + 4 * k + q), bh,
                                  dp.offset, dp.seed_lo, dp.seed_hi);
    uint32_t pk[4];
#pragma unroll
    for (int r = 0; r < 4; ++r)  // byte r of each of the four words
      pk[r] = __byte_perm(__byte_perm(w.x, w.y, 0x40 | r | ((4 + r) << 4)),
                          __byte_perm(w.z, w.w, 0x40 | r | ((4 + r) << 4)),
                          0x5410);
    transpose4_lanes(pk, q);
#pragma unroll
    for (int m = 0; m < 4; ++m) out[4 * k + m] = pk[m];
  }
}

// 1.0f if byte k of `word` is below T, else 0.0f.
__device__ __forceinline__ float keep_of(uint32_t word, int k, uint32_t T) {
  return ((word >> (8 * k)) & 0xFFu) < T ? 1.f : 0.f;
}

}  // namespace fa
