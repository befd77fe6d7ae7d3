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

__device__ __forceinline__ uint32_t word_of(const uint4& w, int k) {
  return k == 0 ? w.x : (k == 1 ? w.y : (k == 2 ? w.z : w.w));
}

// Forward, four key groups at a time: word (i mod 4) of the generator output
// of groups jg0/4 + 4k .. + 3 (keys jg0 + 16k .. + 15), out[m] for group 4k + m.
// The four lanes of a 4-row group each make one of the four calls and pass
// the words to their rows in four shuffle rounds.
__device__ __forceinline__ void dropout_row_words4(const DropoutParams& dp, uint32_t bh, int i,
                                                   int jg0, int k, uint32_t (&out)[4]) {
  const int lane = threadIdx.x & 31, q = lane & 3;
  const int base = lane & ~3;
  const uint4 w = philox4x32_10(uint32_t((jg0 >> 2) + 4 * k + q), uint32_t(i >> 2), bh, dp.offset,
                                dp.seed_lo, dp.seed_hi);
  uint32_t got[4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
    got[t] = __shfl_sync(0xffffffffu, word_of(w, (q + t) & 3), base | ((q - t) & 3));
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int t = (q - m) & 3;
    out[m] = t == 0 ? got[0] : (t == 1 ? got[1] : (t == 2 ? got[2] : got[3]));
  }
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
// Lanes 4t .. 4t + 3 (keys with the same j / 4) share the calls as above.
__device__ __forceinline__ void dropout_col_words(const DropoutParams& dp, uint32_t bh, int j,
                                                  int ig0, uint32_t (&out)[16]) {
  const int lane = threadIdx.x & 31, q = lane & 3;
  const int base = lane & ~3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 w = philox4x32_10(uint32_t(j >> 2), uint32_t((ig0 >> 2) + 4 * k + q), bh,
                                  dp.offset, dp.seed_lo, dp.seed_hi);
    uint32_t got[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      // for receiver lane r = (q + t) mod 4: byte r of each of the four words
      const int r = (q + t) & 3;
      const uint32_t b0 = (w.x >> (8 * r)) & 0xFFu, b1 = (w.y >> (8 * r)) & 0xFFu;
      const uint32_t b2 = (w.z >> (8 * r)) & 0xFFu, b3 = (w.w >> (8 * r)) & 0xFFu;
      const uint32_t packed = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
      got[t] = __shfl_sync(0xffffffffu, packed, base | ((q - t) & 3));
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = (q - m) & 3;
      out[4 * k + m] = t == 0 ? got[0] : (t == 1 ? got[1] : (t == 2 ? got[2] : got[3]));
    }
  }
}

// 1.0f if byte k of `word` is below T, else 0.0f.
__device__ __forceinline__ float keep_of(uint32_t word, int k, uint32_t T) {
  return ((word >> (8 * k)) & 0xFFu) < T ? 1.f : 0.f;
}

}  // namespace fa
