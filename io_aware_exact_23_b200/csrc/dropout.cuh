// dropout.cuh -- the counter-based generator behind fused dropout on the
// attention probabilities (forward: P before the PV product; backward: the same
// mask regenerated, never stored).
//
// Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011): ten rounds over a 128-bit counter
// with a 64-bit key; each round multiplies counter words 0 and 2 by the round
// multipliers, combines the 64-bit products' halves with words 1 and 3 and the
// key, and advances the key by the two Weyl increments.
//
// Mask layout: for head bh, query row i and key j the counter is
// (i, j >> 4, bh, offset), the key is the 64-bit seed (low word, high word);
// the 8-bit draw of key j is byte (j & 3) of output word ((j & 15) >> 2), so
// one call serves 16 keys, and the key is kept iff the draw is >= T =
// floor(rate * 256).  Kept entries are scaled by 256 / (256 - T).
#pragma once

#include <cstdint>

namespace fa {

struct DropoutParams {
  uint32_t T;        // drop a key when its 8-bit draw is below T
  uint32_t seed_lo;  // Philox key
  uint32_t seed_hi;
  uint32_t offset;   // counter word 3 (e.g. the training step)
  float inv_keep;    // 256 / (256 - T)
};

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// The four output words for query row i and keys 16*jblk .. 16*jblk+15.
__device__ __forceinline__ uint4 dropout_words(const DropoutParams &dp, uint32_t i, uint32_t jblk, uint32_t bh) {
  return philox4x32_10(make_uint4(i, jblk, bh, dp.offset), dp.seed_lo, dp.seed_hi);
}

// Keep bits of keys 16*jblk + t (bit t), t = 0..15.
__device__ __forceinline__ uint32_t dropout_keep16(const DropoutParams &dp, uint32_t i, uint32_t jblk, uint32_t bh) {
  const uint4 w = dropout_words(dp, i, jblk, bh);
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t bits = 0;
#pragma unroll
  for (int t = 0; t < 16; ++t) bits |= static_cast<uint32_t>(((ws[t >> 2] >> (8 * (t & 3))) & 0xFFu) >= dp.T) << t;
  return bits;
}

// Mask for a packed bf16 pair whose low half is key 16*jblk + 2t and high half
// key 16*jblk + 2t + 1 (t = 0..7), straight from that generator call's words w:
// 0xFFFF in each half whose key is kept.  The pair's two draw bytes are spread
// into the two 16-bit halves; adding c256 = (256 - T) * 0x00010001 sets bit 8 of
// a half exactly when its draw is >= T (the sum stays below 512: no carry
// between the halves).
__device__ __forceinline__ uint32_t dropout_pair_mask(const uint4 &w, int t, uint32_t c256) {
  const uint32_t word = (t >> 1) == 0 ? w.x : (t >> 1) == 1 ? w.y : (t >> 1) == 2 ? w.z : w.w;
  const uint32_t b0 = static_cast<uint32_t>(2 * t) & 3u;
  const uint32_t h = __byte_perm(word, 0u, b0 | (4u << 4) | ((b0 + 1u) << 8) | (4u << 12));
  return (((h + c256) >> 8) & 0x00010001u) * 0xFFFFu;
}

// Bit c of the keep mask, extracted afresh at each use (volatile: the compiler may
// not carry 64 extracted values across a wait to reuse them later).
__device__ __forceinline__ uint32_t keep_bit_fresh(uint64_t keep, int c) {
  uint32_t bit;
  asm volatile("{\n\t.reg .b64 t;\n\tshr.b64 t, %1, %2;\n\tcvt.u32.u64 %0, t;\n\tand.b32 %0, %0, 1;\n\t}"
               : "=r"(bit)
               : "l"(keep), "r"(c));
  return bit;
}

}  // namespace fa
