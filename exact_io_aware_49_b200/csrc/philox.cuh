// philox.cuh -- device Philox4x32-10 and the packed dropout keep mask.
//
// Dropout is Bernoulli per attention score and its pattern is regenerated in
// the backward pass rather than stored ("FlashAttention" glossary, Dropout
// bullet; "Flash Attention" glossary, Key Components).  The mask is a pure
// function of (seed, b, h, i, j):
//   key     (k0, k1)         = (seed mod 2^32, seed >> 32)
//   counter (c0, c1, c2, c3) = (j >> 3, i, h, b)
//   key j uses output word (j >> 1) & 3: low 16 bits for even j, high for odd
//   keep <=> u16 >= t, t = round-half-even(p * 65536)
// Philox4x32 with 10 rounds is the generator of Salmon, Moraes, Dror and Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11); the multipliers and
// key increments below are the constants that paper publishes.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace fa {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

__device__ __forceinline__ void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                              uint32_t k1, uint32_t (&out)[4]) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kPhiloxM0, c0);
    const uint32_t lo0 = kPhiloxM0 * c0;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c2);
    const uint32_t lo1 = kPhiloxM1 * c2;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

// Philox4x32-10 for calls that share counter words c1, c2, c3 and differ in
// c0 only (one query row of one head: counter (j >> 3, i, h, b)).  With c2
// fixed, round 0's second product is the same for every call, and so is round
// 1's first product (its operand is round 0's new c0 = hi(M1 c2) ^ c1 ^ k0);
// the per-row part of both rounds is precomputed once:
//   a2 = c3 ^ k1(0)                       (round 0: c2' = hi(M0 c0) ^ a2)
//   a3 = lo(M1 c2) ^ k0(1)                (round 1: c0'' = hi(M1 c2') ^ a3)
//   a4 = hi(M0 c0') ^ k1(1), b1 = lo(M0 c0')   (round 1: c2'' = lo(M0 c0) ^ a4, c3'' = b1)
// so a call costs 18 multiplies instead of 20 and gives the same words.
struct PhiloxFixed123 {
  uint32_t a2, a3, a4, b1;
};

__device__ __forceinline__ PhiloxFixed123 philox_fix123(uint32_t c1, uint32_t c2, uint32_t c3, const uint32_t* rk) {
  const uint32_t c0r0 = __umulhi(kPhiloxM1, c2) ^ c1 ^ rk[0];  // round 0's new c0 (fixed)
  PhiloxFixed123 f;
  f.a2 = c3 ^ rk[1];
  f.a3 = (kPhiloxM1 * c2) ^ rk[2];
  f.a4 = __umulhi(kPhiloxM0, c0r0) ^ rk[3];
  f.b1 = kPhiloxM0 * c0r0;
  return f;
}

__device__ __forceinline__ void philox4x32_10_c0(uint32_t c0, const PhiloxFixed123& f, const uint32_t* rk,
                                                 uint32_t (&out)[4]) {
  // round 0 (the c2 product is folded into f)
  const uint32_t x2 = __umulhi(kPhiloxM0, c0) ^ f.a2;
  const uint32_t x3 = kPhiloxM0 * c0;
  // round 1 (the c0 product is folded into f)
  uint32_t y0 = __umulhi(kPhiloxM1, x2) ^ f.a3;
  uint32_t y1 = kPhiloxM1 * x2;
  uint32_t y2 = x3 ^ f.a4;
  uint32_t y3 = f.b1;
#pragma unroll
  for (int r = 2; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kPhiloxM0, y0);
    const uint32_t lo0 = kPhiloxM0 * y0;
    const uint32_t hi1 = __umulhi(kPhiloxM1, y2);
    const uint32_t lo1 = kPhiloxM1 * y2;
    y0 = hi1 ^ y1 ^ rk[2 * r];
    y1 = lo1;
    y2 = hi0 ^ y3 ^ rk[2 * r + 1];
    y3 = lo0;
  }
  out[0] = y0;
  out[1] = y1;
  out[2] = y2;
  out[3] = y3;
}

// kNB calls of philox4x32_10_c0 (counters c0, c0 + 1, ..., c0 + kNB - 1)
// computed round by round in lockstep: the kNB independent multiply chains are
// written interleaved, so they overlap in the multiplier pipeline instead of
// running one after another at its latency.
template <int kNB>
__device__ __forceinline__ void philox4x32_10_c0_batch(uint32_t c0, const PhiloxFixed123& f, const uint32_t* rk,
                                                       uint32_t (&out)[kNB][4]) {
  uint32_t y0[kNB], y1[kNB], y2[kNB], y3[kNB];
#pragma unroll
  for (int n = 0; n < kNB; ++n) {
    const uint32_t x2 = __umulhi(kPhiloxM0, c0 + n) ^ f.a2;  // round 0
    const uint32_t x3 = kPhiloxM0 * (c0 + n);
    y0[n] = __umulhi(kPhiloxM1, x2) ^ f.a3;  // round 1
    y1[n] = kPhiloxM1 * x2;
    y2[n] = x3 ^ f.a4;
    y3[n] = f.b1;
  }
#pragma unroll
  for (int r = 2; r < 10; ++r) {
#pragma unroll
    for (int n = 0; n < kNB; ++n) {
      const uint32_t hi0 = __umulhi(kPhiloxM0, y0[n]);
      const uint32_t lo0 = kPhiloxM0 * y0[n];
      const uint32_t hi1 = __umulhi(kPhiloxM1, y2[n]);
      const uint32_t lo1 = kPhiloxM1 * y2[n];
      y0[n] = hi1 ^ y1[n] ^ rk[2 * r];
      y1[n] = lo1;
      y2[n] = hi0 ^ y3[n] ^ rk[2 * r + 1];
      y3[n] = lo0;
    }
  }
#pragma unroll
  for (int n = 0; n < kNB; ++n) {
    out[n][0] = y0[n];
    out[n][1] = y1[n];
    out[n][2] = y2[n];
    out[n][3] = y3[n];
  }
}

// Philox4x32-10 for calls that share counter words c0, c2, c3 and differ in
// c1 only (one key group of one head: counter (j >> 3, i, h, b) over queries
// i).  Round 0 then has no varying product (its new c0 is c1 ^ e0), round 1
// has one (M0 times that c0) and round 2 one (M1 times round 1's new c2); the
// per-key-group parts are precomputed once:
//   e0 = hi(M1 c2) ^ k0(0)                   (round 0: c0' = c1 ^ e0)
//   f2 = lo(M0 c0) ^ k1(1)                   (round 1: c2'' = hi(M0 c0') ^ f2)
//   f3 = lo(M1 (hi(M0 c0) ^ c3 ^ k1(0))) ^ k0(2)     (round 2: c0 = hi(M1 c2'') ^ f3)
//   f4 = hi(M0 (hi(M1 c2') ^ lo(M1 c2) ^ k0(1))) ^ k1(2), g1 = lo(M0 ...)
// so a call costs 16 multiplies instead of 20 and gives the same words.
struct PhiloxFixed023 {
  uint32_t e0, f2, f3, f4, g1;
};

__device__ __forceinline__ PhiloxFixed023 philox_fix023(uint32_t c0, uint32_t c2, uint32_t c3, const uint32_t* rk) {
  // round 0: c1' = lo(M1 c2), c2' = hi(M0 c0) ^ c3 ^ k1(0), c3' = lo(M0 c0) (all fixed)
  const uint32_t r0c1 = kPhiloxM1 * c2;
  const uint32_t r0c2 = __umulhi(kPhiloxM0, c0) ^ c3 ^ rk[1];
  const uint32_t r0c3 = kPhiloxM0 * c0;
  // round 1: c0'' = hi(M1 c2') ^ c1' ^ k0(1), c1'' = lo(M1 c2') (fixed)
  const uint32_t r1c0 = __umulhi(kPhiloxM1, r0c2) ^ r0c1 ^ rk[2];
  const uint32_t r1c1 = kPhiloxM1 * r0c2;
  PhiloxFixed023 f;
  f.e0 = __umulhi(kPhiloxM1, c2) ^ rk[0];
  f.f2 = r0c3 ^ rk[3];
  f.f3 = r1c1 ^ rk[4];
  // round 2: c2 = hi(M0 c0'') ^ c3'' ^ k1(2), c3 = lo(M0 c0'') (the product is fixed)
  f.f4 = __umulhi(kPhiloxM0, r1c0) ^ rk[5];
  f.g1 = kPhiloxM0 * r1c0;
  return f;
}

__device__ __forceinline__ void philox4x32_10_c1(uint32_t c1, const PhiloxFixed023& f, const uint32_t* rk,
                                                 uint32_t (&out)[4]) {
  // round 0: no varying product
  const uint32_t x0 = c1 ^ f.e0;
  // round 1: M0 x0 varies
  const uint32_t y2 = __umulhi(kPhiloxM0, x0) ^ f.f2;
  const uint32_t y3 = kPhiloxM0 * x0;
  // round 2: M1 y2 varies
  uint32_t z0 = __umulhi(kPhiloxM1, y2) ^ f.f3;
  uint32_t z1 = kPhiloxM1 * y2;
  uint32_t z2 = y3 ^ f.f4;
  uint32_t z3 = f.g1;
#pragma unroll
  for (int r = 3; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kPhiloxM0, z0);
    const uint32_t lo0 = kPhiloxM0 * z0;
    const uint32_t hi1 = __umulhi(kPhiloxM1, z2);
    const uint32_t lo1 = kPhiloxM1 * z2;
    z0 = hi1 ^ z1 ^ rk[2 * r];
    z1 = lo1;
    z2 = hi0 ^ z3 ^ rk[2 * r + 1];
    z3 = lo0;
  }
  out[0] = z0;
  out[1] = z1;
  out[2] = z2;
  out[3] = z3;
}

// kNB calls of philox4x32_10_c1 with counter words c1[n], in lockstep (see
// philox4x32_10_c0_batch).
template <int kNB>
__device__ __forceinline__ void philox4x32_10_c1_batch(const uint32_t (&c1)[kNB], const PhiloxFixed023& f,
                                                       const uint32_t* rk, uint32_t (&out)[kNB][4]) {
  uint32_t z0[kNB], z1[kNB], z2[kNB], z3[kNB];
#pragma unroll
  for (int n = 0; n < kNB; ++n) {
    const uint32_t x0 = c1[n] ^ f.e0;                        // round 0
    const uint32_t y2 = __umulhi(kPhiloxM0, x0) ^ f.f2;      // round 1
    const uint32_t y3 = kPhiloxM0 * x0;
    z0[n] = __umulhi(kPhiloxM1, y2) ^ f.f3;                  // round 2
    z1[n] = kPhiloxM1 * y2;
    z2[n] = y3 ^ f.f4;
    z3[n] = f.g1;
  }
#pragma unroll
  for (int r = 3; r < 10; ++r) {
#pragma unroll
    for (int n = 0; n < kNB; ++n) {
      const uint32_t hi0 = __umulhi(kPhiloxM0, z0[n]);
      const uint32_t lo0 = kPhiloxM0 * z0[n];
      const uint32_t hi1 = __umulhi(kPhiloxM1, z2[n]);
      const uint32_t lo1 = kPhiloxM1 * z2[n];
      z0[n] = hi1 ^ z1[n] ^ rk[2 * r];
      z1[n] = lo1;
      z2[n] = hi0 ^ z3[n] ^ rk[2 * r + 1];
      z3[n] = lo0;
    }
  }
#pragma unroll
  for (int n = 0; n < kNB; ++n) {
    out[n][0] = z0[n];
    out[n][1] = z1[n];
    out[n][2] = z2[n];
    out[n][3] = z3[n];
  }
}

__host__ __device__ inline void philox_round_keys(uint64_t seed, uint32_t (&rk)[20]) {
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    rk[2 * r] = k0;
    rk[2 * r + 1] = k1;
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
}

// Constants that turn the threshold t (1..65535) into a two-lane compare.
struct DropConst {
  uint32_t c2;  // per-lane addend, both halves
  uint32_t m0;  // all ones when t <= 0x8000, else zero
};

__host__ __device__ inline DropConst make_drop_const(uint32_t t) {
  const uint32_t c = (t <= 0x8000u) ? (0x8000u - t) : (0x10000u - t);
  DropConst k;
  k.c2 = c | (c << 16);
  k.m0 = (t <= 0x8000u) ? 0xFFFFFFFFu : 0u;
  return k;
}

// For a Philox word w holding two 16-bit draws x_lo, x_hi, returns a mask with
// 0xFFFF in each half whose draw is >= t, 0 otherwise.  With a = w & 0x7FFF7FFF
// and y = a + c2 (no carry crosses a lane), bit 15 of each lane of y is
// (x & 0x7FFF) >= t (t <= 0x8000) or (x & 0x7FFF) >= t - 0x8000 (t > 0x8000);
// combining with the lane's top bit by OR / AND gives x >= t, and PRMT's
// sign-replicate mode spreads bit 15 / bit 31 over the low / high half.
__device__ __forceinline__ uint32_t keep_mask_2x16(uint32_t w, DropConst k) {
  const uint32_t a = w & 0x7FFF7FFFu;
  const uint32_t y = a + k.c2;
  const uint32_t z = (w & y) | ((w | y) & k.m0);
  return prmt(z, 0u, 0xBB99u);
}


// Keep bits of one query row for the 8 * kCalls keys j0 .. j0 + 8 kCalls - 1
// of a tile (jb0 = j0 / 8), packed into kCalls / 4 words: one Philox call per
// 8 keys (counter words c1, c2, c3 of the row fixed in ``f``).  The 16-bit
// pair c of the row's P (keys j0 + 2c, j0 + 2c + 1) uses the low and high half
// of word c & 3 of call c >> 2; the two-lane test leaves their keep bits at
// bits 15 and 31.  Pair c = 16 k + 2 s + e is stored in word k at bits
// 15 - s - 8 e and 31 - s - 8 e (a multiply-high shifts and adds), so that
// after a left shift by s its bits are the sign bits of bytes 1 and 3 (e = 0)
// or 0 and 2 (e = 1), which PRMT's sign-replicate mode turns into a 0 / 0xFFFF
// mask per 16-bit lane (keep_mask_pair).
template <bool kHighT, int kCalls, int kNB = (kCalls < 8) ? kCalls : 8>  // kNB: calls in flight together
__device__ __forceinline__ void draw_keep_words(uint32_t jb0, const PhiloxFixed123& f, const uint32_t* rk,
                                                uint32_t c2, uint32_t (&W)[kCalls / 4]) {
  static_assert(kCalls % 4 == 0, "four calls per packed word");
  static_assert(kCalls % kNB == 0, "whole lockstep batches");
#pragma unroll
  for (int k = 0; k < kCalls / 4; ++k) W[k] = 0u;
#pragma unroll
  for (int g0 = 0; g0 < kCalls; g0 += kNB) {
    uint32_t w[kNB][4];
    philox4x32_10_c0_batch<kNB>(jb0 + g0, f, rk, w);
#pragma unroll
    for (int n = 0; n < kNB; ++n) {
      const int g = g0 + n;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // bit 15 / 31: the low / high 16-bit draw is >= t (see keep_mask_2x16)
        const uint32_t y = (w[n][e] & 0x7FFF7FFFu) + c2;
        const uint32_t zm = (kHighT ? (w[n][e] & y) : (w[n][e] | y)) & 0x80008000u;
        const int sh = 2 * (g & 3) + (e >> 1) + 8 * (e & 1);
        W[g >> 2] = (sh == 0) ? (W[g >> 2] | zm) : mad_hi_u32(zm, 1u << (32 - sh), W[g >> 2]);
      }
    }
  }
}

// 0 / 0xFFFF lane mask of 16-bit pair c from the packed keep words.
template <int kWords>
__device__ __forceinline__ uint32_t keep_mask_pair(const uint32_t (&W)[kWords], int c) {
  const int cc = c & 15;
  return prmt(W[c >> 4] << (cc >> 1), 0u, (cc & 1) ? 0xAA88u : 0xBB99u);
}

// Keep bits of the dropout mask for this lane's key row and 32 kWords
// consecutive queries: bit l of W[w] is keep(key, q0 + 32 w + l).  ``phx``
// holds the per-key-group part of the Philox rounds (counter words key >> 3,
// h, b are fixed, the query varies).
//
// The Philox counter (key >> 3, query, h, b) yields 8 keys x 1 query per call,
// so lane l8 of each group of 8 consecutive keys evaluates queries
// q0 + 32 w + 8 j + l8 (j = 0..3) for word w.  Per Philox output word the two
// 16-bit draws are tested against t with three integer ops (the same two-lane
// test as the mask export), and a multiply-high on the FMA pipe moves the two
// keep bits to bits 2e and 16 + 2e of an accumulator.  That gives, per lane,
// four bytes whose bit k' is keep(key 8 g + k', query q0 + 32 w + 8 j + l8); a
// three-stage butterfly of lane shuffles then transposes each 8 x 8 bit block
// so that lane k' holds bit l = keep(its key, query q0 + 32 w + 8 j + l).  The
// 4 kWords Philox calls run in lockstep and the words' butterflies are
// interleaved, for more independent work per warp.
template <bool kHighT, int kWords>
__device__ __forceinline__ void keep_bits(const PhiloxFixed023& phx, uint32_t q0, const uint32_t* rk, uint32_t c2,
                                          int lane, uint32_t (&W)[kWords]) {
  constexpr int kCalls = 4 * kWords;
  const uint32_t l8 = static_cast<uint32_t>(lane & 7);
  uint32_t cq[kCalls];
#pragma unroll
  for (int j = 0; j < kCalls; ++j) cq[j] = q0 + 8 * j + l8;
  uint32_t wv[kCalls][4];
  philox4x32_10_c1_batch<kCalls>(cq, phx, rk, wv);
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    W[w] = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t acc = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = wv[4 * w + j][e];
        const uint32_t y = (x & 0x7FFF7FFFu) + c2;
        const uint32_t zm = (kHighT ? (x & y) : (x | y)) & 0x80008000u;  // keep bits at 15 and 31
        acc = mad_hi_u32(zm, 1u << (17 + 2 * e), acc);                    // -> bits 2e and 16 + 2e
      }
      W[w] |= ((acc | (acc >> 15)) & 0xFFu) << (8 * j);
    }
  }
#pragma unroll
  for (int sh = 4; sh >= 1; sh >>= 1) {
    const uint32_t lo = (sh == 4) ? 0x0F0F0F0Fu : ((sh == 2) ? 0x33333333u : 0x55555555u);
#pragma unroll
    for (int w = 0; w < kWords; ++w) {
      const uint32_t y = __shfl_xor_sync(0xffffffffu, W[w], sh);
      W[w] = (l8 & sh) ? ((W[w] & ~lo) | ((y >> sh) & lo)) : ((W[w] & lo) | ((y << sh) & ~lo));
    }
  }
}

// Marks dropped entries by setting the sign bit of P: for 4 columns whose keep
// bits are the low nibble of ``nib``, spreads the bits to the byte signs with
// one multiply and turns each into a full-word mask with PRMT's sign mode.
__device__ __forceinline__ void mark_dropped4(float* P, uint32_t nib) {
  const uint32_t sp = (nib & 0xFu) * 0x10204080u;  // bit e -> bit 8 e + 7
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t keep = prmt(sp, 0u, 0x8888u + 0x1111u * e);
    P[e] = __uint_as_float(__float_as_uint(P[e]) ^ (~keep & 0x80000000u));
  }
}

}  // namespace fa
