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

// The same generator with its round keys precomputed (they are the same for
// every thread of a launch): rk[2r], rk[2r + 1] = (k0 + r W0, k1 + r W1) mod
// 2^32 for rounds r = 0..9.  ``rk`` points at kernel parameter space, so each
// key is an operand read from the constant bank, not a register.
__device__ __forceinline__ void philox4x32_10_rk(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 const uint32_t* rk, uint32_t (&out)[4]) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kPhiloxM0, c0);
    const uint32_t lo0 = kPhiloxM0 * c0;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c2);
    const uint32_t lo1 = kPhiloxM1 * c2;
    c0 = hi1 ^ c1 ^ rk[2 * r];
    c1 = lo1;
    c2 = hi0 ^ c3 ^ rk[2 * r + 1];
    c3 = lo0;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
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

}  // namespace fa
