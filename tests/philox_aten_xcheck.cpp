// Cross-check helper for the oracle's Philox4x32-10: prints the four output
// words of ATen's header-only philox_engine for (seed, subsequence, offset)
// triples read from stdin.  ATen's engine keys Philox with
// (seed mod 2^32, seed >> 32) and counts with (offset lo, offset hi,
// subsequence lo, subsequence hi), so the dropout counter (c0, c1, c2, c3)
// maps to offset = c1 << 32 | c0 and subsequence = c3 << 32 | c2.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
#include <cinttypes>

int main() {
  unsigned long long seed, subseq, offset;
  while (std::scanf("%llu %llu %llu", &seed, &subseq, &offset) == 3) {
    at::philox_engine e(seed, subseq, offset);
    uint32_t r0 = e(), r1 = e(), r2 = e(), r3 = e();
    std::printf("%u %u %u %u\n", r0, r1, r2, r3);
  }
  return 0;
}
