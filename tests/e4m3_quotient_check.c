/* Exhaustive host check of the quantisation kernel's quotient (E4M3 codes of Q and K, one
 * scale per 128-row tile).  The kernel takes x / scale from the tile's correctly rounded
 * reciprocal r = 1 / scale and one correction step (Markstein, IBM J. Res. Develop. 1990):
 * q0 = x * r, q = fma(fma(-q0, scale, x), r, q0), when scale >= 2^-100, and an IEEE
 * division otherwise.  For every positive finite 16-bit amax (bf16 or fp16), scale =
 * amax / 448 in fp32, and every x of the same type with 0 <= x <= amax (the arithmetic is
 * odd in x), this program checks that q and the IEEE quotient x / scale are the same
 * float, or that both lie at or below 2^-10 in magnitude, where E4M3 (smallest subnormal
 * 2^-9, round to nearest even) gives code 0 for each.
 * Usage: e4m3_quotient_check bf16|fp16; prints "pairs N bad M". */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bf16(uint32_t b) {
  uint32_t u = b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static float from_fp16(uint32_t h) {
  const int e = (h >> 10) & 31, m = h & 1023;
  return e == 0 ? ldexpf((float)m, -24) : ldexpf((float)(m | 1024), e - 25);
}

int main(int argc, char** argv) {
  const int fp16 = argc > 1 && strcmp(argv[1], "fp16") == 0;
  const uint32_t top = fp16 ? 0x7bff : 0x7f7f;
  long long pairs = 0, bad = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, bad)
  for (uint32_t a = 1; a <= top; ++a) {
    const float amax = fp16 ? from_fp16(a) : from_bf16(a);
    const float scale = amax / 448.0f;
    if (!(scale >= 0x1p-100f) || isinf(scale)) continue; /* the kernel divides these tiles */
    const float r = 1.0f / scale;
    for (uint32_t b = 0; b <= a; ++b) {
      const float x = fp16 ? from_fp16(b) : from_bf16(b);
      const float ieee = x / scale;
      const float q0 = x * r;
      const float q = fmaf(fmaf(-q0, scale, x), r, q0);
      ++pairs;
      if (memcmp(&q, &ieee, 4) != 0 && !(fabsf(q) <= 0x1p-10f && fabsf(ieee) <= 0x1p-10f &&
                                         signbit(q) == signbit(ieee)))
        ++bad;
    }
  }
  printf("pairs %lld bad %lld\n", pairs, bad);
  return 0;
}
