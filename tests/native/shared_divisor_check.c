/* CPU check of the shared-divisor division used by quant4_pack: with
 * r = RN(1/s) and q0 = RN(x r), Markstein's correction q = RN(q0 + e r),
 * e = x - s q0 (exact under FMA), must equal the IEEE quotient RN(x / s)
 * for every normal s and |x| <= s, except where the kernel takes the plain
 * division (|x| or |q0| below 2^-100); and, for scales in [2^-60, 1], that
 * the same sequence without that test still gives the code IEEE division
 * gives.  Prints "mismatches N" and exits 1
 * on any mismatch.  Build: cc -O2 -mfma -ffp-contract=off ... -lm */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint64_t st = 88172645463325252ull;
static uint32_t rnd(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return (uint32_t)st; }
static float bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }

static float shared_div(float x, float s) {
  float r = 1.0f / s;
  float q0 = x * r;
  if (fabsf(x) < 0x1p-100f || fabsf(q0) < 0x1p-100f) return x / s;
  float e = fmaf(-q0, s, x);
  return fmaf(e, r, q0);
}

int main(int argc, char** argv) {
  long n = argc > 1 ? atol(argv[1]) : 20000000L;
  long bad = 0, tested = 0;
  for (long it = 0; it < n; ++it) {
    float s = bits(rnd() & 0x7fffffff);
    if (!(s >= 1.17549435e-38f && s <= 3.0e38f)) continue;
    float x = bits(rnd());
    if (!isfinite(x)) continue;
    if (fabsf(x) > s) { x = x / 2; if (fabsf(x) > s) continue; }
    float q = shared_div(x, s), ref = x / s;
    ++tested;
    if (memcmp(&q, &ref, 4)) ++bad;
  }
  /* significands near all ones, x near s, scaled-down x */
  for (uint32_t e = 1; e < 254; ++e)
    for (uint32_t k = 0; k < 4000; ++k) {
      float s = bits((e << 23) | (0x7fffff - (rnd() & 0xff)));
      float x = bits((e << 23) | (rnd() & 0x7fffff));
      if (fabsf(x) > s) x = s;
      if (rnd() & 1) x = -x;
      if (rnd() & 1) x = x * 0x1p-20f;
      float q = shared_div(x, s), ref = x / s;
      ++tested;
      if (memcmp(&q, &ref, 4)) ++bad;
    }
  /* Blocks with a scale in [2^-60, 1] take the division without the guard
   * (no per-element test).  There: for |x| >= 2^-100 the quotient must be
   * the IEEE one bit for bit; below, it must be tiny (under 2^-30, far below
   * the smallest nonzero threshold magnitude of either codebook, 0.005) with
   * the sign the IEEE quotient has, +0 and -0 counting as not positive: the
   * code then depends on that sign alone. */
  long bad_tiny = 0, tested_tiny = 0;
  for (long it = 0; it < n; ++it) {
    float s = bits((uint32_t)(67 + rnd() % 60) << 23 | (rnd() & 0x7fffff));     /* 2^-60 .. 2^-1 */
    if (rnd() % 8 == 0) s = 1.0f;
    uint32_t xb = rnd();
    float x = bits(xb);
    if (!isfinite(x)) continue;
    if (rnd() & 1) x = bits((xb & 0x80000000u) | (rnd() % (27u << 23)));      /* below 2^-100 */
    if (fabsf(x) > s) continue;
    float r = 1.0f / s;
    float q0 = x * r;
    float q = fmaf(fmaf(-q0, s, x), r, q0);
    float ref = x / s;
    if (fabsf(x) >= 0x1p-100f) {
      ++tested;
      if (memcmp(&q, &ref, 4)) ++bad;
    } else {
      ++tested_tiny;
      if (!(fabsf(q) < 0x1p-30f && fabsf(ref) < 0x1p-30f && ((q > 0.0f) == (ref > 0.0f)))) ++bad_tiny;
    }
  }
  printf("unguarded: tiny tested %ld bad %ld\n", tested_tiny, bad_tiny);
  bad += bad_tiny;
  printf("tested %ld mismatches %ld\n", tested, bad);
  return bad ? 1 : 0;
}
