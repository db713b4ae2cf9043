/* CPU check of the shared-divisor division used by quant4_pack: with
 * r = RN(1/s) and q0 = RN(x r), Markstein's correction q = RN(q0 + e r),
 * e = x - s q0 (exact under FMA), must equal the IEEE quotient RN(x / s)
 * for every normal s and |x| <= s, except where the kernel takes the plain
 * division (|x| or |q0| below 2^-100).  Prints "mismatches N" and exits 1
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
  printf("tested %ld mismatches %ld\n", tested, bad);
  return bad ? 1 : 0;
}
