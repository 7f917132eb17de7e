/* Markstein's correction of x * RN(1/s) (IBM J. Res. Develop. 34(1), 1990), in
 * the form the cache writer evaluates it:
 *     q0 = RN(x * y),  y = RN(1 / s)
 *     r  = RN(s * q0 - x)          (exact: one fused multiply-add)
 *     q  = RN(q0 - r * y)          (one fused multiply-add)
 * checked against the correctly rounded x / s on the writer's two domains.
 *   affine: a row of bf16 values in [mn, mx] (mn <= 0 <= mx), scale =
 *           max(RN((mx - mn) / L), FLT_EPSILON), L in {255, 15};
 *   block:  scale = RN(amax / Q), Q in {448, 57344, 127}, amax >= 2^-60, x in
 *           [-amax, amax], with subnormal x.
 * Reports the quotients that differ, the ones that differ while the exact
 * quotient is at least 2^-40 (any smaller one codes to 0 in every format), and
 * the sign mismatches (which would flip an FP8 zero).  Compiled with
 * -ffp-contract=off so that only fmaf fuses.  Usage: markstein_check SEED N. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint64_t st;
static uint64_t rnd(void) { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; }
static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float to_bf16(float x) {  /* round to bf16, nearest-even */
  uint32_t u = u_of(x);
  return f_of((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000u);
}
static float bf16_any(void) {
  for (;;) {
    uint32_t b = (uint32_t)(rnd() & 0xFFFF);
    if (rnd() & 1) b = (b & 0x807F) | ((uint32_t)(110 + rnd() % 40) << 7);
    float f = f_of(b << 16);
    if (isfinite(f)) return f;
  }
}
static uint64_t n, differ, differ_big, sign_bad;
static void check(float x, float s) {
  const float y = 1.0f / s;
  const float q0 = x * y;
  const float r = fmaf(q0, s, -x);
  const float q = fmaf(r, -y, q0);
  const float qt = x / s;
  ++n;
  if (signbit(q) != signbit(qt)) ++sign_bad;
  if (u_of(q) != u_of(qt)) {
    ++differ;
    if (fabsf(qt) >= 0x1p-40f) ++differ_big;
  }
}
int main(int argc, char **argv) {
  st = argc > 1 ? strtoull(argv[1], 0, 10) * 2654435761ull + 88172645463325252ull : 88172645463325252ull;
  const long rows = argc > 2 ? atol(argv[2]) : 100000;
  for (long row = 0; row < rows; ++row) {
    /* affine domain */
    float a = bf16_any(), b = bf16_any();
    float mn = fminf(fminf(a, b), 0.0f), mx = fmaxf(fmaxf(a, b), 0.0f), range = mx - mn;
    if (isfinite(range)) {
      float s = range / ((row & 1) ? 15.0f : 255.0f);
      if (s < 1.1920929e-7f) s = 1.1920929e-7f;
      check(mn, s); check(mx, s); check(0.0f, s); check(-0.0f, s);
      for (int k = 0; k < 28; ++k) {
        float x = to_bf16(mn + ((float)(rnd() % 1000001) / 1000000.0f) * range);
        check(fminf(fmaxf(x, mn), mx), s);
      }
    }
    /* block domain */
    float amax;
    do amax = f_of((uint32_t)(rnd() & 0x7FFF) << 16); while (!isfinite(amax) || amax < 0x1p-60f);
    const float Q = (row % 3 == 0) ? 448.0f : ((row % 3 == 1) ? 57344.0f : 127.0f);
    const float s = amax / Q;
    check(amax, s); check(-amax, s); check(-0.0f, s);
    for (int k = 0; k < 29; ++k) {
      float x = (k < 6) ? f_of((uint32_t)(rnd() & 0x80FF) << 16)   /* subnormal bf16 */
                        : to_bf16((((float)(rnd() % 2000001) / 1000000.0f) - 1.0f) * amax);
      if (fabsf(x) > amax) x = copysignf(amax, x);
      check(x, s);
    }
  }
  printf("pairs %llu differ %llu differ_big %llu sign_bad %llu\n", (unsigned long long)n,
         (unsigned long long)differ, (unsigned long long)differ_big, (unsigned long long)sign_bad);
  return 0;
}
