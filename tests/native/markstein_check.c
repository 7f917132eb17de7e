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
 * quotient is at least 2^-24 (any quotient below 2^-17 codes to +-0 in every
 * format: E5M2's smallest subnormal is 2^-16, and 2^-17 ties to even, to 0),
 * and the sign mismatches (which would flip an FP8 zero).  The quotients that
 * differ all have a subnormal residual s*q0 - x (|x| below about 2^-100).  Compiled with
 * -ffp-contract=off so that only fmaf fuses.
 * Usage: markstein_check SEED N            (N random rows per domain)
 *        markstein_check SEED N exhaustive (N scales, each against every finite
 *                                           bf16 x of its domain, edge scales first) */
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
    if (fabsf(qt) >= 0x1p-24f) ++differ_big;
  }
}
/* every finite bf16 x in [lo, hi] against scale s */
static void all_bf16(float lo, float hi, float s) {
  for (uint32_t b = 0; b < 0x10000u; ++b) {
    const float x = f_of(b << 16);
    if (isfinite(x) && x >= lo && x <= hi) check(x, s);
  }
}
static void affine_scale(float mn, float mx, float L) {
  float s = (mx - mn) / L;
  if (s < 1.1920929e-7f) s = 1.1920929e-7f;
  all_bf16(mn, mx, s);
}
static void block_scale(float amax, float Q) { all_bf16(-amax, amax, amax / Q); }
static void exhaustive(long nscales) {
  const float Ls[2] = {255.0f, 15.0f}, Qs[3] = {448.0f, 57344.0f, 127.0f};
  const float bf16_max = f_of(0x7F7Fu << 16);
  /* edge scales: the epsilon floor, the largest amax and the smallest amax the
     writer divides this way (2^-60; below it the writer divides exactly) of every Q */
  affine_scale(-1e-6f, 1e-6f, 255.0f);
  affine_scale(-1e-6f, 0.0f, 15.0f);
  affine_scale(0.0f, 3e-7f, 255.0f);
  affine_scale(-bf16_max / 2.0f, bf16_max / 2.0f, 255.0f);
  for (int q = 0; q < 3; ++q) {
    block_scale(bf16_max, Qs[q]);
    block_scale(0x1p-60f, Qs[q]);
    block_scale(1.0f, Qs[q]);
    block_scale(f_of(0x3FFFu << 16), Qs[q]); /* 1.9921875: mantissa all ones */
  }
  for (long k = 0; k < nscales; ++k) {
    if (k & 1) {
      float amax;
      do amax = f_of((uint32_t)(rnd() & 0x7FFF) << 16); while (!isfinite(amax) || amax < 0x1p-60f);
      block_scale(amax, Qs[k % 3]);
    } else {
      float a = bf16_any(), b = bf16_any();
      float mn = fminf(fminf(a, b), 0.0f), mx = fmaxf(fmaxf(a, b), 0.0f);
      if (isfinite(mx - mn)) affine_scale(mn, mx, Ls[(k >> 1) & 1]);
    }
  }
}
int main(int argc, char **argv) {
  st = argc > 1 ? strtoull(argv[1], 0, 10) * 2654435761ull + 88172645463325252ull : 88172645463325252ull;
  const long rows = argc > 2 ? atol(argv[2]) : 100000;
  if (argc > 3 && strcmp(argv[3], "exhaustive") == 0) {
    exhaustive(rows);
    printf("pairs %llu differ %llu differ_big %llu sign_bad %llu\n", (unsigned long long)n,
           (unsigned long long)differ, (unsigned long long)differ_big, (unsigned long long)sign_bad);
    return 0;
  }
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
