/* CPU check of the kernels' stochastic-rounding decision (sr_magnitude2 in
 * csrc/common.cuh) against the rule it implements: between the neighbouring
 * E2M1 grid magnitudes lo and hi, round up iff u = (w >> 8) * 2^-24 is below
 * (|y| - lo) / (hi - lo)  ("Pretraining Large Language Models with NVFP4",
 * section 2B.4).  The kernel's arithmetic is restated here one element at a
 * time, with C99 directed rounding for the GPU's fma.rp / add.rp on FP32
 * pairs; the rule is evaluated exactly in double.  Usage: sr_decision_check STRIDE -- every STRIDE-th float in
 * [0, 6.4) (both signs alternate) with two words each: a fixed corner word
 * and a pseudo-random one.  Prints the count of mismatches; exit 1 if any. */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#pragma STDC FENV_ACCESS ON

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float fma_ru(float a, float b, float c) {
  fesetround(FE_UPWARD);
  volatile float r = fmaf(a, b, c);
  fesetround(FE_TONEAREST);
  return r;
}
static float add_ru(float a, float b) {
  fesetround(FE_UPWARD);
  volatile float r = a + b;
  fesetround(FE_TONEAREST);
  return r;
}

/* the kernel's formula: 2s, twice the lattice step, from |y|'s binade (s = 0.5
 * below 2), then ceil_s(RU(|y| - u*s)) by the magic-number add, sign restored */
static float kernel_decision(float y, uint32_t w) {
  const float a = fabsf(y);
  volatile float s2 = u2f(f2u(fmaxf(a, 1.0f)) & 0x7F800000u);
  volatile float k = (float)(w >> 8);
  volatile float st = s2 * -2.98023223876953125e-08f;   /* -s * 2^-24 */
  const float z = fma_ru(k, st, a);
  volatile float m = s2 * 6291456.0f;                    /* 1.5 * 2^23 * s */
  volatile float t = add_ru(z, m);
  const float q = t - m;
  return u2f(f2u(q) | (f2u(y) & 0x80000000u));
}

/* the rule, in exact arithmetic */
static const double kGrid[] = {0, 0.5, 1, 1.5, 2, 3, 4, 6, 8};
static float rule(float y, uint32_t w) {
  const double a = fabs((double)y);
  int i = 0;
  while (!(a >= kGrid[i] && a < kGrid[i + 1])) ++i;
  const double p = (a - kGrid[i]) / (kGrid[i + 1] - kGrid[i]);
  const double u = (double)(w >> 8) / 16777216.0;
  const float q = (float)((u < p) ? kGrid[i + 1] : kGrid[i]);
  return u2f(f2u(q) | (f2u(y) & 0x80000000u));
}

int main(int argc, char** argv) {
  const uint32_t stride = argc > 1 ? (uint32_t)strtoul(argv[1], NULL, 10) : 1u;
  const uint32_t corner[6] = {0u, 0xFFFFFFFFu, 0x80000000u, 0x000000FFu, 0x7FFFFF00u, 0x00000100u};
  const uint32_t top = f2u(6.4f);
  uint64_t state = 0x9E3779B97F4A7C15ull, n = 0, bad = 0;
  for (uint32_t b = 0; b < top; b += stride) {
    const float y = u2f(b | ((b / stride) & 1u ? 0x80000000u : 0u));
    state ^= state << 13; state ^= state >> 7; state ^= state << 17;
    const uint32_t ws[2] = {corner[(b / stride) % 6], (uint32_t)(state >> 16)};
    for (int j = 0; j < 2; ++j) {
      const float got = kernel_decision(y, ws[j]), want = rule(y, ws[j]);
      if (f2u(got) != f2u(want)) {
        if (bad < 5) printf("mismatch y=%a w=%08x: %a vs %a\n", y, ws[j], got, want);
        ++bad;
      }
      ++n;
    }
  }
  printf("%llu pairs, %llu mismatches\n", (unsigned long long)n, (unsigned long long)bad);
  return bad != 0;
}
