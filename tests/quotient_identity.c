/* Host-side check of the division-free quotient used by the per-row E4M3
 * quantizer: with r = RN(1/s), q = RN(x r), e = RN(q s - x) (fma) and
 * q' = RN(q - e r) (fma), q' equals the IEEE fp32 quotient RN(x / s)
 * (Markstein's correction, IBM J. Res. Dev. 34(1), 1990).
 *
 * Part 1 is exhaustive over significands: every bf16 significand of x (8
 * bits) against every fp32 significand of s, with both relative exponent
 * offsets, which covers every quotient whose intermediates stay normal (all
 * results scale exactly by powers of two there).  Part 2 checks signed zeros
 * and part 3 random pairs over the whole range the kernel uses the identity
 * for (s = RN(amax / 448) in [2^-80, 2^126], amax a finite bf16): either q' == RN(x / s), or both are below 2^-10
 * in magnitude with the sign of x (the same E4M3 code, a signed zero).
 * Exit status 0 when every check holds.  Arithmetic is plain IEEE fp32
 * (build with -ffp-contract=off; fmaf is the correctly rounded libm fma). */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float corrected(float x, float s, float r) {
  float q = x * r;
  float e = fmaf(q, s, -x);
  return fmaf(-e, r, q);
}

typedef struct { int t, nt; uint64_t bad, n; } job;

static void* exhaustive(void* p) {
  job* j = (job*)p;
  for (uint32_t m = (uint32_t)j->t; m < (1u << 23); m += (uint32_t)j->nt)
    for (uint32_t se = 0; se < 2; ++se) {
      const float s = u2f((127u + se) << 23 | m);
      const float r = 1.0f / s;
      for (uint32_t mx = 0; mx < 128; ++mx)
        for (uint32_t xe = 0; xe < 2; ++xe) {
          const float x = u2f((127u + xe) << 23 | mx << 16);
          j->n++;
          if (f2u(corrected(x, s, r)) != f2u(x / s)) j->bad++;
        }
    }
  return NULL;
}

static uint64_t rng = 0x9E3779B97F4A7C15ull;
static uint64_t next(void) { rng ^= rng << 13; rng ^= rng >> 7; rng ^= rng << 17; return rng; }

int main(int argc, char** argv) {
  int nt = argc > 1 ? atoi(argv[1]) : 8;
  if (nt < 1) nt = 1;
  if (nt > 64) nt = 64;
  pthread_t th[64];
  job jobs[64];
  for (int i = 0; i < nt; ++i) {
    jobs[i].t = i; jobs[i].nt = nt; jobs[i].bad = 0; jobs[i].n = 0;
    pthread_create(&th[i], NULL, exhaustive, &jobs[i]);
  }
  uint64_t bad = 0, n = 0;
  for (int i = 0; i < nt; ++i) { pthread_join(th[i], NULL); bad += jobs[i].bad; n += jobs[i].n; }
  printf("exhaustive: %llu pairs, %llu mismatches\n", (unsigned long long)n, (unsigned long long)bad);

  /* signed zeros keep their sign */
  uint64_t bad0 = 0;
  for (int i = 0; i < 1000; ++i) {
    const float s = ldexpf(1.0f + (float)(next() % 1000000) / 1e6f, (int)(next() % 207) - 80);
    const float r = 1.0f / s;
    if (f2u(corrected(0.0f, s, r)) != 0u || f2u(corrected(-0.0f, s, r)) != 0x80000000u) bad0++;
  }
  printf("signed zeros: %llu mismatches\n", (unsigned long long)bad0);

  /* random pairs as the kernel forms them: a finite bf16 row maximum amax,
   * s = RN(amax / 448), x a bf16 value with |x| <= amax spread log-uniformly
   * down to the subnormals */
  uint64_t badr = 0, nr = 0, nsmall = 0;
  for (int i = 0; i < 20000000; ++i) {
    const uint32_t abits = (uint32_t)(next() % 0x7F80u) << 16;      /* finite positive bf16 */
    const float amax = u2f(abits);
    const float s = amax / 448.0f;
    if (!(s >= 0x1p-80f && s <= 0x1p126f)) continue;
    float x = amax * ldexpf(1.0f, -(int)(next() % 240)) * (float)(1.0 - (double)(next() % 1000) / 2000.0);
    x = u2f(f2u(x) & 0xFFFF0000u);
    if (next() & 1) x = -x;
    const float r = 1.0f / s;
    const float got = corrected(x, s, r), want = x / s;
    nr++;
    if (f2u(got) == f2u(want)) continue;
    nsmall++;
    const int same_sign = signbit(got) == signbit(x) && signbit(want) == signbit(x);
    if (!(fabsf(got) < 0x1p-10f && fabsf(want) < 0x1p-10f && same_sign)) badr++;
  }
  printf("random: %llu pairs, %llu differ below 2^-10 (same code), %llu mismatches\n",
         (unsigned long long)nr, (unsigned long long)nsmall, (unsigned long long)badr);
  return (bad || bad0 || badr) ? 1 : 0;
}
