/* Exhaustive check of the correctly rounded fp32 division used by the
 * quantizer kernel: with y = RN(1/b),
 *     q0 = RN(a*y);  r = RN(a - b*q0) (fused);  q1 = RN(q0 + r*y) (fused)
 * must equal RN(a/b) (Markstein's iteration, e.g. Muller et al.,
 * "Handbook of Floating-Point Arithmetic", correctly rounded division).
 * Scaling a or b by a power of two scales every step exactly (away from
 * underflow/overflow), so significands in [1,2) cover all normal operands:
 *   mode "bf16": a, b with 8-bit significands (x / smooth_factor),
 *   mode "e4m3": a any fp32 significand, b a 4-bit e4m3 significand (x_hat / scale).
 *   mode "bf16all": every finite bf16 a (zeros and subnormals included) over
 *     every bf16 b with 2^-100 <= b < 2^128, in the two layouts the kernel
 *     uses (a / b with the sign of q0 kept, and a / -b).  Here the scaling
 *     argument fails where b*q0 - a falls below the normal range, so the
 *     result may miss RN(a/b) by one unit in the last place; the check proves
 *     that this happens only where |RN(a/b)| < 2^-19 and never changes the sign.
 *     Such a quotient gets code +-0 for every scale (a nonzero code needs
 *     |x_hat| >= 0.25 * 2^-9) and, as a block's largest magnitude, scale 0
 *     (amax / 6 < 2^-10), so codes and scales stay exact.  Prints
 *     "checked N mismatches 0 (off-by-ulp below 2^-19: C)".
 *   mode "rr_bf16all": the activation quantizer's two-op division
 *     q = RN(a*yh + RN(a*yl)) with yh = RZ(1/b), yl = RN(1/b - yh) carrying the
 *     sign of yh, for every finite bf16 a over every normal bf16 b with
 *     2^-126 <= |b| < 2^117 (both signs): equal to RN(a/b) except, as above,
 *     by one ulp where |RN(a/b)| < 2^-19 with the same sign.
 *   mode "rr_e4m3": the same two-op division, a any fp32 significand (both
 *     signs), b each of the eight e4m3 significands (x_hat / scale, amax / 6).
 * Prints the number of mismatches. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static long check(float a, float b) {
  volatile float y = 1.0f / b;
  volatile float q0 = a * y;
  volatile float r = fmaf(-q0, b, a);
  volatile float q1 = fmaf(r, y, q0);
  volatile float ref = a / b;
  return q1 != ref;
}

static float qdiv(float a, float b, float y, int keep_q0_sign) {
  volatile float q0 = a * y;
  volatile float r = fmaf(-q0, b, a);
  volatile float q1 = fmaf(r, y, q0);
  if (!keep_q0_sign) return q1;
  uint32_t u1, u0;
  float q1f = q1, q0f = q0;
  memcpy(&u1, &q1f, 4); memcpy(&u0, &q0f, 4);
  u1 = (u1 & 0x7FFFFFFFu) | (u0 & 0x80000000u);
  return f_of(u1);
}

/* 0: exact; 1: off but allowed (tiny, same sign); 2: violation.  Quotients the
 * kernel sends to its IEEE path (|q| >= 3e38 or NaN) are not checked. */
static int classify(float got, float ref) {
  if (!(fabsf(got) < 3.0e38f)) return 0;
  uint32_t ug, ur;
  memcpy(&ug, &got, 4); memcpy(&ur, &ref, 4);
  if (ug == ur) return 0;
  if (fabsf(ref) < 0x1p-19f && ((ug ^ ur) & 0x80000000u) == 0) return 1;
  return 2;
}

/* {RZ(1/b), RN(1/b - RZ(1/b)) with the sign of the first}. */
static void recip_pair(float b, float* yh, float* yl) {
  const double inv = 1.0 / (double)b;
  float h = (float)inv;
  if (fabs((double)h) > fabs(inv)) h = nextafterf(h, 0.0f);
  *yh = h;
  *yl = copysignf(fabsf((float)(inv - (double)h)), h);
}

static float rr_div(float a, float yh, float yl) {
  volatile float p = a * yl;
  volatile float q = fmaf(a, yh, p);
  return q;
}

int main(int argc, char** argv) {
  long bad = 0, n = 0;
  if (argc > 1 && strcmp(argv[1], "rr_bf16all") == 0) {
    long tiny = 0;
#pragma omp parallel for reduction(+ : bad, n, tiny) schedule(dynamic, 16)
    for (uint32_t bb = 1u << 7; bb < 0xFF80u; ++bb) {
      if ((bb & 0x7FFFu) < 0x0080u || (bb & 0x7FFFu) >= ((127u + 117u) << 7)) continue;  /* |b| in [2^-126, 2^117) */
      const float b = f_of(bb << 16);
      float yh, yl;
      recip_pair(b, &yh, &yl);
      for (uint32_t ab = 0; ab < 0x10000u; ++ab) {
        if (((ab >> 7) & 0xFFu) == 0xFFu) continue;
        const float a = f_of(ab << 16);
        const int c = classify(rr_div(a, yh, yl), a / b);
        bad += c == 2;
        tiny += c == 1;
        n += 1;
      }
    }
    printf("checked %ld mismatches %ld (off-by-ulp below 2^-19: %ld)\n", n, bad, tiny);
    return bad != 0;
  }
  if (argc > 1 && strcmp(argv[1], "rr_e4m3") == 0) {
    for (uint32_t mb = 0; mb < 8; ++mb) {
      const float b = 1.0f + mb / 8.0f;
      float yh, yl;
      recip_pair(b, &yh, &yl);
#pragma omp parallel for reduction(+ : bad, n)
      for (uint32_t ma = 0; ma < (1u << 23); ++ma) {
        const float a = f_of(0x3F800000u | ma);
        bad += u_of(rr_div(a, yh, yl)) != u_of(a / b);
        bad += u_of(rr_div(-a, yh, yl)) != u_of(-a / b);
        n += 2;
      }
    }
    printf("checked %ld mismatches %ld\n", n, bad);
    return bad != 0;
  }
  if (argc > 1 && strcmp(argv[1], "bf16all") == 0) {
    long tiny = 0;
#pragma omp parallel for reduction(+ : bad, n, tiny) schedule(dynamic, 16)
    for (uint32_t bb = (127u - 100u) << 7; bb < 0x7F80u; ++bb) {
      const float b = f_of(bb << 16);
      const float y = 1.0f / b;
      for (uint32_t ab = 0; ab < 0x10000u; ++ab) {
        if (((ab >> 7) & 0xFFu) == 0xFFu) continue;            /* inf / NaN inputs */
        const float a = f_of(ab << 16);
        const int c1 = classify(qdiv(a, b, y, 1), a / b);
        const int c2 = classify(qdiv(a, -b, -y, 0), a / -b);
        bad += (c1 == 2) + (c2 == 2);
        tiny += (c1 == 1) + (c2 == 1);
        n += 2;
      }
    }
    printf("checked %ld mismatches %ld (off-by-ulp below 2^-19: %ld)\n", n, bad, tiny);
    return bad != 0;
  }
  if (argc > 1 && strcmp(argv[1], "bf16") == 0) {
    for (uint32_t ma = 0; ma < 128; ++ma)
      for (uint32_t mb = 0; mb < 128; ++mb) {
        float a = f_of(0x3F800000u | (ma << 16)), b = f_of(0x3F800000u | (mb << 16));
        bad += check(a, b); bad += check(-a, b); n += 2;
      }
  } else {
    for (uint32_t mb = 0; mb < 8; ++mb) {
      float b = 1.0f + mb / 8.0f;
      for (uint32_t ma = 0; ma < (1u << 23); ++ma) {
        float a = f_of(0x3F800000u | ma);
        bad += check(a, b); ++n;
      }
    }
  }
  printf("checked %ld mismatches %ld\n", n, bad);
  return bad != 0;
}
