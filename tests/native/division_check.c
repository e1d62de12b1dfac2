/* Exhaustive check of the correctly rounded fp32 division used by the
 * quantizer kernel: with y = RN(1/b),
 *     q0 = RN(a*y);  r = RN(a - b*q0) (fused);  q1 = RN(q0 + r*y) (fused)
 * must equal RN(a/b) (Markstein's iteration, e.g. Muller et al.,
 * "Handbook of Floating-Point Arithmetic", correctly rounded division).
 * Scaling a or b by a power of two scales every step exactly (away from
 * underflow/overflow), so significands in [1,2) cover all normal operands:
 *   mode "bf16": a, b with 8-bit significands (x / smooth_factor),
 *   mode "e4m3": a any fp32 significand, b a 4-bit e4m3 significand (x_hat / scale).
 * Prints the number of mismatches. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

static long check(float a, float b) {
  volatile float y = 1.0f / b;
  volatile float q0 = a * y;
  volatile float r = fmaf(-q0, b, a);
  volatile float q1 = fmaf(r, y, q0);
  volatile float ref = a / b;
  return q1 != ref;
}

int main(int argc, char** argv) {
  long bad = 0, n = 0;
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
