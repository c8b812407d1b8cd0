/* The kernels' division of a group's abs-max a by the code range Q (7 for
 * int4, 127 for int8), restated on the host: q0 = a * RN(1/Q), then one
 * residual r = a - Q q0 (an fma, exact), q = q0 + r * RN(1/Q) (an fma),
 * Markstein's division by a known divisor.  Compared with the IEEE quotient
 * a / Q for every non-negative finite float a; prints the number of
 * mismatches per divisor.  Build without contraction (-ffp-contract=off). */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static uint64_t mismatches(float q_div, float z) {
  uint64_t bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
  for (int64_t i = 0; i < 0x7f800000LL; ++i) {
    const float a = from_bits((uint32_t)i);
    const float q0 = a * z;
    const float r = fmaf(-q0, q_div, a);
    const float q = fmaf(r, z, q0);
    if (bits(q) != bits(a / q_div)) ++bad;
  }
  return bad;
}

int main(void) {
  printf("7 %llu\n", (unsigned long long)mismatches(7.0f, 0x1.24924ap-3f));
  printf("127 %llu\n", (unsigned long long)mismatches(127.0f, 0x1.020408p-7f));
  return 0;
}
