// kvq_arith.cuh -- device arithmetic shared by the codec kernels: 16-byte
// global stores, fp16 <-> fp32 conversions, the packed subtraction, abs-max,
// the scale of a group (a / 7 correctly rounded, 1/S, fp16 saturation), code
// packing, and the in-register Walsh-Hadamard butterflies.  Every rounding
// point is one IEEE operation (the translation units are compiled with
// --fmad=false and the packed f32x2 intrinsics are never contracted).
// Included inside each translation unit's anonymous namespace, after the
// unit defines kFullMask (the full-warp shuffle mask).
#pragma once

__device__ __forceinline__ void st_v4(void* p, const uint32_t (&r)[4]) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};"
               :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]) : "memory");
}


__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}
__device__ __forceinline__ uint32_t float2_to_half2_bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);   // .x (low 16 bits) = lo
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}
// a - b with one rounding: fma(b, -1, a).
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}
// max(a, |b|, |c|)
__device__ __forceinline__ float amax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}

// fp32 quotient a / Q for the code range Q = 7 (int4) or 127 (int8),
// correctly rounded: q0 = a * RN(1/Q), then one residual correction
// r = a - Q q0 (exact by fma), q = q0 + r * RN(1/Q) (Markstein's division by
// a known divisor).  Equal to IEEE a / Q for every non-negative finite fp32
// a, checked exhaustively for both divisors.
template <int Q>
__device__ __forceinline__ float div_const_rn(float a) {
  static_assert(Q == 7 || Q == 127, "divisor checked exhaustively");
  const float z = Q == 7 ? 0x1.24924ap-3f : 0x1.020408p-7f;   // RN(1/Q)
  const float q0 = __fmul_rn(a, z);
  const float r = __fmaf_rn(-q0, static_cast<float>(Q), a);
  return __fmaf_rn(r, z, q0);
}
__device__ __forceinline__ float div7_rn(float a) { return div_const_rn<7>(a); }
// fp32 reciprocal of a positive fp16 value s, correctly rounded: approximate
// reciprocal plus one Newton-Raphson step.  1/s lies at least 2^-35 (relative)
// away from every rounding midpoint because s has an 11-bit significand, far
// beyond the step's error.  kvq_selftest_rcp_f16 evaluates it at every
// positive finite fp16 s so that a test can compare it with IEEE 1/s.
__device__ __forceinline__ float rcp_f16val(float s) {
  float r0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
  const float e = __fmaf_rn(-s, r0, 1.0f);
  return __fmaf_rn(r0, e, r0);
}
// Scale of one group: S = fp16_rne(a / Q) saturated to 65504 (satfinite);
// r = 1/S, or 0 when S = 0 (which makes every code of the group 0).
template <int Q>
__device__ __forceinline__ uint16_t group_scale_q(float a, float& r) {
  uint16_t b;
  asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(b) : "f"(div_const_rn<Q>(a)));
  const float sf = half_bits_to_float(b);
  r = (sf == 0.0f) ? 0.0f : rcp_f16val(sf);
  return b;
}
__device__ __forceinline__ uint16_t group_scale(float a, float& r) { return group_scale_q<7>(a, r); }
// Eight codes -> one 32-bit word, code k in bits [4k, 4k+4), each saturated
// to [-8, 7] by the packing conversion.
__device__ __forceinline__ uint32_t pack8(const int (&q)[8]) {
  uint32_t d;
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q[7]), "r"(q[6]), "r"(0u));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q[5]), "r"(q[4]), "r"(d));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q[3]), "r"(q[2]), "r"(d));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q[1]), "r"(q[0]), "r"(d));
  return d;
}
// w * s for fp16 operands, exact in fp32 (a product of two fp16 values has at
// most 22 significant bits); the -0.0 addend keeps the sign of a zero product.
__device__ __forceinline__ float mul_f16_f32(__half w, uint16_t s) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(__half_as_ushort(w)), "h"(s), "f"(-0.0f));
  return d;
}

// ---------------------------------------------------------------------------
// Walsh-Hadamard butterflies (unnormalised, Sylvester order) on one vector
// held as pairs p[m] = (v[m], v[m+HALF]) by LANES lanes, from half-width H0
// upwards (stages below H0 already applied).  The vector's lanes are XS lane
// ids apart: lane `sub` of the vector is lane rin + XS * sub of the warp.
// ---------------------------------------------------------------------------
template <int EPT, int LANES, int H0 = 1, int XS = 1>
__device__ __forceinline__ void fwht_pairs(float2 (&p)[EPT / 2], int sub) {
  constexpr int NP = EPT / 2;
#pragma unroll
  for (int h = H0; h < NP; h <<= 1) {
#pragma unroll
    for (int m = 0; m < NP; ++m) {
      if ((m & h) == 0) {
        const float2 a = p[m];
        const float2 b = p[m + h];
        p[m] = __fadd2_rn(a, b);
        p[m + h] = fsub2(a, b);
      }
    }
  }
  // h = HALF: the two halves of each pair
#pragma unroll
  for (int m = 0; m < NP; ++m) {
    const float a = p[m].x, b = p[m].y;
    p[m] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  // h = EPT (two lanes per vector): the lower lane keeps a + b, the upper one
  // a_partner - b_own = fma(-1, own, partner).
#pragma unroll
  for (int bit = 1; bit < LANES; bit <<= 1) {
    const float sg = (sub & bit) ? -1.0f : 1.0f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int m = 0; m < NP; ++m) {
      float2 o;
      o.x = __shfl_xor_sync(kFullMask, p[m].x, bit * XS);
      o.y = __shfl_xor_sync(kFullMask, p[m].y, bit * XS);
      p[m] = __ffma2_rn(sg2, p[m], o);
    }
  }
}
