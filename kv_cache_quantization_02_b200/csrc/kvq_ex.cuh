// kvq_ex.cuh -- pieces the variant codec's translation units share (the WHT
// variants in kvq_ex.cu, the SRFT in kvq_srft.cu): the kernels' argument
// block, the lambda table of a warp tile and the int8 code packing.  Included
// inside each unit's anonymous namespace, after kvq_arith.cuh.
#pragma once

struct ExArgs {
  const float* lam;                     // [n_lambda][D]
  const int8_t* sgn;                    // [D]
  int64_t n;
  int64_t lambda_rows;
  int n_lambda;
  float c;                              // fp32 1/sqrt(D)
};

// Lambda table of the tile starting at row r0 (every row of a warp tile
// shares it: lambda_rows is a multiple of 32 when there are several tables).
__device__ __forceinline__ int table_id(const ExArgs& a, int64_t r0) {
  return a.n_lambda == 1 ? 0 : static_cast<int>((r0 / a.lambda_rows) % a.n_lambda);
}

// Four codes -> one 32-bit word, code k in byte k, each saturated to [-128, 127].
__device__ __forceinline__ uint32_t pack4_s8(int a0, int a1, int a2, int a3) {
  uint32_t d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a3), "r"(a2), "r"(0u));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a1), "r"(a0), "r"(d));
  return d;
}
