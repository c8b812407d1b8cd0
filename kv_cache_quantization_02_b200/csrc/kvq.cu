// kvq.cu -- fused KV-cache rotate-and-quantize for B200 (sm_100a):
// kernels and the C-ABI launcher declared in include/kvq.h.
//
// Method: "When Quantization Is Free: An int4 KV Cache That Outruns fp16 on
// Apple Silicon" (arXiv 2605.05699), Abstract, and its technical summary
// (gist.science), Methodologie 1-3: per vector, sign-multiply, orthogonal
// transform, per-channel lambda, per-group abs-max, round to signed int4,
// pack two codes per byte.  Transform = SRHT (random +-1 signs, then the
// normalised Walsh-Hadamard transform), which the Abstract reports to be
// indistinguishable in quality from the paper's SRFT.  lambda is applied
// before the rotation and removed last on the inverse, the order of "The
// Kernel That Finally Did Something" (VeloxQuant-MLX blog), "The kernel
// toggle".
//
// Work decomposition.  A vector of D fp16 channels is owned by a team of
// LANES = D/32 consecutive lanes of one warp; lane `sub` of the team holds
// channels [32*sub, 32*sub + 32) in registers as 16 packed fp32 pairs
// p[m] = (v[m], v[m+16]), m = 0..15.  The butterfly with half-width h then
// runs as
//   h = 1, 2, 4, 8   : packed f32x2 adds/subs between pairs p[m], p[m+h];
//   h = 16           : inside each pair;
//   h = 32 .. D/2    : across the team's lanes with __shfl_xor_sync, one
//                      fused multiply-add by +-1 per element.
// Every butterfly output is one IEEE fp32 a+b or a-b of the same operands, in
// the same ascending-h order as the plain sequential loop, so the result is
// bit-identical to it.  Loads and stores are 256-bit (one full 32-byte
// sector per lane); a warp covers 32/LANES vectors per iteration and walks a
// grid-stride loop, so every lane executes every shuffle.
//
// This translation unit is compiled with --fmad=false and uses only _rn
// intrinsics on the contract-sensitive steps, so no multiply is ever fused
// into a following add.

#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "kvq.h"

namespace {

constexpr int kThreads = 256;          // threads per block (8 warps)
constexpr int kChunk = 32;             // channels per lane
constexpr unsigned kFullMask = 0xffffffffu;
constexpr int kMaxDevices = 64;

thread_local int g_last_cuda_error = 0;

// ---------------------------------------------------------------------------
// Memory access helpers (256-bit where a lane moves a whole 32-byte sector).
// ---------------------------------------------------------------------------

__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&r)[8]) {
  asm("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]),
        "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "l"(p));
}

__device__ __forceinline__ void ld_nc_v4(const void* p, uint32_t (&r)[4]) {
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "l"(p));
}

__device__ __forceinline__ void st_v8(void* p, const uint32_t (&r)[8]) {
  asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]),
                  "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void st_v4(void* p, const uint32_t (&r)[4]) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};"
               :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
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

// a - b as one rounding: fma(b, -1, a).
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// ---------------------------------------------------------------------------
// Unnormalised Walsh-Hadamard transform of one vector held by a team of
// LANES lanes, 32 channels per lane as pairs p[m] = (v[m], v[m+16]).
// Stages in ascending half-width h = 1 .. D/2.
// ---------------------------------------------------------------------------

template <int LANES>
__device__ __forceinline__ void fwht_team(float2 (&p)[16], int sub) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      if ((m & h) == 0) {
        const float2 a = p[m];
        const float2 b = p[m + h];
        p[m] = __fadd2_rn(a, b);
        p[m + h] = fsub2(a, b);
      }
    }
  }
  // h = 16: the two halves of each pair.
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const float a = p[m].x, b = p[m].y;
    p[m] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  // h = 32 .. 16*LANES: partner lane sub ^ bit.  The lower partner keeps
  // a + b, the upper one b_partner - a_own = fma(-1, own, partner).
#pragma unroll
  for (int bit = 1; bit < LANES; bit <<= 1) {
    const float sg = (sub & bit) ? -1.0f : 1.0f;
    const float2 sg2 = make_float2(sg, sg);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      float2 o;
      o.x = __shfl_xor_sync(kFullMask, p[m].x, bit);
      o.y = __shfl_xor_sync(kFullMask, p[m].y, bit);
      p[m] = __ffma2_rn(sg2, p[m], o);
    }
  }
}

// Per-channel constant table laid out so that lane `sub` reads its pairs
// (p[2j], p[2j+1]) as one float4 at [j][sub]: conflict-free across subs.
template <int LANES>
__device__ __forceinline__ void fill_pair_table(float4 (*tab)[LANES],
                                                const float* __restrict__ lam,
                                                const int8_t* __restrict__ sg,
                                                bool reciprocal) {
  for (int i = threadIdx.x; i < 8 * LANES; i += blockDim.x) {
    const int j = i / LANES, sub = i % LANES;
    const int base = kChunk * sub + 2 * j;
    const int ch[4] = {base, base + 16, base + 1, base + 17};
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float l = lam[ch[k]];
      if (reciprocal) l = __frcp_rn(l);          // fp32 IEEE 1/lambda
      v[k] = (sg[ch[k]] < 0) ? -l : l;           // exact sign flip
    }
    tab[j][sub] = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// Scale of one group: S = fp16_rne(a / 7) saturated to 65504; r = 1/S
// (r = 0 when S = 0, which makes every code of the group 0).
__device__ __forceinline__ uint16_t group_scale(float a, float& r) {
  const float q = __fdiv_rn(a, 7.0f);
  uint16_t b = __half_as_ushort(__float2half_rn(q));
  if (b == 0x7C00u) b = 0x7BFFu;
  const float sf = half_bits_to_float(b);
  r = (sf == 0.0f) ? 0.0f : __frcp_rn(sf);
  return b;
}

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

// Signed 4-bit field k of w, sign-extended.
__device__ __forceinline__ int nibble(uint32_t w, int k) {
  return static_cast<int>(w << (28 - 4 * k)) >> 28;
}

// ---------------------------------------------------------------------------
// Quantize: fp16 [n][D] -> packed u8 [n][D/2] + fp16 scales [n][D/G].
// ---------------------------------------------------------------------------

template <int D, int G>
__global__ void __launch_bounds__(kThreads)
kvq_quantize_kernel(const uint16_t* __restrict__ x,
                    const float* __restrict__ lam,
                    const int8_t* __restrict__ sgn,
                    int64_t n, float c,
                    uint8_t* __restrict__ packed,
                    uint16_t* __restrict__ scales) {
  constexpr int LANES = D / kChunk;
  constexpr int VPW = 32 / LANES;                 // vectors per warp
  constexpr int GPL = G / kChunk;                 // lanes per group (G >= 32)
  __shared__ float4 ls_tab[8][LANES];             // lambda * s, paired
  fill_pair_table<LANES>(ls_tab, lam, sgn, false);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int sub = lane % LANES;
  const int team = lane / LANES;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const float2 c2 = make_float2(c, c);

  for (int64_t base = warp * VPW; base < n; base += nwarps * VPW) {
    const int64_t row = base + team;
    const bool active = row < n;
    const int64_t rrow = active ? row : n - 1;

    // a1: load 32 fp16 channels, widen, multiply by lambda*s (one rounding).
    const uint16_t* src = x + rrow * D + sub * kChunk;
    uint32_t w[16];
    {
      uint32_t lo[8], hi[8];
      ld_nc_v8(src, lo);
      ld_nc_v8(src + 16, hi);
#pragma unroll
      for (int j = 0; j < 8; ++j) { w[j] = lo[j]; w[8 + j] = hi[j]; }
    }
    float2 p[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 a = half2_bits_to_float2(w[j]);       // channels 2j, 2j+1
      const float2 b = half2_bits_to_float2(w[8 + j]);   // channels 2j+16, 2j+17
      const float4 t = ls_tab[j][sub];
      p[2 * j] = __fmul2_rn(make_float2(a.x, b.x), make_float2(t.x, t.y));
      p[2 * j + 1] = __fmul2_rn(make_float2(a.y, b.y), make_float2(t.z, t.w));
    }

    // a2: transform; a3: normalise.
    fwht_team<LANES>(p, sub);
#pragma unroll
    for (int m = 0; m < 16; ++m) p[m] = __fmul2_rn(p[m], c2);

    // a4: group abs-max.  .x holds channels 0..15 of the chunk, .y 16..31.
    float ax = 0.0f, ay = 0.0f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      ax = fmaxf(ax, fabsf(p[m].x));
      ay = fmaxf(ay, fabsf(p[m].y));
    }
    float rx, ry;
    uint16_t sbx, sby = 0;
    if constexpr (G == 16) {
      sbx = group_scale(ax, rx);
      sby = group_scale(ay, ry);
    } else {
      float a = fmaxf(ax, ay);
#pragma unroll
      for (int bit = 1; bit < GPL; bit <<= 1)
        a = fmaxf(a, __shfl_xor_sync(kFullMask, a, bit));
      sbx = group_scale(a, rx);
      ry = rx;
    }

    // a6: codes = rint(y * r), saturated to [-8, 7] while packing (a7).
    const float2 r2 = make_float2(rx, ry);
    int qx[16], qy[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float2 t = __fmul2_rn(p[m], r2);
      qx[m] = __float2int_rn(t.x);
      qy[m] = __float2int_rn(t.y);
    }
    uint32_t out[4];
    {
      int q8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) q8[k] = qx[k];
      out[0] = pack8(q8);
#pragma unroll
      for (int k = 0; k < 8; ++k) q8[k] = qx[8 + k];
      out[1] = pack8(q8);
#pragma unroll
      for (int k = 0; k < 8; ++k) q8[k] = qy[k];
      out[2] = pack8(q8);
#pragma unroll
      for (int k = 0; k < 8; ++k) q8[k] = qy[8 + k];
      out[3] = pack8(q8);
    }
    if (active) {
      st_v4(packed + row * (D / 2) + sub * 16, out);
      uint16_t* srow = scales + row * (D / G);
      if constexpr (G == 16) {
        srow[2 * sub] = sbx;
        srow[2 * sub + 1] = sby;
      } else if constexpr (G == 32) {
        srow[sub] = sbx;
      } else {
        if (sub % GPL == 0) srow[sub / GPL] = sbx;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Dequantize: packed u8 [n][D/2] + fp16 scales [n][D/G] -> fp16 [n][D].
// ---------------------------------------------------------------------------

template <int D, int G>
__global__ void __launch_bounds__(kThreads)
kvq_dequantize_kernel(const uint8_t* __restrict__ packed,
                      const uint16_t* __restrict__ scales,
                      const float* __restrict__ lam,
                      const int8_t* __restrict__ sgn,
                      int64_t n, float c,
                      uint16_t* __restrict__ x_out) {
  constexpr int LANES = D / kChunk;
  constexpr int VPW = 32 / LANES;
  constexpr int GPL = G / kChunk;
  __shared__ float4 sil_tab[8][LANES];            // s / lambda, paired
  fill_pair_table<LANES>(sil_tab, lam, sgn, true);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int sub = lane % LANES;
  const int team = lane / LANES;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const float2 c2 = make_float2(c, c);

  for (int64_t base = warp * VPW; base < n; base += nwarps * VPW) {
    const int64_t row = base + team;
    const bool active = row < n;
    const int64_t rrow = active ? row : n - 1;

    // a8: 16 bytes of codes (channels 32*sub .. +31) and their scales.
    uint32_t w[4];
    ld_nc_v4(packed + rrow * (D / 2) + sub * 16, w);
    const uint16_t* srow = scales + rrow * (D / G);
    float sx, sy;
    if constexpr (G == 16) {
      sx = half_bits_to_float(srow[2 * sub]);
      sy = half_bits_to_float(srow[2 * sub + 1]);
    } else {
      sx = half_bits_to_float(srow[sub / GPL]);
      sy = sx;
    }
    const float2 s2 = make_float2(sx, sy);
    float2 p[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const float qa = __int2float_rn(nibble(w[m / 8], m % 8));
      const float qb = __int2float_rn(nibble(w[2 + m / 8], m % 8));
      p[m] = __fmul2_rn(make_float2(qa, qb), s2);       // exact
    }

    // a9: inverse rotation (same transform), normalise; a10: s / lambda.
    fwht_team<LANES>(p, sub);
    uint32_t o[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 t = sil_tab[j][sub];
      const float2 a = __fmul2_rn(__fmul2_rn(p[2 * j], c2), make_float2(t.x, t.y));
      const float2 b = __fmul2_rn(__fmul2_rn(p[2 * j + 1], c2), make_float2(t.z, t.w));
      o[j] = float2_to_half2_bits(a.x, b.x);         // channels 2j, 2j+1
      o[8 + j] = float2_to_half2_bits(a.y, b.y);     // channels 2j+16, 2j+17
    }
    if (active) {
      uint16_t* dst = x_out + row * D + sub * kChunk;
      uint32_t lo[8], hi[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) { lo[j] = o[j]; hi[j] = o[8 + j]; }
      st_v8(dst, lo);
      st_v8(dst + 16, hi);
    }
  }
}

// ---------------------------------------------------------------------------
// Launch plumbing.
// ---------------------------------------------------------------------------

struct DeviceInfo {
  std::atomic<int> sms{0};
};
DeviceInfo g_dev[kMaxDevices];

int sm_count(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = g_dev[dev].sms.load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_dev[dev].sms.store(v, std::memory_order_relaxed);
  }
  return v;
}

template <typename Kernel>
int blocks_per_sm(Kernel k, int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 1;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k, kThreads, 0) != cudaSuccess || v < 1)
      v = 1;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

template <typename Kernel>
int grid_for(Kernel k, int64_t n, int D) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const int64_t per_block = static_cast<int64_t>(kThreads / 32) * (32 / (D / kChunk));
  const int64_t need = (n + per_block - 1) / per_block;
  int64_t cap = static_cast<int64_t>(sm_count(dev)) * blocks_per_sm(k, dev);
  if (cap < 1) cap = 1;
  return static_cast<int>(need < cap ? need : cap);
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

int check_shape(int D, int G, int64_t n) {
  if (D != 64 && D != 128 && D != 256) return KVQ_ERR_DIM;
  if (G < 16 || G > D || (G & (G - 1)) != 0) return KVQ_ERR_GROUP;
  if (n < 0) return KVQ_ERR_COUNT;
  return KVQ_OK;
}

float norm_const(int D) { return static_cast<float>(1.0 / std::sqrt(static_cast<double>(D))); }

int finish_launch() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(e);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
}

template <int D, int G>
int launch_quantize(const uint16_t* x, const float* lam, const int8_t* s, int64_t n,
                    uint8_t* packed, uint16_t* scales, cudaStream_t st) {
  auto k = kvq_quantize_kernel<D, G>;
  const int grid = grid_for(k, n, D);
  (void)cudaGetLastError();
  k<<<grid, kThreads, 0, st>>>(x, lam, s, n, norm_const(D), packed, scales);
  return finish_launch();
}

template <int D, int G>
int launch_dequantize(const uint8_t* packed, const uint16_t* scales, const float* lam,
                      const int8_t* s, int64_t n, uint16_t* out, cudaStream_t st) {
  auto k = kvq_dequantize_kernel<D, G>;
  const int grid = grid_for(k, n, D);
  (void)cudaGetLastError();
  k<<<grid, kThreads, 0, st>>>(packed, scales, lam, s, n, norm_const(D), out);
  return finish_launch();
}

#define KVQ_DISPATCH(FN, D, G, ...)                                              \
  do {                                                                           \
    switch (D) {                                                                 \
      case 64:                                                                   \
        switch (G) {                                                             \
          case 16: return FN<64, 16>(__VA_ARGS__);                               \
          case 32: return FN<64, 32>(__VA_ARGS__);                               \
          case 64: return FN<64, 64>(__VA_ARGS__);                               \
        }                                                                        \
        break;                                                                   \
      case 128:                                                                  \
        switch (G) {                                                             \
          case 16: return FN<128, 16>(__VA_ARGS__);                              \
          case 32: return FN<128, 32>(__VA_ARGS__);                              \
          case 64: return FN<128, 64>(__VA_ARGS__);                              \
          case 128: return FN<128, 128>(__VA_ARGS__);                            \
        }                                                                        \
        break;                                                                   \
      case 256:                                                                  \
        switch (G) {                                                             \
          case 16: return FN<256, 16>(__VA_ARGS__);                              \
          case 32: return FN<256, 32>(__VA_ARGS__);                              \
          case 64: return FN<256, 64>(__VA_ARGS__);                              \
          case 128: return FN<256, 128>(__VA_ARGS__);                            \
          case 256: return FN<256, 256>(__VA_ARGS__);                            \
        }                                                                        \
        break;                                                                   \
    }                                                                            \
    return KVQ_ERR_GROUP;                                                        \
  } while (0)

}  // namespace

extern "C" {

int kvq_quantize(const uint16_t* x, const float* lambda, const int8_t* signs,
                 int64_t n_vec, int D, int group, uint8_t* packed, uint16_t* scales,
                 void* stream) {
  const int rc = check_shape(D, group, n_vec);
  if (rc != KVQ_OK) return rc;
  if (n_vec == 0) return KVQ_OK;
  if (!x || !lambda || !signs || !packed || !scales) return KVQ_ERR_NULL;
  if (!aligned(x, 32) || !aligned(packed, 16) || !aligned(scales, 2) || !aligned(lambda, 4))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_DISPATCH(launch_quantize, D, group, x, lambda, signs, n_vec, packed, scales, st);
}

int kvq_dequantize(const uint8_t* packed, const uint16_t* scales, const float* lambda,
                   const int8_t* signs, int64_t n_vec, int D, int group, uint16_t* x_out,
                   void* stream) {
  const int rc = check_shape(D, group, n_vec);
  if (rc != KVQ_OK) return rc;
  if (n_vec == 0) return KVQ_OK;
  if (!packed || !scales || !lambda || !signs || !x_out) return KVQ_ERR_NULL;
  if (!aligned(x_out, 32) || !aligned(packed, 16) || !aligned(scales, 2) || !aligned(lambda, 4))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_DISPATCH(launch_dequantize, D, group, packed, scales, lambda, signs, n_vec, x_out, st);
}

const char* kvq_status_string(int status) {
  switch (status) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_NULL: return "KVQ_ERR_NULL: a required pointer is NULL";
    case KVQ_ERR_ALIGN: return "KVQ_ERR_ALIGN: a pointer is misaligned";
    case KVQ_ERR_DIM: return "KVQ_ERR_DIM: D must be 64, 128 or 256";
    case KVQ_ERR_GROUP: return "KVQ_ERR_GROUP: group must be a power of two in [16, D]";
    case KVQ_ERR_COUNT: return "KVQ_ERR_COUNT: n_vec must be >= 0";
    case KVQ_ERR_LAUNCH: return "KVQ_ERR_LAUNCH: the kernel launch failed";
    default: return "unknown kvq status";
  }
}

int kvq_last_cuda_error(void) { return g_last_cuda_error; }

int kvq_version(void) { return (1 << 16) | 0; }

}  // extern "C"
