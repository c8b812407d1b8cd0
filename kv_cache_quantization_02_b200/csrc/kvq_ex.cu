// kvq_ex.cu -- format variants of the KV-cache codec for B200 (sm_100a):
// kernels and the C-ABI launcher of kvq_quantize_ex / kvq_dequantize_ex
// (include/kvq.h).
//
// The same per-vector method as the base codec ("When Quantization Is Free",
// technical summary, Methodologie 1-3: random signs, Walsh-Hadamard rotation,
// per-channel lambda, per-group abs-max, round to signed integers, pack), with
// three options:
//   * lambda after the rotation: y = lambda . (H diag(s) x) / sqrt(D), the
//     order of the summary's step list (transform of diag(s) x, then the
//     per-channel lambda rescale), besides the VecInfer order of the base
//     codec ("The Kernel That Finally Did Something", "What VecInfer does");
//   * 8-bit codes: S = fp16(max|y| / 127), q in [-128, 127], one byte each;
//   * one lambda table per range of rows: row r uses table
//     (r / lambda_rows) % n_lambda (per-(layer, head) smoothing).
// D = 128; G in {16, 32, 64}.  One lane holds a whole vector as 64 packed
// fp32 pairs (v[m], v[m+64]); each warp streams 32-vector tiles through its
// own double-buffered ring (fp16 rows by swizzled tensor copies, codes and
// scales by bulk copies), and the warps of a block claim tiles from a shared
// counter.  A warp tile lies inside one lambda table (lambda_rows is a
// multiple of 32 when there are several), so the warp rebuilds its per-channel
// table in shared memory when a tile's table differs from the last one's.
// Every step is the oracle's IEEE operation in the oracle's order: the scale is
// a correctly rounded division by 7 or 127, 1/S and 1/lambda correctly rounded
// reciprocals, so results are bit-identical.  Bounded waits as in the base
// kernels (a warp that gives up sets bit 0 of the fault word and returns).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "kvq.h"

namespace {

constexpr unsigned kFullMask = 0xffffffffu;

#include "kvq_async.cuh"
#include "kvq_arith.cuh"

constexpr int kD = 128;                 // channels (one lane per vector)
constexpr int kNP = kD / 2;             // packed pairs (v[m], v[m+64])
constexpr int kXW = 4;                  // warps per block
constexpr int kWR = 32;                 // vectors per warp tile
constexpr int kQB = kWR * 128;          // bytes of one 64-channel quarter of a tile
constexpr int kXStage = 2 * kQB;        // bytes of one fp16 warp tile
constexpr uint32_t kSpinX = 1u << 22;

__device__ unsigned int g_ex_fault = 0;   // bit 0: a bounded wait gave up
thread_local int g_ex_cuda_error = 0;

struct ExMaps {
  CUtensorMap q[2];                     // fp16 rows: two 64-channel quarters
};

struct ExArgs {
  const float* lam;                     // [n_lambda][128]
  const int8_t* sgn;                    // [128]
  int64_t n;
  int64_t lambda_rows;
  int n_lambda;
  float c;                              // fp32 1/sqrt(128)
};

template <int BITS>
struct Fmt {
  static constexpr int CB = BITS == 4 ? kD / 2 : kD;   // code bytes per row
  static constexpr float QMAX = BITS == 4 ? 7.0f : 127.0f;
};

__device__ __forceinline__ int xtile_off(int q, int t, int c) {
  return q * kQB + t * 128 + ((c ^ (t & 7)) << 4);
}

// Table of the tile starting at row r0 (all 32 rows share it).
__device__ __forceinline__ int table_id(const ExArgs& a, int64_t r0) {
  return a.n_lambda == 1 ? 0 : static_cast<int>((r0 / a.lambda_rows) % a.n_lambda);
}

// The warp's per-channel table in the pair layout of the base kernels:
// tab[q] = (t[2q], t[2q+64], t[2q+1], t[2q+65]); mode 0: lambda * s,
// 1: lambda, 2: s * (1/lambda), 3: 1/lambda.  Each lane fills one float4.
__device__ __forceinline__ void build_table(float4* tab, const ExArgs& a, int id, int mode, int lane) {
  const float* lr = a.lam + static_cast<int64_t>(id) * kD;
  const int ch[4] = {2 * lane, 2 * lane + kNP, 2 * lane + 1, 2 * lane + 1 + kNP};
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float l = lr[ch[k]];
    if (mode >= 2) l = __frcp_rn(l);
    v[k] = ((mode == 0 || mode == 2) && a.sgn[ch[k]] < 0) ? -l : l;
  }
  tab[lane] = make_float4(v[0], v[1], v[2], v[3]);
}

// The block's sign table in the same layout, as +-1.0f.
__device__ __forceinline__ void build_signs(float4* stab, const ExArgs& a, int q) {
  const int ch[4] = {2 * q, 2 * q + kNP, 2 * q + 1, 2 * q + 1 + kNP};
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = a.sgn[ch[k]] < 0 ? -1.0f : 1.0f;
  stab[q] = make_float4(v[0], v[1], v[2], v[3]);
}

// Header of a block: per-warp tables (kXW x 512 B), the sign table (512 B),
// then two mbarriers and two tile ids per warp and the claim counter.
constexpr int kHdrBars = kXW * 512 + 512;
constexpr int kHdrBytes = kHdrBars + 24 * kXW + 16;

// Four codes -> one 32-bit word, code k in byte k, each saturated to [-128, 127].
__device__ __forceinline__ uint32_t pack4_s8(int a0, int a1, int a2, int a3) {
  uint32_t d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a3), "r"(a2), "r"(0u));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a1), "r"(a0), "r"(d));
  return d;
}

// ---------------------------------------------------------------------------
// Quantize variants: fp16 [n][128] -> codes [n][CB] + fp16 scales [n][128/G].
// ---------------------------------------------------------------------------
template <int G, int BITS, bool AFTER>
__global__ void __launch_bounds__(kXW * 32, 3)
kvq_quantize_ex_kernel(const __grid_constant__ ExMaps maps, const ExArgs a,
                       uint8_t* __restrict__ codes, uint16_t* __restrict__ scales) {
  using F = Fmt<BITS>;
  constexpr int NGH = kNP / G;          // groups per half of the lane's channels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* wsm = smem + warp * 2 * kXStage;
  uint8_t* hdr = smem + kXW * 2 * kXStage;
  float4* tab = reinterpret_cast<float4*>(hdr) + warp * 32;                       // 512 B per warp
  float4* stab = reinterpret_cast<float4*>(hdr + kXW * 512);                        // +-1, 512 B
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + kHdrBars) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + kHdrBars + 16 * kXW) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + kHdrBars + 24 * kXW);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  if (tid < 32) build_signs(stab, a, tid);
  __syncthreads();

  const int64_t ntiles = (a.n + kWR - 1) / kWR;
  const unsigned int mine = static_cast<unsigned int>((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(blockIdx.x + i * gridDim.x) : -1;
  };
  auto refill = [&](int stage) {
    const int t = claim();
    if (lane == 0) tq[stage] = t;
    if (t < 0 || lane != 0) return;
    mbar_expect_tx(&bar[stage], kXStage);
    tensor_g2s(wsm + stage * kXStage, &maps.q[0], 0, t * kWR, &bar[stage]);
    tensor_g2s(wsm + stage * kXStage + kQB, &maps.q[1], 0, t * kWR, &bar[stage]);
  };
  refill(0);
  refill(1);
  const float2 c2 = make_float2(a.c, a.c);
  int cached = -1;
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinX);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_ex_fault, 1u);
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinX);
      return;
    }
    const int id = table_id(a, tile * kWR);
    if (id != cached) {                 // warp-uniform
      build_table(tab, a, id, AFTER ? 1 : 0, lane);
      cached = id;
      __syncwarp();
    }
    const int64_t row = tile * kWR + lane;
    const bool active = row < a.n;
    const uint8_t* st = wsm + stage * kXStage;
    float2 p[kNP];
#pragma unroll
    for (int j = 0; j < kNP / 8; ++j) {
      const int ea = 8 * j, eb = kNP + 8 * j;
      const uint4 xa = *reinterpret_cast<const uint4*>(st + xtile_off(ea / 64, lane, (ea % 64) / 8));
      const uint4 xb = *reinterpret_cast<const uint4*>(st + xtile_off(eb / 64, lane, (eb % 64) / 8));
      const uint32_t aw[4] = {xa.x, xa.y, xa.z, xa.w}, bw[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 fa = half2_bits_to_float2(aw[t]);
        const float2 fb = half2_bits_to_float2(bw[t]);
        if constexpr (!AFTER) {
          const float4 l = tab[4 * j + t];            // lambda * s
          p[8 * j + 2 * t] = __fmul2_rn(make_float2(fa.x, fb.x), make_float2(l.x, l.y));
          p[8 * j + 2 * t + 1] = __fmul2_rn(make_float2(fa.y, fb.y), make_float2(l.z, l.w));
        } else {                                      // signs only: exact
          const float4 sg = stab[4 * j + t];
          p[8 * j + 2 * t] = __fmul2_rn(make_float2(fa.x, fb.x), make_float2(sg.x, sg.y));
          p[8 * j + 2 * t + 1] = __fmul2_rn(make_float2(fa.y, fb.y), make_float2(sg.z, sg.w));
        }
      }
    }
    __syncwarp();                       // the tile is in registers: refill its stage
    refill(stage);

    fwht_pairs<kD, 1>(p, 0);
#pragma unroll
    for (int m = 0; m < kNP; ++m) p[m] = __fmul2_rn(p[m], c2);
    if constexpr (AFTER) {
#pragma unroll
      for (int q = 0; q < kNP / 2; ++q) {
        const float4 l = tab[q];                      // lambda
        p[2 * q] = __fmul2_rn(p[2 * q], make_float2(l.x, l.y));
        p[2 * q + 1] = __fmul2_rn(p[2 * q + 1], make_float2(l.z, l.w));
      }
    }
    // group abs-max, scale S = fp16(a / QMAX) (saturating), r = 1/S
    float rx[NGH], ry[NGH];
    uint16_t bx[NGH], by[NGH];
#pragma unroll
    for (int j = 0; j < NGH; ++j) {
      float ax = 0.f, ay = 0.f;
#pragma unroll
      for (int m = 0; m < G; m += 2) {
        ax = amax3(ax, p[j * G + m].x, p[j * G + m + 1].x);
        ay = amax3(ay, p[j * G + m].y, p[j * G + m + 1].y);
      }
      asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(bx[j]) : "f"(__fdiv_rn(ax, F::QMAX)));
      asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(by[j]) : "f"(__fdiv_rn(ay, F::QMAX)));
      const float sx = half_bits_to_float(bx[j]), sy = half_bits_to_float(by[j]);
      rx[j] = sx == 0.0f ? 0.0f : __frcp_rn(sx);
      ry[j] = sy == 0.0f ? 0.0f : __frcp_rn(sy);
    }
    // codes = rint(y * r), saturated by the packing conversion
    uint32_t out[F::CB / 4];
    if constexpr (BITS == 4) {
#pragma unroll
      for (int k8 = 0; k8 < kNP / 8; ++k8) {
        int qa[8], qb[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int m = 8 * k8 + t;
          const float2 v = __fmul2_rn(p[m], make_float2(rx[m / G], ry[m / G]));
          qa[t] = __float2int_rn(v.x);
          qb[t] = __float2int_rn(v.y);
        }
        out[k8] = pack8(qa);
        out[k8 + kNP / 8] = pack8(qb);
      }
    } else {
#pragma unroll
      for (int k4 = 0; k4 < kNP / 4; ++k4) {
        int qa[4], qb[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int m = 4 * k4 + t;
          const float2 v = __fmul2_rn(p[m], make_float2(rx[m / G], ry[m / G]));
          qa[t] = __float2int_rn(v.x);
          qb[t] = __float2int_rn(v.y);
        }
        out[k4] = pack4_s8(qa[0], qa[1], qa[2], qa[3]);
        out[k4 + kNP / 4] = pack4_s8(qb[0], qb[1], qb[2], qb[3]);
      }
    }
    if (active) {
      uint8_t* dst = codes + row * F::CB;
#pragma unroll
      for (int k4 = 0; k4 < F::CB / 16; ++k4) {
        const uint32_t t4[4] = {out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3]};
        st_v4(dst + 16 * k4, t4);
      }
      uint16_t* srow = scales + row * (kD / G);
#pragma unroll
      for (int j = 0; j < NGH; ++j) {
        srow[j] = bx[j];
        srow[NGH + j] = by[j];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Dequantize variants: codes [n][CB] + fp16 scales [n][128/G] -> fp16 [n][128].
// ---------------------------------------------------------------------------
template <int G, int BITS>
struct DeqLayout {
  static constexpr int WC = kWR * Fmt<BITS>::CB;          // codes of one warp tile
  static constexpr int SPR = (kD / G) * 2;                // scale bytes per row
  static constexpr int WS = kWR * SPR;                    // scales of one warp tile (<= 512)
  static constexpr int STAGE = WC + WS;
  static constexpr int WARP = 2 * STAGE;
};

template <int G, int BITS, bool AFTER>
__global__ void __launch_bounds__(kXW * 32, 2)
kvq_dequantize_ex_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                         const ExArgs a, uint16_t* __restrict__ out, int scale_copy) {
  using F = Fmt<BITS>;
  using L = DeqLayout<G, BITS>;
  constexpr int NGH = kNP / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* wsm = smem + warp * L::WARP;
  uint8_t* hdr = smem + kXW * L::WARP;
  float4* tab = reinterpret_cast<float4*>(hdr) + warp * 32;
  float4* stab = reinterpret_cast<float4*>(hdr + kXW * 512);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + kHdrBars) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + kHdrBars + 16 * kXW) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + kHdrBars + 24 * kXW);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  if (tid < 32) build_signs(stab, a, tid);
  __syncthreads();

  const int64_t ntiles = (a.n + kWR - 1) / kWR;
  const unsigned int mine = static_cast<unsigned int>((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(blockIdx.x + i * gridDim.x) : -1;
  };
  auto scale_bytes = [&](int64_t t) -> uint32_t {
    if (!scale_copy) return 0;
    const int64_t row0 = t * kWR;
    const int valid = static_cast<int>(a.n - row0 < kWR ? a.n - row0 : kWR);
    return static_cast<uint32_t>(valid * L::SPR) & ~15u;
  };
  auto refill = [&](int stage) {
    const int t = claim();
    if (lane == 0) tq[stage] = t;
    if (t < 0 || lane != 0) return;
    const int64_t row0 = static_cast<int64_t>(t) * kWR;
    const int valid = static_cast<int>(a.n - row0 < kWR ? a.n - row0 : kWR);
    const uint32_t sb = scale_bytes(t);
    mbar_expect_tx(&bar[stage], static_cast<uint32_t>(valid) * F::CB + sb);
    bulk_g2s(wsm + stage * L::STAGE, codes + row0 * F::CB, static_cast<uint32_t>(valid) * F::CB, &bar[stage]);
    if (sb) bulk_g2s(wsm + stage * L::STAGE + L::WC, reinterpret_cast<const uint8_t*>(scales) + row0 * L::SPR, sb, &bar[stage]);
  };
  refill(0);
  refill(1);
  const float2 c2 = make_float2(a.c, a.c);
  int cached = -1;
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;
    const int64_t row = tile * kWR + lane;
    const int64_t rrow = row < a.n ? row : a.n - 1;
    const bool sc_smem = static_cast<uint32_t>((lane + 1) * L::SPR) <= scale_bytes(tile);
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinX);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_ex_fault, 1u);
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinX);
      return;
    }
    const int id = table_id(a, tile * kWR);
    if (id != cached) {
      build_table(tab, a, id, AFTER ? 3 : 2, lane);
      cached = id;
      __syncwarp();
    }
    const uint8_t* st = wsm + stage * L::STAGE;
    const uint16_t* srow = sc_smem ? reinterpret_cast<const uint16_t*>(st + L::WC + lane * L::SPR)
                                   : scales + rrow * (kD / G);
    uint16_t sx[NGH], sy[NGH];
#pragma unroll
    for (int j = 0; j < NGH; ++j) {
      sx[j] = srow[j];
      sy[j] = srow[NGH + j];
    }
    // codes of the pair (m, m+64) as exact fp16 integers, then u = q S exactly
    const uint2* seg = reinterpret_cast<const uint2*>(st + lane * F::CB);
    float2 p[kNP];
    if constexpr (BITS == 4) {
      const __half2 bias = __floats2half2_rn(1032.0f, 1032.0f);
#pragma unroll
      for (int kw = 0; kw < kNP / 8; ++kw) {
        const uint2 da = seg[kw / 2], db = seg[(kw + kNP / 8) / 2];
        const uint32_t wa = ((kw & 1) ? da.y : da.x) ^ 0x88888888u;
        const uint32_t wb = ((kw & 1) ? db.y : db.x) ^ 0x88888888u;
        const uint32_t wa4 = wa >> 4, wb4 = wb >> 4;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t sel = 0x0400u | (t << 8) | t;
          const uint32_t e0 = (__byte_perm(wa, wb, sel) & 0x000F000Fu) | 0x64006400u;
          const uint32_t e1 = (__byte_perm(wa4, wb4, sel) & 0x000F000Fu) | 0x64006400u;
          const __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&e0), bias);
          const __half2 h1 = __hsub2(*reinterpret_cast<const __half2*>(&e1), bias);
          const int m0 = 8 * kw + 2 * t, m1 = m0 + 1;
          p[m0] = make_float2(mul_f16_f32(__low2half(h0), sx[m0 / G]), mul_f16_f32(__high2half(h0), sy[m0 / G]));
          p[m1] = make_float2(mul_f16_f32(__low2half(h1), sx[m1 / G]), mul_f16_f32(__high2half(h1), sy[m1 / G]));
        }
      }
    } else {
      const __half2 bias = __floats2half2_rn(1152.0f, 1152.0f);
#pragma unroll
      for (int kw = 0; kw < kNP / 4; ++kw) {
        const uint2 da = seg[kw / 2], db = seg[(kw + kNP / 4) / 2];
        const uint32_t wa = ((kw & 1) ? da.y : da.x) ^ 0x80808080u;
        const uint32_t wb = ((kw & 1) ? db.y : db.x) ^ 0x80808080u;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t sel = 0x0400u | (t << 8) | t;
          const uint32_t e = (__byte_perm(wa, wb, sel) & 0x00FF00FFu) | 0x64006400u;
          const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&e), bias);
          const int m = 4 * kw + t;
          p[m] = make_float2(mul_f16_f32(__low2half(h), sx[m / G]), mul_f16_f32(__high2half(h), sy[m / G]));
        }
      }
    }
    __syncwarp();                       // codes and scales consumed: refill the stage
    refill(stage);
    if constexpr (AFTER) {
#pragma unroll
      for (int q = 0; q < kNP / 2; ++q) {
        const float4 l = tab[q];                      // 1/lambda
        p[2 * q] = __fmul2_rn(p[2 * q], make_float2(l.x, l.y));
        p[2 * q + 1] = __fmul2_rn(p[2 * q + 1], make_float2(l.z, l.w));
      }
    }
    fwht_pairs<kD, 1>(p, 0);
    uint16_t* dst = out + (row < a.n ? row : 0) * kD;
#pragma unroll
    for (int k4 = 0; k4 < kNP / 8; ++k4) {
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int q = 4 * k4 + t;
        float2 a0 = __fmul2_rn(p[2 * q], c2);
        float2 a1 = __fmul2_rn(p[2 * q + 1], c2);
        if constexpr (AFTER) {                        // signs only: exact
          const float4 sg = stab[q];
          a0 = __fmul2_rn(a0, make_float2(sg.x, sg.y));
          a1 = __fmul2_rn(a1, make_float2(sg.z, sg.w));
        } else {
          const float4 l = tab[q];                    // s * (1/lambda)
          a0 = __fmul2_rn(a0, make_float2(l.x, l.y));
          a1 = __fmul2_rn(a1, make_float2(l.z, l.w));
        }
        lo[t] = float2_to_half2_bits(a0.x, a1.x);    // channels 2q, 2q+1
        hi[t] = float2_to_half2_bits(a0.y, a1.y);    // channels 64+2q, 64+2q+1
      }
      if (row < a.n) {
        st_v4(dst + 8 * k4, lo);
        st_v4(dst + kNP + 8 * k4, hi);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Launch plumbing.
// ---------------------------------------------------------------------------

int ex_sms(int& dev) {
  static std::atomic<int> cache[64];
  dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { dev = 0; return 148; }
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1) v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

template <typename Kernel>
int ex_grid(Kernel k, int64_t n, int smem, std::atomic<int>* ready) {
  int dev = 0;
  const int sms = ex_sms(dev);
  int occ = ready[dev].load(std::memory_order_relaxed);
  if (occ == 0) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kXW * 32, smem) != cudaSuccess || occ < 1) occ = 1;
    ready[dev].store(occ, std::memory_order_relaxed);
  }
  const int64_t tiles = (n + kWR - 1) / kWR;
  const int64_t cap = static_cast<int64_t>(sms) * occ;
  return static_cast<int>(tiles < cap ? tiles : cap);
}

int finish_ex() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_ex_cuda_error = static_cast<int>(e);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
}

int check_ex(int D, int G, int bits, int64_t n, int64_t lambda_rows, int n_lambda) {
  if (D != kD) return KVQ_ERR_DIM;
  if (G != 16 && G != 32 && G != 64) return KVQ_ERR_GROUP;
  if (bits != 4 && bits != 8) return KVQ_ERR_GROUP;
  if (n < 0 || n > (int64_t{1} << 31) - 256 || n_lambda < 1 || lambda_rows < 1 ||
      (n_lambda > 1 && lambda_rows % kWR != 0))
    return KVQ_ERR_COUNT;
  return KVQ_OK;
}

template <int G, int BITS, bool AFTER>
int launch_qex(const uint16_t* x, const ExArgs& a, uint8_t* codes, uint16_t* scales, cudaStream_t st) {
  ExMaps maps;
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  for (int q = 0; q < 2; ++q) {
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(a.n)};
    const cuuint64_t strides[1] = {2 * kD};
    const cuuint32_t box[2] = {64, kWR};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&maps.q[q], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                           const_cast<char*>(reinterpret_cast<const char*>(x)) + 128 * q, dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      g_ex_cuda_error = static_cast<int>(r);
      return KVQ_ERR_LAUNCH;
    }
  }
  auto k = kvq_quantize_ex_kernel<G, BITS, AFTER>;
  constexpr int smem = 1024 + kXW * 2 * kXStage + kHdrBytes;
  static std::atomic<int> ready[64];
  const int grid = ex_grid(k, a.n, smem, ready);
  (void)cudaGetLastError();
  k<<<grid, kXW * 32, smem, st>>>(maps, a, codes, scales);
  return finish_ex();
}

template <int G, int BITS, bool AFTER>
int launch_dex(const uint8_t* codes, const uint16_t* scales, const ExArgs& a, uint16_t* out,
               cudaStream_t st) {
  using L = DeqLayout<G, BITS>;
  auto k = kvq_dequantize_ex_kernel<G, BITS, AFTER>;
  constexpr int smem = 128 + kXW * L::WARP + kHdrBytes;
  static std::atomic<int> ready[64];
  const int grid = ex_grid(k, a.n, smem, ready);
  (void)cudaGetLastError();
  k<<<grid, kXW * 32, smem, st>>>(codes, scales, a, out,
                                  (reinterpret_cast<uintptr_t>(scales) & 15) == 0 ? 1 : 0);
  return finish_ex();
}

#define KVQ_EX_DISPATCH(FN, ...)                                                        \
  switch (group * 100 + bits * 10 + (lambda_after ? 1 : 0)) {                          \
    case 1640: return FN<16, 4, false>(__VA_ARGS__);                                    \
    case 1641: return FN<16, 4, true>(__VA_ARGS__);                                     \
    case 1680: return FN<16, 8, false>(__VA_ARGS__);                                    \
    case 1681: return FN<16, 8, true>(__VA_ARGS__);                                     \
    case 3240: return FN<32, 4, false>(__VA_ARGS__);                                    \
    case 3241: return FN<32, 4, true>(__VA_ARGS__);                                     \
    case 3280: return FN<32, 8, false>(__VA_ARGS__);                                    \
    case 3281: return FN<32, 8, true>(__VA_ARGS__);                                     \
    case 6440: return FN<64, 4, false>(__VA_ARGS__);                                    \
    case 6441: return FN<64, 4, true>(__VA_ARGS__);                                     \
    case 6480: return FN<64, 8, false>(__VA_ARGS__);                                    \
    case 6481: return FN<64, 8, true>(__VA_ARGS__);                                     \
    default: return KVQ_ERR_GROUP;                                                      \
  }

inline bool aligned_to(const void* p, uintptr_t al) { return (reinterpret_cast<uintptr_t>(p) & (al - 1)) == 0; }

}  // namespace

// Read (and optionally clear) the variant kernels' fault word; used by
// kvq_fault_status.
__attribute__((visibility("hidden"))) unsigned int kvq_ex_fault_word(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ex_fault, sizeof(v)) != cudaSuccess) return 0;
  if (clear && v) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_ex_fault, &zero, sizeof(zero));
  }
  return v;
}
__attribute__((visibility("hidden"))) int kvq_ex_last_cuda_error() { return g_ex_cuda_error; }

extern "C" {

int kvq_quantize_ex(const uint16_t* x, const float* lambda, const int8_t* signs, int64_t n_vec,
                    int D, int group, int bits, int lambda_after, int64_t lambda_rows,
                    int n_lambda, uint8_t* codes, uint16_t* scales, void* stream) {
  const int rc = check_ex(D, group, bits, n_vec, lambda_rows, n_lambda);
  if (rc != KVQ_OK) return rc;
  if (n_vec == 0) return KVQ_OK;
  if (!x || !lambda || !signs || !codes || !scales) return KVQ_ERR_NULL;
  if (!aligned_to(x, 16) || !aligned_to(codes, 16) || !aligned_to(scales, 2) || !aligned_to(lambda, 4))
    return KVQ_ERR_ALIGN;
  ExArgs a{lambda, signs, n_vec, lambda_rows, n_lambda,
           static_cast<float>(1.0 / std::sqrt(static_cast<double>(kD)))};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_EX_DISPATCH(launch_qex, x, a, codes, scales, st)
}

int kvq_dequantize_ex(const uint8_t* codes, const uint16_t* scales, const float* lambda,
                      const int8_t* signs, int64_t n_vec, int D, int group, int bits,
                      int lambda_after, int64_t lambda_rows, int n_lambda, uint16_t* x_out,
                      void* stream) {
  const int rc = check_ex(D, group, bits, n_vec, lambda_rows, n_lambda);
  if (rc != KVQ_OK) return rc;
  if (n_vec == 0) return KVQ_OK;
  if (!codes || !scales || !lambda || !signs || !x_out) return KVQ_ERR_NULL;
  if (!aligned_to(codes, 16) || !aligned_to(x_out, 16) || !aligned_to(scales, 2) || !aligned_to(lambda, 4))
    return KVQ_ERR_ALIGN;
  ExArgs a{lambda, signs, n_vec, lambda_rows, n_lambda,
           static_cast<float>(1.0 / std::sqrt(static_cast<double>(kD)))};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_EX_DISPATCH(launch_dex, codes, scales, a, x_out, st)
}

}  // extern "C"
