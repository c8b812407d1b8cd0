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
// Work decomposition.  One lane owns EPT = min(D, 128) channels of a vector
// (a vector is owned by LANES = D / EPT lanes: one, or two at D = 256) and
// holds them in registers as EPT/2 packed fp32 pairs p[m] = (v[m], v[m+EPT/2]).
// The butterfly with half-width h then runs as packed f32x2 adds/subs between
// pair registers for h < EPT/2, inside each pair for h = EPT/2, and across
// the two lanes with __shfl_xor_sync for h = EPT (D = 256 only).  Every
// butterfly output is one IEEE fp32 a+b or a-b of the same operands in the
// same ascending-h order as the plain sequential loop, so the result is
// bit-identical to it.
//
// Data movement.  Each warp streams its own warp tiles (32 / LANES vectors,
// one per lane or lane pair: lane rin + 16 * sub holds part sub of row rin,
// so the eight lanes of a quarter-warp phase hold eight different rows)
// through a private double-buffered ring in
// shared memory, so no block-wide barrier couples the warps.  The warps of a
// block draw their next tile from a shared-memory counter over the block's
// tiles (blockIdx.x + i * gridDim.x): a warp that the scheduler favours takes
// more tiles, and all warps finish together.  Large batches run one block of
// 12 warps per SM; small ones run 4-warp blocks, three per SM.  Each fp16
// tile moves as Q = D/64 tensor copies (one per 64-channel quarter of the
// rows, 2-D maps of 64 channels x n rows with the 128-byte swizzle), issued by
// one lane; chunk c of tile row t lands at chunk c ^ (t mod 8), so lanes
// reading consecutive rows hit distinct bank groups.  The packed codes of a
// warp tile are one 2-D tensor copy (D/2 bytes x the tile's rows) swizzled
// over the row's 32, 64 or 128 bytes the same way.  Quantize: tensor loads
// in; codes out through a staging tile and one tensor store, scales by
// direct stores.  Dequantize: codes by tensor copy and scales by bulk copy
// in; the lanes write their fp16 rows into a swizzled staging tile that
// leaves as Q tensor stores (rows past n are clipped by the copy engine,
// rows past n read as zeros on the way in).  No copy uses multicast.  Every
// mbarrier wait is bounded; a warp that gives up sets a device fault word,
// drains its own copies and returns (kvq_fault_status reads the word).
//
// This translation unit is compiled with --fmad=false and uses only _rn
// intrinsics on the contract-sensitive steps, so no multiply is ever fused
// into a following add.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "kvq.h"

// The other translation units' fault words and last CUDA errors.
unsigned int kvq_attn_fault_word(int clear);
int kvq_attn_last_cuda_error();
unsigned int kvq_ex_fault_word(int clear);
int kvq_ex_last_cuda_error();

namespace {

constexpr int kWarps = 12;                 // warps of a streaming block (one block per SM)
constexpr unsigned kFullMask = 0xffffffffu;
constexpr uint32_t kSpinLimit = 1u << 22;  // bounded mbarrier waits
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxVectors = (int64_t{1} << 31) - 256;  // tensor-copy row coordinates are 32-bit

thread_local int g_last_cuda_error = 0;

// Non-zero once some block gave up a bounded wait (see kvq_fault_status).
__device__ unsigned int g_kvq_fault = 0;

// ---------------------------------------------------------------------------
// Lane geometry of a vector: a lane holds EPT channels as NP fp32 pairs, the
// fp16 rows split into Q quarters of 64 channels (128 bytes).
// ---------------------------------------------------------------------------
template <int D>
struct Tile {
  static constexpr int EPT = D < 128 ? D : 128;    // channels per lane
  static constexpr int LANES = D / EPT;             // lanes per vector
  static constexpr int NP = EPT / 2;                // fp32 pairs per lane
  static constexpr int HALF = EPT / 2;              // pair (m, m + HALF)
  static constexpr int Q = D / 64;                  // 64-channel quarters of a row
  static constexpr int TAB = LANES * NP * 8;        // per-channel pair table
};

// The kernel arguments that describe a tensor copy of the fp16 rows: one 2-D
// map (64 channels x n rows, row stride 2D bytes) per quarter.
struct RowMaps {
  CUtensorMap q[4];
};

// A warp tile: the 32 / LANES vectors one warp holds, one per lane (team).
template <int D>
struct WTile {
  static constexpr int WROWS = 32 / Tile<D>::LANES;   // vectors per warp tile
  static constexpr int WQB = WROWS * 128;             // bytes of one quarter of a warp tile
  static constexpr int WSTAGE = Tile<D>::Q * WQB;     // bytes of one fp16 warp tile
  static constexpr int WPIN = WROWS * (D / 2);        // bytes of one packed warp tile
};
// Byte offset of chunk c of quarter q of row t inside a swizzled warp tile.
template <int D>
__device__ __forceinline__ int wtile_off(int q, int t, int c) {
  return q * WTile<D>::WQB + t * 128 + ((c ^ (t & 7)) << 4);
}

constexpr int kScaleBlock = 512;   // bytes reserved for one warp tile's scales (>= 32 rows x 16 B)

// Shared memory of a streaming block (quantize, dequantize) of NW warps: one
// private buffer per warp (a multiple of 1 KiB, so every tensor-copy
// destination keeps the 1 KiB swizzle alignment), then a header holding the
// per-channel table, two mbarriers and two stage tile ids per warp and the
// tile-claim counter.
template <int D>
struct Stream {
  static constexpr int BARS = Tile<D>::TAB;                 // header offsets
  static constexpr int TQ = BARS + 16 * kWarps;
  static constexpr int NEXT = TQ + 8 * kWarps;
  static constexpr int HDR = NEXT + 16;
  static constexpr int QWARP = 2 * WTile<D>::WSTAGE;        // quantize: two fp16 input stages
  static constexpr int QWARP_S =                            // ... plus the staged codes of one warp tile
      QWARP + (WTile<D>::WROWS * (D / 2) + 1023) / 1024 * 1024;
  static constexpr int DWARP =                              // dequantize: output tile, 2 x (codes, scales)
      (WTile<D>::WSTAGE + 2 * WTile<D>::WPIN + 2 * kScaleBlock + 1023) / 1024 * 1024;
  static constexpr int smem(int per_warp, int warps) { return 1024 + warps * per_warp + HDR; }
};
// Shared memory of a round-trip block: per warp two fp16 stages (a tile's
// input, then its output: the output is written over the input it was
// computed from) and the code block of one warp tile; then a header with the
// quantize and dequantize tables, two mbarriers and two stage tile ids per
// warp and the tile-claim counter.  One block of kRtWarps warps per SM, as
// for the streaming kernels.
constexpr int kRtWarps = kWarps;
template <int D>
struct RStream {
  static constexpr int TABQ = 0;
  static constexpr int TABD = Tile<D>::TAB;
  static constexpr int BARS = 2 * Tile<D>::TAB;
  static constexpr int TQ = BARS + 16 * kRtWarps;
  static constexpr int NEXT = TQ + 8 * kRtWarps;
  static constexpr int HDR = NEXT + 16;
  static constexpr int CST = (WTile<D>::WROWS * (D / 2) + 1023) / 1024 * 1024;
  static constexpr int WARP = 2 * WTile<D>::WSTAGE + CST;
  static constexpr int SMEM = 1024 + kRtWarps * WARP + HDR;
};

// ---------------------------------------------------------------------------
// Asynchronous copies and barriers.
// ---------------------------------------------------------------------------

#include "kvq_async.cuh"

#include "kvq_arith.cuh"

// Per-channel table: tab[sub * NP/2 + q] = (c[2q], c[2q+HALF], c[2q+1],
// c[2q+1+HALF]) over lane `sub`'s channels, c = lambda*s (quantize) or
// s * fp32(1/lambda) (dequantize).  Both products are exact sign flips.
template <int D>
__device__ __forceinline__ void fill_tab(float4* tab, const float* __restrict__ lam,
                                         const int8_t* __restrict__ sg, bool reciprocal) {
  using T = Tile<D>;
  for (int i = threadIdx.x; i < T::LANES * (T::NP / 2); i += blockDim.x) {
    const int sub = i / (T::NP / 2), q = i % (T::NP / 2);
    const int base = T::EPT * sub + 2 * q;
    const int ch[4] = {base, base + T::HALF, base + 1, base + 1 + T::HALF};
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float l = lam[ch[k]];
      if (reciprocal) l = __frcp_rn(l);          // fp32 IEEE 1/lambda
      v[k] = (sg[ch[k]] < 0) ? -l : l;
    }
    tab[i] = make_float4(v[0], v[1], v[2], v[3]);
  }
}


// Group geometry of a lane's pairs: GX pairs per group (G <= EPT/2), NGH
// groups per half-lane, HG = the butterfly half-widths that stay in a group.
template <int D, int G>
struct Grp {
  static constexpr int GX = (G < Tile<D>::HALF) ? G : Tile<D>::HALF;
  static constexpr int NGH = Tile<D>::HALF / GX;
  static constexpr int HG = (G < Tile<D>::NP) ? G : Tile<D>::NP;
};

// a2-a7 on one lane's part of a vector, p = x * lambda * s as pairs
// (v[m], v[m + EPT/2]): butterfly, x c, group abs-max, scales, codes.  out:
// the lane's packed codes in row order (word k: channels 8k .. 8k+7 of the
// lane's EPT, two's-complement nibbles); bx / by: the scales (fp16 bits) of
// the groups in pair halves .x / .y.  XS: lane stride between the parts of a
// vector.
template <int D, int G, int XS>
__device__ __forceinline__ void quantize_regs(float2 (&p)[Tile<D>::NP], int sub, float2 c2,
                                              uint32_t (&out)[Tile<D>::EPT / 8],
                                              uint16_t (&bx)[Grp<D, G>::NGH],
                                              uint16_t (&by)[Grp<D, G>::NGH]) {
  constexpr int EPT = Tile<D>::EPT, LANES = Tile<D>::LANES, NP = Tile<D>::NP, HALF = Tile<D>::HALF;
  constexpr int GX = Grp<D, G>::GX, NGH = Grp<D, G>::NGH;
  // a2, a3: transform, normalise.
  fwht_pairs<EPT, LANES, 1, XS>(p, sub);
#pragma unroll
  for (int m = 0; m < NP; ++m) p[m] = __fmul2_rn(p[m], c2);

  // a4, a5: group abs-max and scales.  Pair .x holds channels [0, HALF) of
  // the lane, .y holds [HALF, EPT).
  float rx[NGH], ry[NGH];
  if constexpr (G <= HALF) {
#pragma unroll
    for (int j = 0; j < NGH; ++j) {
      float ax = 0.f, ay = 0.f;
#pragma unroll
      for (int m = 0; m < GX; m += 2) {
        ax = amax3(ax, p[j * GX + m].x, p[j * GX + m + 1].x);
        ay = amax3(ay, p[j * GX + m].y, p[j * GX + m + 1].y);
      }
      bx[j] = group_scale(ax, rx[j]);
      by[j] = group_scale(ay, ry[j]);
    }
  } else {
    float a = 0.f;
#pragma unroll
    for (int m = 0; m < NP; ++m) a = amax3(a, p[m].x, p[m].y);
#pragma unroll
    for (int bit = 1; bit < G / EPT; bit <<= 1) a = fmaxf(a, __shfl_xor_sync(kFullMask, a, bit * XS));
    bx[0] = group_scale(a, rx[0]);
    ry[0] = rx[0];
    by[0] = bx[0];
  }

  // a6, a7: codes = rint(y * r) (half to even), saturated and packed.
#pragma unroll
  for (int k8 = 0; k8 < NP / 8; ++k8) {
    int qa[8], qb[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int m = 8 * k8 + t;
      const float2 v = __fmul2_rn(p[m], make_float2(rx[m / GX], ry[m / GX]));
      qa[t] = __float2int_rn(v.x);
      qb[t] = __float2int_rn(v.y);
    }
    out[k8] = pack8(qa);
    out[k8 + NP / 8] = pack8(qb);
  }
}

// The lane's codes into a warp tile's code staging block, laid out as the
// swizzled tensor store reads it: 16-byte chunk c of row t at chunk
// c ^ ((t * D/2 / 128) mod D/32), so a quarter-warp's chunks fall in distinct
// banks.
template <int D>
__device__ __forceinline__ void stage_codes(uint8_t* cst, const uint32_t (&out)[Tile<D>::EPT / 8],
                                            int sub, int rin) {
  constexpr int EPT = Tile<D>::EPT, RB = D / 2;   // code bytes per row
  const int swz = ((rin * RB) >> 7) & (D / 32 - 1);
#pragma unroll
  for (int k4 = 0; k4 < EPT / 32; ++k4) {
    const int cidx = sub * (EPT / 32) + k4;
    *reinterpret_cast<uint4*>(cst + rin * RB + ((cidx ^ swz) << 4)) =
        make_uint4(out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3]);
  }
}

// The lane's scales into row `orow` of the scale array: the row's D/G scales
// in one store when the pointer is aligned for it (vec), else one by one.
template <int D, int G>
__device__ __forceinline__ void store_scales(uint16_t* __restrict__ scales, int64_t orow, int sub,
                                             const uint16_t (&bx)[Grp<D, G>::NGH],
                                             const uint16_t (&by)[Grp<D, G>::NGH], bool vec) {
  constexpr int EPT = Tile<D>::EPT, LANES = Tile<D>::LANES, HALF = Tile<D>::HALF;
  constexpr int NGH = Grp<D, G>::NGH;
  uint16_t* srow = scales + orow * (D / G);
  if constexpr (G <= HALF && LANES == 1) {
    uint16_t sa[D / G];
#pragma unroll
    for (int j = 0; j < NGH; ++j) { sa[j] = bx[j]; sa[NGH + j] = by[j]; }
    uint32_t sw[D / G / 2];
#pragma unroll
    for (int i = 0; i < D / G / 2; ++i) sw[i] = uint32_t(sa[2 * i]) | (uint32_t(sa[2 * i + 1]) << 16);
    if (vec) {
      if constexpr (D / G == 2) *reinterpret_cast<uint32_t*>(srow) = sw[0];
      else if constexpr (D / G == 4) *reinterpret_cast<uint2*>(srow) = make_uint2(sw[0], sw[1]);
      else *reinterpret_cast<uint4*>(srow) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
    } else {
#pragma unroll
      for (int j = 0; j < NGH; ++j) {
        srow[j] = bx[j];
        srow[NGH + j] = by[j];
      }
    }
  } else if constexpr (G <= HALF) {
#pragma unroll
    for (int j = 0; j < NGH; ++j) {
      srow[sub * (EPT / G) + j] = bx[j];
      srow[sub * (EPT / G) + NGH + j] = by[j];
    }
  } else {
    if (sub % (G / EPT) == 0) srow[sub / (G / EPT)] = bx[0];
  }
}

// a8 and the butterfly stages inside a group: the lane's code words w (row
// order, nibbles biased to n = q + 8) and scales -> p = u after the stages
// h < HG, as fp32 pairs (m, m + EPT/2).  u = q S is exact, and so is every
// stage inside a group.
//  * One prmt + lop3 puts the codes of a pair (m, m + EPT/2) into two 16-bit
//    lanes holding W + 0x6608, the fp16 encoding of the exact integer
//    W + 1544 (W = n, or its partial butterfly sums).
//  * The first four stages run on those integer lanes: one 32-bit add does
//    a + b - bias (or a - b + bias) for both; every lane stays in [0, 65535].
//  * The remaining in-group stages run in fp16x2 after one hsub2 removes the
//    bias (integers of magnitude <= 8 * 2^stage <= 512: exact).
//  * u = W * S by one mixed-precision fma.rn.f32.f16 (a product of two fp16
//    values is exact in fp32).
template <int D, int G>
__device__ __forceinline__ void dequant_front(const uint32_t (&w)[Tile<D>::EPT / 8],
                                              const uint16_t (&sx)[Grp<D, G>::NGH],
                                              const uint16_t (&sy)[Grp<D, G>::NGH],
                                              float2 (&p)[Tile<D>::NP]) {
  constexpr int NP = Tile<D>::NP, HALF = Tile<D>::HALF;
  constexpr int GX = Grp<D, G>::GX, HG = Grp<D, G>::HG;
  uint32_t iq[NP];
#pragma unroll
  for (int kw = 0; kw < NP / 8; ++kw) {
    const uint32_t wa = w[kw], wb = w[kw + HALF / 8];
    const uint32_t wa4 = wa >> 4, wb4 = wb >> 4;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t sel = 0x0400u | (t << 8) | t;   // byte t of a -> byte 0, of b -> byte 2
      iq[8 * kw + 2 * t] = (__byte_perm(wa, wb, sel) & 0x000F000Fu) | 0x66006600u;
      iq[8 * kw + 2 * t + 1] = (__byte_perm(wa4, wb4, sel) & 0x000F000Fu) | 0x66006600u;
    }
  }
  constexpr int kIntStages = 4;
  constexpr uint32_t kBias2 = 0x66086608u;
  constexpr int HI = (1 << kIntStages) < HG ? (1 << kIntStages) : HG;
#pragma unroll
  for (int h = 1; h < HI; h <<= 1) {
#pragma unroll
    for (int m = 0; m < NP; ++m) {
      if ((m & h) == 0) {
        const uint32_t a = iq[m], b = iq[m + h];
        iq[m] = a + b - kBias2;
        iq[m + h] = a - b + kBias2;
      }
    }
  }
  const __half2 k1544 = __floats2half2_rn(1544.0f, 1544.0f);
  __half2 hq[NP];
#pragma unroll
  for (int m = 0; m < NP; ++m) hq[m] = __hsub2(*reinterpret_cast<const __half2*>(&iq[m]), k1544);
#pragma unroll
  for (int h = HI; h < HG; h <<= 1) {
#pragma unroll
    for (int m = 0; m < NP; ++m) {
      if ((m & h) == 0) {
        const __half2 a = hq[m], b = hq[m + h];
        hq[m] = __hadd2(a, b);
        hq[m + h] = __hsub2(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < NP; ++m)
    p[m] = make_float2(mul_f16_f32(__low2half(hq[m]), sx[m / GX]),
                       mul_f16_f32(__high2half(hq[m]), sy[m / GX]));
}

// a9's normalisation and a10: x c, x s/lambda (per-channel table), fp16,
// written into the warp's swizzled fp16 staging tile (the input's quarter
// layout), which Q tensor stores then write out.
template <int D>
__device__ __forceinline__ void stage_rows(const float2 (&p)[Tile<D>::NP], float2 c2,
                                           const float4* mytab, uint8_t* stage_out, int sub, int rin) {
  constexpr int EPT = Tile<D>::EPT, NP = Tile<D>::NP, HALF = Tile<D>::HALF;
  constexpr int QL = EPT / 64;                   // quarters per lane
#pragma unroll
  for (int j = 0; j < NP / 8; ++j) {
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float4 l = mytab[4 * j + t];
      const float2 a = __fmul2_rn(__fmul2_rn(p[8 * j + 2 * t], c2), make_float2(l.x, l.y));
      const float2 b = __fmul2_rn(__fmul2_rn(p[8 * j + 2 * t + 1], c2), make_float2(l.z, l.w));
      lo[t] = float2_to_half2_bits(a.x, b.x);
      hi[t] = float2_to_half2_bits(a.y, b.y);
    }
    const int ea = 8 * j, eb = HALF + 8 * j;
    *reinterpret_cast<uint4*>(stage_out + wtile_off<D>(sub * QL + ea / 64, rin, (ea % 64) / 8)) =
        make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4*>(stage_out + wtile_off<D>(sub * QL + eb / 64, rin, (eb % 64) / 8)) =
        make_uint4(hi[0], hi[1], hi[2], hi[3]);
  }
}

// ---------------------------------------------------------------------------
// Quantize: fp16 [n][D] -> packed u8 [n][D/2] + fp16 scales [n][D/G].
// ---------------------------------------------------------------------------
template <int D, int G, bool INDEXED, int NW>
__global__ void __launch_bounds__(NW * 32, NW == kWarps ? 1 : 3)
kvq_quantize_kernel(const __grid_constant__ RowMaps maps, const float* __restrict__ lam,
                    const int8_t* __restrict__ sgn, int64_t n, float c,
                    uint8_t* __restrict__ packed, uint16_t* __restrict__ scales,
                    const int64_t* __restrict__ row_idx, int64_t cache_rows, int scale_vec,
                    const __grid_constant__ CUtensorMap cmap) {
  using T = Tile<D>;
  using W = WTile<D>;
  constexpr int EPT = T::EPT, NP = T::NP, HALF = T::HALF;
  constexpr bool STG = !INDEXED;                // codes leave through a staged tensor store
  constexpr int QW = STG ? Stream<D>::QWARP_S : Stream<D>::QWARP;
  extern __shared__ uint8_t smem_raw[];
  // a generic pointer here: this kernel measured 5% faster with it than with
  // the shared-space one of align_smem_1k (the dequantizer, the variant
  // quantizer and the SRFT kernels measured the reverse)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  using L = Stream<D>;
  uint8_t* hdr = smem + NW * QW;
  float4* tabw = reinterpret_cast<float4*>(hdr);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + L::BARS) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + L::TQ) + 2 * warp;   // tile in each stage, -1: none
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + L::NEXT);
  uint8_t* wsm = smem + warp * QW;
  uint8_t* cst = wsm + 2 * W::WSTAGE;            // the warp tile's codes, swizzled (STG)
  const int sub = lane / W::WROWS;               // which part of the vector
  const int rin = lane % W::WROWS;               // which row of the warp tile
  fill_tab<D>(tabw, lam, sgn, false);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  __syncthreads();

  // The block owns warp tiles blockIdx.x + i * gridDim.x; its warps claim the
  // next i from a shared counter, so a warp that runs ahead takes more tiles.
  const int64_t ntiles = (n + W::WROWS - 1) / W::WROWS;
  // (ntiles < 2^31: n < 2^31 and a warp tile holds at least 16 rows)
  const unsigned int mine = static_cast<unsigned int>((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(blockIdx.x + i * gridDim.x) : -1;
  };
  auto issue = [&](int64_t tile, int stage) {
    if (tile < 0 || lane != 0) return;
    mbar_expect_tx(&bar[stage], W::WSTAGE);
#pragma unroll
    for (int q = 0; q < T::Q; ++q)
      tensor_g2s(wsm + stage * W::WSTAGE + q * W::WQB, &maps.q[q], 0, static_cast<int>(tile * W::WROWS), &bar[stage]);
  };
  auto refill = [&](int stage) {
    const int t = claim();
    if (lane == 0) tq[stage] = t;
    issue(t, stage);
  };
  refill(0);
  refill(1);
  const float2 c2 = make_float2(c, c);
  const float4* mytab = tabw + sub * (NP / 2);
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;                         // later claims failed too
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_kvq_fault, 1u);
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);   // the stage that gave up, once more
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinLimit);
      if (STG && lane == 0) bulk_wait0();
      return;
    }
    const int64_t row = tile * W::WROWS + rin;
    bool active = row < n;
    int64_t orow = row;                          // destination row of the codes
    if constexpr (INDEXED) {
      orow = active ? row_idx[row] : 0;
      if (active && (orow < 0 || orow >= cache_rows)) {
        atomicOr(&g_kvq_fault, 4u);              // out-of-range index: skipped
        active = false;
      }
    }

    // a1: widen fp16 and multiply by lambda*s (one rounding per element).
    const uint8_t* st = wsm + stage * W::WSTAGE;
    float2 p[NP];
#pragma unroll
    for (int j = 0; j < NP / 8; ++j) {
      constexpr int QL = EPT / 64;               // quarters per lane
      const int ea = 8 * j, eb = HALF + 8 * j;    // first channel of each chunk
      const uint4 a = *reinterpret_cast<const uint4*>(st + wtile_off<D>(sub * QL + ea / 64, rin, (ea % 64) / 8));
      const uint4 b = *reinterpret_cast<const uint4*>(st + wtile_off<D>(sub * QL + eb / 64, rin, (eb % 64) / 8));
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 fa = half2_bits_to_float2(aw[t]);
        const float2 fb = half2_bits_to_float2(bw[t]);
        const float4 l = mytab[4 * j + t];
        p[8 * j + 2 * t] = __fmul2_rn(make_float2(fa.x, fb.x), make_float2(l.x, l.y));
        p[8 * j + 2 * t + 1] = __fmul2_rn(make_float2(fa.y, fb.y), make_float2(l.z, l.w));
      }
    }
    __syncwarp();             // the warp has its inputs: the stage can be refilled
    refill(stage);

    uint32_t out[EPT / 8];
    uint16_t bx[Grp<D, G>::NGH], by[Grp<D, G>::NGH];
    quantize_regs<D, G, W::WROWS>(p, sub, c2, out, bx, by);

    // The codes of a warp tile are one contiguous block: lane 0 stores the
    // staged tile with one tensor copy that skips rows past n.  Rows
    // scattered by an index are stored by each lane.
    if constexpr (STG) {
      if (lane == 0) bulk_wait_read0();
      __syncwarp();                              // the staging tile is free
      stage_codes<D>(cst, out, sub, rin);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tensor_s2g(&cmap, 0, static_cast<int>(tile * W::WROWS), cst);
        bulk_commit();
      }
    }
    if (active) {
      if constexpr (!STG) {
        uint8_t* dst = packed + orow * (D / 2) + sub * (EPT / 2);
#pragma unroll
        for (int k4 = 0; k4 < EPT / 32; ++k4) {
          const uint32_t t4[4] = {out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3]};
          st_v4(dst + 16 * k4, t4);
        }
      }
      store_scales<D, G>(scales, orow, sub, bx, by, scale_vec != 0);
    }
  }
  if (STG && lane == 0) bulk_wait0();
}

// ---------------------------------------------------------------------------
// Dequantize: packed u8 [n][D/2] + fp16 scales [n][D/G] -> fp16 [n][D].
// ---------------------------------------------------------------------------
template <int D, int G, int NW>
__global__ void __launch_bounds__(NW * 32, NW == kWarps ? 1 : 3)
kvq_dequantize_kernel(const __grid_constant__ CUtensorMap cmap, const uint16_t* __restrict__ scales,
                      const float* __restrict__ lam, const int8_t* __restrict__ sgn,
                      int64_t n, float c, const __grid_constant__ RowMaps maps, int scale_copy) {
  using T = Tile<D>;
  using W = WTile<D>;
  constexpr int EPT = T::EPT, LANES = T::LANES, NP = T::NP, HALF = T::HALF;
  constexpr int WROWS = W::WROWS;
  constexpr int WPIN = W::WPIN;
  constexpr int SPR = (D / G) * 2;               // scale bytes per row
  constexpr int WSC = kScaleBlock;
  static_assert(WROWS * SPR <= WSC, "scale block");
  constexpr int NGH = Grp<D, G>::NGH;
  constexpr int HG = Grp<D, G>::HG;               // butterfly stages h < HG stay inside a group
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  using L = Stream<D>;
  uint8_t* hdr = smem + NW * L::DWARP;
  float4* tabw = reinterpret_cast<float4*>(hdr);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + L::BARS) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + L::TQ) + 2 * warp;   // tile in each stage, -1: none
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + L::NEXT);
  uint8_t* stage_out = smem + warp * L::DWARP;                // swizzled fp16 warp tile
  uint8_t* stage_in = stage_out + W::WSTAGE;                  // two packed warp tiles
  uint8_t* stage_sc = stage_in + 2 * WPIN;                    // two scale blocks
  const int sub = lane / WROWS;
  const int rin = lane % WROWS;
  fill_tab<D>(tabw, lam, sgn, true);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  __syncthreads();

  const int64_t ntiles = (n + WROWS - 1) / WROWS;
  // (ntiles < 2^31: n < 2^31 and a warp tile holds at least 16 rows)
  const unsigned int mine = static_cast<unsigned int>((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(blockIdx.x + i * gridDim.x) : -1;
  };
  // bytes of the scale block moved by the copy engine (a multiple of 16)
  auto scale_bytes = [&](int64_t tile) -> uint32_t {
    if (!scale_copy) return 0;
    const int64_t row0 = tile * WROWS;
    const int valid = static_cast<int>(n - row0 < WROWS ? n - row0 : WROWS);
    return static_cast<uint32_t>(valid * SPR) & ~15u;
  };
  auto issue = [&](int64_t tile, int stage) {
    if (tile < 0 || lane != 0) return;
    const int64_t row0 = tile * WROWS;
    const uint32_t sb = scale_bytes(tile);
    mbar_expect_tx(&bar[stage], static_cast<uint32_t>(WPIN) + sb);
    tensor_g2s(stage_in + stage * WPIN, &cmap, 0, static_cast<int>(row0), &bar[stage]);
    if (sb) bulk_g2s(stage_sc + stage * WSC, reinterpret_cast<const uint8_t*>(scales) + row0 * SPR, sb, &bar[stage]);
  };
  auto refill = [&](int stage) {
    const int t = claim();
    if (lane == 0) tq[stage] = t;
    issue(t, stage);
  };
  refill(0);
  refill(1);
  const float2 c2 = make_float2(c, c);
  const float4* mytab = tabw + sub * (NP / 2);
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;                         // later claims failed too
    const int64_t row = tile * WROWS + rin;
    const int64_t rrow = row < n ? row : n - 1;
    const bool sc_smem = static_cast<uint32_t>((rin + 1) * SPR) <= scale_bytes(tile);
    const uint16_t* srow = sc_smem ? reinterpret_cast<const uint16_t*>(stage_sc + stage * WSC + rin * SPR)
                                   : scales + rrow * (D / G);
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_kvq_fault, 1u);
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);   // the stage that gave up, once more
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinLimit);
      if (lane == 0) bulk_wait0();
      return;
    }
    uint16_t sx[NGH], sy[NGH];
    if constexpr (G <= HALF) {
#pragma unroll
      for (int j = 0; j < NGH; ++j) {
        sx[j] = srow[sub * (EPT / G) + j];
        sy[j] = srow[sub * (EPT / G) + NGH + j];
      }
    } else {
      sx[0] = srow[sub / (G / EPT)];
      sy[0] = sx[0];
    }
    // a8: the lane's EPT/2 bytes of codes; nibbles biased to n = q + 8.
    const uint8_t* crow = stage_in + stage * WPIN + rin * (D / 2);
    const int cswz = ((rin * (D / 2)) >> 7) & (D / 32 - 1);
    uint32_t w[EPT / 8];
#pragma unroll
    for (int j = 0; j < EPT / 32; ++j) {
      const uint4 a = *reinterpret_cast<const uint4*>(crow + (((sub * (EPT / 32) + j) ^ cswz) << 4));
      w[4 * j] = a.x ^ 0x88888888u;
      w[4 * j + 1] = a.y ^ 0x88888888u;
      w[4 * j + 2] = a.z ^ 0x88888888u;
      w[4 * j + 3] = a.w ^ 0x88888888u;
    }
    float2 p[NP];
    dequant_front<D, G>(w, sx, sy, p);
    __syncwarp();             // codes and scales consumed: the input stage can be refilled
    refill(stage);
    fwht_pairs<EPT, LANES, HG, WROWS>(p, sub);

    if (lane == 0) bulk_wait_read0();
    __syncwarp();             // the warp's staging tile is free
    stage_rows<D>(p, c2, mytab, stage_out, sub, rin);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < T::Q; ++q)
        tensor_s2g(&maps.q[q], 0, static_cast<int>(tile * WROWS), stage_out + q * W::WQB);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait0();
}


// ---------------------------------------------------------------------------
// Dequantize with the in-group Hadamard on the tensor cores (D = 128, G in
// {16, 32, 64}): the same result as kvq_dequantize_kernel, bit for bit.
//
// H_128 = (H_(128/G) (x) I_G)(I_(128/G) (x) H_G): the butterfly stages with
// half-width h < G act inside a group, and there u = q S stays an exact
// multiple of S, so W = H_G q is a sum of small integers (|W| <= 8 G) that
// any order of addition gets exactly; u = W S is exact in fp32.  The tensor
// cores take that factor: per 16 vectors and 16 channels one m16n8k16 fp16
// MMA with the codes as A (exact small integers) and a 16 x 8 block of
// H_G = H_(G/16) (x) H_16 as B (entries +-1), fp32 accumulation (exact).
// The stages that cross groups (h >= G) then run as fp32 butterflies in the
// oracle's order.  In the accumulator layout a lane holds, for two vectors,
// the channels 8 nt + 2t, 8 nt + 2t + 1 of every n-tile nt, so the partners
// of those stages (channels apart by a multiple of G >= 16) sit in the same
// lane: no shuffle.  Streaming, tiles, tables and the staged tensor stores
// are the butterfly dequantizer's.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte t of the code word w (two nibbles: channel 2b, then 2b + 1) as an
// fp16 pair of exact integers in [-8, 7], low half first.
__device__ __forceinline__ uint32_t code_pair_f16(uint32_t w, int t) {
  const uint32_t wb = w ^ 0x88888888u;
  const uint32_t e = (__byte_perm(wb, wb >> 4, 0x0400u | (t << 8) | t) & 0x000F000Fu) | 0x64006400u;
  const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&e), __floats2half2_rn(1032.0f, 1032.0f));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// (+-1, +-1) fp16 pair: H_16[i][j], H_16[i + 1][j].
__device__ __forceinline__ uint32_t h16_pair(int i, int j) {
  const uint32_t lo = (__popc(i & j) & 1) ? 0xBC00u : 0x3C00u;
  const uint32_t hi = (__popc((i + 1) & j) & 1) ? 0xBC00u : 0x3C00u;
  return lo | (hi << 16);
}

template <int G, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
kvq_dequantize_tc_kernel(const __grid_constant__ CUtensorMap cmap, const uint16_t* __restrict__ scales,
                         const float* __restrict__ lam, const int8_t* __restrict__ sgn,
                         int64_t n, float c, const __grid_constant__ RowMaps maps, int scale_copy) {
  constexpr int D = 128;
  static_assert(G == 16 || G == 32 || G == 64, "in-group Hadamard as 16 x 16 tiles");
  using W = WTile<D>;
  using L = Stream<D>;
  constexpr int WROWS = W::WROWS;                // 32 vectors per warp tile
  constexpr int WPIN = W::WPIN;
  constexpr int NG = D / G;                      // groups per row
  constexpr int SPR = NG * 2;                    // scale bytes per row
  constexpr int WSC = kScaleBlock;
  constexpr int KG = G / 16;                     // k-steps per group
  constexpr int NTG = G / 8;                     // n-tiles per group
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* hdr = smem + NW * L::DWARP;
  float4* tabw = reinterpret_cast<float4*>(hdr);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + L::BARS) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + L::TQ) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + L::NEXT);
  uint8_t* stage_out = smem + warp * L::DWARP;
  uint8_t* stage_in = stage_out + W::WSTAGE;
  uint8_t* stage_sc = stage_in + 2 * WPIN;
  fill_tab<D>(tabw, lam, sgn, true);             // s * fp32(1/lambda), pair layout of the butterfly kernels
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  __syncthreads();

  // B fragments: the two 16 x 8 column blocks of H_16 (and their negatives)
  const uint32_t hb[2][2] = {{h16_pair(2 * t, g), h16_pair(2 * t + 8, g)},
                             {h16_pair(2 * t, 8 + g), h16_pair(2 * t + 8, 8 + g)}};

  const int64_t ntiles = (n + WROWS - 1) / WROWS;
  const unsigned int mine = static_cast<unsigned int>((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(blockIdx.x + i * gridDim.x) : -1;
  };
  auto scale_bytes = [&](int64_t tile) -> uint32_t {
    if (!scale_copy) return 0;
    const int64_t row0 = tile * WROWS;
    const int valid = static_cast<int>(n - row0 < WROWS ? n - row0 : WROWS);
    return static_cast<uint32_t>(valid * SPR) & ~15u;
  };
  auto issue = [&](int64_t tile, int stage) {
    if (tile < 0 || lane != 0) return;
    const int64_t row0 = tile * WROWS;
    const uint32_t sb = scale_bytes(tile);
    mbar_expect_tx(&bar[stage], static_cast<uint32_t>(WPIN) + sb);
    tensor_g2s(stage_in + stage * WPIN, &cmap, 0, static_cast<int>(row0), &bar[stage]);
    if (sb) bulk_g2s(stage_sc + stage * WSC, reinterpret_cast<const uint8_t*>(scales) + row0 * SPR, sb, &bar[stage]);
  };
  auto refill = [&](int stage) {
    const int tt = claim();
    if (lane == 0) tq[stage] = tt;
    issue(tt, stage);
  };
  refill(0);
  refill(1);
  const float2 c2 = make_float2(c, c);
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_kvq_fault, 1u);
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);   // the stage that gave up, once more
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinLimit);
      if (lane == 0) bulk_wait0();
      return;
    }
    const uint32_t sbytes = scale_bytes(tile);
    if (lane == 0) bulk_wait_read0();
    __syncwarp();             // the warp's staging tile is free
#pragma unroll 1
    for (int mt = 0; mt < 2; ++mt) {
      // the lane's rows of this M-tile: 16 mt + g and 16 mt + 8 + g
      uint32_t a[NG * KG][4];
      uint16_t sv[2][NG];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * mt + 8 * hr + g;
        const int64_t row = tile * WROWS + r;
        const int64_t rrow = row < n ? row : n - 1;
        const bool sc_smem = static_cast<uint32_t>((r + 1) * SPR) <= sbytes;
        const uint16_t* srow = sc_smem ? reinterpret_cast<const uint16_t*>(stage_sc + stage * WSC + r * SPR)
                                       : scales + rrow * NG;
#pragma unroll
        for (int j = 0; j < NG; ++j) sv[hr][j] = srow[j];
        // the row's codes: 64 bytes swizzled over the row (16-byte chunk ch at ch ^ ((r >> 1) & 3))
        const uint8_t* crow = stage_in + stage * WPIN + r * (D / 2);
        const int swz = (r >> 1) & 3;
#pragma unroll
        for (int ks = 0; ks < NG * KG; ++ks) {          // 16 channels: bytes 8 ks .. 8 ks + 7
          const uint2 w = *reinterpret_cast<const uint2*>(crow + (((ks >> 1) ^ swz) << 4) + 8 * (ks & 1));
          a[ks][hr] = code_pair_f16(w.x, t);             // channels 16 ks + 2t, + 1
          a[ks][2 + hr] = code_pair_f16(w.y, t);         // channels 16 ks + 8 + 2t, + 1
        }
      }
      float acc[16][4];
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
      // W = H_G q per group: k-step (group gi, ks), n-tile (gi, ntl), block
      // H_(G/16)[ks][ntl / 2] * H_16[., 8 (ntl & 1) ..]
#pragma unroll
      for (int gi = 0; gi < NG; ++gi)
#pragma unroll
        for (int ks = 0; ks < KG; ++ks)
#pragma unroll
          for (int ntl = 0; ntl < NTG; ++ntl) {
            const bool neg = __popc(ks & (ntl >> 1)) & 1;
            const uint32_t b0 = hb[ntl & 1][0] ^ (neg ? 0x80008000u : 0u);
            const uint32_t b1 = hb[ntl & 1][1] ^ (neg ? 0x80008000u : 0u);
            mma_f16_16816(acc[gi * NTG + ntl], a[gi * KG + ks], b0, b1);
          }
      // u = W S (exact), then the stages that cross groups, in fp32
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const float s0 = half_bits_to_float(sv[0][nt / NTG]), s1 = half_bits_to_float(sv[1][nt / NTG]);
        acc[nt][0] = __fmul_rn(acc[nt][0], s0);
        acc[nt][1] = __fmul_rn(acc[nt][1], s0);
        acc[nt][2] = __fmul_rn(acc[nt][2], s1);
        acc[nt][3] = __fmul_rn(acc[nt][3], s1);
      }
#pragma unroll
      for (int h = G; h < D; h <<= 1) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          if (((8 * nt) & h) == 0) {
            const int mt2 = nt + h / 8;
            const float2 a0 = make_float2(acc[nt][0], acc[nt][1]), b0 = make_float2(acc[mt2][0], acc[mt2][1]);
            const float2 a1 = make_float2(acc[nt][2], acc[nt][3]), b1 = make_float2(acc[mt2][2], acc[mt2][3]);
            const float2 s0 = __fadd2_rn(a0, b0), d0 = fsub2(a0, b0);
            const float2 s1 = __fadd2_rn(a1, b1), d1 = fsub2(a1, b1);
            acc[nt][0] = s0.x; acc[nt][1] = s0.y; acc[nt][2] = s1.x; acc[nt][3] = s1.y;
            acc[mt2][0] = d0.x; acc[mt2][1] = d0.y; acc[mt2][2] = d1.x; acc[mt2][3] = d1.y;
          }
        }
      }
      // x c, x s (1/lambda), fp16: channels 8 nt + 2t, + 1 of rows 16 mt + g (+ 8)
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int ch = 8 * nt + 2 * t;
        const float4 tv = tabw[(ch & 63) >> 1];       // (c[2q], c[2q+64], c[2q+1], c[2q+65])
        const float2 f = ch < 64 ? make_float2(tv.x, tv.z) : make_float2(tv.y, tv.w);
        const float2 v0 = __fmul2_rn(__fmul2_rn(make_float2(acc[nt][0], acc[nt][1]), c2), f);
        const float2 v1 = __fmul2_rn(__fmul2_rn(make_float2(acc[nt][2], acc[nt][3]), c2), f);
        const int q = nt >> 3, cc = nt & 7;
        const int r0 = 16 * mt + g, r1 = r0 + 8;
        *reinterpret_cast<uint32_t*>(stage_out + wtile_off<D>(q, r0, cc) + 4 * t) = float2_to_half2_bits(v0.x, v0.y);
        *reinterpret_cast<uint32_t*>(stage_out + wtile_off<D>(q, r1, cc) + 4 * t) = float2_to_half2_bits(v1.x, v1.y);
      }
    }
    __syncwarp();             // codes and scales consumed: the input stage can be refilled
    refill(stage);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < 2; ++q)
        tensor_s2g(&maps.q[q], 0, static_cast<int>(tile * WROWS), stage_out + q * W::WQB);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait0();
}

// ---------------------------------------------------------------------------
// Round trip: fp16 [n][D] -> x_hat = dequantize(quantize(x)) fp16 [n][D], and
// optionally the codes and scales, in one pass (the quantise-then-dequantise
// shape used to simulate the cache's error).  Each warp streams its tiles as
// the quantize kernel does, runs the quantize arithmetic, then the
// dequantize arithmetic straight from the packed code words still in its
// registers (the same words the dequantize kernel would load), so x_hat is
// bit-identical to the two kernels back to back.
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kRtWarps * 32, 1)
kvq_roundtrip_kernel(const __grid_constant__ RowMaps in_maps, const __grid_constant__ RowMaps out_maps,
                     const __grid_constant__ CUtensorMap cmap, const float* __restrict__ lam,
                     const int8_t* __restrict__ sgn, int64_t n, float c,
                     uint16_t* __restrict__ scales, int with_codes, int scale_vec) {
  using T = Tile<D>;
  using W = WTile<D>;
  using L = RStream<D>;
  constexpr int EPT = T::EPT, LANES = T::LANES, NP = T::NP, HALF = T::HALF;
  constexpr int NGH = Grp<D, G>::NGH, HG = Grp<D, G>::HG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  uint8_t* hdr = smem + kRtWarps * L::WARP;
  float4* tab_q = reinterpret_cast<float4*>(hdr + L::TABQ);
  float4* tab_d = reinterpret_cast<float4*>(hdr + L::TABD);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + L::BARS) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + L::TQ) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + L::NEXT);
  uint8_t* wsm = smem + warp * L::WARP;          // two fp16 stages
  uint8_t* cst = wsm + 2 * W::WSTAGE;            // the codes
  const int sub = lane / W::WROWS;
  const int rin = lane % W::WROWS;
  fill_tab<D>(tab_q, lam, sgn, false);
  fill_tab<D>(tab_d, lam, sgn, true);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  __syncthreads();

  const int64_t ntiles = (n + W::WROWS - 1) / W::WROWS;
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
    mbar_expect_tx(&bar[stage], W::WSTAGE);
#pragma unroll
    for (int q = 0; q < T::Q; ++q)
      tensor_g2s(wsm + stage * W::WSTAGE + q * W::WQB, &in_maps.q[q], 0, t * W::WROWS, &bar[stage]);
  };
  refill(0);
  refill(1);
  const float2 c2 = make_float2(c, c);
  const float4* myq = tab_q + sub * (NP / 2);
  const float4* myd = tab_d + sub * (NP / 2);
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_kvq_fault, 1u);
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinLimit);   // the stage that gave up, once more
      // only the first iteration has the other stage's copy in flight
      if (k == 0 && tq[1] >= 0) mbar_wait(&bar[1], 0, kSpinLimit);
      if (lane == 0) bulk_wait0();
      return;
    }
    if (k > 0) {
      // the other stage holds the previous tile's output: once its stores
      // have read it, it takes the next tile
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
      refill(stage ^ 1);
    }
    const int64_t row = tile * W::WROWS + rin;
    uint8_t* st = wsm + stage * W::WSTAGE;
    float2 p[NP];
#pragma unroll
    for (int j = 0; j < NP / 8; ++j) {
      constexpr int QL = EPT / 64;
      const int ea = 8 * j, eb = HALF + 8 * j;
      const uint4 a = *reinterpret_cast<const uint4*>(st + wtile_off<D>(sub * QL + ea / 64, rin, (ea % 64) / 8));
      const uint4 b = *reinterpret_cast<const uint4*>(st + wtile_off<D>(sub * QL + eb / 64, rin, (eb % 64) / 8));
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 fa = half2_bits_to_float2(aw[t]);
        const float2 fb = half2_bits_to_float2(bw[t]);
        const float4 l = myq[4 * j + t];
        p[8 * j + 2 * t] = __fmul2_rn(make_float2(fa.x, fb.x), make_float2(l.x, l.y));
        p[8 * j + 2 * t + 1] = __fmul2_rn(make_float2(fa.y, fb.y), make_float2(l.z, l.w));
      }
    }
    uint32_t out[EPT / 8];
    uint16_t bx[NGH], by[NGH];
    quantize_regs<D, G, W::WROWS>(p, sub, c2, out, bx, by);
    if (with_codes && row < n) store_scales<D, G>(scales, row, sub, bx, by, scale_vec != 0);

    // inverse, from the packed words: the same unpacking, stages and
    // epilogue as the dequantize kernel
    uint32_t w[EPT / 8];
#pragma unroll
    for (int i = 0; i < EPT / 8; ++i) w[i] = out[i] ^ 0x88888888u;
    dequant_front<D, G>(w, bx, by, p);
    fwht_pairs<EPT, LANES, HG, W::WROWS>(p, sub);
    // every lane has read its input and the previous stores have read the
    // code block (waited above): write this tile's output over its input
    __syncwarp();
    if (with_codes) stage_codes<D>(cst, out, sub, rin);
    stage_rows<D>(p, c2, myd, st, sub, rin);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < T::Q; ++q)
        tensor_s2g(&out_maps.q[q], 0, static_cast<int>(tile * W::WROWS), st + q * W::WQB);
      if (with_codes) tensor_s2g(&cmap, 0, static_cast<int>(tile * W::WROWS), cst);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait0();
}

// A barrier that nothing completes, waited on with a short limit: exercises
// the bounded-wait give-up path (fault word) without any real copy.
__global__ void kvq_wait_timeout_kernel(uint32_t limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) { mbar_init(&bar, 1); mbar_fence_init(); }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0, limit);
  if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicOr(&g_kvq_fault, 2u);
}

// The kernels' reciprocal of a group scale, rcp_f16val, evaluated at every
// positive finite fp16 value (bit patterns 0x0001 .. 0x7BFF): out[i] is the
// reciprocal of the fp16 value with bits i + 1, for the host to compare with
// the IEEE quotient.
constexpr int kRcpCount = 0x7BFF;
__global__ void kvq_rcp_table_kernel(float* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < kRcpCount) out[i] = rcp_f16val(half_bits_to_float(static_cast<uint16_t>(i + 1)));
}

// ---------------------------------------------------------------------------
// Launch plumbing.
// ---------------------------------------------------------------------------

std::atomic<int> g_sms[kMaxDevices];

int sm_count(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = g_sms[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Resident blocks per SM of one kernel instance at one block shape on one
// device.  The first call for an instance raises its dynamic shared-memory
// limit to `attr_smem` (the largest shape it is launched with) and asks for
// the largest shared-memory carveout, so kernels launched back to back do not
// make the SMs repartition L1.
template <int KIND, int D, int G, int SHAPE = 0, typename Kernel>
int blocks_per_sm(Kernel k, int dev, int attr_smem, int smem, int threads) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 1;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, attr_smem);
    cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, k, threads, smem) != cudaSuccess || v < 1)
      v = 1;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Launch shape of a streaming kernel (quantize, dequantize) for n vectors.
// Large batches run one block of kWarps warps per SM, whose warps share one
// tile counter.  Batches with fewer than two tiles per such warp run blocks of
// kSmallWarps warps, several per SM, which spreads the few tiles over more SMs
// and starts sooner.  Never more blocks than warp tiles.
constexpr int kSmallWarps = 4;

template <int D>
bool stream_big(int64_t n, int sms) {
  const int64_t tiles = (n + WTile<D>::WROWS - 1) / WTile<D>::WROWS;
  return tiles >= static_cast<int64_t>(sms) * kWarps * 2;
}

template <int KIND, int D, int G, int NW, typename Kernel>
int stream_grid(Kernel k, int dev, int sms, int64_t n, int smem) {
  const int64_t tiles = (n + WTile<D>::WROWS - 1) / WTile<D>::WROWS;
  const int64_t cap = static_cast<int64_t>(sms) * blocks_per_sm<KIND, D, G, NW>(k, dev, smem, smem, NW * 32);
  return static_cast<int>(tiles < cap ? tiles : cap);
}

inline int current_device_sms(int& dev) {
  dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const int sms = sm_count(dev);
  return sms < 1 ? 1 : sms;
}



// One 2-D map per 64-channel quarter of the fp16 rows at `base`: 64 channels
// x n rows, row stride 2D bytes, box 64 x box_rows (one warp tile), 128-byte swizzle.
template <int D>
int make_row_maps(RowMaps& m, const void* base, int64_t n, int box_rows) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  for (int q = 0; q < D / 64; ++q) {
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(2 * D)};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&m.q[q], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                           const_cast<char*>(static_cast<const char*>(base)) + 128 * q, dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      g_last_cuda_error = static_cast<int>(r);
      return KVQ_ERR_LAUNCH;
    }
  }
  return KVQ_OK;
}

// The packed codes at `base` as one 2-D map: D/2 bytes x n rows, box
// D/2 x (one warp tile), swizzled over the row's width (32, 64 or 128 bytes).
template <int D>
int make_code_map(CUtensorMap& m, void* base, int64_t n) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D / 2), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D / 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(D / 2), static_cast<cuuint32_t>(WTile<D>::WROWS)};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = D == 64 ? CU_TENSOR_MAP_SWIZZLE_32B
                               : D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

int check_shape(int D, int G, int64_t n) {
  if (D != 64 && D != 128 && D != 256) return KVQ_ERR_DIM;
  if (G < 16 || G > D || (G & (G - 1)) != 0) return KVQ_ERR_GROUP;
  if (n < 0 || n > kMaxVectors) return KVQ_ERR_COUNT;
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

template <int D, int G, bool INDEXED, int NW>
int launch_quantize_nw(const RowMaps& maps, int dev, int sms, const float* lam, const int8_t* s,
                       int64_t n, uint8_t* packed, uint16_t* scales, const int64_t* row_idx,
                       int64_t cache_rows, cudaStream_t st) {
  auto k = kvq_quantize_kernel<D, G, INDEXED, NW>;
  constexpr bool STG = !INDEXED;
  constexpr int smem = Stream<D>::smem(STG ? Stream<D>::QWARP_S : Stream<D>::QWARP, NW);
  const int grid = stream_grid<INDEXED ? 2 : 0, D, G, NW>(k, dev, sms, n, smem);
  CUtensorMap cmap;
  memset(&cmap, 0, sizeof(cmap));
  if (STG) {
    const int rc = make_code_map<D>(cmap, packed, n);
    if (rc != KVQ_OK) return rc;
  }
  constexpr uintptr_t kScaleRow = (D / G) * 2 < 16 ? (D / G) * 2 : 16;   // bytes of one scale store
  const int svec = (reinterpret_cast<uintptr_t>(scales) % kScaleRow) == 0;
  (void)cudaGetLastError();
  k<<<grid, NW * 32, smem, st>>>(maps, lam, s, n, norm_const(D), packed, scales, row_idx, cache_rows,
                                 svec, cmap);
  return finish_launch();
}

template <int D, int G, bool INDEXED>
int launch_quantize_t(const uint16_t* x, const float* lam, const int8_t* s, int64_t n,
                      uint8_t* packed, uint16_t* scales, const int64_t* row_idx,
                      int64_t cache_rows, cudaStream_t st) {
  RowMaps maps;
  const int rc = make_row_maps<D>(maps, x, n, WTile<D>::WROWS);
  if (rc != KVQ_OK) return rc;
  int dev = 0;
  const int sms = current_device_sms(dev);
  if (stream_big<D>(n, sms))
    return launch_quantize_nw<D, G, INDEXED, kWarps>(maps, dev, sms, lam, s, n, packed, scales,
                                                     row_idx, cache_rows, st);
  return launch_quantize_nw<D, G, INDEXED, kSmallWarps>(maps, dev, sms, lam, s, n, packed, scales,
                                                        row_idx, cache_rows, st);
}

template <int D, int G>
int launch_quantize(const uint16_t* x, const float* lam, const int8_t* s, int64_t n,
                    uint8_t* packed, uint16_t* scales, cudaStream_t st) {
  return launch_quantize_t<D, G, false>(x, lam, s, n, packed, scales, nullptr, n, st);
}

template <int D, int G>
int launch_quantize_rows(const uint16_t* x, const float* lam, const int8_t* s, int64_t n,
                         uint8_t* packed, uint16_t* scales, const int64_t* row_idx,
                         int64_t cache_rows, cudaStream_t st) {
  return launch_quantize_t<D, G, true>(x, lam, s, n, packed, scales, row_idx, cache_rows, st);
}

template <int D, int G, int NW>
int launch_dequantize_nw(const RowMaps& maps, int dev, int sms, const uint8_t* packed,
                         const uint16_t* scales, const float* lam, const int8_t* s, int64_t n,
                         cudaStream_t st) {
  auto k = kvq_dequantize_kernel<D, G, NW>;
  constexpr int smem = Stream<D>::smem(Stream<D>::DWARP, NW);
  const int grid = stream_grid<1, D, G, NW>(k, dev, sms, n, smem);
  CUtensorMap cmap;
  const int rc = make_code_map<D>(cmap, const_cast<uint8_t*>(packed), n);
  if (rc != KVQ_OK) return rc;
  (void)cudaGetLastError();
  k<<<grid, NW * 32, smem, st>>>(cmap, scales, lam, s, n, norm_const(D), maps,
                                 (reinterpret_cast<uintptr_t>(scales) & 15) == 0 ? 1 : 0);
  return finish_launch();
}

template <int D, int G>
int launch_dequantize(const uint8_t* packed, const uint16_t* scales, const float* lam,
                      const int8_t* s, int64_t n, uint16_t* out, cudaStream_t st) {
  RowMaps maps;
  const int rc = make_row_maps<D>(maps, out, n, WTile<D>::WROWS);
  if (rc != KVQ_OK) return rc;
  int dev = 0;
  const int sms = current_device_sms(dev);
  if (stream_big<D>(n, sms))
    return launch_dequantize_nw<D, G, kWarps>(maps, dev, sms, packed, scales, lam, s, n, st);
  return launch_dequantize_nw<D, G, kSmallWarps>(maps, dev, sms, packed, scales, lam, s, n, st);
}

// The tensor-core dequantizer: one block of kWarps warps per SM (or fewer
// blocks than SMs for small batches: never more blocks than warp tiles).
template <int G>
int launch_dequantize_tc(const uint8_t* packed, const uint16_t* scales, const float* lam,
                         const int8_t* s, int64_t n, uint16_t* out, cudaStream_t st) {
  constexpr int D = 128;
  RowMaps maps;
  int rc = make_row_maps<D>(maps, out, n, WTile<D>::WROWS);
  if (rc != KVQ_OK) return rc;
  CUtensorMap cmap;
  rc = make_code_map<D>(cmap, const_cast<uint8_t*>(packed), n);
  if (rc != KVQ_OK) return rc;
  int dev = 0;
  const int sms = current_device_sms(dev);
  auto k = kvq_dequantize_tc_kernel<G, kWarps>;
  constexpr int smem = Stream<D>::smem(Stream<D>::DWARP, kWarps);
  const int grid = stream_grid<3, D, G, kWarps>(k, dev, sms, n, smem);
  (void)cudaGetLastError();
  k<<<grid, kWarps * 32, smem, st>>>(cmap, scales, lam, s, n, norm_const(D), maps,
                                     (reinterpret_cast<uintptr_t>(scales) & 15) == 0 ? 1 : 0);
  return finish_launch();
}

template <int D, int G>
int launch_roundtrip(const uint16_t* x, const float* lam, const int8_t* s, int64_t n,
                     uint16_t* x_hat, uint8_t* packed, uint16_t* scales, cudaStream_t st) {
  auto k = kvq_roundtrip_kernel<D, G>;
  constexpr int smem = RStream<D>::SMEM;
  RowMaps in_maps, out_maps;
  int rc = make_row_maps<D>(in_maps, x, n, WTile<D>::WROWS);
  if (rc == KVQ_OK) rc = make_row_maps<D>(out_maps, x_hat, n, WTile<D>::WROWS);
  if (rc != KVQ_OK) return rc;
  CUtensorMap cmap;
  memset(&cmap, 0, sizeof(cmap));
  if (packed != nullptr) {
    rc = make_code_map<D>(cmap, packed, n);
    if (rc != KVQ_OK) return rc;
  }
  constexpr uintptr_t kScaleRow = (D / G) * 2 < 16 ? (D / G) * 2 : 16;
  const int svec = (reinterpret_cast<uintptr_t>(scales) % kScaleRow) == 0;
  int dev = 0;
  const int sms = current_device_sms(dev);
  const int grid = stream_grid<3, D, G, kRtWarps>(k, dev, sms, n, smem);
  (void)cudaGetLastError();
  k<<<grid, kRtWarps * 32, smem, st>>>(in_maps, out_maps, cmap, lam, s, n, norm_const(D), scales,
                                       packed != nullptr ? 1 : 0, svec);
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
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(scales, 2) || !aligned(lambda, 4))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_DISPATCH(launch_quantize, D, group, x, lambda, signs, n_vec, packed, scales, st);
}

int kvq_quantize_rows(const uint16_t* x, const float* lambda, const int8_t* signs,
                      int64_t n_vec, int D, int group, const int64_t* row_idx,
                      int64_t cache_rows, uint8_t* packed, uint16_t* scales, void* stream) {
  const int rc = check_shape(D, group, n_vec);
  if (rc != KVQ_OK) return rc;
  if (cache_rows < 0) return KVQ_ERR_COUNT;
  if (n_vec == 0) return KVQ_OK;
  if (!x || !lambda || !signs || !row_idx || !packed || !scales) return KVQ_ERR_NULL;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(scales, 2) || !aligned(lambda, 4) ||
      !aligned(row_idx, 8))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_DISPATCH(launch_quantize_rows, D, group, x, lambda, signs, n_vec, packed, scales, row_idx,
               cache_rows, st);
}

int kvq_dequantize(const uint8_t* packed, const uint16_t* scales, const float* lambda,
                   const int8_t* signs, int64_t n_vec, int D, int group, uint16_t* x_out,
                   void* stream) {
  const int rc = check_shape(D, group, n_vec);
  if (rc != KVQ_OK) return rc;
  if (n_vec == 0) return KVQ_OK;
  if (!packed || !scales || !lambda || !signs || !x_out) return KVQ_ERR_NULL;
  if (!aligned(x_out, 16) || !aligned(packed, 16) || !aligned(scales, 2) || !aligned(lambda, 4))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_DISPATCH(launch_dequantize, D, group, packed, scales, lambda, signs, n_vec, x_out, st);
}

int kvq_roundtrip(const uint16_t* x, const float* lambda, const int8_t* signs, int64_t n_vec,
                  int D, int group, uint16_t* x_hat, uint8_t* packed, uint16_t* scales,
                  void* stream) {
  const int rc = check_shape(D, group, n_vec);
  if (rc != KVQ_OK) return rc;
  if (n_vec == 0) return KVQ_OK;
  if (!x || !lambda || !signs || !x_hat) return KVQ_ERR_NULL;
  if ((packed == nullptr) != (scales == nullptr)) return KVQ_ERR_NULL;
  if (!aligned(x, 16) || !aligned(x_hat, 16) || !aligned(lambda, 4) ||
      (packed && (!aligned(packed, 16) || !aligned(scales, 2))))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  KVQ_DISPATCH(launch_roundtrip, D, group, x, lambda, signs, n_vec, x_hat, packed, scales, st);
}

int kvq_fault_status(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kvq_fault, sizeof v) != cudaSuccess) return -1;
  if (clear && v) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_kvq_fault, &zero, sizeof zero) != cudaSuccess) return -1;
  }
  return static_cast<int>(v | kvq_attn_fault_word(clear) | kvq_ex_fault_word(clear));
}

int kvq_selftest_wait_timeout(uint32_t limit, void* stream) {
  (void)cudaGetLastError();
  kvq_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit);
  return finish_launch();
}

int kvq_dequantize_tc(const uint8_t* packed, const uint16_t* scales, const float* lambda,
                      const int8_t* signs, int64_t n_vec, int D, int group, uint16_t* x_out,
                      void* stream) {
  const int rc = check_shape(D, group, n_vec);
  if (rc != KVQ_OK) return rc;
  if (D != 128) return KVQ_ERR_DIM;
  if (group != 16 && group != 32 && group != 64) return KVQ_ERR_GROUP;
  if (n_vec == 0) return KVQ_OK;
  if (!packed || !scales || !lambda || !signs || !x_out) return KVQ_ERR_NULL;
  if (!aligned(x_out, 16) || !aligned(packed, 16) || !aligned(scales, 2) || !aligned(lambda, 4))
    return KVQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (group) {
    case 16: return launch_dequantize_tc<16>(packed, scales, lambda, signs, n_vec, x_out, st);
    case 32: return launch_dequantize_tc<32>(packed, scales, lambda, signs, n_vec, x_out, st);
    default: return launch_dequantize_tc<64>(packed, scales, lambda, signs, n_vec, x_out, st);
  }
}

int kvq_selftest_rcp_f16(float* out, void* stream) {
  if (out == nullptr) return KVQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(out) & 3) != 0) return KVQ_ERR_ALIGN;
  (void)cudaGetLastError();
  kvq_rcp_table_kernel<<<(kRcpCount + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(out);
  return finish_launch();
}

const char* kvq_status_string(int status) {
  switch (status) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_NULL: return "KVQ_ERR_NULL: a required pointer is NULL";
    case KVQ_ERR_ALIGN: return "KVQ_ERR_ALIGN: a pointer is misaligned";
    case KVQ_ERR_DIM: return "KVQ_ERR_DIM: D must be 64, 128 or 256";
    case KVQ_ERR_GROUP: return "KVQ_ERR_GROUP: group must be a power of two in [16, D]";
    case KVQ_ERR_COUNT: return "KVQ_ERR_COUNT: n_vec must be in [0, 2^31 - 256]";
    case KVQ_ERR_LAUNCH: return "KVQ_ERR_LAUNCH: the kernel launch failed";
    default: return "unknown kvq status";
  }
}

int kvq_last_cuda_error(void) {
  if (g_last_cuda_error) return g_last_cuda_error;
  if (const int e = kvq_attn_last_cuda_error()) return e;
  return kvq_ex_last_cuda_error();
}

int kvq_version(void) { return (1 << 16) | 2; }

}  // extern "C"
