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
// The rotation is the SRHT above, or (flags bit KVQ_SRFT) the SRFT of the same
// summary: pack(F diag(s) x), F the unitary DFT, as a 64-point Stockham FFT
// of the channel pairs plus the Hermitian unpacking.
//
// D = 128; G in {16, 32, 64}.  One lane holds a whole vector as 64 packed
// fp32 pairs; each warp streams 32-vector tiles through its own
// double-buffered ring, and the 12 warps of a block (one block per SM) claim
// tiles of a contiguous range from a shared counter.  fp16 rows move by
// swizzled tensor copies; the codes leave the quantisers through the stage
// their tile came from and one tensor store, and enter the dequantisers by a
// swizzled tensor copy; scales move by bulk copies.  A warp tile lies inside one lambda
// table (lambda_rows is a multiple of 32 when there are several), so the warp
// rebuilds its per-channel table in shared memory when a tile's table differs
// from the last one's.  Every step is the oracle's IEEE operation in the
// oracle's order: the scale is a correctly rounded division by 7 or 127, 1/S
// and 1/lambda correctly rounded reciprocals, so results are bit-identical.
// Bounded waits as in the base kernels (a warp that gives up sets bit 0 of the
// fault word and returns).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "kvq.h"

namespace {

constexpr unsigned kFullMask = 0xffffffffu;

#include "kvq_async.cuh"
#include "kvq_arith.cuh"
#include "kvq_ex.cuh"

constexpr int kD = 128;                 // channels (one lane per vector)
constexpr int kNP = kD / 2;             // packed pairs (v[m], v[m+64])
constexpr int kQW = 12;                 // warps of a WHT quantize block (one per SM, 170 registers)
constexpr int kWR = 32;                 // vectors per warp tile
constexpr int kQB = kWR * 128;          // bytes of one 64-channel quarter of a tile
constexpr int kXStage = 2 * kQB;        // bytes of one fp16 warp tile
constexpr uint32_t kSpinX = 1u << 22;

__device__ unsigned int g_ex_fault = 0;   // bit 0: a bounded wait gave up
thread_local int g_ex_cuda_error = 0;

struct ExMaps {
  CUtensorMap q[2];                     // fp16 rows: two 64-channel quarters
};

template <int BITS>
struct Fmt {
  static constexpr int CB = BITS == 4 ? kD / 2 : kD;   // code bytes per row
  static constexpr int QMAX = BITS == 4 ? 7 : 127;
};

__device__ __forceinline__ int xtile_off(int q, int t, int c) {
  return q * kQB + t * 128 + ((c ^ (t & 7)) << 4);
}

// The warp's per-channel table in the pair layout of the base kernels:
// tab[q] = (t[2q], t[2q+64], t[2q+1], t[2q+65]); mode 0: lambda * s,
// 1: fp32(lambda c) (lambda after the rotation: lambda and the normalisation
// are one factor), 2: s * (1/lambda), 3: fp32(c / lambda) (its inverse,
// applied before the transform).  Each lane fills one float4.
__device__ __forceinline__ void build_table(float4* tab, const ExArgs& a, int id, int mode, int lane) {
  const float* lr = a.lam + static_cast<int64_t>(id) * kD;
  const int ch[4] = {2 * lane, 2 * lane + kNP, 2 * lane + 1, 2 * lane + 1 + kNP};
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float l = lr[ch[k]];
    float t;
    if (mode == 0) t = l;
    else if (mode == 1) t = __fmul_rn(l, a.c);
    else if (mode == 2) t = __frcp_rn(l);
    else t = __fdiv_rn(a.c, l);
    v[k] = ((mode == 0 || mode == 2) && a.sgn[ch[k]] < 0) ? -t : t;
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

// Header of a block of nw warps: per-warp tables (nw x 512 B), the sign
// table (512 B), then two mbarriers and two tile ids per warp and the claim
// counter.
__host__ __device__ constexpr int hdr_bars(int nw) { return nw * 512 + 512; }
__host__ __device__ constexpr int hdr_bytes(int nw) { return hdr_bars(nw) + 24 * nw + 16; }

// ---------------------------------------------------------------------------
// Quantize variants: fp16 [n][128] -> codes [n][CB] + fp16 scales [n][128/G].
// ---------------------------------------------------------------------------
template <int G, int BITS, bool AFTER>
__global__ void __launch_bounds__(kQW * 32, 1)
kvq_quantize_ex_kernel(const __grid_constant__ ExMaps maps, const ExArgs a,
                       const __grid_constant__ CUtensorMap cmap, uint16_t* __restrict__ scales) {
  using F = Fmt<BITS>;
  constexpr int NGH = kNP / G;          // groups per half of the lane's channels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* wsm = smem + warp * 2 * kXStage;
  uint8_t* hdr = smem + kQW * 2 * kXStage;
  float4* tab = reinterpret_cast<float4*>(hdr) + warp * 32;                       // 512 B per warp
  float4* stab = reinterpret_cast<float4*>(hdr + kQW * 512);                        // +-1, 512 B
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + hdr_bars(kQW)) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + hdr_bars(kQW) + 16 * kQW) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + hdr_bars(kQW) + 24 * kQW);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  if (tid < 32) build_signs(stab, a, tid);
  __syncthreads();

  const int64_t ntiles = (a.n + kWR - 1) / kWR;
  // The block owns a contiguous range of tiles, so a warp's tiles stay in one
  // lambda table for long stretches (a table spans lambda_rows / 32 tiles).
  const int64_t per = ntiles / gridDim.x, rem = ntiles % gridDim.x;
  const int64_t first = blockIdx.x * per + (blockIdx.x < rem ? blockIdx.x : rem);
  const unsigned int mine = static_cast<unsigned int>(per + (blockIdx.x < rem ? 1 : 0));
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(first + i) : -1;
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
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinX);   // the stage that gave up, once more
      // only the first tile has the other stage's copy in flight
      if (k == 0 && tq[1] >= 0) mbar_wait(&bar[1], 0, kSpinX);
      if (lane == 0) bulk_wait0();
      return;
    }
    if (k > 0) {
      // the other stage holds the previous tile's staged codes: once their
      // store has read them, it takes the next tile
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
      refill(stage ^ 1);
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

    fwht_pairs<kD, 1>(p, 0);
    if constexpr (AFTER) {
#pragma unroll
      for (int q = 0; q < kNP / 2; ++q) {
        const float4 l = tab[q];                      // fp32(lambda c)
        p[2 * q] = __fmul2_rn(p[2 * q], make_float2(l.x, l.y));
        p[2 * q + 1] = __fmul2_rn(p[2 * q + 1], make_float2(l.z, l.w));
      }
    } else {
#pragma unroll
      for (int m = 0; m < kNP; ++m) p[m] = __fmul2_rn(p[m], c2);
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
      bx[j] = group_scale_q<F::QMAX>(ax, rx[j]);
      by[j] = group_scale_q<F::QMAX>(ay, ry[j]);
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
    // the codes leave through the stage this tile came from (every lane has
    // read it), swizzled as code_chunk reads, by one tensor store that skips
    // rows past n
    __syncwarp();
    {
      uint8_t* cst = wsm + stage * kXStage;
      const int swz = ((lane * F::CB) >> 7) & (F::CB / 16 - 1);
#pragma unroll
      for (int k4 = 0; k4 < F::CB / 16; ++k4)
        *reinterpret_cast<uint4*>(cst + lane * F::CB + ((k4 ^ swz) << 4)) =
            make_uint4(out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3]);
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tensor_s2g(&cmap, 0, static_cast<int>(tile * kWR), cst);
        bulk_commit();
      }
    }
    if (active) {
      uint16_t* srow = scales + row * (kD / G);
#pragma unroll
      for (int j = 0; j < NGH; ++j) {
        srow[j] = bx[j];
        srow[NGH + j] = by[j];
      }
    }
  }
  if (lane == 0) bulk_wait0();
}

// ---------------------------------------------------------------------------
// Dequantize variants: codes [n][CB] + fp16 scales [n][128/G] -> fp16 [n][128].
// ---------------------------------------------------------------------------
// A warp's shared memory: the swizzled fp16 staging tile its tensor stores
// read (first, 1 KiB aligned), the two stages' code tiles (each a multiple
// of 1 KiB, so the copy engine's swizzle lines up with code_chunk), then the
// two stages' scales.
template <int G, int BITS>
struct DeqLayout {
  static constexpr int WC = kWR * Fmt<BITS>::CB;          // codes of one warp tile: 2 or 4 KiB
  static constexpr int SPR = (kD / G) * 2;                // scale bytes per row
  static constexpr int WS = kWR * SPR;                    // scales of one warp tile (<= 512)
  static constexpr int SC = 2 * WC;                       // offset of the scales after the staging tile
  static constexpr int WARP = (kXStage + 2 * WC + 2 * WS + 1023) / 1024 * 1024;
};

// Warps of a dequantize block (one block per SM): 12, at most 168 registers a
// thread (the codes are unpacked, staged and converted a block of pairs at a
// time, so that only that block's fp16 halves sit beside the fp32 row).
__host__ __device__ constexpr int deq_warps(bool) { return 12; }

// 16-byte chunk c of lane `lane`'s row of a code tile written by a tensor copy
// swizzled over the row's CB bytes (64 or 128): chunk c of row t sits at
// chunk c ^ ((t * CB / 128) mod CB/16), so the eight rows a quarter-warp
// reads fall in distinct banks.
template <int CB>
__device__ __forceinline__ uint4 code_chunk(const uint8_t* tile, int lane, int c) {
  const int swz = ((lane * CB) >> 7) & (CB / 16 - 1);
  return *reinterpret_cast<const uint4*>(tile + lane * CB + ((c ^ swz) << 4));
}

template <int G, int BITS, bool AFTER>
__global__ void __launch_bounds__(deq_warps(AFTER) * 32, 1)
kvq_dequantize_ex_kernel(const __grid_constant__ CUtensorMap cmap,
                         const uint16_t* __restrict__ scales,
                         const ExArgs a, const __grid_constant__ ExMaps omaps, int scale_copy) {
  using F = Fmt<BITS>;
  using L = DeqLayout<G, BITS>;
  constexpr int NW = deq_warps(AFTER);
  constexpr int NGH = kNP / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* stage_out = smem + warp * L::WARP;              // swizzled fp16 staging tile
  uint8_t* wsm = stage_out + kXStage;                      // two code tiles, then two scale blocks
  uint8_t* hdr = smem + NW * L::WARP;
  float4* tab = reinterpret_cast<float4*>(hdr) + warp * 32;
  float4* stab = reinterpret_cast<float4*>(hdr + NW * 512);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + hdr_bars(NW)) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + hdr_bars(NW) + 16 * NW) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + hdr_bars(NW) + 24 * NW);
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  if (tid < 32) build_signs(stab, a, tid);
  __syncthreads();

  const int64_t ntiles = (a.n + kWR - 1) / kWR;
  // The block owns a contiguous range of tiles, so a warp's tiles stay in one
  // lambda table for long stretches (a table spans lambda_rows / 32 tiles).
  const int64_t per = ntiles / gridDim.x, rem = ntiles % gridDim.x;
  const int64_t first = blockIdx.x * per + (blockIdx.x < rem ? blockIdx.x : rem);
  const unsigned int mine = static_cast<unsigned int>(per + (blockIdx.x < rem ? 1 : 0));
  auto claim = [&]() -> int {
    unsigned int i = 0;
    if (lane == 0) i = atomicAdd(next, 1u);
    i = __shfl_sync(kFullMask, i, 0);
    return i < mine ? static_cast<int>(first + i) : -1;
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
    const uint32_t sb = scale_bytes(t);
    // swizzled tensor copy of the code rows: the copy engine fills the whole
    // box (zeros past the last row)
    mbar_expect_tx(&bar[stage], static_cast<uint32_t>(L::WC) + sb);
    tensor_g2s(wsm + stage * L::WC, &cmap, 0, static_cast<int>(row0), &bar[stage]);
    if (sb) bulk_g2s(wsm + L::SC + stage * L::WS, reinterpret_cast<const uint8_t*>(scales) + row0 * L::SPR, sb, &bar[stage]);
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
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinX);   // the stage that gave up, once more
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinX);
      if (lane == 0) bulk_wait0();
      return;
    }
    const int id = table_id(a, tile * kWR);
    if (id != cached) {
      build_table(tab, a, id, AFTER ? 3 : 2, lane);
      cached = id;
      __syncwarp();
    }
    const uint8_t* st = wsm + stage * L::WC;
    const uint16_t* srow = sc_smem ? reinterpret_cast<const uint16_t*>(wsm + L::SC + stage * L::WS + lane * L::SPR)
                                   : scales + rrow * (kD / G);
    uint16_t sx[NGH], sy[NGH];
#pragma unroll
    for (int j = 0; j < NGH; ++j) {
      sx[j] = srow[j];
      sy[j] = srow[NGH + j];
    }
    // With lambda before the rotation u = q S, and every butterfly stage inside
    // a group keeps u an exact multiple of S: the stages h < HF run on the fp16
    // integers (sums of at most 8 * 64 = 512 for int4 through all in-group
    // stages, 128 * 16 = 2048 for int8 through four), then u = W S exactly by
    // one mixed fma (W S has at most 23 significant bits), the same fp32
    // values as the oracle's stage-by-stage sums.  With lambda after, 1/lambda
    // comes before the transform and every stage runs in fp32: u = q S
    // (exact), then u fp32(c / lambda).
    constexpr int HF = AFTER ? 1 : (BITS == 4 ? (G < kNP ? G : kNP) : 16);
    constexpr int PW = BITS == 4 ? 8 : 4;               // pairs a code word (of each half) holds
    constexpr int HB = HF > PW ? HF : PW;               // pairs unpacked, staged and converted at a time
    // The codes of the pair (m, m+64) as exact fp16 integers, one block of HB
    // pairs at a time (the in-group stages stay inside a block), so that only
    // a block's halves sit beside the fp32 row.  Word w of a row is word w % 4
    // of its swizzled 16-byte chunk w / 4.
    __half2 hq[kNP];
    float2 p[kNP];
    auto to_row = [&](int m) {
      p[m] = make_float2(mul_f16_f32(__low2half(hq[m]), sx[m / G]), mul_f16_f32(__high2half(hq[m]), sy[m / G]));
      if constexpr (AFTER) {
        const float4 l = tab[m / 2];                  // fp32(c / lambda) of the pairs 2q, 2q + 1
        p[m] = __fmul2_rn(p[m], (m & 1) ? make_float2(l.z, l.w) : make_float2(l.x, l.y));
      }
    };
    uint32_t ra[4], rb[4];
    auto unpack_word = [&](int kw) {                    // the pairs PW kw .. PW kw + PW - 1
      if constexpr (BITS == 4) {
        const __half2 bias = __floats2half2_rn(1032.0f, 1032.0f);
        if (kw % 4 == 0) {              // channels 8 kw .. 8 kw + 31 and 64 + the same
          const uint4 ca = code_chunk<F::CB>(st, lane, kw / 4), cb = code_chunk<F::CB>(st, lane, 2 + kw / 4);
          ra[0] = ca.x; ra[1] = ca.y; ra[2] = ca.z; ra[3] = ca.w;
          rb[0] = cb.x; rb[1] = cb.y; rb[2] = cb.z; rb[3] = cb.w;
        }
        const uint32_t wa = ra[kw % 4] ^ 0x88888888u;
        const uint32_t wb = rb[kw % 4] ^ 0x88888888u;
        const uint32_t wa4 = wa >> 4, wb4 = wb >> 4;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t sel = 0x0400u | (t << 8) | t;
          const uint32_t e0 = (__byte_perm(wa, wb, sel) & 0x000F000Fu) | 0x64006400u;
          const uint32_t e1 = (__byte_perm(wa4, wb4, sel) & 0x000F000Fu) | 0x64006400u;
          hq[8 * kw + 2 * t] = __hsub2(*reinterpret_cast<const __half2*>(&e0), bias);
          hq[8 * kw + 2 * t + 1] = __hsub2(*reinterpret_cast<const __half2*>(&e1), bias);
        }
      } else {
        const __half2 bias = __floats2half2_rn(1152.0f, 1152.0f);
        const uint4 ca = code_chunk<F::CB>(st, lane, kw >> 2);
        const uint4 cb = code_chunk<F::CB>(st, lane, (kw + kNP / 4) >> 2);
        const uint32_t xa[4] = {ca.x, ca.y, ca.z, ca.w}, xb[4] = {cb.x, cb.y, cb.z, cb.w};
        const uint32_t wa = xa[kw & 3] ^ 0x80808080u;
        const uint32_t wb = xb[kw & 3] ^ 0x80808080u;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t sel = 0x0400u | (t << 8) | t;
          const uint32_t e = (__byte_perm(wa, wb, sel) & 0x00FF00FFu) | 0x64006400u;
          hq[4 * kw + t] = __hsub2(*reinterpret_cast<const __half2*>(&e), bias);
        }
      }
    };
#pragma unroll
    for (int b0 = 0; b0 < kNP; b0 += HB) {
#pragma unroll
      for (int kw = b0 / PW; kw < (b0 + HB) / PW; ++kw) unpack_word(kw);
#pragma unroll
      for (int h = 1; h < HF; h <<= 1) {
#pragma unroll
        for (int m = b0; m < b0 + HB; ++m) {
          if ((m & h) == 0) {
            const __half2 a2 = hq[m], b2 = hq[m + h];
            hq[m] = __hadd2(a2, b2);
            hq[m + h] = __hsub2(a2, b2);
          }
        }
      }
#pragma unroll
      for (int m = b0; m < b0 + HB; ++m) to_row(m);
    }
    __syncwarp();                       // codes and scales consumed: refill the stage
    refill(stage);
    fwht_pairs<kD, 1, HF>(p, 0);
    if (lane == 0) bulk_wait_read0();   // the previous tile's stores have read the staging tile
    __syncwarp();
#pragma unroll
    for (int k4 = 0; k4 < kNP / 8; ++k4) {
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int q = 4 * k4 + t;
        float2 a0, a1;
        if constexpr (AFTER) {                        // signs only: exact
          const float4 sg = stab[q];
          a0 = __fmul2_rn(p[2 * q], make_float2(sg.x, sg.y));
          a1 = __fmul2_rn(p[2 * q + 1], make_float2(sg.z, sg.w));
        } else {
          const float4 l = tab[q];                    // s * (1/lambda)
          a0 = __fmul2_rn(__fmul2_rn(p[2 * q], c2), make_float2(l.x, l.y));
          a1 = __fmul2_rn(__fmul2_rn(p[2 * q + 1], c2), make_float2(l.z, l.w));
        }
        lo[t] = float2_to_half2_bits(a0.x, a1.x);    // channels 2q, 2q+1
        hi[t] = float2_to_half2_bits(a0.y, a1.y);    // channels 64+2q, 64+2q+1
      }
      *reinterpret_cast<uint4*>(stage_out + xtile_off(0, lane, k4)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(stage_out + xtile_off(1, lane, k4)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
    fence_proxy_async();                // generic-proxy writes -> visible to the tensor stores
    __syncwarp();
    if (lane == 0) {
      tensor_s2g(&omaps.q[0], 0, static_cast<int>(tile * kWR), stage_out);
      tensor_s2g(&omaps.q[1], 0, static_cast<int>(tile * kWR), stage_out + kQB);
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait0();
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
int ex_grid(Kernel k, int64_t n, int smem, int threads, std::atomic<int>* ready) {
  int dev = 0;
  const int sms = ex_sms(dev);
  int occ = ready[dev].load(std::memory_order_relaxed);
  if (occ == 0) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, threads, smem) != cudaSuccess || occ < 1) occ = 1;
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

// D: 128 with the Walsh-Hadamard rotation; 64, 96, 128 or 256 with the SRFT.
int check_ex(int D, int G, int bits, int64_t n, int64_t lambda_rows, int n_lambda, bool srft) {
  if (srft ? (D != 64 && D != 96 && D != 128 && D != 256) : D != kD) return KVQ_ERR_DIM;
  if ((G != 16 && G != 32 && G != 64) || D % G != 0) return KVQ_ERR_GROUP;
  if (bits != 4 && bits != 8) return KVQ_ERR_GROUP;
  if (n < 0 || n > (int64_t{1} << 31) - 256 || n_lambda < 1 || lambda_rows < 1 ||
      (n_lambda > 1 && lambda_rows % kWR != 0))
    return KVQ_ERR_COUNT;
  return KVQ_OK;
}

int encode_x_maps(ExMaps& maps, const uint16_t* x, int64_t n);
int encode_code_map(CUtensorMap& map, const uint8_t* codes, int64_t n, int cb);

template <int G, int BITS, bool AFTER>
int launch_qex(const uint16_t* x, const ExArgs& a, uint8_t* codes, uint16_t* scales, cudaStream_t st) {
  ExMaps maps;
  const int rc = encode_x_maps(maps, x, a.n);
  if (rc != KVQ_OK) return rc;
  auto k = kvq_quantize_ex_kernel<G, BITS, AFTER>;
  constexpr int smem = 1024 + kQW * 2 * kXStage + hdr_bytes(kQW);
  static std::atomic<int> ready[64];
  const int grid = ex_grid(k, a.n, smem, kQW * 32, ready);
  CUtensorMap cmap;
  const int rc2 = encode_code_map(cmap, codes, a.n, Fmt<BITS>::CB);
  if (rc2 != KVQ_OK) return rc2;
  (void)cudaGetLastError();
  k<<<grid, kQW * 32, smem, st>>>(maps, a, cmap, scales);
  return finish_ex();
}

template <int G, int BITS, bool AFTER>
int launch_dex(const uint8_t* codes, const uint16_t* scales, const ExArgs& a, uint16_t* out,
               cudaStream_t st) {
  using L = DeqLayout<G, BITS>;
  ExMaps omaps;
  const int rc = encode_x_maps(omaps, out, a.n);
  if (rc != KVQ_OK) return rc;
  auto k = kvq_dequantize_ex_kernel<G, BITS, AFTER>;
  constexpr int NW = deq_warps(AFTER);
  constexpr int smem = 1024 + NW * L::WARP + hdr_bytes(NW);
  static std::atomic<int> ready[64];
  const int grid = ex_grid(k, a.n, smem, NW * 32, ready);
  CUtensorMap cmap;
  const int rc2 = encode_code_map(cmap, codes, a.n, Fmt<BITS>::CB);
  if (rc2 != KVQ_OK) return rc2;
  (void)cudaGetLastError();
  k<<<grid, NW * 32, smem, st>>>(cmap, scales, a, omaps,
                                  (reinterpret_cast<uintptr_t>(scales) & 15) == 0 ? 1 : 0);
  return finish_ex();
}


int encode_x_maps(ExMaps& maps, const uint16_t* x, int64_t n) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  for (int q = 0; q < 2; ++q) {
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(n)};
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
  return KVQ_OK;
}

// The codes [n][cb] (cb = 64 or 128 bytes) as one 2-D map with a box of one
// warp tile, swizzled over the row's cb bytes (the layout code_chunk reads).
// Every variant quantiser stores its codes through it, and the int8
// dequantisers read them through it (the int4 dequantisers, whose arithmetic
// leaves shared memory idle, measured faster with plain bulk copies of the
// linear 64-byte rows).
int encode_code_map(CUtensorMap& map, const uint8_t* codes, int64_t n, int cb) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cb), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cb)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(cb), kWR};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         cb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_ex_cuda_error = static_cast<int>(r);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
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

// The SRFT codec, one translation unit per D (kvq_srft_d<D>.cu), after the
// checks below.
#define KVQ_SRFT_DECL(D)                                                                          \
  int kvq_srft_quantize_##D(const uint16_t* x, const float* lambda, const int8_t* signs, int64_t n, \
                            int group, int bits, bool after, int64_t lambda_rows, int n_lambda,      \
                            uint8_t* codes, uint16_t* scales, cudaStream_t st);                      \
  int kvq_srft_dequantize_##D(const uint8_t* codes, const uint16_t* scales, const float* lambda,     \
                              const int8_t* signs, int64_t n, int group, int bits, bool after,       \
                              int64_t lambda_rows, int n_lambda, uint16_t* out, cudaStream_t st);    \
  unsigned int kvq_srft_fault_word_##D(int clear);                                                   \
  int kvq_srft_last_cuda_error_##D();
KVQ_SRFT_DECL(64)
KVQ_SRFT_DECL(96)
KVQ_SRFT_DECL(128)
KVQ_SRFT_DECL(256)

// Read (and optionally clear) the variant kernels' fault words; used by
// kvq_fault_status.  The SRFT units' words are included.
__attribute__((visibility("hidden"))) unsigned int kvq_ex_fault_word(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ex_fault, sizeof(v)) != cudaSuccess) return 0;
  if (clear && v) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_ex_fault, &zero, sizeof(zero));
  }
  return v | kvq_srft_fault_word_64(clear) | kvq_srft_fault_word_96(clear) |
         kvq_srft_fault_word_128(clear) | kvq_srft_fault_word_256(clear);
}
__attribute__((visibility("hidden"))) int kvq_ex_last_cuda_error() {
  if (g_ex_cuda_error) return g_ex_cuda_error;
  if (const int e = kvq_srft_last_cuda_error_64()) return e;
  if (const int e = kvq_srft_last_cuda_error_96()) return e;
  if (const int e = kvq_srft_last_cuda_error_128()) return e;
  return kvq_srft_last_cuda_error_256();
}

extern "C" {

int kvq_quantize_ex(const uint16_t* x, const float* lambda, const int8_t* signs, int64_t n_vec,
                    int D, int group, int bits, int flags, int64_t lambda_rows,
                    int n_lambda, uint8_t* codes, uint16_t* scales, void* stream) {
  const int rc = check_ex(D, group, bits, n_vec, lambda_rows, n_lambda, (flags & 2) != 0);
  if (rc != KVQ_OK) return rc;
  if ((flags & ~3) != 0) return KVQ_ERR_GROUP;
  if (n_vec == 0) return KVQ_OK;
  if (!x || !lambda || !signs || !codes || !scales) return KVQ_ERR_NULL;
  if (!aligned_to(x, 16) || !aligned_to(codes, 16) || !aligned_to(scales, 2) || !aligned_to(lambda, 4))
    return KVQ_ERR_ALIGN;
  ExArgs a{lambda, signs, n_vec, lambda_rows, n_lambda,
           static_cast<float>(1.0 / std::sqrt(static_cast<double>(kD)))};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool lambda_after = (flags & 1) != 0;
  if (flags & 2) {
#define KVQ_SRFT_Q(DD) \
  return kvq_srft_quantize_##DD(x, lambda, signs, n_vec, group, bits, lambda_after, lambda_rows, n_lambda, codes, scales, st)
    switch (D) {
      case 64: KVQ_SRFT_Q(64);
      case 96: KVQ_SRFT_Q(96);
      case 128: KVQ_SRFT_Q(128);
      default: KVQ_SRFT_Q(256);
    }
#undef KVQ_SRFT_Q
  }
  KVQ_EX_DISPATCH(launch_qex, x, a, codes, scales, st)
}

int kvq_dequantize_ex(const uint8_t* codes, const uint16_t* scales, const float* lambda,
                      const int8_t* signs, int64_t n_vec, int D, int group, int bits,
                      int flags, int64_t lambda_rows, int n_lambda, uint16_t* x_out,
                      void* stream) {
  const int rc = check_ex(D, group, bits, n_vec, lambda_rows, n_lambda, (flags & 2) != 0);
  if (rc != KVQ_OK) return rc;
  if ((flags & ~3) != 0) return KVQ_ERR_GROUP;
  if (n_vec == 0) return KVQ_OK;
  if (!codes || !scales || !lambda || !signs || !x_out) return KVQ_ERR_NULL;
  if (!aligned_to(codes, 16) || !aligned_to(x_out, 16) || !aligned_to(scales, 2) || !aligned_to(lambda, 4))
    return KVQ_ERR_ALIGN;
  ExArgs a{lambda, signs, n_vec, lambda_rows, n_lambda,
           static_cast<float>(1.0 / std::sqrt(static_cast<double>(kD)))};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool lambda_after = (flags & 1) != 0;
  if (flags & 2) {
#define KVQ_SRFT_DQ(DD) \
  return kvq_srft_dequantize_##DD(codes, scales, lambda, signs, n_vec, group, bits, lambda_after, lambda_rows, n_lambda, x_out, st)
    switch (D) {
      case 64: KVQ_SRFT_DQ(64);
      case 96: KVQ_SRFT_DQ(96);
      case 128: KVQ_SRFT_DQ(128);
      default: KVQ_SRFT_DQ(256);
    }
#undef KVQ_SRFT_DQ
  }
  KVQ_EX_DISPATCH(launch_dex, codes, scales, a, x_out, st)
}

}  // extern "C"
