// kvq_srft.cuh -- the SRFT rotation of the variant codec for B200 (sm_100a):
// the kernels behind kvq_quantize_ex / kvq_dequantize_ex with flags bit
// KVQ_SRFT (include/kvq.h), at D = 64, 96, 128 and 256, group sizes 16, 32
// and 64, int4 or int8 codes, lambda before or after the rotation, one lambda
// table per range of rows.  Each kvq_srft_d<D>.cu includes this file with
// KVQ_SRFT_D set and instantiates that head dimension, so the four compile in
// parallel; every unit has its own fault word, read through its
// kvq_srft_fault_word_<D>.
//
// Streaming as in the other codec kernels: each warp streams warp tiles (32
// vectors, 16 at D = 256) through its own double-buffered shared-memory ring
// and the warps of a block (8, one block per SM) claim tiles of a contiguous
// range from a shared counter.  fp16 rows arrive by swizzled tensor copies
// (one per 64-channel box, plus a 32-channel box at D = 96); the codes leave
// the quantiser through the stage their tile came from and one tensor store,
// and enter the dequantiser by a bulk copy; the dequantiser's fp16 rows leave
// through a swizzled staging tile and tensor stores.  No copy uses multicast.
// Every mbarrier wait is bounded: a warp that gives up sets the fault word,
// drains its copies and returns.  Compiled with --fmad=false; every rounding
// is one IEEE operation in the order the oracle states.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "kvq.h"

#ifndef KVQ_SRFT_D
#error "define KVQ_SRFT_D (64, 96, 128 or 256) before including kvq_srft.cuh"
#endif

namespace {

constexpr unsigned kFullMask = 0xffffffffu;

#include "kvq_async.cuh"
#include "kvq_arith.cuh"
#include "kvq_ex.cuh"
#include "kvq_fft.cuh"

// Warps of a block (one block per SM): 12, whose 168 registers a thread the
// kernels fit with at most a few bytes of spill; 16 at D = 64, whose kernels
// need fewer than 128.
template <int D, bool DEQ>
__host__ __device__ constexpr int sr_warps() { return D == 64 ? 16 : 12; }
constexpr uint32_t kSpinX = 1u << 22;   // bounded mbarrier waits

__device__ unsigned int g_ex_fault = 0;   // bit 0: a bounded wait gave up

// ---------------------------------------------------------------------------
// The SRFT variants (flags bit KVQ_SRFT).  SRFT(x) = pack(F diag(s) x), F the
// unitary DFT ("When Quantization Is Free", technical summary, Methodologie
// 1), computed as the paper's kernel does (Methodologie 2): the length-N =
// D/2 complex FFT of the channel pairs z_n = v_2n + i v_2n+1 in Stockham
// stages (radix 2 while the length is even, then one radix-3 stage: the
// abstract picks the SRFT for mixed radix, so D = 96 runs 2 2 2 2 3), then the
// Hermitian unpacking into y0 = X_0, y1 = X_N, (y_2k, y_2k+1) =
// sqrt(2) (Re, Im) X_k, all / sqrt(D).  The arithmetic is, operation for
// operation, the reading the oracle states:
//   * twiddles are the fp32 values nearest the exact roots of unity (built on
//     the host); a product by 1, -1, i or -i is exact (the operand, negated or
//     with its parts swapped); in any other complex product each part is one
//     rounded product and one fused multiply-add;
//   * the unpacking forms bins k and N-k together: E = Z_k + conj Z_(N-k),
//     O = (Z_k - conj Z_(N-k)) / i, T = omega_D^k O, 2 X_k = E + T,
//     2 X_(N-k) = conj(E - T); its factor 1/2 sits in the normalisation,
//     fp32(1/sqrt(2D)) (fp32(1/sqrt(D)) on X_0 and X_N);
//   * the inverse is the transpose, step by step in reverse order: the
//     scaling, the adjoint unpacking (Z_k = E + iT, Z_(N-k) = conj(E - iT),
//     T = (U_k - conj U_(N-k)) conj(omega_D^k)), the adjoint (DIT) stages;
//   * with lambda after the rotation, lambda and the normalisation are one
//     per-channel factor fp32(lambda_i c_i) (inverse: fp32(c_i / lambda_i)
//     before the transform), and the signs are exact sign-bit flips of the
//     fp16 input and output.
// One lane holds a whole vector (D <= 128) as N packed fp32 pairs, or (D =
// 256) two lanes l and l ^ 16 share one: the first stage, which pairs z_p with
// z_(p+64), reads the whole row from shared memory and lane `sub` keeps the
// outputs of parity sub, so each lane then runs a 64-point FFT on its own bins
// (the even or the odd ones); the inverse's last stage, the one transpose
// stage that pairs the two lanes' bins, exchanges half of them by shuffles.
// ---------------------------------------------------------------------------

template <int D>
struct Sr {
  static_assert(D == 64 || D == 96 || D == 128 || D == 256, "SRFT lengths");
  static constexpr int N = D / 2;                   // complex FFT length
  static constexpr int LANES = D == 256 ? 2 : 1;    // lanes per vector
  static constexpr int NL = N / LANES;              // complex values a lane holds
  static constexpr int WR = 32 / LANES;             // vectors per warp tile
  static constexpr int NB = D / 64;                 // 64-channel boxes of a row (128 B each)
  static constexpr int TAIL = D % 64;               // 0, or a 32-channel box (64 B a row)
  static constexpr int NMAP = NB + (TAIL ? 1 : 0);
  static constexpr int TILE = WR * 2 * D;           // bytes of one fp16 warp tile
};

template <int D, int BITS>
struct SrFmt {
  static constexpr int CB = BITS == 4 ? D / 2 : D;  // code bytes per row
  static constexpr int QMAX = BITS == 4 ? 7 : 127;
  // swizzle of the code tiles' tensor copies: over the row's 64 or 128 bytes
  // where the row is that wide, none otherwise
  static constexpr int SWZ = CB == 64 ? 64 : CB == 128 ? 128 : 0;
};

struct SrMaps {
  CUtensorMap q[4];                     // fp16 rows: up to four 64-channel boxes (or 64 + 32)
};

template <int D>
struct SrTw {
  float2 wn[D / 2];                     // omega_N^k, k < N
  float2 wd[D / 2 + 1];                 // omega_D^k, k <= N
};

// Byte offset of 16-byte chunk c (channels 8c .. 8c+7) of row t in an fp16
// warp tile: 64-channel boxes with the 128-byte swizzle, then (D = 96) a
// 32-channel box with the 64-byte swizzle.
template <int D>
__device__ __forceinline__ int sr_off(int t, int c) {
  using S = Sr<D>;
  if (c < 8 * S::NB) return (c >> 3) * (S::WR * 128) + t * 128 + (((c & 7) ^ (t & 7)) << 4);
  const int cc = c - 8 * S::NB;
  return S::NB * (S::WR * 128) + t * 64 + ((cc ^ ((t >> 1) & 3)) << 4);
}

// Byte offset of 16-byte chunk k of row t of a code tile, in the layout the
// code map's tensor copies use.
template <int CB, int SWZ>
__device__ __forceinline__ int sr_code_off(int t, int k) {
  if constexpr (SWZ == 128) return t * CB + ((k ^ (t & 7)) << 4);
  else if constexpr (SWZ == 64) return t * CB + ((k ^ ((t >> 1) & 3)) << 4);
  else return t * CB + (k << 4);
}

// Header of an SRFT block of nw warps: per-warp tables (nw x 4D bytes), the
// sign-bit masks (D/2 words), then two mbarriers and two tile ids per warp and
// the claim counter.
template <int D>
__host__ __device__ constexpr int sr_hdr_bars(int nw) { return nw * 4 * D + (2 * D + 15) / 16 * 16; }
template <int D>
__host__ __device__ constexpr int sr_hdr_bytes(int nw) {
  return sr_hdr_bars<D>(nw) + 24 * nw + 16 + (D / 2 + 1) * 8;   // ... then the omega_D table
}
// Offset of the block's copy of omega_D^k, k <= D/2, in the header: the
// two-lane unpacking (D = 256) picks its twiddles by the lane's parity, at
// run time, which shared memory serves in one load.
template <int D>
__host__ __device__ constexpr int sr_hdr_wd(int nw) { return sr_hdr_bars<D>(nw) + 24 * nw + 16; }

// The warp's per-channel table for one lambda table, D floats in channel
// order.  mode 0: lambda s (forward, lambda before); 1: fp32(lambda c_i), with
// the odd position of every bin above N/2 negated (forward, lambda after: the
// unpacking writes those bins as conj(E - T) through it); 2: s (1/lambda)
// (inverse, lambda before); 3: fp32(c_i / lambda) (inverse, lambda after).
// c_i = c0 at positions 0, 1, c1h elsewhere.
template <int D>
__device__ __forceinline__ void sr_build_table(float* tab, const ExArgs& a, int id, int mode, float c0,
                                               float c1h, int lane) {
  const float* lr = a.lam + static_cast<int64_t>(id) * D;
  for (int i = lane; i < D; i += 32) {
    const float l = lr[i];
    const float ci = i < 2 ? c0 : c1h;
    const bool neg = a.sgn[i] < 0;
    float v;
    if (mode == 0) {
      v = neg ? -l : l;
    } else if (mode == 1) {
      v = __fmul_rn(l, ci);
      if ((i & 1) && (i >> 1) > D / 4) v = -v;
    } else if (mode == 2) {
      v = __frcp_rn(l);
      if (neg) v = -v;
    } else {
      v = __fdiv_rn(ci, l);
    }
    tab[i] = v;
  }
}

// Sign-bit masks of the channel pairs: bit 15 (bit 31) set when the even (odd)
// channel's sign is negative, to flip fp16 values exactly.
template <int D>
__device__ __forceinline__ void sr_build_masks(uint32_t* mk, const ExArgs& a, int tid, int nthreads) {
  for (int n = tid; n < D / 2; n += nthreads)
    mk[n] = (a.sgn[2 * n] < 0 ? 0x8000u : 0u) | (a.sgn[2 * n + 1] < 0 ? 0x80000000u : 0u);
}

// ---- the Hermitian unpacking, two lanes per vector (D = 256) ---------------
// Lane `sub` holds bins k = 2j + sub of the 128-point spectrum in z[j].  The
// pairs (k, 128 - k) are (j, 64 - j) on lane 0, which also holds X_0 / X_128
// (j = 0) and the lone bin 64 (j = 32), and (j, 63 - j) on lane 1.  Both
// lanes run one loop over j; where their steps differ, both values are formed
// and a select keeps the lane's own, so every product is still the one the
// oracle forms.  ft: the factor table in channel order (fwd: the forward one,
// with the odd positions of bins above 64 negated), or null for the constant
// normalisation (c0 on positions 0, 1, c1h elsewhere).
__device__ __forceinline__ float2 sr256_fac(const float* ft, int k, float c0, float c1h, bool fwd) {
  if (ft != nullptr) return reinterpret_cast<const float2*>(ft)[k];
  if (k == 0) return make_float2(c0, c0);
  return make_float2(c1h, (fwd && k > 64) ? -c1h : c1h);
}

__device__ __forceinline__ void unpack_fwd256(float2 (&z)[64], const float2* wd, const float* ft,
                                              float c0, float c1h, int sub) {
  const bool odd = sub != 0;
  // j = 0: lane 0 forms y0 = X_0, y1 = X_128; lane 1 the pair (1, 127)
  {
    const float2 z0 = z[0];
    const float2 dc = __fmul2_rn(make_float2(__fadd_rn(z0.x, z0.y), __fsub_rn(z0.x, z0.y)),
                                 sr256_fac(ft, 0, c0, c1h, true));
    const float2 A = z[0], Bz = z[63];
    const float2 E = __ffma2_rn(Bz, make_float2(1.0f, -1.0f), A);
    const float2 Dd = __ffma2_rn(Bz, make_float2(-1.0f, 1.0f), A);
    const float2 T = twmul_odiv_rt(Dd, wd[1]);
    const float2 xk = __fmul2_rn(__fadd2_rn(E, T), sr256_fac(ft, 1, c0, c1h, true));
    const float2 xm = __fmul2_rn(fsub2(E, T), sr256_fac(ft, 127, c0, c1h, true));
    z[0] = odd ? xk : dc;
    z[63] = odd ? xm : z[63];
  }
#pragma unroll
  for (int j = 1; j < 32; ++j) {
    const int k = 2 * j + sub;
    const float2 A = z[j];
    const float2 Bz = odd ? z[63 - j] : z[64 - j];
    const float2 w = odd ? wd[2 * j + 1] : wd[2 * j];
    const float2 E = __ffma2_rn(Bz, make_float2(1.0f, -1.0f), A);
    const float2 Dd = __ffma2_rn(Bz, make_float2(-1.0f, 1.0f), A);
    const float2 T = twmul_odiv_rt(Dd, w);
    z[j] = __fmul2_rn(__fadd2_rn(E, T), sr256_fac(ft, k, c0, c1h, true));
    const float2 xm = __fmul2_rn(fsub2(E, T), sr256_fac(ft, 128 - k, c0, c1h, true));
    z[63 - j] = odd ? xm : z[63 - j];
    z[64 - j] = odd ? z[64 - j] : xm;
  }
  // j = 32: lane 0's lone bin 64 (omega_256^64 = -i, exact); lane 1 already
  // wrote z[32] as the partner of j = 31
  {
    const float2 A = z[32];
    const float2 E = __ffma2_rn(A, make_float2(1.0f, -1.0f), A);
    const float2 Dd = __ffma2_rn(A, make_float2(-1.0f, 1.0f), A);
    const float2 T = twmul_odiv<64, 256>(Dd, wd);
    const float2 x = __fmul2_rn(__fadd2_rn(E, T), sr256_fac(ft, 64, c0, c1h, true));
    z[32] = odd ? z[32] : x;
  }
}

__device__ __forceinline__ void unpack_inv256(float2 (&z)[64], const float2* wd, const float* ft,
                                              float c0, float c1h, int sub) {
  const bool odd = sub != 0;
  {
    const float2 u0 = __fmul2_rn(z[0], sr256_fac(ft, 0, c0, c1h, false));
    const float2 dc = make_float2(__fadd_rn(u0.x, u0.y), __fsub_rn(u0.x, u0.y));
    const float2 A = __fmul2_rn(z[0], sr256_fac(ft, 1, c0, c1h, false));
    const float2 Bu = __fmul2_rn(z[63], sr256_fac(ft, 127, c0, c1h, false));
    const float2 E = __ffma2_rn(Bu, make_float2(1.0f, -1.0f), A);
    const float2 Dd = __ffma2_rn(Bu, make_float2(-1.0f, 1.0f), A);
    const float2 T = twmul_conj_rt(Dd, wd[1]);
    const float2 zk = make_float2(__fsub_rn(E.x, T.y), __fadd_rn(E.y, T.x));
    const float2 zm = make_float2(__fadd_rn(E.x, T.y), -__fsub_rn(E.y, T.x));
    z[0] = odd ? zk : dc;
    z[63] = odd ? zm : z[63];
  }
#pragma unroll
  for (int j = 1; j < 32; ++j) {
    const int k = 2 * j + sub;
    const float2 A = __fmul2_rn(z[j], sr256_fac(ft, k, c0, c1h, false));
    const float2 Braw = odd ? z[63 - j] : z[64 - j];
    const float2 Bu = __fmul2_rn(Braw, sr256_fac(ft, 128 - k, c0, c1h, false));
    const float2 w = odd ? wd[2 * j + 1] : wd[2 * j];
    const float2 E = __ffma2_rn(Bu, make_float2(1.0f, -1.0f), A);
    const float2 Dd = __ffma2_rn(Bu, make_float2(-1.0f, 1.0f), A);
    const float2 T = twmul_conj_rt(Dd, w);
    z[j] = make_float2(__fsub_rn(E.x, T.y), __fadd_rn(E.y, T.x));
    const float2 zm = make_float2(__fadd_rn(E.x, T.y), -__fsub_rn(E.y, T.x));
    z[63 - j] = odd ? zm : z[63 - j];
    z[64 - j] = odd ? z[64 - j] : zm;
  }
  {
    const float2 A = __fmul2_rn(z[32], sr256_fac(ft, 64, c0, c1h, false));
    const float2 E = __ffma2_rn(A, make_float2(1.0f, -1.0f), A);
    const float2 Dd = __ffma2_rn(A, make_float2(-1.0f, 1.0f), A);
    const float2 T = twmul<64, 256, true>(Dd, wd);                  // conj(-i) = i, exact
    const float2 x = make_float2(__fsub_rn(E.x, T.y), __fadd_rn(E.y, T.x));
    z[32] = odd ? z[32] : x;
  }
}

// ---- quantize ------------------------------------------------------------
template <int D, int G, int BITS, bool AFTER>
__global__ void __launch_bounds__(sr_warps<D, false>() * 32, 1)
kvq_quantize_srft_kernel(const __grid_constant__ SrMaps maps, const ExArgs a,
                         const __grid_constant__ SrTw<D> tw, float c0, float c1h,
                         const __grid_constant__ CUtensorMap cmap, uint16_t* __restrict__ scales) {
  using S = Sr<D>;
  using F = SrFmt<D, BITS>;
  constexpr int kDW = sr_warps<D, false>();
  constexpr int NG = D / G;             // groups per row
  constexpr int GL = G / 2 / S::LANES;  // pairs of a group a lane holds
  constexpr int NLW = F::CB / 4 / S::LANES;   // code words a lane forms
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = S::LANES == 1 ? 0 : lane / S::WR, rin = S::LANES == 1 ? lane : lane % S::WR;
  uint8_t* wsm = smem + warp * 2 * S::TILE;
  uint8_t* hdr = smem + kDW * 2 * S::TILE;
  float* tab = reinterpret_cast<float*>(hdr) + warp * D;
  const uint32_t* mk = reinterpret_cast<const uint32_t*>(hdr + kDW * 4 * D);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + sr_hdr_bars<D>(kDW)) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + sr_hdr_bars<D>(kDW) + 16 * kDW) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + sr_hdr_bars<D>(kDW) + 24 * kDW);
  float2* wds = reinterpret_cast<float2*>(hdr + sr_hdr_wd<D>(kDW));
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  sr_build_masks<D>(const_cast<uint32_t*>(mk), a, tid, blockDim.x);
  for (int i = tid; i <= D / 2; i += blockDim.x) wds[i] = tw.wd[i];
  __syncthreads();

  const int64_t ntiles = (a.n + S::WR - 1) / S::WR;
  // a contiguous range of tiles per block, so a warp's tiles stay in one
  // lambda table for long stretches
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
    mbar_expect_tx(&bar[stage], S::TILE);
#pragma unroll
    for (int q = 0; q < S::NMAP; ++q)
      tensor_g2s(wsm + stage * S::TILE + q * (S::WR * 128), &maps.q[q], 0, t * S::WR, &bar[stage]);
  };
  refill(0);
  refill(1);
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
    const int id = table_id(a, tile * S::WR);
    if (id != cached) {
      __syncwarp();
      sr_build_table<D>(tab, a, id, AFTER ? 1 : 0, c0, c1h, lane);
      cached = id;
      __syncwarp();
    }
    const int64_t row = tile * S::WR + rin;
    const bool active = row < a.n;
    const uint8_t* st = wsm + stage * S::TILE;
    const float4* tab4 = reinterpret_cast<const float4*>(tab);
    float2 z[S::NL];
    if constexpr (S::LANES == 1) {
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {           // chunk c: channels 8c .. 8c+7 = pairs 4c .. 4c+3
        const uint4 xv = *reinterpret_cast<const uint4*>(st + sr_off<D>(rin, c));
        uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        if constexpr (AFTER) {
          const uint4 m4 = reinterpret_cast<const uint4*>(mk)[c];
          xw[0] ^= m4.x; xw[1] ^= m4.y; xw[2] ^= m4.z; xw[3] ^= m4.w;
#pragma unroll
          for (int j = 0; j < 4; ++j) z[4 * c + j] = half2_bits_to_float2(xw[j]);
        } else {
          const float4 l0 = tab4[2 * c], l1 = tab4[2 * c + 1];    // lambda s
          z[4 * c] = __fmul2_rn(half2_bits_to_float2(xw[0]), make_float2(l0.x, l0.y));
          z[4 * c + 1] = __fmul2_rn(half2_bits_to_float2(xw[1]), make_float2(l0.z, l0.w));
          z[4 * c + 2] = __fmul2_rn(half2_bits_to_float2(xw[2]), make_float2(l1.x, l1.y));
          z[4 * c + 3] = __fmul2_rn(half2_bits_to_float2(xw[3]), make_float2(l1.z, l1.w));
        }
      }
      fft_fwd_from<S::N, S::N, S::N>(z, tw.wn);
      const float2* ft = reinterpret_cast<const float2*>(tab);
      unpack_fwd1<D>(z, tw.wd, [&](int n) -> float2 {
        if constexpr (AFTER) return ft[n];
        else return n == 0 ? make_float2(c0, c0) : make_float2(c1h, n > D / 4 ? -c1h : c1h);
      });
    } else {
      // the first stage from the whole row: lane sub keeps output parity sub,
      // y[2p] = a + b (sub 0), y[2p+1] = (a - b) omega_128^p (sub 1)
      const float sg = sub ? -1.0f : 1.0f;
      sfor<0, 16>([&](auto Cc) {
        constexpr int c = decltype(Cc)::value;
        const uint4 av = *reinterpret_cast<const uint4*>(st + sr_off<D>(rin, c));
        const uint4 bv = *reinterpret_cast<const uint4*>(st + sr_off<D>(rin, c + 16));
        uint32_t aw[4] = {av.x, av.y, av.z, av.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
        float2 fa[4], fb[4];
        if constexpr (AFTER) {
          const uint4 ma = reinterpret_cast<const uint4*>(mk)[c], mb = reinterpret_cast<const uint4*>(mk)[c + 16];
          aw[0] ^= ma.x; aw[1] ^= ma.y; aw[2] ^= ma.z; aw[3] ^= ma.w;
          bw[0] ^= mb.x; bw[1] ^= mb.y; bw[2] ^= mb.z; bw[3] ^= mb.w;
#pragma unroll
          for (int j = 0; j < 4; ++j) { fa[j] = half2_bits_to_float2(aw[j]); fb[j] = half2_bits_to_float2(bw[j]); }
        } else {
          const float4 la0 = tab4[2 * c], la1 = tab4[2 * c + 1], lb0 = tab4[2 * c + 32], lb1 = tab4[2 * c + 33];
          fa[0] = __fmul2_rn(half2_bits_to_float2(aw[0]), make_float2(la0.x, la0.y));
          fa[1] = __fmul2_rn(half2_bits_to_float2(aw[1]), make_float2(la0.z, la0.w));
          fa[2] = __fmul2_rn(half2_bits_to_float2(aw[2]), make_float2(la1.x, la1.y));
          fa[3] = __fmul2_rn(half2_bits_to_float2(aw[3]), make_float2(la1.z, la1.w));
          fb[0] = __fmul2_rn(half2_bits_to_float2(bw[0]), make_float2(lb0.x, lb0.y));
          fb[1] = __fmul2_rn(half2_bits_to_float2(bw[1]), make_float2(lb0.z, lb0.w));
          fb[2] = __fmul2_rn(half2_bits_to_float2(bw[2]), make_float2(lb1.x, lb1.y));
          fb[3] = __fmul2_rn(half2_bits_to_float2(bw[3]), make_float2(lb1.z, lb1.w));
        }
        sfor<0, 4>([&](auto Jc) {
          constexpr int j = decltype(Jc)::value;
          const float2 t = __ffma2_rn(fb[j], make_float2(sg, sg), fa[j]);     // a + b or a - b
          // lane 0's product is discarded: it only keeps lane-uniform code
          // (quantisation does not see the sign of a zero)
          const float2 m = twmul<4 * c + j, 128, false>(t, tw.wn);
          z[4 * c + j] = sub ? m : t;
        });
      });
      fft_fwd_from<64, 64, 128>(z, tw.wn);
      unpack_fwd256(z, wds, AFTER ? tab : nullptr, c0, c1h, sub);
    }
    // group abs-max (across the two lanes at D = 256), S = fp16(a / QMAX), r = 1/S
    float r[NG];
    uint16_t b[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float am = 0.0f;
#pragma unroll
      for (int m = 0; m < GL; ++m) am = amax3(am, z[g * GL + m].x, z[g * GL + m].y);
      if constexpr (S::LANES == 2) am = fmaxf(am, __shfl_xor_sync(kFullMask, am, 16));
      b[g] = group_scale_q<F::QMAX>(am, r[g]);
    }
    uint32_t out[NLW];
    if constexpr (BITS == 4) {
#pragma unroll
      for (int w8 = 0; w8 < NLW; ++w8) {
        int qv[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int m = 4 * w8 + t;
          const float2 v = __fmul2_rn(z[m], make_float2(r[m / GL], r[m / GL]));
          qv[2 * t] = __float2int_rn(v.x);
          qv[2 * t + 1] = __float2int_rn(v.y);
        }
        out[w8] = pack8(qv);
      }
    } else {
#pragma unroll
      for (int w4 = 0; w4 < NLW; ++w4) {
        const float2 v0 = __fmul2_rn(z[2 * w4], make_float2(r[(2 * w4) / GL], r[(2 * w4) / GL]));
        const float2 v1 = __fmul2_rn(z[2 * w4 + 1], make_float2(r[(2 * w4 + 1) / GL], r[(2 * w4 + 1) / GL]));
        out[w4] = pack4_s8(__float2int_rn(v0.x), __float2int_rn(v0.y), __float2int_rn(v1.x), __float2int_rn(v1.y));
      }
    }
    // the codes leave through the stage this tile came from (every lane has
    // read it) by one tensor store that skips rows past n
    __syncwarp();
    uint8_t* cst = wsm + stage * S::TILE;
    if constexpr (S::LANES == 1) {
#pragma unroll
      for (int k4 = 0; k4 < F::CB / 16; ++k4)
        *reinterpret_cast<uint4*>(cst + sr_code_off<F::CB, F::SWZ>(rin, k4)) =
            make_uint4(out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3]);
    } else {
      // lane 0 holds the row's even code bytes (int4) or halfwords (int8),
      // lane 1 the odd ones: lane sub assembles words [sub NLW, (sub+1) NLW)
      constexpr int HW = NLW / 2;
      uint32_t full[NLW];
#pragma unroll
      for (int i = 0; i < HW; ++i) {
        const uint32_t send = sub ? out[i] : out[HW + i];
        const uint32_t recv = __shfl_xor_sync(kFullMask, send, 16);
        const uint32_t lo = sub ? recv : out[i];            // lane 0's word of this part
        const uint32_t hi = sub ? out[HW + i] : recv;       // lane 1's
        if constexpr (BITS == 4) {
          full[2 * i] = __byte_perm(lo, hi, 0x5140);
          full[2 * i + 1] = __byte_perm(lo, hi, 0x7362);
        } else {
          full[2 * i] = __byte_perm(lo, hi, 0x5410);
          full[2 * i + 1] = __byte_perm(lo, hi, 0x7632);
        }
      }
#pragma unroll
      for (int k4 = 0; k4 < NLW / 4; ++k4)
        *reinterpret_cast<uint4*>(cst + sr_code_off<F::CB, F::SWZ>(rin, sub * (NLW / 4) + k4)) =
            make_uint4(full[4 * k4], full[4 * k4 + 1], full[4 * k4 + 2], full[4 * k4 + 3]);
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      tensor_s2g(&cmap, 0, static_cast<int>(tile * S::WR), cst);
      bulk_commit();
    }
    if (active) {
      uint16_t* srow = scales + row * NG;
      constexpr int PER = NG / S::LANES;
#pragma unroll
      for (int g = 0; g < NG; ++g)
        if (g / PER == sub) srow[g] = b[g];
    }
  }
  if (lane == 0) bulk_wait0();
}


// ---- dequantize ------------------------------------------------------------
// A warp's shared memory: the fp16 staging tile its tensor stores read, the
// two stages' code tiles (rows as the bulk copies leave them, CB bytes
// apart), then the two stages' scales.
template <int D, int G, int BITS>
struct SrDeq {
  using S = Sr<D>;
  static constexpr int CB = SrFmt<D, BITS>::CB;
  static constexpr int WC = S::WR * CB;                  // codes of one warp tile
  static constexpr int WCA = (WC + 127) / 128 * 128;
  static constexpr int SPR = (D / G) * 2;                // scale bytes per row
  static constexpr int WS = S::WR * SPR;                 // scales of one warp tile
  static_assert(WS % 16 == 0, "scale blocks stay 16-byte aligned");
  static constexpr int SC = S::TILE + 2 * WCA;           // offset of the scales
  static constexpr int WARP = (SC + 2 * WS + 1023) / 1024 * 1024;
};

// Codes of one lane's pairs as exact fp16 integers times the group scale:
// z[j] = (q_2j S, q_2j+1 S) for the lane's 4-word (int4) or 2-word (int8)
// unit; w is the lane's word of codes (int4: pairs 4u .. 4u+3, one byte each;
// int8: pairs 2u, 2u+1, one halfword each).
template <int BITS>
__device__ __forceinline__ void sr_decode_word(uint32_t w, float2* z, const uint16_t* sv, int g0, int gl) {
  if constexpr (BITS == 4) {
    const __half2 bias = __floats2half2_rn(1032.0f, 1032.0f);
    const uint32_t wb = w ^ 0x88888888u, w4 = wb >> 4;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t sel = 0x0400u | (t << 8) | t;
      const uint32_t e = (__byte_perm(wb, w4, sel) & 0x000F000Fu) | 0x64006400u;
      const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&e), bias);
      const uint16_t s = sv[(g0 + t) / gl];
      z[t] = make_float2(mul_f16_f32(__low2half(h), s), mul_f16_f32(__high2half(h), s));
    }
  } else {
    const __half2 bias = __floats2half2_rn(1152.0f, 1152.0f);
    const uint32_t wb = w ^ 0x80808080u;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t sel = static_cast<uint32_t>(2 * t) | ((2u * t + 1) << 8);
      const uint32_t e = (__byte_perm(wb, 0u, sel) & 0x00FF00FFu) | 0x64006400u;
      const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&e), bias);
      const uint16_t s = sv[(g0 + t) / gl];
      z[t] = make_float2(mul_f16_f32(__low2half(h), s), mul_f16_f32(__high2half(h), s));
    }
  }
}

template <int D, int G, int BITS, bool AFTER>
__global__ void __launch_bounds__(sr_warps<D, true>() * 32, 1)
kvq_dequantize_srft_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                           const ExArgs a, const __grid_constant__ SrTw<D> tw, float c0, float c1h,
                           const __grid_constant__ SrMaps omaps, int scale_copy,
                           const __grid_constant__ CUtensorMap cmap) {
  using S = Sr<D>;
  using L = SrDeq<D, G, BITS>;
  using F = SrFmt<D, BITS>;
  constexpr int kDW = sr_warps<D, true>();
  constexpr int NG = D / G;
  constexpr int GL = G / 2 / S::LANES;  // pairs of a group a lane holds
  constexpr int CB = L::CB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = S::LANES == 1 ? 0 : lane / S::WR, rin = S::LANES == 1 ? lane : lane % S::WR;
  uint8_t* stage_out = smem + warp * L::WARP;
  uint8_t* hdr = smem + kDW * L::WARP;
  float* tab = reinterpret_cast<float*>(hdr) + warp * D;
  const uint32_t* mk = reinterpret_cast<const uint32_t*>(hdr + kDW * 4 * D);
  uint64_t* bar = reinterpret_cast<uint64_t*>(hdr + sr_hdr_bars<D>(kDW)) + 2 * warp;
  int* tq = reinterpret_cast<int*>(hdr + sr_hdr_bars<D>(kDW) + 16 * kDW) + 2 * warp;
  unsigned int* next = reinterpret_cast<unsigned int*>(hdr + sr_hdr_bars<D>(kDW) + 24 * kDW);
  float2* wds = reinterpret_cast<float2*>(hdr + sr_hdr_wd<D>(kDW));
  if (lane == 0) { mbar_init(&bar[0], 1); mbar_init(&bar[1], 1); mbar_fence_init(); }
  if (tid == 0) *next = 0;
  sr_build_masks<D>(const_cast<uint32_t*>(mk), a, tid, blockDim.x);
  for (int i = tid; i <= D / 2; i += blockDim.x) wds[i] = tw.wd[i];
  __syncthreads();

  const int64_t ntiles = (a.n + S::WR - 1) / S::WR;
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
    const int64_t row0 = t * S::WR;
    const int valid = static_cast<int>(a.n - row0 < S::WR ? a.n - row0 : S::WR);
    return static_cast<uint32_t>(valid * L::SPR) & ~15u;
  };
  auto refill = [&](int stage) {
    const int t = claim();
    if (lane == 0) tq[stage] = t;
    if (t < 0 || lane != 0) return;
    const int64_t row0 = static_cast<int64_t>(t) * S::WR;
    const uint32_t sb = scale_bytes(t);
    if constexpr (F::SWZ != 0) {
      // 64- or 128-byte code rows: one tensor copy of the whole tile, swizzled
      // over the row so that the lanes' 16-byte reads of consecutive rows
      // fall in distinct banks (rows past n read as zeros)
      mbar_expect_tx(&bar[stage], static_cast<uint32_t>(S::WR * CB) + sb);
      tensor_g2s(stage_out + S::TILE + stage * L::WCA, &cmap, 0, static_cast<int>(row0), &bar[stage]);
    } else {
      const uint32_t cbytes = static_cast<uint32_t>(a.n - row0 < S::WR ? a.n - row0 : S::WR) * CB;
      mbar_expect_tx(&bar[stage], cbytes + sb);
      bulk_g2s(stage_out + S::TILE + stage * L::WCA, codes + row0 * CB, cbytes, &bar[stage]);
    }
    if (sb) bulk_g2s(stage_out + L::SC + stage * L::WS, reinterpret_cast<const uint8_t*>(scales) + row0 * L::SPR, sb, &bar[stage]);
  };
  refill(0);
  refill(1);
  int cached = -1;
  for (uint32_t k = 0;; ++k) {
    const int stage = k & 1;
    __syncwarp();
    const int64_t tile = tq[stage];
    if (tile < 0) break;
    const int64_t row = tile * S::WR + rin;
    const int64_t rrow = row < a.n ? row : a.n - 1;
    const bool sc_smem = static_cast<uint32_t>((rin + 1) * L::SPR) <= scale_bytes(tile);
    const bool ok = mbar_wait(&bar[stage], (k >> 1) & 1, kSpinX);
    if (__any_sync(kFullMask, !ok)) {
      if (lane == 0) atomicOr(&g_ex_fault, 1u);
      mbar_wait(&bar[stage], (k >> 1) & 1, kSpinX);   // the stage that gave up, once more
      if (tq[stage ^ 1] >= 0) mbar_wait(&bar[stage ^ 1], ((k + 1) >> 1) & 1, kSpinX);
      if (lane == 0) bulk_wait0();
      return;
    }
    const int id = table_id(a, tile * S::WR);
    if (id != cached) {
      __syncwarp();
      sr_build_table<D>(tab, a, id, AFTER ? 3 : 2, c0, c1h, lane);
      cached = id;
      __syncwarp();
    }
    const uint8_t* cst = stage_out + S::TILE + stage * L::WCA;   // the tile's codes (row rin)
    const uint16_t* srow = sc_smem ? reinterpret_cast<const uint16_t*>(stage_out + L::SC + stage * L::WS + rin * L::SPR)
                                   : scales + rrow * NG;
    uint16_t sv[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) sv[g] = srow[g];
    float2 z[S::NL];
    if constexpr (S::LANES == 1) {
      constexpr int PW = BITS == 4 ? 4 : 2;            // pairs per code word
#pragma unroll
      for (int c = 0; c < CB / 16; ++c) {
        const uint4 cv = *reinterpret_cast<const uint4*>(cst + sr_code_off<CB, F::SWZ>(rin, c));
        const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) sr_decode_word<BITS>(cw[t], &z[(4 * c + t) * PW], sv, (4 * c + t) * PW, GL);
      }
    } else {
      // lane sub keeps the row's code bytes (int4) or halfwords (int8) of parity sub
      constexpr int PW = BITS == 4 ? 4 : 2;
      const uint32_t sel = BITS == 4 ? (sub ? 0x7531u : 0x6420u) : (sub ? 0x7632u : 0x5410u);
#pragma unroll
      for (int c = 0; c < CB / 16; ++c) {
        const uint4 cv = *reinterpret_cast<const uint4*>(cst + sr_code_off<CB, F::SWZ>(rin, c));
        const uint32_t w0 = __byte_perm(cv.x, cv.y, sel), w1 = __byte_perm(cv.z, cv.w, sel);
        sr_decode_word<BITS>(w0, &z[(2 * c) * PW], sv, (2 * c) * PW, GL);
        sr_decode_word<BITS>(w1, &z[(2 * c + 1) * PW], sv, (2 * c + 1) * PW, GL);
      }
    }
    __syncwarp();                       // codes and scales consumed: refill the stage
    refill(stage);

    const float2* ft = reinterpret_cast<const float2*>(tab);
    if constexpr (S::LANES == 1) {
      unpack_inv1<D>(z, tw.wd, [&](int n) -> float2 {
        if constexpr (AFTER) return ft[n];
        else return n == 0 ? make_float2(c0, c0) : make_float2(c1h, c1h);
      });
      fft_inv_from<S::N, S::N, S::N>(z, tw.wn);
      if (lane == 0) bulk_wait_read0();   // the previous tile's stores have read the staging tile
      __syncwarp();
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint32_t hv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int n = 4 * c + j;
          if constexpr (AFTER) {
            hv[j] = float2_to_half2_bits(z[n].x, z[n].y) ^ mk[n];          // the signs, exact
          } else {
            const float2 v = __fmul2_rn(z[n], ft[n]);                     // s (1/lambda)
            hv[j] = float2_to_half2_bits(v.x, v.y);
          }
        }
        *reinterpret_cast<uint4*>(stage_out + sr_off<D>(rin, c)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
    } else {
      unpack_inv256(z, wds, AFTER ? tab : nullptr, c0, c1h, sub);
      fft_inv_from<64, 64, 128>(z, tw.wn);
      // the transpose of the first stage: c_p = Y_2p+1 conj(omega_128^p) (lane
      // 1's bins), z_p = Y_2p + c_p, z_(p+64) = Y_2p - c_p; lane 0 forms
      // p < 32, lane 1 p >= 32, half of each lane's values crossing by shuffle
      sfor<0, 64>([&](auto Pc) {
        constexpr int p = decltype(Pc)::value;
        const float2 m = twmul<p, 128, true>(z[p], tw.wn);
        z[p] = sub ? m : z[p];
      });
      if (lane == 0) bulk_wait_read0();   // the previous tile's stores have read the staging tile
      __syncwarp();
      // z_p (pairs 32 sub + i: quarter sub of the row) and z_(p+64) (quarter
      // 2 + sub), four pairs (one 16-byte chunk of each quarter) at a time
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t ha[4], hb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 4 * cc + j;
          const float2 send = sub ? z[i] : z[32 + i];
          float2 recv;
          recv.x = __shfl_xor_sync(kFullMask, send.x, 16);
          recv.y = __shfl_xor_sync(kFullMask, send.y, 16);
          const float2 P = sub ? recv : z[i];          // Y_2p
          const float2 Q = sub ? z[32 + i] : recv;     // c_p
          const float2 oa = __fadd2_rn(P, Q), ob = fsub2(P, Q);
          const int na = 32 * sub + i, nb = 64 + 32 * sub + i;
          if constexpr (AFTER) {
            ha[j] = float2_to_half2_bits(oa.x, oa.y) ^ mk[na];
            hb[j] = float2_to_half2_bits(ob.x, ob.y) ^ mk[nb];
          } else {
            const float2 va = __fmul2_rn(oa, ft[na]), vb = __fmul2_rn(ob, ft[nb]);
            ha[j] = float2_to_half2_bits(va.x, va.y);
            hb[j] = float2_to_half2_bits(vb.x, vb.y);
          }
        }
        *reinterpret_cast<uint4*>(stage_out + sr_off<D>(rin, 8 * sub + cc)) = make_uint4(ha[0], ha[1], ha[2], ha[3]);
        *reinterpret_cast<uint4*>(stage_out + sr_off<D>(rin, 8 * (2 + sub) + cc)) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
      }
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < S::NMAP; ++q)
        tensor_s2g(&omaps.q[q], 0, static_cast<int>(tile * S::WR), stage_out + q * (S::WR * 128));
      bulk_commit();
    }
  }
  if (lane == 0) bulk_wait0();
}


// ---------------------------------------------------------------------------
// Launch plumbing.
// ---------------------------------------------------------------------------

template <int D>
const SrTw<D>& sr_twiddles() {
  static const SrTw<D> tw = [] {
    SrTw<D> t{};
    for (int k = 0; k < D / 2; ++k) t.wn[k] = root_f32(k, D / 2);
    for (int k = 0; k <= D / 2; ++k) t.wd[k] = root_f32(k, D);
    return t;
  }();
  return tw;
}

thread_local int g_srft_cuda_error = 0;

int sr_fail(int code) {
  g_srft_cuda_error = code;
  return KVQ_ERR_LAUNCH;
}

// fp16 rows [n][D]: one map per 64-channel box (128-byte swizzle) and, at
// D = 96, one for the last 32 channels (64-byte swizzle); a box is one warp
// tile of rows.
template <int D>
int sr_encode_x_maps(SrMaps& maps, const uint16_t* x, int64_t n) {
  using S = Sr<D>;
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  memset(&maps, 0, sizeof(maps));
  for (int q = 0; q < S::NMAP; ++q) {
    const bool tail = q == S::NB;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(tail ? 32 : 64), static_cast<cuuint64_t>(n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(2 * D)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(tail ? 32 : 64), static_cast<cuuint32_t>(S::WR)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&maps.q[q], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                           const_cast<char*>(reinterpret_cast<const char*>(x)) + 128 * q, dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           tail ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return sr_fail(static_cast<int>(r));
  }
  return KVQ_OK;
}

// The codes [n][CB] as one map with a box of one warp tile, in the layout
// sr_code_off writes (swizzled over 64- or 128-byte rows, plain otherwise).
template <int D, int BITS>
int sr_encode_code_map(CUtensorMap& map, const uint8_t* codes, int64_t n) {
  using F = SrFmt<D, BITS>;
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(F::CB), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(F::CB)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(F::CB), static_cast<cuuint32_t>(Sr<D>::WR)};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = F::SWZ == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : F::SWZ == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return sr_fail(static_cast<int>(r));
  return KVQ_OK;
}

int sr_sms(int& dev) {
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

// Grid: one block per resident slot, at most one per warp tile.
template <typename Kernel>
int sr_grid(Kernel k, int64_t tiles, int smem, int threads, std::atomic<int>* ready) {
  int dev = 0;
  const int sms = sr_sms(dev);
  int occ = ready[dev].load(std::memory_order_relaxed);
  if (occ == 0) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, threads, smem) != cudaSuccess || occ < 1) occ = 1;
    ready[dev].store(occ, std::memory_order_relaxed);
  }
  const int64_t cap = static_cast<int64_t>(sms) * occ;
  return static_cast<int>(tiles < cap ? tiles : cap);
}

int sr_finish() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KVQ_OK : sr_fail(static_cast<int>(e));
}

float sr_c0(int D) { return static_cast<float>(1.0 / std::sqrt(static_cast<double>(D))); }
float sr_c1h(int D) { return static_cast<float>(1.0 / std::sqrt(2.0 * static_cast<double>(D))); }

template <int D, int G, int BITS, bool AFTER>
int launch_sq(const uint16_t* x, const ExArgs& a, uint8_t* codes, uint16_t* scales, cudaStream_t st) {
  using S = Sr<D>;
  SrMaps maps;
  int rc = sr_encode_x_maps<D>(maps, x, a.n);
  if (rc != KVQ_OK) return rc;
  CUtensorMap cmap;
  rc = sr_encode_code_map<D, BITS>(cmap, codes, a.n);
  if (rc != KVQ_OK) return rc;
  auto k = kvq_quantize_srft_kernel<D, G, BITS, AFTER>;
  constexpr int nw = sr_warps<D, false>();
  constexpr int smem = 1024 + nw * 2 * S::TILE + sr_hdr_bytes<D>(nw);
  static_assert(smem <= 227 * 1024, "shared memory");
  static std::atomic<int> ready[64];
  const int grid = sr_grid(k, (a.n + S::WR - 1) / S::WR, smem, nw * 32, ready);
  (void)cudaGetLastError();
  k<<<grid, nw * 32, smem, st>>>(maps, a, sr_twiddles<D>(), sr_c0(D), sr_c1h(D), cmap, scales);
  return sr_finish();
}

template <int D, int G, int BITS, bool AFTER>
int launch_sd(const uint8_t* codes, const uint16_t* scales, const ExArgs& a, uint16_t* out,
              cudaStream_t st) {
  using S = Sr<D>;
  using L = SrDeq<D, G, BITS>;
  SrMaps omaps;
  int rc = sr_encode_x_maps<D>(omaps, out, a.n);
  if (rc != KVQ_OK) return rc;
  CUtensorMap cmap;
  memset(&cmap, 0, sizeof(cmap));
  if (SrFmt<D, BITS>::SWZ != 0) {
    rc = sr_encode_code_map<D, BITS>(cmap, codes, a.n);
    if (rc != KVQ_OK) return rc;
  }
  auto k = kvq_dequantize_srft_kernel<D, G, BITS, AFTER>;
  constexpr int nw = sr_warps<D, true>();
  constexpr int smem = 1024 + nw * L::WARP + sr_hdr_bytes<D>(nw);
  static_assert(smem <= 227 * 1024, "shared memory");
  static std::atomic<int> ready[64];
  const int grid = sr_grid(k, (a.n + S::WR - 1) / S::WR, smem, nw * 32, ready);
  (void)cudaGetLastError();
  k<<<grid, nw * 32, smem, st>>>(codes, scales, a, sr_twiddles<D>(), sr_c0(D), sr_c1h(D), omaps,
                                  (reinterpret_cast<uintptr_t>(scales) & 15) == 0 ? 1 : 0, cmap);
  return sr_finish();
}

template <int D, template <int, int, int, bool> class Op, typename... Args>
int sr_dispatch_g(int group, int bits, bool after, Args... args) {
  switch (group * 100 + bits * 10 + (after ? 1 : 0)) {
    case 1640: return Op<D, 16, 4, false>::run(args...);
    case 1641: return Op<D, 16, 4, true>::run(args...);
    case 1680: return Op<D, 16, 8, false>::run(args...);
    case 1681: return Op<D, 16, 8, true>::run(args...);
    case 3240: return Op<D, 32, 4, false>::run(args...);
    case 3241: return Op<D, 32, 4, true>::run(args...);
    case 3280: return Op<D, 32, 8, false>::run(args...);
    case 3281: return Op<D, 32, 8, true>::run(args...);
    default: break;
  }
  if constexpr (D % 64 == 0) {
    switch (group * 100 + bits * 10 + (after ? 1 : 0)) {
      case 6440: return Op<D, 64, 4, false>::run(args...);
      case 6441: return Op<D, 64, 4, true>::run(args...);
      case 6480: return Op<D, 64, 8, false>::run(args...);
      case 6481: return Op<D, 64, 8, true>::run(args...);
      default: break;
    }
  }
  return KVQ_ERR_GROUP;
}

template <int D, int G, int BITS, bool AFTER>
struct QuantOp {
  static int run(const uint16_t* x, ExArgs a, uint8_t* codes, uint16_t* scales, cudaStream_t st) {
    return launch_sq<D, G, BITS, AFTER>(x, a, codes, scales, st);
  }
};
template <int D, int G, int BITS, bool AFTER>
struct DequantOp {
  static int run(const uint8_t* codes, const uint16_t* scales, ExArgs a, uint16_t* out, cudaStream_t st) {
    return launch_sd<D, G, BITS, AFTER>(codes, scales, a, out, st);
  }
};

}  // namespace

#define KVQ_SRFT_CAT2(a, b) a##b
#define KVQ_SRFT_CAT(a, b) KVQ_SRFT_CAT2(a, b)

// Entry points behind kvq_quantize_ex / kvq_dequantize_ex with flags bit
// KVQ_SRFT at D = KVQ_SRFT_D (kvq_ex.cu checks every argument first).
__attribute__((visibility("hidden"))) int KVQ_SRFT_CAT(kvq_srft_quantize_, KVQ_SRFT_D)(
    const uint16_t* x, const float* lambda, const int8_t* signs, int64_t n, int group, int bits,
    bool after, int64_t lambda_rows, int n_lambda, uint8_t* codes, uint16_t* scales, cudaStream_t st) {
  const ExArgs a{lambda, signs, n, lambda_rows, n_lambda, sr_c0(KVQ_SRFT_D)};
  return sr_dispatch_g<KVQ_SRFT_D, QuantOp>(group, bits, after, x, a, codes, scales, st);
}

__attribute__((visibility("hidden"))) int KVQ_SRFT_CAT(kvq_srft_dequantize_, KVQ_SRFT_D)(
    const uint8_t* codes, const uint16_t* scales, const float* lambda, const int8_t* signs, int64_t n,
    int group, int bits, bool after, int64_t lambda_rows, int n_lambda, uint16_t* out, cudaStream_t st) {
  const ExArgs a{lambda, signs, n, lambda_rows, n_lambda, sr_c0(KVQ_SRFT_D)};
  return sr_dispatch_g<KVQ_SRFT_D, DequantOp>(group, bits, after, codes, scales, a, out, st);
}

// Read (and optionally clear) this unit's fault word; used by kvq_fault_status.
__attribute__((visibility("hidden"))) unsigned int KVQ_SRFT_CAT(kvq_srft_fault_word_, KVQ_SRFT_D)(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ex_fault, sizeof(v)) != cudaSuccess) return 0;
  if (clear && v) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_ex_fault, &zero, sizeof(zero));
  }
  return v;
}
__attribute__((visibility("hidden"))) int KVQ_SRFT_CAT(kvq_srft_last_cuda_error_, KVQ_SRFT_D)() {
  return g_srft_cuda_error;
}
