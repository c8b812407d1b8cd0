// kvq_attn.cu -- fused decode attention over the int4 rotated-domain KV cache
// for B200 (sm_100a): kernels and the C-ABI launcher of kvq_attention_decode
// (include/kvq.h).
//
// Method: "The Kernel That Finally Did Something -- And Didn't Quite Agree
// With Itself" (VeloxQuant-MLX blog), "Fused group-affine (KIVI-style)
// attention": the quantised keys and values are reconstructed in registers
// inside a FlashAttention-style online softmax, so no dequantised K or V ever
// reaches memory, and the key axis is split flash-decoding style when there
// are few sequences.  The cache rows here are int4 codes of the rotated vector
// y = H diag(s) (lambda . x) / sqrt(D) with fp16 group scales ("When
// Quantization Is Free", technical summary, Methodologie 1-3), so the rotation
// moves to the query, once per head, instead of running once per key:
//     <q, x_t> = <q~, y_t>,   q~ = H diag(s_K) (q / lambda_K) / sqrt(D),
// and the values are summed in the rotated domain and rotated back once:
//     o = (diag(s_V) H (sum_t p_t y_t) / sqrt(D)) / lambda_V
// (H is symmetric with H H = D I, and s_i^2 = 1).
//
// Work decomposition.  A block of four warps owns one (sequence, KV head,
// key split); each warp streams 64-key blocks (codes and scales of K and V,
// four bulk copies into a private double-buffered ring) and keeps its own
// online-softmax state, updated once per block; the block merges the four
// states at the end.
// Both products run on the tensor cores as m16n8k16 fp16 MMAs with fp32
// accumulation, the query heads of the KV head on the M rows:
//   * scores: rows 0..R-1 hold the fp16 high parts of q~, rows 8..8+R-1 the
//     fp16 residuals (q~ = hi + lo to ~2^-22), the N columns are 8 keys and
//     the K dimension 16 channels.  The channel order inside each 32-channel
//     block is permuted so that a lane's B fragments for two k-steps are the
//     four nibble pairs of one 32-bit word of codes (nibbles k and k + 16 of
//     the word), and every k-step stays inside one scale group: the group's
//     scale multiplies the per-group partial sums, key by key, after the MMA.
//   * values: the score fragments are already in the A layout of the value
//     product (rows = heads, K dimension = 16 keys), so p * S_V (split hi/lo
//     the same way) feeds it directly, one A fragment per scale group; the B
//     fragments pair the same channel of two keys.
// A biased code n = q + 8 in [0, 15] is used as the fp16 subnormal n 2^-24,
// exact and made by one mask-and-xor: sum_k a_k q_k = 2^24 sum_k a_k n_k 2^-24
// - 8 sum_k a_k.  The key side starts its accumulators at -8 2^-24 sum a (a
// constant of the query); the value side keeps the running sum of p * S_V per
// group and subtracts it once at the end.
//
// Every mbarrier wait is bounded; a warp that gives up sets the fault word
// and the block still finishes (its output is then meaningless).  A sequence
// length outside [0, T] is clamped and flagged.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "kvq.h"

namespace {

constexpr unsigned kFullMask = 0xffffffffu;

#include "kvq_async.cuh"
#include "kvq_arith.cuh"
#include "kvq_fft.cuh"

constexpr int kAW = 4;                       // warps per block
constexpr int kBK = 64;                      // keys per streamed block
constexpr int kAStages = 2;                  // ring depth per warp
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kSpin = 1u << 22;         // bounded mbarrier waits
constexpr int kMaxRows = 8;                  // query heads per KV head (M rows of one MMA half)

__device__ unsigned int g_attn_fault = 0;    // bit 0: a wait gave up; bit 3: bad sequence length

// Scratch of kvq_attention_decode_static: the partial (max, sum, rotated
// output) rows of the key splits, 8 MiB per device.  Nothing in it has to
// start at zero: every split writes its own slots before the merge kernel,
// later on the same stream, reads them.  Calls that overlap in time (other
// streams, other host threads) share it and race.
constexpr int64_t kStaticScratchBytes = int64_t{8} << 20;
static __device__ __align__(256) unsigned char g_attn_static_scratch[kStaticScratchBytes];
thread_local int g_attn_cuda_error = 0;

struct AttnParams {
  const uint16_t* q;            // fp16 [B][Hq][D]
  const uint8_t* kp;            // [B][Hkv][T][D/2]
  const uint16_t* ks;           // fp16 [B][Hkv][T][D/G]
  const uint8_t* vp;
  const uint16_t* vs;
  const int32_t* seq_len;       // [B]
  const float* lam_k;
  const int8_t* s_k;
  const float* lam_v;
  const int8_t* s_v;
  uint16_t* out;                // fp16 [B][Hq][D]
  float* part;                  // [B*Hkv*nsplit][R][D + 4] when nsplit > 1
  int Hkv, T, R, nsplit, chunk;
  float scale_log2;             // sm_scale * log2(e) * 2^24 (the key product comes out scaled by 2^-24)
  float c;                      // fp32 1/sqrt(D)
  float c1h;                    // fp32 1/sqrt(2D): the SRFT's normalisation of 2 X_k
  float2 wn[64];                // SRFT twiddles omega_(D/2)^k, k < D/2 (SRFT caches only)
  float2 wd[65];                // omega_D^k, k <= D/2
};

// Cache formats (the codec variants' flags): bit 0 lambda after the rotation,
// bit 1 the SRFT rotation.
constexpr int kFmtAfter = 1, kFmtSrft = 2;

template <int D, int G>
struct Attn {
  static constexpr int NB = D / 32;                 // 32-channel blocks of a row
  static constexpr int KS = D / 16;                 // k-steps of the score product
  static constexpr int NT = D / 8;                  // n-tiles of the value product
  static constexpr int NG = D / G;                  // scale groups of a row
  static constexpr int W32 = D / 8;                 // 32-bit words of one code row
  static constexpr int CB = kBK * D / 2;            // code bytes of one block
  static constexpr int SB = kBK * NG * 2;           // scale bytes of one block
  static constexpr int STAGE = 2 * CB + 2 * SB;     // K codes, V codes, K scales, V scales
  static constexpr int QT = 2 * kMaxRows * D * 2;   // q~ hi and lo rows, fp16
  static constexpr int COMB = kAW * kMaxRows * D * 4;
  static constexpr int RING = kAW * kAStages * STAGE;
  static constexpr int AREA = RING > COMB ? RING : COMB;   // the merge reuses the ring
  static constexpr int SMEM = AREA + QT + kAW * kAStages * 8 + kAW * kMaxRows * 8;
  static constexpr int DPL = D / 32;                // channels per lane in the row transforms
};

// A biased code pair as fp16 subnormals: nibbles at bits 0-3 and 16-19 of x,
// n = q + 8 (xor 8 of the two's-complement nibble), value n 2^-24, exact.
__device__ __forceinline__ uint32_t sub_pair(uint32_t x) {
  return (x & 0x000F000Fu) ^ 0x00080008u;
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Unnormalised Walsh-Hadamard transform of one D-vector held by a warp, lane
// l holding channels DPL*l .. DPL*l + DPL-1 (ascending half-width h).
template <int D>
__device__ __forceinline__ void warp_fwht(float (&v)[D / 32], int lane) {
  constexpr int DPL = D / 32;
#pragma unroll
  for (int h = 1; h < DPL; h <<= 1) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int h = DPL; h < D; h <<= 1) {
    const int lb = h / DPL;
    const bool upper = (lane & lb) != 0;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const float o = __shfl_xor_sync(kFull, v[i], lb);
      v[i] = upper ? o - v[i] : v[i] + o;
    }
  }
}

// One head's output from its merged rotated-domain sum y = o / l, back in
// the cache's format:
//   lambda before: out = fp16((s_V . R^T y) / lambda_V),
//   lambda after:  out = fp16(s_V . R^T (y / lambda_V)),
// R^T = H / sqrt(D) (a warp-wide butterfly over the lanes' channels) or the
// SRFT transpose (the codec's adjoint unpacking and transposed FFT, run by one
// lane on the row gathered in `scr`, D floats of this warp's shared memory).
template <int D, int FMT>
__device__ __forceinline__ void finish_head(const AttnParams& P, float (&v)[D / 32], float l,
                                            uint16_t* out_row, int lane, float* scr) {
  constexpr int DPL = D / 32;
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) v[i] *= inv;
  if constexpr ((FMT & kFmtSrft) == 0) {
    if constexpr (FMT & kFmtAfter) {
#pragma unroll
      for (int i = 0; i < DPL; ++i) v[i] /= P.lam_v[DPL * lane + i];
    }
    warp_fwht<D>(v, lane);
    uint16_t h[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = DPL * lane + i;
      const float z = v[i] * P.c;
      const float zs = P.s_v[d] < 0 ? -z : z;
      h[i] = __half_as_ushort(__float2half_rn((FMT & kFmtAfter) ? zs : zs / P.lam_v[d]));
    }
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2*>(out_row + DPL * lane) =
          make_uint2(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16));
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) out_row[DPL * lane + i] = h[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < DPL; ++i) scr[DPL * lane + i] = v[i];
    __syncwarp();
    if (lane == 0) {
      float2 z[D / 2];
#pragma unroll
      for (int n = 0; n < D / 2; ++n) z[n] = make_float2(scr[2 * n], scr[2 * n + 1]);
      unpack_inv1<D>(z, P.wd, [&](int n) -> float2 {
        float2 f = n == 0 ? make_float2(P.c, P.c) : make_float2(P.c1h, P.c1h);
        if constexpr (FMT & kFmtAfter) f = make_float2(f.x / P.lam_v[2 * n], f.y / P.lam_v[2 * n + 1]);
        return f;
      });
      fft_inv_from<D / 2, D / 2, D / 2>(z, P.wn);
#pragma unroll
      for (int n = 0; n < D / 2; ++n) {
        float a = P.s_v[2 * n] < 0 ? -z[n].x : z[n].x;
        float b = P.s_v[2 * n + 1] < 0 ? -z[n].y : z[n].y;
        if constexpr ((FMT & kFmtAfter) == 0) {
          a = a / P.lam_v[2 * n];
          b = b / P.lam_v[2 * n + 1];
        }
        reinterpret_cast<uint32_t*>(out_row)[n] = float2_to_half2_bits(a, b);
      }
    }
    __syncwarp();
  }
}

template <int D, int G, int FMT>
__global__ void __launch_bounds__(kAW * 32, 2)
kvq_attn_kernel(const __grid_constant__ AttnParams P) {
  using A = Attn<D, G>;
  constexpr int NB = A::NB, KS = A::KS, NT = A::NT, NG = A::NG, W32 = A::W32, DPL = A::DPL;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* ring = sm;                                            // [warp][stage][STAGE]
  __half* qt = reinterpret_cast<__half*>(sm + A::AREA);           // [2][8][D]: hi rows, lo rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + A::AREA + A::QT);
  float* ml = reinterpret_cast<float*>(bars + kAW * kAStages);    // [warp][8][2]: m, l
  float* comb = reinterpret_cast<float*>(sm);                     // [warp][8][D], after the key loop

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int item = blockIdx.x;
  const int split = item % P.nsplit;
  const int bh = item / P.nsplit;                                 // b * Hkv + kv head
  const int b = bh / P.Hkv, kvh = bh % P.Hkv;
  const int R = P.R;
  int L = P.seq_len[b];
  if (L < 0 || L > P.T) {
    if (tid == 0) atomicOr(&g_attn_fault, 8u);
    L = L < 0 ? 0 : P.T;
  }
  const int k0 = split * P.chunk;
  const int k1 = min(L, k0 + P.chunk);
  const int nkeys = k1 > k0 ? k1 - k0 : 0;
  const int nblk = (nkeys + kBK - 1) / kBK;

  uint64_t* bar = bars + kAStages * warp;
  if (lane == 0) {
    for (int s = 0; s < kAStages; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  // The rotated query, split into fp16 hi + lo: q~ = R (s_K . (q / lambda_K))
  // with lambda before the rotation, q~ = R (s_K . q) / lambda_K with lambda
  // after it (so that <q, x_t> = <q~, y_t>), R = H / sqrt(D) or the SRFT.
  for (int r = warp; r < kMaxRows; r += kAW) {
    if constexpr (FMT & kFmtSrft) {
      if (lane == 0) {
        float2 z[D / 2];
        if (r < R) {
          const uint32_t* qr = reinterpret_cast<const uint32_t*>(
              P.q + (static_cast<int64_t>(b) * P.Hkv * R + kvh * R + r) * D);
#pragma unroll
          for (int n = 0; n < D / 2; ++n) {
            float2 x = half2_bits_to_float2(qr[n]);
            if constexpr ((FMT & kFmtAfter) == 0) x = make_float2(x.x / P.lam_k[2 * n], x.y / P.lam_k[2 * n + 1]);
            z[n] = make_float2(P.s_k[2 * n] < 0 ? -x.x : x.x, P.s_k[2 * n + 1] < 0 ? -x.y : x.y);
          }
          fft_fwd_from<D / 2, D / 2, D / 2>(z, P.wn);
          unpack_fwd1<D>(z, P.wd, [&](int n) -> float2 {
            float2 f = n == 0 ? make_float2(P.c, P.c) : make_float2(P.c1h, P.c1h);
            if constexpr (FMT & kFmtAfter) f = make_float2(f.x / P.lam_k[2 * n], f.y / P.lam_k[2 * n + 1]);
            if (n > D / 4) f.y = -f.y;                 // bins above N/2 come as conj(E - T)
            return f;
          });
        } else {
#pragma unroll
          for (int n = 0; n < D / 2; ++n) z[n] = make_float2(0.0f, 0.0f);
        }
#pragma unroll
        for (int n = 0; n < D / 2; ++n) {
          const __half2 hi = __floats2half2_rn(z[n].x, z[n].y);
          const float2 hf = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(z[n].x - hf.x, z[n].y - hf.y);
          reinterpret_cast<__half2*>(qt + r * D)[n] = hi;
          reinterpret_cast<__half2*>(qt + (kMaxRows + r) * D)[n] = lo;
        }
      }
      continue;
    }
    float v[DPL];
    if (r < R) {
      const uint16_t* qr = P.q + (static_cast<int64_t>(b) * P.Hkv * R + kvh * R + r) * D;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const int d = DPL * lane + i;
        float x = __half2float(__ushort_as_half(qr[d]));
        if constexpr ((FMT & kFmtAfter) == 0) x = x / P.lam_k[d];
        v[i] = P.s_k[d] < 0 ? -x : x;
      }
      warp_fwht<D>(v, lane);
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) v[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = DPL * lane + i;
      float y = v[i] * P.c;
      if constexpr (FMT & kFmtAfter) y = y / P.lam_k[d];
      const __half hi = __float2half_rn(y);
      const __half lo = __float2half_rn(y - __half2float(hi));
      qt[r * D + d] = hi;
      qt[(kMaxRows + r) * D + d] = lo;
    }
  }
  __syncthreads();

  // Score-product A fragments.  k-step j = (32-channel block bb = j/2, half
  // h = j%2); with c0 = 32 bb + 8 t + 2 h, k-indices (2t, 2t+1) are channels
  // (c0, c0 + 4) and (2t+8, 2t+9) are (c0 + 1, c0 + 5): nibbles (k, k + 16)
  // of the lane's code word 4 bb + t, k = 0, 4 (h = 0) or 8, 12 (h = 1).
  auto qpair = [&](int row, int d0, int d1) -> uint32_t {
    return static_cast<uint32_t>(__half_as_ushort(qt[row * D + d0])) |
           (static_cast<uint32_t>(__half_as_ushort(qt[row * D + d1])) << 16);
  };
  uint32_t Aq[KS][4];
#pragma unroll
  for (int j = 0; j < KS; ++j) {
    const int c0 = 32 * (j >> 1) + 8 * t + 2 * (j & 1);
    Aq[j][0] = qpair(g, c0, c0 + 4);
    Aq[j][1] = qpair(kMaxRows + g, c0, c0 + 4);
    Aq[j][2] = qpair(g, c0 + 1, c0 + 5);
    Aq[j][3] = qpair(kMaxRows + g, c0 + 1, c0 + 5);
  }
  // Bias of the biased codes: -8 2^-24 times each row's sum over a group.
  float bias_hi[NG], bias_lo[NG];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    float sh = 0.0f, sl = 0.0f;
    for (int d = gi * G; d < (gi + 1) * G; ++d) {
      sh += __half2float(qt[g * D + d]);
      sl += __half2float(qt[(kMaxRows + g) * D + d]);
    }
    bias_hi[gi] = -8.0f * 0x1p-24f * sh;
    bias_lo[gi] = -8.0f * 0x1p-24f * sl;
  }

  const int64_t row_base = static_cast<int64_t>(bh) * P.T;
  auto issue = [&](int blk, int stage) {
    if (blk >= nblk || lane != 0) return;
    const int kb = k0 + blk * kBK;
    const int nk = min(kBK, k1 - kb);
    const int nk16 = (nk + 15) & ~15;                            // stays inside T (T % 16 == 0)
    const int64_t row0 = row_base + kb;
    uint8_t* st = ring + (warp * kAStages + stage) * A::STAGE;
    const uint32_t cb = static_cast<uint32_t>(nk16 * (D / 2));
    const uint32_t sb = static_cast<uint32_t>(nk16 * NG * 2);
    mbar_expect_tx(&bar[stage], 2 * cb + 2 * sb);
    bulk_g2s(st, P.kp + row0 * (D / 2), cb, &bar[stage]);
    bulk_g2s(st + A::CB, P.vp + row0 * (D / 2), cb, &bar[stage]);
    bulk_g2s(st + 2 * A::CB, P.ks + row0 * NG, sb, &bar[stage]);
    bulk_g2s(st + 2 * A::CB + A::SB, P.vs + row0 * NG, sb, &bar[stage]);
  };
  for (int s = 0; s < kAStages; ++s) issue(warp + s * kAW, s);

  float O[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.0f;
  float psum[NG];                      // running sum of p * S_V per group (this lane's keys)
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) psum[gi] = 0.0f;
  float m = -INFINITY, l = 0.0f;
  bool failed = false;
  int k = 0;
  for (int blk = warp; blk < nblk; blk += kAW, ++k) {
    const int stage = k % kAStages;
    const bool ok = mbar_wait(&bar[stage], (k / kAStages) & 1, kSpin);
    if (__any_sync(kFull, !ok)) {
      failed = true;
      break;
    }
    const uint8_t* st = ring + (warp * kAStages + stage) * A::STAGE;
    const uint32_t* kc = reinterpret_cast<const uint32_t*>(st);
    const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + A::CB);
    const __half* ksc = reinterpret_cast<const __half*>(st + 2 * A::CB);
    const __half* vsc = reinterpret_cast<const __half*>(st + 2 * A::CB + A::SB);
    const int nk = min(kBK, k1 - (k0 + blk * kBK));

    // Scores of the block's 64 keys, in log2 units: z[sb][nt][e] for key
    // 16 sb + 8 nt + 2 t + e of head g.
    float z[kBK / 16][2][2];
#pragma unroll
    for (int sb = 0; sb < kBK / 16; ++sb) {
      float acc[NG][2][4];
#pragma unroll
      for (int gi = 0; gi < NG; ++gi)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          acc[gi][nt][0] = acc[gi][nt][1] = bias_hi[gi];
          acc[gi][nt][2] = acc[gi][nt][3] = bias_lo[gi];
        }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int kk = 16 * sb + 8 * nt + g;
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) {
          const uint32_t w = kc[kk * W32 + 4 * bb + t];
          mma16816(acc[(32 * bb) / G][nt], Aq[2 * bb], sub_pair(w), sub_pair(w >> 4));
          mma16816(acc[(32 * bb) / G][nt], Aq[2 * bb + 1], sub_pair(w >> 8), sub_pair(w >> 12));
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = 16 * sb + 8 * nt + 2 * t + e;
          float zz = 0.0f;
#pragma unroll
          for (int gi = 0; gi < NG; ++gi)
            zz += __half2float(ksc[key * NG + gi]) * (acc[gi][nt][e] + acc[gi][nt][2 + e]);
          z[sb][nt][e] = (key < nk && g < R) ? zz * P.scale_log2 : -INFINITY;
        }
      }
    }
    // Online softmax: new running max, rescale what is accumulated.
    float mx = -INFINITY;
#pragma unroll
    for (int sb = 0; sb < kBK / 16; ++sb)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) mx = fmaxf(mx, fmaxf(z[sb][nt][0], z[sb][nt][1]));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float mnew = fmaxf(m, mx);
    const float alpha = (mnew == -INFINITY) ? 1.0f : exp2f(m - mnew);
    m = mnew;
    if (__any_sync(kFull, alpha != 1.0f)) {     // skipped once the running maxima settle
      l *= alpha;
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) psum[gi] *= alpha;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        O[n][0] *= alpha; O[n][1] *= alpha; O[n][2] *= alpha; O[n][3] *= alpha;
      }
    }
#pragma unroll
    for (int sb = 0; sb < kBK / 16; ++sb) {
      float p[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          p[nt][e] = (z[sb][nt][e] == -INFINITY) ? 0.0f : exp2f(z[sb][nt][e] - m);
          l += p[nt][e];
        }
      // A fragments of the value product, one per scale group: p * S_V as hi + lo.
      uint32_t Ap[NG][4];
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int key = 16 * sb + 8 * nt + 2 * t;
          // masked keys may sit on stale scale bytes: keep their weight exactly 0
          const float pa = p[nt][0] == 0.0f ? 0.0f : p[nt][0] * __half2float(vsc[key * NG + gi]);
          const float pb = p[nt][1] == 0.0f ? 0.0f : p[nt][1] * __half2float(vsc[(key + 1) * NG + gi]);
          psum[gi] += pa + pb;
          const __half2 hi = __floats2half2_rn(pa, pb);
          const float2 hf = __half22float2(hi);
          Ap[gi][2 * nt] = h2bits(hi);
          Ap[gi][2 * nt + 1] = h2bits(__floats2half2_rn(pa - hf.x, pb - hf.y));
        }
      }
      // B fragments: n-tile nu = 4 bb + u, column g <-> channel 32 bb + 4 g + u,
      // i.e. nibble u & 1 of byte 16 bb + 2 g + (u >> 1).
      const int ka = 16 * sb + 2 * t;
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        const int wi = 4 * bb + (g >> 1);
        const uint32_t a0 = vc[ka * W32 + wi], a1 = vc[(ka + 1) * W32 + wi];
        const uint32_t c0 = vc[(ka + 8) * W32 + wi], c1 = vc[(ka + 9) * W32 + wi];
        const uint32_t sel0 = static_cast<uint32_t>(2 * (g & 1)) | ((4u + 2 * (g & 1)) << 8);
        const uint32_t sel1 = sel0 + 0x101u;
        const uint32_t xa0 = __byte_perm(a0, a1, sel0), xa1 = __byte_perm(a0, a1, sel1);
        const uint32_t xc0 = __byte_perm(c0, c1, sel0), xc1 = __byte_perm(c0, c1, sel1);
        const int gi = (32 * bb) / G;
        mma16816(O[4 * bb + 0], Ap[gi], sub_pair(xa0), sub_pair(xc0));
        mma16816(O[4 * bb + 1], Ap[gi], sub_pair(xa0 >> 4), sub_pair(xc0 >> 4));
        mma16816(O[4 * bb + 2], Ap[gi], sub_pair(xa1), sub_pair(xc1));
        mma16816(O[4 * bb + 3], Ap[gi], sub_pair(xa1 >> 4), sub_pair(xc1 >> 4));
      }
    }
    __syncwarp();                      // the stage is consumed: refill it
    issue(blk + kAStages * kAW, stage);
  }
  bool lost = false;                   // a copy may still land in this warp's ring
  if (failed) {
    if (lane == 0) atomicOr(&g_attn_fault, 1u);
    // drain whatever this warp still has in flight, the stage that gave up
    // included, before the ring is reused
    for (int s = 0; s < kAStages; ++s) {
      const int kk2 = k + s;
      if (warp + kk2 * kAW < nblk && !mbar_wait(&bar[kk2 % kAStages], (kk2 / kAStages) & 1, kSpin))
        lost = true;
    }
    lost = __any_sync(kFull, lost);
  }
  l += __shfl_xor_sync(kFull, l, 1);
  l += __shfl_xor_sync(kFull, l, 2);
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    psum[gi] += __shfl_xor_sync(kFull, psum[gi], 1);
    psum[gi] += __shfl_xor_sync(kFull, psum[gi], 2);
  }
  // every warp is out of the ring: reuse it for the merge, unless a copy may
  // still land there (the fault word is set; the block writes nothing)
  if (__syncthreads_or(lost)) return;
  if (g < R) {
    float* cw = comb + (warp * kMaxRows + g) * D;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int bb = n >> 2, u = n & 3;
      const float corr = 8.0f * psum[(32 * bb) / G];
      cw[32 * bb + 8 * t + u] = __fmaf_rn(O[n][0] + O[n][2], 0x1p24f, -corr);
      cw[32 * bb + 8 * t + 4 + u] = __fmaf_rn(O[n][1] + O[n][3], 0x1p24f, -corr);
    }
    if (t == 0) {
      ml[(warp * kMaxRows + g) * 2] = m;
      ml[(warp * kMaxRows + g) * 2 + 1] = l;
    }
  }
  __syncthreads();
  for (int r = warp; r < R; r += kAW) {
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < kAW; ++w2) M = fmaxf(M, ml[(w2 * kMaxRows + r) * 2]);
    float lsum = 0.0f, v[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) v[i] = 0.0f;
#pragma unroll
    for (int w2 = 0; w2 < kAW; ++w2) {
      const float mw = ml[(w2 * kMaxRows + r) * 2];
      const float e = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
      lsum += e * ml[(w2 * kMaxRows + r) * 2 + 1];
#pragma unroll
      for (int i = 0; i < DPL; ++i) v[i] += e * comb[(w2 * kMaxRows + r) * D + DPL * lane + i];
    }
    if (P.nsplit == 1) {
      uint16_t* orow = P.out + (static_cast<int64_t>(b) * P.Hkv * R + kvh * R + r) * D;
      finish_head<D, FMT>(P, v, lsum, orow, lane, comb + r * D);   // row r's first slot: read above
    } else {
      float* pr = P.part + (static_cast<int64_t>(item) * R + r) * (D + 4);
      if (lane == 0) { pr[0] = M; pr[1] = lsum; }
#pragma unroll
      for (int i = 0; i < DPL; ++i) pr[4 + DPL * lane + i] = v[i];
    }
  }
}

// Merge of the key splits of one (sequence, KV head): one warp per head.
template <int D, int FMT>
__global__ void __launch_bounds__(kMaxRows * 32)
kvq_attn_combine_kernel(const __grid_constant__ AttnParams P) {
  __shared__ float scr[kMaxRows][D];
  constexpr int DPL = D / 32;
  const int bh = blockIdx.x, b = bh / P.Hkv, kvh = bh % P.Hkv;
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (r >= P.R) return;
  const int64_t stride = static_cast<int64_t>(P.R) * (D + 4);
  const float* base = P.part + (static_cast<int64_t>(bh) * P.nsplit * P.R + r) * (D + 4);
  float M = -INFINITY;
  for (int s = 0; s < P.nsplit; ++s) M = fmaxf(M, base[s * stride]);
  float lsum = 0.0f, v[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) v[i] = 0.0f;
  for (int s = 0; s < P.nsplit; ++s) {
    const float* pr = base + s * stride;
    const float e = (pr[0] == -INFINITY) ? 0.0f : exp2f(pr[0] - M);
    lsum += e * pr[1];
#pragma unroll
    for (int i = 0; i < DPL; ++i) v[i] += e * pr[4 + DPL * lane + i];
  }
  uint16_t* orow = P.out + (static_cast<int64_t>(b) * P.Hkv * P.R + kvh * P.R + r) * D;
  finish_head<D, FMT>(P, v, lsum, orow, lane, scr[r]);
}

// ---------------------------------------------------------------------------
// Launch plumbing.
// ---------------------------------------------------------------------------

int attn_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1) v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Key-axis split: enough blocks for about four waves of two blocks per SM,
// but at least one 64-key block per warp in every split.
struct Split {
  int nsplit, chunk;
};
Split choose_split(int64_t pairs, int T) {
  if (T <= 0 || pairs <= 0) return Split{1, T > 0 ? T : kBK};
  const int64_t target = static_cast<int64_t>(attn_sms()) * 2 * 4;
  int64_t ns = (target + pairs - 1) / pairs;
  const int64_t max_ns = (T + kBK * kAW - 1) / (kBK * kAW);
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  int64_t chunk = (T + ns - 1) / ns;
  chunk = (chunk + kBK - 1) / kBK * kBK;
  ns = (T + chunk - 1) / chunk;
  return Split{static_cast<int>(ns), static_cast<int>(chunk)};
}

int64_t part_bytes(int64_t pairs, int R, int D, int nsplit) {
  return nsplit > 1 ? pairs * nsplit * R * (D + 4) * static_cast<int64_t>(sizeof(float)) : 0;
}

int check_attn(int B, int Hq, int Hkv, int T, int D, int G) {
  if (D != 64 && D != 128) return KVQ_ERR_DIM;
  if ((G != 32 && G != 64 && G != 128) || G > D) return KVQ_ERR_GROUP;
  if (B < 0 || T < 0 || (T % 16) != 0 || Hkv < 1 || Hq < Hkv || (Hq % Hkv) != 0 ||
      Hq / Hkv > kMaxRows)
    return KVQ_ERR_COUNT;
  if (static_cast<int64_t>(B) * Hkv * T >= (int64_t{1} << 40)) return KVQ_ERR_COUNT;
  return KVQ_OK;
}

template <int D, int G, int FMT>
int launch_attn(const AttnParams& P, int64_t pairs, cudaStream_t st) {
  using A = Attn<D, G>;
  auto k = kvq_attn_kernel<D, G, FMT>;
  static std::atomic<int> ready[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev >= 0 && dev < 64 && ready[dev].load(std::memory_order_relaxed) == 0) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, A::SMEM);
    ready[dev].store(1, std::memory_order_relaxed);
  }
  const int64_t items = pairs * P.nsplit;
  (void)cudaGetLastError();
  k<<<static_cast<unsigned>(items), kAW * 32, A::SMEM, st>>>(P);
  if (P.nsplit > 1)
    kvq_attn_combine_kernel<D, FMT><<<static_cast<unsigned>(pairs), kMaxRows * 32, 0, st>>>(P);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_attn_cuda_error = static_cast<int>(e);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
}

template <int D, int G>
int launch_fmt(const AttnParams& P, int64_t pairs, int flags, cudaStream_t st) {
  switch (flags) {
    case 0: return launch_attn<D, G, 0>(P, pairs, st);
    case 1: return launch_attn<D, G, 1>(P, pairs, st);
    case 2: return launch_attn<D, G, 2>(P, pairs, st);
    default: return launch_attn<D, G, 3>(P, pairs, st);
  }
}

// The SRFT's twiddles at length D (built once per D).
template <int D>
void attn_twiddles(AttnParams& P) {
  struct Tw { float2 wn[D / 2]; float2 wd[D / 2 + 1]; };
  static const Tw tw = [] {
    Tw t{};
    for (int k = 0; k < D / 2; ++k) t.wn[k] = root_f32(k, D / 2);
    for (int k = 0; k <= D / 2; ++k) t.wd[k] = root_f32(k, D);
    return t;
  }();
  memcpy(P.wn, tw.wn, sizeof(tw.wn));
  memcpy(P.wd, tw.wd, sizeof(tw.wd));
}

}  // namespace

// Read (and optionally clear) the attention kernels' fault word; used by
// kvq_fault_status.
__attribute__((visibility("hidden"))) unsigned int kvq_attn_fault_word(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_fault, sizeof(v)) != cudaSuccess) return 0;
  if (clear && v) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_attn_fault, &zero, sizeof(zero));
  }
  return v;
}
__attribute__((visibility("hidden"))) int kvq_attn_last_cuda_error() { return g_attn_cuda_error; }

// Device address of the static scratch, looked up once per device (on the
// first kvq_attention_decode_static call that needs it on that device) and
// kept for the life of the process: a cudaDeviceReset rebuilds the module and
// leaves the cached address stale, so the entry point is not for use across
// a device reset.  Internal linkage: the library exports only its C ABI.
static void* static_scratch(int& rc) {
  static std::atomic<void*> cache[64];
  int dev = 0;
  rc = KVQ_OK;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    rc = KVQ_ERR_LAUNCH;
    return nullptr;
  }
  void* p = cache[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_static_scratch);
    if (e != cudaSuccess || p == nullptr) {
      g_attn_cuda_error = static_cast<int>(e);
      rc = KVQ_ERR_LAUNCH;
      return nullptr;
    }
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

extern "C" {

int64_t kvq_attention_workspace_bytes(int B, int Hq, int Hkv, int T, int D, int group) {
  if (check_attn(B, Hq, Hkv, T, D, group) != KVQ_OK) return -1;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  const Split sp = choose_split(pairs, T);
  return part_bytes(pairs, Hq / Hkv, D, sp.nsplit);
}

int kvq_attention_decode_ex(const uint16_t* q, const uint8_t* k_packed, const uint16_t* k_scales,
                            const uint8_t* v_packed, const uint16_t* v_scales, const int32_t* seq_len,
                            const float* lambda_k, const int8_t* signs_k, const float* lambda_v,
                            const int8_t* signs_v, int B, int Hq, int Hkv, int T, int D, int group,
                            int flags, float sm_scale, uint16_t* out, void* workspace,
                            int64_t workspace_bytes, void* stream) {
  const int rc = check_attn(B, Hq, Hkv, T, D, group);
  if (rc != KVQ_OK) return rc;
  if ((flags & ~3) != 0) return KVQ_ERR_GROUP;
  if (B == 0) return KVQ_OK;
  if (!q || !k_packed || !k_scales || !v_packed || !v_scales || !seq_len || !lambda_k ||
      !signs_k || !lambda_v || !signs_v || !out)
    return KVQ_ERR_NULL;
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (!al(q, 16) || !al(k_packed, 16) || !al(v_packed, 16) || !al(k_scales, 16) ||
      !al(v_scales, 16) || !al(out, 16) || !al(lambda_k, 4) || !al(lambda_v, 4) || !al(seq_len, 4))
    return KVQ_ERR_ALIGN;
  if (!std::isfinite(sm_scale)) return KVQ_ERR_COUNT;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  Split sp = choose_split(pairs, T);
  if (sp.nsplit > 1 && (workspace == nullptr || !al(workspace, 16) ||
                        workspace_bytes < part_bytes(pairs, Hq / Hkv, D, sp.nsplit)))
    sp = Split{1, T > 0 ? T : kBK};                      // no room for partials: no split
  if (pairs * sp.nsplit > 0x7fffffffLL) return KVQ_ERR_COUNT;
  AttnParams P;
  P.q = q; P.kp = k_packed; P.ks = k_scales; P.vp = v_packed; P.vs = v_scales;
  P.seq_len = seq_len; P.lam_k = lambda_k; P.s_k = signs_k; P.lam_v = lambda_v; P.s_v = signs_v;
  P.out = out;
  P.part = static_cast<float*>(workspace);
  P.Hkv = Hkv; P.T = T; P.R = Hq / Hkv; P.nsplit = sp.nsplit; P.chunk = sp.chunk;
  // scores come out of the key product scaled by 2^-24 (subnormal codes)
  P.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634 * 16777216.0);
  P.c = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  P.c1h = static_cast<float>(1.0 / std::sqrt(2.0 * static_cast<double>(D)));
  memset(P.wn, 0, sizeof(P.wn));
  memset(P.wd, 0, sizeof(P.wd));
  if (flags & kFmtSrft) {
    if (D == 64) attn_twiddles<64>(P);
    else attn_twiddles<128>(P);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (D * 1000 + group) {
    case 64032: return launch_fmt<64, 32>(P, pairs, flags, st);
    case 64064: return launch_fmt<64, 64>(P, pairs, flags, st);
    case 128032: return launch_fmt<128, 32>(P, pairs, flags, st);
    case 128064: return launch_fmt<128, 64>(P, pairs, flags, st);
    case 128128: return launch_fmt<128, 128>(P, pairs, flags, st);
    default: return KVQ_ERR_GROUP;
  }
}

int kvq_attention_decode(const uint16_t* q, const uint8_t* k_packed, const uint16_t* k_scales,
                         const uint8_t* v_packed, const uint16_t* v_scales, const int32_t* seq_len,
                         const float* lambda_k, const int8_t* signs_k, const float* lambda_v,
                         const int8_t* signs_v, int B, int Hq, int Hkv, int T, int D, int group,
                         float sm_scale, uint16_t* out, void* workspace, int64_t workspace_bytes,
                         void* stream) {
  return kvq_attention_decode_ex(q, k_packed, k_scales, v_packed, v_scales, seq_len, lambda_k,
                                 signs_k, lambda_v, signs_v, B, Hq, Hkv, T, D, group, 0, sm_scale,
                                 out, workspace, workspace_bytes, stream);
}

int kvq_attention_decode_static(const uint16_t* q, const uint8_t* k_packed, const uint16_t* k_scales,
                                const uint8_t* v_packed, const uint16_t* v_scales,
                                const int32_t* seq_len, const float* lambda_k,
                                const int8_t* signs_k, const float* lambda_v,
                                const int8_t* signs_v, int B, int Hq, int Hkv, int T, int D,
                                int group, float sm_scale, uint16_t* out, void* stream) {
  const int rc = check_attn(B, Hq, Hkv, T, D, group);
  if (rc != KVQ_OK) return rc;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  const int64_t need = part_bytes(pairs, Hq / Hkv, D, choose_split(pairs, T).nsplit);
  if (need > kStaticScratchBytes) return KVQ_ERR_COUNT;      // more than the static scratch holds
  void* ws = nullptr;
  if (need > 0 && B > 0) {
    int src = KVQ_OK;
    ws = static_scratch(src);
    if (src != KVQ_OK) return src;
  }
  return kvq_attention_decode(q, k_packed, k_scales, v_packed, v_scales, seq_len, lambda_k, signs_k,
                              lambda_v, signs_v, B, Hq, Hkv, T, D, group, sm_scale, out, ws, need,
                              stream);
}

}  // extern "C"
