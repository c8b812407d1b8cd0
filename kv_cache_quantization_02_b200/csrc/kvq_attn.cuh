// kvq_attn.cuh -- fused decode attention over the int4 rotated-domain KV
// cache for B200 (sm_100a): the kernels behind kvq_attention_decode[_ex]
// (include/kvq.h) at one head dimension, D = KVQ_ATTN_D; kvq_attn_d<D>.cu
// instantiate it and kvq_attn.cu holds the C ABI.
//
// Method: "The Kernel That Finally Did Something -- And Didn't Quite Agree
// With Itself" (VeloxQuant-MLX blog), "Fused group-affine (KIVI-style)
// attention": the quantised keys and values are reconstructed in registers
// inside a FlashAttention-style online softmax, so no dequantised K or V ever
// reaches memory, and the key axis is split flash-decoding style when there
// are few sequences.  The cache rows here are int4 codes of the rotated vector
// y = R diag(s) (lambda . x) (or R diag(s) x / lambda with lambda after the
// rotation; R = H / sqrt(D) or the SRFT) with fp16 group scales ("When
// Quantization Is Free", technical summary, Methodologie 1-3), so the rotation
// moves to the query, once per head, instead of running once per key:
//     <q, x_t> = <q~, y_t>,   q~ = R diag(s_K) (q / lambda_K),
// and the values are summed in the rotated domain and rotated back once:
//     o = (diag(s_V) R^T (sum_t p_t y_t)) / lambda_V.
//
// Work decomposition.  A block of four warps owns one (sequence, KV head,
// key split); each warp streams 32-key blocks (codes and scales of K and V,
// four bulk copies into a private ring of 3 stages, 2 at G = 16) and keeps
// its own online-softmax state; the block merges the four states at the end.
// At D = 256 the warps work in pairs: both warps of a pair take the same
// blocks (one ring of 2 stages, the 128-byte code rows by swizzled tensor
// copies), each the channels of one half, and they add their partial scores
// through shared memory before the softmax.
// Both products run on the tensor cores as m16n8k16 fp16 MMAs with fp32
// accumulation, with the N dimension = 4 query heads x 2 parts (q~ and p S_V
// each as an fp16 value plus its fp16 remainder, ~2^-22 together):
//   * scores: M = 16 keys, K = 16 channels.  A lane reads one 32-bit code
//     word per key and 32 channels; its four nibble pairs are the A fragments
//     of two k-steps (low nibbles as n 2^-24, high nibbles as 16 n 2^-24,
//     their query entries divided by 16), and every k-step stays inside one
//     scale group (G = 16: a k-step spans two groups and runs once per group
//     with the other group's entries zero).  The group's scale multiplies
//     the per-group partial sums key by key after the MMA.  In the
//     accumulator layout lane (g, t) holds keys g and g + 8 of head t, both
//     parts: every lane's epilogue is useful work.
//   * values: M = 16 channels, K = 16 keys: the probabilities pass through a
//     per-warp shared-memory row so that lane (g, t) gets keys 2t, 2t+1,
//     2t+8, 2t+9 of head g/2; p S_V per scale group is the B fragment, and
//     byte permutes pair a channel's codes of four keys.  The output columns
//     of lane (g, t) are head t again, so the softmax rescale needs no
//     exchange.
// A biased code n = q + 8 in [0, 15] is the fp16 subnormal n 2^-24, exact,
// made by one mask-and-xor.  The key side adds -8 2^-24 times the query's
// group sums to each group's partial score before its scale multiplies it;
// the value side keeps the running sum of p S_V per group and subtracts 8
// times it once at the end.  The rotations of the query and of the output
// are one warp's work per head: the fast Walsh-Hadamard transform across the
// lanes, or the SRFT as a warp-wide real FFT.
//
// Every mbarrier wait is bounded; a warp that gives up sets the fault word
// and the block writes nothing.  A sequence length outside [0, T] is clamped
// and flagged.  Compiled with --fmad=true: the result is checked against the
// oracle to a derived tolerance, and a contracted multiply-add only removes a
// rounding.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "kvq.h"
#include "kvq_attn_common.cuh"

#ifndef KVQ_ATTN_D
#error "define KVQ_ATTN_D (64, 128 or 256) before including kvq_attn.cuh"
#endif

namespace {

using namespace kvqa;
constexpr unsigned kFullMask = 0xffffffffu;

#include "kvq_async.cuh"
#include "kvq_arith.cuh"

constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kSpin = 1u << 22;         // bounded mbarrier waits

__device__ unsigned int g_attn_fault = 0;    // bit 0: a wait gave up; bit 3: bad sequence length

// ---- the SRFT of one row across a warp ---------------------------------------
// y = M x: y_0 = X_0 / sqrt(D), y_1 = X_(D/2) / sqrt(D), (y_2k, y_2k+1) =
// sqrt(2) (Re, Im) X_k / sqrt(D), X the length-D DFT of x with the root
// omega_D = exp(-2 pi i / D) ("When Quantization Is Free", technical summary,
// Methodologie 1).  M is orthogonal.  The real DFT runs as a complex one of
// length N = D/2 on z_n = x_2n + i x_2n+1, lane L holding z_(ZPL L + j) (j <
// ZPL = N / 32), in four steps (n = j + ZPL L, k = k1 + 32 k2): 32-point
// butterflies across the lanes for each j (decimation in frequency, so lane
// L ends with k1 = bitrev5(L)), a twiddle omega_N^(j k1), ZPL-point DFTs in
// the lane over j; then the Hermitian unpacking, 2 X_k = (Z_k + conj Z_(N-k))
// - i omega_D^k (Z_k - conj Z_(N-k)).  The adjoint runs the same steps
// backwards with conjugate roots.  tw holds omega_D^e, e in [0, D/2].

// omega_D^e, e in [0, D), from the half table: omega_D^(e + D/2) = -omega_D^e.
template <int D>
__device__ __forceinline__ float2 tw_pow(const float2* tw, int e) {
  if (e <= D / 2) return tw[e];
  const float2 w = tw[e - D / 2];
  return make_float2(-w.x, -w.y);
}
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ __forceinline__ float2 cmul_conj(float2 a, float2 b) {     // a conj(b)
  return make_float2(a.x * b.x + a.y * b.y, a.y * b.x - a.x * b.y);
}
__device__ __forceinline__ float2 shfl_xor2(float2 v, int m) {
  return make_float2(__shfl_xor_sync(kFull, v.x, m), __shfl_xor_sync(kFull, v.y, m));
}

// This warp's table of omega_D^e, e in [0, D/2] (shared memory).
template <int D>
__device__ __forceinline__ void build_roots(float2* tw, int lane) {
  for (int e = lane; e <= D / 2; e += 32) {
    float sn, cs;
    sincospif(2.0f * static_cast<float>(e) / static_cast<float>(D), &sn, &cs);
    tw[e] = make_float2(cs, -sn);
  }
  __syncwarp();
}

// In the lane: Z_k2 = sum_j omega_ZPL^(+-j k2) z_j (INV: the + sign).
template <int ZPL, bool INV>
__device__ __forceinline__ void lane_dft(float2 (&z)[ZPL]) {
  if constexpr (ZPL == 2) {
    const float2 a = z[0], b = z[1];
    z[0] = make_float2(a.x + b.x, a.y + b.y);
    z[1] = make_float2(a.x - b.x, a.y - b.y);
  } else if constexpr (ZPL == 4) {
    const float2 a = make_float2(z[0].x + z[2].x, z[0].y + z[2].y), b = make_float2(z[0].x - z[2].x, z[0].y - z[2].y);
    const float2 c = make_float2(z[1].x + z[3].x, z[1].y + z[3].y), d = make_float2(z[1].x - z[3].x, z[1].y - z[3].y);
    const float2 id = INV ? make_float2(-d.y, d.x) : make_float2(d.y, -d.x);     // (+-i) d
    z[0] = make_float2(a.x + c.x, a.y + c.y);
    z[2] = make_float2(a.x - c.x, a.y - c.y);
    z[1] = make_float2(b.x + id.x, b.y + id.y);
    z[3] = make_float2(b.x - id.x, b.y - id.y);
  }
}

// y = M x for one row in shared memory, written over x; y_i / div[i] when
// div is not null.
template <int D>
__device__ __forceinline__ void warp_srft_fwd(float* row, const float2* tw, const float* div, float c,
                                              float c1h, int lane) {
  constexpr int N = D / 2, ZPL = N / 32;
  float2 z[ZPL];
#pragma unroll
  for (int j = 0; j < ZPL; ++j) z[j] = *reinterpret_cast<const float2*>(row + 2 * (ZPL * lane + j));
  __syncwarp();
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1) {
    const bool hi = (lane & h) != 0;
    const float2 w = hi ? tw[(lane & (h - 1)) * (D / (2 * h))] : make_float2(1.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < ZPL; ++j) {
      const float2 u = shfl_xor2(z[j], h);
      const float2 v = hi ? make_float2(u.x - z[j].x, u.y - z[j].y) : make_float2(z[j].x + u.x, z[j].y + u.y);
      z[j] = cmul(v, w);
    }
  }
  const int k1 = static_cast<int>(__brev(static_cast<unsigned>(lane)) >> 27);
#pragma unroll
  for (int j = 1; j < ZPL; ++j) z[j] = cmul(z[j], tw_pow<D>(tw, 2 * j * k1));
  lane_dft<ZPL, false>(z);
  // z[k2] = Z_(k1 + 32 k2); Z_(N-k) is register ZPL-1-k2 of lane bitrev5(32 - k1)
  // (k1 > 0), or register (ZPL - k2) mod ZPL of this lane (k1 = 0)
  const int src = static_cast<int>(__brev(static_cast<unsigned>((32 - k1) & 31)) >> 27);
  float2 zp[ZPL];
#pragma unroll
  for (int k2 = 0; k2 < ZPL; ++k2) {
    const float2 v = make_float2(__shfl_sync(kFull, z[ZPL - 1 - k2].x, src), __shfl_sync(kFull, z[ZPL - 1 - k2].y, src));
    zp[k2] = k1 == 0 ? z[(ZPL - k2) % ZPL] : v;
  }
#pragma unroll
  for (int k2 = 0; k2 < ZPL; ++k2) {
    const int k = k1 + 32 * k2;
    float y0, y1;
    if (k == 0) {                                  // X_0 and X_N, both real
      y0 = c * (z[0].x + z[0].y);
      y1 = c * (z[0].x - z[0].y);
    } else {
      const float2 e = make_float2(z[k2].x + zp[k2].x, z[k2].y - zp[k2].y);    // Z_k + conj Z_(N-k)
      const float2 f = make_float2(z[k2].x - zp[k2].x, z[k2].y + zp[k2].y);    // Z_k - conj Z_(N-k)
      const float2 tt = cmul(f, tw[k]);
      y0 = c1h * (e.x + tt.y);                     // (e - i tt) / sqrt(2 D)
      y1 = c1h * (e.y - tt.x);
    }
    if (div != nullptr) { y0 /= div[2 * k]; y1 /= div[2 * k + 1]; }
    *reinterpret_cast<float2*>(row + 2 * k) = make_float2(y0, y1);
  }
}

// o = M^T y for one row: y read from shared memory, lane L gets o_(DPL L + i)
// in o[i].  With X_0 = y_0, X_N = y_1, X_k = (y_2k + i y_2k+1) / sqrt 2, o_2m +
// i o_2m+1 = z_m / sqrt(D), z the inverse length-N DFT of Z_k = (X_k + conj
// X_(N-k)) + i omega_D^-k (X_k - conj X_(N-k)).
template <int D>
__device__ __forceinline__ void warp_srft_adj(float (&o)[D / 32], const float* row, const float2* tw, float c,
                                              float c1h, int lane) {
  constexpr int N = D / 2, ZPL = N / 32;
  const int k1 = static_cast<int>(__brev(static_cast<unsigned>(lane)) >> 27);
  float2 z[ZPL];
#pragma unroll
  for (int k2 = 0; k2 < ZPL; ++k2) {
    const int k = k1 + 32 * k2;
    if (k == 0) {
      const float y0 = row[0], y1 = row[1];
      z[k2] = make_float2(c * (y0 + y1), c * (y0 - y1));
    } else {
      const float2 yk = *reinterpret_cast<const float2*>(row + 2 * k);
      const float2 yp = *reinterpret_cast<const float2*>(row + 2 * (N - k));
      const float2 e = make_float2(yk.x + yp.x, yk.y - yp.y);
      const float2 f = make_float2(yk.x - yp.x, yk.y + yp.y);
      const float2 tt = cmul_conj(f, tw[k]);
      z[k2] = make_float2(c1h * (e.x - tt.y), c1h * (e.y + tt.x));     // (e + i tt) / sqrt(2 D)
    }
  }
  lane_dft<ZPL, true>(z);
#pragma unroll
  for (int j = 1; j < ZPL; ++j) z[j] = cmul_conj(z[j], tw_pow<D>(tw, 2 * j * k1));
#pragma unroll
  for (int h = 1; h <= 16; h <<= 1) {
    const bool hi = (lane & h) != 0;
    const float2 w = hi ? tw[(lane & (h - 1)) * (D / (2 * h))] : make_float2(1.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < ZPL; ++j) {
      const float2 tt = cmul_conj(z[j], w);
      const float2 u = shfl_xor2(tt, h);
      z[j] = hi ? make_float2(u.x - tt.x, u.y - tt.y) : make_float2(z[j].x + u.x, z[j].y + u.y);
    }
  }
#pragma unroll
  for (int j = 0; j < ZPL; ++j) { o[2 * j] = z[j].x; o[2 * j + 1] = z[j].y; }
}
thread_local int g_attn_cuda_error = 0;

template <int D, int G>
struct Attn {
  // D = 256 runs in warp pairs: the two warps of a pair take the same key
  // blocks, each the channels of one half, and add their partial scores
  // through shared memory; the pair streams one ring of key blocks.
  static constexpr bool PAIR = D == 256;
  static constexpr int NRG = PAIR ? kAW / 2 : kAW;  // key-block streams (rings) per block
  static constexpr int DH = PAIR ? D / 2 : D;       // channels of one warp
  static constexpr int NG = D / G;                  // scale groups of a row
  static constexpr int NGH = DH / G;                // scale groups of one warp
  static constexpr int NBK = DH / 32;               // 32-channel blocks (score k-step pairs) of one warp
  static constexpr int KS = DH / 16;                // k-steps of one warp's score product
  static constexpr int NCT = DH / 16;               // 16-channel tiles of one warp's value product
  static constexpr int W32 = D / 8;                 // 32-bit words of one code row
  static constexpr int ST = (D >= 256 || G == 16) ? 2 : 3;   // ring depth
  static constexpr int CB = kBK * D / 2;            // code bytes of one block
  static constexpr int SB = kBK * NG * 2;           // scale bytes of one block
  // K codes, V codes, K scales, V scales; in pairs (128-byte code rows, which
  // arrive by 128-byte-swizzled tensor copies) a multiple of 1 KiB, the
  // swizzle's period
  static constexpr int STAGE = PAIR ? (2 * CB + 2 * SB + 1023) / 1024 * 1024 : 2 * CB + 2 * SB;
  static constexpr int RING = NRG * ST * STAGE;
  static constexpr int COMB = NRG * kMaxRows * D * 4;
  static constexpr int AREA = RING > COMB ? RING : COMB;   // the merge reuses the ring
  static constexpr int QF = kMaxRows * D * 4;       // rotated query rows, fp32
  static constexpr int SC = 2 * kBK * NGH * 4;      // per warp: the block's K and V scales, fp32
  static constexpr int PS = kBK + 8;                // row stride of the probability rows
  static constexpr int PB = kMaxRows * PS * 4;      // per warp: probabilities [head][key]
  static constexpr int XZ = PAIR ? NRG * 2 * 2 * 2 * 4 * 32 * 4 : 0;   // partial scores [ring][parity][half][2 head tiles][4][lane]
  static constexpr int NBAR = PAIR ? NRG * (2 * ST + 1) : kAW * ST;     // full (and empty, exchange) barriers
  static constexpr int SMEM = AREA + QF + kAW * (SC + PB) + XZ + NBAR * 8 + kAW * kMaxRows * 8 + (PAIR ? 1024 : 0);
  static constexpr int DPL = D / 32;                // channels per lane in the row transforms
  static_assert(STAGE % 16 == 0 && (SC + PB) % 16 == 0, "16-byte aligned areas");
};

// Biased code pairs as fp16 subnormals.  A word of codes xor 0x88888888
// holds n = q + 8 in [0, 15] in every nibble (the two's-complement nibble q
// xor 8); of such a word x, lo_pair takes the nibbles at bits 0-3 and 16-19
// (the low nibbles of bytes 0 and 2) and hi_pair those at bits 4-7 and 20-23
// (the high nibbles): the half holding n (low) or 16 n (high) is the
// subnormal n 2^-24 or 16 n 2^-24, exact, in one mask.
constexpr uint32_t kBias8 = 0x88888888u;
__device__ __forceinline__ uint32_t lo_pair(uint32_t x) { return x & 0x000F000Fu; }
__device__ __forceinline__ uint32_t hi_pair(uint32_t x) { return x & 0x00F000F0u; }

// d = a b + d on the tensor cores (m16n8k16, fp16 operands, fp32 accumulate),
// and d = a b.
__device__ __forceinline__ void mma_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_init(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

// Four 8x8 matrices of 16-bit elements from shared memory (ldmatrix): lane
// i gives the address of row i % 8 of matrix i / 8 (16 bytes, 16-byte
// aligned).  Lane (g, t) = (i / 4, i % 4) receives, of matrix j, elements
// (g, 2t) and (g, 2t + 1) (plain: the 32-bit word t of row g), or with .trans
// elements (2t, g) and (2t + 1, g) (the 16-bit column g of rows 2t, 2t + 1).
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(row)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(row)));
}

// The two parts of a pair: (x0, x1) as fp16 (part 0), or their fp16
// remainders x - fp16(x) (part 1; negp = -1 as fp16 bits, else -0).  The
// remainder comes from one mixed-precision multiply-add per value with the
// packed fp16 value as operand (exact: x and fp16(x) agree to 11 bits), so
// no conversion back to fp32 is needed.
__device__ __forceinline__ uint32_t part_pair(float x0, float x1, uint16_t negp) {
  const uint32_t h = float2_to_half2_bits(x0, x1);
  float d0, d1;
  asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "fma.rn.f32.f16 %0, a, %3, %4;\n\tfma.rn.f32.f16 %1, b, %3, %5;\n\t}"
      : "=f"(d0), "=f"(d1) : "r"(h), "h"(negp), "f"(x0), "f"(x1));
  return float2_to_half2_bits(d0, d1);
}

// 2^x by the SFU's approximation (relative error about 2^-22, results below
// 2^-126 flushed to 0, 2^-inf = +0); the softmax weights need no more.
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// v as fp16 (part 0) or the fp16 remainder v - fp16(v) (part 1): the two parts
// sum to v within 2^-22 |v|.
__device__ __forceinline__ uint16_t f16_part(float v, int part) {
  const __half h = __float2half_rn(v);
  return __half_as_ushort(part ? __float2half_rn(v - __half2float(h)) : h);
}

// N consecutive floats of shared memory into registers, in 16-byte loads
// where N allows (the rows are 16-byte aligned when N is a multiple of 4).
template <int N>
__device__ __forceinline__ void load_row(float (&r)[N], const float* p) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const float4 v = *reinterpret_cast<const float4*>(p + i);
      r[i] = v.x; r[i + 1] = v.y; r[i + 2] = v.z; r[i + 3] = v.w;
    }
  } else if constexpr (N == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    r[0] = v.x; r[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) r[i] = p[i];
  }
}

// N fp16 scales from shared memory as fp32, in the widest loads their
// alignment allows (the N halves start at a multiple of 2N bytes).
template <int N>
__device__ __forceinline__ void load_scales(float (&r)[N], const uint16_t* p) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(p + i);
      const float2 a = half2_bits_to_float2(u.x), b = half2_bits_to_float2(u.y);
      r[i] = a.x; r[i + 1] = a.y; r[i + 2] = b.x; r[i + 3] = b.y;
    }
  } else if constexpr (N == 2) {
    const float2 a = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(p));
    r[0] = a.x; r[1] = a.y;
  } else {
    r[0] = __half2float(__ushort_as_half(p[0]));
  }
}

// N floats into shared memory (16-byte aligned when N is a multiple of 4).
template <int N>
__device__ __forceinline__ void store_row(float* p, const float (&r)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) *reinterpret_cast<float4*>(p + i) = make_float4(r[i], r[i + 1], r[i + 2], r[i + 3]);
  } else if constexpr (N == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(r[0], r[1]);
  } else {
    p[0] = r[0];
  }
}

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
// SRFT's transpose (the warp-wide adjoint above, the row gathered in `scr`,
// D floats of this warp's shared memory; tw this warp's table of roots).
template <int D>
__device__ __forceinline__ void finish_head(const AttnParams& P, float (&v)[D / 32], float l,
                                            uint16_t* out_row, int lane, float* scr, const float2* tw) {
  constexpr int DPL = D / 32;
  const bool after = (P.fmt & kFmtAfter) != 0;
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) v[i] *= inv;
  if ((P.fmt & kFmtSrft) == 0) {
    if (after) {
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
      h[i] = __half_as_ushort(__float2half_rn(after ? zs : zs / P.lam_v[d]));
    }
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2*>(out_row + DPL * lane) =
          make_uint2(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16));
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) out_row[DPL * lane + i] = h[i];
    }
  } else {
    // y (the merged rotated-domain sum) through shared memory, then
    // out_i = s_V,i sum_j M[j][i] y_j (lambda after: y / lambda_V first, per j)
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = DPL * lane + i;
      scr[d] = after ? v[i] / P.lam_v[d] : v[i];
    }
    __syncwarp();
    float o[DPL];
    warp_srft_adj<D>(o, scr, tw, P.c, P.c1h, lane);
    uint16_t h[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = DPL * lane + i;
      const float zs = P.s_v[d] < 0 ? -o[i] : o[i];
      h[i] = __half_as_ushort(__float2half_rn(after ? zs : zs / P.lam_v[d]));
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) out_row[DPL * lane + i] = h[i];
    __syncwarp();
  }
}

// One block of four warps per (sequence, KV head, key split); head tiles of
// four query heads (NH = 1 for up to four heads per KV head, 2 for up to 8).
template <int D, int G, int NH>
__global__ void __launch_bounds__(kAW * 32, (NH > 1) ? 2 : 3)
kvq_attn_kernel(const __grid_constant__ AttnParams P, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap) {
  using A = Attn<D, G>;
  constexpr bool PAIR = A::PAIR;
  constexpr int NRG = A::NRG, DH = A::DH;
  constexpr int NG = A::NG, NGH = A::NGH, NBK = A::NBK, KS = A::KS, NCT = A::NCT, DPL = A::DPL;
  constexpr int ST = A::ST, PS = A::PS;
  constexpr int CPG = (G >= 32) ? G / 32 : 1;     // score k-step pairs per group (G = 16: two groups per pair)
  extern __shared__ __align__(128) uint8_t sm_raw[];
  uint8_t* sm = PAIR ? align_smem_1k(sm_raw) : sm_raw;   // pairs: 1 KiB-aligned stages
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = PAIR ? warp >> 1 : warp;          // this warp's ring (key-block stream)
  const int half = PAIR ? warp & 1 : 0;            // the channel half of a pair's warp
  const bool issuer = half == 0;                   // the warp that issues the ring's copies
  const int cofs = half * DH, gofs = cofs / G;     // this warp's first channel and group
  uint8_t* ring = sm;                                                  // [ring][stage][STAGE]
  float* qf = reinterpret_cast<float*>(sm + A::AREA);                  // [8][D]
  float* scw = qf + kMaxRows * D + warp * ((A::SC + A::PB) / 4);       // this warp's area:
  float* sk = scw;                                                     //   K scales [kBK][NGH], fp32
  float* sv = scw + kBK * NGH;                                         //   V scales [kBK][NGH], fp32
  float* pw = scw + A::SC / 4;                                         //   probabilities [8][PS]
  float* xz = reinterpret_cast<float*>(sm + A::AREA + A::QF + kAW * (A::SC + A::PB));   // pairs' partial scores
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + A::AREA + A::QF + kAW * (A::SC + A::PB) + A::XZ);
  float* ml = reinterpret_cast<float*>(bars + A::NBAR);               // [ring][8][2]: m, l
  float* comb = reinterpret_cast<float*>(sm);                          // [ring][8][D], after the key loop

  const int g = lane >> 2, t = lane & 3;
  const int item = blockIdx.x;
  const int split = item % P.nsplit;
  const int bh = item / P.nsplit;                                      // b * Hkv + kv head
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

  uint64_t* bar = bars + ST * rg;                  // the ring's stages are full
  uint64_t* empty = bars + NRG * ST + ST * rg;     // pairs: both warps are done with a stage
  uint64_t* xch = bars + 2 * NRG * ST + rg;        // pairs: both warps wrote their partial scores
  if (lane == 0 && issuer) {
    for (int s = 0; s < ST; ++s) mbar_init(&bar[s], 1);
    if constexpr (PAIR) {
      for (int s = 0; s < ST; ++s) mbar_init(&empty[s], 2);
      mbar_init(xch, 64);
    }
    mbar_fence_init();
  }
  const int64_t row_base = static_cast<int64_t>(bh) * P.T;
  // The ring's blocks are rg, rg + NRG, ...; each issue copies the next one
  // into the given stage, the sources advancing by NRG blocks of rows.
  int next_blk = rg, next_kb = k0 + rg * kBK;
  const uint8_t* kp_next = P.kp + (row_base + next_kb) * (D / 2);
  const uint8_t* vp_next = P.vp + (row_base + next_kb) * (D / 2);
  const uint16_t* ks_next = P.ks + (row_base + next_kb) * NG;
  const uint16_t* vs_next = P.vs + (row_base + next_kb) * NG;
  auto issue = [&](int stage) {
    if (next_blk < nblk && lane == 0 && issuer) {
      const int nk = min(kBK, k1 - next_kb);
      const int nk16 = (nk + 15) & ~15;                          // stays inside T (T % 16 == 0)
      uint8_t* st = ring + (rg * ST + stage) * A::STAGE;
      const uint32_t cb = static_cast<uint32_t>(nk16 * (D / 2));
      const uint32_t sb = static_cast<uint32_t>(nk16 * NG * 2);
      if constexpr (PAIR) {        // whole 32-row boxes (rows past the split are masked)
        mbar_expect_tx(&bar[stage], 2 * A::CB + 2 * sb);
        const int y = static_cast<int>(row_base + next_kb);
        tensor_g2s(st, &kmap, 0, y, &bar[stage]);
        tensor_g2s(st + A::CB, &vmap, 0, y, &bar[stage]);
      } else {
        mbar_expect_tx(&bar[stage], 2 * cb + 2 * sb);
        bulk_g2s(st, kp_next, cb, &bar[stage]);
        bulk_g2s(st + A::CB, vp_next, cb, &bar[stage]);
      }
      bulk_g2s(st + 2 * A::CB, ks_next, sb, &bar[stage]);
      bulk_g2s(st + 2 * A::CB + A::SB, vs_next, sb, &bar[stage]);
    }
    next_blk += NRG;
    next_kb += NRG * kBK;
    kp_next += NRG * kBK * (D / 2);
    vp_next += NRG * kBK * (D / 2);
    ks_next += NRG * kBK * NG;
    vs_next += NRG * kBK * NG;
  };
  __syncwarp();
  for (int s = 0; s < ST; ++s) issue(s);

  // The rotated query, fp32: q~ = R (s_K . (q / lambda_K)) with lambda before
  // the rotation, q~ = R (s_K . q) / lambda_K with lambda after it (so that
  // <q, x_t> = <q~, y_t>), R = H / sqrt(D) or the SRFT; rows R..7 are zero.
  const bool after = (P.fmt & kFmtAfter) != 0;
  float2* tw = reinterpret_cast<float2*>(scw);          // the SRFT's roots, in this warp's scale area until the key loop
  if (P.fmt & kFmtSrft) build_roots<D>(tw, lane);
  for (int r = warp; r < kMaxRows; r += kAW) {
    float* qr_out = qf + r * D;
    if (P.fmt & kFmtSrft) {
      // q' = s_K . q (lambda before: . / lambda_K) in this row's qf slot, then
      // q~_j = sum_i M[j][i] q'_i (lambda after: / lambda_K,j)
      if (r < R) {
        const uint16_t* qr = P.q + (static_cast<int64_t>(b) * P.Hkv * R + kvh * R + r) * D;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
          const int d = DPL * lane + i;
          float x = __half2float(__ushort_as_half(qr[d]));
          if (!after) x = x / P.lam_k[d];
          qr_out[d] = P.s_k[d] < 0 ? -x : x;
        }
        __syncwarp();
        warp_srft_fwd<D>(qr_out, tw, after ? P.lam_k : nullptr, P.c, P.c1h, lane);
        __syncwarp();
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) qr_out[DPL * lane + i] = 0.0f;
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
        if (!after) x = x / P.lam_k[d];
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
      if (after) y = y / P.lam_k[d];
      qr_out[d] = y;
    }
  }
  __syncthreads();

  // Score B fragments.  k-step j = 2 bb + s of 32-channel block bb: lane
  // (g, t) reads code word w = 4 bb + t of its two keys, and the k-indices
  // (2t, 2t+1) are channels 8w + 2s, 8w + 2s + 4 (low nibbles), (2t+8, 2t+9)
  // are 8w + 2s + 1, 8w + 2s + 5 (high nibbles, which arrive as 16 n: their
  // query entries are divided by 16).  Column g is head 4 ht + g/2, part g & 1
  // (the fp16 value, or its fp16 remainder).  With G = 16 a k-step spans two
  // groups (lanes t < 2 and t >= 2), and runs once per group with the other
  // group's k-indices zero in B.
  constexpr int BQ = (G == 16) ? 2 : 1;
  uint32_t bq[NH][KS][BQ][2];
#pragma unroll
  for (int ht = 0; ht < NH; ++ht)
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      const float* qr = qf + (4 * ht + (g >> 1)) * D;
      const int c0 = cofs + 8 * (4 * (j >> 1) + t) + 2 * (j & 1);
      const int part = g & 1;
      const uint32_t b0 = f16_part(qr[c0], part) | (uint32_t(f16_part(qr[c0 + 4], part)) << 16);
      const uint32_t b1 = f16_part(qr[c0 + 1] * 0.0625f, part) |
                          (uint32_t(f16_part(qr[c0 + 5] * 0.0625f, part)) << 16);
      if constexpr (G == 16) {
        const bool upper = t >= 2;
        bq[ht][j][0][0] = upper ? 0u : b0;
        bq[ht][j][0][1] = upper ? 0u : b1;
        bq[ht][j][1][0] = upper ? b0 : 0u;
        bq[ht][j][1][1] = upper ? b1 : 0u;
      } else {
        bq[ht][j][0][0] = b0;
        bq[ht][j][0][1] = b1;
      }
    }
  // The bias of the biased codes in a group's partial score: -8 2^-24 times
  // the group's sum of the B entries (times 16 for the high-nibble entries),
  // both parts, of this lane's score head 4 ht + t.  The eight lanes of a
  // head split the group's channels and add up by shuffles.
  float bias[NH][NGH];
#pragma unroll
  for (int ht = 0; ht < NH; ++ht) {
    const float* qr = qf + (4 * ht + t) * D;
#pragma unroll
    for (int gi = 0; gi < NGH; ++gi) {
      float s0 = 0.0f, s1 = 0.0f;
      for (int c = (gofs + gi) * G + g; c < (gofs + gi + 1) * G; c += 8) {
        const bool odd = c & 1;
        const float v = odd ? qr[c] * 0.0625f : qr[c];
        const float w = odd ? 16.0f : 1.0f;
        s0 += w * __half2float(__ushort_as_half(f16_part(v, 0)));
        s1 += w * __half2float(__ushort_as_half(f16_part(v, 1)));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        s0 += __shfl_xor_sync(kFull, s0, o);
        s1 += __shfl_xor_sync(kFull, s1, o);
      }
      bias[ht][gi] = -8.0f * 0x1p-24f * (s0 + s1);
    }
  }
  const uint16_t neg_part = (g & 1) ? 0xBC00u : 0x8000u;   // -1 or -0 as fp16

  float O[NH][NCT][4];
#pragma unroll
  for (int ht = 0; ht < NH; ++ht)
#pragma unroll
    for (int n = 0; n < NCT; ++n) O[ht][n][0] = O[ht][n][1] = O[ht][n][2] = O[ht][n][3] = 0.0f;
  float m[NH], l[NH];
#pragma unroll
  for (int ht = 0; ht < NH; ++ht) { m[ht] = -INFINITY; l[ht] = 0.0f; }
  // sum of p S_V per group over this lane's keys, head 4 ht + g/2: the value
  // product runs on biased codes, and 8 times this is its bias
  float pc[NH][NGH];
#pragma unroll
  for (int ht = 0; ht < NH; ++ht)
#pragma unroll
    for (int gi = 0; gi < NGH; ++gi) pc[ht][gi] = 0.0f;
  bool head_ok[NH];                    // this lane's score head is a real head
#pragma unroll
  for (int ht = 0; ht < NH; ++ht) head_ok[ht] = 4 * ht + t < R;
  const float scale = P.scale_log2;
  // byte offset of 16-byte chunk c of code row r in a stage's code tile (pairs:
  // the tensor copy's 128-byte swizzle puts it at chunk c ^ (r mod 8))
  auto code_at = [](int r, int c) -> int { return r * (D / 2) + ((PAIR ? (c ^ (r & 7)) : c) << 4); };
  bool failed = false;
  int k = 0;
  int stage = 0;
  uint32_t phase = 0;                  // parity of the stage's current fill
  for (int blk = rg; blk < nblk; blk += NRG, ++k) {
    const bool ok = mbar_wait(&bar[stage], phase, kSpin);
    if (__any_sync(kFull, !ok)) {
      failed = true;
      break;
    }
    const uint8_t* st = ring + (rg * ST + stage) * A::STAGE;
    const uint32_t* kc = reinterpret_cast<const uint32_t*>(st);
    const uint32_t* vc = reinterpret_cast<const uint32_t*>(st + A::CB);
    const uint16_t* ksh = reinterpret_cast<const uint16_t*>(st + 2 * A::CB);
    const uint16_t* vsh = reinterpret_cast<const uint16_t*>(st + 2 * A::CB + A::SB);
    const int nk = min(kBK, k1 - (k0 + blk * kBK));

    const bool tail = nk < kBK;          // the split's last block may hold fewer keys

    // The block's scales as fp32; in a tail block, keys at or past nk (stale
    // or unwritten rows) get 0, so that their zero weights stay exactly 0.
    if constexpr (PAIR) {
      // lane = key: the scales of this warp's groups
      const bool live = !tail || lane < nk;
      float kf[NGH], vf[NGH];
      load_scales<NGH>(kf, ksh + lane * NG + gofs);
      load_scales<NGH>(vf, vsh + lane * NG + gofs);
#pragma unroll
      for (int e = 0; e < NGH; ++e) {
        kf[e] = live ? kf[e] : 0.0f;
        vf[e] = live ? vf[e] : 0.0f;
      }
      store_row<NGH>(sk + lane * NGH, kf);
      store_row<NGH>(sv + lane * NGH, vf);
    } else {
#pragma unroll
    for (int i0 = 0; i0 < kBK * NG; i0 += 128) {
      const int i = i0 + 4 * lane;
      if (i < kBK * NG) {
        const uint2 kw = *reinterpret_cast<const uint2*>(ksh + i);
        const uint2 vw = *reinterpret_cast<const uint2*>(vsh + i);
        const float2 k01 = half2_bits_to_float2(kw.x), k23 = half2_bits_to_float2(kw.y);
        const float2 v01 = half2_bits_to_float2(vw.x), v23 = half2_bits_to_float2(vw.y);
        float ko[4] = {k01.x, k01.y, k23.x, k23.y}, vo[4] = {v01.x, v01.y, v23.x, v23.y};
        if (tail) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool live = (i + e) / NG < nk;
            ko[e] = live ? ko[e] : 0.0f;
            vo[e] = live ? vo[e] : 0.0f;
          }
        }
        *reinterpret_cast<float4*>(sk + i) = make_float4(ko[0], ko[1], ko[2], ko[3]);
        *reinterpret_cast<float4*>(sv + i) = make_float4(vo[0], vo[1], vo[2], vo[3]);
      }
    }
    }
    __syncwarp();

    // Scores, log2 units: zs[ht][mt][r] for key 16 mt + g + 8 r of head 4 ht + t.
    // A group's partial products fold into the score (times the key's group
    // scale) as soon as its last k-step is done, so one group's accumulators
    // (two at G = 16) are live at a time.
    float zs[NH][2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      constexpr int GPB = (G == 16) ? 2 : 1;          // groups finished per 32-channel block
      float acc[NH][GPB][4];
      float s0[NGH], s1[NGH];
      load_row<NGH>(s0, sk + (16 * mt + g) * NGH);
      load_row<NGH>(s1, sk + (16 * mt + 8 + g) * NGH);
      float z0[NH], z1[NH];
#pragma unroll
      for (int ht = 0; ht < NH; ++ht) z0[ht] = z1[ht] = 0.0f;
      uint32_t kw[4];
#pragma unroll
      for (int bb = 0; bb < NBK; ++bb) {
        // words 4 bb + t of keys g and g + 8, two blocks bb per load: matrix
        // j = (keys 8 (j & 1) .. + 7 of the M-tile, 16-byte chunk bb + j / 2)
        if (bb % 2 == 0)
          ldsm_x4(kw, reinterpret_cast<const uint8_t*>(kc) +
                          code_at(16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1), half * NBK + bb + (lane >> 4)));
        const uint32_t w0 = kw[2 * (bb & 1)] ^ kBias8;
        const uint32_t w1 = kw[2 * (bb & 1) + 1] ^ kBias8;
        const uint32_t a0[4] = {lo_pair(w0), lo_pair(w1), hi_pair(w0), hi_pair(w1)};
        const uint32_t a1[4] = {lo_pair(w0 >> 8), lo_pair(w1 >> 8), hi_pair(w0 >> 8), hi_pair(w1 >> 8)};
#pragma unroll
        for (int ht = 0; ht < NH; ++ht) {
          if constexpr (G == 16) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              mma_init(acc[ht][h2], a0, bq[ht][2 * bb][h2][0], bq[ht][2 * bb][h2][1]);
              mma_acc(acc[ht][h2], a1, bq[ht][2 * bb + 1][h2][0], bq[ht][2 * bb + 1][h2][1]);
            }
          } else {
            if (bb % CPG == 0)
              mma_init(acc[ht][0], a0, bq[ht][2 * bb][0][0], bq[ht][2 * bb][0][1]);
            else
              mma_acc(acc[ht][0], a0, bq[ht][2 * bb][0][0], bq[ht][2 * bb][0][1]);
            mma_acc(acc[ht][0], a1, bq[ht][2 * bb + 1][0][0], bq[ht][2 * bb + 1][0][1]);
          }
          // z += S_K (both parts + the codes' bias) for each group done here
          if (G == 16 || bb % CPG == CPG - 1) {
#pragma unroll
            for (int h2 = 0; h2 < GPB; ++h2) {
              const int gi = (G == 16) ? 2 * bb + h2 : bb / CPG;
              z0[ht] = __fmaf_rn(s0[gi], (acc[ht][h2][0] + acc[ht][h2][1]) + bias[ht][gi], z0[ht]);
              z1[ht] = __fmaf_rn(s1[gi], (acc[ht][h2][2] + acc[ht][h2][3]) + bias[ht][gi], z1[ht]);
            }
          }
        }
      }
#pragma unroll
      for (int ht = 0; ht < NH; ++ht) {
        zs[ht][mt][0] = z0[ht];
        zs[ht][mt][1] = z1[ht];
      }
    }
    if constexpr (PAIR) {
      // the two halves' partial scores through shared memory (one buffer per
      // block parity, so that a warp one block ahead writes the other one),
      // added in the same order by both warps
      float* xo = xz + ((rg * 2 + (k & 1)) * 2 + half) * 256;
      const float* xi = xz + ((rg * 2 + (k & 1)) * 2 + (half ^ 1)) * 256;
#pragma unroll
      for (int ht = 0; ht < NH; ++ht)
#pragma unroll
        for (int i = 0; i < 4; ++i) xo[(ht * 4 + i) * 32 + lane] = zs[ht][i >> 1][i & 1];
      mbar_arrive(xch);
      const bool okx = mbar_wait(xch, k & 1, kSpin);
      if (__any_sync(kFull, !okx)) {
        failed = true;
        break;
      }
#pragma unroll
      for (int ht = 0; ht < NH; ++ht)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float o = xi[(ht * 4 + i) * 32 + lane];
          float& z = zs[ht][i >> 1][i & 1];
          z = half ? o + z : z + o;
        }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int ht = 0; ht < NH; ++ht) {
        zs[ht][mt][0] *= scale;
        zs[ht][mt][1] *= scale;
        if (tail || !head_ok[ht]) {          // keys past nk and padded heads weigh 0
          if (!head_ok[ht] || 16 * mt + g >= nk) zs[ht][mt][0] = -INFINITY;
          if (!head_ok[ht] || 16 * mt + 8 + g >= nk) zs[ht][mt][1] = -INFINITY;
        }
      }

    // Online softmax per head, over the block's 32 keys: the eight lanes of a
    // head (same t) hold four keys each.
#pragma unroll
    for (int ht = 0; ht < NH; ++ht) {
      float mx = fmaxf(fmaxf(zs[ht][0][0], zs[ht][0][1]), fmaxf(zs[ht][1][0], zs[ht][1][1]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      const float mnew = fmaxf(m[ht], mx);
      const float alpha = (mnew == -INFINITY) ? 1.0f : exp2_fast(m[ht] - mnew);
      m[ht] = mnew;
      if (__any_sync(kFull, alpha != 1.0f)) {   // skipped once the running maxima settle
        l[ht] *= alpha;
#pragma unroll
        for (int n = 0; n < NCT; ++n) {       // this lane's output columns are head 4 ht + t
          O[ht][n][0] *= alpha; O[ht][n][1] *= alpha; O[ht][n][2] *= alpha; O[ht][n][3] *= alpha;
        }
        const float alpha_b = __shfl_sync(kFull, alpha, g >> 1);   // head 4 ht + g/2
#pragma unroll
        for (int gi = 0; gi < NGH; ++gi) pc[ht][gi] *= alpha_b;
      }
      // key 16 mt + 8 r + g goes to slot 16 mt + 8 r + g (G >= 32), or to
      // 16 mt + 8 r + 2 (g & 3) + (g >> 2) (G = 16, whose value product's
      // lane t reads keys t, t + 4 and t + 8, t + 12 of each 16 as 8-byte pairs)
      float* prow = pw + (4 * ht + t) * PS + ((G == 16) ? 2 * (g & 3) + (g >> 2) : g);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          // a real head has a finite maximum from its first block on, so a
          // masked key gives 2^-inf = 0; a padded head's weights are never read
          const float p = exp2_fast(zs[ht][mt][r] - mnew);
          l[ht] += p;
          prow[16 * mt + 8 * r] = p;
        }
    }
    __syncwarp();

    // Values, per 16-key step: O[ht][ct] (rows = 16 channels of tile ct,
    // columns = head 4 ht + c/2, part c & 1) += V codes x (p S_V).  G >= 32:
    // the k-indices (2t, 2t+1, 2t+8, 2t+9) are keys 2t, 2t+1, 2t+8, 2t+9 of
    // the step, and a transposing ldmatrix gives lane (g, t) bytes 2g, 2g+1
    // of a 16-byte chunk of keys 2t and 2t+1 in one word (the same channel of
    // both keys at bits 0-3 and 16-19).  G = 16: they are keys t, t + 4,
    // t + 8, t + 12, gathered with byte permutes from word reads (the four
    // lanes t of a read then hit rows of both parities: two-way, not
    // four-way, bank conflicts on 64-byte rows).
    constexpr int KSTEP = (G == 16) ? 4 : 1;         // key stride inside a k-index pair
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int ka = 16 * ks + ((G == 16) ? t : 2 * t);   // keys ka, ka + KSTEP (+ 8)
      float2 pa[NH], pb[NH];
#pragma unroll
      for (int ht = 0; ht < NH; ++ht) {
        const float* prow = pw + (4 * ht + (g >> 1)) * PS + 16 * ks + 2 * t;
        pa[ht] = *reinterpret_cast<const float2*>(prow);
        pb[ht] = *reinterpret_cast<const float2*>(prow + 8);
      }
      constexpr int GC = NGH < 4 ? NGH : 4;           // groups per scale load
      float sq[4][GC];
      uint32_t vw[4];                                 // two chunks of V codes, transposed
#pragma unroll
      for (int gi = 0; gi < NGH; ++gi) {
        // B fragments of this group: p S_V for the four keys, as part g & 1
        if (gi % GC == 0) {
          load_row<GC>(sq[0], sv + ka * NGH + gi);
          load_row<GC>(sq[1], sv + (ka + KSTEP) * NGH + gi);
          load_row<GC>(sq[2], sv + (ka + 8) * NGH + gi);
          load_row<GC>(sq[3], sv + (ka + 8 + KSTEP) * NGH + gi);
        }
        const float s0 = sq[0][gi % GC], s1 = sq[1][gi % GC], s2 = sq[2][gi % GC], s3 = sq[3][gi % GC];
        uint32_t bv[NH][2];
#pragma unroll
        for (int ht = 0; ht < NH; ++ht) {
          const float x0 = pa[ht].x * s0, x1 = pa[ht].y * s1, x2 = pb[ht].x * s2, x3 = pb[ht].y * s3;
          pc[ht][gi] += (x0 + x1) + (x2 + x3);
          bv[ht][0] = part_pair(x0, x1, neg_part);
          bv[ht][1] = part_pair(x2, x3, neg_part);
        }
        if constexpr (G == 16) {
          // tile gi: channels 16 gi + 2 g (low nibble, row g) and + 1 (row g + 8):
          // byte g & 3 of word 2 gi + g / 4
          const int wv = half * (DH / 8) + 2 * gi + (g >> 2), by = g & 3;
          auto word = [&](int r) { return vc[code_at(r, wv >> 2) / 4 + (wv & 3)]; };
          const uint32_t w0 = word(ka), w1 = word(ka + 4), w2 = word(ka + 8), w3 = word(ka + 12);
          const uint32_t sel = static_cast<uint32_t>(by | ((4 + by) << 4));
          const uint32_t x = __byte_perm(__byte_perm(w0, w1, sel), __byte_perm(w2, w3, sel), 0x5140u) ^ kBias8;
          const uint32_t av[4] = {lo_pair(x), hi_pair(x), lo_pair(x >> 8), hi_pair(x >> 8)};
#pragma unroll
          for (int ht = 0; ht < NH; ++ht) mma_acc(O[ht][gi], av, bv[ht][0], bv[ht][1]);
        } else {
          // tile pair j (16-byte chunk j: 32 channels, in group gi): tile 2j
          // holds channels 32j + 4g (row g, low nibble of byte 2g) and + 1 (row
          // g + 8), tile 2j + 1 channels + 2 and + 3 (byte 2g + 1)
#pragma unroll
          for (int j = gi * (G / 32); j < (gi + 1) * (G / 32); ++j) {
            // matrix m = (keys 8 (m & 1) .. + 7 of the step, chunk (j & ~1) + m / 2)
            if (j % 2 == 0)
              ldsm_x4_t(vw, reinterpret_cast<const uint8_t*>(vc) +
                                code_at(16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1),
                                        half * (DH / 32) + (j & ~1) + (lane >> 4)));
            const uint32_t x0 = vw[2 * (j & 1)] ^ kBias8;       // keys 2t, 2t + 1
            const uint32_t x1 = vw[2 * (j & 1) + 1] ^ kBias8;   // keys 2t + 8, 2t + 9
            const uint32_t aa[4] = {lo_pair(x0), hi_pair(x0), lo_pair(x1), hi_pair(x1)};
            const uint32_t ab[4] = {lo_pair(x0 >> 8), hi_pair(x0 >> 8), lo_pair(x1 >> 8), hi_pair(x1 >> 8)};
#pragma unroll
            for (int ht = 0; ht < NH; ++ht) {
              mma_acc(O[ht][2 * j], aa, bv[ht][0], bv[ht][1]);
              mma_acc(O[ht][2 * j + 1], ab, bv[ht][0], bv[ht][1]);
            }
          }
        }
      }
    }
    __syncwarp();                      // the stage and the probability rows are consumed
    if constexpr (PAIR) {
      // the issuing warp refills the stage once its partner is done with it too
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (issuer) {
        const bool oke = mbar_wait(&empty[stage], phase, kSpin);
        if (__any_sync(kFull, !oke)) {
          failed = true;
          break;
        }
      }
    }
    issue(stage);
    if (++stage == ST) { stage = 0; phase ^= 1u; }
  }
  bool lost = false;                   // a copy may still land in this warp's ring
  if (failed) {
    if (lane == 0) atomicOr(&g_attn_fault, 1u);
    // drain whatever this warp still has in flight, the stage that gave up
    // included, before the ring is reused
    for (int s = 0; s < ST; ++s) {
      const int kk2 = k + s;
      if (issuer && rg + kk2 * NRG < nblk && !mbar_wait(&bar[kk2 % ST], (kk2 / ST) & 1, kSpin))
        lost = true;
    }
    lost = __any_sync(kFull, lost);
  }
#pragma unroll
  for (int ht = 0; ht < NH; ++ht) {
    l[ht] += __shfl_xor_sync(kFull, l[ht], 4);
    l[ht] += __shfl_xor_sync(kFull, l[ht], 8);
    l[ht] += __shfl_xor_sync(kFull, l[ht], 16);
  }
  // the bias sums of head 4 ht + t (lanes 8t .. 8t + 3 hold them after the
  // reduction over t)
  float bsum[NH][NGH];
#pragma unroll
  for (int ht = 0; ht < NH; ++ht)
#pragma unroll
    for (int gi = 0; gi < NGH; ++gi) {
      float v = pc[ht][gi];
      v += __shfl_xor_sync(kFull, v, 1);
      v += __shfl_xor_sync(kFull, v, 2);
      bsum[ht][gi] = 8.0f * __shfl_sync(kFull, v, 8 * t);
    }
  // every warp is out of the ring: reuse it for the merge, unless a copy may
  // still land there (the fault word is set; the block writes nothing)
  if (__syncthreads_or(lost)) return;
  // this warp's rotated-domain sums: y = 2^24 (both parts), high-nibble rows
  // / 16, less the bias of the biased codes
#pragma unroll
  for (int ht = 0; ht < NH; ++ht) {
    const int h = 4 * ht + t;
    if (h < R) {
      float* cw = comb + (rg * kMaxRows + h) * D + cofs;
#pragma unroll
      for (int ct = 0; ct < NCT; ++ct) {
        const int byte = (G == 16) ? 8 * ct + g : 16 * (ct >> 1) + 2 * g + (ct & 1);
        const float bz = bsum[ht][(G == 16) ? ct : (32 * (ct >> 1)) / G];
        cw[2 * byte] = __fmaf_rn(O[ht][ct][0] + O[ht][ct][1], 0x1p24f, -bz);
        cw[2 * byte + 1] = __fmaf_rn(O[ht][ct][2] + O[ht][ct][3], 0x1p20f, -bz);
      }
      if (g == 0 && issuer) {
        ml[(rg * kMaxRows + h) * 2] = m[ht];
        ml[(rg * kMaxRows + h) * 2 + 1] = l[ht];
      }
    }
  }
  __syncthreads();
  if ((P.fmt & kFmtSrft) && P.nsplit == 1) build_roots<D>(tw, lane);   // the scale area is free again
  for (int r = warp; r < R; r += kAW) {
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < NRG; ++w2) M = fmaxf(M, ml[(w2 * kMaxRows + r) * 2]);
    float lsum = 0.0f, v[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) v[i] = 0.0f;
#pragma unroll
    for (int w2 = 0; w2 < NRG; ++w2) {
      const float mw = ml[(w2 * kMaxRows + r) * 2];
      const float e = (mw == -INFINITY) ? 0.0f : exp2f(mw - M);
      lsum += e * ml[(w2 * kMaxRows + r) * 2 + 1];
#pragma unroll
      for (int i = 0; i < DPL; ++i) v[i] += e * comb[(w2 * kMaxRows + r) * D + DPL * lane + i];
    }
    if (P.nsplit == 1) {
      uint16_t* orow = P.out + (static_cast<int64_t>(b) * P.Hkv * R + kvh * R + r) * D;
      finish_head<D>(P, v, lsum, orow, lane, comb + r * D, tw);   // row r's first slot: read above
    } else {
      float* pr = P.part + (static_cast<int64_t>(item) * R + r) * (D + 4);
      if (lane == 0) { pr[0] = M; pr[1] = lsum; }
#pragma unroll
      for (int i = 0; i < DPL; ++i) pr[4 + DPL * lane + i] = v[i];
    }
  }
}

// Merge of the key splits of one (sequence, KV head): one warp per head.
template <int D>
__global__ void __launch_bounds__(kMaxRows * 32)
kvq_attn_combine_kernel(const __grid_constant__ AttnParams P) {
  __shared__ float scr[kMaxRows][D];
  __shared__ float2 tws[kMaxRows][D / 2 + 1];
  constexpr int DPL = D / 32;
  const int bh = blockIdx.x, b = bh / P.Hkv, kvh = bh % P.Hkv;
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (r >= P.R) return;
  if (P.fmt & kFmtSrft) build_roots<D>(tws[r], lane);
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
  finish_head<D>(P, v, lsum, orow, lane, scr[r], tws[r]);
}


// ---------------------------------------------------------------------------
// Launch plumbing.
// ---------------------------------------------------------------------------

// A tensor map over the code rows [rows][D/2 bytes] in 32-row boxes with the
// 128-byte swizzle (D = 256, whose rows are 128 bytes).
int encode_code_rows(CUtensorMap& map, const uint8_t* codes, int64_t rows) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return KVQ_ERR_LAUNCH;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(KVQ_ATTN_D / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(KVQ_ATTN_D / 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(KVQ_ATTN_D / 2), static_cast<cuuint32_t>(kBK)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_attn_cuda_error = static_cast<int>(r);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
}

template <int D, int G, int NH>
int launch_attn(const AttnParams& P, int64_t pairs, cudaStream_t st) {
  using A = Attn<D, G>;
  auto k = kvq_attn_kernel<D, G, NH>;
  CUtensorMap kmap, vmap;                        // pairs only: the code tiles' tensor copies
  memset(&kmap, 0, sizeof(kmap));
  memset(&vmap, 0, sizeof(vmap));
  if constexpr (A::PAIR) {
    const int64_t rows = pairs * P.T;
    if (rows >= (int64_t{1} << 31)) return KVQ_ERR_COUNT;   // tensor-copy row coordinates are int32
    int rc = encode_code_rows(kmap, P.kp, rows);
    if (rc == KVQ_OK) rc = encode_code_rows(vmap, P.vp, rows);
    if (rc != KVQ_OK) return rc;
  }
  static std::atomic<int> ready[64];             // the shared-memory opt-in, once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev < 0 || dev >= 64 || ready[dev].load(std::memory_order_relaxed) == 0) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, A::SMEM);
    if (dev >= 0 && dev < 64) ready[dev].store(1, std::memory_order_relaxed);
  }
  const int64_t items = pairs * P.nsplit;
  (void)cudaGetLastError();
  k<<<static_cast<unsigned>(items), kAW * 32, A::SMEM, st>>>(P, kmap, vmap);
  if (P.nsplit > 1)
    kvq_attn_combine_kernel<D><<<static_cast<unsigned>(pairs), kMaxRows * 32, 0, st>>>(P);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_attn_cuda_error = static_cast<int>(e);
    return KVQ_ERR_LAUNCH;
  }
  return KVQ_OK;
}

template <int D, int G>
int launch_nh(const AttnParams& P, int64_t pairs, cudaStream_t st) {
  return P.R <= 4 ? launch_attn<D, G, 1>(P, pairs, st) : launch_attn<D, G, 2>(P, pairs, st);
}

}  // namespace

#define KVQA_CAT2(a, b) a##b
#define KVQA_CAT(a, b) KVQA_CAT2(a, b)

__attribute__((visibility("hidden"))) int KVQA_CAT(kvq_attn_launch_, KVQ_ATTN_D)(
    const kvqa::AttnParams& P, int64_t pairs, int group, cudaStream_t st) {
  constexpr int D = KVQ_ATTN_D;
  switch (group) {
    case 16: return launch_nh<D, 16>(P, pairs, st);
    case 32: return launch_nh<D, 32>(P, pairs, st);
    case 64: return launch_nh<D, 64>(P, pairs, st);
    default:
      if constexpr (D >= 128) return launch_nh<D, 128>(P, pairs, st);
      return KVQ_ERR_GROUP;
  }
}

// Read (and optionally clear) this unit's fault word.
__attribute__((visibility("hidden"))) unsigned int KVQA_CAT(kvq_attn_fault_word_, KVQ_ATTN_D)(int clear) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_fault, sizeof(v)) != cudaSuccess) return 0;
  if (clear && v) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_attn_fault, &zero, sizeof(zero));
  }
  return v;
}
__attribute__((visibility("hidden"))) int KVQA_CAT(kvq_attn_last_cuda_error_, KVQ_ATTN_D)() {
  return g_attn_cuda_error;
}
