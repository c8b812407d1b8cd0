// kvq_attn.cu -- the C-ABI launcher of the fused decode attention over the
// int4 rotated-domain KV cache (include/kvq.h: kvq_attention_decode,
// kvq_attention_decode_ex, kvq_attention_decode_static,
// kvq_attention_workspace_bytes): argument checks, the key-axis split, the
// static scratch, and the dispatch to the unit of the head dimension
// (kvq_attn.cuh, compiled once per D in kvq_attn_d<D>.cu).

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "kvq.h"
#include "kvq_attn_common.cuh"

namespace {

using namespace kvqa;

// Scratch of kvq_attention_decode_static: the partial (max, sum, rotated
// output) rows of the key splits, 8 MiB per device.  Nothing in it has to
// start at zero: every split writes its own slots before the merge kernel,
// later on the same stream, reads them.  Calls that overlap in time (other
// streams, other host threads) share it and race.
constexpr int64_t kStaticScratchBytes = int64_t{8} << 20;
static __device__ __align__(256) unsigned char g_attn_static_scratch[kStaticScratchBytes];
thread_local int g_attn_host_error = 0;

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

// Key-axis split: enough blocks for about four waves of three blocks per SM,
// but at least one 32-key block per warp in every split.
struct Split {
  int nsplit, chunk;
};
Split choose_split(int64_t pairs, int T) {
  if (T <= 0 || pairs <= 0) return Split{1, T > 0 ? T : kBK};
  const int64_t target = static_cast<int64_t>(attn_sms()) * 3 * 4;
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
  if (D != 64 && D != 128 && D != 256) return KVQ_ERR_DIM;
  if ((G != 16 && G != 32 && G != 64 && G != 128) || G > D) return KVQ_ERR_GROUP;
  if (B < 0 || T < 0 || (T % 16) != 0 || Hkv < 1 || Hq < Hkv || (Hq % Hkv) != 0 ||
      Hq / Hkv > kMaxRows)
    return KVQ_ERR_COUNT;
  if (static_cast<int64_t>(B) * Hkv * T >= (int64_t{1} << 40)) return KVQ_ERR_COUNT;
  return KVQ_OK;
}

}  // namespace

// Read (and optionally clear) the attention kernels' fault words (one per
// head-dimension unit); used by kvq_fault_status.
__attribute__((visibility("hidden"))) unsigned int kvq_attn_fault_word(int clear) {
  return kvq_attn_fault_word_64(clear) | kvq_attn_fault_word_128(clear) | kvq_attn_fault_word_256(clear);
}
__attribute__((visibility("hidden"))) int kvq_attn_last_cuda_error() {
  if (g_attn_host_error) return g_attn_host_error;
  if (const int e = kvq_attn_last_cuda_error_64()) return e;
  if (const int e = kvq_attn_last_cuda_error_128()) return e;
  return kvq_attn_last_cuda_error_256();
}

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
      g_attn_host_error = static_cast<int>(e);
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
  memset(&P, 0, sizeof(P));
  P.q = q; P.kp = k_packed; P.ks = k_scales; P.vp = v_packed; P.vs = v_scales;
  P.seq_len = seq_len; P.lam_k = lambda_k; P.s_k = signs_k; P.lam_v = lambda_v; P.s_v = signs_v;
  P.out = out;
  P.part = static_cast<float*>(workspace);
  P.Hkv = Hkv; P.T = T; P.R = Hq / Hkv; P.nsplit = sp.nsplit; P.chunk = sp.chunk;
  P.fmt = flags;
  // scores come out of the key product scaled by 2^-24 (subnormal codes)
  P.scale_log2 = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634 * 16777216.0);
  P.c = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  P.c1h = static_cast<float>(1.0 / std::sqrt(2.0 * static_cast<double>(D)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 64: return kvq_attn_launch_64(P, pairs, group, st);
    case 128: return kvq_attn_launch_128(P, pairs, group, st);
    default: return kvq_attn_launch_256(P, pairs, group, st);
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
