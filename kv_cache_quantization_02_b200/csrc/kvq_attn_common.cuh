// kvq_attn_common.cuh -- what the decode-attention units share with the
// C-ABI launcher in kvq_attn.cu: the launch parameters, the block and key
// tiling the workspace size depends on, and the per-head-dimension entry
// points (kvq_attn_d64.cu, kvq_attn_d128.cu, kvq_attn_d256.cu each compile
// kvq_attn.cuh for one D, so the three build in parallel).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace kvqa {

constexpr int kAW = 4;                       // warps per block
constexpr int kBK = 32;                      // keys per streamed block
constexpr int kMaxRows = 8;                  // query heads per KV head

// Cache formats (the codec variants' flags): bit 0 lambda after the rotation,
// bit 1 the SRFT rotation.
constexpr int kFmtAfter = 1, kFmtSrft = 2;

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
  int fmt;                      // kFmtAfter | kFmtSrft
  float scale_log2;             // sm_scale * log2(e) * 2^24 (the key product comes out scaled by 2^-24)
  float c;                      // fp32 1/sqrt(D)
  float c1h;                    // fp32 1/sqrt(2D): the SRFT's normalisation of 2 X_k
};

}  // namespace kvqa

// One unit per head dimension: launch (group 16, 32, 64 or 128, arguments
// already checked), and that unit's fault word and last CUDA error.
#define KVQA_UNIT_DECL(D)                                                                        \
  __attribute__((visibility("hidden"))) int kvq_attn_launch_##D(const kvqa::AttnParams& P,       \
                                                                int64_t pairs, int group,       \
                                                                cudaStream_t st);               \
  __attribute__((visibility("hidden"))) unsigned int kvq_attn_fault_word_##D(int clear);         \
  __attribute__((visibility("hidden"))) int kvq_attn_last_cuda_error_##D();
KVQA_UNIT_DECL(64)
KVQA_UNIT_DECL(128)
KVQA_UNIT_DECL(256)
#undef KVQA_UNIT_DECL
