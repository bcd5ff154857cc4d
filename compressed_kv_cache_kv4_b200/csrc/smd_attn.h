// smd_attn.h -- parameter block and launcher of the learner-side masked attention.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kv4 {

struct SmdParams {
  const __nv_bfloat16 *q;   // [B][T][Hq][D]
  const __nv_bfloat16 *k;   // [B][T][Hkv][D]
  const __nv_bfloat16 *v;   // [B][T][Hkv][D]
  const int32_t *lens;      // nullable [B]
  const uint32_t *mask;     // nullable [B][Hkv][T][mask_stride]
  int B, T, Hq, Hkv, G, mask_stride;
  float scale_log2;         // softmax_scale * log2(e)
  void *out;                // [B][T][Hq][D] bf16 or fp32
  int out_fp32;
  uint32_t *err;            // nullable error word
};

// Longest sequence: the per-CTA list of active 64-key blocks lives in shared memory.
constexpr int kMaxSmdT = 65536;
constexpr int kMaxSmdBlocks = kMaxSmdT / 64;

size_t smd_smem_bytes(int D, int T);
cudaError_t launch_smd(const SmdParams &p, int D, cudaStream_t stream);

}  // namespace kv4
