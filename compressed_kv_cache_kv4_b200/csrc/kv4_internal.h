// kv4_internal.h -- kernel parameter blocks and launchers inside libkv4.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kv4 {

struct AppendParams {
  const __nv_bfloat16 *k;   // [T][Hkv][D]
  const __nv_bfloat16 *v;
  const int32_t *offsets;   // [B+1]
  const int32_t *lens_old;  // [B]
  const int32_t *page_table;
  int pt_stride, B, Hkv, sink, recent, num_pages;
  long long T;
  uint8_t *pool;
  uint8_t *side;
  long long page_bytes, head_bytes, side_stride;
  uint32_t *err;
  int page_kernel;          // 1: pages filled completely by this append go through append_pages_kernel
};

struct DecodeParams {
  int B, Hq, Hkv, G, sink, recent, num_pages, pt_stride, mask_stride;
  int num_workers, slot_floats, slot_o_off, int8_units;
  const __nv_bfloat16 *q;       // [B][Hq][D]
  const int32_t *seq_lens;      // [B]
  const int32_t *page_table;    // [B][pt_stride]
  const uint32_t *mask;         // nullable [B][Hkv][mask_stride]
  const uint8_t *pool;          // INT4 or bf16 pages
  const uint8_t *side;          // INT8 side blocks
  long long page_bytes, head_bytes, side_stride;
  float scale_log2;             // softmax_scale * log2(e)
  int *plan;                    // [B+1] prefix of attended INT4/bf16 page-heads
  int *first;                   // [2*B*Hkv] worker owning the first item of each range
  int *last;                    // [2*B*Hkv] worker owning the last item of each range
  float *slots;                 // [2*B*Hkv + num_workers][slot_floats] partials
  void *out;
  int out_fp32;
  uint32_t *err;
  long long wait_cap;           // 0 = simulate a copy that never lands
};

struct TopkParams {
  const float *scores;
  long long score_stride;
  const int32_t *seq_lens;
  int B, Hkv, permille, sink, recent, max_len, mask_stride;
  uint32_t *mask;
  int32_t *count;
};

// Largest batch kv4_decode_attn accepts (the per-CTA plan lives in shared memory).
constexpr int kMaxBatch = 8192;

struct DecodeLaunch {
  int smem_bytes;
  int blocks_per_sm;
};

// Launch with programmatic stream serialization: the kernel may start while
// the previous grid in the stream finishes; it calls pdl_wait() before
// touching anything that grid produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

cudaError_t launch_append(const AppendParams &p, int D, cudaStream_t stream);
cudaError_t decode_prepare(int D, int G, bool bf16, DecodeLaunch *out);
int decode_smem_bytes(int D, bool bf16, int B);
cudaError_t launch_decode(const DecodeParams &p, int D, bool bf16, cudaStream_t stream, cudaEvent_t ev0,
                          cudaEvent_t ev1);
cudaError_t launch_topk(const TopkParams &p, cudaStream_t stream);
// Exact merge of the decode partials (np8 = INT8 side pages per (sequence, head)).
cudaError_t launch_merge(const DecodeParams &p, int D, int np8, cudaStream_t stream);

}  // namespace kv4
