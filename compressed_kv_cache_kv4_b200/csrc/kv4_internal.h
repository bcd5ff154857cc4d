// kv4_internal.h -- kernel parameter blocks and launchers inside libkv4.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

struct kv4_cache;

namespace kv4 {

// Device a kv4_cache was created on (-1 for NULL).
int cache_device(const kv4_cache *cache);

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
  int num_sms;              // SMs of the device (grid of the page kernel)
};

struct DecodeParams {
  int B, Hq, Hkv, G, sink, recent, num_pages, pt_stride, mask_stride;
  int num_workers, slot_floats, slot_o_off, int8_units;
  // KV4 kernel: HB warps (KV heads) per CTA, NVB = B * Hkv / HB virtual
  // sequences, NS ring stages, np8 side pages per (sequence, head), n_cta CTAs
  int HB, NVB, NS, np8, n_cta;
  const __nv_bfloat16 *q;       // [B][Hq][D]
  const int32_t *seq_lens;      // [B]
  const int32_t *page_table;    // [B][pt_stride]
  const uint32_t *mask;         // nullable [B][Hkv][mask_stride]
  const uint8_t *pool;          // INT4 or bf16 pages
  const uint8_t *side;          // INT8 side blocks
  long long page_bytes, head_bytes, side_stride;
  float scale_log2;             // softmax_scale * log2(e)
  // KV4: plan [NVB+1] (INT4 pages before each virtual sequence), first/last
  // CTA of each (region, virtual sequence) range [2*NVB], partial slots
  // [2*NVB + n_cta][HB][slot_floats]. bf16: plan [B+1] (page-heads before
  // each sequence), first/last warp of each (sequence, head) range [2*B*Hkv],
  // slots [2*B*Hkv + num_workers][slot_floats].
  int *plan;
  int *first;
  int *last;
  float *slots;
  void *out;
  int out_fp32;
  // page-range shard of every sequence (nullable, KV4 only): INT4 pages
  // [page_begin[b], page_end[b]) of the INT4 region are attended
  const int32_t *page_begin;
  const int32_t *page_end;
  float *partials;              // non-null: the merge writes (m, l, o) partials [B][Hq][D+4] instead of out
  uint32_t *err;
  long long wait_cap;           // 0 = simulate a copy that never lands
};

struct TopkParams {
  const float *scores;
  long long score_stride;
  const int32_t *seq_lens;
  int B, Hkv, permille, sink, recent, max_len, mask_stride;
  int vec_ok;                   // scores 16-byte aligned and score_stride % 4 == 0
  uint32_t *mask;
  int32_t *count;
};

// Largest batch kv4_decode_attn accepts (the per-CTA plan lives in shared
// memory; item descriptors hold a virtual sequence in 13 bits).
constexpr int kMaxBatch = 8192;
// Largest page-table row of the KV4 kernel (page index in 17 bits).
constexpr int kMaxPtStride = 1 << 17;

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
// KV4 kernel: raise its dynamic shared-memory limit on the current device;
// resident CTAs per SM at HB warps and `smem` bytes per CTA.
cudaError_t kv4_decode_set_smem_limit(int D, int G, int smem);
cudaError_t kv4_decode_occupancy(int D, int G, int HB, int smem, int *blocks_per_sm);
int kv4_smem_bytes(int D, int HB, int NS, int NVB);
cudaError_t bf16_decode_prepare(int D, int G, DecodeLaunch *out);
int bf16_smem_bytes(int D, int B);
cudaError_t launch_decode(const DecodeParams &p, int D, bool bf16, cudaStream_t stream, cudaEvent_t ev0,
                          cudaEvent_t ev1);
cudaError_t launch_topk(const TopkParams &p, cudaStream_t stream);

// Masked decode with the retained rows gathered on chip (kv4_masked.cu counts,
// kv4_decode.cu gathers and attends).
struct GatherParams {
  const uint32_t *mask;         // [B][Hkv][mask_stride]
  const int32_t *seq_lens;      // [B]
  int B, Hkv, sink, recent, pt_stride, mask_stride;
  int max_retained;             // rows attended per (sequence, head), at most
  int words;                    // prefix entries per row: ceil(pt_stride * 16 / 32)
  int *wpre;                    // [B][Hkv][words] inclusive retained counts per mask word
  int *counts;                  // [B][Hkv]
  uint32_t *err;
};
// Counts and per-word prefix counts of the retained INT4-region rows.
cudaError_t launch_masked_count(const GatherParams &p, cudaStream_t stream);
// Gathered masked decode of the INT4 region: one partial per warp into
// parts [masked_decode_warps()][B][Hq][D+4] (the layout of kv4_decode_partials).
cudaError_t launch_masked_decode(const DecodeParams &p, const GatherParams &g, float *parts, int D,
                                 cudaStream_t stream);
int masked_decode_warps();
// Exact merge of the decode partials of kv4_decode_kernel or bf16_decode_kernel.
cudaError_t launch_merge(const DecodeParams &p, int D, bool bf16, cudaStream_t stream);
// Exact merge of N gathered (m, l, o) partials [N][rows][D+4] into out [rows][D].
cudaError_t launch_merge_partials(const float *partials, int N, long long rows, int D, void *out, int out_fp32,
                                  cudaStream_t stream);

}  // namespace kv4
