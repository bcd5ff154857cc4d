// kv4_evict.h -- parameter block and launcher of the page-eviction kernel.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kv4 {

struct EvictParams {
  const float *scores;          // [B][Hkv][score_stride]
  long long score_stride;
  int32_t *seq_lens;            // [B], rewritten
  int32_t *page_table;          // [B][pt_stride], rewritten
  int32_t *freed;               // [B][pt_stride], evicted ids first
  int32_t *freed_count;         // [B]
  int pt_stride, B, Hkv, permille, sink, recent;
  uint8_t *side;                // INT8 side blocks, ring pages rotated in place
  long long side_stride, side_page_bytes;
  uint32_t *err;
};

// Ring pages per (sequence, head) at most (recent <= 128).
constexpr int kMaxRingPages = 8;
// Longest page-table row kv4_evict_pages accepts (its keys and the staged row
// live in shared memory).
constexpr int kEvictMaxPages = 16384;

size_t evict_smem_bytes(int pt_stride);
cudaError_t launch_evict(const EvictParams &p, bool vec, cudaStream_t stream);

}  // namespace kv4
