// kv4_masked.cu -- counting pass of the masked decode with gathered rows.
//
// Shadow Mask Distillation, sec. 1 and Figure 1: eviction is recorded as a
// binary mask that attention applies instead of slicing the cache.
//
// A mask keeps positions scattered over almost every page (an H2O-style
// top-10% keeps a row in about four of five (page, head) blocks), so skipping
// whole pages saves almost nothing, and the page kernel's work per page does
// not shrink with the rows it keeps. masked_decode_kernel (kv4_decode.cu)
// therefore gathers the retained rows of each (sequence, KV head) into dense
// 16-row pages on chip; this kernel counts them and gives every mask word the
// number of retained positions up to and including it, so that the gathering
// CTA can list its positions without a search.
#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

namespace {

__device__ __forceinline__ void region(const GatherParams &p, int b, int &L, int &c0, int &c1) {
  L = p.seq_lens[b];
  const int cap = p.pt_stride * kPageTokens;
  L = L < 0 ? 0 : (L > cap ? cap : L);
  c0 = min(p.sink, L);
  c1 = max(c0, L - p.recent);
}

// Bits of mask word w that lie in [c0, c1).
__device__ __forceinline__ uint32_t in_range(int w, int c0, int c1) {
  const int a = max(c0 - 32 * w, 0), z = min(c1 - 32 * w, 32);
  if (z <= a) return 0u;
  return (z >= 32 ? 0xFFFFFFFFu : ((1u << z) - 1u)) & ~((1u << a) - 1u);
}

}  // namespace

// One CTA per (sequence, KV head): inclusive prefix counts of the retained
// INT4-region positions per mask word and the row's count (capped at
// max_retained, which is reported).
__global__ void __launch_bounds__(256) masked_count_kernel(GatherParams p) {
  __shared__ int wsum[8];
  __shared__ int carry_sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x, b = row / p.Hkv;
  int L, c0, c1;
  region(p, b, L, c0, c1);
  const uint32_t *mrow = p.mask + (long long)row * p.mask_stride;
  int *wpre = p.wpre + (long long)row * p.words;
  const int nw = (L + 31) / 32;
  if (tid == 0) carry_sh = 0;
  __syncthreads();
  for (int w0 = 0; w0 < nw; w0 += 256) {
    const int w = w0 + tid;
    const int v = w < nw ? __popc(mrow[w] & in_range(w, c0, c1)) : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int off = carry_sh;
    for (int k = 0; k < warp; ++k) off += wsum[k];
    if (w < nw) wpre[w] = off + incl;
    __syncthreads();
    if (tid == 255) carry_sh = off + incl;
    __syncthreads();
  }
  if (tid == 0) {
    int n = carry_sh;
    if (n > p.max_retained) {
      n = p.max_retained;
      set_error(p.err, kErrCapacity);
    }
    p.counts[row] = n;
  }
}

cudaError_t launch_masked_count(const GatherParams &p, cudaStream_t stream) {
  if (p.B * p.Hkv == 0) return cudaSuccess;
  return launch_pdl(masked_count_kernel, dim3(p.B * p.Hkv), dim3(256), 0, stream, p);
}

}  // namespace kv4
