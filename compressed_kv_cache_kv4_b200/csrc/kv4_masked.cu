// kv4_masked.cu -- decode attention under a retained-position mask with the
// work and the bytes of the INT4 region following the retained count.
//
// Shadow Mask Distillation, sec. 1 and Figure 1: eviction is recorded as a
// binary mask that attention applies instead of slicing the cache. KV4-RL
// review, sec. 3: the INT4 region and the INT8 region are attended separately
// and merged exactly.
//
// A mask keeps positions scattered over almost every page (an H2O-style
// top-10% keeps a row in about four of five (page, head) blocks), so skipping
// whole pages saves nothing, and the decode kernel's work per page does not
// shrink with the rows it keeps. The gather below packs the retained rows of
// the INT4 region of every (sequence, KV head), in position order, into dense
// pages of the ordinary layout (a "compact" cache): K rows and their scales
// are copied whole, a V row's nibbles are moved byte by byte between the
// fragment positions of its source row and of its compact row (a byte holds
// the two nibbles of one row). The ordinary decode kernel then attends the
// compact pages (INT4 only, a mask marking each head's valid rows), the INT8
// region is attended from the original side cache, and the two partials are
// merged. Rows past a head's count in its last compact pages are zero, so
// they are finite and masked out.
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
// INT4-region positions per mask word, the row's count (capped at
// max_retained), the compact length of its sequence (max over heads) and the
// sequence's compact page-table row.
__global__ void __launch_bounds__(256) masked_count_kernel(GatherParams p) {
  __shared__ int wsum[8];
  __shared__ int carry_sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x, b = row / p.Hkv, h = row - b * p.Hkv;
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
    atomicMax(&p.lens_c[b], n);
  }
  if (h == 0)
    for (int j = tid; j < p.PPS; j += 256) p.pt_c[(long long)b * p.PPS + j] = b * p.PPS + j;
}

// One CTA per (sequence, KV head). The row's retained positions are listed in
// shared memory, kChunk at a time, straight from the prefix counts (each
// thread places the positions of its mask words). A warp then assembles one
// compact page of the head at a time: lanes i and i + 16 fetch the two halves
// of row i's data (K codes, K or V scales, and the 16-byte pieces of the V
// block that hold the row's bytes) with all loads in flight together, place
// them at row i of the page image in shared memory, and the warp writes the
// image out. Compact pages past the row's count are written as zeros.
constexpr int kGatherThreads = 512, kGatherChunk = 4096;

template <int D>
__global__ void __launch_bounds__(kGatherThreads) masked_gather_kernel(GatherParams p) {
  constexpr int WARPS = kGatherThreads / 32, HEAD = 18 * D, KROW = D / 2, NP = D / 16;   // NP: V pieces per half row
  extern __shared__ __align__(16) uint8_t gsm[];
  int *list = reinterpret_cast<int *>(gsm);                           // [kGatherChunk]
  uint8_t *img_all = gsm + 4 * kGatherChunk;                          // [WARPS][HEAD]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x, b = row / p.Hkv, h = row - b * p.Hkv;
  int L, c0, c1;
  region(p, b, L, c0, c1);
  const int n = p.counts[row];
  const int npg = (p.lens_c[b] + kPageTokens - 1) / kPageTokens;   // compact pages of the sequence
  const uint32_t *mrow = p.mask + (long long)row * p.mask_stride;
  const int *wpre = p.wpre + (long long)row * p.words;
  const int nw = (L + 31) / 32;
  uint8_t *im = img_all + warp * HEAD;
  const int i = lane & 15, half = lane >> 4;
  for (int t0 = 0; t0 < npg * kPageTokens; t0 += kGatherChunk) {
    const int t1 = min(t0 + kGatherChunk, n);
    __syncthreads();   // the previous chunk's list is no longer read
    for (int w = tid; w < nw; w += kGatherThreads) {
      const int hi_ = wpre[w], lo_ = w > 0 ? wpre[w - 1] : 0;   // retained indices [lo_, hi_) lie in word w
      if (hi_ <= t0 || lo_ >= t1) continue;
      uint32_t bits = mrow[w] & in_range(w, c0, c1);
      for (int k = lo_; bits; ++k) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        if (k >= t0 && k < t1) list[k - t0] = 32 * w + bit;
      }
    }
    __syncthreads();
    const int pg_end = min(npg, (t0 + kGatherChunk) / kPageTokens);
    for (int j = t0 / kPageTokens + warp; j < pg_end; j += WARPS) {
      for (int q = lane; q < HEAD / 16; q += 32) reinterpret_cast<uint4 *>(im)[q] = make_uint4(0, 0, 0, 0);
      const int t = kPageTokens * j + i;
      int page = -1, r = 0;
      if (t < n) {
        const int pos = list[t - t0];
        r = pos % kPageTokens;
        page = p.page_table[(long long)b * p.pt_stride + pos / kPageTokens];
        if (page < 0 || page >= p.num_pages) {
          if (half == 0) set_error(p.err, kErrBounds);
          page = -1;   // the row stays zero
        }
      }
      __syncwarp();
      if (page >= 0) {
        const uint8_t *src = p.pool + (long long)page * p.page_bytes + (long long)h * p.head_bytes;
        // K codes: this lane's half of the row (D/4 bytes)
        uint4 kc[D / 64];
#pragma unroll
        for (int u = 0; u < D / 64; ++u)
          kc[u] = __ldg(reinterpret_cast<const uint4 *>(src + r * KROW + half * (KROW / 2)) + u);
        // K scales (half 0) or V scales (half 1): D/16 bytes
        const int sb = half ? 17 * D : 16 * D;
        uint2 sc = make_uint2(0, 0);
        if constexpr (D == 128) sc = __ldg(reinterpret_cast<const uint2 *>(src + sb + r * (D / 16)));
        else sc.x = __ldg(reinterpret_cast<const uint32_t *>(src + sb + r * (D / 16)));
        // V: the 16-byte pieces (m/4, dm8) holding the row's bytes: word
        // (m/4)*128 + 4*(4*dm8 + (r%8)/2) + m%4 has the row's byte 2*(r%2) + r/8.
        // D = 128: this half takes m/4 = half (8 pieces); D = 64: dm8 in [4 half, 4 half + 4)
        uint4 vp[NP];
#pragma unroll
        for (int u = 0; u < NP; ++u) {
          const int m4 = D == 128 ? half : 0, dm8 = D == 128 ? u : 4 * half + u;
          vp[u] = __ldg(reinterpret_cast<const uint4 *>(src + 8 * D + 16 * (m4 * 32 + 4 * dm8 + (r % 8) / 2)));
        }
#pragma unroll
        for (int u = 0; u < D / 64; ++u)
          reinterpret_cast<uint4 *>(im + i * KROW + half * (KROW / 2))[u] = kc[u];
        if constexpr (D == 128) *reinterpret_cast<uint2 *>(im + sb + i * (D / 16)) = sc;
        else *reinterpret_cast<uint32_t *>(im + sb + i * (D / 16)) = sc.x;
        const int sh_src = 8 * (2 * (r % 2) + r / 8), b_dst = 2 * (i % 2) + i / 8;
#pragma unroll
        for (int u = 0; u < NP; ++u) {
          const int m4 = D == 128 ? half : 0, dm8 = D == 128 ? u : 4 * half + u;
          uint8_t *dst = im + 8 * D + 16 * (m4 * 32 + 4 * dm8 + (i % 8) / 2) + b_dst;
          dst[0] = static_cast<uint8_t>(vp[u].x >> sh_src);
          dst[4] = static_cast<uint8_t>(vp[u].y >> sh_src);
          dst[8] = static_cast<uint8_t>(vp[u].z >> sh_src);
          dst[12] = static_cast<uint8_t>(vp[u].w >> sh_src);
        }
      }
      __syncwarp();
      uint4 *dst = reinterpret_cast<uint4 *>(p.pool_c + ((long long)b * p.PPS + j) * p.page_bytes +
                                             (long long)h * p.head_bytes);
      for (int q = lane; q < HEAD / 16; q += 32) dst[q] = reinterpret_cast<const uint4 *>(im)[q];
      __syncwarp();
    }
  }
  uint32_t *mc = p.mask_c + (long long)row * p.mask_stride_c;
  for (int w = tid; w < p.mask_stride_c; w += kGatherThreads) mc[w] = in_range(w, 0, n);
}

cudaError_t launch_masked_gather(const GatherParams &p, int D, cudaStream_t stream) {
  const int rows = p.B * p.Hkv;
  if (rows == 0) return cudaSuccess;
  cudaError_t e = launch_pdl(masked_count_kernel, dim3(rows), dim3(256), 0, stream, p);
  if (e != cudaSuccess) return e;
  const size_t smem = 4 * kGatherChunk + (size_t)(kGatherThreads / 32) * 18 * D;
  auto kern = D == 128 ? masked_gather_kernel<128> : masked_gather_kernel<64>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(rows), dim3(kGatherThreads), smem, stream, p);
}

}  // namespace kv4
