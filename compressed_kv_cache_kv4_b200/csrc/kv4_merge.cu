// kv4_merge.cu -- exact softmax merge of the decode kernel's partials.
//
// KV4-RL review, sec. 3: the INT4 and INT8 regions are attended separately and
// their (max, sum, output) partials are joined by an exact softmax merge. For
// partials (m_c, l_c, o_c) of one (sequence, query head), m in log2 units and
// o already divided by l:
//   M = max_c m_c,  W_c = l_c 2^(m_c - M),  out = sum_c W_c o_c / sum_c W_c,
// and out = 0 when every partial is empty (l_c = 0).
//
// One warp per (sequence b, query head hq); lane k owns output elements
// [k D/32, (k+1) D/32). The decode kernels record, per range of the work
// space (KV4: a region of a virtual sequence, all heads of its block; bf16: a
// (sequence, KV head)), the first and last worker whose segment touched it;
// the partial of worker w sits in slot (range index + w) * (heads per range)
// + head. Workers between the first and the last wrote a partial for the
// range (an empty one, l = 0, if nothing of it was attended). Every lane loads (m, l) and its
// slice of o for a batch of up to kBatch partials at once, so a batch costs a
// single round trip to L2 (the partials were written moments ago by other SMs;
// all loads bypass L1).
#include <math.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

namespace {

constexpr int kBatch = 8;

template <int DPL>
struct Vec;
template <>
struct Vec<4> {
  static __device__ __forceinline__ void load(const float *src, float (&v)[4]) {
    const float4 x = __ldcg(reinterpret_cast<const float4 *>(src));
    v[0] = x.x;
    v[1] = x.y;
    v[2] = x.z;
    v[3] = x.w;
  }
};
template <>
struct Vec<2> {
  static __device__ __forceinline__ void load(const float *src, float (&v)[2]) {
    const float2 x = __ldcg(reinterpret_cast<const float2 *>(src));
    v[0] = x.x;
    v[1] = x.y;
  }
};

}  // namespace

template <int D, int G, bool kKv4>
__global__ void __launch_bounds__(128) merge_kernel(DecodeParams p) {
  constexpr int DPL = D / 32;
  const long long task = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();                 // the worker grid has finished and its writes are visible
  pdl_launch_dependents();
  if (task >= (long long)p.B * p.Hq) return;
  const int b = static_cast<int>(task / p.Hq), hq = static_cast<int>(task % p.Hq);
  const int h = hq / G, g = hq % G;
  // Ranges of this query head and their slots; the partial of worker w for
  // range r sits in slot (r + w) * HB + hh.
  //   KV4: v = virtual sequence hb * B + b (hh = head within the block), its
  //        INT8 range 2v and INT4 range 2v + 1; plan[v] = first item of v
  //        (n8 INT8 items, then its INT4 pages); workers = CTAs.
  //   bf16: v = b * Hkv + h, HB = 1; one range B * Hkv + v; plan[b] = first
  //        page-head of sequence b; workers = warps.
  int HB, hh;
  long long r8, r4, nw;
  bool has8, has4;
  if constexpr (kKv4) {
    HB = p.HB;
    const int hb = h / HB;
    hh = h - hb * HB;
    const int v = hb * p.B + b;
    const int n8 = p.int8_units ? 2 * p.np8 : 0;
    const long long T = __ldcg(&p.plan[p.NVB]);
    const int pb0 = __ldcg(&p.plan[v]), pb1 = __ldcg(&p.plan[v + 1]);
    nw = T > 0 ? min((long long)p.n_cta, max(1LL, T >> 1)) : 0;   // CTAs that took part
    r8 = 2LL * v;
    r4 = 2LL * v + 1;
    has8 = n8 > 0;
    has4 = pb1 - pb0 > n8;
  } else {
    HB = 1;
    hh = 0;
    const long long T4 = __ldcg(&p.plan[p.B]);
    const int pb0 = __ldcg(&p.plan[b]), pb1 = __ldcg(&p.plan[b + 1]);
    nw = active_workers(p.num_workers, 0, T4);
    r8 = 0;
    r4 = (long long)p.B * p.Hkv + (long long)b * p.Hkv + h;
    has8 = false;
    has4 = pb1 > pb0;
  }
  const int f8 = has8 ? __ldcg(&p.first[r8]) : -1, l8 = has8 ? __ldcg(&p.last[r8]) : -1;
  const int f4 = has4 ? __ldcg(&p.first[r4]) : -1, l4 = has4 ? __ldcg(&p.last[r4]) : -1;
  // A range is used only if it has items; bounds outside [0, nw) (possible only
  // after a worker stopped on an error) drop the range instead of being read.
  const bool ok8 = has8 && f8 >= 0 && f8 <= l8 && l8 < nw;
  const bool ok4 = has4 && f4 >= 0 && f4 <= l4 && l4 < nw;
  const int n8r = ok8 ? l8 - f8 + 1 : 0;
  const int n = n8r + (ok4 ? l4 - f4 + 1 : 0);

  float M = -INFINITY, den = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int c0 = 0; c0 < n; c0 += kBatch) {
    float mk[kBatch], lk[kBatch], ok[kBatch][DPL];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int i = c0 + k;
      mk[k] = -INFINITY;
      lk[k] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) ok[k][e] = 0.f;
      if (i < n) {
        const long long w = i < n8r ? f8 + i : f4 + (i - n8r);
        const float *slot = p.slots + (((i < n8r ? r8 : r4) + w) * HB + hh) * p.slot_floats;
        mk[k] = __ldcg(slot + g);
        lk[k] = __ldcg(slot + G + g);
        Vec<DPL>::load(slot + p.slot_o_off + g * D + lane * DPL, ok[k]);
      }
    }
    float mc = -INFINITY;
#pragma unroll
    for (int k = 0; k < kBatch; ++k)
      if (lk[k] > 0.f) mc = fmaxf(mc, mk[k]);
    if (mc > M) {
      const float f = ex2(M - mc);
      den *= f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] *= f;
      M = mc;
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (!(lk[k] > 0.f)) continue;
      const float wk = lk[k] * ex2(mk[k] - M);
      den += wk;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wk, ok[k][e], acc[e]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  if (p.partials) {
    // the merged partial of this call, for a merge with other shards' partials:
    // m (log2 units), l, two pad words, o (normalised)
    float *pr = p.partials + ((long long)b * p.Hq + hq) * (D + 4);
    if (lane == 0) *reinterpret_cast<float4 *>(pr) = make_float4(den > 0.f ? M : -INFINITY, den, 0.f, 0.f);
#pragma unroll
    for (int e = 0; e < DPL; ++e) pr[4 + lane * DPL + e] = acc[e] * inv;
    return;
  }
  const long long obase = ((long long)b * p.Hq + hq) * D + lane * DPL;
  if (p.out_fp32) {
    float *o = reinterpret_cast<float *>(p.out) + obase;
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4 *>(o) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    } else {
      *reinterpret_cast<float2 *>(o) = make_float2(acc[0] * inv, acc[1] * inv);
    }
  } else {
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.out) + obase;
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2 *>(o) =
          make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    } else {
      *reinterpret_cast<uint32_t *>(o) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
  }
}

template <int D, bool kKv4>
static cudaError_t launch_merge_d(const DecodeParams &p, cudaStream_t stream) {
  const long long warps = (long long)p.B * p.Hq;
  if (warps == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((warps + 3) / 4);
  switch (p.G) {
    case 1: return launch_pdl(merge_kernel<D, 1, kKv4>, dim3(blocks), dim3(128), 0, stream, p);
    case 2: return launch_pdl(merge_kernel<D, 2, kKv4>, dim3(blocks), dim3(128), 0, stream, p);
    default: return launch_pdl(merge_kernel<D, 4, kKv4>, dim3(blocks), dim3(128), 0, stream, p);
  }
}

// ---------------------------------------------------------------------------
// Merge of N gathered partials [N][rows][D+4] (m, l, pad, pad, o) into the
// final output: the same exact merge, one warp per row, shards in order.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) merge_partials_kernel(const float *partials, int N, long long rows, void *out,
                                                             int out_fp32) {
  constexpr int DPL = D / 32;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  if (row >= rows) return;
  float M = -INFINITY, den = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  for (int c0 = 0; c0 < N; c0 += kBatch) {
    float mk[kBatch], lk[kBatch], ok[kBatch][DPL];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      mk[k] = -INFINITY;
      lk[k] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) ok[k][e] = 0.f;
      if (c0 + k < N) {
        const float *pr = partials + ((long long)(c0 + k) * rows + row) * (D + 4);
        mk[k] = pr[0];
        lk[k] = pr[1];
        Vec<DPL>::load(pr + 4 + lane * DPL, ok[k]);
      }
    }
    float mc = -INFINITY;
#pragma unroll
    for (int k = 0; k < kBatch; ++k)
      if (lk[k] > 0.f) mc = fmaxf(mc, mk[k]);
    if (mc > M) {
      const float f = ex2(M - mc);
      den *= f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] *= f;
      M = mc;
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (!(lk[k] > 0.f)) continue;
      const float wk = lk[k] * ex2(mk[k] - M);
      den += wk;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wk, ok[k][e], acc[e]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const long long obase = row * D + lane * DPL;
  if (out_fp32) {
    float *o = reinterpret_cast<float *>(out) + obase;
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[e] = acc[e] * inv;
  } else {
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(out) + obase;
#pragma unroll
    for (int e = 0; e < DPL; e += 2) *reinterpret_cast<uint32_t *>(o + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  }
}

cudaError_t launch_merge_partials(const float *partials, int N, long long rows, int D, void *out, int out_fp32,
                                  cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((rows + 3) / 4);
  if (D == 128)
    return launch_pdl(merge_partials_kernel<128>, dim3(blocks), dim3(128), 0, stream, partials, N, rows, out, out_fp32);
  return launch_pdl(merge_partials_kernel<64>, dim3(blocks), dim3(128), 0, stream, partials, N, rows, out, out_fp32);
}

cudaError_t launch_merge(const DecodeParams &p, int D, bool bf16, cudaStream_t stream) {
  if (bf16) return D == 128 ? launch_merge_d<128, false>(p, stream) : launch_merge_d<64, false>(p, stream);
  return D == 128 ? launch_merge_d<128, true>(p, stream) : launch_merge_d<64, true>(p, stream);
}

}  // namespace kv4
