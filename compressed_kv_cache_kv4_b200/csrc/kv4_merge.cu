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
// [k D/32, (k+1) D/32). The decode kernel records, per (region, sequence, KV
// head) range, the first and last worker whose segment touched it; partial c
// of worker w sits in slot (range index + w). Every lane loads (m, l) and its
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

template <int D, int G>
__global__ void __launch_bounds__(128) merge_kernel(DecodeParams p, int np8) {
  constexpr int DPL = D / 32;
  const long long task = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  pdl_wait();                 // the worker grid has finished and its writes are visible
  pdl_launch_dependents();
  if (task >= (long long)p.B * p.Hq) return;
  const int b = static_cast<int>(task / p.Hq), hq = static_cast<int>(task % p.Hq);
  const int h = hq / G, g = hq % G;
  const long long nbh = (long long)p.B * p.Hkv, r = (long long)b * p.Hkv + h;

  // Range bounds and the plan entries, all independent loads.
  const int pb0 = __ldcg(&p.plan[b]), pb1 = __ldcg(&p.plan[b + 1]);
  const long long T4 = __ldcg(&p.plan[p.B]);
  const int f8 = __ldcg(&p.first[r]), l8 = __ldcg(&p.last[r]);
  const int f4 = __ldcg(&p.first[nbh + r]), l4 = __ldcg(&p.last[nbh + r]);
  const long long T8 = nbh * np8;
  // the decode kernel's worker count; every one of them owns at least one item
  const long long nw = active_workers(p.num_workers, T8, T4);
  // A range is used only if it has items; bounds outside [0, nw) (possible only
  // after a worker stopped on an error) drop the range instead of being read.
  const bool ok8 = np8 > 0 && f8 >= 0 && f8 <= l8 && l8 < nw;
  const bool ok4 = pb1 > pb0 && f4 >= 0 && f4 <= l4 && l4 < nw;
  const int n8 = ok8 ? l8 - f8 + 1 : 0;
  const int n = n8 + (ok4 ? l4 - f4 + 1 : 0);

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
        const long long w = i < n8 ? f8 + i : f4 + (i - n8);
        const float *slot = p.slots + ((i < n8 ? r : nbh + r) + w) * p.slot_floats;
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

template <int D>
static cudaError_t launch_merge_d(const DecodeParams &p, int np8, cudaStream_t stream) {
  const long long warps = (long long)p.B * p.Hq;
  if (warps == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((warps + 3) / 4);
  switch (p.G) {
    case 1: return launch_pdl(merge_kernel<D, 1>, dim3(blocks), dim3(128), 0, stream, p, np8);
    case 2: return launch_pdl(merge_kernel<D, 2>, dim3(blocks), dim3(128), 0, stream, p, np8);
    default: return launch_pdl(merge_kernel<D, 4>, dim3(blocks), dim3(128), 0, stream, p, np8);
  }
}

cudaError_t launch_merge(const DecodeParams &p, int D, int np8, cudaStream_t stream) {
  return D == 128 ? launch_merge_d<128>(p, np8, stream) : launch_merge_d<64>(p, np8, stream);
}

}  // namespace kv4
