// kv_topk.cu -- per (sequence, KV head) retained-position mask.
//
// KVP promo (arXiv 2602.10238), core mechanism, and TTKV promo (arXiv
// 2604.19769), insight 1: eviction is ranking -- score each position, sort,
// truncate at the budget; one ranking per attention head serves every budget.
// KV4-RL review, sec. 3: the first 16 and the last 128 positions are always
// kept. Shadow Mask Distillation, sec. 1: the result is a binary mask.
//
// One CTA per row. Scores become order-preserving 32-bit keys (larger score ->
// larger key, -0 folded into +0). A 3-pass radix select with 11-, 11- and
// 10-bit digits finds the key T of the k-th best non-forced position in O(L)
// work; positions with key > T are kept, and among keys == T the lowest
// indices fill the remainder (a scan over 32-position tiles gives each tie its
// rank in index order). The first digit covers the sign, the exponent and the
// top two mantissa bits, so scores that share an exponent still spread over
// four bins and scores of one magnitude class do not pile onto a handful of
// shared-memory counters. The forced positions are two contiguous ranges, so
// the passes run over the candidate range between them only, four keys per
// thread step. The row is held in shared memory when it fits, otherwise re-read
// from global memory on each pass.
#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

constexpr int kTopkThreads = 512;
constexpr int kTopkBins = 2048;            // 4 bins per thread in the scan
constexpr int kTopkSmemKeys = 49152;   // rows up to this length are staged in shared memory

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Keys of candidate positions [c0, c1) in steps of four per thread: f(i, key)
// for each. With the row in shared memory four keys come from one 16-byte load
// (c0 rounded down to a multiple of four); only the first and the last step
// of the range test each index, the steps between hold four candidates.
template <bool kSmem, typename F>
__device__ __forceinline__ void for_candidates(const uint32_t *keys, const float *srow, int c0, int c1, int tid,
                                               F &&f) {
  const int base = c0 & ~3;
  const int lo = (c0 + 3) & ~3, hi = c1 & ~3;   // [lo, hi): whole steps inside [c0, c1)
  for (int i = base + 4 * tid; i < c1; i += 4 * kTopkThreads) {
    uint32_t k[4];
    if constexpr (kSmem) {
      const uint4 v = *reinterpret_cast<const uint4 *>(keys + i);
      k[0] = v.x;
      k[1] = v.y;
      k[2] = v.z;
      k[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) k[e] = i + e < c1 ? score_key(srow[i + e]) : 0u;
    }
    if (i >= lo && i < hi) {
#pragma unroll
      for (int e = 0; e < 4; ++e) f(i + e, k[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (i + e >= c0 && i + e < c1) f(i + e, k[e]);
    }
  }
}

template <bool kSmem>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint32_t dyn[];
  __shared__ uint32_t hist[kTopkBins];
  __shared__ int wsum[kTopkThreads / 32];
  __shared__ int sh_digit, sh_rem, sh_cnt;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NWARP = kTopkThreads / 32;
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x;
  const int b = row / p.Hkv;
  int L = p.seq_lens[b];
  L = L < 0 ? 0 : (L > p.max_len ? p.max_len : L);
  const float *srow = p.scores + (long long)row * p.score_stride;
  const int S = p.sink, R = p.recent;
  const int nt = (L + 31) / 32;
  // keys [round_up(max_len, 4)] when staged, then the tile ranks [nt]
  uint32_t *keys = dyn;
  int *tile_rank = reinterpret_cast<int *>(dyn + (kSmem ? (p.max_len + 3) / 4 * 4 : 0));

  // forced positions are [0, min(S, L)) and [max(S, L - R), L); the candidates
  // are the positions between them
  const int c0 = min(S, L), c1 = max(c0, L - R);
  auto forced = [&](int pos) { return pos < c0 || pos >= c1; };
  const int nF = L - (c1 - c0);
  const long long kb = (long long)L * p.permille / 1000;
  long long ksel = kb - nF;
  if (ksel < 0) ksel = 0;
  if (ksel > c1 - c0) ksel = c1 - c0;

  // mode: 0 = select none, 1 = select all, 2 = threshold
  const int mode = ksel == 0 ? 0 : (ksel == c1 - c0 ? 1 : 2);
  if (kSmem && mode == 2) {
    const int base = c0 & ~3;
    if (p.vec_ok) {
      // 16-byte loads: the row starts 16-byte aligned and its stride is a
      // multiple of four, so the last vector ends inside the row's storage
      for (int i = base + 4 * tid; i < c1; i += 4 * kTopkThreads) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(srow + i));
        *reinterpret_cast<uint4 *>(keys + i) =
            make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
      }
    } else {
      for (int i = base + tid; i < c1; i += kTopkThreads) keys[i] = score_key(srow[i]);
    }
  }
  __syncthreads();

  uint32_t T = 0;
  int need_eq = 0;
  bool ties = false;
  if (mode == 2) {
    uint32_t prefix = 0, pmask = 0;
    int rem = static_cast<int>(ksel);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const uint32_t dmask = pass == 2 ? 1023u : 2047u;
      for (int i = tid; i < kTopkBins; i += kTopkThreads) hist[i] = 0;
      __syncthreads();
      if (pass == 0) {
        for_candidates<kSmem>(keys, srow, c0, c1, tid,
                              [&](int, uint32_t k) { atomicAdd(&hist[k >> shift], 1u); });
      } else {
        for_candidates<kSmem>(keys, srow, c0, c1, tid, [&](int, uint32_t k) {
          if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & dmask], 1u);
        });
      }
      __syncthreads();
      // thread i owns bins kTopkBins-1-4i .. kTopkBins-4-4i (highest first):
      // block-wide exclusive scan of the per-thread counts from the top
      int cnt[4], tot = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cnt[j] = hist[kTopkBins - 1 - 4 * tid - j];
        tot += cnt[j];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      int c = incl - tot;
      for (int w = 0; w < warp; ++w) c += wsum[w];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (c < rem && rem <= c + cnt[j]) {
          sh_digit = kTopkBins - 1 - 4 * tid - j;
          sh_rem = rem - c;
          sh_cnt = cnt[j];
        }
        c += cnt[j];
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(sh_digit) << shift;
      pmask |= dmask << shift;
      rem = sh_rem;
      __syncthreads();
    }
    T = prefix;
    need_eq = rem;
    // sh_cnt = keys equal to T; ranks among them are needed only when some of
    // them stay out: count per 32-position tile, then scan
    ties = need_eq < sh_cnt;
    if (ties) {
      for (int w = warp; w < nt; w += NWARP) {
        const int pos = 32 * w + lane;
        const bool eq = pos >= c0 && pos < c1 && (kSmem ? keys[pos] : score_key(srow[pos])) == T;
        const uint32_t bal = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) tile_rank[w] = __popc(bal);
      }
      __syncthreads();
      if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < nt; base += 32) {
          const int w = base + lane;
          const int v = w < nt ? tile_rank[w] : 0;
          int incl = v;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          if (w < nt) tile_rank[w] = carry + incl - v;
          carry += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
      __syncthreads();
    }
  }

  // mask words: a warp builds 32 consecutive words (lane i keeps word i) and
  // stores them together
  uint32_t *mrow = p.mask + (long long)row * p.mask_stride;
  for (int w0 = 32 * warp; w0 < nt; w0 += 32 * NWARP) {
    uint32_t mine = 0;
    const int n = min(32, nt - w0);
    for (int i = 0; i < n; ++i) {
      const int w = w0 + i;
      const int pos = 32 * w + lane;
      bool sel = pos < L && (forced(pos) || mode == 1);
      if (mode == 2) {
        const bool cand = pos >= c0 && pos < c1;
        const uint32_t k = cand ? (kSmem ? keys[pos] : score_key(srow[pos])) : 0u;
        if (cand) sel = k > T || (!ties && k == T);
        if (ties) {
          const bool eq = cand && k == T;
          const uint32_t eqbal = __ballot_sync(0xffffffffu, eq);
          if (eq) sel = tile_rank[w] + __popc(eqbal & ((1u << lane) - 1u)) < need_eq;
        }
      }
      const uint32_t word = __ballot_sync(0xffffffffu, sel);
      if (lane == i) mine = word;
    }
    if (lane < n) mrow[w0 + lane] = mine;
  }
  if (tid == 0 && p.count) p.count[row] = nF + static_cast<int>(ksel);
}

cudaError_t launch_topk(const TopkParams &p, cudaStream_t stream) {
  const int rows = p.B * p.Hkv;
  if (rows == 0) return cudaSuccess;
  const bool use_smem = p.max_len <= kTopkSmemKeys;
  const size_t smem = (use_smem ? (size_t)(p.max_len + 3) / 4 * 16 : 0) + (size_t)((p.max_len + 31) / 32) * 4;
  auto kern = use_smem ? topk_kernel<true> : topk_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(rows), dim3(kTopkThreads), smem, stream, p);
}

}  // namespace kv4
