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
#include <algorithm>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

constexpr int kTopkThreads = 512;
constexpr int kTopkBins = 2048;            // 4 bins per thread in the scan
constexpr int kTopkSmemKeys = 49152;   // rows up to this length are staged in shared memory
constexpr int kStageVec = 8;           // 16-byte loads in flight per thread while staging

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Keys of candidate positions [c0, c1) in steps of four per thread: f(i, key)
// for each. With the row in shared memory four keys come from one 16-byte load
// (c0 rounded down to a multiple of four); only the first and the last step
// of the range test each index, the steps between hold four candidates.
template <bool kSmem, int NT, typename F>
__device__ __forceinline__ void for_candidates(const uint32_t *keys, const float *srow, int c0, int c1, int tid,
                                               F &&f) {
  const int base = c0 & ~3;
  const int lo = (c0 + 3) & ~3, hi = c1 & ~3;   // [lo, hi): whole steps inside [c0, c1)
  for (int i = base + 4 * tid; i < c1; i += 4 * NT) {
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

// Shared state of one row's selection.
struct TopkShared {
  uint32_t hist[kTopkBins];
  int wsum[32];
  int digit, rem, cnt, listn, kmin, kmax;
};

// The whole selection of one row by a CTA of NT threads, with the row staged
// as 32-bit keys in shared memory (kSmem) or re-read from global memory on
// every pass. dyn: keys [round_up(max_len, 4)] when staged, then tile ranks.
template <bool kSmem, int NT>
__device__ void topk_row(const TopkParams &p, int row, uint32_t *dyn, TopkShared &sh) {
  uint32_t *hist = sh.hist;
  int *wsum = sh.wsum;
  int &sh_digit = sh.digit, &sh_rem = sh.rem, &sh_cnt = sh.cnt;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NWARP = NT / 32, BPT = kTopkBins / NT;
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
  // with the row staged in shared memory, the first pass's histogram is taken
  // while staging
  const bool fused = kSmem && mode == 2;
  if (fused) {
    for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0;
    __syncthreads();
    const int base = c0 & ~3;
    if (p.vec_ok) {
      // 16-byte loads, kStageVec of them in flight per thread: the row starts
      // 16-byte aligned and its stride is a multiple of four, so the last
      // vector ends inside the row's storage
      const int nvec = (c1 - base + 3) >> 2;
      const float4 *src = reinterpret_cast<const float4 *>(srow + base);
      for (int v0 = tid; v0 < nvec; v0 += kStageVec * NT) {
        float4 buf[kStageVec];
#pragma unroll
        for (int u = 0; u < kStageVec; ++u) {
          const int v = v0 + u * NT;
          if (v < nvec) buf[u] = __ldg(src + v);
        }
#pragma unroll
        for (int u = 0; u < kStageVec; ++u) {
          const int v = v0 + u * NT;
          if (v < nvec) {
            const int i = base + 4 * v;
            const uint4 k4 = make_uint4(score_key(buf[u].x), score_key(buf[u].y), score_key(buf[u].z),
                                        score_key(buf[u].w));
            *reinterpret_cast<uint4 *>(keys + i) = k4;
            if (i >= c0 && i + 4 <= c1) {
              atomicAdd(&hist[k4.x >> 21], 1u);
              atomicAdd(&hist[k4.y >> 21], 1u);
              atomicAdd(&hist[k4.z >> 21], 1u);
              atomicAdd(&hist[k4.w >> 21], 1u);
            } else {
              const uint32_t ka[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (i + e >= c0 && i + e < c1) atomicAdd(&hist[ka[e] >> 21], 1u);
            }
          }
        }
      }
    } else {
      for (int i = base + tid; i < c1; i += NT) {
        const uint32_t k = score_key(srow[i]);
        keys[i] = k;
        if (i >= c0) atomicAdd(&hist[k >> 21], 1u);
      }
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
      if (pass > 0 || !fused) {
        for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0;
        __syncthreads();
      }
      if (pass == 0) {
        if (!fused)
          for_candidates<kSmem, NT>(keys, srow, c0, c1, tid,
                                [&](int, uint32_t k) { atomicAdd(&hist[k >> shift], 1u); });
      } else {
        for_candidates<kSmem, NT>(keys, srow, c0, c1, tid, [&](int, uint32_t k) {
          if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & dmask], 1u);
        });
      }
      __syncthreads();
      // thread i owns bins kTopkBins-1-BPT*i .. kTopkBins-BPT-BPT*i (highest
      // first): block-wide exclusive scan of the per-thread counts from the top
      int cnt[BPT], tot = 0;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        cnt[j] = hist[kTopkBins - 1 - BPT * tid - j];
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
      for (int j = 0; j < BPT; ++j) {
        if (c < rem && rem <= c + cnt[j]) {
          sh_digit = kTopkBins - 1 - BPT * tid - j;
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

  uint32_t *mrow = p.mask + (long long)row * p.mask_stride;
  if (kSmem && mode == 2) {
    // mask words from the staged keys: a warp covers 128 positions (4 words)
    // per step, lane l positions 4l .. 4l+3 from one 16-byte load; the 8 lanes
    // of a word OR their 4-bit pieces together
    const int sub = lane & 7;
    for (int it = warp; 4 * it < nt; it += NWARP) {
      const int pos = 128 * it + 4 * lane;
      uint4 k4 = make_uint4(0, 0, 0, 0);
      if (pos + 4 > c0 && pos < c1) k4 = *reinterpret_cast<const uint4 *>(keys + pos);
      const uint32_t ka[4] = {k4.x, k4.y, k4.z, k4.w};
      uint32_t sel = 0, eq = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = pos + e;
        const bool cand = q >= c0 && q < c1;
        const bool f = q < L && !cand;
        sel |= static_cast<uint32_t>(f || (cand && (ka[e] > T || (!ties && ka[e] == T)))) << e;
        eq |= static_cast<uint32_t>(cand && ties && ka[e] == T) << e;
      }
      sel <<= 4 * sub;
      eq <<= 4 * sub;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        sel |= __shfl_xor_sync(0xffffffffu, sel, o);
        eq |= __shfl_xor_sync(0xffffffffu, eq, o);
      }
      const int w = 4 * it + (lane >> 3);
      if (ties) {   // uniform over the CTA
        // equal keys in index order take the remaining places
        uint32_t mine = (eq >> (4 * sub)) & 15u;
        if (mine) {
          const int r0 = tile_rank[w];
          while (mine) {
            const int b = 4 * sub + __ffs(mine) - 1;
            mine &= mine - 1;
            if (r0 + __popc(eq & ((1u << b) - 1u)) < need_eq) sel |= 1u << b;
          }
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) sel |= __shfl_xor_sync(0xffffffffu, sel, o);
      }
      if (sub == 0 && w < nt) mrow[w] = sel;
    }
    if (tid == 0 && p.count) p.count[row] = nF + static_cast<int>(ksel);
    return;
  }
  // mask words: a warp builds 32 consecutive words (lane i keeps word i) and
  // stores them together
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

// ---------------------------------------------------------------------------
// Rows of up to kFastMaxLen positions with 16-byte aligned scores: the row is
// staged as the top 16 bits of its keys (so four CTAs share an SM and a batch
// of rows runs in one wave). The first histogram bins the candidates' key
// prefixes relative to the row's own range, (prefix - P0) >> s over 2048 bins:
// scores that span a few octaves spread over about a thousand counters instead
// of the few dozen that fixed sign and exponent bits would give, so the
// shared-memory atomics rarely collide. The prefixes are counted as they are
// staged, with the range estimated from the first step of loads (see phase A).
// One pass over the staged prefixes then writes every mask bit except those of
// the threshold bin and lists that bin's positions; the exact threshold is
// selected among the listed keys (full keys re-read from global memory, cached
// in L2 by then; one warp ranks them when at most 32 are listed) and their
// bits are set last. A threshold bin larger than
// kListCap, or an end bin that also counted prefixes outside the estimated
// range, falls back to the general path.
// ---------------------------------------------------------------------------
constexpr int kFastThreads = 256;
constexpr int kFastMaxLen = 16384;
constexpr int kListCap = 2048;
constexpr int kFastStageVec = 4;   // 16-byte loads in flight per thread while staging

// score_key with -0 folded by adding +0 (rounding to nearest gives +0).
__device__ __forceinline__ uint32_t score_key2(float f) {
  const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
  return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

// Bits of the positions [lo, hi) that fall in mask word w.
__device__ __forceinline__ uint32_t range_bits(int w, int lo, int hi) {
  const int a = max(lo - 32 * w, 0), z = min(hi - 32 * w, 32);
  if (z <= a) return 0u;
  return (z >= 32 ? 0xFFFFFFFFu : ((1u << z) - 1u)) & ~((1u << a) - 1u);
}

// Block-wide: the bin (highest first) holding the rem-th largest key of the
// histogram, the rank left inside it and its count, into sh.digit / rem / cnt.
template <int NT>
__device__ void select_bin(TopkShared &sh, int rem, int tid) {
  constexpr int BPT = kTopkBins / NT;
  const int lane = tid & 31, warp = tid >> 5;
  int cnt[BPT], tot = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    cnt[j] = sh.hist[kTopkBins - 1 - BPT * tid - j];
    tot += cnt[j];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.wsum[warp] = incl;
  __syncthreads();
  int c = incl - tot;
  for (int w = 0; w < warp; ++w) c += sh.wsum[w];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    if (c < rem && rem <= c + cnt[j]) {
      sh.digit = kTopkBins - 1 - BPT * tid - j;
      sh.rem = rem - c;
      sh.cnt = cnt[j];
    }
    c += cnt[j];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kFastThreads, 4) topk_fast_kernel(TopkParams p) {
  constexpr int NT = kFastThreads, NWARP = NT / 32;
  extern __shared__ __align__(16) uint8_t dynb[];
  __shared__ TopkShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x;
  const int b = row / p.Hkv;
  int L = p.seq_lens[b];
  L = L < 0 ? 0 : (L > p.max_len ? p.max_len : L);
  const float *srow = p.scores + (long long)row * p.score_stride;
  const int nt = (L + 31) / 32;
  const int c0 = min(p.sink, L), c1 = max(c0, L - p.recent);
  const int nF = L - (c1 - c0);
  const long long kb = (long long)L * p.permille / 1000;
  long long ksel = kb - nF;
  if (ksel < 0) ksel = 0;
  if (ksel > c1 - c0) ksel = c1 - c0;
  const int mode = ksel == 0 ? 0 : (ksel == c1 - c0 ? 1 : 2);
  uint32_t *mrow = p.mask + (long long)row * p.mask_stride;
  if (mode != 2) {
    // no selection: the forced positions, or every position
    for (int w = tid; w < nt; w += NT)
      mrow[w] = mode == 1 ? range_bits(w, 0, L) : (range_bits(w, 0, c0) | range_bits(w, c1, L));
    if (tid == 0 && p.count) p.count[row] = nF + static_cast<int>(ksel);
    return;
  }
  // shared memory: key prefixes [KR] u16 | mask words [round_up(nt_max, 4)] |
  // listed keys [kListCap] u32 | listed positions [kListCap] u16
  // (the prefix area also holds 2 * NTW words of tie bookkeeping later)
  const int NTW = ((p.max_len + 31) / 32 + 3) & ~3, KR = max((p.max_len + 7) & ~7, 4 * NTW);
  uint16_t *keys16 = reinterpret_cast<uint16_t *>(dynb);
  uint32_t *maskw = reinterpret_cast<uint32_t *>(dynb + 2 * KR);
  uint32_t *list_key = maskw + NTW;
  uint16_t *list_pos = reinterpret_cast<uint16_t *>(list_key + kListCap);

  // A. stage the key prefixes and count them into the first histogram as
  // they arrive, so that its shared-memory atomics overlap the row's loads.
  // The bins need the candidates' prefix range before the last loads land:
  // the first step's vectors (one block of NT in every kFastStageVec, spread
  // over the row) give an estimate [emin, emax], widened by a quarter of its
  // span on each side to [P0, P0 + 2048 * 2^S); a prefix outside it counts in
  // the end bin on its side. The exact range follows from the whole pass: a
  // threshold in an end bin that received such prefixes takes the general
  // path, every other bin holds exactly the prefixes of its nominal range.
  for (int i = tid; i < kTopkBins; i += NT) sh.hist[i] = 0;
  if (tid == 0) sh.listn = 0;
  uint32_t kmin = 0xFFFFu, kmax = 0u;   // candidate prefix range of this thread
  uint32_t kmin2 = 0xFFFFFFFFu, kmax2 = 0u;   // the same over whole vectors, two 16-bit lanes
  const int base = c0 & ~3;
  const int nvec = (c1 - base + 3) >> 2;
  const int nblk = (nvec + NT - 1) / NT, nstep = (nblk + kFastStageVec - 1) / kFastStageVec;
  const float4 *src = reinterpret_cast<const float4 *>(srow + base);
  uint32_t P0 = 0, S = 0;
  int negP0 = 0, top = 0;   // -P0, and the last prefix offset of the top bin
  auto bin_of = [&](uint32_t kp) -> uint32_t {
    // max(min(kp - P0, top), 0) >> S: one clamped add, one shift
    return static_cast<uint32_t>(__viaddmin_s32_relu(static_cast<int>(kp), negP0, top)) >> S;
  };
  // the 4 prefixes of a vector whose positions are all candidates
  auto count4 = [&](uint32_t p01, uint32_t p23) {
    atomicAdd(&sh.hist[bin_of(p01 & 0xFFFFu)], 1u);
    atomicAdd(&sh.hist[bin_of(p01 >> 16)], 1u);
    atomicAdd(&sh.hist[bin_of(p23 & 0xFFFFu)], 1u);
    atomicAdd(&sh.hist[bin_of(p23 >> 16)], 1u);
  };
  // vectors [v_in0, v_in1) hold candidates only; the first and the last
  // vector may also hold forced positions and are finished after the pass
  const int v_in0 = base < c0 ? 1 : 0, v_in1 = (c1 - base) >> 2;
  // block-wide min / max of the threads' kmin / kmax into sh.kmin / sh.kmax
  auto reduce_range = [&]() {
    uint32_t a = min(kmin, min(kmin2 & 0xFFFFu, kmin2 >> 16)), z = max(kmax, max(kmax2 & 0xFFFFu, kmax2 >> 16));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
      z = max(z, __shfl_xor_sync(0xffffffffu, z, o));
    }
    if (lane == 0) {
      sh.wsum[warp] = static_cast<int>(a);
      sh.wsum[16 + warp] = static_cast<int>(z);
    }
    __syncthreads();
    if (tid == 0) {
      int x = sh.wsum[0], y = sh.wsum[16];
      for (int w = 1; w < NWARP; ++w) {
        x = min(x, sh.wsum[w]);
        y = max(y, sh.wsum[16 + w]);
      }
      sh.kmin = x;
      sh.kmax = y;
    }
    __syncthreads();
  };
  for (int st = 0; st < nstep; ++st) {
    float4 buf[kFastStageVec];
#pragma unroll
    for (int u = 0; u < kFastStageVec; ++u) {
      const int v = (st + nstep * u) * NT + tid;
      if (v < nvec) buf[u] = __ldg(src + v);
    }
#pragma unroll
    for (int u = 0; u < kFastStageVec; ++u) {
      const int v = (st + nstep * u) * NT + tid;
      if (v < nvec) {
        const uint32_t k0 = score_key2(buf[u].x), k1 = score_key2(buf[u].y), k2 = score_key2(buf[u].z),
                       k3 = score_key2(buf[u].w);
        const uint2 pk = make_uint2(__byte_perm(k0, k1, 0x7632), __byte_perm(k2, k3, 0x7632));
        *reinterpret_cast<uint2 *>(keys16 + base + 4 * v) = pk;
        if (v >= v_in0 && v < v_in1) {
          kmin2 = __vimin3_u16x2(kmin2, pk.x, pk.y);
          kmax2 = __vimax3_u16x2(kmax2, pk.x, pk.y);
          if (st > 0) count4(pk.x, pk.y);
        }
      }
    }
    if (st == 0) {
      // the bins, from the first step's range (no candidate there: the whole
      // prefix range)
      reduce_range();
      int lo = 0, hi = 0x10000;
      if (sh.kmin <= sh.kmax) {
        const int emin = sh.kmin, emax = sh.kmax, q = (emax - emin) >> 2;
        lo = max(emin - q, 0);
        hi = min(emax + q + 1, 0x10000);
      }
      P0 = static_cast<uint32_t>(lo);
      while (static_cast<uint32_t>(hi - lo) > (static_cast<uint32_t>(kTopkBins) << S)) ++S;
      negP0 = -lo;
      top = (kTopkBins << S) - 1;
#pragma unroll
      for (int u = 0; u < kFastStageVec; ++u) {
        const int v = nstep * u * NT + tid;
        if (v >= v_in0 && v < v_in1) {
          const uint2 k2 = *reinterpret_cast<const uint2 *>(keys16 + base + 4 * v);
          count4(k2.x, k2.y);
        }
      }
    }
  }
  __syncthreads();   // the last vector may have been staged by another thread
  if (tid < 2) {
    // the first and the last vector when they hold forced positions
    const int v = tid == 0 ? 0 : nvec - 1;
    if ((v < v_in0 || v >= v_in1) && (tid == 0 || v > 0)) {
      const uint2 k2 = *reinterpret_cast<const uint2 *>(keys16 + base + 4 * v);
      const uint32_t kp[4] = {k2.x & 0xFFFFu, k2.x >> 16, k2.y & 0xFFFFu, k2.y >> 16};
      for (int e = 0; e < 4; ++e) {
        const int q = base + 4 * v + e;
        if (q >= c0 && q < c1) {
          kmin = min(kmin, kp[e]);
          kmax = max(kmax, kp[e]);
          atomicAdd(&sh.hist[bin_of(kp[e])], 1u);
        }
      }
    }
  }
  reduce_range();   // the exact range: were prefixes counted in an end bin from outside it?
  const bool low_out = static_cast<uint32_t>(sh.kmin) < P0;
  const bool high_out = static_cast<uint32_t>(sh.kmax) >= P0 + (static_cast<uint32_t>(kTopkBins) << S);
  const uint32_t pmin = P0;
  const int sh16 = static_cast<int>(S);
  __syncthreads();
  select_bin<NT>(sh, static_cast<int>(ksel), tid);
  const uint32_t d0 = static_cast<uint32_t>(sh.digit);
  const int rem0 = sh.rem, n0 = sh.cnt;
  if (n0 > kListCap || (d0 == 0 && low_out) || (d0 == kTopkBins - 1 && high_out)) {
    // a crowded threshold bin, or an end bin wider than its nominal range:
    // the general path, keys re-read from global memory
    __syncthreads();
    topk_row<false, NT>(p, row, reinterpret_cast<uint32_t *>(dynb), sh);
    return;
  }
  // C. mask bits of every position outside bin d0; bin d0's positions listed
  // (their full keys are fetched after the pass, from L2).
  // A warp covers 128 positions (4 words) per step: lane l positions 4l..4l+3
  // from one 8-byte load; the 8 lanes of a word OR their 4-bit pieces.
  // Bin d0 holds the prefixes [lo16, lo16 + W), W = 2^s: with u = prefix - lo16
  // as an unsigned 32-bit difference (a prefix below the bin wraps past 2^31),
  // the prefix is in the bin iff u < W and above it iff W <= u < 2^31 (every
  // prefix is below 2^16).
  const int sub = lane & 7;
  const uint32_t lo16 = pmin + (d0 << sh16), hi16 = lo16 + (1u << sh16);
  const uint32_t W = 1u << sh16;   // bin d0 is [lo16, lo16 + W)
  // bin d0's positions p + stride * e of the set bits e of lst listed
  // (warp-wide slots, one shared-memory atomic per warp)
  auto list_lane = [&](uint32_t lst, int p, int stride) {
    if (!__any_sync(0xffffffffu, lst != 0)) return;
    const int nl = __popc(lst);
    int excl = nl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, excl, o);
      if (lane >= o) excl += y;
    }
    const int total = __shfl_sync(0xffffffffu, excl, 31);
    excl -= nl;
    int at = 0;
    if (lane == 0 && total) at = atomicAdd(&sh.listn, total);
    at = __shfl_sync(0xffffffffu, at, 0) + excl;
    while (lst) {
      const int e = __ffs(lst) - 1;
      lst &= lst - 1;
      list_pos[at++] = static_cast<uint16_t>(p + stride * e);
    }
  };
  // the word pieces of a step (lane l: positions 4l..4l+3) ORed and stored
  auto store_pieces = [&](int it, uint32_t sel) {
    sel <<= 4 * sub;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) sel |= __shfl_xor_sync(0xffffffffu, sel, o);
    const int w = 4 * it + (lane >> 3);
    if (sub == 0 && w < nt) maskw[w] = sel;
  };
  // steps [it_in0, it_in1) lie inside [c0, c1)
  const int nstp = (nt + 3) / 4;
  const int it_in0 = min((c0 + 127) / 128, nstp), it_in1 = max(it_in0, c1 / 128);
  // (lane l takes positions l, l + 32, l + 64, l + 96 of the step, so that a
  // ballot is a whole mask word)
  for (int it = it_in0 + warp; it < it_in1; it += NWARP) {
    const int p0 = 128 * it + lane;
    uint32_t sw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t u = static_cast<uint32_t>(keys16[p0 + 32 * e]) - lo16;   // below the bin: wraps past 2^31
      sw[e] = __ballot_sync(0xffffffffu, u - W < 0x80000000u - W);
      lw[e] = __ballot_sync(0xffffffffu, u < W);
    }
    if (lane == 0) *reinterpret_cast<uint4 *>(maskw + 4 * it) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
    if ((lw[0] | lw[1] | lw[2] | lw[3]) == 0u) continue;
    uint32_t lst = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) lst |= ((lw[e] >> lane) & 1u) << e;
    list_lane(lst, p0, 32);
  }
  // the other steps: forced positions, the ends of the candidate range
  const int n_edge = it_in0 + (nstp - it_in1);
  for (int j = warp; j < n_edge; j += NWARP) {
    const int it = j < it_in0 ? j : it_in1 + (j - it_in0);
    const int pos = 128 * it + 4 * lane;
    uint2 k2 = make_uint2(0, 0);
    if (pos + 4 > c0 && pos < c1) k2 = *reinterpret_cast<const uint2 *>(keys16 + pos);
    const uint32_t kp[4] = {k2.x & 0xFFFFu, k2.x >> 16, k2.y & 0xFFFFu, k2.y >> 16};
    uint32_t sel = 0, lst = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int q = pos + e;
      const bool cand = q >= c0 && q < c1;
      const bool above = kp[e] >= hi16, inbin = kp[e] >= lo16 && !above;
      sel |= static_cast<uint32_t>((q < L && !cand) || (cand && above)) << e;
      lst |= static_cast<uint32_t>(cand && inbin) << e;
    }
    store_pieces(it, sel);
    list_lane(lst, pos, 1);
  }
  __syncthreads();
  // the listed positions' full keys, all loads in flight together
  for (int i = tid; i < n0; i += NT) list_key[i] = score_key2(srow[list_pos[i]]);
  __syncthreads();
  // D. the exact threshold inside bin d0. Up to 32 listed keys: one warp
  // ranks them against each other (keys above and equal to each). More: its
  // keys lie in [kbase, kbase + 2^(16+s)) with s <= 5, so two 11-bit digits of
  // key - kbase finish the selection.
  const int n = n0;
  uint32_t T;
  int need_eq;
  bool ties;
  if (n <= 32) {
    if (warp == 0) {
      const bool valid = lane < n;
      const uint32_t k = valid ? list_key[lane] : 0u;
      int gt = 0, eq = 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, k, j);
        gt += kj > k ? 1 : 0;
        eq += kj == k ? 1 : 0;
      }
      // T: the key with gt < rem0 <= gt + eq (every lane holding it agrees)
      const uint32_t bal = __ballot_sync(0xffffffffu, valid && gt < rem0 && rem0 <= gt + eq);
      const int src = __ffs(bal) - 1;
      const uint32_t t_key = __shfl_sync(0xffffffffu, k, src);
      const int t_gt = __shfl_sync(0xffffffffu, gt, src), t_eq = __shfl_sync(0xffffffffu, eq, src);
      if (lane == 0) {
        sh.digit = static_cast<int>(t_key);
        sh.rem = rem0 - t_gt;
        sh.cnt = t_eq;
      }
    }
    __syncthreads();
    T = static_cast<uint32_t>(sh.digit);
  } else {
    const uint32_t kbase = (pmin + (d0 << sh16)) << 16;
    for (int i = tid; i < kTopkBins; i += NT) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) atomicAdd(&sh.hist[(list_key[i] - kbase) >> 11], 1u);
    __syncthreads();
    select_bin<NT>(sh, rem0, tid);
    const uint32_t d1 = static_cast<uint32_t>(sh.digit);
    const int rem1 = sh.rem;
    __syncthreads();
    for (int i = tid; i < kTopkBins; i += NT) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
      const uint32_t k = list_key[i] - kbase;
      if ((k >> 11) == d1) atomicAdd(&sh.hist[k & 2047u], 1u);
    }
    __syncthreads();
    select_bin<NT>(sh, rem1, tid);
    T = kbase + (d1 << 11) + static_cast<uint32_t>(sh.digit);
  }
  need_eq = sh.rem;
  ties = need_eq < sh.cnt;
  // E. bits of the listed positions: keys above T, and keys equal to T by
  // index order (ranks from a bitmap of the equal keys and a scan over words)
  if (!ties) {
    for (int i = tid; i < n; i += NT)
      if (list_key[i] >= T) {
        const int q = list_pos[i];
        atomicOr(&maskw[q >> 5], 1u << (q & 31));
      }
  } else {
    uint32_t *eqw = reinterpret_cast<uint32_t *>(dynb);   // the key prefixes are no longer needed
    int *tile_rank = reinterpret_cast<int *>(eqw + NTW);
    for (int w = tid; w < nt; w += NT) eqw[w] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += NT)
      if (list_key[i] == T) {
        const int q = list_pos[i];
        atomicOr(&eqw[q >> 5], 1u << (q & 31));
      }
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
      for (int w0 = 0; w0 < nt; w0 += 32) {
        const int w = w0 + lane;
        const int v = w < nt ? __popc(eqw[w]) : 0;
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
    for (int i = tid; i < n; i += NT) {
      const uint32_t k = list_key[i];
      const int q = list_pos[i], w = q >> 5;
      bool take = k > T;
      if (k == T) take = tile_rank[w] + __popc(eqw[w] & ((1u << (q & 31)) - 1u)) < need_eq;
      if (take) atomicOr(&maskw[w], 1u << (q & 31));
    }
  }
  __syncthreads();
  for (int w = tid; w < nt; w += NT) mrow[w] = maskw[w];
  if (tid == 0 && p.count) p.count[row] = nF + static_cast<int>(ksel);
}

template <bool kSmem>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint32_t dyn[];
  __shared__ TopkShared sh;
  pdl_wait();
  pdl_launch_dependents();
  topk_row<kSmem, kTopkThreads>(p, blockIdx.x, dyn, sh);
}

size_t topk_fast_smem(int max_len) {
  const size_t NTW = ((size_t)(max_len + 31) / 32 + 3) & ~(size_t)3;
  const size_t KR = std::max((size_t)(max_len + 7) & ~(size_t)7, 4 * NTW);
  return 2 * KR + 4 * NTW + 6 * (size_t)kListCap;
}

cudaError_t launch_topk(const TopkParams &p, cudaStream_t stream) {
  const int rows = p.B * p.Hkv;
  if (rows == 0) return cudaSuccess;
  if (p.vec_ok && p.max_len <= kFastMaxLen) {
    const size_t smem = topk_fast_smem(p.max_len);
    cudaError_t e = cudaFuncSetAttribute(topk_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_fast_kernel, dim3(rows), dim3(kFastThreads), smem, stream, p);
  }
  const bool use_smem = p.max_len <= kTopkSmemKeys;
  const size_t smem = (use_smem ? (size_t)(p.max_len + 3) / 4 * 16 : 0) + (size_t)((p.max_len + 31) / 32) * 4;
  auto kern = use_smem ? topk_kernel<true> : topk_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(rows), dim3(kTopkThreads), smem, stream, p);
}

}  // namespace kv4
