// kv4_decode.cu -- decode-step attention over the KV4-RL compressed cache.
//
// KV4-RL review, sec. 3: the INT4 region and the INT8-protected region (first
// 16 and last 128 positions) are attended independently; their partial
// (max, sum, output) triples are combined by an exact softmax merge, so no
// full-precision cache is rebuilt. Shadow Mask Distillation, sec. 1 / Figure 1:
// a retained-position mask is applied inside attention.
//
// Two launches on the caller's stream:
//   kv4_decode_kernel  page-major workers: a CTA with one warp per KV head
//                      streams whole pages (every head of a page in one bulk
//                      copy, the TMA engine, mbarrier completion, bounded
//                      waits) and side pages through a ring of shared-memory
//                      stages shared by its warps. Per page and head, q.K and
//                      P.V are small tensor-core tiles (mma.sync m16n8k16,
//                      fp32 accumulate). Each warp writes one (m, l, o)
//                      partial per (region, sequence) range its CTA touches.
//   merge_kernel       (kv4_merge.cu) one warp per (sequence, query head)
//                      merges the partials exactly.
// The uncompressed comparison (bf16 pages) keeps per-warp workers over
// (sequence, head) page ranges (bf16_decode_kernel).
//
// Softmax bookkeeping runs in the log2 domain (scores scaled by tau*log2 e).
// P.V takes P*scale_V as two fp16 terms (hi + lo), which carries 22
// significant bits into fp32 accumulation; the running max is exact (P <= 1),
// so P*scale_V stays in the fp16 range.
#include <math.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

// Per-warp ring of the bf16 comparison kernel.
template <int D>
struct Bf16Cfg {
  static constexpr int NS = 3;                              // stages per warp
  static constexpr int ROWB = 2 * D + 16;                   // padded bf16 row in shared memory
  static constexpr int STAGE = 2 * kPageTokens * ROWB;
  static constexpr int WARP_SMEM = NS * STAGE;
  static constexpr int RINGS = kWarps * (WARP_SMEM + NS * 8);
};


// ---------------------------------------------------------------------------
// Partial slot: m[G] | l[G] | pad | o[G][D]   (m in log2 units, o normalised)
// ---------------------------------------------------------------------------

// Running-max start: the lowest finite float, so that score - max needs no
// test for an empty state. Only -inf (excluded) scores and scores equal to it
// leave it in place; they get weights 0 and 1, as against a true maximum. A
// state that attended nothing keeps l = 0 and is written as empty.
constexpr float kNoMax = -3.40282347e38f;

// Online-softmax state of one warp for the 8 MMA columns (4 "hi" + 4 "lo"
// copies of up to 4 query heads). Thread (g, t) owns columns 2t and 2t+1.
template <int NMT>
struct SoftmaxState {
  float m[2], l[2];
  float o[NMT][4];   // O^T fragments: rows = head_dim, columns = MMA columns
  __device__ __forceinline__ void reset() {
    m[0] = m[1] = kNoMax;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) o[mt][c] = 0.f;
  }
};

// Scores s[0..3] for (token g, col 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1) are
// in log2 units; -inf marks excluded positions. Updates m, l, rescales o and
// returns the probabilities. kSlack = 8: the reference max moves only when a
// page max exceeds it by more than 8 (probabilities stay <= 2^8); kSlack = 0:
// exact running max (probabilities <= 1).
template <int NMT, int kSlack>
__device__ __forceinline__ void softmax_update(SoftmaxState<NMT> &st, const float (&s)[4], float (&pr)[4]) {
  float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
  // The page's column max exceeds the reference exactly when some lane's own
  // max does, so the warp-wide max (three shuffle rounds) is only formed on
  // pages that move the reference.
  const bool up = mx0 > st.m[0] + static_cast<float>(kSlack) || mx1 > st.m[1] + static_cast<float>(kSlack);
  if (__any_sync(0xffffffffu, up)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (mx0 > st.m[0] + static_cast<float>(kSlack)) {
      const float f = ex2(st.m[0] - mx0);
      st.l[0] *= f;
#pragma unroll
      for (int mt = 0; mt < NMT; ++mt) {
        st.o[mt][0] *= f;
        st.o[mt][2] *= f;
      }
      st.m[0] = mx0;
    }
    if (mx1 > st.m[1] + static_cast<float>(kSlack)) {
      const float f = ex2(st.m[1] - mx1);
      st.l[1] *= f;
#pragma unroll
      for (int mt = 0; mt < NMT; ++mt) {
        st.o[mt][1] *= f;
        st.o[mt][3] *= f;
      }
      st.m[1] = mx1;
    }
  }
  const float2 r = make_float2(st.m[0], st.m[1]);   // kNoMax while nothing is attended: every p is 0
  const float2 d01 = __fadd2_rn(make_float2(s[0], s[1]), make_float2(-r.x, -r.y));
  const float2 d23 = __fadd2_rn(make_float2(s[2], s[3]), make_float2(-r.x, -r.y));
  pr[0] = ex2(d01.x);
  pr[1] = ex2(d01.y);
  pr[2] = ex2(d23.x);
  pr[3] = ex2(d23.y);
  const float2 l = __fadd2_rn(make_float2(st.l[0], st.l[1]),
                              __fadd2_rn(make_float2(pr[0], pr[1]), make_float2(pr[2], pr[3])));
  st.l[0] = l.x;
  st.l[1] = l.y;
}

// Weights w for (token g, col 2t/2t+1) and (token g+8, ...) -> the B fragment
// (k = tokens, n = columns) of the P.V tile. Lanes with t < 2 contribute the
// 16-bit rounding of w ("hi" columns 0-3); lanes with t >= 2 the 16-bit
// rounding of the remainder ("lo" columns 4-7).
__device__ __forceinline__ void weights_bf16(float2 w01, float2 w23, float2 neg_sel, uint32_t &b0, uint32_t &b1) {
  uint32_t h01 = pack_bf16x2(w01.x, w01.y);
  uint32_t h23 = pack_bf16x2(w23.x, w23.y);
  const float2 r01 = __ffma2_rn(neg_sel, make_float2(bf16lo_to_f32(h01), bf16hi_to_f32(h01)), w01);
  const float2 r23 = __ffma2_rn(neg_sel, make_float2(bf16lo_to_f32(h23), bf16hi_to_f32(h23)), w23);
  b0 = movmatrix_t(pack_bf16x2(r01.x, r01.y));
  b1 = movmatrix_t(pack_bf16x2(r23.x, r23.y));
}

// fp16 variant of weights_bf16 (hi + lo carry 22 significant bits). The
// remainder w - hi comes from a mixed-precision FMA (fp16 factors, fp32
// addend, one rounding), so the hi halves need no conversion back to fp32.
// neg_sel is -1 (0xBC00) on the "lo" lanes and 0 on the "hi" lanes.
__device__ __forceinline__ float fma_f16_f32(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}
__device__ __forceinline__ void weights_f16x2(float2 w01, float2 w23, uint16_t neg_sel, uint32_t &b0, uint32_t &b1) {
  const uint32_t h01 = pack_f16x2(w01.x, w01.y);
  const uint32_t h23 = pack_f16x2(w23.x, w23.y);
  const float r0 = fma_f16_f32(static_cast<uint16_t>(h01), neg_sel, w01.x);
  const float r1 = fma_f16_f32(static_cast<uint16_t>(h01 >> 16), neg_sel, w01.y);
  const float r2 = fma_f16_f32(static_cast<uint16_t>(h23), neg_sel, w23.x);
  const float r3 = fma_f16_f32(static_cast<uint16_t>(h23 >> 16), neg_sel, w23.y);
  b0 = movmatrix_t(pack_f16x2(r0, r1));
  b1 = movmatrix_t(pack_f16x2(r2, r3));
}
__device__ __forceinline__ uint16_t f16_neg_sel(bool lo) { return lo ? static_cast<uint16_t>(0xBC00u) : 0; }

// Reduce and write the worker's partial for one piece.
template <int D, int NMT>
__device__ __forceinline__ void write_partial(const DecodeParams &p, SoftmaxState<NMT> &st, float *slot, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    st.l[0] += __shfl_xor_sync(0xffffffffu, st.l[0], o);
    st.l[1] += __shfl_xor_sync(0xffffffffu, st.l[1], o);
  }
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
    for (int c = 0; c < 4; ++c) st.o[mt][c] += __shfl_xor_sync(0xffffffffu, st.o[mt][c], 2);
  if (t < 2) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int head = 2 * t + c;
      if (head < p.G) {
        const bool nonempty = st.l[c] > 0.f;
        const float inv = nonempty ? 1.f / st.l[c] : 0.f;
        float *o = slot + p.slot_o_off + head * D;
#pragma unroll
        for (int mt = 0; mt < NMT; ++mt) {
          o[16 * mt + g] = st.o[mt][c] * inv;
          o[16 * mt + g + 8] = st.o[mt][c + 2] * inv;
        }
        if (g == 0) {
          slot[head] = nonempty ? st.m[c] : -INFINITY;
          slot[p.G + head] = st.l[c];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Per-warp stage ring: item[0] is the next item to consume, in stage `s`.
// ---------------------------------------------------------------------------
template <int NS>
struct Ring {
  int item[NS];
  int s;
  __device__ __forceinline__ void push_rotate(int nxt) {
#pragma unroll
    for (int k = 0; k < NS - 1; ++k) item[k] = item[k + 1];
    item[NS - 1] = nxt;
    s = (s + 1 == NS) ? 0 : s + 1;
  }
};

// All lanes wait for stage s; false if the bounded wait ran out (then every
// copy still in flight is drained with the default limit).
template <int NS>
__device__ __forceinline__ bool ring_wait(const Ring<NS> &r, uint64_t *bars, uint32_t &phase, long long cap,
                                          uint32_t *err, int lane) {
  const bool ok = cap != 0 && mbar_wait_bounded(&bars[r.s], (phase >> r.s) & 1u, cap);
  if (__all_sync(0xffffffffu, ok)) {
    phase ^= 1u << r.s;
    return true;
  }
  if (lane == 0) set_error(err, kErrTimeout);
#pragma unroll
  for (int k = 0; k < NS; ++k) {
    const int st = (r.s + k) % NS;
    if (r.item[k] >= 0) {
      mbar_wait_bounded(&bars[st], (phase >> st) & 1u, kDefaultWaitCycles);
      phase ^= 1u << st;
    }
  }
  return false;
}

// ---------------------------------------------------------------------------
// Page cursor over INT4 / bf16 pages [pg0, pg1) of one (sequence, KV head).
// ---------------------------------------------------------------------------
struct PageCursor {
  int pg1, cursor, batch_base;
  int pid_reg;        // page id of page batch_base + lane
  uint32_t okbits;    // pages in the batch with at least one attended position
};

__device__ __forceinline__ void load_batch(PageCursor &c, int base, const int32_t *ptrow, int lo_tok, int hi_tok,
                                           const uint32_t *mrow, const DecodeParams &p, int lane) {
  c.batch_base = base;
  const int pg = base + lane;
  bool ok = pg < c.pg1;
  int pid = -1;
  if (ok) {
    const int t0 = max(pg * kPageTokens, lo_tok) - pg * kPageTokens;
    const int t1 = min(pg * kPageTokens + kPageTokens, hi_tok) - pg * kPageTokens;
    ok = t0 < t1;
    if (ok && mrow) {
      const uint32_t bits16 = (mrow[pg >> 1] >> ((pg & 1) * 16)) & 0xFFFFu;
      const uint32_t win = ((1u << t1) - 1u) & ~((1u << t0) - 1u);
      ok = (bits16 & win) != 0u;
    }
    if (ok) {
      pid = ptrow[pg];
      if (pid < 0 || pid >= p.num_pages) {
        set_error(p.err, kErrBounds);
        ok = false;
      }
    }
  }
  c.pid_reg = pid;
  c.okbits = __ballot_sync(0xffffffffu, ok);
}

__device__ __forceinline__ int next_page(PageCursor &c, int &pid, const int32_t *ptrow, int lo_tok, int hi_tok,
                                         const uint32_t *mrow, const DecodeParams &p, int lane) {
  // common case: the next page is in the loaded batch and has work
  const int idx0 = c.cursor - c.batch_base;
  if (c.cursor < c.pg1 && idx0 < 32 && ((c.okbits >> idx0) & 1u)) {
    pid = __shfl_sync(0xffffffffu, c.pid_reg, idx0);
    return c.cursor++;
  }
  while (c.cursor < c.pg1) {
    if (c.cursor >= c.batch_base + 32) load_batch(c, c.cursor, ptrow, lo_tok, hi_tok, mrow, p, lane);
    const int idx = c.cursor - c.batch_base;
    const uint32_t rem = c.okbits >> idx;
    if (rem) {
      const int k = __ffs(rem) - 1;
      pid = __shfl_sync(0xffffffffu, c.pid_reg, idx + k);
      const int pg = c.cursor + k;
      c.cursor = pg + 1;
      return pg;
    }
    c.cursor = c.batch_base + 32;
  }
  return -1;
}

// ===========================================================================
// KV4 decode kernel: INT4 pages and INT8 side pages, page-major.
//
// A CTA has one warp per KV head of a head block (HB heads, HB <= 8; with
// more KV heads each block of HB heads is a "virtual sequence" vb = hb * B + b
// of its own). Work items form one flat, ordered space, virtual sequence by
// virtual sequence: first its INT8 side pages (2 * np8 items, the K half then
// the V half of each side page), then its INT4 pages in page order. CTA c
// takes items [c T / nc, (c+1) T / nc), a bound that would part the two
// halves of a side page moved down by one, so every CTA holds its share of
// side-page work and both halves of a side page stay in one CTA. An item
// always covers every head of the block: one bulk copy of the page's HB head
// blocks (INT4; they are contiguous in a page) or HB copies of one side-page
// half, into a stage of an NS-stage ring shared by the CTA. Warp hh computes
// head hh's slice. The warp that releases a stage last (a counter per stage,
// acquire-release shared atomics) refills it with the item NS places ahead,
// so nobody waits for a producer and no warp keeps ring or cursor state
// beyond the stage index. Ranges: (virtual sequence vb, region) has range id
// 2 * vb (INT8) or 2 * vb + 1 (INT4), increasing along the item space.
//
// Item descriptors (kind | vb | page or side page, page id) are prepared per
// chunk of up to kChunk items by the whole CTA: classification, page-table
// reads, bounds checks and the skip of pages without an attended position
// all happen there, in parallel, and the kept items are compacted.
// ===========================================================================
constexpr int kChunk = 256;
constexpr int kItemInt4 = 0, kItemInt8K = 1, kItemInt8V = 2;

// Per-warp query area: D/32 chunks of 512 bytes (the B fragments of the q.K
// tiles, one 16-byte piece per lane) and, for INT4 ranges, the accumulator
// start of every (group, query head): D/32 x 4 floats.
__host__ __device__ constexpr int kv4_q_bytes(int D) { return (D / 32) * 512 + (D / 32) * 32; }

// Shared-memory layout of the KV4 kernel (bytes), for HB heads, NS stages and
// NVB virtual sequences.
struct Kv4Layout {
  int bars, cnt, iss, flag, desc, q, plan, wtot, total;
};

__host__ __device__ inline Kv4Layout kv4_layout(int D, int HB, int NS, int NVB) {
  Kv4Layout l;
  int o = NS * HB * 18 * D;
  l.bars = o;
  o += NS * 8;
  l.cnt = o;   // "empty" mbarriers: every warp arrives when it is done with a stage
  o += NS * 8;
  l.iss = o;
  o += NS * 4;
  l.flag = o;
  o += 4;
  o = (o + 15) & ~15;
  l.desc = o;
  o += kChunk * 8;
  l.q = o;
  o += HB * kv4_q_bytes(D);
  l.plan = o;
  o += (NVB + 1) * 4;
  l.wtot = o;
  o += 8 * 4;
  l.total = o;
  return l;
}

// Largest i in [0, n) with a[i] <= y (a non-decreasing, a[0] <= y).
__device__ __forceinline__ int upper_index(const int *a, int n, long long y) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= y) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Side page j of a sequence of length L holds at least one attended row:
// the sink page (j < js) when L > 0, a ring page when its 16 slots meet the
// slots {p mod R : p in [max(S, L - R), L)}, a cyclic run of min(L - S, R).
__device__ __forceinline__ bool side_page_attended(int j, int L, int S, int R) {
  const int js = S > 0 ? 1 : 0;
  if (L <= 0) return false;
  if (j < js) return true;
  const int r0 = max(S, L - R), nv = L - r0;
  if (nv <= 0) return false;
  if (nv >= R) return true;
  const int lo = 16 * (j - js), a = r0 % R;
  return ((lo - a + R) % R) < nv || ((a - lo + R) % R) < 16;
}

// INT4 pages of sequence b attended by this call: the INT4 region's pages
// [sink/16, ceil((L - recent)/16)), clipped to the shard [page_begin[b],
// page_end[b]) when the call decodes one page-range shard of each sequence.
__device__ __forceinline__ void int4_page_range(const DecodeParams &p, int b, int L, int &pg0, int &pg1) {
  pg0 = int4_first_page(p.sink);
  pg1 = pg0 + int4_num_pages(L, p.sink, p.recent);
  if (p.page_begin) {
    pg0 = max(pg0, p.page_begin[b]);
    pg1 = max(pg0, min(pg1, p.page_end[b]));
  }
}

// Descriptor of flat item x, or false if the item has nothing to attend
// (or names a page outside the pool, which is reported). n8 = INT8 items per
// virtual sequence (0 without side pages).
template <int D>
__device__ bool classify_item(const DecodeParams &p, const int *plan, int n8, long long x, int2 &d) {
  const int NVB = p.NVB, HB = p.HB, cap = p.pt_stride * kPageTokens;
  const int vb = upper_index(plan, NVB, x);
  const int off = static_cast<int>(x - plan[vb]);
  const int hb = vb / p.B, b = vb - hb * p.B;
  if (off < n8) {
    const int j = off >> 1;
    const int L = eff_len(p.seq_lens[b], cap);
    if (!side_page_attended(j, L, p.sink, p.recent)) return false;
    d.x = ((off & 1) ? kItemInt8V : kItemInt8K) | (vb << 2) | (j << 15);
    d.y = 0;
    return true;
  }
  int pg0, pg1;
  int4_page_range(p, b, eff_len(p.seq_lens[b], cap), pg0, pg1);
  const int pg = pg0 + off - n8;
  if (p.mask) {
    const int L = eff_len(p.seq_lens[b], cap);
    const int lo_tok = p.sink, hi_tok = L - p.recent;
    const int t0 = max(pg * kPageTokens, lo_tok) - pg * kPageTokens;
    const int t1 = min(pg * kPageTokens + kPageTokens, hi_tok) - pg * kPageTokens;
    const uint32_t win = ((t1 >= 16 ? 0xFFFFFFFFu : (1u << t1) - 1u)) & ~((1u << t0) - 1u);
    uint32_t any = 0;
    for (int hh = 0; hh < HB; ++hh) {
      const uint32_t *mrow = p.mask + ((long long)b * p.Hkv + hb * HB + hh) * p.mask_stride;
      any |= (mrow[pg >> 1] >> ((pg & 1) * 16)) & win;
    }
    if (!(any & 0xFFFFu)) return false;
  }
  const int pid = p.page_table[(long long)b * p.pt_stride + pg];
  if (pid < 0 || pid >= p.num_pages) {
    set_error(p.err, kErrBounds);
    return false;
  }
  d.x = kItemInt4 | (vb << 2) | (pg << 15);
  d.y = pid;
  return true;
}

// Prepare the descriptors of flat items [cx, cx + n): classified in parallel
// and compacted in order. Returns the number kept (the same in every thread).
template <int D>
__device__ int prepare_chunk(const DecodeParams &p, const int *plan, int n8, long long cx, int n, int2 *desc,
                             int *wtot, int tid, int nthr) {
  const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
  int base = 0;
  for (int r = 0; r < n; r += nthr) {
    const int k = r + tid;
    int2 d = make_int2(0, 0);
    const bool keep = k < n && classify_item<D>(p, plan, n8, cx + k, d);
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) wtot[warp] = __popc(bal);
    __syncthreads();
    int off = base, tot = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int c = wtot[w];
      off += w < warp ? c : 0;
      tot += c;
    }
    if (keep) desc[off + __popc(bal & ((1u << lane) - 1u))] = d;
    __syncthreads();
    base += tot;
  }
  return base;
}

// Issue the copies of item d into a stage (one thread). INT4: the HB head
// blocks of the page, contiguous in the pool; INT8: one half of side page j
// for each of the HB heads.
template <int D>
__device__ __forceinline__ void issue_item(const DecodeParams &p, int2 d, uint8_t *stage, uint64_t *bar) {
  const int kind = d.x & 3, vb = (d.x >> 2) & 0x1FFF, pj = static_cast<int>(static_cast<uint32_t>(d.x) >> 15);
  const int HB = p.HB, hb = vb / p.B, b = vb - hb * p.B;
  if (kind == kItemInt4) {
    const uint32_t bytes = static_cast<uint32_t>(HB * 18 * D);
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(stage, p.pool + (long long)d.y * p.page_bytes + (long long)hb * HB * p.head_bytes, bytes, bar);
  } else {
    constexpr uint32_t KHALF = 16 * D + 64, VHALF = 16 * D;
    const uint32_t bytes = kind == kItemInt8K ? KHALF : VHALF;
    const long long off = (long long)pj * (32 * D + 64) + (kind == kItemInt8K ? 0 : KHALF);
    const uint8_t *src = p.side + ((long long)b * p.Hkv + (long long)hb * HB) * p.side_stride + off;
    mbar_arrive_expect_tx(bar, bytes * HB);
    for (int hh = 0; hh < HB; ++hh) bulk_g2s(stage + hh * 18 * D, src + hh * p.side_stride, bytes, bar);
  }
}

// First/last CTA of every range met by [x0, x1), and an empty partial
// (m = -inf, l = 0) for each of its heads, overwritten by the real one when a
// warp closes the range.
template <int G>
__device__ void mark_ranges(const DecodeParams &p, const int *plan, int n8, long long x0, long long x1, int c,
                            int tid, int nthr) {
  const int NVB = p.NVB, HB = p.HB;
  const int va = upper_index(plan, NVB, x0), vz = upper_index(plan, NVB, x1 - 1);
  const int nr = 2 * (vz - va + 1);
  for (int i = tid; i < nr * HB * G; i += nthr) {
    const int ri = i / (HB * G), hh = (i / G) % HB, g = i % G;
    const int vb = va + (ri >> 1), region = ri & 1;
    const long long s = (long long)plan[vb] + (region ? n8 : 0);
    const long long e = region ? (long long)plan[vb + 1] : (long long)plan[vb] + n8;
    if (s == e || e <= x0 || s >= x1) continue;
    const int rid = 2 * vb + region;
    if (hh == 0 && g == 0) {
      if (s >= x0) p.first[rid] = c;
      if (e <= x1) p.last[rid] = c;
    }
    float *slot = p.slots + ((long long)(rid + c) * HB + hh) * p.slot_floats;
    slot[g] = -INFINITY;
    slot[G + g] = 0.f;
  }
}

// Query fragments of one (virtual sequence, head) into the warp's q area.
// INT4 format (per group i, 512 bytes): q as the B operand of the two q.K
// tiles -- bf16 pairs of the even elements, fp16 pairs of the odd ones --
// then, after the NG group chunks, the accumulator starts
// -(136 * sum of even q + 72 * sum of odd q) of each group as ready-made C
// register quads [group][t & 1] = {c(h), c(h + 1), c(h), c(h + 1)}, h = 2 (t & 1),
// which one 16-byte load hands to the MMA without register moves.
// INT8 format: fp16 fragments of the D/16 tiles of the side-page q.K.
// Every query element must lie in the fp16 range (it enters fp16 tiles);
// one that does not is reported as KV4_ERR_RANGE.
template <int D, int G>
__device__ __forceinline__ void load_q(const DecodeParams &p, int b, int h, bool int4, uint8_t *qsm, int lane) {
  constexpr int NG = D / 32;
  const int g = lane >> 2, t = lane & 3;
  const int head = g & 3;
  const bool hv = head < G;
  const __nv_bfloat16 *qrow = p.q + ((long long)b * p.Hq + h * G + (hv ? head : 0)) * D;
  bool big = false;
  if (int4) {
    const uint4 *qh = reinterpret_cast<const uint4 *>(qrow);
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      const uint4 e = hv ? qh[4 * i + t] : make_uint4(0, 0, 0, 0);
      const float e0 = bf16lo_to_f32(e.x), e1 = bf16hi_to_f32(e.x), e2 = bf16lo_to_f32(e.y), e3 = bf16hi_to_f32(e.y);
      const float e4 = bf16lo_to_f32(e.z), e5 = bf16hi_to_f32(e.z), e6 = bf16lo_to_f32(e.w), e7 = bf16hi_to_f32(e.w);
      const float mx = fmaxf(fmaxf(fmaxf(fabsf(e0), fabsf(e1)), fmaxf(fabsf(e2), fabsf(e3))),
                             fmaxf(fmaxf(fabsf(e4), fabsf(e5)), fmaxf(fabsf(e6), fabsf(e7))));
      big |= !(mx <= 65504.f);
      *reinterpret_cast<uint4 *>(qsm + i * 512 + lane * 16) =
          make_uint4(__byte_perm(e.x, e.z, 0x5410), __byte_perm(e.y, e.w, 0x5410), pack_f16x2(e1, e5),
                     pack_f16x2(e3, e7));
      float part = -136.f * ((e0 + e2) + (e4 + e6)) - 72.f * ((e1 + e3) + (e5 + e7));
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      // lanes 4c..4c+3 now hold the offset of column c, i.e. of query head c & 3
      if (t == 0 && g < 4) {
        // the accumulator start of MMA columns (2t, 2t + 1) for rows g and g + 8,
        // as the four C registers {c0, c1, c0, c1} of lanes with t & 1 = g >> 1
        float *quad = reinterpret_cast<float *>(qsm + NG * 512) + 8 * i + 4 * (g >> 1) + (g & 1);
        quad[0] = part;
        quad[2] = part;
      }
    }
  } else {
    constexpr int NJ = D / 16;
    const uint32_t *qh = reinterpret_cast<const uint32_t *>(qrow);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int d = t * (D / 4) + 4 * j;
      const uint32_t e01 = hv ? qh[d / 2] : 0u, e23 = hv ? qh[d / 2 + 1] : 0u;
      const float x0 = bf16lo_to_f32(e01), x1 = bf16hi_to_f32(e01), x2 = bf16lo_to_f32(e23), x3 = bf16hi_to_f32(e23);
      big |= !(fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3))) <= 65504.f);
      *reinterpret_cast<uint2 *>(qsm + (j / 2) * 512 + lane * 16 + (j % 2) * 8) =
          make_uint2(pack_f16x2(x0, x2), pack_f16x2(x1, x3));
    }
  }
  if (__any_sync(0xffffffffu, big) && lane == 0) set_error(p.err, kErrRange);
  __syncwarp();
}

// Per-range context of a warp.
struct RangeCtx {
  int b, h, L, lo_tok, hi_tok, r0;
  int pin0, pspan;   // pages [pin0, pin0 + pspan) have every slot attended (none under a mask)
  const uint32_t *mrow;
};

// One INT4 page of head h: q.K on bf16/fp16 tiles with offset codes (the
// accumulator start removes the offsets), exact running-max softmax, P.V on
// fp16 tiles with V^T codes and P * scale_V as hi + lo fp16 columns.
template <int D, int G>
__device__ __forceinline__ void int4_item(const DecodeParams &p, uint32_t stg, uint32_t qsm, int pg,
                                          const RangeCtx &rc, SoftmaxState<D / 16> &st, int lane) {
  constexpr int NG = D / 32, NMT = D / 16, NSW = (NG + 1) / 2;
  const int g = lane >> 2, t = lane & 3;
  uint32_t kw0[NG], kw1[NG], ksw0[NSW], ksw1[NSW], vsw0[NSW], vsw1[NSW];
  if constexpr (NG == 4) {
    const uint4 a0 = lds128(stg + g * (D / 2) + t * (D / 8));
    const uint4 a1 = lds128(stg + (g + 8) * (D / 2) + t * (D / 8));
    kw0[0] = a0.x; kw0[1] = a0.y; kw0[2] = a0.z; kw0[3] = a0.w;
    kw1[0] = a1.x; kw1[1] = a1.y; kw1[2] = a1.z; kw1[3] = a1.w;
    const uint2 s0 = lds64(stg + 16 * D + g * 8);
    const uint2 s1 = lds64(stg + 16 * D + (g + 8) * 8);
    const uint2 u0 = lds64(stg + 17 * D + g * 8);
    const uint2 u1 = lds64(stg + 17 * D + (g + 8) * 8);
    ksw0[0] = s0.x; ksw0[1] = s0.y; ksw1[0] = s1.x; ksw1[1] = s1.y;
    vsw0[0] = u0.x; vsw0[1] = u0.y; vsw1[0] = u1.x; vsw1[1] = u1.y;
  } else {
    const uint2 a0 = lds64(stg + g * (D / 2) + t * (D / 8));
    const uint2 a1 = lds64(stg + (g + 8) * (D / 2) + t * (D / 8));
    kw0[0] = a0.x; kw0[1] = a0.y;
    kw1[0] = a1.x; kw1[1] = a1.y;
    ksw0[0] = lds32(stg + 16 * D + g * 4);
    ksw1[0] = lds32(stg + 16 * D + (g + 8) * 4);
    vsw0[0] = lds32(stg + 17 * D + g * 4);
    vsw1[0] = lds32(stg + 17 * D + (g + 8) * 4);
  }
  float ks0[NG], ks1[NG], vs0a[NG], vs1a[NG];
#pragma unroll
  for (int c = 0; c < NSW; ++c) {
    const float2 a0 = f16x2_to_f32x2(ksw0[c]), a1 = f16x2_to_f32x2(ksw1[c]);
    const float2 b0 = f16x2_to_f32x2(vsw0[c]), b1 = f16x2_to_f32x2(vsw1[c]);
    ks0[2 * c] = a0.x; ks1[2 * c] = a1.x; vs0a[2 * c] = b0.x; vs1a[2 * c] = b1.x;
    if (2 * c + 1 < NG) {
      ks0[2 * c + 1] = a0.y; ks1[2 * c + 1] = a1.y; vs0a[2 * c + 1] = b0.y; vs1a[2 * c + 1] = b1.y;
    }
  }
  float2 sc01 = make_float2(0.f, 0.f), sc23 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < NG; ++i) {
    const uint4 qv = lds128(qsm + i * 512 + lane * 16);
    // accumulator start of columns 2t, 2t+1 (query heads 2t & 3, (2t & 3) + 1)
    const uint4 qi = lds128(qsm + NG * 512 + 32 * i + 16 * (t & 1));
    float acc[4];
    const uint32_t k80 = kw0[i] >> 8, k81 = kw1[i] >> 8;
    {   // elements 0, 4 (k-slots 2t, 2t+1) and 2, 6 (2t+8, 2t+9): bf16, 136 + c
      const uint32_t a[4] = {i4x2_biased(kw0[i]), i4x2_biased(kw1[i]), i4x2_biased(k80), i4x2_biased(k81)};
      mma_bf16_c4(acc, a, qv.x, qv.y, qi);
    }
    {   // elements 1, 5 and 3, 7: fp16, 72 + c (bits 4-7 convert in place)
      const uint32_t a[4] = {i4x2_hi_biased_f16(kw0[i]), i4x2_hi_biased_f16(kw1[i]), i4x2_hi_biased_f16(k80),
                             i4x2_hi_biased_f16(k81)};
      mma_f16(acc, a, qv.z, qv.w);
    }
    const float k0 = ks0[i], k1 = ks1[i];
    sc01 = __ffma2_rn(make_float2(k0, k0), make_float2(acc[0], acc[1]), sc01);
    sc23 = __ffma2_rn(make_float2(k1, k1), make_float2(acc[2], acc[3]), sc23);
  }
  const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
  sc01 = __fmul2_rn(sc01, sl2);
  sc23 = __fmul2_rn(sc23, sl2);
  float sl[4] = {sc01.x, sc01.y, sc23.x, sc23.y};
  // which of the page's slots are attended (all of them on interior pages)
  if (static_cast<uint32_t>(pg - rc.pin0) >= static_cast<uint32_t>(rc.pspan)) {
    const int tok0 = pg * kPageTokens + g, tok1 = tok0 + 8;
    bool v0 = tok0 >= rc.lo_tok && tok0 < rc.hi_tok;
    bool v1 = tok1 >= rc.lo_tok && tok1 < rc.hi_tok;
    if (rc.mrow) {
      const uint32_t mw = rc.mrow[pg >> 1] >> ((pg & 1) * 16);
      v0 = v0 && ((mw >> g) & 1u);
      v1 = v1 && ((mw >> (g + 8)) & 1u);
    }
    if (!v0) sl[0] = sl[1] = -INFINITY;
    if (!v1) sl[2] = sl[3] = -INFINITY;
  }
  float pr[4];
  softmax_update<NMT, 0>(st, sl, pr);

  const uint16_t neg_sel = f16_neg_sel(t >= 2);
  uint32_t wb[NG][2];
#pragma unroll
  for (int i = 0; i < NG; ++i) {
    const float vs0 = vs0a[i], vs1 = vs1a[i];
    weights_f16x2(__fmul2_rn(make_float2(pr[0], pr[1]), make_float2(vs0, vs0)),
                  __fmul2_rn(make_float2(pr[2], pr[3]), make_float2(vs1, vs1)), neg_sel, wb[i][0], wb[i][1]);
  }
  uint32_t vw[NMT];
  // lane (g, t) = 4 g + t keeps its V words at position 8 t + (g ^ 2 t)
  const int vpos = 8 * t + (g ^ (2 * t));
#pragma unroll
  for (int q4 = 0; q4 < NMT / 4; ++q4) {
    const uint4 w = lds128(stg + 8 * D + q4 * 512 + vpos * 16);
    vw[4 * q4 + 0] = w.x;
    vw[4 * q4 + 1] = w.y;
    vw[4 * q4 + 2] = w.z;
    vw[4 * q4 + 3] = w.w;
  }
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    const uint32_t v8 = vw[mt] >> 8;
    const uint32_t a[4] = {i4x2_lo_to_f16x2(vw[mt]), i4x2_hi_to_f16x2(vw[mt]), i4x2_lo_to_f16x2(v8),
                           i4x2_hi_to_f16x2(v8)};
    mma_f16(st.o[mt], a, wb[mt >> 1][0], wb[mt >> 1][1]);
  }
}

// Position held by row r of side page j for the range, or -1 when the row is
// not attended (unused slot, or not retained by the mask).
__device__ __forceinline__ int side_row_pos(const DecodeParams &p, const RangeCtx &rc, int j, int r) {
  const int S = p.sink, R = p.recent, js = S > 0 ? 1 : 0;
  int pos;
  if (j < js) {
    pos = r < min(S, rc.L) ? r : -1;
  } else {
    const int slotr = 16 * (j - js) + r;
    const int off = ((slotr - rc.r0) % R + R) % R;
    pos = rc.r0 + off < rc.L ? rc.r0 + off : -1;
  }
  if (pos >= 0 && rc.mrow && !((rc.mrow[pos >> 5] >> (pos & 31)) & 1u)) pos = -1;
  return pos;
}

// K half of INT8 side page j: q.K on fp16 tiles (codes exact in fp16), softmax,
// and the P * scale_V weights (hi + lo) kept for the V half that follows.
template <int D>
__device__ __forceinline__ void int8k_item(const DecodeParams &p, uint32_t stg, uint32_t qsm, int j,
                                           const RangeCtx &rc, SoftmaxState<D / 16> &st, uint32_t &wb0,
                                           uint32_t &wb1, int lane) {
  constexpr int NJ = D / 16, NMT = D / 16, NW = D / 8;
  const int g = lane >> 2, t = lane & 3;
  uint32_t kw[NW];
#pragma unroll
  for (int c = 0; c < NW / 4; ++c) {
    const uint4 w = lds128(stg + c * 512 + lane * 16);
    kw[4 * c + 0] = w.x;
    kw[4 * c + 1] = w.y;
    kw[4 * c + 2] = w.z;
    kw[4 * c + 3] = w.w;
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int jj = 0; jj < NJ; jj += 2) {
    const uint4 qv = lds128(qsm + (jj / 2) * 512 + lane * 16);
    const uint32_t a0[4] = {i8x2_to_f16x2(kw[jj]), i8x2_to_f16x2(kw[NJ + jj]), i8x2_to_f16x2(kw[jj] >> 8),
                            i8x2_to_f16x2(kw[NJ + jj] >> 8)};
    mma_f16(acc, a0, qv.x, qv.y);
    const uint32_t a1[4] = {i8x2_to_f16x2(kw[jj + 1]), i8x2_to_f16x2(kw[NJ + jj + 1]),
                            i8x2_to_f16x2(kw[jj + 1] >> 8), i8x2_to_f16x2(kw[NJ + jj + 1] >> 8)};
    mma_f16(acc, a1, qv.z, qv.w);
  }
  const float k0 = half_bits_to_f32(lds16(stg + 16 * D + 2 * g)) * p.scale_log2;
  const float k1 = half_bits_to_f32(lds16(stg + 16 * D + 2 * (g + 8))) * p.scale_log2;
  const bool v0 = side_row_pos(p, rc, j, g) >= 0, v1 = side_row_pos(p, rc, j, g + 8) >= 0;
  float sl[4];
  sl[0] = v0 ? acc[0] * k0 : -INFINITY;
  sl[1] = v0 ? acc[1] * k0 : -INFINITY;
  sl[2] = v1 ? acc[2] * k1 : -INFINITY;
  sl[3] = v1 ? acc[3] * k1 : -INFINITY;
  float pr[4];
  softmax_update<NMT, 0>(st, sl, pr);
  const float s0 = half_bits_to_f32(lds16(stg + 16 * D + 32 + 2 * g));
  const float s1 = half_bits_to_f32(lds16(stg + 16 * D + 32 + 2 * (g + 8)));
  weights_f16x2(make_float2(pr[0] * s0, pr[1] * s0), make_float2(pr[2] * s1, pr[3] * s1), f16_neg_sel(t >= 2), wb0,
                wb1);
}

// V half of an INT8 side page: P.V on fp16 tiles with the weights of the K half.
template <int D>
__device__ __forceinline__ void int8v_item(uint32_t stg, SoftmaxState<D / 16> &st, uint32_t wb0, uint32_t wb1,
                                           int lane) {
  constexpr int NMT = D / 16, NW = D / 8;
  uint32_t vw[NW];
#pragma unroll
  for (int c = 0; c < NW / 4; ++c) {
    const uint4 w = lds128(stg + c * 512 + lane * 16);
    vw[4 * c + 0] = w.x;
    vw[4 * c + 1] = w.y;
    vw[4 * c + 2] = w.z;
    vw[4 * c + 3] = w.w;
  }
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    const uint32_t a[4] = {i8x2_to_f16x2(vw[2 * mt]), i8x2_to_f16x2(vw[2 * mt] >> 8),
                           i8x2_to_f16x2(vw[2 * mt + 1]), i8x2_to_f16x2(vw[2 * mt + 1] >> 8)};
    mma_f16(st.o[mt], a, wb0, wb1);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(256, 2) kv4_decode_kernel(DecodeParams p) {
  constexpr int NMT = D / 16, QB = kv4_q_bytes(D);
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthr = blockDim.x, HB = p.HB, NS = p.NS, NVB = p.NVB;
  const Kv4Layout lay = kv4_layout(D, HB, NS, NVB);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bars);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + lay.cnt);
  uint32_t *iss = reinterpret_cast<uint32_t *>(smem + lay.iss);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + lay.flag);
  int2 *desc = reinterpret_cast<int2 *>(smem + lay.desc);
  uint8_t *qsm = smem + lay.q + warp * QB;
  int *plan = reinterpret_cast<int *>(smem + lay.plan);   // [NVB + 1]
  int *wtot = reinterpret_cast<int *>(smem + lay.wtot);   // [8]
  const int stage_bytes = HB * 18 * D;
  const uint32_t smem_base = smem_u32(smem), qsm_u32 = smem_u32(qsm);

  if (tid < NS) {
    mbar_init(&full[tid], 1);
    mbar_init(&empty[tid], HB);
    fence_mbar_init();
    iss[tid] = 0;
  }
  if (tid == 0) *abort_flag = 0;
  pdl_wait();                 // inputs and cache writes of earlier grids are visible from here
  pdl_launch_dependents();    // the merge grid may queue behind the workers

  // plan[vb] = first item of virtual sequence vb: n8 INT8 items and its INT4
  // pages per virtual sequence before it
  const int cap = p.pt_stride * kPageTokens;
  const int n8 = p.int8_units ? 2 * p.np8 : 0;
  {
    const int chunk = (NVB + nthr - 1) / nthr;
    const int v0 = min(NVB, tid * chunk), v1 = min(NVB, v0 + chunk);
    int mine = 0;
    for (int vb = v0; vb < v1; ++vb) {
      int pg0, pg1;
      int4_page_range(p, vb % p.B, eff_len(p.seq_lens[vb % p.B], cap), pg0, pg1);
      mine += n8 + pg1 - pg0;
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    int run = incl - mine;
    for (int w = 0; w < warp; ++w) run += wtot[w];
    for (int vb = v0; vb < v1; ++vb) {
      plan[vb] = run;
      int pg0, pg1;
      int4_page_range(p, vb % p.B, eff_len(p.seq_lens[vb % p.B], cap), pg0, pg1);
      run += n8 + pg1 - pg0;
    }
    if (tid == nthr - 1) plan[NVB] = run;
    __syncthreads();
  }
  if (blockIdx.x == 0) {
    for (int vb = tid; vb <= NVB; vb += nthr) p.plan[vb] = plan[vb];
    for (int b = tid; b < p.B; b += nthr)
      if (p.seq_lens[b] < 0 || p.seq_lens[b] > cap) set_error(p.err, kErrCapacity);
  }
  const long long T = plan[NVB];
  if (T == 0) return;
  // at most T/2 CTAs, so that every segment keeps >= 1 item after a bound
  // inside a side page moves down by one
  const long long nc = min((long long)gridDim.x, max(1LL, T >> 1));
  if ((long long)blockIdx.x >= nc) return;
  const int c = blockIdx.x;
  auto bound = [&](long long x) -> long long {
    if (x >= T) return T;
    const int vb = upper_index(plan, NVB, x);
    const long long off = x - plan[vb];
    return (off < n8 && (off & 1)) ? x - 1 : x;
  };
  const long long x0 = bound((long long)c * T / nc), x1 = bound((long long)(c + 1) * T / nc);

  SoftmaxState<NMT> st;
  st.reset();
  RangeCtx rc{};
  int cur = -1;              // open range: region * NVB + vb
  uint32_t wb0 = 0, wb1 = 0;  // INT8 weights, K half -> V half
  int s = 0, rnd = 0;        // ring stage of the next item, and how often the ring went round
  uint32_t phase = 0;
  for (long long cx = x0; cx < x1; cx += kChunk) {
    __syncthreads();         // previous chunk consumed; empty partials written
    if (*abort_flag) break;
    const int n = static_cast<int>(min((long long)kChunk, x1 - cx));
    const int m = prepare_chunk<D>(p, plan, n8, cx, n, desc, wtot, tid, nthr);
    if (warp == 0 && lane < min(NS, m)) {
      const int sl = (s + lane) % NS;
      iss[sl] += 1;
      fence_proxy_async();
      issue_item<D>(p, desc[lane], smem + sl * stage_bytes, &full[sl]);
    }
    if (cx == x0) {
      // with the first copies in flight: first/last CTA and empty partials of
      // every range of the segment, before any warp writes a partial
      mark_ranges<G>(p, plan, n8, x0, x1, c, tid, nthr);
      __syncthreads();
    }
    int2 dnext = desc[0];
    int duty = HB - 1;       // warp that refills after the current item: (k - 1) mod HB
    for (int k = 0; k < m; ++k) {
      const int2 d = dnext;
      if (k + 1 < m) dnext = desc[k + 1];
      const int kind = d.x & 3, vb = (d.x >> 2) & 0x1FFF;
      const int pj = static_cast<int>(static_cast<uint32_t>(d.x) >> 15);
      const int rid = 2 * vb + (kind == kItemInt4 ? 1 : 0);
      if (rid != cur) {
        if (cur >= 0) write_partial<D, NMT>(p, st, p.slots + ((long long)(cur + c) * HB + warp) * p.slot_floats, lane);
        st.reset();
        cur = rid;
        const int hb = vb / p.B;
        rc.b = vb - hb * p.B;
        rc.h = hb * HB + warp;
        rc.L = eff_len(p.seq_lens[rc.b], cap);
        rc.lo_tok = p.sink;
        rc.hi_tok = rc.L - p.recent;
        rc.r0 = max(p.sink, rc.L - p.recent);
        rc.mrow = p.mask ? p.mask + ((long long)rc.b * p.Hkv + rc.h) * p.mask_stride : nullptr;
        rc.pin0 = (rc.lo_tok + kPageTokens - 1) / kPageTokens;
        rc.pspan = rc.mrow ? 0 : max(0, (rc.hi_tok >= 0 ? rc.hi_tok / kPageTokens : -1) - rc.pin0);
        load_q<D, G>(p, rc.b, rc.h, kind == kItemInt4, qsm, lane);
      }
      const bool ok = p.wait_cap != 0 && mbar_wait_bounded(&full[s], (phase >> s) & 1u, p.wait_cap);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          set_error(p.err, kErrTimeout);
          *abort_flag = 1;
        }
        break;
      }
      phase ^= 1u << s;
      const uint32_t stg = smem_base + s * stage_bytes + warp * 18 * D;
      if (kind == kItemInt4) int4_item<D, G>(p, stg, qsm_u32, pj, rc, st, lane);
      else if (kind == kItemInt8K) int8k_item<D>(p, stg, qsm_u32, pj, rc, st, wb0, wb1, lane);
      else int8v_item<D>(stg, st, wb0, wb1, lane);
      // release the stage (no result to wait for); one warp per item, in
      // turn, refills the stage of the item before this one once every warp
      // has released it -- normally long done by then
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (k > 0 && k - 1 + NS < m && duty == warp) {
        const int sp = s == 0 ? NS - 1 : s - 1;
        const int up = s == 0 ? rnd - 1 : rnd;   // how often stage sp was used before that item
        const bool freed = mbar_wait_bounded(&empty[sp], static_cast<uint32_t>(up) & 1u, p.wait_cap);
        if (!__all_sync(0xffffffffu, freed)) {
          if (lane == 0) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
          }
          break;
        }
        if (lane == 0) {
          fence_proxy_async();
          iss[sp] += 1;
          issue_item<D>(p, desc[k - 1 + NS], smem + sp * stage_bytes, &full[sp]);
        }
      }
      if (++s == NS) {
        s = 0;
        ++rnd;
      }
      if (++duty == HB) duty = 0;
    }
  }
  __syncthreads();
  if (*abort_flag) {
    // a copy never landed: wait (bounded) for every copy still in flight, then
    // leave; this CTA's ranges keep their empty partials
    if (tid < NS && iss[tid] > 0) mbar_wait_bounded(&full[tid], (iss[tid] - 1) & 1u, kDefaultWaitCycles);
    return;
  }
  if (cur >= 0) write_partial<D, NMT>(p, st, p.slots + ((long long)(cur + c) * HB + warp) * p.slot_floats, lane);
}

// ---------------------------------------------------------------------------
// Masked decode with the retained rows gathered on chip (Shadow Mask
// Distillation, sec. 1 and Figure 1: the mask is applied inside attention).
// One CTA per (sequence, KV head). Its retained INT4-region positions, in
// order, form "compact pages" of 16 rows; a warp at a time gathers one compact
// page of the head into a shared-memory image of the ordinary head-block
// layout (the K rows, the K and V scale rows, and the 16-byte pieces of the
// V block that hold each row's bytes, loaded with the lanes spread over few
// lines per instruction; the V bytes are moved to the row's place in the
// fragment order) and runs the ordinary page computation on it, with the next
// page's rows already in flight. Rows past the count are zero and not
// attended. The head's INT8 side pages (sink and recent window, under the
// same mask) go through the same image and softmax state. Reads and work of
// the INT4 region follow the retained count; nothing is written back but one
// (m, l, o) partial per warp, in the layout of kv4_decode_partials.
// ---------------------------------------------------------------------------
constexpr int kMaskedWarps = 4, kMaskedChunk = 4096;

__device__ __forceinline__ uint32_t word_bits_in(int w, int c0, int c1) {
  const int a = max(c0 - 32 * w, 0), z = min(c1 - 32 * w, 32);
  if (z <= a) return 0u;
  return (z >= 32 ? 0xFFFFFFFFu : ((1u << z) - 1u)) & ~((1u << a) - 1u);
}

// The partial of a warp's softmax state for query heads h*G .. h*G+G-1 in the
// layout of kv4_decode_partials: m (log2 units), l, two unused words, o.
template <int D, int NMT>
__device__ __forceinline__ void write_cp_partial(int G, SoftmaxState<NMT> &st, float *pr, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    st.l[0] += __shfl_xor_sync(0xffffffffu, st.l[0], o);
    st.l[1] += __shfl_xor_sync(0xffffffffu, st.l[1], o);
  }
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
    for (int c = 0; c < 4; ++c) st.o[mt][c] += __shfl_xor_sync(0xffffffffu, st.o[mt][c], 2);
  if (t < 2) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int head = 2 * t + c;
      if (head < G) {
        const bool nonempty = st.l[c] > 0.f;
        const float inv = nonempty ? 1.f / st.l[c] : 0.f;
        float *ph = pr + head * (D + 4);
#pragma unroll
        for (int mt = 0; mt < NMT; ++mt) {
          ph[4 + 16 * mt + g] = st.o[mt][c] * inv;
          ph[4 + 16 * mt + g + 8] = st.o[mt][c + 2] * inv;
        }
        if (g == 0) {
          ph[0] = nonempty ? st.m[c] : -INFINITY;
          ph[1] = st.l[c];
          ph[2] = 0.f;
          ph[3] = 0.f;
        }
      }
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kMaskedWarps * 32, 4) masked_decode_kernel(DecodeParams p, GatherParams gp,
                                                                             float *parts) {
  constexpr int NMT = D / 16, HEAD = 18 * D, KROW = D / 2, QB = kv4_q_bytes(D);
  extern __shared__ __align__(128) uint8_t msm[];
  int *list = reinterpret_cast<int *>(msm);                 // [kMaskedChunk]
  uint8_t *qarea = msm + 4 * kMaskedChunk;                 // [QB] INT4 query format, shared by the warps
  uint8_t *q8area = qarea + QB;                            // [QB] INT8 query format
  uint8_t *img_all = q8area + QB;                          // [kMaskedWarps][HEAD]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NT = kMaskedWarps * 32;
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x, b = row / p.Hkv, h = row - b * p.Hkv;
  const int cap = p.pt_stride * kPageTokens;
  int L = p.seq_lens[b];
  L = L < 0 ? 0 : (L > cap ? cap : L);
  const int c0 = min(p.sink, L), c1 = max(c0, L - p.recent);
  const int n = gp.counts[row];
  const int npg = (n + kPageTokens - 1) / kPageTokens;
  const uint32_t *mrow = gp.mask + (long long)row * gp.mask_stride;
  const int *wpre = gp.wpre + (long long)row * gp.words;
  const int nw = (L + 31) / 32;
  uint8_t *im = img_all + warp * HEAD;
  if (warp == 0) load_q<D, G>(p, b, h, true, qarea, lane);
  if (warp == 1 % kMaskedWarps && p.int8_units) load_q<D, G>(p, b, h, false, q8area, lane);
  SoftmaxState<NMT> st;
  st.reset();
  RangeCtx rc{};
  rc.b = b;
  rc.h = h;
  rc.L = n;
  rc.lo_tok = 0;
  rc.hi_tok = n;   // rows of compact page j are retained indices 16 j .. 16 j + 15
  rc.mrow = nullptr;
  rc.pin0 = 0;
  rc.pspan = n / kPageTokens;
  const uint32_t im_u32 = smem_u32(im), q_u32 = smem_u32(qarea);
  const int i = lane & 15, half = lane >> 4;
  for (int t0 = 0; t0 < npg * kPageTokens; t0 += kMaskedChunk) {
    const int t1 = min(t0 + kMaskedChunk, n);
    __syncthreads();   // the query is in place; the previous chunk's list is no longer read
    for (int w = tid; w < nw; w += NT) {
      const int hi_ = wpre[w], lo_ = w > 0 ? wpre[w - 1] : 0;   // retained indices [lo_, hi_) lie in word w
      if (hi_ <= t0 || lo_ >= t1) continue;
      uint32_t bits = mrow[w] & word_bits_in(w, c0, c1);
      for (int k = lo_; bits; ++k) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        if (k >= t0 && k < t1) list[k - t0] = 32 * w + bit;
      }
    }
    __syncthreads();
    const int pg_end = min(npg, (t0 + kMaskedChunk) / kPageTokens);
    // Software pipeline over the warp's compact pages j, j + W, ...: the page
    // ids of page j + 2W and the row data of page j + W are in flight while
    // page j is attended. Row i of a compact page is retained position
    // 16 j + i; lanes i and i + 16 look its page up, as pr = page * 16 + slot
    // (-1: no position, or a page id out of range).
    auto row_page = [&](int jj) -> int {
      const int t = kPageTokens * jj + i;
      if (jj >= pg_end || t >= n) return -1;
      const int pos = list[t - t0];
      const int page = p.page_table[(long long)b * p.pt_stride + pos / kPageTokens];
      if (page < 0 || page >= p.num_pages) {
        if (half == 0) set_error(p.err, kErrBounds);
        return -1;   // the row stays zero
      }
      return page * kPageTokens + pos % kPageTokens;
    };
    // The loads are spread so that one warp instruction touches few 128-byte
    // lines: K, 16-byte piece Q = 32u + lane of the page's 16 rows (D/32 per
    // row); V, piece lane % 8 of the 128-byte group span of row 4k + lane/8 in
    // each 512-byte block (k < 4); scales, lane (i, half): the K (half 0) or V
    // (half 1) scale row of row i.
    // V layout: word (m/4)*128 + 4*P + m%4 with P = 8*tt + (g ^ 2*tt),
    // tt = (r%8)/2, holds byte 2*(r%2) + r/8 of row r; a row's bytes in a
    // 512-byte block lie in the 8 pieces of its group span [128 tt, 128 tt + 128).
    constexpr int KPR = D / 32, NK = D / 64, NV = D / 16;
    uint4 kc[NK], vp[NV];
    uint2 sc = make_uint2(0, 0);
    auto row_src = [&](int pr) -> const uint8_t * {
      return p.pool + (long long)(pr / kPageTokens) * p.page_bytes + (long long)h * p.head_bytes;
    };
    auto issue_rows = [&](int prl) {   // prl: this lane's row (lane & 15)
#pragma unroll
      for (int u = 0; u < NK; ++u) {
        const int q = 32 * u + lane, row = q / KPR, y = q % KPR;
        const int pr = __shfl_sync(0xffffffffu, prl, row);
        if (pr >= 0) kc[u] = __ldg(reinterpret_cast<const uint4 *>(row_src(pr) + (pr % kPageTokens) * KROW) + y);
      }
      if (prl >= 0) {
        const int sb = half ? 17 * D : 16 * D;   // K scales (half 0) or V scales (half 1)
        const uint8_t *src = row_src(prl) + sb + (prl % kPageTokens) * (D / 16);
        if constexpr (D == 128) sc = __ldg(reinterpret_cast<const uint2 *>(src));
        else sc.x = __ldg(reinterpret_cast<const uint32_t *>(src));
      }
      // V: rows k*4 + lane/8 (k < 4), each over its D/64 blocks
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int pr = __shfl_sync(0xffffffffu, prl, 4 * k + (lane >> 3));
        if (pr >= 0) {
          const uint4 *src = reinterpret_cast<const uint4 *>(row_src(pr) + 8 * D + 128 * ((pr % 8) / 2)) + (lane & 7);
#pragma unroll
          for (int m4 = 0; m4 < D / 64; ++m4) vp[4 * m4 + k] = __ldg(src + 32 * m4);
        }
      }
    };
    int j = t0 / kPageTokens + warp;
    int pra = row_page(j), prb = row_page(j + kMaskedWarps);
    issue_rows(pra);
    for (; j < pg_end; j += kMaskedWarps) {
      const int prc = row_page(j + 2 * kMaskedWarps);
      // the image of page j: zero first unless every row holds a position
      if (!__all_sync(0xffffffffu, pra >= 0)) {
        for (int q = lane; q < HEAD / 16; q += 32) reinterpret_cast<uint4 *>(im)[q] = make_uint4(0, 0, 0, 0);
        __syncwarp();
      }
#pragma unroll
      for (int u = 0; u < NK; ++u) {
        const int q = 32 * u + lane, row = q / KPR, y = q % KPR;
        if (__shfl_sync(0xffffffffu, pra, row) >= 0) reinterpret_cast<uint4 *>(im + row * KROW)[y] = kc[u];
      }
      if (pra >= 0) {
        const int sb = half ? 17 * D : 16 * D;
        if constexpr (D == 128) *reinterpret_cast<uint2 *>(im + sb + i * (D / 16)) = sc;
        else *reinterpret_cast<uint32_t *>(im + sb + i * (D / 16)) = sc.x;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = 4 * k + (lane >> 3);
        const int pr = __shfl_sync(0xffffffffu, pra, row);
        if (pr >= 0) {
          // source piece x = lane % 8 of the row's span holds g = x ^ 2 tt;
          // the row's byte of word c goes to the image piece of g for row `row`
          const int r = pr % kPageTokens, tts = (r % 8) / 2, g = (lane & 7) ^ (2 * tts);
          const int ttd = (row % 8) / 2, sh_src = 8 * (2 * (r % 2) + r / 8), b_dst = 2 * (row % 2) + row / 8;
          uint8_t *dst = im + 8 * D + 16 * (8 * ttd + (g ^ (2 * ttd))) + b_dst;
#pragma unroll
          for (int m4 = 0; m4 < D / 64; ++m4) {
            const uint4 w = vp[4 * m4 + k];
            dst[512 * m4 + 0] = static_cast<uint8_t>(w.x >> sh_src);
            dst[512 * m4 + 4] = static_cast<uint8_t>(w.y >> sh_src);
            dst[512 * m4 + 8] = static_cast<uint8_t>(w.z >> sh_src);
            dst[512 * m4 + 12] = static_cast<uint8_t>(w.w >> sh_src);
          }
        }
      }
      __syncwarp();
      // the rows of page j + W load while page j is attended
      issue_rows(prb);
      int4_item<D, G>(p, im_u32, q_u32, j, rc, st, lane);
      __syncwarp();
      pra = prb;
      prb = prc;
    }
  }
  // The INT8 region: this head's side pages, a warp per side page, the K half
  // and then the V half through the page image, into the same softmax state.
  if (p.int8_units) {
    __syncthreads();   // the INT8 query is in place
    RangeCtx r8{};
    r8.b = b;
    r8.h = h;
    r8.L = L;
    r8.lo_tok = p.sink;
    r8.hi_tok = L - p.recent;
    r8.r0 = max(p.sink, L - p.recent);
    r8.mrow = mrow;
    const uint32_t q8_u32 = smem_u32(q8area);
    const uint8_t *sbase = p.side + ((long long)b * p.Hkv + h) * p.side_stride;
    constexpr int KHALF = 16 * D + 64, VHALF = 16 * D, PAGE8 = 32 * D + 64;
    uint32_t wb0 = 0, wb1 = 0;
    for (int j = warp; j < p.np8; j += kMaskedWarps) {
      if (!side_page_attended(j, L, p.sink, p.recent)) continue;
      const uint4 *ks = reinterpret_cast<const uint4 *>(sbase + (long long)j * PAGE8);
      for (int q = lane; q < KHALF / 16; q += 32) reinterpret_cast<uint4 *>(im)[q] = __ldg(ks + q);
      __syncwarp();
      int8k_item<D>(p, im_u32, q8_u32, j, r8, st, wb0, wb1, lane);
      __syncwarp();
      const uint4 *vs = reinterpret_cast<const uint4 *>(sbase + (long long)j * PAGE8 + KHALF);
      for (int q = lane; q < VHALF / 16; q += 32) reinterpret_cast<uint4 *>(im)[q] = __ldg(vs + q);
      __syncwarp();
      int8v_item<D>(im_u32, st, wb0, wb1, lane);
      __syncwarp();
    }
  }
  write_cp_partial<D, NMT>(G, st, parts + (((long long)warp * p.B + b) * p.Hq + h * G) * (D + 4), lane);
}

size_t masked_decode_smem(int D) { return 4 * kMaskedChunk + 2 * kv4_q_bytes(D) + (size_t)kMaskedWarps * 18 * D; }

template <int D>
static cudaError_t launch_masked_d(const DecodeParams &p, const GatherParams &g, float *parts, cudaStream_t s) {
  const size_t smem = masked_decode_smem(D);
  auto kern = p.G == 1 ? masked_decode_kernel<D, 1> : (p.G == 2 ? masked_decode_kernel<D, 2> : masked_decode_kernel<D, 4>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(p.B * p.Hkv), dim3(kMaskedWarps * 32), smem, s, p, g, parts);
}

cudaError_t launch_masked_decode(const DecodeParams &p, const GatherParams &g, float *parts, int D, cudaStream_t s) {
  if (p.B * p.Hkv == 0) return cudaSuccess;
  return D == 128 ? launch_masked_d<128>(p, g, parts, s) : launch_masked_d<64>(p, g, parts, s);
}

int masked_decode_warps() { return kMaskedWarps; }

// ---------------------------------------------------------------------------
// bf16 pages of one piece (the uncompressed comparison).
// Head block in a page: K[16][D] bf16 then V[16][D] bf16. Each row is copied
// to a padded shared-memory row so ldmatrix reads are conflict-free.
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ bool bf16_piece(const DecodeParams &p, int b, int h, int L, int pg0, int pg1, uint8_t *wsm,
                           uint64_t *bars, uint32_t &phase, float *slot, int lane) {
  using C = Bf16Cfg<D>;
  constexpr int NS = C::NS, NK = D / 16, NMT = D / 16, ROWB = C::ROWB;
  const int g = lane >> 2, t = lane & 3;

  uint32_t qf[NK][2];
  {
    const int head = g & 3;
    const bool hv = head < G;
    const uint32_t *qh =
        reinterpret_cast<const uint32_t *>(p.q + ((long long)b * p.Hq + h * G + (hv ? head : 0)) * D);
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      qf[j][0] = hv ? qh[(16 * j + 2 * t) / 2] : 0u;
      qf[j][1] = hv ? qh[(16 * j + 2 * t + 8) / 2] : 0u;
    }
  }
  const int32_t *ptrow = p.page_table + (long long)b * p.pt_stride;
  const uint8_t *hbase = p.pool + (long long)h * p.head_bytes;
  const float2 neg_sel = t >= 2 ? make_float2(-1.f, -1.f) : make_float2(0.f, 0.f);

  SoftmaxState<NMT> st;
  st.reset();
  PageCursor cur;
  cur.pg1 = pg1;
  cur.cursor = pg0;
  load_batch(cur, pg0, ptrow, 0, L, nullptr, p, lane);

  // lane < 16 copies K row `lane`, lane >= 16 copies V row `lane - 16`
  const int crow = lane & 15;
  const long long src_off = (lane < 16 ? 0 : 32LL * D) + (long long)crow * 2 * D;
  const int dst_off = (lane < 16 ? 0 : kPageTokens * ROWB) + crow * ROWB;
  auto issue = [&](int s, int pid) {
    if (lane == 0) mbar_arrive_expect_tx(&bars[s], 64 * D);
    __syncwarp();
    bulk_g2s(wsm + s * C::STAGE + dst_off, hbase + (long long)pid * p.page_bytes + src_off, 2 * D, &bars[s]);
  };

  Ring<NS> ring;
  ring.s = 0;
#pragma unroll
  for (int k = 0; k < NS; ++k) {
    int pid = -1;
    ring.item[k] = next_page(cur, pid, ptrow, 0, L, nullptr, p, lane);
    if (ring.item[k] >= 0) issue(k, pid);
  }

  const int mi = lane >> 3, ri = lane & 7;
  while (ring.item[0] >= 0) {
    if (!ring_wait<NS>(ring, bars, phase, p.wait_cap, p.err, lane)) return false;
    const uint32_t stg = smem_u32(wsm + ring.s * C::STAGE);
    const int pg = ring.item[0];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      uint32_t a[4];
      ldmatrix_x4(a, stg + (ri + (mi & 1) * 8) * ROWB + (16 * j + (mi >> 1) * 8) * 2);
      mma_bf16(acc, a, qf[j][0], qf[j][1]);
    }
    const int tok0 = pg * kPageTokens + g, tok1 = tok0 + 8;
    const bool v0 = tok0 < L, v1 = tok1 < L;
    float sl[4];
    sl[0] = v0 ? acc[0] * p.scale_log2 : -INFINITY;
    sl[1] = v0 ? acc[1] * p.scale_log2 : -INFINITY;
    sl[2] = v1 ? acc[2] * p.scale_log2 : -INFINITY;
    sl[3] = v1 ? acc[3] * p.scale_log2 : -INFINITY;
    float pr[4];
    softmax_update<NMT, 8>(st, sl, pr);
    uint32_t wb0, wb1;
    weights_bf16(make_float2(pr[0], pr[1]), make_float2(pr[2], pr[3]), neg_sel, wb0, wb1);
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a, stg + kPageTokens * ROWB + (ri + (mi >> 1) * 8) * ROWB + (16 * mt + (mi & 1) * 8) * 2);
      mma_bf16(st.o[mt], a, wb0, wb1);
    }
    __syncwarp();
    int pid = -1;
    const int nxt = next_page(cur, pid, ptrow, 0, L, nullptr, p, lane);
    if (nxt >= 0) {
      fence_proxy_async();
      issue(ring.s, pid);
    }
    ring.push_rotate(nxt);
  }
  write_partial<D, NMT>(p, st, slot, lane);
  return true;
}

// ---------------------------------------------------------------------------
// bf16 comparison kernel: persistent warp workers over the flat space of
// (sequence, KV head) page ranges, weighted equally per page.
// ---------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kWarps * 32, 4) bf16_decode_kernel(DecodeParams p) {
  using C = Bf16Cfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t *wsm = smem + warp * C::WARP_SMEM;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kWarps * C::WARP_SMEM) + warp * C::NS;
  int *plan = reinterpret_cast<int *>(smem + C::RINGS);   // [B + 1]
  __shared__ int wtot[kWarps];

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < C::NS; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  pdl_wait();
  pdl_launch_dependents();

  // plan[b] = sum over b' < b of (pages of b') * Hkv, computed by the CTA
  const int cap = p.pt_stride * kPageTokens;
  const int chunk = (p.B + kWarps * 32 - 1) / (kWarps * 32);
  const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
  int mine = 0;
  for (int b = b0; b < b1; ++b) mine += (eff_len(p.seq_lens[b], cap) + kPageTokens - 1) / kPageTokens;
  mine *= p.Hkv;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  int run = incl - mine;
  for (int w = 0; w < warp; ++w) run += wtot[w];
  for (int b = b0; b < b1; ++b) {
    plan[b] = run;
    run += (eff_len(p.seq_lens[b], cap) + kPageTokens - 1) / kPageTokens * p.Hkv;
  }
  if (tid == kWarps * 32 - 1) plan[p.B] = run;
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int b = tid; b <= p.B; b += kWarps * 32) {
      p.plan[b] = plan[b];
      if (b < p.B && (p.seq_lens[b] < 0 || p.seq_lens[b] > cap)) set_error(p.err, kErrCapacity);
    }
  }

  const long long wid = (long long)blockIdx.x * kWarps + warp;
  const long long T4 = plan[p.B];
  const long long NWk = active_workers(p.num_workers, 0, T4);
  if (wid >= NWk) return;
  long long x = worker_first_item(wid, NWk, 0, T4);
  const long long z = worker_first_item(wid + 1, NWk, 0, T4);
  const long long nbh = (long long)p.B * p.Hkv;
  if (x >= z) return;

  uint32_t phase = 0;
  int b = 0;
  bool located = false;
  while (x < z) {
    const int y = static_cast<int>(x);
    if (!located) {   // sequence holding y: largest b with plan[b] <= y
      int lo = 0, hi = p.B - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (plan[mid] <= y) lo = mid;
        else hi = mid - 1;
      }
      b = lo;
      located = true;
    }
    while (plan[b + 1] <= y) ++b;
    const int per = (plan[b + 1] - plan[b]) / p.Hkv;
    const int h = (y - plan[b]) / per;
    const int off = (y - plan[b]) % per;
    const long long e = min(z, (long long)plan[b] + (long long)(h + 1) * per);
    const int L = eff_len(p.seq_lens[b], cap);
    float *slot = p.slots + (nbh + (long long)b * p.Hkv + h + wid) * p.slot_floats;
    if (lane == 0) {
      if (off == 0) p.first[nbh + (long long)b * p.Hkv + h] = static_cast<int>(wid);
      if (e == (long long)plan[b] + (long long)(h + 1) * per) p.last[nbh + (long long)b * p.Hkv + h] = static_cast<int>(wid);
    }
    if (!bf16_piece<D, G>(p, b, h, L, off, off + static_cast<int>(e - x), wsm, bars, phase, slot, lane)) return;
    x = e;
  }
}

// ---------------------------------------------------------------------------
// Host side launchers.
// ---------------------------------------------------------------------------
int kv4_smem_bytes(int D, int HB, int NS, int NVB) { return kv4_layout(D, HB, NS, NVB).total; }

int bf16_smem_bytes(int D, int B) {
  return (D == 128 ? Bf16Cfg<128>::RINGS : Bf16Cfg<64>::RINGS) + 4 * (B + 1);
}

template <int D, int G>
static cudaError_t kv4_prepare_one(int HB, int smem, int *blocks_per_sm) {
  if (blocks_per_sm == nullptr)
    return cudaFuncSetAttribute(kv4_decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, kv4_decode_kernel<D, G>, HB * 32, smem);
}

static cudaError_t kv4_prepare(int D, int G, int HB, int smem, int *blocks_per_sm) {
  if (D == 128) {
    switch (G) {
      case 1: return kv4_prepare_one<128, 1>(HB, smem, blocks_per_sm);
      case 2: return kv4_prepare_one<128, 2>(HB, smem, blocks_per_sm);
      case 4: return kv4_prepare_one<128, 4>(HB, smem, blocks_per_sm);
    }
  } else if (D == 64) {
    switch (G) {
      case 1: return kv4_prepare_one<64, 1>(HB, smem, blocks_per_sm);
      case 2: return kv4_prepare_one<64, 2>(HB, smem, blocks_per_sm);
      case 4: return kv4_prepare_one<64, 4>(HB, smem, blocks_per_sm);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t kv4_decode_set_smem_limit(int D, int G, int smem) { return kv4_prepare(D, G, 1, smem, nullptr); }

cudaError_t kv4_decode_occupancy(int D, int G, int HB, int smem, int *blocks_per_sm) {
  return kv4_prepare(D, G, HB, smem, blocks_per_sm);
}

template <int D, int G>
static cudaError_t bf16_prepare_one(DecodeLaunch *out) {
  const int smem_max = bf16_smem_bytes(D, kMaxBatch);
  cudaError_t e = cudaFuncSetAttribute(bf16_decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_max);
  if (e != cudaSuccess) return e;
  int nb = 0;
  // occupancy at batches up to 1024 sequences; larger batches only add plan bytes
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, bf16_decode_kernel<D, G>, kWarps * 32,
                                                    bf16_smem_bytes(D, 1024));
  if (e != cudaSuccess) return e;
  out->smem_bytes = bf16_smem_bytes(D, 1024);
  out->blocks_per_sm = nb > 0 ? nb : 1;
  return cudaSuccess;
}

cudaError_t bf16_decode_prepare(int D, int G, DecodeLaunch *out) {
  if (D == 128) {
    switch (G) {
      case 1: return bf16_prepare_one<128, 1>(out);
      case 2: return bf16_prepare_one<128, 2>(out);
      case 4: return bf16_prepare_one<128, 4>(out);
    }
  } else if (D == 64) {
    switch (G) {
      case 1: return bf16_prepare_one<64, 1>(out);
      case 2: return bf16_prepare_one<64, 2>(out);
      case 4: return bf16_prepare_one<64, 4>(out);
    }
  }
  return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t launch_kv4_d(const DecodeParams &p, cudaStream_t stream) {
  const dim3 grid(p.n_cta), block(p.HB * 32);
  const int smem = kv4_smem_bytes(D, p.HB, p.NS, p.NVB);
  switch (p.G) {
    case 1: return launch_pdl(kv4_decode_kernel<D, 1>, grid, block, smem, stream, p);
    case 2: return launch_pdl(kv4_decode_kernel<D, 2>, grid, block, smem, stream, p);
    default: return launch_pdl(kv4_decode_kernel<D, 4>, grid, block, smem, stream, p);
  }
}

template <int D>
static cudaError_t launch_bf16_d(const DecodeParams &p, cudaStream_t stream) {
  const dim3 grid(p.num_workers / kWarps), block(kWarps * 32);
  const int smem = bf16_smem_bytes(D, p.B);
  switch (p.G) {
    case 1: return launch_pdl(bf16_decode_kernel<D, 1>, grid, block, smem, stream, p);
    case 2: return launch_pdl(bf16_decode_kernel<D, 2>, grid, block, smem, stream, p);
    default: return launch_pdl(bf16_decode_kernel<D, 4>, grid, block, smem, stream, p);
  }
}

cudaError_t launch_decode(const DecodeParams &p, int D, bool bf16, cudaStream_t stream, cudaEvent_t ev0,
                          cudaEvent_t ev1) {
  if (ev0) cudaEventRecord(ev0, stream);
  cudaError_t e;
  if (bf16) e = D == 128 ? launch_bf16_d<128>(p, stream) : launch_bf16_d<64>(p, stream);
  else e = D == 128 ? launch_kv4_d<128>(p, stream) : launch_kv4_d<64>(p, stream);
  if (e != cudaSuccess) return e;
  if (ev1) cudaEventRecord(ev1, stream);
  return launch_merge(p, D, bf16, stream);
}

}  // namespace kv4
