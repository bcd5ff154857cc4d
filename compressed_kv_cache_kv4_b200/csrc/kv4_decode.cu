// kv4_decode.cu -- decode-step attention over the KV4-RL compressed cache.
//
// KV4-RL review, sec. 3: the INT4 region and the INT8-protected region (first
// 16 and last 128 positions) are attended independently; their partial
// (max, sum, output) triples are combined by an exact softmax merge, so no
// full-precision cache is rebuilt. Shadow Mask Distillation, sec. 1 / Figure 1:
// a retained-position mask is applied inside attention.
//
// Two launches on the caller's stream:
//   decode_kernel  persistent warp workers over one flat, weighted item space:
//                  first every (sequence, KV head)'s INT8 side pages (16 rows
//                  each; a sink page and recent/16 ring pages), then every
//                  (sequence, KV head)'s INT4 pages. Each worker owns one
//                  contiguous segment. Pages stream through a per-warp ring of
//                  shared-memory stages filled by 1-D bulk copies (TMA engine,
//                  mbarrier completion, bounded waits). Per page, q.K and P.V
//                  are small tensor-core tiles (mma.sync m16n8k16, fp32
//                  accumulate): q.K of INT4 pages on bf16 tiles (codes
//                  unpacked in registers), P.V of INT4 pages and all of the
//                  INT8 pages on fp16 tiles (the codes are exact in fp16).
//                  Each worker writes one (m, l, o) partial per
//                  (region, sequence, KV head) piece of its segment.
//   merge_kernel   (kv4_merge.cu) one warp per (sequence, query head) merges
//                  its partials exactly.
//
// Softmax bookkeeping runs in the log2 domain (scores scaled by tau*log2 e).
// P.V takes P*scale_V as two fp16 terms (hi + lo), which carries 22
// significant bits into fp32 accumulation; the running max is exact (P <= 1),
// so P*scale_V stays in the fp16 range.
#include <math.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

#ifndef KV4_INT4_STAGES
#define KV4_INT4_STAGES 4
#endif
#ifndef KV4_MIN_BLOCKS
#define KV4_MIN_BLOCKS 4
#endif

template <int D, bool kBF16>
struct Cfg {
  static constexpr int NS = kBF16 ? 3 : KV4_INT4_STAGES;    // stages per warp
  static constexpr int ROWB = 2 * D + 16;                   // padded bf16 row in shared memory
  static constexpr int STAGE = kBF16 ? 2 * kPageTokens * ROWB : 18 * D;
  static constexpr int WARP_SMEM = NS * STAGE;
  // per-warp query operands: [chunk][lane][16 bytes]; INT4 pieces use D/32
  // chunks of q fragments and (D/32 + 1)/2 chunks of accumulator starts,
  // INT8 pieces D/32 chunks of fp16 q fragments
  static constexpr int QCHUNKS = kBF16 ? 0 : D / 32 + (D / 32 + 1) / 2;
  static constexpr int QBYTES = QCHUNKS * 512;
  static constexpr int RINGS = kWarps * (WARP_SMEM + NS * 8 + QBYTES);
};


// ---------------------------------------------------------------------------
// Partial slot: m[G] | l[G] | pad | o[G][D]   (m in log2 units, o normalised)
// ---------------------------------------------------------------------------

// Online-softmax state of one warp for the 8 MMA columns (4 "hi" + 4 "lo"
// copies of up to 4 query heads). Thread (g, t) owns columns 2t and 2t+1.
template <int NMT>
struct SoftmaxState {
  float m[2], l[2];
  float o[NMT][4];   // O^T fragments: rows = head_dim, columns = MMA columns
  __device__ __forceinline__ void reset() {
    m[0] = m[1] = -INFINITY;
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
  const float2 r = make_float2(st.m[0] == -INFINITY ? 0.f : st.m[0], st.m[1] == -INFINITY ? 0.f : st.m[1]);
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

// fp16 variant of weights_bf16 (hi + lo carry 22 significant bits).
__device__ __forceinline__ void weights_f16x2(float2 w01, float2 w23, float2 neg_sel, uint32_t &b0, uint32_t &b1) {
  const uint32_t h01 = pack_f16x2(w01.x, w01.y);
  const uint32_t h23 = pack_f16x2(w23.x, w23.y);
  const float2 r01 = __ffma2_rn(neg_sel, f16x2_to_f32x2(h01), w01);
  const float2 r23 = __ffma2_rn(neg_sel, f16x2_to_f32x2(h23), w23);
  b0 = movmatrix_t(pack_f16x2(r01.x, r01.y));
  b1 = movmatrix_t(pack_f16x2(r23.x, r23.y));
}

__device__ __forceinline__ void weights_f16(float w0, float w1, float w2, float w3, float lo_sel, uint32_t &b0,
                                            uint32_t &b1) {
  uint32_t h01 = pack_f16x2(w0, w1);
  uint32_t h23 = pack_f16x2(w2, w3);
  h01 = pack_f16x2(fmaf(-lo_sel, f16lo_to_f32(h01), w0), fmaf(-lo_sel, f16hi_to_f32(h01), w1));
  h23 = pack_f16x2(fmaf(-lo_sel, f16lo_to_f32(h23), w2), fmaf(-lo_sel, f16hi_to_f32(h23), w3));
  b0 = movmatrix_t(h01);
  b1 = movmatrix_t(h23);
}

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

// ---------------------------------------------------------------------------
// INT4 pages of one piece (sequence b, KV head h, pages [pg0, pg1)).
// Returns false if a bounded wait ran out (the worker must stop).
//
// q.K: A = K codes (rows = slots g, g+8), B = q. Per group two MMAs: a bf16
// one over elements 32i+8t+{0, 4} (k-slots 2t, 2t+1) and {2, 6} (2t+8, 2t+9),
// whose codes enter as 136 + c, and an fp16 one over {1, 5} and {3, 7}, whose
// codes enter as 72 + c -- the nibble order of the K words; one shift by 8
// serves both. The accumulator starts at -(136 * sum of q over the even
// elements + 72 * sum over the odd ones), which removes the offsets.
// P.V: A = V^T codes (rows = head_dim, k = slots), B = P * scale_V (hi + lo).
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ bool int4_piece(const DecodeParams &p, int b, int h, int L, int pg0, int pg1, uint8_t *wsm,
                           uint64_t *bars, uint8_t *qsm, uint32_t &phase, float *slot, int lane) {
  using C = Cfg<D, false>;
  constexpr int NS = C::NS, NG = D / 32, NMT = D / 16, NSW = (NG + 1) / 2;
  const int g = lane >> 2, t = lane & 3;

  // q as the B operand, and -136 * (sum of q over group i) for columns 2t and
  // 2t+1, parked in the warp's shared-memory q area for the whole piece
  {
    const int head = g & 3;
    const bool hv = head < G;
    const uint4 *qh = reinterpret_cast<const uint4 *>(p.q + ((long long)b * p.Hq + h * G + (hv ? head : 0)) * D);
    float qinit[NG][2];
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      const uint4 e = hv ? qh[4 * i + t] : make_uint4(0, 0, 0, 0);
      // e.x = (e0, e1), e.y = (e2, e3), e.z = (e4, e5), e.w = (e6, e7)
      // e.x = (e0, e1), e.y = (e2, e3), e.z = (e4, e5), e.w = (e6, e7). Codes of
      // even elements enter a bf16 MMA as 136 + c, codes of odd elements an
      // fp16 MMA as 72 + c (see the q.K below), so the bf16 pairs (e0, e4),
      // (e2, e6) and the fp16 pairs (e1, e5), (e3, e7) are stored.
      const float e0 = bf16lo_to_f32(e.x), e1 = bf16hi_to_f32(e.x), e2 = bf16lo_to_f32(e.y), e3 = bf16hi_to_f32(e.y);
      const float e4 = bf16lo_to_f32(e.z), e5 = bf16hi_to_f32(e.z), e6 = bf16lo_to_f32(e.w), e7 = bf16hi_to_f32(e.w);
      *reinterpret_cast<uint4 *>(qsm + i * 512 + lane * 16) =
          make_uint4(__byte_perm(e.x, e.z, 0x5410), __byte_perm(e.y, e.w, 0x5410), pack_f16x2(e1, e5),
                     pack_f16x2(e3, e7));
      float part = -136.f * ((e0 + e2) + (e4 + e6)) - 72.f * ((e1 + e3) + (e5 + e7));
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      // lanes 4c..4c+3 hold the group offset of column c; this lane needs columns 2t, 2t+1
      qinit[i][0] = __shfl_sync(0xffffffffu, part, 8 * t);
      qinit[i][1] = __shfl_sync(0xffffffffu, part, 8 * t + 4);
    }
#pragma unroll
    for (int c = 0; c < (NG + 1) / 2; ++c) {
      const float a0 = qinit[2 * c][0], a1 = qinit[2 * c][1];
      const float a2 = 2 * c + 1 < NG ? qinit[(2 * c + 1) % NG][0] : 0.f;
      const float a3 = 2 * c + 1 < NG ? qinit[(2 * c + 1) % NG][1] : 0.f;
      *reinterpret_cast<float4 *>(qsm + (NG + c) * 512 + lane * 16) = make_float4(a0, a1, a2, a3);
    }
    __syncwarp();
  }

  const int lo_tok = p.sink, hi_tok = L - p.recent;
  const uint32_t *mrow = p.mask ? p.mask + ((long long)b * p.Hkv + h) * p.mask_stride : nullptr;
  const int32_t *ptrow = p.page_table + (long long)b * p.pt_stride;
  const uint8_t *hbase = p.pool + (long long)h * p.head_bytes;
  const float2 neg_sel = t >= 2 ? make_float2(-1.f, -1.f) : make_float2(0.f, 0.f);

  SoftmaxState<NMT> st;
  st.reset();
  PageCursor cur;
  cur.pg1 = pg1;
  cur.cursor = pg0;
  load_batch(cur, pg0, ptrow, lo_tok, hi_tok, mrow, p, lane);

  Ring<NS> ring;
  ring.s = 0;
#pragma unroll
  for (int k = 0; k < NS; ++k) {
    int pid = -1;
    ring.item[k] = next_page(cur, pid, ptrow, lo_tok, hi_tok, mrow, p, lane);
    if (ring.item[k] >= 0 && lane == 0) {
      mbar_arrive_expect_tx(&bars[k], C::STAGE);
      bulk_g2s(wsm + k * C::STAGE, hbase + (long long)pid * p.page_bytes, C::STAGE, &bars[k]);
    }
  }

  while (ring.item[0] >= 0) {
    if (!ring_wait<NS>(ring, bars, phase, p.wait_cap, p.err, lane)) return false;
    const uint8_t *stg = wsm + ring.s * C::STAGE;
    const int pg = ring.item[0];

    // ---- q.K
    uint32_t kw0[NG], kw1[NG], ksw0[NSW], ksw1[NSW], vsw0[NSW], vsw1[NSW];
    if constexpr (NG == 4) {
      const uint4 a0 = *reinterpret_cast<const uint4 *>(stg + g * (D / 2) + t * (D / 8));
      const uint4 a1 = *reinterpret_cast<const uint4 *>(stg + (g + 8) * (D / 2) + t * (D / 8));
      kw0[0] = a0.x; kw0[1] = a0.y; kw0[2] = a0.z; kw0[3] = a0.w;
      kw1[0] = a1.x; kw1[1] = a1.y; kw1[2] = a1.z; kw1[3] = a1.w;
      const uint2 s0 = *reinterpret_cast<const uint2 *>(stg + 16 * D + g * 8);
      const uint2 s1 = *reinterpret_cast<const uint2 *>(stg + 16 * D + (g + 8) * 8);
      const uint2 u0 = *reinterpret_cast<const uint2 *>(stg + 17 * D + g * 8);
      const uint2 u1 = *reinterpret_cast<const uint2 *>(stg + 17 * D + (g + 8) * 8);
      ksw0[0] = s0.x; ksw0[1] = s0.y; ksw1[0] = s1.x; ksw1[1] = s1.y;
      vsw0[0] = u0.x; vsw0[1] = u0.y; vsw1[0] = u1.x; vsw1[1] = u1.y;
    } else {
      const uint2 a0 = *reinterpret_cast<const uint2 *>(stg + g * (D / 2) + t * (D / 8));
      const uint2 a1 = *reinterpret_cast<const uint2 *>(stg + (g + 8) * (D / 2) + t * (D / 8));
      kw0[0] = a0.x; kw0[1] = a0.y;
      kw1[0] = a1.x; kw1[1] = a1.y;
      ksw0[0] = *reinterpret_cast<const uint32_t *>(stg + 16 * D + g * 4);
      ksw1[0] = *reinterpret_cast<const uint32_t *>(stg + 16 * D + (g + 8) * 4);
      vsw0[0] = *reinterpret_cast<const uint32_t *>(stg + 17 * D + g * 4);
      vsw1[0] = *reinterpret_cast<const uint32_t *>(stg + 17 * D + (g + 8) * 4);
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
      const uint4 qv = *reinterpret_cast<const uint4 *>(qsm + i * 512 + lane * 16);
      const float2 qi = *reinterpret_cast<const float2 *>(qsm + (NG + i / 2) * 512 + lane * 16 + (i & 1) * 8);
      float acc[4] = {qi.x, qi.y, qi.x, qi.y};
      const uint32_t k80 = kw0[i] >> 8, k81 = kw1[i] >> 8;
      {   // elements 0, 4 (k-slots 2t, 2t+1) and 2, 6 (2t+8, 2t+9): bf16, 136 + c
        const uint32_t a[4] = {i4x2_biased(kw0[i]), i4x2_biased(kw1[i]), i4x2_biased(k80), i4x2_biased(k81)};
        mma_bf16(acc, a, qv.x, qv.y);
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
    // ---- which of the page's slots are attended (all of them on interior pages)
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    sc01 = __fmul2_rn(sc01, sl2);
    sc23 = __fmul2_rn(sc23, sl2);
    float sl[4] = {sc01.x, sc01.y, sc23.x, sc23.y};
    if (mrow || pg * kPageTokens < lo_tok || pg * kPageTokens + kPageTokens > hi_tok) {
      const int tok0 = pg * kPageTokens + g, tok1 = tok0 + 8;
      bool v0 = tok0 >= lo_tok && tok0 < hi_tok;
      bool v1 = tok1 >= lo_tok && tok1 < hi_tok;
      if (mrow) {
        const uint32_t mw = mrow[pg >> 1] >> ((pg & 1) * 16);
        v0 = v0 && ((mw >> g) & 1u);
        v1 = v1 && ((mw >> (g + 8)) & 1u);
      }
      if (!v0) sl[0] = sl[1] = -INFINITY;
      if (!v1) sl[2] = sl[3] = -INFINITY;
    }
    // exact running max: probabilities <= 1, so P * scale_V fits fp16
    float pr[4];
    softmax_update<NMT, 0>(st, sl, pr);

    // ---- P.V
    uint32_t wb[NG][2];
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      const float vs0 = vs0a[i], vs1 = vs1a[i];
      weights_f16x2(__fmul2_rn(make_float2(pr[0], pr[1]), make_float2(vs0, vs0)),
                    __fmul2_rn(make_float2(pr[2], pr[3]), make_float2(vs1, vs1)), neg_sel, wb[i][0], wb[i][1]);
    }
    uint32_t vw[NMT];
#pragma unroll
    for (int q4 = 0; q4 < NMT / 4; ++q4) {
      const uint4 w = *reinterpret_cast<const uint4 *>(stg + 8 * D + q4 * 512 + lane * 16);
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

    // ---- refill this stage
    __syncwarp();
    int pid = -1;
    const int nxt = next_page(cur, pid, ptrow, lo_tok, hi_tok, mrow, p, lane);
    if (nxt >= 0 && lane == 0) {
      fence_proxy_async();
      mbar_arrive_expect_tx(&bars[ring.s], C::STAGE);
      bulk_g2s(wsm + ring.s * C::STAGE, hbase + (long long)pid * p.page_bytes, C::STAGE, &bars[ring.s]);
    }
    ring.push_rotate(nxt);
  }
  write_partial<D, NMT>(p, st, slot, lane);
  return true;
}

// ---------------------------------------------------------------------------
// INT8 side pages [j0, j1) of one (sequence b, KV head h): fp16 tensor-core
// tiles. Each page streams as two items: the K half (codes + both scale
// arrays) and the V half (codes).
//
// q.K: A = int8 K codes (exact in fp16; LOP3 gives 1152 + c, one HSUB2
// removes 1152), B = q in fp16. With one scale per row, any element order is
// allowed: MMA j covers elements tD/4 + 4j + {0, 2} (k-slots 2t, 2t+1) and
// tD/4 + 4j + {1, 3} (k-slots 2t+8, 2t+9).
// P.V: A = V^T codes (fp16), B = P * scale_V (fp16 hi + lo). The running max
// is exact (P <= 1), so P * scale_V never exceeds the fp16 range.
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ bool int8_piece(const DecodeParams &p, int b, int h, int L, int j0, int j1, uint8_t *wsm,
                           uint64_t *bars, uint8_t *qsm, uint32_t &phase, float *slot, int lane) {
  using C = Cfg<D, false>;
  constexpr int NS = C::NS, NJ = D / 16, NMT = D / 16, NW = D / 8;   // MMAs, M-tiles, words per lane
  constexpr int KHALF = 16 * D + 64, VHALF = 16 * D;
  const int g = lane >> 2, t = lane & 3;
  const int S = p.sink, R = p.recent;
  const int js = S > 0 ? 1 : 0;
  const int r0 = max(S, L - R);

  // fp16 q fragments of MMA j at q area chunk j/2, words 2*(j%2) + {0, 1}
  {
    const int head = g & 3;
    const bool hv = head < G;
    const uint32_t *qh =
        reinterpret_cast<const uint32_t *>(p.q + ((long long)b * p.Hq + h * G + (hv ? head : 0)) * D);
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int d = t * (D / 4) + 4 * j;
      const uint32_t e01 = hv ? qh[d / 2] : 0u, e23 = hv ? qh[d / 2 + 1] : 0u;
      *reinterpret_cast<uint2 *>(qsm + (j / 2) * 512 + lane * 16 + (j % 2) * 8) =
          make_uint2(pack_f16x2(bf16lo_to_f32(e01), bf16lo_to_f32(e23)),    // (q[d], q[d+2])
                     pack_f16x2(bf16hi_to_f32(e01), bf16hi_to_f32(e23)));   // (q[d+1], q[d+3])
    }
    __syncwarp();
  }
  const uint32_t *mrow = p.mask ? p.mask + ((long long)b * p.Hkv + h) * p.mask_stride : nullptr;
  const uint8_t *blk = p.side + ((long long)b * p.Hkv + h) * p.side_stride;
  const long long page_bytes8 = 32LL * D + 64;
  const float lo_sel = t >= 2 ? 1.f : 0.f;
  (void)G;

  // position held by row r of page j, or -1 when the row is not attended
  auto row_pos = [&](int j, int r) -> int {
    int pos;
    if (j < js) {
      pos = r < min(S, L) ? r : -1;
    } else {
      const int slotr = 16 * (j - js) + r;
      const int off = ((slotr - r0) % R + R) % R;
      pos = r0 + off < L ? r0 + off : -1;
    }
    if (pos >= 0 && mrow && !((mrow[pos >> 5] >> (pos & 31)) & 1u)) pos = -1;
    return pos;
  };

  SoftmaxState<NMT> st;
  st.reset();
  // item = 2*j + half; pages without an attended row are skipped
  int cursor = 2 * j0;
  auto next_item = [&]() -> int {
    while (cursor < 2 * j1) {
      const int it = cursor++;
      if (it & 1) return it;
      const bool any = __any_sync(0xffffffffu, lane < 16 && row_pos(it >> 1, lane) >= 0);
      if (any) return it;
      ++cursor;   // skip this page's V half too
    }
    return -1;
  };
  auto issue = [&](int stage, int it) {
    if (lane == 0) {
      const uint8_t *src = blk + (long long)(it >> 1) * page_bytes8 + ((it & 1) ? KHALF : 0);
      const uint32_t bytes = (it & 1) ? VHALF : KHALF;
      mbar_arrive_expect_tx(&bars[stage], bytes);
      bulk_g2s(wsm + stage * C::STAGE, src, bytes, &bars[stage]);
    }
  };

  Ring<NS> ring;
  ring.s = 0;
#pragma unroll
  for (int k = 0; k < NS; ++k) {
    ring.item[k] = next_item();
    if (ring.item[k] >= 0) issue(k, ring.item[k]);
  }

  uint32_t wb0 = 0, wb1 = 0;
  while (ring.item[0] >= 0) {
    if (!ring_wait<NS>(ring, bars, phase, p.wait_cap, p.err, lane)) return false;
    const uint8_t *stg = wsm + ring.s * C::STAGE;
    const int it = ring.item[0];
    if ((it & 1) == 0) {
      // ---- K half: scores, softmax, weights
      const int j = it >> 1;
      uint32_t kw[NW];
#pragma unroll
      for (int c = 0; c < NW / 4; ++c) {
        const uint4 w = *reinterpret_cast<const uint4 *>(stg + c * 512 + lane * 16);
        kw[4 * c + 0] = w.x;
        kw[4 * c + 1] = w.y;
        kw[4 * c + 2] = w.z;
        kw[4 * c + 3] = w.w;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int jj = 0; jj < NJ; jj += 2) {
        const uint4 qv = *reinterpret_cast<const uint4 *>(qsm + (jj / 2) * 512 + lane * 16);
        const uint32_t a0[4] = {i8x2_to_f16x2(kw[jj]), i8x2_to_f16x2(kw[NJ + jj]), i8x2_to_f16x2(kw[jj] >> 8),
                                i8x2_to_f16x2(kw[NJ + jj] >> 8)};
        mma_f16(acc, a0, qv.x, qv.y);
        const uint32_t a1[4] = {i8x2_to_f16x2(kw[jj + 1]), i8x2_to_f16x2(kw[NJ + jj + 1]),
                                i8x2_to_f16x2(kw[jj + 1] >> 8), i8x2_to_f16x2(kw[NJ + jj + 1] >> 8)};
        mma_f16(acc, a1, qv.z, qv.w);
      }
      const __half *ks = reinterpret_cast<const __half *>(stg + 16 * D);
      const __half *vs = reinterpret_cast<const __half *>(stg + 16 * D + 32);
      const float k0 = __half2float(ks[g]) * p.scale_log2, k1 = __half2float(ks[g + 8]) * p.scale_log2;
      const bool v0 = row_pos(j, g) >= 0, v1 = row_pos(j, g + 8) >= 0;
      float sl[4];
      sl[0] = v0 ? acc[0] * k0 : -INFINITY;
      sl[1] = v0 ? acc[1] * k0 : -INFINITY;
      sl[2] = v1 ? acc[2] * k1 : -INFINITY;
      sl[3] = v1 ? acc[3] * k1 : -INFINITY;
      float pr[4];
      softmax_update<NMT, 0>(st, sl, pr);
      const float s0 = __half2float(vs[g]), s1 = __half2float(vs[g + 8]);
      weights_f16(pr[0] * s0, pr[1] * s0, pr[2] * s1, pr[3] * s1, lo_sel, wb0, wb1);
    } else {
      // ---- V half: P.V
      uint32_t vw[NW];
#pragma unroll
      for (int c = 0; c < NW / 4; ++c) {
        const uint4 w = *reinterpret_cast<const uint4 *>(stg + c * 512 + lane * 16);
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
    __syncwarp();
    const int nxt = next_item();
    if (nxt >= 0) {
      if (lane == 0) fence_proxy_async();
      issue(ring.s, nxt);
    }
    ring.push_rotate(nxt);
  }
  write_partial<D, NMT>(p, st, slot, lane);
  return true;
}

// ---------------------------------------------------------------------------
// bf16 pages of one piece (the uncompressed comparison).
// Head block in a page: K[16][D] bf16 then V[16][D] bf16. Each row is copied
// to a padded shared-memory row so ldmatrix reads are conflict-free.
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ bool bf16_piece(const DecodeParams &p, int b, int h, int L, int pg0, int pg1, uint8_t *wsm,
                           uint64_t *bars, uint32_t &phase, float *slot, int lane) {
  using C = Cfg<D, true>;
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
// Persistent worker kernel.
// ---------------------------------------------------------------------------
template <int D, int G, bool kBF16>
__global__ void __launch_bounds__(kWarps * 32, KV4_MIN_BLOCKS) decode_kernel(DecodeParams p) {
  using C = Cfg<D, kBF16>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t *wsm = smem + warp * C::WARP_SMEM;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kWarps * C::WARP_SMEM) + warp * C::NS;
  uint8_t *qsm = smem + kWarps * (C::WARP_SMEM + C::NS * 8) + warp * C::QBYTES;
  int *plan = reinterpret_cast<int *>(smem + C::RINGS);   // [B + 1]
  __shared__ int wtot[kWarps];

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < C::NS; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  pdl_wait();                 // inputs and cache writes of earlier grids are visible from here
  pdl_launch_dependents();    // the merge grid may queue behind the workers

  // plan[b] = sum over b' < b of (attended pages of b') * Hkv, computed by the CTA
  const int cap = p.pt_stride * kPageTokens;
  const int chunk = (p.B + kWarps * 32 - 1) / (kWarps * 32);
  const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
  int mine = 0;
  for (int b = b0; b < b1; ++b) {
    const int L = eff_len(p.seq_lens[b], cap);
    mine += kBF16 ? (L + kPageTokens - 1) / kPageTokens : int4_num_pages(L, p.sink, p.recent);
  }
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
    const int L = eff_len(p.seq_lens[b], cap);
    run += (kBF16 ? (L + kPageTokens - 1) / kPageTokens : int4_num_pages(L, p.sink, p.recent)) * p.Hkv;
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
  const int np8 = (!kBF16 && p.int8_units) ? side_pages(p.sink, p.recent) : 0;
  const long long T8 = (long long)p.B * p.Hkv * np8;
  const long long T4 = plan[p.B];
  const long long NWk = active_workers(p.num_workers, T8, T4);
  if (wid >= NWk) return;
  long long x = worker_first_item(wid, NWk, T8, T4);
  const long long z = worker_first_item(wid + 1, NWk, T8, T4);
  const long long nbh = (long long)p.B * p.Hkv;
  if (x >= z) return;

  uint32_t phase = 0;
  const int first_page = kBF16 ? 0 : int4_first_page(p.sink);
  int b = 0;
  bool located = false;
  while (x < z) {
    bool ok;
    bool int8_item = false;
    if constexpr (!kBF16) int8_item = x < T8;
    if (int8_item) {
      if constexpr (!kBF16) {
        const int r8 = static_cast<int>(x / np8);
        const int j0 = static_cast<int>(x % np8);
        const long long e = min(z, (long long)(r8 + 1) * np8);
        const int L = eff_len(p.seq_lens[r8 / p.Hkv], cap);
        float *slot = p.slots + ((long long)r8 + wid) * p.slot_floats;
        if (lane == 0) {
          if (j0 == 0) p.first[r8] = static_cast<int>(wid);
          if (e == (long long)(r8 + 1) * np8) p.last[r8] = static_cast<int>(wid);
        }
        ok = int8_piece<D, G>(p, r8 / p.Hkv, r8 % p.Hkv, L, j0, j0 + static_cast<int>(e - x), wsm, bars, qsm,
                              phase, slot, lane);
        x = e;
      }
    } else {
      const int y = static_cast<int>(x - T8);
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
      const long long e = min(z, T8 + plan[b] + (long long)(h + 1) * per);
      const int L = eff_len(p.seq_lens[b], cap);
      float *slot = p.slots + (nbh + (long long)b * p.Hkv + h + wid) * p.slot_floats;
      const int pg0 = first_page + off;
      const int pg1 = pg0 + static_cast<int>(e - x);
      if (lane == 0) {
        if (off == 0) p.first[nbh + (long long)b * p.Hkv + h] = static_cast<int>(wid);
        if (e == T8 + plan[b] + (long long)(h + 1) * per) p.last[nbh + (long long)b * p.Hkv + h] = static_cast<int>(wid);
      }
      if constexpr (kBF16) ok = bf16_piece<D, G>(p, b, h, L, pg0, pg1, wsm, bars, phase, slot, lane);
      else ok = int4_piece<D, G>(p, b, h, L, pg0, pg1, wsm, bars, qsm, phase, slot, lane);
      x = e;
    }
    if (!ok) return;
  }
}

// ---------------------------------------------------------------------------
// Host side launchers.
// ---------------------------------------------------------------------------
int decode_smem_bytes(int D, bool bf16, int B) {
  const int rings = D == 128 ? (bf16 ? Cfg<128, true>::RINGS : Cfg<128, false>::RINGS)
                             : (bf16 ? Cfg<64, true>::RINGS : Cfg<64, false>::RINGS);
  return rings + 4 * (B + 1);
}

template <int D, int G, bool kBF16>
static cudaError_t prepare_one(DecodeLaunch *out) {
  const int smem_max = decode_smem_bytes(D, kBF16, kMaxBatch);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_max);
  if (e != cudaSuccess) return e;
  int nb = 0;
  // occupancy at batches up to 1024 sequences; larger batches only add plan bytes
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, decode_kernel<D, G, kBF16>, kWarps * 32,
                                                    decode_smem_bytes(D, kBF16, 1024));
  if (e != cudaSuccess) return e;
  out->smem_bytes = decode_smem_bytes(D, kBF16, 1024);
  out->blocks_per_sm = nb > 0 ? nb : 1;
  return cudaSuccess;
}

template <int D, bool kBF16>
static cudaError_t prepare_d(int G, DecodeLaunch *out) {
  switch (G) {
    case 1: return prepare_one<D, 1, kBF16>(out);
    case 2: return prepare_one<D, 2, kBF16>(out);
    case 4: return prepare_one<D, 4, kBF16>(out);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t decode_prepare(int D, int G, bool bf16, DecodeLaunch *out) {
  if (D == 128) return bf16 ? prepare_d<128, true>(G, out) : prepare_d<128, false>(G, out);
  if (D == 64) return bf16 ? prepare_d<64, true>(G, out) : prepare_d<64, false>(G, out);
  return cudaErrorInvalidValue;
}

template <int D, int G, bool kBF16>
static cudaError_t launch_main(const DecodeParams &p, cudaStream_t stream) {
  return launch_pdl(decode_kernel<D, G, kBF16>, dim3(p.num_workers / kWarps), dim3(kWarps * 32),
                    decode_smem_bytes(D, kBF16, p.B), stream, p);
}

template <int D, bool kBF16>
static cudaError_t launch_main_d(const DecodeParams &p, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_main<D, 1, kBF16>(p, stream);
    case 2: return launch_main<D, 2, kBF16>(p, stream);
    default: return launch_main<D, 4, kBF16>(p, stream);
  }
}

cudaError_t launch_decode(const DecodeParams &p, int D, bool bf16, cudaStream_t stream, cudaEvent_t ev0,
                          cudaEvent_t ev1) {
  if (ev0) cudaEventRecord(ev0, stream);
  cudaError_t e;
  if (D == 128) e = bf16 ? launch_main_d<128, true>(p, stream) : launch_main_d<128, false>(p, stream);
  else e = bf16 ? launch_main_d<64, true>(p, stream) : launch_main_d<64, false>(p, stream);
  if (e != cudaSuccess) return e;
  if (ev1) cudaEventRecord(ev1, stream);
  const int np8 = (!bf16 && p.int8_units) ? side_pages(p.sink, p.recent) : 0;
  return launch_merge(p, D, np8, stream);
}

}  // namespace kv4
