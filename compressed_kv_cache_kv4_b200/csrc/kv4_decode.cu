// kv4_decode.cu -- decode-step attention over the KV4-RL compressed cache.
//
// KV4-RL review, sec. 3: the INT4 region and the INT8-protected region (first
// 16 and last 128 positions) are attended independently; their partial
// (max, sum, output) triples are combined by an exact softmax merge, so no
// full-precision cache is rebuilt. Shadow Mask Distillation, sec. 1 / Figure 1:
// a retained-position mask is applied inside attention.
//
// Three launches on the caller's stream:
//   plan_kernel    prefix over sequences of attended pages x KV heads
//   decode_kernel  persistent warp workers. Each worker first attends its
//                  share of INT8 units (one (sequence, KV head) protected set
//                  each, fp32 SIMT arithmetic), then one contiguous segment of
//                  the flat (sequence, KV head, page) space of the INT4 region.
//                  Pages stream through a per-warp ring of shared-memory stages
//                  filled by 1-D bulk copies (TMA engine, mbarrier completion,
//                  bounded waits). Per page, q.K and P.V are two small
//                  tensor-core tiles (mma.sync m16n8k16, bf16 in, fp32
//                  accumulate); INT4 codes are unpacked to bf16 in registers.
//                  Each worker writes one (m, l, o) partial per (sequence, KV
//                  head) piece of its segment.
//   merge_kernel   one warp per (sequence, query head) merges the partials.
//
// Softmax bookkeeping runs in the log2 domain (scores scaled by tau*log2 e).
// The P.V tile takes P*scale_V as two bf16 terms (hi + lo), which carries
// 16 significant bits into fp32 accumulation.
#include <math.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

template <int D, bool kBF16>
struct Cfg {
  static constexpr int NS = kBF16 ? 3 : 4;                  // stages per warp
  static constexpr int ROWB = 2 * D + 16;                   // padded bf16 row in shared memory
  static constexpr int STAGE = kBF16 ? 2 * kPageTokens * ROWB : 18 * D;
  static constexpr int WARP_SMEM = NS * STAGE;
  static constexpr int SMEM = kWarps * (WARP_SMEM + NS * 8);
};

// ---------------------------------------------------------------------------
// plan: plan[b] = sum_{b' < b} pages(b') * Hkv, plan[B] = total.
// ---------------------------------------------------------------------------
template <bool kBF16>
__global__ void __launch_bounds__(1024) plan_kernel(DecodeParams p) {
  __shared__ long long wsum[32];
  __shared__ long long carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  const int cap = p.pt_stride * kPageTokens;
  for (int base = 0; base < p.B; base += 1024) {
    const int b = base + tid;
    long long v = 0;
    if (b < p.B) {
      const int L = p.seq_lens[b];
      if (L < 0 || L > cap) set_error(p.err, kErrCapacity);
      const int Le = eff_len(L, cap);
      const int np = kBF16 ? (Le + kPageTokens - 1) / kPageTokens : int4_num_pages(Le, p.sink, p.recent);
      v = (long long)np * p.Hkv;
    }
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      long long s = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;
    }
    __syncthreads();
    if (b < p.B) p.plan[b] = carry + (warp ? wsum[warp - 1] : 0) + x - v;
    __syncthreads();
    if (tid == 0) carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) p.plan[p.B] = carry;
}

// ---------------------------------------------------------------------------
// Partial slot: m[G] | l[G] | pad | o[G][D]   (m in log2 units, o normalised)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void write_empty_slot(const DecodeParams &p, float *slot, int D, int lane) {
  for (int i = lane; i < p.G; i += 32) {
    slot[i] = -INFINITY;
    slot[p.G + i] = 0.f;
  }
  for (int i = lane; i < p.G * D; i += 32) slot[p.slot_o_off + i] = 0.f;
}

// ---------------------------------------------------------------------------
// INT8 unit: the protected positions of one (sequence, KV head), fp32 SIMT.
// Positions: [0, min(sink, L)) from the sink rows, [max(sink, L - recent), L)
// from ring row sink + p mod recent. Exact two-pass softmax over <= 144 rows.
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ void int8_unit(const DecodeParams &p, int u, uint8_t *wsm, int lane) {
  constexpr int EPL = D / 32;
  const int b = u / p.Hkv, h = u % p.Hkv;
  float *slot = p.slots8 + (long long)u * p.slot_floats;
  const int L = eff_len(p.seq_lens[b], p.pt_stride * kPageTokens);
  const int S = p.sink, R = p.recent;
  const int ns = min(S, L);
  const int r0 = max(S, L - R);
  const int nr = max(0, L - r0);
  const int n8 = ns + nr;
  if (n8 == 0) {
    write_empty_slot(p, slot, D, lane);
    return;
  }
  float *qs = reinterpret_cast<float *>(wsm);   // [G][D]
  float *sc = qs + G * D;                       // [n8][G]
  const __nv_bfloat16 *qg = p.q + ((long long)b * p.Hq + h * G) * D;
  for (int i = lane; i < G * D; i += 32) qs[i] = __bfloat162float(qg[i]);
  __syncwarp();
  const uint8_t *blk = p.side + (long long)u * p.side_stride;
  const int rows = S + R;
  const int8_t *kc = reinterpret_cast<const int8_t *>(blk);
  const int8_t *vc = kc + (long long)rows * D;
  const __half *ksc = reinterpret_cast<const __half *>(blk + 2LL * rows * D);
  const __half *vsc = ksc + rows;
  const uint32_t *mrow = p.mask ? p.mask + ((long long)b * p.Hkv + h) * p.mask_stride : nullptr;

  // scores: one lane per position
  for (int j = lane; j < n8; j += 32) {
    const int pos = j < ns ? j : r0 + (j - ns);
    const int row = j < ns ? j : S + pos % R;
    const bool keep = !mrow || ((mrow[pos >> 5] >> (pos & 31)) & 1u);
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.f;
    if (keep) {
      const int4 *kr = reinterpret_cast<const int4 *>(kc + (long long)row * D);
#pragma unroll 2
      for (int c = 0; c < D / 16; ++c) {
        const int4 w = kr[c];
        const int32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float kv = static_cast<float>(static_cast<int8_t>((wv[e >> 2] >> (8 * (e & 3))) & 0xFF));
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g] = fmaf(qs[g * D + 16 * c + e], kv, acc[g]);
        }
      }
      const float s = __half2float(ksc[row]) * p.scale_log2;
#pragma unroll
      for (int g = 0; g < G; ++g) sc[j * G + g] = acc[g] * s;
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) sc[j * G + g] = -INFINITY;
    }
  }
  __syncwarp();
  // max and probabilities per head
  float m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float mx = -INFINITY;
    for (int j = lane; j < n8; j += 32) mx = fmaxf(mx, sc[j * G + g]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    m[g] = mx;
  }
  __syncwarp();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float sum = 0.f;
    for (int j = lane; j < n8; j += 32) {
      const float s = sc[j * G + g];
      const float pr = (s == -INFINITY) ? 0.f : ex2(s - m[g]);
      sc[j * G + g] = pr;
      sum += pr;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    l[g] = sum;
  }
  __syncwarp();
  // P.V: lane owns EPL consecutive elements
  float o[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[g][e] = 0.f;
  for (int j = 0; j < n8; ++j) {
    float pr[G];
    bool any = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      pr[g] = sc[j * G + g];
      any |= pr[g] != 0.f;
    }
    if (!any) continue;
    const int pos = j < ns ? j : r0 + (j - ns);
    const int row = j < ns ? j : S + pos % R;
    const float vs = __half2float(vsc[row]);
    float v[EPL];
    if constexpr (EPL == 4) {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(vc + (long long)row * D + lane * 4);
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = static_cast<float>(static_cast<int8_t>((w >> (8 * e)) & 0xFF)) * vs;
    } else {
      const uint16_t w = *reinterpret_cast<const uint16_t *>(vc + (long long)row * D + lane * 2);
#pragma unroll
      for (int e = 0; e < 2; ++e) v[e] = static_cast<float>(static_cast<int8_t>((w >> (8 * e)) & 0xFF)) * vs;
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[g][e] = fmaf(pr[g], v[e], o[g][e]);
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const bool nonempty = l[g] > 0.f;
    const float inv = nonempty ? 1.f / l[g] : 0.f;
    if (lane == 0) {
      slot[g] = nonempty ? m[g] : -INFINITY;
      slot[G + g] = l[g];
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) slot[p.slot_o_off + g * D + lane * EPL + e] = o[g][e] * inv;
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Page streaming state shared by the INT4 and bf16 page loops.
// ---------------------------------------------------------------------------
struct PageCursor {
  int pg1, cursor, batch_base;
  int pid_reg;        // page id of page batch_base + lane
  uint32_t okbits;    // pages in the batch with at least one attended position
};

// Load the page ids and "has work" bits of pages [base, base + 32).
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
      const uint32_t win = ((t1 >= 32 ? 0xFFFFFFFFu : ((1u << t1) - 1u))) & ~((1u << t0) - 1u);
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

// Next page with work at or after the cursor; -1 when the piece is exhausted.
__device__ __forceinline__ int next_page(PageCursor &c, int &pid, const int32_t *ptrow, int lo_tok, int hi_tok,
                                         const uint32_t *mrow, const DecodeParams &p, int lane) {
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

// Online-softmax state of one warp for the 8 MMA columns (4 "hi" + 4 "lo"
// copies of up to 4 query heads). Thread (g, t) owns columns 2t and 2t+1.
template <int NMT>
struct SoftmaxState {
  float m[2], l[2];
  float o[NMT][4];   // O^T fragments: rows = head_dim, columns = MMA columns
};

// Scores s[0..3] for (token g, col 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1) are
// in log2 units; -inf marks excluded positions. Updates m, l, rescales o, and
// returns the probabilities.
template <int NMT>
__device__ __forceinline__ void softmax_update(SoftmaxState<NMT> &st, float (&s)[4], float (&pr)[4]) {
  float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  // Lazy rescale: keep the reference max unless the page max exceeds it by
  // more than 8 (probabilities stay <= 2^8, far inside fp32 and bf16 range).
  if (mx0 > st.m[0] + 8.f) {
    const float f = ex2(st.m[0] - mx0);
    st.l[0] *= f;
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt) {
      st.o[mt][0] *= f;
      st.o[mt][2] *= f;
    }
    st.m[0] = mx0;
  }
  if (mx1 > st.m[1] + 8.f) {
    const float f = ex2(st.m[1] - mx1);
    st.l[1] *= f;
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt) {
      st.o[mt][1] *= f;
      st.o[mt][3] *= f;
    }
    st.m[1] = mx1;
  }
  const float r0 = st.m[0] == -INFINITY ? 0.f : st.m[0];
  const float r1 = st.m[1] == -INFINITY ? 0.f : st.m[1];
  pr[0] = ex2(s[0] - r0);
  pr[1] = ex2(s[1] - r1);
  pr[2] = ex2(s[2] - r0);
  pr[3] = ex2(s[3] - r1);
  st.l[0] += pr[0] + pr[2];
  st.l[1] += pr[1] + pr[3];
}

// Weights w for (token g, col 2t/2t+1) and (token g+8, ...) -> the B fragment
// (k = tokens, n = columns) of the P.V tile. Lanes with t < 2 contribute the
// bf16 rounding of w ("hi" columns 0-3); lanes with t >= 2 the bf16 rounding of
// the remainder ("lo" columns 4-7).
__device__ __forceinline__ void weights_to_bfrag(float w0, float w1, float w2, float w3, float lo_sel,
                                                 uint32_t &b0, uint32_t &b1) {
  uint32_t h01 = pack_bf16x2(w0, w1);
  uint32_t h23 = pack_bf16x2(w2, w3);
  h01 = pack_bf16x2(fmaf(-lo_sel, bf16lo_to_f32(h01), w0) , fmaf(-lo_sel, bf16hi_to_f32(h01), w1));
  h23 = pack_bf16x2(fmaf(-lo_sel, bf16lo_to_f32(h23), w2), fmaf(-lo_sel, bf16hi_to_f32(h23), w3));
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

// Drain copies still in flight after a failed wait, then report.
template <int NS>
__device__ __forceinline__ void drain(const int (&pgs)[NS], uint64_t *bars, uint32_t phase) {
#pragma unroll
  for (int s = 0; s < NS; ++s)
    if (pgs[s] >= 0) mbar_wait_bounded(&bars[s], (phase >> s) & 1u, kDefaultWaitCycles);
}

// ---------------------------------------------------------------------------
// INT4 pages of one piece (sequence b, KV head h, pages [pg0, pg1)).
// Returns false if a bounded wait ran out (the worker must stop).
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ bool int4_piece(const DecodeParams &p, int b, int h, int L, int pg0, int pg1, uint8_t *wsm,
                           uint64_t *bars, uint32_t &phase, float *slot, int lane) {
  using C = Cfg<D, false>;
  constexpr int NS = C::NS, NG = D / 32, NMT = D / 16;
  const int g = lane >> 2, t = lane & 3;

  // q as the B operand of the q.K tile: column n = g reads head g % 4; the
  // k-slots of MMA (group i, half j) hold elements 32i+8t+{2j, 2j+4, 2j+1, 2j+5},
  // matching the nibble order of the K words.
  uint32_t qf[NG][2][2];
  {
    const int head = g & 3;
    const bool hv = head < G;
    const uint4 *qh = reinterpret_cast<const uint4 *>(p.q + ((long long)b * p.Hq + h * G + (hv ? head : 0)) * D);
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      uint4 e = hv ? qh[(32 * i + 8 * t) / 8] : make_uint4(0, 0, 0, 0);
      // e.x = (e0, e1), e.y = (e2, e3), e.z = (e4, e5), e.w = (e6, e7)
      qf[i][0][0] = __byte_perm(e.x, e.z, 0x5410);   // (e0, e4)
      qf[i][0][1] = __byte_perm(e.x, e.z, 0x7632);   // (e1, e5)
      qf[i][1][0] = __byte_perm(e.y, e.w, 0x5410);   // (e2, e6)
      qf[i][1][1] = __byte_perm(e.y, e.w, 0x7632);   // (e3, e7)
    }
  }

  const int lo_tok = p.sink, hi_tok = L - p.recent;
  const uint32_t *mrow = p.mask ? p.mask + ((long long)b * p.Hkv + h) * p.mask_stride : nullptr;
  const int32_t *ptrow = p.page_table + (long long)b * p.pt_stride;
  const uint8_t *hbase = p.pool + (long long)h * p.head_bytes;
  const float lo_sel = t >= 2 ? 1.f : 0.f;

  SoftmaxState<NMT> st;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
    for (int c = 0; c < 4; ++c) st.o[mt][c] = 0.f;

  PageCursor cur;
  cur.pg1 = pg1;
  cur.cursor = pg0;
  load_batch(cur, pg0, ptrow, lo_tok, hi_tok, mrow, p, lane);

  int pgs[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    int pid = -1;
    pgs[s] = next_page(cur, pid, ptrow, lo_tok, hi_tok, mrow, p, lane);
    if (pgs[s] >= 0 && lane == 0) {
      mbar_arrive_expect_tx(&bars[s], C::STAGE);
      bulk_g2s(wsm + s * C::STAGE, hbase + (long long)pid * p.page_bytes, C::STAGE, &bars[s]);
    }
  }

  for (;;) {
    bool done = false;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      if (pgs[s] < 0) {
        done = true;
        break;
      }
      const bool ok = p.wait_cap != 0 && mbar_wait_bounded(&bars[s], (phase >> s) & 1u, p.wait_cap);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) set_error(p.err, kErrTimeout);
        drain<NS>(pgs, bars, phase);
        return false;
      }
      phase ^= 1u << s;
      const uint8_t *stg = wsm + s * C::STAGE;
      const int pg = pgs[s];

      // ---- q.K: A = K codes (rows = slots g, g+8), one accumulator per group
      uint32_t kw0[NG], kw1[NG];
      if constexpr (NG == 4) {
        const uint4 a0 = *reinterpret_cast<const uint4 *>(stg + g * (D / 2) + t * (D / 8));
        const uint4 a1 = *reinterpret_cast<const uint4 *>(stg + (g + 8) * (D / 2) + t * (D / 8));
        kw0[0] = a0.x; kw0[1] = a0.y; kw0[2] = a0.z; kw0[3] = a0.w;
        kw1[0] = a1.x; kw1[1] = a1.y; kw1[2] = a1.z; kw1[3] = a1.w;
      } else {
        const uint2 a0 = *reinterpret_cast<const uint2 *>(stg + g * (D / 2) + t * (D / 8));
        const uint2 a1 = *reinterpret_cast<const uint2 *>(stg + (g + 8) * (D / 2) + t * (D / 8));
        kw0[0] = a0.x; kw0[1] = a0.y;
        kw1[0] = a1.x; kw1[1] = a1.y;
      }
      const __half *ksp = reinterpret_cast<const __half *>(stg + 16 * D);
      const __half *vsp = reinterpret_cast<const __half *>(stg + 17 * D);
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < NG; ++i) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t a[4] = {i4x2_to_bf16x2(kw0[i] >> (8 * j)), i4x2_to_bf16x2(kw1[i] >> (8 * j)),
                                 i4x2_to_bf16x2(kw0[i] >> (8 * j + 4)), i4x2_to_bf16x2(kw1[i] >> (8 * j + 4))};
          mma_bf16(acc, a, qf[i][j][0], qf[i][j][1]);
        }
        const float k0 = __half2float(ksp[g * NG + i]);
        const float k1 = __half2float(ksp[(g + 8) * NG + i]);
        sc[0] = fmaf(k0, acc[0], sc[0]);
        sc[1] = fmaf(k0, acc[1], sc[1]);
        sc[2] = fmaf(k1, acc[2], sc[2]);
        sc[3] = fmaf(k1, acc[3], sc[3]);
      }
      // ---- which of the page's slots are attended
      const int tok0 = pg * kPageTokens + g, tok1 = tok0 + 8;
      bool v0 = tok0 >= lo_tok && tok0 < hi_tok;
      bool v1 = tok1 >= lo_tok && tok1 < hi_tok;
      if (mrow) {
        const uint32_t mw = mrow[pg >> 1] >> ((pg & 1) * 16);
        v0 = v0 && ((mw >> g) & 1u);
        v1 = v1 && ((mw >> (g + 8)) & 1u);
      }
      float sl[4];
      sl[0] = v0 ? sc[0] * p.scale_log2 : -INFINITY;
      sl[1] = v0 ? sc[1] * p.scale_log2 : -INFINITY;
      sl[2] = v1 ? sc[2] * p.scale_log2 : -INFINITY;
      sl[3] = v1 ? sc[3] * p.scale_log2 : -INFINITY;
      float pr[4];
      softmax_update<NMT>(st, sl, pr);

      // ---- P.V: A = V^T codes (rows = head_dim, k = slots), B = P * scale_V
      uint32_t wb[NG][2];
#pragma unroll
      for (int i = 0; i < NG; ++i) {
        const float vs0 = __half2float(vsp[g * NG + i]);
        const float vs1 = __half2float(vsp[(g + 8) * NG + i]);
        weights_to_bfrag(pr[0] * vs0, pr[1] * vs0, pr[2] * vs1, pr[3] * vs1, lo_sel, wb[i][0], wb[i][1]);
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
        const uint32_t a[4] = {i4x2_to_bf16x2(vw[mt]), i4x2_to_bf16x2(vw[mt] >> 4), i4x2_to_bf16x2(vw[mt] >> 8),
                               i4x2_to_bf16x2(vw[mt] >> 12)};
        mma_bf16(st.o[mt], a, wb[mt >> 1][0], wb[mt >> 1][1]);
      }

      // ---- refill this stage
      __syncwarp();
      int pid = -1;
      pgs[s] = next_page(cur, pid, ptrow, lo_tok, hi_tok, mrow, p, lane);
      if (pgs[s] >= 0 && lane == 0) {
        fence_proxy_async();
        mbar_arrive_expect_tx(&bars[s], C::STAGE);
        bulk_g2s(wsm + s * C::STAGE, hbase + (long long)pid * p.page_bytes, C::STAGE, &bars[s]);
      }
    }
    if (done) break;
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
  const float lo_sel = t >= 2 ? 1.f : 0.f;

  SoftmaxState<NMT> st;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
    for (int c = 0; c < 4; ++c) st.o[mt][c] = 0.f;

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

  int pgs[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    int pid = -1;
    pgs[s] = next_page(cur, pid, ptrow, 0, L, nullptr, p, lane);
    if (pgs[s] >= 0) issue(s, pid);
  }

  const int mi = lane >> 3, ri = lane & 7;
  for (;;) {
    bool done = false;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      if (pgs[s] < 0) {
        done = true;
        break;
      }
      const bool ok = p.wait_cap != 0 && mbar_wait_bounded(&bars[s], (phase >> s) & 1u, p.wait_cap);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) set_error(p.err, kErrTimeout);
        drain<NS>(pgs, bars, phase);
        return false;
      }
      phase ^= 1u << s;
      const uint32_t stg = smem_u32(wsm + s * C::STAGE);
      const int pg = pgs[s];

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
      softmax_update<NMT>(st, sl, pr);
      uint32_t wb0, wb1;
      weights_to_bfrag(pr[0], pr[1], pr[2], pr[3], lo_sel, wb0, wb1);
#pragma unroll
      for (int mt = 0; mt < NMT; ++mt) {
        uint32_t a[4];
        ldmatrix_x4_trans(a, stg + kPageTokens * ROWB + (ri + (mi >> 1) * 8) * ROWB + (16 * mt + (mi & 1) * 8) * 2);
        mma_bf16(st.o[mt], a, wb0, wb1);
      }
      __syncwarp();
      int pid = -1;
      pgs[s] = next_page(cur, pid, ptrow, 0, L, nullptr, p, lane);
      if (pgs[s] >= 0) {
        fence_proxy_async();
        issue(s, pid);
      }
    }
    if (done) break;
  }
  write_partial<D, NMT>(p, st, slot, lane);
  return true;
}

// ---------------------------------------------------------------------------
// Persistent worker kernel.
// ---------------------------------------------------------------------------
template <int D, int G, bool kBF16>
__global__ void __launch_bounds__(kWarps * 32) decode_kernel(DecodeParams p) {
  using C = Cfg<D, kBF16>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *wsm = smem + warp * C::WARP_SMEM;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kWarps * C::WARP_SMEM) + warp * C::NS;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < C::NS; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const long long wid = (long long)blockIdx.x * kWarps + warp;
  const long long NW = p.num_workers;
  const int cap = p.pt_stride * kPageTokens;
  const long long U8 = (!kBF16 && p.int8_units) ? (long long)p.B * p.Hkv : 0;
  if constexpr (!kBF16) {
    for (long long u = wid; u < U8; u += NW) int8_unit<D, G>(p, static_cast<int>(u), wsm, lane);
  }

  const long long T4 = p.plan[p.B];
  long long x = seg_start(wid, T4, U8, NW, kInt8UnitWeight);
  const long long z = seg_start(wid + 1, T4, U8, NW, kInt8UnitWeight);
  if (x >= z) return;
  // sequence holding x: largest b with plan[b] <= x
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.plan[mid] <= x) lo = mid;
    else hi = mid - 1;
  }
  int b = lo;
  uint32_t phase = 0;
  const int first_page = kBF16 ? 0 : int4_first_page(p.sink);
  while (x < z) {
    while (p.plan[b + 1] <= x) ++b;
    const long long base = p.plan[b];
    const long long per = (p.plan[b + 1] - base) / p.Hkv;
    const int h = static_cast<int>((x - base) / per);
    const int off = static_cast<int>((x - base) % per);
    const long long e = min(z, base + (long long)(h + 1) * per);
    const int L = eff_len(p.seq_lens[b], cap);
    const int r = b * p.Hkv + h;
    float *slot = p.slots4 + (long long)(r + wid) * p.slot_floats;
    const int pg0 = first_page + off;
    const int pg1 = pg0 + static_cast<int>(e - x);
    bool ok;
    if constexpr (kBF16) ok = bf16_piece<D, G>(p, b, h, L, pg0, pg1, wsm, bars, phase, slot, lane);
    else ok = int4_piece<D, G>(p, b, h, L, pg0, pg1, wsm, bars, phase, slot, lane);
    if (!ok) return;
    x = e;
  }
}

// ---------------------------------------------------------------------------
// Exact merge of the partials of one (sequence, query head):
// M = max m_c, W_c = l_c 2^(m_c - M), out = sum W_c o_c / sum W_c.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) merge_kernel(DecodeParams p, int has8) {
  constexpr int EPL = D / 32;
  const long long task = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (task >= (long long)p.B * p.Hq) return;
  const int b = static_cast<int>(task / p.Hq), hq = static_cast<int>(task % p.Hq);
  const int h = hq / p.G, gq = hq % p.G;
  const int r = b * p.Hkv + h;
  float M = -INFINITY, den = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  auto add = [&](const float *slot) {
    const float l = slot[p.G + gq];
    if (!(l > 0.f)) return;
    const float m = slot[gq];
    if (m > M) {
      const float f = ex2(M - m);
      den *= f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] *= f;
      M = m;
    }
    const float w = l * ex2(m - M);
    den += w;
    const float *o = slot + p.slot_o_off + gq * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, o[e], acc[e]);
  };
  if (has8) add(p.slots8 + (long long)r * p.slot_floats);
  const long long base = p.plan[b];
  const long long per = (p.plan[b + 1] - base) / p.Hkv;
  if (per > 0) {
    const long long start = base + (long long)h * per, end = start + per;
    const long long T4 = p.plan[p.B], NW = p.num_workers;
    const long long U8 = has8 ? (long long)p.B * p.Hkv : 0;
    long long lo = 0, hi = NW - 1;   // largest w with seg_start(w) <= start
    while (lo < hi) {
      const long long mid = (lo + hi + 1) >> 1;
      if (seg_start(mid, T4, U8, NW, kInt8UnitWeight) <= start) lo = mid;
      else hi = mid - 1;
    }
    long long a = seg_start(lo, T4, U8, NW, kInt8UnitWeight);
    for (long long w = lo; w < NW && a < end; ++w) {
      const long long a1 = seg_start(w + 1, T4, U8, NW, kInt8UnitWeight);
      if (a1 > a && a1 > start) add(p.slots4 + (r + w) * p.slot_floats);
      a = a1;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const long long obase = ((long long)b * p.Hq + hq) * D + lane * EPL;
  if (p.out_fp32) {
    float *o = reinterpret_cast<float *>(p.out) + obase;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = acc[e] * inv;
  } else {
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.out) + obase;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = __float2bfloat16_rn(acc[e] * inv);
  }
}

// ---------------------------------------------------------------------------
// Host side launchers.
// ---------------------------------------------------------------------------
template <int D, int G, bool kBF16>
static cudaError_t prepare_one(DecodeLaunch *out) {
  using C = Cfg<D, kBF16>;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  int nb = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, decode_kernel<D, G, kBF16>, kWarps * 32, C::SMEM);
  if (e != cudaSuccess) return e;
  out->smem_bytes = C::SMEM;
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
static void launch_main(const DecodeParams &p, cudaStream_t stream) {
  using C = Cfg<D, kBF16>;
  decode_kernel<D, G, kBF16><<<p.num_workers / kWarps, kWarps * 32, C::SMEM, stream>>>(p);
}

template <int D, bool kBF16>
static void launch_main_d(const DecodeParams &p, cudaStream_t stream) {
  switch (p.G) {
    case 1: launch_main<D, 1, kBF16>(p, stream); break;
    case 2: launch_main<D, 2, kBF16>(p, stream); break;
    default: launch_main<D, 4, kBF16>(p, stream); break;
  }
}

cudaError_t launch_decode(const DecodeParams &p, int D, bool bf16, cudaStream_t stream, cudaEvent_t ev0,
                          cudaEvent_t ev1) {
  if (bf16) plan_kernel<true><<<1, 1024, 0, stream>>>(p);
  else plan_kernel<false><<<1, 1024, 0, stream>>>(p);
  if (ev0) cudaEventRecord(ev0, stream);
  if (D == 128) {
    if (bf16) launch_main_d<128, true>(p, stream);
    else launch_main_d<128, false>(p, stream);
  } else {
    if (bf16) launch_main_d<64, true>(p, stream);
    else launch_main_d<64, false>(p, stream);
  }
  if (ev1) cudaEventRecord(ev1, stream);
  const long long warps = (long long)p.B * p.Hq;
  const unsigned blocks = static_cast<unsigned>((warps + 3) / 4);
  const int has8 = (!bf16 && p.int8_units) ? 1 : 0;
  if (D == 128) merge_kernel<128><<<blocks, 128, 0, stream>>>(p, has8);
  else merge_kernel<64><<<blocks, 128, 0, stream>>>(p, has8);
  return cudaGetLastError();
}

}  // namespace kv4
