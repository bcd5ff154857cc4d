// kv4_append.cu -- quantise new K/V positions into the paged INT4 pool and the
// INT8 sink / recent-window side cache.
//
// KV4-RL review, sec. 3: the full context is stored as paged INT4; the first 16
// and the 128 most recent positions are also kept in an INT8 side cache.
// Quantiser (stated reading): symmetric; INT4 per group of 32 consecutive
// head_dim elements, INT8 per token row; scale = max|x| / qmax rounded toward
// +inf to fp16; code = x / scale rounded to nearest-even.
//
// Three kernels. append_pages_kernel takes every page the append fills
// completely (a prefill, or a multi-token append that crosses page
// boundaries): one warp per (page, KV head) at a time on resident CTAs, the
// page's 16 bf16 rows of K, then of V, brought into a per-warp shared-memory
// stage by the bulk-copy engine one half-unit ahead; lane l quantises half a
// group (16 elements) of row l % 16 -- the two lanes of a group combine their
// maxima with one shuffle -- into a shared-memory image of the 18*D-byte head
// block, which the warp writes out with 16-byte stores. append_tokens_kernel
// follows: one warp per INT8 side page that the append writes whole (the sink
// page, ring pages whose rows all hold a position), then one warp per new
// position with other work left (INT4 slots of partly filled pages, INT8 rows
// of partly filled side pages), over its KV heads and K / V. When no page is
// filled completely (a decode step) append_kernel takes everything: one warp
// per new position, KV head and K or V. In the row paths lane l holds D/32
// consecutive elements of the row.
//
// Scale: fp32 IEEE division then round-up to fp16 equals rounding the exact
// quotient a/7 (a/127) up: for a bf16 numerator the quotient is either exact
// or has a periodic binary expansion whose bits past the fp16 precision are
// never all zero, so the fp32 rounding cannot land on an fp16 value. The
// division is one multiply and two fmas (div_by_const).
// Code: x/s is either a half-integer or more than 2^-12 away from every
// half-integer, so x * r (r an approximate 1/s) snapped to a 2^-13 grid keeps
// the exact half-integers and the side of every other value, and one more
// addition rounds it to the nearest integer with ties to even (biased_code2).
// The codes stay biased by 1.5 * 2^23, whose low mantissa bits are then the
// two's-complement code, so nibbles and bytes come straight from the bits.
#include <algorithm>
#include <type_traits>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

__device__ __forceinline__ uint32_t nib(int c) { return static_cast<uint32_t>(c) & 0xFu; }

// a / d rounded to nearest for a constant d, given y = RN(1/d): q0 = RN(a*y)
// is within an ulp of a/d, the residual a - d*q0 is exact in one fma, and the
// corrected q0 + r*y rounds to the correctly rounded quotient (Markstein's
// division by reciprocal with one fma correction). For d = 7 and d = 127 the
// result equals IEEE division for every positive finite fp32 a (checked
// exhaustively against the C library's division).
__device__ __forceinline__ float div_by_const(float a, float d, float y) {
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-d, q0, a);
  return __fmaf_rn(r, y, q0);
}

// 1/s to within an ulp or two (fp32 approximate reciprocal).
__device__ __forceinline__ float rcp_approx(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  return r;
}

// Codes kept biased: kCodeBias + c is an fp32 integer in [2^23, 2^24), where
// consecutive integers have consecutive bit patterns and the pattern of
// kCodeBias ends in 4 zero bits, so its low 4 bits are c mod 16.
constexpr float kCodeBias = 12582912.f;   // 1.5 * 2^23

// kCodeBias + (x/s rounded to the nearest integer, ties to even) for two values,
// given r within 4 ulps of 1/s (rcp.approx is within one) and |x/s| <= 127.5;
// r = 0 gives 0 for x = 0. x/s is a half-integer or more than 2^-12 from every
// half-integer: with x = X 2^ex (|X| < 2^8) and s = S 2^es (S < 2^11),
// 2x - (2k+1)s is a multiple of 2^min(ex+1, es), which over 2s is at least
// 1/(2S) if ex + 1 >= es, and otherwise, where |x/s| >= 1/4, at least 1/(4|X|).
// x*r is within 127.5 * 2^-21 < 2^-14 of x/s, and x*r + 1536 is rounded once
// to the 2^-13 spacing of fp32 in [1024, 2048): the result is exactly k + 1/2
// at a half-integer x/s, and elsewhere it stays more than 2^-12 - 2^-14 - 2^-14
// > 0 away on the same side of every half-integer. Adding 1.5 * 2^23 - 1536
// then rounds to the nearest integer, ties to even. (Checked exhaustively on
// the CPU: every positive fp16 s and every bf16 x with |x| <= 7s, and with
// |x| <= 127s, for r = RN(1/s) and r moved by 2 and 4 ulps either way.)
__device__ __forceinline__ float2 biased_code2(float2 x, float r) {
  const float2 t = __ffma2_rn(x, make_float2(r, r), make_float2(1536.f, 1536.f));
  return __fadd2_rn(t, make_float2(kCodeBias - 1536.f, kCodeBias - 1536.f));
}

// Byte of two biased codes: lo in the low nibble, hi in the high nibble.
__device__ __forceinline__ uint32_t nib_pair(float lo, float hi) {
  return (__float_as_uint(lo) & 0xFu) | ((__float_as_uint(hi) << 4) & 0xF0u);
}

// Quantise this lane's EPL values with a scale shared by `span` lanes
// (span = lanes per group for INT4, 32 for INT8) to codes in [-QMAX, QMAX].
// Returns the fp16 scale bits.
template <int EPL, int QMAX>
__device__ __forceinline__ uint16_t quant_lane(const float (&x)[EPL], int span, int (&c)[EPL], uint32_t *err) {
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) a = fmaxf(a, fabsf(x[e]));
  for (int off = 1; off < span; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if (a == 0.f) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) c[e] = 0;
    return 0;
  }
  constexpr float qm = static_cast<float>(QMAX);
  uint16_t bits = __half_as_ushort(__float2half_ru(div_by_const(a, qm, 1.f / qm)));
  const bool sat = bits == 0x7C00u;
  if (sat) {                       // a/qmax > 65504: saturate and flag
    bits = 0x7BFFu;
    set_error(err, kErrRange);
  }
  const float r = rcp_approx(half_bits_to_f32(bits));
  float cb[EPL];
#pragma unroll
  for (int e = 0; e < EPL; e += 2) {
    const float2 v = biased_code2(make_float2(x[e], x[e + 1]), r);
    cb[e] = v.x;
    cb[e + 1] = v.y;
  }
  // s >= max|x| / qmax makes |x / s| <= qmax: a clamp only when s saturated
  if (sat) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) cb[e] = fminf(fmaxf(cb[e], kCodeBias - qm), kCodeBias + qm);
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) c[e] = static_cast<int>(__float_as_uint(cb[e]) - __float_as_uint(kCodeBias));
  return bits;
}

// Sequence b owning packed row j, the row's position and the sequence's new length.
__device__ __forceinline__ void locate_row(const AppendParams &p, long long j, int &b, int &pos, int &L_new) {
  if (p.offsets) {
    // largest b with offsets[b] <= j
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.offsets[mid] <= j) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
    pos = p.lens_old[b] + static_cast<int>(j - p.offsets[b]);
    L_new = p.lens_old[b] + (p.offsets[b + 1] - p.offsets[b]);
  } else {
    b = static_cast<int>(j);   // one new position per sequence
    pos = p.lens_old[b];
    L_new = pos + 1;
  }
}

// Position pos lies in a page that the append [L_old, L_new) fills completely.
__device__ __forceinline__ bool in_full_page(int pos, int L_old, int L_new) {
  const int f0 = (L_old + kPageTokens - 1) / kPageTokens * kPageTokens;
  const int f1 = L_new / kPageTokens * kPageTokens;
  return pos >= f0 && pos < f1;
}

constexpr int kAppendWarps = 8;

// Shared-memory pitch of one staged bf16 row: 2*D bytes plus 16, so that the
// 16 rows of a page start 4 banks apart and the lanes' 16-byte reads of one
// instruction take the minimum of 4 wavefronts.
template <int D>
constexpr int kStageRow = 2 * D + 16;

// append_pages_kernel's dynamic shared memory: per warp a stage of 16 rows and
// the 18*D-byte image of one head block, per warp an mbarrier, then the plan.
template <int D>
constexpr size_t append_pages_smem(int B) {
  return (size_t)kAppendWarps * (16 * kStageRow<D> + 18 * D + 8) + (size_t)(B + 1) * 4;
}

// (page the append fills completely, KV head) number u -> sequence b, head h,
// page index pg within the sequence, and j, the first of its 16 new rows.
__device__ __forceinline__ void locate_page_unit(const AppendParams &p, const int *fplan, long long u, int &b,
                                                 int &h, int &pg, long long &j) {
  const int unit = static_cast<int>(u / p.Hkv);
  h = static_cast<int>(u % p.Hkv);
  int lo = 0, hi = p.B - 1;   // sequence: largest b with fplan[b] <= unit
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (fplan[mid] <= unit) lo = mid;
    else hi = mid - 1;
  }
  b = lo;
  const int L_old = p.lens_old[b];
  pg = (L_old + kPageTokens - 1) / kPageTokens + (unit - fplan[b]);
  j = p.offsets[b] + ((long long)pg * kPageTokens - L_old);
}

// Lanes 0..15 copy row j + lane of KV head h (K or V) into the warp's stage
// with the bulk-copy engine; lane 0 arms the stage's barrier for the bytes.
template <int D>
__device__ __forceinline__ void stage_rows(const AppendParams &p, long long j, int h, int kv, uint8_t *stage,
                                           uint64_t *bar, int lane) {
  if (lane == 0) mbar_arrive_expect_tx(bar, 16 * 2 * D);
  if (lane < 16) {
    const __nv_bfloat16 *src = (kv == 0 ? p.k : p.v) + ((j + lane) * p.Hkv + h) * D;
    bulk_g2s(stage + lane * kStageRow<D>, src, 2 * D, bar);
  }
}

// Quantise the 16 rows of one KV head's K (kv = 0) or V (kv = 1) of a page
// into the image of its head block. Lane (r, hh) holds row r, elements
// [16 hh, 16 hh + 16) of every group of 32: raw[2i], raw[2i+1] for group i.
template <int D>
__device__ __forceinline__ void quant_page_rows(const uint4 (&raw)[D / 16], int kv, uint8_t *im, int r, int hh,
                                                uint32_t *err) {
  constexpr int NG = D / kGroup;
  uint32_t kword[2][NG], sc_pair[(NG + 1) / 2] = {};
#pragma unroll
  for (int i = 0; i < NG; ++i) {
    float x[16];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 w = raw[2 * i + q];
      x[8 * q + 0] = bf16lo_to_f32(w.x);
      x[8 * q + 1] = bf16hi_to_f32(w.x);
      x[8 * q + 2] = bf16lo_to_f32(w.y);
      x[8 * q + 3] = bf16hi_to_f32(w.y);
      x[8 * q + 4] = bf16lo_to_f32(w.z);
      x[8 * q + 5] = bf16hi_to_f32(w.z);
      x[8 * q + 6] = bf16lo_to_f32(w.w);
      x[8 * q + 7] = bf16hi_to_f32(w.w);
    }
    // scale of the group: max |x| over both lanes of the pair (lane ^ 16)
    float a = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(x[e]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 16));
    uint32_t sbits = 0;
    float rc = 0.f;   // a == 0: every code is 0
    bool sat = false;
    if (a != 0.f) {
      sbits = __half_as_ushort(__float2half_ru(div_by_const(a, 7.f, 1.f / 7.f)));
      sat = sbits == 0x7C00u;
      if (sat) {                       // a/7 > 65504: saturate and flag
        sbits = 0x7BFFu;
        if (hh == 0) set_error(err, kErrRange);
      }
      rc = rcp_approx(half_bits_to_f32(static_cast<uint16_t>(sbits)));
    }
    float cb[16];   // biased codes 1.5 * 2^23 + c
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const float2 v = biased_code2(make_float2(x[e], x[e + 1]), rc);
      cb[e] = v.x;
      cb[e + 1] = v.y;
    }
    // sc >= max|x| / 7 makes |x / sc| <= 7: a clamp only when sc saturated
    if (sat) {
#pragma unroll
      for (int e = 0; e < 16; ++e) cb[e] = fminf(fmaxf(cb[e], kCodeBias - 7.f), kCodeBias + 7.f);
    }
    if (kv == 0) {
      // K: element 32i + 8t + k of row r is nibble k of the word at
      // r*D/2 + t*D/8 + 4i; this lane's elements are chunks t = 2hh, 2hh+1
#pragma unroll
      for (int q = 0; q < 2; ++q)
        kword[q][i] = nib_pair(cb[8 * q], cb[8 * q + 1]) | nib_pair(cb[8 * q + 2], cb[8 * q + 3]) << 8 |
                      nib_pair(cb[8 * q + 4], cb[8 * q + 5]) << 16 | nib_pair(cb[8 * q + 6], cb[8 * q + 7]) << 24;
    } else {
      // V: the byte of (slot r, element d) pairs d and d+8 (low, high nibble);
      // this lane's d = 32i + 16hh + e, e < 8 (m = 2i + hh, d mod 8 = e)
      const int m = 2 * i + hh, tt = (r % 8) / 2;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int word = (m / 4) * 128 + (8 * tt + (e ^ (2 * tt))) * 4 + (m % 4);
        im[8 * D + 4 * word + 2 * (r % 2) + r / 8] = static_cast<uint8_t>(nib_pair(cb[e], cb[e + 8]));
      }
    }
    sc_pair[i / 2] |= sbits << (16 * (i % 2));
  }
  if (kv == 0) {
    // chunk t = 2hh + q of row r: the words of groups 0 .. NG-1, 16 (D = 128) or 8 bytes
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint8_t *kd = im + r * (D / 2) + (2 * hh + q) * (D / 8);
      if constexpr (NG == 4) *reinterpret_cast<uint4 *>(kd) = make_uint4(kword[q][0], kword[q][1], kword[q][2], kword[q][3]);
      else *reinterpret_cast<uint2 *>(kd) = make_uint2(kword[q][0], kword[q][1]);
    }
  }
  // the NG fp16 scales of row r, K at 16D, V at 17D
  if (hh == 0) {
    uint8_t *sd = im + (16 + kv) * D + 2 * NG * r;
    if constexpr (NG == 4) *reinterpret_cast<uint2 *>(sd) = make_uint2(sc_pair[0], sc_pair[1]);
    else *reinterpret_cast<uint32_t *>(sd) = sc_pair[0];
  }
}

// One warp per (page the append fills completely, KV head) at a time, over a
// grid of resident CTAs. Every CTA first forms, in shared memory, the prefix
// over sequences of their completely filled pages, then maps its warps' units
// onto (sequence, page, head). Each warp streams its units' rows through a
// one-stage buffer: as soon as its lanes hold the staged K (V) rows in
// registers, the bulk-copy engine fetches the V rows (the next unit's K rows)
// into the same stage while the lanes quantise.
template <int D>
__global__ void __launch_bounds__(256, 3) append_pages_kernel(AppendParams p) {
  constexpr int WARPS = kAppendWarps;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int wtot[WARPS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t *stage = smem + warp * 16 * kStageRow<D>;
  uint8_t *im = smem + WARPS * 16 * kStageRow<D> + warp * 18 * D;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + WARPS * (16 * kStageRow<D> + 18 * D));
  int *fplan = reinterpret_cast<int *>(bars + WARPS);
  if (tid < WARPS) mbar_init(&bars[tid], 1);
  fence_mbar_init();
  pdl_wait();
  pdl_launch_dependents();

  auto full_pages = [&](int b) {
    const int L_old = p.lens_old[b];
    if (L_old < 0) return 0;
    const int L_new = L_old + (p.offsets[b + 1] - p.offsets[b]);
    const int f0 = (L_old + kPageTokens - 1) / kPageTokens, f1 = L_new / kPageTokens;
    return f1 > f0 ? f1 - f0 : 0;
  };
  const int chunk = (p.B + WARPS * 32 - 1) / (WARPS * 32);
  const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
  int mine = 0;
  for (int b = b0; b < b1; ++b) mine += full_pages(b);
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
    fplan[b] = run;
    run += full_pages(b);
  }
  if (tid == WARPS * 32 - 1) fplan[p.B] = run;
  __syncthreads();

  const long long units = (long long)fplan[p.B] * p.Hkv;
  const long long stride = (long long)gridDim.x * WARPS;
  long long u = (long long)blockIdx.x * WARPS + warp;
  if (u >= units) return;
  uint64_t *bar = &bars[warp];
  // lane (r, hh): row r of the page, elements [16 hh, 16 hh + 16) of each group
  const int r = lane & 15, hh = lane >> 4;
  const uint32_t sa = smem_u32(stage) + r * kStageRow<D> + 32 * hh;
  int b, h, pg;
  long long j;
  locate_page_unit(p, fplan, u, b, h, pg, j);
  stage_rows<D>(p, j, h, 0, stage, bar, lane);
  uint32_t phase = 0;
  for (;;) {
    const long long un = u + stride;
    int nb = 0, nh = 0, npg = 0;
    long long nj = 0;
    if (un < units) locate_page_unit(p, fplan, un, nb, nh, npg, nj);
    const int page = pg < p.pt_stride ? p.page_table[(long long)b * p.pt_stride + pg] : -1;
#pragma unroll 1
    for (int kv = 0; kv < 2; ++kv) {
      const bool ok = mbar_wait_bounded(bar, phase, kDefaultWaitCycles);
      if (!__all_sync(0xffffffffu, ok)) {   // the copy did not land: flag, drain it, stop
        if (lane == 0) set_error(p.err, kErrTimeout);
        mbar_wait_bounded(bar, phase, kDefaultWaitCycles);
        return;
      }
      phase ^= 1u;
      uint4 raw[D / 16];
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        raw[2 * i] = lds128(sa + 64 * i);
        raw[2 * i + 1] = lds128(sa + 64 * i + 16);
      }
      // the stage is read: order the reads before the next bulk write into it
      fence_proxy_async();
      __syncwarp();
      if (kv == 0) stage_rows<D>(p, j, h, 1, stage, bar, lane);
      else if (un < units) stage_rows<D>(p, nj, nh, 0, stage, bar, lane);
      quant_page_rows<D>(raw, kv, im, r, hh, p.err);
    }
    __syncwarp();
    if (pg >= p.pt_stride) {
      if (lane == 0) set_error(p.err, kErrCapacity);
    } else if (page < 0 || page >= p.num_pages) {
      if (lane == 0) set_error(p.err, kErrBounds);
    } else {
      uint4 *dst = reinterpret_cast<uint4 *>(p.pool + (long long)page * p.page_bytes + (long long)h * p.head_bytes);
      const uint4 *srci = reinterpret_cast<const uint4 *>(im);
      for (int q = lane; q < 18 * D / 16; q += 32) dst[q] = srci[q];
    }
    __syncwarp();
    if (un >= units) break;
    u = un;
    b = nb;
    h = nh;
    pg = npg;
    j = nj;
  }
}

// INT8 side pages that an append with the page kernel writes whole, one warp
// per (page, KV head) in append_tokens_kernel instead of row by row: the sink
// page when the sequence starts with this append and fills all 16 of its rows,
// and, when every position of the recent window is new, each ring page whose
// 16 rows all hold a position (all of them once L_new >= recent). Every other
// INT8 row is written by the row path, so no byte outside a row is touched.
__device__ __forceinline__ bool sink_whole(const AppendParams &p, int L_old, int L_new) {
  return p.page_kernel && p.sink == kPageTokens && L_old == 0 && L_new >= kPageTokens;
}
// Number of whole ring pages (ring pages 0 .. n-1).
__device__ __forceinline__ int ring_whole(const AppendParams &p, int L_old, int L_new) {
  const bool fresh = p.page_kernel && p.recent > 0 && L_old >= 0 && L_old <= max(L_new - p.recent, 0);
  return fresh ? min(p.recent, L_new) / kPageTokens : 0;
}
__device__ __forceinline__ int side_pages_whole(const AppendParams &p, int L_old, int L_new) {
  return (sink_whole(p, L_old, L_new) ? 1 : 0) + ring_whole(p, L_old, L_new);
}

// Where the rows of position pos of sequence b go: the INT4 slot r of `page`
// (unless the page kernel owns the page) and the INT8 sink and ring rows.
struct RowTarget {
  int sink_row, ring_row, r, page;
  bool skip4;
};

// False if the position has nothing to write here, or if its page id is out
// of range (flagged).
__device__ __forceinline__ bool row_target(const AppendParams &p, int b, int pos, int L_new, int lane, RowTarget &t) {
  const int S = p.sink, R = p.recent, L_old = p.lens_old[b];
  t.sink_row = (pos < S && !sink_whole(p, L_old, L_new)) ? pos : -1;
  t.ring_row = (R > 0 && pos >= L_new - R && (pos % R) / kPageTokens >= ring_whole(p, L_old, L_new))
                   ? (S > 0 ? 16 : 0) + pos % R
                   : -1;
  // INT4 slots of pages this append fills completely belong to append_pages_kernel
  t.skip4 = p.page_kernel && in_full_page(pos, L_old, L_new);
  if (t.skip4 && t.sink_row < 0 && t.ring_row < 0) return false;
  t.page = p.page_table[(long long)b * p.pt_stride + pos / kPageTokens];
  if (t.page < 0 || t.page >= p.num_pages) {
    if (lane == 0) set_error(p.err, kErrBounds);
    return false;
  }
  t.r = pos % kPageTokens;
  return true;
}

// This lane's D/32 consecutive bf16 elements of row (j, head h, K or V), packed.
template <int D>
using RowRaw = typename std::conditional<D / 32 == 4, uint2, uint32_t>::type;

template <int D>
__device__ __forceinline__ RowRaw<D> load_row_raw(const AppendParams &p, long long j, int h, int kv, int lane) {
  const __nv_bfloat16 *src = (kv == 0 ? p.k : p.v) + (j * p.Hkv + h) * D + lane * (D / 32);
  return *reinterpret_cast<const RowRaw<D> *>(src);
}

__device__ __forceinline__ void unpack_row(uint2 raw, float (&x)[4]) {
  x[0] = bf16lo_to_f32(raw.x);
  x[1] = bf16hi_to_f32(raw.x);
  x[2] = bf16lo_to_f32(raw.y);
  x[3] = bf16hi_to_f32(raw.y);
}

__device__ __forceinline__ void unpack_row(uint32_t raw, float (&x)[2]) {
  x[0] = bf16lo_to_f32(raw);
  x[1] = bf16hi_to_f32(raw);
}

// Quantise and store one row (head h, K or V) of position pos of sequence b,
// given by its lanes' elements x: the INT4 slot (unless the page kernel owns
// the page) and the INT8 side rows. One warp; lane l holds D/32 consecutive
// elements.
template <int D>
__device__ __forceinline__ void store_row(const AppendParams &p, const RowTarget &t, const float (&x)[D / 32], int h,
                                          int kv, int b, int lane) {
  constexpr int EPL = D / 32;              // elements per lane
  constexpr int LPG = kGroup / EPL;        // lanes per INT4 group
  const int sink_row = t.sink_row, ring_row = t.ring_row, r = t.r;
  const bool skip4 = t.skip4;
  uint8_t *blk = p.pool + (long long)t.page * p.page_bytes + (long long)h * p.head_bytes;
  const int d0 = lane * EPL;
  const int grp = d0 / kGroup;
  uint8_t *sblk = p.side + ((long long)b * p.Hkv + h) * p.side_stride;
  const long long spage = 32LL * D + 64;

  {
    // ---- INT4 copy, one scale per group of 32
    int c[EPL];
    const uint16_t s4 = skip4 ? 0 : quant_lane<EPL, 7>(x, LPG, c, p.err);
    if (skip4) {
    } else if (kv == 0) {
      // K: element d at row r, chunk (d%32)/8, word d/32, nibble d%8
      const int t = (d0 % kGroup) / 8, k0 = d0 % 8;
      uint8_t *dst = blk + r * (D / 2) + t * (D / 8) + 4 * grp + k0 / 2;
      if constexpr (EPL == 4) {
        const uint32_t v16 = nib(c[0]) | nib(c[1]) << 4 | nib(c[2]) << 8 | nib(c[3]) << 12;
        *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(v16);
      } else {
        *dst = static_cast<uint8_t>(nib(c[0]) | nib(c[1]) << 4);
      }
      if (d0 % kGroup == 0) *reinterpret_cast<uint16_t *>(blk + 16 * D + 2 * (r * (D / 32) + grp)) = s4;
    } else {
      // V: the byte of (slot r, element d) pairs d and d+8, held 8/EPL lanes up
      int partner[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) partner[e] = __shfl_down_sync(0xffffffffu, c[e], 8 / EPL);
      if ((d0 % 16) < 8) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int d = d0 + e;
          const int m = d / 16, g = d % 8, tt = (r % 8) / 2;
          const int word = (m / 4) * 128 + (8 * tt + (g ^ (2 * tt))) * 4 + (m % 4);
          blk[8 * D + 4 * word + 2 * (r % 2) + r / 8] = static_cast<uint8_t>(nib(c[e]) | nib(partner[e]) << 4);
        }
      }
      if (d0 % kGroup == 0) *reinterpret_cast<uint16_t *>(blk + 17 * D + 2 * (r * (D / 32) + grp)) = s4;
    }

    // ---- INT8 side cache (sink row and/or ring row), one scale per token row
    if (sink_row >= 0 || ring_row >= 0) {
      int c8[EPL];
      const uint16_t s8 = quant_lane<EPL, 127>(x, 32, c8, p.err);
      int partner8[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) partner8[e] = __shfl_down_sync(0xffffffffu, c8[e], 8 / EPL);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const int row = which == 0 ? sink_row : ring_row;
        if (row < 0) continue;
        uint8_t *pg = sblk + (long long)(row / 16) * spage;
        const int rr = row % 16;
        if (kv == 0) {
          // K row rr, element d: lane 4*(rr%8) + d/(D/4), word (rr/8)*(D/16) + (d%(D/4))/4, byte d%4
          const int t = d0 / (D / 4), jw = (d0 % (D / 4)) / 4;
          const int lanek = 4 * (rr % 8) + t;
          const int w = (rr / 8) * (D / 16) + jw;
          uint8_t *dst = pg + (w / 4) * 512 + lanek * 16 + (w % 4) * 4 + d0 % 4;
          if constexpr (EPL == 4) {
            uint32_t packed = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) packed |= (static_cast<uint32_t>(c8[e]) & 0xFFu) << (8 * e);
            *reinterpret_cast<uint32_t *>(dst) = packed;
          } else {
            *reinterpret_cast<uint16_t *>(dst) =
                static_cast<uint16_t>((static_cast<uint32_t>(c8[0]) & 0xFFu) | (static_cast<uint32_t>(c8[1]) & 0xFFu) << 8);
          }
          if (lane == 0) *reinterpret_cast<uint16_t *>(pg + 16 * D + 2 * rr) = s8;
        } else {
          // V row rr, element d: lane 4*(d%8) + (rr%8)/2, word 2*(d/16) + rr/8,
          // bytes 2*(rr%2) + {0: d, 1: d+8}
          if ((d0 % 16) < 8) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
              const int d = d0 + e;
              const int lanev = 4 * (d % 8) + (rr % 8) / 2;
              const int w = 2 * (d / 16) + rr / 8;
              const uint32_t pair = (static_cast<uint32_t>(c8[e]) & 0xFFu) | (static_cast<uint32_t>(partner8[e]) & 0xFFu) << 8;
              *reinterpret_cast<uint16_t *>(pg + 16 * D + 64 + (w / 4) * 512 + lanev * 16 + (w % 4) * 4 +
                                            2 * (rr % 2)) = static_cast<uint16_t>(pair);
            }
          }
          if (lane == 0) *reinterpret_cast<uint16_t *>(pg + 16 * D + 32 + 2 * rr) = s8;
        }
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (task >= p.T * p.Hkv * 2) return;
  const int kv = static_cast<int>(task & 1);   // 0: K, 1: V
  const long long j = (task >> 1) / p.Hkv;
  const int h = static_cast<int>((task >> 1) % p.Hkv);
  // the row's load is in flight while its place in the cache is looked up
  const RowRaw<D> raw = load_row_raw<D>(p, j, h, kv, lane);
  int b, pos, L_new;
  locate_row(p, j, b, pos, L_new);
  if (pos < 0 || pos >= p.pt_stride * kPageTokens) {
    if (lane == 0) set_error(p.err, kErrCapacity);
    return;
  }
  RowTarget t;
  if (!row_target(p, b, pos, L_new, lane, t)) return;
  float x[D / 32];
  unpack_row(raw, x);
  store_row<D>(p, t, x, h, kv, b, lane);
}

// Positions of sequence b that have work outside the pages the append fills
// completely: the slots of partly filled pages and the INT8 sink and ring
// rows not written page-wise. They form [L_old, a_end) and [b_start, L_new)
// (one range if these meet); returns their number.
__device__ __forceinline__ int token_work(const AppendParams &p, int b, int &L_old, int &a_end, int &b_start) {
  L_old = p.lens_old[b];
  const int L_new = L_old + (p.offsets[b + 1] - p.offsets[b]);
  if (L_old < 0) {                 // invalid length: every position (the row kernel flags it)
    a_end = b_start = L_new;
    return L_new - L_old;
  }
  const int f0 = (L_old + kPageTokens - 1) / kPageTokens * kPageTokens;
  const int f1 = L_new / kPageTokens * kPageTokens;
  // (ring rows of positions below f1 sit in whole ring pages when any ring page is whole)
  a_end = min(L_new, max(f0, sink_whole(p, L_old, L_new) ? 0 : min(p.sink, f1)));
  b_start = max(L_old, min(f1, max(ring_whole(p, L_old, L_new) > 0 ? f1 : L_new - p.recent, f0)));
  if (a_end >= b_start) {
    a_end = b_start = L_new;
    return L_new - L_old;
  }
  return (a_end - L_old) + (L_new - b_start);
}

// One INT8 side page j of (sequence b, KV head h) written whole (one warp):
// lane (r, hh) quantises row r -- elements [16 hh, 16 hh + 16) of every group
// of 32 -- of K, then of V, into a shared-memory image of the 32*D + 64-byte
// page, written out with 16-byte stores. Row r of the sink page holds
// position r; row r of ring page k holds the position of the recent window
// congruent to 16 k + r modulo recent.
template <int D>
__device__ void append_side_page(const AppendParams &p, int b, int h, int j, int L_old, int L_new, uint8_t *im,
                                 int lane) {
  constexpr int NG = D / kGroup;
  const int r = lane & 15, hh = lane >> 4;
  const int js = p.sink > 0 ? 1 : 0;
  // (every row of a whole page holds a position)
  const int pos = j < js ? r : L_new - 1 - (L_new - 1 - (kPageTokens * (j - js) + r)) % p.recent;
  const long long row = p.offsets[b] + (pos - L_old);
#pragma unroll 1
  for (int kv = 0; kv < 2; ++kv) {
    uint4 raw[D / 16];
    const __nv_bfloat16 *src = (kv == 0 ? p.k : p.v) + (row * p.Hkv + h) * D + 16 * hh;
#pragma unroll
    for (int i = 0; i < NG; ++i) {
#pragma unroll
      for (int q = 0; q < 2; ++q)
        raw[2 * i + q] = *reinterpret_cast<const uint4 *>(src + kGroup * i + 8 * q);
    }
    // row scale: max |x| over the row (this lane's half, then lane ^ 16)
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) a = fmaxf(a, fmaxf(fabsf(bf16lo_to_f32(w[e])), fabsf(bf16hi_to_f32(w[e]))));
    }
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 16));
    uint32_t sbits = 0;
    float rc = 0.f;   // a == 0: every code is 0
    bool sat = false;
    if (a != 0.f) {
      sbits = __half_as_ushort(__float2half_ru(div_by_const(a, 127.f, 1.f / 127.f)));
      sat = sbits == 0x7C00u;
      if (sat) {                       // a/127 > 65504: saturate and flag
        sbits = 0x7BFFu;
        if (hh == 0) set_error(p.err, kErrRange);
      }
      rc = rcp_approx(half_bits_to_f32(static_cast<uint16_t>(sbits)));
    }
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      float cb[16];   // biased codes of elements d = 32i + 16hh + e
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint4 w = raw[2 * i + q];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = biased_code2(make_float2(bf16lo_to_f32(ww[e]), bf16hi_to_f32(ww[e])), rc);
          cb[8 * q + 2 * e] = v.x;
          cb[8 * q + 2 * e + 1] = v.y;
        }
      }
      if (sat) {
#pragma unroll
        for (int e = 0; e < 16; ++e) cb[e] = fminf(fmaxf(cb[e], kCodeBias - 127.f), kCodeBias + 127.f);
      }
      const int d0 = kGroup * i + 16 * hh;
      if (kv == 0) {
        // K row r, element d: byte d%4 of word (r/8)*(D/16) + (d%(D/4))/4 of
        // lane 4*(r%8) + d/(D/4); 4 consecutive elements make one word
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int d = d0 + 4 * c;
          const int lk = 4 * (r % 8) + d / (D / 4), w = (r / 8) * (D / 16) + (d % (D / 4)) / 4;
          const uint32_t lo = __byte_perm(__float_as_uint(cb[4 * c]), __float_as_uint(cb[4 * c + 1]), 0x0040);
          const uint32_t hi = __byte_perm(__float_as_uint(cb[4 * c + 2]), __float_as_uint(cb[4 * c + 3]), 0x0040);
          *reinterpret_cast<uint32_t *>(im + (w / 4) * 512 + lk * 16 + (w % 4) * 4) = __byte_perm(lo, hi, 0x5410);
        }
      } else {
        // V row r, element d (d%16 < 8): bytes 2(r%2) and 2(r%2)+1 of word
        // 2(d/16) + r/8 of lane 4(d%8) + (r%8)/2 hold the codes of d and d+8
        const int w = 2 * (d0 / 16) + r / 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int lv = 4 * e + (r % 8) / 2;
          const uint32_t pair = __byte_perm(__float_as_uint(cb[e]), __float_as_uint(cb[e + 8]), 0x0040);
          *reinterpret_cast<uint16_t *>(im + 16 * D + 64 + (w / 4) * 512 + lv * 16 + (w % 4) * 4 + 2 * (r % 2)) =
              static_cast<uint16_t>(pair);
        }
      }
    }
    if (hh == 0) *reinterpret_cast<uint16_t *>(im + 16 * D + 32 * kv + 2 * r) = static_cast<uint16_t>(sbits);
  }
  __syncwarp();
  uint4 *dst = reinterpret_cast<uint4 *>(p.side + ((long long)b * p.Hkv + h) * p.side_stride +
                                         (long long)j * (32 * D + 64));
  const uint4 *srci = reinterpret_cast<const uint4 *>(im);
  for (int q = lane; q < (32 * D + 64) / 16; q += 32) dst[q] = srci[q];
  __syncwarp();
}

// Used with append_pages_kernel: one warp per INT8 side page written whole
// (append_side_page), then one warp per position that has work outside the
// pages the append fills completely, over its KV heads and K / V. Every CTA
// forms the prefixes over sequences of both counts in shared memory.
template <int D>
__global__ void __launch_bounds__(256) append_tokens_kernel(AppendParams p) {
  constexpr int WARPS = 8;
  __shared__ int wtot[2][WARPS];
  __shared__ __align__(16) uint8_t img[WARPS][32 * D + 64];
  extern __shared__ int tplan[];   // [B + 1] positions, then [B + 1] side pages
  int *splan = tplan + p.B + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  auto side_count = [&](int b) {
    const int L_old = p.lens_old[b];
    return side_pages_whole(p, L_old, L_old + (p.offsets[b + 1] - p.offsets[b]));
  };
  const int chunk = (p.B + WARPS * 32 - 1) / (WARPS * 32);
  const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
  int mine = 0, mine_s = 0, lo_, ae_, bs_;
  for (int b = b0; b < b1; ++b) {
    mine += token_work(p, b, lo_, ae_, bs_);
    mine_s += side_count(b);
  }
  int incl = mine, incl_s = mine_s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    const int z = __shfl_up_sync(0xffffffffu, incl_s, o);
    if (lane >= o) {
      incl += y;
      incl_s += z;
    }
  }
  if (lane == 31) {
    wtot[0][warp] = incl;
    wtot[1][warp] = incl_s;
  }
  __syncthreads();
  int run = incl - mine, run_s = incl_s - mine_s;
  for (int w = 0; w < warp; ++w) {
    run += wtot[0][w];
    run_s += wtot[1][w];
  }
  for (int b = b0; b < b1; ++b) {
    tplan[b] = run;
    splan[b] = run_s;
    run += token_work(p, b, lo_, ae_, bs_);
    run_s += side_count(b);
  }
  if (tid == WARPS * 32 - 1) {
    tplan[p.B] = run;
    splan[p.B] = run_s;
  }
  __syncthreads();

  const long long nside = (long long)splan[p.B] * p.Hkv;
  const long long total = nside + tplan[p.B];
  for (long long u = (long long)blockIdx.x * WARPS + warp; u < total; u += (long long)gridDim.x * WARPS) {
    if (u < nside) {
      const int q = static_cast<int>(u / p.Hkv), h = static_cast<int>(u % p.Hkv);
      int lo = 0, hi = p.B - 1;   // sequence: largest b with splan[b] <= q
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (splan[mid] <= q) lo = mid;
        else hi = mid - 1;
      }
      const int b = lo, L_old = p.lens_old[b], L_new = L_old + (p.offsets[b + 1] - p.offsets[b]);
      const int js = p.sink > 0 ? 1 : 0;
      const int k = q - splan[b];   // which of the sequence's whole side pages
      const int j = sink_whole(p, L_old, L_new) ? (k == 0 ? 0 : js + (k - 1)) : js + k;
      append_side_page<D>(p, b, h, j, L_old, L_new, img[warp], lane);
      continue;
    }
    const int tu = static_cast<int>(u - nside);
    int lo = 0, hi = p.B - 1;   // sequence: largest b with tplan[b] <= tu
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tplan[mid] <= tu) lo = mid;
      else hi = mid - 1;
    }
    const int b = lo;
    int L_old, a_end, b_start;
    token_work(p, b, L_old, a_end, b_start);
    const int k = tu - tplan[b];
    const int pos = k < a_end - L_old ? L_old + k : b_start + (k - (a_end - L_old));
    const int L_new = L_old + (p.offsets[b + 1] - p.offsets[b]);
    const long long j = p.offsets[b] + (pos - L_old);
    if (pos < 0 || pos >= p.pt_stride * kPageTokens) {
      if (lane == 0) set_error(p.err, kErrCapacity);
      continue;
    }
    RowTarget t;
    if (!row_target(p, b, pos, L_new, lane, t)) continue;
    // the position's rows (KV head, K / V) in batches of 8, each batch's loads in flight together
    for (int hk0 = 0; hk0 < 2 * p.Hkv; hk0 += 8) {
      RowRaw<D> raw[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (hk0 + e < 2 * p.Hkv) raw[e] = load_row_raw<D>(p, j, (hk0 + e) >> 1, (hk0 + e) & 1, lane);
      const int n = min(8, 2 * p.Hkv - hk0);
#pragma unroll 1
      for (int e = 0; e < n; ++e) {   // row hk0 + e sits in raw[0]: the batch shifts down
        float x[D / 32];
        unpack_row(raw[0], x);
        store_row<D>(p, t, x, (hk0 + e) >> 1, (hk0 + e) & 1, b, lane);
#pragma unroll
        for (int k = 0; k < 7; ++k) raw[k] = raw[k + 1];
      }
    }
  }
}

template <int D>
cudaError_t launch_append_pages(unsigned blocks, const AppendParams &p, cudaStream_t stream) {
  const size_t smem = append_pages_smem<D>(p.B);
  const cudaError_t attr = cudaFuncSetAttribute(append_pages_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
  if (attr != cudaSuccess) return attr;
  return launch_pdl(append_pages_kernel<D>, dim3(blocks), dim3(32 * kAppendWarps), smem, stream, p);
}

template <int D>
cudaError_t launch_append_tokens(unsigned blocks, const AppendParams &p, cudaStream_t stream) {
  const size_t smem = (size_t)(p.B + 1) * 8;   // the two plans
  const cudaError_t attr = cudaFuncSetAttribute(append_tokens_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)smem);
  if (attr != cudaSuccess) return attr;
  return launch_pdl(append_tokens_kernel<D>, dim3(blocks), dim3(32 * kAppendWarps), smem, stream, p);
}

cudaError_t launch_append(const AppendParams &p_in, int D, cudaStream_t stream) {
  AppendParams p = p_in;
  const long long tasks = p.T * p.Hkv * 2;
  if (tasks == 0) return cudaSuccess;
  const int warps_per_block = 8;
  // Pages can only be filled completely by a multi-position append; the page
  // kernel reads rows with 16-byte loads and keeps its plan in shared memory.
  const bool aligned16 = ((reinterpret_cast<uintptr_t>(p.k) | reinterpret_cast<uintptr_t>(p.v)) & 15u) == 0;
  // (the plan, 4 bytes per sequence, and the stages stay within 227 KB of shared memory)
  p.page_kernel = (p.offsets && p.T >= kPageTokens && aligned16 && p.B <= 7168) ? 1 : 0;
  if (!p.page_kernel) {
    const unsigned blocks = static_cast<unsigned>((tasks + warps_per_block - 1) / warps_per_block);
    if (D == 128) return launch_pdl(append_kernel<128>, dim3(blocks), dim3(32 * warps_per_block), 0, stream, p);
    return launch_pdl(append_kernel<64>, dim3(blocks), dim3(32 * warps_per_block), 0, stream, p);
  }
  // resident CTAs only (3 per SM): each warp keeps its stage busy over several units
  const long long units = (p.T / kPageTokens) * p.Hkv;   // upper bound on (full page, head) units
  const unsigned pblocks = static_cast<unsigned>(std::max(
      1LL, std::min((units + warps_per_block - 1) / warps_per_block, 3LL * std::max(p.num_sms, 1))));
  cudaError_t e = D == 128 ? launch_append_pages<128>(pblocks, p, stream) : launch_append_pages<64>(pblocks, p, stream);
  if (e != cudaSuccess) return e;
  // upper bound on the warp units left: per sequence and KV head the whole side
  // pages, then the positions with work left (all of them, or per sequence two
  // partial pages plus the sink and ring rows)
  const long long tw = std::min<long long>(p.T, (long long)p.B * (2 * kPageTokens + p.sink + p.recent)) +
                       (long long)p.B * p.Hkv * (1 + p.recent / kPageTokens);
  // resident CTAs only (2 per SM), so that each CTA's plan serves several units
  const unsigned tblocks = static_cast<unsigned>(
      std::max(1LL, std::min((tw + warps_per_block - 1) / warps_per_block, 2LL * std::max(p.num_sms, 1))));
  return D == 128 ? launch_append_tokens<128>(tblocks, p, stream) : launch_append_tokens<64>(tblocks, p, stream);
}

}  // namespace kv4
