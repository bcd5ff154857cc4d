// kv4_append.cu -- quantise new K/V positions into the paged INT4 pool and the
// INT8 sink / recent-window side cache.
//
// KV4-RL review, sec. 3: the full context is stored as paged INT4; the first 16
// and the 128 most recent positions are also kept in an INT8 side cache.
// Quantiser (stated reading): symmetric; INT4 per group of 32 consecutive
// head_dim elements, INT8 per token row; scale = max|x| / qmax rounded toward
// +inf to fp16; code = x / scale rounded to nearest-even.
//
// Two kernels. append_pages_kernel takes every page the append fills
// completely (a prefill, or a multi-token append that crosses page
// boundaries): one warp per (page, KV head); for K, then for V, lane l
// quantises half a group (16 elements) of row l % 16 -- the two lanes of a
// group combine their maxima with one shuffle -- into a shared-memory image
// of the 18*D-byte head block, which the warp then writes out with 16-byte
// stores. Codes are packed arithmetically: with u = c + 8 in [1, 15], four
// codes make an exact fp32 integer u0 + 16 u1 + 256 u2 + 4096 u3 whose bits
// an added 2^23 exposes, and XOR with 0x8 per nibble gives c mod 16.
// append_kernel takes the rest: one warp per (new position, KV head, K or V),
// lane l holding D/32 consecutive elements, for the INT4 slots of partially
// filled pages and for every INT8 side-cache row.
//
// Scale: fp32 IEEE division then round-up to fp16 equals rounding the exact
// quotient a/7 (a/127) up: for a bf16 numerator the quotient is either exact
// or has a periodic binary expansion whose bits past the fp16 precision are
// never all zero, so the fp32 rounding cannot land on an fp16 value.
// Code: x/s differs from every half-integer it is not equal to by at least
// 2^-10, while x * r, with r = 1/s rounded (or approximated to an ulp or two),
// differs from x/s by less than 2^-19 for |x/s| <= 7, so rounding x * r to the
// nearest integer is exact except at true half-way points; those are detected
// exactly through the residual c*s - x (exact in fp32) and resolved to the
// even code.
#include <algorithm>

#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

__device__ __forceinline__ uint32_t nib(int c) { return static_cast<uint32_t>(c) & 0xFu; }

// Nearest-even integer to x/s (s > 0), given r = RN(1/s).
__device__ __forceinline__ float round_code(float x, float s, float r) {
  float c = rintf(x * r);
  const float d = fmaf(c, s, -x);   // c*s - x, exact
  if (2.f * fabsf(d) == s) {        // half-way: x/s = c - sign(d)/2; keep the even one
    if (static_cast<int>(c) & 1) c -= copysignf(1.f, d);
  }
  return c;
}

// The same for two values with one scale (packed f32x2 arithmetic); r only
// has to be within 2^-20 of 1/s (an approximate reciprocal will do): the
// half-way test uses the exact residual, not r.
__device__ __forceinline__ float2 round_code2(float2 x, float s, float r) {
  const float2 q = __fmul2_rn(x, make_float2(r, r));
  // nearest-even integer of q (|q| < 2^22): adding 1.5 * 2^23 rounds q to an
  // integer in the last mantissa place, subtracting it again is exact
  float2 c = __fadd2_rn(__fadd2_rn(q, make_float2(12582912.f, 12582912.f)), make_float2(-12582912.f, -12582912.f));
  const float2 d = __ffma2_rn(c, make_float2(s, s), make_float2(-x.x, -x.y));   // c*s - x, exact
  if (2.f * fabsf(d.x) == s || 2.f * fabsf(d.y) == s) {   // rare: an exact half-way point
    if (2.f * fabsf(d.x) == s && (static_cast<int>(c.x) & 1)) c.x -= copysignf(1.f, d.x);
    if (2.f * fabsf(d.y) == s && (static_cast<int>(c.y) & 1)) c.y -= copysignf(1.f, d.y);
  }
  return c;
}

// 1/s to within an ulp or two (fp32 approximate reciprocal).
__device__ __forceinline__ float rcp_approx(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  return r;
}

// Codes c0..c3 in [-7, 7] -> 16 bits of four 4-bit two's-complement nibbles
// (c0 lowest). With u = c + 8 in [1, 15], u0 + 16 u1 + 256 u2 + 4096 u3 is an
// integer below 2^16, exact in fp32; adding 2^23 puts it in the low mantissa
// bits, and nibble u ^ 8 = c mod 16 (the caller XORs 0x8888).
__device__ __forceinline__ uint32_t nib4_biased(float c0, float c1, float c2, float c3) {
  const float v = fmaf(c3, 4096.f, fmaf(c2, 256.f, fmaf(c1, 16.f, c0 + 34952.f)));   // 34952 = 8 * 0x1111
  return __float_as_uint(v + 8388608.f);
}

// Quantise this lane's EPL values with a scale shared by `span` lanes
// (span = lanes per group for INT4, 32 for INT8). Returns the fp16 scale bits.
template <int EPL>
__device__ __forceinline__ uint16_t quant_lane(const float (&x)[EPL], int span, float qmax, int (&c)[EPL],
                                               uint32_t *err) {
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) a = fmaxf(a, fabsf(x[e]));
  for (int off = 1; off < span; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if (a == 0.f) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) c[e] = 0;
    return 0;
  }
  uint16_t bits = __half_as_ushort(__float2half_ru(__fdiv_rn(a, qmax)));
  if (bits == 0x7C00u) {           // a/qmax > 65504: saturate and flag
    bits = 0x7BFFu;
    set_error(err, kErrRange);
  }
  const float s = half_bits_to_f32(bits);
  const float r = __frcp_rn(s);
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const float v = fminf(fmaxf(round_code(x[e], s, r), -qmax), qmax);
    c[e] = static_cast<int>(v);
  }
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

// Scale bits and codes of one group of 32 values held by one thread (the same
// quantiser as quant_lane, without lanes to combine).
__device__ __forceinline__ uint16_t quant_group32(const float (&x)[kGroup], int (&c)[kGroup], uint32_t *err) {
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < kGroup; ++e) a = fmaxf(a, fabsf(x[e]));
  if (a == 0.f) {
#pragma unroll
    for (int e = 0; e < kGroup; ++e) c[e] = 0;
    return 0;
  }
  uint16_t bits = __half_as_ushort(__float2half_ru(__fdiv_rn(a, 7.f)));
  const bool sat = bits == 0x7C00u;
  if (sat) {                       // a/7 > 65504: saturate and flag
    bits = 0x7BFFu;
    set_error(err, kErrRange);
  }
  const float s = half_bits_to_f32(bits);
  const float r = __frcp_rn(s);
  // s >= max|x| / 7 makes |x / s| <= 7, so the codes need a clamp only when
  // the scale saturated
#pragma unroll
  for (int e = 0; e < kGroup; ++e) {
    const float v = round_code(x[e], s, r);
    c[e] = static_cast<int>(sat ? fminf(fmaxf(v, -7.f), 7.f) : v);
  }
  return bits;
}

// One warp per (page the append fills completely, KV head). Every CTA first
// forms, in shared memory, the prefix over sequences of their completely
// filled pages, then maps its warps' units onto (sequence, page, head).
template <int D>
__global__ void __launch_bounds__(256, 4) append_pages_kernel(AppendParams p) {
  constexpr int WARPS = 8, NG = D / kGroup;
  __shared__ __align__(16) uint8_t img[WARPS][18 * D];
  __shared__ int wtot[WARPS];
  extern __shared__ int fplan[];   // [B + 1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  uint8_t *im = img[warp];
  // lane (r, hh): row r of the page, elements [16 hh, 16 hh + 16) of each group;
  // K first, then V, so that the whole warp runs one code path at a time
  const int r = lane & 15, hh = lane >> 4;
  for (long long u = (long long)blockIdx.x * WARPS + warp; u < units; u += (long long)gridDim.x * WARPS) {
    const int unit = static_cast<int>(u / p.Hkv), h = static_cast<int>(u % p.Hkv);
    int lo = 0, hi = p.B - 1;   // sequence: largest b with fplan[b] <= unit
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (fplan[mid] <= unit) lo = mid;
      else hi = mid - 1;
    }
    const int b = lo;
    const int L_old = p.lens_old[b];
    const int pg = (L_old + kPageTokens - 1) / kPageTokens + (unit - fplan[b]);
    if (pg >= p.pt_stride) {
      if (lane == 0) set_error(p.err, kErrCapacity);
      continue;
    }
    const int page = p.page_table[(long long)b * p.pt_stride + pg];
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) set_error(p.err, kErrBounds);
      continue;
    }
    // rows j .. j+15 are the page's slots 0..15 (all new, all of sequence b)
    const long long j = p.offsets[b] + (pg * kPageTokens - L_old);
#pragma unroll 1
    for (int kv = 0; kv < 2; ++kv) {
      const __nv_bfloat16 *src = (kv == 0 ? p.k : p.v) + ((j + r) * p.Hkv + h) * D + 16 * hh;
#pragma unroll
      for (int i = 0; i < NG; ++i) {   // unrolled: the groups' loads are in flight together
        float x[16];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 w = *reinterpret_cast<const uint4 *>(src + kGroup * i + 8 * q);
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
        uint16_t sbits = 0;
        float c[16];
        if (a == 0.f) {
#pragma unroll
          for (int e = 0; e < 16; ++e) c[e] = 0.f;
        } else {
          sbits = __half_as_ushort(__float2half_ru(__fdiv_rn(a, 7.f)));
          const bool sat = sbits == 0x7C00u;
          if (sat) {                       // a/7 > 65504: saturate and flag
            sbits = 0x7BFFu;
            if (hh == 0) set_error(p.err, kErrRange);
          }
          const float sc = half_bits_to_f32(sbits);
          const float rc = rcp_approx(sc);
          // sc >= max|x| / 7 makes |x / sc| <= 7: a clamp only when sc saturated
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float2 v = round_code2(make_float2(x[e], x[e + 1]), sc, rc);
            if (sat) v = make_float2(fminf(fmaxf(v.x, -7.f), 7.f), fminf(fmaxf(v.y, -7.f), 7.f));
            c[e] = v.x;
            c[e + 1] = v.y;
          }
        }
        if (kv == 0) {
          // K: element 32i + 8t + k of row r is nibble k of the word at
          // r*D/2 + t*D/8 + 4i; this lane's elements are chunks t = 2hh, 2hh+1
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint32_t w = __byte_perm(nib4_biased(c[8 * q], c[8 * q + 1], c[8 * q + 2], c[8 * q + 3]),
                                           nib4_biased(c[8 * q + 4], c[8 * q + 5], c[8 * q + 6], c[8 * q + 7]),
                                           0x5410) ^ 0x88888888u;
            *reinterpret_cast<uint32_t *>(im + r * (D / 2) + (2 * hh + q) * (D / 8) + 4 * i) = w;
          }
          if (hh == 0) *reinterpret_cast<uint16_t *>(im + 16 * D + 2 * (r * NG + i)) = sbits;
        } else {
          // V: the byte of (slot r, element d) pairs d and d+8 (low, high nibble);
          // this lane's d = 32i + 16hh + e, e < 8 (m = 2i + hh, d mod 8 = e)
          const int m = 2 * i + hh, tt = (r % 8) / 2;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int word = (m / 4) * 128 + (8 * tt + (e ^ (2 * tt))) * 4 + (m % 4);
            const uint32_t byte = (__float_as_uint(fmaf(c[e + 8], 16.f, c[e] + 136.f) + 8388608.f) & 0xFFu) ^ 0x88u;
            im[8 * D + 4 * word + 2 * (r % 2) + r / 8] = static_cast<uint8_t>(byte);
          }
          if (hh == 0) *reinterpret_cast<uint16_t *>(im + 17 * D + 2 * (r * NG + i)) = sbits;
        }
      }
    }
    __syncwarp();
    uint4 *dst = reinterpret_cast<uint4 *>(p.pool + (long long)page * p.page_bytes + (long long)h * p.head_bytes);
    const uint4 *srci = reinterpret_cast<const uint4 *>(im);
    for (int q = lane; q < 18 * D / 16; q += 32) dst[q] = srci[q];
    __syncwarp();
  }
}

// Quantise and store row (j, head h, K or V) of position pos of sequence b:
// the INT4 slot (unless the page kernel owns the page) and the INT8 side rows.
// One warp; lane l holds D/32 consecutive elements.
template <int D>
__device__ __forceinline__ void append_row(const AppendParams &p, long long j, int h, int kv, int b, int pos,
                                           int L_new, int lane) {
  constexpr int EPL = D / 32;              // elements per lane
  constexpr int LPG = kGroup / EPL;        // lanes per INT4 group
  const int S = p.sink, R = p.recent;
  const int sink_row = pos < S ? pos : -1;
  const int ring_row = (R > 0 && pos >= L_new - R) ? (S > 0 ? 16 : 0) + pos % R : -1;
  // INT4 slots of pages this append fills completely belong to append_pages_kernel
  const bool skip4 = p.page_kernel && in_full_page(pos, p.lens_old[b], L_new);
  if (skip4 && sink_row < 0 && ring_row < 0) return;
  const int page = p.page_table[(long long)b * p.pt_stride + pos / kPageTokens];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0 && kv == 0) set_error(p.err, kErrBounds);
    return;
  }
  const int r = pos % kPageTokens;
  uint8_t *blk = p.pool + (long long)page * p.page_bytes + (long long)h * p.head_bytes;
  const int d0 = lane * EPL;
  const int grp = d0 / kGroup;
  uint8_t *sblk = p.side + ((long long)b * p.Hkv + h) * p.side_stride;
  const long long spage = 32LL * D + 64;

  {
    const __nv_bfloat16 *src = (kv == 0 ? p.k : p.v) + (j * p.Hkv + h) * D + d0;
    float x[EPL];
    if constexpr (EPL == 4) {
      const uint2 raw = *reinterpret_cast<const uint2 *>(src);
      x[0] = bf16lo_to_f32(raw.x);
      x[1] = bf16hi_to_f32(raw.x);
      x[2] = bf16lo_to_f32(raw.y);
      x[3] = bf16hi_to_f32(raw.y);
    } else {
      const uint32_t raw = *reinterpret_cast<const uint32_t *>(src);
      x[0] = bf16lo_to_f32(raw);
      x[1] = bf16hi_to_f32(raw);
    }

    // ---- INT4 copy, one scale per group of 32
    int c[EPL];
    const uint16_t s4 = skip4 ? 0 : quant_lane<EPL>(x, LPG, 7.f, c, p.err);
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
      const uint16_t s8 = quant_lane<EPL>(x, 32, 127.f, c8, p.err);
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
  int b, pos, L_new;
  locate_row(p, j, b, pos, L_new);
  if (pos < 0 || pos >= p.pt_stride * kPageTokens) {
    if (lane == 0) set_error(p.err, kErrCapacity);
    return;
  }
  append_row<D>(p, j, h, kv, b, pos, L_new, lane);
}

// Positions of sequence b that have work outside the pages the append fills
// completely: the slots of partly filled pages and the INT8 sink and ring
// rows. They form [L_old, a_end) and [b_start, L_new) (one range if these
// meet); returns their number.
__device__ __forceinline__ int token_work(const AppendParams &p, int b, int &L_old, int &a_end, int &b_start) {
  L_old = p.lens_old[b];
  const int L_new = L_old + (p.offsets[b + 1] - p.offsets[b]);
  if (L_old < 0) {                 // invalid length: every position (the row kernel flags it)
    a_end = b_start = L_new;
    return L_new - L_old;
  }
  const int f0 = (L_old + kPageTokens - 1) / kPageTokens * kPageTokens;
  const int f1 = L_new / kPageTokens * kPageTokens;
  a_end = min(L_new, max(f0, min(p.sink, f1)));
  b_start = max(L_old, min(f1, max(L_new - p.recent, f0)));
  if (a_end >= b_start) {
    a_end = b_start = L_new;
    return L_new - L_old;
  }
  return (a_end - L_old) + (L_new - b_start);
}

// Used with append_pages_kernel: one warp per position that has work outside
// the pages the append fills completely, looping over the KV heads and K / V.
// Every CTA forms the prefix of those positions over sequences in shared memory.
template <int D>
__global__ void __launch_bounds__(256) append_tokens_kernel(AppendParams p) {
  constexpr int WARPS = 8;
  __shared__ int wtot[WARPS];
  extern __shared__ int tplan[];   // [B + 1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int chunk = (p.B + WARPS * 32 - 1) / (WARPS * 32);
  const int b0 = min(p.B, tid * chunk), b1 = min(p.B, b0 + chunk);
  int mine = 0, lo_, ae_, bs_;
  for (int b = b0; b < b1; ++b) mine += token_work(p, b, lo_, ae_, bs_);
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
    tplan[b] = run;
    run += token_work(p, b, lo_, ae_, bs_);
  }
  if (tid == WARPS * 32 - 1) tplan[p.B] = run;
  __syncthreads();

  const int total = tplan[p.B];
  for (long long u = (long long)blockIdx.x * WARPS + warp; u < total; u += (long long)gridDim.x * WARPS) {
    int lo = 0, hi = p.B - 1;   // sequence: largest b with tplan[b] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tplan[mid] <= u) lo = mid;
      else hi = mid - 1;
    }
    const int b = lo;
    int L_old, a_end, b_start;
    token_work(p, b, L_old, a_end, b_start);
    const int k = static_cast<int>(u - tplan[b]);
    const int pos = k < a_end - L_old ? L_old + k : b_start + (k - (a_end - L_old));
    const int L_new = L_old + (p.offsets[b + 1] - p.offsets[b]);
    const long long j = p.offsets[b] + (pos - L_old);
    if (pos < 0 || pos >= p.pt_stride * kPageTokens) {
      if (lane == 0) set_error(p.err, kErrCapacity);
      continue;
    }
    for (int hk = 0; hk < 2 * p.Hkv; ++hk) append_row<D>(p, j, hk >> 1, hk & 1, b, pos, L_new, lane);
  }
}

cudaError_t launch_append(const AppendParams &p_in, int D, cudaStream_t stream) {
  AppendParams p = p_in;
  const long long tasks = p.T * p.Hkv * 2;
  if (tasks == 0) return cudaSuccess;
  const int warps_per_block = 8;
  // Pages can only be filled completely by a multi-position append; the page
  // kernel reads rows with 16-byte loads and keeps its plan in shared memory.
  const bool aligned16 = ((reinterpret_cast<uintptr_t>(p.k) | reinterpret_cast<uintptr_t>(p.v)) & 15u) == 0;
  // (the plan, 4 bytes per sequence, stays within the default 48 KB with the page images)
  p.page_kernel = (p.offsets && p.T >= kPageTokens && aligned16 && p.B <= 7168) ? 1 : 0;
  if (!p.page_kernel) {
    const unsigned blocks = static_cast<unsigned>((tasks + warps_per_block - 1) / warps_per_block);
    if (D == 128) return launch_pdl(append_kernel<128>, dim3(blocks), dim3(32 * warps_per_block), 0, stream, p);
    return launch_pdl(append_kernel<64>, dim3(blocks), dim3(32 * warps_per_block), 0, stream, p);
  }
  const long long units = (p.T / kPageTokens) * p.Hkv;   // upper bound on (full page, head) units
  const unsigned pblocks = static_cast<unsigned>(
      std::max(1LL, std::min((units + warps_per_block - 1) / warps_per_block, 8192LL)));
  const size_t plan_bytes = (size_t)(p.B + 1) * 4;
  cudaError_t e = D == 128 ? launch_pdl(append_pages_kernel<128>, dim3(pblocks), dim3(32 * warps_per_block),
                                        plan_bytes, stream, p)
                           : launch_pdl(append_pages_kernel<64>, dim3(pblocks), dim3(32 * warps_per_block),
                                        plan_bytes, stream, p);
  if (e != cudaSuccess) return e;
  // upper bound on the positions with work left: all of them, or per sequence
  // two partial pages plus the sink and ring rows
  const long long tw = std::min<long long>(p.T, (long long)p.B * (2 * kPageTokens + p.sink + p.recent));
  const unsigned tblocks = static_cast<unsigned>(
      std::max(1LL, std::min((tw + warps_per_block - 1) / warps_per_block, 8192LL)));
  if (D == 128)
    return launch_pdl(append_tokens_kernel<128>, dim3(tblocks), dim3(32 * warps_per_block), plan_bytes, stream, p);
  return launch_pdl(append_tokens_kernel<64>, dim3(tblocks), dim3(32 * warps_per_block), plan_bytes, stream, p);
}

}  // namespace kv4
