// kv4_append.cu -- quantise new K/V positions into the paged INT4 pool and the
// INT8 sink / recent-window side cache.
//
// KV4-RL review, sec. 3: the full context is stored as paged INT4; the first 16
// and the 128 most recent positions are also kept in an INT8 side cache.
// Quantiser (stated reading): symmetric; INT4 per group of 32 consecutive
// head_dim elements, INT8 per token row; scale = max|x| / qmax rounded toward
// +inf to fp16; code = x / scale rounded to nearest-even.
//
// One warp per (new position, KV head). Lane l holds D/32 consecutive
// elements. fp32 IEEE division followed by round-up to fp16 equals rounding
// the exact quotient a/7 (a/127) up: a bf16 numerator over 7 (127) is never an
// fp16 value unless exact, so the fp32 rounding cannot land on the boundary.
// x/scale in fp32 is at least 2^-10 away from any half-integer it is not equal
// to, so rintf of the fp32 quotient is the exact nearest-even code.
#include "kv4_common.cuh"
#include "kv4_internal.h"

namespace kv4 {

template <int D>
struct AppendLane {
  static constexpr int EPL = D / 32;          // elements per lane
  static constexpr int LPG = kGroup / EPL;    // lanes per INT4 group
};

__device__ __forceinline__ uint32_t nib(int c) { return static_cast<uint32_t>(c) & 0xFu; }

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
  __half hs = __float2half_ru(__fdiv_rn(a, qmax));
  uint16_t bits = __half_as_ushort(hs);
  if (bits == 0x7C00u) {           // a/qmax > 65504: saturate and flag
    bits = 0x7BFFu;
    set_error(err, kErrRange);
  }
  const float s = half_bits_to_f32(bits);
  const int q = static_cast<int>(qmax);
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    int v = static_cast<int>(rintf(__fdiv_rn(x[e], s)));
    c[e] = v > q ? q : (v < -q ? -q : v);
  }
  return bits;
}

template <int D>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  constexpr int EPL = AppendLane<D>::EPL;
  constexpr int LPG = AppendLane<D>::LPG;
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (task >= p.T * p.Hkv) return;
  const long long j = task / p.Hkv;
  const int h = static_cast<int>(task % p.Hkv);

  // sequence owning row j: largest b with offsets[b] <= j
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.offsets[mid] <= j) lo = mid;
    else hi = mid - 1;
  }
  const int b = lo;
  const int n_new = p.offsets[b + 1] - p.offsets[b];
  const int pos = p.lens_old[b] + static_cast<int>(j - p.offsets[b]);
  const int L_new = p.lens_old[b] + n_new;
  if (pos < 0 || pos >= p.pt_stride * kPageTokens) {
    if (lane == 0) set_error(p.err, kErrCapacity);
    return;
  }
  const int page = p.page_table[(long long)b * p.pt_stride + pos / kPageTokens];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0) set_error(p.err, kErrBounds);
    return;
  }
  const int r = pos % kPageTokens;
  uint8_t *blk = p.pool + (long long)page * p.page_bytes + (long long)h * p.head_bytes;
  const int d0 = lane * EPL;
  const int grp = d0 / kGroup;

  const int S = p.sink, R = p.recent;
  const int sink_row = pos < S ? pos : -1;
  const int ring_row = (R > 0 && pos >= L_new - R) ? S + pos % R : -1;
  const int rows = S + R;
  uint8_t *sblk = p.side + ((long long)b * p.Hkv + h) * p.side_stride;

#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
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
    const uint16_t s4 = quant_lane<EPL>(x, LPG, 7.f, c, p.err);
    if (kv == 0) {
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
      // V: the byte of (slot r, element d) pairs d and d+8; its partner lane is
      // 8/EPL lanes up.
      int partner[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) partner[e] = __shfl_down_sync(0xffffffffu, c[e], 8 / EPL);
      if ((d0 % 16) < 8) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int d = d0 + e;
          const int m = d / 16, g = d % 8, tt = (r % 8) / 2;
          const int lanev = 4 * g + tt;
          const int word = (m / 4) * 128 + lanev * 4 + (m % 4);
          blk[8 * D + 4 * word + 2 * (r % 2) + r / 8] = static_cast<uint8_t>(nib(c[e]) | nib(partner[e]) << 4);
        }
      }
      if (d0 % kGroup == 0) *reinterpret_cast<uint16_t *>(blk + 17 * D + 2 * (r * (D / 32) + grp)) = s4;
    }

    // ---- INT8 side cache (sink row and/or ring row), one scale per token row
    if (sink_row >= 0 || ring_row >= 0) {
      int c8[EPL];
      const uint16_t s8 = quant_lane<EPL>(x, 32, 127.f, c8, p.err);
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < EPL; ++e) packed |= (static_cast<uint32_t>(c8[e]) & 0xFFu) << (8 * e);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const int row = which == 0 ? sink_row : ring_row;
        if (row < 0) continue;
        uint8_t *cdst = sblk + (long long)kv * rows * D + (long long)row * D + d0;
        if constexpr (EPL == 4) *reinterpret_cast<uint32_t *>(cdst) = packed;
        else *reinterpret_cast<uint16_t *>(cdst) = static_cast<uint16_t>(packed);
        if (lane == 0)
          *reinterpret_cast<uint16_t *>(sblk + 2LL * rows * D + 2LL * kv * rows + 2LL * row) = s8;
      }
    }
  }
}

cudaError_t launch_append(const AppendParams &p, int D, cudaStream_t stream) {
  const long long tasks = p.T * p.Hkv;
  if (tasks == 0) return cudaSuccess;
  const int warps_per_block = 8;
  const long long blocks = (tasks + warps_per_block - 1) / warps_per_block;
  if (D == 128) append_kernel<128><<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(p);
  else append_kernel<64><<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kv4
