// kv4_common.cuh -- device helpers shared by the libkv4 kernels (sm_100a).
//
// Inline PTX for: mbarrier + 1-D bulk copies (the TMA engine, one CTA per copy),
// warp-level bf16 tensor-core MMA (m16n8k16) and 8x8 fragment transposes,
// LOP3 nibble -> bf16 unpacking, ex2.approx.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kv4 {

constexpr int kPageTokens = 16;
constexpr int kGroup = 32;
constexpr int kWarps = 4;                       // warps per CTA in the decode kernels
constexpr long long kDefaultWaitCycles = 1ll << 32;

// Device error bits: bit (1 << status) for the kv4_status values of kv4.h.
constexpr uint32_t kErrCapacity = 1u << 3;
constexpr uint32_t kErrBounds = 1u << 4;
constexpr uint32_t kErrRange = 1u << 5;
constexpr uint32_t kErrTimeout = 1u << 6;

__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- programmatic dependent launch
// Wait until the grids this one depends on (earlier work in the stream) have
// completed and their writes are visible; a no-op without the launch attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid in the stream to start launching (it still waits in pdl_wait).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- mbarrier + bulk copy
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Arrive on `bar` (release semantics at CTA scope); the state token is discarded.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most `cap` SM cycles.
// cap <= 0 gives up immediately unless the phase is already complete.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, long long cap) {
  if (mbar_try_wait(bar, parity)) return true;
  if (cap <= 0) return false;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > cap) return false;
  }
  return true;
}

// 1-D bulk copy global -> shared through the TMA engine; completion is
// counted in bytes on `bar`. dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- shared-memory loads by 32-bit address
// (volatile: they stay behind the mbarrier wait that makes the data visible)
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint16_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

// ---------------------------------------------------------------- tensor-core fragments
// D = A * B + C with A 16x16 (row), B 16x8 (col) bf16, C/D fp32.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A * B + C with the four C registers given (fp32 bit patterns), A 16x16
// (row), B 16x8 (col) bf16, C/D fp32.
__device__ __forceinline__ void mma_bf16_c4(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                            uint4 c) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(__uint_as_float(c.x)),
        "f"(__uint_as_float(c.y)), "f"(__uint_as_float(c.z)), "f"(__uint_as_float(c.w)));
}

// Transpose an 8x8 matrix of 16-bit elements held one row per 4 lanes.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Two signed 4-bit codes at bits 0-3 and 16-19 of w -> bf16x2 of 136 + c.
// LOP3 computes (w & 0x000F000F) ^ 0x43084308: flipping bit 3 turns the
// two's-complement nibble c into c + 8, and 0x43 above it makes the bf16
// value 128 + (c + 8). The offset 136 is removed elsewhere (through the MMA
// accumulator's initial value).
__device__ __forceinline__ uint32_t i4x2_biased(uint32_t w) {
  uint32_t t;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x000F000Fu), "r"(0x43084308u));
  return t;
}

// Two signed 4-bit codes at bits 0-3 and 16-19 of w -> fp16x2 of the codes.
// LOP3 computes (w & 0x000F000F) ^ 0x64086408: flipping bit 3 turns c into
// c + 8 under fp16's 1024, giving 1032 + c; subtracting 1032 is exact.
__device__ __forceinline__ uint32_t i4x2_lo_to_f16x2(uint32_t w) {
  uint32_t t, d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x000F000Fu), "r"(0x64086408u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(t), "r"(0x64086408u));
  return d;
}

// Two signed 4-bit codes at bits 4-7 and 20-23 of w -> fp16x2, with no shift:
// fp16 has ten mantissa bits, so under an exponent of 64 (0x5400) the field
// at bits 4-7 has weight 1. (w & 0x00F000F0) ^ 0x54805480 is 72 + c.
__device__ __forceinline__ uint32_t i4x2_hi_to_f16x2(uint32_t w) {
  uint32_t t, d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x00F000F0u), "r"(0x54805480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(t), "r"(0x54805480u));
  return d;
}

// The same LOP3 as i4x2_hi_to_f16x2 without the subtraction: fp16x2 of 72 + c
// for the codes at bits 4-7 and 20-23 (the offset is removed elsewhere).
__device__ __forceinline__ uint32_t i4x2_hi_biased_f16(uint32_t w) {
  uint32_t t;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x00F000F0u), "r"(0x54805480u));
  return t;
}

// Two signed 8-bit codes at bits 0-7 and 16-23 of w -> fp16x2 of the codes.
// LOP3 computes (w & 0x00FF00FF) ^ 0x64806480: flipping bit 7 turns c into
// c + 128, and 0x64 above it makes the fp16 value 1024 + (c + 128).
// Subtracting 1152 (fp16 0x6480) is exact.
__device__ __forceinline__ uint32_t i8x2_to_f16x2(uint32_t w) {
  uint32_t t, d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x00FF00FFu), "r"(0x64806480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(t), "r"(0x64806480u));
  return d;
}

// D = A * B + C with A 16x16 (row), B 16x8 (col) fp16, C/D fp32.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float f16lo_to_f32(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
}
__device__ __forceinline__ float f16hi_to_f32(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
}

// Both fp16 halves of a 32-bit word as floats (low half in .x).
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2 *>(&v));
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float half_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// ---------------------------------------------------------------- region arithmetic
// Effective length: negative or beyond the page-table capacity counts as empty.
__device__ __forceinline__ int eff_len(int L, int cap) { return (L < 0 || L > cap) ? 0 : L; }

// INT4-attended positions are [sink, L - recent); the rest of [0, L) is the
// INT8-protected set (KV4-RL review, sec. 3). Pages of the INT4 region:
// [sink/16, ceil((L - recent)/16)).
__device__ __forceinline__ int int4_first_page(int sink) { return sink / kPageTokens; }
__device__ __forceinline__ int int4_num_pages(int L, int sink, int recent) {
  const int hi = L - recent;
  if (hi <= sink) return 0;
  return (hi + kPageTokens - 1) / kPageTokens - sink / kPageTokens;
}

// ---------------------------------------------------------------- split of the decode work
// Weights of one item when splitting work among workers: an INT4 page-head
// (18*D bytes) counts 4, an INT8 side page (32*D + 64 bytes) counts 7.
constexpr long long kW4 = 4, kW8 = 7;

// First item of worker w among nw: items 0..T8-1 are INT8 pages (weight kW8),
// then T4 INT4/bf16 pages (weight kW4); worker w starts at the first item whose
// weighted start is >= floor(w * total / nw).
__device__ __forceinline__ long long worker_first_item(long long w, long long nw, long long T8, long long T4) {
  if (w >= nw) return T8 + T4;
  const long long total = kW8 * T8 + kW4 * T4;
  const long long a = w * total / nw;
  if (a <= kW8 * T8) return (a + kW8 - 1) / kW8;
  return T8 + (a - kW8 * T8 + kW4 - 1) / kW4;
}

// Number of workers that take part: at most one per kW8 weight units of work,
// so that the share of each of them holds at least one item (a share spans at
// least kW8 weight units and item starts are at most kW8 apart).
__device__ __forceinline__ long long active_workers(long long nw, long long T8, long long T4) {
  const long long cap = (kW8 * T8 + kW4 * T4) / kW8;
  return cap < 1 ? 1 : (nw < cap ? nw : cap);
}

__host__ __device__ __forceinline__ int side_pages(int sink, int recent) { return (sink > 0 ? 1 : 0) + recent / 16; }

}  // namespace kv4
