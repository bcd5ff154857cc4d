// smd_attn.cu -- learner-side causal attention under the recorded shadow mask.
//
// Shadow Mask Distillation, sec. 1 and Figure 1: during the sparse rollout the
// KV eviction records, for the query at every position, a binary mask of the
// positions it kept; the learner injects that mask into its causal attention,
// so each learner row reproduces exactly what the rollout attended to (the
// pages' pi_sparse == pi_shadow). Query t of head hq (KV head h = hq / G)
// attends to {p <= t : bit p of mask row (h, t)} over the bf16 K and V; an
// empty set gives 0.
//
// Flash-attention style on the 5th-generation tensor cores (tcgen05). A CTA
// of one warpgroup (128 threads) takes one KV head and 128/G query positions:
// tile row r = g (128/G) + position, so the G query heads of a KV head share
// every K/V tile and mask row, and thread r owns row r (TMEM lane r) for the
// whole softmax. Before the loop the CTA ORs its mask rows per 64-key block;
// blocks with no kept key for any of its rows are never loaded. Per active
// block: S = Q K^T by tcgen05.mma (Q, K in shared memory, S in 64 TMEM
// columns); each thread reads its S row (tcgen05.ld), applies the mask bits,
// causality and the length, and takes the exponentials against its running
// maximum; P goes to shared memory as bf16 hi + lo parts (P keeps 16
// significant bits) and O += P V accumulates in TMEM (two MMAs per 16 keys, V
// as an MN-major operand). O is rescaled in TMEM only when a row's maximum
// grows by more than 2^8 since it was last used (the exponentials stay below
// 256, the result is the same softmax). MMAs are issued by one thread and
// signal an mbarrier through tcgen05.commit; every wait is bounded. One CTA
// barrier per block: after it the issuing thread queues P V of this block and
// then S of the next. K tiles of the next block load (cp.async) while the
// softmax runs, V tiles while S is computed. Operands use the no-swizzle
// core-matrix layout: 8 rows of 16 bytes per core matrix.
#include <math.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"
#include "smd_attn.h"

namespace kv4 {

namespace {

constexpr int kTcThreads = 128;   // one warpgroup: TMEM lanes 0..127
constexpr int kTcRows = 128;      // tile rows (M of every MMA)
constexpr int kKeyBlock = 64;     // keys per block (N of S, K of P V)

// x - hi for a bf16 hi: a mixed-precision FMA (bf16 factors, fp32 addend, one
// rounding), so hi needs no conversion back to fp32.
constexpr uint16_t kBf16MinusOne = 0xBF80u;
__device__ __forceinline__ float fma_bf16_f32(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle: start, leading and stride byte
// offsets in 16-byte units, descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(const void *p, uint32_t lbo, uint32_t sbo) {
  const uint32_t a = smem_u32(p);
  return (uint64_t)((a >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, A
// K-major, B K-major or MN-major, shape M x N.
__device__ __forceinline__ uint32_t umma_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// 32 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}
__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// A bounded wait; once one has run out on this thread the later ones give up
// at once, so control flow stays the same on every thread and the total wait
// stays bounded. The CTA checks the outcome once, at the end.
__device__ __forceinline__ void sticky_wait(uint64_t *bar, uint32_t parity, long long cap, bool &ok) {
  ok = mbar_wait_bounded(bar, parity, ok ? cap : 0) && ok;
}

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads) smd_attn_kernel(SmdParams p) {
  constexpr int QP = kTcRows / G;                          // query positions per CTA
  constexpr int CH = D / 8;                                // 16-byte chunks of a row
  constexpr int QBYTES = kTcRows * D * 2;
  constexpr int KVBYTES = kKeyBlock * D * 2;
  constexpr int PBYTES = kTcRows * kKeyBlock * 2;
  constexpr uint32_t TCOLS = D == 128 ? 256u : 128u;       // S (64 columns) then O (D columns)
  constexpr uint32_t OCOL = kKeyBlock;
  constexpr long long kCap = 1ll << 31;                    // cycles per wait (about a second)
  extern __shared__ __align__(1024) uint8_t smem[];
  // Q: element (row, d) at ((d/8)*16 + row/8)*128 + (row%8)*16 + (d%8)*2
  // K, V: element (key, d) at ((d/8)*8 + key/8)*128 + (key%8)*16 + (d%8)*2
  // P: element (row, key) at ((key/8)*16 + row/8)*128 + (row%8)*16 + (key%8)*2
  uint8_t *sq = smem;
  uint8_t *sk = sq + QBYTES;
  uint8_t *sv = sk + KVBYTES;
  uint8_t *sph = sv + KVBYTES;
  uint8_t *spl = sph + PBYTES;
  int *blist = reinterpret_cast<int *>(spl + PBYTES);      // [T/64 + 1]
  __shared__ uint32_t active[kMaxSmdBlocks / 32];
  __shared__ int nact;
  __shared__ __align__(8) uint64_t bar_s, bar_o;
  __shared__ uint32_t tslot;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z, h = blockIdx.y;
  const int ntile = (p.T + QP - 1) / QP;
  const int t0 = (ntile - 1 - static_cast<int>(blockIdx.x)) * QP;   // longest rows first
  pdl_wait();
  pdl_launch_dependents();
  int L = p.T;
  if (p.lens) {
    L = p.lens[b];
    if (L < 0 || L > p.T) {
      if (tid == 0 && p.err) set_error(p.err, kErrCapacity);
      L = L < 0 ? 0 : p.T;
    }
  }
  const int r = tid;                                       // tile row = TMEM lane
  const int g = r / QP, t = t0 + r % QP, hq = h * G + g;
  const bool live = t < L;

  // ---- active key blocks of this CTA's rows
  const int tlast = min(t0 + QP, L) - 1;
  const int nblk = tlast >= 0 ? tlast / kKeyBlock + 1 : 0;
  for (int i = tid; i < (nblk + 31) / 32; i += kTcThreads) active[i] = 0u;
  __syncthreads();
  if (p.mask) {
    const int nw = 2 * nblk;
    const int rows = tlast - t0 + 1;
    for (int idx = tid; idx < rows * nw; idx += kTcThreads) {
      const int rr = idx / nw, w = idx % nw;
      const uint32_t word = w < p.mask_stride
                                ? __ldg(p.mask + (((long long)b * p.Hkv + h) * p.T + t0 + rr) * p.mask_stride + w)
                                : 0u;
      if (word) atomicOr(&active[(w >> 1) >> 5], 1u << ((w >> 1) & 31));
    }
  } else {
    for (int j = tid; j < nblk; j += kTcThreads) atomicOr(&active[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < nblk; base += 32) {
      const int j = base + lane;
      const bool on = j < nblk && ((active[j >> 5] >> (j & 31)) & 1u);
      const uint32_t bal = __ballot_sync(0xffffffffu, on);
      if (on) blist[run + __popc(bal & ((1u << lane) - 1u))] = j;
      run += __popc(bal);
    }
    if (lane == 0) nact = run;
  }
  __syncthreads();
  const int na = nact;
  const long long orow = (((long long)b * p.T + t) * p.Hq + hq) * D;

  if (na == 0) {   // nothing visible to any row of the CTA: the rows are 0
    if (t < p.T) {
      if (p.out_fp32) {
        float4 *o = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + orow);
        for (int c = 0; c < D / 4; ++c) o[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        uint4 *o = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.out) + orow);
        for (int c = 0; c < D / 8; ++c) o[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }

  // ---- TMEM, barriers, Q tile, first K and V tiles
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tslot)),
                 "n"(TCOLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    fence_mbar_init();
  }
  {
    const __nv_bfloat16 *qrow = p.q + orow;
#pragma unroll 4
    for (int c = 0; c < CH; ++c) {
      const uint4 v = live ? *reinterpret_cast<const uint4 *>(qrow + c * 8) : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4 *>(sq + (c * 16 + r / 8) * 128 + (r % 8) * 16) = v;
    }
  }
  auto load_kv = [&](uint8_t *dst_tile, const __nv_bfloat16 *src_base, int j) {
    const int kb = j * kKeyBlock;
    for (int e = tid; e < kKeyBlock * CH; e += kTcThreads) {
      const int n = e / CH, c = e % CH;
      const int pos = kb + n;
      const bool in = pos < L;
      const __nv_bfloat16 *src = src_base + (((long long)b * p.T + (in ? pos : 0)) * p.Hkv + h) * D + c * 8;
      cp_async16(smem_u32(dst_tile + (c * 8 + n / 8) * 128 + (n % 8) * 16), src, in ? 16u : 0u);
    }
    cp_async_commit();
  };
  load_kv(sk, p.k, blist[0]);
  load_kv(sv, p.v, blist[0]);
  cp_async_wait<0>();
  fence_async_smem();
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tslot;
  const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);   // this warp's lane quarter
  const uint32_t idesc_s = umma_idesc(kTcRows, kKeyBlock, false);
  const uint32_t idesc_o = umma_idesc(kTcRows, D, true);
  const uint32_t *mrow = p.mask && live ? p.mask + (((long long)b * p.Hkv + h) * p.T + t) * p.mask_stride : nullptr;
  auto issue_qk = [&]() {
#pragma unroll
    for (int st = 0; st < D / 16; ++st)
      umma_bf16(tmem, umma_desc(sq + st * 2 * 2048, 2048, 128), umma_desc(sk + st * 2 * 1024, 1024, 128), idesc_s,
                st > 0 ? 1u : 0u);
    umma_commit(&bar_s);
  };
  if (tid == 0) issue_qk();

  float m_used = -INFINITY, l = 0.f;
  uint32_t ph_s = 0, ph_o = 0;
  bool ok = true;
  for (int i = 0; i < na; ++i) {
    const int j = blist[i], kb = j * kKeyBlock;
    // this row's mask words for the block, loaded while the MMAs run
    uint32_t w0 = 0xffffffffu, w1 = 0xffffffffu;
    if (p.mask) {
      const int wi = kb >> 5;
      w0 = mrow && wi < p.mask_stride ? __ldg(mrow + wi) : 0u;
      w1 = mrow && wi + 1 < p.mask_stride ? __ldg(mrow + wi + 1) : 0u;
    }
    if (i > 0) {   // P V of the previous block: its P tiles, V tile and O are free/stable after this
      sticky_wait(&bar_o, ph_o, kCap, ok);
      ph_o ^= 1u;
      tc_after_sync();
      load_kv(sv, p.v, j);
    }
    sticky_wait(&bar_s, ph_s, kCap, ok);   // S = Q K^T of this block
    ph_s ^= 1u;
    tc_after_sync();
    float x[kKeyBlock];
    {
      uint32_t sr[32];
      tmem_ld32(trow, sr);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) x[k] = __uint_as_float(sr[k]);
      tmem_ld32(trow + 32, sr);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) x[32 + k] = __uint_as_float(sr[k]);
    }
    if (i + 1 < na) load_kv(sk, p.k, blist[i + 1]);   // S is read: the K tile is free

    // visibility: live row, key <= query, mask bit set
    float mloc = -INFINITY;
#pragma unroll
    for (int k = 0; k < kKeyBlock; ++k) {
      const bool vis = live && kb + k <= t && (((k < 32 ? w0 : w1) >> (k & 31)) & 1u);
      x[k] = vis ? x[k] * p.scale_log2 : -INFINITY;
      mloc = fmaxf(mloc, x[k]);
    }
    float corr = 1.f;
    bool resc = false;
    if (mloc > m_used + 8.f) {   // also true when the first visible key arrives
      if (m_used != -INFINITY) {
        resc = true;
        corr = ex2(m_used - mloc);
      }
      m_used = mloc;
    }
    const float base = m_used == -INFINITY ? 0.f : m_used;
    float lsum = 0.f;
#pragma unroll
    for (int k = 0; k < kKeyBlock; ++k) {
      x[k] = ex2(x[k] - base);
      lsum += x[k];
    }
    l = l * corr + lsum;
    if (__any_sync(0xffffffffu, resc)) {   // this warp's O rows in TMEM (settled: P V of i - 1 is done)
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(trow + OCOL + c0, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * corr);
        tmem_st32(trow + OCOL + c0, o);
      }
      tmem_wait_st();
    }
    // P as bf16 hi + lo, row r
#pragma unroll
    for (int c = 0; c < kKeyBlock / 8; ++c) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = x[c * 8 + 2 * e], x1 = x[c * 8 + 2 * e + 1];
        hw[e] = pack_bf16x2(x0, x1);
        lw[e] = pack_bf16x2(fma_bf16_f32(static_cast<uint16_t>(hw[e]), kBf16MinusOne, x0),
                            fma_bf16_f32(static_cast<uint16_t>(hw[e] >> 16), kBf16MinusOne, x1));
      }
      const int off = (c * 16 + r / 8) * 128 + (r % 8) * 16;
      *reinterpret_cast<uint4 *>(sph + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4 *>(spl + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    // V(i) and K(i + 1) have landed; P(i) is written; S(i) has been read
    cp_async_wait<0>();
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < kKeyBlock / 16; ++kk) {
        const uint64_t dv = umma_desc(sv + kk * 2 * 128, 128, 1024);
        umma_bf16(tmem + OCOL, umma_desc(sph + kk * 2 * 2048, 2048, 128), dv, idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        umma_bf16(tmem + OCOL, umma_desc(spl + kk * 2 * 2048, 2048, 128), dv, idesc_o, 1u);
      }
      umma_commit(&bar_o);
      if (i + 1 < na) issue_qk();   // S of the next block, queued behind this P V
    }
  }
  sticky_wait(&bar_o, ph_o, kCap, ok);   // the last P V
  if (__syncthreads_or(!ok)) {
    if (tid == 0 && p.err) set_error(p.err, kErrTimeout);
  } else {
    tc_after_sync();
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(trow + OCOL + c0, o);
      tmem_wait_ld();
      if (t < p.T) {
        if (p.out_fp32) {
          float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + orow + c0);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                                 __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.out) + orow + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * k]) * inv, __uint_as_float(o[8 * k + 1]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv));
        }
      }
    }
  }
  cp_async_wait<0>();
  tc_before_sync();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(TCOLS));
}

size_t smd_smem_bytes(int D, int T) {
  const size_t q = (size_t)128 * D * 2, kv = (size_t)64 * D * 2, pt = (size_t)128 * 64 * 2;
  return q + 2 * kv + 2 * pt + ((size_t)(T + 63) / 64 + 1) * 4;
}

template <int D, int G>
static cudaError_t launch_smd_dg(const SmdParams &p, cudaStream_t stream) {
  constexpr int QP = kTcRows / G;
  const size_t smem = smd_smem_bytes(D, p.T);
  cudaError_t e = cudaFuncSetAttribute(smd_attn_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.T + QP - 1) / QP, p.Hkv, p.B);
  return launch_pdl(smd_attn_kernel<D, G>, grid, dim3(kTcThreads), smem, stream, p);
}

template <int D>
static cudaError_t launch_smd_d(const SmdParams &p, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_smd_dg<D, 1>(p, stream);
    case 2: return launch_smd_dg<D, 2>(p, stream);
    default: return launch_smd_dg<D, 4>(p, stream);
  }
}

cudaError_t launch_smd(const SmdParams &p, int D, cudaStream_t stream) {
  if (p.B == 0 || p.T == 0) return cudaSuccess;
  return D == 128 ? launch_smd_d<128>(p, stream) : launch_smd_d<64>(p, stream);
}

}  // namespace kv4
