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
// Flash-attention style, on mma.sync m16n8k16 bf16 tiles. A CTA of four warps
// takes one KV head and 16 * 4/G query positions; warp w owns query head
// g = w % G for positions 16 (w / G) .. +15, so the G heads of a KV head share
// every K/V tile and every mask row. Before the loop the CTA ORs its mask rows
// per 64-key block; blocks with no retained key for any of its rows are never
// loaded. Active blocks stream through a two-stage cp.async ring of K and V
// tiles (rows padded to D + 8 elements so that fragment loads are free of bank
// conflicts). Per block: S = Q K^T (Q fragments held in registers, K fragments
// by ldmatrix), masked
// keys and keys after the query set to -inf, online softmax in base 2, then
// O += P V with P split into bf16 hi + lo parts (two MMAs) so that P keeps
// 16 significant bits; V fragments come from ldmatrix.trans.
#include <math.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"
#include "smd_attn.h"

namespace kv4 {

namespace {

constexpr int kSmdWarps = 4;
constexpr int kSmdThreads = kSmdWarps * 32;
constexpr int kKeyBlock = 64;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kSmdThreads) smd_attn_kernel(SmdParams p) {
  constexpr int QP = 16 * (kSmdWarps / G);   // query positions per CTA
  constexpr int PITCH = D + 8;               // smem row pitch in elements
  constexpr int TILE = kKeyBlock * PITCH;    // elements per K or V tile
  constexpr int CH = D / 8;                  // 16-byte chunks per row
  constexpr int KS = D / 16;                 // k-steps of q.K
  constexpr int ND = D / 8;                  // n-tiles of the output
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16 *ks = reinterpret_cast<__nv_bfloat16 *>(smem);     // [2][TILE]
  __nv_bfloat16 *vs = ks + 2 * TILE;                                 // [2][TILE]
  int *blist = reinterpret_cast<int *>(vs + 2 * TILE);               // [T/64 + 1]
  __shared__ uint32_t active[kMaxSmdBlocks / 32];
  __shared__ int nact;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 2, tig = lane & 3;
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
  const int g = warp % G, pg = warp / G;
  const int hq = h * G + g;
  const int ta = t0 + 16 * pg + grp, tb = ta + 8;   // this lane's two query rows

  // ---- active key blocks of this CTA's rows
  const int tlast = min(t0 + QP, L) - 1;            // last query row that exists
  const int nblk = tlast >= 0 ? tlast / kKeyBlock + 1 : 0;
  for (int i = tid; i < (nblk + 31) / 32; i += kSmdThreads) active[i] = 0u;
  __syncthreads();
  if (p.mask) {
    const int nw = 2 * nblk;                        // mask words covering the blocks
    const int rows = tlast - t0 + 1;
    for (int idx = tid; idx < rows * nw; idx += kSmdThreads) {
      const int r = idx / nw, w = idx % nw;
      const uint32_t word = w < p.mask_stride
                                ? __ldg(p.mask + (((long long)b * p.Hkv + h) * p.T + t0 + r) * p.mask_stride + w)
                                : 0u;
      if (word) atomicOr(&active[(w >> 1) >> 5], 1u << ((w >> 1) & 31));
    }
  } else {
    for (int j = tid; j < nblk; j += kSmdThreads) atomicOr(&active[j >> 5], 1u << (j & 31));
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

  // ---- Q fragments (rows beyond the length are zero)
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16 *qra = p.q + (((long long)b * p.T + ta) * p.Hq + hq) * D;
    const __nv_bfloat16 *qrb = p.q + (((long long)b * p.T + tb) * p.Hq + hq) * D;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const int d = s * 16 + 2 * tig;
      qa[s][0] = ta < L ? *reinterpret_cast<const uint32_t *>(qra + d) : 0u;
      qa[s][1] = tb < L ? *reinterpret_cast<const uint32_t *>(qrb + d) : 0u;
      qa[s][2] = ta < L ? *reinterpret_cast<const uint32_t *>(qra + d + 8) : 0u;
      qa[s][3] = tb < L ? *reinterpret_cast<const uint32_t *>(qrb + d + 8) : 0u;
    }
  }

  auto load_block = [&](int j, int stage) {
    const int kb = j * kKeyBlock;
    for (int c = tid; c < 2 * kKeyBlock * CH; c += kSmdThreads) {
      const int which = c / (kKeyBlock * CH), rem = c % (kKeyBlock * CH);
      const int row = rem / CH, ch = rem % CH;
      const int pos = kb + row;
      const bool in = pos < L;
      const __nv_bfloat16 *base = which ? p.v : p.k;
      const __nv_bfloat16 *src = base + (((long long)b * p.T + (in ? pos : 0)) * p.Hkv + h) * D + ch * 8;
      __nv_bfloat16 *dst = (which ? vs : ks) + stage * TILE + row * PITCH + ch * 8;
      cp_async16(smem_u32(dst), src, in ? 16u : 0u);
    }
    cp_async_commit();
  };

  float o[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
  const uint32_t *mra = p.mask ? p.mask + (((long long)b * p.Hkv + h) * p.T + ta) * p.mask_stride : nullptr;
  const uint32_t *mrb = p.mask ? p.mask + (((long long)b * p.Hkv + h) * p.T + tb) * p.mask_stride : nullptr;

  if (na > 0) load_block(blist[0], 0);
  for (int i = 0; i < na; ++i) {
    if (i + 1 < na) {
      load_block(blist[i + 1], (i + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int j = blist[i], kb = j * kKeyBlock, stage = i & 1;
    const __nv_bfloat16 *kt = ks + stage * TILE;
    const __nv_bfloat16 *vt = vs + stage * TILE;

    // S = Q K^T over the 64 keys of the block
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
    // K fragments by ldmatrix: matrices (keys 8n.., d 16st), (8n.., 16st + 8),
    // (8n + 8.., 16st), (8n + 8.., 16st + 8) give b0, b1 of n-tiles n and n + 1
    const int kmi = lane >> 3, kri = lane & 7;
#pragma unroll
    for (int st = 0; st < KS; ++st) {
#pragma unroll
      for (int n = 0; n < 8; n += 2) {
        uint32_t bk[4];
        ldmatrix_x4(bk, smem_u32(kt + ((n + (kmi >> 1)) * 8 + kri) * PITCH + st * 16 + (kmi & 1) * 8));
        mma_bf16(s[n], qa[st], bk[0], bk[1]);
        mma_bf16(s[n + 1], qa[st], bk[2], bk[3]);
      }
    }

    // visibility: query row < L, key <= query (so key < L), mask bit set
    uint32_t wa0 = 0xffffffffu, wa1 = 0xffffffffu, wb0 = 0xffffffffu, wb1 = 0xffffffffu;
    if (p.mask) {
      const int w0 = kb >> 5;
      wa0 = ta < L && w0 < p.mask_stride ? __ldg(mra + w0) : 0u;
      wa1 = ta < L && w0 + 1 < p.mask_stride ? __ldg(mra + w0 + 1) : 0u;
      wb0 = tb < L && w0 < p.mask_stride ? __ldg(mrb + w0) : 0u;
      wb1 = tb < L && w0 + 1 < p.mask_stride ? __ldg(mrb + w0 + 1) : 0u;
    }
    float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kk = n * 8 + 2 * tig + e;          // key offset in the block
        const int key = kb + kk;
        const uint32_t bit = 1u << (kk & 31);
        const bool va = ta < L && key <= ta && ((kk < 32 ? wa0 : wa1) & bit);
        const bool vb = tb < L && key <= tb && ((kk < 32 ? wb0 : wb1) & bit);
        s[n][e] = va ? s[n][e] * p.scale_log2 : -INFINITY;
        s[n][2 + e] = vb ? s[n][2 + e] * p.scale_log2 : -INFINITY;
        mxa = fmaxf(mxa, s[n][e]);
        mxb = fmaxf(mxb, s[n][2 + e]);
      }
    }
#pragma unroll
    for (int x = 1; x < 4; x <<= 1) {
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, x));
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, x));
    }
    const float mna = fmaxf(ma, mxa), mnb = fmaxf(mb, mxb);
    // a row with nothing visible so far keeps m = -inf, weights 0, factor 1
    const float ca = mna == -INFINITY ? 1.f : ex2(ma - mna);
    const float cb = mnb == -INFINITY ? 1.f : ex2(mb - mnb);
    const float ba = mna == -INFINITY ? 0.f : mna, bb = mnb == -INFINITY ? 0.f : mnb;
    ma = mna;
    mb = mnb;
    la *= ca;
    lb *= cb;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      o[n][0] *= ca;
      o[n][1] *= ca;
      o[n][2] *= cb;
      o[n][3] *= cb;
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      s[n][0] = ex2(s[n][0] - ba);
      s[n][1] = ex2(s[n][1] - ba);
      s[n][2] = ex2(s[n][2] - bb);
      s[n][3] = ex2(s[n][3] - bb);
      la += s[n][0] + s[n][1];
      lb += s[n][2] + s[n][3];
    }

    // O += P V, P as bf16 hi + lo
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      uint32_t ph[4], pl[4];
      const float *s0 = s[2 * kc], *s1 = s[2 * kc + 1];
      const float f[8] = {s0[0], s0[1], s0[2], s0[3], s1[0], s1[1], s1[2], s1[3]};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // a0: row a keys 2tig..; a1: row b; a2: row a keys 8 + 2tig..; a3: row b
        const float x0 = f[(r & 1) * 2 + (r >> 1) * 4], x1 = f[(r & 1) * 2 + (r >> 1) * 4 + 1];
        ph[r] = pack_bf16x2(x0, x1);
        pl[r] = pack_bf16x2(x0 - bf16lo_to_f32(ph[r]), x1 - bf16hi_to_f32(ph[r]));
      }
#pragma unroll
      for (int n = 0; n < ND; n += 2) {
        uint32_t bv[4];
        const int mi = lane >> 3, ri = lane & 7;
        const __nv_bfloat16 *vr = vt + (kc * 16 + (mi & 1) * 8 + ri) * PITCH + (n + (mi >> 1)) * 8;
        ldmatrix_x4_trans(bv, smem_u32(vr));
        mma_bf16(o[n], ph, bv[0], bv[1]);
        mma_bf16(o[n], pl, bv[0], bv[1]);
        mma_bf16(o[n + 1], ph, bv[2], bv[3]);
        mma_bf16(o[n + 1], pl, bv[2], bv[3]);
      }
    }
    __syncthreads();   // the stage is refilled by the next iteration's prefetch
  }

  // ---- normalise and store
#pragma unroll
  for (int x = 1; x < 4; x <<= 1) {
    la += __shfl_xor_sync(0xffffffffu, la, x);
    lb += __shfl_xor_sync(0xffffffffu, lb, x);
  }
  const float ia = la > 0.f ? 1.f / la : 0.f, ib = lb > 0.f ? 1.f / lb : 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int t = half ? tb : ta;
    if (t >= p.T) continue;
    const float inv = half ? ib : ia;
    const long long base = (((long long)b * p.T + t) * p.Hq + hq) * D + 2 * tig;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const float y0 = o[n][2 * half] * inv, y1 = o[n][2 * half + 1] * inv;
      if (p.out_fp32) {
        *reinterpret_cast<float2 *>(reinterpret_cast<float *>(p.out) + base + n * 8) = make_float2(y0, y1);
      } else {
        *reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(p.out) + base + n * 8) =
            pack_bf16x2(y0, y1);
      }
    }
  }
}

size_t smd_smem_bytes(int D, int T) {
  const size_t tile = (size_t)64 * (D + 8) * 2;
  return 4 * tile + ((size_t)(T + 63) / 64 + 1) * 4;
}

template <int D, int G>
static cudaError_t launch_smd_dg(const SmdParams &p, cudaStream_t stream) {
  constexpr int QP = 16 * (kSmdWarps / G);
  const size_t smem = smd_smem_bytes(D, p.T);
  cudaError_t e = cudaFuncSetAttribute(smd_attn_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.T + QP - 1) / QP, p.Hkv, p.B);
  return launch_pdl(smd_attn_kernel<D, G>, grid, dim3(kSmdThreads), smem, stream, p);
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
