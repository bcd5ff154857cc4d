// kv4_evict.cu -- page-granular eviction and compaction of a KV4 cache.
//
// KVP promo (arXiv 2602.10238), engineering-limitations section, third item:
// a paged (vLLM-style) cache holds 16-position blocks, so a token ranking is
// applied per block on the mean of the block's scores and whole blocks are
// dropped. KV-streams summary page, method details (core idea): after the
// compaction the cache keeps streaming -- later positions are appended into
// the surviving pages, nothing is flushed or prefilled again. KV4-RL review,
// sec. 3: the first 16 and the last 128 positions keep their INT8 copies.
//
// Per sequence b with L positions in n = ceil(L/16) logical pages:
//  - candidates are the full pages holding no INT8-protected position
//    (p < sink or p >= L - recent): logical pages [jlo, jhi);
//  - a page's key is the fp64 sum of its 16 * Hkv scores, head by head and
//    slot by slot (every candidate has the same count, so the sum orders the
//    pages as their mean does);
//  - k = floor(n * permille / 1000) pages are kept, the n - nc non-candidates
//    counted toward k; the best max(0, k - (n - nc)) candidates by (key
//    descending, index ascending) stay, the other e candidates are evicted;
//  - the page-table row becomes the surviving entries in order, then the
//    entries past page n - 1 (mapped ahead for later appends), then e times
//    -1; the evicted ids go to the free list; the length drops by 16 e;
//  - positions after an evicted page move down 16 each, so the recent window
//    moves down 16 e and ring page q of every head moves to ring page
//    (q - e) mod (recent / 16); the INT4 pages themselves are not touched.
//
// One thread-block cluster of kEvictCluster CTAs per sequence. All of them
// compute page keys and store them into rank 0's shared memory (distributed
// shared memory); after one cluster barrier rank 0 runs the selection and the
// row rewrite while the other ranks rotate the ring (the shift e is known
// before any key is). Selection: a 64-bit radix select (8-bit digits,
// double-buffered histograms) finds the key T of the last kept candidate; it
// stops early once the bin it descends into is kept whole, T then being that
// bin's smallest key. Ties
// at T go to the lower page index (a per-32-page tile scan), and a second tile
// scan numbers the evicted pages, which places every entry of the rewritten
// row. The row is staged in shared memory before any entry is written back.
// The ring rotation has each thread own one 16-byte column of a head's ring
// pages: it loads the column from every ring page, then stores each piece at
// its new page, so the rotation needs no staging buffer.
#include <cooperative_groups.h>

#include "kv4_common.cuh"
#include "kv4_internal.h"
#include "kv4_evict.h"

namespace cg = cooperative_groups;

namespace kv4 {

constexpr int kEvictThreads = 256;
constexpr int kEvictCluster = 4;

namespace {

__device__ __forceinline__ unsigned long long page_key(double s) {
  unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(s));
  if (u == 0x8000000000000000ull) u = 0ull;   // -0 ranks with +0
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Exclusive prefix over v[0..n) in place (warp 0 of the CTA).
__device__ __forceinline__ void tile_scan(int *v, int n, int lane) {
  int carry = 0;
  for (int base = 0; base < n; base += 32) {
    const int w = base + lane;
    const int x = w < n ? v[w] : 0;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (w < n) v[w] = carry + incl - x;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
}

}  // namespace

template <bool kVec>
__global__ void __cluster_dims__(kEvictCluster, 1, 1) __launch_bounds__(kEvictThreads, 2)
    evict_pages_kernel(EvictParams p) {
  extern __shared__ __align__(16) unsigned long long ev_smem[];
  __shared__ unsigned int hist[2][256];
  __shared__ int sh_digit[2], sh_rem[2], sh_whole[2];
  __shared__ unsigned long long sh_min;
  constexpr int NWARP = kEvictThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / kEvictCluster;
  pdl_wait();
  pdl_launch_dependents();
  // Every branch below depends on this sequence's length only, so the CTAs of
  // a cluster take the same ones and meet at the same barriers.
  const int L = p.seq_lens[b];
  if (L < 0 || L > p.pt_stride * kPageTokens || (long long)L > p.score_stride) {
    if (rank == 0 && tid == 0) {
      set_error(p.err, kErrCapacity);
      p.freed_count[b] = 0;
    }
    return;
  }
  const int n = (L + kPageTokens - 1) / kPageTokens;
  const int jlo = p.sink > 0 ? 1 : 0;
  const int jhi = max(jlo, (L - p.recent) / kPageTokens);   // a negative quotient rounds up to <= 0
  const int nc = jhi - jlo;
  long long ksel = (long long)n * p.permille / 1000 - (n - nc);
  ksel = ksel < 0 ? 0 : (ksel > nc ? nc : ksel);
  const int e = nc - static_cast<int>(ksel);
  if (e == 0) {   // nothing leaves: the row, the length and the ring stay as they are
    if (rank == 0 && tid == 0) p.freed_count[b] = 0;
    return;
  }

  const int ntiles = (p.pt_stride + 31) / 32;
  unsigned long long *keys = ev_smem;                                  // [pt_stride], index j - jlo
  int *row = reinterpret_cast<int *>(ev_smem + p.pt_stride);           // [pt_stride]
  int *tile_eq = row + p.pt_stride;                                    // [ntiles]
  int *tile_ev = tile_eq + ntiles;                                     // [ntiles]
  uint32_t *ev_word = reinterpret_cast<uint32_t *>(tile_ev + ntiles);  // [ntiles]
  int32_t *gt = p.page_table + (long long)b * p.pt_stride;
  // rank 0's shared memory may be written only once every CTA of the cluster
  // runs: arrive now, wait just before the first remote store
  cluster.barrier_arrive();
  if (rank == 0)
    for (int j = tid; j < p.pt_stride; j += kEvictThreads) row[j] = gt[j];
  cluster.barrier_wait();

  // page keys of the candidates (only needed when some but not all stay),
  // spread over the cluster; the loads of four heads are issued before their
  // adds, which keep the order
  if (ksel > 0) {
    unsigned long long *keys0 = cluster.map_shared_rank(keys, 0);
    const float *srow = p.scores + (long long)b * p.Hkv * p.score_stride;
    for (int c = rank * kEvictThreads + tid; c < nc; c += kEvictCluster * kEvictThreads) {
      const float *s0 = srow + (long long)(jlo + c) * kPageTokens;
      double acc = 0.0;
      for (int h0 = 0; h0 < p.Hkv; h0 += 4) {
        float v[4][16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (h0 + i < p.Hkv) {
            const float *s = s0 + (long long)(h0 + i) * p.score_stride;
            if constexpr (kVec) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 x = __ldg(reinterpret_cast<const float4 *>(s) + q);
                v[i][4 * q] = x.x;
                v[i][4 * q + 1] = x.y;
                v[i][4 * q + 2] = x.z;
                v[i][4 * q + 3] = x.w;
              }
            } else {
#pragma unroll
              for (int r = 0; r < 16; ++r) v[i][r] = __ldg(s + r);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (h0 + i < p.Hkv) {
#pragma unroll
            for (int r = 0; r < 16; ++r) acc += (double)v[i][r];
          }
        }
      }
      keys0[c] = page_key(acc);
    }
  }

  if (rank != 0) {
    // The keys are in rank 0 once this arrival (a release) completes; the
    // ring pages of every head move down by e mod (recent / 16) meanwhile.
    cluster.barrier_arrive();
    const int nring = p.recent / kPageTokens;
    const int sh = nring > 0 ? e % nring : 0;
    if (sh != 0) {
      const int cols = static_cast<int>(p.side_page_bytes / 16);
      const long long ring0 = p.sink > 0 ? p.side_page_bytes : 0;
      const int tasks = p.Hkv * cols;
      const int g = (rank - 1) * kEvictThreads + tid, G = (kEvictCluster - 1) * kEvictThreads;
      // two columns per step: every load of both is in flight before a store
      for (int t0 = g; t0 < tasks; t0 += 2 * G) {
        uint4 v[2][kMaxRingPages];
        uint8_t *base[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int t = t0 + u * G;
          base[u] = nullptr;
          if (t < tasks) {
            const int h = t / cols, c = t % cols;
            base[u] = p.side + ((long long)b * p.Hkv + h) * p.side_stride + ring0 + 16LL * c;
#pragma unroll
            for (int q = 0; q < kMaxRingPages; ++q)
              if (q < nring) v[u][q] = *reinterpret_cast<const uint4 *>(base[u] + q * p.side_page_bytes);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (base[u] == nullptr) continue;
#pragma unroll
          for (int q = 0; q < kMaxRingPages; ++q) {
            if (q < nring) {
              const int dst = q >= sh ? q - sh : q - sh + nring;
              *reinterpret_cast<uint4 *>(base[u] + dst * p.side_page_bytes) = v[u][q];
            }
          }
        }
      }
    }
    cluster.barrier_wait();
    return;
  }
  cluster.sync();   // rank 0: every key has landed

  // key T of the ksel-th best candidate and how many keys equal to T stay
  unsigned long long T = 0ull;
  int need_eq = 0;
  if (ksel > 0) {
    for (int i = tid; i < 512; i += kEvictThreads) hist[i >> 8][i & 255] = 0u;
    __syncthreads();
    unsigned long long prefix = 0ull, pmask = 0ull;
    int rem = static_cast<int>(ksel);
    bool whole = false;   // every key under `prefix` is kept
    for (int pass = 0; pass < 8 && !whole; ++pass) {
      const int shift = 56 - 8 * pass, cur = pass & 1;
      // warp-strided so that a warp's lanes take one step together; a warp
      // whose matching keys share a digit adds them with one atomic
      for (int c0 = 32 * warp; c0 < nc; c0 += kEvictThreads) {
        const int c = c0 + lane;
        bool m = false;
        unsigned int dig = 0u;
        if (c < nc) {
          const unsigned long long k = keys[c];
          m = (k & pmask) == prefix;
          dig = static_cast<unsigned int>((k >> shift) & 255ull);
        }
        const uint32_t act = __ballot_sync(0xffffffffu, m);
        if (act == 0u) continue;
        const int leader = __ffs(act) - 1;
        const unsigned int d0 = __shfl_sync(0xffffffffu, dig, leader);
        if (__all_sync(0xffffffffu, !m || dig == d0)) {
          if (lane == leader) atomicAdd(&hist[cur][d0], static_cast<unsigned int>(__popc(act)));
        } else if (m) {
          atomicAdd(&hist[cur][dig], 1u);
        }
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins 255-8l .. 248-8l, highest first
        unsigned int hv[8];
        int tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hv[i] = hist[cur][255 - 8 * lane - i];
          tot += static_cast<int>(hv[i]);
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int above = incl - tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int cnt = static_cast<int>(hv[i]);
          if (above < rem && rem <= above + cnt) {
            sh_digit[cur] = 255 - 8 * lane - i;
            sh_rem[cur] = rem - above;
            sh_whole[cur] = rem - above == cnt;
          }
          above += cnt;
        }
      } else if (warp == 1) {
        // the other histogram was last read in the previous pass
        for (int i = lane; i < 256; i += 32) hist[cur ^ 1][i] = 0u;
      }
      __syncthreads();
      prefix |= static_cast<unsigned long long>(sh_digit[cur]) << shift;
      pmask |= 255ull << shift;
      rem = sh_rem[cur];
      whole = sh_whole[cur] != 0 && pass < 7;
    }
    if (whole) {
      // The chosen bin is taken whole: T is its smallest key and every key
      // equal to T stays (keys under a smaller prefix are all below T).
      if (tid == 0) sh_min = ~0ull;
      __syncthreads();
      unsigned long long mn = ~0ull;
      for (int c = tid; c < nc; c += kEvictThreads) {
        const unsigned long long k = keys[c];
        if ((k & pmask) == prefix && k < mn) mn = k;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, mn, o);
        mn = y < mn ? y : mn;
      }
      if (lane == 0) atomicMin(&sh_min, mn);
      __syncthreads();
      T = sh_min;
      need_eq = nc;
    } else {
      T = prefix;
      need_eq = rem;
    }
  }

  // ties at T in page order: per-tile counts, then an exclusive scan
  auto is_cand = [&](int j) { return j >= jlo && j < jhi; };
  for (int w = warp; w < ntiles; w += NWARP) {
    const int j = 32 * w + lane;
    const bool eq = ksel > 0 && is_cand(j) && keys[j - jlo] == T;
    const uint32_t bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) tile_eq[w] = __popc(bal);
  }
  __syncthreads();
  if (warp == 0) tile_scan(tile_eq, ntiles, lane);
  __syncthreads();

  // evicted pages: a bit per page, counts per tile, then their scan
  for (int w = warp; w < ntiles; w += NWARP) {
    const int j = 32 * w + lane;
    bool keep = true, eq = false;
    if (is_cand(j)) {
      if (ksel == 0) {
        keep = false;
      } else {
        const unsigned long long k = keys[j - jlo];
        keep = k > T;
        eq = k == T;
      }
    }
    const uint32_t eqbal = __ballot_sync(0xffffffffu, eq);
    if (eq) keep = tile_eq[w] + __popc(eqbal & ((1u << lane) - 1u)) < need_eq;
    const uint32_t evbal = __ballot_sync(0xffffffffu, !keep);
    if (lane == 0) {
      ev_word[w] = evbal;
      tile_ev[w] = __popc(evbal);
    }
  }
  __syncthreads();
  if (warp == 0) tile_scan(tile_ev, ntiles, lane);
  __syncthreads();

  // rewrite the row (every read comes from the staged copy)
  int32_t *gfree = p.freed + (long long)b * p.pt_stride;
  for (int j = tid; j < p.pt_stride; j += kEvictThreads) {
    const int w = j >> 5, bit = j & 31;
    const uint32_t word = ev_word[w];
    if (j < n) {
      const int before = tile_ev[w] + __popc(word & ((1u << bit) - 1u));
      if ((word >> bit) & 1u) gfree[before] = row[j];
      else gt[j - before] = row[j];
    } else {
      gt[j - e] = row[j];
    }
  }
  for (int t = p.pt_stride - e + tid; t < p.pt_stride; t += kEvictThreads) gt[t] = -1;
  if (tid == 0) {
    p.seq_lens[b] = L - kPageTokens * e;
    p.freed_count[b] = e;
  }
}

size_t evict_smem_bytes(int pt_stride) {
  const size_t ntiles = (size_t)(pt_stride + 31) / 32;
  return (size_t)pt_stride * 8 + (size_t)pt_stride * 4 + ntiles * 12;
}

cudaError_t launch_evict(const EvictParams &p, bool vec, cudaStream_t stream) {
  if (p.B == 0) return cudaSuccess;
  const size_t smem = evict_smem_bytes(p.pt_stride);
  auto kern = vec ? evict_pages_kernel<true> : evict_pages_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(p.B * kEvictCluster), dim3(kEvictThreads), smem, stream, p);
}

}  // namespace kv4
