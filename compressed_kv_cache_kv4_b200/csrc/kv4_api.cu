// kv4_api.cu -- the extern "C" boundary of libkv4 (declared in include/kv4.h).
//
// Host-side argument validation, workspace layout, worker planning and kernel
// launches on the caller's stream. No device memory is allocated except the
// 4-byte error word of a kv4_cache.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "../../include/kv4.h"
#include "kv4_common.cuh"
#include "kv4_internal.h"
#include "kv4_evict.h"
#include "smd_attn.h"

using namespace kv4;

struct kv4_cache {
  kv4_config cfg;
  uint8_t *pool;
  size_t pool_bytes;
  uint8_t *side;
  size_t side_bytes;
  uint32_t *err;
  int device;
  int num_sms;
  long long wait_cap;
};

int kv4::cache_device(const kv4_cache *cache) { return cache ? cache->device : -1; }

namespace {

constexpr size_t kAlign = 256;

// Last CUDA runtime error seen by a libkv4 call of this thread (kv4_last_cuda_error).
thread_local cudaError_t g_last_cuda = cudaSuccess;

// True (and recorded) if e is an error.
bool bad(cudaError_t e) {
  if (e == cudaSuccess) return false;
  g_last_cuda = e;
  return true;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

long long page_head_bytes(int D) { return 18LL * D; }

// INT8 side block of one (sequence, KV head): a sink page (when sink > 0) and
// recent/16 ring pages of 32*D + 64 bytes each.
long long side_head_bytes(int D, int sink, int recent) {
  return (long long)((sink > 0 ? 1 : 0) + recent / 16) * (32LL * D + 64);
}

int slot_o_off(int G) { return (int)round_up((size_t)(2 * G), 4); }
int slot_floats(int G, int D) { return slot_o_off(G) + G * D; }

kv4_status check_config(const kv4_config *c) {
  if (!c) return KV4_ERR_INVALID;
  if (c->num_kv_heads < 1 || c->max_seqs < 1 || c->num_pages < 1) return KV4_ERR_INVALID;
  if (c->page_tokens != kPageTokens || c->group != kGroup) return KV4_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return KV4_ERR_UNSUPPORTED;
  if (c->sink < 0 || c->sink > 16 || c->recent < 0 || c->recent > 128 || c->recent % 16) return KV4_ERR_UNSUPPORTED;
  return KV4_OK;
}

// ---------------------------------------------------------------- launch geometry, per device
struct DeviceInfo {
  int sms = 0, smem_sm = 0, smem_reserved = 0, smem_optin = 0;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;
std::map<std::tuple<int, int, int>, cudaError_t> g_kv4_attr;             // (device, D, G)
std::map<std::tuple<int, int, int, int, int>, int> g_kv4_occ;            // (device, D, G, HB, smem)
std::map<std::tuple<int, int, int>, std::pair<cudaError_t, DecodeLaunch>> g_bf16_geo;   // (device, D, G)

// Attributes of the current device (looked up once per device).
cudaError_t device_info(int *dev_out, DeviceInfo *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  auto it = g_dev.find(dev);
  if (it == g_dev.end()) {
    DeviceInfo d;
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    it = g_dev.emplace(dev, d).first;
  }
  *dev_out = dev;
  *out = it->second;
  return cudaSuccess;
}

// Heads per CTA of the KV4 kernel: the largest divisor of Hkv that is <= 8.
int kv4_head_block(int Hkv) {
  for (int hb = Hkv < 8 ? Hkv : 8; hb > 1; --hb)
    if (Hkv % hb == 0) return hb;
  return 1;
}

struct Kv4Plan {
  int HB, NVB, NS, smem, n_cta;
};

// Launch plan of the KV4 kernel for B sequences on the current device: as
// many ring stages (up to 6) as let 16 warps (16 / HB CTAs) share an SM, and
// by default as many CTAs as are resident at once (num_workers > 0: that many
// warps, i.e. ceil(num_workers / HB) CTAs).
kv4_status kv4_plan(int D, int G, int Hkv, int B, int num_workers, Kv4Plan *out) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev = 0;
  DeviceInfo di;
  if (bad(device_info(&dev, &di))) return KV4_ERR_CUDA;
  Kv4Plan pl{};
  pl.HB = kv4_head_block(Hkv);
  const long long nvb = (long long)B * (Hkv / pl.HB);
  if (nvb > kMaxBatch) return KV4_ERR_UNSUPPORTED;
  pl.NVB = static_cast<int>(nvb);
  const int target = 16 / pl.HB > 0 ? 16 / pl.HB : 1;
  const int budget = (di.smem_sm - target * di.smem_reserved) / target;
  pl.NS = 6;
  while (pl.NS > 2 && kv4_smem_bytes(D, pl.HB, pl.NS, pl.NVB) > budget) --pl.NS;
  pl.smem = kv4_smem_bytes(D, pl.HB, pl.NS, pl.NVB);
  if (pl.smem > di.smem_optin) return KV4_ERR_UNSUPPORTED;
  const auto key = std::make_tuple(dev, D, G, pl.HB, pl.smem);
  auto it = g_kv4_occ.find(key);
  if (it == g_kv4_occ.end()) {
    // the dynamic shared-memory limit is raised once per (device, D, G) to
    // the device's opt-in maximum, which covers every plan
    const auto akey = std::make_tuple(dev, D, G);
    if (g_kv4_attr.find(akey) == g_kv4_attr.end())
      g_kv4_attr.emplace(akey, kv4_decode_set_smem_limit(D, G, di.smem_optin));
    if (bad(g_kv4_attr[akey])) return KV4_ERR_CUDA;
    int nb = 0;
    if (bad(kv4_decode_occupancy(D, G, pl.HB, pl.smem, &nb))) return KV4_ERR_CUDA;
    it = g_kv4_occ.emplace(key, nb > 0 ? nb : 1).first;
  }
  const long long def = (long long)it->second * di.sms;
  const long long want = num_workers > 0 ? ((long long)num_workers + pl.HB - 1) / pl.HB : def;
  pl.n_cta = static_cast<int>(want < 1 ? 1 : (want > (1 << 20) ? (1 << 20) : want));
  *out = pl;
  return KV4_OK;
}

// bf16 comparison kernel geometry, per device.
cudaError_t bf16_geometry(int D, int G, DecodeLaunch *out, int *num_sms) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev = 0;
  DeviceInfo di;
  cudaError_t e = device_info(&dev, &di);
  if (e != cudaSuccess) return e;
  const auto key = std::make_tuple(dev, D, G);
  auto it = g_bf16_geo.find(key);
  if (it == g_bf16_geo.end()) {
    DecodeLaunch l{};
    const cudaError_t pe = bf16_decode_prepare(D, G, &l);
    it = g_bf16_geo.emplace(key, std::make_pair(pe, l)).first;
  }
  if (it->second.first != cudaSuccess) return it->second.first;
  *out = it->second.second;
  *num_sms = di.sms;
  return cudaSuccess;
}

int bf16_workers(int requested, const DecodeLaunch &l, int num_sms) {
  const int nw = requested > 0 ? requested : num_sms * l.blocks_per_sm * kWarps;
  return (nw + kWarps - 1) / kWarps * kWarps;
}

// KV4 workspace: plan int32 [NVB+1] | first, last int32 [2*NVB] each |
// partial slots [2*NVB + n_cta][HB][slot_floats] (INT8 ranges, then INT4
// ranges, each offset by the CTA index).
size_t kv4_ws_bytes(const Kv4Plan &pl, int G, int D) {
  const size_t slot = (size_t)slot_floats(G, D) * 4;
  return round_up((size_t)(pl.NVB + 1) * 4, kAlign) + 2 * round_up((size_t)2 * pl.NVB * 4, kAlign) +
         round_up(((size_t)2 * pl.NVB + pl.n_cta) * pl.HB * slot, kAlign);
}

// bf16 workspace: plan int32 [B+1] | first, last int32 [2*B*Hkv] each |
// partial slots [2*B*Hkv + nw][slot_floats].
size_t bf16_ws_bytes(int B, int Hkv, int G, int D, int nw) {
  const size_t slot = (size_t)slot_floats(G, D) * 4;
  return round_up((size_t)(B + 1) * 4, kAlign) + 2 * round_up((size_t)2 * B * Hkv * 4, kAlign) +
         round_up(((size_t)2 * B * Hkv + nw) * slot, kAlign);
}

// Carve a workspace with `nplan` plan entries and `nrange` ranges.
void carve_workspace(DecodeParams &p, void *ws, size_t nplan, size_t nrange) {
  uint8_t *w = static_cast<uint8_t *>(ws);
  p.plan = reinterpret_cast<int *>(w);
  w += round_up(nplan * 4, kAlign);
  p.first = reinterpret_cast<int *>(w);
  w += round_up(nrange * 4, kAlign);
  p.last = reinterpret_cast<int *>(w);
  w += round_up(nrange * 4, kAlign);
  p.slots = reinterpret_cast<float *>(w);
}

kv4_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return KV4_OK;
  g_last_cuda = e;
  return KV4_ERR_CUDA;
}

// Timing hook state: per kind, a fixed pool of event pairs filled in call order.
struct Timing {
  bool on = false;
  int max_records = 0;
  int every = 1;          // record every `every`-th call of a kind
  int used[2] = {0, 0};
  long long calls[2] = {0, 0};
  std::vector<cudaEvent_t> ev[2];   // 2 * max_records events per kind
};
Timing g_timing;
std::mutex g_timing_mu;

void timing_pair(int kind, cudaEvent_t *e0, cudaEvent_t *e1) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  *e0 = *e1 = nullptr;
  if (!g_timing.on || g_timing.used[kind] >= g_timing.max_records) return;
  if (g_timing.calls[kind]++ % g_timing.every != 0) return;
  const int i = g_timing.used[kind]++;
  *e0 = g_timing.ev[kind][2 * i];
  *e1 = g_timing.ev[kind][2 * i + 1];
}

void timing_free() {
  for (int k = 0; k < 2; ++k) {
    for (cudaEvent_t e : g_timing.ev[k]) cudaEventDestroy(e);
    g_timing.ev[k].clear();
    g_timing.used[k] = 0;
    g_timing.calls[k] = 0;
  }
  g_timing.on = false;
  g_timing.max_records = 0;
}

}  // namespace

extern "C" {

const char *kv4_last_cuda_error(void) {
  return g_last_cuda == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda);
}

const char *kv4_status_string(kv4_status s) {
  switch (s) {
    case KV4_OK: return "KV4_OK";
    case KV4_ERR_INVALID: return "KV4_ERR_INVALID";
    case KV4_ERR_UNSUPPORTED: return "KV4_ERR_UNSUPPORTED";
    case KV4_ERR_CAPACITY: return "KV4_ERR_CAPACITY";
    case KV4_ERR_BOUNDS: return "KV4_ERR_BOUNDS";
    case KV4_ERR_RANGE: return "KV4_ERR_RANGE";
    case KV4_ERR_TIMEOUT: return "KV4_ERR_TIMEOUT";
    case KV4_ERR_CUDA: return "KV4_ERR_CUDA";
  }
  return "KV4_ERR_UNKNOWN";
}

kv4_status kv4_cache_bytes(const kv4_config *cfg, size_t *page_pool_bytes, size_t *side_cache_bytes) {
  const kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  if (!page_pool_bytes || !side_cache_bytes) return KV4_ERR_INVALID;
  *page_pool_bytes = (size_t)cfg->num_pages * cfg->num_kv_heads * page_head_bytes(cfg->head_dim);
  *side_cache_bytes =
      (size_t)cfg->max_seqs * cfg->num_kv_heads * side_head_bytes(cfg->head_dim, cfg->sink, cfg->recent);
  return KV4_OK;
}

kv4_status kv4_cache_create(const kv4_config *cfg, void *page_pool, size_t pool_bytes, void *side_cache,
                            size_t side_bytes, kv4_cache **out) {
  size_t need_pool = 0, need_side = 0;
  const kv4_status st = kv4_cache_bytes(cfg, &need_pool, &need_side);
  if (st != KV4_OK) return st;
  if (!out || !page_pool || pool_bytes < need_pool) return KV4_ERR_INVALID;
  if (need_side > 0 && (!side_cache || side_bytes < need_side)) return KV4_ERR_INVALID;
  if (!aligned(page_pool, 16) || (side_cache && !aligned(side_cache, 16))) return KV4_ERR_INVALID;
  kv4_cache *c = new kv4_cache();
  c->cfg = *cfg;
  c->pool = static_cast<uint8_t *>(page_pool);
  c->pool_bytes = pool_bytes;
  c->side = static_cast<uint8_t *>(side_cache);
  c->side_bytes = side_bytes;
  c->wait_cap = kDefaultWaitCycles;
  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (e == cudaSuccess) e = cudaMalloc(&c->err, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(c->err, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    if (c->err) cudaFree(c->err);
    delete c;
    return KV4_ERR_CUDA;
  }
  *out = c;
  return KV4_OK;
}

void kv4_cache_destroy(kv4_cache *cache) {
  if (!cache) return;
  if (cache->err) cudaFree(cache->err);
  delete cache;
}

kv4_status kv4_append(kv4_cache *cache, void *stream, const void *k_new, const void *v_new,
                      const int32_t *new_offsets, const int32_t *seq_lens_old, const int32_t *page_table,
                      int32_t pt_stride, int32_t B, int64_t total_new) {
  if (!cache) return KV4_ERR_INVALID;
  if (B < 0 || total_new < 0 || pt_stride < 1) return KV4_ERR_INVALID;
  if (B == 0 || total_new == 0) return KV4_OK;
  if (B > cache->cfg.max_seqs) return KV4_ERR_CAPACITY;
  if (!k_new || !v_new || !seq_lens_old || !page_table) return KV4_ERR_INVALID;
  if (!new_offsets && total_new != B) return KV4_ERR_INVALID;
  const int D = cache->cfg.head_dim;
  if (!aligned(k_new, 8) || !aligned(v_new, 8)) return KV4_ERR_INVALID;
  AppendParams p{};
  p.k = static_cast<const __nv_bfloat16 *>(k_new);
  p.v = static_cast<const __nv_bfloat16 *>(v_new);
  p.offsets = new_offsets;
  p.lens_old = seq_lens_old;
  p.page_table = page_table;
  p.pt_stride = pt_stride;
  p.B = B;
  p.Hkv = cache->cfg.num_kv_heads;
  p.sink = cache->cfg.sink;
  p.recent = cache->cfg.recent;
  p.num_pages = cache->cfg.num_pages;
  p.T = total_new;
  p.pool = cache->pool;
  p.side = cache->side;
  p.head_bytes = page_head_bytes(D);
  p.page_bytes = p.head_bytes * p.Hkv;
  p.side_stride = side_head_bytes(D, p.sink, p.recent);
  p.err = cache->err;
  p.num_sms = cache->num_sms;
  return cuda_status(launch_append(p, D, static_cast<cudaStream_t>(stream)));
}

kv4_status kv4_workspace_bytes(const kv4_cache *cache, int32_t B, int32_t num_q_heads, int32_t num_workers,
                               size_t *bytes) {
  if (!cache || !bytes || B < 0 || num_workers < 0) return KV4_ERR_INVALID;
  const int Hkv = cache->cfg.num_kv_heads;
  if (num_q_heads < 1 || num_q_heads % Hkv) return KV4_ERR_INVALID;
  const int G = num_q_heads / Hkv;
  if (G != 1 && G != 2 && G != 4) return KV4_ERR_UNSUPPORTED;
  if (B == 0) {
    *bytes = 0;
    return KV4_OK;
  }
  Kv4Plan pl{};
  const kv4_status st = kv4_plan(cache->cfg.head_dim, G, Hkv, B, num_workers, &pl);
  if (st != KV4_OK) return st;
  *bytes = kv4_ws_bytes(pl, G, cache->cfg.head_dim);
  return KV4_OK;
}

}  // extern "C"

namespace {

// kv4_decode_attn and kv4_decode_partials: the whole INT4 region and the INT8
// region of every sequence, or one page-range shard of the INT4 region
// (page_begin/page_end) with or without the INT8 region.
kv4_status decode_call(kv4_cache *cache, void *stream, const void *q, int32_t Hq, const int32_t *seq_lens,
                       const int32_t *page_table, int32_t pt_stride, const int32_t *page_begin,
                       const int32_t *page_end, int32_t with_int8, const uint32_t *retain_mask, int32_t mask_stride,
                       float softmax_scale, int32_t num_workers, void *workspace, size_t ws_bytes, void *out,
                       int32_t out_is_fp32, float *partials, int32_t B) {
  if (!cache || B < 0 || pt_stride < 1 || num_workers < 0) return KV4_ERR_INVALID;
  if (B == 0) return KV4_OK;
  if (B > cache->cfg.max_seqs) return KV4_ERR_CAPACITY;
  if (B > kMaxBatch) return KV4_ERR_UNSUPPORTED;
  const int Hkv = cache->cfg.num_kv_heads, D = cache->cfg.head_dim;
  if (Hq < 1 || Hq % Hkv) return KV4_ERR_INVALID;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4) return KV4_ERR_UNSUPPORTED;
  if (!q || !seq_lens || !page_table || !workspace || (!out && !partials)) return KV4_ERR_INVALID;
  if (!aligned(q, 16) || (out && !aligned(out, 16)) || (partials && !aligned(partials, 16)) ||
      !aligned(workspace, 16))
    return KV4_ERR_INVALID;
  if ((page_begin == nullptr) != (page_end == nullptr)) return KV4_ERR_INVALID;
  if (retain_mask && (long long)mask_stride * 32 < (long long)pt_stride * kPageTokens) return KV4_ERR_INVALID;
  if (!isfinite(softmax_scale)) return KV4_ERR_INVALID;
  if (pt_stride > kMaxPtStride) return KV4_ERR_UNSUPPORTED;
  int dev = -1;
  if (bad(cudaGetDevice(&dev))) return KV4_ERR_CUDA;
  if (dev != cache->device) return KV4_ERR_INVALID;
  Kv4Plan pl{};
  const kv4_status ps = kv4_plan(D, G, Hkv, B, num_workers, &pl);
  if (ps != KV4_OK) return ps;
  const bool has8 = cache->cfg.sink + cache->cfg.recent > 0 && with_int8;
  if (ws_bytes < kv4_ws_bytes(pl, G, D)) return KV4_ERR_INVALID;

  DecodeParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.sink = cache->cfg.sink;
  p.recent = cache->cfg.recent;
  p.num_pages = cache->cfg.num_pages;
  p.pt_stride = pt_stride;
  p.mask_stride = mask_stride;
  p.num_workers = pl.n_cta * pl.HB;
  p.slot_floats = slot_floats(G, D);
  p.slot_o_off = slot_o_off(G);
  p.int8_units = has8 ? 1 : 0;
  p.HB = pl.HB;
  p.NVB = pl.NVB;
  p.NS = pl.NS;
  p.np8 = side_pages(p.sink, p.recent);
  p.n_cta = pl.n_cta;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.mask = retain_mask;
  p.pool = cache->pool;
  p.side = cache->side;
  p.head_bytes = page_head_bytes(D);
  p.page_bytes = p.head_bytes * Hkv;
  p.side_stride = side_head_bytes(D, p.sink, p.recent);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.out_fp32 = out_is_fp32 ? 1 : 0;
  p.page_begin = page_begin;
  p.page_end = page_end;
  p.partials = partials;
  p.err = cache->err;
  p.wait_cap = cache->wait_cap;
  carve_workspace(p, workspace, (size_t)pl.NVB + 1, (size_t)2 * pl.NVB);
  cudaEvent_t e0, e1;
  timing_pair(0, &e0, &e1);
  return cuda_status(launch_decode(p, D, false, static_cast<cudaStream_t>(stream), e0, e1));
}

}  // namespace

extern "C" {

kv4_status kv4_decode_attn(kv4_cache *cache, void *stream, const void *q, int32_t Hq, const int32_t *seq_lens,
                           const int32_t *page_table, int32_t pt_stride, const uint32_t *retain_mask,
                           int32_t mask_stride, float softmax_scale, int32_t num_workers, void *workspace,
                           size_t ws_bytes, void *out, int32_t out_is_fp32, int32_t B) {
  if (!out && B > 0) return KV4_ERR_INVALID;
  return decode_call(cache, stream, q, Hq, seq_lens, page_table, pt_stride, nullptr, nullptr, 1, retain_mask,
                     mask_stride, softmax_scale, num_workers, workspace, ws_bytes, out, out_is_fp32, nullptr, B);
}

kv4_status kv4_decode_partials(kv4_cache *cache, void *stream, const void *q, int32_t Hq, const int32_t *seq_lens,
                               const int32_t *page_table, int32_t pt_stride, const int32_t *page_begin,
                               const int32_t *page_end, int32_t with_int8, const uint32_t *retain_mask,
                               int32_t mask_stride, float softmax_scale, int32_t num_workers, void *workspace,
                               size_t ws_bytes, float *partials, int32_t B) {
  if (!partials && B > 0) return KV4_ERR_INVALID;
  return decode_call(cache, stream, q, Hq, seq_lens, page_table, pt_stride, page_begin, page_end, with_int8,
                     retain_mask, mask_stride, softmax_scale, num_workers, workspace, ws_bytes, nullptr, 0, partials,
                     B);
}

}  // extern "C"

namespace {

// Workspace of kv4_decode_attn_masked: counts [B*Hkv] | word prefix counts
// [B*Hkv*words] | partials [W][B][Hq][D+4] (one per warp of the gathering
// kernel).
struct MaskedLayout {
  size_t counts, wpre, parts, total;
  int words, nparts;
};

MaskedLayout masked_layout(const kv4_cache *cache, int B, int Hq, int pt_stride) {
  const int D = cache->cfg.head_dim, Hkv = cache->cfg.num_kv_heads;
  MaskedLayout l{};
  l.words = (pt_stride * kPageTokens + 31) / 32;
  l.nparts = masked_decode_warps();
  size_t o = 0;
  l.counts = o;
  o += round_up((size_t)B * Hkv * 4, kAlign);
  l.wpre = o;
  o += round_up((size_t)B * Hkv * l.words * 4, kAlign);
  l.parts = o;
  o += round_up((size_t)l.nparts * B * Hq * (D + 4) * 4, kAlign);
  l.total = o;
  return l;
}

kv4_status masked_check(const kv4_cache *cache, int B, int Hq, int pt_stride, int max_retained, Kv4Plan *pl) {
  if (!cache || B < 0 || Hq < 1 || pt_stride < 1 || max_retained < 0) return KV4_ERR_INVALID;
  const int Hkv = cache->cfg.num_kv_heads, D = cache->cfg.head_dim;
  if (Hq % Hkv) return KV4_ERR_INVALID;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4) return KV4_ERR_UNSUPPORTED;
  if (B > cache->cfg.max_seqs) return KV4_ERR_CAPACITY;
  if (B > kMaxBatch || pt_stride > kMaxPtStride) return KV4_ERR_UNSUPPORTED;
  return kv4_plan(D, G, Hkv, B > 0 ? B : 1, 0, pl);
}

}  // namespace

extern "C" {

kv4_status kv4_masked_workspace_bytes(const kv4_cache *cache, int32_t B, int32_t Hq, int32_t pt_stride,
                                      int32_t max_retained, size_t *bytes) {
  if (!bytes) return KV4_ERR_INVALID;
  Kv4Plan pl{};
  const kv4_status st = masked_check(cache, B, Hq, pt_stride, max_retained, &pl);
  if (st != KV4_OK) return st;
  *bytes = masked_layout(cache, B, Hq, pt_stride).total;
  return KV4_OK;
}

kv4_status kv4_decode_attn_masked(kv4_cache *cache, void *stream, const void *q, int32_t Hq,
                                  const int32_t *seq_lens, const int32_t *page_table, int32_t pt_stride,
                                  const uint32_t *retain_mask, int32_t mask_stride, int32_t max_retained,
                                  float softmax_scale, void *workspace, size_t ws_bytes, void *out,
                                  int32_t out_is_fp32, int32_t B) {
  Kv4Plan pl{};
  const kv4_status st = masked_check(cache, B, Hq, pt_stride, max_retained, &pl);
  if (st != KV4_OK) return st;
  if (B == 0) return KV4_OK;
  if (!q || !seq_lens || !page_table || !retain_mask || !workspace || !out) return KV4_ERR_INVALID;
  if (!aligned(workspace, kAlign) || !aligned(out, 16) || !aligned(q, 16)) return KV4_ERR_INVALID;
  if ((long long)mask_stride * 32 < (long long)pt_stride * kPageTokens) return KV4_ERR_INVALID;
  if (!isfinite(softmax_scale)) return KV4_ERR_INVALID;
  int dev = -1;
  if (bad(cudaGetDevice(&dev))) return KV4_ERR_CUDA;
  if (dev != cache->device) return KV4_ERR_INVALID;
  const MaskedLayout l = masked_layout(cache, B, Hq, pt_stride);
  if (ws_bytes < l.total) return KV4_ERR_INVALID;
  const int D = cache->cfg.head_dim, Hkv = cache->cfg.num_kv_heads, G = Hq / Hkv;
  uint8_t *w = static_cast<uint8_t *>(workspace);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *parts = reinterpret_cast<float *>(w + l.parts);
  // 1. retained INT4-region rows per (sequence, head), and prefix counts per mask word
  GatherParams g{};
  g.mask = retain_mask;
  g.seq_lens = seq_lens;
  g.B = B;
  g.Hkv = Hkv;
  g.sink = cache->cfg.sink;
  g.recent = cache->cfg.recent;
  g.pt_stride = pt_stride;
  g.mask_stride = mask_stride;
  g.max_retained = max_retained;
  g.words = l.words;
  g.wpre = reinterpret_cast<int *>(w + l.wpre);
  g.counts = reinterpret_cast<int *>(w + l.counts);
  g.err = cache->err;
  if (bad(launch_masked_count(g, s))) return KV4_ERR_CUDA;
  // 2. the retained rows gathered on chip and attended, one partial per warp
  DecodeParams dp{};
  dp.B = B;
  dp.Hq = Hq;
  dp.Hkv = Hkv;
  dp.G = G;
  dp.sink = cache->cfg.sink;
  dp.recent = cache->cfg.recent;
  dp.num_pages = cache->cfg.num_pages;
  dp.pt_stride = pt_stride;
  dp.q = static_cast<const __nv_bfloat16 *>(q);
  dp.seq_lens = seq_lens;
  dp.page_table = page_table;
  dp.pool = cache->pool;
  dp.head_bytes = page_head_bytes(D);
  dp.page_bytes = dp.head_bytes * Hkv;
  dp.scale_log2 = softmax_scale * 1.4426950408889634f;
  dp.err = cache->err;
  dp.side = cache->side;
  dp.side_stride = side_head_bytes(D, dp.sink, dp.recent);
  dp.np8 = side_pages(dp.sink, dp.recent);
  dp.int8_units = dp.sink + dp.recent > 0 ? 1 : 0;
  if (bad(launch_masked_decode(dp, g, parts, D, s))) return KV4_ERR_CUDA;
  // 3. the exact merge of the warps' partials
  return cuda_status(launch_merge_partials(parts, l.nparts, (long long)B * Hq, D, out, out_is_fp32 ? 1 : 0, s));
}

kv4_status kv4_merge_partials(void *stream, const float *partials, int32_t N, int32_t B, int32_t Hq, int32_t D,
                              void *out, int32_t out_is_fp32) {
  if (N < 0 || B < 0 || Hq < 1) return KV4_ERR_INVALID;
  if (D != 64 && D != 128) return KV4_ERR_UNSUPPORTED;
  if (B == 0) return KV4_OK;
  if (!out || (N > 0 && !partials)) return KV4_ERR_INVALID;
  if (!aligned(out, 16) || (partials && !aligned(partials, 16))) return KV4_ERR_INVALID;
  return cuda_status(launch_merge_partials(partials, N, (long long)B * Hq, D, out, out_is_fp32 ? 1 : 0,
                                           static_cast<cudaStream_t>(stream)));
}

kv4_status kv_topk_retain(void *stream, const float *scores, int64_t score_stride, const int32_t *seq_lens,
                          int32_t B, int32_t Hkv, int32_t budget_permille, int32_t sink, int32_t recent,
                          uint32_t *mask_out, int32_t mask_stride, int32_t *count_out, int32_t max_len) {
  if (B < 0 || Hkv < 1 || max_len < 0) return KV4_ERR_INVALID;
  if (B == 0) return KV4_OK;
  if (!scores || !seq_lens || !mask_out) return KV4_ERR_INVALID;
  if (budget_permille < 0 || budget_permille > 1000 || sink < 0 || recent < 0) return KV4_ERR_INVALID;
  if (score_stride < max_len || (long long)mask_stride * 32 < max_len) return KV4_ERR_INVALID;
  if (max_len > 1500000) return KV4_ERR_UNSUPPORTED;
  TopkParams p{};
  p.scores = scores;
  p.score_stride = score_stride;
  p.seq_lens = seq_lens;
  p.B = B;
  p.Hkv = Hkv;
  p.permille = budget_permille;
  p.sink = sink;
  p.recent = recent;
  p.max_len = max_len;
  p.mask_stride = mask_stride;
  p.vec_ok = (aligned(scores, 16) && score_stride % 4 == 0) ? 1 : 0;
  p.mask = mask_out;
  p.count = count_out;
  return cuda_status(launch_topk(p, static_cast<cudaStream_t>(stream)));
}

kv4_status bf16_paged_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t num_workers,
                                      size_t *bytes) {
  if (!bytes || B < 0 || Hkv < 1 || Hq < 1 || Hq % Hkv || num_workers < 0) return KV4_ERR_INVALID;
  const int G = Hq / Hkv;
  if ((G != 1 && G != 2 && G != 4) || (D != 64 && D != 128)) return KV4_ERR_UNSUPPORTED;
  DecodeLaunch l{};
  int sms = 0;
  if (bad(bf16_geometry(D, G, &l, &sms))) return KV4_ERR_CUDA;
  *bytes = bf16_ws_bytes(B, Hkv, G, D, bf16_workers(num_workers, l, sms));
  return KV4_OK;
}

kv4_status bf16_paged_decode_attn(void *stream, const void *q, int32_t Hq, int32_t Hkv, int32_t D,
                                  const void *kv_pages, int32_t num_pages, const int32_t *page_table,
                                  int32_t pt_stride, const int32_t *seq_lens, float softmax_scale,
                                  int32_t num_workers, void *workspace, size_t ws_bytes, void *out,
                                  int32_t out_is_fp32, int32_t B, uint32_t *error_word) {
  if (B < 0 || Hkv < 1 || Hq < 1 || Hq % Hkv || pt_stride < 1 || num_pages < 1 || num_workers < 0)
    return KV4_ERR_INVALID;
  if (B == 0) return KV4_OK;
  if (B > kMaxBatch) return KV4_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if ((G != 1 && G != 2 && G != 4) || (D != 64 && D != 128)) return KV4_ERR_UNSUPPORTED;
  if (!q || !kv_pages || !page_table || !seq_lens || !workspace || !out) return KV4_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 16) || !aligned(kv_pages, 16))
    return KV4_ERR_INVALID;
  if (!isfinite(softmax_scale)) return KV4_ERR_INVALID;
  DecodeLaunch l{};
  int sms = 0;
  if (bad(bf16_geometry(D, G, &l, &sms))) return KV4_ERR_CUDA;
  const int nw = bf16_workers(num_workers, l, sms);
  if (ws_bytes < bf16_ws_bytes(B, Hkv, G, D, nw)) return KV4_ERR_INVALID;
  DecodeParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.num_pages = num_pages;
  p.pt_stride = pt_stride;
  p.num_workers = nw;
  p.slot_floats = slot_floats(G, D);
  p.slot_o_off = slot_o_off(G);
  p.int8_units = 0;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.pool = static_cast<const uint8_t *>(kv_pages);
  p.head_bytes = 64LL * D;
  p.page_bytes = p.head_bytes * Hkv;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.out_fp32 = out_is_fp32 ? 1 : 0;
  p.err = error_word;
  p.wait_cap = kDefaultWaitCycles;
  carve_workspace(p, workspace, (size_t)B + 1, (size_t)2 * B * Hkv);
  cudaEvent_t e0, e1;
  timing_pair(1, &e0, &e1);
  return cuda_status(launch_decode(p, D, true, static_cast<cudaStream_t>(stream), e0, e1));
}

kv4_status kv4_evict_pages(kv4_cache *cache, void *stream, const float *scores, int64_t score_stride,
                           int32_t budget_permille, int32_t *seq_lens, int32_t *page_table, int32_t pt_stride,
                           int32_t *freed_pages, int32_t *freed_count, int32_t B) {
  if (!cache) return KV4_ERR_INVALID;
  if (B < 0 || pt_stride < 1 || score_stride < 0) return KV4_ERR_INVALID;
  if (budget_permille < 0 || budget_permille > 1000) return KV4_ERR_INVALID;
  if (B == 0) return KV4_OK;
  if (B > cache->cfg.max_seqs) return KV4_ERR_CAPACITY;
  if (!scores || !seq_lens || !page_table || !freed_pages || !freed_count) return KV4_ERR_INVALID;
  if (!aligned(scores, 4)) return KV4_ERR_INVALID;
  if (pt_stride > kEvictMaxPages) return KV4_ERR_UNSUPPORTED;
  EvictParams p{};
  p.scores = scores;
  p.score_stride = score_stride;
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.freed = freed_pages;
  p.freed_count = freed_count;
  p.pt_stride = pt_stride;
  p.B = B;
  p.Hkv = cache->cfg.num_kv_heads;
  p.permille = budget_permille;
  p.sink = cache->cfg.sink;
  p.recent = cache->cfg.recent;
  p.side = cache->side;
  p.side_stride = side_head_bytes(cache->cfg.head_dim, p.sink, p.recent);
  p.side_page_bytes = 32LL * cache->cfg.head_dim + 64;
  p.err = cache->err;
  const bool vec = aligned(scores, 16) && score_stride % 4 == 0;
  return cuda_status(launch_evict(p, vec, static_cast<cudaStream_t>(stream)));
}

kv4_status smd_masked_attn(void *stream, const void *q, const void *k, const void *v, int32_t B, int32_t T,
                           int32_t Hq, int32_t Hkv, int32_t D, const int32_t *seq_lens, const uint32_t *mask,
                           int32_t mask_stride, float softmax_scale, void *out, int32_t out_is_fp32,
                           uint32_t *error_word) {
  if (B < 0 || T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv) return KV4_ERR_INVALID;
  if (B == 0 || T == 0) return KV4_OK;
  if (!q || !k || !v || !out) return KV4_ERR_INVALID;
  const int G = Hq / Hkv;
  if ((G != 1 && G != 2 && G != 4) || (D != 64 && D != 128)) return KV4_ERR_UNSUPPORTED;
  if (T > kMaxSmdT || B > 65535 || Hkv > 65535) return KV4_ERR_UNSUPPORTED;
  if (mask && (long long)mask_stride * 32 < T) return KV4_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return KV4_ERR_INVALID;
  if (mask && !aligned(mask, 4)) return KV4_ERR_INVALID;
  SmdParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.k = static_cast<const __nv_bfloat16 *>(k);
  p.v = static_cast<const __nv_bfloat16 *>(v);
  p.lens = seq_lens;
  p.mask = mask;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.mask_stride = mask ? mask_stride : 0;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.out = out;
  p.out_fp32 = out_is_fp32 ? 1 : 0;
  p.err = error_word;
  return cuda_status(launch_smd(p, D, static_cast<cudaStream_t>(stream)));
}

kv4_status kv4_get_error(kv4_cache *cache, void *stream, uint32_t *bits) {
  if (!cache) return KV4_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t w = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&w, cache->err, sizeof(w), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(cache->err, 0, sizeof(uint32_t));
  if (bad(e)) return KV4_ERR_CUDA;
  if (bits) *bits = w;
  if (w & (1u << KV4_ERR_TIMEOUT)) return KV4_ERR_TIMEOUT;
  if (w & (1u << KV4_ERR_BOUNDS)) return KV4_ERR_BOUNDS;
  if (w & (1u << KV4_ERR_CAPACITY)) return KV4_ERR_CAPACITY;
  if (w & (1u << KV4_ERR_RANGE)) return KV4_ERR_RANGE;
  return KV4_OK;
}

kv4_status kv4_debug_set_wait_limit(kv4_cache *cache, int64_t cycles) {
  if (!cache) return KV4_ERR_INVALID;
  cache->wait_cap = cycles < 0 ? kDefaultWaitCycles : cycles;
  return KV4_OK;
}

kv4_status kv4_device_info(int32_t *num_sms, int32_t *default_workers_out) {
  // the decode kernel at D = 128, 32 query / 8 KV heads, 64 sequences
  Kv4Plan pl{};
  const kv4_status st = kv4_plan(128, 4, 8, 64, 0, &pl);
  if (st != KV4_OK) return st;
  int dev = 0;
  DeviceInfo di;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (bad(device_info(&dev, &di))) return KV4_ERR_CUDA;
  }
  if (num_sms) *num_sms = di.sms;
  if (default_workers_out) *default_workers_out = pl.n_cta * pl.HB;
  return KV4_OK;
}

kv4_status kv4_timing_enable(int32_t max_records, int32_t every) {
  if (max_records < 1 || every < 1) return KV4_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  timing_free();
  for (int k = 0; k < 2; ++k) {
    g_timing.ev[k].resize(2 * (size_t)max_records, nullptr);
    for (auto &e : g_timing.ev[k]) {
      if (bad(cudaEventCreate(&e))) {
        timing_free();
        return KV4_ERR_CUDA;
      }
    }
  }
  g_timing.max_records = max_records;
  g_timing.every = every;
  g_timing.on = true;
  return KV4_OK;
}

kv4_status kv4_timing_read(int32_t kind, double *total_ms, int32_t *count) {
  if (kind < 0 || kind > 1 || !total_ms || !count) return KV4_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  double sum = 0.0;
  const int n = g_timing.used[kind];
  for (int i = 0; i < n; ++i) {
    float ms = 0.f;
    if (bad(cudaEventSynchronize(g_timing.ev[kind][2 * i + 1]))) return KV4_ERR_CUDA;
    if (bad(cudaEventElapsedTime(&ms, g_timing.ev[kind][2 * i], g_timing.ev[kind][2 * i + 1])))
      return KV4_ERR_CUDA;
    sum += ms;
  }
  g_timing.used[kind] = 0;
  *total_ms = sum;
  *count = n;
  return KV4_OK;
}

kv4_status kv4_timing_read_each(int32_t kind, float *ms_out, int32_t cap, int32_t *count) {
  if (kind < 0 || kind > 1 || !count || cap < 0 || (cap > 0 && !ms_out)) return KV4_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  const int n = g_timing.used[kind];
  for (int i = 0; i < n; ++i) {
    float ms = 0.f;
    if (bad(cudaEventSynchronize(g_timing.ev[kind][2 * i + 1]))) return KV4_ERR_CUDA;
    if (bad(cudaEventElapsedTime(&ms, g_timing.ev[kind][2 * i], g_timing.ev[kind][2 * i + 1])))
      return KV4_ERR_CUDA;
    if (i < cap) ms_out[i] = ms;
  }
  g_timing.used[kind] = 0;
  *count = n;
  return KV4_OK;
}

kv4_status kv4_timing_disable(void) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  timing_free();
  return KV4_OK;
}

}  // extern "C"
