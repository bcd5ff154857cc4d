// kv4_noalloc.cu -- kv4_decode_attn_noalloc: the decode step of
// kv4_decode_attn with its scratch taken from a fixed array inside the
// library instead of a workspace the caller allocates.
//
// Who needs it: a caller that cannot hand the library device memory of its
// own, e.g. C code with no access to the application's device allocator, or a
// serving loop that must not call cudaMalloc / cudaFree between steps (both
// may synchronise the whole device). The method itself has no such call; this
// is plumbing around the same kernels.
//
// The array is an ordinary __device__ variable of the library's module: the
// CUDA runtime reserves it on each device when it loads the module there, and
// nothing here allocates or frees memory at run time. Its address on a device
// is looked up once (cudaGetSymbolAddress, which also makes the runtime load
// the module on that device) and cached.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "kv4.h"
#include "kv4_internal.h"

namespace {

static_assert(KV4_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

// One copy per device, zero-initialised when the module is loaded. The decode
// kernels write every word of their scratch before reading it, so nothing in
// it has to start at zero and nothing is cleared between calls.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KV4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_ptr[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of g_noalloc_scratch on the current device; the first call
// per device performs the lookup. The cached address assumes the device's
// primary context lives as long as the process: after a cudaDeviceReset the
// module is loaded again and the address may change, so a process that resets
// a device must not call this entry point on it afterwards.
kv4_status scratch_on_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return KV4_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return KV4_ERR_UNSUPPORTED;
  void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return KV4_ERR_CUDA;
      }
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return KV4_OK;
}

}  // namespace

extern "C" kv4_status kv4_decode_attn_noalloc(kv4_cache *cache, void *stream, const void *q, int32_t Hq,
                                              const int32_t *seq_lens, const int32_t *page_table,
                                              int32_t pt_stride, const uint32_t *retain_mask,
                                              int32_t mask_stride, float softmax_scale, int32_t num_workers,
                                              void *out, int32_t out_is_fp32, int32_t B) {
  if (!cache || B < 0 || num_workers < 0) return KV4_ERR_INVALID;
  if (B == 0) return KV4_OK;
  // The scratch handed to the kernels is the current device's copy of the
  // array, so the current device must be the one the cache lives on.
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return KV4_ERR_CUDA;
  }
  if (dev != kv4::cache_device(cache)) return KV4_ERR_INVALID;
  // The scratch this call needs, from the same sizing rule as the workspace
  // of kv4_decode_attn; refuse before touching the device if it does not fit.
  size_t need = 0;
  const kv4_status st = kv4_workspace_bytes(cache, B, Hq, num_workers, &need);
  if (st != KV4_OK) return st;
  if (need > (size_t)KV4_NOALLOC_SCRATCH_BYTES) return KV4_ERR_CAPACITY;
  void *scratch = nullptr;
  const kv4_status su = scratch_on_current_device(&scratch);
  if (su != KV4_OK) return su;
  return kv4_decode_attn(cache, stream, q, Hq, seq_lens, page_table, pt_stride, retain_mask, mask_stride,
                         softmax_scale, num_workers, scratch, (size_t)KV4_NOALLOC_SCRATCH_BYTES, out, out_is_fp32,
                         B);
}
