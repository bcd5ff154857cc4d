"""Python binding of libkv4 (include/kv4.h): decode attention over a KV4-RL
compressed KV cache on B200.

Argument marshalling only: every computation runs in libkv4's CUDA kernels.
torch supplies device memory and the current CUDA stream. If libkv4.so has not
been built, importing the compute entry points raises ImportError; there is no
fallback implementation.

Names mirror the C ABI (kv4_cache_bytes, kv4_cache_create, kv4_append,
kv4_workspace_bytes, kv4_decode_attn, kv4_decode_partials, kv4_merge_partials,
kv4_masked_workspace_bytes, kv4_decode_attn_masked,
kv_topk_retain, kv4_evict_pages, smd_masked_attn, bf16_paged_decode_attn,
kv4_get_error); ``KV4Cache`` bundles the buffers and handle of one cache;
``cp`` holds the context-parallel plumbing (shard plan, gather of partials).
"""
import ctypes as C
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkv4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "kv4.h")

STATUS = {0: "KV4_OK", 1: "KV4_ERR_INVALID", 2: "KV4_ERR_UNSUPPORTED", 3: "KV4_ERR_CAPACITY",
          4: "KV4_ERR_BOUNDS", 5: "KV4_ERR_RANGE", 6: "KV4_ERR_TIMEOUT", 7: "KV4_ERR_CUDA"}
KV4_OK, KV4_ERR_INVALID, KV4_ERR_UNSUPPORTED, KV4_ERR_CAPACITY = 0, 1, 2, 3
KV4_ERR_BOUNDS, KV4_ERR_RANGE, KV4_ERR_TIMEOUT, KV4_ERR_CUDA = 4, 5, 6, 7


class Kv4Error(RuntimeError):
    def __init__(self, status, what=""):
        super().__init__("%s: %s" % (what, STATUS.get(status, status)))
        self.status = status


class kv4_config(C.Structure):
    _fields_ = [("num_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("page_tokens", C.c_int32),
                ("group", C.c_int32), ("sink", C.c_int32), ("recent", C.c_int32),
                ("max_seqs", C.c_int32), ("num_pages", C.c_int32)]


_lib = None
_P, _I32, _I64, _SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t


def lib():
    """Load libkv4.so (built in-tree by compressed_kv_cache_kv4_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libkv4.so is not built; run `python -m compressed_kv_cache_kv4_b200.build`")
    L = C.CDLL(LIB_PATH)
    sig = {
        "kv4_status_string": (C.c_char_p, [C.c_int]),
        "kv4_last_cuda_error": (C.c_char_p, []),
        "kv4_cache_bytes": (C.c_int, [C.POINTER(kv4_config), C.POINTER(_SZ), C.POINTER(_SZ)]),
        "kv4_cache_create": (C.c_int, [C.POINTER(kv4_config), _P, _SZ, _P, _SZ, C.POINTER(_P)]),
        "kv4_cache_destroy": (None, [_P]),
        "kv4_append": (C.c_int, [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I64]),
        "kv4_workspace_bytes": (C.c_int, [_P, _I32, _I32, _I32, C.POINTER(_SZ)]),
        "kv4_decode_attn": (C.c_int, [_P, _P, _P, _I32, _P, _P, _I32, _P, _I32, C.c_float, _I32, _P, _SZ,
                                      _P, _I32, _I32]),
        "kv4_decode_attn_noalloc": (C.c_int, [_P, _P, _P, _I32, _P, _P, _I32, _P, _I32, C.c_float, _I32,
                                              _P, _I32, _I32]),
        "kv4_decode_partials": (C.c_int, [_P, _P, _P, _I32, _P, _P, _I32, _P, _P, _I32, _P, _I32, C.c_float,
                                          _I32, _P, _SZ, _P, _I32]),
        "kv4_merge_partials": (C.c_int, [_P, _P, _I32, _I32, _I32, _I32, _P, _I32]),
        "kv4_masked_workspace_bytes": (C.c_int, [_P, _I32, _I32, _I32, _I32, C.POINTER(_SZ)]),
        "kv4_decode_attn_masked": (C.c_int, [_P, _P, _P, _I32, _P, _P, _I32, _P, _I32, _I32, C.c_float, _P, _SZ,
                                             _P, _I32, _I32]),
        "kv_topk_retain": (C.c_int, [_P, _P, _I64, _P, _I32, _I32, _I32, _I32, _I32, _P, _I32, _P, _I32]),
        "kv4_evict_pages": (C.c_int, [_P, _P, _P, _I64, _I32, _P, _P, _I32, _P, _P, _I32]),
        "smd_masked_attn": (C.c_int, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P, _P, _I32, C.c_float,
                                      _P, _I32, _P]),
        "bf16_paged_workspace_bytes": (C.c_int, [_I32, _I32, _I32, _I32, _I32, C.POINTER(_SZ)]),
        "bf16_paged_decode_attn": (C.c_int, [_P, _P, _I32, _I32, _I32, _P, _I32, _P, _I32, _P, C.c_float,
                                             _I32, _P, _SZ, _P, _I32, _I32, _P]),
        "kv4_get_error": (C.c_int, [_P, _P, C.POINTER(C.c_uint32)]),
        "kv4_debug_set_wait_limit": (C.c_int, [_P, _I64]),
        "kv4_device_info": (C.c_int, [C.POINTER(_I32), C.POINTER(_I32)]),
        "kv4_timing_enable": (C.c_int, [_I32, _I32]),
        "kv4_timing_read": (C.c_int, [_I32, C.POINTER(C.c_double), C.POINTER(_I32)]),
        "kv4_timing_read_each": (C.c_int, [_I32, _P, _I32, C.POINTER(_I32)]),
        "kv4_timing_disable": (C.c_int, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def header_symbols():
    """Function names declared in include/kv4.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)))


def _check(st, what):
    if st != KV4_OK:
        if st == KV4_ERR_CUDA:
            what = "%s (%s)" % (what, lib().kv4_last_cuda_error().decode())
        raise Kv4Error(st, what)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def make_config(num_kv_heads, head_dim, max_seqs, num_pages, sink=16, recent=128):
    return kv4_config(num_kv_heads, head_dim, 16, 32, sink, recent, max_seqs, num_pages)


def kv4_cache_bytes(cfg):
    a, b = _SZ(0), _SZ(0)
    _check(lib().kv4_cache_bytes(C.byref(cfg), C.byref(a), C.byref(b)), "kv4_cache_bytes")
    return a.value, b.value


def kv4_cache_create(cfg, pool, side):
    h = _P()
    _check(lib().kv4_cache_create(C.byref(cfg), _ptr(pool), pool.numel() * pool.element_size(),
                                  _ptr(side), 0 if side is None else side.numel() * side.element_size(),
                                  C.byref(h)), "kv4_cache_create")
    return h


def kv4_cache_destroy(handle):
    lib().kv4_cache_destroy(handle)


def kv4_append(handle, k_new, v_new, new_offsets, seq_lens_old, page_table, stream=None):
    st = lib().kv4_append(handle, _stream(stream), _ptr(k_new), _ptr(v_new), _ptr(new_offsets),
                          _ptr(seq_lens_old), _ptr(page_table), page_table.shape[1],
                          seq_lens_old.numel(), k_new.shape[0])
    _check(st, "kv4_append")


def kv4_workspace_bytes(handle, B, Hq, num_workers=0):
    n = _SZ(0)
    _check(lib().kv4_workspace_bytes(handle, B, Hq, num_workers, C.byref(n)), "kv4_workspace_bytes")
    return n.value


def kv4_decode_attn(handle, q, seq_lens, page_table, softmax_scale, workspace, out, retain_mask=None,
                    num_workers=0, stream=None):
    B, Hq, _ = q.shape
    mstride = 0 if retain_mask is None else retain_mask.shape[-1]
    st = lib().kv4_decode_attn(handle, _stream(stream), _ptr(q), Hq, _ptr(seq_lens), _ptr(page_table),
                               page_table.shape[1], _ptr(retain_mask), mstride, C.c_float(softmax_scale),
                               num_workers, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _ptr(out), 1 if out.dtype == torch.float32 else 0, B)
    _check(st, "kv4_decode_attn")


def kv4_decode_partials(handle, q, seq_lens, page_table, softmax_scale, workspace, partials, page_begin=None,
                        page_end=None, with_int8=True, retain_mask=None, num_workers=0, stream=None):
    """Exact softmax partials (m, l, o) of one page-range shard of every
    sequence: partials is fp32 [B][Hq][D+4] (m, l, two unused words, o)."""
    B, Hq, _ = q.shape
    mstride = 0 if retain_mask is None else retain_mask.shape[-1]
    st = lib().kv4_decode_partials(handle, _stream(stream), _ptr(q), Hq, _ptr(seq_lens), _ptr(page_table),
                                   page_table.shape[1], _ptr(page_begin), _ptr(page_end), 1 if with_int8 else 0,
                                   _ptr(retain_mask), mstride, C.c_float(softmax_scale), num_workers, _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _ptr(partials), B)
    _check(st, "kv4_decode_partials")


def kv4_merge_partials(partials, out, stream=None):
    """Exact merge of partials [N][B][Hq][D+4] into out [B][Hq][D] (bf16 or fp32)."""
    N, B, Hq, D4 = partials.shape
    st = lib().kv4_merge_partials(_stream(stream), _ptr(partials), N, B, Hq, D4 - 4, _ptr(out),
                                  1 if out.dtype == torch.float32 else 0)
    _check(st, "kv4_merge_partials")


def kv4_masked_workspace_bytes(handle, B, Hq, pt_stride, max_retained):
    n = _SZ()
    _check(lib().kv4_masked_workspace_bytes(handle, B, Hq, pt_stride, max_retained, C.byref(n)),
           "kv4_masked_workspace_bytes")
    return n.value


def kv4_decode_attn_masked(handle, q, seq_lens, page_table, softmax_scale, retain_mask, max_retained, workspace, out,
                           stream=None):
    """Masked decode with the INT4 region's retained rows gathered into compact
    pages first (reads and work follow the retained count); out [B][Hq][D]
    bf16 or fp32."""
    B, Hq, _ = q.shape
    st = lib().kv4_decode_attn_masked(handle, _stream(stream), _ptr(q), Hq, _ptr(seq_lens), _ptr(page_table),
                                      page_table.shape[1], _ptr(retain_mask), retain_mask.shape[-1], max_retained,
                                      C.c_float(softmax_scale), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _ptr(out),
                                      1 if out.dtype == torch.float32 else 0, B)
    _check(st, "kv4_decode_attn_masked")


# Size of the fixed per-device scratch of kv4_decode_attn_noalloc (KV4_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 16 << 20


def kv4_decode_attn_noalloc(handle, q, seq_lens, page_table, softmax_scale, out, retain_mask=None,
                            num_workers=0, stream=None):
    """kv4_decode_attn with the library's fixed scratch instead of a caller
    workspace (for callers that cannot allocate device memory). Calls whose
    kernels may overlap in time on one device must not be issued: they share
    the scratch."""
    B, Hq, _ = q.shape
    mstride = 0 if retain_mask is None else retain_mask.shape[-1]
    st = lib().kv4_decode_attn_noalloc(handle, _stream(stream), _ptr(q), Hq, _ptr(seq_lens), _ptr(page_table),
                                       page_table.shape[1], _ptr(retain_mask), mstride, C.c_float(softmax_scale),
                                       num_workers, _ptr(out), 1 if out.dtype == torch.float32 else 0, B)
    if st == KV4_ERR_CAPACITY:
        need = kv4_workspace_bytes(handle, B, Hq, num_workers)
        if need > NOALLOC_SCRATCH_BYTES:
            raise Kv4Error(st, "kv4_decode_attn_noalloc: needs %d bytes of scratch, the fixed area holds %d"
                           % (need, NOALLOC_SCRATCH_BYTES))
    _check(st, "kv4_decode_attn_noalloc")


def kv_topk_retain(scores, seq_lens, budget_permille, mask_out, count_out=None, sink=16, recent=128,
                   max_len=None, stream=None):
    B, Hkv, stride = scores.shape
    max_len = stride if max_len is None else max_len
    st = lib().kv_topk_retain(_stream(stream), _ptr(scores), stride, _ptr(seq_lens), B, Hkv, budget_permille,
                              sink, recent, _ptr(mask_out), mask_out.shape[-1], _ptr(count_out), max_len)
    _check(st, "kv_topk_retain")


def kv4_evict_pages(handle, scores, budget_permille, seq_lens, page_table, freed_pages, freed_count,
                    stream=None):
    """Page-granular eviction and compaction: rewrites seq_lens, page_table and
    the side cache's ring pages in place; freed_pages[b, :freed_count[b]] get the
    evicted physical page ids."""
    B, _, stride = scores.shape
    st = lib().kv4_evict_pages(handle, _stream(stream), _ptr(scores), stride, budget_permille, _ptr(seq_lens),
                               _ptr(page_table), page_table.shape[1], _ptr(freed_pages), _ptr(freed_count), B)
    _check(st, "kv4_evict_pages")


def smd_masked_attn(q, k, v, softmax_scale, out, seq_lens=None, mask=None, error_word=None, stream=None):
    """Learner-side causal attention under the shadow mask. q [B][T][Hq][D],
    k/v [B][T][Hkv][D] bf16; mask None or int32/uint32 [B][Hkv][T][mask_stride];
    out [B][T][Hq][D] bf16 or fp32."""
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    st = lib().smd_masked_attn(_stream(stream), _ptr(q), _ptr(k), _ptr(v), B, T, Hq, Hkv, D, _ptr(seq_lens),
                               _ptr(mask), 0 if mask is None else mask.shape[-1], C.c_float(softmax_scale),
                               _ptr(out), 1 if out.dtype == torch.float32 else 0, _ptr(error_word))
    _check(st, "smd_masked_attn")


def bf16_paged_workspace_bytes(B, Hq, Hkv, D, num_workers=0):
    n = _SZ(0)
    _check(lib().bf16_paged_workspace_bytes(B, Hq, Hkv, D, num_workers, C.byref(n)), "bf16_paged_workspace_bytes")
    return n.value


def bf16_paged_decode_attn(q, kv_pages, page_table, seq_lens, softmax_scale, workspace, out, Hkv,
                           num_workers=0, error_word=None, stream=None):
    B, Hq, D = q.shape
    st = lib().bf16_paged_decode_attn(_stream(stream), _ptr(q), Hq, Hkv, D, _ptr(kv_pages), kv_pages.shape[0],
                                      _ptr(page_table), page_table.shape[1], _ptr(seq_lens),
                                      C.c_float(softmax_scale), num_workers, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _ptr(out),
                                      1 if out.dtype == torch.float32 else 0, B, _ptr(error_word))
    _check(st, "bf16_paged_decode_attn")


def kv4_get_error(handle, stream=None):
    bits = C.c_uint32(0)
    st = lib().kv4_get_error(handle, _stream(stream), C.byref(bits))
    return st, bits.value


def kv4_debug_set_wait_limit(handle, cycles):
    _check(lib().kv4_debug_set_wait_limit(handle, int(cycles)), "kv4_debug_set_wait_limit")


def kv4_device_info():
    a, b = _I32(0), _I32(0)
    _check(lib().kv4_device_info(C.byref(a), C.byref(b)), "kv4_device_info")
    return a.value, b.value


def kv4_timing_enable(max_records, every=1):
    _check(lib().kv4_timing_enable(int(max_records), int(every)), "kv4_timing_enable")


def kv4_timing_read(kind):
    """(total_ms, count) of recorded worker-kernel launches; kind 0 = kv4, 1 = bf16."""
    ms, n = C.c_double(0), _I32(0)
    _check(lib().kv4_timing_read(int(kind), C.byref(ms), C.byref(n)), "kv4_timing_read")
    return ms.value, n.value


def kv4_timing_read_each(kind, cap=4096):
    """Per-launch durations (ms, oldest first) of the recorded worker-kernel launches."""
    buf = (C.c_float * max(int(cap), 1))()
    n = _I32(0)
    _check(lib().kv4_timing_read_each(int(kind), buf, int(cap), C.byref(n)), "kv4_timing_read_each")
    return [float(buf[i]) for i in range(min(n.value, int(cap)))]


def kv4_timing_disable():
    _check(lib().kv4_timing_disable(), "kv4_timing_disable")


class KV4Cache:
    """One compressed cache: caller-side torch buffers plus the library handle."""

    def __init__(self, num_kv_heads, head_dim, max_seqs, num_pages, sink=16, recent=128, device="cuda",
                 fill=None):
        self.cfg = make_config(num_kv_heads, head_dim, max_seqs, num_pages, sink, recent)
        pool_bytes, side_bytes = kv4_cache_bytes(self.cfg)

        def buf(n):
            if fill is None:
                return torch.empty(n, dtype=torch.uint8, device=device)
            return torch.full((n,), fill, dtype=torch.uint8, device=device)

        self.pool = buf(pool_bytes)
        self.side = buf(side_bytes) if side_bytes else None
        self.handle = kv4_cache_create(self.cfg, self.pool, self.side)
        self._ws = {}

    def close(self):
        if self.handle:
            kv4_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, B, Hq, num_workers=0):
        key = (B, Hq, num_workers)
        if key not in self._ws:
            n = kv4_workspace_bytes(self.handle, B, Hq, num_workers)
            self._ws[key] = torch.zeros(n, dtype=torch.uint8, device=self.pool.device)
        return self._ws[key]

    def append(self, k_new, v_new, new_offsets, seq_lens_old, page_table, stream=None):
        kv4_append(self.handle, k_new, v_new, new_offsets, seq_lens_old, page_table, stream)

    def decode(self, q, seq_lens, page_table, softmax_scale, out=None, out_fp32=False, retain_mask=None,
               num_workers=0, stream=None):
        B, Hq, D = q.shape
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
        ws = self.workspace(B, Hq, num_workers)
        kv4_decode_attn(self.handle, q, seq_lens, page_table, softmax_scale, ws, out, retain_mask,
                        num_workers, stream)
        return out

    def decode_masked(self, q, seq_lens, page_table, softmax_scale, retain_mask, max_retained, out=None,
                      out_fp32=False, stream=None):
        """kv4_decode_attn_masked: the retained INT4 rows gathered into compact
        pages first; max_retained bounds the retained INT4-region positions of
        any (sequence, head)."""
        B, Hq, D = q.shape
        if out is None:
            out = torch.empty((B, Hq, D), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
        key = ("masked", B, Hq, page_table.shape[1], max_retained)
        if key not in self._ws:
            n = kv4_masked_workspace_bytes(self.handle, B, Hq, page_table.shape[1], max_retained)
            self._ws[key] = torch.zeros(n, dtype=torch.uint8, device=self.pool.device)
        kv4_decode_attn_masked(self.handle, q, seq_lens, page_table, softmax_scale, retain_mask, max_retained,
                               self._ws[key], out, stream)
        return out

    def evict_pages(self, scores, budget_permille, seq_lens, page_table, stream=None):
        """Evict whole pages in place; returns (freed_pages [B][pt_stride], freed_count [B])."""
        B = seq_lens.shape[0]
        freed = torch.full((B, page_table.shape[1]), -1, dtype=torch.int32, device=page_table.device)
        count = torch.zeros(B, dtype=torch.int32, device=page_table.device)
        kv4_evict_pages(self.handle, scores, budget_permille, seq_lens, page_table, freed, count, stream)
        return freed, count

    def get_error(self, stream=None):
        return kv4_get_error(self.handle, stream)
