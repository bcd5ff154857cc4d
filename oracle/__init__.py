"""Python view of the fp64 CPU oracle (oracle/kv4_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of bench.py. The product path
never imports it. It shares no code with the CUDA library; inputs reach both
sides from the seeded generators in ``compressed_kv_cache_kv4_b200.synth``.

bf16 and fp16 values cross this boundary as their raw 16-bit patterns
(numpy uint16), so nothing is rounded on the way in.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class Shape(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("D", C.c_int32),
                ("sink", C.c_int32), ("recent", C.c_int32)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.kv4o_fp16_round_up.restype = C.c_uint16
        L.kv4o_fp16_round_up.argtypes = [C.c_double]
        L.kv4o_fp16_to_double.restype = C.c_double
        L.kv4o_fp16_to_double.argtypes = [C.c_uint16]
        L.kv4o_bf16_to_double.restype = C.c_double
        L.kv4o_bf16_to_double.argtypes = [C.c_uint16]
        L.kv4o_round_half_even.restype = C.c_double
        L.kv4o_round_half_even.argtypes = [C.c_double]
        for f in (L.kv4o_quant_int4, L.kv4o_quant_int8):
            f.restype = C.c_int
            f.argtypes = [P, C.c_int, P, P]
        L.kv4o_page_head_bytes.restype = C.c_int64
        L.kv4o_page_head_bytes.argtypes = [C.c_int]
        for f in (L.kv4o_k_code_byte, L.kv4o_v_code_byte):
            f.restype = C.c_int64
            f.argtypes = [C.c_int, C.c_int, C.c_int, C.POINTER(C.c_int)]
        for f in (L.kv4o_k_scale_byte, L.kv4o_v_scale_byte):
            f.restype = C.c_int64
            f.argtypes = [C.c_int, C.c_int, C.c_int]
        L.kv4o_side_head_bytes.restype = C.c_int64
        L.kv4o_side_head_bytes.argtypes = [C.c_int, C.c_int, C.c_int]
        L.kv4o_side_pages.restype = C.c_int
        L.kv4o_side_pages.argtypes = [C.c_int, C.c_int]
        L.kv4o_side_page_bytes.restype = C.c_int64
        L.kv4o_side_page_bytes.argtypes = [C.c_int]
        for f in (L.kv4o_side_k_byte, L.kv4o_side_v_byte):
            f.restype = C.c_int64
            f.argtypes = [C.c_int, C.c_int, C.c_int]
        for f in (L.kv4o_side_ks_byte, L.kv4o_side_vs_byte):
            f.restype = C.c_int64
            f.argtypes = [C.c_int, C.c_int]
        L.kv4o_write_cache.restype = C.c_int
        L.kv4o_write_cache.argtypes = [C.POINTER(Shape), P, P, C.c_int, P, P, C.c_int,
                                       P, C.c_int64, P, C.c_int64]
        L.kv4o_dequant_rows.restype = None
        L.kv4o_dequant_rows.argtypes = [C.POINTER(Shape), P, P, C.c_int, P, C.c_int, C.c_int, P, P]
        L.kv4o_decode.restype = None
        L.kv4o_decode.argtypes = [C.POINTER(Shape), P, P, P, C.c_int, P, P, C.c_int,
                                  C.c_float, C.c_int, P]
        L.kv4o_attend_rows.restype = None
        L.kv4o_attend_rows.argtypes = [C.c_int, P, P, P, C.c_int, C.c_double, P, P, P]
        L.kv4o_merge.restype = None
        L.kv4o_merge.argtypes = [C.c_int, C.c_int, P, P, P, P]
        L.kv4o_topk.restype = None
        L.kv4o_topk.argtypes = [P, C.c_int64, P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                P, C.c_int, P]
        L.kv4o_evict_pages.restype = None
        L.kv4o_evict_pages.argtypes = [P, C.c_int64, P, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                       C.c_int, P, C.c_int, P, P, P]
        L.kv4o_masked_attn.restype = None
        L.kv4o_masked_attn.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, P, P, P, P, P, C.c_int,
                                       C.c_float, P]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def fp16_round_up(y: float) -> int:
    return int(lib().kv4o_fp16_round_up(float(y)))


def fp16_to_float(bits: int) -> float:
    return float(lib().kv4o_fp16_to_double(int(bits)))


def bf16_to_float(bits: int) -> float:
    return float(lib().kv4o_bf16_to_double(int(bits)))


def round_half_even(x: float) -> float:
    return float(lib().kv4o_round_half_even(float(x)))


# ---------------------------------------------------------------- quantiser
def quant_int4(x_bits):
    """x_bits: uint16 bf16 patterns, length n (a group). -> (scale_bits, codes int8, overflow)."""
    x = _c(x_bits, np.uint16)
    sc = np.zeros(1, np.uint16)
    codes = np.zeros(x.size, np.int8)
    ov = lib().kv4o_quant_int4(_p(x), x.size, _p(sc), _p(codes))
    return int(sc[0]), codes, int(ov)


def quant_int8(x_bits):
    x = _c(x_bits, np.uint16)
    sc = np.zeros(1, np.uint16)
    codes = np.zeros(x.size, np.int8)
    ov = lib().kv4o_quant_int8(_p(x), x.size, _p(sc), _p(codes))
    return int(sc[0]), codes, int(ov)


# ---------------------------------------------------------------- layout
def page_head_bytes(D):
    return int(lib().kv4o_page_head_bytes(D))


def k_code_byte(D, r, d):
    nib = C.c_int(0)
    off = lib().kv4o_k_code_byte(D, r, d, C.byref(nib))
    return int(off), int(nib.value)


def v_code_byte(D, r, d):
    nib = C.c_int(0)
    off = lib().kv4o_v_code_byte(D, r, d, C.byref(nib))
    return int(off), int(nib.value)


def k_scale_byte(D, r, grp):
    return int(lib().kv4o_k_scale_byte(D, r, grp))


def v_scale_byte(D, r, grp):
    return int(lib().kv4o_v_scale_byte(D, r, grp))


def side_head_bytes(D, sink, recent):
    return int(lib().kv4o_side_head_bytes(D, sink, recent))


def side_pages(sink, recent):
    return int(lib().kv4o_side_pages(sink, recent))


def side_page_bytes(D):
    return int(lib().kv4o_side_page_bytes(D))


def side_k_byte(D, row, d):
    return int(lib().kv4o_side_k_byte(D, row, d))


def side_v_byte(D, row, d):
    return int(lib().kv4o_side_v_byte(D, row, d))


def side_ks_byte(D, row):
    return int(lib().kv4o_side_ks_byte(D, row))


def side_vs_byte(D, row):
    return int(lib().kv4o_side_vs_byte(D, row))


def shape(B, Hq, Hkv, D, sink=16, recent=128):
    return Shape(B, Hq, Hkv, D, sink, recent)


def write_cache(sh, k_bits, v_bits, lens, page_table, num_pages, fill=0xA5):
    """Byte image of the page pool and side cache after appending every
    position. k_bits/v_bits: uint16 [B][Lmax][Hkv][D]. Returns (pool, side, flags)."""
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    lens = _c(lens, np.int32)
    pt = _c(page_table, np.int32)
    Lmax = k.shape[1]
    pool = np.full(num_pages * page_head_bytes(sh.D) * sh.Hkv, fill, np.uint8)
    side = np.full(sh.B * sh.Hkv * side_head_bytes(sh.D, sh.sink, sh.recent), fill, np.uint8)
    flags = lib().kv4o_write_cache(C.byref(sh), _p(k), _p(v), Lmax, _p(lens), _p(pt), pt.shape[1],
                                   _p(pool), pool.size, _p(side), side.size)
    return pool, side, int(flags)


def dequant_rows(sh, k_bits, v_bits, lens, b, h):
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    lens = _c(lens, np.int32)
    L = int(lens[b])
    kh = np.zeros((max(L, 1), sh.D), np.float64)
    vh = np.zeros((max(L, 1), sh.D), np.float64)
    lib().kv4o_dequant_rows(C.byref(sh), _p(k), _p(v), k.shape[1], _p(lens), b, h, _p(kh), _p(vh))
    return kh[:L], vh[:L]


# ---------------------------------------------------------------- attention
def decode(sh, q_bits, k_bits, v_bits, lens, softmax_scale, mask=None, mode=0):
    """mode 0: KV4 values (INT4 + INT8 protection); mode 1: plain bf16 values."""
    q = _c(q_bits, np.uint16)
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    lens = _c(lens, np.int32)
    out = np.zeros((sh.B, sh.Hq, sh.D), np.float64)
    m = None if mask is None else _c(mask, np.uint32)
    ms = 0 if m is None else m.shape[-1]
    lib().kv4o_decode(C.byref(sh), _p(q), _p(k), _p(v), k.shape[1], _p(lens), _p(m), ms,
                      C.c_float(softmax_scale), mode, _p(out))
    return out


def attend_rows(q, krows, vrows, scale):
    q = _c(q, np.float64)
    kr = _c(krows, np.float64).reshape(-1, q.size)
    vr = _c(vrows, np.float64).reshape(-1, q.size)
    m = np.zeros(1)
    l = np.zeros(1)
    o = np.zeros(q.size)
    lib().kv4o_attend_rows(q.size, _p(q), _p(kr), _p(vr), kr.shape[0], float(scale), _p(m), _p(l), _p(o))
    return float(m[0]), float(l[0]), o


def merge(ms, ls, os_):
    ms = _c(ms, np.float64)
    ls = _c(ls, np.float64)
    o = _c(os_, np.float64)
    D = o.shape[-1]
    out = np.zeros(D)
    lib().kv4o_merge(D, ms.size, _p(ms), _p(ls), _p(o.reshape(-1, D)), _p(out))
    return out


# ---------------------------------------------------------------- top-k
def topk(scores, lens, permille, sink=16, recent=128):
    """scores: float32 [B][Hkv][stride]. -> (mask uint32 [B][Hkv][ceil(stride/32)], count int32 [B][Hkv])."""
    s = _c(scores, np.float32)
    B, Hkv, stride = s.shape
    lens = _c(lens, np.int32)
    mstride = (stride + 31) // 32
    mask = np.zeros((B, Hkv, mstride), np.uint32)
    count = np.zeros((B, Hkv), np.int32)
    lib().kv4o_topk(_p(s), stride, _p(lens), B, Hkv, permille, sink, recent, _p(mask), mstride, _p(count))
    return mask, count


# ---------------------------------------------------------------- page eviction
def evict_pages(scores, lens, page_table, side, D, permille, sink=16, recent=128):
    """Page-granular eviction and compaction on copies of the inputs.
    scores: float32 [B][Hkv][stride]; lens int32 [B]; page_table int32 [B][pt_stride];
    side: uint8 side-cache image (or None to skip the ring rotation check).
    -> (lens, page_table, freed [B][pt_stride] (-1 past the count), freed_count, side)."""
    s = _c(scores, np.float32)
    B, Hkv, stride = s.shape
    lens = np.array(lens, np.int32, copy=True)
    pt = np.array(page_table, np.int32, copy=True)
    freed = np.full(pt.shape, -1, np.int32)
    cnt = np.zeros(B, np.int32)
    if side is None:
        side = np.zeros(B * Hkv * side_head_bytes(D, sink, recent), np.uint8)
    side = np.array(side, np.uint8, copy=True)
    assert np.all(lens <= stride) and np.all(lens <= 16 * pt.shape[1])
    lib().kv4o_evict_pages(_p(s), stride, _p(lens), B, Hkv, D, permille, sink, recent, _p(pt),
                           pt.shape[1], _p(freed), _p(cnt), _p(side))
    return lens, pt, freed, cnt, side


# ---------------------------------------------------------------- learner-side masked attention
def masked_attn(q_bits, k_bits, v_bits, softmax_scale, lens=None, mask=None):
    """q_bits uint16 [B][T][Hq][D]; k_bits, v_bits uint16 [B][T][Hkv][D];
    mask None or uint32 [B][Hkv][T][mask_stride]. -> float64 [B][T][Hq][D]."""
    q = _c(q_bits, np.uint16)
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    ln = None if lens is None else _c(lens, np.int32)
    m = None if mask is None else _c(mask, np.uint32)
    ms = 0 if m is None else m.shape[-1]
    out = np.zeros((B, T, Hq, D), np.float64)
    lib().kv4o_masked_attn(B, T, Hq, Hkv, D, _p(q), _p(k), _p(v), _p(ln), _p(m), ms,
                           C.c_float(softmax_scale), _p(out))
    return out
