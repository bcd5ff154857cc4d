"""The C ABI without a GPU: the library loads, exports every function declared
in include/kv4.h, and rejects bad arguments on the host before any CUDA call."""
import ctypes as C

import pytest

import compressed_kv_cache_kv4_b200 as K


def test_exports_every_declared_symbol():
    L = K.lib()
    names = K.header_symbols()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    L = K.lib()
    for code, name in K.STATUS.items():
        assert L.kv4_status_string(code).decode() == name


def test_cache_bytes():
    cfg = K.make_config(8, 128, 64, 1000)
    pool, side = K.kv4_cache_bytes(cfg)
    assert pool == 1000 * 8 * 18 * 128               # 18*D bytes per (page, head)
    assert side == 64 * 8 * 37440                    # (16 + 128) rows of 2*(128 + 2) bytes
    cfg = K.make_config(2, 64, 2, 30, 0, 0)
    assert K.kv4_cache_bytes(cfg) == (30 * 2 * 1152, 0)


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, K.KV4_ERR_UNSUPPORTED), ("page_tokens", 32, K.KV4_ERR_UNSUPPORTED),
    ("group", 64, K.KV4_ERR_UNSUPPORTED), ("sink", 17, K.KV4_ERR_UNSUPPORTED),
    ("recent", 129, K.KV4_ERR_UNSUPPORTED), ("num_kv_heads", 0, K.KV4_ERR_INVALID),
    ("num_pages", 0, K.KV4_ERR_INVALID)])
def test_cache_bytes_rejects(field, value, status):
    cfg = K.make_config(8, 128, 64, 1000)
    setattr(cfg, field, value)
    a, b = C.c_size_t(0), C.c_size_t(0)
    assert K.lib().kv4_cache_bytes(C.byref(cfg), C.byref(a), C.byref(b)) == status


def test_host_validation_without_launch():
    L = K.lib()
    assert L.kv4_append(None, None, None, None, None, None, None, 1, 1, 1) == K.KV4_ERR_INVALID
    assert L.kv4_decode_attn(None, None, None, 32, None, None, 1, None, 0, C.c_float(0.1), 0, None, 0,
                             None, 0, 1) == K.KV4_ERR_INVALID
    # budget outside 0..1000, stride too small, null pointers
    fake = C.c_void_p(0x1000)
    assert L.kv_topk_retain(None, fake, 100, fake, 1, 1, 1001, 16, 128, fake, 4, None, 100) == K.KV4_ERR_INVALID
    assert L.kv_topk_retain(None, fake, 50, fake, 1, 1, 500, 16, 128, fake, 4, None, 100) == K.KV4_ERR_INVALID
    assert L.kv_topk_retain(None, None, 100, fake, 1, 1, 500, 16, 128, fake, 4, None, 100) == K.KV4_ERR_INVALID
    # B = 0 is a no-op
    assert L.kv_topk_retain(None, None, 0, None, 0, 1, 500, 16, 128, None, 0, None, 0) == K.KV4_OK
    n = C.c_size_t(0)
    assert L.bf16_paged_workspace_bytes(4, 12, 4, 128, 0, C.byref(n)) == K.KV4_ERR_UNSUPPORTED   # G = 3
    assert L.bf16_paged_workspace_bytes(4, 8, 4, 96, 0, C.byref(n)) == K.KV4_ERR_UNSUPPORTED     # D = 96
    assert L.kv4_evict_pages(None, None, fake, 100, 500, fake, fake, 8, fake, fake, 1) == K.KV4_ERR_INVALID
    # smd_masked_attn: argument checks before any launch
    f = C.c_float(0.1)
    a16 = C.c_void_p(0x10000)
    args = lambda q=a16, Hq=8, Hkv=2, D=128, mask=None, ms=0, out=a16, T=100: (
        None, q, a16, a16, 1, T, Hq, Hkv, D, None, mask, ms, f, out, 0, None)
    assert L.smd_masked_attn(*args(q=None)) == K.KV4_ERR_INVALID            # null q
    assert L.smd_masked_attn(*args(Hq=6, Hkv=4)) == K.KV4_ERR_INVALID       # Hq % Hkv != 0
    assert L.smd_masked_attn(*args(Hq=24, Hkv=3)) == K.KV4_ERR_UNSUPPORTED  # G = 8
    assert L.smd_masked_attn(*args(D=96)) == K.KV4_ERR_UNSUPPORTED          # head_dim
    assert L.smd_masked_attn(*args(T=70000)) == K.KV4_ERR_UNSUPPORTED       # longer than 65536
    assert L.smd_masked_attn(*args(mask=fake, ms=3)) == K.KV4_ERR_INVALID   # 3 words < ceil(100/32)
    assert L.smd_masked_attn(*args(out=C.c_void_p(0x10008))) == K.KV4_ERR_INVALID   # misaligned out
    assert L.smd_masked_attn(*args(T=0)) == K.KV4_OK                        # nothing to do
    assert L.kv4_get_error(None, None, None) == K.KV4_ERR_INVALID
    assert L.kv4_debug_set_wait_limit(None, 0) == K.KV4_ERR_INVALID


def test_compute_entry_points_need_the_library(monkeypatch):
    """No fallback: without libkv4.so the binding raises instead of computing."""
    monkeypatch.setattr(K, "_lib", None)
    monkeypatch.setattr(K, "LIB_PATH", "/nonexistent/libkv4.so")
    with pytest.raises(ImportError):
        K.lib()
