"""kv4_decode_attn_masked: masked decode with the retained INT4 rows gathered
into compact pages, against the oracle's masked decode and against the
page-granular masked path of kv4_decode_attn (Shadow Mask Distillation, sec. 1
and Figure 1: the mask is applied inside attention)."""
import numpy as np
import pytest
import torch

import compressed_kv_cache_kv4_b200 as K

from helpers import Case, assert_bf16_output, assert_close
from test_gpu_parity import small_wl

pytestmark = pytest.mark.gpu


def _bits(mask_np):
    """Mask words [B][H][W] -> bits [B][H][32 W] (bit p % 32 of word p / 32)."""
    B, H, W = mask_np.shape
    return ((mask_np[..., None].astype(np.uint64) >> np.arange(32, dtype=np.uint64)) & 1).reshape(B, H, W * 32)


def _words(bits):
    B, H, N = bits.shape
    w = bits.reshape(B, H, N // 32, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64)
    return w.sum(axis=-1).astype(np.uint32)


def _counts(mask_np, lens, sink, recent):
    """Retained positions of the INT4 region per (sequence, head)."""
    bits = _bits(mask_np)
    out = np.zeros(mask_np.shape[:2], np.int64)
    for b in range(mask_np.shape[0]):
        L = int(lens[b])
        c0 = min(sink, L)
        c1 = max(c0, L - recent)
        out[b] = bits[b, :, c0:c1].sum(axis=1)
    return out


@pytest.mark.parametrize("geom", ["qwen", "small_heads", "pure_int4", "odd_window"])
@pytest.mark.parametrize("kind", ["full", "empty", "random10", "random50", "sparse_pages"])
def test_masked_gather_matches_oracle(geom, kind):
    lens = [3000, 150, 40, 1800, 1, 145, 161, 2049]
    kw = {"qwen": {}, "small_heads": dict(Hq=8, Hkv=2, D=64), "pure_int4": dict(sink=0, recent=0),
          "odd_window": dict(sink=5, recent=16)}[geom]
    wl = small_wl(lens, seed=61, **kw)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    mstride = (c.pt_np.shape[1] * 16 + 31) // 32
    rng = np.random.default_rng(["qwen", "small_heads", "pure_int4", "odd_window"].index(geom) * 10
                                + ["full", "empty", "random10", "random50", "sparse_pages"].index(kind))
    if kind == "full":
        m = np.full((wl.B, wl.Hkv, mstride), 0xFFFFFFFF, np.uint32)
    elif kind == "empty":
        m = np.zeros((wl.B, wl.Hkv, mstride), np.uint32)
    elif kind == "sparse_pages":
        m = np.zeros((wl.B, wl.Hkv, mstride), np.uint32)
        m[:, :, 5::7] = rng.integers(0, 2 ** 32, size=m[:, :, 5::7].shape, dtype=np.uint64).astype(np.uint32)
    else:
        p = 0.1 if kind == "random10" else 0.5
        m = _words(rng.random((wl.B, wl.Hkv, mstride * 32)) < p)
    cnt = _counts(m, wl.lens, wl.sink, wl.recent)
    bound = int(cnt.max())
    mt = torch.as_tensor(m.view(np.int32), device="cuda")
    q = c.q.to("cuda")
    out32 = c.cache.decode_masked(q, c.lens, c.pt, wl.softmax_scale, mt, bound, out_fp32=True)
    out16 = c.cache.decode_masked(q, c.lens, c.pt, wl.softmax_scale, mt, bound + 37)
    st, bits = c.cache.get_error()
    assert st == K.KV4_OK, (st, bits)
    ref = c.oracle_decode(mask=m)
    assert_close(out32.cpu().numpy(), ref, what="%s %s gathered" % (geom, kind))
    assert_bf16_output(out16, out32, ref)
    # the page-granular masked path gives the same attention
    assert_close(out32.cpu().numpy(), c.decode(mask=mt).cpu().numpy(), what="%s %s vs page path" % (geom, kind))
    if kind == "empty":
        assert not out32.any()


def test_masked_gather_topk_mask_and_capacity():
    """Masks from kv_topk_retain (equal counts over heads), and a bound below
    the retained count: KV4_ERR_CAPACITY."""
    wl = small_wl([5000, 3001, 700, 2048], seed=62)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    Lmax = int(wl.lens.max())
    rng = np.random.default_rng(5)
    sc = rng.standard_normal((wl.B, wl.Hkv, Lmax)).astype(np.float32)
    mstride = (c.pt_np.shape[1] * 16 + 31) // 32
    mask = torch.zeros((wl.B, wl.Hkv, mstride), dtype=torch.int32, device="cuda")
    count = torch.zeros((wl.B, wl.Hkv), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(torch.as_tensor(sc, device="cuda"), c.lens, 200, mask, count, sink=wl.sink,
                     recent=wl.recent, max_len=Lmax)
    m = mask.cpu().numpy().view(np.uint32)
    cnt = _counts(m, wl.lens, wl.sink, wl.recent)
    assert (cnt == cnt[:, :1]).all()          # one count per sequence
    bound = int(np.floor(wl.lens.max() * 200 / 1000))
    q = c.q.to("cuda")
    out = c.cache.decode_masked(q, c.lens, c.pt, wl.softmax_scale, mask, bound, out_fp32=True)
    assert c.cache.get_error()[0] == K.KV4_OK
    assert_close(out.cpu().numpy(), c.oracle_decode(mask=m), what="top-k mask gathered")
    c.cache.decode_masked(q, c.lens, c.pt, wl.softmax_scale, mask, int(cnt.max()) - 1, out_fp32=True)
    st, bits = c.cache.get_error()
    assert st == K.KV4_ERR_CAPACITY
