"""GPU parity of every hot-path step against the fp64 oracle, through the C ABI.

Bit-exact: INT4/INT8 codes, scale bits and page/side-cache layout written by
kv4_append; retained-position masks and counts from kv_topk_retain.
Tolerance (helpers.py): attention outputs of kv4_decode_attn and
bf16_paged_decode_attn against the oracle on the same dequantised values.
"""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth
import compressed_kv_cache_kv4_b200 as K

from helpers import Case, assert_close, assert_bf16_output, bf16_pages

pytestmark = pytest.mark.gpu


def small_wl(lens, Hq=32, Hkv=8, D=128, seed=77, sink=16, recent=128):
    wl = synth.workload("qwen8b", B=len(lens))
    wl.lens = np.asarray(lens, np.int32)
    wl.B = len(lens)
    wl.Hq, wl.Hkv, wl.D, wl.seed = Hq, Hkv, D, seed
    wl.sink, wl.recent = sink, recent
    wl.softmax_scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    return wl


# ------------------------------------------------------------------ append
@pytest.mark.parametrize("name,chunks", [("tiny", 1), ("tiny", 3), ("mixed128", 1), ("mixed128", 4)])
def test_append_bytes_match_oracle(name, chunks):
    wl = synth.workload("tiny") if name == "tiny" else small_wl([1, 15, 16, 17, 143, 144, 145, 300, 1000])
    c = Case(wl)
    c.make_cache()
    c.append_all(chunks=chunks)
    pool, side, flags = c.oracle_cache()
    assert flags == 0
    st, bits = c.cache.get_error()
    assert st == K.KV4_OK, bits
    gp = c.cache.pool.cpu().numpy()
    assert np.array_equal(gp, pool), "page pool differs at %s" % np.flatnonzero(gp != pool)[:10]
    gs = c.cache.side.cpu().numpy()
    assert np.array_equal(gs, side), "side cache differs at %s" % np.flatnonzero(gs != side)[:10]


@pytest.mark.parametrize("sink,recent,D", [(16, 128, 128), (5, 16, 64), (0, 0, 64), (16, 0, 64), (0, 32, 128),
                                            (16, 48, 64)])
@pytest.mark.parametrize("chunks", [1, 3])
def test_append_side_windows_match_oracle(sink, recent, D, chunks):
    """INT8 side pages written whole by the page path (a sink page of 16 rows,
    ring pages whose rows all hold a position) and by rows (a shorter sink,
    partly filled ring pages, appends that do not renew the whole window),
    every pool and side byte against the oracle."""
    wl = small_wl([3, 16, 20, 47, 130, 257, 700], Hq=8, Hkv=2, D=D, seed=sink + recent + chunks, sink=sink,
                  recent=recent)
    c = Case(wl)
    c.make_cache()
    c.append_all(chunks=chunks)
    pool, side, flags = c.oracle_cache()
    assert flags == 0
    st, bits = c.cache.get_error()
    assert st == K.KV4_OK, bits
    gp = c.cache.pool.cpu().numpy()
    assert np.array_equal(gp, pool), "page pool differs at %s" % np.flatnonzero(gp != pool)[:10]
    if c.cache.side is not None:
        gs = c.cache.side.cpu().numpy()
        assert np.array_equal(gs, side), "side cache differs at %s" % np.flatnonzero(gs != side)[:10]


def test_append_unaligned_rows_match_oracle():
    """k_new / v_new 8- but not 16-byte aligned: whole pages go through the
    per-position kernel instead of the page kernel; the bytes are the same."""
    wl = small_wl([40, 64, 17, 200], Hq=8, Hkv=2)
    c = Case(wl)
    c.make_cache()
    T = c.k.shape[0]
    kbuf = torch.zeros(T * wl.Hkv * wl.D + 4, dtype=torch.bfloat16, device="cuda")
    vbuf = torch.zeros_like(kbuf)
    k = kbuf[4:].view(T, wl.Hkv, wl.D)
    v = vbuf[4:].view(T, wl.Hkv, wl.D)
    k.copy_(c.k.to("cuda"))
    v.copy_(c.v.to("cuda"))
    assert k.data_ptr() % 16 == 8
    c.cache.append(k, v, torch.as_tensor(c.off.astype(np.int32), device="cuda"),
                   torch.zeros(wl.B, dtype=torch.int32, device="cuda"), c.pt)
    torch.cuda.synchronize()
    pool, side, flags = c.oracle_cache()
    assert flags == 0 and c.cache.get_error()[0] == K.KV4_OK
    assert np.array_equal(c.cache.pool.cpu().numpy(), pool)
    assert np.array_equal(c.cache.side.cpu().numpy(), side)


def test_append_single_token_steps_ring():
    """Prefill, then one token per step: the ring keeps the last 128 positions
    exactly as the oracle's image of the final lengths."""
    steps = 20
    wl = small_wl(np.array([40, 150, 290]) + steps, seed=5)
    c = Case(wl)
    c.make_cache()
    k, v = c.k.cuda(), c.v.cuda()
    pre = (wl.lens - steps).astype(np.int64)
    idx = np.concatenate([np.arange(c.off[b], c.off[b] + pre[b]) for b in range(wl.B)])
    offs = np.zeros(wl.B + 1, np.int32)
    offs[1:] = np.cumsum(pre)
    it = torch.as_tensor(idx, device="cuda")
    c.cache.append(k[it].contiguous(), v[it].contiguous(), torch.as_tensor(offs, device="cuda"),
                   torch.zeros(wl.B, dtype=torch.int32, device="cuda"), c.pt)
    for s in range(steps):
        it = torch.as_tensor([int(c.off[b] + pre[b] + s) for b in range(wl.B)], device="cuda")
        c.cache.append(k[it].contiguous(), v[it].contiguous(), torch.arange(wl.B + 1, dtype=torch.int32, device="cuda"),
                       torch.as_tensor((pre + s).astype(np.int32), device="cuda"), c.pt)
    torch.cuda.synchronize()
    pool, side, _ = c.oracle_cache()
    assert np.array_equal(c.cache.pool.cpu().numpy(), pool)
    assert np.array_equal(c.cache.side.cpu().numpy(), side)


# ------------------------------------------------------------------ decode
def test_decode_tiny_end_to_end():
    wl = synth.workload("tiny")
    c = Case(wl)
    c.make_cache()
    c.append_all()
    ref = c.oracle_decode()
    out32 = c.decode(out_fp32=True)
    out16 = c.decode(out_fp32=False)
    assert_close(out32.cpu().numpy(), ref, what="tiny fp32")
    assert_bf16_output(out16, out32, ref)
    assert c.cache.get_error()[0] == K.KV4_OK


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 4, 2), (128, 8, 8), (64, 8, 4), (64, 4, 4), (128, 4, 2)])
def test_decode_from_oracle_bytes(D, Hq, Hkv):
    """The decode kernel reading bytes written by the oracle's own layout writer."""
    wl = small_wl([1, 16, 17, 100, 144, 145, 160, 161, 700, 2049, 3001], Hq=Hq, Hkv=Hkv, D=D, seed=D + Hq)
    c = Case(wl)
    c.make_cache()
    c.load_oracle_bytes()
    ref = c.oracle_decode()
    out = c.decode(out_fp32=True)
    assert_close(out.cpu().numpy(), ref, what="D=%d G=%d" % (D, Hq // Hkv))


@pytest.mark.parametrize("workers", [4, 8, 12, 60, 0, 4000])
def test_worker_count_invariance(workers):
    wl = small_wl([3000, 2, 0, 500, 145, 4100, 900, 1600, 33], seed=11)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    ref = c.oracle_decode()
    out = c.decode(num_workers=workers)
    assert_close(out.cpu().numpy(), ref, what="workers=%d" % workers)


def test_deterministic_run_to_run():
    wl = small_wl([2500, 700, 3100], seed=12)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    a = c.decode()
    b = c.decode()
    assert torch.equal(a, b)


def test_short_context_ignores_int4_pages():
    """L <= 144 is entirely INT8: poisoning the INT4 pages changes nothing."""
    wl = small_wl([144, 37, 1, 100], seed=13)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    a = c.decode()
    c.cache.pool.copy_(torch.randint(0, 256, c.cache.pool.shape, dtype=torch.uint8, device="cuda"))
    b = c.decode()
    assert torch.equal(a, b)
    assert_close(a.cpu().numpy(), c.oracle_decode(), what="short")


def test_protected_positions_ignore_int4_codes():
    """L > 144: the INT4 copies of sink and recent positions are never read."""
    wl = small_wl([400], seed=14, Hq=8, Hkv=2)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    a = c.decode()
    pool = c.cache.pool.view(c.num_pages, wl.Hkv, 18 * wl.D)
    # page 0 = positions 0..15 (sink); pages 17..24 hold positions >= 272 = L - 128
    for lp in [0] + list(range(17, 25)):
        pool[int(c.pt_np[0, lp])] = torch.randint(0, 256, pool[0].shape, dtype=torch.uint8, device="cuda")
    b = c.decode()
    assert torch.equal(a, b)


def test_pure_kv4_mode():
    wl = small_wl([1, 0, 300, 1700], seed=15, sink=0, recent=0)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    assert c.cache.side is None
    assert_close(c.decode().cpu().numpy(), c.oracle_decode(), what="pure kv4")


def test_mask_full_empty_random():
    wl = small_wl([3000, 150, 40, 1800], seed=16)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    mstride = (c.pt_np.shape[1] * 16 + 31) // 32
    full = torch.full((wl.B, wl.Hkv, mstride), -1, dtype=torch.int32, device="cuda")
    base = c.decode()
    assert torch.equal(c.decode(mask=full), base)
    zero = torch.zeros_like(full)
    assert not c.decode(mask=zero).any()
    rng = np.random.default_rng(3)
    rnd = rng.integers(0, 2 ** 32, size=(wl.B, wl.Hkv, mstride), dtype=np.uint64).astype(np.uint32)
    rnd[:, :, :3] = 0                       # whole pages without a retained position
    out = c.decode(mask=torch.as_tensor(rnd.view(np.int32), device="cuda"))
    assert_close(out.cpu().numpy(), c.oracle_decode(mask=rnd), what="random mask")


# ------------------------------------------------------------------ top-k
@pytest.mark.parametrize("permille", [0, 100, 300, 500, 900, 1000])
def test_topk_matches_oracle(permille):
    rng = np.random.default_rng(permille + 1)
    B, Hkv, Lmax = 5, 3, 5000
    lens = np.array([5000, 1, 145, 2000, 4097], np.int32)
    sc = rng.standard_normal((B, Hkv, Lmax)).astype(np.float32)
    sc[0, 0] = np.round(sc[0, 0] * 2) / 2           # heavy ties
    sc[1, 1, :] = 0.0
    sc[2, 2, ::3] = -0.0
    mstride = (Lmax + 31) // 32 + 1
    mask = torch.full((B, Hkv, mstride), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    count = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(torch.as_tensor(sc, device="cuda"), torch.as_tensor(lens, device="cuda"), permille,
                     mask, count)
    m_ref, c_ref = O.topk(sc, lens, permille)
    got = mask.cpu().numpy().view(np.uint32)
    for b in range(B):
        nw = (int(lens[b]) + 31) // 32
        assert np.array_equal(got[b, :, :nw], m_ref[b, :, :nw]), (b, permille)
        assert np.all(got[b, :, nw:] == 0x5A5A5A5A)          # words past L untouched
    assert np.array_equal(count.cpu().numpy(), c_ref)


@pytest.mark.parametrize("permille", [100, 500])
def test_topk_crowded_threshold_bin(permille):
    """Rows whose threshold bin (sign, exponent and two mantissa bits) holds
    more keys than the short list of the staged path: equal scores, one large
    block of equal scores among random ones, and distinct scores that all lie
    in [1, 1.25). The selection falls back to the general path and must give
    the same masks."""
    rng = np.random.default_rng(permille + 7)
    B, Hkv, Lmax = 2, 2, 6000
    lens = np.array([6000, 5003], np.int32)
    sc = rng.standard_normal((B, Hkv, Lmax)).astype(np.float32)
    sc[0, 0, :] = 1.0
    sc[0, 1, 1000:4000] = 2.0
    sc[1, 0, :] = (1.0 + 0.25 * rng.random(Lmax)).astype(np.float32)
    sc[1, 1, :] = np.float32(1.0) + np.float32(2.0 ** -20) * rng.integers(0, 64, Lmax).astype(np.float32)
    mstride = (Lmax + 31) // 32
    mask = torch.zeros((B, Hkv, mstride), dtype=torch.int32, device="cuda")
    count = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(torch.as_tensor(sc, device="cuda"), torch.as_tensor(lens, device="cuda"), permille, mask, count)
    m_ref, c_ref = O.topk(sc, lens, permille)
    got = mask.cpu().numpy().view(np.uint32)
    for b in range(B):
        nw = (int(lens[b]) + 31) // 32
        assert np.array_equal(got[b, :, :nw], m_ref[b, :, :nw]), b
    assert np.array_equal(count.cpu().numpy(), c_ref)


@pytest.mark.parametrize("permille", [10, 100, 990])
def test_topk_range_off_the_first_loads(permille):
    """Rows whose values depend strongly on the position, so that a part of the
    row alone misjudges the range of the whole: tail outliers far above or far
    below the rest, an exponential ramp, and blocks of 1024 positions with
    scales from 1e-20 to 1e20. Thresholds among the outliers fall outside any
    range estimated without them; the masks must still equal the oracle's."""
    rng = np.random.default_rng(permille + 31)
    B, Hkv, Lmax = 2, 4, 16384
    lens = np.array([16384, 9001], np.int32)
    sc = rng.standard_normal((B, Hkv, Lmax)).astype(np.float32)
    for b, L in enumerate(lens):
        sc[b, 0, L - 428:L - 128] = np.float32(1e30) * (1.0 + rng.random(300)).astype(np.float32)
        sc[b, 1, L - 428:L - 128] = np.float32(-1e30) * (1.0 + rng.random(300)).astype(np.float32)
        sc[b, 2, :] = np.exp2(np.arange(Lmax) / 256.0).astype(np.float32)
        scale = 10.0 ** rng.uniform(-20, 20, (Lmax + 1023) // 1024)
        sc[b, 3, :] = (sc[b, 3, :] * np.repeat(scale, 1024)[:Lmax]).astype(np.float32)
    mstride = (Lmax + 31) // 32
    mask = torch.zeros((B, Hkv, mstride), dtype=torch.int32, device="cuda")
    count = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(torch.as_tensor(sc, device="cuda"), torch.as_tensor(lens, device="cuda"), permille, mask, count)
    m_ref, c_ref = O.topk(sc, lens, permille)
    got = mask.cpu().numpy().view(np.uint32)
    for b in range(B):
        nw = (int(lens[b]) + 31) // 32
        assert np.array_equal(got[b, :, :nw], m_ref[b, :, :nw]), b
    assert np.array_equal(count.cpu().numpy(), c_ref)


@pytest.mark.parametrize("permille", [100, 300])
def test_topk_threshold_bin_sizes(permille):
    """Rows whose threshold bin holds few keys (the exact selection among them
    by one warp) or a few dozen to a few hundred (by digit histograms): a
    block of equal scores of 8, 31, 33 or 60 positions placed at the budget's
    quantile, and a coarse value grid (about 128 equal keys per value)."""
    rng = np.random.default_rng(permille + 41)
    B, Hkv, Lmax = 2, 5, 16384
    lens = np.array([16384, 7001], np.int32)
    sc = rng.standard_normal((B, Hkv, Lmax)).astype(np.float32)
    for b, L in enumerate(lens):
        c = np.arange(16, L - 128)
        for h, run in enumerate((8, 31, 33, 60)):
            row = sc[b, h]
            q = np.sort(row[c])[::-1][int(L) * permille // 1000 - 144]
            pos = rng.choice(c, run, replace=False)
            row[pos] = q
        sc[b, 4, :] = (np.round(sc[b, 4, :] * 16) / 16).astype(np.float32)
    mstride = (Lmax + 31) // 32
    mask = torch.zeros((B, Hkv, mstride), dtype=torch.int32, device="cuda")
    count = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(torch.as_tensor(sc, device="cuda"), torch.as_tensor(lens, device="cuda"), permille, mask, count)
    m_ref, c_ref = O.topk(sc, lens, permille)
    got = mask.cpu().numpy().view(np.uint32)
    for b in range(B):
        nw = (int(lens[b]) + 31) // 32
        assert np.array_equal(got[b, :, :nw], m_ref[b, :, :nw]), b
    assert np.array_equal(count.cpu().numpy(), c_ref)


def test_topk_long_rows_global_path():
    rng = np.random.default_rng(9)
    B, Hkv, Lmax = 1, 2, 70000
    lens = np.array([70000], np.int32)
    sc = rng.standard_normal((B, Hkv, Lmax)).astype(np.float32)
    sc[0, 1] = np.round(sc[0, 1] * 4) / 4
    mstride = (Lmax + 31) // 32
    mask = torch.zeros((B, Hkv, mstride), dtype=torch.int32, device="cuda")
    K.kv_topk_retain(torch.as_tensor(sc, device="cuda"), torch.as_tensor(lens, device="cuda"), 500, mask)
    m_ref, _ = O.topk(sc, lens, 500)
    assert np.array_equal(mask.cpu().numpy().view(np.uint32), m_ref)


# ------------------------------------------------------------------ bf16 comparison kernel
@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 4, 2)])
def test_bf16_paged_decode(D, Hq, Hkv):
    wl = small_wl([1, 15, 16, 17, 500, 2049], Hq=Hq, Hkv=Hkv, D=D, seed=21)
    c = Case(wl)
    pages = bf16_pages(c)
    pt = torch.as_tensor(c.pt_np, device="cuda")
    lens = torch.as_tensor(wl.lens, device="cuda")
    ws = torch.zeros(K.bf16_paged_workspace_bytes(wl.B, Hq, Hkv, D), dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.B, Hq, D), dtype=torch.float32, device="cuda")
    K.bf16_paged_decode_attn(c.q.cuda(), pages, pt, lens, wl.softmax_scale, ws, out, Hkv)
    assert_close(out.cpu().numpy(), c.oracle_decode(mode=1), what="bf16 kernel")


# ------------------------------------------------------------------ error paths (no fault)
def test_bad_page_id_is_reported():
    wl = small_wl([600, 300], seed=31)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    assert c.cache.get_error()[0] == K.KV4_OK
    bad = c.pt.clone()
    bad[0, 10] = c.num_pages + 5
    bad[1, 3] = -7
    c.cache.decode(c.q.cuda(), c.lens, bad, wl.softmax_scale, out_fp32=True)
    st, bits = c.cache.get_error()
    assert st == K.KV4_ERR_BOUNDS and bits & (1 << K.KV4_ERR_BOUNDS)
    assert c.cache.get_error()[0] == K.KV4_OK          # cleared
    assert_close(c.decode().cpu().numpy(), c.oracle_decode(), what="after bounds error")


def test_length_beyond_capacity_is_reported():
    wl = small_wl([600], seed=32)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    too_long = torch.as_tensor([c.pt_np.shape[1] * 16 + 1], dtype=torch.int32, device="cuda")
    out = c.cache.decode(c.q.cuda(), too_long, c.pt, wl.softmax_scale, out_fp32=True)
    st, _ = c.cache.get_error()
    assert st == K.KV4_ERR_CAPACITY and not out.any()


def test_wait_timeout_is_reported_and_context_survives():
    wl = small_wl([900, 500], seed=33)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    K.kv4_debug_set_wait_limit(c.cache.handle, 0)
    c.decode()
    st, _ = c.cache.get_error()
    assert st == K.KV4_ERR_TIMEOUT
    K.kv4_debug_set_wait_limit(c.cache.handle, -1)
    assert_close(c.decode().cpu().numpy(), c.oracle_decode(), what="after timeout")
    assert c.cache.get_error()[0] == K.KV4_OK


def test_range_overflow_flag():
    wl = small_wl([20], seed=34, Hq=4, Hkv=1)
    c = Case(wl)
    c.k[3, 0, 5] = 6.0e5                   # |x| > 458,528: scale overflows fp16
    c.make_cache()
    c.append_all()
    st, _ = c.cache.get_error()
    assert st == K.KV4_ERR_RANGE
    pool, side, flags = c.oracle_cache()
    assert flags == 1
    assert np.array_equal(c.cache.pool.cpu().numpy(), pool)
    assert np.array_equal(c.cache.side.cpu().numpy(), side)


def test_append_exact_ties():
    """Rows built so that x/scale is exactly k + 1/2 for many elements (INT4 and
    INT8 scales that are powers of two): codes must round half to even."""
    wl = small_wl([40], seed=35, Hq=4, Hkv=1)
    c = Case(wl)
    D = wl.D
    rng = np.random.default_rng(0)
    rows = []
    for p in range(40):
        e = float(2.0 ** int(rng.integers(-6, 4)))
        row = np.zeros(D, np.float32)
        for grp in range(D // 32):
            vals = (rng.integers(-7, 7, size=32) + 0.5) * e          # ties for an INT4 scale of e
            vals[int(rng.integers(0, 32))] = 7 * e * (1 if rng.random() < 0.5 else -1)
            row[32 * grp: 32 * grp + 32] = vals
        if p % 2:                                                   # INT8 ties: max 127 e
            row = ((rng.integers(-127, 127, size=D) + 0.5) * e).astype(np.float32)
            row[int(rng.integers(0, D))] = 127 * e
        rows.append(row)
    kt = torch.as_tensor(np.stack(rows)[:, None, :]).to(torch.bfloat16)
    assert torch.equal(kt.float(), torch.as_tensor(np.stack(rows)[:, None, :]))   # exact in bf16
    c.k = kt
    c.v = -kt
    c.make_cache()
    c.append_all()
    pool, side, _ = c.oracle_cache()
    assert np.array_equal(c.cache.pool.cpu().numpy(), pool)
    assert np.array_equal(c.cache.side.cpu().numpy(), side)


# ------------------------------------------------------------------ query magnitude
def _scaled_queries(q, scale, spike_channels, spike):
    """q * scale, with `spike_channels` channels of every query head multiplied by `spike` more
    (queries after a QK-norm are far from N(0, 1) per channel)."""
    x = q.float() * scale
    if spike_channels:
        g = torch.Generator().manual_seed(99)
        ch = torch.randperm(q.shape[-1], generator=g)[:spike_channels]
        x[..., ch] *= spike
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("scale,spike_channels,spike", [(8.0, 0, 1.0), (32.0, 0, 1.0), (1.0, 3, 100.0),
                                                         (8.0, 4, 100.0), (0.01, 0, 1.0)])
def test_decode_large_queries(scale, spike_channels, spike):
    """q·K with queries far from N(0, 1): large magnitudes (peaky softmax, scores in the
    hundreds), a few channels two orders of magnitude above the rest, and tiny queries
    (near-uniform softmax). Outputs stay within the tolerance of the fp64 oracle."""
    wl = small_wl([1, 17, 145, 300, 1000, 2049, 3001], seed=41)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    q = _scaled_queries(c.q, scale, spike_channels, spike)
    assert torch.isfinite(q.float()).all()
    c.q = q
    ref = c.oracle_decode()
    out32 = c.decode(out_fp32=True)
    out16 = c.decode(out_fp32=False)
    assert c.cache.get_error()[0] == K.KV4_OK
    assert_close(out32.cpu().numpy(), ref, what="q x%g, %d channels x%g" % (scale, spike_channels, spike))
    assert_bf16_output(out16, out32, ref)


def test_decode_query_beyond_fp16_range_is_reported():
    """A query element whose magnitude exceeds the fp16 range cannot enter the fp16 tiles:
    the kernel reports KV4_ERR_RANGE instead of returning silently wrong scores."""
    wl = small_wl([300, 40], seed=42, Hq=8, Hkv=2)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    q = c.q.clone()
    q[0, 1, 5] = 1.0e5
    c.decode(q=q)
    st, bits = c.cache.get_error()
    assert st == K.KV4_ERR_RANGE and bits & (1 << K.KV4_ERR_RANGE)
    assert c.cache.get_error()[0] == K.KV4_OK
