"""GPU parity of kv4_evict_pages (page-granular eviction and compaction)
against the fp64 oracle, through the C ABI.

Bit-exact: the rewritten page tables, lengths, free lists and counts, the
rotated side cache (every byte), the untouched page pool. Within the attention
tolerance: decode of the compacted cache against the oracle's decode of the
compacted sequences, and the same after one more appended position (the
compacted cache keeps streaming into its surviving pages).
"""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth
import compressed_kv_cache_kv4_b200 as K

from helpers import Case, assert_close
from test_gpu_parity import small_wl

pytestmark = pytest.mark.gpu

EXTRA = 40   # positions mapped ahead of each sequence's length


def _scores(wl, stride, seed, ties):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((wl.B, wl.Hkv, stride)).astype(np.float32)
    if ties:   # small integers: many pages with equal sums
        s = rng.integers(0, 3, size=s.shape).astype(np.float32)
    s[0, :, 16:32] = -0.0       # a page of negative zeros
    return s


def _compacted(case, b, freed_ids, pt_np):
    """Surviving positions of sequence b (rows of the original packed K/V)."""
    L = int(case.wl.lens[b])
    ev = {j for j in range(pt_np.shape[1]) if int(pt_np[b, j]) in freed_ids}
    keep = [p for p in range(L) if p // 16 not in ev]
    return np.asarray(case.off[b] + np.asarray(keep, np.int64), np.int64)


def _pad(rows_list, x, Lmax):
    out = torch.zeros((len(rows_list), max(Lmax, 1)) + tuple(x.shape[1:]), dtype=x.dtype)
    for i, r in enumerate(rows_list):
        out[i, : len(r)] = x[torch.as_tensor(r, dtype=torch.long)]
    return out


def _side(case):
    side = case.cache.side
    return np.zeros(0, np.uint8) if side is None else side.cpu().numpy()


CONFIGS = [
    # D, Hq, Hkv, sink, recent
    (128, 32, 8, 16, 128),
    (64, 4, 2, 16, 128),
    (64, 8, 4, 0, 64),
    (128, 8, 2, 5, 16),
    (64, 4, 1, 0, 0),
]


@pytest.mark.parametrize("cfg", CONFIGS)
@pytest.mark.parametrize("permille", [0, 250, 600, 1000])
def test_evict_matches_oracle(cfg, permille):
    D, Hq, Hkv, sink, recent = cfg
    lens = [300, 0, 5, 160, 161, 700, 2049, 3001, 1200]
    wl = small_wl(lens, Hq=Hq, Hkv=Hkv, D=D, seed=D + Hkv + sink, sink=sink, recent=recent)
    c = Case(wl, extra_tokens=EXTRA)
    c.make_cache()
    c.append_all(chunks=2)
    stride = int(max(lens)) + 12                          # stride % 4 == 0: vector loads
    sc = _scores(wl, stride, seed=permille + D, ties=(permille == 600))
    pool0, side0, _ = c.oracle_cache()
    gpool = c.cache.pool.clone()

    freed, cnt = c.cache.evict_pages(torch.as_tensor(sc, device="cuda"), permille, c.lens, c.pt)
    st, bits = c.cache.get_error()
    assert st == K.KV4_OK, bits
    l2, pt2, fr, cnt_ref, side_ref = O.evict_pages(sc, wl.lens, c.pt_np, side0, D, permille, sink, recent)
    assert np.array_equal(c.lens.cpu().numpy(), l2)
    assert np.array_equal(c.pt.cpu().numpy(), pt2)
    assert np.array_equal(cnt.cpu().numpy(), cnt_ref)
    gfr = freed.cpu().numpy()
    for b in range(wl.B):
        assert np.array_equal(gfr[b, : cnt_ref[b]], fr[b, : cnt_ref[b]]), b
        assert np.all(gfr[b, cnt_ref[b]:] == -1), b        # entries past the count untouched
    gs = _side(c)
    assert np.array_equal(gs, side_ref), "side differs at %s" % np.flatnonzero(gs != side_ref)[:10]
    assert torch.equal(c.cache.pool, gpool)

    # decode of the compacted cache
    rows = [_compacted(c, b, set(int(x) for x in fr[b, : cnt_ref[b]]), c.pt_np) for b in range(wl.B)]
    Lmax = int(l2.max())
    kb = synth.bf16_bits(_pad(rows, c.k, Lmax))
    vb = synth.bf16_bits(_pad(rows, c.v, Lmax))
    qb = synth.bf16_bits(c.q)
    ref = O.decode(c.shape(), qb, kb, vb, l2, wl.softmax_scale)
    out = c.cache.decode(c.q.cuda(), c.lens, c.pt, wl.softmax_scale, out_fp32=True)
    assert_close(out.cpu().numpy(), ref, what="compacted decode")

    # one more position per sequence goes into the surviving (or mapped-ahead) pages
    gen = torch.Generator().manual_seed(99)
    kn = torch.randn((wl.B, Hkv, D), generator=gen).to(torch.bfloat16)
    vn = torch.randn((wl.B, Hkv, D), generator=gen).to(torch.bfloat16)
    old = c.lens.clone()
    K.kv4_append(c.cache.handle, kn.cuda(), vn.cuda(), None, old, c.pt)
    new_lens = l2 + 1
    c.lens = torch.as_tensor(new_lens.astype(np.int32), device="cuda")
    kb2 = np.zeros((wl.B, Lmax + 1, Hkv, D), np.uint16)
    vb2 = np.zeros_like(kb2)
    kb2[:, :Lmax] = kb[:, :Lmax]
    vb2[:, :Lmax] = vb[:, :Lmax]
    knb, vnb = synth.bf16_bits(kn), synth.bf16_bits(vn)
    for b in range(wl.B):
        kb2[b, l2[b]] = knb[b]
        vb2[b, l2[b]] = vnb[b]
    ref2 = O.decode(c.shape(), qb, kb2, vb2, new_lens, wl.softmax_scale)
    out2 = c.cache.decode(c.q.cuda(), c.lens, c.pt, wl.softmax_scale, out_fp32=True)
    assert_close(out2.cpu().numpy(), ref2, what="append after compaction")
    # bytes a fresh append of the compacted sequences writes (equal under two fills)
    pa, sa, _ = O.write_cache(c.shape(), kb2, vb2, new_lens, pt2, c.num_pages, fill=0xA5)
    pb, sb, _ = O.write_cache(c.shape(), kb2, vb2, new_lens, pt2, c.num_pages, fill=0x5A)
    gp, gs = c.cache.pool.cpu().numpy(), _side(c)
    wp, ws = pa == pb, sa == sb
    assert np.array_equal(gp[wp], pa[wp])
    assert np.array_equal(gs[ws], sa[ws])
    assert c.cache.get_error()[0] == K.KV4_OK
    c.cache.close()


def test_evict_scalar_score_path_and_bad_length():
    """Scores at an odd row stride take the scalar loads; a length beyond the
    score stride is reported and leaves its sequence as it was."""
    lens = [700, 2049, 400]
    wl = small_wl(lens, Hq=8, Hkv=2, D=64, seed=3)
    c = Case(wl, extra_tokens=EXTRA)
    c.make_cache()
    c.append_all()
    stride = 2049 + 3                                      # odd stride
    sc = _scores(wl, stride, seed=5, ties=False)
    pool0, side0, _ = c.oracle_cache()
    freed, cnt = c.cache.evict_pages(torch.as_tensor(sc, device="cuda"), 300, c.lens, c.pt)
    assert c.cache.get_error()[0] == K.KV4_OK
    l2, pt2, fr, cnt_ref, side_ref = O.evict_pages(sc, wl.lens, c.pt_np, side0, 64, 300)
    assert np.array_equal(c.lens.cpu().numpy(), l2) and np.array_equal(c.pt.cpu().numpy(), pt2)
    assert np.array_equal(cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(c.cache.side.cpu().numpy(), side_ref)

    # lengths now l2; claim sequence 1 is longer than the score rows
    bad = c.lens.clone()
    bad[1] = stride + 1
    pt_before = c.pt.clone()
    side_before = c.cache.side.clone()
    sc_small = torch.as_tensor(sc, device="cuda")
    freed, cnt = c.cache.evict_pages(sc_small, 0, bad, c.pt)
    st, bits = c.cache.get_error()
    assert st == K.KV4_ERR_CAPACITY
    assert int(cnt[1]) == 0 and int(bad[1]) == stride + 1
    assert torch.equal(c.pt[1], pt_before[1])
    blk = side_before.numel() // wl.B
    assert torch.equal(c.cache.side[blk: 2 * blk], side_before[blk: 2 * blk])
    c.cache.close()
