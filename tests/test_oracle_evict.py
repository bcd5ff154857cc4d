"""Pins for the oracle's page-granular eviction and compaction.

Pages: KVP promo (arXiv 2602.10238), engineering-limitations section, third
item -- a paged cache with 16-position blocks ranks and evicts whole blocks on
the mean of their positions' scores; KV-streams summary page, method details
(core idea) -- the compacted cache keeps streaming; KV4-RL review sec. 3 --
the first 16 and last 128 positions stay INT8-protected. Build readings: only
full pages outside the INT8 set are candidates, k = floor(n * permille /
1000) pages with the kept non-candidates counted toward k, ties to the lower
page index; later positions move down 16 per evicted page.

Each check reaches the expected result by a route other than the oracle's own
sort and rewrite: hand-worked tables, a pairwise order check on integer scores
(page sums exact in any order), decode of the compacted sequence against masked
decode of the original, and the rotated side image against re-appending the
surviving positions from scratch.
"""
import numpy as np
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth


def _page_scores(values_per_page, Hkv, stride):
    """scores [1][Hkv][stride] with every position of page j equal to values_per_page[j]."""
    s = np.zeros((1, Hkv, stride), np.float32)
    for j, c in enumerate(values_per_page):
        s[0, :, 16 * j: 16 * j + 16] = c
    return s


def test_hand_worked_tables():
    # L = 200, sink 16, recent 128: pages 0..12, page 12 partial (8 positions).
    # Candidates: pages 1, 2, 3 (page 4 holds position 72 = L - 128).
    L, Hkv, pt_stride = 200, 2, 16
    vals = [0.0, 2.0, 5.0, 5.0] + [0.0] * 9
    sc = _page_scores(vals, Hkv, 208)
    pt = (100 + np.arange(pt_stride, dtype=np.int32))[None, :].copy()   # entries 13..15 mapped ahead
    # permille 1000: k = 13 -> keep all.
    lens, pt2, fr, cnt, _ = O.evict_pages(sc, [L], pt, None, 64, 1000)
    assert lens[0] == 200 and cnt[0] == 0 and np.array_equal(pt2, pt)
    # permille 900: k = 11, 10 kept non-candidates -> keep 1 candidate: pages 2
    # and 3 tie on 5.0, the lower index wins; pages 1 and 3 are evicted.
    lens, pt2, fr, cnt, _ = O.evict_pages(sc, [L], pt, None, 64, 900)
    assert lens[0] == 200 - 32 and cnt[0] == 2
    assert list(fr[0, :2]) == [101, 103] and np.all(fr[0, 2:] == -1)
    assert list(pt2[0]) == [100, 102] + list(range(104, 116)) + [-1, -1]
    # permille 0: every candidate goes.
    lens, pt2, fr, cnt, _ = O.evict_pages(sc, [L], pt, None, 64, 0)
    assert lens[0] == 152 and list(fr[0, :3]) == [101, 102, 103]
    assert list(pt2[0]) == [100] + list(range(104, 116)) + [-1, -1, -1]


def test_no_candidates_and_degenerate_lengths():
    Hkv = 2
    sc = np.random.default_rng(1).standard_normal((5, Hkv, 160)).astype(np.float32)
    lens = np.array([0, 5, 16, 144, 159], np.int32)
    pt = np.arange(5 * 10, dtype=np.int32).reshape(5, 10)
    for permille in (0, 500, 1000):
        l2, pt2, fr, cnt, _ = O.evict_pages(sc, lens, pt, None, 64, permille)
        # L <= 159: the INT8 set [0,16) u [L-128, L) leaves no full page between.
        assert np.array_equal(l2, lens) and np.array_equal(pt2, pt) and np.all(cnt == 0)
    # L = 160: page 1 = [16, 32) lies below L - 128 = 32 -> one candidate.
    l2, pt2, fr, cnt, _ = O.evict_pages(sc[:1], [160], pt[:1], None, 64, 0)
    assert l2[0] == 144 and cnt[0] == 1 and fr[0, 0] == 1


def test_partial_last_page_is_never_evicted():
    # sink = recent = 0: every full page is a candidate, the partial one is not.
    Hkv, L = 1, 1000                     # 62 full pages + 8 positions
    vals = [float(j % 7) for j in range(63)]
    sc = _page_scores(vals, Hkv, 1008)
    pt = np.arange(64, dtype=np.int32)[None, :].copy()
    lens, pt2, fr, cnt, _ = O.evict_pages(sc, [L], pt, None, 64, 500, sink=0, recent=0)
    # k = floor(63 * 0.5) = 31; the partial page counts toward it -> 30 full pages kept.
    assert cnt[0] == 32 and lens[0] == L - 32 * 16
    assert pt2[0, 30] == 62          # the partial page is the last surviving entry
    assert pt2[0, 31] == 63 and np.all(pt2[0, 32:] == -1)


def test_pairwise_order_on_exact_sums():
    """Every kept candidate beats every evicted candidate by (page mean desc,
    index asc); the number kept follows the floor rule. Integer scores make
    every page sum exact, so the order is checked on int64 sums."""
    rng = np.random.default_rng(7)
    B, Hkv, stride = 6, 3, 1600
    for trial in range(8):
        levels = int(rng.integers(1, 6))
        sc = rng.integers(-levels, levels + 1, size=(B, Hkv, stride)).astype(np.float32)
        lens = rng.integers(0, stride + 1, size=B).astype(np.int32)
        sink, recent = [(16, 128), (0, 0), (16, 0), (0, 64), (5, 32)][trial % 5]
        permille = int(rng.integers(0, 1001))
        pt_stride = stride // 16 + 3
        pt = rng.permutation(B * pt_stride).astype(np.int32).reshape(B, pt_stride)
        l2, pt2, fr, cnt, _ = O.evict_pages(sc, lens, pt, None, 64, permille, sink, recent)
        for b in range(B):
            L = int(lens[b])
            n = (L + 15) // 16
            cand = [j for j in range(n)
                    if 16 * j + 16 <= L and 16 * j >= sink and 16 * j + 16 <= L - recent]
            # a page with a protected position lies partly below sink or past L - recent
            sums = {j: int(sc[b, :, 16 * j: 16 * j + 16].astype(np.int64).sum()) for j in cand}
            freed = set(int(x) for x in fr[b, : cnt[b]])
            ev = [j for j in cand if int(pt[b, j]) in freed]
            kept = [j for j in cand if j not in ev]
            assert len(freed) == cnt[b] == len(ev)
            want_kept = max(0, min(len(cand), n * permille // 1000 - (n - len(cand))))
            assert len(kept) == want_kept, (trial, b)
            for a in kept:
                for d in ev:
                    assert sums[a] > sums[d] or (sums[a] == sums[d] and a < d), (trial, b, a, d)
            assert l2[b] == L - 16 * len(ev)
            surv = [int(pt[b, j]) for j in range(pt_stride) if not (j < n and j in ev)]
            assert list(pt2[b]) == surv + [-1] * len(ev)
            assert list(fr[b, : cnt[b]]) == [int(pt[b, j]) for j in ev]


def _compacted_rows(kb, vb, L, evicted_pages):
    keep = [p for p in range(L) if p // 16 not in set(evicted_pages)]
    return kb[keep], vb[keep]


def test_compacted_decode_equals_masked_decode_and_side_image():
    """Decode of the compacted sequences (re-appended from scratch) equals
    decode of the original sequences with the evicted pages masked out; the
    oracle's rotated side image and its rewritten page table equal what a
    fresh append of the surviving positions writes."""
    rng = np.random.default_rng(11)
    for (sink, recent, D, Hkv) in [(16, 128, 64, 2), (16, 64, 128, 1), (0, 32, 64, 2), (7, 16, 64, 1)]:
        lens = np.array([1200, 37, 0, 700, 161, 2000], np.int32)
        B, Hq = len(lens), 2 * Hkv
        Lmax = int(lens.max())
        g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
        q = synth.bf16_bits(torch.randn((B, Hq, D), generator=g).to(torch.bfloat16))
        kt = torch.randn((B, Lmax, Hkv, D), generator=g).to(torch.bfloat16)
        vt = torch.randn((B, Lmax, Hkv, D), generator=g).to(torch.bfloat16)
        kb, vb = synth.bf16_bits(kt), synth.bf16_bits(vt)
        sc = rng.standard_normal((B, Hkv, Lmax)).astype(np.float32)
        pt_stride = (Lmax + 15) // 16 + 2
        num_pages = B * pt_stride
        pt = rng.permutation(num_pages).astype(np.int32).reshape(B, pt_stride)
        sh = O.shape(B, Hq, Hkv, D, sink, recent)
        pool0, side0, _ = O.write_cache(sh, kb, vb, lens, pt, num_pages)
        for permille in (0, 300, 800):
            l2, pt2, fr, cnt, side1 = O.evict_pages(sc, lens, pt, side0, D, permille, sink, recent)
            # 1. decode: compacted rows vs masked original
            ck = np.zeros_like(kb)
            cv = np.zeros_like(vb)
            mstride = (Lmax + 31) // 32
            mask = np.zeros((B, Hkv, mstride), np.uint32)
            for b in range(B):
                ev_ids = set(int(x) for x in fr[b, : cnt[b]])
                ev_pages = [j for j in range(pt_stride) if int(pt[b, j]) in ev_ids]
                rk, rv = _compacted_rows(kb[b], vb[b], int(lens[b]), ev_pages)
                assert rk.shape[0] == l2[b]
                ck[b, : rk.shape[0]] = rk
                cv[b, : rv.shape[0]] = rv
                for p in range(int(lens[b])):
                    if p // 16 not in ev_pages:
                        mask[b, :, p // 32] |= np.uint32(1 << (p % 32))
            out_c = O.decode(sh, q, ck, cv, l2, 0.125)
            out_m = O.decode(sh, q, kb, vb, lens, 0.125, mask=mask)
            assert np.array_equal(out_c, out_m), (sink, recent, permille)
            # 2. side image and page table: a fresh append of the compacted rows
            # through the rewritten table; bytes it writes are those it leaves
            # equal under two different fill values.
            pa, sa, _ = O.write_cache(sh, ck, cv, l2, pt2, num_pages, fill=0xA5)
            pb, sb, _ = O.write_cache(sh, ck, cv, l2, pt2, num_pages, fill=0x5A)
            ws = sa == sb
            assert np.array_equal(side1[ws], sa[ws]), (sink, recent, permille)
            wp = pa == pb
            assert np.array_equal(pool0[wp], pa[wp]), (sink, recent, permille)
