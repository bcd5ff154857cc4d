"""Pins for the oracle's attention, merge and region split.

What the pages fix (KV4-RL review, sec. 3): the INT4 region and the INT8
region (first 16, last 128 positions) are attended independently and their
partials are combined by an exact softmax merge, so the merge of the partials
equals one softmax over the union; a context of at most 144 positions is
entirely INT8. SMD (sec. 1, Figure 1): a binary mask of retained positions is
applied inside attention, so a full mask reproduces unmasked attention.
Closed forms (equal scores, zero query, dominant key, two keys) pin the
single-pass definition itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth


def _bits(x):
    return synth.bf16_bits(torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16))


def _tiny_inputs(lens, Hq=4, Hkv=2, D=64, seed=0, sink=16, recent=128):
    g = torch.Generator().manual_seed(seed)
    B, Lmax = len(lens), max(lens)
    q = torch.randn((B, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Lmax, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Lmax, Hkv, D), generator=g).to(torch.bfloat16)
    sh = O.shape(B, Hq, Hkv, D, sink, recent)
    return sh, synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), np.array(lens, np.int32)


def test_merge_equals_single_softmax_random_chunkings():
    rng = np.random.default_rng(3)
    for trial in range(50):
        n, D = int(rng.integers(1, 300)), 16
        q = rng.standard_normal(D)
        kr = rng.standard_normal((n, D)) * 3
        vr = rng.standard_normal((n, D))
        m, l, o = O.attend_rows(q, kr, vr, 0.25)
        cuts = np.sort(rng.integers(0, n + 1, size=int(rng.integers(0, 6))))
        edges = [0, *cuts.tolist(), n]
        parts = [O.attend_rows(q, kr[a:b], vr[a:b], 0.25) for a, b in zip(edges[:-1], edges[1:])]
        merged = O.merge([p[0] for p in parts], [p[1] for p in parts], np.stack([p[2] for p in parts]))
        assert np.allclose(merged, o, rtol=1e-12, atol=1e-13), trial


def test_decode_equals_merge_of_int4_and_int8_partials():
    """The KV4-RL reading: partial over P4 (INT4 values) merged with partial over
    P8 (INT8 values) equals the oracle's single pass over all positions."""
    sh, q, k, v, lens = _tiny_inputs([300, 145, 144, 150, 17])
    out = O.decode(sh, q, k, v, lens, 0.125)
    G = sh.Hq // sh.Hkv
    for b in range(sh.B):
        L = int(lens[b])
        p8 = [p for p in range(L) if p < 16 or p >= L - 128]
        p4 = [p for p in range(L) if p not in p8]
        for h in range(sh.Hkv):
            kh, vh = O.dequant_rows(sh, k, v, lens, b, h)
            for g in range(G):
                qd = np.array([O.bf16_to_float(x) for x in q[b, h * G + g]])
                parts = [O.attend_rows(qd, kh[idx], vh[idx], 0.125) for idx in (p4, p8)]
                merged = O.merge([p[0] for p in parts], [p[1] for p in parts],
                                 np.stack([p[2] for p in parts]))
                assert np.allclose(merged, out[b, h * G + g], rtol=1e-12, atol=1e-13)


def test_short_context_is_entirely_int8():
    sh, q, k, v, lens = _tiny_inputs([144, 37, 1])
    for b in range(sh.B):
        kh, vh = O.dequant_rows(sh, k, v, lens, b, 1)
        for p in range(int(lens[b])):
            sc, codes, _ = O.quant_int8(k[b, p, 1])
            assert np.array_equal(kh[p], codes * O.fp16_to_float(sc))
    # one more position makes position 16 leave the protected set (INT4 values)
    sh, q, k, v, lens = _tiny_inputs([145])
    kh, _ = O.dequant_rows(sh, k, v, lens, 0, 0)
    sc, codes, _ = O.quant_int4(k[0, 16, 0, :32])
    assert np.array_equal(kh[16, :32], codes * O.fp16_to_float(sc))


def test_closed_forms():
    D = 8
    rng = np.random.default_rng(5)
    vr = rng.standard_normal((6, D))
    # equal scores -> mean of V
    kr = np.tile(rng.standard_normal(D), (6, 1))
    _, _, o = O.attend_rows(rng.standard_normal(D), kr, vr, 0.5)
    assert np.allclose(o, vr.mean(axis=0), rtol=1e-14, atol=1e-15)
    # zero query -> mean of V for any keys
    _, l, o = O.attend_rows(np.zeros(D), rng.standard_normal((6, D)), vr, 0.5)
    assert l == 6.0 and np.allclose(o, vr.mean(axis=0), rtol=1e-14, atol=1e-15)
    # one dominant key (gap > 700 in the exponent) -> that row of V
    q = np.zeros(D)
    q[0] = 1.0
    kr = np.zeros((6, D))
    kr[3, 0] = 3000.0
    _, _, o = O.attend_rows(q, kr, vr, 0.25)
    assert np.array_equal(o, vr[3])
    # two keys with score gap delta: o = (v1 + e^-delta v2) / (1 + e^-delta)
    kr = np.zeros((2, D))
    kr[0, 0], kr[1, 0] = 2.0, 0.5
    delta = 0.25 * 1.5
    _, _, o = O.attend_rows(q, kr, vr[:2], 0.25)
    want = (vr[0] + math.exp(-delta) * vr[1]) / (1 + math.exp(-delta))
    assert np.allclose(o, want, rtol=1e-14, atol=1e-15)
    # empty set -> (-inf, 0, 0)
    m, l, o = O.attend_rows(q, np.zeros((0, D)), np.zeros((0, D)), 1.0)
    assert m == -math.inf and l == 0.0 and not o.any()
    assert not O.merge([-math.inf], [0.0], np.zeros((1, D))).any()


def test_gqa_head_mapping_and_bf16_mode():
    """Query head hq reads KV head hq // G: compare each head with a one-head
    problem holding only that KV head."""
    sh, q, k, v, lens = _tiny_inputs([60, 9], Hq=6, Hkv=3, D=32)
    out = O.decode(sh, q, k, v, lens, 0.3, mode=1)
    for hq in range(6):
        h = hq // 2
        sh1 = O.shape(sh.B, 1, 1, 32, 16, 128)
        out1 = O.decode(sh1, q[:, hq: hq + 1], k[:, :, h: h + 1], v[:, :, h: h + 1], lens, 0.3, mode=1)
        assert np.array_equal(out1[:, 0], out[:, hq])
    # mode 1 of a single position returns that V exactly
    sh1 = O.shape(1, 1, 1, 32, 16, 128)
    o1 = O.decode(sh1, q[:1, :1], k[:1, :1, :1], v[:1, :1, :1], np.array([1], np.int32), 0.3, mode=1)
    assert np.array_equal(o1[0, 0], [O.bf16_to_float(x) for x in v[0, 0, 0]])


def test_mask_full_and_empty_and_subset():
    sh, q, k, v, lens = _tiny_inputs([300, 40])
    base = O.decode(sh, q, k, v, lens, 0.125)
    full = np.full((sh.B, sh.Hkv, 10), 0xFFFFFFFF, np.uint32)
    assert np.array_equal(O.decode(sh, q, k, v, lens, 0.125, mask=full), base)
    empty = np.zeros_like(full)
    assert not O.decode(sh, q, k, v, lens, 0.125, mask=empty).any()
    rng = np.random.default_rng(1)
    sub = rng.integers(0, 2 ** 32, size=full.shape, dtype=np.uint64).astype(np.uint32)
    out = O.decode(sh, q, k, v, lens, 0.125, mask=sub)
    G = sh.Hq // sh.Hkv
    for b in range(sh.B):
        for h in range(sh.Hkv):
            keep = [p for p in range(int(lens[b])) if (sub[b, h, p // 32] >> (p % 32)) & 1]
            kh, vh = O.dequant_rows(sh, k, v, lens, b, h)
            for g in range(G):
                qd = np.array([O.bf16_to_float(x) for x in q[b, h * G + g]])
                _, _, o = O.attend_rows(qd, kh[keep], vh[keep], 0.125)
                assert np.allclose(o, out[b, h * G + g], rtol=1e-12, atol=1e-13)


def test_protection_reduces_error_against_bf16():
    """Fidelity proxy (reported, not a page-fixed number): INT8 protection of
    sink + recent lowers the error against unquantised attention."""
    wl = synth.workload("tiny")
    k, v, off = synth.gen_kv(wl)
    q = synth.bf16_bits(synth.gen_q(wl))
    kb = synth.bf16_bits(synth.pad_batch(k, off, range(wl.B)))
    vb = synth.bf16_bits(synth.pad_batch(v, off, range(wl.B)))
    ref = O.decode(O.shape(2, 4, 2, 64, 16, 128), q, kb, vb, wl.lens, 0.125, mode=1)
    prot = O.decode(O.shape(2, 4, 2, 64, 16, 128), q, kb, vb, wl.lens, 0.125, mode=0)
    pure = O.decode(O.shape(2, 4, 2, 64, 0, 0), q, kb, vb, wl.lens, 0.125, mode=0)
    assert np.abs(prot - ref).max() < np.abs(pure - ref).max()
