"""Pins for the oracle's byte writer (page pool and INT8 side cache).

The layout is this build's own definition (the pages only say "paged INT4"
with 16-token pages and an INT8 side cache for 16 sink + 128 recent
positions). These tests check the writer against (a) hand-computed offsets of
the stated layout, (b) a bijection argument, and (c) a decode of the bytes
through the array view the GPU kernels use (32-bit words carrying the
register fragments), which is a different statement of the same layout.
"""
import numpy as np
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth


def test_hand_computed_offsets():
    # D = 128: head block = 2304 bytes = K codes 1024 | V codes 1024 | K scales 128 | V scales 128
    assert O.page_head_bytes(128) == 2304 and O.page_head_bytes(64) == 1152
    # K, slot 5, dim 37: group i=1, chunk t=0, element k=5 -> byte 5*64 + 0*16 + 4*1 + 2, high nibble
    assert O.k_code_byte(128, 5, 37) == (326, 1)
    # K, slot 15, dim 127: i=3, t=3, k=7 -> 15*64 + 3*16 + 12 + 3 = 1023, high nibble
    assert O.k_code_byte(128, 15, 127) == (1023, 1)
    # V, slot 5, dim 37: m=2, g=5, upper-8 flag 0; t=2, odd slot, first half -> lane 22 at
    # position 8*2 + (5 xor 4) = 17, word 17*4 + 2 = 70 -> byte 1024 + 280 + 2 = 1306, low nibble
    assert O.v_code_byte(128, 5, 37) == (1306, 0)
    # V, slot 9, dim 120: m=7 (second 512-byte half), g=0, upper-8 flag 1; t=0, odd, r8=1
    # -> position 0, word 128 + 0 + 3 = 131 -> byte 1024 + 524 + 2 + 1 = 1551, high nibble
    assert O.v_code_byte(128, 9, 120) == (1551, 1)
    # V, slot 14, dim 3: m=0, g=3, t=3, even slot, r8=1 -> position 24 + (3 xor 6) = 29,
    # word 116 -> byte 1024 + 464 + 1 = 1489, low nibble
    assert O.v_code_byte(128, 14, 3) == (1489, 0)
    # scales: slot r, group i at 2*(4r + i) after the codes
    assert O.k_scale_byte(128, 3, 2) == 2048 + 28
    assert O.v_scale_byte(128, 3, 2) == 2176 + 28
    # D = 64: rows of 32 bytes, chunks of 8 bytes
    assert O.k_code_byte(64, 1, 40) == (32 + 8 + 4 + 0, 0)
    # INT8 side block: 1 sink page + 8 ring pages of 2*(16*D + 32) bytes
    assert O.side_head_bytes(128, 16, 128) == 9 * 4160 == 37440
    assert O.side_head_bytes(64, 16, 128) == 9 * 2112 and O.side_page_bytes(128) == 4160
    assert O.side_head_bytes(128, 0, 0) == 0 and O.side_pages(0, 128) == 8
    # side K, row 21 (ring page 1, row 5), element 70: t = 2, j = 1, e = 2; lane 22,
    # word 1 -> 4160 + 0*512 + 22*16 + 4 + 2
    assert O.side_k_byte(128, 21, 70) == 4160 + 352 + 6
    # side V, row 9, element 37: m = 2, g = 5, t = 0, odd row, r/8 = 1 -> lane 20,
    # word 5 -> 2112 (after K codes and both scale arrays) + 512 + 320 + 4 + 2 + 0
    assert O.side_v_byte(128, 9, 37) == 2112 + 512 + 320 + 4 + 2
    assert O.side_ks_byte(128, 17) == 4160 + 2048 + 2
    assert O.side_vs_byte(128, 17) == 4160 + 2048 + 32 + 2


def test_side_layout_is_a_bijection():
    for D in (64, 128):
        pb = O.side_page_bytes(D)
        seen = set()
        for row in range(16):
            for d in range(D):
                seen.add(O.side_k_byte(D, row, d))
                seen.add(O.side_v_byte(D, row, d))
            seen.add(O.side_ks_byte(D, row))
            seen.add(O.side_ks_byte(D, row) + 1)
            seen.add(O.side_vs_byte(D, row))
            seen.add(O.side_vs_byte(D, row) + 1)
        assert seen == set(range(pb))


def test_v_rows_of_a_group_are_contiguous():
    """The V codes of the rows {2a, 2a+1, 2a+8, 2a+9} fill 128 contiguous bytes of
    each 512-byte block of the V area, so they can be read without the other rows."""
    for D in (64, 128):
        for a in range(4):
            got = {O.v_code_byte(D, r, d)[0] for r in (2 * a, 2 * a + 1, 2 * a + 8, 2 * a + 9) for d in range(D)}
            want = {8 * D + 512 * blk + 128 * a + k for blk in range(D // 64) for k in range(128)}
            assert got == want, (D, a)


def test_layout_is_a_bijection():
    for D in (64, 128):
        seen = set()
        for r in range(16):
            for d in range(D):
                for f in (O.k_code_byte, O.v_code_byte):
                    seen.add(f(D, r, d))
        assert seen == {(b, n) for b in range(16 * D) for n in (0, 1)}
        sc = {f(D, r, i) for r in range(16) for i in range(D // 32) for f in (O.k_scale_byte, O.v_scale_byte)}
        assert sc == set(range(16 * D, 18 * D, 2))


def _nibbles(words):
    w = words.astype(np.uint32)
    out = np.stack([(w >> (4 * k)) & 0xF for k in range(8)], axis=-1)
    return np.where(out >= 8, out.astype(np.int32) - 16, out.astype(np.int32))


def _decode_block_via_fragments(blk, D):
    """Read a head block the way the tensor-core fragments read it."""
    words = blk[: 16 * D].view(np.uint32)
    # K: [row 16][chunk t 4][word i D/32] -> nibble k is dim 32i + 8t + k
    kw = words[: 2 * D].reshape(16, 4, D // 32)
    kn = _nibbles(kw)                               # [16][t][i][k]
    K = kn.transpose(0, 2, 1, 3).reshape(16, D)     # [row][i][t][k] -> dim
    # V: word (lane, m) at (m//4)*128 + P*4 + m%4, lane = 4g + t stored at
    # position P = 8t + (g xor 2t); nibbles
    # n0 (2t, 16m+g) n1 (2t, 16m+g+8) n2 (2t+8, g) n3 (2t+8, g+8) n4 (2t+1, g)
    # n5 (2t+1, g+8) n6 (2t+9, g) n7 (2t+9, g+8) -- the A fragment of V^T
    vw = words[2 * D: 4 * D]
    V = np.zeros((16, D), np.int32)
    for lane in range(32):
        g, t = lane // 4, lane % 4
        for m in range(D // 16):
            n = _nibbles(vw[(m // 4) * 128 + (8 * t + (g ^ (2 * t))) * 4 + m % 4])
            for j, (tok, dd) in enumerate([(2 * t, g), (2 * t, g + 8), (2 * t + 8, g), (2 * t + 8, g + 8),
                                           (2 * t + 1, g), (2 * t + 1, g + 8), (2 * t + 9, g), (2 * t + 9, g + 8)]):
                V[tok, 16 * m + dd] = n[j]
    ks = blk[16 * D: 17 * D].view(np.uint16).reshape(16, D // 32)
    vs = blk[17 * D: 18 * D].view(np.uint16).reshape(16, D // 32)
    return K, V, ks, vs


def test_writer_matches_quantiser_through_fragment_view():
    wl = synth.workload("tiny")
    k, v, off = synth.gen_kv(wl)
    pt, npages = synth.gen_page_table(wl)
    sh = O.shape(wl.B, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)
    kb = synth.bf16_bits(synth.pad_batch(k, off, range(wl.B)))
    vb = synth.bf16_bits(synth.pad_batch(v, off, range(wl.B)))
    pool, side, flags = O.write_cache(sh, kb, vb, wl.lens, pt, npages)
    assert flags == 0
    D, Hkv = wl.D, wl.Hkv
    hb = O.page_head_bytes(D)
    for b in range(wl.B):
        L = int(wl.lens[b])
        for p in range(0, L, 7):
            page, r = pt[b, p // 16], p % 16
            for h in range(Hkv):
                blk = pool[(page * Hkv + h) * hb: (page * Hkv + h + 1) * hb]
                K, V, ks, vs = _decode_block_via_fragments(blk, D)
                for grp in range(D // 32):
                    sc, codes, _ = O.quant_int4(kb[b, p, h, 32 * grp: 32 * grp + 32])
                    assert ks[r, grp] == sc and np.array_equal(K[r, 32 * grp: 32 * grp + 32], codes)
                    sc, codes, _ = O.quant_int4(vb[b, p, h, 32 * grp: 32 * grp + 32])
                    assert vs[r, grp] == sc and np.array_equal(V[r, 32 * grp: 32 * grp + 32], codes)


def _decode_side_page_via_fragments(page, D):
    """Read one INT8 side page the way the fp16 tensor-core fragments read it."""
    w = page.view(np.uint32)
    nk = 4 * D                                   # K codes: 16*D bytes = 4*D words
    K = np.zeros((16, D), np.int32)
    V = np.zeros((16, D), np.int32)
    kw = w[: nk].reshape(D // 32, 32, 4)          # [chunk][lane][word in chunk]
    vw = w[nk + 16: 2 * nk + 16].reshape(D // 32, 32, 4)
    sb = lambda x, k: ((int(x) >> (8 * k)) & 0xFF) - (256 if (int(x) >> (8 * k)) & 0x80 else 0)
    for lane in range(32):
        g, t = lane // 4, lane % 4
        for wi in range(D // 8):
            # K: words 0..D/16-1 are row g, the rest row g+8; word j holds elements
            # t*D/4 + 4j + (0..3) in bytes 0..3
            x = kw[wi // 4, lane, wi % 4]
            row = g + 8 * (wi // (D // 16))
            j = wi % (D // 16)
            for e in range(4):
                K[row, t * (D // 4) + 4 * j + e] = sb(x, e)
            # V: word 2m + r8 holds (slot 2t+8r8, dim 16m+g), (2t+8r8, 16m+g+8),
            # (2t+8r8+1, 16m+g), (2t+8r8+1, 16m+g+8) in bytes 0..3
            y = vw[wi // 4, lane, wi % 4]
            m, r8 = wi // 2, wi % 2
            for e, (tok, dd) in enumerate([(2 * t + 8 * r8, g), (2 * t + 8 * r8, g + 8),
                                           (2 * t + 8 * r8 + 1, g), (2 * t + 8 * r8 + 1, g + 8)]):
                V[tok, 16 * m + dd] = sb(y, e)
    ks = page[16 * D: 16 * D + 32].view(np.uint16)
    vs = page[16 * D + 32: 16 * D + 64].view(np.uint16)
    return K, V, ks, vs


def test_side_cache_sink_and_ring():
    wl = synth.workload("tiny")
    k, v, off = synth.gen_kv(wl)
    pt, npages = synth.gen_page_table(wl)
    sh = O.shape(wl.B, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)
    kb = synth.bf16_bits(synth.pad_batch(k, off, range(wl.B)))
    vb = synth.bf16_bits(synth.pad_batch(v, off, range(wl.B)))
    _, side, _ = O.write_cache(sh, kb, vb, wl.lens, pt, npages, fill=0x5A)
    S, R, D = wl.sink, wl.recent, wl.D
    stride = O.side_head_bytes(D, S, R)
    pb = O.side_page_bytes(D)
    for b in range(wl.B):
        L = int(wl.lens[b])
        for h in range(wl.Hkv):
            blk = side[(b * wl.Hkv + h) * stride: (b * wl.Hkv + h + 1) * stride]
            pages = [_decode_side_page_via_fragments(blk[i * pb: (i + 1) * pb], D) for i in range(stride // pb)]
            # sink rows (page 0) hold positions 0..15
            for p in range(min(S, L)):
                sc, codes, _ = O.quant_int8(kb[b, p, h])
                assert pages[0][2][p] == sc and np.array_equal(pages[0][0][p], codes)
            # ring slot p % R (page 1 + slot/16) holds the latest position with that residue
            for p in range(max(0, L - R), L):
                slot = p % R
                sc, codes, _ = O.quant_int8(vb[b, p, h])
                pg = pages[1 + slot // 16]
                assert pg[3][slot % 16] == sc and np.array_equal(pg[1][slot % 16], codes)
            # ring slots never written keep the fill byte (sequence of 37 tokens)
            if L < R:
                for slot in range(L, R):
                    assert blk[O.side_k_byte(D, 16 + slot, 0)] == 0x5A
