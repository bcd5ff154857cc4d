"""Parity at the full workload sizes, in the launch configuration the benchmark
times (default worker count, bf16 output, whole batch in one call), on sampled
outputs the oracle computes sequence by sequence.

- qwen8b: B = 64, L ~ U[1024, 8192].
- async: B = 256, log-normal lengths up to 32768, 64 steps of
  one-token append + decode; checked at steps 0, 31 and 63.
- long: B = 4, L = 131072; the split-K partials of each sequence
  against the single-pass oracle.
- evict: B = 64, L = 16384; top-k masks bit-exact at every budget,
  masked decode at 10% and 50% on sampled sequences, 100% = unmasked bitwise.
- long, context parallel: the same four 128K sequences decoded as four
  page-range shards (kv4_decode_partials, the INT8 region with the last) and
  merged (kv4_merge_partials), against the oracle.
- prefill bytes: the benchmark's prefill of the qwen8b and async prompts in one
  kv4_append; page and side-cache bytes of sampled sequences (the first and the
  last ones of the batch among them, which only later grid-stride passes of the
  page kernel reach) bit-exact against the oracle's writer.
"""
import gc

import numpy as np
import pytest
import torch

import oracle as O
import compressed_kv_cache_kv4_b200 as K
from compressed_kv_cache_kv4_b200 import synth

from helpers import assert_close, assert_bf16_output

pytestmark = pytest.mark.gpu


def _sample(lens, n_random, seed):
    lens = np.asarray(lens)
    rng = np.random.default_rng(seed)
    pick = {int(np.argmin(lens)), int(np.argmax(lens))}
    pick.update(int(x) for x in rng.choice(len(lens), size=n_random, replace=False))
    return sorted(pick)


def _oracle(wl, rows_k, rows_v, q_rows, lens, mask=None):
    """fp64 oracle over the given sequences: rows_k/rows_v lists of [L][Hkv][D] bf16 (CPU)."""
    n = len(rows_k)
    Lmax = max(int(x) for x in lens)
    kb = torch.zeros((n, max(Lmax, 1), wl.Hkv, wl.D), dtype=torch.bfloat16)
    vb = torch.zeros_like(kb)
    for i in range(n):
        kb[i, : rows_k[i].shape[0]] = rows_k[i]
        vb[i, : rows_v[i].shape[0]] = rows_v[i]
    sh = O.shape(n, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)
    return O.decode(sh, synth.bf16_bits(q_rows), synth.bf16_bits(kb), synth.bf16_bits(vb),
                    np.asarray(lens, np.int32), wl.softmax_scale, mask=mask)


def _prefill(wl, lens, cap):
    k, v, off = synth.gen_kv(wl, device="cuda", lens=lens)
    pt, npages = synth.gen_page_table(wl, cap)
    cache = K.KV4Cache(wl.Hkv, wl.D, wl.B, npages, wl.sink, wl.recent)
    ptd = torch.as_tensor(pt, device="cuda")
    cache.append(k, v, torch.as_tensor(off.astype(np.int32), device="cuda"),
                 torch.zeros(wl.B, dtype=torch.int32, device="cuda"), ptd)
    return cache, ptd, k, v, off


def _check(wl, cache, ptd, lens_np, q, seqs, rows_k, rows_v, what):
    lens = torch.as_tensor(np.asarray(lens_np, np.int32), device="cuda")
    out16 = cache.decode(q, lens, ptd, wl.softmax_scale)                 # the benchmark's call
    out32 = cache.decode(q, lens, ptd, wl.softmax_scale, out_fp32=True)
    st, bits = cache.get_error()
    assert st == K.KV4_OK, (what, st, bits)
    ref = _oracle(wl, rows_k, rows_v, q[seqs].cpu(), [int(lens_np[b]) for b in seqs])
    assert_close(out32[seqs].cpu().numpy(), ref, what=what)
    assert_bf16_output(out16[seqs], out32[seqs], ref)


def _cleanup():
    gc.collect()
    torch.cuda.empty_cache()


def test_qwen8b_full_size():
    wl = synth.workload("qwen8b")
    cache, ptd, k, v, off = _prefill(wl, wl.lens, wl.lens)
    q = synth.gen_q(wl, device="cuda")
    seqs = _sample(wl.lens, 4, 21)
    rows_k = [k[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    rows_v = [v[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    _check(wl, cache, ptd, wl.lens, q, seqs, rows_k, rows_v, "qwen8b")
    cache.close()
    del cache, k, v
    _cleanup()


def test_async_full_size_64_steps():
    wl = synth.workload("async")
    steps = 64
    L0 = wl.lens.astype(np.int64)
    lens_pre = np.maximum(L0 - steps, 0).astype(np.int32)
    cache, ptd, k, v, off = _prefill(wl, lens_pre, L0)
    seqs = _sample(L0, 2, 23)
    rows_k = [k[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    rows_v = [v[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    del k, v
    _cleanup()
    for c in range(steps):
        kn, vn = synth.gen_step_kv(wl, c, device="cuda")
        old = torch.as_tensor(lens_pre + c, dtype=torch.int32, device="cuda")
        K.kv4_append(cache.handle, kn.contiguous(), vn.contiguous(), None, old, ptd)
        for i, b in enumerate(seqs):
            rows_k[i] = torch.cat([rows_k[i], kn[b: b + 1].cpu()])
            rows_v[i] = torch.cat([rows_v[i], vn[b: b + 1].cpu()])
        q = synth.gen_q(wl, step=c, device="cuda")
        if c in (0, 31, 63):
            _check(wl, cache, ptd, lens_pre + c + 1, q, seqs, rows_k, rows_v, "async step %d" % c)
        else:
            cache.decode(q, torch.as_tensor(lens_pre + c + 1, dtype=torch.int32, device="cuda"), ptd,
                         wl.softmax_scale)
    cache.close()
    del cache
    _cleanup()


def test_long_context_full_size():
    wl = synth.workload("long")
    cache, ptd, k, v, off = _prefill(wl, wl.lens, wl.lens)
    q = synth.gen_q(wl, device="cuda")
    seqs = list(range(wl.B))
    rows_k = [k[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    rows_v = [v[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    del k, v
    _cleanup()
    _check(wl, cache, ptd, wl.lens, q, seqs, rows_k, rows_v, "long")
    cache.close()
    del cache
    _cleanup()


def test_long_context_parallel_full_size():
    from compressed_kv_cache_kv4_b200 import cp
    wl = synth.workload("long")
    cache, ptd, k, v, off = _prefill(wl, wl.lens, wl.lens)
    q = synth.gen_q(wl, device="cuda")
    seqs = list(range(wl.B))
    rows_k = [k[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    rows_v = [v[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    del k, v
    _cleanup()
    lens = torch.as_tensor(wl.lens, device="cuda")
    n = 4
    pb, pe = cp.shard_pages(wl.lens, n, wl.sink, wl.recent)
    parts = torch.empty((n, wl.B, wl.Hq, wl.D + 4), dtype=torch.float32, device="cuda")
    ws = cache.workspace(wl.B, wl.Hq)
    for r in range(n):
        K.kv4_decode_partials(cache.handle, q, lens, ptd, wl.softmax_scale, ws, parts[r],
                              torch.as_tensor(pb[r], device="cuda"), torch.as_tensor(pe[r], device="cuda"),
                              with_int8=(r == n - 1))
    out32 = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    K.kv4_merge_partials(parts, out32)
    K.kv4_merge_partials(parts, out16)
    st, bits = cache.get_error()
    assert st == K.KV4_OK, (st, bits)
    ref = _oracle(wl, rows_k, rows_v, q.cpu(), [int(x) for x in wl.lens])
    assert_close(out32.cpu().numpy(), ref, what="long, 4 shards")
    assert_bf16_output(out16, out32, ref)
    cache.close()
    del cache
    _cleanup()


def test_evict_full_size():
    wl = synth.workload("evict")
    cache, ptd, k, v, off = _prefill(wl, wl.lens, wl.lens)
    scores = synth.gen_scores(wl, k, off, device="cuda")
    q = synth.gen_q(wl, device="cuda")
    seqs = _sample(wl.lens, 2, 25)
    rows_k = [k[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    rows_v = [v[int(off[b]): int(off[b + 1])].cpu() for b in seqs]
    del k, v
    _cleanup()
    lens = torch.as_tensor(wl.lens, device="cuda")
    L = int(wl.lens.max())
    mstride = (ptd.shape[1] * 16 + 31) // 32
    mask = torch.zeros((wl.B, wl.Hkv, mstride), dtype=torch.int32, device="cuda")
    count = torch.zeros((wl.B, wl.Hkv), dtype=torch.int32, device="cuda")
    sc_np = scores.cpu().numpy()
    unmasked = cache.decode(q, lens, ptd, wl.softmax_scale, out_fp32=True)
    for permille in (100, 300, 500, 900, 1000):
        K.kv_topk_retain(scores, lens, permille, mask, count, max_len=L)
        torch.cuda.synchronize()
        m_ref, c_ref = O.topk(sc_np, wl.lens, permille)
        got = mask.cpu().numpy().view(np.uint32)[:, :, : m_ref.shape[-1]]
        assert np.array_equal(got, m_ref), permille
        assert np.array_equal(count.cpu().numpy(), c_ref), permille
        if permille in (100, 500):
            out32 = cache.decode(q, lens, ptd, wl.softmax_scale, out_fp32=True, retain_mask=mask)
            out16 = cache.decode(q, lens, ptd, wl.softmax_scale, retain_mask=mask)
            ref = _oracle(wl, rows_k, rows_v, q[seqs].cpu(), [int(wl.lens[b]) for b in seqs],
                          mask=np.ascontiguousarray(m_ref[seqs]))
            assert_close(out32[seqs].cpu().numpy(), ref, what="evict %d" % permille)
            assert_bf16_output(out16[seqs], out32[seqs], ref)
            # the gathered path at full size, under the same mask
            g32 = cache.decode_masked(q, lens, ptd, wl.softmax_scale, mask, L * permille // 1000, out_fp32=True)
            assert_close(g32[seqs].cpu().numpy(), ref, what="evict gathered %d" % permille)
            assert_close(g32.cpu().numpy(), out32.cpu().numpy(), what="evict gathered vs page path %d" % permille)
        if permille == 1000:
            full = cache.decode(q, lens, ptd, wl.softmax_scale, out_fp32=True, retain_mask=mask)
            assert torch.equal(full, unmasked)
    st, bits = cache.get_error()
    assert st == K.KV4_OK, (st, bits)
    cache.close()
    del cache
    _cleanup()


@pytest.mark.parametrize("name", ["qwen8b", "async"])
def test_prefill_bytes_full_size(name):
    wl = synth.workload(name)
    L0 = wl.lens.astype(np.int64)
    lens_pre = np.maximum(L0 - 64, 0).astype(np.int32)        # the benchmark's prefill lengths
    k, v, off = synth.gen_kv(wl, device="cuda", lens=lens_pre)
    pt, npages = synth.gen_page_table(wl, L0 + 64)
    cache = K.KV4Cache(wl.Hkv, wl.D, wl.B, npages, wl.sink, wl.recent, fill=0xA5)
    ptd = torch.as_tensor(pt, device="cuda")
    cache.append(k, v, torch.as_tensor(off.astype(np.int32), device="cuda"),
                 torch.zeros(wl.B, dtype=torch.int32, device="cuda"), ptd)
    torch.cuda.synchronize()
    st, bits = cache.get_error()
    assert st == K.KV4_OK, (st, bits)
    seqs = sorted(set(_sample(lens_pre, 3, 27)) | {0, 1, wl.B // 2, wl.B - 2, wl.B - 1})
    n = len(seqs)
    lens_s = lens_pre[seqs].astype(np.int32)
    Lmax = int(lens_s.max())
    kb = torch.zeros((n, Lmax, wl.Hkv, wl.D), dtype=torch.bfloat16)
    vb = torch.zeros_like(kb)
    for i, b in enumerate(seqs):
        kb[i, : lens_s[i]] = k[int(off[b]): int(off[b + 1])].cpu()
        vb[i, : lens_s[i]] = v[int(off[b]): int(off[b + 1])].cpu()
    del k, v
    _cleanup()
    # the sampled sequences' pages renumbered into a compact pool for the oracle
    npg = [(int(L) + 15) // 16 for L in lens_s]
    pt_s = np.full((n, max(npg)), -1, np.int32)
    nxt = 0
    for i in range(n):
        pt_s[i, : npg[i]] = np.arange(nxt, nxt + npg[i])
        nxt += npg[i]
    sh = O.shape(n, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)
    pool_ref, side_ref, flags = O.write_cache(sh, synth.bf16_bits(kb), synth.bf16_bits(vb), lens_s, pt_s,
                                              max(nxt, 1), fill=0xA5)
    assert flags == 0
    page_bytes = wl.Hkv * 18 * wl.D
    side_blk = cache.side.numel() // wl.B
    pool = cache.pool.view(npages, page_bytes)
    side = cache.side.view(wl.B, side_blk)
    for i, b in enumerate(seqs):
        ids = torch.as_tensor(pt[b, : npg[i]].astype(np.int64), device="cuda")
        got = pool.index_select(0, ids).cpu().numpy()
        want = pool_ref.reshape(-1, page_bytes)[pt_s[i, : npg[i]]]
        assert np.array_equal(got, want), "%s: pages of sequence %d differ" % (name, b)
        assert np.array_equal(side[b].cpu().numpy(), side_ref.reshape(n, side_blk)[i]), \
            "%s: side cache of sequence %d differs" % (name, b)
    cache.close()
    del cache
    _cleanup()
