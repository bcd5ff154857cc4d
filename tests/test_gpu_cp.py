"""Context-parallel decode through the C ABI: each call attends one page-range
shard of every sequence (kv4_decode_partials), and the exact merge of the
shards' partials (kv4_merge_partials) is compared with the fp64 oracle.

On one GPU the shards run one after another on the same cache; on several
GPUs each rank runs its own shard and the partials are all-gathered first
(compressed_kv_cache_kv4_b200.cp; the exchange itself is covered on CPU in
test_multi_rank_cpu.py).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import compressed_kv_cache_kv4_b200 as K
from compressed_kv_cache_kv4_b200 import cp, synth

from helpers import Case, assert_close, assert_bf16_output
from test_gpu_parity import small_wl

pytestmark = pytest.mark.gpu

LOG2E = 1.0 / math.log(2.0)


def _partials(c, pb, pe, int8_rank):
    wl = c.wl
    n = pb.shape[0]
    parts = torch.empty((n, wl.B, wl.Hq, wl.D + 4), dtype=torch.float32, device="cuda")
    ws = c.cache.workspace(wl.B, wl.Hq)
    q = c.q.to("cuda")
    for r in range(n):
        K.kv4_decode_partials(c.cache.handle, q, c.lens, c.pt, wl.softmax_scale, ws, parts[r],
                              torch.as_tensor(pb[r], device="cuda"), torch.as_tensor(pe[r], device="cuda"),
                              with_int8=(r == int8_rank))
    return parts


@pytest.mark.parametrize("n", [1, 2, 3, 5])
def test_shards_merge_to_oracle(n):
    wl = small_wl([5000, 3001, 700, 100, 145, 161], seed=51)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    pb, pe = cp.shard_pages(wl.lens, n, wl.sink, wl.recent)
    parts = _partials(c, pb, pe, n - 1)
    out32 = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32, device="cuda")
    out16 = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    K.kv4_merge_partials(parts, out32)
    K.kv4_merge_partials(parts, out16)
    assert c.cache.get_error()[0] == K.KV4_OK
    ref = c.oracle_decode()
    assert_close(out32.cpu().numpy(), ref, what="%d shards" % n)
    assert_bf16_output(out16, out32, ref)
    # the same attention as the single call
    assert_close(out32.cpu().numpy(), c.decode(out_fp32=True).cpu().numpy(), what="vs one call")


def test_shard_partial_matches_oracle_rows():
    """One middle shard, INT4 positions only: its (m, l, o) against the oracle's
    softmax partial over the same dequantised rows."""
    wl = small_wl([3001, 2049], seed=52, Hq=8, Hkv=2)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    pb, pe = cp.shard_pages(wl.lens, 3, wl.sink, wl.recent)
    parts = _partials(c, pb[1:2], pe[1:2], -1)[0].cpu().numpy()
    sh = c.shape()
    kb = synth.bf16_bits(synth.pad_batch(c.k, c.off, range(wl.B)))
    vb = synth.bf16_bits(synth.pad_batch(c.v, c.off, range(wl.B)))
    q = c.q.float().numpy().astype(np.float64)
    G = wl.Hq // wl.Hkv
    for b in range(wl.B):
        L = int(wl.lens[b])
        pos = np.arange(int(pb[1, b]) * 16, int(pe[1, b]) * 16)
        pos = pos[(pos >= wl.sink) & (pos < L - wl.recent)]
        assert pos.size > 0
        for h in range(wl.Hkv):
            kh, vh = O.dequant_rows(sh, kb, vb, wl.lens, b, h)
            for g in range(G):
                hq = h * G + g
                m, l, o = O.attend_rows(q[b, hq], kh[pos], vh[pos], wl.softmax_scale)
                got = parts[b, hq]
                assert abs(got[0] - m * LOG2E) <= 1e-4 * max(1.0, abs(m * LOG2E)), (b, hq, got[0], m * LOG2E)
                assert abs(got[1] - l) <= 1e-4 * l, (b, hq, got[1], l)
                assert np.abs(got[4:] - o).max() <= 2e-3, (b, hq)


def test_empty_and_int8_only_shards():
    wl = small_wl([2000, 500], seed=53, Hq=8, Hkv=2)
    c = Case(wl)
    c.make_cache()
    c.append_all()
    z = np.zeros((1, wl.B), np.int32)
    empty = _partials(c, z, z, -1)[0].cpu().numpy()
    assert np.all(np.isneginf(empty[..., 0])) and np.all(empty[..., 1] == 0) and np.all(empty[..., 4:] == 0)
    # INT8 region alone + all INT4 pages in a second shard = the whole attention
    first, end = cp.int4_pages(wl.lens, wl.sink, wl.recent)
    pb = np.stack([z[0], first.astype(np.int32)])
    pe = np.stack([z[0], end.astype(np.int32)])
    parts = _partials(c, pb, pe, 0)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32, device="cuda")
    K.kv4_merge_partials(parts, out)
    assert_close(out.cpu().numpy(), c.oracle_decode(), what="int8 shard + int4 shard")
