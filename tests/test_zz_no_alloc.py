"""kv4_decode_attn_noalloc: the decode step with the library's fixed scratch
instead of a caller workspace, checked against kv4_decode_attn.

Collected last on purpose (file name), so it also runs after every other GPU
test has used the library in the same process.
"""
import os
import re

import numpy as np
import pytest
import torch

import compressed_kv_cache_kv4_b200 as K
from compressed_kv_cache_kv4_b200 import synth

from helpers import Case


def _case():
    # mixed lengths: empty-INT4 short sequences, page-boundary lengths, a ragged tail
    wl = synth.workload("qwen8b", B=9)
    wl.lens = np.array([1, 15, 144, 145, 300, 1000, 1777, 2048, 3001], np.int32)
    wl.B = 9
    c = Case(wl)
    c.make_cache()
    c.append_all()
    return c


def test_scratch_size_matches_header():
    src = open(os.path.join(os.path.dirname(__file__), "..", "include", "kv4.h")).read()
    m = re.search(r"#define\s+KV4_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "KV4_NOALLOC_SCRATCH_BYTES not found in kv4.h"
    assert (int(m.group(1)) << int(m.group(2))) == K.NOALLOC_SCRATCH_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("out_fp32", [True, False])
def test_noalloc_matches_workspace_call(out_fp32):
    c = _case()
    wl = c.wl
    dt = torch.float32 if out_fp32 else torch.bfloat16
    g = torch.Generator(device="cpu")
    g.manual_seed(4242)
    for call in range(2):   # two consecutive calls with different queries
        q = (c.q if call == 0 else torch.randn(c.q.shape, generator=g).to(torch.bfloat16)).to("cuda")
        want = c.cache.decode(q, c.lens, c.pt, wl.softmax_scale, out_fp32=out_fp32)
        got = torch.full((wl.B, wl.Hq, wl.D), float("nan"), dtype=dt, device="cuda")
        K.kv4_decode_attn_noalloc(c.cache.handle, q, c.lens, c.pt, wl.softmax_scale, got)
        torch.cuda.synchronize()
        st, bits = c.cache.get_error()
        assert st == K.KV4_OK and bits == 0
        assert torch.isfinite(got.float()).all()
        # same kernels, same worker count, same data: the outputs agree bit for bit
        assert torch.equal(got.view(torch.int32 if out_fp32 else torch.int16),
                           want.view(torch.int32 if out_fp32 else torch.int16)), "call %d" % call


@pytest.mark.gpu
def test_noalloc_rejects_oversized_scratch():
    c = _case()
    wl = c.wl
    # enough workers that the partial slots alone exceed the fixed area
    nw = K.NOALLOC_SCRATCH_BYTES // 1024
    assert K.kv4_workspace_bytes(c.cache.handle, wl.B, wl.Hq, nw) > K.NOALLOC_SCRATCH_BYTES
    out = torch.zeros((wl.B, wl.Hq, wl.D), dtype=torch.float32, device="cuda")
    with pytest.raises(K.Kv4Error) as ei:
        K.kv4_decode_attn_noalloc(c.cache.handle, c.q.to("cuda"), c.lens, c.pt, wl.softmax_scale, out,
                                  num_workers=nw)
    assert ei.value.status == K.KV4_ERR_CAPACITY
    assert "fixed area" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0   # nothing was enqueued
