"""GPU parity of smd_masked_attn (learner-side attention under the shadow
mask) against the fp64 oracle, through the C ABI.

Small cases: every output element against kv4o_masked_attn, for D 64/128, GQA
groups 1/2/4, dense causal, recorded-eviction masks, very sparse masks (whole
64-key blocks skipped), empty rows and ragged lengths. Full size (the learner
workload: 4 sequences of 8192 positions, 32/8 heads, D = 128): sampled rows
against the rollout's decode-step attention under the same mask row, which the
oracle pins equal to the learner's row. Tolerance as for decode (helpers.py):
fp32 output max-abs 2e-3 and relative L2 5e-3; the bf16 output is the
round-to-nearest-even bf16 of the fp32 output.
"""
import numpy as np
import pytest
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth
import compressed_kv_cache_kv4_b200 as K

from helpers import assert_close, assert_bf16_output

pytestmark = pytest.mark.gpu


def _case(B, T, Hq, Hkv, D, seed):
    wl = synth.workload("learner", B=B, T=T)
    wl.Hq, wl.Hkv, wl.D, wl.seed = Hq, Hkv, D, seed
    wl.softmax_scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    q, k, v = synth.gen_learner_qkv(wl, T)
    return wl, q, k, v


def _run(q, k, v, tau, lens=None, mask=None, fp32=True):
    B, T, Hq, D = q.shape
    out = torch.empty((B, T, Hq, D), dtype=torch.float32 if fp32 else torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.smd_masked_attn(q.cuda(), k.cuda(), v.cuda(), tau, out,
                      seq_lens=None if lens is None else torch.as_tensor(lens, device="cuda"),
                      mask=None if mask is None else mask.cuda(), error_word=err)
    torch.cuda.synchronize()
    return out, int(err.item())


def _oracle(q, k, v, tau, lens=None, mask=None):
    return O.masked_attn(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), tau, lens=lens,
                         mask=None if mask is None else mask.numpy().view(np.uint32))


@pytest.mark.parametrize("B,T,Hq,Hkv,D", [(2, 200, 8, 2, 64), (1, 333, 32, 8, 128), (2, 150, 2, 2, 128),
                                          (1, 257, 4, 2, 64), (3, 64, 4, 1, 128)])
@pytest.mark.parametrize("kind", ["dense", "shadow", "sparse"])
def test_matches_oracle(B, T, Hq, Hkv, D, kind):
    wl, q, k, v = _case(B, T, Hq, Hkv, D, seed=T + D + Hq)
    tau = wl.softmax_scale
    mask = None
    if kind == "shadow":
        mask = synth.gen_shadow_mask(wl, T)
    elif kind == "sparse":
        # a few keys only: most 64-key blocks of most CTAs are empty
        mask = synth.gen_shadow_mask(wl, T, sink=0, recent=0)
        rng = np.random.default_rng(T)
        mm = mask.numpy().view(np.uint32)
        mm &= rng.integers(0, 2 ** 32, size=mm.shape, dtype=np.uint64).astype(np.uint32) & np.uint32(0x01010101)
        mm[:, :, 3] = 0                                           # an empty row
        mask = torch.from_numpy(mm.view(np.int32).copy())
    lens = np.array([T, max(T - 37, 0), 1][:B], np.int32) if B > 1 else None
    ref = _oracle(q, k, v, tau, lens=lens, mask=mask)
    out32, err = _run(q, k, v, tau, lens=lens, mask=mask)
    assert err == 0
    assert_close(out32.cpu().numpy(), ref, what="%s B=%d T=%d G=%d D=%d" % (kind, B, T, Hq // Hkv, D))
    out16, _ = _run(q, k, v, tau, lens=lens, mask=mask, fp32=False)
    assert_bf16_output(out16, out32, ref)


def test_length_outside_range_is_reported_and_clamped():
    wl, q, k, v = _case(2, 96, 4, 2, 64, seed=9)
    lens = np.array([200, -3], np.int32)
    out, err = _run(q, k, v, wl.softmax_scale, lens=lens)
    assert err == 1 << K.KV4_ERR_CAPACITY
    ref = _oracle(q, k, v, wl.softmax_scale, lens=np.array([96, 0], np.int32))
    assert_close(out.cpu().numpy(), ref, what="clamped lengths")


def test_learner_full_size_rows_equal_rollout_decode():
    """The learner workload at full size; sampled query rows against the
    oracle's decode-step attention of the rollout at length t + 1 under mask
    row t (over bf16 values)."""
    wl = synth.workload("learner")
    T = int(wl.lens.max())
    q, k, v = synth.gen_learner_qkv(wl, T, device="cuda")
    mask = synth.gen_shadow_mask(wl, T, device="cuda")
    out = torch.empty((wl.B, T, wl.Hq, wl.D), dtype=torch.float32, device="cuda")
    K.smd_masked_attn(q, k, v, wl.softmax_scale, out, mask=mask)
    torch.cuda.synchronize()
    rows = [0, 1, 15, 16, 63, 64, 127, 128, 1000, 4095, 4096, 6001, T - 2, T - 1]
    sh = O.shape(wl.B, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)
    kc, vc, qc = synth.bf16_bits(k), synth.bf16_bits(v), synth.bf16_bits(q)
    mc = mask[:, :, rows].cpu().numpy().view(np.uint32)
    got = out[:, rows].cpu().numpy()
    for i, t in enumerate(rows):
        L = t + 1
        ref = O.decode(sh, np.ascontiguousarray(qc[:, t]), np.ascontiguousarray(kc[:, :L]),
                       np.ascontiguousarray(vc[:, :L]), np.full(wl.B, L, np.int32), wl.softmax_scale,
                       mask=np.ascontiguousarray(mc[:, :, i]), mode=1)
        assert_close(got[:, i], ref, what="row %d" % t)
    del q, k, v, mask, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("D,Hq,Hkv", [(64, 4, 2), (128, 8, 2)])
@pytest.mark.parametrize("div", [16.0, 160.0])
def test_growing_scores_rescale_the_accumulator(D, Hq, Hkv, div):
    """K rows scaled up along the sequence: a row's running maximum grows by
    about 60 (div 16) or 5-12 (div 160) base-2 units per 64-key block, so the
    accumulator is rescaled in place, every block or only some; results still
    match the oracle."""
    T = 640
    wl, q, k, v = _case(2, T, Hq, Hkv, D, seed=31 + D)
    gain = (1.0 + torch.arange(T, dtype=torch.float32) / div)[None, :, None, None]
    k = (k.float() * gain).to(torch.bfloat16)
    q = (q.float().abs()).to(torch.bfloat16)          # positive queries ...
    k = k.float().abs().to(torch.bfloat16)            # ... and keys: scores grow with the key position
    mask = synth.gen_shadow_mask(wl, T)
    for m in (None, mask):
        ref = _oracle(q, k, v, wl.softmax_scale, mask=m)
        out, err = _run(q, k, v, wl.softmax_scale, mask=m)
        assert err == 0
        assert_close(out.cpu().numpy(), ref, what="growing scores D=%d" % D)
