"""Pins for the oracle's learner-side attention under the shadow mask.

Shadow Mask Distillation, sec. 1 and Figure 1: the rollout records, for every
generated position, the binary mask of the positions its KV eviction kept; the
learner applies that mask inside its causal attention, so that its policy and
the sparse rollout's coincide. Build readings: row t of the mask belongs to
the query at position t and covers keys p <= t; the learner attends over the
bf16 K and V; an empty row gives 0.

The pins reach the result by other routes: torch float64 softmax on small
cases, closed forms, and the rollout's own decode-step attention (the
oracle's kv4o_decode over bf16 values at length t + 1 under mask row t).
"""
import numpy as np
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth


def _inputs(B, T, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, T, Hq, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, T, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, T, Hkv, D), generator=g).to(torch.bfloat16)
    return q, k, v


def _mask(B, Hkv, T, density, seed):
    rng = np.random.default_rng(seed)
    W = (T + 31) // 32 + 1
    bits = rng.random((B, Hkv, T, T)) < density
    m = np.zeros((B, Hkv, T, W), np.uint32)
    for w in range(W):
        for i in range(32):
            p = 32 * w + i
            if p < T:
                m[..., w] |= bits[..., p].astype(np.uint32) << np.uint32(i)
    return m, bits


def _torch_ref(q, k, v, tau, bits=None, lens=None):
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    qd, kd, vd = q.double(), k.double(), v.double()
    out = torch.zeros((B, T, Hq, D), dtype=torch.float64)
    causal = torch.tril(torch.ones(T, T, dtype=torch.bool))
    for b in range(B):
        L = T if lens is None else int(lens[b])
        for hq in range(Hq):
            h = hq // G
            s = tau * qd[b, :, hq] @ kd[b, :, h].T                     # [T][T]
            allow = causal.clone()
            if bits is not None:
                allow &= torch.as_tensor(bits[b, h])
            allow[:, L:] = False
            s = s.masked_fill(~allow, float("-inf"))
            w = torch.softmax(s, dim=-1)
            w = torch.nan_to_num(w, nan=0.0)                            # empty rows
            o = w @ vd[b, :, h]
            o[L:] = 0.0
            out[b, :, hq] = o
    return out.numpy()


def test_dense_causal_matches_torch():
    q, k, v = _inputs(2, 37, 4, 2, 32, 1)
    got = O.masked_attn(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), 0.25)
    ref = _torch_ref(q, k, v, float(np.float32(0.25)))
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_masked_and_ragged_match_torch():
    B, T, Hq, Hkv, D = 3, 45, 8, 2, 32
    q, k, v = _inputs(B, T, Hq, Hkv, D, 2)
    m, bits = _mask(B, Hkv, T, 0.4, 3)
    lens = np.array([45, 30, 1], np.int32)
    tau = float(np.float32(1.0 / np.sqrt(D)))
    got = O.masked_attn(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), tau, lens=lens, mask=m)
    ref = _torch_ref(q, k, v, tau, bits=bits, lens=lens)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_closed_forms():
    B, T, Hq, Hkv, D = 1, 20, 2, 1, 32
    q, k, v = _inputs(B, T, Hq, Hkv, D, 4)
    W = 1
    # diagonal-only mask: every query sees itself only -> its own value row
    diag = np.zeros((B, Hkv, T, W), np.uint32)
    for t in range(T):
        diag[0, 0, t, 0] = np.uint32(1 << t)
    got = O.masked_attn(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), 0.3, mask=diag)
    vv = v.double().numpy()
    for hq in range(Hq):
        assert np.array_equal(got[0, :, hq], vv[0, :, 0])
    # only future bits set: causally nothing is visible -> 0
    fut = np.zeros((B, Hkv, T, W), np.uint32)
    for t in range(T - 1):
        fut[0, 0, t, 0] = np.uint32((0xFFFFF << (t + 1)) & 0xFFFFF)
    got = O.masked_attn(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), 0.3, mask=fut)
    assert np.all(got[0, : T - 1] == 0.0)
    # equal keys: the output is the mean of the visible values
    k1 = k.clone()
    k1[:] = k[0, 0, 0]
    got = O.masked_attn(synth.bf16_bits(q), synth.bf16_bits(k1), synth.bf16_bits(v), 0.3)
    for t in range(T):
        assert np.allclose(got[0, t, 0], vv[0, : t + 1, 0].mean(axis=0), rtol=1e-12, atol=1e-13)


def test_row_t_equals_the_rollout_decode_step():
    """pi_shadow == pi_sparse: query t under mask row t gives the decode-step
    attention of the rollout at length t + 1 under the same retained set."""
    B, T, Hq, Hkv, D = 2, 70, 8, 2, 64
    q, k, v = _inputs(B, T, Hq, Hkv, D, 5)
    m, _ = _mask(B, Hkv, T, 0.5, 6)
    tau = float(np.float32(1.0 / np.sqrt(D)))
    qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v)
    learner = O.masked_attn(qb, kb, vb, tau, mask=m)
    sh = O.shape(B, Hq, Hkv, D, 16, 128)
    for t in (0, 1, 17, 40, 69):
        rollout = O.decode(sh, np.ascontiguousarray(qb[:, t]), kb, vb, np.full(B, t + 1, np.int32), tau,
                           mask=np.ascontiguousarray(m[:, :, t]), mode=1)
        assert np.allclose(learner[:, t], rollout, rtol=1e-12, atol=1e-13), t
