"""Checks of the seeded input generators that the parity tests and the
benchmark share (CPU only): the shadow mask a rollout's eviction records, and
the learner inputs. None of the method's arithmetic is involved."""
import numpy as np

from compressed_kv_cache_kv4_b200 import synth


def _bits(mask, T):
    m = mask.numpy().view(np.uint32)
    out = np.zeros(m.shape[:-1] + (T,), bool)
    for p in range(T):
        out[..., p] = (m[..., p // 32] >> np.uint32(p % 32)) & 1
    return out


def test_shadow_mask_is_causal_monotone_and_keeps_sink_and_recent():
    wl = synth.workload("learner", B=2)
    T = 400
    bits = _bits(synth.gen_shadow_mask(wl, T), T)             # [B][Hkv][T][T]
    t = np.arange(T)[:, None]
    p = np.arange(T)[None, :]
    assert not (bits & (p > t)).any()                          # nothing after the query
    forced = (p <= t) & ((p < wl.sink) | (p >= t - wl.recent + 1))
    assert (bits | ~forced).all()                              # sink and recent always kept
    # monotone eviction: once a position is gone from row t it stays gone
    # from every later row, except that nothing leaves the recent window early
    gone = (~bits) & (p <= t)
    for tt in range(T - 1):
        assert not (gone[..., tt, :] & bits[..., tt + 1, :]).any(), tt
    # away from the forced positions, p survives to row t with probability
    # P(floor(2 p u) >= t - p) = max(0, 1 - (t - p) / (2 p)) (u uniform)
    tt, pp = np.meshgrid(np.arange(300, T), np.arange(wl.sink, 300 - wl.recent), indexing="ij")
    want = np.clip(1.0 - (tt - pp) / (2.0 * pp), 0.0, 1.0).mean()
    got = bits[..., 300:, wl.sink: 300 - wl.recent].mean()
    assert abs(got - want) < 0.04, (got, want)


def test_shadow_mask_rows_subset_equals_full():
    wl = synth.workload("learner", B=1)
    T = 200
    full = synth.gen_shadow_mask(wl, T).numpy()
    rows = [0, 5, 63, 64, 199]
    part = synth.gen_shadow_mask(wl, T, rows=rows).numpy()
    assert np.array_equal(part, full[:, :, rows])


def test_learner_inputs_are_seeded_and_shaped():
    wl = synth.workload("learner", B=2)
    q1, k1, v1 = synth.gen_learner_qkv(wl, T=64)
    q2, k2, v2 = synth.gen_learner_qkv(wl, T=64)
    assert q1.shape == (2, 64, 32, 128) and k1.shape == (2, 64, 8, 128) and v1.shape == k1.shape
    assert q1.equal(q2) and k1.equal(k2) and v1.equal(v2)
    # the outlier channels of each KV head carry the gain
    chans = synth.outlier_channels(wl)
    kf = k1.float()
    for h in range(wl.Hkv):
        big = kf[:, :, h, chans[h]].abs().mean()
        rest = np.delete(np.arange(wl.D), chans[h])
        small = kf[:, :, h, rest].abs().mean()
        assert big > 5 * small
