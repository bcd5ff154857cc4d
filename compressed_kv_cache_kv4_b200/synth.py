"""Seeded synthetic inputs for the five decode-attention workloads.

This module holds input synthesis only: shapes, seeds and value distributions.
None of the method's arithmetic (quantisation, attention, merge, selection)
lives here. Both the CUDA path and the CPU oracle receive the tensors made
here, so the two never share anything but their inputs.

Workloads (the pages run RL rollouts of Qwen3-4B/8B-Base, which are not
available; these synthetic shapes stand in for them):

- ``tiny``   B=2, L=(200, 37), 4 query / 2 KV heads, D=64, outlier K channels
              3 and 17 scaled x8, softmax scale 1/8.
- ``qwen8b`` B=64, L ~ U{1024..8192}, 32/8 heads, D=128, per KV head 4 random
              K channels scaled x10, pages randomly permuted.
- ``async``  B=256, L0 = clip(round(exp(N(ln 4096, 1))), 256, 32768), same
              heads; 64 decode steps of one appended token per sequence.
- ``long``   B=4, L=131072, same heads.
- ``evict``  B=64, L=16384, same heads; per-position scores are the summed
              softmax attention of 32 random N(0,1) queries at the 32 positions
              before the current one (H2O-style accumulated attention).
- ``learner`` B=4 sequences of T=8192 positions, same heads, for the
              learner-side attention under the shadow mask: q, K, V of every
              position and the mask the rollout's eviction recorded per query
              position (``gen_shadow_mask``).

Random values depend on the device the generator runs on (torch's CPU and CUDA
generators differ); every comparison hands the same tensors to both sides.
"""
from dataclasses import dataclass, field
import math

import numpy as np
import torch

PAGE_TOKENS = 16


@dataclass
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    lens: np.ndarray              # int32 [B], context length after this step's append
    softmax_scale: float
    sink: int = 16
    recent: int = 128
    outlier_channels: tuple = ()  # fixed channels (tiny workload), else random per KV head
    outlier_count: int = 4
    outlier_gain: float = 10.0
    steps: int = 1                # decode steps the workload runs
    budgets: tuple = ()           # permille budgets (evict workload)
    extra: dict = field(default_factory=dict)

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def total_len(self):
        return int(self.lens.astype(np.int64).sum())


def _gen(seed, purpose, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + int(purpose))
    return g


def _f32_inv_sqrt(D):
    return float(np.float32(1.0) / np.sqrt(np.float32(D)))


def workload(name, **over):
    """Build one of the five workloads; keyword overrides shrink it for tests."""
    if name == "tiny":
        wl = Workload("tiny", 1001, 2, 4, 2, 64, np.array([200, 37], np.int32), 0.125,
                      outlier_channels=(3, 17), outlier_gain=8.0)
    elif name == "qwen8b":
        B = over.pop("B", 64)
        lo, hi = over.pop("len_range", (1024, 8192))
        g = _gen(1002, 0)
        lens = torch.randint(lo, hi + 1, (B,), generator=g).numpy().astype(np.int32)
        wl = Workload("qwen8b", 1002, B, 32, 8, 128, lens, _f32_inv_sqrt(128))
    elif name == "async":
        B = over.pop("B", 256)
        med, lo, hi = over.pop("len_dist", (4096, 256, 32768))
        g = _gen(1003, 0)
        z = torch.randn(B, generator=g, dtype=torch.float64).numpy()
        lens = np.clip(np.round(np.exp(math.log(med) + 1.0 * z)), lo, hi).astype(np.int32)
        wl = Workload("async", 1003, B, 32, 8, 128, lens, _f32_inv_sqrt(128), steps=64)
    elif name == "long":
        B = over.pop("B", 4)
        L = over.pop("L", 131072)
        wl = Workload("long", 1004, B, 32, 8, 128, np.full(B, L, np.int32), _f32_inv_sqrt(128))
    elif name == "learner":
        B = over.pop("B", 4)
        T = over.pop("T", 8192)
        wl = Workload("learner", 1006, B, 32, 8, 128, np.full(B, T, np.int32), _f32_inv_sqrt(128))
    elif name == "evict":
        B = over.pop("B", 64)
        L = over.pop("L", 16384)
        wl = Workload("evict", 1005, B, 32, 8, 128, np.full(B, L, np.int32), _f32_inv_sqrt(128),
                      budgets=(100, 300, 500, 900, 1000))
    else:
        raise ValueError(name)
    for k, v in over.items():
        setattr(wl, k, v)
    wl.lens = np.asarray(wl.lens, np.int32)
    wl.B = int(wl.lens.size)
    return wl


def outlier_channels(wl):
    """[Hkv][n] channel indices whose K values are scaled by ``outlier_gain``."""
    if wl.outlier_channels:
        return np.tile(np.array(wl.outlier_channels, np.int64), (wl.Hkv, 1))
    g = _gen(wl.seed, 2)
    return np.stack([torch.randperm(wl.D, generator=g)[: wl.outlier_count].numpy()
                     for _ in range(wl.Hkv)])


def offsets_of(lens):
    off = np.zeros(len(lens) + 1, np.int64)
    off[1:] = np.cumsum(np.asarray(lens, np.int64))
    return off


def gen_kv(wl, device="cpu", lens=None, purpose=1):
    """Packed bf16 K and V: [T][Hkv][D] with T = sum(lens), plus int64 offsets [B+1].
    K ~ N(0,1) with the outlier channels scaled; V ~ N(0,1)."""
    lens = wl.lens if lens is None else np.asarray(lens, np.int32)
    off = offsets_of(lens)
    T = int(off[-1])
    g = _gen(wl.seed, purpose, device)
    k = torch.randn((T, wl.Hkv, wl.D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((T, wl.Hkv, wl.D), generator=g, device=device, dtype=torch.float32)
    gain = torch.ones((wl.Hkv, wl.D), device=device, dtype=torch.float32)
    for h, chans in enumerate(outlier_channels(wl)):
        gain[h, torch.as_tensor(chans, device=device)] = wl.outlier_gain
    k.mul_(gain)
    return k.to(torch.bfloat16), v.to(torch.bfloat16), off


def gen_step_kv(wl, step, device="cpu"):
    """New K/V for one decode step, one token per sequence: [B][Hkv][D] bf16."""
    g = _gen(wl.seed, 100 + 2 * step, device)
    k = torch.randn((wl.B, wl.Hkv, wl.D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((wl.B, wl.Hkv, wl.D), generator=g, device=device, dtype=torch.float32)
    gain = torch.ones((wl.Hkv, wl.D), device=device, dtype=torch.float32)
    for h, chans in enumerate(outlier_channels(wl)):
        gain[h, torch.as_tensor(chans, device=device)] = wl.outlier_gain
    k.mul_(gain)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def gen_q(wl, step=0, device="cpu"):
    """Query of one decode step: [B][Hq][D] bf16, N(0,1)."""
    g = _gen(wl.seed, 3 + 2 * step, device)
    return torch.randn((wl.B, wl.Hq, wl.D), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def gen_page_table(wl, capacity_tokens=None, extra_pages=0):
    """Random physical page assignment. capacity_tokens[b] positions are mapped for
    sequence b (defaults to lens). Unmapped entries hold -1.
    Returns (page_table int32 [B][pt_stride], num_pages)."""
    cap = wl.lens if capacity_tokens is None else np.asarray(capacity_tokens, np.int64)
    npg = (np.asarray(cap, np.int64) + PAGE_TOKENS - 1) // PAGE_TOKENS
    total = int(npg.sum()) + extra_pages
    g = _gen(wl.seed, 4)
    perm = torch.randperm(total, generator=g).numpy().astype(np.int32)
    stride = int(max(1, npg.max()))
    pt = np.full((wl.B, stride), -1, np.int32)
    pos = 0
    for b in range(wl.B):
        pt[b, : npg[b]] = perm[pos: pos + npg[b]]
        pos += int(npg[b])
    return pt, total


def gen_scores(wl, k, off, device="cpu", n_queries=32, chunk=8):
    """H2O-style accumulated attention scores, fp32 [B][Hkv][Lmax]: for each
    (b, h), the sum over 32 random N(0,1) queries q_j placed at positions
    t_j = L-33+j (j = 1..32) of softmax over p <= t_j of tau * q_j . K_p.
    Positions beyond L_b are 0."""
    Lmax = int(wl.lens.max())
    out = torch.zeros((wl.B, wl.Hkv, Lmax), device=device, dtype=torch.float32)
    g = _gen(wl.seed, 5, device)
    for b in range(wl.B):
        L = int(wl.lens[b])
        kb = k[int(off[b]): int(off[b + 1])].to(device=device, dtype=torch.float32)  # [L][Hkv][D]
        qj = torch.randn((wl.Hkv, n_queries, wl.D), generator=g, device=device, dtype=torch.float32)
        t = torch.arange(L - 33 + 1, L - 33 + n_queries + 1, device=device)          # t_j
        logits = torch.einsum("hjd,phd->hjp", qj, kb) * wl.softmax_scale
        pos = torch.arange(L, device=device)
        logits = logits.masked_fill(pos[None, None, :] > t[None, :, None], float("-inf"))
        out[b, :, :L] = torch.softmax(logits, dim=-1).sum(dim=1)
    return out


def pad_batch(x, off, seqs, Lmax=None):
    """Packed [T][...] -> padded [len(seqs)][Lmax][...] (zeros past each length)."""
    lens = [int(off[b + 1] - off[b]) for b in seqs]
    Lmax = max(lens) if Lmax is None else Lmax
    out = torch.zeros((len(seqs), max(Lmax, 1)) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    for i, b in enumerate(seqs):
        out[i, : lens[i]] = x[int(off[b]): int(off[b + 1])]
    return out


def bf16_bits(t):
    """bf16 tensor -> numpy uint16 bit patterns (CPU)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def gen_learner_qkv(wl, T=None, device="cpu"):
    """Learner inputs for B sequences of T positions: q [B][T][Hq][D], K and V
    [B][T][Hkv][D] in bf16, N(0,1) with the outlier K channels scaled."""
    T = int(wl.lens.max()) if T is None else T
    g = _gen(wl.seed, 7, device)
    q = torch.randn((wl.B, T, wl.Hq, wl.D), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((wl.B, T, wl.Hkv, wl.D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((wl.B, T, wl.Hkv, wl.D), generator=g, device=device, dtype=torch.float32)
    gain = torch.ones((wl.Hkv, wl.D), device=device, dtype=torch.float32)
    for h, chans in enumerate(outlier_channels(wl)):
        gain[h, torch.as_tensor(chans, device=device)] = wl.outlier_gain
    k.mul_(gain)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def gen_shadow_mask(wl, T=None, device="cpu", sink=None, recent=None, rows=None):
    """The mask a rollout's eviction records, int32 [B][Hkv][T][ceil(T/32)]
    (bit p % 32 of word p / 32 of row t: position p kept at query position t).

    Eviction is monotone: position p of (b, h) stays until step
    e = p + 1 + floor(2 p u), u ~ U[0, 1), and never returns; the first `sink`
    and the last `recent` positions are always kept. Away from those, p is
    still kept in row t with probability max(0, 1 - (t - p) / (2 p)); over the
    causal triangle of 8192 positions 45.5% of the (query, key) pairs are kept.
    Bits above t are clear. `rows` limits the
    output to those query positions (then [B][Hkv][len(rows)][words])."""
    T = int(wl.lens.max()) if T is None else T
    sink = wl.sink if sink is None else sink
    recent = wl.recent if recent is None else recent
    g = _gen(wl.seed, 8, device)
    u = torch.rand((wl.B, wl.Hkv, T), generator=g, device=device, dtype=torch.float64)
    pos = torch.arange(T, device=device, dtype=torch.float64)
    evict_at = (pos + 1 + torch.floor(2 * pos * u)).to(torch.int64)       # [B][Hkv][T]
    W = (T + 31) // 32
    trows = torch.arange(T, device=device) if rows is None else torch.as_tensor(rows, device=device)
    out = torch.zeros((wl.B, wl.Hkv, len(trows), W), dtype=torch.int32, device=device)
    shifts = torch.arange(32, device=device, dtype=torch.int64)
    p = torch.arange(W * 32, device=device)
    pe = torch.full((wl.B, wl.Hkv, W * 32), -1, dtype=torch.int64, device=device)
    pe[..., :T] = evict_at
    chunk = 256
    for c0 in range(0, len(trows), chunk):
        t = trows[c0: c0 + chunk].to(torch.int64)[:, None]                    # [c][1]
        keep = (p[None, :] <= t) & ((p[None, :] < sink) | (p[None, :] >= t - recent + 1)
                                    | (pe[:, :, None, :] > t))                  # [B][Hkv][c][W*32]
        keep &= p[None, :] < T
        words = (keep.view(wl.B, wl.Hkv, -1, W, 32).to(torch.int64) << shifts).sum(-1)
        out[:, :, c0: c0 + chunk] = (words & 0xFFFFFFFF).to(torch.int32)
    return out
