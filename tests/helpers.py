"""Shared test plumbing: build caches from the seeded inputs, run the oracle on
selected sequences, and compare within the stated tolerances.

Tolerances (the attention outputs of kv4_decode_attn against the fp64 oracle on
the same dequantised values): max-abs <= 2e-3 and relative L2 <= 5e-3, checked
on the kernel's fp32 output mode. The bf16 output must equal the
round-to-nearest-even bf16 of that fp32 output, and lie within 2e-3 plus half a
bf16 ulp of the oracle (a bf16 half-ulp alone exceeds 2e-3 once |o| >= 1).
"""
import numpy as np
import torch

import oracle as O
from compressed_kv_cache_kv4_b200 import synth
import compressed_kv_cache_kv4_b200 as K

ATOL = 2e-3
RTOL_L2 = 5e-3


def assert_close(got, ref, atol=ATOL, rl2=RTOL_L2, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got - ref))
    assert mx <= atol and rel <= rl2, "%s max_abs=%.3e rel_l2=%.3e" % (what, mx, rel)
    return mx, rel


def bf16_ulp(x):
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_output(out_bf16, out_fp32, ref):
    want = out_fp32.to(torch.bfloat16)
    assert torch.equal(out_bf16.view(torch.int16), want.view(torch.int16)), "bf16 output != RNE(fp32 output)"
    got = out_bf16.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= ATOL + 0.5 * bf16_ulp(ref)), "bf16 output outside tolerance"


class Case:
    """A workload laid out for both sides: packed K/V, query, page table and a
    GPU cache filled by kv4_append (or by copying oracle-written bytes)."""

    def __init__(self, wl, gen_device="cpu", fill=0xA5, extra_tokens=0, num_pages_extra=0):
        self.wl = wl
        self.k, self.v, self.off = synth.gen_kv(wl, device=gen_device)
        self.q = synth.gen_q(wl, device=gen_device)
        cap = wl.lens.astype(np.int64) + extra_tokens
        self.pt_np, self.num_pages = synth.gen_page_table(wl, cap, extra_pages=num_pages_extra)
        self.fill = fill

    # ---------------------------------------------------------------- GPU side
    def make_cache(self):
        wl = self.wl
        self.cache = K.KV4Cache(wl.Hkv, wl.D, wl.B, self.num_pages, wl.sink, wl.recent, fill=self.fill)
        self.pt = torch.as_tensor(self.pt_np, device="cuda")
        self.lens = torch.as_tensor(wl.lens, device="cuda")
        return self.cache

    def append_all(self, chunks=1):
        """Append every position with kv4_append, in `chunks` calls per sequence."""
        wl = self.wl
        k = self.k.to("cuda")
        v = self.v.to("cuda")
        lens_done = np.zeros(wl.B, np.int64)
        for c in range(chunks):
            upto = np.array([(int(L) * (c + 1)) // chunks for L in wl.lens], np.int64)
            n_new = upto - lens_done
            offs = np.zeros(wl.B + 1, np.int64)
            offs[1:] = np.cumsum(n_new)
            idx = np.concatenate([np.arange(self.off[b] + lens_done[b], self.off[b] + upto[b])
                                  for b in range(wl.B)]).astype(np.int64)
            idx_t = torch.as_tensor(idx, device="cuda")
            kk = k.index_select(0, idx_t).contiguous()
            vv = v.index_select(0, idx_t).contiguous()
            self.cache.append(kk, vv, torch.as_tensor(offs.astype(np.int32), device="cuda"),
                              torch.as_tensor(lens_done.astype(np.int32), device="cuda"), self.pt)
            lens_done = upto
        torch.cuda.synchronize()

    def load_oracle_bytes(self):
        pool, side, _ = self.oracle_cache()
        self.cache.pool.copy_(torch.as_tensor(pool))
        if self.cache.side is not None:
            self.cache.side.copy_(torch.as_tensor(side))

    def decode(self, out_fp32=True, mask=None, num_workers=0, q=None):
        q = (self.q if q is None else q).to("cuda")
        return self.cache.decode(q, self.lens, self.pt, self.wl.softmax_scale, out_fp32=out_fp32,
                                 retain_mask=mask, num_workers=num_workers)

    # ---------------------------------------------------------------- oracle side
    def shape(self, seqs=None):
        wl = self.wl
        n = wl.B if seqs is None else len(seqs)
        return O.shape(n, wl.Hq, wl.Hkv, wl.D, wl.sink, wl.recent)

    def oracle_cache(self):
        wl = self.wl
        kb = synth.bf16_bits(synth.pad_batch(self.k, self.off, range(wl.B)))
        vb = synth.bf16_bits(synth.pad_batch(self.v, self.off, range(wl.B)))
        return O.write_cache(self.shape(), kb, vb, wl.lens, self.pt_np, self.num_pages, fill=self.fill)

    def oracle_decode(self, seqs=None, mask=None, mode=0):
        wl = self.wl
        seqs = list(range(wl.B)) if seqs is None else list(seqs)
        kb = synth.bf16_bits(synth.pad_batch(self.k, self.off, seqs))
        vb = synth.bf16_bits(synth.pad_batch(self.v, self.off, seqs))
        qb = synth.bf16_bits(self.q[seqs])
        lens = wl.lens[seqs]
        m = None if mask is None else np.ascontiguousarray(np.asarray(mask)[seqs])
        return O.decode(self.shape(seqs), qb, kb, vb, lens, wl.softmax_scale, mask=m, mode=mode)


def bf16_pages(case):
    """bf16 page pool for the comparison kernel: [num_pages][Hkv][K|V][16][D]."""
    wl = case.wl
    pages = torch.zeros((case.num_pages, wl.Hkv, 2, 16, wl.D), dtype=torch.bfloat16, device="cuda")
    k = case.k.to("cuda")
    v = case.v.to("cuda")
    for b in range(wl.B):
        L = int(wl.lens[b])
        pos = torch.arange(L, device="cuda")
        pid = torch.as_tensor(case.pt_np[b], device="cuda")[pos // 16].long()
        slot = (pos % 16).long()
        kb = k[int(case.off[b]): int(case.off[b]) + L]        # [L][Hkv][D]
        vb = v[int(case.off[b]): int(case.off[b]) + L]
        pages[pid, :, 0, slot, :] = kb
        pages[pid, :, 1, slot, :] = vb
    return pages
