"""Host-side helpers of bench.py that turn measurements into reported figures
(CPU only): the set-bit count of a mask (visible pairs of the learner row) and
the algorithmic bytes of one page-eviction launch."""
import importlib.util
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_mask_popcount_matches_python_count():
    b = _bench()
    rng = np.random.default_rng(3)
    words = rng.integers(0, 2 ** 32, size=(3, 5, 7), dtype=np.uint64).astype(np.uint32)
    words[0, 0, 0] = 0xFFFFFFFF
    words[0, 0, 1] = 0x80000000
    want = sum(bin(int(w)).count("1") for w in words.reshape(-1))
    got = b.mask_popcount(torch.from_numpy(words.view(np.int32).copy()))
    assert got == want


def test_page_evict_bytes_by_hand():
    b = _bench()
    from compressed_kv_cache_kv4_b200 import synth
    wl = synth.workload("evict", B=2, L=16384)
    # L = 16384: n = 1024 pages, candidates 1..1015 (1015), kept non-candidates 9
    # 10%: k = 102 -> 93 candidates kept, e = 922, e mod 8 = 2 -> ring rotates
    per_seq = 8 + 4 + 1015 * 16 * 8 * 4 + 2 * 1024 * 4 + 922 * 4 + 2 * 8 * 8 * (32 * 128 + 64)
    assert b.page_evict_bytes(wl, wl.lens, 1024, 100, 8) == 2 * per_seq
    # 50%: k = 512 -> 503 kept, e = 512, a multiple of 8 -> the ring stays
    per_seq = 8 + 4 + 1015 * 16 * 8 * 4 + 2 * 1024 * 4 + 512 * 4
    assert b.page_evict_bytes(wl, wl.lens, 1024, 500, 8) == 2 * per_seq
    # 100%: nothing leaves, only the length and the count
    assert b.page_evict_bytes(wl, wl.lens, 1024, 1000, 8) == 2 * 12
