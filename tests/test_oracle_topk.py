"""Pins for the oracle's retained-position selection.

Pages: KVP promo (arXiv 2602.10238), core mechanism -- a continuous score per
token, rank, truncate at any budget from 10% to 90% with one policy; TTKV promo
(arXiv 2604.19769), insight 1 -- eviction as ranking, per head. KV4-RL review
sec. 3 -- the first 16 and last 128 positions are always kept. Build readings:
k = floor(L * permille / 1000), forced positions count toward k, ties go to
the lower index.
"""
import itertools

import numpy as np
import pytest

import oracle as O


def _bits_of(mask_row, L):
    return [p for p in range(L) if (mask_row[p // 32] >> (p % 32)) & 1]


def _brute(scores, L, permille, sink, recent):
    forced = {p for p in range(L) if p < sink or p >= L - recent}
    cand = [p for p in range(L) if p not in forced]
    k = L * permille // 1000
    take = max(0, min(k - len(forced), len(cand)))
    valid = []
    for sub in itertools.combinations(cand, take):
        s = set(sub)
        kept, dropped = [p for p in cand if p in s], [p for p in cand if p not in s]
        if all((scores[a] > scores[d]) or (scores[a] == scores[d] and a < d)
               for a in kept for d in dropped):
            valid.append(s)
    assert len(valid) == 1
    return sorted(forced | valid[0])


def test_brute_force_tiny():
    rng = np.random.default_rng(2)
    for trial in range(120):
        L = int(rng.integers(1, 13))
        sink, recent = int(rng.integers(0, 3)), int(rng.integers(0, 4))
        permille = int(rng.integers(0, 1001))
        levels = int(rng.integers(1, 4))                 # few levels -> many ties
        sc = rng.integers(0, levels, size=L).astype(np.float32)
        if trial % 3 == 0:
            sc = rng.standard_normal(L).astype(np.float32)
        scores = np.zeros((1, 1, 16), np.float32)
        scores[0, 0, :L] = sc
        mask, count = O.topk(scores, np.array([L], np.int32), permille, sink, recent)
        want = _brute(sc, L, permille, sink, recent)
        assert _bits_of(mask[0, 0], L) == want, (trial, L, permille)
        assert count[0, 0] == len(want)


def test_nested_budgets_and_forced_set():
    rng = np.random.default_rng(4)
    B, H, L = 3, 2, 2000
    scores = rng.standard_normal((B, H, L)).astype(np.float32)
    scores[:, :, ::5] = 0.5                               # plenty of exact ties
    lens = np.array([2000, 1000, 150], np.int32)
    prev = None
    for permille in (100, 300, 500, 900, 1000):
        mask, count = O.topk(scores, lens, permille)
        for b in range(B):
            Lb = int(lens[b])
            forced = min(Lb, 16 + 128) if Lb > 16 else Lb
            kept = _bits_of(mask[b, 0], Lb)
            assert set(range(16)) <= set(kept) and set(range(max(0, Lb - 128), Lb)) <= set(kept)
            assert count[b, 0] == max(Lb * permille // 1000, forced)
            if prev is not None:
                assert set(_bits_of(prev[b, 0], Lb)) <= set(kept)
        prev = mask
    assert all(count[b, 0] == lens[b] for b in range(B))  # 100% keeps everything


def test_budget_counts_golden():
    """k at L = 16384 for the evict workload budgets (tests/golden/budget_counts.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "budget_counts.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    scores = np.random.default_rng(0).standard_normal((1, 1, 16384)).astype(np.float32)
    for L, permille, want in ((int(a), int(b), int(c)) for a, b, c in rows):
        _, count = O.topk(scores, np.array([L], np.int32), permille)
        assert count[0, 0] == want


def test_negative_zero_equals_zero():
    scores = np.zeros((1, 1, 8), np.float32)
    scores[0, 0, 2] = -0.0
    scores[0, 0, 5] = 0.0
    scores[0, 0, 6] = -1.0
    mask, _ = O.topk(scores, np.array([8], np.int32), 250, 0, 0)   # k = 2
    assert _bits_of(mask[0, 0], 8) == [0, 1]                        # all zeros tie: lowest indices
    mask, _ = O.topk(scores, np.array([8], np.int32), 875, 0, 0)   # k = 7: drop only the -1
    assert _bits_of(mask[0, 0], 8) == [0, 1, 2, 3, 4, 5, 7]
