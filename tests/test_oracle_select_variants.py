"""Pins of the Local + TopK and top-p-with-floor selection rules (CPU)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "select_variant_cases.json")))


def _rows(csr):
    return [list(map(int, r)) for r in oracle.csr_rows(*csr)]


def test_local_topk_golden():
    for g in GOLD["local_topk"]:
        x = np.asarray(g["scores"], dtype=np.float32)[None, None]
        for c in g["cases"]:
            assert _rows(oracle.select_local_topk(x, c["k"])) == c["rows"], c["why"]


def test_topp_floor_golden():
    for g in GOLD["topp_floor"]:
        x = np.asarray(g["scores"], dtype=np.float32)[None, None]
        assert oracle.floor_of_head(g["counts"], g["n_valid"], g["block"]) == g["floor"]
        assert _rows(oracle.select_topp_floor(x, g["p"], g["n_valid"], g["block"])) == g["rows"], g["why"]
        assert [len(r) for r in oracle.csr_rows(*oracle.select_contract(x, g["p"], "row"))] == g["counts"]


def _rank_pairwise(row, exclude):
    """Rank of every id among the others by pairwise comparison (no sort)."""
    bits = row.view(np.uint32).astype(np.int64)
    n = len(row)
    rank = {}
    for j in range(n):
        if j == exclude:
            continue
        rank[j] = sum(1 for t in range(n) if t != exclude and t != j and
                      (bits[t] > bits[j] or (bits[t] == bits[j] and t < j)))
    return rank


@pytest.mark.parametrize("seed", range(6))
def test_local_topk_matches_pairwise_ranking(seed):
    rng = np.random.default_rng(seed)
    nB = int(rng.integers(1, 12))
    vals = np.array([0.0, 2.0 ** -20, 0.125, 0.25, 0.25 + 2.0 ** -10, 0.5, 1.0, 1.5], dtype=np.float32)
    x = rng.choice(vals, size=(1, 2, nB, nB)).astype(np.float32)
    for k in (0, 1, 2, 3, nB - 1, nB + 3):
        if k < 0:
            continue
        got = _rows(oracle.select_local_topk(x, k))
        r = 0
        for h in range(2):
            for i in range(nB):
                rank = _rank_pairwise(x[0, h, i], i)
                expect = sorted([i] + [j for j, rk in rank.items() if rk < k])
                assert got[r] == expect
                r += 1


@pytest.mark.parametrize("seed", range(6))
def test_topp_floor_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    block = 64
    nB = int(rng.integers(2, 9))
    n_valid = (nB - 1) * block + int(rng.integers(1, block + 1))
    p = float(rng.choice([0.3, 0.5, 0.9, 0.99]))
    x = (rng.random((1, 3, nB, nB)) ** 6).astype(np.float32)
    x[0, 1, :, 0] = 0.0                                   # zero-weight blocks
    x[0, 2] = np.float32(0.25)                            # all ties
    base = oracle.csr_rows(*oracle.select_contract(x, p, "row"))
    got = oracle.csr_rows(*oracle.select_topp_floor(x, p, n_valid, block))
    v = [min(block, n_valid - i * block) for i in range(nB)]
    for h in range(3):
        c = [len(base[h * nB + i]) for i in range(nB)]
        K = oracle.floor_of_head(c, n_valid, block)
        mean = Fraction(sum(vi * ci for vi, ci in zip(v, c)), sum(v))
        assert K - 1 < mean <= K                               # the ceiling, by exact rationals
        for i in range(nB):
            row = x[0, h, i]
            n = max(c[i], min(K, nB))
            rank = _rank_pairwise(row, -1)
            expect = sorted(j for j, rk in rank.items() if rk < n)
            assert list(got[h * nB + i]) == expect             # a prefix of the ranked order
            assert set(base[h * nB + i]) <= set(expect)        # extends the threshold set


def test_variants_reject_bad_input():
    with pytest.raises(oracle.InvalidScores):
        oracle.select_local_topk(np.full((1, 1, 2, 2), -1.0, np.float32), 1)
    with pytest.raises(ValueError):
        oracle.select_topp_floor(np.full((1, 1, 2, 2), 0.5, np.float32), 0.5, 200, 64)   # n_valid past the grid
