"""Pins for oracle.select (CPU): hand-worked cases, brute force, invariants."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from block_sparse_attention_16_b200.workload import get_workload, make_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "select_cases.json")


def _rows(csr):
    return [list(map(int, r)) for r in oracle.csr_rows(*csr)]


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_cases(case):
    s = np.asarray(case["scores"], dtype=np.float32)
    got = _rows(oracle.select_contract(s, case["p"], case["scope"]))
    assert got == case["expected"]
    # the same dyadic cases through the fp64 sequential rule
    assert _rows(oracle.select_fp64(s.astype(np.float64), case["p"], case["scope"])) == case["expected"]


def _w(x32):
    return [int(math.floor(float(v) * 2.0 ** 32)) for v in x32]


def _brute_force_min_size(w, T):
    """Smallest subset size whose weight sum reaches T, and the best sum at that size."""
    n = len(w)
    for k in range(0, n + 1):
        best = max((sum(w[i] for i in c) for c in itertools.combinations(range(n), k)), default=0)
        if best >= T:
            return k, best
    return n, sum(w)


def _check_segment(x32, kept, p):
    w = _w(x32)
    T = oracle.threshold_fixed_point(p, sum(w))
    k_star, best = _brute_force_min_size(w, T)
    k_star = max(k_star, 1)
    assert len(kept) == k_star
    if k_star >= 1 and T > 0:
        assert sum(w[i] for i in kept) == best          # the kept set is a heaviest set of its size
    # ranking property: no dropped element outranks a kept one
    dropped = [i for i in range(len(x32)) if i not in set(kept)]
    for a in kept:
        for b in dropped:
            assert not (x32[b] > x32[a]) and not (x32[b] == x32[a] and b < a)


def test_brute_force_random_rows():
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 10))
        x = rng.random(n).astype(np.float32)
        if trial % 3 == 0:                                 # ties and zeros
            x = rng.choice(np.array([0.0, 0.125, 0.25, 0.3, 0.5], dtype=np.float32), n)
        x = (x / max(float(x.sum()), 1e-30)).astype(np.float32) if trial % 5 else x
        p = float(rng.choice([0.25, 0.5, 0.9, 0.99, 0.999, 0.3]))
        rp, col = oracle.select_contract(x[None, None, None, :], p, "row")
        _check_segment(x, list(map(int, col)), p)


def test_brute_force_tiny_workload_rows_and_heads():
    wl = get_workload("tiny")
    q, k, _ = make_qkv(wl)
    m = oracle.block_mass(q.numpy(), k.numpy(), wl.n_valid, wl.block).astype(np.float32)
    for p in (0.5, 0.9, 0.99):
        rows = oracle.csr_rows(*oracle.select_contract(m, p, "row"))
        for h in range(wl.H):
            for i in range(wl.n_blocks):
                _check_segment(m[0, h, i], list(map(int, rows[h * wl.n_blocks + i])), p)
        # head scope: 16 pairs -> 65,536 subsets
        rows = oracle.csr_rows(*oracle.select_contract(m / 4.0, p, "head"))
        for h in range(wl.H):
            flat = [i * 4 + int(j) for i in range(4) for j in rows[h * 4 + i]]
            _check_segment((m[0, h] / 4.0).reshape(-1).astype(np.float32), flat, p)


def test_invariants_retained_minimal_and_fraction():
    rng = np.random.default_rng(7)
    x = rng.random((2, 3, 16, 16)).astype(np.float32) ** 4
    for scope in ("row", "head"):
        for p in (0.25, 0.9, 0.99):
            rows = oracle.csr_rows(*oracle.select_contract(x, p, scope))
            segs = ([(b, h, i) for b in range(2) for h in range(3) for i in range(16)]
                    if scope == "row" else [(b, h) for b in range(2) for h in range(3)])
            for s in segs:
                if scope == "row":
                    b, h, i = s
                    vals = x[b, h, i]
                    kept = list(map(int, rows[(b * 3 + h) * 16 + i]))
                else:
                    b, h = s
                    vals = x[b, h].reshape(-1)
                    kept = [i * 16 + int(j) for i in range(16) for j in rows[(b * 3 + h) * 16 + i]]
                w = np.floor(vals.astype(np.float64) * 2.0 ** 32).astype(np.int64)
                T = oracle.threshold_fixed_point(p, int(w.sum()))
                kw = sorted((int(w[i]) for i in kept))
                assert sum(kw) >= T                                  # retained >= p
                assert sum(kw) - kw[0] < T                           # dropping the lowest falls below
                n = len(vals)
                assert (len(kept) - 1) < p * n                       # kept fraction bound
                # real-valued retained mass, up to the 2^-32 quantum per element
                assert vals[kept].astype(np.float64).sum() >= p * vals.astype(np.float64).sum() - n * 2.0 ** -32 - 1e-7


def test_p_one_keeps_everything_and_invalid_scores_rejected():
    x = np.zeros((1, 1, 3, 3), dtype=np.float32)
    rp, col = oracle.select_contract(x, 1.0, "row")
    assert list(rp) == [0, 3, 6, 9]
    for bad in (np.nan, -1.0, 2.0, np.inf, -0.0):
        y = np.full((1, 1, 2, 2), 0.25, dtype=np.float32)
        y[0, 0, 1, 1] = bad
        with pytest.raises(oracle.InvalidScores):
            oracle.select_contract(y, 0.9, "row")
    with pytest.raises(ValueError):
        oracle.select_contract(x, 0.0, "row")
    with pytest.raises(ValueError):
        oracle.select_contract(x, 1.5, "row")


def test_fixed_point_threshold_values():
    # p = 0.99 quantises to 16,609,444 / 2^24
    assert oracle.threshold_fixed_point(0.99, 1 << 24) == 16609444
    assert oracle.threshold_fixed_point(1.0, 12345) == 12345
    assert oracle.threshold_fixed_point(0.5, 3) == 2                # ceil(1.5)
    assert oracle.threshold_fixed_point(0.25, 1 << 40) == 1 << 38


def test_fractional_weights_are_floored():
    # Scores below 2^-9 have fp32 bits finer than 2^-32, so their weight
    # x * 2^32 has a fractional part, which the contract floors.  Hand-worked:
    # x = (0.25, 0.25, 3 * 2^-34) gives w = (2^30, 2^30, floor(0.75) = 0),
    # W = 2^31 and, at p = 1/2, T = ceil(2^23 * 2^31 / 2^24) = 2^30, which the
    # first 0.25 reaches alone.  (Rounded weights would make W = 2^31 + 1 and
    # T = 2^30 + 1, so both 0.25 blocks; real arithmetic keeps both as well,
    # since 0.25 < (0.5 + 3 * 2^-34) / 2: the quantum is part of the contract.)
    tiny = np.float32(3.0 * 2.0 ** -34)
    assert float(tiny) * 2.0 ** 32 == 0.75
    x = np.array([[[[0.25, 0.25, tiny]]]], dtype=np.float32)
    assert _rows(oracle.select_contract(x, 0.5, "row")) == [[0]]
    assert _rows(oracle.select_fp64(x.astype(np.float64), 0.5, "row")) == [[0, 1]]
    # scores below the 2^-32 quantum weigh nothing: five 2^-33 (weight
    # floor(1/2) = 0 each) beside one 2^-20 (weight 2^12) give W = 2^12 and, at
    # p = 0.999 (P = 16,760,439), T = ceil(P * 2^12 / 2^24) = 4092 <= 2^12
    y = np.full((1, 1, 1, 6), np.float32(2.0 ** -33), dtype=np.float32)
    y[0, 0, 0, 4] = np.float32(2.0 ** -20)
    assert _rows(oracle.select_contract(y, 0.999, "row")) == [[4]]


def test_fp64_rule_agrees_on_tiny_workload():
    wl = get_workload("tiny")
    q, k, _ = make_qkv(wl)
    m = oracle.block_mass(q.numpy(), k.numpy(), wl.n_valid, wl.block)
    for p in (0.5, 0.9, 0.99, 0.999):
        a = oracle.select_contract(m.astype(np.float32), p, "row")
        b = oracle.select_fp64(m, p, "row")
        assert _rows(a) == _rows(b)
