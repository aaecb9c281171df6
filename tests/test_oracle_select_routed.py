"""Pins of the entropy-routed selection oracle (EG-Sparse abstract, readsearch.ai
page of arXiv 2610.14672): hand-worked golden cases, scipy's entropy, closed
forms, reductions to the row rule, and brute force over tiny pools."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.stats

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "select_routed_cases.json")))


def _rows(csr):
    return [list(map(int, r)) for r in oracle.csr_rows(*csr)]


def test_golden_entropy_route_rows():
    x = np.asarray(GOLD["scores"], dtype=np.float32)[None]
    e = oracle.head_entropy(x)
    np.testing.assert_allclose(e[0], GOLD["entropy"], rtol=0, atol=1e-12, err_msg=GOLD["entropy_why"])
    for c in GOLD["cases"]:
        assert oracle.route_heads(e, c["threshold"], c["group"])[0].tolist() == c["route"], c["why"]
        assert _rows(oracle.select_routed(x, c["p"], c["threshold"], c["group"])) == c["rows"], c["why"]


@pytest.mark.parametrize("seed", range(4))
def test_entropy_against_scipy(seed):
    rng = np.random.default_rng(seed)
    nB = int(rng.integers(2, 40))
    x = (rng.random((2, 3, nB, nB)) ** 4).astype(np.float32)
    x[0, 1, :, ::3] = 0.0                                  # zero entries: 0 ln 0 = 0
    x[1, 2] *= np.float32(1e-3)                            # rows not summing to 1
    e = oracle.head_entropy(x)
    for b in range(2):
        for h in range(3):
            rows = [scipy.stats.entropy(x[b, h, i].astype(np.float64)) for i in range(nB)]
            assert abs(e[b, h] - np.mean(rows) / math.log(nB)) < 1e-12


def test_entropy_closed_forms():
    nB = 7
    x = np.zeros((1, 4, nB, nB), dtype=np.float32)
    x[0, 0] = 1.0 / nB                                     # uniform rows: 1
    for i in range(nB):
        x[0, 1, i, (3 * i) % nB] = 1.0                     # one-hot rows: 0
        x[0, 2, i, i] = x[0, 2, i, (i + 1) % nB] = 0.5     # two halves: ln 2 / ln nB
    x[0, 3, : nB // 2] = 1.0 / nB                          # half uniform, half all-zero rows
    e = oracle.head_entropy(x)[0]
    assert abs(e[0] - 1.0) < 1e-6 and e[1] == 0.0
    assert abs(e[2] - math.log(2) / math.log(nB)) < 1e-12
    assert abs(e[3] - (nB // 2) / nB * e[0]) < 1e-12
    assert oracle.head_entropy(np.ones((1, 2, 1, 1), dtype=np.float32)).tolist() == [[0.0, 0.0]]
    # scale invariance: the row is normalised first
    np.testing.assert_allclose(oracle.head_entropy(x * np.float32(0.25)), oracle.head_entropy(x), atol=1e-12)


def test_route_heads_groups():
    e = np.array([[0.1, 0.9, 0.2, 0.3, 0.95, 0.05, 0.4]])
    assert oracle.route_heads(e, 0.5, 2).tolist() == [[0, -1, 0, 1, -1, 1, 2]]
    assert oracle.route_heads(e, 0.5, 10).tolist() == [[0, -1, 0, 0, -1, 0, 0]]
    assert oracle.route_heads(e, 0.05, 1).tolist() == [[-1] * 7]          # strict <
    assert oracle.route_heads(e, 1.5, 3).tolist() == [[0, 0, 0, 1, 1, 1, 2]]
    with pytest.raises(ValueError):
        oracle.route_heads(e, 0.5, 0)


@pytest.mark.parametrize("seed", range(4))
def test_reduces_to_row_rule(seed):
    rng = np.random.default_rng(10 + seed)
    nB = int(rng.integers(1, 20))
    x = (rng.random((1, 5, nB, nB)) ** 3).astype(np.float32)
    p = float(rng.choice([0.3, 0.9, 0.99, 1.0]))
    row = _rows(oracle.select_contract(x, p, "row"))
    assert _rows(oracle.select_routed(x, p, -1.0, 3)) == row              # nothing routed
    assert _rows(oracle.select_routed(x, p, 2.0, 1)) == row               # every pool one head


def _brute_min_count_max_weight(w, T):
    n = len(w)
    for k in range(1, n + 1):
        best = max(sum(w[list(c)]) for c in itertools.combinations(range(n), k))
        if best >= T:
            return k, best
    return n, int(sum(w))


@pytest.mark.parametrize("seed", range(8))
def test_pools_brute_force(seed):
    rng = np.random.default_rng(200 + seed)
    H, nB = int(rng.integers(2, 5)), int(rng.integers(1, 5))
    group = int(rng.integers(2, H + 1))
    vals = np.array([0.0, 2.0 ** -12, 0.125, 0.25, 0.375, 0.5, 0.75, 1.0], dtype=np.float32)
    x = rng.choice(vals, size=(1, H, nB, nB)).astype(np.float32)
    p = float(rng.choice([0.25, 0.5, 0.7, 0.9]))
    rows = oracle.csr_rows(*oracle.select_routed(x, p, 2.0, group))
    w = np.floor(x.astype(np.float64) * 2.0 ** 32).astype(np.int64)
    pools = [list(range(s, min(s + group, H))) for s in range(0, H, group)]
    for members in pools:
        for i in range(nB):
            seg = np.concatenate([w[0, h, i] for h in members])
            T = oracle.threshold_fixed_point(p, int(seg.sum()))
            kept = [m * nB + int(j) for m, h in enumerate(members) for j in rows[h * nB + i]]
            k, best = _brute_min_count_max_weight(seg, T)
            assert len(kept) == max(k, 1)
            assert int(seg[kept].sum()) == best or (T == 0 and len(kept) == 1)
            # ties at the cut go to the lower flat index
            bits = np.concatenate([x[0, h, i] for h in members]).view(np.uint32)
            for a in kept:
                for b in range(len(seg)):
                    if b not in kept:
                        assert bits[b] < bits[a] or (bits[b] == bits[a] and b > a)


def test_pooled_mass_and_empty_rows():
    rng = np.random.default_rng(7)
    nB = 16
    z = rng.standard_normal((1, 6, nB, nB)) * np.array([6, 6, 6, 0.3, 0.3, 0.3])[None, :, None, None]
    x = np.exp(z - z.max(-1, keepdims=True))
    x = (x / x.sum(-1, keepdims=True)).astype(np.float32)       # rows sum to 1, like exact block masses
    e = oracle.head_entropy(x)
    assert (e[0, :3] < e[0, 3:].min()).all()                   # peaked heads have the lower entropy
    thr = float((e[0, :3].max() + e[0, 3:].min()) / 2)
    p = 0.9
    rows = oracle.csr_rows(*oracle.select_routed(x, p, thr, 3))
    for i in range(nB):
        kept = sum(float(x[0, h, i, rows[h * nB + i]].sum()) for h in range(3))
        assert kept >= p * float(x[0, :3, i].sum()) - 1e-6
    for h in range(3, 6):
        for i in range(nB):
            r = rows[h * nB + i]
            assert float(x[0, h, i, r].sum()) >= p * float(x[0, h, i].sum()) - 1e-6 and len(r) >= 1


def test_invalid_scores_rejected():
    x = np.full((1, 2, 3, 3), 0.25, dtype=np.float32)
    x[0, 1, 2, 0] = np.nan
    with pytest.raises(oracle.InvalidScores):
        oracle.select_routed(x, 0.5, 2.0, 2)
