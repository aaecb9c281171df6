"""The algorithmic work bench.py divides by (its TFLOP/s and roofline figures
rest on it): attention FLOPs on kept block pairs and on kept (token, key block)
pairs, and the CSR-to-mask expansion, against brute-force loops over tokens and
closed forms.  No GPU."""
from types import SimpleNamespace

import numpy as np
import pytest

import bench
import oracle


def _wl(H, n_valid, d=64, block=64, B=1):
    return SimpleNamespace(B=B, H=H, n_valid=n_valid, d=d, block=block, n_blocks=-(-n_valid // block))


def _valid(wl):
    return [min(wl.block, wl.n_valid - j * wl.block) for j in range(wl.n_blocks)]


@pytest.mark.parametrize("seed", range(5))
def test_attention_flops_brute_force(seed):
    rng = np.random.default_rng(seed)
    wl = _wl(H=3, n_valid=int(rng.integers(1, 700)), d=int(rng.choice([64, 128])), block=int(rng.choice([64, 128])))
    nB = wl.n_blocks
    m = (rng.random((wl.H, nB, nB)) < 0.4).astype(np.float64)
    v = _valid(wl)
    want = 0
    for h in range(wl.H):
        for i in range(nB):
            for j in range(nB):
                if m[h, i, j]:
                    want += 4 * wl.d * v[i] * v[j]          # every valid query row times every valid key
    assert bench.attention_flops(m, nB, wl.block, wl.n_valid, wl.d) == want
    assert bench.attention_flops(m.reshape(-1, nB), nB, wl.block, wl.n_valid, wl.d) == want


def test_attention_flops_dense_closed_form():
    wl = _wl(H=2, n_valid=32760, d=128)
    nB = wl.n_blocks
    ones = np.ones((wl.H, nB, nB))
    assert bench.attention_flops(ones, nB, wl.block, wl.n_valid, wl.d) == 4.0 * wl.d * wl.n_valid ** 2 * wl.H


def test_kept_mask_from_csr():
    rng = np.random.default_rng(3)
    rows = [sorted(rng.choice(9, size=int(rng.integers(0, 10)), replace=False).tolist()) for _ in range(7)]
    rp, col = oracle.csr_from_rows(rows)
    m = bench.kept_mask(rp, col, 7, 9)
    for r, c in enumerate(rows):
        assert [j for j in range(9) if m[r, j]] == c


def _token_layout(keep, wl):
    """Library layout of a per-token blockset from keep[g, r, j] (token r of
    head g keeps key block j): per (g, query block) the ascending key blocks
    kept by at least one of its tokens, each with its 64-bit token set."""
    G, nB = keep.shape[0], wl.n_blocks
    counts = np.zeros(G * nB, dtype=np.int64)
    cols = np.zeros((G * nB, nB), dtype=np.int64)
    masks = np.zeros((G * nB, nB), dtype=np.uint64)
    for g in range(G):
        for qb in range(nB):
            r = g * nB + qb
            toks = range(qb * 64, min((qb + 1) * 64, wl.n_valid))
            for j in range(nB):
                bits = 0
                for t in toks:
                    if keep[g, t, j]:
                        bits |= 1 << (t - qb * 64)
                if bits:
                    cols[r, counts[r]] = j
                    masks[r, counts[r]] = np.uint64(bits)
                    counts[r] += 1
    return counts, cols, masks


@pytest.mark.parametrize("seed", range(4))
def test_token_flops_brute_force(seed):
    rng = np.random.default_rng(10 + seed)
    wl = _wl(H=2, n_valid=int(rng.integers(65, 400)), d=128)
    nB = wl.n_blocks
    keep = rng.random((wl.H, wl.n_valid, nB)) < 0.2
    keep[0, :5] = False                                        # tokens that keep nothing
    v = _valid(wl)
    fl_want = sum(4 * wl.d * v[j] for g in range(wl.H) for t in range(wl.n_valid) for j in range(nB) if keep[g, t, j])
    dens_want = keep.sum() / (wl.H * wl.n_valid * nB)
    empty_want = float((~keep.any(axis=2)).mean())
    fl, dens, empty = bench.token_flops_of(*_token_layout(keep, wl), wl)
    assert fl == fl_want
    assert abs(dens - dens_want) < 1e-15 and abs(empty - empty_want) < 1e-15


def test_token_flops_closed_forms():
    wl = _wl(H=1, n_valid=130, d=64)
    nB = wl.n_blocks
    everything = np.ones((1, wl.n_valid, nB), dtype=bool)
    fl, dens, empty = bench.token_flops_of(*_token_layout(everything, wl), wl)
    assert fl == 4.0 * wl.d * wl.n_valid ** 2 and dens == 1.0 and empty == 0.0
    nothing = np.zeros((1, wl.n_valid, nB), dtype=bool)
    assert bench.token_flops_of(*_token_layout(nothing, wl), wl) == (0.0, 0.0, 1.0)


def test_median_entropy_threshold():
    assert bench.median_entropy(np.array([0.9, 0.1, 0.5, 0.3])) == 0.4
    assert bench.median_entropy(np.array([0.9, 0.1, 0.5])) == 0.5
    e = np.array([0.39, 0.94, 0.52, 0.83, 0.70, 0.41, 0.9998, 0.9995, 0.9998, 0.9998, 0.9995, 0.9997])
    thr = bench.median_entropy(e)
    assert (e < thr).sum() == 6                           # half the heads pooled


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    # profiles/traffic.json holds ncu DRAM bytes with a hash of the kernel's
    # source files; a changed source must turn the figure into None (null in
    # the bench line), an unchanged one must give the stored bytes
    import json
    import os
    import shutil
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    name = next(k for k, v in d.items() if isinstance(v, dict) and "source_hash" in v and bench.load_traffic(k))
    files = d[name]["files"]
    (tmp_path / "profiles").mkdir()
    shutil.copy(os.path.join(bench.ROOT, "profiles", "traffic.json"), tmp_path / "profiles" / "traffic.json")
    csrc = tmp_path / "block_sparse_attention_16_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in files:
        shutil.copy(os.path.join(bench.ROOT, "block_sparse_attention_16_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = bench.load_traffic(name)
    assert before == d[name]["bytes"]
    with open(csrc / files[0], "a") as fh:
        fh.write("\n// edited\n")
    assert bench.load_traffic(name) is None
    assert bench.load_traffic("no such kernel") is None
    # the stored figure comes back exactly when the sources are the ones hashed
    with open(csrc / files[0], "rb") as fh:
        data = fh.read()
    with open(csrc / files[0], "wb") as fh:
        fh.write(data[: -len(b"\n// edited\n")])
    assert bench.load_traffic(name) == before
