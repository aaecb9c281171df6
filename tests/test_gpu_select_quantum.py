"""Selection at the 2^-32 quantum on the GPU, through every block scope.

The selection contract weighs a score x by w = floor(x * 2^32).  Scores below
2^-9 have fp32 bits finer than 2^-32, so their x * 2^32 has a fractional part.
Here every score other than the planted ones is k * 2^-34 with k in 0..3:
weight floor(k / 4) = 0, but 1 under rounding (k = 3) or a ceiling (k >= 1).
Each segment (a row, a head, a pool row) then holds a few planted 0.25 scores,
and p = 0.5.  With floored weights, W is exactly the planted mass and the
cut falls exactly on a planted score.  Any other weight moves the threshold
one quantum higher and keeps one more planted score.  So the kept counts
below hold only for floored weights.  Beside the counts, each case must be
bit-exact against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from parity import assert_csr_equal, gpu_csr

pytestmark = pytest.mark.gpu

QUARTER = np.float32(0.25)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _background(rng, shape):
    x = (rng.integers(0, 4, size=shape) * 2.0 ** -34).astype(np.float32)
    assert np.all(np.floor(x.astype(np.float64) * 2.0 ** 32) == 0) and np.any(x == np.float32(3 * 2.0 ** -34))
    return x


def _plant_rows(rng, x, per_row):
    """per_row planted 0.25 scores at distinct random columns of every row."""
    B, H, nQ, nB = x.shape
    for b in range(B):
        for h in range(H):
            for i in range(nQ):
                x[b, h, i, rng.choice(nB, size=per_row, replace=False)] = QUARTER
    return x


def _counts(csr):
    return np.diff(csr[0])


@pytest.mark.parametrize("nB", [3, 40, 512, 1100])
def test_row_scope_floors_fractional_weights(nB):
    # two planted scores a row: floored weights keep the first alone
    rng = np.random.default_rng(700 + nB)
    B, H = 1, (2 if nB <= 512 else 1)
    x = _plant_rows(rng, _background(rng, (B, H, nB, nB)), 2)
    bs = lbsa.lbsa_select(torch.from_numpy(x).cuda(), 64, 0.5, "row")
    got = gpu_csr(bs)
    assert np.all(_counts(got) == 1)
    assert_csr_equal(got, oracle.select_contract(x, 0.5, "row"))
    assert lbsa.lbsa_get_status(bs) == 0


@pytest.mark.parametrize("nB", [24, 600])
def test_head_scope_floors_fractional_weights(nB):
    # two planted scores a head (flat positions): floored weights keep the first alone;
    # nB = 24 takes the one-launch cluster path, nB = 600 the multi-launch radix path
    rng = np.random.default_rng(800 + nB)
    B, H = 2, 2
    x = _background(rng, (B, H, nB, nB))
    for b in range(B):
        for h in range(H):
            flat = rng.choice(nB * nB, size=2, replace=False)
            x[b, h].reshape(-1)[flat] = QUARTER
    bs = lbsa.lbsa_select(torch.from_numpy(x).cuda(), 64, 0.5, "head")
    got = gpu_csr(bs)
    assert np.all(_counts(got).reshape(B * H, nB).sum(1) == 1)
    assert_csr_equal(got, oracle.select_contract(x, 0.5, "head"))
    assert lbsa.lbsa_get_status(bs) == 0


def test_topp_floor_rule_floors_fractional_weights():
    # the row rule keeps one block a row, so the head's floor is 1 and nothing grows
    rng = np.random.default_rng(900)
    nB = 48
    x = _plant_rows(rng, _background(rng, (1, 3, nB, nB)), 2)
    bs = lbsa.lbsa_select_rule(torch.from_numpy(x).cuda(), 64, "topp_floor", n_valid=nB * 64, p=0.5)
    got = gpu_csr(bs)
    assert np.all(_counts(got) == 1)
    assert_csr_equal(got, oracle.select_topp_floor(x, 0.5, nB * 64, 64))


def test_routed_pools_floor_fractional_weights():
    # every head routed (threshold above any normalised entropy), pools of two heads:
    # a pool row holds four planted scores, and floored weights keep the first two
    rng = np.random.default_rng(901)
    nB, H = 40, 4
    x = _plant_rows(rng, _background(rng, (1, H, nB, nB)), 2)
    bs, ent, dom = lbsa.lbsa_select_routed(torch.from_numpy(x).cuda(), 64, 0.5, 2.0, 2)
    got = gpu_csr(bs)
    c = _counts(got).reshape(H, nB)
    assert np.all(c[0::2] + c[1::2] == 2)
    assert dom.cpu().numpy().tolist() == [[0, 0, 1, 1]]
    assert_csr_equal(got, oracle.select_routed(x, 0.5, 2.0, 2, entropy=ent.cpu().numpy()))
