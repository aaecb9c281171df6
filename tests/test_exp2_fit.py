"""Provenance of the FMA-pipe exp2 polynomials in csrc/lbsa_device.cuh (no GPU).

Both polynomials approximate 2^f on [-1/2, 1/2] after round-to-nearest range
reduction.  Their coefficients come from a minimax fit of the relative error,
computed by iteratively reweighted least squares (Lawson's algorithm) on
Chebyshev nodes.  This test parses the shipped fp32 coefficients out of the
header, redoes the fit in fp64, and checks that (1) the shipped coefficients
are that fit, rounded to fp32, and (2) their worst relative error over a dense
grid stays within the bound each function's comment states.
"""
import os
import re

import numpy as np
import pytest

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "block_sparse_attention_16_b200", "csrc", "lbsa_device.cuh")


def _coefficients(fn: str):
    src = open(HEADER).read()
    body = src[re.search(r"__device__ __forceinline__ \w+(?: \w+)* " + fn + r"\(", src).start():]
    body = body[:body.index("\n}\n")]
    # Horner chain, from the line that starts q: the leading coefficient comes
    # first, then the addends in order (the packed form writes each literal twice,
    # once per lane)
    body = body[re.search(r"(unsigned long long|float) q =", body).start():]
    lits = [float(x) for x in re.findall(r"(?<![\w.])(-?[0-9]+\.[0-9]+(?:e[+-]?[0-9]+)?)f", body)]
    if "f2_as_u64" in body:
        lits = lits[::2]
    return np.array(lits[::-1])                      # c0 .. cn


def _fit(deg: int, n: int = 4001, iters: int = 400):
    k = np.arange(n)
    x = 0.5 * np.cos(np.pi * (k + 0.5) / n)          # Chebyshev nodes on [-1/2, 1/2]
    A = np.vander(x, deg + 1, increasing=True) / np.exp2(x)[:, None]
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        e = np.abs(A @ c - 1.0)
        w = w * e
        w /= w.sum()
    return c


@pytest.mark.parametrize("fn,deg,bound", [("exp2_poly2", 4, 2.7e-6), ("exp2_poly3", 3, 8.0e-5)])
def test_shipped_coefficients_are_the_minimax_fit(fn, deg, bound):
    shipped = _coefficients(fn)
    assert shipped.shape == (deg + 1,)
    refit = _fit(deg)
    assert np.allclose(shipped, refit.astype(np.float32).astype(np.float64), rtol=2e-6, atol=1e-8), (shipped, refit)
    x = np.linspace(-0.5, 0.5, 400001)
    rel = np.abs(np.polyval(shipped[::-1], x) / np.exp2(x) - 1.0).max()
    assert rel <= bound, rel
    # the fit is (near) equioscillating: the error at the interval ends is close to the maximum
    ends = np.abs(np.polyval(shipped[::-1], np.array([-0.5, 0.5])) / np.exp2([-0.5, 0.5]) - 1.0)
    assert ends.min() > 0.5 * rel
