"""GPU parity at the edges of the supported sizes and at degenerate token counts.

Maximum sizes: 4096 blocks a head for attention and head-scope selection,
1024 for row-scope selection, 1024 blocks (65,536 tokens) for the exact
scorer.  Degenerate inputs: a single token, a single partial block, exactly
one full block, one token past it.  Everything against the fp64 oracle with
the tolerances of the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import make_qkv, small_workload
from parity import assert_csr_equal, assert_out_close, assert_scores_close, gpu_csr, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    lbsa.lbsa_device_status(clear=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("n", [1, 7, 64, 65])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_degenerate_token_counts(n, dtype):
    """A grid of n tokens (1 x 1 x n): scores, selection and attention of the
    whole path, p = 0.99 row scope and the dense p = 1."""
    wl = small_workload(f"deg{n}", 1, 2, 64, (1, 1, n), 64, dtype=dtype, wid=400 + n)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores = lbsa.lbsa_score(q, k, 64)
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.block_mass(qh, kh, n, 64))
    for p in (0.99, 1.0):
        bs = lbsa.lbsa_select(scores, 64, p, "row")
        out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
        torch.cuda.synchronize()
        assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
        csr = gpu_csr(bs)
        assert_csr_equal(csr, oracle.select_contract(host(scores), p, "row"))
        ref_o, ref_l = oracle.sparse_attention(qh, kh, vh, n, 64, *csr)
        assert_out_close(host(out), ref_o[:, :, :n], q.dtype)
        tol = 1e-2 if dtype == "bf16" else 1e-5
        assert np.max(np.abs(host(lse) - ref_l[:, :, :n])) <= tol
    if n == 1:
        # one token attends to itself only: out = v
        assert np.max(np.abs(host(out) - vh)) <= (2e-2 if dtype == "bf16" else 1e-6)


def test_attention_at_4096_blocks():
    """nB = 4096 (262,144 tokens, 64-token blocks): the largest block count the
    attention kernel takes; random lists of up to 12 blocks, sampled query
    blocks against the oracle."""
    nB, block, d = 4096, 64, 64
    n = nB * block - 37                                   # ragged last block
    g = torch.Generator(device="cuda").manual_seed(41)
    q, k, v = (torch.randn(1, 1, n, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3))
    rng = np.random.default_rng(42)
    rows = [np.sort(rng.choice(nB, size=int(rng.integers(0, 13)), replace=False)) for _ in range(nB)]
    rows[nB - 1] = np.array([0, nB - 1])
    rp, col = oracle.csr_from_rows(rows)
    bs = lbsa.lbsa_blockset_from_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(), 1, 1, nB, block)
    out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
    qb = np.array([0, 1, 1777, 2048, nB - 2, nB - 1])
    ref_o, ref_l = oracle.sparse_attention(host(q), host(k), host(v), n, block, rp, col, qblocks=qb)
    rows_idx = np.concatenate([np.arange(i * block, min(i * block + block, n)) for i in qb])
    ref_rows = np.concatenate([np.arange(j * block, j * block + min(block, n - i * block))
                               for j, i in enumerate(qb)])
    assert_out_close(host(out)[:, :, rows_idx], ref_o[:, :, ref_rows], torch.bfloat16)
    gl, rl = host(lse)[:, :, rows_idx], ref_l[:, :, ref_rows]
    assert np.array_equal(np.isneginf(gl), np.isneginf(rl))
    fin = np.isfinite(rl)
    assert np.max(np.abs(gl[fin] - rl[fin])) <= 1e-2


def test_head_selection_at_4096_blocks():
    nB = 4096
    rng = np.random.default_rng(43)
    z = rng.standard_normal((1, 1, nB, nB)) * 2
    x = np.exp(z - z.max())
    x = (x / x.sum()).astype(np.float32)
    s = torch.from_numpy(x).cuda()
    for p in (0.25, 0.5):
        bs = lbsa.lbsa_select(s, 64, p, "head")
        assert_csr_equal(gpu_csr(bs), oracle.select_contract(x, p, "head"))
        assert lbsa.lbsa_get_status(bs) == 0


def test_row_selection_at_1024_blocks():
    nB = 1024
    rng = np.random.default_rng(44)
    x = rng.dirichlet(np.ones(nB) * 0.2, size=(1, 2, nB)).astype(np.float32)
    s = torch.from_numpy(x).cuda()
    for p in (0.5, 0.99):
        bs = lbsa.lbsa_select(s, 64, p, "row")
        assert_csr_equal(gpu_csr(bs), oracle.select_contract(x, p, "row"))
        assert lbsa.lbsa_get_status(bs) == 0


def test_exact_scores_at_1024_blocks():
    """65,536 tokens in one head (1024 blocks): the scorer's strips span 1024
    chunks; sampled query blocks of the masses against the oracle."""
    wl = small_workload("big", 1, 1, 128, (16, 64, 64), 64, dtype="bf16", wid=450)     # 65,536 tokens
    q, k, _ = make_qkv(wl, device="cuda")
    scores = lbsa.lbsa_score(q, k, 64)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    qb = [0, 511, 1023]
    ref = oracle.block_mass(host(q), host(k), wl.n_valid, 64, qblocks=qb)
    assert_scores_close(host(scores)[:, :, qb], ref)
    assert np.max(np.abs(host(scores).astype(np.float64).sum(-1) - 1.0)) < 1e-3
