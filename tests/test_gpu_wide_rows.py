"""GPU parity of every selection rule on rows wider than 1024 key blocks (the
CTA-per-row path): nB = 1857, a HunyuanVideo-size grid (118,800 tokens) in
64-token blocks.  Index sets bit for bit against the oracle's selectors on the
same fp32 scores; ties, a zero-mass row and an invalid score included."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from parity import assert_csr_equal, gpu_csr

from test_gpu_routed import _mixed_scores
from test_gpu_token_proxy import token_csr

pytestmark = pytest.mark.gpu

NB = 1857                       # ceil(118800 / 64)
N_VALID = 118800


def _rows(H, seed, nB=NB):
    rng = np.random.default_rng(seed)
    x = np.empty((1, H, nB, nB))
    z = rng.standard_normal((H // 2, nB, nB)) * 5
    x[0, :H // 2] = np.exp(z - z.max(-1, keepdims=True))
    x[0, H // 2:] = rng.choice(np.array([0.0, 1 / 64, 1 / 32, 3 / 64, 1 / 8]), size=(H - H // 2, nB, nB))
    x[0, -1, 3] = 0.0                                 # a row with no mass at all
    x /= np.maximum(x.sum(-1, keepdims=True), 1e-30)
    return x.astype(np.float32)


def test_row_rule_bit_exact():
    x = _rows(2, 11)
    s = torch.from_numpy(x).cuda()
    for p in (0.5, 0.99, 1.0):
        bs = lbsa.lbsa_select(s, 64, p, "row")
        assert_csr_equal(gpu_csr(bs), oracle.select_contract(x, p, "row"))
        assert lbsa.lbsa_get_status(bs) == 0


def test_row_rule_flags_an_invalid_score():
    x = _rows(2, 12)
    x[0, 1, 7, 100] = np.nan
    bs = lbsa.lbsa_select(torch.from_numpy(x).cuda(), 64, 0.9, "row")
    rp, col = gpu_csr(bs)
    r = NB + 7
    assert lbsa.lbsa_get_status(bs) == lbsa.LBSA_ERR_INVALID_SCORES
    assert np.array_equal(col[rp[r]:rp[r + 1]], np.arange(NB))          # the row keeps every block
    clean = x.copy()
    clean[0, 1, 7] = 1.0 / NB
    want_rp, want_col = oracle.select_contract(clean, 0.9, "row")
    keep = np.ones(2 * NB, dtype=bool)
    keep[r] = False
    got_rows = [col[rp[i]:rp[i + 1]] for i in range(2 * NB) if keep[i]]
    want_rows = [want_col[want_rp[i]:want_rp[i + 1]] for i in range(2 * NB) if keep[i]]
    assert all(np.array_equal(a, b) for a, b in zip(got_rows, want_rows))


def test_rank_rules_bit_exact():
    x = _rows(2, 13)
    s = torch.from_numpy(x).cuda()
    for k in (2, 6, 18):
        bs = lbsa.lbsa_select_rule(s, 64, "local_topk", n_valid=N_VALID, k=k)
        assert_csr_equal(gpu_csr(bs), oracle.select_local_topk(x, k))
    for p in (0.5, 0.9):
        bs = lbsa.lbsa_select_rule(s, 64, "topp_floor", n_valid=N_VALID, p=p)
        assert_csr_equal(gpu_csr(bs), oracle.select_topp_floor(x, p, N_VALID, 64))
        assert lbsa.lbsa_get_status(bs) == 0


def test_routed_rule_bit_exact():
    x = _mixed_scores(1, 4, NB, 14)
    s = torch.from_numpy(x).cuda()
    e = oracle.head_entropy(x)
    thr = float(np.median(e))
    bs, ent, dom = lbsa.lbsa_select_routed(s, 64, 0.99, thr, 2)
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == 0
    assert_csr_equal(gpu_csr(bs), oracle.select_routed(x, 0.99, thr, 2, entropy=ent.cpu().numpy()))


def test_per_token_rule_bit_exact():
    """Per-token scope with 1100 key blocks (70,390 tokens): one head's token x
    block scores, softmax-like rows, head-scope threshold."""
    nB, n_valid = 1100, 1099 * 64 + 54
    rng = np.random.default_rng(15)
    z = rng.standard_normal((n_valid, nB)).astype(np.float32) * 3
    x = np.exp(z - z.max())
    x = (x / x.sum(dtype=np.float64)).astype(np.float32)[None, None]
    s = torch.from_numpy(x).cuda()
    bs = lbsa.lbsa_select_tokens(s, 64, 0.25)
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == 0
    assert_csr_equal(token_csr(bs, n_valid), oracle.select_contract(x, 0.25, "head"))
