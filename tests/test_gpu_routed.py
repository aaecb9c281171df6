"""GPU parity of entropy-routed selection (EG-Sparse abstract, readsearch.ai page
of arXiv 2610.14672): head entropies against the fp64 oracle within the error
of fp32 logarithms, routing and index sets bit-exact (the oracle routes on the
GPU's entropies, so both sides take the floating-point decision on the same
values), and attention over the routed blockset."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, small_workload
from parity import assert_csr_equal, assert_out_close, gpu_csr, host

pytestmark = pytest.mark.gpu

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "select_routed_cases.json")))
# |E_gpu - E_oracle|: each fp32 logarithm is within a few ulp (relative 2.4e-7),
# and sum_j pi_j |ln x_j| / ln nB stays within a small multiple of 1 for these inputs
ENT_TOL = 2e-6


def _check(x, p, thr, group):
    s = torch.from_numpy(x).cuda()
    bs, ent, dom = lbsa.lbsa_select_routed(s, 64, p, thr, group)
    e = ent.cpu().numpy()
    np.testing.assert_allclose(e, oracle.head_entropy(x), rtol=0, atol=ENT_TOL)
    assert np.array_equal(dom.cpu().numpy(), oracle.route_heads(e, thr, group))
    assert_csr_equal(gpu_csr(bs), oracle.select_routed(x, p, thr, group, entropy=e))
    assert lbsa.lbsa_get_status(bs) == 0
    return bs, e, dom.cpu().numpy()


def test_golden_cases():
    x = np.asarray(GOLD["scores"], dtype=np.float32)[None]
    for c in GOLD["cases"]:
        bs, e, dom = _check(x, c["p"], c["threshold"], c["group"])
        np.testing.assert_allclose(e[0], GOLD["entropy"], rtol=0, atol=ENT_TOL)
        assert dom[0].tolist() == c["route"], c["why"]
        rp, col = gpu_csr(bs)
        assert [list(map(int, col[rp[r]:rp[r + 1]])) for r in range(len(rp) - 1)] == c["rows"], c["why"]


def _mixed_scores(B, H, nB, seed):
    """Heads alternate between peaked rows (low entropy), Dirichlet rows and
    rows of a few repeated values (ties across the members of a pool)."""
    rng = np.random.default_rng(seed)
    x = np.empty((B, H, nB, nB))
    for h in range(H):
        kind = h % 3
        if kind == 0:
            z = rng.standard_normal((B, nB, nB)) * 6
            r = np.exp(z - z.max(-1, keepdims=True))
        elif kind == 1:
            r = rng.dirichlet(np.ones(nB) * 0.5, size=(B, nB))
        else:
            r = rng.choice(np.array([0.0, 1 / 64, 1 / 32, 1 / 8]), size=(B, nB, nB))
            r[..., 0] += 1 / 64
        x[:, h] = r / r.sum(-1, keepdims=True)
    return x.astype(np.float32)


@pytest.mark.parametrize("nB", [1, 5, 33, 100, 512])
@pytest.mark.parametrize("group", [1, 2, 4, 64])
def test_random_bit_exact(nB, group):
    B, H = 2, 7
    x = _mixed_scores(B, H, nB, 500 + nB * 7 + group)
    e = oracle.head_entropy(x)
    thresholds = (-1.0, float(np.median(e)), 2.0) if nB <= 100 else (float(np.median(e)),)
    ps = (0.25, 0.9, 0.99, 1.0) if nB <= 100 else (0.9, 0.99)
    for thr in thresholds:
        for p in ps:
            _check(x, p, thr, group)


def test_invalid_scores_flag_their_domain():
    nB, H = 8, 4
    x = np.zeros((1, H, nB, nB), dtype=np.float32)
    for h in range(H):
        for i in range(nB):
            x[0, h, i, (i + h) % nB] = 1.0                   # one-hot rows: entropy 0
    x[0, 0, 2, 5] = 3.0                                      # >= 2 in a routed head: its pool's row 2
    x[0, 3, 4, 1] = np.nan                                   # NaN: entropy NaN, never routed
    s = torch.from_numpy(x).cuda()
    bs, ent, dom = lbsa.lbsa_select_routed(s, 64, 0.9, 0.5, 2)
    assert lbsa.lbsa_get_status(bs) == lbsa.LBSA_ERR_INVALID_SCORES
    e, d = ent.cpu().numpy()[0], dom.cpu().numpy()[0]
    assert np.isnan(e[3]) and d.tolist() == [0, 0, 1, -1]
    rp, col = gpu_csr(bs)
    rows = [list(map(int, col[rp[r]:rp[r + 1]])) for r in range(len(rp) - 1)]
    full = list(range(nB))
    assert rows[0 * nB + 2] == full and rows[1 * nB + 2] == full       # the pool's domain at row 2
    assert rows[3 * nB + 4] == full                                     # the NaN row, selected per row
    for h in range(H):                                                  # every other row: its one-hot block
        for i in range(nB):
            if (h, i) not in ((0, 2), (1, 2), (3, 4)):
                assert rows[h * nB + i] == [(i + h) % nB]


def test_pipeline_and_attention():
    """Exact scores of a small bf16 layer -> routed selection -> attention, against the oracle."""
    wl = small_workload("routed", 1, 4, 128, (4, 8, 12), 64, dtype="bf16", wid=150)   # 384 tokens, 6 blocks
    q, k, v = (t.cuda() for t in make_qkv(wl))
    scores = lbsa.lbsa_score(q, k, wl.block)
    sh = host(scores)
    thr = float(np.median(oracle.head_entropy(sh)))
    for p, group in ((0.5, 2), (0.9, 4)):
        bs, ent, dom = lbsa.lbsa_select_routed(scores, wl.block, p, thr, group)
        csr = gpu_csr(bs)
        assert_csr_equal(csr, oracle.select_routed(sh, p, thr, group, entropy=ent.cpu().numpy()))
        out = lbsa.lbsa_attend(q, k, v, bs)
        ref_o, _ = oracle.sparse_attention(host(q), host(k), host(v), wl.n_valid, wl.block, *csr)
        assert_out_close(host(out), ref_o[:, :, :wl.n_valid], torch.bfloat16)


def test_wan_skew_full_size():
    """The Wan-like layer with half its heads peaked: exact scores, routed
    selection at p = 0.99 with the median entropy as threshold, every row
    bit-exact, attention on sampled query blocks."""
    wl = get_workload("wan_skew")
    T, Hg, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, Hg, W, "3d", tile=(4, 4, 4), device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    scores = lbsa.lbsa_score(qp, kp, wl.block)
    sh = host(scores)
    e_ref = oracle.head_entropy(sh)
    thr = float(np.median(e_ref))
    nB = wl.n_blocks
    for group in (3, wl.H):
        bs, ent, dom = _check(sh, 0.99, thr, group)
        assert (dom >= 0).sum() >= 1
        if group == 3:
            op = lbsa.lbsa_attend(qp, kp, vp, bs)
            csr = gpu_csr(bs)
            for h in (0, 11):
                qh, kh, vh = (host(t[:, h:h + 1]) for t in (qp, kp, vp))
                a, b = csr[0][h * nB], csr[0][(h + 1) * nB]
                hrp, hcol = csr[0][h * nB:(h + 1) * nB + 1] - a, csr[1][a:b]
                ref_o, _ = oracle.sparse_attention(qh, kh, vh, wl.n_valid, wl.block, hrp, hcol, qblocks=[42])
                got = host(op[:, h:h + 1, 42 * wl.block:43 * wl.block])
                assert_out_close(got, ref_o[:, :, :wl.block], torch.bfloat16)
