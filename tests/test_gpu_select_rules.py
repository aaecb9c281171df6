"""GPU parity of the Local + TopK and top-p-with-per-head-floor selection rules."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import make_qkv, small_workload
from parity import assert_csr_equal, assert_out_close, gpu_csr, host

pytestmark = pytest.mark.gpu


def _scores(kind, nB, H, seed):
    rng = np.random.default_rng(seed)
    if kind == "dirichlet":
        x = rng.dirichlet(np.ones(nB) * 0.3, size=(1, H, nB))
    elif kind == "ties":
        x = rng.choice(np.array([0.0, 1 / 64, 1 / 32, 3 / 64, 1 / 8]), size=(1, H, nB, nB))
    else:
        z = rng.standard_normal((1, H, nB, nB)) * 6
        x = np.exp(z - z.max(-1, keepdims=True))
        x /= x.sum(-1, keepdims=True)
    return x.astype(np.float32)


@pytest.mark.parametrize("nB", [1, 5, 33, 100, 512, 929])
@pytest.mark.parametrize("kind", ["dirichlet", "ties", "peaked"])
def test_local_topk_bit_exact(nB, kind):
    x = _scores(kind, nB, 3, 300 + nB)
    s = torch.from_numpy(x).cuda()
    ks = (0, 2, 6, 18, nB - 1, nB + 4) if nB <= 100 else (2, 18)
    for k in ks:
        if k < 0:
            continue
        bs = lbsa.lbsa_select_rule(s, 64, "local_topk", n_valid=nB * 64, k=k)
        assert_csr_equal(gpu_csr(bs), oracle.select_local_topk(x, k))
        assert lbsa.lbsa_get_status(bs) == 0


@pytest.mark.parametrize("nB", [1, 5, 33, 100, 512, 929])
@pytest.mark.parametrize("kind", ["dirichlet", "ties", "peaked"])
def test_topp_floor_bit_exact(nB, kind):
    x = _scores(kind, nB, 3, 400 + nB)
    s = torch.from_numpy(x).cuda()
    cases = ((64, 64), (64, 17), (128, 1)) if nB <= 100 else ((64, 17),)
    for block, tail in cases:
        n_valid = (nB - 1) * block + tail
        for p in ((0.25, 0.9, 0.99) if nB <= 100 else (0.9,)):
            bs = lbsa.lbsa_select_rule(s, block, "topp_floor", n_valid=n_valid, p=p)
            assert_csr_equal(gpu_csr(bs), oracle.select_topp_floor(x, p, n_valid, block))
            assert lbsa.lbsa_get_status(bs) == 0


def test_rules_on_the_pipeline_and_attention():
    """Exact scores of a small bf16 layer -> each rule -> attention, against the oracle."""
    wl = small_workload("rules", 1, 2, 128, (4, 8, 12), 64, dtype="bf16", wid=140)   # 384 tokens, 6 blocks
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores = lbsa.lbsa_score(q, k, wl.block)
    sh = host(scores)
    for bs, ref in ((lbsa.lbsa_select_rule(scores, wl.block, "local_topk", n_valid=wl.n_valid, k=2),
                     oracle.select_local_topk(sh, 2)),
                    (lbsa.lbsa_select_rule(scores, wl.block, "topp_floor", n_valid=wl.n_valid, p=0.5),
                     oracle.select_topp_floor(sh, 0.5, wl.n_valid, wl.block))):
        csr = gpu_csr(bs)
        assert_csr_equal(csr, ref)
        out = lbsa.lbsa_attend(q, k, v, bs)
        ref_o, _ = oracle.sparse_attention(host(q), host(k), host(v), wl.n_valid, wl.block, *csr)
        assert_out_close(host(out), ref_o[:, :, :wl.n_valid], torch.bfloat16)


def test_rule_arguments_are_validated():
    s = torch.full((1, 1, 4, 4), 0.25, device="cuda")
    with pytest.raises(lbsa.LbsaError):
        lbsa.lbsa_select_rule(s, 64, "topp_floor", n_valid=300, p=0.5)        # past the block grid
    with pytest.raises(lbsa.LbsaError):
        lbsa.lbsa_select_rule(s, 64, "topp_floor", n_valid=192, p=0.5)        # short of the last block
    with pytest.raises(lbsa.LbsaError):
        lbsa.lbsa_select_rule(s, 64, "local_topk", n_valid=256, k=-1)
    with pytest.raises(lbsa.LbsaError):
        lbsa.lbsa_select_rule(s, 64, "topp_floor", n_valid=256, p=0.0)
