"""GPU parity of the fused dense step: dense attention + exact block masses in one sweep."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, small_workload
from parity import assert_csr_equal, assert_out_close, assert_scores_close, gpu_csr, host

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, d, grid, block
    ("f64_d128_ragged", 2, 2, 128, (3, 8, 12), 64),     # 288 tokens, 5 blocks, last 32 valid
    ("f128_d128_ragged", 1, 3, 128, (4, 9, 10), 128),   # 360 tokens, 3 blocks, last 104 valid
    ("f64_d64_ragged", 1, 2, 64, (5, 6, 7), 64),        # 210 tokens, 4 blocks, last 18 valid
    ("f128_d64_odd", 2, 1, 64, (3, 7, 31), 128),        # 651 tokens, 6 blocks, last 11 valid (a half-empty last step)
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_fused_dense_step_matches_oracle(case):
    name, B, H, d, grid, block = case
    wl = small_workload(name, B, H, d, grid, block, dtype="bf16", wid=150 + CASES.index(case))
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores, out, lse = lbsa.lbsa_score_attend(q, k, v, block, want_lse=True)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.block_mass(qh, kh, wl.n_valid, block))
    ref_o, ref_l = oracle.dense_attention(qh, kh, vh, wl.n_valid)
    assert_out_close(host(out), ref_o, torch.bfloat16)
    assert np.max(np.abs(host(lse) - ref_l)) <= 1e-2
    # the masses drive the same selection as the scorer's (bit-exact contract on these scores)
    bs = lbsa.lbsa_select(scores, block, 0.9, "row")
    assert_csr_equal(gpu_csr(bs), oracle.select_contract(host(scores), 0.9, "row"))


def test_fused_dense_step_many_key_blocks():
    """128-token blocks, nB = 153 > 128 (each mass thread takes two key blocks),
    ragged last block: every mass against the exact scorer, sampled query blocks
    against the fp64 oracle, O against attention over the dense blockset."""
    wl = small_workload("f128_nb153", 1, 2, 128, (5, 30, 130), 128, dtype="bf16", wid=161)   # 19500 tokens
    assert wl.n_blocks == 153
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores, out = lbsa.lbsa_score_attend(q, k, v, wl.block)
    ref_scores = lbsa.lbsa_score(q, k, wl.block)
    ref_out = lbsa.lbsa_attend(q, k, v, lbsa.lbsa_select(ref_scores, wl.block, 1.0, "row"))
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    assert_scores_close(host(scores), host(ref_scores))
    assert_out_close(host(out), host(ref_out), torch.bfloat16)
    sc = host(scores)
    for h, qb in ((0, 0), (1, 77), (1, 152)):
        ref = oracle.block_mass(host(q[:, h:h + 1]), host(k[:, h:h + 1]), wl.n_valid, wl.block, qblocks=[qb])
        assert_scores_close(sc[:, h:h + 1, qb:qb + 1], ref)


def test_fused_dense_step_on_the_wan_layer():
    """Full Wan-like layer: masses agree with the scorer's; O agrees with attention over
    the dense blockset (a different kernel, so within the bf16 tolerance, not bit for bit)
    and with the fp64 oracle on sampled rows."""
    wl = get_workload("wan")
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    scores, out = lbsa.lbsa_score_attend(qp, kp, vp, wl.block)
    ref_scores = lbsa.lbsa_score(qp, kp, wl.block)
    dense = lbsa.lbsa_select(ref_scores, wl.block, 1.0, "row")
    ref_out = lbsa.lbsa_attend(qp, kp, vp, dense)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    assert_scores_close(host(scores), host(ref_scores))
    assert_out_close(host(out), host(ref_out), torch.bfloat16)
    rows = np.array([0, 1, 4095, 20000, wl.n_valid - 1])
    for h in (0, 7):
        sl = slice(h, h + 1)
        ref_o, _ = oracle.dense_attention(host(qp[:, sl]), host(kp[:, sl]), host(vp[:, sl]), wl.n_valid, rows=rows)
        assert_out_close(host(out[:, sl, rows]), ref_o, torch.bfloat16)
        assert_out_close(host(ref_out[:, sl, rows]), ref_o, torch.bfloat16)
    # sampled query blocks against the fp64 oracle directly
    sc = host(scores)
    for h, qb in ((0, 0), (5, 211), (11, wl.n_blocks - 1)):
        ref = oracle.block_mass(host(qp[:, h:h + 1]), host(kp[:, h:h + 1]), wl.n_valid, wl.block, qblocks=[qb])
        assert_scores_close(sc[:, h:h + 1, qb:qb + 1], ref)
