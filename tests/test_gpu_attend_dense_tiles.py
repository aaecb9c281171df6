"""GPU parity of the dense-blockset attention path (two 128-row query tiles per
CTA, 128-key steps): p = 1 blocksets against the fp64 oracle's dense attention.

Shapes cover an odd number of query tiles (a CTA whose second tile is absent),
ragged last blocks, a step whose second 64-key half is empty (odd block count),
both block sizes, both head dims, batch > 1 and strided [B, N, H, d] views.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import make_qkv, small_workload
from parity import assert_out_close, host

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, d, grid, block
    ("t64_d128_odd_tiles", 1, 2, 128, (3, 9, 13), 64),     # 351 tokens: 6 blocks, 3 tiles, last block 31 valid
    ("t64_d128_one_tile", 2, 1, 128, (1, 5, 20), 64),      # 100 tokens: 2 blocks, 1 tile
    ("t64_d64_odd_blocks", 1, 3, 64, (4, 7, 11), 64),      # 308 tokens: 5 blocks (a half-empty last step)
    ("t128_d128_ragged", 1, 2, 128, (5, 9, 11), 128),      # 495 tokens: 4 blocks, last 111 valid
    ("t128_d64_odd_tiles", 2, 2, 64, (3, 8, 21), 128),     # 504 tokens: 4 blocks; 5 tiles of 128 rows (odd)
    ("t64_d128_many", 1, 1, 128, (8, 16, 33), 64),         # 4224 tokens: 66 blocks, 33 tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_dense_blockset_matches_dense_attention(case):
    name, B, H, d, grid, block = case
    wl = small_workload(name, B, H, d, grid, block, dtype="bf16", wid=170 + CASES.index(case))
    q, k, v = (x.cuda() for x in make_qkv(wl))
    nB = wl.n_blocks
    scores = torch.full((B, H, nB, nB), 1.0 / nB, device="cuda")
    bs = lbsa.lbsa_select(scores, block, 1.0, "row")
    out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0 and lbsa.lbsa_get_status(bs) == 0
    ref_o, ref_l = oracle.dense_attention(host(q), host(k), host(v), wl.n_valid)
    assert_out_close(host(out), ref_o, torch.bfloat16)
    assert np.max(np.abs(host(lse) - ref_l)) <= 1e-2


def test_dense_blockset_on_strided_view():
    """[B, N, H, d] storage viewed as [B, H, N, d]: the output keeps q's strides."""
    wl = small_workload("t_strided", 1, 3, 128, (3, 9, 13), 64, dtype="bf16", wid=190)
    q, k, v = (x.cuda().transpose(1, 2).contiguous().transpose(1, 2) for x in make_qkv(wl))
    nB = wl.n_blocks
    bs = lbsa.lbsa_select(torch.full((1, 3, nB, nB), 1.0 / nB, device="cuda"), 64, 1.0, "row")
    out = torch.empty_like(q)
    lbsa.lbsa_attend(q, k, v, bs, out=out)
    torch.cuda.synchronize()
    assert out.stride() == q.stride()
    ref_o, _ = oracle.dense_attention(host(q), host(k), host(v), wl.n_valid)
    assert_out_close(host(out), ref_o, torch.bfloat16)


def test_dense_and_sparse_paths_agree_on_a_full_list():
    """The same full lists through both attention kernels (the p = 1 blockset and
    a CSR import of it, which takes the 64-key kernel) agree within tolerance."""
    wl = small_workload("t_both", 1, 2, 128, (3, 9, 13), 64, dtype="bf16", wid=191)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    nB = wl.n_blocks
    dense = lbsa.lbsa_select(torch.full((1, 2, nB, nB), 1.0 / nB, device="cuda"), 64, 1.0, "row")
    rp, col = lbsa.lbsa_blockset_export(dense)
    imported = lbsa.lbsa_blockset_from_csr(rp, col, 1, 2, nB, 64)
    o1 = lbsa.lbsa_attend(q, k, v, dense)
    o2 = lbsa.lbsa_attend(q, k, v, imported)
    torch.cuda.synchronize()
    assert_out_close(host(o1), host(o2).astype(np.float64), torch.bfloat16)
