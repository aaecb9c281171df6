"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

Block scores and outputs are checked on sampled query blocks (each sample is a
full row sweep in the fp64 oracle); index sets are checked bit-exact on every
row; permutations are checked element by element.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, make_qkv_f32, redraw_qkv
from parity import assert_csr_equal, assert_out_close, assert_scores_close, gpu_csr, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    lbsa.lbsa_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def head_csr(rp, col, h, nB):
    """CSR rows of head h (batch 0) re-based to a one-head CSR."""
    a, b = rp[h * nB], rp[(h + 1) * nB]
    return rp[h * nB:(h + 1) * nB + 1] - a, col[a:b]


def check_sampled(q, k, v, scores, csr, wl, heads, qblocks, check_scores=True, out=None):
    nB = wl.n_blocks
    for h in heads:
        qh, kh, vh = (host(x[:, h:h + 1]) for x in (q, k, v))
        if check_scores:
            ref = oracle.block_mass(qh, kh, wl.n_valid, wl.block, qblocks=qblocks)
            assert_scores_close(host(scores[:, h:h + 1, qblocks]), ref)
        if out is not None:
            hrp, hcol = head_csr(csr[0], csr[1], h, nB)
            ref_o, _ = oracle.sparse_attention(qh, kh, vh, wl.n_valid, wl.block, hrp, hcol, qblocks=qblocks)
            got = np.concatenate([host(out[:, h:h + 1, i * wl.block:min((i + 1) * wl.block, wl.n_valid)])
                                  for i in qblocks], axis=2)
            want = np.concatenate([ref_o[:, :, n * wl.block:n * wl.block + min(wl.block, wl.n_valid - i * wl.block)]
                                   for n, i in enumerate(qblocks)], axis=2)
            assert_out_close(got, want, torch.bfloat16)


def test_wan_3d_exact_p099():
    wl = get_workload("wan")
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", tile=(4, 4, 4), device="cuda")
    assert np.array_equal(perm.cpu().numpy(), oracle.perm_3d_tiles(T, H, W, 4, 4, 4))
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    pl = perm.long()
    assert torch.equal(qp, q[:, :, pl]) and torch.equal(vp, v[:, :, pl])
    scores = lbsa.lbsa_score(qp, kp, wl.block)
    bs = lbsa.lbsa_select(scores, wl.block, 0.99, "row")
    op = lbsa.lbsa_attend(qp, kp, vp, bs)
    o = lbsa.lbsa_permute([op], perm, inverse=True)[0]
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0 and lbsa.lbsa_get_status(bs) == 0
    assert torch.equal(o[:, :, pl], op)
    csr = gpu_csr(bs)
    assert_csr_equal(csr, oracle.select_contract(host(scores), 0.99, "row"))
    nB = wl.n_blocks
    check_sampled(qp, kp, vp, scores, csr, wl, heads=[0, 5, 11], qblocks=[0, 137, nB - 1], out=op)
    check_sampled(qp, kp, vp, scores, csr, wl, heads=[3, 8], qblocks=[300, 301], out=op)
    density = (np.diff(csr[0]).sum()) / (wl.H * nB * nB)
    assert 0.0 < density <= 1.0


def test_wan_skew_p_sweep():
    wl = get_workload("wan_skew")
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", tile=(4, 4, 4), device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    scores = lbsa.lbsa_score(qp, kp, wl.block)
    sh = host(scores)
    check_sampled(qp, kp, vp, scores, None, wl, heads=[0, 11], qblocks=[5, wl.n_blocks - 1], out=None)
    nB = wl.n_blocks
    dens = []
    for p in wl.extra["p_sweep"]:
        bs = lbsa.lbsa_select(scores, wl.block, p, "row")
        op = lbsa.lbsa_attend(qp, kp, vp, bs)
        torch.cuda.synchronize()
        csr = gpu_csr(bs)
        assert_csr_equal(csr, oracle.select_contract(sh, p, "row"))
        if p in (0.9, 0.999):
            check_sampled(qp, kp, vp, scores, csr, wl, heads=[1, 10], qblocks=[42], check_scores=False, out=op)
        per_head = np.diff(csr[0]).reshape(wl.H, nB).sum(1) / (nB * nB)
        dens.append(per_head)
    dens = np.array(dens)
    assert np.all(np.diff(dens, axis=0) >= 0)          # density grows with p, per head


def test_wan_proxy_cycle_head_scope():
    wl = get_workload("wan_proxy")
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    nB = wl.n_blocks
    for call in range(3):
        kind = oracle.PARTITION_CYCLE[call % 3]
        perm = lbsa.lbsa_partition_perm(T, H, W, kind, tile=(4, 4, 4), frame_tile=(8, 8), device="cuda")
        assert np.array_equal(perm.cpu().numpy(), oracle.perm_for_call(call, T, H, W))
        qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
        scores = lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool")
        bs = lbsa.lbsa_select(scores, wl.block, 0.25, "head")
        op = lbsa.lbsa_attend(qp, kp, vp, bs)
        o = lbsa.lbsa_permute([op], perm, inverse=True)[0]
        torch.cuda.synchronize()
        assert lbsa.lbsa_get_status(bs) == 0
        sh = host(scores)
        assert_scores_close(sh, oracle.meanpool_scores(host(qp), host(kp), wl.n_valid, wl.block))
        csr = gpu_csr(bs)
        assert_csr_equal(csr, oracle.select_contract(sh, 0.25, "head"))
        counts = np.diff(csr[0]).reshape(wl.H, nB)
        assert np.all(counts.sum(1) - 1 < 0.25 * nB * nB)      # kept fraction bound of the global rule
        rows = [i for i in (0, nB // 2, nB - 1)]
        check_sampled(qp, kp, vp, scores, csr, wl, heads=[2, 9], qblocks=rows, check_scores=False, out=op)
        assert torch.equal(o[:, :, perm.long()], op)


def test_hunyuan_frozen_reuse():
    wl = get_workload("hunyuan")
    q32, k32, v32 = make_qkv_f32(wl, device="cuda")
    q, k, v = (x.to(torch.bfloat16) for x in (q32, k32, v32))
    scores = lbsa.lbsa_score(q, k, wl.block)
    bs = lbsa.lbsa_select(scores, wl.block, 0.99, "row")
    torch.cuda.synchronize()
    nB = wl.n_blocks
    csr = gpu_csr(bs)
    assert_csr_equal(csr, oracle.select_contract(host(scores), 0.99, "row"))
    check_sampled(q, k, v, scores, csr, wl, heads=[0, 23], qblocks=[nB - 1, 400], out=None)
    for t in range(1, wl.extra["steps"] + 1):
        q, k, v = redraw_qkv(wl, q32, k32, v32, t)
        out = lbsa.lbsa_attend(q, k, v, bs)
        if t in (1, 25, 49):
            torch.cuda.synchronize()
            check_sampled(q, k, v, scores, csr, wl, heads=[3, 7, 12, 16, 22], qblocks=[0, 401, nB - 1],
                          check_scores=False, out=out)
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
