"""GPU parity of the per-token proxy path (VMoBA's literal scoring): every
query token scores the key-block means, head-scope threshold selection over a
head's (token, key block) pairs, attention of each token over its own kept
blocks.  Scores against the fp64 oracle within the score tolerance; the
token lists bit for bit against the oracle's selector run on the GPU's own
scores; outputs within the bf16 / fp32 output tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, small_workload
from parity import assert_csr_equal, assert_out_close, assert_scores_close, host

pytestmark = pytest.mark.gpu

TAU = 0.25


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    lbsa.lbsa_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def token_csr(bs, n_valid, heads=None):
    """Per-token CSR of a per-token blockset (rows (b*H + h)*n_valid + t over
    the heads g in `heads`), checking its block-level structure on the way:
    ascending ids and a non-empty token set per listed entry."""
    counts, cols = (x.cpu().numpy() for x in lbsa.lbsa_blockset_views(bs))
    masks = lbsa.lbsa_blockset_masks(bs).cpu().numpy().view(np.uint64)
    nB = bs.nB
    heads = range(bs.B * bs.H) if heads is None else heads
    rows = []
    for g in heads:
        for i in range(nB):
            r = g * nB + i
            c = int(counts[r])
            ids, ms = cols[r, :c], masks[r, :c]
            assert np.all(np.diff(ids) > 0) and np.all(ms != 0)
            t0, t1 = i * 64, min(i * 64 + 64, n_valid)
            bits = (ms[None, :] >> np.arange(t1 - t0, dtype=np.uint64)[:, None]) & np.uint64(1)
            assert not np.any(ms >> np.uint64(t1 - t0)) if t1 - t0 < 64 else True
            rows.extend(ids[bits[u].astype(bool)] for u in range(t1 - t0))
    return oracle.csr_from_rows(rows)


def _run(q, k, v, block=64):
    scores = lbsa.lbsa_score(q, k, block, mode="meanpool_token")
    bs = lbsa.lbsa_select_tokens(scores, block, TAU)
    out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0 and lbsa.lbsa_get_status(bs) == 0
    return scores, bs, out, lse


CASES = [
    ("bf16_d128", 1, 3, 128, (3, 8, 12), "bf16"),        # 288 tokens, 5 blocks, last 32 valid
    ("bf16_d64_ragged", 2, 2, 64, (5, 6, 7), "bf16"),    # 210 tokens, 4 blocks, last 18 valid
    ("f32_d128_ragged", 1, 2, 128, (3, 5, 9), "f32"),    # 135 tokens, 3 blocks, last 7 valid
    ("f32_d64", 1, 2, 64, (4, 8, 8), "f32"),             # 256 tokens, 4 full blocks
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_token_proxy_pipeline_matches_oracle(case):
    name, B, H, d, grid, dtype = case
    wl = small_workload(name, B, H, d, grid, 64, dtype=dtype, wid=310 + CASES.index(case))
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores, bs, out, lse = _run(q, k, v)
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.token_meanpool_scores(qh, kh, wl.n_valid, 64))
    csr = token_csr(bs, wl.n_valid)
    assert_csr_equal(csr, oracle.select_contract(host(scores), TAU, "head"))
    ref_o, ref_l = oracle.token_sparse_attention(qh, kh, vh, wl.n_valid, 64, *csr)
    assert_out_close(host(out), ref_o, q.dtype)
    gl = host(lse)
    assert np.array_equal(np.isneginf(gl), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    assert np.max(np.abs(gl[fin] - ref_l[fin])) <= (1e-2 if dtype == "bf16" else 1e-5)
    empty = np.isneginf(ref_l)
    assert np.all(host(out)[empty] == 0)


@pytest.mark.parametrize("d", [128, 64])
def test_token_scores_over_several_chunks(d):
    """Tensor-core logits (bf16 token rows): 8,261 tokens (65 tiles of 128, the
    last 69 rows), nB = 130 key blocks (two chunks of 128, the second with 2
    valid columns; rows not a multiple of 4 floats): every score against the
    fp64 oracle, and the head-scope selection on them bit-exact."""
    wl = small_workload(f"tokchunks{d}", 1, 2, d, (11, 751, 1), 64, dtype="bf16", wid=330 + d)
    assert wl.n_blocks == 130
    q, k = (x.cuda() for x in make_qkv(wl)[:2])
    scores = lbsa.lbsa_score(q, k, 64, mode="meanpool_token")
    bs = lbsa.lbsa_select_tokens(scores, 64, TAU)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0 and lbsa.lbsa_get_status(bs) == 0
    sc = host(scores)
    assert_scores_close(sc, oracle.token_meanpool_scores(host(q), host(k), wl.n_valid, 64))
    assert_csr_equal(token_csr(bs, wl.n_valid), oracle.select_contract(sc, TAU, "head"))


def test_token_proxy_p1_keeps_every_pair_and_is_dense():
    wl = small_workload("tokdense", 1, 2, 128, (3, 8, 12), 64, dtype="bf16", wid=320)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores = lbsa.lbsa_score(q, k, 64, mode="meanpool_token")
    bs = lbsa.lbsa_select_tokens(scores, 64, 1.0)
    out = lbsa.lbsa_attend(q, k, v, bs)
    torch.cuda.synchronize()
    counts, _ = lbsa.lbsa_blockset_views(bs)
    assert torch.all(counts == bs.nB)
    ref_o, _ = oracle.dense_attention(host(q), host(k), host(v), wl.n_valid)
    assert_out_close(host(out), ref_o, torch.bfloat16)


def test_token_proxy_on_the_wan_proxy_layer():
    """Full Wan-like proxy shape (3D tiles): scores and token lists of two heads
    in full, outputs of sampled tokens."""
    wl = get_workload("wan_proxy")
    T, Hg, Wg = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, Hg, Wg, "3d", device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    scores, bs, out, _ = _run(qp, kp, vp)
    heads = [0, 7]
    qh, kh, vh = (host(x[:, heads]) for x in (qp, kp, vp))
    sc = host(scores[:, heads])
    assert_scores_close(sc, oracle.token_meanpool_scores(qh, kh, wl.n_valid, 64))
    csr = token_csr(bs, wl.n_valid, heads=heads)
    assert_csr_equal(csr, oracle.select_contract(sc, TAU, "head"))
    rng = np.random.default_rng(5)
    toks = np.sort(rng.choice(wl.n_valid, size=96, replace=False))
    rows = oracle.csr_rows(*csr)
    sub_rows = [rows[h * wl.n_valid + t] for h in range(2) for t in toks]
    ref_o, _ = oracle.token_sparse_attention(qh[:, :, toks], kh, vh, wl.n_valid, 64,
                                             *oracle.csr_from_rows(_scatter(sub_rows, len(toks), wl.n_valid)),
                                             tokens=np.arange(len(toks)))
    assert_out_close(host(out[:, heads][:, :, toks]), ref_o, torch.bfloat16)


def _scatter(sub_rows, n_tok, n_valid):
    """Rows for token_sparse_attention over a [B, 2, n_tok, d] query slice: the
    CSR is indexed (b*H + h)*n_valid + t, so pad each head to n_valid rows."""
    rows = []
    for h in range(2):
        rows.extend(sub_rows[h * n_tok:(h + 1) * n_tok])
        rows.extend(np.zeros(0, dtype=np.int64) for _ in range(n_valid - n_tok))
    return rows
