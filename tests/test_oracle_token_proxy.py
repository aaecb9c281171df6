"""Pins for the oracle's per-token proxy path (CPU): VMoBA's literal scoring,
where every query token scores every key-block mean, global selection over a
head's (token, key block) pairs, and attention over per-token block lists.

Each function is checked against something other than itself: torch routines,
the already-pinned block-granular functions through closed forms, dense
attention, and a brute-force selector written with Python integers.
"""
import math

import numpy as np
import torch

import oracle
from block_sparse_attention_16_b200.workload import make_qkv, small_workload


def _token_scores_by_torch(q, k, n_valid, block):
    """Key-block means by padding + masked sum, one matmul, softmax over the flattened head."""
    q = torch.as_tensor(np.asarray(q, dtype=np.float64))[:, :, :n_valid]
    k = torch.as_tensor(np.asarray(k, dtype=np.float64))[:, :, :n_valid]
    B, H, _, d = q.shape
    nB = -(-n_valid // block)
    kp = torch.zeros(B, H, nB * block, d, dtype=torch.float64)
    kp[:, :, :n_valid] = k
    cnt = torch.clamp(n_valid - torch.arange(nB) * block, max=block).to(torch.float64)
    kbar = kp.reshape(B, H, nB, block, d).sum(3) / cnt[None, None, :, None]
    s = q @ kbar.transpose(-1, -2) / math.sqrt(d)
    return torch.softmax(s.reshape(B, H, -1), dim=-1).reshape(B, H, n_valid, nB).numpy()


def test_token_scores_match_torch_with_ragged_tail():
    wl = small_workload("tok", 2, 2, 32, (3, 5, 7), 16, dtype="f32", wid=300)     # 105 tokens, 7 blocks
    q, k, _ = make_qkv(wl)
    s = oracle.token_meanpool_scores(q.numpy(), k.numpy(), wl.n_valid, 16)
    assert s.shape == (2, 2, 105, 7)
    assert np.max(np.abs(s - _token_scores_by_torch(q.numpy(), k.numpy(), wl.n_valid, 16))) < 1e-15
    assert np.max(np.abs(s.reshape(2, 2, -1).sum(-1) - 1.0)) < 1e-12


def test_token_scores_never_read_padding_rows():
    # rows at or past n_valid are padding: large values there change no score
    wl = small_workload("tok", 2, 2, 32, (3, 5, 7), 16, dtype="f32", wid=300)     # 105 tokens, 7 blocks
    q, k, _ = (x.numpy().astype(np.float64) for x in make_qkv(wl))
    pad = np.full((2, 2, 7, 32), 1e3)
    a = oracle.token_meanpool_scores(q, k, wl.n_valid, 16)
    b = oracle.token_meanpool_scores(np.concatenate([q, pad], 2), np.concatenate([k, -pad], 2), wl.n_valid, 16)
    assert np.array_equal(a, b)


def test_identical_tokens_reduce_to_block_means_over_block_size():
    # every query token of a (full) block equal to the block's mean: the token
    # score matrix repeats each block row `block` times, so it is the
    # block-granular proxy divided by the block size
    rng = np.random.default_rng(1)
    block, nB, d = 8, 5, 16
    qb = rng.standard_normal((1, 3, nB, d))
    q = np.repeat(qb, block, axis=2)
    k = rng.standard_normal((1, 3, nB * block, d))
    tok = oracle.token_meanpool_scores(q, k, nB * block, block)
    blk = oracle.meanpool_scores(q, k, nB * block, block)
    assert np.max(np.abs(tok - np.repeat(blk, block, axis=2) / block)) < 1e-15


def _block_csr_to_tokens(row_ptr, col, B, H, nB, block, n_valid):
    rows = []
    for b in range(B):
        for h in range(H):
            for t in range(n_valid):
                r = (b * H + h) * nB + t // block
                rows.append(np.asarray(col[row_ptr[r]:row_ptr[r + 1]]))
    return oracle.csr_from_rows(rows)


def test_token_attention_with_block_lists_equals_block_attention():
    wl = small_workload("tokatt", 1, 2, 32, (2, 5, 9), 16, dtype="f32", wid=301)   # 90 tokens, 6 blocks
    q, k, v = (x.numpy() for x in make_qkv(wl))
    nB = 6
    rng = np.random.default_rng(2)
    rows = [np.sort(rng.choice(nB, size=int(rng.integers(0, nB + 1)), replace=False)) for _ in range(2 * nB)]
    rp, col = oracle.csr_from_rows(rows)
    ref_o, ref_l = oracle.sparse_attention(q, k, v, wl.n_valid, 16, rp, col)
    trp, tcol = _block_csr_to_tokens(rp, col, 1, 2, nB, 16, wl.n_valid)
    o, l = oracle.token_sparse_attention(q, k, v, wl.n_valid, 16, trp, tcol)
    assert np.max(np.abs(o - ref_o[:, :, :wl.n_valid])) < 1e-13
    fin = np.isfinite(ref_l[:, :, :wl.n_valid])
    assert np.array_equal(np.isfinite(l), fin)
    assert np.max(np.abs(l[fin] - ref_l[:, :, :wl.n_valid][fin])) < 1e-13


def test_token_attention_full_lists_is_dense_and_empty_is_zero():
    wl = small_workload("tokd", 1, 1, 32, (2, 4, 9), 16, dtype="f32", wid=302)     # 72 tokens, 5 blocks
    q, k, v = (x.numpy() for x in make_qkv(wl))
    nB = 5
    rows = [np.arange(nB) if t % 3 else np.zeros(0, dtype=np.int64) for t in range(wl.n_valid)]
    rp, col = oracle.csr_from_rows(rows)
    o, l = oracle.token_sparse_attention(q, k, v, wl.n_valid, 16, rp, col)
    dense_o, dense_l = oracle.dense_attention(q, k, v, wl.n_valid)
    full = np.arange(wl.n_valid) % 3 != 0
    assert np.max(np.abs(o[0, 0, full] - dense_o[0, 0, full])) < 1e-13
    assert np.max(np.abs(l[0, 0, full] - dense_l[0, 0, full])) < 1e-13
    assert np.all(o[0, 0, ~full] == 0) and np.all(np.isneginf(l[0, 0, ~full]))


def test_token_attention_single_block_is_torch_sdpa_over_that_block():
    wl = small_workload("toks", 1, 1, 32, (2, 4, 9), 16, dtype="f32", wid=303)
    q, k, v = (x.numpy() for x in make_qkv(wl))
    rows = [np.array([(t * 7) % 5]) for t in range(wl.n_valid)]
    rp, col = oracle.csr_from_rows(rows)
    o, _ = oracle.token_sparse_attention(q, k, v, wl.n_valid, 16, rp, col)
    for t in (0, 13, 71):
        j = (t * 7) % 5
        keys = np.arange(j * 16, min(j * 16 + 16, wl.n_valid))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.as_tensor(q[0, 0, t:t + 1], dtype=torch.float64)[None],
            torch.as_tensor(k[0, 0, keys], dtype=torch.float64)[None],
            torch.as_tensor(v[0, 0, keys], dtype=torch.float64)[None])[0, 0].numpy()
        assert np.max(np.abs(o[0, 0, t] - ref)) < 1e-13


def test_token_rows_follow_batch_head_token_order_and_token_subset():
    # CSR row r = (b*H + h)*n_valid + t, one list per (batch, head, token)
    wl = small_workload("tokr", 2, 2, 16, (2, 4, 9), 16, dtype="f32", wid=306)   # 72 tokens, 5 blocks
    q, k, v = (x.numpy() for x in make_qkv(wl))
    B, H, n, nB = 2, 2, wl.n_valid, 5
    rng = np.random.default_rng(9)
    rows = [np.sort(rng.choice(nB, size=int(rng.integers(1, nB + 1)), replace=False)) for _ in range(B * H * n)]
    rp, col = oracle.csr_from_rows(rows)
    o, _ = oracle.token_sparse_attention(q, k, v, n, 16, rp, col)
    for b in range(B):
        for h in range(H):
            for t in (0, 17, 40, 71):
                keys = np.concatenate([np.arange(j * 16, min(j * 16 + 16, n)) for j in rows[(b * H + h) * n + t]])
                ref = torch.nn.functional.scaled_dot_product_attention(
                    torch.as_tensor(q[b, h, t:t + 1], dtype=torch.float64)[None],
                    torch.as_tensor(k[b, h, keys], dtype=torch.float64)[None],
                    torch.as_tensor(v[b, h, keys], dtype=torch.float64)[None])[0, 0].numpy()
                assert np.max(np.abs(o[b, h, t] - ref)) < 1e-13
    sub, _ = oracle.token_sparse_attention(q, k, v, n, 16, rp, col, tokens=[40, 3])
    assert np.array_equal(sub[:, :, 0], o[:, :, 40]) and np.array_equal(sub[:, :, 1], o[:, :, 3])


def _brute_head_select(x32, tau):
    """Fixed-point head selection written out with Python integers and sorted()."""
    flat = x32.reshape(-1)
    bits = flat.view(np.uint32).astype(np.int64)
    w = [math.floor(float(v) * 2 ** 32) for v in flat.astype(np.float64)]
    W = sum(w)
    P = round(tau * 2 ** 24)
    T = -((-(P * W)) // 2 ** 24)
    order = sorted(range(len(flat)), key=lambda i: (-int(bits[i]), i))
    acc, k = 0, len(flat)
    for pos, i in enumerate(order):
        acc += w[i]
        if acc >= T:
            k = pos + 1
            break
    return sorted(order[:max(k, 1)])


def test_token_head_selection_matches_integer_brute_force_and_bounds():
    wl = small_workload("toksel", 1, 2, 32, (2, 4, 9), 16, dtype="f32", wid=304)   # 72 tokens x 5 blocks
    q, k, _ = make_qkv(wl)
    s32 = oracle.token_meanpool_scores(q.numpy(), k.numpy(), wl.n_valid, 16).astype(np.float32)
    rp, col = oracle.select_contract(s32, 0.25, "head")
    nQ, nB = wl.n_valid, 5
    assert len(rp) == 2 * nQ + 1
    for h in range(2):
        kept = [(r - h * nQ) * nB + int(c) for r in range(h * nQ, (h + 1) * nQ) for c in col[rp[r]:rp[r + 1]]]
        assert kept == _brute_head_select(s32[0, h], 0.25)
        n = nQ * nB
        assert (len(kept) - 1) < 0.25 * n                 # kept count bound of global threshold selection
        got = float(s32[0, h].reshape(-1)[kept].astype(np.float64).sum())
        assert got >= 0.25 * float(s32[0, h].astype(np.float64).sum()) - n * 2.0 ** -32
