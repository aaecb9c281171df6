"""Pins for oracle.attention against library routines and closed forms (CPU)."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, small_workload


def _sdpa64(q, k, v):
    """torch's own fp64 SDPA on CPU (a library routine, not the oracle's formula)."""
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()


def _tiny():
    wl = get_workload("tiny")
    q, k, v = make_qkv(wl)
    return wl, q.numpy(), k.numpy(), v.numpy()


def test_dense_matches_torch_sdpa_fp64():
    wl, q, k, v = _tiny()
    O, lse = oracle.dense_attention(q, k, v, wl.n_valid)
    ref = _sdpa64(q, k, v)
    assert np.max(np.abs(O - ref)) < 1e-12
    # lse against torch.logsumexp of the scaled logits
    z = torch.as_tensor(q, dtype=torch.float64) @ torch.as_tensor(k, dtype=torch.float64).transpose(-1, -2)
    ref_lse = torch.logsumexp(z / math.sqrt(wl.d), dim=-1).numpy()
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


def test_dense_rows_subset_returns_those_rows():
    wl, q, k, v = _tiny()
    O, lse = oracle.dense_attention(q, k, v, wl.n_valid)
    rows = [7, 2, wl.n_valid - 1]
    Os, ls = oracle.dense_attention(q, k, v, wl.n_valid, rows=rows)
    # (a matmul over fewer rows may round in another order: equal to 1e-14)
    assert np.max(np.abs(Os - O[:, :, rows])) < 1e-14 and np.max(np.abs(ls - lse[:, :, rows])) < 1e-14


def test_dense_equal_keys_gives_mean_of_values():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 1, 10, 16))
    k = np.tile(rng.standard_normal((1, 1, 1, 16)), (1, 1, 37, 1))
    v = rng.standard_normal((1, 1, 37, 16))
    O, lse = oracle.dense_attention(q, k, v, 37, rows=np.arange(10))
    assert np.allclose(O[0, 0], v[0, 0].mean(axis=0)[None, :], atol=1e-13)
    expect = np.log(37.0) + (q[0, 0] @ k[0, 0, 0]) / 4.0
    assert np.allclose(lse[0, 0], expect, atol=1e-12)


def test_dense_one_dominant_key_returns_its_value():
    d = 8
    q = np.zeros((1, 1, 1, d)); q[..., 0] = 100.0
    k = np.zeros((1, 1, 5, d)); k[0, 0, 3, 0] = 100.0
    v = np.arange(5 * d, dtype=np.float64).reshape(1, 1, 5, d)
    O, _ = oracle.dense_attention(q, k, v, 5, rows=[0])
    assert np.allclose(O[0, 0, 0], v[0, 0, 3], atol=1e-9)


def test_dense_ignores_padding_rows():
    wl, q, k, v = _tiny()
    nv = 200
    O1, l1 = oracle.dense_attention(q, k, v, nv)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, nv:] = 1e6
    v2[:, :, nv:] = np.nan
    O2, l2 = oracle.dense_attention(q, k2, v2, nv)
    assert np.array_equal(O1, O2) and np.array_equal(l1, l2)
    ref = _sdpa64(q[:, :, :nv], k[:, :, :nv], v[:, :, :nv])
    assert np.max(np.abs(O1 - ref)) < 1e-12


def _full_csr(B, H, nB):
    rows = [np.arange(nB) for _ in range(B * H * nB)]
    return oracle.csr_from_rows(rows)


def test_sparse_all_blocks_equals_dense():
    wl, q, k, v = _tiny()
    rp, col = _full_csr(wl.B, wl.H, wl.n_blocks)
    Os, ls = oracle.sparse_attention(q, k, v, wl.n_valid, wl.block, rp, col)
    Od, ld = oracle.dense_attention(q, k, v, wl.n_valid)
    assert np.max(np.abs(Os - Od)) < 1e-12 and np.max(np.abs(ls - ld)) < 1e-12


def test_sparse_single_block_is_softmax_over_that_block():
    wl, q, k, v = _tiny()
    nB, b = wl.n_blocks, wl.block
    rows = [np.array([(i * 3 + h) % nB]) for h in range(wl.H) for i in range(nB)]
    rp, col = oracle.csr_from_rows(rows)
    O, _ = oracle.sparse_attention(q, k, v, wl.n_valid, b, rp, col)
    for h in range(wl.H):
        for i in range(nB):
            j = (i * 3 + h) % nB
            ref = _sdpa64(q[:, h:h + 1, i * b:(i + 1) * b], k[:, h:h + 1, j * b:(j + 1) * b],
                          v[:, h:h + 1, j * b:(j + 1) * b])
            assert np.max(np.abs(O[:, h:h + 1, i * b:(i + 1) * b] - ref)) < 1e-12


def test_sparse_union_of_blocks_matches_sdpa_on_gathered_keys():
    wl = small_workload("t", 1, 1, 32, (3, 5, 7), 16, dtype="f32")   # 105 tokens, ragged tail
    q, k, v = (x.numpy() for x in make_qkv(wl))
    nB = wl.n_blocks
    rng = np.random.default_rng(3)
    rows = [np.sort(rng.choice(nB, size=rng.integers(1, nB + 1), replace=False)) for _ in range(nB)]
    rp, col = oracle.csr_from_rows(rows)
    O, _ = oracle.sparse_attention(q, k, v, wl.n_valid, wl.block, rp, col)
    for i in range(nB):
        keys = np.concatenate([np.arange(j * 16, min(j * 16 + 16, wl.n_valid)) for j in rows[i]])
        r1 = min(i * 16 + 16, wl.n_valid)
        ref = _sdpa64(q[:, :, i * 16:r1], k[:, :, keys], v[:, :, keys])
        assert np.max(np.abs(O[:, :, i * 16:r1] - ref)) < 1e-12
    # padded rows of the last block stay zero
    assert np.all(O[:, :, wl.n_valid:] == 0)


def test_sparse_rows_follow_batch_head_block_order_and_qblocks_subset():
    # CSR row r = (b*H + h)*nB + i: every (batch, head, query block) has its own
    # list here, so a row numbered any other way attends to the wrong keys
    wl = small_workload("t", 2, 3, 16, (2, 5, 7), 16, dtype="f32", wid=305)   # 70 tokens, 5 blocks
    q, k, v = (x.numpy() for x in make_qkv(wl))
    B, H, nB, blk = 2, 3, wl.n_blocks, 16
    rng = np.random.default_rng(8)
    rows = [np.sort(rng.choice(nB, size=int(rng.integers(1, nB + 1)), replace=False)) for _ in range(B * H * nB)]
    rp, col = oracle.csr_from_rows(rows)
    O, lse = oracle.sparse_attention(q, k, v, wl.n_valid, blk, rp, col)
    for b in range(B):
        for h in range(H):
            for i in range(nB):
                keys = np.concatenate([np.arange(j * blk, min(j * blk + blk, wl.n_valid))
                                       for j in rows[(b * H + h) * nB + i]])
                r0, r1 = i * blk, min(i * blk + blk, wl.n_valid)
                ref = _sdpa64(q[b:b + 1, h:h + 1, r0:r1], k[b:b + 1, h:h + 1, keys], v[b:b + 1, h:h + 1, keys])
                assert np.max(np.abs(O[b, h, r0:r1] - ref[0, 0])) < 1e-12
                z = torch.as_tensor(q[b, h, r0:r1], dtype=torch.float64) @ \
                    torch.as_tensor(k[b, h, keys], dtype=torch.float64).T
                ref_l = torch.logsumexp(z / math.sqrt(16), dim=-1).numpy()
                assert np.max(np.abs(lse[b, h, r0:r1] - ref_l)) < 1e-12
    # a subset of query blocks, in any order, returns those blocks' slices
    Os, ls = oracle.sparse_attention(q, k, v, wl.n_valid, blk, rp, col, qblocks=[4, 1])
    assert np.array_equal(Os[:, :, :blk], O[:, :, 4 * blk:5 * blk])
    assert np.array_equal(Os[:, :, blk:], O[:, :, blk:2 * blk])
    assert np.array_equal(ls[:, :, blk:], lse[:, :, blk:2 * blk])


def test_sparse_empty_row_outputs_zero_and_neg_inf_lse():
    wl, q, k, v = _tiny()
    nB = wl.n_blocks
    rows = [np.array([], dtype=np.int64) if i == 1 else np.arange(nB)
            for h in range(wl.H) for i in range(nB)]
    rp, col = oracle.csr_from_rows(rows)
    O, lse = oracle.sparse_attention(q, k, v, wl.n_valid, wl.block, rp, col)
    b = wl.block
    assert np.all(O[:, :, b:2 * b] == 0) and np.all(np.isneginf(lse[:, :, b:2 * b]))
    assert np.all(np.isfinite(lse[:, :, :b]))
