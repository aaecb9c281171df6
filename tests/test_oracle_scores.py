"""Pins for oracle.scores (CPU): invariants, library routines, closed forms."""
import math

import numpy as np
import torch

import oracle
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, small_workload


def _mass_by_torch(q, k, n_valid, block):
    """Block-summed torch.softmax with a key mask, reshaped (independent route)."""
    q = torch.as_tensor(np.asarray(q, dtype=np.float64))
    k = torch.as_tensor(np.asarray(k, dtype=np.float64))
    B, H, S, d = q.shape
    nB = -(-n_valid // block)
    Sp = nB * block
    qp = torch.zeros(B, H, Sp, d, dtype=torch.float64); qp[:, :, :n_valid] = q[:, :, :n_valid]
    kp = torch.zeros(B, H, Sp, d, dtype=torch.float64); kp[:, :, :n_valid] = k[:, :, :n_valid]
    z = qp @ kp.transpose(-1, -2) / math.sqrt(d)
    z[..., n_valid:] = -torch.inf
    P = torch.softmax(z, dim=-1)
    rowmass = P.reshape(B, H, Sp, nB, block).sum(-1)            # [B,H,Sp,nB]
    valid = torch.zeros(Sp, dtype=torch.float64); valid[:n_valid] = 1
    rowmass = rowmass * valid[None, None, :, None]
    num = rowmass.reshape(B, H, nB, block, nB).sum(3)
    cnt = valid.reshape(nB, block).sum(1)
    return (num / cnt[None, None, :, None]).numpy()


def test_block_mass_rows_sum_to_one():
    wl = get_workload("tiny")
    q, k, _ = make_qkv(wl)
    m = oracle.block_mass(q.numpy(), k.numpy(), wl.n_valid, wl.block)
    assert m.shape == (1, 2, 4, 4)
    assert np.max(np.abs(m.sum(-1) - 1.0)) < 1e-12
    assert np.all(m >= 0)


def test_block_mass_matches_blocked_torch_softmax():
    wl = get_workload("tiny")
    q, k, _ = make_qkv(wl)
    m = oracle.block_mass(q.numpy(), k.numpy(), wl.n_valid, wl.block)
    assert np.max(np.abs(m - _mass_by_torch(q.numpy(), k.numpy(), wl.n_valid, wl.block))) < 1e-13


def test_block_mass_ragged_tail_matches_torch():
    wl = small_workload("t", 1, 2, 32, (3, 5, 7), 16, dtype="f32")      # 105 tokens, 7 blocks
    q, k, _ = make_qkv(wl)
    m = oracle.block_mass(q.numpy(), k.numpy(), wl.n_valid, wl.block)
    assert np.max(np.abs(m - _mass_by_torch(q.numpy(), k.numpy(), wl.n_valid, 16))) < 1e-13
    assert np.max(np.abs(m.sum(-1) - 1.0)) < 1e-12
    sub = oracle.block_mass(q.numpy(), k.numpy(), wl.n_valid, 16, qblocks=[6, 2])
    assert np.array_equal(sub, m[:, :, [6, 2]])


def test_block_mass_uniform_keys_is_block_fraction():
    # all keys equal -> every row attends uniformly -> mass = |J_j| / n_valid
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 1, 50, 8))
    k = np.tile(rng.standard_normal((1, 1, 1, 8)), (1, 1, 50, 1))
    m = oracle.block_mass(q, k, 50, 16)
    expect = np.array([16, 16, 16, 2]) / 50.0
    assert np.allclose(m[0, 0], expect[None, :], atol=1e-14)


def test_meanpool_identical_tokens_closed_form():
    # every token of a block equals one vector -> the block mean is that vector
    rng = np.random.default_rng(5)
    nB, b, d = 5, 4, 8
    qv = rng.standard_normal((nB, d)); kv = rng.standard_normal((nB, d))
    q = np.repeat(qv, b, axis=0)[None, None]
    k = np.repeat(kv, b, axis=0)[None, None]
    s = oracle.meanpool_scores(q, k, nB * b, b)[0, 0]
    logits = qv @ kv.T / math.sqrt(d)
    expect = np.exp(logits) / np.exp(logits).sum()
    assert np.max(np.abs(s - expect)) < 1e-14


def test_meanpool_matches_torch_pooling_and_softmax():
    wl = small_workload("t", 1, 2, 32, (3, 5, 7), 16, dtype="f32")
    q, k, _ = make_qkv(wl)
    s = oracle.meanpool_scores(q.numpy(), k.numpy(), wl.n_valid, 16)
    assert np.max(np.abs(s.sum(axis=(2, 3)) - 1.0)) < 1e-12
    qt, kt = q.double(), k.double()
    for h in range(2):
        bounds = [(j * 16, min(j * 16 + 16, wl.n_valid)) for j in range(wl.n_blocks)]
        qb = torch.stack([qt[0, h, a:e].mean(0) for a, e in bounds])
        kb = torch.stack([kt[0, h, a:e].mean(0) for a, e in bounds])
        ref = torch.softmax((qb @ kb.T).flatten() / math.sqrt(32), 0).reshape(len(bounds), -1)
        assert np.max(np.abs(s[0, h] - ref.numpy())) < 1e-14


def test_scores_never_read_padding_rows():
    # Arrays may be longer than n_valid (a buffer padded to whole blocks); rows
    # at or past n_valid are not tokens, so filling them with large values must
    # change no score: the ragged last block holds 9 of 16 tokens here.
    wl = small_workload("t", 1, 2, 32, (3, 5, 7), 16, dtype="f32")      # 105 tokens, 7 blocks
    q, k, _ = (x.numpy().astype(np.float64) for x in make_qkv(wl))
    pad = np.full((1, 2, 7, 32), 1e3)
    qp, kp = np.concatenate([q, pad], axis=2), np.concatenate([k, -pad], axis=2)
    assert qp.shape[2] == 112
    for fn in (oracle.block_mass, oracle.meanpool_scores):
        a = fn(q, k, wl.n_valid, 16)
        b = fn(qp, kp, wl.n_valid, 16)
        assert np.array_equal(a, b), fn.__name__


def test_meanpool_zero_keys_uniform():
    q = np.random.default_rng(2).standard_normal((1, 1, 24, 8))
    k = np.zeros((1, 1, 24, 8))
    s = oracle.meanpool_scores(q, k, 24, 8)
    assert np.allclose(s, 1.0 / 9.0, atol=1e-15)
