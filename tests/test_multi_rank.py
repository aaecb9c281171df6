"""World-size-2 gloo tests (CPU) of the multi-rank host logic."""
import itertools
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_16_b200.multi import (barrier, lpt_shards, max_over_ranks, run_sharded_layer,
                                                 shard_loads)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, weights, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shards = lpt_shards(weights, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, shards)
        assert all(g == shards for g in gathered), "ranks disagree on the split"
        mine = shards[rank]
        t = 10.0 + 5.0 * rank + 0.25 * len(mine)
        tmax = max_over_ranks(t)
        barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{tmax} {','.join(map(str, mine))}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_and_reduce(tmp_path):
    rng = np.random.default_rng(0)
    weights = (rng.random(12) * 100).round(3).tolist()       # kept pairs per (batch, head)
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, weights, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    lines = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(2)]
    shards = lpt_shards(weights, 2)
    expect_max = max(10.0 + 5.0 * r + 0.25 * len(shards[r]) for r in range(2))
    for r, (tmax, mine) in enumerate(lines):
        assert float(tmax) == expect_max
        assert list(map(int, mine.split(","))) == shards[r]


def test_lpt_is_a_partition_and_within_four_thirds_of_optimal():
    rng = np.random.default_rng(1)
    for trial in range(40):
        n = int(rng.integers(1, 11))
        world = int(rng.integers(1, 4))
        w = rng.integers(1, 50, size=n).tolist()
        shards = lpt_shards(w, world)
        assert sorted(i for s in shards for i in s) == list(range(n))
        best = min(max(sum(w[i] for i in range(n) if a[i] == r) for r in range(world))
                   for a in itertools.product(range(world), repeat=n))
        assert max(shard_loads(w, shards)) <= (4 / 3 - 1 / (3 * world)) * best + 1e-9


def test_single_process_helpers_are_identity():
    assert max_over_ranks(3.5) == 3.5
    assert lpt_shards([5, 5, 5], 1) == [[0, 1, 2]]
    with pytest.raises(ValueError):
        lpt_shards([1], 0)


# ---------------------------------------------------------------- one layer split over two ranks
def _tiny_layer():
    """A tiny fp64 layer (B=2, H=3, 256 tokens, d=64), its oracle blockset at
    p = 0.9, and the kept pairs per (batch, head) unit."""
    import torch
    import oracle
    rng = np.random.default_rng(7)
    q, k, v = (torch.from_numpy(rng.standard_normal((2, 3, 256, 64))) for _ in range(3))
    masses = oracle.block_mass(q.numpy(), k.numpy(), 256, 64)
    rp, col = oracle.select_contract(masses.astype(np.float32), 0.9, "row")
    weights = np.diff(rp).reshape(6, 4).sum(1).tolist()
    return q, k, v, rp, col, weights


def _oracle_units(rp, col):
    """The host stand-in of the GPU attention: the oracle's block-sparse
    attention of each listed unit with its rows of the CSR."""
    import torch
    import oracle

    def compute(qu, ku, vu, units):
        outs = []
        for n, u in enumerate(units):
            a = rp[u * 4]
            urp, ucol = rp[u * 4:u * 4 + 5] - a, col[a:rp[u * 4 + 4]]
            o, _ = oracle.sparse_attention(qu[n:n + 1][None].numpy(), ku[n:n + 1][None].numpy(),
                                           vu[n:n + 1][None].numpy(), 256, 64, urp, ucol)
            outs.append(torch.from_numpy(o[0, 0]))
        return torch.stack(outs) if outs else qu[:0]
    return compute


def _layer_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, rp, col, weights = _tiny_layer()
        out = run_sharded_layer(q, k, v, weights, _oracle_units(rp, col))
        units, mine = run_sharded_layer(q, k, v, weights, _oracle_units(rp, col), gather=False)
        np.save(os.path.join(out_dir, f"full{rank}.npy"), out.numpy())
        np.save(os.path.join(out_dir, f"units{rank}.npy"), np.array(units))
    finally:
        dist.destroy_process_group()


def test_sharded_layer_on_two_gloo_ranks_equals_one_process(tmp_path):
    """Shard by LPT on kept pairs, compute each rank's heads, all_gather: every
    rank ends with exactly the one-process layer output."""
    q, k, v, rp, col, weights = _tiny_layer()
    ref = _oracle_units(rp, col)(q.reshape(6, 256, 64), k.reshape(6, 256, 64), v.reshape(6, 256, 64),
                                 list(range(6))).reshape(2, 3, 256, 64).numpy()
    mp.start_processes(_layer_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    shards = lpt_shards(weights, 2)
    for r in range(2):
        assert np.array_equal(np.load(tmp_path / f"full{r}.npy"), ref)
        assert np.load(tmp_path / f"units{r}.npy").tolist() == shards[r]
    assert sorted(shards[0] + shards[1]) == list(range(6)) and shards[0] and shards[1]


def test_more_ranks_than_units():
    """Three ranks, two units: one rank holds none, computes nothing (no library
    call) and the gather still returns the whole layer on every rank."""
    from block_sparse_attention_16_b200.multi import attend_units
    import torch
    shards = lpt_shards([5.0, 3.0], 3)
    assert sorted(len(sh) for sh in shards) == [0, 1, 1]

    class NoLibrary:
        def __getattr__(self, name):
            raise AssertionError(f"{name} called for a rank without units")

    compute = attend_units(NoLibrary(), None, [])
    q = torch.zeros(0, 16, 8)
    assert compute(q, q, q, []).shape == (0, 16, 8)


def _uneven_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, H, N, d = 1, 2, 8, 4
        q = torch.arange(B * H * N * d, dtype=torch.float64).reshape(B, H, N, d)
        out = run_sharded_layer(q, q, q, [2.0, 1.0], lambda qu, ku, vu, units: qu * 2)
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy())
    finally:
        dist.destroy_process_group()


def test_sharded_layer_with_an_idle_rank(tmp_path):
    """Three gloo ranks over two units: every rank ends with the whole layer."""
    import torch
    mp.start_processes(_uneven_worker, args=(3, _free_port(), str(tmp_path)), nprocs=3, join=True,
                       start_method="spawn")
    want = (torch.arange(64, dtype=torch.float64).reshape(1, 2, 8, 4) * 2).numpy()
    for r in range(3):
        assert np.array_equal(np.load(tmp_path / f"out{r}.npy"), want)
