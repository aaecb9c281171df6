"""GPU side of a layer split over ranks by (batch, head) unit: the library's
attention on a subset of a blockset's units (through a blockset of just their
rows) gives exactly the rows the whole-layer call gives, and the one-rank flow
of run_sharded_layer returns the whole layer's output unchanged."""
import numpy as np
import pytest
import torch

import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.multi import attend_units, layer_shards, run_sharded_layer
from block_sparse_attention_16_b200.workload import make_qkv, small_workload

pytestmark = pytest.mark.gpu


def test_units_subset_and_one_rank_flow_are_exact():
    wl = small_workload("shard", 2, 3, 128, (3, 9, 13), 64, dtype="bf16", wid=195)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores = lbsa.lbsa_score(q, k, wl.block)
    bs = lbsa.lbsa_select(scores, wl.block, 0.9, "row")
    full = lbsa.lbsa_attend(q, k, v, bs)
    counts, _ = lbsa.lbsa_blockset_views(bs)
    weights = counts.view(wl.B * wl.H, wl.n_blocks).sum(1).tolist()
    flat = [x.reshape(wl.B * wl.H, wl.n_valid, wl.d) for x in (q, k, v, full)]
    units = [1, 4]
    sub = attend_units(lbsa, bs, units)(flat[0][units], flat[1][units], flat[2][units], units)
    assert torch.equal(sub, flat[3][units])
    shards = layer_shards(weights)                       # one process: every unit on rank 0
    assert shards == [list(range(wl.B * wl.H))]
    out = run_sharded_layer(q, k, v, weights, attend_units(lbsa, bs, shards[0]))
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    assert torch.equal(out, full)
