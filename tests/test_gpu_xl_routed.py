"""Entropy-routed selection at the HunyuanVideo-like size (24 heads, 929 key
blocks of 128 tokens): one pool of all 24 heads puts 22,296 scores of a query
block in one domain (89 KB of shared memory per pool row, above the 48 KB
default), bit-exact against the oracle run on the GPU's entropies."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from parity import assert_csr_equal, gpu_csr

pytestmark = pytest.mark.gpu


def test_all_head_pool_hunyuan_size():
    H, nB = 24, 929
    rng = np.random.default_rng(929)
    conc = np.where(np.arange(H) < H // 2, 0.05, 2.0)          # half peaked, half diffuse heads
    x = np.stack([rng.dirichlet(np.full(nB, c), size=nB) for c in conc])[None].astype(np.float32)
    s = torch.from_numpy(x).cuda()
    for thr, group, p in ((2.0, H, 0.99), (2.0, H, 0.5), (float(np.median(oracle.head_entropy(x))), 5, 0.99)):
        bs, ent, dom = lbsa.lbsa_select_routed(s, 128, p, thr, group)
        e = ent.cpu().numpy()
        np.testing.assert_allclose(e, oracle.head_entropy(x), rtol=0, atol=2e-6)
        assert np.array_equal(dom.cpu().numpy(), oracle.route_heads(e, thr, group))
        assert_csr_equal(gpu_csr(bs), oracle.select_routed(x, p, thr, group, entropy=e))
        assert lbsa.lbsa_get_status(bs) == 0
