"""Allocation-free head-scope selection against the allocating entry point.

lbsa_select_head_noalloc exists for callers that may not allocate device
memory (an allocator that forbids cudaMalloc, a fixed memory budget): its
scratch is a static device array and its outputs are caller buffers.  This
file runs last so that a failure here leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_16_b200 as lbsa
from parity import gpu_csr

pytestmark = pytest.mark.gpu


def _scores(B, H, nB, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    z = torch.randn(B, H, nB * nB, generator=g, device="cuda") * 3
    return torch.softmax(z, dim=-1).reshape(B, H, nB, nB).contiguous()


def _call(scores, p, counts, cols, status):
    B, H, nB, _ = scores.shape
    lib = lbsa.load_library()
    rc = lib.lbsa_select_head_noalloc(ctypes.c_void_p(scores.data_ptr()), B, H, nB, p,
                                      ctypes.c_void_p(counts.data_ptr()), ctypes.c_void_p(cols.data_ptr()),
                                      ctypes.c_void_p(status.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == lbsa.LBSA_OK, lbsa.lbsa_last_error()


def test_noalloc_matches_lbsa_select_twice_in_a_row():
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    # two calls in a row with different shapes: stale scratch from the first
    # call would corrupt the second
    for B, H, nB, p, seed in ((1, 12, 512, 0.25, 1), (2, 3, 100, 0.5, 2)):
        scores = _scores(B, H, nB, seed)
        counts = torch.full((B * H * nB,), -1, dtype=torch.int32, device="cuda")
        cols = torch.full((B * H * nB * nB,), -1, dtype=torch.int32, device="cuda")
        status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
        _call(scores, p, counts, cols, status)
        bs = lbsa.lbsa_select(scores, 64, p, "head")
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        rp, col = gpu_csr(bs)
        c = counts.cpu().numpy().astype(np.int64)
        assert np.array_equal(c, np.diff(rp))
        cl = cols.cpu().numpy().reshape(-1, nB)
        got = np.concatenate([cl[r, :c[r]] for r in range(len(c))])
        assert np.array_equal(got, col)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    torch.cuda.set_device(0)
    lib = lbsa.load_library()
    # 200 heads x nB = 1024 need ~2.4 MB of scratch (> the 1 MiB array).  The
    # buffers match the requested shape, so even a wrongly accepted call
    # would stay in bounds.
    B, H, nB = 1, 200, 1024
    scores = torch.full((B, H, nB, nB), 1.0 / (nB * nB), dtype=torch.float32, device="cuda")
    counts = torch.zeros(B * H * nB, dtype=torch.int32, device="cuda")
    cols = torch.zeros(B * H * nB * nB, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p
    rc = lib.lbsa_select_head_noalloc(p(scores.data_ptr()), B, H, nB, 0.5, p(counts.data_ptr()),
                                      p(cols.data_ptr()), p(status.data_ptr()),
                                      p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == lbsa.LBSA_ERR_UNSUPPORTED
    assert "static array" in lbsa.lbsa_last_error()
    del scores, cols
    torch.cuda.empty_cache()
