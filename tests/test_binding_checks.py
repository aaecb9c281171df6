"""The Python binding passes the library device pointers only: a tensor that is
not on a CUDA device, not on the current device, or smaller than the library
will index is rejected before any call reaches the library."""
import numpy as np
import pytest
import torch

import block_sparse_attention_16_b200 as lbsa


def _raises_invalid(fn):
    with pytest.raises(lbsa.LbsaError) as e:
        fn()
    assert e.value.code == lbsa.LBSA_ERR_INVALID_ARG


def test_selection_rejects_host_scores():
    s = torch.full((1, 2, 4, 4), 0.25)
    _raises_invalid(lambda: lbsa.lbsa_select(s, 64, 0.9, "row"))
    _raises_invalid(lambda: lbsa.lbsa_select_rule(s, 64, "local_topk", n_valid=256, k=2))
    _raises_invalid(lambda: lbsa.lbsa_select_routed(s, 64, 0.9, 0.5, 2))
    _raises_invalid(lambda: lbsa.lbsa_select_head_noalloc(s, 0.25))
    _raises_invalid(lambda: lbsa.lbsa_select_tokens(torch.full((1, 2, 256, 4), 0.25), 64, 0.25))


def test_csr_import_rejects_host_arrays():
    rp = torch.tensor([0, 1, 2], dtype=torch.int32)
    col = torch.tensor([0, 1], dtype=torch.int32)
    _raises_invalid(lambda: lbsa.lbsa_blockset_from_csr(rp, col, 1, 1, 2, 64))


def test_scores_and_attention_reject_host_tensors():
    q = torch.zeros(1, 1, 64, 64)
    _raises_invalid(lambda: lbsa.lbsa_score(q, q, 64))
    _raises_invalid(lambda: lbsa.lbsa_score_attend(q, q, q, 64))
    _raises_invalid(lambda: lbsa.lbsa_permute([q], torch.zeros(64, dtype=torch.int32)))


@pytest.mark.gpu
def test_undersized_outputs_and_short_perm_are_rejected():
    dev = torch.device("cuda", torch.cuda.current_device())
    q = torch.randn(1, 2, 200, 64, device=dev)
    _raises_invalid(lambda: lbsa.lbsa_score(q, q, 64, scores=torch.empty(1, 2, 4, 3, device=dev)))
    _raises_invalid(lambda: lbsa.lbsa_score(q, q, 64, lse=torch.empty(1, 2, 199, device=dev)))
    _raises_invalid(lambda: lbsa.lbsa_score(q, q, 64, mode="meanpool_token", scores=torch.empty(1, 2, 4, 4, device=dev)))
    _raises_invalid(lambda: lbsa.lbsa_permute([q], torch.arange(199, dtype=torch.int32, device=dev)))
    _raises_invalid(lambda: lbsa.lbsa_permute([q], torch.arange(200, dtype=torch.int64, device=dev)))


@pytest.mark.gpu
def test_out_of_range_perm_skips_rows_and_reports_bad_index():
    dev = torch.device("cuda", torch.cuda.current_device())
    q = torch.randn(1, 2, 200, 64, device=dev)
    lbsa.lbsa_device_status(clear=True)
    perm = torch.arange(200, dtype=torch.int32, device=dev).flip(0).contiguous()
    perm[7] = 200
    perm[9] = -1
    y = torch.zeros_like(q)
    lbsa.lbsa_permute([q], perm, outs=[y])
    assert lbsa.lbsa_device_status(clear=True) == lbsa.LBSA_ERR_BAD_INDEX
    good = torch.ones(200, dtype=torch.bool)
    good[7] = good[9] = False
    ref = q.flip(2)
    assert torch.equal(y[:, :, good.to(dev)], ref[:, :, good.to(dev)])
    assert not y[:, :, 7].any() and not y[:, :, 9].any()
    lbsa.lbsa_permute([q], torch.arange(200, dtype=torch.int32, device=dev).flip(0).contiguous(), outs=[y])
    assert lbsa.lbsa_device_status(clear=True) == lbsa.LBSA_OK


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_tensors_of_another_device_are_rejected():
    torch.cuda.set_device(0)
    q = torch.randn(1, 1, 64, 64, device="cuda:1")
    _raises_invalid(lambda: lbsa.lbsa_score(q, q, 64))
    _raises_invalid(lambda: lbsa.lbsa_permute([q], torch.arange(64, dtype=torch.int32, device="cuda:1")))
