"""The Python binding passes the library device pointers only: a tensor that is
not on a CUDA device is rejected before any call reaches the library.  No GPU."""
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
