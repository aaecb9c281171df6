"""Tolerances and comparison helpers shared by the GPU parity tests.

Tolerances (stated once, used everywhere):
  block scores   |gpu - oracle| <= max(1e-4 * |oracle|, 1e-12)
                 (relative 1e-4; masses below 1e-8 may underflow in fp32, so
                 an absolute floor of 1e-12 applies there)
  index sets     bit-exact: the GPU blockset equals the oracle's fixed-point
                 selector run on the GPU's own fp32 scores
  outputs        bf16 inputs: max-abs <= 2e-2 and relative Frobenius <= 1e-2
                 fp32 inputs: max-abs <= 1e-5 and relative Frobenius <= 1e-5
                 (both against the fp64 oracle on the same input bytes)
"""
import numpy as np
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa

SCORE_REL, SCORE_FLOOR = 1e-4, 1e-12
OUT_TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-5, 1e-5)}


def assert_scores_close(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = np.maximum(SCORE_REL * np.abs(ref), SCORE_FLOOR)
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} scores out of tolerance; worst rel "
                           f"{(err / np.maximum(np.abs(ref), 1e-300)).max():.3e}, "
                           f"example gpu={gpu[bad][0]!r} ref={ref[bad][0]!r}")


def assert_out_close(gpu, ref, dtype):
    abs_tol, fro_tol = OUT_TOL[dtype]
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    max_abs = float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0
    denom = float(np.linalg.norm(ref))
    fro = float(np.linalg.norm(gpu - ref)) / denom if denom > 0 else float(np.linalg.norm(gpu))
    assert max_abs <= abs_tol, f"max-abs {max_abs:.3e} > {abs_tol}"
    assert fro <= fro_tol, f"rel-Frobenius {fro:.3e} > {fro_tol}"
    return max_abs, fro


def gpu_csr(bs):
    rp, col = lbsa.lbsa_blockset_export(bs)
    return rp.cpu().numpy().astype(np.int64), col.cpu().numpy().astype(np.int64)


def assert_csr_equal(got, want):
    rp_g, col_g = got
    rp_w, col_w = want
    assert np.array_equal(rp_g, rp_w), f"row counts differ in {np.sum(np.diff(rp_g) != np.diff(rp_w))} rows"
    assert np.array_equal(col_g, col_w), "column ids differ"


def host(x):
    return x.detach().float().cpu().numpy() if x.dtype == torch.bfloat16 else x.detach().cpu().numpy()
