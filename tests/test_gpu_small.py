"""GPU parity on small shapes: every path of the C ABI against the fp64 oracle.

Shapes span several 128-row tiles, ragged last blocks, both block sizes, both
head dims, batch > 1, empty rows, p = 1 (dense) and the status-word paths.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_16_b200 as lbsa
from block_sparse_attention_16_b200.workload import get_workload, make_qkv, small_workload
from parity import assert_csr_equal, assert_out_close, assert_scores_close, gpu_csr, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    lbsa.lbsa_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def _pipeline(wl, p, scope="row", mode="exact"):
    q, k, v = (x.cuda() for x in make_qkv(wl))
    scores, lse_d = (lbsa.lbsa_score(q, k, wl.block, mode=mode, want_lse=True) if mode == "exact"
                     else (lbsa.lbsa_score(q, k, wl.block, mode=mode), None))
    bs = lbsa.lbsa_select(scores, wl.block, p, scope)
    out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    assert lbsa.lbsa_get_status(bs) == 0
    return q, k, v, scores, lse_d, bs, out, lse


# ------------------------------------------------------------------ plumbing
def test_bounded_wait_reports_timeout():
    assert lbsa.lbsa_selftest_wait(2000) == lbsa.LBSA_ERR_TIMEOUT


@pytest.mark.parametrize("grid", [(4, 8, 8), (21, 30, 52), (5, 7, 9)])
def test_device_partition_perm_matches_oracle(grid):
    T, H, W = grid
    for kind, ref in (("1d", oracle.perm_1d_temporal(T, H, W)), ("2d", oracle.perm_2d_frame_tiles(T, H, W)),
                      ("3d", oracle.perm_3d_tiles(T, H, W)), ("raster", oracle.perm_raster(T, H, W))):
        got = lbsa.lbsa_partition_perm(T, H, W, kind, device="cuda").cpu().numpy()
        assert np.array_equal(got, ref), kind


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_permute_gather_scatter(dtype, d):
    T, H, W = 5, 7, 9
    n = T * H * W
    g = torch.Generator(device="cuda").manual_seed(3)
    xs = [torch.randn(2, 3, n, d, generator=g, device="cuda").to(dtype) for _ in range(3)]
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", device="cuda")
    ys = lbsa.lbsa_permute(xs, perm)
    pl = perm.long()
    for x, y in zip(xs, ys):
        assert torch.equal(y, x[:, :, pl])
    back = lbsa.lbsa_permute(ys, perm, inverse=True)
    for x, b in zip(xs, back):
        assert torch.equal(b, x)


# ------------------------------------------------------------------ fp32 path (true fp32)
@pytest.mark.parametrize("p", [0.5, 0.9, 0.99, 1.0])
def test_tiny_fp32_pipeline(p):
    wl = get_workload("tiny")
    q, k, v, scores, lse_d, bs, out, lse = _pipeline(wl, p)
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.block_mass(qh, kh, wl.n_valid, wl.block))
    _, ref_lse = oracle.dense_attention(qh, kh, vh, wl.n_valid)
    assert np.max(np.abs(host(lse_d) - ref_lse)) <= 1e-5
    csr = gpu_csr(bs)
    assert_csr_equal(csr, oracle.select_contract(host(scores), p, "row"))
    ref_o, ref_l = oracle.sparse_attention(qh, kh, vh, wl.n_valid, wl.block, *csr)
    assert_out_close(host(out), ref_o[:, :, :wl.n_valid], torch.float32)
    assert np.max(np.abs(host(lse) - ref_l[:, :, :wl.n_valid])) <= 1e-5


def test_fp32_ragged_multi_batch():
    wl = small_workload("f32r", 2, 2, 128, (3, 5, 9), 64, dtype="f32", wid=101)   # 135 tokens, last block 7
    q, k, v, scores, _, bs, out, lse = _pipeline(wl, 0.95)
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.block_mass(qh, kh, wl.n_valid, wl.block))
    csr = gpu_csr(bs)
    assert_csr_equal(csr, oracle.select_contract(host(scores), 0.95, "row"))
    ref_o, _ = oracle.sparse_attention(qh, kh, vh, wl.n_valid, wl.block, *csr)
    assert_out_close(host(out), ref_o[:, :, :wl.n_valid], torch.float32)


# ------------------------------------------------------------------ bf16 tensor-core path
BF16_CASES = [
    # name, B, H, d, grid, block
    ("b64_d128_ragged", 2, 2, 128, (3, 8, 12), 64),       # 288 tokens: 5 blocks, last 32 valid, 3 tiles
    ("b128_d128_ragged", 1, 3, 128, (4, 9, 10), 128),     # 360 tokens: 3 blocks, last 104 valid
    ("b64_d64_ragged", 1, 2, 64, (5, 6, 7), 64),          # 210 tokens: 4 blocks, last 18 valid
    ("b64_d128_16blk", 1, 2, 128, (4, 16, 16), 64),       # 1024 tokens: 16 blocks, 8 tiles
    ("b128_d64_odd", 2, 1, 64, (3, 7, 31), 128),          # 651 tokens: 6 blocks, last 11 valid
]


@pytest.mark.parametrize("case", BF16_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("p", [0.9, 0.99])
def test_bf16_pipeline(case, p):
    name, B, H, d, grid, block = case
    wl = small_workload(name, B, H, d, grid, block, dtype="bf16", wid=110 + BF16_CASES.index(case))
    q, k, v, scores, lse_d, bs, out, lse = _pipeline(wl, p)
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.block_mass(qh, kh, wl.n_valid, wl.block))
    _, ref_dl = oracle.dense_attention(qh, kh, vh, wl.n_valid)
    assert np.max(np.abs(host(lse_d) - ref_dl)) <= 1e-3
    csr = gpu_csr(bs)
    assert_csr_equal(csr, oracle.select_contract(host(scores), p, "row"))
    ref_o, ref_l = oracle.sparse_attention(qh, kh, vh, wl.n_valid, wl.block, *csr)
    assert_out_close(host(out), ref_o[:, :, :wl.n_valid], torch.bfloat16)
    assert np.max(np.abs(host(lse) - ref_l[:, :, :wl.n_valid])) <= 1e-2


@pytest.mark.parametrize("mode,scope,p", [("exact", "row", 0.9), ("meanpool", "head", 0.25)])
def test_token_major_views_match_contiguous(mode, scope, p):
    """[B, N, H, d] storage seen as [B, H, N, d] views (strided heads and rows):
    every stage reads and writes through the strides, bit for bit as on copies."""
    wl = small_workload("strided", 2, 3, 128, (3, 8, 12), 64, dtype="bf16", wid=130)
    q, k, v = (x.cuda() for x in make_qkv(wl))
    qs, ks, vs = (x.transpose(1, 2).contiguous().transpose(1, 2) for x in (q, k, v))
    assert qs.stride(2) == wl.H * wl.d and not qs.is_contiguous()
    perm = lbsa.lbsa_partition_perm(*wl.grid, "3d", device="cuda")
    outs = []
    for a, b_, c in ((q, k, v), (qs, ks, vs)):
        ap, bp, cp = lbsa.lbsa_permute([a, b_, c], perm)
        sc = lbsa.lbsa_score(ap, bp, wl.block, mode=mode)
        bs = lbsa.lbsa_select(sc, wl.block, p, scope)
        o = lbsa.lbsa_attend(ap, bp, cp, bs)
        back = lbsa.lbsa_permute([o], perm, inverse=True)[0]
        torch.cuda.synchronize()
        assert lbsa.lbsa_device_status() == 0 and lbsa.lbsa_get_status(bs) == 0
        outs.append((ap, sc, gpu_csr(bs), o, back))
    (a0, s0, c0, o0, b0), (a1, s1, c1, o1, b1) = outs
    assert torch.equal(a0, a1)
    assert torch.equal(s0, s1)
    assert_csr_equal(c1, c0)
    assert torch.equal(o0, o1) and torch.equal(b0, b1)


@pytest.mark.parametrize("case", BF16_CASES[:3], ids=lambda c: c[0])
def test_bf16_dense_p1_equals_dense_attention(case):
    name, B, H, d, grid, block = case
    wl = small_workload(name, B, H, d, grid, block, dtype="bf16", wid=120)
    q, k, v, scores, _, bs, out, lse = _pipeline(wl, 1.0)
    rp, col = gpu_csr(bs)
    assert np.all(np.diff(rp) == wl.n_blocks)
    ref_o, ref_l = oracle.dense_attention(host(q), host(k), host(v), wl.n_valid)
    assert_out_close(host(out), ref_o, torch.bfloat16)
    assert np.max(np.abs(host(lse) - ref_l)) <= 1e-2


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("block", [64, 128])
def test_hand_built_lists_with_empty_rows(dtype, block):
    wl = small_workload("csr", 1, 2, 128, (4, 10, 16), block, dtype=dtype, wid=130)    # 640 tokens
    q, k, v = (x.cuda() for x in make_qkv(wl))
    nB = wl.n_blocks
    rng = np.random.default_rng(block)
    rows = []
    for h in range(wl.H):
        for i in range(nB):
            r = rng.random()
            if r < 0.25:
                rows.append(np.zeros(0, dtype=np.int64))                      # empty row
            elif r < 0.5:
                rows.append(np.array([int(rng.integers(nB))]))                 # single block
            else:
                rows.append(np.sort(rng.choice(nB, size=int(rng.integers(1, nB + 1)), replace=False)))
    rp, col = oracle.csr_from_rows(rows)
    bs = lbsa.lbsa_blockset_from_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(),
                                     wl.B, wl.H, nB, block)
    out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == 0
    assert_csr_equal(gpu_csr(bs), (rp, col))
    ref_o, ref_l = oracle.sparse_attention(host(q), host(k), host(v), wl.n_valid, block, rp, col)
    assert_out_close(host(out), ref_o[:, :, :wl.n_valid], q.dtype)
    gl = host(lse)
    rl = ref_l[:, :, :wl.n_valid]
    assert np.array_equal(np.isneginf(gl), np.isneginf(rl))
    fin = np.isfinite(rl)
    assert np.max(np.abs(gl[fin] - rl[fin])) <= 1e-2
    empty = np.isneginf(rl)
    assert np.all(host(out)[empty] == 0)



@pytest.mark.parametrize("block", [64, 128])
def test_running_max_rescales_within_and_across_steps(block):
    """Logits that climb steeply along the key axis (head 0) make the running
    max grow inside a 128-key step and at every step, so P already written and
    O are rescaled; falling logits (head 1) never rescale after the first key.
    Dense lists and random lists with empty rows, against the fp64 oracle."""
    B, H, d, n_valid = 1, 2, 128, 600            # 10 (b=64) or 5 (b=128) blocks, ragged last block
    nB = (n_valid + block - 1) // block
    g = torch.Generator().manual_seed(140 + block)
    q = torch.randn(B, H, n_valid, d, generator=g) * 0.5
    k = torch.randn(B, H, n_valid, d, generator=g) * 0.5
    v = torch.randn(B, H, n_valid, d, generator=g)
    ramp = torch.arange(n_valid, dtype=torch.float32) * 0.35 * (d ** 0.5) / (8.0 * 1.4426950408889634)
    q[:, :, :, 0] = 8.0
    k[0, 0, :, 0] = ramp                          # +0.35 per key in log2 units: +22 over a 64-key half
    k[0, 1, :, 0] = ramp.flip(0)
    q, k, v = (x.to(torch.bfloat16).cuda() for x in (q, k, v))
    rng = np.random.default_rng(block)
    dense = [np.arange(nB) for _ in range(B * H * nB)]
    sparse = []
    for _ in range(B * H * nB):
        r = rng.random()
        sparse.append(np.zeros(0, dtype=np.int64) if r < 0.2 else
                      np.sort(rng.choice(nB, size=int(rng.integers(1, nB + 1)), replace=False)))
    for rows in (dense, sparse):
        rp, col = oracle.csr_from_rows(rows)
        bs = lbsa.lbsa_blockset_from_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(), B, H, nB, block)
        out, lse = lbsa.lbsa_attend(q, k, v, bs, want_lse=True)
        torch.cuda.synchronize()
        assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
        ref_o, ref_l = oracle.sparse_attention(host(q), host(k), host(v), n_valid, block, rp, col)
        assert_out_close(host(out), ref_o[:, :, :n_valid], torch.bfloat16)
        gl, rl = host(lse), ref_l[:, :, :n_valid]
        assert np.array_equal(np.isneginf(gl), np.isneginf(rl))
        fin = np.isfinite(rl)
        assert np.max(np.abs(gl[fin] - rl[fin])) <= 1e-2

def test_bad_block_index_is_flagged_and_skipped():
    wl = small_workload("bad", 1, 1, 128, (2, 8, 16), 64, dtype="bf16", wid=131)   # 256 tokens, 4 blocks
    q, k, v = (x.cuda() for x in make_qkv(wl))
    rows = [np.array([0, 1]), np.array([1, 7]), np.array([2]), np.array([0, 3])]   # 7 is out of range
    rp, col = oracle.csr_from_rows(rows)
    bs = lbsa.lbsa_blockset_from_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(col).cuda(), 1, 1, 4, 64)
    out = lbsa.lbsa_attend(q, k, v, bs)
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs, clear=True) == lbsa.LBSA_ERR_BAD_INDEX
    assert lbsa.lbsa_get_status(bs) == 0
    clean = [np.array([0, 1]), np.array([1]), np.array([2]), np.array([0, 3])]
    crp, ccol = oracle.csr_from_rows(clean)
    ref_o, _ = oracle.sparse_attention(host(q), host(k), host(v), wl.n_valid, 64, crp, ccol)
    assert_out_close(host(out), ref_o, torch.bfloat16)


def test_invalid_scores_keep_all_and_flag():
    scores = torch.full((1, 2, 8, 8), 1.0 / 8, device="cuda")
    scores[0, 1, 3, 5] = float("nan")
    bs = lbsa.lbsa_select(scores, 64, 0.5, "row")
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == lbsa.LBSA_ERR_INVALID_SCORES
    rp, col = gpu_csr(bs)
    counts = np.diff(rp)
    assert counts[8 + 3] == 8                        # the poisoned row keeps everything
    assert np.all(counts[:8] == 4)                   # 4 x 1/8 = 0.5 reaches p = 0.5
    bs2 = lbsa.lbsa_select(scores, 64, 0.5, "head")
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs2) == lbsa.LBSA_ERR_INVALID_SCORES
    rp2, _ = gpu_csr(bs2)
    assert np.all(np.diff(rp2)[8:] == 8)             # the poisoned head keeps everything


# ------------------------------------------------------------------ selection on synthetic score matrices
@pytest.mark.parametrize("nB", [1, 4, 33, 100, 512, 929])
@pytest.mark.parametrize("kind", ["dirichlet", "ties", "peaked"])
def test_select_row_bit_exact(nB, kind):
    rng = np.random.default_rng(nB)
    H = 3
    if kind == "dirichlet":
        x = rng.dirichlet(np.ones(nB) * 0.3, size=(1, H, nB))
    elif kind == "ties":
        x = rng.choice(np.array([0.0, 1 / 64, 1 / 32, 3 / 64, 1 / 8]), size=(1, H, nB, nB))
    else:
        z = rng.standard_normal((1, H, nB, nB)) * 6
        x = np.exp(z - z.max(-1, keepdims=True))
        x /= x.sum(-1, keepdims=True)
    x = x.astype(np.float32)
    s = torch.from_numpy(x).cuda()
    for p in (0.25, 0.9, 0.99, 0.999):
        bs = lbsa.lbsa_select(s, 64, p, "row")
        assert_csr_equal(gpu_csr(bs), oracle.select_contract(x, p, "row"))
        assert lbsa.lbsa_get_status(bs) == 0


@pytest.mark.parametrize("nB", [1, 31, 32, 33, 100])
def test_block_bitmask_round_trip(nB):
    """Bitmask export sets exactly the kept ids of each row (checked against the
    oracle's CSR of the same selection); importing it gives the same blockset; a
    stray bit past nB is dropped and flagged."""
    rng = np.random.default_rng(90 + nB)
    x = rng.random((2, 3, nB, nB)).astype(np.float32)
    x /= x.sum(-1, keepdims=True)
    s = torch.from_numpy(x).cuda()
    bs = lbsa.lbsa_select(s, 64, 0.6, "row")
    bits = lbsa.lbsa_blockset_export_bitmask(bs)
    torch.cuda.synchronize()
    rp, col = oracle.select_contract(x, 0.6, "row")
    W = (nB + 31) // 32
    words = bits.cpu().numpy().view(np.uint32).reshape(-1, W)
    for r in range(2 * 3 * nB):
        want = np.zeros(W, dtype=np.uint32)
        for j in col[rp[r]:rp[r + 1]]:
            want[j >> 5] |= np.uint32(1) << np.uint32(j & 31)
        assert np.array_equal(words[r], want), r
    back = lbsa.lbsa_blockset_from_bitmask(bits, 64)
    assert_csr_equal(gpu_csr(back), (rp, col))
    assert lbsa.lbsa_get_status(back) == 0
    if nB % 32:
        stray = bits.clone()
        stray[0, 0, 0, W - 1] |= torch.tensor(-(1 << 31), dtype=torch.int32, device="cuda")   # bit 31: past nB
        bad = lbsa.lbsa_blockset_from_bitmask(stray, 64)
        assert_csr_equal(gpu_csr(bad), (rp, col))
        assert lbsa.lbsa_get_status(bad) == lbsa.LBSA_ERR_BAD_INDEX


@pytest.mark.parametrize("nB", [2, 16, 100, 512, 568, 576])
@pytest.mark.parametrize("kind", ["softmax", "ties"])
def test_select_head_bit_exact(nB, kind):
    """Head scope against the oracle; nB = 568 is the largest the one-launch cluster
    path holds (71 rows of 568 scores a CTA in shared memory), 576 takes the
    multi-kernel path."""
    rng = np.random.default_rng(7 + nB)
    H = 2
    if kind == "softmax":
        z = rng.standard_normal((1, H, nB, nB)) * 3
        x = np.exp(z - z.max(axis=(2, 3), keepdims=True))
        x /= x.sum(axis=(2, 3), keepdims=True)
    else:
        x = rng.choice(np.array([0.0, 2.0 ** -20, 2.0 ** -16, 2.0 ** -14]), size=(1, H, nB, nB))
    x = x.astype(np.float32)
    s = torch.from_numpy(x).cuda()
    for p in (0.1, 0.25, 0.5, 0.9, 1.0):
        bs = lbsa.lbsa_select(s, 64, p, "head")
        assert_csr_equal(gpu_csr(bs), oracle.select_contract(x, p, "head"))
        assert lbsa.lbsa_get_status(bs) == 0


# ------------------------------------------------------------------ block-mean proxy + head scope
@pytest.mark.parametrize("d", [128, 64])
def test_meanpool_scores_on_tensor_cores(d):
    """Block-mean proxy with bf16 inputs and nB a multiple of 4 (the tensor-core
    logits): 8,448 tokens, nB = 132 (two 128-row tiles and two 128-column
    chunks, each 4 wide in the second), every score against the fp64 oracle,
    head scope bit-exact on them."""
    wl = small_workload(f"mptc{d}", 1, 2, d, (1, 8, 1056), 64, dtype="bf16", wid=140 + d)
    assert wl.n_blocks == 132
    q, k = (x.cuda() for x in make_qkv(wl)[:2])
    scores = lbsa.lbsa_score(q, k, wl.block, mode="meanpool")
    bs = lbsa.lbsa_select(scores, wl.block, 0.25, "head")
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0 and lbsa.lbsa_get_status(bs) == 0
    sc = host(scores)
    assert_scores_close(sc, oracle.meanpool_scores(host(q), host(k), wl.n_valid, wl.block))
    assert_csr_equal(gpu_csr(bs), oracle.select_contract(sc, 0.25, "head"))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_meanpool_head_scope_pipeline(dtype):
    wl = small_workload("mp", 1, 3, 128, (4, 12, 20), 64, dtype=dtype, wid=140)   # 960 tokens: 15 blocks
    q, k, v, scores, _, bs, out, lse = _pipeline(wl, 0.25, scope="head", mode="meanpool")
    qh, kh, vh = host(q), host(k), host(v)
    assert_scores_close(host(scores), oracle.meanpool_scores(qh, kh, wl.n_valid, wl.block))
    csr = gpu_csr(bs)
    assert_csr_equal(csr, oracle.select_contract(host(scores), 0.25, "head"))
    ref_o, _ = oracle.sparse_attention(qh, kh, vh, wl.n_valid, wl.block, *csr)
    assert_out_close(host(out), ref_o[:, :, :wl.n_valid], q.dtype)


@pytest.mark.gpu
def test_fma_pipe_exp2_within_its_error_bound():
    """The scorer's FMA-pipe exponential against 2^v in fp64 over its domain."""
    v = torch.cat([torch.linspace(-125.0, 0.0, 1_000_001, dtype=torch.float64),
                   -30.0 * torch.rand(200_001, dtype=torch.float64, generator=torch.Generator().manual_seed(7)),
                   torch.tensor([-0.5, 0.5 - 1.0, -1e-30, 0.0], dtype=torch.float64)]).float()
    out = lbsa.lbsa_selftest_exp2(v.cuda()).cpu().double()
    ref = torch.exp2(v.double())
    rel = ((out - ref).abs() / ref).max().item()
    assert rel < 3e-6, rel
    # below the clamp the result is 2^-125 (tiny, never negative or garbage)
    low = lbsa.lbsa_selftest_exp2(torch.tensor([-126.0, -500.0, -1e30], device="cuda")).cpu().double()
    assert torch.all((low - 2.0 ** -125).abs() <= 1e-6 * 2.0 ** -125), low
