"""Benchmark of block-sparse video attention on B200.

One step = one block-sparse attention call over one Wan-like attention layer
(B=1, H=12, d=128, 21x30x52 = 32,760 tokens in 3D-tile order, bf16, 64-token
blocks) with block indices selected once at p = 0.99 from exact block masses
and then frozen: LoSA's steady state, and the metric's own quantity.  Inputs
are resident in HBM when timing starts (302 MB of Q/K/V, larger than the
126 MB L2, so no extra flush is needed between calls).

value  = TFLOP/s on the kept pairs, summed over ranks: 4*d*sum_kept(valid_q *
         valid_k) per call, divided by the max-over-ranks device time per call.
The same JSON line carries, measured in the same run (single GPU):
  attend    ms/call, TFLOP/s and fraction of the measured burst bf16 peak
  dense     our kernel at p = 1 and torch SDPA on the same layer
  step0     LoSA's one dense step: fused dense attention + exact masses, then
            selection; and the exact scorer alone
  hot_path  one pass of the whole path: permute, exact masses, selection,
            attention, inverse permute
  config2   HunyuanVideo-like layer: indices from step 0, then 49 re-drawn
            attention calls with them frozen (median, p10, p90 per call)
  config4   skewed heads, p in {0.90, 0.95, 0.99, 0.999}: ms, TFLOP/s, density
  config3   mean-pooled proxy with head-scope tau = 0.25, per partition (1D,
            2D, 3D): the whole call
  config0   the tiny fp32 case: scorer, selection, attention
Multi-GPU (--gpus N under torchrun): every rank runs its own layer (the path
shards by (batch, head) with no exchange step), so scaling is weak and there is
no data-path collective.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference]
                  [--no-extra] [--clocks-csv PATH]

--impl reference times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "block-sparse attn ms/call & achieved TFLOP/s at p=0.99, frac of B200 roofline"
WORKLOAD = "wan"
P = 0.99


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "source": "of measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "of fallback"}


def attention_flops(counts, nB, block, n_valid, d):
    """4*d*sum over kept (query block, key block) of valid_q * valid_k."""
    valid = np.full(nB, block, dtype=np.float64)
    valid[-1] = n_valid - (nB - 1) * block
    c = np.asarray(counts).reshape(-1, nB, nB)          # [G, nB, nB] or flat [G*nB, nB]
    return 4.0 * d * float(np.einsum("gij,i,j->", c, valid, valid))


def token_flops(lbsa, bs, wl):
    """token_flops_of on a per-token blockset's device arrays."""
    counts, cols = (x.cpu().numpy() for x in lbsa.lbsa_blockset_views(bs))
    masks = lbsa.lbsa_blockset_masks(bs).cpu().numpy().view(np.uint64)
    return token_flops_of(counts, cols, masks, wl)


def token_flops_of(counts, cols, masks, wl):
    """Attention FLOPs on the kept (token, key block) pairs of a per-token blockset
    (counts [R], cols and masks [R, nB] as the library lays them out), 4*d*sum
    over tokens of their kept blocks' valid keys; also the kept-pair density and
    the fraction of tokens that keep nothing."""
    nB, blk = wl.n_blocks, wl.block
    counts = np.asarray(counts).reshape(-1)
    cols = np.asarray(cols).reshape(-1, nB)
    masks = np.asarray(masks, dtype=np.uint64).reshape(-1, nB)
    valid = np.full(nB, blk, dtype=np.float64)
    valid[-1] = wl.n_valid - (nB - 1) * blk
    slot = np.arange(nB)[None, :] < counts[:, None]
    m = np.where(slot, masks, np.uint64(0))
    pop = np.unpackbits(m.view(np.uint8), axis=1).reshape(m.shape[0], nB, 64).sum(-1)     # tokens per entry
    kept = float(pop.sum())
    fl = 4.0 * wl.d * float((pop * valid[np.where(slot, cols, 0)]).sum())
    per_tok = np.zeros((m.shape[0], 64), dtype=np.uint64)
    for u in range(64):
        per_tok[:, u] = ((m >> np.uint64(u)) & np.uint64(1)).max(axis=1)
    G = wl.B * wl.H
    n_tok = G * wl.n_valid
    has = per_tok.reshape(G, nB * 64)[:, :wl.n_valid].sum()
    return fl, kept / (n_tok * nB), 1.0 - float(has) / n_tok


def median_entropy(ent):
    """Routing threshold of the entropy-routed sweep lines: the median of one batch
    element's head entropies (mean of the two middle values for an even count), so
    that the heads strictly below it (half of them when the values are distinct) are
    pooled."""
    e = np.sort(np.asarray(ent.cpu() if hasattr(ent, "cpu") else ent, dtype=np.float64).reshape(-1))
    n = e.shape[0]
    return float(e[n // 2]) if n % 2 else float((e[n // 2 - 1] + e[n // 2]) / 2)


def kept_mask(row_ptr, col, rows, nB):
    m = np.zeros((rows, nB), dtype=np.float64)
    r = np.repeat(np.arange(rows), np.diff(row_ptr))
    m[r, col] = 1.0
    return m


class Clocks:
    """nvidia-smi sampler for the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, path):
        self.path = path
        self.proc = None
        try:
            self.f = open(path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # start timing only once the sampler is writing (nvidia-smi takes a moment to start)
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(path) == 0 and self.proc.poll() is None:
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- oracle (CPU) sample
def oracle_attention_sample(q, k, v, wl, row_ptr, col, heads_qblocks):
    """The fp64 oracle's block-sparse attention on sampled (head, query block)
    units of a blockset (CSR over B*H*nB rows); returns (kept-pair FLOPs, seconds)."""
    import oracle
    nB, b, n, d = wl.n_blocks, wl.block, wl.n_valid, wl.d
    flops = 0.0
    t0 = time.perf_counter()
    for h, qbs in heads_qblocks:
        qh = q[:, h:h + 1].float().numpy()
        kh = k[:, h:h + 1].float().numpy()
        vh = v[:, h:h + 1].float().numpy()
        rp = row_ptr[h * nB:(h + 1) * nB + 1] - row_ptr[h * nB]
        cl = col[row_ptr[h * nB]:row_ptr[(h + 1) * nB]]
        oracle.sparse_attention(qh, kh, vh, n, b, rp, cl, qblocks=qbs)
        for i in qbs:
            vq = min(b, n - i * b)
            vk = sum(min(b, n - j * b) for j in cl[rp[i]:rp[i + 1]])
            flops += 4.0 * d * vq * vk
    return flops, time.perf_counter() - t0


def oracle_frozen_rows(q, k, wl, heads_qblocks, p=P):
    """Step 0 on the host: exact masses of the sampled query blocks and the
    fixed-point selection (the untimed set-up of the reference arm); returns a
    CSR over all B*H*nB rows whose other rows are empty."""
    import oracle
    nB, b, n = wl.n_blocks, wl.block, wl.n_valid
    rows = [np.zeros(0, dtype=np.int64)] * (wl.H * nB)
    for h, qbs in heads_qblocks:
        mass = oracle.block_mass(q[:, h:h + 1].float().numpy(), k[:, h:h + 1].float().numpy(), n, b, qblocks=qbs)
        for t, i in enumerate(qbs):
            _, c = oracle.select_contract(mass[:, :, t:t + 1, :].astype(np.float32), p, "row")
            rows[h * nB + i] = c
    return oracle.csr_from_rows(rows)


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from block_sparse_attention_16_b200.workload import get_workload, make_qkv
    wl = get_workload(WORKLOAD)
    q, k, v = make_qkv(wl, device="cpu")
    import oracle
    T, H, W = wl.grid
    perm = oracle.perm_3d_tiles(T, H, W, 4, 4, 4)
    q, k, v = (x[:, :, torch.from_numpy(perm)] for x in (q, k, v))
    rng = np.random.default_rng(0)
    per_step = 4

    def sample(step):
        h = step % wl.H
        return [(h, sorted(rng.choice(wl.n_blocks, per_step, replace=False).tolist()))]

    samples = [sample(s) for s in range(args.warmup + args.steps)]
    # set-up (untimed, as the frozen indices are for the GPU arm): step 0's masses
    # and selection for every sampled query block
    rp, col = oracle_frozen_rows(q, k, wl, [u for smp in samples for u in smp])
    for s in range(args.warmup):
        oracle_attention_sample(q, k, v, wl, rp, col, samples[s])
    tot_f, tot_t = 0.0, 0.0
    for s in range(args.steps):
        f, t = oracle_attention_sample(q, k, v, wl, rp, col, samples[args.warmup + s])
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    n_cores = cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": n_cores, "kind": "oracle",
                         "sample": f"block-sparse attention of {per_step} query blocks of one head per step, "
                                   f"indices from the oracle's exact masses and p = {P} selection (untimed set-up), "
                                   f"3D-tile-ordered Wan-like layer"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl, world):
    T, H, W = wl.grid
    return {"workload": f"Wan-like layer {T}x{H}x{W} ({wl.n_valid} tokens), H={wl.H}, d={wl.d}, "
                        f"{wl.block}-token blocks, 3D 4x4x4 tiles: one block-sparse attention call with "
                        f"indices selected at p={P} from exact block masses and frozen",
            "B": wl.B, "H": wl.H, "d": wl.d, "n_valid": wl.n_valid, "block": wl.block, "p": P,
            "partition": "3d tiles 4x4x4", "l2": "inputs larger than L2 (302 MB Q/K/V per call)",
            "parallelism": f"replicas x{world} (independent layers, no collective)"}


# ---------------------------------------------------------------- own arm
def blockset_flops(lbsa, bs, wl):
    """Kept-pair attention FLOPs and density of a row- or head-scope blockset."""
    rp, col = lbsa.lbsa_blockset_export(bs)
    rp, col = rp.cpu().numpy(), col.cpu().numpy()
    R = wl.B * wl.H * wl.n_blocks
    mask = kept_mask(rp, col, R, wl.n_blocks).reshape(wl.B * wl.H, wl.n_blocks, wl.n_blocks)
    return attention_flops(mask, wl.n_blocks, wl.block, wl.n_valid, wl.d), float(mask.mean()), rp, col


def dense_flops(wl):
    return 4.0 * wl.d * wl.n_valid ** 2 * wl.H * wl.B


def extra_measurements(lbsa, wl, dev, qp, kp, vp, perm, q, k, v, pk):
    """Everything the line reports beside the contract's timed calls (single GPU)."""
    from block_sparse_attention_16_b200.workload import get_workload, make_qkv, make_qkv_f32, redraw_qkv

    def tf(fl, ms):
        return fl / (ms * 1e-3) / 1e12

    out = {}
    # dense attention on the same layer: our kernel at p = 1 (every block) and torch SDPA
    nB = wl.n_blocks
    full = torch.full((wl.B, wl.H, nB, nB), 1.0 / nB, device=dev)
    bs1 = lbsa.lbsa_select(full, wl.block, 1.0, "row")
    fd = dense_flops(wl)
    # LoSA's one dense step (fused dense attention + exact masses, then selection),
    # timed alternately with our dense attention so that their ratio is free of drift
    sc_f, o_f = lbsa.lbsa_score_attend(qp, kp, vp, wl.block)
    t_own, t_fused = _timer_pair(lambda: lbsa.lbsa_attend(qp, kp, vp, bs1),
                                 lambda: lbsa.lbsa_score_attend(qp, kp, vp, wl.block, scores=sc_f, out=o_f))
    t_sdpa = _timer(lambda: torch.nn.functional.scaled_dot_product_attention(qp, kp, vp))["median"]
    out["dense"] = {"own_p1_ms": t_own, "own_p1_tflops": tf(fd, t_own), "torch_sdpa_ms": t_sdpa,
                    "torch_sdpa_tflops": tf(fd, t_sdpa), "flops": fd}
    t_sel = _timer(lambda: lbsa.lbsa_select(sc_f, wl.block, P, "row"))["median"]
    sc = lbsa.lbsa_score(qp, kp, wl.block)
    t_score = _timer(lambda: lbsa.lbsa_score(qp, kp, wl.block, scores=sc))["median"]
    out["step0"] = {"fused_dense_step_ms": t_fused, "select_ms": t_sel, "total_ms": t_fused + t_sel,
                    "fused_vs_own_dense": t_fused / t_own, "exact_scorer_ms": t_score,
                    "exact_scorer_tflops": tf(2.0 * wl.n_valid ** 2 * wl.d * wl.H, t_score)}

    # one pass of the whole path
    def hot():
        a_, b_, c_ = lbsa.lbsa_permute([q, k, v], perm)
        s_ = lbsa.lbsa_score(a_, b_, wl.block)
        x_ = lbsa.lbsa_select(s_, wl.block, P, "row")
        o_ = lbsa.lbsa_attend(a_, b_, c_, x_)
        return lbsa.lbsa_permute([o_], perm, inverse=True)[0]
    out["hot_path"] = {"ms": _timer(hot)["median"],
                       "stages": "3D permute of Q, K, V; exact masses; row selection p=0.99; attention; "
                                 "inverse permute of O"}

    # config 2: HunyuanVideo-like layer, indices from step 0, 49 re-drawn calls with them frozen
    wh = get_workload("hunyuan")
    q32, k32, v32 = make_qkv_f32(wh, device=dev)
    qh, kh, vh = (x.to(torch.bfloat16) for x in (q32, k32, v32))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    sch, _ = lbsa.lbsa_score_attend(qh, kh, vh, wh.block)
    bsh = lbsa.lbsa_select(sch, wh.block, P, "row")
    e1.record()
    torch.cuda.synchronize()
    t_step0 = e0.elapsed_time(e1)
    flh, densh, _, _ = blockset_flops(lbsa, bsh, wh)
    calls = []
    for t in range(1, wh.extra["steps"] + 1):
        qh, kh, vh = redraw_qkv(wh, q32, k32, v32, t)
        e0.record()
        lbsa.lbsa_attend(qh, kh, vh, bsh)
        e1.record()
        e1.synchronize()
        calls.append(e0.elapsed_time(e1))
    calls.sort()
    med = calls[len(calls) // 2]
    t_sdpa_h = _timer(lambda: torch.nn.functional.scaled_dot_product_attention(qh, kh, vh), n=3, warm=1)["median"]
    out["config2"] = {"workload": "HunyuanVideo-like 33x45x80 (118800 tokens), H=24, d=128, 128-token blocks, raster",
                      "step0_ms": t_step0, "calls": len(calls), "density": densh, "ms_per_call_median": med,
                      "ms_per_call_p10": calls[max(0, len(calls) // 10)],
                      "ms_per_call_p90": calls[min(len(calls) - 1, 9 * len(calls) // 10)],
                      "tflops_median": tf(flh, med), "frac_of_burst": tf(flh, med) / pk["bf16"],
                      "torch_sdpa_dense_ms": t_sdpa_h, "torch_sdpa_dense_tflops": tf(dense_flops(wh), t_sdpa_h)}
    assert lbsa.lbsa_get_status(bsh) == 0
    del q32, k32, v32, qh, kh, vh, sch, bsh

    # config 4: skewed heads, p sweep
    ws = get_workload("wan_skew")
    T, H, W = ws.grid
    qs, ks, vs = make_qkv(ws, device=dev)
    perm_s = lbsa.lbsa_partition_perm(T, H, W, "3d", device=dev)
    qs, ks, vs = lbsa.lbsa_permute([qs, ks, vs], perm_s)
    scs = lbsa.lbsa_score(qs, ks, ws.block)
    rows = []
    for p_ in ws.extra["p_sweep"]:
        bsp = lbsa.lbsa_select(scs, ws.block, p_, "row")
        fl, dens, _, _ = blockset_flops(lbsa, bsp, ws)
        ta = _timer(lambda: lbsa.lbsa_attend(qs, ks, vs, bsp))["median"]
        rows.append({"p": p_, "density": dens, "attend_ms": ta, "tflops": tf(fl, ta), "frac_of_burst": tf(fl, ta) / pk["bf16"]})
    t_d = _timer(lambda: torch.nn.functional.scaled_dot_product_attention(qs, ks, vs))["median"]
    out["config4"] = {"workload": "skewed heads (half alpha in [2,4], half in [0.25,0.5]), Wan-like shape",
                      "rows": rows, "torch_sdpa_dense_ms": t_d}
    del qs, ks, vs, scs

    # config 3: mean-pooled proxy, head scope tau = 0.25, one whole call per partition
    wp = get_workload("wan_proxy")
    T, H, W = wp.grid
    qq, kk, vv = make_qkv(wp, device=dev)
    prow = {}
    for part in ("1d", "2d", "3d"):
        pm = lbsa.lbsa_partition_perm(T, H, W, part, device=dev)

        def call():
            a_, b_, c_ = lbsa.lbsa_permute([qq, kk, vv], pm)
            s_ = lbsa.lbsa_score(a_, b_, wp.block, mode="meanpool")
            x_ = lbsa.lbsa_select(s_, wp.block, wp.p, "head")
            o_ = lbsa.lbsa_attend(a_, b_, c_, x_)
            return lbsa.lbsa_permute([o_], pm, inverse=True)[0]
        prow[part] = _timer(call)["median"]
    # the 3D call's stages, and the per-token proxy (every query token against the key-block means)
    pm = lbsa.lbsa_partition_perm(T, H, W, "3d", device=dev)
    a3, b3, c3 = lbsa.lbsa_permute([qq, kk, vv], pm)
    s3 = lbsa.lbsa_score(a3, b3, wp.block, mode="meanpool")
    x3 = lbsa.lbsa_select(s3, wp.block, wp.p, "head")
    stages = {"score_ms": _timer(lambda: lbsa.lbsa_score(a3, b3, wp.block, mode="meanpool", scores=s3))["median"],
              "select_ms": _timer(lambda: lbsa.lbsa_select(s3, wp.block, wp.p, "head"))["median"],
              "attend_ms": _timer(lambda: lbsa.lbsa_attend(a3, b3, c3, x3))["median"]}
    st3 = lbsa.lbsa_score(a3, b3, wp.block, mode="meanpool_token")
    xt3 = lbsa.lbsa_select_tokens(st3, wp.block, wp.p)
    token = {"score_ms": _timer(lambda: lbsa.lbsa_score(a3, b3, wp.block, mode="meanpool_token",
                                                        scores=st3))["median"],
             "select_ms": _timer(lambda: lbsa.lbsa_select_tokens(st3, wp.block, wp.p))["median"],
             "attend_ms": _timer(lambda: lbsa.lbsa_attend(a3, b3, c3, xt3))["median"]}
    out["config3"] = {"workload": "mean-pooled proxy, head scope tau=0.25, Wan-like shape",
                      "call_ms": prow, "call_ms_mean_of_cycle": sum(prow.values()) / 3,
                      "stages_3d_ms": stages, "per_token_3d_ms": token}
    del qq, kk, vv, a3, b3, c3, s3, x3, st3, xt3

    # config 0: tiny fp32 case
    wt = get_workload("tiny")
    qt, kt, vt = (x.to(dev) for x in make_qkv(wt))
    sct = lbsa.lbsa_score(qt, kt, wt.block)
    bst = lbsa.lbsa_select(sct, wt.block, P, "row")
    out["config0"] = {"workload": "tiny fp32 (2 heads, 256 tokens, d=64)",
                      "score_ms": _timer(lambda: lbsa.lbsa_score(qt, kt, wt.block, scores=sct))["median"],
                      "select_ms": _timer(lambda: lbsa.lbsa_select(sct, wt.block, P, "row"))["median"],
                      "attend_ms": _timer(lambda: lbsa.lbsa_attend(qt, kt, vt, bst))["median"]}
    torch.cuda.synchronize()
    assert lbsa.lbsa_device_status() == 0
    return out


def run_own(args, rank, world):
    import block_sparse_attention_16_b200 as lbsa
    from block_sparse_attention_16_b200.build import build
    from block_sparse_attention_16_b200.multi import barrier, max_over_ranks
    from block_sparse_attention_16_b200.workload import get_workload, make_qkv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    if rank == 0:
        build()
    barrier(dev)
    lbsa.load_library()
    wl = get_workload(WORKLOAD)
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device=dev)
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", tile=(4, 4, 4), device=dev)
    stream = torch.cuda.current_stream()

    # step 0 (untimed): 3D-tile order, exact masses, selection at p = 0.99; the
    # indices are then frozen for every timed call (LoSA's schedule)
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    scores = lbsa.lbsa_score(qp, kp, wl.block)
    bs = lbsa.lbsa_select(scores, wl.block, P, "row")
    att_flops, density, rp, col = blockset_flops(lbsa, bs, wl)
    out = torch.empty_like(qp)

    for _ in range(args.warmup):
        lbsa.lbsa_attend(qp, kp, vp, bs, out=out)
    torch.cuda.synchronize()
    clocks_path = args.clocks_csv or f"/tmp/lbsa_clocks_rank{rank}.csv"
    clocks = Clocks(dev.index, clocks_path)
    barrier(dev)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        lbsa.lbsa_attend(qp, kp, vp, bs, out=out)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    clk = clocks.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    ms_per_step = total_ms / args.steps
    value = world * att_flops * args.steps / (total_ms * 1e-3) / 1e12
    assert lbsa.lbsa_get_status(bs) == 0

    pk = peaks()
    att_tflops = att_flops / (ms_per_step * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attend", "achieved": att_tflops, "peak": pk["bf16"],
                "unit": "TFLOP/s", "frac": att_tflops / pk["bf16"], "traffic": load_traffic("attend"),
                "peak_source": pk["source"] + " (bf16 burst: the attention call is the whole timed step)"}

    # end to end through the public API: every step uploads its Q, K, V (block
    # order) from pinned host memory, runs the attention call with the frozen
    # indices and downloads O.  Two steps are in flight: step i+1's inputs upload
    # (copy stream) while step i computes, and step i's output downloads (second
    # copy stream) while step i+1 computes.
    qh, kh, vh = (x.cpu().pin_memory() for x in (qp, kp, vp))
    ohs = [torch.empty_like(qh).pin_memory() for _ in range(2)]
    ins = [[torch.empty_like(qp) for _ in range(3)] for _ in range(2)]
    outs = [torch.empty_like(qp) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]      # slot's inputs have landed
    ev_free = [torch.cuda.Event() for _ in range(2)]    # slot's inputs consumed
    ev_out = [torch.cuda.Event() for _ in range(2)]     # slot's output ready on the device
    ev_down = [torch.cuda.Event() for _ in range(2)]    # slot's output downloaded
    started = [False, False]

    def upload(i):
        sl = i % 2
        if started[sl]:
            h2d.wait_event(ev_free[sl])
        with torch.cuda.stream(h2d):
            for d_, h_ in zip(ins[sl], (qh, kh, vh)):
                d_.copy_(h_, non_blocking=True)
        ev_in[sl].record(h2d)

    def compute(i):
        sl = i % 2
        stream.wait_event(ev_in[sl])
        if started[sl]:
            stream.wait_event(ev_down[sl])
        lbsa.lbsa_attend(*ins[sl], bs, out=outs[sl])
        ev_free[sl].record(stream)
        ev_out[sl].record(stream)
        d2h.wait_event(ev_out[sl])
        with torch.cuda.stream(d2h):
            ohs[sl].copy_(outs[sl], non_blocking=True)
        ev_down[sl].record(d2h)
        started[sl] = True

    def e2e_run(n, e_begin=None):
        if e_begin is not None:
            e_begin.record(stream)
            h2d.wait_event(e_begin)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
        stream.wait_event(ev_down[(n - 1) % 2])

    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    bytes_in = 3 * q.numel() * q.element_size()
    bytes_out = q.numel() * q.element_size()
    del qh, kh, vh, ohs, ins, outs

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qc, kc, vc = (x.cpu() for x in (qp, kp, vp))
        rng = np.random.default_rng(1)
        sample = [(h, sorted(rng.choice(wl.n_blocks, 4, replace=False).tolist())) for h in range(0, wl.H, 2)]
        f, t = oracle_attention_sample(qc, kc, vc, wl, rp.astype(np.int64), col.astype(np.int64), sample)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cores(), "kind": "oracle",
               "sample": f"block-sparse attention of {sum(len(x[1]) for x in sample)} query blocks over "
                         f"{len(sample)} heads with the frozen indices, {t:.1f} s"}

    extra = None
    if rank == 0 and world == 1 and not args.no_extra:
        extra = extra_measurements(lbsa, wl, dev, qp, kp, vp, perm, q, k, v, pk)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(wl, world),
            "attend": {"ms_per_call": ms_per_step, "tflops": att_tflops, "frac_of_burst": att_tflops / pk["bf16"],
                       "flops_per_call": att_flops, "density": density},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": world * att_flops * args.steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms / args.steps,
                    "h2d_bytes_per_step": bytes_in, "d2h_bytes_per_step": bytes_out,
                    "overlap": "two steps in flight: uploads and downloads on two copy streams"},
            "gpu_launches": args.steps,
            "clocks": clk,
        }
        if extra:
            line.update(extra)
        print(json.dumps(line), flush=True)
    return 0


def load_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's sources changed since those counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(kernel)
    if not d:
        return None
    h = hashlib.sha256()
    for f in d["files"]:
        h.update(open(os.path.join(ROOT, "block_sparse_attention_16_b200", "csrc", f), "rb").read())
    return d["bytes"] if h.hexdigest()[:16] == d["source_hash"] else None


def run_profile(kernel):
    """A small case for ncu: 6 heads of the Wan-like layer (151 MB of Q/K/V, more
    than L2), one warm-up pass of the path, then two launches of `kernel`
    ("dense": attention over the p = 1 blockset, the two-tile kernel; "fused":
    the fused dense step); or,
    for "proxy", one mean-pooled proxy call per partition on the full shape; for
    "token", one call of each per-token proxy stage on the full shape (3D tiles)."""
    import dataclasses

    import block_sparse_attention_16_b200 as lbsa
    from block_sparse_attention_16_b200.build import build
    from block_sparse_attention_16_b200.workload import get_workload, make_qkv

    build()
    if kernel == "token":
        # per-token proxy path of the Wan-like shape (3D tiles), one call of each stage
        wl = get_workload("wan_proxy")
        T, H, W = wl.grid
        q, k, v = make_qkv(wl, device="cuda")
        perm = lbsa.lbsa_partition_perm(T, H, W, "3d", device="cuda")
        qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
        sc = lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool_token")
        bs = lbsa.lbsa_select_tokens(sc, wl.block, 0.25)
        lbsa.lbsa_attend(qp, kp, vp, bs)
        torch.cuda.synchronize()
        assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
        print("profile case token: ok")
        return 0
    if kernel == "routed":
        # entropy-routed selection on the skewed Wan-like layer's exact scores:
        # heads below the median entropy pooled 3 at a time, p = 0.99; two calls
        wl = get_workload("wan_skew")
        T, H, W = wl.grid
        q, k, v = make_qkv(wl, device="cuda")
        perm = lbsa.lbsa_partition_perm(T, H, W, "3d", device="cuda")
        qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
        sc = lbsa.lbsa_score(qp, kp, wl.block)
        _, ent, _ = lbsa.lbsa_select_routed(sc, wl.block, 0.99, -1.0, 1)
        thr = median_entropy(ent[0])
        for _ in range(2):
            bs, _, _ = lbsa.lbsa_select_routed(sc, wl.block, 0.99, thr, 3)
        lbsa.lbsa_attend(qp, kp, vp, bs)
        torch.cuda.synchronize()
        assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
        print("profile case routed: ok")
        return 0
    if kernel == "proxy":
        # mean-pooled proxy path of the Wan-like shape, one call per partition
        wl = get_workload("wan_proxy")
        T, H, W = wl.grid
        q, k, v = make_qkv(wl, device="cuda")
        for part in ("1d", "2d", "3d"):
            perm = lbsa.lbsa_partition_perm(T, H, W, part, device="cuda")
            qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
            sc = lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool")
            bs = lbsa.lbsa_select(sc, wl.block, wl.p, "head")
            lbsa.lbsa_attend(qp, kp, vp, bs)
        torch.cuda.synchronize()
        assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
        print("profile case proxy: ok")
        return 0
    wl = dataclasses.replace(get_workload(WORKLOAD), H=6)
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", tile=(4, 4, 4), device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    scores = lbsa.lbsa_score(qp, kp, wl.block)
    bs = lbsa.lbsa_select(scores, wl.block, P, "row")
    lbsa.lbsa_attend(qp, kp, vp, bs)
    dense = lbsa.lbsa_select(scores, wl.block, 1.0, "row") if kernel == "dense" else None
    for _ in range(2):
        if kernel == "attend":
            lbsa.lbsa_attend(qp, kp, vp, bs)
        elif kernel == "dense":
            lbsa.lbsa_attend(qp, kp, vp, dense)
        elif kernel == "fused":
            lbsa.lbsa_score_attend(qp, kp, vp, wl.block)
        elif kernel == "score":
            lbsa.lbsa_score(qp, kp, wl.block, scores=scores)
        elif kernel == "select":
            lbsa.lbsa_select(scores, wl.block, P, "row")
    torch.cuda.synchronize()
    assert lbsa.lbsa_get_status(bs) == 0 and lbsa.lbsa_device_status() == 0
    print(f"profile case {kernel}: ok")
    return 0


def _timer(fn, n=10, warm=3, flush=None):
    """Median device time (ms) of fn() over n runs, CUDA events on the current stream."""
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(n):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    ts.sort()
    return {"median": ts[len(ts) // 2], "p10": ts[max(0, len(ts) // 10)], "p90": ts[min(len(ts) - 1, (9 * len(ts)) // 10)]}


def _timer_pair(fa, fb, n=10, warm=3):
    """Median device times (ms) of fa() and fb(), timed alternately (a, b, a, b, ...)
    so that clock drift under the power cap weighs on both alike."""
    for _ in range(warm):
        fa()
        fb()
    ta, tb = [], []
    for _ in range(n):
        for f, ts in ((fa, ta), (fb, tb)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
    ta.sort()
    tb.sort()
    return ta[len(ta) // 2], tb[len(tb) // 2]


def run_sweep(args):
    """Per-stage timings on every workload (one JSON line per measurement)."""
    import block_sparse_attention_16_b200 as lbsa
    from block_sparse_attention_16_b200.build import build
    from block_sparse_attention_16_b200.workload import get_workload, make_qkv, make_qkv_f32, redraw_qkv

    build()
    torch.cuda.set_device(0)
    pk = peaks()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")   # 256 MB L2 flush
    out = []

    def emit(**kw):
        line = json.dumps(kw)
        out.append(line)
        print(line, flush=True)

    def flops_of(bs, wl):
        rp, col = lbsa.lbsa_blockset_export(bs)
        rp, col = rp.cpu().numpy(), col.cpu().numpy()
        m = kept_mask(rp, col, wl.B * wl.H * wl.n_blocks, wl.n_blocks).reshape(wl.B * wl.H, wl.n_blocks, wl.n_blocks)
        return attention_flops(m, wl.n_blocks, wl.block, wl.n_valid, wl.d), m

    def hbm(nbytes, ms):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"GB/s": gbs, "frac_hbm": gbs / pk["hbm_gbs"]}

    def tfl(fl, ms):
        t = fl / (ms * 1e-3) / 1e12
        return {"TFLOP/s": t, "frac_bf16_sustained": t / pk["bf16_sustained"], "frac_bf16_burst": t / pk["bf16"]}

    # tiny fp32 workload (true-fp32 SIMT kernels)
    wl = get_workload("tiny")
    q, k, v = make_qkv(wl, device="cuda")
    sc = lbsa.lbsa_score(q, k, wl.block)
    bs = lbsa.lbsa_select(sc, wl.block, P, "row")
    emit(workload="tiny", stage="score_f32", **_timer(lambda: lbsa.lbsa_score(q, k, wl.block, scores=sc)))
    emit(workload="tiny", stage="select_row", **_timer(lambda: lbsa.lbsa_select(sc, wl.block, P, "row")))
    emit(workload="tiny", stage="attend_f32", **_timer(lambda: lbsa.lbsa_attend(q, k, v, bs)))

    # Wan-like layer, exact mass, 3D tiles
    wl = get_workload("wan")
    T, H, W = wl.grid
    q, k, v = make_qkv(wl, device="cuda")
    perm = lbsa.lbsa_partition_perm(T, H, W, "3d", device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    sc = lbsa.lbsa_score(qp, kp, wl.block)
    bs = lbsa.lbsa_select(sc, wl.block, P, "row")
    fl, _ = flops_of(bs, wl)
    qkv_bytes = 3 * q.numel() * q.element_size()
    t = _timer(lambda: lbsa.lbsa_permute([q, k, v], perm, outs=[qp, kp, vp]), flush=flush)
    emit(workload="wan", stage="permute_qkv", **t, **hbm(2 * qkv_bytes, t["median"]))
    t = _timer(lambda: lbsa.lbsa_score(qp, kp, wl.block, scores=sc))
    emit(workload="wan", stage="score_exact", **t, **tfl(2.0 * wl.n_valid ** 2 * wl.d * wl.H, t["median"]))
    t = _timer(lambda: lbsa.lbsa_select(sc, wl.block, P, "row"), flush=flush)
    emit(workload="wan", stage="select_row", **t, **hbm(sc.numel() * 4, t["median"]))
    t = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, bs))
    emit(workload="wan", stage="attend", density=fl / (4.0 * wl.d * wl.n_valid ** 2 * wl.H), **t, **tfl(fl, t["median"]))
    dense = lbsa.lbsa_select(sc, wl.block, 1.0, "row")
    fld, _ = flops_of(dense, wl)
    t = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, dense))
    emit(workload="wan", stage="attend_dense_p1", **t, **tfl(fld, t["median"]))
    t = _timer(lambda: torch.nn.functional.scaled_dot_product_attention(qp, kp, vp))
    emit(workload="wan", stage="torch_sdpa_dense (library reference)", **t, **tfl(fld, t["median"]))
    # the fused dense step: dense O and the exact block masses from one sweep
    sc_f, o_f = lbsa.lbsa_score_attend(qp, kp, vp, wl.block)
    t = _timer(lambda: lbsa.lbsa_score_attend(qp, kp, vp, wl.block, scores=sc_f, out=o_f))
    emit(workload="wan", stage="fused_dense_step (dense O + exact masses)", **t, **tfl(fld, t["median"]))
    del sc_f, o_f
    del q, k, v, qp, kp, vp, sc, bs, dense

    # skewed heads: p sweep
    wl = get_workload("wan_skew")
    q, k, v = make_qkv(wl, device="cuda")
    qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
    sc = lbsa.lbsa_score(qp, kp, wl.block)
    for p in wl.extra["p_sweep"]:
        bs = lbsa.lbsa_select(sc, wl.block, p, "row")
        fl, m = flops_of(bs, wl)
        ta = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, bs))
        ts = _timer(lambda: lbsa.lbsa_select(sc, wl.block, p, "row"), flush=flush)
        emit(workload="wan_skew", stage="attend", p=p, density=float(m.mean()),
             density_per_head=[round(float(x), 4) for x in m.mean(axis=(1, 2))], **ta, **tfl(fl, ta["median"]),
             select_ms=ts["median"])
    # the two further rules on the same scores: SCOPE-style floor over row top-p,
    # and VMoBA's Local + TopK at the pages' k values
    rules = [("topp_floor", dict(p=p_)) for p_ in (0.9, 0.99)] + [("local_topk", dict(k=k_)) for k_ in (2, 6, 18)]
    for rule, kw in rules:
        bs = lbsa.lbsa_select_rule(sc, wl.block, rule, n_valid=wl.n_valid, **kw)
        fl, m = flops_of(bs, wl)
        ta = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, bs))
        ts = _timer(lambda: lbsa.lbsa_select_rule(sc, wl.block, rule, n_valid=wl.n_valid, **kw), flush=flush)
        emit(workload="wan_skew", stage="attend", rule=rule, **kw, density=float(m.mean()),
             density_per_head=[round(float(x), 4) for x in m.mean(axis=(1, 2))], **ta, **tfl(fl, ta["median"]),
             select_ms=ts["median"], **{"select_" + k2: v2 for k2, v2 in hbm(sc.numel() * 4, ts["median"]).items()})
    # entropy-routed competition domains (EG-Sparse): heads below the median
    # entropy pooled `group` at a time, the rest per row, p = 0.99; and the
    # all-head pool of the abstract's diagnostic (every head routed, one pool)
    _, ent, _ = lbsa.lbsa_select_routed(sc, wl.block, 0.99, -1.0, 1)
    thr = median_entropy(ent[0])
    for thr_, group in ((thr, 3), (thr, 6), (thr, wl.H), (2.0, wl.H)):
        bs, _, dom = lbsa.lbsa_select_routed(sc, wl.block, 0.99, thr_, group)
        fl, m = flops_of(bs, wl)
        ta = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, bs))
        ts = _timer(lambda: lbsa.lbsa_select_routed(sc, wl.block, 0.99, thr_, group), flush=flush)
        emit(workload="wan_skew", stage="attend", rule="routed", p=0.99, entropy_threshold=round(thr_, 6),
             group=group, routed_heads=int((dom >= 0).sum()), entropy=[round(float(x), 4) for x in ent[0]],
             density=float(m.mean()), density_per_head=[round(float(x), 4) for x in m.mean(axis=(1, 2))],
             empty_rows=float((m.sum(axis=2) == 0).mean()), **ta, **tfl(fl, ta["median"]), select_ms=ts["median"],
             **{"select_" + k2: v2 for k2, v2 in hbm(sc.numel() * 4, ts["median"]).items()})
    del q, k, v, qp, kp, vp, sc

    # proxy mode: 1D / 2D / 3D cycle, head-scope selection at tau = 0.25
    wl = get_workload("wan_proxy")
    q, k, v = make_qkv(wl, device="cuda")
    for call in range(3):
        kind = ("1d", "2d", "3d")[call]
        perm = lbsa.lbsa_partition_perm(T, H, W, kind, device="cuda")
        qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
        sc = lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool")
        bs = lbsa.lbsa_select(sc, wl.block, 0.25, "head")
        fl, m = flops_of(bs, wl)

        def full_call():
            a, b_, c = lbsa.lbsa_permute([q, k, v], perm)
            s2 = lbsa.lbsa_score(a, b_, wl.block, mode="meanpool")
            bsx = lbsa.lbsa_select(s2, wl.block, 0.25, "head")
            o = lbsa.lbsa_attend(a, b_, c, bsx)
            lbsa.lbsa_permute([o], perm, inverse=True)

        tm = _timer(lambda: lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool", scores=sc), flush=flush)
        th = _timer(lambda: lbsa.lbsa_select(sc, wl.block, 0.25, "head"), flush=flush)
        ta = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, bs))
        tc = _timer(full_call, flush=flush)
        empty = float((m.sum(axis=2) == 0).mean())
        emit(workload="wan_proxy", partition=kind, stage="meanpool", **tm, **hbm(2 * q.numel() * 2 + sc.numel() * 4, tm["median"]))
        emit(workload="wan_proxy", partition=kind, stage="select_head", **th, **hbm(3 * sc.numel() * 4, th["median"]))
        emit(workload="wan_proxy", partition=kind, stage="attend", density=float(m.mean()), empty_rows=empty, **ta,
             **tfl(fl, ta["median"]))
        emit(workload="wan_proxy", partition=kind, stage="full_call", **tc)
    del q, k, v, qp, kp, vp, sc

    # per-token proxy (VMoBA's literal scoring): every query token scores the key-block
    # means, head-scope selection at tau = 0.25 over the (token, key block) pairs
    wl = get_workload("wan_proxy")
    q, k, v = make_qkv(wl, device="cuda")
    for kind in ("1d", "2d", "3d"):
        perm = lbsa.lbsa_partition_perm(T, H, W, kind, device="cuda")
        qp, kp, vp = lbsa.lbsa_permute([q, k, v], perm)
        sc = lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool_token")
        bs = lbsa.lbsa_select_tokens(sc, wl.block, 0.25)
        fl, dens, empty = token_flops(lbsa, bs, wl)
        tm = _timer(lambda: lbsa.lbsa_score(qp, kp, wl.block, mode="meanpool_token", scores=sc), flush=flush)
        th = _timer(lambda: lbsa.lbsa_select_tokens(sc, wl.block, 0.25), flush=flush)
        ta = _timer(lambda: lbsa.lbsa_attend(qp, kp, vp, bs))
        emit(workload="wan_proxy_token", partition=kind, stage="meanpool_token", **tm,
             **hbm(2 * q.numel() * 2 + sc.numel() * 4, tm["median"]))
        emit(workload="wan_proxy_token", partition=kind, stage="select_tokens", **th, **hbm(sc.numel() * 4, th["median"]))
        emit(workload="wan_proxy_token", partition=kind, stage="attend", density=dens, empty_tokens=empty, **ta,
             **tfl(fl, ta["median"]))
        del sc, bs
    del q, k, v, qp, kp, vp

    # HunyuanVideo-like layer: select once, 49 re-drawn attend calls on the frozen blockset
    wl = get_workload("hunyuan")
    q32, k32, v32 = make_qkv_f32(wl, device="cuda")
    q, k, v = (x.to(torch.bfloat16) for x in (q32, k32, v32))
    t = _timer(lambda: lbsa.lbsa_score(q, k, wl.block), n=3, warm=1)
    sc = lbsa.lbsa_score(q, k, wl.block)
    emit(workload="hunyuan", stage="score_exact", **t, **tfl(2.0 * wl.n_valid ** 2 * wl.d * wl.H, t["median"]))
    bs = lbsa.lbsa_select(sc, wl.block, P, "row")
    t = _timer(lambda: lbsa.lbsa_select(sc, wl.block, P, "row"), flush=flush)
    emit(workload="hunyuan", stage="select_row", **t, **hbm(sc.numel() * 4, t["median"]))
    fl, m = flops_of(bs, wl)
    times = []
    for step in range(1, wl.extra["steps"] + 1):
        q, k, v = redraw_qkv(wl, q32, k32, v32, step)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lbsa.lbsa_attend(q, k, v, bs)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ts = sorted(times)
    med = ts[len(ts) // 2]
    emit(workload="hunyuan", stage="attend_frozen_x49", density=float(m.mean()), median=med, p10=ts[4], p90=ts[44],
         **tfl(fl, med))
    dense = lbsa.lbsa_select(sc, wl.block, 1.0, "row")
    fld, _ = flops_of(dense, wl)
    t = _timer(lambda: lbsa.lbsa_attend(q, k, v, dense), n=3, warm=1)
    emit(workload="hunyuan", stage="attend_dense_p1", **t, **tfl(fld, t["median"]))
    t = _timer(lambda: torch.nn.functional.scaled_dot_product_attention(q, k, v), n=3, warm=1)
    emit(workload="hunyuan", stage="torch_sdpa_dense (library reference)", **t, **tfl(fld, t["median"]))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="leave out the measurements beside the contract's timed calls (dense, step 0, configs 0-4)")
    ap.add_argument("--clocks-csv", default=None, help="where the nvidia-smi clock samples go (default under /tmp)")
    ap.add_argument("--profile", choices=["attend", "dense", "fused", "score", "select", "proxy", "token", "routed"],
                    help="run the small ncu case for one kernel instead of the benchmark")
    ap.add_argument("--sweep", action="store_true", help="per-stage timings on every workload (not the contract line)")
    args = ap.parse_args()
    if args.profile:
        return run_profile(args.profile)
    if args.sweep:
        return run_sweep(args)
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # the CPU oracle on rank 0 alone: no process group, no device
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_own(args, rank, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
