"""Planted mistakes in the oracle are caught by its pins (CPU only).

The oracle is trusted because its pins (library routines, closed forms, brute
force, hand-worked cases under tests/golden/) would notice a plausible mistake
in it.  This file checks that claim directly.  Each case takes the source of
one oracle function, makes one plausible mistake in it by a textual edit (a
dropped term, a wrong sign or index, a transposed operand, > where the reading
is >=, a floor where it is a ceiling, ...), executes the edited copy in the
namespace of the function's own module and swaps it in for the real function
while the pin tests of that module run.  At least one pin must then fail.

The edit must match the source exactly once, so a case cannot pass vacuously
after the oracle is reworded; and the same runner, with nothing planted, must
see every pin pass.
"""
import importlib
import inspect
import textwrap

import numpy as np
import pytest

import oracle

import test_oracle_attention
import test_oracle_partition
import test_oracle_scores
import test_oracle_select
import test_oracle_select_routed
import test_oracle_select_variants
import test_oracle_token_proxy

# the submodules by name (the package re-exports a function called select_routed,
# which shadows the submodule of that name as an attribute)
A, S, SEL, V, R, P = (importlib.import_module("oracle." + m) for m in
                      ("attention", "scores", "select", "select_variants", "select_routed", "partition"))

# oracle module -> the test modules that pin it
PINS = {
    A: (test_oracle_attention, test_oracle_token_proxy),
    S: (test_oracle_scores, test_oracle_token_proxy),
    SEL: (test_oracle_select,),
    V: (test_oracle_select_variants,),
    R: (test_oracle_select_routed,),
    P: (test_oracle_partition,),
}

# (module, function, text in its source, replacement, the mistake in words)
PLANTED = [
    # exact block mass (LoSA)
    (S, "block_mass", "@ kk.T) * scale", "@ kk.T)", "logits without 1/sqrt(d)"),
    (S, "block_mass", ".sum(axis=1).mean()", ".sum(axis=1).sum()", "block rows summed, not averaged"),
    (S, "block_mass", "kk = k[b, h, :n_valid]", "kk = q[b, h, :n_valid]", "queries in place of keys"),
    (S, "block_mass", "kk = k[b, h, :n_valid]", "kk = k[b, h]", "padding keys inside the softmax"),
    (S, "block_mass", "e / e.sum(axis=1, keepdims=True)", "e / e.sum(axis=0, keepdims=True)",
     "softmax over the query axis"),
    (S, "block_mass", "c0, c1 = j * block, min(", "c0, c1 = j * block + 1, min(",
     "key block starts one token late"),
    (S, "block_mass", "r0, r1 = int(i) * block, min((int(i) + 1) * block, n_valid)",
     "r0, r1 = n * block, min((n + 1) * block, n_valid)", "query block taken by its position in qblocks, not its id"),
    # block-mean proxy (VMoBA)
    (S, "meanpool_scores", "out[b, h] = e / e.sum()", "out[b, h] = e / e.sum(axis=1, keepdims=True)",
     "softmax per query block instead of over the head"),
    (S, "meanpool_scores", "s = (qbar @ kbar.T) / np.sqrt(d)", "s = qbar @ kbar.T", "logits without 1/sqrt(d)"),
    (S, "meanpool_scores", "qbar = np.stack([q[b, h,", "qbar = np.stack([k[b, h,", "key means in place of query means"),
    (S, "meanpool_scores", "kbar = np.stack([k[b, h, j * block:min((j + 1) * block, n_valid)]",
     "kbar = np.stack([k[b, h, j * block:(j + 1) * block]", "ragged key block averaged over padding"),
    (S, "meanpool_scores", "e = np.exp(s - s.max())", "e = np.exp(s.max() - s)", "wrong sign in the exponent"),
    # per-token proxy
    (S, "token_meanpool_scores", "out[b, h] = e / e.sum()", "out[b, h] = e / e.sum(axis=1, keepdims=True)",
     "softmax per token instead of over the head"),
    (S, "token_meanpool_scores", "s = (q[b, h, :n_valid] @ kbar.T) / np.sqrt(d)", "s = q[b, h, :n_valid] @ kbar.T",
     "logits without 1/sqrt(d)"),
    (S, "token_meanpool_scores", "k[b, h, j * block:min((j + 1) * block, n_valid)]", "k[b, h, j * block:(j + 1) * block]",
     "ragged key block averaged over padding"),
    # dense attention
    (A, "dense_attention", "@ k[b, h, :n_valid].T) * scale", "@ k[b, h, :n_valid].T)", "logits without 1/sqrt(d)"),
    (A, "dense_attention", "lse[b, h] = (m + np.log(l))[:, 0]", "lse[b, h] = np.log(l)[:, 0]",
     "log-sum-exp without the row maximum"),
    (A, "dense_attention", "(e / l) @ v[b, h, :n_valid]", "(e / l) @ k[b, h, :n_valid]", "keys in place of values"),
    (A, "dense_attention", "O[b, h] = (e / l) @", "O[b, h] = e @", "probabilities not normalised"),
    (A, "dense_attention", "z = (q[b, h, rows] @", "z = (q[b, h, :len(rows)] @", "the first rows in place of the asked ones"),
    # block-sparse attention
    (A, "sparse_attention", "l = e.sum(axis=1, keepdims=True)", "l = e.sum(axis=1, keepdims=True) + 1.0",
     "normaliser with a stray term (not renormalised over the kept keys)"),
    (A, "sparse_attention", "np.arange(j * block, min((j + 1) * block, n_valid))", "np.arange(j * block, (j + 1) * block)",
     "padding keys of a ragged last block attended"),
    (A, "sparse_attention", "r0, r1 = int(i) * block, min(", "r0, r1 = int(i) * block + 1, min(",
     "query rows shifted by one"),
    (A, "sparse_attention", "lse = np.full((B, H, len(qblocks) * block), -np.inf)",
     "lse = np.zeros((B, H, len(qblocks) * block))", "empty rows get lse 0"),
    (A, "sparse_attention", "z = (q[b, h, r0:r1] @ k[b, h, keys].T) * scale", "z = (q[b, h, r0:r1] @ k[b, h, keys].T)",
     "logits without 1/sqrt(d)"),
    (A, "token_sparse_attention", "z = (k[b, h, keys] @ q[b, h, int(t)]) * scale", "z = (k[b, h, keys] @ q[b, h, int(t)])",
     "logits without 1/sqrt(d)"),
    (A, "token_sparse_attention", "O[b, h, n] = (e / l) @ v[b, h, keys]", "O[b, h, n] = (e / l) @ k[b, h, keys]",
     "keys in place of values"),
    (A, "sparse_attention", "r = (b * H + h) * nB + int(i)", "r = (h * B + b) * nB + int(i)",
     "CSR row numbered head-major across the batch"),
    (A, "sparse_attention", "o0 = n * block", "o0 = int(i) * block", "output placed by block id, not position"),
    (A, "token_sparse_attention", "r = (b * H + h) * n_valid + int(t)", "r = (h * B + b) * n_valid + int(t)",
     "CSR row numbered head-major across the batch"),
    # fixed-point selection contract
    (SEL, "threshold_fixed_point", "return -((-num) >> 24)", "return num >> 24", "threshold floored, not ceiled"),
    (SEL, "threshold_fixed_point", "P = round(float(p) * (1 << 24))", "P = int(float(p) * (1 << 24))",
     "p truncated to 24 bits, not rounded"),
    (SEL, "_segment_keep", "csum >= T", "csum > T", "strict > where the rule reads >="),
    (SEL, "_segment_keep", "np.lexsort((idx, -bits", "np.lexsort((-idx, -bits", "ties go to the higher index"),
    (SEL, "_segment_keep", "np.lexsort((idx, -bits.astype(np.int64)))", "np.lexsort((idx, bits.astype(np.int64)))",
     "ascending sort"),
    (SEL, "_segment_keep", "k = int(hit[0]) + 1 if len(hit) else n", "k = int(hit[0]) if len(hit) else n",
     "prefix one short"),
    (SEL, "_segment_keep", "if p >= 1.0:", "if p > 1.0:", "p = 1 not the dense set"),
    (SEL, "_weights", "np.floor(x32.astype(np.float64) * 4294967296.0)", "np.round(x32.astype(np.float64) * 4294967296.0)",
     "weights rounded, not floored"),
    (SEL, "_weights", "if np.any(bits >= np.uint32(0x40000000)):", "if False:", "invalid scores accepted"),
    (SEL, "select_contract", "per[int(f) // nK].append(int(f) % nK)", "per[int(f) % nQ].append(int(f) // nQ)",
     "head scope: flat index split transposed"),
    (SEL, "select_contract", "_segment_keep(bits[b, h].reshape(-1), w[b, h].reshape(-1), p)",
     "_segment_keep(bits[b, h].T.reshape(-1), w[b, h].T.reshape(-1), p)", "head scope: pairs flattened key-block major"),
    (SEL, "select_fp64", "if c >= p * total:", "if c > p * total:", "fp64 rule: strict > where it reads >="),
    (SEL, "select_fp64", "order = np.lexsort((np.arange(n), -seg))", "order = np.lexsort((-np.arange(n), -seg))",
     "fp64 rule: ties go to the higher index"),
    (SEL, "csr_from_rows", "row_ptr[r + 1] = row_ptr[r] + len(c)", "row_ptr[r + 1] = len(c)",
     "CSR offsets not accumulated"),
    # Local + TopK and the per-head floor
    (V, "_order", "np.lexsort((np.arange(n), -bits_row", "np.lexsort((-np.arange(n), -bits_row",
     "ties go to the higher id"),
    (V, "select_local_topk", "order = [j for j in _order(bits[b, h, i]) if j != i]",
     "order = [j for j in _order(bits[b, h, i])]", "the diagonal block counted among the top k"),
    (V, "select_local_topk", "np.asarray([i] + order[:k]", "np.asarray(order[:k + 1]", "the diagonal block not forced"),
    (V, "floor_of_head", "return -((-num) // den)", "return num // den", "floor mean rounded down"),
    (V, "floor_of_head", "v = [min(block, n_valid - i * block) for i in range(nQ)]", "v = [block for i in range(nQ)]",
     "floor mean not weighted by the ragged block's size"),
    (V, "select_topp_floor", "n = max(counts[i], min(K, nK))", "n = min(K, nK)", "floor replaces a longer row"),
    # entropy-routed domains
    (R, "head_entropy", "out[b, h] = total / nQ / math.log(nB)", "out[b, h] = total / nQ",
     "entropy not normalised by log nB"),
    (R, "head_entropy", "pi = row[row > 0.0] / s", "pi = row[row > 0.0]", "row not normalised to a distribution"),
    (R, "head_entropy", "out[b, h] = total / nQ / math.log(nB)", "out[b, h] = total / math.log(nB)",
     "rows summed, not averaged"),
    (R, "route_heads", "e[b, h] < threshold", "e[b, h] > threshold", "high-entropy heads pooled"),
    (R, "route_heads", "pool[b, h] = rank // group", "pool[b, h] = rank % group", "pools dealt round-robin"),
    (R, "select_routed", "mine = kept[(kept // nB) == m] % nB", "mine = kept[(kept % nB) == m] // nB",
     "pool member index and block id transposed"),
    # token orders
    (P, "perm_1d_temporal", "(t * H + h) * W + w", "(h * T + t) * W + w", "1D order indexes a transposed grid"),
    (P, "perm_2d_frame_tiles", "for h in range(h0, min(h0 + th, H)):", "for h in range(h0, h0 + th):",
     "frame tiles not truncated at the edge"),
    (P, "perm_2d_frame_tiles", "for h0 in range(0, H, th):\n            for w0 in range(0, W, tw):",
     "for w0 in range(0, W, tw):\n            for h0 in range(0, H, th):", "frame tiles walked column by column"),
    (P, "perm_3d_tiles", "for w in range(w0, min(w0 + tw, W)):", "for w in range(w0, W):",
     "3D tiles run to the row end"),
    (P, "perm_3d_tiles", "for t in range(t0, min(t0 + tt, T)):\n                    for h in range(h0, min(h0 + th, H)):",
     "for h in range(h0, min(h0 + th, H)):\n                    for t in range(t0, min(t0 + tt, T)):",
     "3D tile walks h before t"),
    (P, "perm_for_call", "PARTITION_CYCLE[call % 3]", "PARTITION_CYCLE[(call + 1) % 3]", "cycle starts at 2D"),
]


def _planted(module, name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(module, name)))
    assert src.count(old) == 1, f"{module.__name__}.{name}: the edit must match its source once: {old!r}"
    ns = dict(vars(module))
    exec(compile(src.replace(old, new), f"<planted {module.__name__}.{name}>", "exec"), ns)
    return ns[name]


def _pin_calls(test_module):
    """Every pin test of a module as (id, zero-argument call), parametrisations expanded."""
    for name, fn in sorted(vars(test_module).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            yield name, fn
            continue
        assert len(marks) == 1 and "," not in marks[0].args[0], name
        arg = marks[0].args[0]
        for n, val in enumerate(marks[0].args[1]):
            yield f"{name}[{n}]", (lambda f=fn, a=arg, x=val: f(**{a: x}))


def _failing_pins(module):
    failed = []
    for test_module in PINS[module]:
        for pid, call in _pin_calls(test_module):
            try:
                with np.errstate(all="ignore"):
                    call()
            except (Exception, pytest.fail.Exception):
                failed.append(f"{test_module.__name__}::{pid}")
    return failed


@pytest.mark.parametrize("module", list(PINS), ids=lambda m: m.__name__)
def test_runner_sees_every_pin_pass_with_nothing_planted(module):
    assert _failing_pins(module) == []


@pytest.mark.parametrize("module,name,old,new,what", PLANTED,
                         ids=[f"{m.__name__.split('.')[-1]}.{n}:{w}" for m, n, _, _, w in PLANTED])
def test_planted_mistake_fails_a_pin(module, name, old, new, what, monkeypatch):
    mutant = _planted(module, name, old, new)
    monkeypatch.setattr(module, name, mutant)
    if getattr(oracle, name, None) is not None:
        monkeypatch.setattr(oracle, name, mutant)
    failed = _failing_pins(module)
    assert failed, f"no pin notices: {what} ({module.__name__}.{name})"
