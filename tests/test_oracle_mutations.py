"""The oracle's pins have teeth: each test plants one plausible mistake (a dropped
term, a wrong sign, an off-by-one, a flipped tie rule, a transposed operand) in a
copy of the oracle, on the CPU, and checks that the pins of tests/test_oracle_pins.py
relevant to it fail.  The library is never touched.  CPU only."""
import inspect
import os
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle", "dsa_oracle.py")

ASHAPE = "ashape or empty or attention"
VSK = "vs_estimate or superset or planted"
SEL = "moba or threshold or block_score"
ATT = "attention or empty or dense or ashape or pairs"
RUNS = "slash or window or mirrored"

# (name, original text, planted text, pins to run)
MUTANTS = [
    ("ashape window off by one", "(i - j < window)", "(i - j <= window)", ASHAPE),
    ("ashape sink off by one", "(j < sink)", "(j <= sink)", ASHAPE),
    ("ashape not causal", "return (j <= i) & ((j < sink)", "return ((j < sink)", ASHAPE),
    ("vs estimate without tau", "logits = tau * (Kh[: i + 1] @ Qh[i])\n        p",
     "logits = (Kh[: i + 1] @ Qh[i])\n        p", VSK),
    ("vs estimate drops the diagonal key", "logits = tau * (Kh[: i + 1] @ Qh[i])\n        p",
     "logits = tau * (Kh[: i + 1] @ Qh[i])\n        logits[-1] = -np.inf if i > 0 else logits[-1]\n        p", VSK),
    ("vs slash offset sign", "s[i - np.arange(i + 1)] += p", "s[np.arange(i + 1)] += p", VSK),
    ("vs estimate one row short", "for i in range(max(0, N - last_q), N):",
     "for i in range(max(0, N - last_q + 1), N):", VSK),
    ("vs estimate unnormalised", "        p /= p.sum()\n        v[: i + 1] += p", "        v[: i + 1] += p", VSK),
    ("top-k ties to the higher index", "order = np.lexsort((np.arange(x.size), -x))",
     "order = np.lexsort((-np.arange(x.size), -x))", "topk"),
    ("top-k of the smallest", "order = np.lexsort((np.arange(x.size), -x))",
     "order = np.lexsort((np.arange(x.size), x))", "topk or planted"),
    ("distances floor only", "D = np.union1d(S // B, -((-S) // B))", "D = np.unique(S // B)", "distance or superset"),
    ("distances not clipped", "return D[D < nkb].astype(np.int64)", "return D.astype(np.int64)", "distance"),
    ("columns visible one block late", "if j <= qb * B + B - 1 and (qb - j // B) not in Dset]",
     "if j <= qb * B and (qb - j // B) not in Dset]", "superset"),
    ("columns keep covered keys", "if j <= qb * B + B - 1 and (qb - j // B) not in Dset]",
     "if j <= qb * B + B - 1]", "superset"),
    ("partial block pooled over B", "out[b] = X[b * B: min(N, b * B + B)].mean(axis=0)",
     "out[b] = X[b * B: min(N, b * B + B)].sum(axis=0) / B", "mean_pool or block_score"),
    ("block scores without tau", "return (qbar @ kbar.T) / math.sqrt(d)", "return (qbar @ kbar.T)", "block_score"),
    ("block scores transposed", "return (qbar @ kbar.T) / math.sqrt(d)", "return (kbar @ qbar.T) / math.sqrt(d)",
     "block_score"),
    ("key conv without residual", "return Kh + silu(conv + bias[None, :])", "return silu(conv + bias[None, :])",
     "key_conv"),
    ("key conv without bias", "return Kh + silu(conv + bias[None, :])", "return Kh + silu(conv)", "key_conv"),
    ("key conv anti-causal", "shifted[t:] = Kh[: N - t] if t < N else 0.0",
     "shifted[: N - t] = Kh[t:] if t < N else 0.0", "key_conv"),
    ("silu sign", "return x / (1.0 + np.exp(-x))", "return x / (1.0 + np.exp(x))", "key_conv"),
    ("block top-k without the own block", "return topk_indices(scores_row[: I + 1], k)",
     "return topk_indices(scores_row[: I], k) if I > 0 else np.zeros(0, np.int64)", SEL),
    ("moba without the own block", "return np.union1d(past, [I]).astype(np.int64)",
     "return past.astype(np.int64)", SEL),
    ("moba ranks the own block", "past = topk_indices(scores_row[:I], k) if I > 0",
     "past = topk_indices(scores_row[:I + 1], k) if I >= 0", SEL),
    ("threshold strict", "kept = np.nonzero(P >= alpha * P.max())[0]", "kept = np.nonzero(P > alpha * P.max())[0]",
     SEL),
    ("threshold without the sink", "extra = ([0] if keep_sink else [])", "extra = ([])", SEL),
    ("threshold on logits", "kept = np.nonzero(P >= alpha * P.max())[0]",
     "kept = np.nonzero(logits >= alpha * logits.max())[0]", SEL),
    ("attention without tau", "logits = tau * (Kh[J] @ Qh[i])", "logits = (Kh[J] @ Qh[i])", ATT),
    ("lse without the max", "lse[r] = m + math.log(w.sum())", "lse[r] = math.log(w.sum())", ATT),
    ("attention not causal", "keys = keys[(keys <= i) & (keys < hi.N)]", "keys = keys[(keys < hi.N)]", ATT),
    ("attention ignores the A-shape predicate", "keys = keys[ashape_allowed(i, keys, hi.sink, hi.window)]",
     "keys = keys", ATT),
    ("empty row attends to itself", "        if J.size == 0:\n            continue",
     "        if J.size == 0:\n            J = np.array([i])", ATT),
    ("pair count off by one", "total += allowed_keys(hi, i).size",
     "total += allowed_keys(hi, i).size + (1 if i == 0 else 0)", "pairs"),
    ("block pair count excludes the diagonal key", 'upto_i = np.searchsorted(keys, rows, side="right")',
     'upto_i = np.searchsorted(keys, rows, side="left")', "pairs_by_block"),
    ("block pair count adds the sink twice", "total += int((sink_n + win_n - both_n).sum())",
     "total += int((sink_n + win_n).sum())", "pairs_by_block"),
    ("block pair count window one short", "win_lo = rows - hi.window + 1", "win_lo = rows - hi.window + 2",
     "pairs_by_block"),
    ("unified vertical sums over the keys", "V = P.sum(axis=0)", "V = P.sum(axis=1)", "unified"),
    ("unified diagonal above the main one", "G = np.array([np.trace(P, offset=-dd) for dd in range(nqb)])",
     "G = np.array([np.trace(P, offset=dd) for dd in range(nqb)])", "unified"),
    ("unified diagonal block one off", "I - diag[diag <= I]", "I - diag[diag <= I] - 1", "unified"),
    ("slash runs: touching windows not merged", "if runs and a <= runs[-1][1] + 1:",
     "if runs and a <= runs[-1][1]:", RUNS),
    ("slash runs: window end from r0 + B", "a, b = max(0, r0 - o), r1 - o", "a, b = max(0, r0 - o), r0 + B - 1 - o",
     RUNS),
    ("slash runs: no clip at key 0", "a, b = max(0, r0 - o), r1 - o", "a, b = r0 - o, r1 - o", RUNS),
    ("slash runs: columns keep run keys", "if j <= qb * B + B - 1 and not any(a <= j <= b for a, b in runs)]",
     "if j <= qb * B + B - 1]", RUNS),
]


def _load_mutant(src: str):
    """The oracle's source with one mistake planted, as a fresh module object."""
    name = "oracle._dsa_oracle_mutant"
    mod = types.ModuleType(name)
    mod.__file__ = ORACLE
    sys.modules[name] = mod  # dataclasses resolve annotations through sys.modules
    try:
        exec(compile(src, ORACLE, "exec"), mod.__dict__)
    finally:
        del sys.modules[name]
    return mod


def _calls(fn):
    """Every argument set pytest would call a pin with (its parametrize marks
    expanded; the seeded rng fixture as conftest defines it)."""
    cases = [{}]
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names = [n.strip() for n in mark.args[0].split(",")]
        expanded = []
        for case in cases:
            for vals in mark.args[1]:
                vals = vals if len(names) > 1 else (vals,)
                expanded.append(dict(case, **dict(zip(names, vals))))
        cases = expanded
    if "rng" in inspect.signature(fn).parameters:
        cases = [dict(c, rng=np.random.default_rng(12345)) for c in cases]
    return cases


def _pins_fail(mutant, keywords: str) -> bool:
    from tests import test_oracle_pins as pins
    words = [w.strip() for w in keywords.split(" or ")]
    selected = [getattr(pins, n) for n in dir(pins)
                if n.startswith("test_") and any(w in n for w in words)]
    assert selected, keywords
    saved = pins.orc
    pins.orc = mutant
    try:
        for fn in selected:
            for kwargs in _calls(fn):
                try:
                    fn(**kwargs)
                except Exception:
                    return True
        return False
    finally:
        pins.orc = saved


@pytest.mark.parametrize("name,original,planted,pins", MUTANTS, ids=[m[0].replace(" ", "_") for m in MUTANTS])
def test_pins_catch_planted_mistake(name, original, planted, pins):
    src = open(ORACLE, encoding="utf-8").read()
    assert src.count(original) == 1, f"the oracle no longer holds the text this mutant replaces: {name}"
    assert _pins_fail(_load_mutant(src.replace(original, planted)), pins), f"pins did not catch '{name}'"


def test_unmutated_oracle_passes_the_same_pins():
    src = open(ORACLE, encoding="utf-8").read()
    for kw in sorted({m[3] for m in MUTANTS}):
        assert not _pins_fail(_load_mutant(src), kw), kw
