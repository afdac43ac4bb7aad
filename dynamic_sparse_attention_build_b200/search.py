"""Kernel-aware per-head pattern search.

The MInference 1.0 summary (section "オフライン探索", offline search) assigns every
attention head one sparse pattern ahead of time, choosing among the pattern
types by what the GPU kernels actually cost, subject to keeping the attention
the head really pays.  This module does that with this library's own kernels:

* for each head and each candidate pattern, the head alone is run as a
  one-head problem through ``build_indices`` and ``sparse_prefill``; the time is
  the median of a few CUDA-event timings of the two calls;
* the candidate is scored by attention recall, the share of each row's softmax
  mass that the pattern's mask keeps:
      recall_i = sum_{j in M_i} p_ij = exp(LSE_sparse,i - LSE_dense,i),
  with p the causal softmax of the row and the dense log-sum-exp from the same
  kernel over every causal block (rows whose mask is empty have recall 0);
* the chosen pattern is the fastest candidate whose mean recall reaches the
  target; the dense candidate (every causal block) closes every list, so some
  candidate always qualifies.

Inputs are the layer's Q, K, V on the GPU ([heads, tokens, d], bf16); for a
real model these would be calibration activations, here they are the synthetic
workloads.  Nothing in the search runs on the CPU except the bookkeeping.
"""
from __future__ import annotations

import statistics
from dataclasses import dataclass

import torch

from . import api


def default_candidates(N: int, block: int) -> list[dict]:
    """Pattern candidates of the three MInference types (A-shape, Vertical-Slash,
    block-sparse) plus the FlashPrefill threshold, sized for N tokens, and the
    dense pattern last."""
    nb = -(-N // block)
    c = [dict(kind="ashape", sink=64, window=w) for w in (256, 1024, 4096) if w < N]
    c += [dict(kind="vs", last_q=64, n_vert=v, n_slash=s) for v, s in ((100, 400), (500, 2000), (1000, 6096))
          if v + s < N]
    c += [dict(kind="block_topk", topk=k) for k in (8, 32, 100) if k < nb]
    c += [dict(kind="block_threshold", alpha=0.5, keep_sink=1, keep_local=1)]
    c += [dense_pattern(N, block)]
    return c


def dense_pattern(N: int, block: int) -> dict:
    """Every causal key block (block top-k with k = number of blocks)."""
    return dict(kind="block_topk", topk=-(-N // block))


def attention_recall(lse_sparse: torch.Tensor, lse_dense: torch.Tensor) -> torch.Tensor:
    """Per-row share of the causal softmax mass inside the sparse mask:
    exp(LSE_sparse - LSE_dense), 0 where the mask keeps no key (LSE = -inf)."""
    r = torch.exp(lse_sparse.double() - lse_dense.double())
    return torch.where(torch.isfinite(lse_sparse.double()), r, torch.zeros_like(r))


@dataclass
class Trial:
    head: int
    pattern: dict
    ms: float          # median time of build_indices + sparse_prefill for this head
    recall: float      # mean attention recall over the head's rows
    min_recall: float  # lowest row recall
    pairs: int         # allowed (query, key) pairs of the mask


def choose(trials: list[Trial], recall_target: float) -> Trial:
    """The fastest trial whose mean recall reaches the target; if none does,
    the one with the highest recall (ties: the faster one)."""
    ok = [t for t in trials if t.recall >= recall_target]
    if ok:
        return min(ok, key=lambda t: (t.ms, -t.recall))
    return max(trials, key=lambda t: (t.recall, -t.ms))


def _time_head(Qh, Kh, Vh, pattern, block, repeats):
    idx = api.build_indices(Qh, Kh, [pattern], block)
    O, lse = api.sparse_prefill(Qh, Kh, Vh, idx, want_lse=True)
    times = []
    for _ in range(repeats):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        api.build_indices(Qh, Kh, [pattern], block, bufs=idx)
        api.sparse_prefill(Qh, Kh, Vh, idx, O=O, lse=lse)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    pairs = int(api.count_pairs(Qh, Kh, idx).item())
    return statistics.median(times), lse[0], pairs


def search_patterns(Q, K, V, block, candidates=None, recall_target=0.95, repeats=3, heads=None):
    """Chooses one pattern per q-head.  Returns (patterns, trials): the list of
    chosen pattern dicts (one per head, ready for ``build_indices``) and every
    Trial, in (head, candidate) order.  ``heads`` limits the search to some
    heads (the others get the dense pattern)."""
    if not Q.is_cuda:
        raise RuntimeError("search_patterns runs the library's CUDA kernels: Q, K, V must be on the GPU")
    Hq, N, _ = Q.shape
    G = Hq // K.shape[0]
    cands = list(candidates) if candidates is not None else default_candidates(N, block)
    dense = dense_pattern(N, block)
    if dense not in cands:
        cands.append(dense)
    heads = range(Hq) if heads is None else heads
    chosen = [dict(dense) for _ in range(Hq)]
    trials = []
    for h in heads:
        kvh = h // G
        Qh, Kh, Vh = Q[h:h + 1], K[kvh:kvh + 1], V[kvh:kvh + 1]
        _, lse_d, _ = _time_head(Qh, Kh, Vh, dense, block, 1)
        lse_d = lse_d.clone()
        ht = []
        for c in cands:
            ms, lse_s, pairs = _time_head(Qh, Kh, Vh, c, block, repeats)
            r = attention_recall(lse_s, lse_d)
            ht.append(Trial(h, dict(c), ms, float(r.mean()), float(r.min()), pairs))
        trials += ht
        chosen[h] = dict(choose(ht, recall_target).pattern)
    return chosen, trials


def summary(trials: list[Trial], chosen: list[dict]) -> str:
    """One line per head: the chosen pattern and its time / recall."""
    lines = []
    by_head = {}
    for t in trials:
        by_head.setdefault(t.head, []).append(t)
    for h, ts in sorted(by_head.items()):
        c = next(t for t in ts if t.pattern == chosen[h])
        lines.append(f"head {h}: {c.pattern} {c.ms:.3f} ms recall {c.recall:.4f} (min {c.min_recall:.4f}), "
                     f"density {c.pairs / max(1, _causal_pairs(ts)):.4f}")
    return "\n".join(lines)


def _causal_pairs(ts: list[Trial]) -> int:
    # the dense trial keeps every causal pair
    return max(t.pairs for t in ts)


__all__ = ["Trial", "attention_recall", "choose", "default_candidates", "dense_pattern", "search_patterns",
           "summary"]


def _main():
    """python -m dynamic_sparse_attention_build_b200.search [--workload k] [--N n]
    [--heads a-b] [--target r]: the search on a seeded synthetic workload; prints
    one line per head and a JSON summary line."""
    import argparse
    import json
    import os
    import sys
    import time

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--N", type=int, default=0)
    ap.add_argument("--heads", default="0-7")
    ap.add_argument("--target", type=float, default=0.95)
    ap.add_argument("--repeats", type=int, default=3)
    args = ap.parse_args()
    w = synth.workload(args.workload, **({"N": args.N} if args.N else {}))
    Q, K, V, _ = synth.make_inputs(w, device="cuda")
    a, _, b = args.heads.partition("-")
    heads = list(range(int(a), int(b or a) + 1))
    t0 = time.perf_counter()
    chosen, trials = search_patterns(Q, K, V, w["B"], recall_target=args.target, repeats=args.repeats, heads=heads)
    secs = time.perf_counter() - t0
    print(summary(trials, chosen))
    print(json.dumps({"workload": w["name"], "N": w["N"], "heads": heads, "target": args.target,
                      "seconds": secs, "trials": len(trials),
                      "chosen": {h: chosen[h] for h in heads}}))


if __name__ == "__main__":
    _main()
