"""Test helpers bridging oracle results and the library's index buffers."""
import math

import numpy as np
import torch

from oracle import dsa_oracle as orc

# Output tolerances for bf16 inputs against the fp64 oracle, given identical indices.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Index sets may differ only on entries within this relative band of the cut.
TIE_REL = 1e-3


def oracle_heads_to_lists(heads):
    """Oracle HeadIndex list -> dicts accepted by ``indices_from_lists``."""
    out = []
    for hi in heads:
        d = dict(kind=hi.kind, sink=hi.sink, window=hi.window,
                 blocks=[np.asarray(b) for b in hi.blocks],
                 cols=[np.asarray(c) for c in hi.cols])
        if hi.kind == orc.VS and hi.runs is not None:
            d["kind"] = "vs_windows"
            d["dist"] = runs_list_from_slashes(hi.S, hi.B, hi.N)
        elif hi.kind == orc.VS:
            d["dist"] = np.asarray(hi.D)
        out.append(d)
    return out


def gpu_lists_to_oracle_heads(bufs, N, B):
    """Library index buffers -> oracle HeadIndex objects (VS blocks rebuilt from D
    with the oracle's own rule, so the oracle evaluates exactly the GPU's mask)."""
    kinds = {0: orc.ASHAPE, 1: orc.VS, 2: orc.BLOCK_TOPK, 3: orc.BLOCK_THRESHOLD, 4: orc.MOBA, 5: orc.UNIFIED,
             6: orc.VS}
    heads = []
    nqb = (N + B - 1) // B
    for hl in bufs.host_lists():
        hi = orc.HeadIndex(kind=kinds[hl["kind"]], B=B, N=N, sink=hl["sink"], window=hl["window"])
        if hl["kind"] == 6:
            hi.runs = [runs_of_block(hl["dist"], qb, B, N) for qb in range(nqb)]
            hi.blocks = [np.zeros(0, np.int64)] * nqb
        elif hi.kind == orc.VS:
            D = np.asarray(hl["dist"], np.int64)
            hi.D = D
            hi.blocks = [np.sort(qb - D[D <= qb]) for qb in range(nqb)]
        else:
            hi.blocks = [np.asarray(b, np.int64) for b in hl["blocks"]]
        hi.cols = [np.asarray(c, np.int64) for c in hl["cols"]]
        heads.append(hi)
    return heads


def runs_list_from_slashes(S, B, N):
    """The library's slash-run list of a VS_WINDOWS head from its slash offsets
    S: [n, n_last, then (a, b) offset intervals [o, o + L - 1] merged when they
    overlap or touch, for blocks of height B, then for the last block's height]."""
    S = np.sort(np.asarray(S, np.int64))
    nqb = (N + B - 1) // B
    out = []
    counts = []
    for L in (B, N - (nqb - 1) * B):
        iv = []
        for o in S:
            if iv and o <= iv[-1][1] + 1:
                iv[-1][1] = max(iv[-1][1], int(o) + L - 1)
            else:
                iv.append([int(o), int(o) + L - 1])
        counts.append(len(iv))
        out += [x for p in iv for x in p]
    return np.asarray(counts + out, np.int64)


def runs_of_block(lst, qb, B, N):
    """Key runs [first, last] (ascending) of query block qb from a slash-run list."""
    lst = np.asarray(lst, np.int64)
    n, n_last = int(lst[0]), int(lst[1])
    nqb = (N + B - 1) // B
    last = qb == nqb - 1
    iv = lst[2 + (2 * n if last else 0): 2 + 2 * n + (2 * n_last if last else 0)].reshape(-1, 2)
    r1 = min(N - 1, qb * B + B - 1)
    runs = [[max(0, r1 - b), r1 - a] for a, b in iv if r1 - a >= 0]
    return np.asarray(sorted(runs), np.int64).reshape(-1, 2)


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close_outputs(O_gpu, O_ref, what=""):
    err = np.abs(O_gpu - O_ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max abs {mx:.3e}, mean abs {mean:.3e}"
    return mx, mean


def assert_lse_close(lse_gpu, lse_ref, what=""):
    both_inf = np.isneginf(lse_gpu) & np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), np.isneginf(lse_ref)), f"{what}: empty-row sets differ"
    d = np.abs(lse_gpu[~both_inf] - lse_ref[~both_inf])
    assert d.size == 0 or d.max() < 2e-3, f"{what}: lse max diff {d.max():.3e}"


def topk_set_ok(gpu_sel, ref_sel, scores, k, rel=TIE_REL, logit=False):
    """Sets of top-k indices agree except for entries whose oracle score lies
    within the tie band of the k-th largest score (relative for positive sums,
    absolute in logit units, i.e. relative in probability space, for logits)."""
    gpu_sel = set(int(x) for x in gpu_sel)
    ref_sel = set(int(x) for x in ref_sel)
    if gpu_sel == ref_sel:
        return True, ""
    n = scores.size
    kk = min(k, n)
    cut = np.sort(scores)[::-1][kk - 1]
    band = rel if logit else rel * abs(cut)
    bad = [e for e in gpu_sel ^ ref_sel if abs(scores[e] - cut) > band]
    if len(gpu_sel) != len(ref_sel):
        return False, f"sizes {len(gpu_sel)} vs {len(ref_sel)}"
    return (not bad), f"entries outside the tie band: {bad[:10]} (cut {cut})"


def threshold_set_ok(gpu_sel, ref_sel, logits, I, alpha, forced, rel=TIE_REL):
    gpu_sel = set(int(x) for x in gpu_sel)
    ref_sel = set(int(x) for x in ref_sel)
    if gpu_sel == ref_sel:
        return True, ""
    row = logits[: I + 1]
    ratio = np.exp(row - row.max())
    bad = [e for e in gpu_sel ^ ref_sel if e not in forced and abs(ratio[e] - alpha) > rel * alpha]
    return (not bad), f"entries outside the tie band: {bad[:10]}"
