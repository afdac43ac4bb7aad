"""Host-side checks of the kernel-aware pattern search: the recall formula
against its definition (brute-force sums of the causal softmax inside the mask,
computed with the oracle), and the selection rule."""
import math

import numpy as np
import torch

import synth
from dynamic_sparse_attention_build_b200 import search
from oracle import dsa_oracle as orc


def _brute_recall(q, k, hi, i):
    """sum over the mask's keys of the causal softmax of row i (fp64)."""
    d = q.shape[1]
    lg = (k[: i + 1] @ q[i]) / math.sqrt(d)
    p = np.exp(lg - lg.max())
    p /= p.sum()
    J = orc.allowed_keys(hi, i)
    return float(p[J].sum()) if J.size else 0.0


def test_recall_is_softmax_mass_inside_mask():
    N, d, B = 192, 16, 64
    Q, K, V = synth.random_qkv(1, 1, N, d, seed=21, scale=2.0)
    q, k, v = (t[0].double().numpy() for t in (Q, K, V))
    _, lse_d = orc.dense_causal_attention(q, k, v)
    for pat in (dict(kind="ashape", sink=16, window=40), dict(kind="block_topk", topk=1),
                dict(kind="vs", last_q=32, n_vert=5, n_slash=3)):
        hi = orc.build_head_index(q, k, pat, B)
        _, lse_s = orc.attention_rows(q, k, v, hi, np.arange(N))
        r = search.attention_recall(torch.tensor(lse_s), torch.tensor(lse_d)).numpy()
        want = np.array([_brute_recall(q, k, hi, i) for i in range(N)])
        np.testing.assert_allclose(r, want, rtol=1e-10, atol=1e-12)
        assert (r <= 1 + 1e-12).all() and (r >= 0).all()
    # a row whose mask is empty has recall 0 (LSE = -inf there)
    r = search.attention_recall(torch.tensor([-np.inf, 0.0]), torch.tensor([1.0, 0.0]))
    assert r.tolist() == [0.0, 1.0]


def _t(ms, recall, i=0):
    return search.Trial(0, dict(kind="block_topk", topk=i), ms, recall, recall, 0)


def test_choose_fastest_qualifying_else_best_recall():
    ts = [_t(1.0, 0.90, 1), _t(2.0, 0.97, 2), _t(1.5, 0.96, 3), _t(3.0, 1.0, 4)]
    assert search.choose(ts, 0.95).pattern["topk"] == 3          # fastest with recall >= 0.95
    assert search.choose(ts, 0.999).pattern["topk"] == 4
    ts2 = [_t(1.0, 0.5, 1), _t(2.0, 0.8, 2), _t(0.5, 0.8, 3)]
    assert search.choose(ts2, 0.9).pattern["topk"] == 3          # none qualifies: best recall, then faster


def test_default_candidates_end_dense():
    c = search.default_candidates(4096, 64)
    assert c[-1] == search.dense_pattern(4096, 64) == dict(kind="block_topk", topk=64)
    kinds = {x["kind"] for x in c}
    assert {"ashape", "vs", "block_topk", "block_threshold"} <= kinds
    assert all(x["n_vert"] + x["n_slash"] < 4096 for x in c if x["kind"] == "vs")
