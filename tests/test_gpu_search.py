"""The kernel-aware pattern search on the GPU: its recall against the oracle's
(same indices), and the invariants of its choice."""
import numpy as np
import pytest
import torch

import synth
from oracle import dsa_oracle as orc
from tests._parity import gpu_lists_to_oracle_heads, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


def test_search_choice_and_recall_parity(dsa):
    from dynamic_sparse_attention_build_b200 import search
    N, d, B = 2048, 128, 64
    # the mixed layer's data (planted vertical keys and periodic slashes) at 2048 tokens
    w = synth.workload(2, N=N)
    Q, K, V, _ = synth.make_inputs(w)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    target = 0.9
    heads = [0, 1, 2, 3]
    chosen, trials = search.search_patterns(Qd, Kd, Vd, B, recall_target=target, repeats=2, heads=heads)
    cands = search.default_candidates(N, B)
    assert len(trials) == len(heads) * len(cands)
    assert all(chosen[h] == search.dense_pattern(N, B) for h in range(Q.shape[0]) if h not in heads)
    for h in heads:
        ts = [t for t in trials if t.head == h]
        dense = [t for t in ts if t.pattern == search.dense_pattern(N, B)][0]
        assert abs(dense.recall - 1.0) < 1e-6 and abs(dense.min_recall - 1.0) < 1e-6
        c = [t for t in ts if t.pattern == chosen[h]][0]
        assert c.recall >= target
        assert all(c.ms <= t.ms for t in ts if t.recall >= target)
    print("\n" + search.summary(trials, chosen))

    # recall of two candidates on head 0, GPU vs oracle on the library's own indices
    q, k, v = to64(Q)[0], to64(K)[0], to64(V)[0]
    _, lse_d = orc.dense_causal_attention(q, k, v)
    rows = np.linspace(0, N - 1, 96).astype(np.int64)
    for pat in (dict(kind="vs", last_q=64, n_vert=100, n_slash=400), dict(kind="ashape", sink=64, window=256)):
        idx = dsa.build_indices(Qd[:1], Kd[:1], [pat], B)  # head 0 reads KV head 0
        _, lse_g = dsa.sparse_prefill(Qd[:1], Kd[:1], Vd[:1], idx, want_lse=True)
        idx_d = dsa.build_indices(Qd[:1], Kd[:1], [search.dense_pattern(N, B)], B)
        _, lse_gd = dsa.sparse_prefill(Qd[:1], Kd[:1], Vd[:1], idx_d, want_lse=True)
        r_gpu = search.attention_recall(lse_g[0], lse_gd[0]).cpu().numpy()[rows]
        hi = gpu_lists_to_oracle_heads(idx, N, B)[0]
        _, lse_s = orc.attention_rows(q, k, v, hi, rows)
        r_ref = search.attention_recall(torch.tensor(lse_s), torch.tensor(lse_d[rows])).numpy()
        # LSEs agree within 2e-3, so recalls within ~2e-3 relative
        np.testing.assert_allclose(r_gpu, r_ref, rtol=5e-3, atol=1e-6)
        trial = [t for t in trials if t.head == 0 and t.pattern == pat][0]
        full = search.attention_recall(lse_g[0], lse_gd[0]).mean().item()
        assert abs(trial.recall - full) < 1e-9  # the search scored exactly this
