"""Pins of the CPU oracle against things other than itself: hand-worked examples
from the pages' definitions (tests/golden/), brute force on tiny inputs written as
explicit loops, closed forms, and library routines (torch SDPA in float64).
CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as orc
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- A-shape
def test_ashape_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "ashape_hand_example.json")))
    N, sink, window, B = g["N"], g["sink"], g["window"], g["block"]
    want = np.array([[c == "1" for c in row] for row in g["mask_rows"]])
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    assert (orc.ashape_allowed(i, j, sink, window) == want).all()
    hi = orc.HeadIndex(kind=orc.ASHAPE, B=B, N=N, sink=sink, window=window)
    hi.blocks = [orc.ashape_blocks(qb, B, N, sink, window) for qb in range(2)]
    hi.cols = [np.zeros(0, np.int64)] * 2
    assert [list(b) for b in hi.blocks] == g["blocks_per_query_block"]
    assert (orc.index_mask_dense(hi) == want).all()


@pytest.mark.parametrize("N,B,sink,window", [(50, 8, 3, 5), (64, 16, 0, 17), (37, 4, 9, 1),
                                             (100, 32, 40, 64), (20, 64, 4, 4)])
def test_ashape_blocks_bruteforce(N, B, sink, window):
    nqb = (N + B - 1) // B
    for qb in range(nqb):
        want = set()
        for i in range(qb * B, min(N, qb * B + B)):
            for j in range(N):
                if j <= i and (j < sink or i - j < window):
                    want.add(j // B)
        assert list(orc.ashape_blocks(qb, B, N, sink, window)) == sorted(want)
    hi = orc.build_head_index(np.zeros((N, 4)), np.zeros((N, 4)),
                              dict(kind="ashape", sink=sink, window=window), B)
    M = orc.index_mask_dense(hi)
    for i in range(N):
        for j in range(N):
            assert M[i, j] == (j <= i and (j < sink or i - j < window))


# --------------------------------------------------------------------------- VS
def _vs_bruteforce(Q, K, last_q):
    N, d = K.shape
    v = [0.0] * N
    s = [0.0] * N
    for i in range(max(0, N - last_q), N):
        logit = [sum(Q[i, c] * K[j, c] for c in range(d)) / math.sqrt(d) for j in range(i + 1)]
        m = max(logit)
        e = [math.exp(x - m) for x in logit]
        z = sum(e)
        for j in range(i + 1):
            v[j] += e[j] / z
            s[i - j] += e[j] / z
    return np.array(v), np.array(s)


@pytest.mark.parametrize("N,d,last_q", [(23, 4, 5), (16, 8, 40), (31, 3, 31)])
def test_vs_estimate_bruteforce(rng, N, d, last_q):
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d))
    v, s = orc.vs_estimate(Q, K, last_q)
    vb, sb = _vs_bruteforce(Q, K, last_q)
    np.testing.assert_allclose(v, vb, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(s, sb, rtol=1e-12, atol=1e-14)
    # each row's probabilities sum to one
    assert abs(v.sum() - min(last_q, N)) < 1e-9
    assert abs(s.sum() - min(last_q, N)) < 1e-9


def test_vs_estimate_zero_query_closed_form():
    N, d, last_q = 40, 6, 7
    K = np.random.default_rng(1).standard_normal((N, d))
    v, s = orc.vs_estimate(np.zeros((N, d)), K, last_q)
    rows = range(N - last_q, N)
    v_cf = np.array([sum(1.0 / (i + 1) for i in rows if i >= j) for j in range(N)])
    s_cf = np.array([sum(1.0 / (i + 1) for i in rows if i >= o) for o in range(N)])
    np.testing.assert_allclose(v, v_cf, rtol=1e-13)
    np.testing.assert_allclose(s, s_cf, rtol=1e-13)


def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(50):
        n = int(rng.integers(1, 40))
        x = rng.integers(0, 6, n).astype(float)  # many ties
        k = int(rng.integers(1, 45))
        remaining = list(range(n))
        picked = []
        for _ in range(min(k, n)):
            best = remaining[0]
            for idx in remaining:
                if x[idx] > x[best]:
                    best = idx  # strict: the earlier (lower) index wins a tie
            picked.append(best)
            remaining.remove(best)
        assert list(orc.topk_indices(x, k)) == sorted(picked)


@pytest.mark.parametrize("B", [4, 8, 16])
def test_distance_set_covers_slash_cells(B):
    rng = np.random.default_rng(B)
    N = 150
    nb = (N + B - 1) // B
    for trial in range(20):
        S = np.sort(rng.choice(N, size=int(rng.integers(1, 12)), replace=False))
        D = orc.vs_distance_set(S, B, nb)
        for qb in range(nb):
            rows = range(qb * B, min(N, qb * B + B))
            dist = {qb - (i - o) // B for i in rows for o in S if i - o >= 0}
            assert dist <= set(int(x) for x in D)
            full = qb * B + B <= N and qb * B - int(S.max()) >= 0
            if full:
                assert dist == set(int(x) for x in D)


@pytest.mark.parametrize("B", [4, 8, 16])
def test_distance_set_is_exactly_the_reached_distances(B):
    # With N a multiple of B the last query block is full, so every distance in D
    # is reached by some block's slash cells and no other distance is: D holds
    # nothing that can never apply (no distance >= the number of key blocks).
    rng = np.random.default_rng(50 + B)
    N = 160
    nb = N // B
    for trial in range(20):
        S = rng.choice(N, size=int(rng.integers(1, 12)), replace=False)
        reached = set()
        for qb in range(nb):
            for i in range(qb * B, qb * B + B):
                for o in S:
                    if i - o >= 0:
                        reached.add(qb - (i - int(o)) // B)
        assert set(int(x) for x in orc.vs_distance_set(S, B, nb)) == reached


def _vs_head(rng, N, d, B, last_q, n_vert, n_slash):
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d))
    return orc.build_head_index(Q, K, dict(kind="vs", last_q=last_q, n_vert=n_vert,
                                           n_slash=n_slash), B)


@pytest.mark.parametrize("N,B,nv,ns", [(64, 8, 5, 4), (77, 16, 9, 3), (50, 4, 2, 20)])
def test_vs_index_superset_and_no_double_count(rng, N, B, nv, ns):
    hi = _vs_head(rng, N, 6, B, 10, nv, ns)
    M = orc.index_mask_dense(hi)
    Vs, Ss = set(int(x) for x in hi.V), set(int(x) for x in hi.S)
    for i in range(N):
        for j in range(N):
            exact = j <= i and (j in Vs or (i - j) in Ss)
            if exact:
                assert M[i, j]
            if M[i, j]:
                assert j <= i
    Dset = set(int(x) for x in hi.D)
    for qb in range(len(hi.blocks)):
        # explicit column rule, written as a loop
        want = [j for j in sorted(Vs) if j <= qb * B + B - 1 and (qb - j // B) not in Dset]
        assert list(hi.cols[qb]) == want
        assert list(hi.blocks[qb]) == sorted(qb - x for x in Dset if x <= qb)
        covered = set(int(b) for b in hi.blocks[qb])
        assert not any(j // B in covered for j in hi.cols[qb])


def test_vs_slash_windows_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "vs_slash_windows_hand_example.json")))
    N, B, S, V = g["N"], g["block"], np.array(g["S"]), np.array(g["V"])
    nqb = (N + B - 1) // B
    hi = orc.HeadIndex(kind=orc.VS, B=B, N=N, V=V, S=S)
    hi.runs = [orc.vs_slash_runs(S, qb, B, N) for qb in range(nqb)]
    hi.blocks = [np.zeros(0, np.int64)] * nqb
    hi.cols = [orc.vs_window_columns(V, hi.runs[qb], qb, B) for qb in range(nqb)]
    assert [r.tolist() for r in hi.runs] == g["runs_per_query_block"]
    assert [list(c) for c in hi.cols] == g["columns_per_query_block"]
    assert list(orc.allowed_keys(hi, 10)) == g["row_10_keys"]


@pytest.mark.parametrize("B", [4, 8, 16])
def test_vs_slash_runs_are_the_slash_cells_of_each_block(B):
    rng = np.random.default_rng(100 + B)
    N = 150
    for trial in range(20):
        S = rng.choice(N, size=int(rng.integers(1, 15)), replace=False)
        for qb in range((N + B - 1) // B):
            runs = orc.vs_slash_runs(S, qb, B, N)
            got = set()
            for a, b in runs:
                got |= set(range(a, b + 1))
            want = set()
            for i in range(qb * B, min(N, qb * B + B)):
                for o in S:
                    if i - o >= 0:
                        want.add(int(i - o))
            assert got == want
            # ascending, disjoint and not touching (maximal runs)
            for (a0, b0), (a1, b1) in zip(runs[:-1], runs[1:]):
                assert a0 <= b0 < a1 - 1 < b1


@pytest.mark.parametrize("B", [4, 16, 64])
def test_vs_slash_runs_are_the_dilated_offsets_mirrored(B):
    # Key j is reached from rows r0..r1 on slash o iff r0 - o <= j <= r1 - o, i.e.
    # r1 - j lies in [o, o + L - 1] with L = r1 - r0 + 1.  So the runs of a query
    # block are the merged intervals of those dilated offsets, mirrored at r1 and
    # clipped at key 0: one per-head list serves every query block of height L.
    rng = np.random.default_rng(7 * B)
    N = 700
    for trial in range(10):
        S = rng.choice(N, size=int(rng.integers(1, 40)), replace=False)
        for qb in range((N + B - 1) // B):
            r0, r1 = qb * B, min(N, qb * B + B) - 1
            L = r1 - r0 + 1
            ivs = []
            for o in sorted(int(x) for x in S):  # merged [o, o + L - 1], ascending
                if ivs and o <= ivs[-1][1] + 1:
                    ivs[-1][1] = max(ivs[-1][1], o + L - 1)
                else:
                    ivs.append([o, o + L - 1])
            mirrored = [[max(0, r1 - hi), r1 - lo] for lo, hi in reversed(ivs) if r1 - lo >= 0]
            assert orc.vs_slash_runs(S, qb, B, N).tolist() == mirrored


@pytest.mark.parametrize("N,B,nv,ns", [(64, 8, 5, 4), (77, 16, 9, 3), (50, 4, 2, 20), (90, 8, 0, 7)])
def test_vs_window_mask_between_exact_and_aligned_blocks(N, B, nv, ns):
    rng = np.random.default_rng(N + B)
    Q = rng.standard_normal((N, 6))
    K = rng.standard_normal((N, 6))
    pat = dict(kind="vs", last_q=10, n_vert=nv, n_slash=ns)
    hw = orc.build_head_index(Q, K, dict(pat, slash_cover="windows"), B)
    hb = orc.build_head_index(Q, K, pat, B)
    assert list(hw.V) == list(hb.V) and list(hw.S) == list(hb.S)
    Mw, Mb = orc.index_mask_dense(hw), orc.index_mask_dense(hb)
    Vs, Ss = set(int(x) for x in hw.V), set(int(x) for x in hw.S)
    for i in range(N):
        for j in range(N):
            exact = j <= i and (j in Vs or (i - j) in Ss)
            assert not exact or Mw[i, j]      # every exact VS cell is kept
            assert not Mw[i, j] or Mb[i, j]   # the runs never go past the aligned blocks
    for qb in range(len(hw.runs)):
        in_runs = lambda j: any(a <= j <= b for a, b in hw.runs[qb])
        want = [j for j in sorted(Vs) if j <= qb * B + B - 1 and not in_runs(j)]
        assert list(hw.cols[qb]) == want
    assert orc.selected_pairs(hw) <= orc.selected_pairs(hb)


def test_vs_estimate_picks_planted_verticals():
    w = synth.workload(1)
    Q, K, V, planted = synth.make_inputs(w)
    q = Q[0].double().numpy()
    k = K[0].double().numpy()
    v, s = orc.vs_estimate(q, k, w["vs"]["last_q"])
    Vsel = set(orc.topk_indices(v, w["vs"]["n_vert"]).tolist())
    assert set(planted["vert"][0].tolist()) <= Vsel


# --------------------------------------------------------------------------- block scoring
def test_mean_pool_partial_block():
    X = np.arange(30, dtype=float).reshape(10, 3)
    P = orc.mean_pool(X, 4)
    np.testing.assert_allclose(P[0], X[0:4].mean(0))
    np.testing.assert_allclose(P[2], X[8:10].mean(0))
    assert P.shape == (3, 3)


@pytest.mark.parametrize("N,B,d", [(32, 8, 5), (29, 8, 3), (40, 16, 7)])
def test_block_score_is_mean_token_logit(rng, N, B, d):
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d))
    S = orc.block_logits(orc.mean_pool(Q, B), orc.mean_pool(K, B), d)
    nb = (N + B - 1) // B
    for I in range(nb):
        for J in range(nb):
            tot, cnt = 0.0, 0
            for i in range(I * B, min(N, I * B + B)):
                for j in range(J * B, min(N, J * B + B)):
                    tot += sum(Q[i, c] * K[j, c] for c in range(d)) / math.sqrt(d)
                    cnt += 1
            assert abs(S[I, J] - tot / cnt) < 1e-12


def test_key_conv_bruteforce(rng):
    N, d, W = 13, 4, 4
    K = rng.standard_normal((N, d))
    w = rng.standard_normal((d, W)) * 0.5
    b = rng.standard_normal(d) * 0.1
    out = orc.key_conv(K, w, b)
    for j in range(N):
        for c in range(d):
            acc = b[c]
            for t in range(W):
                if j - t >= 0:
                    acc += w[c, t] * K[j - t, c]
            want = K[j, c] + acc / (1.0 + math.exp(-acc))
            assert abs(out[j, c] - want) < 1e-12
    np.testing.assert_array_equal(orc.key_conv(K, np.zeros((d, W)), np.zeros(d)), K)


def test_threshold_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "threshold_hand_example.json")))
    row = np.array(g["logits"])
    for c in g["cases"]:
        kept = orc.select_threshold(row, g["I"], c["alpha"], c["keep_sink"], c["keep_local"])
        assert list(kept) == c["kept"], c


def test_threshold_limits(rng):
    row = rng.standard_normal(20)
    for I in range(20):
        assert list(orc.select_threshold(row, I, 1e-300, 0, 0)) == list(range(I + 1))
        top = set(np.nonzero(row[: I + 1] == row[: I + 1].max())[0].tolist())
        assert set(orc.select_threshold(row, I, 1.0, 1, 1).tolist()) == top | {0, I}


def test_moba_and_block_topk_selection(rng):
    row = rng.standard_normal(30)
    for I in range(30):
        m = orc.select_moba(row, I, 8)
        past = sorted(range(I), key=lambda J: (-row[J], J))[:8]
        assert list(m) == sorted(set(past) | {I})
        t = orc.select_block_topk(row, I, 5)
        assert list(t) == sorted(sorted(range(I + 1), key=lambda J: (-row[J], J))[:5])


# --------------------------------------------------------------------------- attention
def _sdpa_causal(Q, K, V):
    q = torch.from_numpy(Q)[None, None]
    k = torch.from_numpy(K)[None, None]
    v = torch.from_numpy(V)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    L = (q @ k.transpose(-1, -2)) / math.sqrt(Q.shape[1])
    L = L.masked_fill(torch.triu(torch.ones(Q.shape[0], Q.shape[0], dtype=torch.bool), 1), -math.inf)
    return o[0, 0].numpy(), torch.logsumexp(L, -1)[0, 0].numpy()


@pytest.mark.parametrize("N,B,d", [(64, 16, 8), (70, 16, 8), (33, 64, 4)])
def test_all_blocks_equal_dense_causal(rng, N, B, d):
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    nb = (N + B - 1) // B
    hi = orc.build_head_index(Q, K, dict(kind="block_topk", topk=nb), B)
    O, lse = orc.attention_rows(Q, K, V, hi, np.arange(N))
    O_ref, lse_ref = _sdpa_causal(Q, K, V)
    np.testing.assert_allclose(O, O_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12)
    O2, lse2 = orc.dense_causal_attention(Q, K, V)
    np.testing.assert_allclose(O2, O_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse2, lse_ref, rtol=1e-12)


def test_attention_bruteforce_and_closed_forms(rng):
    N, B, d = 40, 8, 5
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    hi = orc.build_head_index(Q, K, dict(kind="vs", last_q=6, n_vert=4, n_slash=3), B)
    O, lse = orc.attention_rows(Q, K, V, hi, np.arange(N))
    M = orc.index_mask_dense(hi)
    for i in range(N):
        J = [j for j in range(N) if M[i, j]]
        if not J:
            assert np.all(O[i] == 0) and lse[i] == -math.inf
            continue
        lg = [sum(Q[i, c] * K[j, c] for c in range(d)) / math.sqrt(d) for j in J]
        m = max(lg)
        e = [math.exp(x - m) for x in lg]
        want = [sum(e[t] * V[J[t], c] for t in range(len(J))) / sum(e) for c in range(d)]
        np.testing.assert_allclose(O[i], want, rtol=1e-11, atol=1e-13)
        assert abs(lse[i] - (m + math.log(sum(e)))) < 1e-11
    # Q = 0: uniform weights over the allowed set
    O0, _ = orc.attention_rows(np.zeros_like(Q), K, V, hi, np.arange(N))
    for i in range(N):
        J = np.nonzero(M[i])[0]
        if J.size:
            np.testing.assert_allclose(O0[i], V[J].mean(0), rtol=1e-12, atol=1e-14)
    # V = c: O = c wherever a key is allowed
    Oc, _ = orc.attention_rows(Q, K, np.full_like(V, 0.75), hi, np.arange(N))
    rows = [i for i in range(N) if M[i].any()]
    np.testing.assert_allclose(Oc[rows], 0.75, rtol=1e-13)


def test_empty_rows_and_duplicates():
    N, B, d = 16, 4, 3
    rng = np.random.default_rng(3)
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    hi = orc.HeadIndex(kind=orc.VS, B=B, N=N)
    hi.blocks = [np.zeros(0, np.int64), np.array([0]), np.array([1]), np.array([2, 3])]
    hi.cols = [np.array([2]), np.array([1, 2]), np.zeros(0, np.int64), np.array([12, 13])]
    O, lse = orc.attention_rows(Q, K, V, hi, np.arange(N))
    # rows 0 and 1 see nothing (column 2 is in the future)
    assert np.all(O[:2] == 0) and np.all(np.isneginf(lse[:2]))
    # duplicates between block 0 and columns 1, 2 of query block 1 count once
    hi2 = orc.HeadIndex(kind=orc.VS, B=B, N=N, blocks=hi.blocks,
                        cols=[hi.cols[0], np.zeros(0, np.int64), hi.cols[2], np.zeros(0, np.int64)])
    O2, lse2 = orc.attention_rows(Q, K, V, hi2, np.arange(4, N))
    np.testing.assert_array_equal(O[4:], O2)
    np.testing.assert_array_equal(lse[4:], lse2)


def test_selected_pairs_counts_mask(rng):
    hi = _vs_head(rng, 48, 4, 8, 5, 3, 4)
    assert orc.selected_pairs(hi) == int(orc.index_mask_dense(hi).sum())


@pytest.mark.parametrize("N,B", [(200, 16), (131, 8), (64, 64), (97, 32)])
def test_selected_pairs_by_block_equals_the_mask_count(rng, N, B):
    """The block-wise count (one sorted key set per query block, binary search
    per row, the A-shape predicate by inclusion-exclusion) equals the number of
    True entries of the dense index mask, for every pattern kind, slash runs
    and columns that repeat keys of listed blocks included."""
    d = 8
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d))
    pats = [dict(kind="ashape", sink=5, window=11), dict(kind="ashape", sink=0, window=1),
            dict(kind="ashape", sink=N, window=3), dict(kind="ashape", sink=2 * B + 3, window=B + 1),
            dict(kind="vs", last_q=16, n_vert=9, n_slash=7),
            dict(kind="vs", last_q=16, n_vert=9, n_slash=7, slash_cover="windows"),
            dict(kind="block_topk", topk=3), dict(kind="block_threshold", alpha=0.4),
            dict(kind="moba", topk=2)]
    for p in pats:
        hi = orc.build_head_index(Q, K, p, B)
        if p["kind"] == "block_topk":  # columns inside listed blocks must count once
            hi.cols = [np.sort(rng.choice(min(N, qb * B + B), size=min(5, qb * B + B), replace=False))
                       for qb in range(len(hi.blocks))]
        want = int(orc.index_mask_dense(hi).sum())
        assert orc.selected_pairs_by_block(hi) == want, p
        assert orc.selected_pairs(hi) == want, p


# --------------------------------------------------------------------------- unified discovery
def _lower(rows):
    n = len(rows)
    sc = np.full((n, n), -7.0)  # above the diagonal: never read
    for I, r in enumerate(rows):
        sc[I, : I + 1] = r
    return sc


def test_unified_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "unified_discovery_hand_example.json")))
    sc = _lower(g["logits_lower"])
    P, V, G = orc.unified_pattern_scores(sc)
    for I, row in enumerate(g["P"]):
        np.testing.assert_allclose(P[I, : I + 1], row, rtol=1e-12)
    np.testing.assert_allclose(V, g["V"], rtol=1e-12)
    np.testing.assert_allclose(G, g["G"], rtol=1e-12)
    blocks, vert, diag = orc.select_unified(sc, g["alpha"], False, False)
    assert list(vert) == g["verticals"] and list(diag) == g["diagonals"]
    assert [list(b) for b in blocks] == g["blocks"]


def test_unified_sums_bruteforce_and_limits(rng):
    """V and G against explicit loops over (I, J); alpha -> 0 keeps every J <= I,
    alpha = 1 keeps the argmax sets; the per-row rule is the threshold kind's."""
    n = 13
    sc = rng.standard_normal((n, n)) * 2
    P, V, G = orc.unified_pattern_scores(sc)
    for I in range(n):
        w = [math.exp(sc[I, J]) for J in range(I + 1)]
        for J in range(I + 1):
            assert abs(P[I, J] - w[J] / sum(w)) < 1e-12
    for J in range(n):
        assert abs(V[J] - sum(P[I, J] for I in range(J, n))) < 1e-12
    for dd in range(n):
        assert abs(G[dd] - sum(P[I, I - dd] for I in range(dd, n))) < 1e-12
    blocks, vert, diag = orc.select_unified(sc, 1e-300, False, False)
    assert all(list(b) == list(range(I + 1)) for I, b in enumerate(blocks))
    blocks, vert, diag = orc.select_unified(sc, 1.0, False, False)
    assert list(vert) == [int(np.argmax(V))] and list(diag) == [int(np.argmax(G))]
    for I in range(n):
        thr = orc.select_threshold(sc[I], I, 0.3, False, False)
        b, _, _ = orc.select_unified(sc, 0.3, False, False)
        assert set(thr) <= set(b[I])


def test_unified_finds_planted_vertical_and_diagonal(rng):
    """A key block that every query block favours is a vertical; a block
    distance every query block favours is a diagonal; both reach every row."""
    n = 40
    sc = rng.standard_normal((n, n)) * 0.1
    for I in range(n):
        if I >= 7:
            sc[I, 7] += 6.0          # planted vertical at key block 7
        if I >= 3:
            sc[I, I - 3] += 6.0      # planted diagonal at distance 3
    blocks, vert, diag = orc.select_unified(sc, 0.5, True, True)
    assert 7 in vert and 3 in diag
    for I in range(10, n):
        assert {0, 7, I - 3, I} <= set(blocks[I])


def test_runs_list_helpers_match_the_oracle_runs(rng):
    """The test helpers that read the library's slash-run lists (offset intervals
    merged at the block height, mirrored at a block's last row) give exactly the
    oracle's runs for every query block, ragged last block included."""
    from tests._parity import runs_list_from_slashes, runs_of_block
    for N, B, ns in ((300, 16, 7), (257, 32, 40), (100, 64, 3), (1000, 64, 200)):
        S = np.sort(rng.choice(N, size=ns, replace=False))
        lst = runs_list_from_slashes(S, B, N)
        for qb in range((N + B - 1) // B):
            assert np.array_equal(runs_of_block(lst, qb, B, N), orc.vs_slash_runs(S, qb, B, N)), (N, B, qb)
