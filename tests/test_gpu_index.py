"""GPU parity of dsa_build_indices against the fp64 oracle.

Index sets must match exactly, except for entries whose oracle score lies within
1e-3 (relative) of the top-k / threshold cut.  Integer steps that follow a
selection (VS distances and columns) are compared bit-exactly against the
oracle's rule applied to the GPU's own selection, so a near-tie cannot cascade.
The attention output with the GPU's indices is then checked against the oracle
evaluating the same indices."""
import numpy as np
import pytest
import torch

import synth
from oracle import dsa_oracle as orc
from tests._parity import (assert_close_outputs, assert_lse_close, gpu_lists_to_oracle_heads, runs_list_from_slashes,
                           runs_of_block, threshold_set_ok, to64, topk_set_ok)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


def check_indices(bufs, ref_heads, pats, N, B, convs_ref=None):
    gl = bufs.host_lists()
    nqb = (N + B - 1) // B
    for h, (g, r, p) in enumerate(zip(gl, ref_heads, pats)):
        kind = p["kind"]
        if kind == "ashape":
            assert g["kind"] == 0 and g["sink"] == p["sink"] and g["window"] == p["window"]
            for qb in range(nqb):
                assert list(g["blocks"][qb]) == list(r.blocks[qb]), (h, qb)
        elif kind == "vs":
            ok, msg = topk_set_ok(g["vert"], r.V, r.vscore, p["n_vert"])
            assert ok, f"head {h} verticals: {msg}"
            ok, msg = topk_set_ok(g["slash"], r.S, r.sscore, p["n_slash"])
            assert ok, f"head {h} slashes: {msg}"
            assert list(g["vert"]) == sorted(g["vert"]) and list(g["slash"]) == sorted(g["slash"])
            D = orc.vs_distance_set(np.asarray(g["slash"], np.int64), B, nqb)
            assert list(g["dist"]) == list(D), f"head {h} distances"
            for qb in range(nqb):
                want = orc.vs_columns(np.asarray(g["vert"], np.int64), D, qb, B)
                assert list(g["cols"][qb]) == list(want), (h, qb)
        elif kind == "vs_windows":
            ok, msg = topk_set_ok(g["vert"], r.V, r.vscore, p["n_vert"])
            assert ok, f"head {h} verticals: {msg}"
            ok, msg = topk_set_ok(g["slash"], r.S, r.sscore, p["n_slash"])
            assert ok, f"head {h} slashes: {msg}"
            S = np.asarray(g["slash"], np.int64)
            assert list(g["dist"]) == list(runs_list_from_slashes(S, B, N)), f"head {h} run list"
            for qb in range(nqb):
                runs = runs_of_block(g["dist"], qb, B, N)
                assert np.array_equal(runs, orc.vs_slash_runs(S, qb, B, N)), (h, qb)
                want = orc.vs_window_columns(np.asarray(g["vert"], np.int64), runs, qb, B)
                assert list(g["cols"][qb]) == list(want), (h, qb)
        elif kind == "unified":
            # the kept verticals and diagonals against the oracle's (tie-aware at
            # alpha times the maximum), then each row: its own threshold blocks
            # (tie-aware) plus exactly the GPU's verticals and diagonals
            P, Vs, Gs = orc.unified_pattern_scores(r.block_scores)
            a = p["alpha"]
            for got, want, sums in ((g["vert"], r.vert_blocks, Vs), (g["slash"], r.diag_blocks, Gs)):
                bad = [x for x in set(got.tolist()) ^ set(want.tolist()) if abs(sums[x] / sums.max() - a) > 1e-3 * a]
                assert not bad, f"head {h}: pattern sets differ beyond the tie band at {bad[:10]}"
            gv, gd = np.asarray(g["vert"]), np.asarray(g["slash"])
            for I in range(nqb):
                extra = set(gv[gv <= I].tolist()) | set((I - gd[gd <= I]).tolist())
                forced = extra | ({0} if p.get("keep_sink", 1) else set()) | ({I} if p.get("keep_local", 1) else set())
                row = P[I, : I + 1]
                ref_rows = set(np.nonzero(row >= a * row.max())[0].tolist()) | forced
                ok, msg = threshold_set_ok(g["blocks"][I], sorted(ref_rows), r.block_scores[I], I, a, forced)
                assert ok, f"head {h} block {I}: {msg}"
                assert set(g["blocks"][I].tolist()) >= forced
        else:
            sc = r.block_scores
            for I in range(nqb):
                gs, rs = g["blocks"][I], r.blocks[I]
                assert list(gs) == sorted(set(gs.tolist())), (h, I)
                if kind == "block_threshold":
                    forced = {0, I}
                    ok, msg = threshold_set_ok(gs, rs, sc[I], I, p["alpha"], forced)
                elif kind == "moba":
                    assert I in set(gs.tolist())
                    ok, msg = topk_set_ok([x for x in gs if x != I], [x for x in rs if x != I], sc[I][:I],
                                          p["topk"], logit=True) if I > 0 else (True, "")
                else:
                    ok, msg = topk_set_ok(gs, rs, sc[I][: I + 1], p["topk"], logit=True)
                assert ok, f"head {h} block {I}: {msg}"


def run(dsa, Q, K, V, pats, B, rows=None, convs=None):
    N = Q.shape[1]
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    dpats = []
    G = Q.shape[0] // K.shape[0]
    for h, p in enumerate(pats):
        p = dict(p)
        if convs is not None and p["kind"] == "moba":
            w, b = convs[h // G]
            p["conv"] = (w.cuda(), b.cuda())
        dpats.append(p)
    bufs = dsa.build_indices(Qd, Kd, dpats, B)
    torch.cuda.synchronize()
    st, det = dsa.device_status()
    assert st == 0, (st, det)
    oconvs = None
    if convs is not None:
        oconvs = [(convs[h // G][0].double().numpy(), convs[h // G][1].double().numpy()) for h in range(len(pats))]
    ref = orc.build_indices(to64(Q), to64(K), pats, B, oconvs)
    check_indices(bufs, ref, pats, N, B)
    # attention with the GPU's own indices
    O, lse = dsa.sparse_prefill(Qd, Kd, Vd, bufs, want_lse=True)
    torch.cuda.synchronize()
    heads = gpu_lists_to_oracle_heads(bufs, N, B)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    O_ref, lse_ref = orc.sparse_attention(to64(Q), to64(K), to64(V), heads, rows)
    assert_close_outputs(to64(O)[:, rows], O_ref, "O")
    assert_lse_close(lse.cpu().double().numpy()[:, rows], lse_ref, "lse")
    # exact pair count of the index mask
    pairs = dsa.count_pairs(Qd, Kd, bufs).cpu().numpy()
    if N <= 1500:
        want = [orc.selected_pairs(hh) for hh in heads]
        assert list(pairs) == want
    return bufs


def test_vs_tiny_workload(dsa):
    w = synth.workload(1)
    Q, K, V, planted = synth.make_inputs(w)
    bufs = run(dsa, Q, K, V, synth.head_patterns(w), w["B"])
    assert set(planted["vert"][0].tolist()) <= set(bufs.host_lists()[0]["vert"].tolist())


def test_mixed_gqa_ragged(dsa):
    N, d, B = 1500, 128, 64
    Q, K, V = synth.random_qkv(8, 2, N, d, seed=21)
    pats = [dict(kind="vs", last_q=64, n_vert=60, n_slash=50),
            dict(kind="ashape", sink=100, window=300),
            dict(kind="block_topk", topk=5),
            dict(kind="vs", last_q=20, n_vert=2000, n_slash=7),
            dict(kind="block_threshold", alpha=0.5, keep_sink=1, keep_local=1),
            dict(kind="block_topk", topk=100),
            dict(kind="vs", last_q=128, n_vert=0, n_slash=1),
            dict(kind="ashape", sink=0, window=1)]
    run(dsa, Q, K, V, pats, B)


@pytest.mark.parametrize("B", [64, 128])
def test_vs_windows(dsa, B):
    """Vertical-Slash heads whose slashes are covered by their exact key runs per
    query block (every aligned 64-key unit a run touches, with the run keys as a
    per-half mask) next to every other kind in one layer (the kernel with run
    masks then serves them all), with few, many and clustered slashes, a ragged
    length and GQA."""
    N, d = 1400, 128
    Q, K, V = synth.random_qkv(8, 2, N, d, seed=51 + B)
    pats = [dict(kind="vs_windows", last_q=64, n_vert=40, n_slash=3),
            dict(kind="vs_windows", last_q=32, n_vert=200, n_slash=300),
            dict(kind="ashape", sink=70, window=200),
            dict(kind="vs", last_q=64, n_vert=50, n_slash=20),
            dict(kind="block_topk", topk=3),
            dict(kind="vs_windows", last_q=100, n_vert=0, n_slash=40),
            dict(kind="block_threshold", alpha=0.5),
            dict(kind="unified", alpha=0.6)]
    run(dsa, Q, K, V, pats, B)


def test_vs_row_tiles_d64(dsa):
    """The VS estimate stacks the estimate rows of two VS heads of a KV group
    (64 rows each) into one tensor-core operand, or takes one head of up to 128
    rows alone: five VS heads of one KV group with 64, 30, 100, 1 and 64 rows
    give two pairs and one single head, next to other kinds, at d = 64 and a
    ragged length."""
    N, d, B = 2100, 64, 64
    Q, K, V = synth.random_qkv(8, 1, N, d, seed=41)
    pats = [dict(kind="vs", last_q=64, n_vert=70, n_slash=40),
            dict(kind="vs", last_q=30, n_vert=10, n_slash=300),
            dict(kind="block_topk", topk=4),
            dict(kind="vs", last_q=100, n_vert=128, n_slash=64),
            dict(kind="vs", last_q=1, n_vert=5, n_slash=5),
            dict(kind="ashape", sink=64, window=200),
            dict(kind="vs", last_q=64, n_vert=1, n_slash=1000),
            dict(kind="block_threshold", alpha=0.6)]
    run(dsa, Q, K, V, pats, B, rows=np.r_[0:80, 1000:1100, N - 150:N])


@pytest.mark.parametrize("B", [128, 512])
@pytest.mark.parametrize("conv", [False, True])
def test_moba(dsa, B, conv):
    w = synth.workload(4, N=1400 if B == 128 else 2600, Hq=2, Hkv=2, B=B, conv_width=4 if conv else 0)
    Q, K, V, _ = synth.make_inputs(w)
    convs = synth.conv_weights(w)
    run(dsa, Q, K, V, synth.head_patterns(w), B, convs=convs,
        rows=np.r_[0:64, 500:600, w["N"] - 200:w["N"]])


@pytest.mark.parametrize("d", [64, 128])
def test_moba_conv_widths(dsa, d):
    """Each key-conv width has its own pooling instantiation: five KV heads with
    widths 1, 3, 5 and 8 and one without a conv (five launches), non-zero biases,
    a ragged last block, and runs of rows that start inside the previous block
    (the causal window reaches back across the block boundary)."""
    N, B = 1100, 128
    widths = [1, 3, 5, 8, 0]
    Q, K, V = synth.random_qkv(5, 5, N, d, seed=77 + d)
    g = torch.Generator().manual_seed(5 + d)
    convs = [None if W == 0 else (torch.randn(d, W, generator=g) * 0.5, torch.randn(d, generator=g) * 0.3)
             for W in widths]
    pats = [dict(kind="moba", topk=3) for _ in widths]
    dpats = [dict(p, conv=(c[0].cuda(), c[1].cuda())) if c is not None else p for p, c in zip(pats, convs)]
    bufs = dsa.build_indices(Q.cuda(), K.cuda(), dpats, B)
    torch.cuda.synchronize()
    assert dsa.device_status() == (0, 0)
    oconvs = [None if c is None else (c[0].double().numpy(), c[1].double().numpy()) for c in convs]
    ref = orc.build_indices(to64(Q), to64(K), pats, B, oconvs)
    check_indices(bufs, ref, pats, N, B)


def test_threshold_topics(dsa):
    w = synth.workload(3, N=4096, Hq=4, Hkv=2)
    Q, K, V, planted = synth.make_inputs(w)
    bufs = run(dsa, Q, K, V, synth.head_patterns(w), w["B"], rows=np.r_[0:130, 2000:2100, 3900:4096])
    # same-topic blocks are found: every kept block J < I shares I's topic, and
    # the blocks earlier in the sequence with I's topic are kept
    topic = planted["topic"][0].numpy()
    lists = bufs.host_lists()[0]["blocks"]
    hits = sum(int(all(topic[J] == topic[I] for J in lists[I] if J not in (0, I))) for I in range(len(lists)))
    assert hits >= 0.9 * len(lists)


@pytest.mark.parametrize("wid", [2, 3])
def test_unified_discovery(dsa, wid):
    """FlashPrefill-style discovery of vertical, diagonal and block shapes from one
    pooled block search (DSA_KIND_UNIFIED) on two layers: planted vertical tokens
    and periodic slashes (the mixed layer's data), and per-block topics; with
    another kind in the same KV group and a ragged length."""
    N = 4000 if wid == 2 else 4096
    w = synth.workload(wid, N=N, Hq=4, Hkv=2)
    Q, K, V, _ = synth.make_inputs(w)
    B = w["B"]
    pats = [dict(kind="unified", alpha=0.5), dict(kind="unified", alpha=0.1, keep_sink=0, keep_local=0),
            dict(kind="block_threshold", alpha=0.5), dict(kind="unified", alpha=0.9)]
    bufs = run(dsa, Q, K, V, pats, B, rows=np.r_[0:80, 1800:1900, N - 120:N])
    lists = bufs.host_lists()
    assert all(len(lists[h]["vert"]) > 0 and len(lists[h]["slash"]) > 0 for h in (0, 1, 3))


def test_index_build_is_deterministic(dsa):
    """Two builds of the same layer give the same lists bit for bit: the VS sums
    use no floating-point atomics (each key chunk writes its own window of slash
    sums; windows that overlap are added in a fixed order)."""
    w = synth.workload(2, N=6000, Hq=8, Hkv=2)
    Q, K, V, _ = synth.make_inputs(w)
    pats = synth.head_patterns(w)
    Qd, Kd = Q.cuda(), K.cuda()
    a = dsa.build_indices(Qd, Kd, pats, w["B"])
    b = dsa.build_indices(Qd, Kd, pats, w["B"])
    torch.cuda.synchronize()
    for name in ("head_info", "blk_ptr", "blk_idx", "dist_ptr", "dist", "col_ptr", "col_idx", "vert_idx",
                 "slash_idx"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert any(p["kind"] == "vs" for p in pats)


@pytest.mark.parametrize("N", [70000, 300001])
def test_vs_topk_multi_cta(dsa, N):
    """The VS top-k runs as a cluster of CTAs for long arrays (4 CTAs above 65,536
    keys, 8 above 262,144), each owning a contiguous segment: the selected sets
    against the oracle's scores (tie-aware), ascending, for a large k, a small k
    and k at the array length's scale; two builds give identical lists."""
    pats = [dict(kind="vs", last_q=64, n_vert=1000, n_slash=6096), dict(kind="vs", last_q=32, n_vert=3, n_slash=1),
            dict(kind="vs", last_q=64, n_vert=5000, n_slash=N - 5)]
    Q, K, _ = synth.random_qkv(3, 1, N, 128, seed=N % 97)
    Qd, Kd = Q.cuda(), K.cuda()
    a = dsa.build_indices(Qd, Kd, pats, 64)
    b = dsa.build_indices(Qd, Kd, pats, 64)
    torch.cuda.synchronize()
    assert dsa.device_status() == (0, 0)
    assert torch.equal(a.vert_idx, b.vert_idx) and torch.equal(a.slash_idx, b.slash_idx)
    lists = a.host_lists()
    k64 = to64(K[0])
    for h, p in enumerate(pats):
        v, s = orc.vs_estimate(to64(Q[h]), k64, p["last_q"])
        for got, sc, k in ((lists[h]["vert"], v, p["n_vert"]), (lists[h]["slash"], s, p["n_slash"])):
            assert len(got) == k and np.all(np.diff(got) > 0), (h, k)
            ok, msg = topk_set_ok(got, orc.topk_indices(sc, k), sc, k)
            assert ok, f"head {h}, k {k}: {msg}"
