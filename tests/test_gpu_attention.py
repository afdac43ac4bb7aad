"""GPU parity of dsa_sparse_prefill against the fp64 oracle, given identical
indices (built by the oracle and handed to the library through the C ABI)."""
import numpy as np
import pytest
import torch

import synth
from oracle import dsa_oracle as orc
from tests._parity import (assert_close_outputs, assert_lse_close, oracle_heads_to_lists, to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


def run_case(dsa, Q, K, V, heads, B, rows=None, layout="hnd"):
    """GPU attention with the oracle's indices vs the oracle's attention."""
    N = Q.shape[1]
    dev = "cuda"
    idx = dsa.indices_from_lists(oracle_heads_to_lists(heads), N, B, dev)
    if layout == "nhd":  # [N, H, d] storage viewed as [H, N, d]
        Qd = Q.transpose(0, 1).contiguous().to(dev).transpose(0, 1)
        Kd = K.transpose(0, 1).contiguous().to(dev).transpose(0, 1)
        Vd = V.transpose(0, 1).contiguous().to(dev).transpose(0, 1)
        O = torch.empty(N, Q.shape[0], Q.shape[2], dtype=torch.bfloat16, device=dev).transpose(0, 1)
    else:
        Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
        O = None
    O, lse = dsa.sparse_prefill(Qd, Kd, Vd, idx, O=O, want_lse=True)
    torch.cuda.synchronize()
    st, det = dsa.device_status()
    assert st == 0, (st, det)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    O_ref, lse_ref = orc.sparse_attention(to64(Q), to64(K), to64(V), heads, rows)
    O_g = to64(O)[:, rows]
    lse_g = lse.cpu().double().numpy()[:, rows]
    res = assert_close_outputs(O_g, O_ref, "O")
    assert_lse_close(lse_g, lse_ref, "lse")
    return res


@pytest.mark.parametrize("N,d,B", [(1000, 128, 64), (777, 64, 64), (1300, 128, 128), (640, 128, 512)])
def test_all_blocks_is_dense_causal(dsa, N, d, B):
    Q, K, V = synth.random_qkv(4, 2, N, d, seed=N + d)
    nb = (N + B - 1) // B
    heads = orc.build_indices(to64(Q), to64(K), [dict(kind="block_topk", topk=nb)] * 4, B)
    run_case(dsa, Q, K, V, heads, B)
    # and the oracle's own dense reference agrees with itself on these rows
    O_dense, _ = orc.dense_causal_attention(to64(Q)[0], to64(K)[0], to64(V)[0])
    O_sp, _ = orc.attention_rows(to64(Q)[0], to64(K)[0], to64(V)[0], heads[0], np.arange(N))
    np.testing.assert_allclose(O_sp, O_dense, rtol=1e-9, atol=1e-12)


def test_vs_tiny_workload(dsa):
    w = synth.workload(1)
    Q, K, V, _ = synth.make_inputs(w)
    heads = orc.build_indices(to64(Q), to64(K), synth.head_patterns(w), w["B"])
    run_case(dsa, Q, K, V, heads, w["B"])


@pytest.mark.parametrize("layout", ["hnd", "nhd"])
def test_mixed_kinds_gqa_ragged(dsa, layout):
    N, d, B = 2000, 128, 64
    Q, K, V = synth.random_qkv(8, 2, N, d, seed=5)
    pats = [dict(kind="vs", last_q=64, n_vert=60, n_slash=50),
            dict(kind="ashape", sink=100, window=300),
            dict(kind="block_topk", topk=5),
            dict(kind="vs", last_q=30, n_vert=10, n_slash=8),
            dict(kind="ashape", sink=0, window=64),
            dict(kind="block_threshold", alpha=0.5, keep_sink=1, keep_local=1),
            dict(kind="moba", topk=3),
            dict(kind="ashape", sink=70, window=1)]
    heads = orc.build_indices(to64(Q), to64(K), pats, B)
    run_case(dsa, Q, K, V, heads, B, layout=layout)


@pytest.mark.parametrize("B", [128, 256, 512])
def test_large_blocks(dsa, B):
    N, d = 1700, 128
    Q, K, V = synth.random_qkv(4, 4, N, d, seed=B)
    pats = [dict(kind="block_threshold", alpha=0.3, keep_sink=1, keep_local=1),
            dict(kind="moba", topk=2), dict(kind="block_topk", topk=3),
            dict(kind="ashape", sink=B // 2 + 3, window=B + 17)]
    heads = orc.build_indices(to64(Q), to64(K), pats, B)
    run_case(dsa, Q, K, V, heads, B)


def test_empty_rows_and_duplicates(dsa):
    """VS head with nothing listed for early rows, columns that repeat keys of a
    listed block (must count once), a column list longer than one tile, and an
    odd column count."""
    N, d, B = 700, 128, 64
    Q, K, V = synth.random_qkv(2, 1, N, d, seed=9)
    nqb = (N + B - 1) // B
    rng = np.random.default_rng(0)
    heads = []
    for h in range(2):
        hi = orc.HeadIndex(kind=orc.VS, B=B, N=N)
        hi.D = np.array([0, 3], np.int64) if h == 0 else np.array([5], np.int64)
        hi.blocks = [np.sort(qb - hi.D[hi.D <= qb]) for qb in range(nqb)]
        cols = []
        for qb in range(nqb):
            hi_lim = min(N, qb * B + B)
            c = np.sort(rng.choice(hi_lim, size=min(hi_lim, 150 + qb), replace=False)) if qb % 3 else \
                np.arange(qb * B + 40, min(N, qb * B + 45))
            cols.append(c.astype(np.int64))
        hi.cols = cols
        heads.append(hi)
    run_case(dsa, Q, K, V, heads, B)


def test_tiny_and_single_block(dsa):
    for N in (1, 17, 64, 65, 129):
        Q, K, V = synth.random_qkv(2, 1, N, 64, seed=N)
        heads = orc.build_indices(to64(Q), to64(K), [dict(kind="block_topk", topk=2),
                                                     dict(kind="ashape", sink=3, window=5)], 64)
        run_case(dsa, Q, K, V, heads, 64)


def test_repeat_runs_are_bit_identical(dsa):
    """The kernel has a fixed order of MMAs and softmax steps, so two runs on the
    same inputs must agree bit for bit; a difference means a race (for example a
    barrier phase read too early)."""
    w = synth.workload(2, N=4000, Hq=8, Hkv=2)
    Q, K, V, _ = synth.make_inputs(w, device="cuda")
    pats = synth.head_patterns(w)
    idx = dsa.build_indices(Q, K, pats, w["B"])
    outs = []
    for _ in range(3):
        O, lse = dsa.sparse_prefill(Q, K, V, idx, want_lse=True)
        torch.cuda.synchronize()
        outs.append((O.clone(), lse.clone()))
    for O, lse in outs[1:]:
        assert torch.equal(O, outs[0][0])
        assert torch.equal(lse, outs[0][1])


@pytest.mark.parametrize("kind", ["dense", "vs"])
def test_large_logit_jumps(dsa, kind):
    """Keys with very large logits after a row's first tile: the running max of
    the online softmax then grows by far more than its raise threshold (2^32 in
    base 2), so O and l are rescaled mid-row (and, for the VS head, columns add
    keys after the block tiles)."""
    N, d, B = 640, 128, 64
    Q, K, V = synth.random_qkv(2, 1, N, d, seed=11)
    g = torch.Generator().manual_seed(12)
    u = torch.randn(d, generator=g)
    u = u / u.norm()
    Kf = K.float()
    # keys 200, 333 and 517 point along u with norm 500: logit ~ 44 * (q . u),
    # i.e. jumps of tens of natural units (x 1.44 in base 2) for many rows
    for j, a in ((200, 500.0), (333, -300.0), (517, 700.0)):
        Kf[0, j] = a * u
    K = Kf.to(torch.bfloat16)
    nb = (N + B - 1) // B
    if kind == "dense":
        pats = [dict(kind="block_topk", topk=nb)] * 2
    else:
        pats = [dict(kind="vs", last_q=64, n_vert=40, n_slash=12)] * 2
    heads = orc.build_indices(to64(Q), to64(K), pats, B)
    if kind == "vs":
        # make sure the planted keys are columns of some query blocks
        for hi in heads:
            for qb in range(nb):
                extra = [j for j in (200, 333, 517) if j <= qb * B + B - 1]
                hi.cols[qb] = np.unique(np.concatenate([hi.cols[qb], np.asarray(extra, np.int64)]))
    # the oracle's rows really do see such jumps
    lg = to64(Q)[0] @ to64(K)[0].T / np.sqrt(d)
    assert (lg[:, 517] - lg[:, :64].max(axis=1) > 32 / np.log2(np.e)).sum() > 20
    run_case(dsa, Q, K, V, heads, B)
