"""dsa_build_indices_static: the index builder for callers that cannot allocate
device memory (a plugin inside a runtime that owns all device memory, or a
latency-critical path where cudaMalloc could synchronise the device).  Its
scratch is a fixed buffer inside the library, so the caller passes only inputs
and output index arrays.

Checked through the C ABI against the regular dsa_build_indices on the same
inputs, on two calls in a row, after a call on an unrelated problem (another
seed, length and set of patterns) has left its own data in the shared buffer:
the buffer keeps the previous call's contents, which must not leak into the
next result.  The attention output built from those indices is checked too.
Kept in a file of its own so that it runs last."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import dsa_oracle as orc
from tests._parity import assert_close_outputs, to64, topk_set_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


PATS = [dict(kind="vs", last_q=64, n_vert=60, n_slash=50), dict(kind="ashape", sink=100, window=300),
        dict(kind="block_topk", topk=5), dict(kind="vs", last_q=32, n_vert=20, n_slash=200),
        dict(kind="block_threshold", alpha=0.5, keep_sink=1, keep_local=1), dict(kind="moba", topk=4),
        dict(kind="vs", last_q=64, n_vert=3000, n_slash=7), dict(kind="ashape", sink=0, window=64)]


def same_indices(a, b, Q, K, N, B):
    """Equal lists; VS selections may differ only inside the oracle's tie band,
    and then distances and columns must follow each side's own selection."""
    la, lb = a.host_lists(), b.host_lists()
    G = Q.shape[0] // K.shape[0]
    for h, (x, y) in enumerate(zip(la, lb)):
        assert (x["kind"], x["sink"], x["window"]) == (y["kind"], y["sink"], y["window"])
        if x["kind"] != 1:
            for qb in range(len(x["blocks"])):
                assert np.array_equal(x["blocks"][qb], y["blocks"][qb]), (h, qb)
            continue
        if np.array_equal(x["vert"], y["vert"]) and np.array_equal(x["slash"], y["slash"]):
            assert np.array_equal(x["dist"], y["dist"])
            for qb in range(len(x["cols"])):
                assert np.array_equal(x["cols"][qb], y["cols"][qb]), (h, qb)
            continue
        v, s = orc.vs_estimate(to64(Q[h]), to64(K[h // G]), PATS[h]["last_q"])
        assert topk_set_ok(x["vert"], y["vert"], v, PATS[h]["n_vert"])[0]
        assert topk_set_ok(x["slash"], y["slash"], s, PATS[h]["n_slash"])[0]
        nqb = (N + B - 1) // B
        for z in (x, y):
            D = orc.vs_distance_set(np.asarray(z["slash"], np.int64), B, nqb)
            assert np.array_equal(z["dist"], D)
            vert = np.asarray(z["vert"], np.int64)
            for qb in range(nqb):
                assert np.array_equal(z["cols"][qb], orc.vs_columns(vert, D, qb, B)), (h, qb)


def test_static_workspace_matches_regular_builder(dsa):
    from dynamic_sparse_attention_build_b200 import _binding as Bi
    from dynamic_sparse_attention_build_b200.api import alloc_indices, make_patterns, make_problem

    N, d, B = 3000, 128, 64
    Q, K, V = synth.random_qkv(8, 2, N, d, seed=31)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    pats_c = make_patterns(PATS)
    ref = dsa.build_indices(Qd, Kd, pats_c, B)
    O_ref, _ = dsa.sparse_prefill(Qd, Kd, Vd, ref)
    prob = make_problem(Qd, Kd, block=B)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # an unrelated problem first, so the shared buffer holds other data (other
    # maxima, bitmaps, sums and counts) when the checked calls start
    N2 = 5000
    Q2, K2, _ = synth.random_qkv(8, 4, N2, d, seed=97)
    Q2d, K2d = Q2.cuda() * 3, K2.cuda()
    pats2 = make_patterns([dict(kind="moba", topk=9), dict(kind="vs", last_q=128, n_vert=700, n_slash=900),
                           dict(kind="block_threshold", alpha=0.2, keep_sink=1, keep_local=1),
                           dict(kind="block_topk", topk=40)] * 2)
    prob2 = make_problem(Q2d, K2d, block=B)
    out2 = alloc_indices(prob2, pats2, "cuda")
    st = Bi.dsa_build_indices_static(prob2, ctypes.c_void_p(Q2d.data_ptr()), ctypes.c_void_p(K2d.data_ptr()),
                                     pats2, out2.c, stream)
    assert st == Bi.DSA_OK, Bi.dsa_status_string(st)
    torch.cuda.synchronize()
    assert dsa.device_status() == (0, 0)
    for call in range(2):
        out = alloc_indices(prob, pats_c, "cuda")  # outputs belong to the caller
        out.workspace = None
        st = Bi.dsa_build_indices_static(prob, ctypes.c_void_p(Qd.data_ptr()), ctypes.c_void_p(Kd.data_ptr()),
                                         pats_c, out.c, stream)
        assert st == Bi.DSA_OK, Bi.dsa_status_string(st)
        torch.cuda.synchronize()
        assert dsa.device_status() == (0, 0)
        same_indices(ref, out, Q, K, N, B)
        O, _ = dsa.sparse_prefill(Qd, Kd, Vd, out)
        torch.cuda.synchronize()
        assert_close_outputs(to64(O), to64(O_ref), f"call {call}")


def test_static_workspace_rejects_large_problem(dsa):
    from dynamic_sparse_attention_build_b200 import _binding as Bi
    from dynamic_sparse_attention_build_b200.api import make_patterns

    p = Bi.dsa_problem()
    p.Hq, p.Hkv, p.N, p.d, p.block = 32, 8, 1 << 20, 128, 64
    p.q_head_stride = p.k_head_stride = p.v_head_stride = p.o_head_stride = (1 << 20) * 128
    p.q_token_stride = p.k_token_stride = p.v_token_stride = p.o_token_stride = 128
    pats_c = make_patterns([dict(kind="vs", last_q=64, n_vert=1000, n_slash=6096)] * 32)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    idx = Bi.dsa_indices()
    for f in ("head_info", "blk_ptr", "blk_idx", "dist_ptr", "dist", "col_ptr", "col_idx", "vert_idx",
              "slash_idx"):
        setattr(idx, f, dummy.data_ptr())
    idx.blk_cap = idx.dist_cap = idx.col_cap = 16
    idx.vert_stride = idx.slash_stride = 1
    st = Bi.dsa_build_indices_static(p, ctypes.c_void_p(dummy.data_ptr()), ctypes.c_void_p(dummy.data_ptr()),
                                     pats_c, idx, ctypes.c_void_p(0))
    assert st == Bi.DSA_ERR_CAPACITY
