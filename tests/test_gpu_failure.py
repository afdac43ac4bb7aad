"""Failure paths that a kernel reports without faulting or hanging the GPU: a
bounded wait that runs out, an index outside its range, and capacities that are
too small (rejected on the host before any launch)."""
import numpy as np
import pytest
import torch

import synth
from oracle import dsa_oracle as orc
from tests._parity import oracle_heads_to_lists, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


def test_bounded_wait_reports_timeout(dsa):
    from dynamic_sparse_attention_build_b200 import _binding as B
    import ctypes
    st = B.dsa_selftest_wait_timeout(2000, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == B.DSA_OK
    status, detail = dsa.device_status()
    assert status == B.DSA_ERR_TIMEOUT and detail == 9
    assert dsa.device_status() == (0, 0)  # reading clears it; the context stays usable
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


def test_out_of_range_block_is_reported_and_skipped(dsa):
    from dynamic_sparse_attention_build_b200 import _binding as B
    N, d, Bk = 300, 64, 64
    Q, K, V = synth.random_qkv(1, 1, N, d, seed=3)
    heads = orc.build_indices(to64(Q), to64(K), [dict(kind="block_topk", topk=2)], Bk)
    lists = oracle_heads_to_lists(heads)
    good = dsa.indices_from_lists(lists, N, Bk, "cuda")
    lists[0]["blocks"][3] = np.array([0, 99])  # block 99 does not exist
    bad = dsa.indices_from_lists(lists, N, Bk, "cuda")
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    O_bad, _ = dsa.sparse_prefill(Qd, Kd, Vd, bad)
    status, detail = dsa.device_status()
    assert status == B.DSA_ERR_DEVICE and detail == 30
    O_good, _ = dsa.sparse_prefill(Qd, Kd, Vd, good)
    assert dsa.device_status() == (0, 0)
    # rows of other query blocks are untouched by the bad entry
    assert torch.equal(O_bad[:, :192], O_good[:, :192])
    assert torch.isfinite(O_bad.float()).all()


def test_too_small_capacity_is_rejected_on_the_host(dsa):
    from dynamic_sparse_attention_build_b200 import _binding as B
    from dynamic_sparse_attention_build_b200.api import alloc_indices, make_patterns, make_problem
    N = 1000
    Q, K, _ = synth.random_qkv(2, 1, N, 128, seed=1)
    Qd, Kd = Q.cuda(), K.cuda()
    pats = make_patterns([dict(kind="block_threshold", alpha=0.5), dict(kind="vs", last_q=16, n_vert=8, n_slash=8)])
    prob = make_problem(Qd, Kd, block=64)
    bufs = alloc_indices(prob, pats)
    bufs.blk_idx = bufs.blk_idx[:5]
    bufs.__post_init__()
    with pytest.raises(B.DSAError) as e:
        dsa.build_indices(Qd, Kd, pats, 64, bufs=bufs)
    assert e.value.status == B.DSA_ERR_CAPACITY
    bufs = alloc_indices(prob, pats)
    bufs.workspace = bufs.workspace[:100]
    with pytest.raises(B.DSAError) as e:
        dsa.build_indices(Qd, Kd, pats, 64, bufs=bufs)
    assert e.value.status == B.DSA_ERR_CAPACITY
    assert dsa.device_status() == (0, 0)


def _clone_bufs(dsa, bufs):
    from dynamic_sparse_attention_build_b200.api import IndexBuffers
    return IndexBuffers(Hq=bufs.Hq, N=bufs.N, block=bufs.block, nqb=bufs.nqb,
                        head_info=bufs.head_info.clone(), blk_ptr=bufs.blk_ptr.clone(),
                        blk_idx=bufs.blk_idx.clone(), dist_ptr=bufs.dist_ptr.clone(), dist=bufs.dist.clone(),
                        col_ptr=bufs.col_ptr.clone(), col_idx=bufs.col_idx.clone(),
                        vert_idx=bufs.vert_idx.clone(), slash_idx=bufs.slash_idx.clone(),
                        kinds_present=bufs.kinds_present)


@pytest.mark.parametrize("which", ["blk_past_cap", "blk_negative", "col_past_cap", "col_reversed", "dist_past_cap"])
def test_malformed_rows_are_reported_and_skipped(dsa, which):
    """A CSR row whose pointers leave [0, cap] (or run backwards) is reported as
    DSA_ERR_DEVICE with the list's detail code and treated as empty, by the
    attention kernel and by the pair count; the kernel never reads outside the
    arrays, and every other row is computed as with well-formed lists."""
    from dynamic_sparse_attention_build_b200 import _binding as B
    N, d, Bk = 700, 64, 64
    nqb = (N + Bk - 1) // Bk
    Q, K, V = synth.random_qkv(2, 1, N, d, seed=5)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    pats = [dict(kind="block_topk", topk=3), dict(kind="vs", last_q=16, n_vert=40, n_slash=6)]
    good = dsa.build_indices(Qd, Kd, pats, Bk)
    O_good, _ = dsa.sparse_prefill(Qd, Kd, Vd, good)
    pairs_good = dsa.count_pairs(Qd, Kd, good)
    assert dsa.device_status() == (0, 0)
    bad = _clone_bufs(dsa, good)
    cap_b, cap_c, cap_d = bad.blk_idx.numel(), bad.col_idx.numel(), bad.dist.numel()
    h, qb = (0, 4) if which.startswith("blk") else (1, 6)
    r = h * nqb + qb
    if which == "blk_past_cap":
        bad.blk_ptr[r + 1] = cap_b + 1000       # rows qb and qb + 1 of head 0
        detail, rows = 33, [(0, qb), (0, qb + 1)]
    elif which == "blk_negative":
        bad.blk_ptr[r] = -5                       # rows qb - 1 and qb of head 0
        detail, rows = 33, [(0, qb - 1), (0, qb)]
    elif which == "col_past_cap":
        bad.col_ptr[r + 1] = cap_c + 7
        detail, rows = 34, [(1, qb), (1, qb + 1)]
    elif which == "col_reversed":
        bad.col_ptr[r + 1] = int(bad.col_ptr[r]) - 1   # end before begin
        detail, rows = 34, [(1, qb), (1, qb + 1)]
    else:
        bad.dist_ptr[2] = cap_d + 5               # head 1's distance list
        detail, rows = 35, [(1, q) for q in range(nqb)]
    bad.__post_init__()
    O_bad, _ = dsa.sparse_prefill(Qd, Kd, Vd, bad)
    status, det = dsa.device_status()
    assert status == B.DSA_ERR_DEVICE and det == detail, (status, det)
    pairs_bad = dsa.count_pairs(Qd, Kd, bad)
    status, det = dsa.device_status()
    assert status == B.DSA_ERR_DEVICE and det == detail, (status, det)
    assert dsa.device_status() == (0, 0)
    skipped = np.zeros((2, N), bool)
    for hh, q in rows:
        skipped[hh, q * Bk:min(N, q * Bk + Bk)] = True
    keep = torch.from_numpy(~skipped)
    assert torch.equal(O_bad.cpu()[keep], O_good.cpu()[keep])
    assert torch.isfinite(O_bad.float()).all()
    assert int(pairs_bad[1 - rows[0][0]]) == int(pairs_good[1 - rows[0][0]])
    if which != "col_reversed":  # there the next row reads one column of this one
        assert int(pairs_bad[rows[0][0]]) < int(pairs_good[rows[0][0]])


def test_abort_with_loads_in_flight_leaves_the_next_launch_exact(dsa):
    """With a wait bound of a few microseconds some wait of the attention kernel
    runs out while its CTA still has TMA loads and MMAs in flight; the CTA then
    drains them, frees its tensor memory and exits, the launch reports
    DSA_ERR_TIMEOUT, and the next launch with the default bound is bit-identical
    to a clean run."""
    from dynamic_sparse_attention_build_b200 import _binding as B
    w = synth.workload(2, N=8192, Hq=8, Hkv=2)
    Q, K, V, _ = synth.make_inputs(w, device="cuda")
    pats = synth.head_patterns(w)
    idx = dsa.build_indices(Q, K, pats, w["B"])
    O_ref, lse_ref = dsa.sparse_prefill(Q, K, V, idx, want_lse=True)
    assert dsa.device_status() == (0, 0)
    timeouts = 0
    try:
        for limit_ns in (300, 1000, 3000, 10000, 30000):
            assert B.dsa_set_wait_limit(limit_ns) == B.DSA_OK
            for _ in range(2):
                dsa.sparse_prefill(Q, K, V, idx)
                status, det = dsa.device_status()
                assert status in (B.DSA_OK, B.DSA_ERR_TIMEOUT), (limit_ns, status, det)
                timeouts += status == B.DSA_ERR_TIMEOUT
    finally:
        assert B.dsa_set_wait_limit(0) == B.DSA_OK
    assert timeouts > 0, "no wait ran out: the abort path was not reached"
    O, lse = dsa.sparse_prefill(Q, K, V, idx, want_lse=True)
    assert dsa.device_status() == (0, 0)
    assert torch.equal(O, O_ref) and torch.equal(lse, lse_ref)
    assert B.dsa_set_wait_limit(61 * 10**9) == B.DSA_ERR_INVALID_ARG


@pytest.mark.parametrize("kind", ["vs", "vs_windows"])
def test_kind_missing_from_kinds_present_is_reported(dsa, kind):
    """dsa_sparse_prefill picks its kernel from kinds_present (column tiles only
    with a VS kind, slash-run masks only with VS_WINDOWS).  Lists whose
    kinds_present omits a kind that a head has: that head is reported
    (DSA_ERR_DEVICE, detail 36) and left empty (O = 0, LSE = -inf), the other
    heads equal the run with the right bits."""
    from dynamic_sparse_attention_build_b200 import _binding as B
    N, d, Bk = 700, 64, 64
    Q, K, V = synth.random_qkv(2, 1, N, d, seed=9)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    pats = [dict(kind="block_topk", topk=3), dict(kind=kind, last_q=16, n_vert=20, n_slash=6)]
    good = dsa.build_indices(Qd, Kd, pats, Bk)
    O_good, lse_good = dsa.sparse_prefill(Qd, Kd, Vd, good, want_lse=True)
    assert dsa.device_status() == (0, 0)
    bad = _clone_bufs(dsa, good)
    bad.kinds_present = 1 << B.DSA_KIND_BLOCK_TOPK
    bad.__post_init__()
    O_bad, lse_bad = dsa.sparse_prefill(Qd, Kd, Vd, bad, want_lse=True)
    status, det = dsa.device_status()
    assert status == B.DSA_ERR_DEVICE and det == 36, (status, det)
    assert torch.equal(O_bad[0], O_good[0]) and torch.equal(lse_bad[0], lse_good[0])
    assert not O_bad[1].any() and torch.isinf(lse_bad[1]).all()
    assert dsa.device_status() == (0, 0)
