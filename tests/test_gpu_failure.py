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
