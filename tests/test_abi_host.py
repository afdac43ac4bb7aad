"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
function include/dsa.h declares, validates arguments before any launch, and
sizes its index lists and workspace."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import synth
from oracle import dsa_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from dynamic_sparse_attention_build_b200 import _binding
    if not os.path.exists(_binding.LIB_PATH):
        from dynamic_sparse_attention_build_b200 import build
        build.build()
    _binding.lib()
    return _binding


def header_functions():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_function(B):
    names = header_functions()
    assert len(names) >= 8
    lib = B.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTS)


def problem(B, Hq=4, Hkv=2, N=1000, d=128, block=64):
    p = B.dsa_problem()
    p.Hq, p.Hkv, p.N, p.d, p.block = Hq, Hkv, N, d, block
    p.q_head_stride = p.k_head_stride = p.v_head_stride = p.o_head_stride = N * d
    p.q_token_stride = p.k_token_stride = p.v_token_stride = p.o_token_stride = d
    return p


def pats(B, kinds):
    from dynamic_sparse_attention_build_b200.api import make_patterns
    return make_patterns(kinds)


DEF = [dict(kind="vs", last_q=64, n_vert=10, n_slash=20), dict(kind="ashape", sink=4, window=100),
       dict(kind="block_topk", topk=3), dict(kind="block_threshold", alpha=0.5)]


def status_of(B, p, pp):
    sz = B.dsa_sizes()
    return B.lib().dsa_workspace_size(ctypes.byref(p), pp, ctypes.byref(sz)), sz


def test_problem_validation(B):
    pp = pats(B, DEF)
    assert status_of(B, problem(B), pp)[0] == B.DSA_OK
    assert status_of(B, problem(B, d=96), pp)[0] == B.DSA_ERR_UNSUPPORTED
    assert status_of(B, problem(B, Hq=4, Hkv=3), pp)[0] == B.DSA_ERR_INVALID_ARG
    assert status_of(B, problem(B, block=32), pp)[0] == B.DSA_ERR_INVALID_ARG
    assert status_of(B, problem(B, N=0), pp)[0] == B.DSA_ERR_INVALID_ARG
    p = problem(B)
    p.k_token_stride = 100  # not a multiple of 8 elements
    assert status_of(B, p, pp)[0] == B.DSA_ERR_INVALID_ARG
    p = problem(B)
    p.q_token_stride = 64  # shorter than a row
    assert status_of(B, p, pp)[0] == B.DSA_ERR_INVALID_ARG
    assert B.lib().dsa_workspace_size(None, pp, None) == B.DSA_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(kind="ashape", sink=-1, window=4), dict(kind="ashape", sink=0, window=0),
                                 dict(kind="vs", last_q=0, n_vert=1, n_slash=1),
                                 dict(kind="block_topk", topk=0),
                                 dict(kind="block_threshold", alpha=0.0),
                                 dict(kind="block_threshold", alpha=1.5)])
def test_pattern_validation(B, bad):
    pp = pats(B, [bad] + DEF[1:])
    assert status_of(B, problem(B), pp)[0] == B.DSA_ERR_INVALID_ARG


def test_vs_last_q_limit(B):
    pp = pats(B, [dict(kind="vs", last_q=129, n_vert=1, n_slash=1)] + DEF[1:])
    assert status_of(B, problem(B), pp)[0] == B.DSA_ERR_UNSUPPORTED


def test_conv_must_match_within_group(B):
    w1 = torch.zeros(128, 4)
    w2 = torch.zeros(128, 4)
    b = torch.zeros(128)
    # host tensors stand in for device pointers: only the pointer identity is checked here
    p = [dict(kind="moba", topk=2, conv=(w1, b)), dict(kind="moba", topk=2, conv=(w2, b)),
         dict(kind="moba", topk=2), dict(kind="moba", topk=2)]
    assert status_of(B, problem(B), pats(B, p))[0] == B.DSA_ERR_INVALID_ARG
    p[1] = dict(kind="moba", topk=2, conv=(w1, b))
    assert status_of(B, problem(B), pats(B, p))[0] == B.DSA_OK


def test_capacities_are_exact_or_bounds(B):
    N, Bk = 1000, 64
    p = problem(B, Hq=4, Hkv=2, N=N, block=Bk)
    st, sz = status_of(B, p, pats(B, DEF))
    assert st == 0
    nqb = (N + Bk - 1) // Bk
    assert sz.nqb == nqb and sz.blk_ptr_len == 4 * nqb + 1 and sz.col_ptr_len == 4 * nqb + 1
    # A-shape block count is exact (the oracle's block sets)
    a = sum(orc.ashape_blocks(q, Bk, N, 4, 100).size for q in range(nqb))
    topk = sum(min(3, q + 1) for q in range(nqb))
    thr = sum(q + 1 for q in range(nqb))
    assert sz.blk_cap == a + topk + thr
    assert sz.dist_cap == min(40, nqb)
    assert sz.col_cap == sum(min(10, q * Bk + Bk) for q in range(nqb))
    assert sz.vert_stride == 10 and sz.slash_stride == 20
    assert sz.workspace_bytes > 0 and sz.workspace_bytes % 256 == 0


@pytest.mark.parametrize("N", [129, 1000, 4096, 32768, 100000])
def test_vs_workspace_covers_every_key_chunk(B, N):
    # The VS estimate's key chunk (1024, 768 or 512 keys) is chosen at build time
    # from the device's SM count, so the workspace, sized without a device, must
    # hold the per-chunk row statistics and slash windows of any of them, on top
    # of the v and s sums.
    nvs = 3
    kinds = [dict(kind="vs", last_q=128, n_vert=10, n_slash=20)] * nvs + [dict(kind="ashape", sink=4, window=100)]
    p = problem(B, Hq=4, Hkv=2, N=N, block=64)
    st, sz = status_of(B, p, pats(B, kinds))
    assert st == 0
    need = 2 * nvs * N * 4  # v and s
    for c in (1024, 768, 512):
        nch = -(-N // c)
        parts = nvs * nch * 128 * 2 * 4  # (max, sum) of up to 128 estimate rows per chunk
        wins = nvs * nch * (c + 128) * 4  # slash window per chunk
        assert sz.workspace_bytes >= need + parts + wins, (N, c)


def test_null_pointers_rejected_before_launch(B):
    p = problem(B)
    pp = pats(B, DEF)
    idx = B.dsa_indices()
    lib = B.lib()
    assert lib.dsa_sparse_prefill(ctypes.byref(p), None, None, None, ctypes.byref(idx), None, None, None) \
        == B.DSA_ERR_INVALID_ARG
    assert lib.dsa_build_indices(ctypes.byref(p), None, None, pp, ctypes.byref(idx), None, 0, None) \
        == B.DSA_ERR_INVALID_ARG
    assert lib.dsa_selftest_wait_timeout(0, None) == B.DSA_ERR_INVALID_ARG


def test_status_strings(B):
    for s in range(7):
        assert B.dsa_status_string(s)
    assert B.dsa_status_string(99) == "unknown status"


def test_synth_workloads_are_deterministic():
    w = synth.workload(2, N=256, Hq=4, Hkv=2)
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    kinds = [p["kind"] for p in synth.head_patterns(synth.workload(2))]
    assert kinds.count("ashape") == 6 and kinds.count("block_topk") == 6 and kinds.count("vs") == 20
