"""Head-sharded prefill of one layer through the library's own calls on the GPU
(the multi-GPU partition of whole KV groups, run here on one GPU).

Heads are independent in both calls, so a shard's output must equal the
corresponding heads of the unsharded layer bit for bit: at world size 1, for
each rank of a two-way split computed one after the other in this process, and
through the all-gather of a one-rank NCCL group.  The 32K mixed layer is used
because both halves of its two-way split keep ten Vertical-Slash heads, so the
VS estimate takes the same key chunks as in the whole layer (its sums, and with
them near-tie selections, then agree exactly)."""
import socket

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import dynamic_sparse_attention_build_b200 as m
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_layer_equals_unsharded(dsa):
    from dynamic_sparse_attention_build_b200 import shard
    w = synth.workload(2)
    Q, K, V, _ = synth.make_inputs(w, device="cuda")
    pats = synth.head_patterns(w)
    B = w["B"]
    idx = dsa.build_indices(Q, K, pats, B)
    O_full, _ = dsa.sparse_prefill(Q, K, V, idx)
    torch.cuda.synchronize()
    assert dsa.device_status() == (0, 0)
    kinds = [p["kind"] for p in pats]
    assert kinds[:16].count("vs") == kinds[16:].count("vs") == 10
    # world size 1: the whole layer through the default compute
    O1 = shard.sharded_prefill(Q, K, V, pats, B, rank=0, world=1)
    assert torch.equal(O1, O_full)
    # a two-way split, each rank's KV groups through the library
    parts = []
    for r in range(2):
        q0, q1 = shard.head_range(r, 2, w["Hq"], w["Hkv"])
        Or = shard.sharded_prefill(Q, K, V, pats, B, rank=r, world=2)
        assert Or.shape[0] == q1 - q0
        parts.append(Or)
    assert torch.equal(torch.cat(parts), O_full)
    assert dsa.device_status() == (0, 0)


def test_sharded_gather_one_rank_nccl(dsa):
    import datetime

    import torch.distributed as dist
    from dynamic_sparse_attention_build_b200 import shard
    w = synth.workload(2, N=8192, Hq=8, Hkv=2)
    Q, K, V, _ = synth.make_inputs(w, device="cuda")
    pats = synth.head_patterns(w)
    idx = dsa.build_indices(Q, K, pats, w["B"])
    O_full, _ = dsa.sparse_prefill(Q, K, V, idx)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        O = shard.sharded_prefill(Q, K, V, pats, w["B"], rank=0, world=1, gather=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(O, O_full)
