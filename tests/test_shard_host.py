"""Head-sharded prefill of one layer, host logic on CPU: the KV-group partition
covers every head exactly once with balanced shards, and with the gloo backend
(world sizes 2 and 3) each rank's shard, computed by the fp64 oracle, gathers
into exactly the single-process layer output."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from dynamic_sparse_attention_build_b200 import shard  # noqa: E402


@pytest.mark.parametrize("Hq,Hkv,world", [(32, 8, 8), (32, 8, 3), (16, 16, 4), (8, 2, 2), (4, 4, 3), (6, 3, 4)])
def test_partition_covers_every_head_once(Hq, Hkv, world):
    seen = []
    sizes = []
    for r in range(world):
        k0, k1 = shard.kv_group_range(r, world, Hkv)
        q0, q1 = shard.head_range(r, world, Hq, Hkv)
        assert q0 == k0 * (Hq // Hkv) and q1 == k1 * (Hq // Hkv)
        seen += list(range(q0, q1))
        sizes.append(k1 - k0)
    assert seen == list(range(Hq))
    assert max(sizes) - min(sizes) <= 1


def _oracle_compute(q, k, v, pats, B):
    """Stand-in for the library's two calls on CPU: the oracle, head by head."""
    from oracle import dsa_oracle as orc
    G = q.shape[0] // k.shape[0]
    out = []
    for h in range(q.shape[0]):
        qh, kh, vh = (t.double().numpy() for t in (q[h], k[h // G], v[h // G]))
        hi = orc.build_head_index(qh, kh, pats[h], B)
        O, _ = orc.attention_rows(qh, kh, vh, hi, np.arange(qh.shape[0]))
        out.append(torch.from_numpy(O))
    return torch.stack(out)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _layer():
    import synth
    Q, K, V = synth.random_qkv(6, 3, 160, 16, seed=9)
    pats = [dict(kind="ashape", sink=8, window=40), dict(kind="block_topk", topk=2),
            dict(kind="vs", last_q=16, n_vert=6, n_slash=4), dict(kind="block_threshold", alpha=0.5),
            dict(kind="moba", topk=1), dict(kind="ashape", sink=0, window=64)]
    return Q, K, V, pats


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    from dynamic_sparse_attention_build_b200 import shard as sh
    Q, K, V, pats = _layer()
    O_local = sh.sharded_prefill(Q, K, V, pats, 32, rank, world, compute=_oracle_compute)
    O_full = sh.sharded_prefill(Q, K, V, pats, 32, rank, world, gather=True, compute=_oracle_compute)
    out[rank] = (O_local.numpy(), O_full.numpy())
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gathered_shards_equal_the_layer(world):
    Q, K, V, pats = _layer()
    ref = _oracle_compute(Q, K, V, pats, 32).numpy()
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        O_local, O_full = res[r]
        q0, q1 = shard.head_range(r, world, 6, 3)
        np.testing.assert_array_equal(O_local, ref[q0:q1])
        np.testing.assert_array_equal(O_full, ref)
