"""Head-sharded prefill of one layer over several GPUs (one process per GPU).

Heads are independent in both steps of the path (index building reads a
q-head and its KV head, attention reads the same), so a layer splits by whole
KV groups — the G q-heads that share a KV head travel with it — with no
exchange on the data path.  Each rank runs ``build_indices`` and
``sparse_prefill`` on its own groups; if the caller needs every head's output
on every rank, one all-gather of O at the layer boundary assembles it (NCCL over
NVLink on GPUs).  Ranks own contiguous, balanced runs of KV groups: the first
``Hkv % world`` ranks take one group more.
"""
from __future__ import annotations

import torch


def kv_group_range(rank: int, world: int, Hkv: int) -> tuple[int, int]:
    """[first, last) KV heads of ``rank``: contiguous, sizes differ by at most one."""
    if not (0 <= rank < world) or world < 1:
        raise ValueError(f"rank {rank} not in a world of {world}")
    base, extra = divmod(Hkv, world)
    first = rank * base + min(rank, extra)
    return first, first + base + (1 if rank < extra else 0)


def head_range(rank: int, world: int, Hq: int, Hkv: int) -> tuple[int, int]:
    """[first, last) q-heads of ``rank``: the q-heads of its KV groups."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    k0, k1 = kv_group_range(rank, world, Hkv)
    return k0 * G, k1 * G


def shard_inputs(Q, K, V, patterns, rank: int, world: int):
    """This rank's views of a layer: Q, K, V head slices and its patterns."""
    Hq, Hkv = Q.shape[0], K.shape[0]
    q0, q1 = head_range(rank, world, Hq, Hkv)
    k0, k1 = kv_group_range(rank, world, Hkv)
    return Q[q0:q1], K[k0:k1], V[k0:k1], list(patterns[q0:q1])


def gather_heads(O_local: torch.Tensor, Hq: int, Hkv: int, group=None) -> torch.Tensor:
    """All-gather every rank's [heads, N, d] output into the full [Hq, N, d]
    (one collective; shards may differ in size by one KV group)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    G = Hq // Hkv
    sizes = [(kv_group_range(r, world, Hkv)[1] - kv_group_range(r, world, Hkv)[0]) * G for r in range(world)]
    if O_local.shape[0] != sizes[rank]:
        raise ValueError(f"rank {rank} holds {O_local.shape[0]} heads, expected {sizes[rank]}")
    mx = max(sizes)
    tail = O_local.shape[1:]
    send = O_local
    if O_local.shape[0] < mx:  # equal-sized pieces for one all_gather_into_tensor
        send = torch.cat([O_local, O_local.new_zeros((mx - O_local.shape[0],) + tail)])
    out = O_local.new_empty((world * mx,) + tail)
    dist.all_gather_into_tensor(out, send.contiguous(), group=group)
    return torch.cat([out[r * mx:r * mx + sizes[r]] for r in range(world)])


def sharded_prefill(Q, K, V, patterns, block, rank: int, world: int, gather=False, group=None, compute=None):
    """Builds indices and runs attention for this rank's KV groups; returns this
    rank's O [its heads, N, d] (or the full [Hq, N, d] with ``gather``).
    ``compute(Q, K, V, patterns, block) -> O`` defaults to the library's two calls."""
    Qr, Kr, Vr, pr = shard_inputs(Q, K, V, patterns, rank, world)
    if compute is None:
        from . import api

        def compute(q, k, v, p, b):
            idx = api.build_indices(q, k, p, b)
            return api.sparse_prefill(q, k, v, idx)[0]
    O = compute(Qr, Kr, Vr, pr, block)
    if gather:
        return gather_heads(O, Q.shape[0], K.shape[0], group)
    return O


__all__ = ["gather_heads", "head_range", "kv_group_range", "shard_inputs", "sharded_prefill"]
