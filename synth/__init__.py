"""Seeded synthetic inputs for dynamic sparse attention prefill.

This module only draws random numbers and lays out test data: the Q/K/V tensors
of each workload, its planted vertical / slash / topic structure, the per-head
pattern assignment and the MoBA key-conv weights.  It holds none of the method's
arithmetic, so both the CUDA path's tests and the CPU oracle can take their inputs
from it.

Workloads (all batch 1, causal, bf16):

1. ``vs_tiny_4k``: 1 q / 1 KV head, N=4096, d=64, N(0,1) + RoPE base 1e4,
   Vertical-Slash (last_q 64, 256 vertical, 256 slash, block 64), 8 planted
   vertical tokens.
2. ``llama3_8b_mixed_32k``: 32 q / 8 KV heads, d=128, N=32768, N(0,1) + RoPE base
   5e5; per-head patterns drawn from the seed (20% A-shape sink 128 / window 1024,
   60% Vertical-Slash 64 / 1000 / 6096, 20% block top-100), block 64; 32 planted
   vertical tokens and 4 periodic slash offsets per KV head.
3. ``flashprefill_threshold_128k``: 32 q / 8 KV heads, d=128, N=131072, 512 topic
   vectors, each 128-token block drawn from one topic plus N(0, 0.5^2) noise;
   block threshold alpha=0.5 (probability space) with the sink and local blocks.
4. ``moba_64k``: 16 q / 16 KV heads, d=128, N=65536, N(0,1); MoBA top-8 plus the
   own block, block 512 or 128, optional width-4 causal depthwise key conv.
5. ``vs_1m``: 32 q / 8 KV heads, d=128, N=2^20, N(0,1) + RoPE base 5e5, all heads
   Vertical-Slash (64 / 1000 / 6096, block 64), 64 planted vertical tokens and 4
   periodic slash offsets per KV head.

Every size can be overridden (``N=``, ``Hq=``, ``Hkv=``, ``d=``) to get a small
case with the same structure.
"""
from __future__ import annotations

import math

import torch

WORKLOADS = {
    1: dict(name="vs_tiny_4k", Hq=1, Hkv=1, N=4096, d=64, B=64, rope=1e4,
            n_planted_vert=8, n_planted_slash=0, mix="vs",
            vs=dict(last_q=64, n_vert=256, n_slash=256)),
    2: dict(name="llama3_8b_mixed_32k", Hq=32, Hkv=8, N=32768, d=128, B=64, rope=5e5,
            n_planted_vert=32, n_planted_slash=4, mix="mixed",
            vs=dict(last_q=64, n_vert=1000, n_slash=6096),
            ashape=dict(sink=128, window=1024), block_topk=dict(topk=100)),
    3: dict(name="flashprefill_threshold_128k", Hq=32, Hkv=8, N=131072, d=128, B=128,
            rope=None, topics=512, topic_block=128, noise=0.5, mix="threshold",
            threshold=dict(alpha=0.5, keep_sink=1, keep_local=1)),
    4: dict(name="moba_64k", Hq=16, Hkv=16, N=65536, d=128, B=512, rope=None,
            mix="moba", moba=dict(topk=8), conv_width=0),
    5: dict(name="vs_1m", Hq=32, Hkv=8, N=1 << 20, d=128, B=64, rope=5e5,
            n_planted_vert=64, n_planted_slash=4, mix="vs",
            vs=dict(last_q=64, n_vert=1000, n_slash=6096)),
}


def workload(cfg_id: int, **over) -> dict:
    """A copy of workload ``cfg_id`` with any field overridden."""
    w = dict(WORKLOADS[cfg_id])
    w.update(over)
    w["id"] = cfg_id
    w["seed"] = over.get("seed", 1000 + cfg_id)
    return w


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _rope_(x: torch.Tensor, base: float) -> None:
    """Llama-style rotate-half rotary embedding, in place, on fp32 [N, d]."""
    N, d = x.shape
    half = d // 2
    inv = 1.0 / (base ** (torch.arange(0, half, device=x.device, dtype=torch.float64) / half))
    pos = torch.arange(N, device=x.device, dtype=torch.float64)
    ang = torch.outer(pos, inv)
    cos = torch.cos(ang).to(torch.float32)
    sin = torch.sin(ang).to(torch.float32)
    x1 = x[:, :half].clone()
    x2 = x[:, half:].clone()
    x[:, :half] = x1 * cos - x2 * sin
    x[:, half:] = x2 * cos + x1 * sin


def head_patterns(w: dict) -> list:
    """Per-q-head pattern dicts, drawn from the seed for the mixed workload."""
    Hq = w["Hq"]
    mix = w["mix"]
    B = w["B"]
    if mix == "vs":
        return [dict(kind="vs", **w["vs"]) for _ in range(Hq)]
    if mix == "threshold":
        return [dict(kind="block_threshold", **w["threshold"]) for _ in range(Hq)]
    if mix == "moba":
        return [dict(kind="moba", **w["moba"]) for _ in range(Hq)]
    if mix == "mixed":
        n_a = round(0.2 * Hq)
        n_b = round(0.2 * Hq)
        kinds = ["ashape"] * n_a + ["block_topk"] * n_b + ["vs"] * (Hq - n_a - n_b)
        g = _gen(w["seed"] + 7, "cpu")
        perm = torch.randperm(Hq, generator=g).tolist()
        kinds = [kinds[p] for p in perm]
        out = []
        for k in kinds:
            if k == "ashape":
                out.append(dict(kind="ashape", **w["ashape"]))
            elif k == "block_topk":
                out.append(dict(kind="block_topk", **w["block_topk"]))
            else:
                out.append(dict(kind="vs", **w["vs"]))
        return out
    raise ValueError(mix)


def conv_weights(w: dict, device="cpu"):
    """MoBA key-conv weights per KV head: taps ~ N(0, 1/4) of shape [d, W] and zero
    bias [d], float32; None when the conv is off."""
    W = int(w.get("conv_width", 0) or 0)
    if W == 0:
        return None
    g = _gen(w["seed"] + 11, device)
    out = []
    for _ in range(w["Hkv"]):
        taps = torch.randn(w["d"], W, generator=g, device=device, dtype=torch.float32) * 0.5
        out.append((taps, torch.zeros(w["d"], device=device, dtype=torch.float32)))
    return out


def make_inputs(w: dict, device="cpu"):
    """Q [Hq, N, d], K [Hkv, N, d], V [Hkv, N, d] as bf16 on ``device``, plus a dict
    describing the planted structure (positions and offsets)."""
    Hq, Hkv, N, d = w["Hq"], w["Hkv"], w["N"], w["d"]
    G = Hq // Hkv
    g = _gen(w["seed"], device)
    Q = torch.empty(Hq, N, d, device=device, dtype=torch.bfloat16)
    K = torch.empty(Hkv, N, d, device=device, dtype=torch.bfloat16)
    V = torch.empty(Hkv, N, d, device=device, dtype=torch.bfloat16)
    planted = dict(vert=[], slash=[], topic=[])
    if w["mix"] == "threshold":
        T = w["topics"]
        tb = w["topic_block"]
        nb = (N + tb - 1) // tb
        for kv in range(Hkv):
            topics = torch.randn(T, d, generator=g, device=device, dtype=torch.float32)
            assign = torch.randint(0, T, (nb,), generator=g, device=device)
            base = topics[assign].repeat_interleave(tb, dim=0)[:N]
            planted["topic"].append(assign.cpu())
            for h in range(kv * G, kv * G + G):
                Q[h] = (base + w["noise"] * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16)
            K[kv] = (base + w["noise"] * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16)
            V[kv] = (base + w["noise"] * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16)
        return Q, K, V, planted
    nv = int(w.get("n_planted_vert", 0) or 0)
    ns = int(w.get("n_planted_slash", 0) or 0)
    scale = d ** 0.25
    for kv in range(Hkv):
        kf = torch.randn(N, d, generator=g, device=device, dtype=torch.float32)
        vf = torch.randn(N, d, generator=g, device=device, dtype=torch.float32)
        qf = [torch.randn(N, d, generator=g, device=device, dtype=torch.float32) for _ in range(G)]
        if w.get("rope"):
            _rope_(kf, w["rope"])
            for q in qf:
                _rope_(q, w["rope"])
        u = torch.randn(d, generator=g, device=device, dtype=torch.float32)
        u = u / u.norm()
        pos = torch.zeros(0, dtype=torch.int64)
        if nv > 0:
            pos = torch.randperm(N, generator=g, device=device)[: min(nv, N)].sort().values
            for q in qf:
                q += scale * u
            kf[pos] += 4.0 * scale * u
        planted["vert"].append(pos.cpu())
        offs = []
        if ns > 0:
            P = int(torch.randint(64, 2049, (1,), generator=g, device=device).item())
            qsum = torch.stack(qf).sum(0)
            for m in range(1, ns + 1):
                o = m * P
                if o < N:
                    kf[: N - o] += (4.0 / math.sqrt(d)) * qsum[o:]
                    offs.append(o)
        planted["slash"].append(offs)
        K[kv] = kf.to(torch.bfloat16)
        V[kv] = vf.to(torch.bfloat16)
        for t, q in enumerate(qf):
            Q[kv * G + t] = q.to(torch.bfloat16)
    return Q, K, V, planted


def random_qkv(Hq, Hkv, N, d, seed, device="cpu", scale=1.0):
    """Plain N(0, scale^2) bf16 Q [Hq,N,d], K/V [Hkv,N,d] for small parity cases."""
    g = _gen(seed, device)
    Q = (scale * torch.randn(Hq, N, d, generator=g, device=device)).to(torch.bfloat16)
    K = (scale * torch.randn(Hkv, N, d, generator=g, device=device)).to(torch.bfloat16)
    V = torch.randn(Hkv, N, d, generator=g, device=device).to(torch.bfloat16)
    return Q, K, V
