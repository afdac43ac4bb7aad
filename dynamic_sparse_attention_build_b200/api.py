"""Torch-facing wrappers of the C ABI (marshalling only).

Tensors are bf16 CUDA tensors shaped [heads, tokens, d] (any strides with a
contiguous last dimension; a [tokens, heads, d] tensor viewed with
``.transpose(0, 1)`` works too).  Device memory for indices, workspace and
outputs is allocated here with torch; the library itself allocates nothing.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import numpy as np
import torch

from . import _binding as B


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_problem(Q, K, V=None, O=None, block=64) -> B.dsa_problem:
    Hq, N, d = Q.shape
    Hkv = K.shape[0]
    V = K if V is None else V
    O = Q if O is None else O
    p = B.dsa_problem()
    p.Hq, p.Hkv, p.N, p.d, p.block = Hq, Hkv, N, d, block
    p.q_head_stride, p.q_token_stride = Q.stride(0), Q.stride(1)
    p.k_head_stride, p.k_token_stride = K.stride(0), K.stride(1)
    p.v_head_stride, p.v_token_stride = V.stride(0), V.stride(1)
    p.o_head_stride, p.o_token_stride = O.stride(0), O.stride(1)
    return p


def make_patterns(patterns):
    """list of pattern dicts -> ctypes array of dsa_pattern.  A MoBA dict may hold
    ``conv=(w, b)``: CUDA float32 tensors [d, W] and [d]."""
    arr = (B.dsa_pattern * len(patterns))()
    keep = []
    for h, pd in enumerate(patterns):
        c = arr[h]
        c.kind = B.KIND_CODES[pd["kind"]]
        c.sink = int(pd.get("sink", 0))
        c.window = int(pd.get("window", 1))
        c.last_q = int(pd.get("last_q", 0))
        c.n_vert = int(pd.get("n_vert", 0))
        c.n_slash = int(pd.get("n_slash", 0))
        c.topk = int(pd.get("topk", 0))
        c.alpha = float(pd.get("alpha", 1.0))
        c.keep_sink = int(pd.get("keep_sink", 1))
        c.keep_local = int(pd.get("keep_local", 1))
        conv = pd.get("conv")
        if conv is not None:
            w, b = conv
            w = w.contiguous().float()
            b = b.contiguous().float()
            keep += [w, b]
            c.conv_width = int(w.shape[1])
            c.conv_weight = w.data_ptr()
            c.conv_bias = b.data_ptr()
        else:
            c.conv_width = 0
    arr._keep = keep  # keeps conv tensors alive with the array
    return arr


@dataclass
class IndexBuffers:
    """Device index arrays (see ``dsa_indices`` in include/dsa.h) and their C view."""
    Hq: int
    N: int
    block: int
    nqb: int
    head_info: torch.Tensor
    blk_ptr: torch.Tensor
    blk_idx: torch.Tensor
    dist_ptr: torch.Tensor
    dist: torch.Tensor
    col_ptr: torch.Tensor
    col_idx: torch.Tensor
    vert_idx: torch.Tensor
    slash_idx: torch.Tensor
    workspace: torch.Tensor | None = None
    kinds_present: int = 0  # bit k: some head has kind k (dsa_kind codes)
    c: B.dsa_indices = field(default=None)

    def __post_init__(self):
        c = B.dsa_indices()
        c.head_info = self.head_info.data_ptr()
        c.blk_ptr = self.blk_ptr.data_ptr()
        c.blk_idx = self.blk_idx.data_ptr()
        c.dist_ptr = self.dist_ptr.data_ptr()
        c.dist = self.dist.data_ptr()
        c.col_ptr = self.col_ptr.data_ptr()
        c.col_idx = self.col_idx.data_ptr()
        c.vert_idx = self.vert_idx.data_ptr()
        c.slash_idx = self.slash_idx.data_ptr()
        c.blk_cap = self.blk_idx.numel()
        c.dist_cap = self.dist.numel()
        c.col_cap = self.col_idx.numel()
        c.vert_stride = self.vert_idx.numel() // max(1, self.Hq)
        c.slash_stride = self.slash_idx.numel() // max(1, self.Hq)
        c.kinds_present = self.kinds_present
        self.c = c

    def host_lists(self):
        """Per-head Python view for inspection: dict of numpy arrays."""
        hi = self.head_info.cpu().numpy().reshape(-1, 4)
        bp = self.blk_ptr.cpu().numpy()
        bi = self.blk_idx.cpu().numpy()
        dp = self.dist_ptr.cpu().numpy()
        di = self.dist.cpu().numpy()
        cp = self.col_ptr.cpu().numpy()
        ci = self.col_idx.cpu().numpy()
        vs = self.vert_idx.cpu().numpy().reshape(self.Hq, -1)
        ss = self.slash_idx.cpu().numpy().reshape(self.Hq, -1)
        out = []
        for h in range(self.Hq):
            r0 = h * self.nqb
            out.append(dict(
                kind=int(hi[h, 0]), sink=int(hi[h, 1]), window=int(hi[h, 2]),
                blocks=[bi[bp[r0 + q]:bp[r0 + q + 1]] for q in range(self.nqb)],
                dist=di[dp[h]:dp[h + 1]],
                cols=[ci[cp[r0 + q]:cp[r0 + q + 1]] for q in range(self.nqb)],
                vert=vs[h][vs[h] >= 0], slash=ss[h][ss[h] >= 0]))
        return out


def alloc_indices(problem, pats_c, device="cuda") -> IndexBuffers:
    sz = B.dsa_workspace_size(problem, pats_c)
    i32 = dict(dtype=torch.int32, device=device)
    bufs = IndexBuffers(
        Hq=problem.Hq, N=problem.N, block=problem.block, nqb=sz.nqb,
        head_info=torch.zeros(sz.head_info_len, **i32),
        blk_ptr=torch.zeros(sz.blk_ptr_len, **i32),
        blk_idx=torch.zeros(sz.blk_cap, **i32),
        dist_ptr=torch.zeros(sz.dist_ptr_len, **i32),
        dist=torch.zeros(sz.dist_cap, **i32),
        col_ptr=torch.zeros(sz.col_ptr_len, **i32),
        col_idx=torch.zeros(sz.col_cap, **i32),
        vert_idx=torch.full((problem.Hq * sz.vert_stride,), -1, **i32),
        slash_idx=torch.full((problem.Hq * sz.slash_stride,), -1, **i32),
        workspace=torch.empty(int(sz.workspace_bytes), dtype=torch.uint8, device=device),
        kinds_present=_kinds_mask(int(pats_c[h].kind) for h in range(problem.Hq)),
    )
    return bufs


def _kinds_mask(codes):
    m = 0
    for k in codes:
        m |= 1 << int(k)
    return m


def build_indices(Q, K, patterns, block, bufs: IndexBuffers | None = None, stream=None) -> IndexBuffers:
    """dsa_build_indices on torch tensors; allocates the buffers if none are given."""
    prob = make_problem(Q, K, block=block)
    pats_c = patterns if isinstance(patterns, ctypes.Array) else make_patterns(patterns)
    if bufs is None:
        bufs = alloc_indices(prob, pats_c, Q.device)
    st = B.dsa_build_indices(prob, _ptr(Q), _ptr(K), pats_c, bufs.c, _ptr(bufs.workspace),
                             bufs.workspace.numel(), _stream_ptr(stream))
    B.check(st, "dsa_build_indices")
    bufs._pats = pats_c
    return bufs


def sparse_prefill(Q, K, V, idx: IndexBuffers, O=None, lse=None, want_lse=False, stream=None):
    """dsa_sparse_prefill on torch tensors; returns (O, lse or None)."""
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(Q.shape[0], Q.shape[1], dtype=torch.float32, device=Q.device)
    prob = make_problem(Q, K, V, O, block=idx.block)
    st = B.dsa_sparse_prefill(prob, _ptr(Q), _ptr(K), _ptr(V), idx.c, _ptr(O), _ptr(lse), _stream_ptr(stream))
    B.check(st, "dsa_sparse_prefill")
    return O, lse


def count_pairs(Q, K, idx: IndexBuffers, stream=None) -> torch.Tensor:
    """Exact number of allowed (i, j) pairs per head (int64 tensor [Hq])."""
    pairs = torch.empty(Q.shape[0], dtype=torch.int64, device=Q.device)
    prob = make_problem(Q, K, block=idx.block)
    B.check(B.dsa_count_pairs(prob, idx.c, _ptr(pairs), _stream_ptr(stream)), "dsa_count_pairs")
    return pairs


def device_status(stream=None):
    """(status, detail) of the current device; synchronises the stream."""
    return B.dsa_get_device_status(_stream_ptr(stream))


def indices_from_lists(heads, N, block, device="cuda") -> IndexBuffers:
    """Index buffers from host lists, one dict per head with keys ``kind`` (name),
    ``sink``, ``window``, ``blocks`` (list per query block), ``dist`` (VS),
    ``cols`` (list per query block).  Lets indices from any source reach
    dsa_sparse_prefill."""
    Hq = len(heads)
    nqb = (N + block - 1) // block
    info = np.zeros((Hq, 4), np.int32)
    blk_cnt = np.zeros(Hq * nqb, np.int64)
    col_cnt = np.zeros(Hq * nqb, np.int64)
    dist_cnt = np.zeros(Hq, np.int64)
    blk_all, col_all, dist_all = [], [], []
    for h, hd in enumerate(heads):
        info[h, 0] = B.KIND_CODES[hd["kind"]]
        info[h, 1] = hd.get("sink", 0)
        info[h, 2] = hd.get("window", 0)
        if hd["kind"] in ("vs", "vs_windows"):
            d = np.asarray(hd["dist"], np.int32)
            dist_all.append(d)
            dist_cnt[h] = d.size
        for q in range(nqb):
            if hd["kind"] not in ("vs", "vs_windows"):
                b = np.asarray(hd["blocks"][q], np.int32)
                blk_all.append(b)
                blk_cnt[h * nqb + q] = b.size
            c = np.asarray(hd["cols"][q], np.int32)
            col_all.append(c)
            col_cnt[h * nqb + q] = c.size

    def csr(cnt, parts):
        ptr = np.zeros(cnt.size + 1, np.int32)
        ptr[1:] = np.cumsum(cnt)
        data = np.concatenate(parts).astype(np.int32) if parts else np.zeros(0, np.int32)
        if data.size == 0:
            data = np.zeros(1, np.int32)
        return ptr, data

    bp, bi = csr(blk_cnt, blk_all)
    cp, ci = csr(col_cnt, col_all)
    dp, di = csr(dist_cnt, dist_all)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return IndexBuffers(Hq=Hq, N=N, block=block, nqb=nqb, head_info=t(info.ravel()), blk_ptr=t(bp),
                        blk_idx=t(bi), dist_ptr=t(dp), dist=t(di), col_ptr=t(cp), col_idx=t(ci),
                        vert_idx=torch.full((Hq,), -1, dtype=torch.int32, device=device),
                        slash_idx=torch.full((Hq,), -1, dtype=torch.int32, device=device),
                        kinds_present=_kinds_mask(info[:, 0]))


class HostPrefill:
    """Prefill of one layer whose Q, K, V and O live in pinned host memory, with
    the copies overlapped: the layer's KV groups are split into ``chunks``
    contiguous runs (heads are independent); chunk c's inputs go to the GPU on a
    copy stream while chunk c - 1 computes and chunk c - 2's output comes back on
    another, so a step costs about the largest of the three totals instead of
    their sum.  Device buffers and per-chunk index buffers are allocated once
    and reused by every ``run``; results equal those of the device-resident
    calls head for head."""

    def __init__(self, Hq, Hkv, N, d, patterns, block, chunks=4, device="cuda"):
        from .shard import kv_group_range
        if Hq % Hkv:
            raise ValueError("Hq must be a multiple of Hkv")
        self.G = Hq // Hkv
        self.block = block
        self.device = torch.device(device)
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.Q = torch.empty(Hq, N, d, **bf)
        self.K = torch.empty(Hkv, N, d, **bf)
        self.V = torch.empty(Hkv, N, d, **bf)
        self.O = torch.empty(Hq, N, d, **bf)
        n = max(1, min(chunks, Hkv))
        self.ranges = [kv_group_range(c, n, Hkv) for c in range(n)]
        self.pats = [make_patterns(patterns[k0 * self.G:k1 * self.G]) for k0, k1 in self.ranges]
        # index buffers of every chunk, allocated (and zero-filled on the current
        # stream) here, before any run
        self.bufs = [alloc_indices(make_problem(self.Q[k0 * self.G:k1 * self.G], self.K[k0:k1], block=block),
                                   self.pats[c], self.device) for c, (k0, k1) in enumerate(self.ranges)]
        self.h2d = torch.cuda.Stream(self.device)
        self.comp = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)

    def run(self, Qh, Kh, Vh, Oh):
        """Q/K/V (pinned host, [heads, N, d] bf16) -> Oh (pinned host).  Asynchronous
        with respect to the host; the caller's current stream waits for the last
        output copy, so synchronising it (or an event recorded on it) suffices."""
        cur = torch.cuda.current_stream(self.device)
        # everything the caller's stream did before (including the previous run,
        # which it waits for) happens before this run touches the device buffers
        for s in (self.h2d, self.comp, self.d2h):
            s.wait_stream(cur)
        last = None
        for c, (k0, k1) in enumerate(self.ranges):
            q0, q1 = k0 * self.G, k1 * self.G
            with torch.cuda.stream(self.h2d):
                self.Q[q0:q1].copy_(Qh[q0:q1], non_blocking=True)
                self.K[k0:k1].copy_(Kh[k0:k1], non_blocking=True)
                self.V[k0:k1].copy_(Vh[k0:k1], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(self.h2d)
            self.comp.wait_event(ev_in)
            q, k, v, o = self.Q[q0:q1], self.K[k0:k1], self.V[k0:k1], self.O[q0:q1]
            self.bufs[c] = build_indices(q, k, self.pats[c], self.block, bufs=self.bufs[c], stream=self.comp)
            sparse_prefill(q, k, v, self.bufs[c], O=o, stream=self.comp)
            ev_out = torch.cuda.Event()
            ev_out.record(self.comp)
            self.d2h.wait_event(ev_out)
            with torch.cuda.stream(self.d2h):
                Oh[q0:q1].copy_(o, non_blocking=True)
                last = torch.cuda.Event()
                last.record(self.d2h)
        cur.wait_event(last)
        return Oh

    def status(self):
        """(status, detail) of the kernels that ``run`` enqueued (they run on this
        object's compute stream); synchronises that stream and clears the word."""
        return device_status(self.comp)
