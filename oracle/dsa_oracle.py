"""Plain fp64 CPU oracle for dynamic sparse attention prefill.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may import this module.  It
shares no code with the CUDA path and imports nothing from the product package.

Everything here is written for a reader to check against the pages by eye: numpy
in float64, whole-array library primitives (matmul, sort) as single steps, and no
blocking or fusion beyond what each definition states.

Sources (page title, section):

* [MI]  "MInference 1.0: Accelerating Pre-filling for Long-Context LLMs via Dynamic
        Sparse Attention" (abeam.tech summary) -- sections "3つの疎パターン" (the
        three sparse patterns: A-shape, Vertical-Slash, Block-Sparse) and
        "推論時は軽い近似で動的マスクを作る" (building the dynamic mask at inference
        time from Q[-last_q:] x K, or from mean-pooled Q/K blocks).
* [MIa] MInference abstract (zhuanzhiai.com): each head's index lists are built
        at run time from its fixed pattern, and attention is then computed over
        those lists only.
* [FP]  "FlashPrefill: Instantaneous Pattern Discovery and Thresholding for
        Ultra-Fast Long-Context Prefilling" (gist.science summary) -- section 2.1
        (mean-pooled key per block) and section 2.2, the equation
        thresh_I = alpha * max_{J<=I} Score_{I,J}.
* [MoBA] "Optimizing Mixture of Block Attention" (lifetechia.com summary) --
        "MoBA：長文処理の救世主となるか？" (each query attends to a few KV blocks
        picked by a router) and "2. キーに対する畳み込み適用" (short key conv with
        SiLU and a residual before routing).

Readings where the pages are silent:

* score scale tau = 1/sqrt(d) everywhere;
* block score s_IJ = tau * mean(q_I) . mean(k_J)  (equal, by bilinearity, to the
  mean of the token logits of the block);
* VS aggregation: causal row softmax over j <= i for each of the last ``last_q``
  rows, then v[j] = sum_i p_ij and s[o] = sum_i p_{i,i-o};
* top-k ties go to the lower index; with no more candidates than k, all are kept;
* VS index form: block-distance set D = {floor(o/B), ceil(o/B) : o in S} (clipped
  to [0, nkb)), query block qb keeps key blocks {qb - delta : delta in D, delta <= qb},
  and its columns are the verticals j <= qb*B+B-1 whose block is not already kept;
  with ``slash_cover="windows"`` the slashes are instead covered by the exact keys
  they reach from each query block, merged into runs (not aligned to blocks),
  and the columns are the verticals outside those runs;
* threshold in probability space: keep J <= I with P_IJ >= alpha * max_J P_IJ,
  plus the sink block 0 and the local block I when asked;
* MoBA: top-k over J < I by tau * qbar_I . kbar_J, plus the own block I; the key
  conv is k + SiLU(causal depthwise conv(k) + b), used for routing only;
* a row with no allowed key has O = 0 and LSE = -inf.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against brute force, closed forms or a library routine, and
``tests/test_oracle_mutations.py`` plants plausible mistakes in a copy of this
module to check that each one fails a pin.  Parity unpinned: the VS
aggregation rule and the forced blocks of each kind rest on the readings above,
not on anything the pages fix.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# Pattern kinds (plain names; the C ABI has its own enum and this module never
# sees it).
ASHAPE = "ashape"
VS = "vs"
BLOCK_TOPK = "block_topk"
BLOCK_THRESHOLD = "block_threshold"
MOBA = "moba"
UNIFIED = "unified"
VS_WINDOWS = "vs_windows"   # VS with slash_cover="windows"
KINDS = (ASHAPE, VS, BLOCK_TOPK, BLOCK_THRESHOLD, MOBA, UNIFIED, VS_WINDOWS)


def n_blocks(N: int, B: int) -> int:
    return (N + B - 1) // B


# ---------------------------------------------------------------------------
# A-shape  [MI] "3つの疎パターン" / A-shape: sink tokens plus a local window.
# ---------------------------------------------------------------------------
def ashape_allowed(i, j, sink: int, window: int):
    """The A-shape mask: key j is visible to row i iff j <= i and (j is one of the
    first ``sink`` tokens, or j is within the ``window`` most recent keys of i,
    counting i itself).  Works elementwise on numpy arrays."""
    i = np.asarray(i)
    j = np.asarray(j)
    return (j <= i) & ((j < sink) | (i - j < window))


def ashape_blocks(qb: int, B: int, N: int, sink: int, window: int) -> np.ndarray:
    """Key blocks holding at least one A-shape-allowed key for some row of query
    block ``qb``.  Derived from the row definition: row i sees [0, min(sink, i+1))
    and [max(0, i-window+1), i]; the union over the rows of the block is the union
    of those intervals for its first and last row."""
    r0 = qb * B
    r1 = min(N, r0 + B) - 1
    keys = np.union1d(np.arange(0, min(sink, r1 + 1)),
                      np.arange(max(0, r0 - window + 1), r1 + 1))
    return np.unique(keys // B).astype(np.int64)


# ---------------------------------------------------------------------------
# Vertical-Slash  [MI] "推論時は軽い近似で動的マスクを作る": coarse attention of
# Q[-last_q:] against all of K, then pick vertical lines and slash lines.
# ---------------------------------------------------------------------------
def vs_estimate(Qh: np.ndarray, Kh: np.ndarray, last_q: int):
    """Coarse attention of the last ``last_q`` queries of one head.

    Qh, Kh: [N, d] float64.  Returns (v, s), each float64 [N]:
    v[j] = sum over the last rows i of softmax_{j<=i}(tau q_i.k_j)  (vertical line j)
    s[o] = sum over the last rows i of the same probability at j = i - o
           (slash line with offset o = i - j >= 0).
    """
    N, d = Kh.shape
    tau = 1.0 / math.sqrt(d)
    v = np.zeros(N)
    s = np.zeros(N)
    for i in range(max(0, N - last_q), N):
        logits = tau * (Kh[: i + 1] @ Qh[i])
        p = np.exp(logits - logits.max())
        p /= p.sum()
        v[: i + 1] += p
        s[i - np.arange(i + 1)] += p
    return v, s


def topk_indices(x: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries of x, found by a full sort (score
    descending, index ascending, so ties go to the lower index), returned in
    ascending index order.  With len(x) <= k every index is returned."""
    x = np.asarray(x, dtype=np.float64)
    order = np.lexsort((np.arange(x.size), -x))
    return np.sort(order[: min(k, x.size)]).astype(np.int64)


def vs_distance_set(S: np.ndarray, B: int, nkb: int) -> np.ndarray:
    """Block distances that cover every cell of the chosen slash lines.

    For query block qb (rows qb*B .. qb*B+B-1) the keys of slash o are
    j = i - o, which lie in key blocks qb - ceil(o/B) .. qb - floor(o/B); the set of
    distances does not depend on qb.  Distances >= nkb can never apply."""
    S = np.asarray(S, dtype=np.int64)
    D = np.union1d(S // B, -((-S) // B))
    return D[D < nkb].astype(np.int64)


def vs_columns(V: np.ndarray, D: np.ndarray, qb: int, B: int) -> np.ndarray:
    """Vertical columns that query block qb must add on top of its kept blocks:
    j in V that some row of the block can see (j <= qb*B+B-1) and whose key block
    qb - floor(j/B) is not already covered by a distance in D."""
    V = np.asarray(V, dtype=np.int64)
    Dset = set(int(x) for x in D)
    keep = [int(j) for j in V if j <= qb * B + B - 1 and (qb - j // B) not in Dset]
    return np.asarray(keep, dtype=np.int64)


def vs_slash_runs(S: np.ndarray, qb: int, B: int, N: int) -> np.ndarray:
    """The keys that slash lines S reach from query block qb, as maximal runs.

    Rows r0..r1 of the block meet slash o at keys r0 - o .. r1 - o, a window of the
    block's height; keys below 0 do not exist.  Windows that overlap or touch are
    merged.  Returns an int64 array [n, 2] of (first, last) keys, inclusive, in
    ascending order.  (The unaligned alternative to covering each slash with two
    aligned key blocks; the key set equals {i - o : r0 <= i <= r1, o in S, i >= o}.)"""
    r0 = qb * B
    r1 = min(N, r0 + B) - 1
    runs = []
    # larger offsets start further left: descending o gives ascending windows
    for o in sorted((int(x) for x in S), reverse=True):
        if o > r1:
            continue
        a, b = max(0, r0 - o), r1 - o
        if runs and a <= runs[-1][1] + 1:
            runs[-1][1] = max(runs[-1][1], b)
        else:
            runs.append([a, b])
    return np.asarray(runs, dtype=np.int64).reshape(-1, 2)


def vs_window_columns(V: np.ndarray, runs: np.ndarray, qb: int, B: int) -> np.ndarray:
    """Vertical columns query block qb adds on top of its slash runs: j in V that
    some row of the block can see (j <= qb*B+B-1) and that lies in no run."""
    V = np.asarray(V, dtype=np.int64)
    keep = [int(j) for j in V
            if j <= qb * B + B - 1 and not any(a <= j <= b for a, b in runs)]
    return np.asarray(keep, dtype=np.int64)


# ---------------------------------------------------------------------------
# Block scoring  [MI] (mean-pool Q and K per block, block-level attention),
# [FP] 2.1 (mean-pooled key per block), [MoBA] (router over KV blocks).
# ---------------------------------------------------------------------------
def mean_pool(X: np.ndarray, B: int) -> np.ndarray:
    """Mean of each run of B consecutive rows; a last, partial block is averaged
    over the rows it actually has."""
    N, d = X.shape
    nb = n_blocks(N, B)
    out = np.zeros((nb, d))
    for b in range(nb):
        out[b] = X[b * B: min(N, b * B + B)].mean(axis=0)
    return out


def silu(x):
    return x / (1.0 + np.exp(-x))


def key_conv(Kh: np.ndarray, w: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """[MoBA] "2. キーに対する畳み込み適用": short token-level conv on the keys with
    SiLU and a residual.  Causal and depthwise: channel c of token j mixes
    k[j-t, c] for t = 0..W-1 (zero before the first token).
    Kh [N, d], w [d, W], bias [d]."""
    N, d = Kh.shape
    W = w.shape[1]
    conv = np.zeros_like(Kh)
    for t in range(W):
        shifted = np.zeros_like(Kh)
        shifted[t:] = Kh[: N - t] if t < N else 0.0
        conv += shifted * w[:, t][None, :]
    return Kh + silu(conv + bias[None, :])


def block_logits(qbar: np.ndarray, kbar: np.ndarray, d: int) -> np.ndarray:
    """s_IJ = tau * qbar_I . kbar_J for every pair (the caller keeps J <= I)."""
    return (qbar @ kbar.T) / math.sqrt(d)


def select_block_topk(scores_row: np.ndarray, I: int, k: int) -> np.ndarray:
    """MInference block-sparse: the k best key blocks among J <= I."""
    return topk_indices(scores_row[: I + 1], k)


def select_moba(scores_row: np.ndarray, I: int, k: int) -> np.ndarray:
    """MoBA routing: the k best past blocks J < I, plus the query's own block I."""
    past = topk_indices(scores_row[:I], k) if I > 0 else np.zeros(0, np.int64)
    return np.union1d(past, [I]).astype(np.int64)


def select_threshold(scores_row: np.ndarray, I: int, alpha: float,
                     keep_sink: bool, keep_local: bool) -> np.ndarray:
    """[FP] 2.2: thresh_I = alpha * max_{J<=I} Score_IJ, keep Score_IJ >= thresh_I,
    with Score read as the softmax probability over the candidates J <= I."""
    logits = scores_row[: I + 1]
    P = np.exp(logits - logits.max())
    P /= P.sum()
    kept = np.nonzero(P >= alpha * P.max())[0]
    extra = ([0] if keep_sink else []) + ([I] if keep_local else [])
    return np.union1d(kept, extra).astype(np.int64)


def unified_pattern_scores(scores: np.ndarray):
    """[FP] 2.1: the vertical, diagonal and block shapes are found together from
    one pooled block search.  From the block logits s_IJ (J <= I):
      P_IJ = softmax_{J <= I}(s_IJ)                  (row-normalised block weights),
      V_J  = sum_{I >= J} P_IJ                       (vertical: one key block for every query block),
      G_d  = sum_{I >= d} P_{I, I - d}               (diagonal: one block distance d),
    the block-level counterparts of the VS estimate's column and slash sums.
    Returns (P with zeros above the diagonal, V, G)."""
    nqb = scores.shape[0]
    P = np.zeros((nqb, nqb))
    for I in range(nqb):
        row = scores[I, : I + 1]
        w = np.exp(row - row.max())
        P[I, : I + 1] = w / w.sum()
    V = P.sum(axis=0)
    G = np.array([np.trace(P, offset=-dd) for dd in range(nqb)])
    return P, V, G


def select_unified(scores: np.ndarray, alpha: float, keep_sink: bool, keep_local: bool):
    """The max-based threshold of [FP] 2.2 applied per pattern: verticals
    {J : V_J >= alpha max V}, diagonals {d : G_d >= alpha max G}, and for each
    query block I its blocks {J <= I : P_IJ >= alpha max_J P_IJ}.  Query block I
    keeps the union of its blocks, the verticals J <= I, the blocks I - d of the
    diagonals d <= I, and block 0 / block I when asked.
    Returns (list of ascending block arrays, verticals, diagonals)."""
    P, V, G = unified_pattern_scores(scores)
    vert = np.nonzero(V >= alpha * V.max())[0]
    diag = np.nonzero(G >= alpha * G.max())[0]
    out = []
    for I in range(scores.shape[0]):
        row = P[I, : I + 1]
        parts = [np.nonzero(row >= alpha * row.max())[0], vert[vert <= I], I - diag[diag <= I]]
        if keep_sink:
            parts.append(np.array([0]))
        if keep_local:
            parts.append(np.array([I]))
        out.append(np.unique(np.concatenate(parts)).astype(np.int64))
    return out, vert.astype(np.int64), diag.astype(np.int64)


# ---------------------------------------------------------------------------
# Per-head index construction.
# ---------------------------------------------------------------------------
@dataclass
class HeadIndex:
    """Indices of one q-head.  ``blocks[qb]`` and ``cols[qb]`` are ascending int64
    arrays.  For VS heads ``blocks`` is derived from ``D``; the raw verticals V,
    slashes S and their fp64 scores are kept for tie-aware comparisons."""
    kind: str
    B: int
    N: int
    blocks: list = field(default_factory=list)
    cols: list = field(default_factory=list)
    sink: int = 0
    window: int = 0
    D: np.ndarray | None = None
    V: np.ndarray | None = None
    S: np.ndarray | None = None
    vscore: np.ndarray | None = None
    sscore: np.ndarray | None = None
    block_scores: np.ndarray | None = None   # [nqb, nkb] logits (block kinds)
    vert_blocks: np.ndarray | None = None    # unified: kept vertical key blocks
    diag_blocks: np.ndarray | None = None    # unified: kept diagonal block distances
    runs: list | None = None   # VS with slash_cover "windows": [n, 2] key runs per query block


def build_head_index(Qh, Kh, pattern: dict, B: int, conv=None) -> HeadIndex:
    """Indices for one q-head with its KV head's keys.

    Qh, Kh: [N, d] float64 (the same bf16 values the GPU reads, widened).
    pattern: {"kind": ..., and the fields of that kind}; conv: (w [d,W], b [d])
    for MoBA key conv, or None."""
    N, d = Kh.shape
    nqb = n_blocks(N, B)
    kind = pattern["kind"]
    if kind == VS_WINDOWS:
        pattern = dict(pattern, kind=VS, slash_cover="windows")
        kind = VS
    hi = HeadIndex(kind=kind, B=B, N=N)
    empty = np.zeros(0, np.int64)
    if kind == ASHAPE:
        hi.sink, hi.window = int(pattern["sink"]), int(pattern["window"])
        hi.blocks = [ashape_blocks(qb, B, N, hi.sink, hi.window) for qb in range(nqb)]
        hi.cols = [empty] * nqb
    elif kind == VS:
        v, s = vs_estimate(Qh, Kh, int(pattern["last_q"]))
        hi.vscore, hi.sscore = v, s
        hi.V = topk_indices(v, int(pattern["n_vert"]))
        hi.S = topk_indices(s, int(pattern["n_slash"]))
        cover = pattern.get("slash_cover", "blocks")
        if cover == "blocks":
            hi.D = vs_distance_set(hi.S, B, nqb)
            hi.blocks = [np.sort(qb - hi.D[hi.D <= qb]) for qb in range(nqb)]
            hi.cols = [vs_columns(hi.V, hi.D, qb, B) for qb in range(nqb)]
        elif cover == "windows":
            hi.runs = [vs_slash_runs(hi.S, qb, B, N) for qb in range(nqb)]
            hi.blocks = [empty] * nqb
            hi.cols = [vs_window_columns(hi.V, hi.runs[qb], qb, B) for qb in range(nqb)]
        else:
            raise ValueError(f"unknown slash_cover {cover!r}")
    elif kind == UNIFIED:
        sc = block_logits(mean_pool(Qh, B), mean_pool(Kh, B), d)
        hi.block_scores = sc
        hi.blocks, hi.vert_blocks, hi.diag_blocks = select_unified(
            sc, float(pattern["alpha"]), bool(pattern.get("keep_sink", 1)), bool(pattern.get("keep_local", 1)))
        hi.cols = [empty] * nqb
    elif kind in (BLOCK_TOPK, BLOCK_THRESHOLD, MOBA):
        keys = Kh
        if kind == MOBA and conv is not None:
            keys = key_conv(Kh, conv[0], conv[1])
        sc = block_logits(mean_pool(Qh, B), mean_pool(keys, B), d)
        hi.block_scores = sc
        blocks = []
        for I in range(nqb):
            if kind == BLOCK_TOPK:
                blocks.append(select_block_topk(sc[I], I, int(pattern["topk"])))
            elif kind == MOBA:
                blocks.append(select_moba(sc[I], I, int(pattern["topk"])))
            else:
                blocks.append(select_threshold(sc[I], I, float(pattern["alpha"]),
                                               bool(pattern.get("keep_sink", 1)),
                                               bool(pattern.get("keep_local", 1))))
        hi.blocks = blocks
        hi.cols = [empty] * nqb
    else:
        raise ValueError(f"unknown pattern kind {kind!r}")
    return hi


# ---------------------------------------------------------------------------
# Attention given indices  [MIa]: attention over the index lists of each head's
# pattern; [FP] 2.3 (only listed blocks are visited).
# ---------------------------------------------------------------------------
def allowed_keys(hi: HeadIndex, i: int) -> np.ndarray:
    """The index mask of row i as a sorted set of key positions: keys of the
    listed blocks, slash runs and columns of row i's query block, restricted to j <= i
    (and to the A-shape predicate for A-shape heads).  A key listed twice is one
    key."""
    B = hi.B
    qb = i // B
    blk = np.asarray(hi.blocks[qb], dtype=np.int64)
    from_blocks = (blk[:, None] * B + np.arange(B)[None, :]).ravel() if blk.size else np.zeros(0, np.int64)
    keys = np.union1d(from_blocks, np.asarray(hi.cols[qb], dtype=np.int64))
    if hi.runs is not None and hi.runs[qb].size:
        keys = np.union1d(keys, np.concatenate([np.arange(a, b + 1) for a, b in hi.runs[qb]]))
    keys = keys[(keys <= i) & (keys < hi.N)]
    if hi.kind == ASHAPE:
        keys = keys[ashape_allowed(i, keys, hi.sink, hi.window)]
    return keys


def attention_rows(Qh, Kh, Vh, hi: HeadIndex, rows):
    """Masked softmax attention for the given rows of one head, in float64.

    O_i = sum_{j allowed} exp(l_ij - m_i) v_j / sum_{j allowed} exp(l_ij - m_i),
    l_ij = tau q_i.k_j, LSE_i = m_i + ln(sum exp(l_ij - m_i)).  Rows with no
    allowed key give O_i = 0 and LSE_i = -inf."""
    N, d = Kh.shape
    tau = 1.0 / math.sqrt(d)
    rows = np.asarray(rows, dtype=np.int64)
    O = np.zeros((rows.size, Vh.shape[1]))
    lse = np.full(rows.size, -np.inf)
    for r, i in enumerate(rows):
        J = allowed_keys(hi, int(i))
        if J.size == 0:
            continue
        logits = tau * (Kh[J] @ Qh[i])
        m = logits.max()
        w = np.exp(logits - m)
        O[r] = (w @ Vh[J]) / w.sum()
        lse[r] = m + math.log(w.sum())
    return O, lse


def index_mask_dense(hi: HeadIndex) -> np.ndarray:
    """The whole N x N boolean index mask (tiny N only)."""
    M = np.zeros((hi.N, hi.N), dtype=bool)
    for i in range(hi.N):
        M[i, allowed_keys(hi, i)] = True
    return M


def dense_causal_attention(Qh, Kh, Vh):
    """Textbook dense causal softmax attention in float64 (for the all-blocks
    equivalence): O = softmax(tau Q K^T with j > i masked) V."""
    N, d = Kh.shape
    L = (Qh @ Kh.T) / math.sqrt(d)
    L[np.triu_indices(N, 1)] = -np.inf
    m = L.max(axis=1, keepdims=True)
    W = np.exp(L - m)
    lse = m[:, 0] + np.log(W.sum(axis=1))
    return (W @ Vh) / W.sum(axis=1, keepdims=True), lse


# ---------------------------------------------------------------------------
# Whole layer.
# ---------------------------------------------------------------------------
def build_indices(Q, K, patterns, B, convs=None):
    """Q [Hq, N, d], K [Hkv, N, d] float64; patterns: list of Hq dicts; convs:
    optional list (per q-head) of (w, b) or None.  Returns a list of HeadIndex."""
    Hq, Hkv = Q.shape[0], K.shape[0]
    G = Hq // Hkv
    out = []
    for h in range(Hq):
        conv = convs[h] if convs is not None else None
        out.append(build_head_index(Q[h], K[h // G], patterns[h], B, conv))
    return out


def sparse_attention(Q, K, V, heads, rows=None):
    """O [Hq, len(rows), d] and LSE [Hq, len(rows)] for the given rows (default all)."""
    Hq, N, d = Q.shape
    G = Hq // K.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    O = np.zeros((Hq, rows.size, V.shape[2]))
    lse = np.zeros((Hq, rows.size))
    for h in range(Hq):
        O[h], lse[h] = attention_rows(Q[h], K[h // G], V[h // G], heads[h], rows)
    return O, lse


def selected_pairs(hi: HeadIndex) -> int:
    """|M| of one head: the number of allowed (i, j) pairs of the index mask,
    counted exactly from the block and column lists (used for F_sel = 4 d |M|)."""
    total = 0
    for i in range(hi.N):
        total += allowed_keys(hi, i).size
    return total


def selected_pairs_by_block(hi: HeadIndex) -> int:
    """|M| of one head counted one query block at a time (fast enough for
    full-length layers).  The keys a query block lists (its blocks' keys, its
    slash runs and its columns, as a set) are the same for every row of the
    block; row i keeps those with j <= i, found by a binary search in the sorted
    set, and for A-shape heads only those with j < sink or i - j < window
    ([MI] "3つの疎パターン": sink tokens plus a local window), counted as
    |{j < sink}| + |{j > i - window}| - |{both}| among the keys j <= i."""
    B, N = hi.B, hi.N
    total = 0
    for qb in range(n_blocks(N, B)):
        blk = np.asarray(hi.blocks[qb], dtype=np.int64)
        parts = [(blk[:, None] * B + np.arange(B)[None, :]).ravel(), np.asarray(hi.cols[qb], dtype=np.int64)]
        if hi.runs is not None and hi.runs[qb].size:
            parts += [np.arange(a, b + 1) for a, b in hi.runs[qb]]
        keys = np.unique(np.concatenate(parts))
        keys = keys[keys < N]
        rows = np.arange(qb * B, min(N, qb * B + B), dtype=np.int64)
        upto_i = np.searchsorted(keys, rows, side="right")          # keys j <= i
        if hi.kind != ASHAPE:
            total += int(upto_i.sum())
            continue
        sink_n = np.searchsorted(keys, np.minimum(rows + 1, hi.sink), side="left")   # j <= i, j < sink
        win_lo = rows - hi.window + 1                                               # window: j >= i - window + 1
        win_n = upto_i - np.searchsorted(keys, win_lo, side="left")
        both_hi = np.minimum(rows + 1, hi.sink)                                      # j < min(i + 1, sink)
        both_n = (np.searchsorted(keys, both_hi, side="left")                         # ... and j >= i - window + 1
                  - np.searchsorted(keys, np.minimum(win_lo, both_hi), side="left"))
        total += int((sink_n + win_n - both_n).sum())
    return total
