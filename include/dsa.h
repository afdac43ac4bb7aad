/*
 * dsa.h -- C ABI of the B200 dynamic sparse attention prefill library (libdsa.so).
 *
 * The library does the two steps of dynamic sparse attention for long-context
 * prefill:
 *
 *   dsa_build_indices : per-head sparse indices from Q and K, following the head's
 *                       pattern (A-shape, Vertical-Slash, block top-k, block
 *                       threshold, MoBA routing);
 *   dsa_sparse_prefill: causal FlashAttention-style forward pass over only the
 *                       listed key blocks and key columns.
 *
 * The two calls follow the MInference abstract (zhuanzhiai.com page): a head's
 * pattern is fixed ahead of time, its index lists are built from that pattern
 * when the layer runs, and attention then reads only those lists.  Pattern
 * definitions:
 *   - A-shape, Vertical-Slash, block-sparse: "MInference 1.0" summary (abeam.tech),
 *     sections "3つの疎パターン" and "推論時は軽い近似で動的マスクを作る";
 *   - max-relative block threshold: "FlashPrefill" summary (gist.science), section
 *     2.2, thresh_I = alpha * max_{J<=I} Score_{I,J}, with the mean-pooled key of
 *     section 2.1;
 *   - MoBA routing and the key convolution: "Optimizing Mixture of Block Attention"
 *     summary (lifetechia.com), sections on block routing and "2. キーに対する畳み込み適用".
 *
 * Conventions for every call:
 *   - Every pointer marked "device" is CUDA device memory owned by the caller; the
 *     library allocates nothing, frees nothing and never synchronises, except
 *     dsa_get_device_status, which synchronises the given stream.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and is asynchronous to the host.
 *   - Arguments are validated on the host before any launch; an invalid call
 *     returns an error code and enqueues nothing.  No call throws or aborts.
 *   - Errors a kernel finds (an index list longer than its capacity, an index out
 *     of range, a malformed list, a bounded wait that ran out) are recorded in the
 *     status word of the call's stream and reported by dsa_get_device_status.
 *   - Batch size is one sequence.  Heads are independent.
 *   - Numerics: bf16 Q/K/V/O, tensor-core products with fp32 accumulation, fp32
 *     softmax and scores; P is rounded to bf16 before the P.V product.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dsa_stream; /* same type as cudaStream_t */

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,  /* bad shape, stride, alignment, null pointer, or pattern field */
    DSA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement (e.g. d not 64/128) */
    DSA_ERR_CAPACITY = 3,     /* an output list or workspace is smaller than required */
    DSA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed; see dsa_last_cuda_error */
    DSA_ERR_TIMEOUT = 5,      /* a kernel's bounded wait ran out (reported by the device) */
    DSA_ERR_DEVICE = 6        /* a kernel found an inconsistent index (reported by the device) */
} dsa_status;

typedef enum dsa_kind {
    DSA_KIND_ASHAPE = 0,          /* sink + local window, fixed mask */
    DSA_KIND_VS = 1,              /* Vertical-Slash, estimated from the last last_q queries */
    DSA_KIND_BLOCK_TOPK = 2,      /* MInference block-sparse: top-k pooled block scores, J <= I */
    DSA_KIND_BLOCK_THRESHOLD = 3, /* FlashPrefill: P_IJ >= alpha * max_J P_IJ, plus sink/local */
    DSA_KIND_MOBA = 4,            /* MoBA: top-k over J < I plus the own block I */
    DSA_KIND_UNIFIED = 5,         /* FlashPrefill discovery: vertical, diagonal and block
                                     shapes at once from the pooled block scores */
    DSA_KIND_VS_WINDOWS = 6       /* Vertical-Slash whose slashes are covered by their exact
                                     key runs per query block instead of aligned blocks */
} dsa_kind;

/*
 * One attention layer of one sequence.  Q has Hq heads, K and V have Hkv heads
 * (Hq a multiple of Hkv; q-head h reads KV head h / (Hq/Hkv)).  N tokens, head
 * dimension d in {64, 128}.  `block` is the block size B of both query and key
 * blocks, in {64, 128, 256, 512}; nqb = nkb = ceil(N / B).
 * Strides are in elements; the last (d) dimension must be contiguous.  Token and
 * head strides of Q/K/V must be multiples of 8 elements and all base pointers
 * 16-byte aligned (TMA requirement).  [H, N, d] and [N, H, d] layouts both work.
 */
typedef struct dsa_problem {
    int32_t Hq, Hkv, N, d, block;
    int32_t reserved;
    int64_t q_head_stride, q_token_stride;
    int64_t k_head_stride, k_token_stride;
    int64_t v_head_stride, v_token_stride;
    int64_t o_head_stride, o_token_stride;
} dsa_problem;

/*
 * Pattern of one q-head.  Only the fields of its kind are read.
 *   ASHAPE:          sink >= 0, window >= 1.  Row i sees j <= i with j < sink or i - j < window.
 *   VS:              last_q >= 1, n_vert >= 0, n_slash >= 0 (counts of the top-k vertical
 *                    columns and slash offsets; clipped to N).
 *   BLOCK_TOPK:      topk >= 1 (blocks per query block among J <= I).
 *   BLOCK_THRESHOLD: 0 < alpha <= 1, in probability space; keep_sink / keep_local
 *                    force blocks 0 and I.
 *   UNIFIED:         0 < alpha <= 1; keep_sink / keep_local as for BLOCK_THRESHOLD.  From
 *                    the pooled block scores s_IJ (J <= I) and their row softmax P_IJ:
 *                    vertical sums V_J = sum_I P_IJ, diagonal sums G_d = sum_I P_{I,I-d};
 *                    query block I keeps {J : P_IJ >= alpha max_J P_IJ}, the verticals
 *                    J <= I with V_J >= alpha max V, and the blocks I - d of the
 *                    diagonals d <= I with G_d >= alpha max G ("FlashPrefill" summary,
 *                    sections 2.1 and 2.2, the max-based threshold applied per shape).
 *                    The kept verticals and diagonals are written to vert_idx / slash_idx.
 *   Block kinds (BLOCK_TOPK, BLOCK_THRESHOLD, MOBA, UNIFIED) need nqb = ceil(N / block) <= 2048
 *   (DSA_ERR_UNSUPPORTED otherwise).
 *   MOBA:            topk >= 0 past blocks (J < I) plus the own block I.  Optional
 *                    causal depthwise key conv for routing: conv_width in [0, 8]
 *                    (0 = off); conv_weight: device float [d][conv_width] (tap t
 *                    multiplies k[j - t]); conv_bias: device float [d].  All
 *                    block-kind heads of one KV group must use the same conv
 *                    (same width and pointers).
 */
typedef struct dsa_pattern {
    int32_t kind;
    int32_t sink, window;
    int32_t last_q, n_vert, n_slash;
    int32_t topk;
    float alpha;
    int32_t keep_sink, keep_local;
    int32_t conv_width;
    int32_t reserved;
    const float* conv_weight;
    const float* conv_bias;
} dsa_pattern;

/*
 * Index lists, all device memory owned by the caller, sized from dsa_sizes.
 * Rows of the CSR arrays are r = h * nqb + qb.  All lists are strictly ascending
 * (no entry repeats within one list).  dsa_sparse_prefill checks every row
 * against the capacities (0 <= ptr[r] <= ptr[r+1] <= cap) and every entry
 * against its range; a malformed row or entry is skipped and reported as
 * DSA_ERR_DEVICE by dsa_get_device_status.
 *   head_info [Hq * 4]          : kind, sink, window, 0 for each head.
 *   blk_ptr   [Hq * nqb + 1]    : key blocks of (h, qb) are blk_idx[blk_ptr[r] .. blk_ptr[r+1]).
 *   blk_idx   [blk_cap]         : (empty for VS heads, whose blocks come from dist)
 *   dist_ptr  [Hq + 1]          : VS block distances of head h are dist[dist_ptr[h] .. dist_ptr[h+1]);
 *   dist      [dist_cap]          query block qb keeps key blocks qb - delta for delta <= qb.
 *   col_ptr   [Hq * nqb + 1]    : VS key columns of (h, qb) are col_idx[col_ptr[r] .. col_ptr[r+1]),
 *   col_idx   [col_cap]           none of them inside a block the row already keeps.
 *   vert_idx  [Hq * vert_stride]: chosen vertical columns of VS heads, vertical key blocks of
 *                                 UNIFIED heads (ascending, -1 padded).
 *   slash_idx [Hq * slash_stride]: chosen slash offsets o = i - j of VS heads, diagonal block
 *                                 distances d of UNIFIED heads (ascending, -1 padded).
 * VS_WINDOWS heads keep no blocks; their dist row is the slash-run list
 *   [n, n_last, a_0, b_0, ..., a_{n-1}, b_{n-1}, then n_last pairs]: the merged offset
 *   intervals [a, b] of the chosen slashes dilated by the block height (the first
 *   n for full blocks, the last n_last for a shorter last block); query block qb
 *   (last row r1) keeps the key runs [max(0, r1 - b), r1 - a].  Their columns lie
 *   outside those runs.
 * kinds_present: bit k set when some head has kind k.  dsa_sparse_prefill reads it
 *   to choose its kernel (column tiles only when bit 1 or bit 6 is set, slash-run
 *   masks only when bit 6 is: a VS head met without bit 1, or a VS_WINDOWS head
 *   without bit 6, is reported as DSA_ERR_DEVICE and left empty);
 *   dsa_build_indices does not read it.
 * dsa_sparse_prefill reads only head_info, blk_*, dist*, col_*, kinds_present.
 */
typedef struct dsa_indices {
    int32_t* head_info;
    int32_t* blk_ptr;
    int32_t* blk_idx;
    int32_t* dist_ptr;
    int32_t* dist;
    int32_t* col_ptr;
    int32_t* col_idx;
    int32_t* vert_idx;
    int32_t* slash_idx;
    int64_t blk_cap, dist_cap, col_cap;
    int32_t vert_stride, slash_stride;
    int32_t kinds_present;  /* bit k set when some head has kind k (dsa_kind) */
    int32_t reserved;
} dsa_indices;

/* Sizes for one (problem, patterns) pair: element counts of every index array
 * (upper bounds for the lists) and the bytes of scratch workspace that
 * dsa_build_indices needs. */
typedef struct dsa_sizes {
    int32_t nqb;
    int32_t vert_stride, slash_stride;
    int32_t reserved;
    int64_t head_info_len, blk_ptr_len, blk_cap, dist_ptr_len, dist_cap, col_ptr_len, col_cap;
    int64_t workspace_bytes;
} dsa_sizes;

/* Pure host.  Validates the problem and the Hq patterns and fills *out.
 * Returns DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED on a bad request. */
dsa_status dsa_workspace_size(const dsa_problem* p, const dsa_pattern* pats, dsa_sizes* out);

/* Builds the index lists of every head from its pattern, at run time (the
 * MInference abstract's second step).  Q, K: device bf16 with the problem's
 * strides.  pats: host array [Hq].  out: index arrays with capacities at least those
 * of dsa_workspace_size.  workspace: device scratch of at least
 * sizes.workspace_bytes (256-byte aligned); its contents on entry do not matter.
 * Enqueues kernels on `stream`; returns DSA_ERR_CAPACITY if a capacity or the
 * workspace is too small. */
dsa_status dsa_build_indices(const dsa_problem* p, const void* Q, const void* K,
                             const dsa_pattern* pats, const dsa_indices* out,
                             void* workspace, size_t workspace_bytes, dsa_stream stream);

/* Sparse attention forward (MInference abstract: attention over each head's index
 * lists only; FlashPrefill section 2.3: only listed blocks are visited).
 * Row i of head h attends to key j iff j <= i and (j is in a listed block of its
 * query block, or j is a listed column), and for A-shape heads also
 * (j < sink or i - j < window).  A key listed twice counts once.
 * O: device bf16 written with the problem's o strides.  lse: optional device float
 * [Hq * N] (natural log; -inf for a row with no allowed key, whose O row is 0).
 * The indices may come from dsa_build_indices or from any other source that
 * follows the layout above. */
dsa_status dsa_sparse_prefill(const dsa_problem* p, const void* Q, const void* K,
                              const void* V, const dsa_indices* idx, void* O, float* lse,
                              dsa_stream stream);

/* Counts the allowed (i, j) pairs of each head's index mask, exactly (the
 * selected-work measure: FLOPs = 4 * d * pairs).  pairs: device int64 [Hq],
 * overwritten. */
dsa_status dsa_count_pairs(const dsa_problem* p, const dsa_indices* idx, int64_t* pairs,
                           dsa_stream stream);

/* Synchronises `stream`, then returns and clears the status word that work
 * enqueued on `stream` reports into on the current device: DSA_OK,
 * DSA_ERR_CAPACITY, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE (or DSA_ERR_CUDA if the
 * synchronisation itself failed).  detail (nullable) receives a kernel-specific
 * code: which list overflowed, which wait ran out, or which list was malformed.
 * Each device has 64 status words; a stream's word is chosen by hashing its
 * handle, so streams whose handles fall on the same word share it (an error of
 * one is then reported to a caller of the other).  The first error recorded in a
 * word is kept until this call clears it. */
dsa_status dsa_get_device_status(dsa_stream stream, int32_t* detail);

/* Self-test of the bounded-wait path: one CTA waits on a barrier that nothing
 * will ever complete, with a limit of timeout_us microseconds, then records
 * DSA_ERR_TIMEOUT in the status word and exits normally.  Lets a test check the
 * timeout reporting without faulting or hanging the GPU. */
dsa_status dsa_selftest_wait_timeout(uint32_t timeout_us, dsa_stream stream);

/* dsa_build_indices without a workspace argument, for callers that cannot
 * allocate device memory (a plugin inside another runtime that owns all device
 * memory, or a latency-critical path where cudaMalloc would synchronise the
 * device).  The pages have no counterpart: this is a deployment variant of the
 * same index builder, with identical results.
 * Scratch comes from a 16 MiB buffer compiled into the library: every GPU that
 * loads the library holds it until the process exits.  A problem whose
 * sizes.workspace_bytes exceeds 16 MiB returns DSA_ERR_CAPACITY and enqueues
 * nothing.  The library allocates and frees nothing in this call.
 * The first call on a device (with that device current) looks up the buffer's
 * device address; make that first call before any stream capture.
 * All calls on a device share the buffer and it keeps the previous call's
 * contents (the builder clears what it needs zeroed); calls whose work overlaps
 * on the GPU race on it, so order them (one stream, or events). */
dsa_status dsa_build_indices_static(const dsa_problem* p, const void* Q, const void* K,
                                    const dsa_pattern* pats, const dsa_indices* out,
                                    dsa_stream stream);

/* Sets the bound, in nanoseconds of GPU global time, on every in-kernel wait of
 * the launches that follow, on every device of this process (0 restores the
 * default of 4 s; more than 60 s is DSA_ERR_INVALID_ARG).  A wait that runs out
 * records DSA_ERR_TIMEOUT and its CTA stops its work and exits cleanly; after a
 * timeout the output of that launch is incomplete.  A diagnostic: a short bound
 * makes the abort path reachable without any fault. */
dsa_status dsa_set_wait_limit(uint64_t limit_ns);

/* Static description of a status code. */
const char* dsa_status_string(dsa_status s);

/* The cudaError_t value of the last DSA_ERR_CUDA on this thread (0 if none). */
int32_t dsa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
