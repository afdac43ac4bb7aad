// Causal block-sparse attention forward for sm_100a.
//
// What it computes (MInference abstract: attention restricted to the index lists
// built for each head's pattern; FlashPrefill section 2.3: the kernel jumps straight to the
// listed blocks instead of testing every block): for row i of head h,
//   O_i = sum_{j in M_i} softmax_j(tau q_i.k_j) v_j,
// where M_i holds the keys j <= i of the key blocks listed for i's query block
// (CSR blocks, or qb - delta for the VS distances), plus its listed columns, and
// for A-shape heads only those with j < sink or i - j < window.
//
// Design (persistent: two CTAs per SM; a work item = 128 query rows of one head,
// items handed out by a global counter, latest (heaviest) query tiles first):
//   * the tile's two 64-row halves each belong to one query block (two different
//     blocks when B = 64, the same block otherwise).  Their key lists become two
//     bitmaps over 64-key units in shared memory; the union is walked in
//     ascending order, one unit (64 keys) per KV tile, each unit flagged with the
//     halves that listed it (the other half masks it out);
//   * column lists are gathered into dense 64-key tiles (gather-and-densify); a
//     column inside a block the half already keeps is masked out;
//   * slash runs of VS_WINDOWS heads (exact key runs per query block) join the
//     unit bitmaps: every unit a run touches, carrying each half's run keys as
//     a 64-bit mask;
//   * three instantiations, chosen from the index's kinds_present: block kinds
//     only (no column code), with column tiles, with column tiles and run masks
//     (the smaller code keeps short items out of instruction-cache misses);
//   * warps 2-3 (decoders) fetch items, turn an item's lists into bitmap set
//     (item & 1) up to one item ahead, publish it, and gather its column rows;
//     warp 0 (one thread) loads each item's Q and issues the TMA loads
//     (SWIZZLE_128B boxes of 64 x 64) of its key units into two K and two V
//     buffers; tiles are issued strictly in order (units, then columns, item by
//     item), which keeps every empty-buffer parity wait unambiguous; warp 1 (one
//     thread) issues each tile's tcgen05.mma from one asm block; warps 4-7 run the
//     online softmax (one thread per row) and the epilogue.  Tile and item
//     counters run across items, so every barrier keeps its phase from one item
//     to the next;
//   * TMEM (256 columns per CTA): O at [0, 128), two S buffers of 64 columns at
//     128 and 192.  S(t+1) = Q K(t+1)^T is computed while the softmax works on
//     S(t); the softmax writes P(t) as bf16 pairs over the first 32 columns of its
//     S buffer and O += P(t) V(t) reads it from there; S(t+2) is issued right
//     after that P.V (one thread's MMAs run in order);
//   * the running max is only raised when it grows by more than 2^32; only then
//     does the softmax wait for the previous P.V and rescale O, so in the common
//     case the softmax of one tile overlaps the P.V of the one before;
//   * ~100 KB of shared memory and 256 TMEM columns per CTA let two CTAs share an
//     SM, so one CTA's softmax also overlaps the other's tensor-core work.
// No cluster, no multicast; every wait is bounded (status word + early exit).
#include <cudaTypedefs.h>

#include <atomic>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int BM = 128;            // query rows per CTA
constexpr int UNIT = 64;           // keys per KV tile (one TMA box of rows)
constexpr int BN = UNIT;
constexpr int QSLAB = 128 * 128;   // bytes of one 128-row x 64-column bf16 slab (Q)
constexpr int KSLAB = 64 * 128;    // bytes of one 64-row x 64-column bf16 slab (K, V)
constexpr int NTHREADS = 256;      // warps 0,2,3 load, warp 1 issues MMAs, warps 4-7 softmax
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t S_COL = 128;    // S buffer b at S_COL + 64 b
constexpr int NINFO = 4;           // StageInfo slots (a slot is reused after its softmax ended)
// log2 units.  Scaling every P of a row by one power of two changes no rounding
// (fp32 and bf16 are relative), so a running max that lags the true one is exact
// after the final division; 2^32 leaves P <= 2^32, l and O <= 2^53 |V| for 2^21
// keys, far inside fp32 range, and avoids almost every O rescale.
constexpr float RESCALE_THRESHOLD = 32.0f;
// Waits of the TMA producer and of the MMA thread block in try_wait (the warp
// then takes no issue slots from the softmax warp that shares its scheduler)
// instead of polling.
constexpr bool kLoaderSuspend = true;
constexpr bool kMmaSuspend = true;

struct StageInfo {
  int type;   // 0 = key unit, 1 = column tile, 3 = key unit of slash runs
  int u;      // unit id (types 0 and 3)
  int flags;  // bit h: half h of the rows uses this tile
  int ncols;  // valid columns (type 1)
  uint32_t m[4];  // type 3: the unit's keys inside half h's runs, bits m[2h] | m[2h + 1] << 32
};

struct ItemInfo {
  int h, qt, kind, sink, window, T;  // T: KV tiles of the item
};

// An item as the decoder warps hand it to the TMA producer and to themselves
// (column gathering): bitmap set item & 1 holds its key units.
struct DecInfo {
  int item;    // -1: no more items
  int h, qt, kvh;
  int T_u, T;  // unit tiles, all tiles
  int tg;      // tiles of this CTA's earlier items
  int flags1;  // halves that use half 0's column tiles (3 when both halves share a query block)
  int cc[2], cb[2];  // column count / first column of each half
  // slash runs (VS_WINDOWS heads): per half, the interval list of its query
  // block's height (an index into dist), its length and the block's last row
  int wins;  // the item's head is VS_WINDOWS: its units carry run masks
  int rbeg[2], rn[2], rr1[2];
};

struct AttnArgs {
  int Hq, G, N, B, nqb, n_qtiles, n_units, nwords;
  const int32_t* head_info;
  const int32_t* blk_ptr;
  const int32_t* blk_idx;
  const int32_t* dist_ptr;
  const int32_t* dist;
  const int32_t* col_ptr;
  const int32_t* col_idx;
  int64_t blk_cap, dist_cap, col_cap;  // lengths of blk_idx, dist, col_idx
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t k_hs, k_ts, v_hs, v_ts;
  __nv_bfloat16* O;
  int64_t o_hs, o_ts;
  int o_v8;  // O rows are 32-byte aligned: 256-bit stores
  float* lse;
  float scale_log2;
  unsigned long long* sched;  // item counter: launch epoch (high 32 bits), items handed out (low 32)
  unsigned epoch;             // this launch's epoch (never 0)
  unsigned* status;
  uint64_t wait_limit_ns;
};

template <int D>
struct Smem {
  static constexpr int DS = D / 64;  // 64-column slabs
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + DS * QSLAB;         // [2 buffers][DS slabs]
  static constexpr int V_OFF = K_OFF + 2 * DS * KSLAB;
  static constexpr int COL_OFF = V_OFF + 2 * DS * KSLAB;   // int [NINFO][BN]
  static constexpr int INFO_OFF = COL_OFF + NINFO * BN * 4;
  static constexpr int ITEM_OFF = INFO_OFF + NINFO * (int)sizeof(StageInfo);
  static constexpr int DEC_OFF = ITEM_OFF + 2 * (int)sizeof(ItemInfo);
  static constexpr int BAR_OFF = (DEC_OFF + 2 * (int)sizeof(DecInfo) + 7) & ~7;
  static constexpr int NBAR = 29;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BITS_OFF = MISC_OFF + 64;
  // two bitmap sets (items kc and kc + 1), each two halves of nwords words
  static int bytes(int nwords) { return BITS_OFF + 4 * nwords * 4 + 1024; }
};

// Barrier slots.  Per-buffer barriers (K, V, S, P) complete once per use of their
// buffer, i.e. once per two tiles; B_ODONE completes once per P.V in order; Q
// and O barriers once per item; B_INFO + s when StageInfo slot s (and its column
// list) is written; B_ITEMFULL / B_ITEMFREE + s guard ItemInfo slot s.
enum {
  B_QFULL = 0,
  B_QEMPTY = 1,
  B_KFULL = 2,     // +2
  B_KEMPTY = 4,    // +2
  B_VFULL = 6,     // +2
  B_VEMPTY = 8,    // +2
  B_SFULL = 10,    // +2
  B_PFULL = 12,    // +2
  B_ODONE = 14,
  B_OREADY = 15,
  B_DRAIN = 16,
  B_ITEMFULL = 17,  // +2
  B_ITEMFREE = 19,  // +2
  B_INFO = 21,      // +NINFO
  B_DECFULL = 25,   // +2: bitmap set s and DecInfo s written
  B_UNITS = 27,     // once per item: the producer has issued the item's unit tiles
  B_COLS = 28       // once per item: the gatherers have filled the item's column tiles
};
static_assert(B_COLS + 1 <= 29, "barrier slots");

// One lane waits, the whole warp learns the outcome (keeps warp-collective
// tcgen05 and shuffle instructions converged even when a wait runs out).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit, unsigned* status,
                                          unsigned detail, volatile int* abort_flag) {
  // fast path: every lane probes once, no broadcast needed
  if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, limit, status, detail, abort_flag) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // byte offset inside a slab
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (x0, x1) = (a0, a1) * b + c with one packed f32x2 fused multiply-add
__device__ __forceinline__ void fma2(float a0, float a1, float b, float c, float& x0, float& x1) {
  uint64_t av, bv, cv, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(av) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(bv) : "f"(b), "f"(b));
  asm("mov.b64 %0, {%1, %2};" : "=l"(cv) : "f"(c), "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(av), "l"(bv), "l"(cv));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(r));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// (s0, s1) += (a, b) as one packed f32x2 add
__device__ __forceinline__ void add2(float& s0, float& s1, float a, float b) {
  uint64_t sv, av;
  asm("mov.b64 %0, {%1, %2};" : "=l"(sv) : "f"(s0), "f"(s1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(av) : "f"(a), "f"(b));
  asm("add.rn.f32x2 %0, %0, %1;" : "+l"(sv) : "l"(av));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(s0), "=f"(s1) : "l"(sv));
}

// 32 bytes to global memory in one store (address 32-byte aligned)
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ uint32_t low_bits(int n) {  // n clamped to [0, 32]
  return n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u));
}

// The MMAs of one tile, issued from one asm block (predicates set once; the
// descriptors advance from a base by constant address offsets, the address
// field being bits 0-13 of the descriptor in 16-byte units, which never carries
// for shared-memory addresses below 256 KB).
//   S = Q K^T: NK k-steps of 16 over the head dimension, accumulating after the first.
template <int NK>
__device__ __forceinline__ void mma_qk_tile(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc) {
  static_assert(NK == 4 || NK == 8, "head dimension 64 or 128");
  // k-step kk: 64-column slab kk >> 2 (QSLAB / KSLAB bytes apart), 32 bytes per step inside it
  constexpr uint64_t QS = QSLAB >> 4, KS = KSLAB >> 4;
  const uint32_t zero = 0;
  if constexpr (NK == 4) {
    asm volatile(
        "{\n\t.reg .pred pf, pt;\n\t"
        "setp.ne.b32 pf, %9, 0;\n\tsetp.eq.b32 pt, %9, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %10, pf;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %10, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %10, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %10, pt;\n\t}" ::"r"(d_tmem),
        "l"(a0), "l"(a0 + 2), "l"(a0 + 4), "l"(a0 + 6), "l"(b0), "l"(b0 + 2), "l"(b0 + 4), "l"(b0 + 6),
        "r"(zero), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred pf, pt;\n\t"
        "setp.ne.b32 pf, %17, 0;\n\tsetp.eq.b32 pt, %17, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %18, pf;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %18, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %18, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %18, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %18, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %18, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %18, pt;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %18, pt;\n\t}" ::"r"(d_tmem),
        "l"(a0), "l"(a0 + 2), "l"(a0 + 4), "l"(a0 + 6), "l"(a0 + QS), "l"(a0 + QS + 2), "l"(a0 + QS + 4),
        "l"(a0 + QS + 6), "l"(b0), "l"(b0 + 2), "l"(b0 + 4), "l"(b0 + 6), "l"(b0 + KS), "l"(b0 + KS + 2),
        "l"(b0 + KS + 4), "l"(b0 + KS + 6), "r"(zero), "r"(idesc)
        : "memory");
  }
}
//   O (+)= P V: four k-steps of 16 keys, P read from TMEM (8 columns of packed
//   bf16 per step), V from shared memory (2048 bytes per step); the first step
//   overwrites O when acc_first is 0.
__device__ __forceinline__ void mma_pv_tile(uint32_t d_tmem, uint32_t p_tmem, uint64_t b0, uint32_t idesc,
                                            uint32_t acc_first) {
  constexpr uint64_t VS = 2048 >> 4;
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t"
      "setp.ne.b32 pf, %9, 0;\n\tsetp.eq.b32 pt, %9, %9;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %10, pf;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %10, pt;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %10, pt;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %10, pt;\n\t}" ::"r"(d_tmem),
      "r"(p_tmem), "r"(p_tmem + 8), "r"(p_tmem + 16), "r"(p_tmem + 24), "l"(b0), "l"(b0 + VS), "l"(b0 + 2 * VS),
      "l"(b0 + 3 * VS), "r"(acc_first), "r"(idesc)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Next item index past the first wave.  The counter word carries the epoch of
// the launch that last used it in its high 32 bits.  A launch that finds another
// epoch there (a word left by an earlier launch, even one that ended early)
// restarts the count at its own epoch: one CTA's compare-and-swap succeeds and
// takes item 0, the others see the new epoch and count on from it.  So no launch
// has to clear the word when it ends, and the common case is one atomic add.
static __device__ __noinline__ int sched_restart(unsigned long long* ctr, unsigned epoch, unsigned long long old) {
  while (true) {
    unsigned long long cur = old + 1ull;
    while ((unsigned)(cur >> 32) != epoch) {
      const unsigned long long prev = atomicCAS(ctr, cur, ((unsigned long long)epoch << 32) | 1ull);
      if (prev == cur) return 0;
      cur = prev;
    }
    old = atomicAdd(ctr, 1ull);
    if ((unsigned)(old >> 32) == epoch) return (int)(unsigned)(old & 0xffffffffull);
  }
}
__device__ __forceinline__ int sched_next(unsigned long long* ctr, unsigned epoch) {
  const unsigned long long old = atomicAdd(ctr, 1ull);
  if ((unsigned)(old >> 32) == epoch) return (int)(unsigned)(old & 0xffffffffull);
  return sched_restart(ctr, epoch, old);  // out of line: once per launch and CTA at most
}

// A CSR row [beg, end) is usable only if 0 <= beg <= end <= cap; otherwise the
// row is reported (DSA_ERR_DEVICE, `detail`) and treated as empty, so a
// malformed list never makes the kernel read outside the caller's arrays.
static __device__ __noinline__ void report_bad_row(unsigned* status, unsigned detail) {
  report(status, DSA_ERR_DEVICE, detail);
}
__device__ __forceinline__ void checked_row(int& beg, int& end, int64_t cap, unsigned* status, unsigned detail) {
  if (!(0 <= beg && beg <= end && (int64_t)end <= cap)) {
    report_bad_row(status, detail);
    beg = 0;
    end = 0;
  }
}

// Waits, bounded by the default limit whatever the launch's own limit and
// ignoring the abort flag, for a TMA load this CTA issued to land.  Used after an
// abort, so that no copy can still be writing into the CTA's shared memory when
// the CTA exits.  A wait that runs out has nothing left to report.
static __device__ __noinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// After an abort, the producer drains its loads still in flight.  The MMA
// thread records how far it has seen K, V and Q land (misc[11], [12], [13]); a
// load it has not seen may still be in flight, and no later phase of that
// buffer's barrier can have completed (filling the buffer again needs the load
// consumed first), so the parity wait is unambiguous.
static __device__ __noinline__ void drain_loads(uint64_t* bars, const int* misc, int q_kc, int pk0, int pk1,
                                                int pv0, int pv1) {
  const volatile int* vm = misc;
  if (q_kc >= 0 && vm[13] <= q_kc) mbar_drain(&bars[B_QFULL], q_kc & 1);
  const int pk[2] = {pk0, pk1}, pv[2] = {pv0, pv1};
  for (int b = 0; b < 2; ++b) {
    if (pk[b] >= 0 && vm[11] <= pk[b]) mbar_drain(&bars[B_KFULL + b], (pk[b] >> 1) & 1);
    if (pv[b] >= 0 && vm[12] <= pv[b]) mbar_drain(&bars[B_VFULL + b], (pv[b] >> 1) & 1);
  }
}

// Slash runs (VS_WINDOWS): offset interval [a, b] of a block whose last row is
// r1 is the key run [max(0, r1 - b), r1 - a]; the intervals ascend, so the runs
// descend in key order.  The bits of keys u0 .. u0 + 63 inside the runs; *c is
// a cursor (start: n - 1) for units visited in ascending order.
__device__ __forceinline__ uint64_t unit_run_mask(const int32_t* iv, int n, int r1, int u0, int* c) {
  int k = *c;
  while (k >= 0 && r1 - iv[2 * k] < u0) --k;  // runs wholly below this unit
  *c = k;
  uint64_t m = 0;
  for (; k >= 0; --k) {
    const int lo = max(0, r1 - iv[2 * k + 1]), hi = r1 - iv[2 * k];
    if (lo > u0 + 63) break;
    const int x = max(lo, u0) - u0, y = min(hi, u0 + 63) - u0;
    if (y < x) continue;
    const uint64_t top = (y == 63) ? ~0ull : ((1ull << (y + 1)) - 1ull);
    m |= top & ~((1ull << x) - 1ull);
  }
  return m;
}

// Key j lies in one of the runs of a list (offset intervals [a_k, b_k],
// ascending, of a block whose last row is r1) iff r1 - j falls in an interval.
__device__ __forceinline__ bool key_in_runs(const int32_t* iv, int n, int r1, int j) {
  const int d = r1 - j;
  int lo = 0, hi = n;  // first interval with a > d
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (iv[2 * mid] <= d) lo = mid + 1; else hi = mid;
  }
  return lo > 0 && d <= iv[2 * (lo - 1) + 1];
}

// RUNS: units with slash-run masks (some head is VS_WINDOWS).  COLS: gathered column tiles
// (some head is VS or VS_WINDOWS); without them the decoders, the gatherers and
// the softmax carry no column code, which keeps the kernel's instruction
// footprint small for layers of block kinds only.
template <int D, bool RUNS, bool COLS>
__global__ void __launch_bounds__(NTHREADS, 2)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  pdl_prologue();
  using L = Smem<D>;
  constexpr int DS = L::DS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR_OFF);
  int* misc = reinterpret_cast<int*>(sm + L::MISC_OFF);
  // misc: [0] tmem base, [2] abort, [3] unit count, [9] decoder go flag, [10] current item,
  //       [11] / [12] K / V tiles the MMA thread has seen land, [13] items whose Q it has seen land
  volatile int* abort_flag = misc + 2;
  uint32_t* bits = reinterpret_cast<uint32_t*>(sm + L::BITS_OFF);  // [set][half][nwords]
  DecInfo* dec = reinterpret_cast<DecInfo*>(sm + L::DEC_OFF);
  StageInfo* info = reinterpret_cast<StageInfo*>(sm + L::INFO_OFF);
  ItemInfo* items = reinterpret_cast<ItemInfo*>(sm + L::ITEM_OFF);
  int* colsm = reinterpret_cast<int*>(sm + L::COL_OFF);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_items = a.n_qtiles * a.Hq;

  // ---------------------------------------------------------------- set-up (once per CTA)
  if (tid == 0) {
    for (int i = 0; i < L::NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == B_PFULL || i == B_PFULL + 1) cnt = 4;
      if (i == B_ITEMFREE || i == B_ITEMFREE + 1) cnt = 5;
      mbar_init(&bars[i], cnt);
    }
    fence_barrier_init();
    misc[2] = 0;
    misc[11] = 0;
    misc[12] = 0;
    misc[13] = 0;
  }
  if (warp == 1) {
    tmem_alloc(reinterpret_cast<uint32_t*>(&misc[0]), TMEM_COLS);
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);
  const uint32_t tmem_O = tmem_base;
  const uint64_t limit = a.wait_limit_ns;
  const int upb = a.B / UNIT;  // units per block

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Q of every item and the TMA loads of its key units, walking the bitmap set
    // that the decoder warps filled (up to one item ahead).
    if (lane == 0) {
      // TMA loads issued whose landing this thread has not seen implied yet: the
      // last Q, and the last K / V tile of each buffer (a later load into the same
      // buffer is only issued once the earlier one has been consumed)
      int q_kc = -1, pk[2] = {-1, -1}, pv[2] = {-1, -1};
      for (int kc = 0;; ++kc) {
        const int s = kc & 1;
        if (!mbar_wait_ool(&bars[B_DECFULL + s], (kc >> 1) & 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag,
                       kLoaderSuspend))
          break;
        const DecInfo di = dec[s];
        if (di.item < 0) break;  // no more items
        // Q once every Q K^T of the previous item has finished
        if (kc > 0 && !mbar_wait_ool(&bars[B_QEMPTY], (kc - 1) & 1, limit, a.status, DETAIL_WAIT_Q, abort_flag,
                                 kLoaderSuspend))
          break;
        mbar_arrive_expect_tx(&bars[B_QFULL], DS * QSLAB);
        q_kc = kc;
        for (int c = 0; c < DS; ++c)
          tma_load_3d(sm + L::Q_OFF + c * QSLAB, &tmQ, &bars[B_QFULL], c * 64, di.qt * BM, di.h);
        // Tiles are issued in order (units, then columns, item by item): a buffer's
        // empty barrier is waited on by parity, which is only unambiguous when the
        // tile two before has been issued.  So the previous item's column tiles
        // come first.
        if (kc > 0 && !mbar_wait_ool(&bars[B_COLS], (kc - 1) & 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag,
                                 kLoaderSuspend))
          break;
        const uint32_t* b0 = bits + s * 2 * a.nwords;
        const uint32_t* b1 = b0 + a.nwords;
        bool ok = true;
        int w = 0;
        uint32_t pend = b0[0] | b1[0];
        int rc[2] = {di.rn[0] - 1, di.rn[1] - 1};  // run cursors (VS_WINDOWS items)
        for (int t = 0; t < di.T_u; ++t) {
          const int g = di.tg + t;
          const int b = g & 1;
          const uint32_t use = (g >> 1) & 1;
          if (!mbar_wait_ool(&bars[B_KEMPTY + b], use ^ 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend)) {
            ok = false;
            break;
          }
          while (pend == 0u && w + 1 < a.nwords) {
            ++w;
            pend = b0[w] | b1[w];
          }
          const int bit = __ffs(pend) - 1;  // T_u counts exactly the set bits
          pend &= pend - 1u;
          const int u = w * 32 + bit;
          StageInfo& si = info[g % NINFO];
          si.type = 0;
          si.u = u;
          si.flags = (int)((b0[w] >> bit) & 1u) | ((int)((b1[w] >> bit) & 1u) << 1);
          si.ncols = 0;
          if constexpr (RUNS) {
            if (di.wins) {
              // the unit's keys inside each half's runs (the softmax masks the rest)
              si.type = 3;
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                uint64_t m = 0;
                if ((si.flags >> hh) & 1)
                  m = unit_run_mask(a.dist + di.rbeg[hh], di.rn[hh], di.rr1[hh], u * UNIT, &rc[hh]);
                si.m[2 * hh] = (uint32_t)m;
                si.m[2 * hh + 1] = (uint32_t)(m >> 32);
              }
            }
          }
          mbar_arrive(&bars[B_INFO + g % NINFO]);
          uint8_t* kst = sm + L::K_OFF + b * DS * KSLAB;
          uint8_t* vst = sm + L::V_OFF + b * DS * KSLAB;
          mbar_arrive_expect_tx(&bars[B_KFULL + b], DS * KSLAB);
          pk[b] = g;
          for (int c = 0; c < DS; ++c) tma_load_3d(kst + c * KSLAB, &tmK, &bars[B_KFULL + b], c * 64, u * UNIT, di.kvh);
          if (!mbar_wait_ool(&bars[B_VEMPTY + b], use ^ 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars[B_VFULL + b], DS * KSLAB);
          pv[b] = g;
          for (int c = 0; c < DS; ++c) tma_load_3d(vst + c * KSLAB, &tmV, &bars[B_VFULL + b], c * 64, u * UNIT, di.kvh);
        }
        if (!ok) break;
        mbar_arrive(&bars[B_UNITS]);  // this item's bitmaps are no longer read here
      }
      if (*abort_flag) drain_loads(bars, misc, q_kc, pk[0], pk[1], pv[0], pv[1]);
    }
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ decoders
    // Work items (query tile, head) are dealt latest (heaviest) tiles first: the
    // first item of a CTA is its block index, later ones come from a global
    // counter (dynamic: items differ a lot in cost).  These two warps turn item
    // kc + 1's lists into bitmap set (kc + 1) & 1 before they gather item kc's
    // column tiles, so the lists of an item are read while the item before it
    // still computes.
    const int dtid = (warp - 2) * 32 + lane;  // 0..63
    int next_item = (int)blockIdx.x;          // held by dtid 0
    int tg_dec = 0;                           // tiles of the items decoded so far
    bool go = true;

    // Decodes item kc of this CTA into bitmap set kc & 1 and publishes it.
    // Returns false when there is no such item (end marker published) or on abort.
    // Set kc & 1 is free: these warps gathered item kc - 2's columns, which they
    // only start once the producer has issued that item's units.
    auto decode = [&](int kc) -> bool {
      const int s = kc & 1;
      if (dtid == 0) {
        misc[10] = next_item;
        next_item = (int)gridDim.x + sched_next(a.sched, a.epoch);  // fetched one item ahead
        misc[3] = 0;
      }
      named_barrier(1, 64);
      const int item = misc[10];
      if (item >= n_items) {
        // no more work: end markers for the producer, the MMA and the softmax warps
        if (dtid == 0) {
          const int slot = kc & 1;
          if (kc < 2 || mbar_wait_ool(&bars[B_ITEMFREE + slot], ((kc >> 1) - 1) & 1, limit, a.status,
                                  DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend)) {
            items[slot].T = -1;
            mbar_arrive(&bars[B_ITEMFULL + slot]);
          }
          dec[s].item = -1;
          mbar_arrive(&bars[B_DECFULL + s]);
        }
        return false;  // the previous item's column tiles are still gathered
      }
      const int h = item % a.Hq;
      const int qt = a.n_qtiles - 1 - item / a.Hq;
      const int row0 = qt * BM;
      const int kind = a.head_info[h * 4 + 0];
      uint32_t* b0 = bits + s * 2 * a.nwords;
      uint32_t* b1 = b0 + a.nwords;
      for (int i = dtid; i < 2 * a.nwords; i += 64) b0[i] = 0u;
      int qbh[2], r1h[2];
      bool live[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r0 = row0 + hh * 64;
        live[hh] = r0 < a.N;
        qbh[hh] = r0 / a.B;
        r1h[hh] = min(a.N - 1, r0 + 63);
      }
      const bool shared_qb = live[1] && (qbh[0] == qbh[1]);
      named_barrier(1, 64);
      if (dtid == 32) {
        // column lists: independent of the block lists, read in parallel with them
        int ce0 = 0, ce1 = 0, cb0 = 0, cb1 = 0;
        if (COLS && live[0]) {
          const int r = h * a.nqb + qbh[0];
          cb0 = a.col_ptr[r];
          ce0 = a.col_ptr[r + 1];
          checked_row(cb0, ce0, a.col_cap, a.status, DETAIL_BAD_COLPTR);
        }
        if (COLS && live[1] && !shared_qb) {
          const int r = h * a.nqb + qbh[1];
          cb1 = a.col_ptr[r];
          ce1 = a.col_ptr[r + 1];
          checked_row(cb1, ce1, a.col_cap, a.status, DETAIL_BAD_COLPTR);
        }
        dec[s].cc[0] = ce0 - cb0;
        dec[s].cc[1] = ce1 - cb1;
        dec[s].cb[0] = cb0;
        dec[s].cb[1] = cb1;
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!live[hh]) continue;
        uint32_t* bb = hh ? b1 : b0;
        const int qb = qbh[hh];
        const int r1 = r1h[hh];
        if (kind == DSA_KIND_VS_WINDOWS) {
          if constexpr (RUNS) {
            // the slash runs of the half's query block: every 64-key unit they
            // touch (up to the half's last row) joins the half's unit bitmap; the
            // producer attaches the run keys of each unit as a mask
            int beg = a.dist_ptr[h], end = a.dist_ptr[h + 1];
            checked_row(beg, end, a.dist_cap, a.status, DETAIL_BAD_DISTPTR);
            int n = 0, nl = 0;
            if (end - beg >= 2) {
              n = a.dist[beg];
              nl = a.dist[beg + 1];
            }
            if (end - beg < 2 || n < 0 || nl < 0 || 2 + 2 * ((int64_t)n + nl) != end - beg) {
              report_bad_row(a.status, DETAIL_BAD_DISTPTR);
              n = nl = 0;
            }
            const bool lastb = qb == a.nqb - 1;
            const int r1b = min(a.N - 1, qb * a.B + a.B - 1);
            const int off = beg + 2 + (lastb ? 2 * n : 0);
            const int m = lastb ? nl : n;
            for (int k = dtid; k < m; k += 64) {
              const int hi = r1b - a.dist[off + 2 * k], lo = max(0, r1b - a.dist[off + 2 * k + 1]);
              if (hi < lo) continue;
              const int uhi = min(hi, r1) / UNIT;
              for (int u = lo / UNIT; u <= uhi; ++u) atomicOr(&bb[u >> 5], 1u << (u & 31));
            }
            if (dtid == 0) {
              dec[s].rbeg[hh] = off;
              dec[s].rn[hh] = m;
              dec[s].rr1[hh] = r1b;
            }
          } else {
            report_bad_row(a.status, DETAIL_BAD_KIND);  // this build's kernel has no run masks
          }
        } else if (kind == DSA_KIND_VS) {
          if constexpr (COLS) {
            int beg = a.dist_ptr[h], end = a.dist_ptr[h + 1];
            checked_row(beg, end, a.dist_cap, a.status, DETAIL_BAD_DISTPTR);
            for (int e = beg + dtid; e < end; e += 64) {
              const int delta = a.dist[e];
              if (delta < 0) { report(a.status, DSA_ERR_DEVICE, DETAIL_BAD_DIST); continue; }
              if (delta > qb) continue;
              const int kb = qb - delta;
              for (int u = kb * upb; u < kb * upb + upb; ++u)
                if (u * UNIT <= r1) atomicOr(&bb[u >> 5], 1u << (u & 31));
            }
          } else {
            report_bad_row(a.status, DETAIL_BAD_KIND);  // this build's kernel has no column tiles
          }
        } else {
          const int r = h * a.nqb + qb;
          int beg = a.blk_ptr[r], end = a.blk_ptr[r + 1];
          checked_row(beg, end, a.blk_cap, a.status, DETAIL_BAD_BLKPTR);
          for (int e = beg + dtid; e < end; e += 64) {
            const int kb = a.blk_idx[e];
            if (kb < 0 || kb >= a.nqb) { report(a.status, DSA_ERR_DEVICE, DETAIL_BAD_BLOCK); continue; }
            for (int u = kb * upb; u < kb * upb + upb; ++u)
              if (u * UNIT <= r1) atomicOr(&bb[u >> 5], 1u << (u & 31));
          }
        }
      }
      named_barrier(1, 64);
      {
        int cnt = 0;
        for (int w = dtid; w < a.nwords; w += 64) cnt += __popc(b0[w] | b1[w]);
        cnt = warp_sum_int(cnt);
        if (lane == 0 && cnt) atomicAdd(&misc[3], cnt);
      }
      named_barrier(1, 64);
      if (dtid == 0) {
        DecInfo& di = dec[s];
        di.item = item;
        di.h = h;
        di.qt = qt;
        di.kvh = h / a.G;
        di.T_u = misc[3];  // one tile per unit
        di.flags1 = shared_qb ? 3 : 1;
        di.T = di.T_u + ceil_div(di.cc[0], BN) + ceil_div(di.cc[1], BN);
        di.wins = 0;
        if constexpr (RUNS) {
          const bool wins = kind == DSA_KIND_VS_WINDOWS;
          di.wins = wins ? 1 : 0;
          if (!wins || !live[0]) di.rn[0] = 0;
          if (!wins || !live[1]) di.rn[1] = 0;
        }
        di.tg = tg_dec;
        // publish the item (its slot is free once both consumers read item kc - 2)
        const int slot = kc & 1;
        const bool ok = kc < 2 || mbar_wait_ool(&bars[B_ITEMFREE + slot], ((kc >> 1) - 1) & 1, limit, a.status,
                                            DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend);
        if (ok) {
          ItemInfo& it = items[slot];
          it.h = h;
          it.qt = qt;
          it.kind = kind;
          it.sink = a.head_info[h * 4 + 1];
          it.window = a.head_info[h * 4 + 2];
          it.T = di.T;
          mbar_arrive(&bars[B_ITEMFULL + slot]);
          mbar_arrive(&bars[B_DECFULL + s]);
        }
        misc[9] = ok ? 1 : 0;
      }
      named_barrier(1, 64);
      if (misc[9] == 0) { go = false; return false; }
      tg_dec += dec[s].T;
      return true;
    };

    // Gathers the column tiles of item kc (bitmap set kc & 1) into the K/V
    // buffers: rows loaded into the swizzled layout by all 64 threads.
    auto gather = [&](int kc) {
      const int s = kc & 1;
      const DecInfo di = dec[s];
      const uint32_t* b0 = bits + s * 2 * a.nwords;
      const uint32_t* b1 = b0 + a.nwords;
      // the column tiles follow the item's unit tiles (see the producer)
      if (dtid == 0)
        misc[9] = mbar_wait_ool(&bars[B_UNITS], kc & 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend) ? 1 : 0;
      named_barrier(1, 64);
      if (misc[9] == 0) { go = false; return; }
      int t = di.T_u;
      for (int hh = 0; COLS && go && hh < 2; ++hh) {
        const int nt = ceil_div(di.cc[hh], BN);
        const int cflags = hh ? 2 : di.flags1;
        for (int ct = 0; ct < nt; ++ct, ++t) {
          const int g = di.tg + t;
          const int b = g & 1;
          const uint32_t use = (g >> 1) & 1;
          if (dtid == 0) {
            bool ok = mbar_wait_ool(&bars[B_KEMPTY + b], use ^ 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend);
            ok = ok && mbar_wait_ool(&bars[B_VEMPTY + b], use ^ 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag, kLoaderSuspend);
            misc[9] = ok ? 1 : 0;
          }
          named_barrier(1, 64);
          if (misc[9] == 0) { go = false; break; }
          const int first = di.cb[hh] + ct * BN;
          const int nc = min(BN, di.cc[hh] - ct * BN);
          int* cj = colsm + (g % NINFO) * BN;
          uint8_t* kst = sm + L::K_OFF + b * DS * KSLAB;
          uint8_t* vst = sm + L::V_OFF + b * DS * KSLAB;
          constexpr int CH = D / 8;           // 16-byte chunks per row
          constexpr int PER = BN * CH / 64;   // chunks per thread
          constexpr int UNR = 4;
          static_assert(PER % UNR == 0, "gather unroll");
#pragma unroll 1
          for (int i0 = 0; i0 < PER; i0 += UNR) {
            uint4 kv[UNR], vv[UNR];
            uint32_t off[UNR];
#pragma unroll
            for (int q = 0; q < UNR; ++q) {
              const int i = (i0 + q) * 64 + dtid;
              const int slot = i / CH;
              const int ch = i % CH;
              int j = (slot < nc) ? a.col_idx[first + slot] : -1;
              if (slot < nc && (j < 0 || j >= a.N)) {
                report(a.status, DSA_ERR_DEVICE, DETAIL_BAD_COL);
                j = -1;
              }
              if (ch == 0) {
                // bit 24 / 25: the column's block is already kept for half 0 / half 1,
                // so that half must not count the key a second time
                int v = j;
                if (j >= 0) {
                  const int u = j / UNIT;
                  // (the units of a VS_WINDOWS item hold only its run keys: there the
                  // runs alone decide)
                  int cov = di.wins ? 0
                                    : ((int)((b0[u >> 5] >> (u & 31)) & 1u) | ((int)((b1[u >> 5] >> (u & 31)) & 1u) << 1));
                  if constexpr (RUNS) {
                    // a column inside a slash run of the half counts once
                    if (di.rn[0] > 0 && key_in_runs(a.dist + di.rbeg[0], di.rn[0], di.rr1[0], j)) cov |= 1;
                    if (di.rn[1] > 0 && key_in_runs(a.dist + di.rbeg[1], di.rn[1], di.rr1[1], j)) cov |= 2;
                  }
                  v = j | (cov << 24);
                }
                cj[slot] = v;
              }
              const int jr = j < 0 ? 0 : j;
              kv[q] = __ldg(reinterpret_cast<const uint4*>(a.K + di.kvh * a.k_hs + (int64_t)jr * a.k_ts) + ch);
              vv[q] = __ldg(reinterpret_cast<const uint4*>(a.V + di.kvh * a.v_hs + (int64_t)jr * a.v_ts) + ch);
              off[q] = (ch >> 3) * KSLAB + swz(slot, ch & 7);
            }
#pragma unroll
            for (int q = 0; q < UNR; ++q) {
              *reinterpret_cast<uint4*>(kst + off[q]) = kv[q];
              *reinterpret_cast<uint4*>(vst + off[q]) = vv[q];
            }
          }
          fence_proxy_async_smem();
          named_barrier(1, 64);
          if (dtid == 0) {
            StageInfo& si = info[g % NINFO];
            si.type = 1;
            si.u = -1;
            si.flags = cflags;
            si.ncols = nc;
            mbar_arrive(&bars[B_INFO + g % NINFO]);
            mbar_arrive(&bars[B_KFULL + b]);
            mbar_arrive(&bars[B_VFULL + b]);
          }
        }
      }
      if (go && dtid == 0) mbar_arrive(&bars[B_COLS]);
    };

    // decode(kc) then gather(kc - 1): one call site each keeps the code small
    for (int kc = 0; go; ++kc) {
      const bool have = decode(kc);
      if (kc > 0 && go) gather(kc - 1);
      if (!have) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, 0, 1);
      static_assert(BN == 64, "P.V issues four k-steps of 16 keys");
      const uint64_t q_desc = smem_desc(smem_u32(sm + L::Q_OFF), 16, 1024, SWZ_128B);
      const uint64_t k_desc0 = smem_desc(smem_u32(sm + L::K_OFF), 16, 1024, SWZ_128B);
      const uint64_t k_desc1 = smem_desc(smem_u32(sm + L::K_OFF + DS * KSLAB), 16, 1024, SWZ_128B);
      const uint64_t v_desc0 = smem_desc(smem_u32(sm + L::V_OFF), KSLAB, 1024, SWZ_128B);
      const uint64_t v_desc1 = smem_desc(smem_u32(sm + L::V_OFF + DS * KSLAB), KSLAB, 1024, SWZ_128B);
      bool ok = true;
      int tg = 0;
      volatile int* seen = misc;  // [11] K, [12] V, [13] Q loads seen landed (for the producer's drain)
      for (int kc = 0; ok; ++kc) {
        const int slot = kc & 1;
        if (!mbar_wait_ool(&bars[B_ITEMFULL + slot], (kc >> 1) & 1, limit, a.status, DETAIL_WAIT_Q, abort_flag, kMmaSuspend)) break;
        const int T = items[slot].T;
        mbar_arrive(&bars[B_ITEMFREE + slot]);
        if (T < 0) break;  // no more items
        if (!mbar_wait_ool(&bars[B_QFULL], kc & 1, limit, a.status, DETAIL_WAIT_Q, abort_flag, kMmaSuspend)) break;
        seen[13] = kc + 1;
        if (T == 0) tc_commit(&bars[B_QEMPTY]);
        for (int t = 0; t <= T; ++t) {
          if (t < T) {
            // S(g) = Q K(g)^T into S buffer g & 1
            const int g = tg + t;
            const int b = g & 1;
            const uint32_t use = (g >> 1) & 1;
            if (!mbar_wait_ool(&bars[B_KFULL + b], use, limit, a.status, DETAIL_WAIT_K, abort_flag, kMmaSuspend)) { ok = false; break; }
            seen[11] = g + 1;
            // the buffer still holds P(g-2), which P(g-2) V(g-2) reads; that
            // product was issued by this thread before this one, and the
            // tensor core runs one thread's MMAs in issue order, so its reads of
            // P precede this product's writes of S without a wait here
            tc_fence_after();
            mma_qk_tile<D / 16>(tmem_base + S_COL + 64 * b, q_desc, b ? k_desc1 : k_desc0, IDESC_QK);
            tc_commit(&bars[B_SFULL + b]);
            tc_commit(&bars[B_KEMPTY + b]);
            if (t == T - 1) tc_commit(&bars[B_QEMPTY]);  // Q may be replaced by the next item's
          }
          if (t >= 1) {
            // O += P(g-1) V(g-1); the item's first P.V overwrites O
            const int u = t - 1;
            const int g = tg + u;
            const int b = g & 1;
            const uint32_t use = (g >> 1) & 1;
            if (!mbar_wait_ool(&bars[B_PFULL + b], use, limit, a.status, DETAIL_WAIT_P, abort_flag, kMmaSuspend)) { ok = false; break; }
            if (!mbar_wait_ool(&bars[B_VFULL + b], use, limit, a.status, DETAIL_WAIT_V, abort_flag, kMmaSuspend)) { ok = false; break; }
            seen[12] = g + 1;
            tc_fence_after();
            mma_pv_tile(tmem_O, tmem_base + S_COL + 64 * b, b ? v_desc1 : v_desc0, IDESC_PV, u > 0 ? 1u : 0u);
            tc_commit(&bars[B_ODONE]);
            tc_commit(&bars[B_VEMPTY + b]);
          }
        }
        if (ok && T > 0) tc_commit(&bars[B_OREADY]);  // the item's O is final once this completes
        tg += T;
      }
      // drain every MMA this thread issued before TMEM is released (also after
      // an abort: the wait ignores the abort flag)
      tc_commit(&bars[B_DRAIN]);
      mbar_drain(&bars[B_DRAIN], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;           // TMEM lane quadrant of this warp
    const int r = q4 * 32 + lane;      // row within the tile == TMEM lane
    const int half = r >> 6;
    const int hbit = 1 << half;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bool ok = true;
    int tg = 0, nready = 0;
    for (int kc = 0; ok; ++kc) {
      const int islot = kc & 1;
      if (!warp_wait(&bars[B_ITEMFULL + islot], (kc >> 1) & 1, limit, a.status, DETAIL_WAIT_Q, abort_flag)) break;
      const ItemInfo it = items[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_ITEMFREE + islot]);
      if (it.T < 0) break;  // no more items
      const int T = it.T;
      const int kind = it.kind;
      const int sink = it.sink;
      const int window = it.window;
      const int row = it.qt * BM + r;
      float m = -INFINITY, l = 0.f;
      for (int t = 0; ok && t < T; ++t) {
        const int g = tg + t;
        const int b = g & 1;
        const uint32_t use = (g >> 1) & 1;
        const int slot = g % NINFO;
        // The StageInfo of a tile is published when its K load is issued, before
        // its S can exist, so this wait ends at the first probe whenever S is not
        // ready yet either.  The tile's mask is built while its S load is in flight.
        if (!warp_wait(&bars[B_INFO + slot], (g / NINFO) & 1, limit, a.status, DETAIL_WAIT_K, abort_flag)) {
          ok = false;
          break;
        }
        const StageInfo si = info[slot];
        if (!warp_wait(&bars[B_SFULL + b], use, limit, a.status, DETAIL_WAIT_S, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_t = tmem_base + lane_off + S_COL + 64 * b;
        float s[64];
        tmem_ld32(s_t, s);
        tmem_ld32(s_t + 32, s + 32);
        // allowed-key bits of this row, 32 columns per word
        uint32_t mw[2];
        if (RUNS && si.type == 3) {
          // the unit's keys inside the half's runs, causal
          const bool oks = (si.flags & hbit) != 0;
#pragma unroll
          for (int k = 0; k < 2; ++k) mw[k] = oks ? (si.m[2 * half + k] & low_bits(row - (si.u * UNIT + k * 32) + 1)) : 0u;
        } else if (!COLS || si.type == 0) {
          const bool oks = (si.flags & hbit) != 0;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int j0 = si.u * UNIT + k * 32;
            uint32_t bits = oks ? low_bits(row - j0 + 1) : 0u;
            if (kind == DSA_KIND_ASHAPE) bits &= low_bits(sink - j0) | ~low_bits(row - window + 1 - j0);
            mw[k] = bits;
          }
        } else {
          const int* cj = colsm + slot * BN;
          const bool okh = (si.flags & hbit) != 0;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint32_t bits = 0u;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
              const int v = cj[k * 32 + i];
              const bool al = okh && (k * 32 + i < si.ncols) && (v >= 0) && !((v >> (24 + half)) & 1) &&
                              ((v & 0xFFFFFF) <= row);
              bits |= (al ? 1u : 0u) << i;
            }
            mw[k] = bits;
          }
        }
        tmem_wait_ld();
        // masked keys become -inf, so one code path serves every tile (exp2 of
        // -inf is 0); a tile the whole warp sees fully skips even that
        if (!__all_sync(0xffffffffu, (mw[0] & mw[1]) == 0xffffffffu)) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
#pragma unroll
            for (int i = 0; i < 32; ++i) s[k * 32 + i] = ((mw[k] >> i) & 1u) ? s[k * 32 + i] : -INFINITY;
          }
        }
        // tile max of the allowed raw scores (independent partial maxima)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 32; ++i) mx[i & 3] = max3f(mx[i & 3], s[2 * i], s[2 * i + 1]);
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        const float m_new = fmaxf(m, mt * a.scale_log2);
        // the max moves when it grows by more than the threshold or becomes finite
        // for the first time; O and l only need rescaling in the first case (a
        // row without a finite max so far has O = 0 and l = 0)
        float alpha = 1.f;
        bool need = false;
        if (m_new > m + RESCALE_THRESHOLD) {
          if (m != -INFINITY) {
            alpha = fast_ex2(m - m_new);
            l *= alpha;
            need = true;
          }
          m = m_new;
        }
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          // O must hold every P.V of the item so far before it is rescaled: wait
          // for P(g-1) V(g-1)
          if (!warp_wait(&bars[B_ODONE], (g - 1) & 1, limit, a.status, DETAIL_WAIT_O, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t o_t = tmem_O + lane_off;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(o_t + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(o_t + c * 32, o);
          }
        }
        // P = exp2(s * scale - m) as bf16 pairs over the first 32 columns of the
        // buffer.  A row with no allowed key so far (m = -inf) keeps x = -inf.
        const float negm = (m == -INFINITY) ? 0.f : -m;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1, p0, p1;
            fma2(s[k * 32 + 2 * i], s[k * 32 + 2 * i + 1], a.scale_log2, negm, x0, x1);
            p0 = fast_ex2(x0);
            p1 = fast_ex2(x1);
            add2(ls[(i & 1) * 2], ls[(i & 1) * 2 + 1], p0, p1);
            __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
            pk[i] = *reinterpret_cast<uint32_t*>(&v2);
          }
          tmem_st16(s_t + k * 16, pk);
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_PFULL + b]);
      }
      // epilogue.  The MMA thread commits B_OREADY once per item with tiles,
      // after the item's last P.V; O is read out of TMEM before this warp
      // produces the next item's first P, which is what lets that item's first
      // P.V overwrite it.
      const bool have = ok && T > 0;
      if (have) {
        if (!warp_wait(&bars[B_OREADY], nready & 1, limit, a.status, DETAIL_WAIT_O, abort_flag)) ok = false;
        ++nready;
        tc_fence_after();
      }
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const bool in = row < a.N;
      __nv_bfloat16* orow = a.O + (int64_t)it.h * a.o_hs + (int64_t)(in ? row : 0) * a.o_ts;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (have && ok) {
          tmem_ld32(tmem_O + lane_off + c * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (in) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(o[2 * i] * inv, o[2 * i + 1] * inv);
            pk[i] = *reinterpret_cast<uint32_t*>(&v2);
          }
          if (a.o_v8) {
            st_global_v8(orow + c * 32, pk);
            st_global_v8(orow + c * 32 + 16, pk + 8);
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<uint4*>(orow + c * 32 + v * 8) = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
      if (a.lse != nullptr && in)
        a.lse[(int64_t)it.h * a.N + row] = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      tg += T;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// --------------------------------------------------------------------------
// host side
// --------------------------------------------------------------------------
// Item counters of the persistent attention kernel, one per launch taken
// round-robin from a pool so that launches in flight on different streams do not
// share one (up to kSchedSlots of them).  Each use of a slot gets a larger epoch
// than the one before (sched_next), so a slot needs no clearing between launches.
constexpr int kSchedSlots = 64;
__device__ unsigned long long g_sched[kSchedSlots];

bool sched_slot(unsigned long long** slot, unsigned* epoch) {
  constexpr int kMaxDev = 64;
  static std::atomic<unsigned long long*> base[kMaxDev] = {};
  static std::atomic<unsigned long long> launches{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  unsigned long long* b = base[dev].load();
  if (b == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sched) != cudaSuccess) return false;
    b = static_cast<unsigned long long*>(p);
    base[dev].store(b);  // every thread finds the same address
  }
  const unsigned long long n = launches.fetch_add(1ull);
  *slot = b + (n % kSchedSlots);
  *epoch = (unsigned)(n / kSchedSlots) + 1u;  // 0 is the value of a never-used slot
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over a bf16 tensor [H][N][d] with element strides (token, head); box
// of 64 columns x box_rows rows x 1 head, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* map, const void* base, int d, int N, int H, int64_t ts, int64_t hs, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  if (H == 1 || hs == 0) hs = (int64_t)N * ts;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)ts * 2, (cuuint64_t)hs * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool RUNS, bool COLS>
dsa_status launch_d(const dsa_problem& p, const void* Q, const void* K, const void* V, const dsa_indices& idx,
                    void* O, float* lse, cudaStream_t stream, unsigned* status) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, D, p.N, p.Hq, p.q_token_stride, p.q_head_stride, BM) ||
      !make_map(&mk, K, D, p.N, p.Hkv, p.k_token_stride, p.k_head_stride, UNIT) ||
      !make_map(&mv, V, D, p.N, p.Hkv, p.v_token_stride, p.v_head_stride, UNIT))
    return DSA_ERR_CUDA;
  AttnArgs a;
  a.Hq = p.Hq;
  a.G = p.Hq / p.Hkv;
  a.N = p.N;
  a.B = p.block;
  a.nqb = ceil_div(p.N, p.block);
  a.n_qtiles = ceil_div(p.N, BM);
  a.n_units = ceil_div(p.N, UNIT);
  a.nwords = ceil_div(a.n_units, 32);
  a.head_info = idx.head_info;
  a.blk_ptr = idx.blk_ptr;
  a.blk_idx = idx.blk_idx;
  a.dist_ptr = idx.dist_ptr;
  a.dist = idx.dist;
  a.col_ptr = idx.col_ptr;
  a.col_idx = idx.col_idx;
  a.blk_cap = idx.blk_cap;
  a.dist_cap = idx.dist_cap;
  a.col_cap = idx.col_cap;
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.k_hs = p.k_head_stride;
  a.k_ts = p.k_token_stride;
  a.v_hs = p.v_head_stride;
  a.v_ts = p.v_token_stride;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_hs = p.o_head_stride;
  a.o_ts = p.o_token_stride;
  a.o_v8 = ((reinterpret_cast<uintptr_t>(O) & 31u) == 0 && p.o_token_stride % 16 == 0 && p.o_head_stride % 16 == 0) ? 1 : 0;
  a.lse = lse;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  a.status = status;
  if (!sched_slot(&a.sched, &a.epoch)) return DSA_ERR_CUDA;
  a.wait_limit_ns = wait_limit_ns();
  int smem = Smem<D>::bytes(a.nwords);
  // at most two CTAs per SM: each holds 256 of the 512 TMEM columns
  if (smem < 80 * 1024) smem = 80 * 1024;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D, RUNS, COLS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  const int n_items = a.n_qtiles * p.Hq;
  if (n_items == 0) return DSA_OK;
  // persistent: two CTAs per SM, items dealt round-robin
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const int grid = n_items < 2 * sms ? n_items : 2 * sms;
  e = launch_pdl(sparse_attn_kernel<D, RUNS, COLS>, dim3(grid), dim3(NTHREADS), (size_t)smem, stream, mq, mk, mv, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return DSA_OK;
}

}  // namespace

bool make_tma_map_bf16_3d(CUtensorMap* map, const void* base, int d, int N, int H, int64_t ts, int64_t hs,
                          int box_rows) {
  return make_map(map, base, d, N, H, ts, hs, box_rows);
}

dsa_status launch_sparse_attn(const dsa_problem& p, const void* Q, const void* K, const void* V,
                              const dsa_indices& idx, void* O, float* lse, cudaStream_t stream, unsigned* status) {
  // the kernel with slash-run masks only when a VS_WINDOWS head is present, and
  // with column tiles only when a VS kind is: the other kinds keep the smaller
  // code of the plainer instantiations
  const bool runs = (idx.kinds_present >> DSA_KIND_VS_WINDOWS) & 1;
  const bool cols = runs || ((idx.kinds_present >> DSA_KIND_VS) & 1);
  if (p.d == 128)
    return runs ? launch_d<128, true, true>(p, Q, K, V, idx, O, lse, stream, status)
                : (cols ? launch_d<128, false, true>(p, Q, K, V, idx, O, lse, stream, status)
                        : launch_d<128, false, false>(p, Q, K, V, idx, O, lse, stream, status));
  if (p.d == 64)
    return runs ? launch_d<64, true, true>(p, Q, K, V, idx, O, lse, stream, status)
                : (cols ? launch_d<64, false, true>(p, Q, K, V, idx, O, lse, stream, status)
                        : launch_d<64, false, false>(p, Q, K, V, idx, O, lse, stream, status));
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
