// Sparse-index construction for sm_100a.
//
// Per head, following its pattern (MInference abstract: indices are built
// dynamically from the assigned pattern):
//   A-shape    -- closed-form key blocks of the sink and the local window
//                 ("MInference 1.0" summary, "3つの疎パターン": fixed mask);
//   VS         -- coarse attention of the last last_q queries against all keys,
//                 vertical sums v[j] and slash sums s[o], exact top-k of each,
//                 then block distances D and per-query-block columns
//                 ("推論時は軽い近似で動的マスクを作る");
//   block kinds-- mean-pooled Q and K per block, s_IJ = tau qbar_I . kbar_J over the
//                 causal triangle, then top-k (MInference block-sparse, MoBA routing)
//                 or the max-relative threshold of FlashPrefill section 2.2
//                 (P_IJ >= alpha max_J P_IJ  <=>  s_IJ >= max_J s_IJ + ln alpha);
//                 MoBA may first run a causal depthwise conv with SiLU and a
//                 residual over the keys ("2. キーに対する畳み込み適用").
// Every list is produced by count -> scan -> fill into caller-owned CSR arrays.
// Every kernel is launched with programmatic dependent launch (pdl_prologue in
// dsa_common.cuh), and the build issues no memsets: the count kernels clear the
// pointer entries no other kernel writes, VS pass 1 clears the slash sums.
#include <math.h>
#include <string.h>

#include <algorithm>

#include <cooperative_groups.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int MAXH = 256;     // heads per layer this build accepts
constexpr int MAXKV = 256;
// keys per CTA of the VS estimate: one of VS_CHUNKS, chosen per problem by
// choose_vs_chunk (all multiples of VS_SUB and >= VS_MAXL)
constexpr int VS_CHUNKS[3] = {1024, 768, 512};
constexpr int VS_CHUNK_MAX = 1024;
constexpr int VS_SUB = 128;     // keys per sub-tile
constexpr int VS_MAXL = 128;    // last_q limit
static_assert(VS_CHUNKS[0] == VS_CHUNK_MAX && VS_CHUNKS[0] % VS_SUB == 0 && VS_CHUNKS[1] % VS_SUB == 0 &&
                  VS_CHUNKS[2] % VS_SUB == 0,
              "chunks are whole sub-tiles");
static_assert(VS_CHUNKS[2] >= VS_MAXL, "the keys an offset meets from the estimate rows span at most two chunks");

struct HeadTab {
  int kind[MAXH];
  int sink[MAXH];
  int window[MAXH];
  int last_q[MAXH];
  int n_vert[MAXH];
  int n_slash[MAXH];
  int topk[MAXH];
  float lnalpha[MAXH];
  int keep_sink[MAXH];
  int keep_local[MAXH];
  int bslot[MAXH];  // slot among block-kind heads, -1 otherwise
  int uslot[MAXH];  // slot among unified-discovery heads, -1 otherwise
  int uhead[MAXH];  // q-head of unified slot s
  int vslot[MAXH];  // slot among VS heads, -1 otherwise
  int bhead[MAXH];  // q-head of block slot s
  int vhead[MAXH];  // q-head of VS slot s
};

struct ConvTab {
  const float* w[MAXKV];
  const float* b[MAXKV];
  int width[MAXKV];
  int need[MAXKV];  // K of this KV head is pooled
};

struct Layout {
  int Hq, Hkv, G, N, d, B, nqb, nkw, nbh, nvs, vs_chunk, vs_nchunks, vs_lmax, nuh, sel_ri, sel_nx, dtmp_stride;
  int64_t off_kbar, off_sel, off_v, off_s, off_part, off_stat, off_dtmp, off_dbits, off_spart, off_upart, total;
};

__host__ __device__ inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Vertical-Slash kinds: the estimate and its top-k are shared; they differ in
// how the chosen slashes are covered (aligned blocks, or exact per-block runs).
__host__ __device__ inline bool is_vs_kind(int k) { return k == DSA_KIND_VS || k == DSA_KIND_VS_WINDOWS; }

// order-preserving float -> uint32 key
__device__ __forceinline__ uint32_t fkey(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// CTA-wide helpers (blockDim.x threads, multiple of 32, <= 1024)
// ---------------------------------------------------------------------------
// Exact top-k of vals[0..n) (ties to the lower index), n > k >= 1.  Finds the
// k-th largest key T by three radix passes over the 32-bit key, most
// significant digit first (12, 12 and 8 bits), and how many keys equal to T to
// take.  One 4096-bin histogram for the whole CTA: the first digit is the sign,
// the exponent and the top mantissa bits, so sums of similar magnitude still
// spread over many bins and few lanes of a warp add to the same bin at once
// (an 8-bit first digit is the exponent alone: ~20 lanes of every warp hit one
// bin on the VS sums).  blockDim.x: a power of two, 32..1024.
// hist: shared int[RADIX_BINS]; red: shared int[>= 2 + blockDim.x / 32].
constexpr int RB = 8;  // keys loaded per thread before use in the CTA-wide select
constexpr int RADIX_BINS = 4096;

template <typename Loader>
__device__ void radix_kth(const Loader& load, int n, int k, int* hist, int* red, uint32_t* T_out,
                          int* take_eq_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bpt = RADIX_BINS / blockDim.x;  // bins per thread in the digit search
  uint32_t prefix = 0, mask = 0;
  int need = k;  // keys still to take among those matching prefix (>= 1)
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
    const uint32_t dmask = pass == 2 ? 0xffu : 0xfffu;
    for (int i = threadIdx.x; i < RADIX_BINS; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    // RB independent loads in flight per thread before their keys are counted
    for (int i0 = 0; i0 < n; i0 += RB * blockDim.x) {
      uint32_t key[RB];
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        const int i = i0 + q * blockDim.x + threadIdx.x;
        key[q] = (i < n) ? fkey(load(i)) : 0u;
      }
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        const int i = i0 + q * blockDim.x + threadIdx.x;
        if (i < n && (key[q] & mask) == prefix) atomicAdd(&hist[(key[q] >> shift) & dmask], 1);
      }
    }
    __syncthreads();
    // thread t takes bins RADIX_BINS-1-t*bpt downwards (bins above the digit
    // width are empty); a CTA-wide exclusive scan of the per-thread sums is the
    // count of keys in higher bins; the one thread whose run crosses `need`
    // holds the digit
    const int top = RADIX_BINS - 1 - threadIdx.x * bpt;
    int tot = 0;
    for (int q = 0; q < bpt; ++q) tot += hist[top - q];
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) red[2 + warp] = incl;
    __syncthreads();
    int above = incl - tot;
    for (int w = 0; w < warp; ++w) above += red[2 + w];
    if (above < need && above + tot >= need) {
      for (int q = 0; q < bpt; ++q) {
        const int c = hist[top - q];
        if (above + c >= need) {
          red[0] = top - q;
          red[1] = above;
          break;
        }
        above += c;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)red[0] << shift;
    mask |= dmask << shift;
    need -= red[1];
    __syncthreads();
  }
  *T_out = prefix;
  *take_eq_out = need;
}

// Ordered selection: calls emit(i, rank) for every selected i in ascending i,
// where selected = key > T, or key == T among the first take_eq such keys.
// One warp per contiguous segment; coalesced reads; red: shared int[>= 2*nw+2].
template <typename Loader, typename Emit>
__device__ void ordered_select(const Loader& load, int n, uint32_t T, int take_eq, int* red, const Emit& emit) {
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = ceil_div(ceil_div(n, nw), 32) * 32;
  const int beg = min(n, warp * seg), end = min(n, beg + seg);
  int gt = 0, eq = 0;
  for (int i0 = beg + lane; i0 < end; i0 += 32 * RB) {
    uint32_t key[RB];
#pragma unroll
    for (int q = 0; q < RB; ++q) key[q] = (i0 + 32 * q < end) ? fkey(load(i0 + 32 * q)) : 0u;
#pragma unroll
    for (int q = 0; q < RB; ++q) {
      if (i0 + 32 * q < end) {
        gt += key[q] > T;
        eq += key[q] == T;
      }
    }
  }
  gt = warp_sum_int(gt);
  eq = warp_sum_int(eq);
  if (lane == 0) {
    red[2 * warp] = gt;
    red[2 * warp + 1] = eq;
  }
  __syncthreads();
  int out_base = 0, eq_base = 0;
  for (int w = 0; w < warp; ++w) {
    eq_base += red[2 * w + 1];
  }
  // output position: selected-before = gt of earlier warps + min(eq earlier, take_eq)
  for (int w = 0; w < warp; ++w) out_base += red[2 * w];
  out_base += min(eq_base, take_eq);
  __syncthreads();
  int eq_run = eq_base;
  int pos = out_base;
  uint32_t kb[RB];
  for (int i0 = beg; i0 < end; i0 += 32) {
    const int i = i0 + lane;
    const int q = ((i0 - beg) >> 5) % RB;
    if (q == 0) {
#pragma unroll
      for (int u = 0; u < RB; ++u) kb[u] = (i + 32 * u < end) ? fkey(load(i + 32 * u)) : 0u;
    }
    uint32_t key = kb[0];
#pragma unroll
    for (int u = 1; u < RB; ++u)
      if (q == u) key = kb[u];
    bool sel = false, iseq = false;
    if (i < end) {
      iseq = key == T;
      sel = key > T;
    }
    const unsigned eqm = __ballot_sync(0xffffffffu, iseq);
    const int eq_before = eq_run + __popc(eqm & ((1u << lane) - 1u));
    if (iseq && eq_before < take_eq) sel = true;
    eq_run += __popc(eqm);
    const unsigned sm = __ballot_sync(0xffffffffu, sel);
    if (sel) emit(i, pos + __popc(sm & ((1u << lane) - 1u)));
    pos += __popc(sm);
  }
}

// ---------------------------------------------------------------------------
// head info + A-shape / block counts
// ---------------------------------------------------------------------------
// also clears the distance-list counts of non-VS heads (and the leading zero)
__global__ void k_head_info(const __grid_constant__ HeadTab ht, int Hq, int32_t* head_info, int32_t* dist_ptr) {
  pdl_prologue();
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= Hq) return;
  if (h == 0) dist_ptr[0] = 0;
  if (!is_vs_kind(ht.kind[h])) dist_ptr[1 + h] = 0;
  head_info[h * 4 + 0] = ht.kind[h];
  head_info[h * 4 + 1] = ht.kind[h] == DSA_KIND_ASHAPE ? ht.sink[h] : 0;
  head_info[h * 4 + 2] = ht.kind[h] == DSA_KIND_ASHAPE ? ht.window[h] : 0;
  head_info[h * 4 + 3] = 0;
}

__device__ __forceinline__ void ashape_range(int qb, int B, int N, int sink, int window, int* a, int* w) {
  const int r0 = qb * B;
  const int r1 = min(N - 1, r0 + B - 1);
  *a = ceil_div(min(sink, r1 + 1), B);          // sink blocks [0, a)
  *w = max(0, r0 - window + 1) / B;             // window blocks [w, qb]
}

// Block-list counts of A-shape heads; zero counts for the rows no later kernel
// fills (block lists of VS heads, column lists of non-VS heads) and the leading
// zeros of both pointer arrays.  Block-kind and VS counts are written later.
__global__ void k_ashape_count(const __grid_constant__ HeadTab ht, Layout L, int32_t* blk_ptr, int32_t* col_ptr) {
  pdl_prologue();
  const int h = blockIdx.y;
  const int qb = blockIdx.x * blockDim.x + threadIdx.x;
  if (qb >= L.nqb) return;
  const int kind = ht.kind[h];
  if (h == 0 && qb == 0) {
    blk_ptr[0] = 0;
    col_ptr[0] = 0;
  }
  if (!is_vs_kind(kind)) col_ptr[1 + h * L.nqb + qb] = 0;
  if (is_vs_kind(kind)) blk_ptr[1 + h * L.nqb + qb] = 0;
  if (kind != DSA_KIND_ASHAPE) return;
  int a, w;
  ashape_range(qb, L.B, L.N, ht.sink[h], ht.window[h], &a, &w);
  const int cnt = a + (qb + 1 - max(w, a) > 0 ? qb + 1 - max(w, a) : 0);
  blk_ptr[1 + h * L.nqb + qb] = cnt;
}

// Causal depthwise key conv (width W, SiLU, residual) summed over a contiguous
// run of rows [r0, r1) for this thread's 8 channels: weights in registers, the
// last W rows in a register window, one 16-byte load per row (four in flight).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sum over rows r0 <= r < r1 of k_r + SiLU(conv_r) for 8 channels, where
// conv_r = b + sum_t w_t k_{r - t}.  SiLU(c) = c sigmoid(c) = h + h tanh(h) with
// h = c / 2 (sigmoid(c) = (1 + tanh(c / 2)) / 2): one tanh.approx (relative error
// about 2^-11, far below what routing on pooled keys can see) instead of an
// exponential and a division; the halving is folded into the weights and bias.
// sw: the head's weights as [W][D] and its bias as [D], halved, in shared memory.
// (a.x, a.y) * (b.x, b.y) + (c.x, c.y) and (a.x + b.x, a.y + b.y) as one packed
// f32x2 instruction each (per-lane rounding as fmaf / an add: the same values)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t av, bv, cv, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(av) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(bv) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(cv) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(av), "l"(bv), "l"(cv));
  float2 o;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
  return o;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t av, bv, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(av) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(bv) : "f"(b.x), "f"(b.y));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(av), "l"(bv));
  float2 o;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
  return o;
}
// the two bf16 of a 32-bit word as floats (a bf16 is the high half of its float)
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <int W, int D>
__device__ __forceinline__ void conv_rows_sum(const __nv_bfloat16* X, int64_t ts, int c0, int r0, int r1,
                                              const float* sw, float* acc) {
  // channels in pairs (c0 + 2j, c0 + 2j + 1), j < 4: packed f32x2 arithmetic
  float2 wt[W][4], bias[4], win[W][4], acc2[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    bias[j] = make_float2(sw[W * D + c0 + 2 * j], sw[W * D + c0 + 2 * j + 1]);
    acc2[j] = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < W; ++t) wt[t][j] = make_float2(sw[t * D + c0 + 2 * j], sw[t * D + c0 + 2 * j + 1]);
  }
  // before row r is shifted in, win[t] = k[r - 1 - t] (t < W - 1); after the
  // shift win[t] = k[r - t].  Rows before 0 are zero (causal, zero padded).
#pragma unroll
  for (int t = 0; t < W - 1; ++t) {
    const int rr = r0 - 1 - t;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (rr >= 0 && r0 < r1) raw = __ldg(reinterpret_cast<const uint4*>(X + (int64_t)rr * ts + c0));
    const uint32_t* wv = reinterpret_cast<const uint32_t*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) win[t][j] = bf16x2_to_float2(wv[j]);
  }
  // software pipelined: the next four rows are in flight while these four are
  // computed
  uint4 nxt[4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    nxt[u] = (r0 + u < r1) ? __ldg(reinterpret_cast<const uint4*>(X + (int64_t)(r0 + u) * ts + c0))
                           : make_uint4(0, 0, 0, 0);
  for (int r = r0; r < r1; r += 4) {
    uint4 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      raw[u] = nxt[u];
      nxt[u] = (r + 4 + u < r1) ? __ldg(reinterpret_cast<const uint4*>(X + (int64_t)(r + 4 + u) * ts + c0))
                                : make_uint4(0, 0, 0, 0);
    }
    // rows past r1 (the run's last step) are computed and dropped: no branch
    // between the four rows, so their chains overlap
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float kf = (r + u < r1) ? 1.f : 0.f;
      const float2 keep = make_float2(kf, kf);
#pragma unroll
      for (int t = W - 1; t > 0; --t) {
#pragma unroll
        for (int j = 0; j < 4; ++j) win[t][j] = win[t - 1][j];
      }
      const uint32_t* wv = reinterpret_cast<const uint32_t*>(&raw[u]);
#pragma unroll
      for (int j = 0; j < 4; ++j) win[0][j] = bf16x2_to_float2(wv[j]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 h = bias[j];
#pragma unroll
        for (int t = 0; t < W; ++t) h = ffma2(wt[t][j], win[t][j], h);
        const float2 th = make_float2(tanh_approx(h.x), tanh_approx(h.y));
        // k + SiLU(conv) = k + (h + h tanh h)
        acc2[j] = ffma2(keep, fadd2(win[0][j], ffma2(h, th, h)), acc2[j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    acc[2 * j] = acc2[j].x;
    acc[2 * j + 1] = acc2[j].y;
  }
}

// ---------------------------------------------------------------------------
// key mean pooling (+ optional causal depthwise key conv with SiLU and residual)
// ---------------------------------------------------------------------------
// grid: (ceil(nqb / bpc), Hkv); KV heads that no block head reads are skipped.
// Queries are pooled inside k_block_select.  CW = 0: plain mean, for the KV heads
// without a key conv, one block per CTA (bpc = 1); CW = W in 1..8: the conv of
// width W, for the KV heads with that width (one launch per width present, so
// each instantiation holds exactly the registers its width needs), bpc blocks
// per CTA (see conv_blocks_per_cta).
template <int D, int CW>
__global__ void __launch_bounds__(256) k_pool(const __grid_constant__ ConvTab ct, Layout L,
                                              const __nv_bfloat16* K, int64_t k_hs, int64_t k_ts, uint8_t* ws,
                                              int bpc) {
  pdl_prologue();
  constexpr int TPR = D / 8;          // threads per row, 8 channels each
  constexpr int RG = 256 / TPR;       // rows in flight
  __shared__ float part[RG][D];
  __shared__ float sw[CW > 0 ? (CW + 1) * D : 1];  // conv weights [CW][D] and bias [D], halved
  const int b0 = blockIdx.x * bpc;  // the CTA's first block
  const int kvh = blockIdx.y;
  if (!ct.need[kvh] || ct.width[kvh] != CW) return;
  if constexpr (CW > 0) {
    // coalesced: consecutive threads read consecutive weights (stored [D][CW])
    for (int i = threadIdx.x; i < CW * D; i += blockDim.x) sw[(i % CW) * D + i / CW] = 0.5f * ct.w[kvh][i];
    for (int i = threadIdx.x; i < D; i += blockDim.x) sw[CW * D + i] = 0.5f * ct.b[kvh][i];
    __syncthreads();
  }
  const __nv_bfloat16* X = K + kvh * k_hs;
  const int64_t ts = k_ts;
  // pooled rows as bf16 hi[D] then lo[D], hi + lo ~ the fp32 mean
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(ws + L.off_kbar) + ((int64_t)kvh * L.nqb + b0) * 2 * D;
  const int rg = threadIdx.x / TPR;
  const int c0 = (threadIdx.x % TPR) * 8;
  const int r_beg = b0 * L.B;
  const int r_end = min(L.N, r_beg + bpc * L.B);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if constexpr (CW == 0) {
    // plain mean: eight independent row loads in flight per thread
    int r = r_beg + rg;
    for (; r + 7 * RG < r_end; r += 8 * RG) {
      uint4 raw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) raw[u] = __ldg(reinterpret_cast<const uint4*>(X + (int64_t)(r + u * RG) * ts + c0));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __bfloat162float(e[i]);
      }
    }
    for (; r < r_end; r += RG) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(X + (int64_t)r * ts + c0));
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __bfloat162float(e[i]);
    }
  } else {
    // each row group takes a contiguous run of rows (the conv window slides along
    // it); with several blocks per CTA the runs tile the blocks exactly, so each
    // run lies in one block
    const int run = ceil_div(bpc * L.B, RG);
    const int r0 = min(r_end, r_beg + rg * run), r1 = min(r_end, r0 + run);
    conv_rows_sum<CW, D>(X, ts, c0, r0, r1, sw, acc);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[rg][c0 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < D) {
    const int gpb = RG / bpc;  // row groups per block
    for (int j = 0; j < bpc; ++j) {
      const int rows = min(L.N, r_beg + (j + 1) * L.B) - (r_beg + j * L.B);
      if (rows <= 0) break;
      float s = 0.f;
      for (int g = j * gpb; g < (j + 1) * gpb; ++g) s += part[g][threadIdx.x];
      const float x = s / (float)rows;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      out[(int64_t)j * 2 * D + threadIdx.x] = hi;
      out[(int64_t)j * 2 * D + D + threadIdx.x] = __float2bfloat16_rn(x - __bfloat162float(hi));
    }
  }
}

// Blocks per CTA of the conv pooling: enough for 512 rows when the block size
// divides 512 (32-row runs per row group: the W - 1 rows before each run are
// loaded again, and the CTA's set-up is paid once per 512 rows), else one.
// bpc divides the row groups (16 for d = 128, 32 for d = 64), so a block is an
// exact number of runs.
inline int conv_blocks_per_cta(int B) { return (B < 512 && 512 % B == 0) ? 512 / B : 1; }

// the plain pooling for the KV heads without a conv and one launch per conv width present
template <int D>
cudaError_t launch_pool(const ConvTab& ct, const Layout& L, const __nv_bfloat16* k, int64_t k_hs, int64_t k_ts,
                        uint8_t* ws, cudaStream_t st) {
  bool has[9] = {};
  for (int h = 0; h < L.Hkv; ++h)
    if (ct.need[h]) has[ct.width[h] < 0 || ct.width[h] > 8 ? 0 : ct.width[h]] = true;
  const int bpc = conv_blocks_per_cta(L.B);
  const dim3 grid(L.nqb, L.Hkv), cgrid(ceil_div(L.nqb, bpc), L.Hkv), block(256);
  cudaError_t e = cudaSuccess;
  if (has[0]) e = launch_pdl(k_pool<D, 0>, grid, block, 0, st, ct, L, k, k_hs, k_ts, ws, 1);
#define DSA_CONV_POOL(W) \
  if (e == cudaSuccess && has[W]) e = launch_pdl(k_pool<D, W>, cgrid, block, 0, st, ct, L, k, k_hs, k_ts, ws, bpc);
  DSA_CONV_POOL(1) DSA_CONV_POOL(2) DSA_CONV_POOL(3) DSA_CONV_POOL(4)
  DSA_CONV_POOL(5) DSA_CONV_POOL(6) DSA_CONV_POOL(7) DSA_CONV_POOL(8)
#undef DSA_CONV_POOL
  return e;
}

// ---------------------------------------------------------------------------
// block scores + selection.  One CTA (SEL_NT threads) per (block slot, SEL_RI
// consecutive query blocks).  The scores of those rows against every candidate
// key block are one 16-row tile product q̄_tile x K̄^T on the tensor cores
// (mma.sync m16n8k16, bf16 operands, fp32 accumulation).  The pooled rows are
// stored as bf16 hi + lo pairs and the product keeps hi.hi + hi.lo + lo.hi, so a
// score carries about 16 mantissa bits of each operand (the fp32 means have 24).
// K̄ is read once per SEL_RI rows; each warp takes 8-key-block column tiles in
// turn.  Then one warp per row selects: a max and a compare for the threshold,
// an exact radix select for top-k; the selection bitmap is built one 32-block
// word at a time from warp ballots (only the words up to row I's own block are
// written; the list fill reads no further).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int SEL_RI = 16;  // query blocks per CTA
constexpr int SEL_NT = 512;  // threads per CTA
constexpr int SEL_NW = SEL_NT / 32;
// score row stride in floats: 8 past a multiple of 32 so the 8-byte stores of
// one half-warp (rows g..g+3, columns 2 t4) hit 16 distinct bank pairs
__host__ __device__ constexpr int SEL_RS(int npad) { return npad + 8; }
// query blocks per select CTA: up to 2048 query rows to pool, at most SEL_RI
inline int sel_blocks_per_cta(int B) {
  int ri = SEL_RI;
  while (ri > 1 && ri * B > 2048) ri >>= 1;
  return ri;
}
// dynamic shared memory: the score tile, which first holds the pooling partials
inline size_t sel_smem_bytes(int D, int nkw) {
  const size_t scores = (size_t)SEL_RI * SEL_RS(nkw * 32) * 4;
  const size_t partials = (size_t)(SEL_NT / (D / 8)) * D * 4;
  return scores > partials ? scores : partials;
}

// Warp-level exact top-k of vals[0..n) (ties to the lower index), 0 < k < n.
// hist: this warp's shared int[256].  Returns the k-th largest key and how many
// keys equal to it to take.
__device__ void warp_radix_kth(const float* vals, int n, int k, int* hist, uint32_t* T_out, int* take_eq) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t key = fkey(vals[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncwarp();
    // lane L owns bins 255-8L .. 248-8L (descending); find the bin where the
    // running count from the top reaches `need`
    int c[8], own = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = hist[255 - 8 * lane - q];
      own += c[q];
    }
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = incl - own;
    const bool here = excl < need && incl >= need;
    const unsigned who = __ballot_sync(0xffffffffu, here);
    const int src = __ffs(who) - 1;
    int digit = 0, above = 0;
    if (here) {
      int run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + c[q] >= need) { digit = 255 - 8 * lane - q; break; }
        run += c[q];
      }
      above = run;
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    prefix |= (uint32_t)digit << shift;
    mask |= 255u << shift;
    need -= above;
    __syncwarp();
  }
  *T_out = prefix;
  *take_eq = need;
}

// ri query blocks per CTA (a power of two, at most SEL_RI): their rows are
// mean-pooled here, straight from Q (Q-bar never goes to memory), then scored
// and selected.  Streaming Q is most of the index build's HBM traffic; doing it
// in the CTAs that also score lets one CTA's selection overlap another's loads.
template <int D>
__global__ void __launch_bounds__(SEL_NT) k_block_select(const __grid_constant__ HeadTab ht, Layout L,
                                                      const __nv_bfloat16* Q, int64_t q_hs, int64_t q_ts,
                                                      uint8_t* ws, int32_t* blk_ptr, int ri) {
  pdl_prologue();
  extern __shared__ float sc[];  // [SEL_RI][SEL_RS(npad)] scores of the group's rows
  __shared__ int hist[SEL_NW][256];
  const int npad = L.nkw * 32;
  const int slot = blockIdx.y;
  const int I0 = blockIdx.x * ri;
  const int nI = min(ri, L.nqb - I0);
  const int h = ht.bhead[slot];
  const int kind = ht.kind[h];
  const int kvh = h / L.G;
  const float tau = rsqrtf((float)D);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const __nv_bfloat16* khl = reinterpret_cast<const __nv_bfloat16*>(ws + L.off_kbar) + (int64_t)kvh * L.nqb * 2 * D;
  const int g = lane >> 2, t4 = lane & 3;
  // The contraction runs over the channels in a permuted order (the same on
  // both operands, so the dot products are unchanged): the 16-byte run of
  // channels 32m + 8 t4 .. +7 of a row feeds k-steps 2m and 2m + 1, so every
  // fragment register pair comes from one vector load.
  auto ld16 = [](const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); };
  // the group's 16 pooled query rows (hi then lo) staged in shared memory; the
  // row pitch is 64 bytes past a multiple of 128 so that the 16-byte fragment
  // loads of rows g and g + 1 fall in different banks
  constexpr int QP = 2 * D + 32;
  __shared__ __align__(16) __nv_bfloat16 qs[SEL_RI][QP];
  {
    // mean pooling: thread (row group rg, 8-channel chunk c0); row group rg
    // serves block rg / gpb and takes every gpb-th row of it, eight loads in
    // flight; partial sums meet in shared memory (aliasing the score tile)
    constexpr int CPR = D / 8;         // 16-byte chunks per row
    constexpr int RGS = SEL_NT / CPR;  // row groups
    static_assert(RGS % SEL_RI == 0, "row groups per block");
    const int gpb = RGS / ri;
    const int rg = tid / CPR, c0 = (tid % CPR) * 8;
    const int b = rg / gpb, sub = rg % gpb;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    if (b < nI) {
      const int r_beg = (I0 + b) * L.B, r_end = min(L.N, r_beg + L.B);
      const __nv_bfloat16* X = Q + (int64_t)h * q_hs + c0;
      int r = r_beg + sub;
      for (; r + 7 * gpb < r_end; r += 8 * gpb) {
        uint4 raw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) raw[u] = __ldg(reinterpret_cast<const uint4*>(X + (int64_t)(r + u * gpb) * q_ts));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] += __bfloat162float(e[j]);
        }
      }
      for (; r < r_end; r += gpb) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(X + (int64_t)r * q_ts));
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += __bfloat162float(e[j]);
      }
    }
    float* part = sc;  // [RGS][D]
#pragma unroll
    for (int j = 0; j < 8; ++j) part[rg * D + c0 + j] = acc[j];
    __syncthreads();
    for (int i = tid; i < SEL_RI * D; i += SEL_NT) {
      const int bb = i / D, ch = i % D;
      __nv_bfloat16 hi = __float2bfloat16_rn(0.f), lo = hi;
      if (bb < nI) {
        float sum = 0.f;
        for (int k = 0; k < gpb; ++k) sum += part[(bb * gpb + k) * D + ch];
        const int r_beg = (I0 + bb) * L.B;
        const float x = sum / (float)(min(L.N, r_beg + L.B) - r_beg);
        hi = __float2bfloat16_rn(x);
        lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      }
      qs[bb][ch] = hi;
      qs[bb][D + ch] = lo;
    }
    __syncthreads();  // the score tile may now overwrite the partial sums
  }
  // s = tau (qhi khi + qhi klo + qlo khi): bf16 tensor-core products with fp32
  // accumulation; the dropped qlo klo term is below 2^-16 of |q| |k| per channel.
  // Each warp takes 8-key-block column tiles in turn.
  const int Jend = I0 + nI;  // candidates of the group's last row are J < Jend
  const int ntiles = ceil_div(Jend, 8);
  for (int nt = warp; nt < ntiles; nt += SEL_NW) {
    const int J0 = nt * 8;
    const int Jb = J0 + g;
    const __nv_bfloat16* kp = khl + (int64_t)min(Jb, L.nqb - 1) * 2 * D + 8 * t4;
    uint4 bh[D / 32], bl[D / 32];
#pragma unroll
    for (int m = 0; m < D / 32; ++m) {
      bh[m] = ld16(kp + 32 * m);
      bl[m] = ld16(kp + D + 32 * m);
    }
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < D / 32; ++m) {
      const int cq = 32 * m + 8 * t4;
      const uint4 h0 = *reinterpret_cast<const uint4*>(&qs[g][cq]);
      const uint4 h1 = *reinterpret_cast<const uint4*>(&qs[g + 8][cq]);
      const uint4 l0 = *reinterpret_cast<const uint4*>(&qs[g][D + cq]);
      const uint4 l1 = *reinterpret_cast<const uint4*>(&qs[g + 8][D + cq]);
      const uint32_t ah0[4] = {h0.x, h1.x, h0.y, h1.y}, ah1[4] = {h0.z, h1.z, h0.w, h1.w};
      const uint32_t al0[4] = {l0.x, l1.x, l0.y, l1.y}, al1[4] = {l0.z, l1.z, l0.w, l1.w};
      mma_bf16_16816(c, ah0, bh[m].x, bh[m].y);
      mma_bf16_16816(c, ah0, bl[m].x, bl[m].y);
      mma_bf16_16816(c, al0, bh[m].x, bh[m].y);
      mma_bf16_16816(c, ah1, bh[m].z, bh[m].w);
      mma_bf16_16816(c, ah1, bl[m].z, bl[m].w);
      mma_bf16_16816(c, al1, bh[m].z, bh[m].w);
    }
    // columns J0 + 2 t4, +1 of rows g and g + 8; key blocks past the last
    // real one (clamped loads above) land in columns no row reads
    const int J = J0 + 2 * t4;
    if (g < nI) *reinterpret_cast<float2*>(sc + g * SEL_RS(npad) + J) = make_float2(c[0] * tau, c[1] * tau);
    if (g + 8 < nI) *reinterpret_cast<float2*>(sc + (g + 8) * SEL_RS(npad) + J) = make_float2(c[2] * tau, c[3] * tau);
  }
  __syncthreads();
  // selection: warp w handles rows w, w + SEL_NW, ...
  for (int rr = warp; rr < nI; rr += SEL_NW) {
    const int I = I0 + rr;
    const float* row = sc + rr * SEL_RS(npad);
    uint32_t* sel = reinterpret_cast<uint32_t*>(ws + L.off_sel) + ((int64_t)slot * L.nqb + I) * L.nkw;
    const int ncand = (kind == DSA_KIND_MOBA) ? I : I + 1;
    int count = 0;
    if (kind == DSA_KIND_UNIFIED) {
      // row-normalised weights P_IJ = exp(s_IJ - max) / sum, written over the
      // row's scores for the CTA's column and diagonal sums below; the row's own
      // blocks are those with s_IJ >= max + ln(alpha) (the threshold rule)
      float mx = -INFINITY;
      for (int J = lane; J < ncand; J += 32) mx = fmaxf(mx, row[J]);
      mx = warp_max(mx);
      float sum = 0.f;
      for (int J = lane; J < ncand; J += 32) sum += __expf(row[J] - mx);
      sum = warp_sum(sum);
      const float thr = mx + ht.lnalpha[h];
      const float inv = 1.f / sum;
      float* prow = sc + rr * SEL_RS(npad);
      for (int w0 = 0; w0 <= (I >> 5); ++w0) {
        const int J = w0 * 32 + lane;
        bool keep = J < ncand && row[J] >= thr;
        if (J == 0 && ht.keep_sink[h]) keep = true;
        if (J == I && ht.keep_local[h]) keep = true;
        const float pj = J < ncand ? __expf(row[J] - mx) * inv : 0.f;
        __syncwarp();
        prow[J] = pj;
        const unsigned bits = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) sel[w0] = bits;
        count += __popc(bits);
      }
    } else if (kind == DSA_KIND_BLOCK_THRESHOLD) {
      float mx = -INFINITY;
      for (int J = lane; J < ncand; J += 32) mx = fmaxf(mx, row[J]);
      mx = warp_max(mx);
      const float thr = mx + ht.lnalpha[h];
      for (int w0 = 0; w0 <= (I >> 5); ++w0) {
        const int J = w0 * 32 + lane;
        bool keep = J < ncand && row[J] >= thr;
        if (J == 0 && ht.keep_sink[h]) keep = true;
        if (J == I && ht.keep_local[h]) keep = true;
        const unsigned bits = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) sel[w0] = bits;
        count += __popc(bits);
      }
    } else {
      const int k = ht.topk[h];
      uint32_t T = 0;
      int take_eq = 0;
      const bool all = ncand <= k;
      if (!all && k > 0) warp_radix_kth(row, ncand, k, hist[warp], &T, &take_eq);
      int eq_run = 0;
      for (int w0 = 0; w0 <= (I >> 5); ++w0) {
        const int J = w0 * 32 + lane;
        bool keep = false, iseq = false;
        if (J < ncand && k > 0) {
          if (all) {
            keep = true;
          } else {
            const uint32_t key = fkey(row[J]);
            keep = key > T;
            iseq = key == T;
          }
        }
        const unsigned eqm = __ballot_sync(0xffffffffu, iseq);
        if (iseq && eq_run + __popc(eqm & ((1u << lane) - 1u)) < take_eq) keep = true;
        eq_run += __popc(eqm);
        if (kind == DSA_KIND_MOBA && J == I) keep = true;
        const unsigned bits = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) sel[w0] = bits;
        count += __popc(bits);
      }
    }
    if (lane == 0) blk_ptr[1 + h * L.nqb + I] = count;
  }
  if (kind == DSA_KIND_UNIFIED) {
    // this CTA's share of the vertical sums V_J = sum_I P_IJ and diagonal sums
    // G_d = sum_I P_{I, I-d}, over its rows in ascending order (k_unified_merge
    // adds the CTAs' shares in ascending order: the same sums on every run)
    __syncthreads();
    float* up = reinterpret_cast<float*>(ws + L.off_upart) +
                ((int64_t)ht.uslot[h] * L.sel_nx + blockIdx.x) * 2 * L.nqb;
    for (int x = tid; x < L.nqb; x += SEL_NT) {
      float v = 0.f, gd = 0.f;
      for (int rr = 0; rr < nI; ++rr) {
        const int I = I0 + rr;
        if (x <= I) {
          v += sc[rr * SEL_RS(npad) + x];
          gd += sc[rr * SEL_RS(npad) + (I - x)];
        }
      }
      up[x] = v;
      up[L.nqb + x] = gd;
    }
  }
}

__device__ __forceinline__ uint32_t low_mask_upto(int n) {  // bits 0..n (n in 0..31)
  return n >= 31 ? 0xffffffffu : ((2u << n) - 1u);
}

// Unified discovery, per head: adds the CTAs' shares of the vertical and
// diagonal sums (ascending CTA order), keeps the verticals V_J >= alpha max V
// and diagonals G_d >= alpha max G, and adds to every query block's selection
// the verticals J <= I and the blocks I - d of the diagonals d <= I; the row
// counts are rewritten.  The kept verticals and diagonals are also written,
// ascending and -1 padded, to the vertical / slash lists of the head.
__global__ void __launch_bounds__(1024) k_unified_merge(const __grid_constant__ HeadTab ht, Layout L, uint8_t* ws,
                                                        int32_t* blk_ptr, int32_t* vert_idx, int vert_stride,
                                                        int32_t* slash_idx, int slash_stride) {
  pdl_prologue();
  extern __shared__ float um[];  // V[nqb], G[nqb], then the kept bitmaps as words
  const int uslot = blockIdx.x;
  const int h = ht.uhead[uslot];
  const int nqb = L.nqb;
  float* V = um;
  float* G = um + nqb;
  uint32_t* vb = reinterpret_cast<uint32_t*>(um + 2 * nqb);  // [nkw] vertical bits
  uint32_t* db = vb + L.nkw;                                  // [nkw] diagonal bits
  __shared__ float red[2][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* up = reinterpret_cast<const float*>(ws + L.off_upart) + (int64_t)uslot * L.sel_nx * 2 * nqb;
  float mv = 0.f, mg = 0.f;
  for (int x = tid; x < nqb; x += blockDim.x) {
    float v = 0.f, gd = 0.f;
    for (int c = 0; c < L.sel_nx; ++c) {
      v += up[(int64_t)c * 2 * nqb + x];
      gd += up[(int64_t)c * 2 * nqb + nqb + x];
    }
    V[x] = v;
    G[x] = gd;
    mv = fmaxf(mv, v);
    mg = fmaxf(mg, gd);
  }
  mv = warp_max(mv);
  mg = warp_max(mg);
  if (lane == 0) {
    red[0][warp] = mv;
    red[1][warp] = mg;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    float a = lane < nw ? red[0][lane] : 0.f, b = lane < nw ? red[1][lane] : 0.f;
    a = warp_max(a);
    b = warp_max(b);
    if (lane == 0) {
      red[0][0] = a;
      red[1][0] = b;
    }
  }
  __syncthreads();
  // alpha in probability space: V_J >= alpha max V  <=>  V_J >= exp(ln alpha) max V
  const float alpha = __expf(ht.lnalpha[h]);
  const float tv = alpha * red[0][0], tg = alpha * red[1][0];
  for (int w0 = warp; w0 < L.nkw; w0 += blockDim.x >> 5) {
    const int x = w0 * 32 + lane;
    const unsigned bv = __ballot_sync(0xffffffffu, x < nqb && V[x] >= tv);
    const unsigned bd = __ballot_sync(0xffffffffu, x < nqb && G[x] >= tg);
    if (lane == 0) {
      vb[w0] = bv;
      db[w0] = bd;
    }
  }
  __syncthreads();
  // the kept lists, ascending (warp 0: verticals, warp 1: diagonals)
  if (warp < 2) {
    const uint32_t* bits = warp == 0 ? vb : db;
    int32_t* out = warp == 0 ? vert_idx + (int64_t)h * vert_stride : slash_idx + (int64_t)h * slash_stride;
    const int stride = warp == 0 ? vert_stride : slash_stride;
    int pos = 0;
    for (int w0 = 0; w0 < L.nkw; ++w0) {
      const uint32_t word = bits[w0];
      const int x = w0 * 32 + lane;
      const bool on = (word >> lane) & 1u;
      const int at = pos + __popc(word & ((1u << lane) - 1u));
      if (on && at < stride) out[at] = x;
      pos += __popc(word);
    }
    for (int i = pos + lane; i < stride; i += 32) out[i] = -1;
  }
  // rows: OR in the verticals J <= I and the diagonal blocks I - d (d <= I)
  uint32_t* sel0 = reinterpret_cast<uint32_t*>(ws + L.off_sel) + (int64_t)ht.bslot[h] * nqb * L.nkw;
  for (int I = warp; I < nqb; I += blockDim.x >> 5) {
    uint32_t* sel = sel0 + (int64_t)I * L.nkw;
    int count = 0;
    for (int w0 = 0; w0 <= (I >> 5); ++w0) {
      const int J = w0 * 32 + lane;
      const int dd = I - J;  // J = I - d
      bool keep = J <= I && (((vb[w0] >> lane) & 1u) || (dd >= 0 && ((db[dd >> 5] >> (dd & 31)) & 1u)));
      const unsigned add = __ballot_sync(0xffffffffu, keep);
      uint32_t word = sel[w0];
      word |= add;
      if (w0 == (I >> 5)) word &= low_mask_upto(I & 31);  // candidates J <= I only
      if (lane == 0) sel[w0] = word;
      count += __popc(word);
    }
    if (lane == 0) blk_ptr[1 + h * nqb + I] = count;
  }
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Waits, bounded by the default limit and ignoring the abort flag, for a
// phase to complete (loads or MMAs this CTA issued, before it exits).
static __device__ __noinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// ---------------------------------------------------------------------------
// VS estimate on the tensor cores.  One CTA per (row tile, key chunk): a row
// tile stacks the estimate rows of up to two VS q-heads of one KV group (64
// rows each, or one head of up to 128 rows) into one 128-row operand, so a K
// sub-tile loaded once by TMA feeds both heads.  Per 128-key sub-tile one
// elected thread issues the product into tensor memory (two 128-column buffers,
// so the next product overlaps the work on this one):
//   PASS 1: S = Qrows K^T (lane = row): running max and sum of 2^(x - max) per
//           row over the chunk -> per-chunk partials (merged by k_vs_rowstats);
//   PASS 2: S^T = K Qrows^T (lane = key): p = 2^(x - m_i - log2 l_i) for every
//           row i; v[j] is a sum over the thread's own values.  s[o] is
//           summed along the diagonals of each warp's 32-key x 64-row block by
//           a register that moves up one lane per row (a diagonal enters at
//           lane 0 and is complete when it leaves lane 31), written once into
//           the warp's window and merged in a fixed order into the chunk's window
//           of offsets (no atomics: the sums are the same bit for bit on every run).
// x = tau log2(e) q.k, so every exponential is one ex2.  Warp 0 issues the TMA
// loads, warp 1 the MMAs; eight compute warps: two per TMEM lane quadrant, each
// taking one half (64) of the 128 columns.
// ---------------------------------------------------------------------------
// One lane waits (suspended in try_wait), the warp learns the outcome.
__device__ __forceinline__ bool vt_warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit, unsigned* status,
                                             unsigned detail, volatile int* abort_flag) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_ool(bar, parity, limit, status, detail, abort_flag, true) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}
// Named barrier over n threads that also returns whether `pred` held on all of
// them, so that the warps of a group leave a loop together.
__device__ __forceinline__ bool named_barrier_and(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

constexpr int VT_COMPUTE = 256;             // eight compute warps
constexpr int VT_THREADS = 64 + VT_COMPUTE;
constexpr int VT_ROWS = 128;                // rows of a row tile (the MMA's M or N)
constexpr int VT_HALF = 64;                 // columns per compute warp
constexpr int VT_SLAB = 128 * 128;          // bytes of one 128-row x 64-column bf16 slab
constexpr int VT_WW = VT_ROWS + 32;         // per-warp window

struct VsTiles {
  int n;
  int h0[MAXH];  // first q-head of the tile
  int h1[MAXH];  // second q-head (-1: the tile holds one head)
  int lp[MAXH];  // rows per head slot: 64 (two heads) or 128 (one head)
};

template <int D>
struct VtSmem {
  static constexpr int DS = D / 64;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = DS * VT_SLAB;                  // two stages
  static constexpr int BAR_OFF = K_OFF + 2 * DS * VT_SLAB;    // 10 barriers
  static constexpr int MISC_OFF = BAR_OFF + 10 * 8;           // [0] tmem base, [1] abort
  static constexpr int ROWM_OFF = MISC_OFF + 16;              // float [VT_ROWS]: m_i + log2 l_i (pass 2)
  static constexpr int VSUM_OFF = ROWM_OFF + VT_ROWS * 4;     // float [VT_ROWS] (pass 2)
  // pass 2: float [8 warps][VT_WW] windows; pass 1: float [2][2][VT_ROWS] row partials
  static constexpr int WIN_OFF = VSUM_OFF + VT_ROWS * 4;
  static constexpr int CWIN_OFF = WIN_OFF + 8 * VT_WW * 4;    // float [2 slots][chunk + VT_ROWS]
  static int bytes(int chunk) { return CWIN_OFF + 2 * (chunk + VT_ROWS) * 4 + 1024; }
};
static_assert(8 * VT_WW >= 4 * VT_ROWS, "pass-1 partials fit in the window area");
enum { VB_QFULL = 0, VB_KFULL = 1, VB_KEMPTY = 3, VB_SFULL = 5, VB_SEMPTY = 7, VB_DRAIN = 9 };

template <int D, int PASS>
__global__ void __launch_bounds__(VT_THREADS, 2)
k_vs_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
        const __grid_constant__ HeadTab ht, const __grid_constant__ VsTiles vt, Layout L, uint8_t* ws,
        unsigned* status, uint64_t limit) {
  pdl_prologue();
  using S = VtSmem<D>;
  constexpr int DS = S::DS;
  extern __shared__ uint8_t vt_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(vt_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::BAR_OFF);
  int* misc = reinterpret_cast<int*>(sm + S::MISC_OFF);
  volatile int* abort_flag = misc + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x % vt.n;
  const int chunk = blockIdx.x / vt.n;
  const int CHK = L.vs_chunk;
  const int j0 = chunk * CHK;
  const int j1 = min(L.N, j0 + CHK);
  const int nsub = (j1 - j0 + VT_ROWS - 1) / VT_ROWS;
  const int LP = vt.lp[tile];
  const int hs[2] = {vt.h0[tile], vt.h1[tile]};
  const int kvh = hs[0] / L.G;

  if (tid == 0) {
    for (int i = 0; i < 10; ++i) mbar_init(&bars[i], (i == VB_SEMPTY || i == VB_SEMPTY + 1) ? 8 : 1);
    fence_barrier_init();
    misc[1] = 0;
  }
  if (warp == 1) {
    tmem_alloc(reinterpret_cast<uint32_t*>(&misc[0]), 256);
    tc_fence_before();
  }
  if (tid == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // estimate rows: slot s holds rows [N - Lq, N - Lq + LP) of head hs[s]
      // (rows past N arrive as zeros and are masked)
      const int nslot = hs[1] >= 0 ? 2 : 1;
      mbar_arrive_expect_tx(&bars[VB_QFULL], DS * VT_SLAB);
      for (int s = 0; s < 2; ++s) {
        const int h = s < nslot ? hs[s] : hs[0];
        const int i0 = L.N - min(ht.last_q[h], L.N);
        for (int r = 0; r < (LP == 64 ? 1 : 2) && s * LP + r * 64 < VT_ROWS; ++r)
          for (int c = 0; c < DS; ++c)
            tma_load_3d(sm + S::Q_OFF + c * VT_SLAB + (s * LP + r * 64) * 128, &tmQ, &bars[VB_QFULL], c * 64,
                        i0 + r * 64, h);
      }
      int last[2] = {-1, -1};
      bool ok = true;
      for (int t = 0; t < nsub; ++t) {
        const int b = t & 1;
        if (t >= 2 && !mbar_wait_ool(&bars[VB_KEMPTY + b], ((t >> 1) - 1) & 1, limit, status, DETAIL_WAIT_EMPTY,
                                     abort_flag, true)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[VB_KFULL + b], DS * VT_SLAB);
        last[b] = t;
        for (int c = 0; c < DS; ++c)
          tma_load_3d(sm + S::K_OFF + (b * DS + c) * VT_SLAB, &tmK, &bars[VB_KFULL + b], c * 64,
                      j0 + t * VT_ROWS, kvh);
      }
      if (!ok) {
        // a wait ran out: the loads this thread issued land before the CTA exits
        // (only this thread arms these barriers, so the parities are unambiguous)
        mbar_drain(&bars[VB_QFULL], 0);
        for (int b = 0; b < 2; ++b)
          if (last[b] >= 0) mbar_drain(&bars[VB_KFULL + b], (last[b] >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(VT_ROWS, VT_ROWS, 0, 0);
      const uint64_t qd = smem_desc(smem_u32(sm + S::Q_OFF), 16, 1024, SWZ_128B);
      bool ok = mbar_wait_ool(&bars[VB_QFULL], 0, limit, status, DETAIL_WAIT_Q, abort_flag, true);
      for (int t = 0; ok && t < nsub; ++t) {
        const int b = t & 1;
        const uint32_t use = (t >> 1) & 1;
        if (!mbar_wait_ool(&bars[VB_KFULL + b], use, limit, status, DETAIL_WAIT_K, abort_flag, true)) break;
        if (t >= 2 && !mbar_wait_ool(&bars[VB_SEMPTY + b], use ^ 1, limit, status, DETAIL_WAIT_SFREE, abort_flag, true))
          break;
        tc_fence_after();
        const uint64_t kd = smem_desc(smem_u32(sm + S::K_OFF + b * DS * VT_SLAB), 16, 1024, SWZ_128B);
        // pass 1: rows x keys (A = Q rows); pass 2: keys x rows (A = K)
        const uint64_t a0 = PASS == 1 ? qd : kd, b0 = PASS == 1 ? kd : qd;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)((kk >> 2) * (VT_SLAB >> 4) + (kk & 3) * 2);
          tc_mma_f16(tmem + 128 * b, a0 + off, b0 + off, IDESC, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[VB_SFULL + b]);
        tc_commit(&bars[VB_KEMPTY + b]);
      }
      tc_commit(&bars[VB_DRAIN]);
      mbar_drain(&bars[VB_DRAIN], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute
    const int cw = warp - 2;                  // 0..7
    const int q4 = warp & 3;                  // TMEM lane quadrant
    const int ch = cw >> 2;                   // column half: columns [64 ch, 64 ch + 64)
    const int lr = q4 * 32 + lane;            // this thread's TMEM lane
    const uint32_t col0 = (uint32_t)(VT_HALF * ch);
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sc = 1.4426950408889634f * rsqrtf((float)D);
    const int ctid = tid - 64;                // 0..255
    int lq[2], i0[2], vsl[2];
    for (int s = 0; s < 2; ++s) {
      const int h = hs[s];
      lq[s] = h >= 0 ? min(ht.last_q[h], L.N) : 0;
      i0[s] = L.N - lq[s];
      vsl[s] = h >= 0 ? ht.vslot[h] : 0;
    }
    float* rowm = reinterpret_cast<float*>(sm + S::ROWM_OFF);
    float* vsum = reinterpret_cast<float*>(sm + S::VSUM_OFF);
    float* wins = reinterpret_cast<float*>(sm + S::WIN_OFF);
    float* win = wins + cw * VT_WW;           // this warp's window (pass 2)
    float* cwin = reinterpret_cast<float*>(sm + S::CWIN_OFF);
    // pass 2: this warp's columns are rows [64 ch, 64 ch + 64) of the tile,
    // i.e. head slot wslot, its rows rr = rbase + c (c < 64)
    const int wslot = LP == 64 ? ch : 0;
    const int rbase = LP == 64 ? 0 : VT_HALF * ch;
    if (PASS == 2) {
      const float* stat = reinterpret_cast<const float*>(ws + L.off_stat);
      for (int r = ctid; r < VT_ROWS; r += VT_COMPUTE) {
        const int s = r / LP, rr = r % LP;
        const bool valid = s < 2 && hs[s] >= 0 && rr < lq[s];
        // p = 2^(x - m) / l = 2^(x - (m + log2 l)); rows outside the head: p = 0
        rowm[r] = valid ? stat[((int64_t)vsl[s] * VS_MAXL + rr) * 2 + 0] +
                              __log2f(stat[((int64_t)vsl[s] * VS_MAXL + rr) * 2 + 1])
                        : INFINITY;
      }
      for (int i = ctid; i < 8 * VT_WW; i += VT_COMPUTE) wins[i] = 0.f;
      for (int i = ctid; i < 2 * (CHK + VT_ROWS); i += VT_COMPUTE) cwin[i] = 0.f;
      named_barrier(1, VT_COMPUTE);
    }
    // pass 1 state: this thread's row, over its half of the columns
    const int ps = lr / LP, prr = lr % LP;
    const bool prow = PASS == 1 && ps < 2 && hs[ps] >= 0 && prr < lq[ps];
    const int pi = prow ? i0[ps] + prr : -1;
    float run_m = -INFINITY, run_l = 0.f;
    bool ok = true;
    for (int t = 0; t < nsub; ++t) {
      const int b = t & 1;
      const uint32_t use = (t >> 1) & 1;
      const int jt = j0 + t * VT_ROWS;  // first key of the sub-tile
      ok = vt_warp_wait(&bars[VB_SFULL + b], use, limit, status, DETAIL_WAIT_S, abort_flag);
      if (PASS == 2) ok = named_barrier_and(1, VT_COMPUTE, ok);  // the compute warps leave together
      if (!ok) break;
      tc_fence_after();
      float x[VT_HALF];
      tmem_ld32(tmem + lane_off + 128 * b + col0, x);
      tmem_ld32(tmem + lane_off + 128 * b + col0 + 32, x + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[VB_SEMPTY + b]);  // the buffer is free for sub-tile t + 2
      if (PASS == 1) {
        // row pi against keys jt + 64 ch + c: valid while j <= pi and j < j1
        const int nv = prow ? min(VT_HALF, min(pi + 1, j1) - (jt + VT_HALF * ch)) : 0;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < VT_HALF; ++c) {
          x[c] = c < nv ? x[c] * sc : -INFINITY;
          mx = fmaxf(mx, x[c]);
        }
        if (mx != -INFINITY) {
          if (mx > run_m) {
            run_l = (run_m == -INFINITY) ? 0.f : run_l * ex2_approx(run_m - mx);
            run_m = mx;
          }
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int c = 0; c < VT_HALF; c += 2) {
            s0 += ex2_approx(x[c] - run_m);
            s1 += ex2_approx(x[c + 1] - run_m);
          }
          run_l += s0 + s1;
        }
      } else {
        // key j = jt + lr against rows rr = rbase + c, c = 0..63, of head slot
        // wslot (estimate row i = i0 + rr); the pair counts when j <= i and
        // j < N.  Window index t = c - lane + 31 holds offset o = i - j: the
        // diagonal of (c, lane); dacc carries diagonal t in lane c - t + 31.
        const int j = jt + lr;
        const bool kv = j < j1;
        const int jlim = min(j1, jt + VT_ROWS) - 1;  // the sub-tile's last key
        const bool nomask = jlim <= i0[wslot] && jt + VT_ROWS <= j1;
        const int ilim = i0[wslot] + rbase;  // row of column c is ilim + c
        // two independent chains (columns 0..31 and 32..63) halve the serial
        // shuffle chain: chain A holds diagonals t = 0..62 (win[t]), chain B
        // t = 32..94 (win[64 + t - 32]); the merge adds both
        float va = 0.f, vb = 0.f, da = 0.f, db = 0.f;
        const float4* rm4 = reinterpret_cast<const float4*>(rowm + VT_HALF * ch);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 ma = rm4[c4], mb = rm4[8 + c4];
          const float mma[4] = {ma.x, ma.y, ma.z, ma.w}, mmb[4] = {mb.x, mb.y, mb.z, mb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = c4 * 4 + e;
            const bool oka = nomask || (kv && j <= ilim + c);
            const bool okb = nomask || (kv && j <= ilim + 32 + c);
            const float pa = oka ? ex2_approx(fmaf(x[c], sc, -mma[e])) : 0.f;
            const float pb = okb ? ex2_approx(fmaf(x[32 + c], sc, -mmb[e])) : 0.f;
            va += pa;
            vb += pb;
            da += pa;
            db += pb;
            if (lane == 31) {  // diagonals t = c (chain A) and t = 32 + c (chain B) are complete
              win[c] = da;
              win[64 + c] = db;
            }
            if (c + 1 < 32) {
              da = __shfl_up_sync(0xffffffffu, da, 1);
              db = __shfl_up_sync(0xffffffffu, db, 1);
              if (lane == 0) da = db = 0.f;  // diagonals t = c + 32, c + 64 start
            }
          }
        }
        if (lane < 31) {  // chain A: t = 32 .. 62; chain B: t = 64 .. 94
          win[62 - lane] = da;
          win[64 + 62 - lane] = db;
        }
        const float v = va + vb;
        float vtot = v;
        if (LP != 64) {
          // one head over both column halves: the two warps of a quadrant add
          // their key sums in a fixed order (half 0 + half 1)
          if (ch == 1) vsum[lr] = v;
          named_barrier(1, VT_COMPUTE);
          if (ch == 0) vtot = v + vsum[lr];
        }
        if (kv && (LP == 64 ? hs[wslot] >= 0 : ch == 0)) {
          float* vout = reinterpret_cast<float*>(ws + L.off_v);
          vout[(int64_t)vsl[wslot] * L.N + j] = LP == 64 ? v : vtot;
        }
        named_barrier(1, VT_COMPUTE);
        // merge the warps' windows into the chunk window in a fixed order.
        // Warp (ch, q4) covers keys jt + 32 q4 + lane and rows rbase(ch) + c;
        // its window index t holds chunk-window index
        // t + rbase(ch) + CHK - 32 - (jt - j0) - 32 q4 of slot wslot(ch).
        const int base = CHK - 32 - (jt - j0);
        const int nslot = LP == 64 ? 2 : 1;
        for (int e = ctid; e < nslot * (VT_ROWS + 128); e += VT_COMPUTE) {
          const int s = e / (VT_ROWS + 128);
          const int idx = base - 96 + (e % (VT_ROWS + 128));  // chunk-window index
          if ((LP == 64 && hs[s] < 0) || idx < 0 || idx >= CHK + VT_ROWS) continue;
          float acc = cwin[s * (CHK + VT_ROWS) + idx];
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            const int wch = w >> 2, wq = (w + 2) & 3;  // warp 2 + w: column half, quadrant
            const int ws_ = LP == 64 ? wch : 0;
            if (ws_ != s) continue;
            const int rb = LP == 64 ? 0 : VT_HALF * wch;
            const int tw = idx - (base + rb - 32 * wq);
            if (tw >= 0 && tw <= 62) acc += wins[w * VT_WW + tw];            // chain A
            if (tw >= 32 && tw <= 94) acc += wins[w * VT_WW + 64 + tw - 32];  // chain B
          }
          cwin[s * (CHK + VT_ROWS) + idx] = acc;
        }
        named_barrier(1, VT_COMPUTE);  // every entry t <= 94 is rewritten next sub-tile
      }
    }
    if (PASS == 1) {
      // the two column halves of each row: (m, l) pairs combined in a fixed order
      float* pm = wins;                 // [2][VT_ROWS] max
      float* pl = wins + 2 * VT_ROWS;   // [2][VT_ROWS] sum
      pm[ch * VT_ROWS + lr] = run_m;
      pl[ch * VT_ROWS + lr] = run_l;
      named_barrier(1, VT_COMPUTE);
      if (ch == 0 && prow) {
        const float m0 = pm[lr], m1 = pm[VT_ROWS + lr];
        const float m = fmaxf(m0, m1);
        float l = 0.f;
        if (m0 != -INFINITY) l += pl[lr] * ex2_approx(m0 - m);
        if (m1 != -INFINITY) l += pl[VT_ROWS + lr] * ex2_approx(m1 - m);
        float* part = reinterpret_cast<float*>(ws + L.off_part);
        float* pp = part + (((int64_t)vsl[ps] * L.vs_nchunks + chunk) * VS_MAXL + prr) * 2;
        pp[0] = m;
        pp[1] = l;
      }
    } else if (ok) {
      named_barrier(1, VT_COMPUTE);
      // this chunk's windows of slash sums (offset o at index o - (i0 - (j0 + CHK - 1)))
      for (int s = 0; s < (hs[1] >= 0 ? 2 : 1); ++s) {
        float* wout = reinterpret_cast<float*>(ws + L.off_spart) +
                      ((int64_t)vsl[s] * L.vs_nchunks + chunk) * (CHK + VS_MAXL);
        for (int t = ctid; t < CHK + VS_MAXL; t += VT_COMPUTE)
          wout[t] = (t < CHK + lq[s]) ? cwin[s * (CHK + VT_ROWS) + t] : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// s[o] of one VS head from the windows of the (at most two) key chunks whose
// keys meet offset o from the estimate rows, in ascending chunk order.
__global__ void __launch_bounds__(256) k_vs_slash_combine(const __grid_constant__ HeadTab ht, Layout L, uint8_t* ws) {
  pdl_prologue();
  const int vslot = blockIdx.y;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= L.N) return;
  const int h = ht.vhead[vslot];
  const int Lq = min(ht.last_q[h], L.N);
  const int i0 = L.N - Lq;
  const float* wins =
      reinterpret_cast<const float*>(ws + L.off_spart) + (int64_t)vslot * L.vs_nchunks * (L.vs_chunk + VS_MAXL);
  // chunk c holds the offsets (i0 - (c + 1) C, i0 + Lq - 1 - c C], C = L.vs_chunk
  const int hi = i0 + Lq - 1 - o;  // the largest key an estimate row meets at offset o
  float acc = 0.f;
  if (hi >= 0) {
    const int C = L.vs_chunk;
    const int c_hi = min(L.vs_nchunks - 1, hi / C);
    for (int c = max(0, c_hi - 1); c <= c_hi; ++c) {
      const int t = o - (i0 - (c * C + C - 1));
      if (t >= 0 && t < C + VS_MAXL) acc += wins[(int64_t)c * (C + VS_MAXL) + t];
    }
  }
  reinterpret_cast<float*>(ws + L.off_s)[(int64_t)vslot * L.N + o] = acc;
}

// merge the per-chunk (max, sum) partials (log2 units) into the row softmax statistics
__global__ void k_vs_rowstats(const __grid_constant__ HeadTab ht, Layout L, uint8_t* ws) {
  pdl_prologue();
  const int vslot = blockIdx.x;
  const int h = ht.vhead[vslot];
  const int Lq = min(ht.last_q[h], L.N);
  const float* part = reinterpret_cast<const float*>(ws + L.off_part);
  float* stat = reinterpret_cast<float*>(ws + L.off_stat);
  for (int r = threadIdx.x; r < Lq; r += blockDim.x) {
    float m = -INFINITY;
    for (int c = 0; c < L.vs_nchunks; ++c)
      m = fmaxf(m, part[(((int64_t)vslot * L.vs_nchunks + c) * VS_MAXL + r) * 2]);
    float l = 0.f;
    for (int c = 0; c < L.vs_nchunks; ++c) {
      const float* pp = part + (((int64_t)vslot * L.vs_nchunks + c) * VS_MAXL + r) * 2;
      if (pp[0] != -INFINITY) l += pp[1] * exp2f(pp[0] - m);
    }
    stat[((int64_t)vslot * VS_MAXL + r) * 2 + 0] = m;
    stat[((int64_t)vslot * VS_MAXL + r) * 2 + 1] = l;
  }
}

// Exact top-k of v (blockIdx.y == 0) or s (== 1) of one VS head, ascending, -1
// padded: one cluster of 1 to VT_CL CTAs per (head, array), each CTA owning a
// contiguous segment (one CTA for short arrays, where the cluster's exchanges
// cost more than its bandwidth gains).  Three radix passes of 12, 12 and 8 bits: each CTA counts
// its segment's keys that match the prefix so far into its own 4096-bin
// histogram; CTA 0 of the cluster adds the cluster's histograms through
// distributed shared memory, finds the digit holding the k-th key and hands it
// to every CTA.  Then each CTA counts its keys above the k-th and equal to it,
// learns the counts of the CTAs before it (again through distributed shared
// memory) and writes its selected keys at their ascending positions (ties go to
// the lower index, as in the CTA-wide select).
constexpr int VT_CL = 8;

// CTAs per top-k cluster for arrays of n keys
inline int vs_topk_cluster(int n) { return n <= (1 << 16) ? 1 : (n <= (1 << 18) ? 4 : VT_CL); }

template <typename Loader, typename Emit>
__device__ void ordered_select_range(const Loader& load, int beg_all, int end_all, uint32_t T, int take_eq,
                                     int eq_base0, int out_base0, int* red, const Emit& emit) {
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = end_all - beg_all;
  const int seg = ceil_div(ceil_div(max(n, 1), nw), 32) * 32;
  const int beg = beg_all + min(n, warp * seg), end = beg_all + min(n, warp * seg + seg);
  int gt = 0, eq = 0;
  for (int i = beg + lane; i < end; i += 32) {
    const uint32_t key = fkey(load(i));
    gt += key > T;
    eq += key == T;
  }
  gt = warp_sum_int(gt);
  eq = warp_sum_int(eq);
  if (lane == 0) {
    red[2 * warp] = gt;
    red[2 * warp + 1] = eq;
  }
  __syncthreads();
  int eq_run = eq_base0, gt_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += red[2 * w];
    eq_run += red[2 * w + 1];
  }
  __syncthreads();
  int pos = out_base0 + gt_before + min(eq_run, take_eq) - min(eq_base0, take_eq);
  for (int i0 = beg; i0 < end; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < end ? fkey(load(i)) : 0u;
    const bool iseq = i < end && key == T;
    bool sel = i < end && key > T;
    const unsigned eqm = __ballot_sync(0xffffffffu, iseq);
    if (iseq && eq_run + __popc(eqm & ((1u << lane) - 1u)) < take_eq) sel = true;
    eq_run += __popc(eqm);
    const unsigned sm = __ballot_sync(0xffffffffu, sel);
    if (sel) emit(i, pos + __popc(sm & ((1u << lane) - 1u)));
    pos += __popc(sm);
  }
}

__global__ void __launch_bounds__(1024) k_vs_topk(const __grid_constant__ HeadTab ht, Layout L, uint8_t* ws,
                                                  int32_t* vert_idx, int vert_stride, int32_t* slash_idx,
                                                  int slash_stride) {
  pdl_prologue();
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ int hist[RADIX_BINS];
  __shared__ int red[80];
  __shared__ int xfer[4];  // from CTA 0: digit, keys above it; segment counts gt, eq
  const int rank = (int)cluster.block_rank();
  const int ncl = (int)cluster.num_blocks();
  const int vslot = blockIdx.x / ncl;
  const int which = blockIdx.y;
  const int h = ht.vhead[vslot];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* arr = reinterpret_cast<const float*>(ws + (which == 0 ? L.off_v : L.off_s)) + (int64_t)vslot * L.N;
  const int k = min(which == 0 ? ht.n_vert[h] : ht.n_slash[h], L.N);
  int32_t* out = which == 0 ? vert_idx + (int64_t)h * vert_stride : slash_idx + (int64_t)h * slash_stride;
  const int stride = which == 0 ? vert_stride : slash_stride;
  const int seg = ceil_div(ceil_div(L.N, ncl), 32) * 32;
  const int beg = min(L.N, rank * seg), end = min(L.N, beg + seg);
  for (int i = k + rank * blockDim.x + tid; i < stride; i += ncl * blockDim.x) out[i] = -1;
  if (k <= 0) return;  // the whole cluster leaves together (k is the same for all)
  if (k >= L.N) {
    for (int i = beg + tid; i < end; i += blockDim.x) out[i] = i;
    return;
  }
  uint32_t prefix = 0, mask = 0;
  int need = k;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
    const uint32_t dmask = pass == 2 ? 0xffu : 0xfffu;
    for (int i = tid; i < RADIX_BINS; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i0 = beg; i0 < end; i0 += RB * blockDim.x) {
      uint32_t key[RB];
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        const int i = i0 + q * blockDim.x + tid;
        key[q] = (i < end) ? fkey(arr[i]) : 0u;
      }
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        const int i = i0 + q * blockDim.x + tid;
        if (i < end && (key[q] & mask) == prefix) atomicAdd(&hist[(key[q] >> shift) & dmask], 1);
      }
    }
    cluster.sync();  // every CTA's histogram is complete
    if (rank == 0) {
      // add the other CTAs' histograms into this one, then find the digit:
      // thread t takes bins RADIX_BINS-1-t*bpt downwards; an exclusive scan of
      // the per-thread sums is the count of keys in higher bins
      for (int r = 1; r < ncl; ++r) {
        const int* rh = cluster.map_shared_rank(hist, r);
        for (int i = tid; i < RADIX_BINS; i += blockDim.x) hist[i] += rh[i];
      }
      __syncthreads();
      const int bpt = RADIX_BINS / blockDim.x;
      const int top = RADIX_BINS - 1 - tid * bpt;
      int tot = 0;
      for (int q = 0; q < bpt; ++q) tot += hist[top - q];
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) red[2 + warp] = incl;
      __syncthreads();
      int above = incl - tot;
      for (int w = 0; w < warp; ++w) above += red[2 + w];
      if (above < need && above + tot >= need) {
        for (int q = 0; q < bpt; ++q) {
          const int c = hist[top - q];
          if (above + c >= need) {
            for (int r = 0; r < ncl; ++r) {
              int* rx = cluster.map_shared_rank(xfer, r);
              rx[0] = top - q;
              rx[1] = above;
            }
            break;
          }
          above += c;
        }
      }
    }
    cluster.sync();  // the digit is in every CTA's xfer; CTA 0 is done reading histograms
    prefix |= (uint32_t)xfer[0] << shift;
    mask |= dmask << shift;
    need -= xfer[1];
  }
  const uint32_t T = prefix;
  const int take_eq = need;
  // counts of the segments before this CTA's (none for a one-CTA cluster)
  int gt_before = 0, eq_before = 0;
  if (ncl > 1) {
    int gt = 0, eq = 0;
    for (int i = beg + tid; i < end; i += blockDim.x) {
      const uint32_t key = fkey(arr[i]);
      gt += key > T;
      eq += key == T;
    }
    gt = warp_sum_int(gt);
    eq = warp_sum_int(eq);
    if (lane == 0) {
      red[2 * warp] = gt;
      red[2 * warp + 1] = eq;
    }
    __syncthreads();
    if (tid == 0) {
      int g = 0, e = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        g += red[2 * w];
        e += red[2 * w + 1];
      }
      xfer[2] = g;
      xfer[3] = e;
    }
    cluster.sync();
    for (int r = 0; r < rank; ++r) {
      const int* rx = cluster.map_shared_rank(xfer, r);
      gt_before += rx[2];
      eq_before += rx[3];
    }
    cluster.sync();  // no CTA leaves while another may still read its counts
  }
  __syncthreads();
  auto load = [&](int i) { return arr[i]; };
  ordered_select_range(load, beg, end, T, take_eq, eq_before, gt_before + min(eq_before, take_eq), red,
                       [&](int i, int pos) { out[pos] = i; });
}

// block distances D of one VS head: {floor(o/B), ceil(o/B)} for the chosen
// slashes.  One flag byte per key block (plain stores: every writer writes 1),
// then one bitmap word per 32 blocks from a warp ballot, and the ascending list
// from a scan of the per-word counts.  Dynamic shared memory: nkw * 32 bytes.
// Slash runs of a VS_WINDOWS head (MInference summary, "3つの疎パターン": slash
// lines).  Query block qb (rows r0..r1, height L) reaches on slash o the keys
// i - o for r0 <= i <= r1, i >= o: the window [r0 - o, r1 - o] clipped at key 0,
// i.e. the offset interval [o, o + L - 1] mirrored at r1.  Windows of slashes
// closer than L + 1 touch, so a block's runs are the merged intervals of the
// dilated offsets, mirrored: one list per block height (every block has height
// B except a shorter last one).  Output (n, n_last = intervals of the two
// heights): out[0] = n, out[1] = n_last, out[2 + 2k] = a_k, out[3 + 2k] = b_k
// (k < n, ascending, disjoint, not touching), then the n_last intervals of the
// last block's height the same way; *len = 2 + 2 (n + n_last).  S (ascending, -1 padded) is the head's slash list.
// One CTA of up to 1024 threads.
__device__ void vs_runs(const HeadTab& ht, const Layout& L, const int32_t* S, int32_t* out, int32_t* len) {
  __shared__ int scan[96];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int h = ht.vhead[blockIdx.x];
  const int ns = min(ht.n_slash[h], L.N);
  const int last_h = L.N - (L.nqb - 1) * L.B;  // height of the last block
  int pos = 2;
  for (int pass = 0; pass < 2; ++pass) {
    const int Lh = pass == 0 ? L.B : last_h;
    int base = 0;  // intervals so far in this pass
    for (int k0 = 0; k0 < ns; k0 += blockDim.x) {
      const int k = k0 + tid;
      const int o = k < ns ? S[k] : -1;
      const int op = (k > 0 && k < ns) ? S[k - 1] : -1;
      const bool valid = o >= 0;
      // a new interval starts where the previous window ends more than one key
      // away: o > o_prev + L
      const bool start = valid && (k == 0 || op < 0 || o > op + Lh);
      const int on = (k + 1 < ns) ? S[k + 1] : -1;
      const bool end = valid && (k + 1 >= ns || on < 0 || on > o + Lh);
      // block-wide exclusive scan of `start`
      const unsigned bal = __ballot_sync(0xffffffffu, start);
      if (lane == 0) scan[warp] = __popc(bal);
      __syncthreads();
      if (warp == 0) {
        int c = lane < nw ? scan[lane] : 0;
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += y;
        }
        if (lane < nw) scan[32 + lane] = incl - c;
        if (lane == 31) scan[64] = incl;
      }
      __syncthreads();
      // interval index of k: intervals started before this chunk + those started
      // at or before k in it, minus one (k lies in the last one started)
      const int id = base + scan[32 + warp] + __popc(bal & ((2u << lane) - 1u)) - 1;
      if (start) out[pos + 2 * id] = o;
      if (end) out[pos + 2 * id + 1] = o + Lh - 1;
      base += scan[64];
      __syncthreads();
    }
    if (tid == 0) out[pass] = base;
    pos += 2 * base;
  }
  if (tid == 0) *len = pos;
}

__global__ void __launch_bounds__(1024) k_vs_dist(const __grid_constant__ HeadTab ht, Layout L, uint8_t* ws,
                                                  const int32_t* slash_idx, int slash_stride, int32_t* dist_ptr) {
  pdl_prologue();
  extern __shared__ uint8_t flag[];
  __shared__ int wofs[1025];  // nkw <= 1024 (N <= 2^21, B >= 64)
  const int vslot = blockIdx.x;
  const int h = ht.vhead[vslot];
  uint32_t* dbits = reinterpret_cast<uint32_t*>(ws + L.off_dbits) + (int64_t)vslot * L.nkw;
  int32_t* dtmp = reinterpret_cast<int32_t*>(ws + L.off_dtmp) + (int64_t)vslot * L.dtmp_stride;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (ht.kind[h] == DSA_KIND_VS_WINDOWS) {
    vs_runs(ht, L, slash_idx + (int64_t)h * slash_stride, dtmp, dist_ptr + 1 + h);
    return;
  }
  for (int i = threadIdx.x; i < L.nkw * 8; i += blockDim.x) reinterpret_cast<uint32_t*>(flag)[i] = 0u;
  __syncthreads();
  const int ns = min(ht.n_slash[h], L.N);
  for (int t = threadIdx.x; t < ns; t += blockDim.x) {
    const int o = slash_idx[(int64_t)h * slash_stride + t];
    if (o < 0) continue;
    const int lo = o / L.B, hi = (o + L.B - 1) / L.B;
    if (lo < L.nqb) flag[lo] = 1;
    if (hi < L.nqb) flag[hi] = 1;
  }
  __syncthreads();
  for (int w = warp; w < L.nkw; w += nw) {
    const unsigned bits = __ballot_sync(0xffffffffu, flag[w * 32 + lane] != 0);
    if (lane == 0) {
      dbits[w] = bits;
      wofs[w] = __popc(bits);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scan of the per-word counts
    int carry = 0;
    for (int w0 = 0; w0 < L.nkw; w0 += 32) {
      const int w = w0 + lane;
      const int c = (w < L.nkw) ? wofs[w] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (w < L.nkw) wofs[w] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) dist_ptr[1 + h] = carry;
  }
  __syncthreads();
  for (int w = warp; w < L.nkw; w += nw) {
    const bool f = flag[w * 32 + lane] != 0;
    const unsigned bits = __ballot_sync(0xffffffffu, f);
    if (f) dtmp[wofs[w] + __popc(bits & ((1u << lane) - 1u))] = w * 32 + lane;
  }
}

// Key j lies in a slash run of query block qb (last row r1) iff r1 - j falls in
// one of the block height's offset intervals (vs_runs layout; the last block
// may be shorter and has its own list): a binary search over ascending a_k.
__device__ __forceinline__ bool in_runs(const int32_t* runs, bool last_block, int r1, int j) {
  const int n = runs[0], n_last = runs[1];
  const int32_t* iv = runs + 2 + (last_block ? 2 * n : 0);
  const int m = last_block ? n_last : n;
  const int d = r1 - j;
  int lo = 0, hi = m;  // first interval with a > d
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (iv[2 * mid] <= d) lo = mid + 1; else hi = mid;
  }
  return lo > 0 && d <= iv[2 * (lo - 1) + 1];
}

// columns of (VS head, query block): j in V, j <= qb*B+B-1, (qb - j/B) not in D.
// One warp per query block, eight per CTA; the CTA stages the D bitmap and a
// window of the (ascending) vertical list in shared memory once for its warps.
// FILL=false writes counts, FILL=true writes lists.
template <bool FILL>
__global__ void __launch_bounds__(256) k_vs_cols(const __grid_constant__ HeadTab ht, Layout L, uint8_t* ws,
                                                 const int32_t* vert_idx, int vert_stride, int32_t* col_ptr,
                                                 int32_t* col_idx, int64_t col_cap, unsigned* status) {
  pdl_prologue();
  constexpr int WIN = 1024;
  __shared__ int32_t vwin[WIN];
  __shared__ uint32_t dsh[1024];  // nkw <= 1024
  const int vslot = blockIdx.y;
  const int h = ht.vhead[vslot];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x * 8 + warp;
  const int qb_last = min(L.nqb - 1, blockIdx.x * 8 + 7);
  const int lim_cta = qb_last * L.B + L.B - 1;
  const uint32_t* dbits = reinterpret_cast<const uint32_t*>(ws + L.off_dbits) + (int64_t)vslot * L.nkw;
  for (int w = threadIdx.x; w < L.nkw; w += blockDim.x) dsh[w] = dbits[w];
  const int32_t* V = vert_idx + (int64_t)h * vert_stride;
  const int nv = min(ht.n_vert[h], L.N);
  const int lim = qb * L.B + L.B - 1;
  const int lim_r1 = min(L.N - 1, lim);  // the block's last row
  const int row = h * L.nqb + qb;
  // VS_WINDOWS: the head's run intervals (vs_runs) replace the distance bitmap
  const int32_t* runs = ht.kind[h] == DSA_KIND_VS_WINDOWS
                            ? reinterpret_cast<const int32_t*>(ws + L.off_dtmp) + (int64_t)vslot * L.dtmp_stride
                            : nullptr;
  bool active = qb < L.nqb;
  int pos = 0;
  if (FILL && active) {
    pos = col_ptr[row];
    if (col_ptr[row + 1] > col_cap) {
      if (lane == 0) report(status, DSA_ERR_CAPACITY, DETAIL_CAP_COL);
      active = false;
    }
  }
  for (int c0 = 0; c0 < nv; c0 += WIN) {
    const int cn = min(WIN, nv - c0);
    __syncthreads();  // the previous window is consumed (and dsh is written)
    for (int t = threadIdx.x; t < cn; t += blockDim.x) vwin[t] = V[c0 + t];
    __syncthreads();
    if (active) {
      for (int t0 = 0; t0 < cn; t0 += 32) {
        const int t = t0 + lane;
        const int j = (t < cn) ? vwin[t] : -1;
        bool take = false;
        if (j >= 0 && j <= lim) {
          if (runs != nullptr) {
            take = !in_runs(runs, qb == L.nqb - 1, lim_r1, j);
          } else {
            const int delta = qb - j / L.B;
            take = !((dsh[delta >> 5] >> (delta & 31)) & 1u);
          }
        }
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (FILL && take) col_idx[pos + __popc(m & ((1u << lane) - 1u))] = j;
        pos += __popc(m);
        if (__shfl_sync(0xffffffffu, j, 31) > lim) {  // V is ascending
          active = false;
          break;
        }
      }
    }
    if (vwin[cn - 1] > lim_cta) break;  // no query block of this CTA reads further
  }
  if (!FILL && lane == 0 && qb < L.nqb) col_ptr[1 + row] = pos;
}

// in-place inclusive scan of ptr[0..n) (ptr[0] == 0, ptr[r+1] == count of row r)
__global__ void __launch_bounds__(1024) k_scan(int32_t* p0, int n0, int64_t cap0, int32_t* p1, int n1, int64_t cap1,
                                               int32_t* p2, int n2, int64_t cap2, unsigned* status) {
  pdl_prologue();
  __shared__ int wsum[32];
  int32_t* p = blockIdx.x == 0 ? p0 : (blockIdx.x == 1 ? p1 : p2);
  const int n = blockIdx.x == 0 ? n0 : (blockIdx.x == 1 ? n1 : n2);
  const int64_t cap = blockIdx.x == 0 ? cap0 : (blockIdx.x == 1 ? cap1 : cap2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = ceil_div(ceil_div(n, 32), 32) * 32;
  const int beg = min(n, warp * seg), end = min(n, beg + seg);
  // eight loads in flight per lane in both passes (the segment is too long for
  // shared memory at a million tokens)
  constexpr int U = 8;
  int s = 0;
  for (int i0 = beg; i0 < end; i0 += 32 * U) {
    int v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * 32 + lane;
      v[u] = (i < end) ? p[i] : 0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) s += v[u];
  }
  s = warp_sum_int(s);
  if (lane == 0) wsum[warp] = s;
  __syncthreads();
  int carry = 0;
  for (int w = 0; w < warp; ++w) carry += wsum[w];
  for (int i0 = beg; i0 < end; i0 += 32 * U) {
    int v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * 32 + lane;
      v[u] = (i < end) ? p[i] : 0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * 32 + lane;
      int x = v[u];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < end) p[i] = x + carry;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && n > 0 && (int64_t)p[n - 1] > cap) {
    const unsigned det = blockIdx.x == 0 ? DETAIL_CAP_BLK : (blockIdx.x == 1 ? DETAIL_CAP_COL : DETAIL_CAP_DIST);
    report(status, DSA_ERR_CAPACITY, det);
  }
}

// fill block lists: A-shape closed form, block kinds from the selection bitmap
__global__ void k_blk_fill(const __grid_constant__ HeadTab ht, Layout L, const uint8_t* ws, const int32_t* blk_ptr,
                           int32_t* blk_idx, int64_t blk_cap, unsigned* status) {
  pdl_prologue();
  const int h = blockIdx.y;
  const int kind = ht.kind[h];
  if (is_vs_kind(kind)) return;
  const int qb = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (qb >= L.nqb) return;
  const int row = h * L.nqb + qb;
  const int beg = blk_ptr[row], end = blk_ptr[row + 1];
  if (end > blk_cap) {
    if (lane == 0) report(status, DSA_ERR_CAPACITY, DETAIL_CAP_BLK);
    return;
  }
  if (kind == DSA_KIND_ASHAPE) {
    int a, w;
    ashape_range(qb, L.B, L.N, ht.sink[h], ht.window[h], &a, &w);
    const int w2 = max(w, a);
    const int n = a + max(0, qb + 1 - w2);
    for (int t = lane; t < n && beg + t < end; t += 32) blk_idx[beg + t] = (t < a) ? t : (w2 + t - a);
    return;
  }
  const uint32_t* sel = reinterpret_cast<const uint32_t*>(ws + L.off_sel) + ((int64_t)ht.bslot[h] * L.nqb + qb) * L.nkw;
  int pos = beg;
  const int nw = (qb >> 5) + 1;  // selected blocks satisfy J <= qb; later words are never written
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t bits = (w < nw) ? sel[w] : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int p = pos + incl - c;
    uint32_t b = bits;
    while (b) {
      const int bit = __ffs(b) - 1;
      b &= b - 1u;
      if (p < end) blk_idx[p] = w * 32 + bit;
      ++p;
    }
    pos += __shfl_sync(0xffffffffu, incl, 31);
  }
}

__global__ void k_dist_fill(const __grid_constant__ HeadTab ht, Layout L, const uint8_t* ws, const int32_t* dist_ptr,
                            int32_t* dist, int64_t dist_cap, unsigned* status) {
  pdl_prologue();
  const int vslot = blockIdx.x;
  const int h = ht.vhead[vslot];
  const int beg = dist_ptr[h], end = dist_ptr[h + 1];
  if (end > dist_cap) {
    if (threadIdx.x == 0) report(status, DSA_ERR_CAPACITY, DETAIL_CAP_DIST);
    return;
  }
  const int32_t* dtmp = reinterpret_cast<const int32_t*>(ws + L.off_dtmp) + (int64_t)vslot * L.dtmp_stride;
  for (int t = threadIdx.x; t < end - beg; t += blockDim.x) dist[beg + t] = dtmp[t];
}

// ---------------------------------------------------------------------------
// exact |M| per head (selected pairs), from the lists
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool sorted_contains(const int32_t* a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo < n && a[lo] == x;
}

__device__ __forceinline__ int64_t ashape_pairs_in_block(int kb, int B, int r0, int r1, int sink, int window) {
  // sum over rows i in [r0, r1] of |{j in block kb : j <= i, (j < sink or i - j < window)}|
  int64_t tot = 0;
  const int k0 = kb * B, k1 = kb * B + B - 1;
  for (int i = r0; i <= r1; ++i) {
    const int hi = min(k1, i);
    if (hi < k0) continue;
    // union of [k0, min(hi, sink-1)] and [max(k0, i-window+1), hi]
    const int a_hi = min(hi, sink - 1);
    const int na = a_hi >= k0 ? a_hi - k0 + 1 : 0;
    const int b_lo = max(k0, i - window + 1);
    const int nb = hi >= b_lo ? hi - b_lo + 1 : 0;
    int overlap = 0;
    if (na > 0 && nb > 0) {
      const int olo = max(k0, b_lo), ohi = min(a_hi, hi);
      overlap = ohi >= olo ? ohi - olo + 1 : 0;
    }
    tot += na + nb - overlap;
  }
  return tot;
}

__global__ void k_count_pairs(int Hq, int N, int B, int nqb, const int32_t* head_info, const int32_t* blk_ptr,
                              const int32_t* blk_idx, const int32_t* dist_ptr, const int32_t* dist,
                              const int32_t* col_ptr, const int32_t* col_idx, int64_t blk_cap, int64_t dist_cap,
                              int64_t col_cap, unsigned long long* pairs, unsigned* status) {
  pdl_prologue();
  const int qb = blockIdx.x;
  const int h = blockIdx.y;
  const int kind = head_info[h * 4];
  const int sink = head_info[h * 4 + 1], window = head_info[h * 4 + 2];
  const int r0 = qb * B, r1 = min(N - 1, r0 + B - 1);
  const int nrows = r1 - r0 + 1;
  int64_t tot = 0;
  const int32_t* lst;
  int nl;
  int dsel = 0;
  // a row is used only if 0 <= beg <= end <= cap (else reported and counted empty)
  auto row_ok = [&](int beg, int end, int64_t cap, unsigned detail) {
    if (0 <= beg && beg <= end && (int64_t)end <= cap) return true;
    if (threadIdx.x == 0) report(status, DSA_ERR_DEVICE, detail);
    return false;
  };
  const int32_t* runs = nullptr;  // VS_WINDOWS: the head's run intervals
  if (kind == DSA_KIND_VS_WINDOWS) {
    const int beg = dist_ptr[h], end = dist_ptr[h + 1];
    const bool ok = row_ok(beg, end, dist_cap, DETAIL_BAD_DISTPTR) && end - beg >= 2 &&
                    2 + 2 * ((int64_t)dist[beg] + dist[beg + 1]) == end - beg;
    if (!ok && end - beg >= 0 && threadIdx.x == 0) report(status, DSA_ERR_DEVICE, DETAIL_BAD_DISTPTR);
    runs = ok ? dist + beg : nullptr;
    lst = dist;
    nl = 0;
  } else if (kind == DSA_KIND_VS) {
    const int beg = dist_ptr[h], end = dist_ptr[h + 1];
    const bool ok = row_ok(beg, end, dist_cap, DETAIL_BAD_DISTPTR);
    lst = ok ? dist + beg : dist;
    nl = ok ? end - beg : 0;
    dsel = 1;
  } else {
    const int beg = blk_ptr[h * nqb + qb], end = blk_ptr[h * nqb + qb + 1];
    const bool ok = row_ok(beg, end, blk_cap, DETAIL_BAD_BLKPTR);
    lst = ok ? blk_idx + beg : blk_idx;
    nl = ok ? end - beg : 0;
  }
  for (int e = threadIdx.x; e < nl; e += blockDim.x) {
    const int kb = dsel ? qb - lst[e] : lst[e];
    if (kb < 0 || kb > qb) continue;
    if (e > 0 && (dsel ? lst[e - 1] == lst[e] : lst[e - 1] == lst[e])) continue;  // repeated entry
    if (kind == DSA_KIND_ASHAPE) {
      tot += ashape_pairs_in_block(kb, B, r0, r1, sink, window);
    } else if (kb < qb) {
      tot += (int64_t)nrows * B;
    } else {
      // diagonal block: row i sees keys r0 .. i
      tot += (int64_t)nrows * (nrows + 1) / 2;
    }
  }
  if (runs != nullptr) {
    // run [lo, hi] (keys) of this block: row i counts min(i, hi) - lo + 1 keys
    // when i >= lo, all hi - lo + 1 once i > hi
    const bool lastb = qb == nqb - 1;
    const int nr = lastb ? runs[1] : runs[0];
    const int32_t* iv = runs + 2 + (lastb ? 2 * runs[0] : 0);
    for (int k = threadIdx.x; k < nr; k += blockDim.x) {
      const int hi = r1 - iv[2 * k], lo = max(0, r1 - iv[2 * k + 1]);
      if (hi < lo) continue;
      const int64_t x0 = max(r0, lo) - lo + 1, x1 = min(r1, hi) - lo + 1;
      if (x1 >= x0) tot += (x0 + x1) * (x1 - x0 + 1) / 2;
      const int64_t full_rows = max(0, r1 - max(r0, hi + 1) + 1);
      tot += full_rows * (hi - lo + 1);
    }
  }
  int cb = col_ptr[h * nqb + qb], ce = col_ptr[h * nqb + qb + 1];
  if (!row_ok(cb, ce, col_cap, DETAIL_BAD_COLPTR)) cb = ce = 0;
  for (int e = cb + threadIdx.x; e < ce; e += blockDim.x) {
    const int j = col_idx[e];
    if (j < 0 || j > r1) continue;
    const int kb = j / B;
    const bool covered = runs != nullptr ? in_runs(runs, qb == nqb - 1, r1, j)
                                         : (dsel ? sorted_contains(lst, nl, qb - kb) : sorted_contains(lst, nl, kb));
    if (covered) continue;
    tot += r1 - max(j, r0) + 1;
  }
  __shared__ unsigned long long sh[32];
  unsigned long long v = (unsigned long long)tot;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += sh[i];
    atomicAdd(&pairs[h], s);
  }
}

// ---------------------------------------------------------------------------
// host planning
// ---------------------------------------------------------------------------
dsa_status check_pattern(const dsa_problem& p, const dsa_pattern& q) {
  switch (q.kind) {
    case DSA_KIND_ASHAPE:
      if (q.sink < 0 || q.window < 1) return DSA_ERR_INVALID_ARG;
      return DSA_OK;
    case DSA_KIND_VS:
    case DSA_KIND_VS_WINDOWS:
      if (q.last_q < 1 || q.n_vert < 0 || q.n_slash < 0) return DSA_ERR_INVALID_ARG;
      if (q.last_q > VS_MAXL) return DSA_ERR_UNSUPPORTED;
      return DSA_OK;
    case DSA_KIND_BLOCK_TOPK:
      if (q.topk < 1) return DSA_ERR_INVALID_ARG;
      return DSA_OK;
    case DSA_KIND_BLOCK_THRESHOLD:
    case DSA_KIND_UNIFIED:
      if (!(q.alpha > 0.f && q.alpha <= 1.f)) return DSA_ERR_INVALID_ARG;
      return DSA_OK;
    case DSA_KIND_MOBA:
      if (q.topk < 0 || q.conv_width < 0 || q.conv_width > 8) return DSA_ERR_INVALID_ARG;
      if (q.conv_width > 0 && (q.conv_weight == nullptr || q.conv_bias == nullptr)) return DSA_ERR_INVALID_ARG;
      return DSA_OK;
    default:
      return DSA_ERR_INVALID_ARG;
  }
  (void)p;
}

bool is_block_kind(int k) {
  return k == DSA_KIND_BLOCK_TOPK || k == DSA_KIND_BLOCK_THRESHOLD || k == DSA_KIND_MOBA || k == DSA_KIND_UNIFIED;
}

int vs_rows_pad(int lq) {
  int rt = 1;
  while (rt * 16 < lq) rt *= 2;
  return rt;
}

// Key chunk of the VS estimate.  Its grid is one CTA per (VS head, chunk), two
// resident per SM.  When 1024-key chunks leave SMs idle (fewer CTAs than
// slots), the smallest chunk whose grid still fits in one wave is used: more
// CTAs, each with less to do (4K tokens, one VS head: 0.070 -> 0.057 ms of index
// build).  From one wave up 1024 stays: per-CTA costs (Q rows, statistics, the
// window write) outweigh the shorter tail (32K tokens, 20 VS heads, 768-key
// chunks: 0.340 -> 0.362 ms).
int choose_vs_chunk(int nvs, int N, int sms) {
  const int64_t slots = 2 * (int64_t)std::max(sms, 1);
  if ((int64_t)nvs * ceil_div(N, VS_CHUNK_MAX) >= slots) return VS_CHUNK_MAX;
  for (int i = 2; i >= 1; --i)
    if ((int64_t)nvs * ceil_div(N, VS_CHUNKS[i]) <= slots) return VS_CHUNKS[i];
  return VS_CHUNK_MAX;
}

dsa_status make_layout(const dsa_problem& p, const dsa_pattern* pats, Layout* L, HeadTab* ht, ConvTab* ct,
                       dsa_sizes* sz) {
  if (p.Hq > MAXH || p.Hkv > MAXKV) return DSA_ERR_UNSUPPORTED;
  L->Hq = p.Hq;
  L->Hkv = p.Hkv;
  L->G = p.Hq / p.Hkv;
  L->N = p.N;
  L->d = p.d;
  L->B = p.block;
  L->nqb = ceil_div(p.N, p.block);
  L->nkw = ceil_div(L->nqb, 32);
  L->nbh = 0;
  L->nvs = 0;
  L->nuh = 0;
  L->dtmp_stride = ceil_div(p.N, p.block);
  L->sel_ri = sel_blocks_per_cta(p.block);
  L->sel_nx = ceil_div(L->nqb, L->sel_ri);
  L->vs_lmax = 0;
  L->vs_chunk = VS_CHUNK_MAX;  // launch_build_indices may choose a smaller one
  L->vs_nchunks = ceil_div(p.N, VS_CHUNK_MAX);
  if (ht) memset(ht, 0, sizeof(HeadTab));
  if (ct) memset(ct, 0, sizeof(ConvTab));
  int64_t blk = 0, dcap = 0, ccap = 0;
  int vstride = 1, sstride = 1;
  const int nqb = L->nqb, B = p.block, N = p.N;
  for (int h = 0; h < p.Hq; ++h) {
    const dsa_pattern& q = pats[h];
    dsa_status s = check_pattern(p, q);
    if (s != DSA_OK) return s;
    if (ht) {
      ht->kind[h] = q.kind;
      ht->sink[h] = q.sink;
      ht->window[h] = q.window;
      ht->last_q[h] = q.last_q;
      ht->n_vert[h] = q.n_vert;
      ht->n_slash[h] = q.n_slash;
      ht->topk[h] = q.topk;
      ht->lnalpha[h] = (q.kind == DSA_KIND_BLOCK_THRESHOLD || q.kind == DSA_KIND_UNIFIED) ? logf(q.alpha) : 0.f;
      ht->keep_sink[h] = q.keep_sink;
      ht->keep_local[h] = q.keep_local;
      ht->bslot[h] = -1;
      ht->vslot[h] = -1;
      ht->uslot[h] = -1;
    }
    if (is_block_kind(q.kind)) {
      if (ht) {
        ht->bslot[h] = L->nbh;
        ht->bhead[L->nbh] = h;
        if (q.kind == DSA_KIND_UNIFIED) {
          ht->uslot[h] = L->nuh;
          ht->uhead[L->nuh] = h;
        }
      }
      L->nbh++;
      if (q.kind == DSA_KIND_UNIFIED) {
        L->nuh++;
        vstride = std::max(vstride, nqb);  // kept vertical blocks and diagonals
        sstride = std::max(sstride, nqb);
      }
      const int kvh = h / L->G;
      if (ct) {
        if (ct->need[kvh]) {
          const int w = q.kind == DSA_KIND_MOBA ? q.conv_width : 0;
          if (ct->width[kvh] != w || (w > 0 && (ct->w[kvh] != q.conv_weight || ct->b[kvh] != q.conv_bias)))
            return DSA_ERR_INVALID_ARG;  // block heads of one KV group must share the key conv
        } else {
          ct->need[kvh] = 1;
          ct->width[kvh] = q.kind == DSA_KIND_MOBA ? q.conv_width : 0;
          ct->w[kvh] = ct->width[kvh] ? q.conv_weight : nullptr;
          ct->b[kvh] = ct->width[kvh] ? q.conv_bias : nullptr;
        }
      }
      for (int qb = 0; qb < nqb; ++qb) {
        if (q.kind == DSA_KIND_BLOCK_TOPK) blk += std::min(q.topk, qb + 1);
        else if (q.kind == DSA_KIND_MOBA) blk += std::min(q.topk, qb) + 1;
        else blk += qb + 1;
      }
    } else if (q.kind == DSA_KIND_ASHAPE) {
      for (int qb = 0; qb < nqb; ++qb) {
        const int r0 = qb * B, r1 = std::min(N - 1, r0 + B - 1);
        const int a = ceil_div(std::min(q.sink, r1 + 1), B);
        const int w = std::max(0, r0 - q.window + 1) / B;
        blk += a + std::max(0, qb + 1 - std::max(w, a));
      }
    } else {  // VS
      if (ht) {
        ht->vslot[h] = L->nvs;
        ht->vhead[L->nvs] = h;
      }
      L->nvs++;
      const int nv = std::min(q.n_vert, N), ns = std::min(q.n_slash, N);
      vstride = std::max(vstride, nv);
      sstride = std::max(sstride, ns);
      if (q.kind == DSA_KIND_VS_WINDOWS) {
        // run list: [n, n_last, then n (a, b) offset intervals for full blocks,
        // then n_last for a shorter last block], each at most ns intervals
        dcap += 2 + 4 * (int64_t)ns;
        L->dtmp_stride = std::max<int>(L->dtmp_stride, 2 + 4 * ns);
      } else {
        dcap += std::min<int64_t>(2 * (int64_t)ns, nqb);
      }
      for (int qb = 0; qb < nqb; ++qb) ccap += std::min<int64_t>(nv, (int64_t)qb * B + B);
      L->vs_lmax = std::max(L->vs_lmax, 16 * vs_rows_pad(std::min(q.last_q, N)));
    }
  }
  if (blk > INT32_MAX || ccap > INT32_MAX || (int64_t)p.Hq * nqb + 1 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (L->nbh > 0 && L->nqb > 2048) return DSA_ERR_UNSUPPORTED;  // block scores of 16 rows live in shared memory
  const int64_t d = p.d;
  int64_t off = 0;
  L->off_kbar = off; off = align256(off + (L->nbh ? (int64_t)p.Hkv * nqb * d * 4 : 0));
  L->off_sel = off;  off = align256(off + (int64_t)L->nbh * nqb * L->nkw * 4);
  L->off_v = off;    off = align256(off + (int64_t)L->nvs * N * 4);
  L->off_s = off;    off = align256(off + (int64_t)L->nvs * N * 4);
  // the per-chunk regions are sized for the candidate chunk that needs the most
  int64_t vs_parts = 0, vs_wins = 0;
  for (int c : VS_CHUNKS) {
    vs_parts = std::max<int64_t>(vs_parts, ceil_div(N, c));
    vs_wins = std::max<int64_t>(vs_wins, (int64_t)ceil_div(N, c) * (c + VS_MAXL));
  }
  L->off_part = off; off = align256(off + (int64_t)L->nvs * vs_parts * VS_MAXL * 2 * 4);
  L->off_stat = off; off = align256(off + (int64_t)L->nvs * VS_MAXL * 2 * 4);
  L->off_dtmp = off; off = align256(off + (int64_t)L->nvs * L->dtmp_stride * 4);
  L->off_dbits = off; off = align256(off + (int64_t)L->nvs * L->nkw * 4);
  // per-chunk windows of the slash sums (chunk + VS_MAXL offsets each)
  L->off_spart = off; off = align256(off + (int64_t)L->nvs * vs_wins * 4);
  // unified discovery: each select CTA's shares of the vertical and diagonal sums
  L->off_upart = off; off = align256(off + (int64_t)L->nuh * L->sel_nx * 2 * nqb * 4);
  L->total = std::max<int64_t>(off, 256);
  if (sz) {
    sz->nqb = nqb;
    sz->vert_stride = vstride;
    sz->slash_stride = sstride;
    sz->reserved = 0;
    sz->head_info_len = 4 * (int64_t)p.Hq;
    sz->blk_ptr_len = (int64_t)p.Hq * nqb + 1;
    sz->blk_cap = std::max<int64_t>(blk, 1);
    sz->dist_ptr_len = p.Hq + 1;
    sz->dist_cap = std::max<int64_t>(dcap, 1);
    sz->col_ptr_len = (int64_t)p.Hq * nqb + 1;
    sz->col_cap = std::max<int64_t>(ccap, 1);
    sz->workspace_bytes = L->total;
  }
  return DSA_OK;
}

// Row tiles of the VS estimate: the VS q-heads of each KV group, two per tile
// when both estimate at most 64 rows, one otherwise.
void make_vs_tiles(const HeadTab& ht, const Layout& L, VsTiles* vt) {
  vt->n = 0;
  for (int g = 0; g < L.Hkv; ++g) {
    int pend = -1;  // a head of <= 64 rows waiting for a partner
    for (int h = g * L.G; h < (g + 1) * L.G; ++h) {
      if (!is_vs_kind(ht.kind[h])) continue;
      const int lq = std::min(ht.last_q[h], L.N);
      if (lq > 64) {
        vt->h0[vt->n] = h, vt->h1[vt->n] = -1, vt->lp[vt->n] = VT_ROWS, vt->n++;
      } else if (pend < 0) {
        pend = h;
      } else {
        vt->h0[vt->n] = pend, vt->h1[vt->n] = h, vt->lp[vt->n] = 64, vt->n++;
        pend = -1;
      }
    }
    if (pend >= 0) vt->h0[vt->n] = pend, vt->h1[vt->n] = -1, vt->lp[vt->n] = 64, vt->n++;
  }
}

template <int D>
dsa_status launch_vs(const HeadTab& ht, const VsTiles& vt, const Layout& L, const dsa_problem& p, const void* Q,
                     const void* K, uint8_t* ws, cudaStream_t st, unsigned* status) {
  CUtensorMap mq, mk;
  if (!make_tma_map_bf16_3d(&mq, Q, D, p.N, p.Hq, p.q_token_stride, p.q_head_stride, 64) ||
      !make_tma_map_bf16_3d(&mk, K, D, p.N, p.Hkv, p.k_token_stride, p.k_head_stride, VT_ROWS))
    return DSA_ERR_CUDA;
  const int smem = VtSmem<D>::bytes(L.vs_chunk);
  cudaError_t e = cudaFuncSetAttribute(k_vs_tc<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_vs_tc<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  const dim3 grid(L.vs_nchunks * vt.n);
  const uint64_t limit = wait_limit_ns();
  e = launch_pdl(k_vs_tc<D, 1>, grid, dim3(VT_THREADS), (size_t)smem, st, mq, mk, ht, vt, L, ws, status, limit);
  if (e == cudaSuccess) e = launch_pdl(k_vs_rowstats, dim3(L.nvs), dim3(128), 0, st, ht, L, ws);
  if (e == cudaSuccess)
    e = launch_pdl(k_vs_tc<D, 2>, grid, dim3(VT_THREADS), (size_t)smem, st, mq, mk, ht, vt, L, ws, status, limit);
  if (e == cudaSuccess)
    e = launch_pdl(k_vs_slash_combine, dim3(ceil_div(L.N, 256), L.nvs), dim3(256), 0, st, ht, L, ws);
  if (e != cudaSuccess) return cuda_fail(e);
  return DSA_OK;
}

}  // namespace

dsa_status plan_sizes(const dsa_problem& p, const dsa_pattern* pats, dsa_sizes* out) {
  static thread_local ConvTab ct;  // validates the per-group key conv as well
  Layout L;
  return make_layout(p, pats, &L, nullptr, &ct, out);
}

dsa_status launch_build_indices(const dsa_problem& p, const void* Q, const void* K, const dsa_pattern* pats,
                                const dsa_indices& out, void* ws_v, size_t ws_bytes, cudaStream_t st,
                                unsigned* status) {
  static thread_local HeadTab ht;
  static thread_local ConvTab ct;
  static thread_local VsTiles vt;
  Layout L;
  dsa_sizes sz;
  dsa_status s = make_layout(p, pats, &L, &ht, &ct, &sz);
  if (s != DSA_OK) return s;
  if ((int64_t)ws_bytes < sz.workspace_bytes) return DSA_ERR_CAPACITY;
  if (out.blk_cap < sz.blk_cap || out.dist_cap < sz.dist_cap || out.col_cap < sz.col_cap) return DSA_ERR_CAPACITY;
  if ((L.nvs > 0 || L.nuh > 0) && (!out.vert_idx || !out.slash_idx || out.vert_stride < sz.vert_stride ||
                                   out.slash_stride < sz.slash_stride))
    return DSA_ERR_CAPACITY;
  uint8_t* ws = static_cast<uint8_t*>(ws_v);
  const int nrows = p.Hq * L.nqb + 1;
  cudaError_t e;
  if (L.nvs > 0) {
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    make_vs_tiles(ht, L, &vt);
    L.vs_chunk = choose_vs_chunk(vt.n, p.N, sms);
    L.vs_nchunks = ceil_div(p.N, L.vs_chunk);
  }
#define DSA_CK(x)                          \
  do {                                     \
    e = (x);                               \
    if (e != cudaSuccess) return cuda_fail(e); \
  } while (0)
  // every kernel below starts with pdl_prologue(); the pointer arrays are
  // cleared by k_head_info / k_ashape_count where no count kernel writes them
  DSA_CK(launch_pdl(k_head_info, dim3(ceil_div(p.Hq, 128)), dim3(128), 0, st, ht, p.Hq, out.head_info, out.dist_ptr));
  DSA_CK(launch_pdl(k_ashape_count, dim3(ceil_div(L.nqb, 128), p.Hq), dim3(128), 0, st, ht, L, out.blk_ptr,
                    out.col_ptr));
  const auto* q = static_cast<const __nv_bfloat16*>(Q);
  const auto* k = static_cast<const __nv_bfloat16*>(K);
  if (L.nbh > 0) {
    if (p.d == 128) {
      DSA_CK(launch_pool<128>(ct, L, k, p.k_head_stride, p.k_token_stride, ws, st));
      const int ri = sel_blocks_per_cta(p.block);
      const size_t sel_smem = sel_smem_bytes(128, L.nkw);
      DSA_CK(cudaFuncSetAttribute(k_block_select<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem));
      DSA_CK(launch_pdl(k_block_select<128>, dim3(ceil_div(L.nqb, ri), L.nbh), dim3(SEL_NT), sel_smem, st, ht, L,
                        q, p.q_head_stride, p.q_token_stride, ws, out.blk_ptr, ri));
    } else {
      DSA_CK(launch_pool<64>(ct, L, k, p.k_head_stride, p.k_token_stride, ws, st));
      const int ri = sel_blocks_per_cta(p.block);
      const size_t sel_smem = sel_smem_bytes(64, L.nkw);
      DSA_CK(cudaFuncSetAttribute(k_block_select<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem));
      DSA_CK(launch_pdl(k_block_select<64>, dim3(ceil_div(L.nqb, ri), L.nbh), dim3(SEL_NT), sel_smem, st, ht, L,
                        q, p.q_head_stride, p.q_token_stride, ws, out.blk_ptr, ri));
    }
    if (L.nuh > 0) {
      const size_t um = (size_t)(2 * L.nqb + 2 * L.nkw) * 4;
      DSA_CK(launch_pdl(k_unified_merge, dim3(L.nuh), dim3(1024), um, st, ht, L, ws, out.blk_ptr, out.vert_idx,
                        out.vert_stride, out.slash_idx, out.slash_stride));
    }
  }
  if (L.nvs > 0) {
    s = (p.d == 128) ? launch_vs<128>(ht, vt, L, p, Q, K, ws, st, status)
                     : launch_vs<64>(ht, vt, L, p, Q, K, ws, st, status);
    if (s != DSA_OK) return s;
    const int ncl = vs_topk_cluster(p.N);
    DSA_CK(launch_pdl_cluster(k_vs_topk, dim3(L.nvs * ncl, 2), dim3(1024), ncl, st, ht, L, ws, out.vert_idx,
                              out.vert_stride, out.slash_idx, out.slash_stride));
    DSA_CK(launch_pdl(k_vs_dist, dim3(L.nvs), dim3(1024), (size_t)L.nkw * 32, st, ht, L, ws, out.slash_idx,
                      out.slash_stride, out.dist_ptr));
    DSA_CK(launch_pdl(k_vs_cols<false>, dim3(ceil_div(L.nqb, 8), L.nvs), dim3(256), 0, st, ht, L, ws, out.vert_idx,
                      out.vert_stride, out.col_ptr, out.col_idx, out.col_cap, status));
  }
  DSA_CK(launch_pdl(k_scan, dim3(3), dim3(1024), 0, st, out.blk_ptr, nrows, out.blk_cap, out.col_ptr, nrows,
                    out.col_cap, out.dist_ptr, p.Hq + 1, out.dist_cap, status));
  DSA_CK(launch_pdl(k_blk_fill, dim3(ceil_div(L.nqb, 8), p.Hq), dim3(256), 0, st, ht, L,
                    static_cast<const uint8_t*>(ws), static_cast<const int32_t*>(out.blk_ptr), out.blk_idx,
                    out.blk_cap, status));
  if (L.nvs > 0) {
    DSA_CK(launch_pdl(k_dist_fill, dim3(L.nvs), dim3(256), 0, st, ht, L, static_cast<const uint8_t*>(ws),
                      static_cast<const int32_t*>(out.dist_ptr), out.dist, out.dist_cap, status));
    DSA_CK(launch_pdl(k_vs_cols<true>, dim3(ceil_div(L.nqb, 8), L.nvs), dim3(256), 0, st, ht, L, ws, out.vert_idx,
                      out.vert_stride, out.col_ptr, out.col_idx, out.col_cap, status));
  }
  DSA_CK(cudaGetLastError());
#undef DSA_CK
  return DSA_OK;
}

dsa_status launch_count_pairs(const dsa_problem& p, const dsa_indices& idx, int64_t* pairs, cudaStream_t st,
                              unsigned* status) {
  const int nqb = ceil_div(p.N, p.block);
  cudaError_t e = cudaMemsetAsync(pairs, 0, sizeof(int64_t) * p.Hq, st);
  if (e != cudaSuccess) return cuda_fail(e);
  k_count_pairs<<<dim3(nqb, p.Hq), 128, 0, st>>>(p.Hq, p.N, p.block, nqb, idx.head_info, idx.blk_ptr, idx.blk_idx,
                                                 idx.dist_ptr, idx.dist, idx.col_ptr, idx.col_idx, idx.blk_cap,
                                                 idx.dist_cap, idx.col_cap,
                                                 reinterpret_cast<unsigned long long*>(pairs), status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return DSA_OK;
}

}  // namespace dsa
