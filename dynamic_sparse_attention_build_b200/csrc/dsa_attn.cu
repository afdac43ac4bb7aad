// Causal block-sparse attention forward for sm_100a.
//
// What it computes (MInference abstract: sparse attention "with the pattern and
// sparse indices"; FlashPrefill section 2.3: the kernel jumps straight to the
// listed blocks instead of testing every block): for row i of head h,
//   O_i = sum_{j in M_i} softmax_j(tau q_i.k_j) v_j,
// where M_i holds the keys j <= i of the key blocks listed for i's query block
// (CSR blocks, or qb - delta for the VS distances), plus its listed columns, and
// for A-shape heads only those with j < sink or i - j < window.
//
// Design (one CTA = 128 query rows of one head):
//   * the tile's two 64-row halves each belong to one query block (two different
//     blocks when B = 64, the same block otherwise).  Their key lists are turned
//     into two bitmaps over 64-key units in shared memory; the union is walked
//     in ascending order, two units (128 keys) per KV tile, and each unit carries
//     a 2-bit flag saying which half listed it (the other half masks it out);
//   * column lists are gathered into dense 128-key tiles (gather-and-densify);
//   * warp 0 issues TMA loads of K/V units (SWIZZLE_128B boxes of 64x64),
//     warps 0,2,3 gather column rows, warp 1 issues tcgen05.mma (S = Q K^T into
//     a double-buffered TMEM tile, O += P V into a TMEM accumulator), warps 4-7
//     run the online softmax (one thread per row) and the epilogue;
//   * online softmax keeps a stale running max unless it grows by more than 2^8,
//     which avoids most O rescales and is exact after the final division.
// No cluster, no multicast; every wait is bounded (status word + early exit).
#include <cudaTypedefs.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int BM = 128;          // query rows per CTA
constexpr int UNIT = 64;         // keys per unit (TMA box rows)
constexpr int BN = 128;          // keys per KV tile (2 units)
constexpr int STAGES = 2;
constexpr int SLAB = 128 * 128;  // bytes of one 128-row x 64-column bf16 slab
constexpr int NTHREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

struct StageInfo {
  int type;      // 0 = two units, 1 = column tile
  int u0, u1;    // unit ids (type 0); u1 = -1 when the second slot is padding
  int flags0, flags1;  // half bits for u0/u1 (type 0) or the column tile (flags0)
  int ncols;     // valid columns (type 1)
  int pad[2];
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
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t k_hs, k_ts, v_hs, v_ts;
  __nv_bfloat16* O;
  int64_t o_hs, o_ts;
  float* lse;
  float scale_log2;
  unsigned* status;
  uint64_t wait_limit_ns;
};

template <int D>
struct Smem {
  static constexpr int DS = D / 64;  // 64-column slabs
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + DS * SLAB;
  static constexpr int V_OFF = K_OFF + STAGES * DS * SLAB;
  static constexpr int P_OFF = V_OFF + STAGES * DS * SLAB;
  static constexpr int COL_OFF = P_OFF + 2 * SLAB;
  static constexpr int INFO_OFF = COL_OFF + STAGES * BN * 4;
  static constexpr int BAR_OFF = INFO_OFF + STAGES * (int)sizeof(StageInfo);
  static constexpr int NBAR = 16;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BITS_OFF = MISC_OFF + 64;
  static int bytes(int nwords) { return BITS_OFF + 2 * nwords * 4 + 1024; }
};

// barrier slots
enum { B_QFULL = 0, B_KFULL = 1, B_VFULL = 3, B_EMPTY = 5, B_SFULL = 7, B_SFREE = 9, B_PFULL = 11,
       B_ODONE = 12, B_DRAIN = 13 };

// One lane waits, the whole warp learns the outcome (keeps warp-collective
// tcgen05 and shuffle instructions converged even when a wait runs out).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit, unsigned* status,
                                          unsigned detail, volatile int* abort_flag) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, limit, status, detail, abort_flag) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // byte offset inside a slab
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnArgs a) {
  using L = Smem<D>;
  constexpr int DS = L::DS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR_OFF);
  int* misc = reinterpret_cast<int*>(sm + L::MISC_OFF);
  // misc: [0] tmem base, [1] T total tiles, [2] abort, [3] unit count, [4] col count half0,
  //       [5] col count half1, [6] col base half0, [7] col base half1, [8] shared-list flag
  volatile int* abort_flag = misc + 2;
  uint32_t* bits0 = reinterpret_cast<uint32_t*>(sm + L::BITS_OFF);
  uint32_t* bits1 = bits0 + a.nwords;
  StageInfo* info = reinterpret_cast<StageInfo*>(sm + L::INFO_OFF);
  int* colsm = reinterpret_cast<int*>(sm + L::COL_OFF);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bid = blockIdx.x;
  const int h = bid % a.Hq;
  const int qt = a.n_qtiles - 1 - bid / a.Hq;  // heaviest (latest) tiles first
  const int kvh = h / a.G;
  const int kind = a.head_info[h * 4 + 0];
  const int sink = a.head_info[h * 4 + 1];
  const int window = a.head_info[h * 4 + 2];
  const int row0 = qt * BM;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < L::NBAR; ++i)
      mbar_init(&bars[i], (i == B_SFREE || i == B_SFREE + 1 || i == B_PFULL) ? 4u : 1u);
    fence_barrier_init();
    misc[2] = 0;
    misc[3] = 0;
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
  for (int i = tid; i < 2 * a.nwords; i += NTHREADS) bits0[i] = 0u;
  __syncthreads();
  tc_fence_after();

  // query block and last row of each half
  int qbh[2], r1h[2];
  bool live[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r0 = row0 + hh * 64;
    live[hh] = r0 < a.N;
    qbh[hh] = r0 / a.B;
    r1h[hh] = min(a.N - 1, r0 + 63);
  }
  const int upb = a.B / UNIT;  // units per block
  const bool shared_qb = live[1] && (qbh[0] == qbh[1]);
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    if (!live[hh]) continue;
    uint32_t* bits = hh ? bits1 : bits0;
    const int qb = qbh[hh];
    const int r1 = r1h[hh];
    if (kind == DSA_KIND_VS) {
      const int beg = a.dist_ptr[h], end = a.dist_ptr[h + 1];
      for (int e = beg + tid; e < end; e += NTHREADS) {
        const int delta = a.dist[e];
        if (delta < 0) { report(a.status, DSA_ERR_DEVICE, DETAIL_BAD_DIST); continue; }
        if (delta > qb) continue;
        const int kb = qb - delta;
        for (int u = kb * upb; u < kb * upb + upb; ++u)
          if (u * UNIT <= r1) atomicOr(&bits[u >> 5], 1u << (u & 31));
      }
    } else {
      const int r = h * a.nqb + qb;
      const int beg = a.blk_ptr[r], end = a.blk_ptr[r + 1];
      for (int e = beg + tid; e < end; e += NTHREADS) {
        const int kb = a.blk_idx[e];
        if (kb < 0 || kb >= a.nqb) { report(a.status, DSA_ERR_DEVICE, DETAIL_BAD_BLOCK); continue; }
        for (int u = kb * upb; u < kb * upb + upb; ++u)
          if (u * UNIT <= r1) atomicOr(&bits[u >> 5], 1u << (u & 31));
      }
    }
  }
  __syncthreads();
  {
    int cnt = 0;
    for (int w = tid; w < a.nwords; w += NTHREADS) cnt += __popc(bits0[w] | bits1[w]);
    cnt = warp_sum_int(cnt);
    if (lane == 0 && cnt) atomicAdd(&misc[3], cnt);
  }
  if (tid == 0) {
    int c0 = 0, c1 = 0, b0 = 0, b1 = 0;
    if (live[0]) {
      const int r = h * a.nqb + qbh[0];
      b0 = a.col_ptr[r];
      c0 = a.col_ptr[r + 1] - b0;
    }
    if (live[1] && !shared_qb) {
      const int r = h * a.nqb + qbh[1];
      b1 = a.col_ptr[r];
      c1 = a.col_ptr[r + 1] - b1;
    }
    misc[4] = c0; misc[5] = c1; misc[6] = b0; misc[7] = b1; misc[8] = shared_qb ? 1 : 0;
  }
  __syncthreads();
  const int n_units = misc[3];
  const int T_u = (n_units + 1) >> 1;
  const int ccount[2] = {misc[4], misc[5]};
  const int cbase[2] = {misc[6], misc[7]};
  const int cflags[2] = {misc[8] ? 3 : 1, 2};
  const int T_c0 = ceil_div(ccount[0], BN), T_c1 = ceil_div(ccount[1], BN);
  const int T = T_u + T_c0 + T_c1;

  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);
  const uint32_t tmem_O = tmem_base;
  const uint32_t q_addr = smem_u32(sm + L::Q_OFF);
  const uint64_t limit = a.wait_limit_ns;

  if (warp == 0 || warp == 2 || warp == 3) {
    // ------------------------------------------------------------ loaders
    const int ltid = (warp == 0 ? 0 : warp - 1) * 32 + lane;  // 0..95
    if (warp == 0 && lane == 0) {
      // Q tile
      mbar_arrive_expect_tx(&bars[B_QFULL], DS * SLAB);
      for (int c = 0; c < DS; ++c) tma_load_3d(sm + L::Q_OFF + c * SLAB, &tmQ, &bars[B_QFULL], c * 64, row0, h);
      // unit tiles
      int w = 0;
      uint32_t pend = (a.nwords > 0) ? (bits0[0] | bits1[0]) : 0u;
      auto next_unit = [&](int& fl) -> int {
        while (pend == 0u) {
          if (++w >= a.nwords) return -1;
          pend = bits0[w] | bits1[w];
        }
        const int b = __ffs(pend) - 1;
        pend &= pend - 1u;
        fl = (int)((bits0[w] >> b) & 1u) | ((int)((bits1[w] >> b) & 1u) << 1);
        return w * 32 + b;
      };
      for (int t = 0; t < T_u; ++t) {
        const int st = t % STAGES;
        if (!mbar_wait(&bars[B_EMPTY + st], ((t / STAGES) & 1) ^ 1, limit, a.status, DETAIL_WAIT_EMPTY, abort_flag)) break;
        int f0 = 0, f1 = 0;
        const int u0 = next_unit(f0);
        int u1 = next_unit(f1);
        if (u1 < 0) f1 = 0;
        info[st].type = 0;
        info[st].u0 = u0;
        info[st].u1 = u1;
        info[st].flags0 = f0;
        info[st].flags1 = f1;
        info[st].ncols = 0;
        const int ul = (u1 < 0) ? u0 : u1;
        uint8_t* kst = sm + L::K_OFF + st * DS * SLAB;
        uint8_t* vst = sm + L::V_OFF + st * DS * SLAB;
        mbar_arrive_expect_tx(&bars[B_KFULL + st], DS * SLAB);
        for (int c = 0; c < DS; ++c) {
          tma_load_3d(kst + c * SLAB, &tmK, &bars[B_KFULL + st], c * 64, u0 * UNIT, kvh);
          tma_load_3d(kst + c * SLAB + SLAB / 2, &tmK, &bars[B_KFULL + st], c * 64, ul * UNIT, kvh);
        }
        mbar_arrive_expect_tx(&bars[B_VFULL + st], DS * SLAB);
        for (int c = 0; c < DS; ++c) {
          tma_load_3d(vst + c * SLAB, &tmV, &bars[B_VFULL + st], c * 64, u0 * UNIT, kvh);
          tma_load_3d(vst + c * SLAB + SLAB / 2, &tmV, &bars[B_VFULL + st], c * 64, ul * UNIT, kvh);
        }
      }
    }
    __syncwarp();
    // column tiles: all 96 loader threads gather rows into the swizzled layout
    int t = T_u;
    bool go = true;
    for (int hh = 0; go && hh < 2; ++hh) {
      const int nt = hh ? T_c1 : T_c0;
      for (int ct = 0; ct < nt; ++ct, ++t) {
        const int st = t % STAGES;
        if (ltid == 0)
          misc[9] = mbar_wait(&bars[B_EMPTY + st], ((t / STAGES) & 1) ^ 1, limit, a.status, DETAIL_WAIT_EMPTY,
                              abort_flag) ? 1 : 0;
        named_barrier(1, 96);
        if (misc[9] == 0) { go = false; break; }
        const int first = cbase[hh] + ct * BN;
        const int nc = min(BN, ccount[hh] - ct * BN);
        uint8_t* kst = sm + L::K_OFF + st * DS * SLAB;
        uint8_t* vst = sm + L::V_OFF + st * DS * SLAB;
        constexpr int CH = D / 8;  // 16-byte chunks per row
        for (int i = ltid; i < BN * CH; i += 96) {
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
              const int cov = (int)((bits0[u >> 5] >> (u & 31)) & 1u) | ((int)((bits1[u >> 5] >> (u & 31)) & 1u) << 1);
              v = j | (cov << 24);
            }
            colsm[st * BN + slot] = v;
          }
          const int jr = j < 0 ? 0 : j;
          const uint4 kv = __ldg(reinterpret_cast<const uint4*>(a.K + kvh * a.k_hs + (int64_t)jr * a.k_ts) + ch);
          const uint4 vv = __ldg(reinterpret_cast<const uint4*>(a.V + kvh * a.v_hs + (int64_t)jr * a.v_ts) + ch);
          const uint32_t off = (ch >> 3) * SLAB + swz(slot, ch & 7);
          *reinterpret_cast<uint4*>(kst + off) = kv;
          *reinterpret_cast<uint4*>(vst + off) = vv;
        }
        fence_proxy_async_smem();
        named_barrier(1, 96);
        if (ltid == 0) {
          info[st].type = 1;
          info[st].u0 = -1;
          info[st].u1 = -1;
          info[st].flags0 = cflags[hh];
          info[st].flags1 = 0;
          info[st].ncols = nc;
          mbar_arrive(&bars[B_KFULL + st]);
          mbar_arrive(&bars[B_VFULL + st]);
        }
        named_barrier(1, 96);  // misc[9] is reused by the next tile
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, 0, 1);
      const uint32_t p_addr = smem_u32(sm + L::P_OFF);
      bool ok = mbar_wait(&bars[B_QFULL], 0, limit, a.status, DETAIL_WAIT_Q, abort_flag);
      auto issue_pv = [&](int u) -> bool {
        const int st = u % STAGES;
        if (!mbar_wait(&bars[B_PFULL], u & 1, limit, a.status, DETAIL_WAIT_P, abort_flag)) return false;
        if (!mbar_wait(&bars[B_VFULL + st], (u / STAGES) & 1, limit, a.status, DETAIL_WAIT_V, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm + L::V_OFF + st * DS * SLAB);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t ad = smem_desc(p_addr + (kk >> 2) * SLAB + (kk & 3) * 32, 16, 1024, SWZ_128B);
          const uint64_t bd = smem_desc(v_addr + kk * 2048, SLAB, 1024, SWZ_128B);
          tc_mma_f16(tmem_O, ad, bd, IDESC_PV, (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars[B_ODONE]);
        tc_commit(&bars[B_EMPTY + st]);
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % STAGES;
        const int b = t & 1;
        if (!mbar_wait(&bars[B_KFULL + st], (t / STAGES) & 1, limit, a.status, DETAIL_WAIT_K, abort_flag)) { ok = false; break; }
        if (t >= 2 && !mbar_wait(&bars[B_SFREE + b], ((t >> 1) & 1) ^ 1, limit, a.status, DETAIL_WAIT_SFREE, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm + L::K_OFF + st * DS * SLAB);
        const uint32_t s_tmem = tmem_base + 128 + 128 * b;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc(q_addr + (kk >> 2) * SLAB + (kk & 3) * 32, 16, 1024, SWZ_128B);
          const uint64_t bd = smem_desc(k_addr + (kk >> 2) * SLAB + (kk & 3) * 32, 16, 1024, SWZ_128B);
          tc_mma_f16(s_tmem, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[B_SFULL + b]);
        if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok && T > 0) issue_pv(T - 1);
      // drain every MMA this thread issued before TMEM is released
      tc_commit(&bars[B_DRAIN]);
      mbar_wait(&bars[B_DRAIN], 0, limit, a.status, DETAIL_WAIT_O, abort_flag);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = tid - 128;          // row within the tile == TMEM lane
    const int q4 = warp & 3;          // TMEM lane quadrant of this warp
    const int row = row0 + r;
    const int half = r >> 6;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    uint8_t* p_sm = sm + L::P_OFF;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    float s[BN];
    for (int t = 0; t < T; ++t) {
      const int st = t % STAGES;
      const int b = t & 1;
      if (!warp_wait(&bars[B_KFULL + st], (t / STAGES) & 1, limit, a.status, DETAIL_WAIT_K, abort_flag)) { ok = false; break; }
      const StageInfo si = info[st];
      if (!warp_wait(&bars[B_SFULL + b], (t >> 1) & 1, limit, a.status, DETAIL_WAIT_S, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_tmem = tmem_base + lane_off + 128 + 128 * b;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(s_tmem + c * 32, s + c * 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_SFREE + b]);
      // masks
      const int hbit = 1 << half;
      float mt = -INFINITY;
      if (si.type == 0) {
        const bool ok0 = (si.flags0 & hbit) != 0;
        const bool ok1 = (si.u1 >= 0) && ((si.flags1 & hbit) != 0);
        const int k0 = si.u0 * UNIT, k1 = si.u1 * UNIT;
        const bool full = ok0 && ok1 && (max(k0, k1) + UNIT - 1 <= row) && kind != DSA_KIND_ASHAPE;
        if (full) {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            s[c] *= a.scale_log2;
            mt = fmaxf(mt, s[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const int j = (c < UNIT) ? (k0 + c) : (k1 + c - UNIT);
            bool al = (c < UNIT) ? ok0 : ok1;
            al = al && (j <= row);
            if (kind == DSA_KIND_ASHAPE) al = al && (j < sink || row - j < window);
            s[c] = al ? s[c] * a.scale_log2 : -INFINITY;
            mt = fmaxf(mt, s[c]);
          }
        }
      } else {
        const bool okh = (si.flags0 & hbit) != 0;
        const int* cj = colsm + st * BN;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const int v = cj[c];
          const int j = v & 0xFFFFFF;
          const bool al = okh && (c < si.ncols) && (v >= 0) && !((v >> (24 + half)) & 1) && (j <= row);
          s[c] = al ? s[c] * a.scale_log2 : -INFINITY;
          mt = fmaxf(mt, s[c]);
        }
      }
      const float m_new = fmaxf(m, mt);
      const bool need = m_new > m + RESCALE_THRESHOLD;  // also true for the first finite max
      float alpha = 1.f;
      if (need) {
        alpha = exp2f(m - m_new);
        l *= alpha;
        m = m_new;
      }
      if (t > 0) {
        // P.V of the previous tile must be done before O is rescaled or P is overwritten
        if (!warp_wait(&bars[B_ODONE], (t - 1) & 1, limit, a.status, DETAIL_WAIT_O, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
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
          tmem_wait_st();
        }
      }
      // P = exp2(s - m), rounded to bf16, into the swizzled K-major P tile
      float lsum = 0.f;
      const bool dead = (m == -INFINITY);
#pragma unroll
      for (int c8 = 0; c8 < BN / 8; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = dead ? 0.f : exp2f(s[c8 * 8 + 2 * i] - m);
          const float p1 = dead ? 0.f : exp2f(s[c8 * 8 + 2 * i + 1] - m);
          lsum += p0 + p1;
          __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<uint32_t*>(&v2);
        }
        const uint32_t off = (c8 >> 3) * SLAB + swz(r, c8 & 7);
        *reinterpret_cast<uint4*>(p_sm + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PFULL]);
    }
    // epilogue
    const bool have = ok && T > 0;
    if (have) {
      if (!warp_wait(&bars[B_ODONE], (T - 1) & 1, limit, a.status, DETAIL_WAIT_O, abort_flag)) ok = false;
      tc_fence_after();
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    __nv_bfloat16* orow = a.O + h * a.o_hs + (int64_t)row * a.o_ts;
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
      if (row < a.N) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(o[v * 8 + 2 * i] * inv, o[v * 8 + 2 * i + 1] * inv);
            pk[i] = *reinterpret_cast<uint32_t*>(&v2);
          }
          *reinterpret_cast<uint4*>(orow + c * 32 + v * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    if (a.lse != nullptr && row < a.N)
      a.lse[(int64_t)h * a.N + row] = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    __syncwarp();
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

template <int D>
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
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.k_hs = p.k_head_stride;
  a.k_ts = p.k_token_stride;
  a.v_hs = p.v_head_stride;
  a.v_ts = p.v_token_stride;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_hs = p.o_head_stride;
  a.o_ts = p.o_token_stride;
  a.lse = lse;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  a.status = status;
  a.wait_limit_ns = kWaitLimitNs;
  int smem = Smem<D>::bytes(a.nwords);
  if (smem < 120 * 1024) smem = 120 * 1024;  // one CTA per SM: each CTA holds 512 TMEM columns
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  const int grid = a.n_qtiles * p.Hq;
  if (grid == 0) return DSA_OK;
  sparse_attn_kernel<D><<<grid, NTHREADS, smem, stream>>>(mq, mk, mv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return DSA_OK;
}

}  // namespace

dsa_status launch_sparse_attn(const dsa_problem& p, const void* Q, const void* K, const void* V,
                              const dsa_indices& idx, void* O, float* lse, cudaStream_t stream, unsigned* status) {
  if (p.d == 128) return launch_d<128>(p, Q, K, V, idx, O, lse, stream, status);
  if (p.d == 64) return launch_d<64>(p, Q, K, V, idx, O, lse, stream, status);
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
