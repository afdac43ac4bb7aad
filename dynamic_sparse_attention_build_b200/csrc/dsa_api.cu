// The C ABI: argument validation, the per-device status word, and dispatch to
// the kernel launchers.  Nothing here allocates device memory.
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

// Status words, kStatusSlots per device, each [0] first error code, [1] detail,
// [2] block, [3] spare.  A call uses the word of its stream's slot, so errors of
// work on one stream are not reported to a caller of another (unless their
// handles fall on the same slot).
constexpr int kStatusSlots = 64;
__device__ unsigned g_status[kStatusSlots * 4];

namespace {
thread_local int32_t t_last_cuda_error = 0;
constexpr int kMaxDevices = 64;
std::atomic<unsigned*> g_status_addr[kMaxDevices] = {};

int status_slot(cudaStream_t s) {
  uint64_t x = static_cast<uint64_t>(reinterpret_cast<uintptr_t>(s));
  x ^= x >> 29;
  x *= 0x9E3779B97F4A7C15ull;  // Fibonacci hashing of the handle value
  return static_cast<int>(x >> 58);  // top 6 bits: 0 .. 63
}
static_assert(kStatusSlots == 64, "status_slot returns 6 bits");

__global__ void selftest_wait_kernel(unsigned* status, uint64_t limit_ns) {
  pdl_prologue();
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives: phase 0 never completes
    fence_barrier_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_ns, status, DETAIL_WAIT_SELFTEST, &abort_flag);
  __syncthreads();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

namespace {
std::atomic<uint64_t> g_wait_limit{kWaitLimitNs};
}  // namespace

uint64_t wait_limit_ns() { return g_wait_limit.load(); }

dsa_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = (int32_t)e;
  return DSA_ERR_CUDA;
}

unsigned* status_ptr(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned* base = g_status_addr[dev].load();
  if (base == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    base = static_cast<unsigned*>(p);
    g_status_addr[dev].store(base);  // every thread that races here finds the same address
  }
  return base + 4 * status_slot(stream);
}

dsa_status validate_problem(const dsa_problem* p) {
  if (p == nullptr) return DSA_ERR_INVALID_ARG;
  if (p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv != 0 || p->N < 1) return DSA_ERR_INVALID_ARG;
  if (p->Hq > 4096) return DSA_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return DSA_ERR_UNSUPPORTED;
  if (p->block != 64 && p->block != 128 && p->block != 256 && p->block != 512) return DSA_ERR_INVALID_ARG;
  if (p->N > (1 << 21)) return DSA_ERR_UNSUPPORTED;
  const int64_t ts[4] = {p->q_token_stride, p->k_token_stride, p->v_token_stride, p->o_token_stride};
  const int64_t hs[4] = {p->q_head_stride, p->k_head_stride, p->v_head_stride, p->o_head_stride};
  for (int i = 0; i < 4; ++i) {
    if (ts[i] < p->d || ts[i] % 8 != 0) return DSA_ERR_INVALID_ARG;
    if (hs[i] < 0 || hs[i] % 8 != 0) return DSA_ERR_INVALID_ARG;
  }
  return DSA_OK;
}

dsa_status validate_indices_ptrs(const dsa_indices* idx, bool for_build) {
  if (idx == nullptr) return DSA_ERR_INVALID_ARG;
  if (!idx->head_info || !idx->blk_ptr || !idx->dist_ptr || !idx->col_ptr) return DSA_ERR_INVALID_ARG;
  if (idx->blk_cap < 0 || idx->dist_cap < 0 || idx->col_cap < 0) return DSA_ERR_INVALID_ARG;
  if ((idx->blk_cap > 0 && !idx->blk_idx) || (idx->dist_cap > 0 && !idx->dist) ||
      (idx->col_cap > 0 && !idx->col_idx))
    return DSA_ERR_INVALID_ARG;
  if (for_build && (idx->vert_stride < 0 || idx->slash_stride < 0)) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

}  // namespace dsa

using namespace dsa;

extern "C" {

dsa_status dsa_workspace_size(const dsa_problem* p, const dsa_pattern* pats, dsa_sizes* out) {
  dsa_status s = validate_problem(p);
  if (s != DSA_OK) return s;
  if (pats == nullptr || out == nullptr) return DSA_ERR_INVALID_ARG;
  return plan_sizes(*p, pats, out);
}

dsa_status dsa_build_indices(const dsa_problem* p, const void* Q, const void* K, const dsa_pattern* pats,
                             const dsa_indices* out, void* workspace, size_t workspace_bytes, dsa_stream stream) {
  dsa_status s = validate_problem(p);
  if (s != DSA_OK) return s;
  if (pats == nullptr || !Q || !K || !aligned16(Q) || !aligned16(K)) return DSA_ERR_INVALID_ARG;
  s = validate_indices_ptrs(out, true);
  if (s != DSA_OK) return s;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DSA_ERR_INVALID_ARG;
  unsigned* st = status_ptr((cudaStream_t)stream);
  if (st == nullptr) return cuda_fail(cudaGetLastError());
  return launch_build_indices(*p, Q, K, pats, *out, workspace, workspace_bytes, (cudaStream_t)stream, st);
}

dsa_status dsa_sparse_prefill(const dsa_problem* p, const void* Q, const void* K, const void* V,
                              const dsa_indices* idx, void* O, float* lse, dsa_stream stream) {
  dsa_status s = validate_problem(p);
  if (s != DSA_OK) return s;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return DSA_ERR_INVALID_ARG;
  s = validate_indices_ptrs(idx, false);
  if (s != DSA_OK) return s;
  unsigned* st = status_ptr((cudaStream_t)stream);
  if (st == nullptr) return cuda_fail(cudaGetLastError());
  return launch_sparse_attn(*p, Q, K, V, *idx, O, lse, (cudaStream_t)stream, st);
}

dsa_status dsa_count_pairs(const dsa_problem* p, const dsa_indices* idx, int64_t* pairs, dsa_stream stream) {
  dsa_status s = validate_problem(p);
  if (s != DSA_OK) return s;
  if (pairs == nullptr) return DSA_ERR_INVALID_ARG;
  s = validate_indices_ptrs(idx, false);
  if (s != DSA_OK) return s;
  unsigned* st = status_ptr((cudaStream_t)stream);
  if (st == nullptr) return cuda_fail(cudaGetLastError());
  return launch_count_pairs(*p, *idx, pairs, (cudaStream_t)stream, st);
}

dsa_status dsa_get_device_status(dsa_stream stream, int32_t* detail) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned* st = status_ptr((cudaStream_t)stream);
  if (st == nullptr) return cuda_fail(cudaGetLastError());
  unsigned host[4] = {0, 0, 0, 0};
  e = cudaMemcpy(host, st, sizeof(host), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (host[0] != 0) {
    const unsigned zero[4] = {0, 0, 0, 0};
    e = cudaMemcpy(st, zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (detail) *detail = (int32_t)host[1];
  switch (host[0]) {
    case 0: return DSA_OK;
    case DSA_ERR_CAPACITY: return DSA_ERR_CAPACITY;
    case DSA_ERR_TIMEOUT: return DSA_ERR_TIMEOUT;
    default: return DSA_ERR_DEVICE;
  }
}

dsa_status dsa_selftest_wait_timeout(uint32_t timeout_us, dsa_stream stream) {
  if (timeout_us == 0 || timeout_us > 10000000u) return DSA_ERR_INVALID_ARG;
  unsigned* st = status_ptr((cudaStream_t)stream);
  if (st == nullptr) return cuda_fail(cudaGetLastError());
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(st, (uint64_t)timeout_us * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return DSA_OK;
}

dsa_status dsa_set_wait_limit(uint64_t limit_ns) {
  if (limit_ns > 60ull * 1000000000ull) return DSA_ERR_INVALID_ARG;
  g_wait_limit.store(limit_ns == 0 ? kWaitLimitNs : limit_ns);
  return DSA_OK;
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported";
    case DSA_ERR_CAPACITY: return "capacity exceeded";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_DEVICE: return "device reported an inconsistent index";
  }
  return "unknown status";
}

int32_t dsa_last_cuda_error(void) { return t_last_cuda_error; }

}  // extern "C"
