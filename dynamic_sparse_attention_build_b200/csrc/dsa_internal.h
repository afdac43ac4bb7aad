// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// Device address of the status word (4 x uint32) that work on `stream` reports
// into on the current device, or nullptr on failure.
unsigned* status_ptr(cudaStream_t stream);

// Records a CUDA error for dsa_last_cuda_error and returns DSA_ERR_CUDA.
dsa_status cuda_fail(cudaError_t e);

// Default bound on every in-kernel wait (ns of global time).
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// The bound that launches use now (kWaitLimitNs unless dsa_set_wait_limit changed it).
uint64_t wait_limit_ns();

dsa_status validate_problem(const dsa_problem* p);
dsa_status validate_indices_ptrs(const dsa_indices* idx, bool for_build);

dsa_status launch_sparse_attn(const dsa_problem& p, const void* Q, const void* K, const void* V,
                              const dsa_indices& idx, void* O, float* lse, cudaStream_t stream,
                              unsigned* status);

dsa_status launch_count_pairs(const dsa_problem& p, const dsa_indices& idx, int64_t* pairs,
                              cudaStream_t stream, unsigned* status);

// 3-D TMA map over a bf16 tensor [H][N][d] with element strides (token, head):
// boxes of 64 columns x box_rows rows x 1 head, 128-byte swizzle, zero fill
// outside the tensor.  False if the driver entry point or the encoding fails.
bool make_tma_map_bf16_3d(CUtensorMap* map, const void* base, int d, int N, int H, int64_t ts, int64_t hs,
                          int box_rows);

dsa_status plan_sizes(const dsa_problem& p, const dsa_pattern* pats, dsa_sizes* out);

dsa_status launch_build_indices(const dsa_problem& p, const void* Q, const void* K,
                                const dsa_pattern* pats, const dsa_indices& out, void* ws,
                                size_t ws_bytes, cudaStream_t stream, unsigned* status);

}  // namespace dsa
