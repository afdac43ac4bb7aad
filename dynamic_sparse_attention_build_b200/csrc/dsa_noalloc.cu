// dsa_build_indices_static: index building whose scratch memory is a fixed
// buffer compiled into the library, for callers that must not allocate device
// memory.
//
// Who needs it: code that runs inside a host runtime which owns every byte of
// device memory (a plugin or custom op of another inference engine, a process
// with a hard device-memory budget reserved up front), and latency-critical
// paths where a cudaMalloc is not acceptable because it can synchronise the
// whole device and stall unrelated streams.  Such callers can still pass the
// inputs and the output index arrays they own, but not a workspace.
//
// The scratch is one file-scope array of kStaticWorkspaceBytes on every GPU
// that loads the library, held until the process exits.  Problems whose
// workspace would be larger are rejected with DSA_ERR_CAPACITY.  All calls on a
// device share the array and it keeps the previous call's contents; the index
// builder clears what it accumulates into before each use, so stale contents
// do not matter, but two calls whose work overlaps on the GPU (different
// streams, no ordering between them) race on the array.
#include <atomic>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr size_t kStaticWorkspaceBytes = 16u << 20;  // 16 MiB
constexpr int kMaxDev = 64;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Host code may not use g_static_workspace as a pointer: in host code that name
// is a host-side stand-in, not a device address.  The device address is looked
// up once per device, with that device current (an atomic: host threads that make
// their first call at the same moment store the same address).  It stays valid
// for the life of the device's context, so the library must not be used again
// after a cudaDeviceReset in the same process.
std::atomic<void*> g_ws_addr[kMaxDev] = {};

dsa_status static_workspace(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDev) return DSA_ERR_UNSUPPORTED;
  void* p = g_ws_addr[dev].load();
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return cuda_fail(e);
    g_ws_addr[dev].store(p);
  }
  *out = p;
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_build_indices_static(const dsa_problem* p, const void* Q, const void* K,
                                               const dsa_pattern* pats, const dsa_indices* out,
                                               dsa_stream stream) {
  dsa_status s = validate_problem(p);
  if (s != DSA_OK) return s;
  if (pats == nullptr || !Q || !K) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Q) & 15u) || (reinterpret_cast<uintptr_t>(K) & 15u)) return DSA_ERR_INVALID_ARG;
  s = validate_indices_ptrs(out, true);
  if (s != DSA_OK) return s;
  dsa_sizes sz;
  s = plan_sizes(*p, pats, &sz);
  if (s != DSA_OK) return s;
  if (sz.workspace_bytes > (int64_t)kStaticWorkspaceBytes) return DSA_ERR_CAPACITY;
  void* ws = nullptr;
  s = static_workspace(&ws);
  if (s != DSA_OK) return s;
  unsigned* st = status_ptr((cudaStream_t)stream);
  if (st == nullptr) return cuda_fail(cudaGetLastError());
  return launch_build_indices(*p, Q, K, pats, *out, ws, kStaticWorkspaceBytes, (cudaStream_t)stream, st);
}
