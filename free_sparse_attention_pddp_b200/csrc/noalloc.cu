// Reuse step without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// reuse step: runtimes that reserve all device memory up front and hand out
// only tensor buffers, or plug-ins that must not touch the allocator. For them
// this file keeps the reuse kernel's only scratch -- its status block -- in a
// file-scope static device array instead of the caller's workspace.
//
// The array is small (kScratchBytes) but every GPU that loads the library
// holds one copy until the process exits. All calls share it: each call clears
// it before launching, so calls whose kernels overlap on the GPU (on different
// streams) race on it and may report each other's status.
#include <mutex>

#include "mcs_internal.h"

namespace {

constexpr size_t kScratchBytes = MCS_STATUS_BYTES;  // the status block
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_noalloc_scratch[kScratchBytes / sizeof(int32_t)];

std::mutex g_mu;
int32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device, resolved once
// per device (with that device current) and cached for the process: after a
// cudaDeviceReset the cached address is stale, which the header states.
mcs_status scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MCS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MCS_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<int32_t*>(ptr);
  }
  *out = g_scratch_addr[dev];
  return MCS_OK;
}

}  // namespace

extern "C" mcs_status mcs_sparse_noalloc(const mcs_shape* s, const void* q, const void* k, const void* v,
                                         const int32_t* perm, const int32_t* kv_idx, const void* resid, void* o,
                                         int32_t* info, cudaStream_t stream) {
  if (!s || !q || !k || !v || !perm || !kv_idx || !o) return MCS_ERR_INVALID_ARG;
  const size_t need = mcs_workspace_bytes(s, MCS_OP_SPARSE);
  if (need == 0) {
    // invalid or unsupported shape: let the regular entry point classify it
    return mcs_sparse(s, q, k, v, perm, kv_idx, resid, o, nullptr, 0, stream);
  }
  if (need > kScratchBytes) return MCS_ERR_INVALID_ARG;  // beyond the static scratch
  int32_t* scratch = nullptr;
  mcs_status st = scratch_for_current_device(&scratch);
  if (st != MCS_OK) return st;
  if (cudaMemsetAsync(scratch, 0, kScratchBytes, stream) != cudaSuccess) return MCS_ERR_CUDA;
  st = mcs_sparse(s, q, k, v, perm, kv_idx, resid, o, scratch, kScratchBytes, stream);
  if (st != MCS_OK || !info) return st;
  int32_t words[MCS_INFO_WORDS];
  if (cudaMemcpyAsync(words, scratch, sizeof(words), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MCS_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MCS_ERR_CUDA;
  for (int i = 0; i < MCS_INFO_WORDS; ++i) info[i] = words[i];
  return static_cast<mcs_status>(words[MCS_SW_STATUS]);
}
