// gate_noalloc.cu -- seer_gate_noalloc: the gate with a fixed, library-owned
// scratch buffer, for callers that cannot allocate device memory.
//
// seer_gate needs a scratch workspace (pooled Q/K, projected gate vectors,
// block logits) that its caller allocates.  Some callers cannot do that: a
// plugin running inside a host framework that owns every device allocation,
// code that runs while a CUDA graph is being captured (cudaMalloc is not
// allowed then), or a runtime with a hard "no allocation after start-up"
// policy.  This entry point takes the same inputs and outputs and uses a
// static device buffer instead.
//
// The buffer is a file-scope __device__ array of kNoAllocScratchBytes.  Every
// GPU on which the library's device code is loaded keeps it until the process
// exits.  Host code cannot use the array's name as a device address, so on
// the first call on each device (with that device current) the address is
// resolved once with cudaGetSymbolAddress and cached; make that first call
// before any stream capture.  All calls on a device share the buffer and it
// keeps the previous call's contents: the status word it starts with is
// cleared by every call, and every other byte the kernels read is written
// first by the same call.  Calls whose work overlaps on the GPU (other streams,
// or no ordering between them) race on the buffer.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/seer.h"
#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = SEER_GATE_NOALLOC_MAX_SCRATCH;

static __device__ __align__(256) unsigned char g_gate_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the buffer on the current device (resolved once per
// device).  Returns a CUDA error code.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gate_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" seer_status seer_gate_noalloc(const seer_dims* dims, const void* Q, const void* K,
                                         seer_dtype dtype, const float* Wq, const float* Wk,
                                         int32_t h, float rope_theta, seer_select_mode mode,
                                         float T, int32_t k, float density, float* scores_out,
                                         int32_t* counts, int32_t* indices, int32_t cap,
                                         seer_stream_t stream) {
  const size_t need = seer_gate_workspace_size(dims, h);
  if (need == 0) return SEER_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return SEER_ERR_WORKSPACE;
  void* scratch = nullptr;
  const cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    seer::set_last_cuda_error((int32_t)e);  // what seer_last_cuda_error() returns
    return SEER_ERR_CUDA;
  }
  return seer_gate(dims, Q, K, dtype, Wq, Wk, h, rope_theta, mode, T, k, density, scores_out,
                   counts, indices, cap, scratch, kNoAllocScratchBytes, stream);
}
