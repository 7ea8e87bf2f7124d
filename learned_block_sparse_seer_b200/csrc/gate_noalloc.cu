// gate_noalloc.cu -- seer_gate_noalloc: the gate with a fixed, library-owned
// scratch buffer, for callers that cannot allocate device memory.
//
// seer_gate needs a scratch workspace (pooled Q/K, projected gate vectors,
// block logits) that its caller allocates.  Some callers cannot do that: a
// plugin running inside a host framework that owns every device allocation
// and hands out only its own tensors, or a runtime with a hard "no device
// allocation after start-up" policy (allocation can fail or stall at an
// arbitrary point in the middle of serving).  This entry point takes the same
// inputs and outputs and uses a static device buffer instead.
//
// The buffer is a file-scope __device__ array of kNoAllocScratchBytes.  Every
// GPU on which the library's device code is loaded keeps it until the process
// exits.  Host code cannot use the array's name as a device address, so on
// the first call on each device (with that device current) the address is
// resolved once with cudaGetSymbolAddress and cached; make that first call
// before any stream capture.  The cache is keyed by the current context's
// unique id, so a device reset (which makes a new context and reloads the
// module) resolves the address again.
//
// All calls on a device share the buffer and it keeps the previous call's
// contents: the status word it starts with is cleared by every call, and
// every other byte the kernels read is written first by the same call.  Calls
// whose work overlaps on the GPU (other streams, or no ordering between them)
// race on the buffer.
//
// Device-side failures (a bounded wait that gave up) land in the buffer's
// status word, which the caller cannot read.  So a last kernel checks it and,
// if it is set, overwrites every count with -1: the failure shows up in the
// outputs themselves.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/seer.h"
#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = SEER_GATE_NOALLOC_MAX_SCRATCH;

static __device__ __align__(256) unsigned char g_gate_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_ctx_id[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The unique id of the current context (driver entry points, no link
// dependency on libcuda); 0 if it cannot be read.
unsigned long long current_ctx_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = (CtxGetCurrentFn)f;
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)f;
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the buffer on the current device (resolved once per
// device and context).  Returns a CUDA error code.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long ctx = current_ctx_id();  // 0 before the runtime's first call on this thread
  if (!g_scratch_ptr[dev] || ctx == 0 || g_ctx_id[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gate_scratch);  // makes the device's primary context current
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_ctx_id[dev] = current_ctx_id();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

// If the gate recorded a device-side failure in the buffer's status word,
// every row's count becomes -1 (the outputs are then unusable, and a
// consumer such as seer_sparse_attn rejects them as bad lists).
__global__ void __launch_bounds__(256) mark_failed_rows_kernel(const uint32_t* __restrict__ status,
                                                               int32_t* __restrict__ counts, long long rows) {
  if (*status == 0u) return;  // kDevOk
  for (long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += (long long)gridDim.x * blockDim.x)
    counts[r] = -1;
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
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    seer::set_last_cuda_error((int32_t)e);  // what seer_last_cuda_error() returns
    return SEER_ERR_CUDA;
  }
  const seer_status st = seer_gate(dims, Q, K, dtype, Wq, Wk, h, rope_theta, mode, T, k, density, scores_out,
                                   counts, indices, cap, scratch, kNoAllocScratchBytes, stream);
  if (st != SEER_OK) return st;
  const long long rows = (long long)dims->B * dims->Hq * (dims->n / seer::kBlock);
  const long long blocks = rows / 256 + 1 < 148 ? rows / 256 + 1 : 148;
  mark_failed_rows_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      &reinterpret_cast<const seer::WsHeader*>(scratch)->status, counts, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    seer::set_last_cuda_error((int32_t)e);
    return SEER_ERR_CUDA;
  }
  return SEER_OK;
}
