// common.cuh -- shapes, workspace layout helpers and small device utilities
// shared by the kernels of the SeerAttention prefill library.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/seer.h"
#include "ptx.cuh"

namespace seer {

constexpr int kBlock = 64;  // tokens per gate block and attention tile

// The first 256 bytes of every workspace: the device status word and the
// dynamic work counters of the persistent kernels.
struct WsHeader {
  uint32_t status;        // kDevOk / kDevTimeout / kDevBadIndex ... (ptx.cuh)
  uint32_t bad_value;     // first offending value recorded with a status
  uint32_t work_counter;  // persistent-kernel work index
  uint32_t work_counter2;
  uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// Records the CUDA error reported by seer_last_cuda_error() on this host
// thread (api.cu).
void set_last_cuda_error(int32_t e);

__host__ __device__ constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Carves consecutive 256-byte-aligned regions out of a workspace.
struct WsCarver {
  size_t off = sizeof(WsHeader);
  size_t take(size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  }
};

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code, uint32_t value) {
  if (atomicCAS(status, 0u, code) == 0u) status[1] = value;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Bounded wait (timeout_ns of %globaltimer) for a phase whose completion
// depends on no other warp of the CTA: a bulk copy this thread issued, or
// the commit of MMAs it issued.  Used before a CTA exits, so it does not give
// up when the CTA's abort flag is raised: copies and products in flight
// finish before their shared or tensor memory is released.
__device__ __forceinline__ bool wait_landed(uint64_t* bar, uint32_t parity, uint64_t timeout_ns = 20000000ull) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000u))
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  return true;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace seer
