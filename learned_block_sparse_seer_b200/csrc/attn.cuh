// attn.cuh -- parameters and launcher of the block-sparse attention kernel.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace seer {

struct AttnParams {
  int B, Hq, Hkv, n, d, nb, G, cap;
  long long total_units;     // B * Hq * nb
  const int32_t* counts;     // [B, Hq, nb]
  const int32_t* indices;    // [B, Hq, nb, cap]
  void* O;                   // [B, Hq, n, d] bf16 or fp32
  float* lse;                // [B, Hq, n] or null
  int out_fp32;              // O element type
  float scale_log2;          // softmax scale * log2(e)
  uint32_t* status;          // workspace status word
  uint32_t* work_counter;    // workspace work counter (zeroed per call)
  unsigned long long timeout_ns;
};

// Persistent launch: one CTA per SM (at most one per unit).  tmQ/tmK/tmV are
// 2-D bf16 tensor maps over [rows, d] with 64x64 boxes and 128-byte swizzle.
cudaError_t launch_sparse_attn(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                               const AttnParams& p, int num_sms, cudaStream_t st);

}  // namespace seer
