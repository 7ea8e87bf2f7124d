// attn_tf32.cuh -- block-sparse attention for fp32 Q/K/V on the tf32 tensor
// cores (attn_tf32.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace seer {

struct Tf32AttnParams {
  int Hq, Hkv, n, d, nb, cap;
  long long total_units;   // B * Hq * nb: one CTA each
  const int32_t* counts;   // [B, Hq, nb]
  const int32_t* indices;  // [B, Hq, nb, cap]
  float* O;                // [B, Hq, n, d] fp32
  float* lse;              // [B, Hq, n] or null
  float scale_log2;        // softmax scale * log2(e)
  uint32_t* status;        // workspace status word
  unsigned long long timeout_ns;
};

// V^T per 64-key block into Vt [B*Hkv*nb*d, 64] (fp32).
cudaError_t launch_vt(const float* V, float* Vt, long long BHkv, int n, int d, cudaStream_t st);

// tmQ, tmK: 3-D fp32 panel maps over Q [B*Hq*n, d] and K [B*Hkv*n, d] (box
// {32, 64, d/32}); tmV over Vt [B*Hkv*nb*d, 64] (box {32, d, 2}); all
// 128-byte swizzled.
cudaError_t launch_attn_tf32(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const Tf32AttnParams& p, cudaStream_t st);

}  // namespace seer
