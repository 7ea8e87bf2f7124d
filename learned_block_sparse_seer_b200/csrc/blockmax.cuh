// blockmax.cuh -- parameters and launcher of the max-pooled probability map.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace seer {

struct BmaxParams {
  int B, Hq, Hkv, n, d, nb, G, npairs;
  long long total_units;   // B * Hq * npairs
  float* map;              // [B, Hq, nb, nb] fp32
  float* lse;              // [B, Hq, n] fp32 or null
  float scale_log2;        // softmax scale * log2(e)
  float* r;                // scratch: [ctas, nb, 2, 128] per-row half-block maxima (log2 units)
  uint32_t* status;
  uint32_t* work_counter;
  unsigned long long timeout_ns;
};

// Persistent launch of at most `ctas` CTAs (the scratch holds that many
// slots).  tmQ/tmK are bf16 [rows, d] maps with 64 x 128 boxes.
cudaError_t launch_blockmax(const CUtensorMap& tmQ, const CUtensorMap& tmK, const BmaxParams& p,
                            int ctas, cudaStream_t st);

}  // namespace seer
