// fwd.cuh -- parameters and launcher of the dense causal attention forward
// that also forms the 2D-max-pooled probability map (the training forward).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace seer {

struct FwdParams {
  int B, Hq, Hkv, n, d, nb, G, npairs;
  long long total_units;  // B * Hq * npairs (a unit: one head, two query blocks)
  void* O;                // [B, Hq, n, d] bf16 or fp32
  int out_fp32;
  float* lse;             // [B, Hq, n] fp32 or null
  float* map;             // [B, Hq, nb, nb] fp32 or null (null: attention only)
  float scale_log2;       // softmax scale * log2(e)
  float* r;               // with map: per CTA [nb][2][128] per-row half-block score maxima (log2 units)
  uint32_t* status;
  uint32_t* work_counter;
  unsigned long long timeout_ns;
  // 64-row units (numbered as the sparse kernel numbers them, KV-head-major,
  // query blocks from the last) whose rows scored more than 2^64 above their
  // first step's maximum, for the exact fallback
  uint32_t* redo_count;
  int* redo_list;
  int redo_cap;
  // non-null: the launch does nothing unless (*run_if != 0) == run_if_value
  const uint32_t* run_if;
  uint32_t run_if_value;
};

// Persistent launch of at most `ctas` CTAs (the map scratch holds that many
// slots).  tmQ, tmK, tmV are 3-D bf16 maps over [rows, d] read as 64-dim
// panels (64 dims, rows, d/64) with a 64 x 128 x d/64 box, 128-byte swizzle.
cudaError_t launch_fwd(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const FwdParams& p,
                       int ctas, cudaStream_t st);

}  // namespace seer
