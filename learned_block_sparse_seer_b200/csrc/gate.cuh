// gate.cuh -- host-side launchers of the AttnGate kernels (gate.cu).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/seer.h"

namespace seer {

// Q average-pool (is_k = false) or K [max|min|avg]-pool (is_k = true) of X
// [BH, n, d] into out [BH, n/64, d] or [BH, n/64, 3d] (fp32).  tab: optional
// varlen block table (valid tokens per block).
cudaError_t launch_pool(const void* X, seer_dtype dt, bool is_k, long long BH, int n, int d,
                        float* out, cudaStream_t st, const int2* tab = nullptr);

// Batched C = alpha * A B^T (fp32); see gemm_nt_kernel for the batch mapping.
cudaError_t launch_gemm_nt(const float* A, const float* B, float* C, int M, int N, int K,
                           long long a_bs, long long b_bs, long long c_bs, int ldc, int batch,
                           int zh, int zmul, int zg, float alpha, bool causal, cudaStream_t st);

// Block-level RoPE with base theta / 64 on x [rows, h] (row position = row % nb).
cudaError_t launch_rope(float* x, long long rows, int nb, int h, float theta, cudaStream_t st);

// Causal softmax of logit rows (from_logits) and/or index-list selection.
// mode may carry SEER_SELECT_FORCE_DIAGONAL; tab: optional varlen table.
cudaError_t launch_row_select(const float* in, float* scores, bool from_logits, long long rows,
                              int nb, int mode, float T, int k, float density, int32_t* counts,
                              int32_t* indices, int cap, cudaStream_t st, int row_len = 0,
                              const int2* tab = nullptr);

// Varlen packing: the per-block table (first block of the block's sequence,
// valid tokens) from the sequences' starts and lengths (device arrays).
cudaError_t launch_varlen_table(const int32_t* start, const int32_t* len, int nseq, int n, int2* tab,
                                uint32_t* status, cudaStream_t st);

}  // namespace seer
