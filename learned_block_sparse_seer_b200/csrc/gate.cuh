// gate.cuh -- host-side launchers of the AttnGate kernels (gate.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/seer.h"

namespace seer {

// Q average-pool (is_k = false) or K [max|min|avg]-pool (is_k = true) of X
// [BH, n, d] into out [BH, n/64, d] or [BH, n/64, 3d] (fp32).  tab: optional
// varlen block table (valid tokens per block).
// lo non-null: out receives each pooled value rounded to tf32 and lo the exact
// remainder (the tf32x3 operand split), instead of the fp32 value.
// Inputs of the tensor-core gate, pooled and split in one launch: Q blocks
// (average, [B*Hq*nb, d]) and K blocks ([max | min | avg], [B*Hkv*nb, 3d]),
// each written as tf32 part (qhi, khi) and remainder (qlo, klo), and the
// weights Wq (nwq floats) and Wk (nwk floats) split the same way.  cq and ck
// are the CTAs (8 warps, a block per warp) of the two poolings.
struct GateInputs {
  const void* Q;
  const void* K;
  long long nq, nk, cq, ck;
  int n, d;
  float *qhi, *qlo, *khi, *klo;
  const int2* tab;
  const float* Wq;
  const float* Wk;
  long long nwq, nwk;
  float *wqh, *wql, *wkh, *wkl;
};
cudaError_t launch_gate_inputs(const GateInputs& g, seer_dtype dt, cudaStream_t st);

cudaError_t launch_pool(const void* X, seer_dtype dt, bool is_k, long long BH, int n, int d,
                        float* out, cudaStream_t st, const int2* tab = nullptr, float* lo = nullptr);

// Batched C = alpha * A B^T (fp32); see gemm_nt_kernel for the batch mapping.
cudaError_t launch_gemm_nt(const float* A, const float* B, float* C, int M, int N, int K,
                           long long a_bs, long long b_bs, long long c_bs, int ldc, int batch,
                           int zh, int zmul, int zg, float alpha, bool causal, cudaStream_t st);

// C[z] = alpha * A[z] B[bz]^T on the tensor cores in three tf32 products
// (fp32-level accuracy): the gate's causal logits (causal = 1: tiles above
// the diagonal are skipped) and its projections (causal = 0).  A, B are split
// first: launch_split_tf32 rounds x to tf32 in place and writes the remainder
// to lo (launch_gate_inputs splits the caller's weights into workspace
// buffers).  tmAh/tmAl are fp32 maps over A's hi/lo
// [batch * M rows, K], tmBh/tmBl over B's [(max bz + 1) * N rows, K],
// 32 x 128 boxes, 128-byte swizzle.  K % 32 == 0.
struct Tf32x3Params {
  int M, N, K, ldc, zh, zmul, zg, causal;
  long long c_bs;
  float alpha;
  float* C;
  float* C_lo;  // non-null: C receives the result rounded to tf32 and C_lo the exact remainder
  int tma_out;  // launch_gemm_tf32x3_causal: write C (and C_lo) by TMA stores through tmC (tmClo)
  uint32_t* status;
  unsigned long long timeout_ns;
};
cudaError_t launch_split_tf32(float* x, float* lo, long long n, cudaStream_t st);
// tmC / tmClo (used when p.tma_out): 3-D maps over C / C_lo (N columns, M rows,
// batch; box 32 x 128 x 1, 128-byte swizzle).
cudaError_t launch_gemm_tf32x3_causal(const CUtensorMap& tmAh, const CUtensorMap& tmAl, const CUtensorMap& tmBh,
                                      const CUtensorMap& tmBl, const CUtensorMap& tmC, const CUtensorMap& tmClo,
                                      const Tf32x3Params& p, int batch, cudaStream_t st);

// The causal logits with each 128-row block of A held in tensor memory while
// the B tiles up to the diagonal stream past it (p.causal ignored: always
// causal); persistent, at most num_sms CTAs.  tmAh / tmAl are 3-D panel maps
// over the A parts (box 32 x 128 x K/32), tmBh / tmBl 2-D maps over the B
// parts (box 32 x 128), tmC a 3-D map over C (N columns, M rows, batch; box
// 32 x 128 x 1).  Needs K a multiple of 32 and at most 128, N and c_bs
// multiples of 4 and C 16-byte aligned (gemm_tf32x3_rows_fits).
bool gemm_tf32x3_rows_fits(int K, int N, long long c_bs, const void* C);
cudaError_t launch_gemm_tf32x3_rows(const CUtensorMap& tmAh, const CUtensorMap& tmAl, const CUtensorMap& tmBh,
                                    const CUtensorMap& tmBl, const CUtensorMap& tmC, const Tf32x3Params& p,
                                    int batch, int num_sms, cudaStream_t st);

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
