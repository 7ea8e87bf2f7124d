// decode.cuh -- launchers of the decode-stage gate, the block-sparse decode
// attention and the decode ground truth.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace seer {

// k~ for key blocks j0 .. j0+nnew-1 of every (batch, KV head): K is the cache
// [B*Hkv, n_cap, d] (bf16 or fp32), Wk [Hkv, d, 3d], kt [B*Hkv, n_cap/64, d].
cudaError_t launch_kcache(const void* K, bool fp32, const float* Wk, float* kt, long long BHkv, int Hkv, int n_cap,
                          int d, int j0, int nnew, cudaStream_t st);

// logits [rows, nc] = q . k~_j * scale for the nc candidate blocks
// (q [rows, d] in the cache dtype, rows = B*Hq).
cudaError_t launch_decode_logits(const void* q, bool fp32, const float* kt, float* logits, long long B, int Hq,
                                 int Hkv, int d, int nc, int nb_cap, float scale, cudaStream_t st);

// Splits of each row's list in the decode attention (a function of the row
// count only, so that the workspace size follows from the shape).
int decode_attn_splits(long long rows);

struct DecodeAttnArgs {
  const void* q;
  const void* K;
  const void* V;
  bool fp32;
  const int32_t* counts;
  const int32_t* indices;
  int cap, Hq, Hkv, d, n_cap, seq_len, splits;
  long long rows;
  float scale_log2;
  float* part;      // [rows, splits, d + 2]
  int32_t* ticket;  // [rows], zero on entry; left zero
  void* O;          // [rows, d]
  float* lse;       // [rows] or null
  uint32_t* status;
  unsigned long long timeout_ns;  // bound of every wait
};
cudaError_t launch_decode_attn(const DecodeAttnArgs& a, cudaStream_t st);

// Ground truth: chunks of key blocks per row and the scratch they need.
constexpr int kGtMaxChunks = 256;

// gt [rows, c + 1] and lse [rows] (may be null) of the token at seq_len - 1.
// stats: [rows, kGtMaxChunks, 2] floats; ticket: [B * Hq] ints, zero on
// entry and left zero.
cudaError_t launch_decode_gt(const void* q, const void* K, bool fp32, long long B, int Hq, int Hkv, int d, int n_cap,
                             int seq_len, float scale_log2, float* gt, float* lse, float* stats, int32_t* ticket,
                             uint32_t* status, unsigned long long timeout_ns, cudaStream_t st);

}  // namespace seer
