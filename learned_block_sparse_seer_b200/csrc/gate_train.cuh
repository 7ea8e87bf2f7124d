// gate_train.cuh -- launchers of the AttnGate distillation step (KL loss and
// the gate's weight gradients).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace seer {

// C_z = alpha * sum_{r < R} A_{z,r} B_{z,r}, z = z1 * Z2 + z2 (fp32).
// A(m, k) = A[z1*a_z1 + z2*a_z2 + r*a_r + m*a_m + k*a_k]
// B(k, n) = B[z1*b_z1 + (z2/b_div)*b_z2 + r*b_r + k*b_k + n*b_n]
// C(m, n) = C[z1*c_z1 + z2*c_z2 + m*c_m + n*c_n]
// band: 0 dense; 1 A is zero for k > m; 2 A is zero for k < m (tiles skipped).
struct GemmBatched {
  const float* A;
  const float* B;
  float* C;
  int M, N, K, R, Z1, Z2, b_div, band;
  long long a_m, a_k, a_z1, a_z2, a_r;
  long long b_k, b_n, b_z1, b_z2, b_r;
  long long c_m, c_n, c_z1, c_z2;
  float alpha;
};

// Per causal row of the gate logits: KL(g || softmax(z)) into row_loss and
// dz = (softmax(z) - g) / rows written over the logits (0 for j > i); g is
// the gt row divided by its causal sum.
cudaError_t launch_kl_rows(float* zdz, const float* gt, float* row_loss, long long rows, int nb,
                           cudaStream_t st);
// loss = sum(row_loss) / rows, in a fixed order (one CTA).
cudaError_t launch_loss_sum(const float* row_loss, long long rows, float* loss, cudaStream_t st);
cudaError_t launch_gemm_batched(const GemmBatched& g, cudaStream_t st);

}  // namespace seer
