// gate_train.cu -- the AttnGate's distillation step: KL(gt || score) and the
// gradients of that loss with respect to the gate's two linear layers.
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4, "Loss function: KL-divergence"
// (loss = D_KL(gt || score), score = AttnGate(Q, K), gt the 2D-max-pooled
// attention map) and "Training data and hyperparameters" (only the gate's
// parameters are trained).  Readings: both maps are row distributions over
// the causal key blocks j <= i, so each gt row is divided by its sum; the
// loss is the mean over all (batch, query head, query block) rows.
//
// Kernels (all fp32; the sizes are O(nb^2 h) per head, far below the
// attention's):
//   kl_row_kernel     one CTA per row: softmax of the logits, normalised gt,
//                     the row's KL term, and dz = (score - g) / rows written
//                     over the logits in place (0 above the diagonal)
//   loss_sum_kernel   one CTA: the rows' terms summed in a fixed order
//                     (deterministic), divided by the row count
//   gemm_batched_kernel  C_z = alpha * sum_r A_{z,r} B_{z,r} with arbitrary
//                     element and batch strides: dq~ = dz k~, dk~ = dz^T q~
//                     (summed over a KV head's query heads), dWq = dq~^T qbar,
//                     dWk = dk~^T kbar (summed over the batch)
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "gate_train.cuh"

namespace seer {

// ------------------------------------------------------------- KL rows ---
__global__ void __launch_bounds__(256) kl_row_kernel(float* __restrict__ zdz, const float* __restrict__ gt,
                                                     float* __restrict__ row_loss, int nb, float inv_rows) {
  const long long row = blockIdx.x;  // (b * Hq + hq) * nb + i
  const int i = (int)(row % nb);
  float* z = zdz + row * nb;
  const float* g = gt + row * nb;
  __shared__ float red[8];
  __shared__ float bc;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  auto block_max = [&](float v) -> float {
    v = warp_max(v);
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (tid == 0) {
      float m = red[0];
      for (int k = 1; k < 8; ++k) m = fmaxf(m, red[k]);
      bc = m;
    }
    __syncthreads();
    const float r = bc;
    __syncthreads();
    return r;
  };
  auto block_sum = [&](float v) -> float {
    v = warp_sum(v);
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (tid == 0) {
      float s = 0.f;
      for (int k = 0; k < 8; ++k) s += red[k];
      bc = s;
    }
    __syncthreads();
    const float r = bc;
    __syncthreads();
    return r;
  };
  float m = -INFINITY;
  for (int j = tid; j <= i; j += blockDim.x) m = fmaxf(m, z[j]);
  m = block_max(m);
  float se = 0.f, sg = 0.f;
  for (int j = tid; j <= i; j += blockDim.x) {
    se += expf(z[j] - m);
    sg += g[j];
  }
  se = block_sum(se);
  sg = block_sum(sg);
  const float log_se = logf(se);
  const float inv_sg = 1.0f / sg;
  float term = 0.f;
  for (int j = tid; j < nb; j += blockDim.x) {
    float dz = 0.f;
    if (j <= i) {
      const float logs = z[j] - m - log_se;  // log score
      const float gn = g[j] * inv_sg;
      if (gn > 0.f) term += gn * (logf(gn) - logs);
      dz = (expf(logs) - gn) * inv_rows;
    }
    z[j] = dz;
  }
  term = block_sum(term);
  if (tid == 0) row_loss[row] = term;
}

// One CTA, fixed summation order: each thread a strided slice in index order,
// then a fixed tree.
__global__ void __launch_bounds__(1024) loss_sum_kernel(const float* __restrict__ row_loss, long long rows,
                                                        float* __restrict__ loss) {
  __shared__ double part[1024];
  double s = 0.0;
  for (long long r = threadIdx.x; r < rows; r += blockDim.x) s += (double)row_loss[r];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = (float)(part[0] / (double)rows);
}

// ------------------------------------------------------- strided GEMM ----
// 64 x 64 tile per CTA, 256 threads (4 x 4 outputs each), k in chunks of 32.
// Batch z = blockIdx.z = z1 * Z2 + z2; B's second batch index is z2 / b_div.
// band: 0 none; 1 only k <= m contributes (lower-triangular A); 2 only k >= m.
__global__ void __launch_bounds__(256) gemm_batched_kernel(const GemmBatched g) {
  const int tm = blockIdx.x, tn = blockIdx.y;
  const int z1 = blockIdx.z / g.Z2, z2 = blockIdx.z % g.Z2;
  const float* Ab = g.A + z1 * g.a_z1 + z2 * g.a_z2;
  const float* Bb = g.B + z1 * g.b_z1 + (z2 / g.b_div) * g.b_z2;
  float* Cb = g.C + z1 * g.c_z1 + z2 * g.c_z2;
  __shared__ float As[32][65];
  __shared__ float Bs[32][65];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  const int m_lo = tm * 64, m_hi = min(g.M, m_lo + 64) - 1;
  int k_begin = 0, k_end = g.K;
  if (g.band == 1) k_end = min(g.K, m_hi + 1);
  if (g.band == 2) k_begin = (m_lo / 32) * 32;
  for (int r = 0; r < g.R; ++r) {
    const float* Ar = Ab + r * g.a_r;
    const float* Br = Bb + r * g.b_r;
    for (int k0 = k_begin; k0 < k_end; k0 += 32) {
      for (int e = tid; e < 64 * 32; e += 256) {
        const int rr = e / 32, cc = e % 32;
        const int gk = k0 + cc;
        const int gm = tm * 64 + rr, gn = tn * 64 + rr;
        As[cc][rr] = (gm < g.M && gk < k_end) ? Ar[gm * g.a_m + gk * g.a_k] : 0.f;
        Bs[cc][rr] = (gn < g.N && gk < k_end) ? Br[gk * g.b_k + gn * g.b_n] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < 32; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a[q] = As[kk][ty * 4 + q];
          b[q] = Bs[kk][tx * 4 + q];
        }
#pragma unroll
        for (int pp = 0; pp < 4; ++pp)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[pp][q] = fmaf(a[pp], b[q], acc[pp][q]);
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int pp = 0; pp < 4; ++pp) {
    const int gm = tm * 64 + ty * 4 + pp;
    if (gm >= g.M) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int gn = tn * 64 + tx * 4 + q;
      if (gn < g.N) Cb[gm * g.c_m + gn * g.c_n] = g.alpha * acc[pp][q];
    }
  }
}

cudaError_t launch_kl_rows(float* zdz, const float* gt, float* row_loss, long long rows, int nb,
                           cudaStream_t st) {
  kl_row_kernel<<<(unsigned)rows, 256, 0, st>>>(zdz, gt, row_loss, nb, (float)(1.0 / (double)rows));
  return cudaGetLastError();
}

cudaError_t launch_loss_sum(const float* row_loss, long long rows, float* loss, cudaStream_t st) {
  loss_sum_kernel<<<1, 1024, 0, st>>>(row_loss, rows, loss);
  return cudaGetLastError();
}

cudaError_t launch_gemm_batched(const GemmBatched& g, cudaStream_t st) {
  dim3 grid((unsigned)((g.M + 63) / 64), (unsigned)((g.N + 63) / 64), (unsigned)(g.Z1 * g.Z2));
  gemm_batched_kernel<<<grid, 256, 0, st>>>(g);
  return cudaGetLastError();
}

}  // namespace seer
