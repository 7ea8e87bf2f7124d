// decode.cu -- decode-stage gating and block-sparse decode attention.
//
// Source: the authors' OpenReview rebuttal ("decode-stage evaluation"): for
// decoding the AttnGate drops the Q branch's pooling and projection (each
// token's own query scores the key blocks), keeps a small compressed K cache
// (pooled after RoPE) so that gating never reads the full K cache, loads V
// only for the selected blocks, and is distilled against the 1D max-pooling
// of the token's attention row.  Readings: the compressed cache holds
// k~_j = Wk [max | min | avg](K block j) for the complete blocks j < c, where
// c = (seq_len - 1) / 64 is the current token's block; that block is always
// attended and is not a candidate; no further RoPE; h = d.
//
// Kernels (memory-bound: one query row per (batch, head)):
//   kcache_kernel       one CTA per (batch, KV head, new block): pooling over
//                       the block's 64 keys, then k~ = Wk[g] kbar
//   decode_logits_kernel  one CTA per (batch, query head): q . k~_j / sqrt(d)
//                       for the c candidates (a warp per block); the softmax
//                       and selection then reuse the prefill row kernel
//   decode_attn_kernel  split-KV online softmax: CTA (row, split) walks every
//                       split-th entry of the row's list (selected blocks, then
//                       the current block); partial (m, l, o) per split
//   decode_combine_kernel  merges the splits by log-sum-exp into O and LSE
//   decode_gt_kernel    the 1D ground truth: a warp per key block keeps the
//                       block's raw maximum and an online (m, l); the row's
//                       LSE then turns the maxima into probabilities
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "decode.cuh"
#include "ptx.cuh"

namespace seer {

namespace {
template <typename T>
__device__ __forceinline__ float ld(const T* p, long long i) {
  if constexpr (sizeof(T) == 2)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  else
    return reinterpret_cast<const float*>(p)[i];
}
}  // namespace

// ---------------------------------------------------- compressed K cache --
template <typename T>
__global__ void __launch_bounds__(128) kcache_kernel(const T* __restrict__ K, const float* __restrict__ Wk,
                                                     float* __restrict__ kt, int Hkv, int n_cap, int d, int h,
                                                     int j0, int nnew) {
  extern __shared__ float kb[];  // [3d]: max | min | avg
  const long long bhj = blockIdx.x;
  const int t = (int)(bhj % nnew);
  const long long bh = bhj / nnew;
  const int g = (int)(bh % Hkv);
  const int j = j0 + t;
  const int nb_cap = n_cap / kBlock;
  const long long row0 = (bh * n_cap + (long long)j * kBlock) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float mx = -INFINITY, mn = INFINITY, s = 0.f;
    for (int r = 0; r < kBlock; ++r) {
      const float v = ld(K, row0 + (long long)r * d + c);
      mx = fmaxf(mx, v);
      mn = fminf(mn, v);
      s += v;
    }
    kb[c] = mx;
    kb[d + c] = mn;
    kb[2 * d + c] = s * (1.0f / kBlock);
  }
  __syncthreads();
  for (int o = threadIdx.x; o < h; o += blockDim.x) {
    const float* w = Wk + ((long long)g * h + o) * 3 * d;
    float acc = 0.f;
    for (int e = 0; e < 3 * d; ++e) acc = fmaf(w[e], kb[e], acc);
    kt[(bh * nb_cap + j) * h + o] = acc;
  }
}

// ------------------------------------------------------------ gate logits --
template <typename T>
__global__ void __launch_bounds__(256) decode_logits_kernel(const T* __restrict__ q, const float* __restrict__ kt,
                                                            float* __restrict__ logits, int Hq, int Hkv, int d,
                                                            int nc, int nb_cap, float scale) {
  __shared__ float qs[256];
  const long long row = blockIdx.x;  // b * Hq + hq
  const long long b = row / Hq;
  const int hq = (int)(row % Hq), g = hq / (Hq / Hkv);
  for (int c = threadIdx.x; c < d; c += blockDim.x) qs[c] = ld(q, row * d + c);
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const float* kg = kt + (b * Hkv + g) * (long long)nb_cap * d;
  for (int j = warp; j < nc; j += blockDim.x / 32) {
    float acc = 0.f;
    for (int c = lane; c < d; c += 32) acc = fmaf(qs[c], kg[(long long)j * d + c], acc);
    acc = warp_sum(acc);
    if (lane == 0) logits[row * nc + j] = acc * scale;
  }
}

// ------------------------------------------------------ decode attention --
// 128 threads: for scores two threads per key (each half of d), for PV one
// thread per head dimension.  part: [rows, splits, d + 2] = (o[d], m, l), m
// in the log2 domain.
template <typename T>
__global__ void __launch_bounds__(128) decode_attn_kernel(const T* __restrict__ q, const T* __restrict__ K,
                                                          const T* __restrict__ V, const int32_t* __restrict__ counts,
                                                          const int32_t* __restrict__ indices, int cap, int Hq,
                                                          int Hkv, int d, int n_cap, int seq_len, float scale_log2,
                                                          int splits, float* __restrict__ part,
                                                          uint32_t* __restrict__ status) {
  __shared__ float qs[128];
  __shared__ float ps[64];
  __shared__ float sh_l;
  const long long row = blockIdx.x;
  const int split = blockIdx.y;
  const long long b = row / Hq;
  const int hq = (int)(row % Hq), g = hq / (Hq / Hkv);
  const int tid = threadIdx.x;
  const int c = (seq_len - 1) / kBlock;
  int cnt = counts[row];
  const int lim = min(cap, c);
  if (cnt < 0 || cnt > lim) {
    if (tid == 0 && split == 0) record_status(status, kDevBadIndex, (uint32_t)row);
    cnt = cnt < 0 ? 0 : lim;
  }
  for (int e = tid; e < d; e += blockDim.x) qs[e] = ld(q, row * d + e) * scale_log2;
  const long long head0 = (b * Hkv + g) * (long long)n_cap * d;
  float m = -INFINITY, l = 0.f, o = 0.f;
  const int key = tid >> 1, hp = tid & 1, half = d / 2;
  __syncthreads();
  for (int e = split; e <= cnt; e += splits) {
    int j = c, nkeys = seq_len - c * kBlock;
    if (e < cnt) {
      j = indices[row * cap + e];
      if (j < 0 || j >= c) {
        if (tid == 0) record_status(status, kDevBadIndex, (uint32_t)row);
        j = j < 0 ? 0 : c - 1;
      }
      nkeys = kBlock;
    }
    const long long kbase = head0 + (long long)j * kBlock * d;
    float acc = 0.f;
    if (key < nkeys) {
      const long long r = kbase + (long long)key * d + hp * half;
      for (int x = 0; x < half; ++x) acc = fmaf(qs[hp * half + x], ld(K, r + x), acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);  // the key's two halves
    if (hp == 0) ps[key] = key < nkeys ? acc : -INFINITY;
    __syncthreads();
    float bm = fmaxf(ps[tid & 31], ps[32 + (tid & 31)]);
    bm = warp_max(bm);
    const float mn = fmaxf(m, bm);
    const float alpha = exp2f(m - mn);
    __syncthreads();
    if (tid < kBlock) ps[tid] = exp2f(ps[tid] - mn);  // -inf for absent keys -> 0
    __syncthreads();
    if (tid < 32) {
      const float s = warp_sum(ps[tid] + ps[tid + 32]);
      if (tid == 0) sh_l = s;
    }
    if (tid < d) {
      float acc = 0.f;
      for (int k = 0; k < nkeys; ++k) acc = fmaf(ps[k], ld(V, kbase + (long long)k * d + tid), acc);
      o = o * alpha + acc;
    }
    __syncthreads();
    l = l * alpha + sh_l;
    m = mn;
    __syncthreads();
  }
  float* pp = part + (row * splits + split) * (long long)(d + 2);
  if (tid < d) pp[tid] = o;
  if (tid == 0) {
    pp[d] = m;
    pp[d + 1] = l;
  }
}

template <typename T>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part, int splits, int d,
                                                             T* __restrict__ O, float* __restrict__ lse) {
  const long long row = blockIdx.x;
  const float* pr = part + row * splits * (long long)(d + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, pr[s * (d + 2) + d]);
  float L = 0.f, acc = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = pr[s * (d + 2) + d];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    L += pr[s * (d + 2) + d + 1] * w;
    if ((int)threadIdx.x < d) acc += pr[s * (d + 2) + threadIdx.x] * w;
  }
  if ((int)threadIdx.x < d) {
    const float v = acc / L;
    if constexpr (sizeof(T) == 2)
      reinterpret_cast<__nv_bfloat16*>(O)[row * d + threadIdx.x] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(O)[row * d + threadIdx.x] = v;
  }
  if (threadIdx.x == 0 && lse) lse[row] = (M + log2f(L)) * 0.6931471805599453f;
}

// ------------------------------------------------------ 1D ground truth ---
template <typename T>
__global__ void __launch_bounds__(256) decode_gt_kernel(const T* __restrict__ q, const T* __restrict__ K, int Hq,
                                                        int Hkv, int d, int n_cap, int seq_len, float scale_log2,
                                                        float* __restrict__ gt, float* __restrict__ lse) {
  __shared__ float qs[256];
  __shared__ float wm[8], wl[8];
  __shared__ float sh_lse;
  const long long row = blockIdx.x;
  const long long b = row / Hq;
  const int hq = (int)(row % Hq), g = hq / (Hq / Hkv);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int nbc = (seq_len - 1) / kBlock + 1;  // blocks 0 .. c
  for (int e = threadIdx.x; e < d; e += blockDim.x) qs[e] = ld(q, row * d + e) * scale_log2;
  __syncthreads();
  const long long head0 = (b * Hkv + g) * (long long)n_cap * d;
  float m = -INFINITY, l = 0.f;
  for (int j = warp; j < nbc; j += 8) {
    float s2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int key = j * kBlock + 2 * lane + u;
      float acc = -INFINITY;
      if (key < seq_len) {
        acc = 0.f;
        const long long r = head0 + (long long)key * d;
        for (int x = 0; x < d; ++x) acc = fmaf(qs[x], ld(K, r + x), acc);
      }
      s2[u] = acc;
    }
    const float bm = warp_max(fmaxf(s2[0], s2[1]));
    const float mn = fmaxf(m, bm);
    const float part = warp_sum(exp2f(s2[0] - mn) + exp2f(s2[1] - mn));
    l = l * exp2f(m - mn) + part;
    m = mn;
    if (lane == 0) gt[row * nbc + j] = bm;  // raw maximum for now
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int w = 0; w < 8; ++w) M = fmaxf(M, wm[w]);
    float L = 0.f;
    for (int w = 0; w < 8; ++w)
      if (wm[w] > -INFINITY) L += wl[w] * exp2f(wm[w] - M);
    sh_lse = M + log2f(L);
    if (lse) lse[row] = sh_lse * 0.6931471805599453f;
  }
  __syncthreads();
  const float l2 = sh_lse;
  for (int j = threadIdx.x; j < nbc; j += blockDim.x) gt[row * nbc + j] = exp2f(gt[row * nbc + j] - l2);
}

// ------------------------------------------------------------- launchers --
cudaError_t launch_kcache(const void* K, bool fp32, const float* Wk, float* kt, long long BHkv, int Hkv, int n_cap,
                          int d, int h, int j0, int nnew, cudaStream_t st) {
  const size_t smem = sizeof(float) * 3 * d;
  const unsigned grid = (unsigned)(BHkv * nnew);
  if (fp32)
    kcache_kernel<float><<<grid, 128, smem, st>>>((const float*)K, Wk, kt, Hkv, n_cap, d, h, j0, nnew);
  else
    kcache_kernel<uint16_t><<<grid, 128, smem, st>>>((const uint16_t*)K, Wk, kt, Hkv, n_cap, d, h, j0, nnew);
  return cudaGetLastError();
}

cudaError_t launch_decode_logits(const void* q, bool fp32, const float* kt, float* logits, long long rows, int Hq,
                                 int Hkv, int d, int nc, int nb_cap, float scale, cudaStream_t st) {
  if (fp32)
    decode_logits_kernel<float><<<(unsigned)rows, 256, 0, st>>>((const float*)q, kt, logits, Hq, Hkv, d, nc, nb_cap,
                                                                scale);
  else
    decode_logits_kernel<uint16_t><<<(unsigned)rows, 256, 0, st>>>((const uint16_t*)q, kt, logits, Hq, Hkv, d, nc,
                                                                   nb_cap, scale);
  return cudaGetLastError();
}

cudaError_t launch_decode_attn(const DecodeAttnArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)a.rows, (unsigned)a.splits);
  if (a.fp32) {
    decode_attn_kernel<float><<<grid, 128, 0, st>>>((const float*)a.q, (const float*)a.K, (const float*)a.V,
                                                    a.counts, a.indices, a.cap, a.Hq, a.Hkv, a.d, a.n_cap, a.seq_len,
                                                    a.scale_log2, a.splits, a.part, a.status);
    decode_combine_kernel<float><<<(unsigned)a.rows, 128, 0, st>>>(a.part, a.splits, a.d, (float*)a.O, a.lse);
  } else {
    decode_attn_kernel<uint16_t><<<grid, 128, 0, st>>>((const uint16_t*)a.q, (const uint16_t*)a.K,
                                                       (const uint16_t*)a.V, a.counts, a.indices, a.cap, a.Hq, a.Hkv,
                                                       a.d, a.n_cap, a.seq_len, a.scale_log2, a.splits, a.part,
                                                       a.status);
    decode_combine_kernel<uint16_t><<<(unsigned)a.rows, 128, 0, st>>>(a.part, a.splits, a.d, (uint16_t*)a.O, a.lse);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_gt(const void* q, const void* K, bool fp32, long long rows, int Hq, int Hkv, int d,
                             int n_cap, int seq_len, float scale_log2, float* gt, float* lse, cudaStream_t st) {
  if (fp32)
    decode_gt_kernel<float><<<(unsigned)rows, 256, 0, st>>>((const float*)q, (const float*)K, Hq, Hkv, d, n_cap,
                                                            seq_len, scale_log2, gt, lse);
  else
    decode_gt_kernel<uint16_t><<<(unsigned)rows, 256, 0, st>>>((const uint16_t*)q, (const uint16_t*)K, Hq, Hkv, d,
                                                               n_cap, seq_len, scale_log2, gt, lse);
  return cudaGetLastError();
}

}  // namespace seer
