// gate.cu -- the AttnGate of SeerAttention and the binary block-mask step, as
// CUDA kernels for sm_100a.
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4 ("AttnGate", "Pooling Method
// Selection", "Block-Level RoPE", Eq. 1, "Generating the binary block mask")
// and the OpenReview rebuttal, section 3.3 (top-k indices [S/B, k];
// threshold mask o > threshold).
//
// Kernels (all HBM- or latency-bound; none is a dense contraction worth the
// tensor cores -- the gate is ~1/4096 of the attention map):
//   pool_kernel      Q avg-pool / K [max|min|avg]-pool, one warp per block,
//                    16-byte vector loads, shuffle reductions
//   gemm_nt_kernel   fp32 SIMT tile GEMM: gate projections and the causal
//                    block logits q~ k~^T / sqrt(d) (upper tiles skipped)
//   rope_kernel      optional block-level RoPE on q~ / k~
//   row_select_kernel  one CTA per score row: causal softmax (Eq. 1), optional
//                    score write-out, then threshold compaction or exact top-k
//                    (radix select on the fp32 bit patterns, ties to lower j)
#include <cstdint>

#include "common.cuh"
#include "gate.cuh"

namespace seer {

// ------------------------------------------------------------------ pool --
// One warp per (head, block i).  Every lane loads 16 bytes of a row per step;
// lanes that cover the same columns are combined with shuffles at the end.
template <typename T, bool IS_K>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ X, long long nblocks,
                                                   int n, int d, float* __restrict__ out) {
  constexpr int EPL = 16 / sizeof(T);  // elements per lane per load
  const long long warp = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (warp >= nblocks) return;
  const int lane = threadIdx.x & 31;
  const int nb = n / kBlock;
  const long long bh = warp / nb;
  const int i = (int)(warp % nb);
  const int lpr = d / EPL;    // lanes per row
  const int rpi = 32 / lpr;   // rows per iteration
  const int cg = lane % lpr;  // column group of this lane
  const T* base = X + ((bh * n) + (long long)i * kBlock) * d + cg * EPL;

  float sum[EPL], mx[EPL], mn[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    sum[e] = 0.f;
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
  for (int r = lane / lpr; r < kBlock; r += rpi) {
    uint4 v = *reinterpret_cast<const uint4*>(base + (long long)r * d);
    float f[EPL];
    if constexpr (sizeof(T) == 2) {
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    } else {
      f[0] = __uint_as_float(v.x);
      f[1] = __uint_as_float(v.y);
      f[2] = __uint_as_float(v.z);
      f[3] = __uint_as_float(v.w);
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sum[e] += f[e];
      if (IS_K) {
        mx[e] = fmaxf(mx[e], f[e]);
        mn[e] = fminf(mn[e], f[e]);
      }
    }
  }
  for (int o = lpr; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], o);
      if (IS_K) {
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], o));
        mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], o));
      }
    }
  }
  if (lane < lpr) {
    if (!IS_K) {
      float* o = out + ((bh * nb) + i) * (long long)d + cg * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = sum[e] * (1.0f / kBlock);
    } else {
      float* o = out + ((bh * nb) + i) * (long long)(3 * d) + cg * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        o[e] = mx[e];
        o[d + e] = mn[e];
        o[2 * d + e] = sum[e] * (1.0f / kBlock);
      }
    }
  }
}

// ------------------------------------------------------------------ gemm --
// C[z][m][c] = alpha * sum_k A[z][m][k] * B[bz][c][k]; A is M x K and B is
// N x K (both row-major), C has leading dimension ldc.  The B batch index is
// bz = (z / zh) * zmul + (z % zh) / zg (per-head weights, or the KV head of a
// query head).  With CAUSAL, tiles strictly above the diagonal are skipped.
template <bool CAUSAL>
__global__ void __launch_bounds__(256) gemm_nt_kernel(const float* __restrict__ A,
                                                      const float* __restrict__ B,
                                                      float* __restrict__ C, int M, int N, int K,
                                                      long long a_bs, long long b_bs,
                                                      long long c_bs, int ldc, int zh, int zmul,
                                                      int zg, float alpha) {
  const int tm = blockIdx.x, tn = blockIdx.y, z = blockIdx.z;
  if (CAUSAL && tn > tm) return;
  const float* Ab = A + z * a_bs;
  const int bz = (z / zh) * zmul + (z % zh) / zg;
  const float* Bb = B + bz * b_bs;
  float* Cb = C + z * c_bs;
  __shared__ float As[32][65];
  __shared__ float Bs[32][65];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int e = tid; e < 64 * 32; e += 256) {
      const int r = e / 32, c = e % 32;
      const int gk = k0 + c;
      const int gm = tm * 64 + r, gn = tn * 64 + r;
      As[c][r] = (gm < M && gk < K) ? Ab[(long long)gm * K + gk] : 0.f;
      Bs[c][r] = (gn < N && gk < K) ? Bb[(long long)gn * K + gk] : 0.f;
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
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int gm = tm * 64 + ty * 4 + p;
    if (gm >= M) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int gn = tn * 64 + tx * 4 + q;
      if (gn < N) Cb[(long long)gm * ldc + gn] = alpha * acc[p][q];
    }
  }
}

// ------------------------------------------------------------------ rope --
// Block-level RoPE (summary page, "Block-Level RoPE": theta' = theta / B,
// applied after the projections, at block positions).  Pairs (c, c + h/2);
// the frequency of pair c is base'^(-2c/h); in place on x [rows, h].
__global__ void rope_kernel(float* __restrict__ x, long long rows, int nb, int h, float base) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int half = h / 2;
  if (t >= rows * half) return;
  const long long row = t / half;
  const int c = (int)(t % half);
  const int pos = (int)(row % nb);
  const double freq = pow((double)base, -2.0 * c / (double)h);
  double sn, cs;
  sincos((double)pos * freq, &sn, &cs);
  float* v = x + row * h;
  const float a = v[c], b = v[c + half];
  v[c] = (float)(a * cs - b * sn);
  v[c + half] = (float)(b * cs + a * sn);
}

// ----------------------------------------------------------- row select --
constexpr int kRowThreads = 256;

// Exclusive scan of one int per thread across the CTA; returns the prefix and
// writes the total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh /*[32]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sh[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int before = warp > 0 ? sh[warp - 1] : 0;
  const int tot = sh[nw - 1];
  __syncthreads();
  *total = tot;
  return before + x - v;
}

__device__ __forceinline__ float block_reduce_max(float v, float* sh) {
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, sh[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* sh) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += sh[w];
  __syncthreads();
  return r;
}

// Order-preserving map of an fp32 bit pattern to uint32 (larger float ->
// larger key).
__device__ __forceinline__ uint32_t f2key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Number of blocks row i keeps under a top-k mode.
__device__ __forceinline__ int topk_count(int i, int mode, int k, float density) {
  int ki;
  if (mode == SEER_SELECT_TOPK_K) {
    ki = k;
  } else {
    ki = (int)ceilf(__fmul_rn(density, (float)(i + 1)));
    if (ki < 1) ki = 1;
  }
  return ki < i + 1 ? ki : i + 1;
}

// One CTA per score row r (query block i = r % nb).  With FROM_LOGITS the row
// holds causal logits q~.k~/sqrt(d): it is turned into Eq. 1's softmax over
// j <= i (written to `scores` when non-null; j > i written as 0).  Otherwise
// the row already holds scores.  Then the active blocks are written as an
// ascending list.
template <bool FROM_LOGITS>
__global__ void __launch_bounds__(kRowThreads) row_select_kernel(
    const float* in, float* scores, int nb, int mode, float T, int k,
    float density, int32_t* __restrict__ counts, int32_t* __restrict__ indices, int cap, int row_len) {
  extern __shared__ float sv[];  // [nb]
  __shared__ int sh_i[32];
  __shared__ float sh_f[32];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel_prefix, sel_remaining;

  const long long row = blockIdx.x;
  // causal prefill rows: query block i = row % nb; row_len > 0: every row
  // has row_len candidates (the decode gate)
  const int i = row_len > 0 ? row_len - 1 : (int)(row % nb);
  const int len = i + 1;
  const int tid = threadIdx.x;
  const float* src = in + row * (long long)nb;

  for (int j = tid; j < len; j += kRowThreads) sv[j] = src[j];
  __syncthreads();

  if (FROM_LOGITS) {
    float m = -INFINITY;
    for (int j = tid; j < len; j += kRowThreads) m = fmaxf(m, sv[j]);
    m = block_reduce_max(m, sh_f);
    float s = 0.f;
    for (int j = tid; j < len; j += kRowThreads) {
      const float e = expf(sv[j] - m);
      sv[j] = e;
      s += e;
    }
    s = block_reduce_sum(s, sh_f);
    for (int j = tid; j < len; j += kRowThreads) sv[j] = sv[j] / s;
    __syncthreads();
    if (scores != nullptr) {
      float* dst = scores + row * (long long)nb;
      for (int j = tid; j < nb; j += kRowThreads) dst[j] = j < len ? sv[j] : 0.f;
    }
  }

  // Each thread owns a contiguous chunk so that compaction keeps ascending j.
  const int chunk = (len + kRowThreads - 1) / kRowThreads;
  const int j0 = tid * chunk;
  const int j1 = min(j0 + chunk, len);
  int32_t* out = indices + row * (long long)cap;

  if (mode == SEER_SELECT_THRESHOLD) {
    int c = 0;
    for (int j = j0; j < j1; ++j) c += sv[j] > T;
    int total;
    int pos = block_exclusive_scan(c, sh_i, &total);
    for (int j = j0; j < j1; ++j)
      if (sv[j] > T) out[pos++] = j;
    if (tid == 0) counts[row] = total;
    return;
  }

  const int ki = topk_count(i, mode, k, density);
  if (ki >= len) {  // every causal block is kept
    for (int j = tid; j < len; j += kRowThreads) out[j] = j;
    if (tid == 0) counts[row] = len;
    return;
  }

  // Radix select of the ki-th largest key, 8 bits at a time from the top.
  uint32_t prefix = 0, pmask = 0;
  uint32_t remaining = (uint32_t)ki;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kRowThreads) hist[b] = 0;
    __syncthreads();
    // Scores of a row share their top bits, so most keys fall into a few
    // bins: lanes with the same bin are counted by one atomic (match_any).
    for (int j0 = 0; j0 < len; j0 += kRowThreads) {
      const int j = j0 + tid;
      uint32_t bin = 0x100u;  // not counted
      if (j < len) {
        const uint32_t key = f2key(sv[j]);
        if ((key & pmask) == prefix) bin = (key >> shift) & 0xffu;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0x100u && (tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      uint32_t cnt[8];
      uint32_t part = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = hist[255 - 8 * tid - q];
        part += cnt[q];
      }
      uint32_t incl = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const uint32_t excl = incl - part;
      if (excl < remaining && remaining <= incl) {
        uint32_t before = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (before < remaining && remaining <= before + cnt[q]) {
            sel_prefix = prefix | ((uint32_t)(255 - 8 * tid - q) << shift);
            sel_remaining = remaining - before;
          }
          before += cnt[q];
        }
      }
    }
    __syncthreads();
    prefix = sel_prefix;
    remaining = sel_remaining;
    pmask |= 0xffu << shift;
    __syncthreads();
  }
  // keys > prefix are all kept; of the keys == prefix, the `remaining` ones
  // with the lowest j are kept.
  int eq = 0;
  for (int j = j0; j < j1; ++j) eq += f2key(sv[j]) == prefix;
  int eq_total;
  int eq_rank = block_exclusive_scan(eq, sh_i, &eq_total);
  int c = 0;
  {
    int r = eq_rank;
    for (int j = j0; j < j1; ++j) {
      const uint32_t key = f2key(sv[j]);
      if (key > prefix) {
        ++c;
      } else if (key == prefix) {
        if ((uint32_t)r < remaining) ++c;
        ++r;
      }
    }
  }
  int total;
  int pos = block_exclusive_scan(c, sh_i, &total);
  {
    int r = eq_rank;
    for (int j = j0; j < j1; ++j) {
      const uint32_t key = f2key(sv[j]);
      bool keep = false;
      if (key > prefix) {
        keep = true;
      } else if (key == prefix) {
        keep = (uint32_t)r < remaining;
        ++r;
      }
      if (keep) out[pos++] = j;
    }
  }
  if (tid == 0) counts[row] = total;
}

// --------------------------------------------------------------- launchers --
cudaError_t launch_pool(const void* X, seer_dtype dt, bool is_k, long long BH, int n, int d,
                        float* out, cudaStream_t st) {
  const long long nblocks = BH * (n / kBlock);
  const int warps = 8;
  const unsigned grid = (unsigned)((nblocks + warps - 1) / warps);
  if (dt == SEER_BF16) {
    if (is_k)
      pool_kernel<uint16_t, true><<<grid, warps * 32, 0, st>>>((const uint16_t*)X, nblocks, n, d, out);
    else
      pool_kernel<uint16_t, false><<<grid, warps * 32, 0, st>>>((const uint16_t*)X, nblocks, n, d, out);
  } else {
    if (is_k)
      pool_kernel<float, true><<<grid, warps * 32, 0, st>>>((const float*)X, nblocks, n, d, out);
    else
      pool_kernel<float, false><<<grid, warps * 32, 0, st>>>((const float*)X, nblocks, n, d, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm_nt(const float* A, const float* B, float* C, int M, int N, int K,
                           long long a_bs, long long b_bs, long long c_bs, int ldc, int batch,
                           int zh, int zmul, int zg, float alpha, bool causal, cudaStream_t st) {
  dim3 grid((M + 63) / 64, (N + 63) / 64, batch);
  if (causal)
    gemm_nt_kernel<true><<<grid, 256, 0, st>>>(A, B, C, M, N, K, a_bs, b_bs, c_bs, ldc, zh, zmul,
                                               zg, alpha);
  else
    gemm_nt_kernel<false><<<grid, 256, 0, st>>>(A, B, C, M, N, K, a_bs, b_bs, c_bs, ldc, zh, zmul,
                                                zg, alpha);
  return cudaGetLastError();
}

cudaError_t launch_rope(float* x, long long rows, int nb, int h, float theta, cudaStream_t st) {
  const long long total = rows * (h / 2);
  const unsigned grid = (unsigned)((total + 255) / 256);
  rope_kernel<<<grid, 256, 0, st>>>(x, rows, nb, h, theta / (float)kBlock);
  return cudaGetLastError();
}

cudaError_t launch_row_select(const float* in, float* scores, bool from_logits, long long rows,
                              int nb, int mode, float T, int k, float density, int32_t* counts,
                              int32_t* indices, int cap, cudaStream_t st, int row_len) {
  const size_t smem = (size_t)nb * sizeof(float);
  if (from_logits) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(row_select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
    row_select_kernel<true><<<(unsigned)rows, kRowThreads, smem, st>>>(
        in, scores, nb, mode, T, k, density, counts, indices, cap, row_len);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(row_select_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
    row_select_kernel<false><<<(unsigned)rows, kRowThreads, smem, st>>>(
        in, nullptr, nb, mode, T, k, density, counts, indices, cap, row_len);
  }
  return cudaGetLastError();
}

}  // namespace seer
