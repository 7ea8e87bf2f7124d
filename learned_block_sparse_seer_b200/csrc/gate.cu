// gate.cu -- the AttnGate of SeerAttention and the binary block-mask step, as
// CUDA kernels for sm_100a.
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4 ("AttnGate", "Pooling Method
// Selection", "Block-Level RoPE", Eq. 1, "Generating the binary block mask")
// and the OpenReview rebuttal, section 3.3 (top-k indices [S/B, k];
// threshold mask o > threshold).
//
// Kernels (the gate is ~1/4096 of the attention map; pooling is HBM-bound,
// the rest small):
//   pool_kernel      Q avg-pool / K [max|min|avg]-pool, one warp per block,
//                    16-byte vector loads, shuffle reductions
//   gemm_nt_kernel   fp32 SIMT tile GEMM: gate projections, and the causal
//                    block logits q~ k~^T / sqrt(d) (upper tiles skipped) when
//                    h is not a multiple of 32; gemm_nt128_kernel is its
//                    128 x 128-tile form for K % 16 == 0
//   split_tf32_kernel + gemm_tf32x3_kernel
//                    the causal block logits on the tf32 tensor cores (tcgen05)
//                    when h % 32 == 0: three products of tf32 parts (hi*hi +
//                    hi*lo + lo*hi) keep fp32-level accuracy
//   rope_kernel      optional block-level RoPE on q~ / k~
//   row_select_warp_kernel / row_select_kernel
//                    one warp (many rows of <= 2048 candidates) or one CTA per
//                    score row: causal softmax (Eq. 1), optional score
//                    write-out, then threshold compaction or exact top-k
//                    (radix select on the fp32 bit patterns, ties to lower j)
#include <cstdint>

#include "common.cuh"
#include "gate.cuh"
#include "ptx.cuh"
#include "tf32mma.cuh"

namespace seer {

// ------------------------------------------------------------------ pool --
// One warp per (head, block i).  Every lane loads 16 bytes of a row per step;
// lanes that cover the same columns are combined with shuffles at the end.
// With a varlen table, block i pools only its tab[i].y valid tokens (the
// sequence's last block may be partial); a block of no sequence writes 0.
template <typename T, bool IS_K>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ X, long long nblocks,
                                                   int n, int d, float* __restrict__ out,
                                                   const int2* __restrict__ tab) {
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
  const int valid = tab ? tab[i].y : kBlock;  // tokens of the block that belong to a sequence

  float sum[EPL], mx[EPL], mn[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    sum[e] = 0.f;
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
  for (int r = lane / lpr; r < valid; r += rpi) {
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
    const float inv = valid > 0 ? 1.0f / (float)valid : 0.f;
    if (!IS_K) {
      float* o = out + ((bh * nb) + i) * (long long)d + cg * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = sum[e] * inv;
    } else {
      float* o = out + ((bh * nb) + i) * (long long)(3 * d) + cg * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        o[e] = valid > 0 ? mx[e] : 0.f;
        o[d + e] = valid > 0 ? mn[e] : 0.f;
        o[2 * d + e] = sum[e] * inv;
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

// The same product with 128 x 128 tiles, for K % 16 == 0 and 16-byte aligned
// A/B rows: 256 threads, each owning an 8 x 8 block of outputs (rows
// 4*ty + {0..3} and 64 + 4*ty + {0..3}, columns likewise with tx), so every
// k step takes four 16-byte shared loads for 64 FMAs.  k slices of 16 are
// staged transposed ([k][m]) in two shared buffers; the next slice's global
// loads are in flight while the current one is multiplied.
template <bool CAUSAL>
__global__ void __launch_bounds__(256, 1) gemm_nt128_kernel(const float* __restrict__ A,
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
  __shared__ __align__(16) float As[2][16][132];
  __shared__ __align__(16) float Bs[2][16][132];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // this thread's two 16-byte global loads per operand and slice: float4
  // f = tid + 256 s covers row f / 4, k offset 4 * (f % 4)
  float4 ra[2], rb[2];
  auto gload = [&](int k0) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int f = tid + 256 * s, r = f >> 2, kq = (f & 3) * 4;
      const int gm = tm * 128 + r, gn = tn * 128 + r;
      ra[s] = gm < M ? *reinterpret_cast<const float4*>(Ab + (long long)gm * K + k0 + kq)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
      rb[s] = gn < N ? *reinterpret_cast<const float4*>(Bb + (long long)gn * K + k0 + kq)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto sstore = [&](int buf) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int f = tid + 256 * s, r = f >> 2, kq = (f & 3) * 4;
      As[buf][kq][r] = ra[s].x;
      As[buf][kq + 1][r] = ra[s].y;
      As[buf][kq + 2][r] = ra[s].z;
      As[buf][kq + 3][r] = ra[s].w;
      Bs[buf][kq][r] = rb[s].x;
      Bs[buf][kq + 1][r] = rb[s].y;
      Bs[buf][kq + 2][r] = rb[s].z;
      Bs[buf][kq + 3][r] = rb[s].w;
    }
  };
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  gload(0);
  sstore(0);
  __syncthreads();
  const int nk = K / 16;
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) gload((kt + 1) * 16);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    // the other buffer was last read in the previous slice, before the
    // barrier that ended it
    if (kt + 1 < nk) sstore(buf ^ 1);
    __syncthreads();
  }
  const bool vec = (ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(Cb) & 15) == 0;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int gm = tm * 128 + (p >> 2) * 64 + ty * 4 + (p & 3);
    if (gm >= M) continue;
    float* crow = Cb + (long long)gm * ldc;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gn = tn * 128 + h * 64 + tx * 4;
      if (vec && gn + 3 < N) {
        *reinterpret_cast<float4*>(crow + gn) = make_float4(alpha * acc[p][4 * h], alpha * acc[p][4 * h + 1],
                                                            alpha * acc[p][4 * h + 2], alpha * acc[p][4 * h + 3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (gn + q < N) crow[gn + q] = alpha * acc[p][4 * h + q];
      }
    }
  }
}

// ------------------------------------------------------ tf32x3 logits --
// The causal block logits on the tensor cores with fp32-level accuracy: each
// fp32 operand is split into a tf32 part and its remainder (hi = x rounded
// to tf32, lo = x - hi, both exact in fp32) and C = alpha (Ah Bh^T + Ah Bl^T
// + Al Bh^T); the dropped Al Bl^T term and lo's own tf32 rounding leave a
// relative error near 2^-21 per product.  One CTA per 128 x 128 tile of C
// (tiles strictly above the diagonal skipped): warp 0 loads 32-column
// k slices of the four operands by TMA (no cluster multicast) into a
// 3-stage ring, warp 1 issues the tcgen05 MMAs into a 128-column TMEM
// accumulator, then all four warps read it back (TMEM lane = tile row).
__global__ void split_tf32_kernel(float* __restrict__ x, float* __restrict__ lo, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = x[i];
    uint32_t h;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(v));
    const float hi = __uint_as_float(h);
    x[i] = hi;
    lo[i] = v - hi;
  }
}

__global__ void split_tf32_copy_kernel(const float* __restrict__ x, float* __restrict__ hi_out,
                                       float* __restrict__ lo, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = x[i];
    uint32_t h;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(v));
    const float hi = __uint_as_float(h);
    hi_out[i] = hi;
    lo[i] = v - hi;
  }
}

namespace gt3 {
// One stage of 64 KB per CTA: three CTAs share an SM, so one tile's loads,
// products and epilogue overlap the others' (a tile is only four 32-float
// slices deep, too short to pipeline within one CTA).
constexpr int kStages = 1;
constexpr uint32_t kOp = 128u * 128u;                 // one operand slice: 128 rows x 32 floats
constexpr uint32_t kStage = 4u * kOp;                 // Ah, Al, Bh, Bl
constexpr uint32_t kSmem = kStages * kStage + 1024u;  // + slack to align the ring to 1024 bytes
}  // namespace gt3

__global__ void __launch_bounds__(128, 1) gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmAh,
                                                             const __grid_constant__ CUtensorMap tmAl,
                                                             const __grid_constant__ CUtensorMap tmBh,
                                                             const __grid_constant__ CUtensorMap tmBl,
                                                             const Tf32x3Params p) {
  using namespace gt3;
  const int tm = blockIdx.x, tn = blockIdx.y, z = blockIdx.z;
  if (p.causal && tn > tm) return;  // causal: tiles strictly above the diagonal are never read
  extern __shared__ uint8_t gt3_raw[];
  uint8_t* const ring = gt3_raw + ((1024u - (smem_u32(gt3_raw) & 1023u)) & 1023u);
  __shared__ uint64_t full[kStages], empty[kStages], done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int issued, consumed;  // slices whose copies went out / whose products were issued
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_p = &abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    issued = consumed = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int nk = p.K / 32;
  const int arow = z * p.M + tm * 128;
  const int bz = (z / p.zh) * p.zmul + (z % p.zh) / p.zg;
  const int brow = bz * p.N + tn * 128;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmAh);
    prefetch_tmap(&tmAl);
    prefetch_tmap(&tmBh);
    prefetch_tmap(&tmBl);
    for (int c = 0; c < nk; ++c) {
      const int s = c % kStages;
      if (c >= kStages && !mbar_wait(&empty[s], ((c / kStages) - 1) & 1, abort_p, p.status, p.timeout_ns)) break;
      mbar_arrive_expect_tx(&full[s], kStage);
      uint8_t* const st = ring + s * kStage;
      tma_load_2d(st, &tmAh, &full[s], c * 32, arow);
      tma_load_2d(st + kOp, &tmAl, &full[s], c * 32, arow);
      tma_load_2d(st + 2 * kOp, &tmBh, &full[s], c * 32, brow);
      tma_load_2d(st + 3 * kOp, &tmBl, &full[s], c * 32, brow);
      issued = c + 1;
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = make_idesc_tf32(128, 128, 0, 0);  // A and B K-major
    const uint32_t rbase = smem_u32(ring);
    for (int c = 0; c < nk; ++c) {
      const int s = c % kStages;
      if (!mbar_wait(&full[s], (c / kStages) & 1, abort_p, p.status, p.timeout_ns)) break;
      tc_fence_after();
      const uint64_t dAh = make_sw128_desc(rbase + s * kStage, 16, 1024);
      const uint64_t dAl = dAh + (kOp >> 4), dBh = dAh + ((2 * kOp) >> 4), dBl = dAh + ((3 * kOp) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t off = (uint64_t)((kk * 32) >> 4);  // 8 floats = 32 bytes per k step
        mma_tf32_ss(tmem, dAh + off, dBh + off, idesc, (c > 0 || kk > 0) ? 1u : 0u);
        mma_tf32_ss(tmem, dAh + off, dBl + off, idesc, 1u);
        mma_tf32_ss(tmem, dAl + off, dBh + off, idesc, 1u);
      }
      mma_commit(&empty[s]);
      consumed = c + 1;
    }
    // issued even after a failed wait: it arrives once this thread's MMAs are done
    mma_commit(&done);
  }
  __syncwarp();
  const bool ok = mbar_wait(&done, 0, abort_p, p.status, p.timeout_ns) && *abort_p == 0;
  tc_fence_after();
  const int r = warp * 32 + lane;  // TMEM lane = tile row
  const int gm = tm * 128 + r;
  float* const crow = p.C + (long long)z * p.c_bs + (long long)gm * p.ldc;
  const bool vec = (p.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(p.C + (long long)z * p.c_bs) & 15) == 0;
#pragma unroll 1
  for (int c0 = 0; c0 < 128; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    const int gn = tn * 128 + c0;
    if (ok && gm < p.M && gn < p.N) {
      if (vec && gn + 32 <= p.N) {
#pragma unroll
        for (int q = 0; q < 32; q += 4)
          *reinterpret_cast<float4*>(crow + gn + q) =
              make_float4(p.alpha * __uint_as_float(v[q]), p.alpha * __uint_as_float(v[q + 1]),
                          p.alpha * __uint_as_float(v[q + 2]), p.alpha * __uint_as_float(v[q + 3]));
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (gn + q < p.N) crow[gn + q] = p.alpha * __uint_as_float(v[q]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 128);
  // After an abort, the copies of slices that were issued but never consumed
  // may still be in flight: each completes its stage's full phase (armed by
  // the loader alone), so wait (bounded) for those phases before the shared
  // memory is released.
  if (threadIdx.x == 0 && *abort_p) {
    for (int c = consumed > issued - kStages ? consumed : issued - kStages; c < issued; ++c) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_sleep(&full[c % kStages], (c / kStages) & 1, 20000u))
        if (globaltimer_ns() - t0 > 20000000ull) break;
    }
  }
}

cudaError_t launch_gemm_tf32x3_causal(const CUtensorMap& tmAh, const CUtensorMap& tmAl, const CUtensorMap& tmBh,
                                      const CUtensorMap& tmBl, const Tf32x3Params& p, int batch, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gemm_tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gt3::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.M + 127) / 128, (p.N + 127) / 128, batch);
  gemm_tf32x3_kernel<<<grid, 128, gt3::kSmem, st>>>(tmAh, tmAl, tmBh, tmBl, p);
  return cudaGetLastError();
}

cudaError_t launch_split_tf32(float* x, float* lo, long long n, cudaStream_t st) {
  split_tf32_kernel<<<1184, 256, 0, st>>>(x, lo, n);
  return cudaGetLastError();
}

cudaError_t launch_split_tf32_copy(const float* x, float* hi, float* lo, long long n, cudaStream_t st) {
  split_tf32_copy_kernel<<<592, 256, 0, st>>>(x, hi, lo, n);
  return cudaGetLastError();
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
//  * mode carries SEER_SELECT_FORCE_DIAGONAL as a flag: block i joins the
//    list whatever its score.
//  * row_len > 0 (the decode gate): every row has row_len candidates.
//  * tab (varlen packing): row i's candidates are its own sequence's blocks
//    f .. i with f = tab[i].x (none when f < 0); k_i is taken at the local
//    row i - f, and the list holds global block indices.
template <bool FROM_LOGITS, int NT>
__global__ void __launch_bounds__(NT) row_select_kernel(
    const float* in, float* scores, int nb, int mode_flags, float T, int k,
    float density, int32_t* __restrict__ counts, int32_t* __restrict__ indices, int cap, int row_len,
    const int2* __restrict__ tab) {
  extern __shared__ float sv[];  // [nb]
  __shared__ int sh_i[32];
  __shared__ float sh_f[32];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel_prefix, sel_remaining;

  const int mode = mode_flags & 0xff;
  const bool force_diag = (mode_flags & SEER_SELECT_FORCE_DIAGONAL) != 0;
  const long long row = blockIdx.x;
  const int ig = row_len > 0 ? row_len - 1 : (int)(row % nb);  // query block (global)
  const int off = tab ? tab[ig].x : 0;  // first candidate block
  const int tid = threadIdx.x;
  if (off < 0) {  // a block of no sequence: no candidates
    if (FROM_LOGITS && scores != nullptr) {
      float* dst = scores + row * (long long)nb;
      for (int j = tid; j < nb; j += NT) dst[j] = 0.f;
    }
    if (tid == 0) counts[row] = 0;
    return;
  }
  const int i = ig - off;  // local query block: candidates are local 0 .. i
  const int len = i + 1;
  const float* src = in + row * (long long)nb + off;

  for (int j = tid; j < len; j += NT) sv[j] = src[j];
  __syncthreads();

  if (FROM_LOGITS) {
    float m = -INFINITY;
    for (int j = tid; j < len; j += NT) m = fmaxf(m, sv[j]);
    m = block_reduce_max(m, sh_f);
    float s = 0.f;
    for (int j = tid; j < len; j += NT) {
      const float e = expf(sv[j] - m);
      sv[j] = e;
      s += e;
    }
    s = block_reduce_sum(s, sh_f);
    for (int j = tid; j < len; j += NT) sv[j] = sv[j] / s;
    __syncthreads();
    if (scores != nullptr) {
      float* dst = scores + row * (long long)nb;
      for (int j = tid; j < nb; j += NT) dst[j] = (j >= off && j - off < len) ? sv[j - off] : 0.f;
    }
  }

  // Each thread owns a contiguous chunk so that compaction keeps ascending j.
  const int chunk = (len + NT - 1) / NT;
  const int j0 = tid * chunk;
  const int j1 = min(j0 + chunk, len);
  int32_t* out = indices + row * (long long)cap;

  if (mode == SEER_SELECT_THRESHOLD) {
    int c = 0;
    for (int j = j0; j < j1; ++j) c += sv[j] > T || (force_diag && j == i);
    int total;
    int pos = block_exclusive_scan(c, sh_i, &total);
    for (int j = j0; j < j1; ++j)
      if (sv[j] > T || (force_diag && j == i)) out[pos++] = j + off;
    if (tid == 0) counts[row] = total;
    return;
  }

  const int ki = topk_count(i, mode, k, density);
  if (ki >= len) {  // every causal block is kept
    for (int j = tid; j < len; j += NT) out[j] = j + off;
    if (tid == 0) counts[row] = len;
    return;
  }

  // Radix select of the ki-th largest key, 8 bits at a time from the top.
  uint32_t prefix = 0, pmask = 0;
  uint32_t remaining = (uint32_t)ki;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += NT) hist[b] = 0;
    __syncthreads();
    // Scores of a row share their top bits, so most keys fall into a few
    // bins: lanes with the same bin are counted by one atomic (match_any).
    for (int j0 = 0; j0 < len; j0 += NT) {
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
      bool keep = force_diag && j == i;
      if (key > prefix) {
        keep = true;
      } else if (key == prefix) {
        keep = keep || (uint32_t)r < remaining;
        ++r;
      }
      c += keep;
    }
  }
  int total;
  int pos = block_exclusive_scan(c, sh_i, &total);
  {
    int r = eq_rank;
    for (int j = j0; j < j1; ++j) {
      const uint32_t key = f2key(sv[j]);
      bool keep = force_diag && j == i;
      if (key > prefix) {
        keep = true;
      } else if (key == prefix) {
        keep = keep || (uint32_t)r < remaining;
        ++r;
      }
      if (keep) out[pos++] = j + off;
    }
  }
  if (tid == 0) counts[row] = total;
}

// The same selection with one warp per row, for many rows of at most
// kSelMaxWidth candidates (the prefill gate): the row lives in shared memory
// (one buffer per warp; lane l owns candidates j = 32 t + l), reductions are
// warp shuffles, the radix histogram is the warp's own 256 shared bins, and
// the ascending lists are compacted with ballots, so no CTA barrier is taken.
// Every loop over the row is a short rolled loop: fully unrolled register
// copies of the row made the kernel wait on instruction fetch.  The softmax
// multiplies by the reciprocal of the row sum; the key order, ties to the
// lower j, the forced diagonal and varlen windows follow row_select_kernel.
constexpr int kSelWarps = 8;
constexpr int kSelMaxWidth = 4096;
template <bool FROM_LOGITS>
__global__ void __launch_bounds__(32 * kSelWarps) row_select_warp_kernel(
    const float* in, float* scores, long long rows, int nb, int mode_flags, float T, int k, float density,
    int32_t* __restrict__ counts, int32_t* __restrict__ indices, int cap, int row_len, const int2* __restrict__ tab) {
  extern __shared__ uint32_t sel_smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kSelWarps + wid;
  if (row >= rows) return;  // whole warps only: no CTA barrier follows
  const int width = row_len > 0 ? row_len : nb;  // candidates of a row, at most
  uint32_t* const hist = sel_smem + wid * 256;
  float* const buf = reinterpret_cast<float*>(sel_smem + kSelWarps * 256) + (size_t)wid * width;
  uint32_t* const key = reinterpret_cast<uint32_t*>(buf);
  const unsigned lt = (1u << lane) - 1u;

  const int mode = mode_flags & 0xff;
  const bool force_diag = (mode_flags & SEER_SELECT_FORCE_DIAGONAL) != 0;
  const int ig = row_len > 0 ? row_len - 1 : (int)(row % nb);
  const int off = tab ? tab[ig].x : 0;
  float* const dst = (FROM_LOGITS && scores != nullptr) ? scores + row * (long long)nb : nullptr;
  if (off < 0) {
    if (dst)
      for (int j = lane; j < nb; j += 32) dst[j] = 0.f;
    if (lane == 0) counts[row] = 0;
    return;
  }
  const int i = ig - off;
  const int len = i + 1;
  const int nt = (len + 31) >> 5;  // 32-candidate chunks
  const float* src = in + row * (long long)nb + off;
  // The row into shared memory.  Lane sums run in the same candidate order
  // as the per-row kernels' (j = lane, lane + 32, ...), then one butterfly.
  float m = -INFINITY;
#pragma unroll 4
  for (int j = lane; j < len; j += 32) {
    const float x = src[j];
    buf[j] = x;
    m = fmaxf(m, x);
  }
  if (FROM_LOGITS) {
    m = warp_max(m);
    float sum = 0.f;
#pragma unroll 4
    for (int j = lane; j < len; j += 32) {
      const float e = expf(buf[j] - m);
      buf[j] = e;
      sum += e;
    }
    const float inv = 1.0f / warp_sum(sum);
#pragma unroll 4
    for (int j = lane; j < len; j += 32) {
      const float v = buf[j] * inv;
      buf[j] = v;
      if (dst) dst[off + j] = v;
    }
    if (dst)
      for (int j = lane; j < nb; j += 32)
        if (j < off || j >= off + len) dst[j] = 0.f;
  }
  int32_t* out = indices + row * (long long)cap;

  if (mode == SEER_SELECT_THRESHOLD) {
    int base = 0;
    for (int t = 0; t < nt; ++t) {
      const int j = 32 * t + lane;
      const bool keep = j < len && (buf[j] > T || (force_diag && j == i));
      const unsigned km = __ballot_sync(0xffffffffu, keep);
      if (keep) out[base + __popc(km & lt)] = j + off;
      base += __popc(km);
    }
    if (lane == 0) counts[row] = base;
    return;
  }

  const int ki = topk_count(i, mode, k, density);
  if (ki >= len) {
    for (int j = lane; j < len; j += 32) out[j] = j + off;
    if (lane == 0) counts[row] = len;
    return;
  }

  // Order-preserving keys replace the values.  Radix select of the ki-th
  // largest key, 8 bits at a time.  Bits that all of the row's keys share
  // are fixed at once (a warp AND / OR of the keys): a softmax row's values
  // lie close together, so its keys agree on the sign, the exponent and the
  // top of the mantissa, and the first digit starts at the highest bit where
  // they differ.  The search also stops as soon as the bin holding the ki-th
  // key is taken whole.
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll 4
  for (int j = lane; j < len; j += 32) {
    const uint32_t kk = f2key(buf[j]);
    key[j] = kk;
    kand &= kk;
    kor |= kk;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    kor |= __shfl_xor_sync(0xffffffffu, kor, o);
  }
  const uint32_t kdiff = kand ^ kor;
  const int hb = kdiff ? 31 - __clz(kdiff) : -1;  // highest bit where keys differ
  // bits above hb are fixed (all of them when every key is equal)
  uint32_t pmask = hb < 0 ? 0xffffffffu : (hb >= 31 ? 0u : ~((2u << hb) - 1u));
  uint32_t prefix = kand & pmask, remaining = (uint32_t)ki;
#pragma unroll 1
  for (int shift = hb >= 7 ? hb - 7 : 0; hb >= 0;) {
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[8 * lane + q] = 0;
    __syncwarp();
#pragma unroll 4
    for (int j = lane; j < len; j += 32) {
      const uint32_t kt = key[j];
      // plain shared atomics: measured faster here than first aggregating
      // the lanes of equal bins with a warp match
      if ((kt & pmask) == prefix) atomicAdd(&hist[(kt >> shift) & 0xffu], 1u);
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l (descending)
    uint32_t cnt[8], part = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      cnt[q] = hist[255 - 8 * lane - q];
      part += cnt[q];
    }
    uint32_t incl = part;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - part;
    uint32_t sel_bin = 0, sel_rem = 0, sel_cnt = 0;
    const bool mine = excl < remaining && remaining <= incl;
    if (mine) {
      uint32_t before = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (before < remaining && remaining <= before + cnt[q]) {
          sel_bin = (uint32_t)(255 - 8 * lane - q);
          sel_rem = remaining - before;
          sel_cnt = cnt[q];
        }
        before += cnt[q];
      }
    }
    const int owner = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    sel_bin = __shfl_sync(0xffffffffu, sel_bin, owner);
    sel_rem = __shfl_sync(0xffffffffu, sel_rem, owner);
    sel_cnt = __shfl_sync(0xffffffffu, sel_cnt, owner);
    prefix |= sel_bin << shift;
    remaining = sel_rem;
    pmask |= 0xffu << shift;
    __syncwarp();  // the bins are cleared again only after every lane read them
    // (when the digit overlaps bits fixed earlier, those bits of sel_bin equal
    // the prefix's: every counted key shares them)
    if (sel_cnt == sel_rem || shift == 0) break;  // the bin is taken whole, or every bit is fixed
    shift = shift >= 8 ? shift - 8 : 0;
  }
  // keys above the prefix (on the bits fixed so far) are all kept; of the
  // keys equal to it the `remaining` ones with the lowest j; the diagonal
  // joins when forced
  int base = 0;
  uint32_t eq_before = 0;
  for (int t = 0; t < nt; ++t) {
    const int j = 32 * t + lane;
    const uint32_t kt = j < len ? key[j] & pmask : 0u;
    const bool eq = j < len && kt == prefix;
    const unsigned em = __ballot_sync(0xffffffffu, eq);
    const uint32_t rank = eq_before + __popc(em & lt);
    eq_before += __popc(em);
    const bool keep = j < len && (kt > prefix || (eq && rank < remaining) || (force_diag && j == i));
    const unsigned km = __ballot_sync(0xffffffffu, keep);
    if (keep) out[base + __popc(km & lt)] = j + off;
    base += __popc(km);
  }
  if (lane == 0) counts[row] = base;
}

// ---------------------------------------------------------- varlen table --
// Packed variable-length prefill: sequence s occupies tokens
// start[s] .. start[s] + len[s] - 1 of the packed buffer, start[s] a multiple
// of 64, the sequences in ascending order without overlap.  tab[i] = (first
// block of block i's sequence, tokens of block i inside it), or (-1, 0) for a
// block of no sequence.  Thread s also checks sequence s; a bad entry is
// recorded in the status word and its blocks are treated as gaps.
__global__ void varlen_table_kernel(const int32_t* __restrict__ start, const int32_t* __restrict__ len, int nseq,
                                    int n, int2* __restrict__ tab, uint32_t* __restrict__ status) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int nb = n / kBlock;
  if (t < nseq) {
    const int a = start[t], l = len[t];
    const int lim = t + 1 < nseq ? start[t + 1] : n;
    if (a < 0 || (a % kBlock) != 0 || l < 1 || a + l > lim || a + l > n) record_status(status, kDevBadIndex, (uint32_t)t);
  }
  if (t >= nb) return;
  const int p = t * kBlock;  // first token of block t
  // last sequence whose start is <= p (starts ascending)
  int lo = 0, hi = nseq - 1, s = -1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    if (start[mid] <= p) {
      s = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  int2 v = make_int2(-1, 0);
  if (s >= 0) {
    const int a = start[s], l = len[s];
    const int lim = s + 1 < nseq ? start[s + 1] : n;
    const bool ok = a >= 0 && (a % kBlock) == 0 && l >= 1 && a + l <= lim && a + l <= n;
    if (ok && p < a + l) v = make_int2(a / kBlock, min(kBlock, a + l - p));
  }
  tab[t] = v;
}

// --------------------------------------------------------------- launchers --
cudaError_t launch_pool(const void* X, seer_dtype dt, bool is_k, long long BH, int n, int d,
                        float* out, cudaStream_t st, const int2* tab) {
  const long long nblocks = BH * (n / kBlock);
  const int warps = 8;
  const unsigned grid = (unsigned)((nblocks + warps - 1) / warps);
  if (dt == SEER_BF16) {
    if (is_k)
      pool_kernel<uint16_t, true><<<grid, warps * 32, 0, st>>>((const uint16_t*)X, nblocks, n, d, out, tab);
    else
      pool_kernel<uint16_t, false><<<grid, warps * 32, 0, st>>>((const uint16_t*)X, nblocks, n, d, out, tab);
  } else {
    if (is_k)
      pool_kernel<float, true><<<grid, warps * 32, 0, st>>>((const float*)X, nblocks, n, d, out, tab);
    else
      pool_kernel<float, false><<<grid, warps * 32, 0, st>>>((const float*)X, nblocks, n, d, out, tab);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm_nt(const float* A, const float* B, float* C, int M, int N, int K,
                           long long a_bs, long long b_bs, long long c_bs, int ldc, int batch,
                           int zh, int zmul, int zg, float alpha, bool causal, cudaStream_t st) {
  const bool big = K % 16 == 0 && a_bs % 4 == 0 && b_bs % 4 == 0 && (reinterpret_cast<uintptr_t>(A) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(B) & 15) == 0;
  if (big) {
    dim3 grid((M + 127) / 128, (N + 127) / 128, batch);
    if (causal)
      gemm_nt128_kernel<true><<<grid, 256, 0, st>>>(A, B, C, M, N, K, a_bs, b_bs, c_bs, ldc, zh, zmul, zg, alpha);
    else
      gemm_nt128_kernel<false><<<grid, 256, 0, st>>>(A, B, C, M, N, K, a_bs, b_bs, c_bs, ldc, zh, zmul, zg, alpha);
    return cudaGetLastError();
  }
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

namespace {
template <bool FROM_LOGITS, int NT>
cudaError_t row_select_launch(const float* in, float* scores, long long rows, int nb, int mode, float T, int k,
                              float density, int32_t* counts, int32_t* indices, int cap, cudaStream_t st,
                              int row_len, const int2* tab) {
  const size_t smem = (size_t)nb * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(row_select_kernel<FROM_LOGITS, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  row_select_kernel<FROM_LOGITS, NT><<<(unsigned)rows, NT, smem, st>>>(in, FROM_LOGITS ? scores : nullptr, nb, mode,
                                                                       T, k, density, counts, indices, cap, row_len,
                                                                       tab);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_row_select(const float* in, float* scores, bool from_logits, long long rows,
                              int nb, int mode, float T, int k, float density, int32_t* counts,
                              int32_t* indices, int cap, cudaStream_t st, int row_len, const int2* tab) {
  // Few rows (the decode gate, small batches) leave most SMs idle and each
  // row's latency exposed: then 1024 threads share a row's work.
  const bool wide = rows < 2LL * 148;
  // Many rows of at most kSelMaxWidth candidates: one warp per row, the row
  // in shared memory
  const int width = row_len > 0 ? row_len : nb;
  if (!wide && rows >= 8LL * 148 && width <= kSelMaxWidth) {
    const unsigned grid = (unsigned)((rows + kSelWarps - 1) / kSelWarps);
    const size_t smem = sizeof(uint32_t) * (size_t)kSelWarps * (256 + width);
    auto kern = from_logits ? row_select_warp_kernel<true> : row_select_warp_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 32 * kSelWarps, smem, st>>>(in, from_logits ? scores : nullptr, rows, nb, mode, T, k, density,
                                             counts, indices, cap, row_len, tab);
    return cudaGetLastError();
  }
  if (from_logits)
    return wide ? row_select_launch<true, 1024>(in, scores, rows, nb, mode, T, k, density, counts, indices, cap, st,
                                                row_len, tab)
                : row_select_launch<true, kRowThreads>(in, scores, rows, nb, mode, T, k, density, counts, indices,
                                                       cap, st, row_len, tab);
  return wide ? row_select_launch<false, 1024>(in, scores, rows, nb, mode, T, k, density, counts, indices, cap, st,
                                               row_len, tab)
              : row_select_launch<false, kRowThreads>(in, scores, rows, nb, mode, T, k, density, counts, indices, cap,
                                                      st, row_len, tab);
}

}  // namespace seer

namespace seer {
cudaError_t launch_varlen_table(const int32_t* start, const int32_t* len, int nseq, int n, int2* tab,
                                uint32_t* status, cudaStream_t st) {
  const int nb = n / kBlock;
  const int m = nb > nseq ? nb : nseq;
  varlen_table_kernel<<<(m + 255) / 256, 256, 0, st>>>(start, len, nseq, n, tab, status);
  return cudaGetLastError();
}
}  // namespace seer
