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
//                    16-byte vector loads, shuffle reductions; optionally
//                    writes its result split into tf32 part and remainder
//   gate_inputs_kernel
//                    for the tensor-core gate: the Q and K pooling (split)
//                    and the tf32 split of Wq and Wk in one launch
//   gemm_nt_kernel   fp32 SIMT tile GEMM: gate projections and the causal
//                    block logits when h or d is not a multiple of 32;
//                    gemm_nt128_kernel is its 128 x 128-tile form
//   gemm_tf32x3_kernel
//                    the gate projections on the tf32 tensor cores (tcgen05):
//                    three products of tf32 parts (hi*hi + hi*lo + lo*hi)
//                    keep fp32-level accuracy; the epilogue writes q~ / k~
//                    already split for the logits, by TMA stores
//   gemm_tf32x3_rows_kernel
//                    the causal block logits q~ k~^T / sqrt(d) the same way,
//                    persistent: each q~ row block is copied into TMEM once
//                    and the key tiles up to the diagonal stream past it
//   split_tf32_kernel
//                    the tf32 split of q~ / k~ after RoPE, in place
//   rope_kernel      optional block-level RoPE on q~ / k~
//   row_select_warp4_kernel / row_select_warp_kernel / row_select_kernel
//                    one warp (many rows of <= 4096 candidates; 16-byte
//                    vectors when rows are aligned) or one CTA per score row:
//                    causal softmax (Eq. 1), optional score write-out, then
//                    threshold compaction or exact top-k (radix select on
//                    the fp32 bit patterns, ties to lower j)
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
// With lo non-null the result is written split for the tf32x3 products: the
// value rounded to tf32 into out, the exact remainder into lo.
__device__ __forceinline__ float tf32_hi(float v) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(v));
  return __uint_as_float(h);
}

// One warp pools block `warp` (the warp-uniform index over B*H*nb blocks).
template <typename T, bool IS_K>
__device__ __forceinline__ void pool_block(const T* __restrict__ X, long long warp, int n, int d,
                                           float* __restrict__ out, const int2* __restrict__ tab,
                                           float* __restrict__ lo) {
  constexpr int EPL = 16 / sizeof(T);  // elements per lane per load
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
#pragma unroll 8
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
    const int w = IS_K ? 3 * d : d;
    const long long at = ((bh * nb) + i) * (long long)w + cg * EPL;
    // EPL consecutive floats per part, 16-byte aligned: float4 stores
    auto put = [&](int c, const float (&v)[EPL]) {
#pragma unroll
      for (int e = 0; e < EPL; e += 4) {
        float4 x = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        if (lo) {
          const float4 hv = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
          *reinterpret_cast<float4*>(lo + at + c + e) = make_float4(x.x - hv.x, x.y - hv.y, x.z - hv.z, x.w - hv.w);
          x = hv;
        }
        *reinterpret_cast<float4*>(out + at + c + e) = x;
      }
    };
    float v[EPL];
    if (!IS_K) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) v[e] = sum[e] * inv;
      put(0, v);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) v[e] = valid > 0 ? mx[e] : 0.f;
      put(0, v);
#pragma unroll
      for (int e = 0; e < EPL; ++e) v[e] = valid > 0 ? mn[e] : 0.f;
      put(d, v);
#pragma unroll
      for (int e = 0; e < EPL; ++e) v[e] = sum[e] * inv;
      put(2 * d, v);
    }
  }
}

template <typename T, bool IS_K>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ X, long long nblocks,
                                                   int n, int d, float* __restrict__ out,
                                                   const int2* __restrict__ tab, float* __restrict__ lo) {
  const long long warp = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (warp >= nblocks) return;
  pool_block<T, IS_K>(X, warp, n, d, out, tab, lo);
}

// The gate's inputs in one launch, for the tensor-core projections: CTAs
// [0, cq) pool Q (warp per block), [cq, cq + ck) pool K, and the rest split
// Wq and Wk into their tf32 parts and remainders.  All three read HBM only,
// so they share the launch's bandwidth instead of running one after another.
template <typename T>
__global__ void __launch_bounds__(256, 4) gate_inputs_kernel(GateInputs g) {
  const long long cta = blockIdx.x;
  if (cta < g.cq) {
    const long long warp = cta * 8 + threadIdx.x / 32;
    if (warp < g.nq) pool_block<T, false>((const T*)g.Q, warp, g.n, g.d, g.qhi, g.tab, g.qlo);
  } else if (cta < g.cq + g.ck) {
    const long long warp = (cta - g.cq) * 8 + threadIdx.x / 32;
    if (warp < g.nk) pool_block<T, true>((const T*)g.K, warp, g.n, g.d, g.khi, g.tab, g.klo);
  } else {
    const long long t0 = (cta - g.cq - g.ck) * 256 + threadIdx.x;
    const long long stride = (gridDim.x - g.cq - g.ck) * 256ll;
    for (long long i = t0; i < g.nwq + g.nwk; i += stride) {
      const bool isq = i < g.nwq;
      const long long j = isq ? i : i - g.nwq;
      const float v = isq ? g.Wq[j] : g.Wk[j];
      const float hi = tf32_hi(v);
      (isq ? g.wqh : g.wkh)[j] = hi;
      (isq ? g.wql : g.wkl)[j] = v - hi;
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

namespace gt3 {
// With one stage of 64 KB per CTA, three CTAs share an SM, so one tile's
// loads, products and epilogue overlap the others' (for many shallow tiles).
// Few deep tiles (a projection with K = 3d) take three stages instead, so
// that one CTA's slices stream while it multiplies.
constexpr uint32_t kOp = 128u * 128u;                 // one operand slice: 128 rows x 32 floats
constexpr uint32_t kStage = 4u * kOp;                 // Ah, Al, Bh, Bl
constexpr uint32_t smem_bytes(int stages) { return (uint32_t)stages * kStage + 1024u; }  // + alignment slack
}  // namespace gt3

template <int kStages>
__global__ void __launch_bounds__(128, 1) gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmAh,
                                                             const __grid_constant__ CUtensorMap tmAl,
                                                             const __grid_constant__ CUtensorMap tmBh,
                                                             const __grid_constant__ CUtensorMap tmBl,
                                                             const __grid_constant__ CUtensorMap tmC,
                                                             const __grid_constant__ CUtensorMap tmClo,
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
  if (p.tma_out) {
    // Every product is done, so the ring is free: 32-column chunks go through
    // 128-byte-swizzled staging tiles there (two per output, alternating)
    // and leave by TMA stores, clipped at the matrix's edges.
    const bool all_ok = __syncthreads_and(ok) != 0;
#pragma unroll 1
    for (int c = 0; c < 4 && all_ok; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(32 * c), v);
      tmem_wait_ld();
      uint8_t* const sh = ring + (c & 1) * 16384;
      uint8_t* const sl = ring + 32768 + (c & 1) * 16384;
      if (threadIdx.x == 0 && c >= 2) bulk_wait_group_read<1>();  // the slot's previous store has read it
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float4 x = make_float4(p.alpha * __uint_as_float(v[4 * k]), p.alpha * __uint_as_float(v[4 * k + 1]),
                               p.alpha * __uint_as_float(v[4 * k + 2]), p.alpha * __uint_as_float(v[4 * k + 3]));
        const uint32_t at = (uint32_t)(r * 128 + ((k ^ (r & 7)) << 4));
        if (p.C_lo) {
          const float4 hv = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
          *reinterpret_cast<float4*>(sl + at) = make_float4(x.x - hv.x, x.y - hv.y, x.z - hv.z, x.w - hv.w);
          x = hv;
        }
        *reinterpret_cast<float4*>(sh + at) = x;
      }
      fence_async_shared();
      __syncthreads();
      if (threadIdx.x == 0) {
        tma_store_3d(&tmC, sh, tn * 128 + 32 * c, tm * 128, z);
        if (p.C_lo) tma_store_3d(&tmClo, sl, tn * 128 + 32 * c, tm * 128, z);
        bulk_commit_group();
      }
    }
    if (threadIdx.x == 0) bulk_wait_group<0>();
  }
#pragma unroll 1
  for (int c0 = 0; c0 < 128 && !p.tma_out; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    const int gn = tn * 128 + c0;
    if (ok && gm < p.M && gn < p.N) {
      if (p.C_lo && vec && gn + 32 <= p.N) {
        // split output: tf32 part into C, exact remainder into C_lo
        float* const lrow = p.C_lo + (long long)z * p.c_bs + (long long)gm * p.ldc;
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          const float4 x = make_float4(p.alpha * __uint_as_float(v[q]), p.alpha * __uint_as_float(v[q + 1]),
                                       p.alpha * __uint_as_float(v[q + 2]), p.alpha * __uint_as_float(v[q + 3]));
          const float4 hv = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
          *reinterpret_cast<float4*>(crow + gn + q) = hv;
          *reinterpret_cast<float4*>(lrow + gn + q) = make_float4(x.x - hv.x, x.y - hv.y, x.z - hv.z, x.w - hv.w);
        }
      } else if (p.C_lo) {
        float* const lrow = p.C_lo + (long long)z * p.c_bs + (long long)gm * p.ldc;
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (gn + q < p.N) {
            const float x = p.alpha * __uint_as_float(v[q]);
            const float hv = tf32_hi(x);
            crow[gn + q] = hv;
            lrow[gn + q] = x - hv;
          }
      } else if (vec && gn + 32 <= p.N) {
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
                                      const CUtensorMap& tmBl, const CUtensorMap& tmC, const CUtensorMap& tmClo,
                                      const Tf32x3Params& p, int batch, cudaStream_t st) {
  dim3 grid((p.M + 127) / 128, (p.N + 127) / 128, batch);
  // deep tiles (more than four slices) stream through three stages
  const bool deep = p.K > 128;
  auto kern = deep ? gemm_tf32x3_kernel<3> : gemm_tf32x3_kernel<1>;
  const uint32_t smem = gt3::smem_bytes(deep ? 3 : 1);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 128, smem, st>>>(tmAh, tmAl, tmBh, tmBl, tmC, tmClo, p);
  return cudaGetLastError();
}

// ---------------------------------------- tf32x3 causal logits, by rows --
// The causal logits with the query side held on chip: a CTA takes one
// 128-row block of q~ at a time, copies its tf32 parts and remainders into
// tensor memory (tcgen05.cp; A of TS-form MMAs), and sweeps the key tiles
// tn = 0..tm up to the diagonal, so each q~ row block crosses L2 once and
// the MMAs read only the key slices from shared memory.  Warp 0 loads by
// TMA (no cluster multicast), warp 1 issues the copies and MMAs into one of
// two TMEM accumulators while warps 2..5 drain the other: each 32-column
// chunk goes through a 128-byte-swizzled staging tile in shared memory and
// leaves by a TMA store (clipped at the matrix's edges).  Work items
// (z, tm), tm + 1 tiles each, are dealt out statically: largest first, in
// snake order across the CTAs so that each CTA's total is close to the mean.
namespace gtr {
constexpr int kBStages = 4;
constexpr uint32_t kSlice = 128u * 128u;            // 128 rows x 32 floats
constexpr int kMaxSlices = 4;                       // h <= 128
constexpr uint32_t kAStage = kMaxSlices * kSlice;   // one part of the q~ block: 64 KB
constexpr uint32_t kBStage = 2u * kSlice;           // one 32-column slice of a k~ tile, both parts: 32 KB
constexpr uint32_t kOut = kSlice;                   // one 128 x 32 output chunk: 16 KB
constexpr uint32_t kSmem = kAStage + kBStages * kBStage + 2u * kOut + 1024u;
constexpr int kThreads = 224;                        // warps: 0 key loads, 1 MMA, 2..5 epilogue, 6 q~ loads
constexpr uint32_t kColAh = 256, kColAl = 384;      // TMEM: accumulators at 0 and 128
}  // namespace gtr

// Item w of this CTA's r-th round (snake order), or -1 past the end.
__device__ __forceinline__ int gtr_item(int r, int items) {
  const int G = (int)gridDim.x, b = (int)blockIdx.x;
  const int w = r * G + ((r & 1) ? G - 1 - b : b);
  return w < items ? w : -1;
}

__global__ void __launch_bounds__(gtr::kThreads, 1)
    gemm_tf32x3_rows_kernel(const __grid_constant__ CUtensorMap tmAh, const __grid_constant__ CUtensorMap tmAl,
                            const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmBl,
                            const __grid_constant__ CUtensorMap tmC, const Tf32x3Params p, int batch) {
  using namespace gtr;
  extern __shared__ uint8_t gtr_raw[];
  uint8_t* const sA = gtr_raw + ((1024u - (smem_u32(gtr_raw) & 1023u)) & 1023u);
  uint8_t* const sB = sA + kAStage;
  uint8_t* const sO = sB + kBStages * kBStage;
  __shared__ uint64_t a_full, a_free, atm_free, b_full[kBStages], b_empty[kBStages], acc_full[2], acc_empty[2], done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  // teardown accounting: q~ parts and key slices whose copies went out / were consumed
  __shared__ int a_issued, a_used, b_issued, b_used;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_p = &abort_flag;
  const uint64_t tmo = p.timeout_ns;
  const int nk = p.K / 32;  // 32-column slices, at most kMaxSlices
  const int T = (p.M + 127) / 128;
  const int items = T * batch;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    a_issued = a_used = b_issued = b_used = 0;
    mbar_init(&a_full, 1);
    mbar_init(&a_free, 1);
    mbar_init(&atm_free, 1);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);
    }
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 6) {
    // ------------------------------------------------------- q~ loads ----
    if (lane == 0) {
      prefetch_tmap(&tmAh);
      prefetch_tmap(&tmAl);
      const uint32_t a_bytes = (uint32_t)nk * kSlice;
      int su = 0;  // staging uses of the q~ buffer
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = gtr_item(r, items);
        if (w < 0) break;
        const int tm = T - 1 - w / batch, z = w % batch;
        const int arow = z * p.M + tm * 128;
        // the two parts, one at a time through the staging buffer (free once
        // the previous part was copied into TMEM)
        for (int part = 0; part < 2 && ok; ++part) {
          if (su > 0 && !mbar_wait(&a_free, (su - 1) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&a_full, a_bytes);
          tma_load_3d(sA, part ? &tmAl : &tmAh, &a_full, 0, arow, 0);
          a_issued = ++su;
        }
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------- key loads ---
    if (lane == 0) {
      prefetch_tmap(&tmBh);
      prefetch_tmap(&tmBl);
      int cs = 0;  // key slices
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = gtr_item(r, items);
        if (w < 0) break;
        const int tm = T - 1 - w / batch, z = w % batch;
        const int bz = (z / p.zh) * p.zmul + (z % p.zh) / p.zg;
        for (int tn = 0; tn <= tm && ok; ++tn) {
          const int brow = bz * p.N + tn * 128;
          for (int c = 0; c < nk; ++c) {
            const int s = cs % kBStages;
            if (cs >= kBStages && !mbar_wait(&b_empty[s], ((cs / kBStages) - 1) & 1, abort_p, p.status, tmo)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&b_full[s], kBStage);
            tma_load_2d(sB + s * kBStage, &tmBh, &b_full[s], c * 32, brow);
            tma_load_2d(sB + s * kBStage + kSlice, &tmBl, &b_full[s], c * 32, brow);
            b_issued = ++cs;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- copies and MMAs ---
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_tf32(128, 128, 0, 0);  // A (TMEM) and B K-major
      const uint64_t dA0 = make_sw128_desc(smem_u32(sA), 16, 1024);
      const uint64_t dB0 = make_sw128_desc(smem_u32(sB), 16, 1024);
      int it = 0, su = 0, cs = 0, tile = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int w = gtr_item(r, items);
        if (w < 0) break;
        const int tm = T - 1 - w / batch;
        // the previous item's products must be done before its q~ is overwritten
        if (it > 0 && !mbar_wait(&atm_free, (it - 1) & 1, abort_p, p.status, tmo)) break;
        // one part of the q~ block from the staging buffer into TMEM
        auto copy_part = [&](int part) -> bool {
          if (!mbar_wait(&a_full, su & 1, abort_p, p.status, tmo)) return false;
          tc_fence_after();
          const uint32_t ta = tmem + (part ? kColAl : kColAh);
          for (int c = 0; c < nk; ++c)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tmem_cp_128x256b(ta + (uint32_t)(c * 32 + kk * 8),
                               dA0 + (uint64_t)((c * kSlice + kk * 32) >> 4));
          mma_commit(&a_free);  // the staging buffer is free once these copies are done
          a_used = ++su;
          return true;
        };
        if (!copy_part(0)) break;
        // The item's first tile takes its tf32-part products while the
        // remainder part is still loading (its nk <= kBStages slices all stay
        // resident), then the remainder's products.
        {
          const int buf = tile & 1;
          if (tile >= 2 && !mbar_wait(&acc_empty[buf], ((tile >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
          tc_fence_after();
          const uint32_t acc = tmem + (uint32_t)buf * 128u;
          for (int c = 0; c < nk && ok; ++c) {
            const int s = (cs + c) % kBStages;
            if (!mbar_wait(&b_full[s], ((cs + c) / kBStages) & 1, abort_p, p.status, tmo)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t dBh = dB0 + (uint64_t)((s * kBStage) >> 4);
            const uint64_t dBl = dBh + (uint64_t)(kSlice >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t off = (uint64_t)((kk * 32) >> 4);
              const uint32_t col = (uint32_t)(c * 32 + kk * 8);
              mma_tf32_ts(acc, tmem + kColAh + col, dBh + off, idesc, (c > 0 || kk > 0) ? 1u : 0u);
              mma_tf32_ts(acc, tmem + kColAh + col, dBl + off, idesc, 1u);
            }
          }
          if (!ok || !copy_part(1)) break;
          for (int c = 0; c < nk; ++c) {
            const int s = cs % kBStages;
            const uint64_t dBh = dB0 + (uint64_t)((s * kBStage) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_tf32_ts(acc, tmem + kColAl + (uint32_t)(c * 32 + kk * 8), dBh + (uint64_t)((kk * 32) >> 4), idesc,
                          1u);
            mma_commit(&b_empty[s]);
            b_used = ++cs;
          }
          mma_commit(&acc_full[buf]);
          ++tile;
        }
        for (int tn = 1; tn <= tm && ok; ++tn, ++tile) {
          const int buf = tile & 1;
          if (tile >= 2 && !mbar_wait(&acc_empty[buf], ((tile >> 1) - 1) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem + (uint32_t)buf * 128u;
          for (int c = 0; c < nk; ++c) {
            const int s = cs % kBStages;
            if (!mbar_wait(&b_full[s], (cs / kBStages) & 1, abort_p, p.status, tmo)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t dBh = dB0 + (uint64_t)((s * kBStage) >> 4);
            const uint64_t dBl = dBh + (uint64_t)(kSlice >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t off = (uint64_t)((kk * 32) >> 4);  // 8 floats = 32 bytes per k step
              const uint32_t col = (uint32_t)(c * 32 + kk * 8);
              mma_tf32_ts(acc, tmem + kColAh + col, dBh + off, idesc, (c > 0 || kk > 0) ? 1u : 0u);
              mma_tf32_ts(acc, tmem + kColAh + col, dBl + off, idesc, 1u);
              mma_tf32_ts(acc, tmem + kColAl + col, dBh + off, idesc, 1u);
            }
            mma_commit(&b_empty[s]);
            b_used = ++cs;
          }
          if (!ok) break;
          mma_commit(&acc_full[buf]);
        }
        if (!ok) break;
        mma_commit(&atm_free);
        ++it;
      }
      // arrives once every copy and MMA this thread issued is done (even after a failed wait)
      mma_commit(&done);
    }
  } else if (warp >= 2 && warp <= 5) {
    // --------------------------------------------------------- epilogue --
    const int q = warp & 3;        // TMEM sub-partition: rows 32q .. 32q+31
    const int rr = q * 32 + lane;  // tile row
    const bool storer = warp == 2 && lane == 0;
    int tile = 0, chunk = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int w = gtr_item(r, items);
      if (w < 0) break;
      const int tm = T - 1 - w / batch, z = w % batch;
      for (int tn = 0; tn <= tm; ++tn, ++tile) {
        const int buf = tile & 1;
        ok = mbar_wait(&acc_full[buf], (tile >> 1) & 1, abort_p, p.status, tmo);
        // every epilogue thread leaves together: the named barriers below have no timeout
        if (bar_red_or(1, 128, !ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the whole 128-column row in registers with one wait, then the
        // accumulator is free for the MMA warp
        uint32_t v[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 128 + 32 * c), v[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
#pragma unroll
        for (int c = 0; c < 4; ++c, ++chunk) {
          uint8_t* const so = sO + (chunk & 1) * kOut;
          // the staging tile's previous store has finished reading it
          if (storer) bulk_wait_group_read<1>();
          named_barrier_sync(2, 128);
          // row rr, 16-byte piece k at (k ^ (rr & 7)) (128-byte swizzle)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(so + rr * 128 + ((k ^ (rr & 7)) << 4)) =
                make_float4(p.alpha * __uint_as_float(v[c][4 * k]), p.alpha * __uint_as_float(v[c][4 * k + 1]),
                            p.alpha * __uint_as_float(v[c][4 * k + 2]), p.alpha * __uint_as_float(v[c][4 * k + 3]));
          fence_async_shared();
          named_barrier_sync(2, 128);
          if (storer) {
            tma_store_3d(&tmC, so, tn * 128 + 32 * c, tm * 128, z);
            bulk_commit_group();
          }
        }
      }
    }
    if (storer) bulk_wait_group<0>();  // every store complete before the CTA exits
  }

  // every copy and MMA done before TMEM is released (bounded; the MMA warp always commits)
  __syncwarp();
  {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(&done, 0, 20000u))
      if (globaltimer_ns() - t0 > 20000000ull) break;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
  // After an abort, copies that were issued but never consumed may still be
  // in flight: each completes its stage's full phase (armed by the loader
  // alone), so wait (bounded) for those phases before shared memory is
  // released.  A loader arms slice c only after slice c - kBStages was
  // consumed, so only the last kBStages can be open; likewise the staging
  // buffer holds at most one part.
  if (threadIdx.x == 0 && *abort_p) {
    for (int c = b_used > b_issued - kBStages ? b_used : b_issued - kBStages; c < b_issued; ++c) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_sleep(&b_full[c % kBStages], (c / kBStages) & 1, 20000u))
        if (globaltimer_ns() - t0 > 20000000ull) break;
    }
    if (a_used < a_issued) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_sleep(&a_full, (a_issued - 1) & 1, 20000u))
        if (globaltimer_ns() - t0 > 20000000ull) break;
    }
  }
}

bool gemm_tf32x3_rows_fits(int K, int N, long long c_bs, const void* C) {
  return K % 32 == 0 && K / 32 <= gtr::kMaxSlices && N % 4 == 0 && c_bs % 4 == 0 &&
         (reinterpret_cast<uintptr_t>(C) & 15) == 0;
}

cudaError_t launch_gemm_tf32x3_rows(const CUtensorMap& tmAh, const CUtensorMap& tmAl, const CUtensorMap& tmBh,
                                    const CUtensorMap& tmBl, const CUtensorMap& tmC, const Tf32x3Params& p,
                                    int batch, int num_sms, cudaStream_t st) {
  if (!gemm_tf32x3_rows_fits(p.K, p.N, p.c_bs, p.C)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_tf32x3_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gtr::kSmem);
  if (e != cudaSuccess) return e;
  const long long items = (long long)((p.M + 127) / 128) * batch;
  const int grid = (int)(items < num_sms ? items : num_sms);
  gemm_tf32x3_rows_kernel<<<grid < 1 ? 1 : grid, gtr::kThreads, gtr::kSmem, st>>>(tmAh, tmAl, tmBh, tmBl, tmC, p,
                                                                                  batch);
  return cudaGetLastError();
}

cudaError_t launch_split_tf32(float* x, float* lo, long long n, cudaStream_t st) {
  split_tf32_kernel<<<1184, 256, 0, st>>>(x, lo, n);
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
// is exp2-based (one FMA and one MUFU exponential per candidate) and
// multiplies by the reciprocal of the row sum; the key order, ties to the
// lower j, the forced diagonal and varlen windows follow row_select_kernel.
//
// Three passes over the row before the radix select: (A) load, maximum and
// minimum; (B) exponentials and their sum; (C) probabilities, their
// order-preserving keys and the first radix histogram.  The first digit's
// position is predicted from the keys of the two extreme candidates (the
// keys of a row share every bit above the highest bit where its largest and
// smallest keys differ); the true AND / OR of all keys, formed in the same
// pass, confirms the prediction, and otherwise the first histogram is built
// again in a pass of its own.
constexpr int kSelWarps = 8;
constexpr int kSelMaxWidth = 4096;

// Shared-memory counter increment with the condition as a predicate (no
// branch around the atomic).
__device__ __forceinline__ void red_shared_add1_if(uint32_t* addr, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "@p red.shared.add.u32 [%0], 1;\n\t}" ::"r"(smem_u32(addr)),
      "r"((uint32_t)pred)
      : "memory");
}

// Global int32 store with the condition as a predicate.
__device__ __forceinline__ void st_global_if(int32_t* addr, int32_t v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "@p st.global.b32 [%0], %1;\n\t}" ::"l"(addr),
      "r"(v), "r"((uint32_t)pred)
      : "memory");
}

__device__ __forceinline__ float ex2_approx_full(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));  // keeps subnormal results
  return y;
}

// Bits above the highest bit where the keys differ (kd = AND ^ OR of the
// keys, or of the two extreme keys): the mask of fixed bits and the shift of
// the first 8-bit digit below them.
__device__ __forceinline__ void fixed_bits(uint32_t kd, int& hb, uint32_t& pmask, int& shift) {
  hb = kd ? 31 - __clz(kd) : -1;
  pmask = hb < 0 ? 0xffffffffu : (hb >= 31 ? 0u : ~((2u << hb) - 1u));
  shift = hb >= 7 ? hb - 7 : 0;
}

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
  int32_t* out = indices + row * (long long)cap;
  const bool threshold = mode == SEER_SELECT_THRESHOLD;
  const int ki = threshold ? 0 : topk_count(i, mode, k, density);
  if (!threshold && ki >= len && !dst) {
    for (int j = lane; j < len; j += 32) out[j] = j + off;
    if (lane == 0) counts[row] = len;
    return;
  }

  // (A) the row into shared memory, its maximum and minimum
  float m = -INFINITY, mn = INFINITY;
#pragma unroll 4
  for (int j = lane; j < len; j += 32) {
    const float x = src[j];
    buf[j] = x;
    m = fmaxf(m, x);
    mn = fminf(mn, x);
  }
  m = warp_max(m);
  mn = -warp_max(-mn);
  constexpr float kLog2e = 1.4426950408889634f;
  const float mc = m * kLog2e;
  float inv = 1.f;
  if (FROM_LOGITS) {
    // (B) exponentials 2^(x log2(e) - m log2(e)) and their sum, summed in
    // the same candidate order as the per-row kernel (j = lane, lane + 32,
    // ...), then one butterfly
    float sum = 0.f;
#pragma unroll 4
    for (int j = lane; j < len; j += 32) {
      const float e = ex2_approx_full(fmaf(buf[j], kLog2e, -mc));
      buf[j] = e;
      sum += e;
    }
    inv = 1.0f / warp_sum(sum);
  }
  const bool radix = !threshold && ki < len;
  // predicted fixed bits and first digit, from the extreme candidates' keys
  // (formed exactly as every candidate's below)
  const float vhi = FROM_LOGITS ? ex2_approx_full(fmaf(m, kLog2e, -mc)) * inv : m;
  const float vlo = FROM_LOGITS ? ex2_approx_full(fmaf(mn, kLog2e, -mc)) * inv : mn;
  int hb_p, shift_p;
  uint32_t pmask_p;
  fixed_bits(f2key(vhi) ^ f2key(vlo), hb_p, pmask_p, shift_p);
  const bool first_hist = radix && hb_p >= 0;
  if (first_hist) {
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[8 * lane + q] = 0;
    __syncwarp();
  }
  // (C) probabilities (written out when asked for), keys, their AND / OR and
  // the first histogram on the predicted digit
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll 4
  for (int j = lane; j < len; j += 32) {
    const float v = FROM_LOGITS ? buf[j] * inv : buf[j];
    if (dst) dst[off + j] = v;
    if (threshold) {
      buf[j] = v;
    } else {
      const uint32_t kk = f2key(v);
      key[j] = kk;
      kand &= kk;
      kor |= kk;
      red_shared_add1_if(&hist[(kk >> shift_p) & 0xffu], first_hist);
    }
  }
  if (dst)
    for (int j = lane; j < nb; j += 32)
      if (j < off || j >= off + len) dst[j] = 0.f;

  if (threshold) {
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
  if (!radix) {
    for (int j = lane; j < len; j += 32) out[j] = j + off;
    if (lane == 0) counts[row] = len;
    return;
  }

  // Radix select of the ki-th largest key, 8 bits at a time.  Bits that all
  // of the row's keys share are fixed at once (a warp AND / OR of the keys):
  // a softmax row's values lie close together, so its keys agree on the
  // sign, the exponent and the top of the mantissa, and the first digit
  // starts at the highest bit where they differ.  The search also stops as
  // soon as the bin holding the ki-th key is taken whole.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    kor |= __shfl_xor_sync(0xffffffffu, kor, o);
  }
  int hb, shift;
  uint32_t pmask;
  fixed_bits(kand ^ kor, hb, pmask, shift);
  uint32_t prefix = kand & pmask, remaining = (uint32_t)ki;
  // the histogram of pass C is the first pass's when the prediction held
  bool have = first_hist && hb == hb_p && prefix == (f2key(vhi) & pmask_p);
  __syncwarp();
#pragma unroll 1
  for (; hb >= 0;) {
    if (!have) {
#pragma unroll
      for (int q = 0; q < 8; ++q) hist[8 * lane + q] = 0;
      __syncwarp();
#pragma unroll 4
      for (int j = lane; j < len; j += 32) {
        const uint32_t kt = key[j];
        red_shared_add1_if(&hist[(kt >> shift) & 0xffu], (kt & pmask) == prefix);
      }
      __syncwarp();
    }
    have = false;
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
    st_global_if(out + base + __popc(km & lt), j + off, keep);
    base += __popc(km);
  }
  if (lane == 0) counts[row] = base;
}

// The same selection with 16-byte vectors: lane l owns candidates
// 128 t + 4 l .. 128 t + 4 l + 3, so every pass over the row moves four
// candidates per shared-memory access and per loop step.  For rows that
// start 16-byte aligned (nb a multiple of 4, no varlen table).  The passes
// are those of row_select_warp_kernel; the final compaction ranks a lane's
// four candidates with a warp prefix sum, and skips the tie ranking when the
// radix search ended on a bin taken whole (the usual case).
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, int lane, uint32_t& total) {
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  total = __shfl_sync(0xffffffffu, incl, 31);
  return incl - v;
}

template <bool FROM_LOGITS>
__global__ void __launch_bounds__(32 * kSelWarps) row_select_warp4_kernel(
    const float* in, float* scores, long long rows, int nb, int mode_flags, float T, int k, float density,
    int32_t* __restrict__ counts, int32_t* __restrict__ indices, int cap, long long v0, long long v1, int width) {
  extern __shared__ uint32_t sel_smem[];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Rows are taken query block by query block across all heads (the
  // warps of a CTA get rows of equal length; the first rows taken are the
  // shortest, whose logits the logits kernel wrote last and L2 still holds).
  // This launch takes rows v0 .. v1 - 1 of that order, none longer than
  // width (a multiple of 4: each warp's row buffer).
  const long long vrow = v0 + (long long)blockIdx.x * kSelWarps + wid;
  if (vrow >= v1) return;  // whole warps only: no CTA barrier follows
  // 32-bit division when the row count allows it (always, in practice)
  const long long heads = rows / nb;
  long long hq, ib;
  if (rows <= 0x7fffffffLL) {
    const uint32_t vr = (uint32_t)vrow, hd = (uint32_t)heads;
    ib = vr / hd;
    hq = vr - (uint32_t)ib * hd;
  } else {
    ib = vrow / heads;
    hq = vrow - ib * heads;
  }
  const long long row = hq * nb + ib;
  uint32_t* const hist = sel_smem + wid * 256;
  float4* const buf = reinterpret_cast<float4*>(sel_smem + kSelWarps * 256) + (size_t)wid * (width / 4);
  uint4* const key = reinterpret_cast<uint4*>(buf);

  const int mode = mode_flags & 0xff;
  const bool force_diag = (mode_flags & SEER_SELECT_FORCE_DIAGONAL) != 0;
  const int i = (int)ib;  // the row's query block
  const int len = i + 1;
  const int nc = (len + 127) >> 7;  // 128-candidate chunks
  const float4* src = reinterpret_cast<const float4*>(in + row * (long long)nb);
  float* const dst = (FROM_LOGITS && scores != nullptr) ? scores + row * (long long)nb : nullptr;
  int32_t* out = indices + row * (long long)cap;
  const bool threshold = mode == SEER_SELECT_THRESHOLD;
  const int ki = threshold ? 0 : topk_count(i, mode, k, density);
  if (!threshold && ki >= len && !dst) {
    for (int j = lane; j < len; j += 32) out[j] = j;
    if (lane == 0) counts[row] = len;
    return;
  }
  // Lane l owns the vectors v = 32 t + l, i.e. candidates 4v .. 4v + 3.  The
  // nfull vectors below len are whole; at most one more (vector nfull, of
  // lane nfull % 32) holds the row's last rem < 4 candidates.  Every pass
  // runs its whole vectors unmasked and the partial one separately.
  const int nfull = len >> 2, rem = len & 3;
  const bool tail = rem != 0 && lane == (nfull & 31);
  // order-preserving key; probabilities are never negative
  auto key_of = [](float x) { return FROM_LOGITS ? (__float_as_uint(x) | 0x80000000u) : f2key(x); };

  // (A) the row into shared memory, its maximum and minimum; from logits
  // also each lane's running softmax sum (relative to its running maximum,
  // rescaled when that grows).  Four vectors per lane in flight at a time.
  constexpr float kLog2e = 1.4426950408889634f;
  float m = -INFINITY, mn = INFINITY, sl = 0.f, mcl = -INFINITY;  // mcl = m log2(e)
  auto fold = [&](float4 x, int nv) {
    if (nv < 4) {  // the row's partial vector: repeat its first candidate for the extremes
      if (nv < 2) x.y = x.x;
      if (nv < 3) x.z = x.x;
      x.w = x.x;
    }
    const float vm = fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w));
    mn = fminf(mn, fminf(fminf(x.x, x.y), fminf(x.z, x.w)));
    if (FROM_LOGITS) {
      if (vm > m) {
        sl *= ex2_approx((m - vm) * kLog2e);
        m = vm;
        mcl = m * kLog2e;
      }
      float e = ex2_approx(fmaf(x.x, kLog2e, -mcl));
      if (nv > 1) e += ex2_approx(fmaf(x.y, kLog2e, -mcl));
      if (nv > 2) e += ex2_approx(fmaf(x.z, kLog2e, -mcl));
      if (nv > 3) e += ex2_approx(fmaf(x.w, kLog2e, -mcl));
      sl += e;
    } else {
      m = fmaxf(m, vm);
    }
  };
  for (int v0 = lane; v0 < nfull; v0 += 128) {
    float4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (v0 + 32 * u < nfull) x[u] = src[v0 + 32 * u];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (v0 + 32 * u < nfull) {
        buf[v0 + 32 * u] = x[u];
        fold(x[u], 4);
      }
  }
  if (tail) {  // the row has nb >= 4 nfull + 4 entries: the whole vector is readable
    const float4 x = src[nfull];
    buf[nfull] = x;
    fold(x, rem);
  }
  const float m_lane = m;
  m = warp_max(m);
  mn = -warp_max(-mn);
  const float mc = m * kLog2e;
  float inv = 1.f;
  if (FROM_LOGITS) {
    // lanes' sums onto the row maximum (a lane with no candidate adds 0)
    inv = 1.0f / warp_sum(sl * ex2_approx((m_lane - m) * kLog2e));
  }
  const bool radix = !threshold && ki < len;
  const float vhi = FROM_LOGITS ? ex2_approx(fmaf(m, kLog2e, -mc)) * inv : m;
  const float vlo = FROM_LOGITS ? ex2_approx(fmaf(mn, kLog2e, -mc)) * inv : mn;
  int hb_p, shift_p;
  uint32_t pmask_p;
  fixed_bits(key_of(vhi) ^ key_of(vlo), hb_p, pmask_p, shift_p);
  const bool first_hist = radix && hb_p >= 0;
  if (first_hist) {
#pragma unroll
    for (int q = 0; q < 8; ++q) hist[8 * lane + q] = 0;
    __syncwarp();
  }
  // (C) probabilities, keys, AND / OR, the first histogram on the predicted digit
  uint32_t kand = 0xffffffffu, kor = 0u;
  auto probv = [&](int v, int nv) {
    const float4 x = buf[v];
    float4 pv;
    pv.x = FROM_LOGITS ? ex2_approx(fmaf(x.x, kLog2e, -mc)) * inv : x.x;
    pv.y = FROM_LOGITS ? ex2_approx(fmaf(x.y, kLog2e, -mc)) * inv : x.y;
    pv.z = FROM_LOGITS ? ex2_approx(fmaf(x.z, kLog2e, -mc)) * inv : x.z;
    pv.w = FROM_LOGITS ? ex2_approx(fmaf(x.w, kLog2e, -mc)) * inv : x.w;
    if (dst) {
      if (nv == 4) {
        *reinterpret_cast<float4*>(dst + 4 * v) = pv;
      } else {
        dst[4 * v] = pv.x;
        if (nv > 1) dst[4 * v + 1] = pv.y;
        if (nv > 2) dst[4 * v + 2] = pv.z;
      }
    }
    if (threshold) {
      buf[v] = pv;
      return;
    }
    const uint4 kk = make_uint4(key_of(pv.x), key_of(pv.y), key_of(pv.z), key_of(pv.w));
    key[v] = kk;
    kand &= kk.x;
    kor |= kk.x;
    if (nv > 1) kand &= kk.y, kor |= kk.y;
    if (nv > 2) kand &= kk.z, kor |= kk.z;
    if (nv > 3) kand &= kk.w, kor |= kk.w;
    if (first_hist) {
      atomicAdd(&hist[(kk.x >> shift_p) & 0xffu], 1u);
      if (nv > 1) atomicAdd(&hist[(kk.y >> shift_p) & 0xffu], 1u);
      if (nv > 2) atomicAdd(&hist[(kk.z >> shift_p) & 0xffu], 1u);
      if (nv > 3) atomicAdd(&hist[(kk.w >> shift_p) & 0xffu], 1u);
    }
  };
#pragma unroll 2
  for (int v = lane; v < nfull; v += 32) probv(v, 4);
  if (tail) probv(nfull, rem);
  if (dst)
    for (int j = len + lane; j < nb; j += 32) dst[j] = 0.f;
  // candidates of this lane's vector in chunk t (0 past the row)
  auto nvalid = [&](int v) { return v < nfull ? 4 : (v == nfull ? rem : 0); };

  if (threshold) {
    int base = 0;
    for (int t = 0; t < nc; ++t) {
      const int v = 32 * t + lane;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      const int nv = nvalid(v);
      if (nv > 0) x = buf[v];
      const int j0 = 4 * v;
      const bool k0 = nv > 0 && (x.x > T || (force_diag && j0 == i));
      const bool k1 = nv > 1 && (x.y > T || (force_diag && j0 + 1 == i));
      const bool k2 = nv > 2 && (x.z > T || (force_diag && j0 + 2 == i));
      const bool k3 = nv > 3 && (x.w > T || (force_diag && j0 + 3 == i));
      uint32_t tot;
      const uint32_t pos = base + warp_excl_scan((uint32_t)k0 + k1 + k2 + k3, lane, tot);
      uint32_t q = pos;
      st_global_if(out + q, j0, k0);
      q += k0;
      st_global_if(out + q, j0 + 1, k1);
      q += k1;
      st_global_if(out + q, j0 + 2, k2);
      q += k2;
      st_global_if(out + q, j0 + 3, k3);
      base += (int)tot;
    }
    if (lane == 0) counts[row] = base;
    return;
  }
  if (!radix) {
    for (int j = lane; j < len; j += 32) out[j] = j;
    if (lane == 0) counts[row] = len;
    return;
  }

  // radix select of the ki-th largest key (as in row_select_warp_kernel)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    kor |= __shfl_xor_sync(0xffffffffu, kor, o);
  }
  int hb, shift;
  uint32_t pmask;
  fixed_bits(kand ^ kor, hb, pmask, shift);
  uint32_t prefix = kand & pmask, remaining = (uint32_t)ki;
  bool whole = hb < 0;  // the keys equal to the final prefix are all kept
  if (hb < 0) whole = remaining >= (uint32_t)len;
  bool have = first_hist && hb == hb_p && prefix == (key_of(vhi) & pmask_p);
  __syncwarp();
#pragma unroll 1
  for (; hb >= 0;) {
    if (!have) {
#pragma unroll
      for (int q = 0; q < 8; ++q) hist[8 * lane + q] = 0;
      __syncwarp();
      auto countv = [&](int v, int nv) {
        const uint4 kk = key[v];
        red_shared_add1_if(&hist[(kk.x >> shift) & 0xffu], (kk.x & pmask) == prefix);
        red_shared_add1_if(&hist[(kk.y >> shift) & 0xffu], nv > 1 && (kk.y & pmask) == prefix);
        red_shared_add1_if(&hist[(kk.z >> shift) & 0xffu], nv > 2 && (kk.z & pmask) == prefix);
        red_shared_add1_if(&hist[(kk.w >> shift) & 0xffu], nv > 3 && (kk.w & pmask) == prefix);
      };
#pragma unroll 2
      for (int v = lane; v < nfull; v += 32) countv(v, 4);
      if (tail) countv(nfull, rem);
      __syncwarp();
    }
    have = false;
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
    __syncwarp();
    if (sel_cnt == sel_rem) {
      whole = true;
      break;
    }
    if (shift == 0) break;
    shift = shift >= 8 ? shift - 8 : 0;
  }
  // keys above the prefix are kept; of those equal to it, the `remaining`
  // with the lowest j (all of them when the bin was taken whole); the
  // diagonal joins when forced
  int base = 0;
  uint32_t eq_before = 0;
  // chunks whose 32 vectors are all whole: with the bin taken whole (and no
  // forced diagonal) a key is kept iff it is at least the prefix, whose bits
  // below the fixed ones are zero
  const int nfc = whole && !force_diag ? nfull >> 5 : 0;
  for (int t = 0; t < nfc; ++t) {
    const int v = 32 * t + lane;
    const uint4 kk = key[v];
    const bool k0 = kk.x >= prefix, k1 = kk.y >= prefix, k2 = kk.z >= prefix, k3 = kk.w >= prefix;
    uint32_t tot;
    uint32_t q = base + warp_excl_scan((uint32_t)k0 + k1 + k2 + k3, lane, tot);
    const int j0 = 4 * v;
    st_global_if(out + q, j0, k0);
    q += k0;
    st_global_if(out + q, j0 + 1, k1);
    q += k1;
    st_global_if(out + q, j0 + 2, k2);
    q += k2;
    st_global_if(out + q, j0 + 3, k3);
    base += (int)tot;
  }
  for (int t = nfc; t < nc; ++t) {
    const int v = 32 * t + lane;
    const int nv = nvalid(v);
    uint4 kk = make_uint4(0u, 0u, 0u, 0u);
    if (nv > 0) kk = key[v];
    const uint32_t a0 = kk.x & pmask, a1 = kk.y & pmask, a2 = kk.z & pmask, a3 = kk.w & pmask;
    const int j0 = 4 * v;
    bool k0, k1, k2, k3;
    if (whole) {
      k0 = nv > 0 && a0 >= prefix;
      k1 = nv > 1 && a1 >= prefix;
      k2 = nv > 2 && a2 >= prefix;
      k3 = nv > 3 && a3 >= prefix;
    } else {
      const bool e0 = nv > 0 && a0 == prefix, e1 = nv > 1 && a1 == prefix;
      const bool e2 = nv > 2 && a2 == prefix, e3 = nv > 3 && a3 == prefix;
      uint32_t etot;
      const uint32_t r0 = eq_before + warp_excl_scan((uint32_t)e0 + e1 + e2 + e3, lane, etot);
      const uint32_t r1 = r0 + e0, r2 = r1 + e1, r3 = r2 + e2;
      eq_before += etot;
      k0 = nv > 0 && (a0 > prefix || (e0 && r0 < remaining));
      k1 = nv > 1 && (a1 > prefix || (e1 && r1 < remaining));
      k2 = nv > 2 && (a2 > prefix || (e2 && r2 < remaining));
      k3 = nv > 3 && (a3 > prefix || (e3 && r3 < remaining));
    }
    if (force_diag) {
      k0 = k0 || (nv > 0 && j0 == i);
      k1 = k1 || (nv > 1 && j0 + 1 == i);
      k2 = k2 || (nv > 2 && j0 + 2 == i);
      k3 = k3 || (nv > 3 && j0 + 3 == i);
    }
    uint32_t tot;
    uint32_t q = base + warp_excl_scan((uint32_t)k0 + k1 + k2 + k3, lane, tot);
    st_global_if(out + q, j0, k0);
    q += k0;
    st_global_if(out + q, j0 + 1, k1);
    q += k1;
    st_global_if(out + q, j0 + 2, k2);
    q += k2;
    st_global_if(out + q, j0 + 3, k3);
    base += (int)tot;
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
                        float* out, cudaStream_t st, const int2* tab, float* lo) {
  const long long nblocks = BH * (n / kBlock);
  const int warps = 8;
  const unsigned grid = (unsigned)((nblocks + warps - 1) / warps);
  if (dt == SEER_BF16) {
    if (is_k)
      pool_kernel<uint16_t, true><<<grid, warps * 32, 0, st>>>((const uint16_t*)X, nblocks, n, d, out, tab, lo);
    else
      pool_kernel<uint16_t, false><<<grid, warps * 32, 0, st>>>((const uint16_t*)X, nblocks, n, d, out, tab, lo);
  } else {
    if (is_k)
      pool_kernel<float, true><<<grid, warps * 32, 0, st>>>((const float*)X, nblocks, n, d, out, tab, lo);
    else
      pool_kernel<float, false><<<grid, warps * 32, 0, st>>>((const float*)X, nblocks, n, d, out, tab, lo);
  }
  return cudaGetLastError();
}

cudaError_t launch_gate_inputs(const GateInputs& g, seer_dtype dt, cudaStream_t st) {
  const long long wsplit = 148;  // CTAs that split the weights (grid-stride)
  const long long grid = g.cq + g.ck + wsplit;
  if (dt == SEER_BF16)
    gate_inputs_kernel<uint16_t><<<(unsigned)grid, 256, 0, st>>>(g);
  else
    gate_inputs_kernel<float><<<(unsigned)grid, 256, 0, st>>>(g);
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
    if (!tab && row_len <= 0 && nb % 4 == 0 && (reinterpret_cast<uintptr_t>(in) & 15) == 0 &&
        (!scores || (reinterpret_cast<uintptr_t>(scores) & 15) == 0)) {
      // rows start 16-byte aligned: four candidates per lane and access.  Two
      // launches: the shorter half of the rows (query blocks below nb / 2)
      // with half-size row buffers, so more warps share an SM, then the rest.
      auto kern4 = from_logits ? row_select_warp4_kernel<true> : row_select_warp4_kernel<false>;
      const long long heads = rows / nb;
      const int half_w = ((nb / 2 + 3) / 4) * 4;
      const long long split = heads * (long long)(nb / 2);
      const long long lo[2] = {0, split}, hi[2] = {split, rows};
      const int wd[2] = {half_w, nb};
      for (int c = 0; c < 2; ++c) {
        if (hi[c] <= lo[c]) continue;
        const size_t sm = sizeof(uint32_t) * (size_t)kSelWarps * (256 + wd[c]);
        cudaError_t e = cudaFuncSetAttribute(kern4, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        const unsigned g = (unsigned)((hi[c] - lo[c] + kSelWarps - 1) / kSelWarps);
        kern4<<<g, 32 * kSelWarps, sm, st>>>(in, from_logits ? scores : nullptr, rows, nb, mode, T, k, density,
                                            counts, indices, cap, lo[c], hi[c], wd[c]);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
      }
      return cudaSuccess;
    }
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
