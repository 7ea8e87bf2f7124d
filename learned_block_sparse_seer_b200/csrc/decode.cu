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
// Everything here is bound by HBM (one query row per (batch, head), so no
// contraction is large enough for the tensor cores).  The common pattern is
// the "slab": a warp reads 8 x 512 contiguous bytes with one 16-byte load per
// lane per row chunk (lane l takes chunk l % LPR of row i * RPI + l / LPR in
// load i), multiplies its chunk by the matching chunk of the query in
// registers, and a butterfly reduce-scatter over the LPR lanes of a row
// leaves every lane with the full dot product of one row (7 shuffles for 8
// rows instead of 8 full reductions).
//
// Kernels:
//   kcache_kernel       CTA per (batch, KV head, 16 blocks): pooling by slabs,
//                       then the projection k~ = Wk[g] kbar as a shared-memory
//                       tiled product in packed f32x2 FMAs (Wk read once per
//                       16 blocks, each 32-feature slice loaded one slice
//                       ahead)
//   decode_logits_kernel  CTA per (batch, KV head, head group, row chunk):
//                       q . k~_j / sqrt(d) for GT query heads of the group at
//                       once (k~ read once for them); the softmax and the
//                       selection then reuse the prefill row kernel
//   decode_attn_kernel  split-KV: CTA (row, split) takes a contiguous range of
//                       the row's list (selected blocks, then the current
//                       block); each warp runs its own online softmax over
//                       16..64-row slabs with K and V loads issued together;
//                       the last CTA of a row (atomic ticket) merges the splits
//                       by log-sum-exp into O and LSE
//   decode_gt_kernel    CTA per (batch, KV head, head group, chunk of key
//                       blocks): scores of GT query heads per K read, each
//                       block's raw maximum and the chunk's (m, l); the last
//                       CTA of the group turns the maxima into probabilities
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "decode.cuh"
#include "ptx.cuh"

namespace seer {

namespace dec {

// 16-byte chunk conversions.
template <typename T>
struct Chunk;
template <>
struct Chunk<uint16_t> {  // bf16
  static constexpr int N = 8;
  __device__ static __forceinline__ void cvt(const uint4& u, float (&x)[8]) {
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
    x[4] = __uint_as_float(u.z << 16);
    x[5] = __uint_as_float(u.z & 0xffff0000u);
    x[6] = __uint_as_float(u.w << 16);
    x[7] = __uint_as_float(u.w & 0xffff0000u);
  }
};
template <>
struct Chunk<float> {
  static constexpr int N = 4;
  __device__ static __forceinline__ void cvt(const uint4& u, float (&x)[4]) {
    x[0] = __uint_as_float(u.x);
    x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z);
    x[3] = __uint_as_float(u.w);
  }
};

template <typename T, int D>
struct Slab {
  static constexpr int EPC = Chunk<T>::N;   // elements per 16-byte chunk
  static constexpr int LPR = D / EPC;       // lanes (chunks) per row
  static constexpr int RPI = 32 / LPR;      // rows per load instruction
  static constexpr int ROWS = 8 * RPI;      // rows per slab
  static_assert(LPR >= 8 && LPR <= 32, "a row must be 8..32 chunks");
  // lane's row within the slab for load i, and its chunk
  __device__ static __forceinline__ int row(int i, int lane) { return i * RPI + lane / LPR; }
  __device__ static __forceinline__ int chunk(int lane) { return lane % LPR; }
};

// Streaming 16-byte read-only load (no L1 allocation).
__device__ __forceinline__ uint4 ldg16(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

template <typename T>
__device__ __forceinline__ float ld1(const T* p, long long i) {
  if constexpr (sizeof(T) == 2)
    return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(p)[i] << 16);
  else
    return p[i];
}

// Butterfly reduce-scatter of 8 load-rows x GT heads over the LPR lanes that
// hold a row's chunks.  On return v[0][h] is the full dot product, for head
// h, of the lane's row; the function returns that row's load index (the row
// is Slab::row(index, lane)).
template <int LPR, int GT>
__device__ __forceinline__ int reduce_rows(float (&v)[8][GT], int lane) {
  constexpr int O1 = LPR / 2, O2 = LPR / 4, O3 = LPR / 8;
  const bool a = lane & O1, b = lane & O2, c = lane & O3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < GT; ++h) {
      const float send = a ? v[i][h] : v[i + 4][h];
      const float keep = a ? v[i + 4][h] : v[i][h];
      v[i][h] = keep + __shfl_xor_sync(0xffffffffu, send, O1);
    }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int h = 0; h < GT; ++h) {
      const float send = b ? v[i][h] : v[i + 2][h];
      const float keep = b ? v[i + 2][h] : v[i][h];
      v[i][h] = keep + __shfl_xor_sync(0xffffffffu, send, O2);
    }
#pragma unroll
  for (int h = 0; h < GT; ++h) {
    const float send = c ? v[0][h] : v[1][h];
    const float keep = c ? v[1][h] : v[0][h];
    v[0][h] = keep + __shfl_xor_sync(0xffffffffu, send, O3);
  }
#pragma unroll
  for (int o = O3 / 2; o > 0; o >>= 1)
#pragma unroll
    for (int h = 0; h < GT; ++h) v[0][h] += __shfl_xor_sync(0xffffffffu, v[0][h], o);
  return 4 * (int)a + 2 * (int)b + (int)c;
}

// The lane of this lane's row group that holds load-row i after reduce_rows.
template <int LPR>
__device__ __forceinline__ int holder(int i, int lane) {
  return (lane & ~(LPR - 1)) | (((i >> 2) & 1) * (LPR / 2)) | (((i >> 1) & 1) * (LPR / 4)) | ((i & 1) * (LPR / 8));
}

// True on exactly one lane of each row's LPR lanes after reduce_rows.
template <int LPR>
__device__ __forceinline__ bool row_owner(int lane) {
  return (lane & (LPR / 8 - 1)) == 0;
}

}  // namespace dec

// ---------------------------------------------------- compressed K cache --
namespace {
constexpr int kKcBlocks = 16;  // key blocks per CTA
constexpr int kKcThreads = 256;
}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(kKcThreads, 4) kcache_kernel(const T* __restrict__ K, const float* __restrict__ Wk,
                                                            float* __restrict__ kt, int Hkv, int n_cap, int j0,
                                                            int nnew) {
  using S = dec::Slab<T, D>;
  constexpr int E = S::EPC;
  constexpr int NG = kKcThreads / D;   // output groups
  constexpr int BPG = kKcBlocks / NG;  // blocks per output group (4 or 8)
  constexpr int SPB = kBlock / S::ROWS;
  constexpr int WS = D + 1;            // padded row of the weight tile
  extern __shared__ __align__(16) float sm[];
  float* kbarT = sm;                   // [3D][kKcBlocks]: pooled features, blocks contiguous
  float* wt = sm + 3 * D * kKcBlocks;  // [32][D + 1]: a 32-feature slice of Wk[g]^T
  const int nch = (nnew + kKcBlocks - 1) / kKcBlocks;
  const long long bh = blockIdx.x / nch;
  const int ch = (int)(blockIdx.x % nch);
  const int g = (int)(bh % Hkv);
  const int jb = j0 + ch * kKcBlocks;
  const int nblk = min(kKcBlocks, j0 + nnew - jb);
  const int nb_cap = n_cap / kBlock;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- pooling: warp w takes blocks w, w + 8; two slabs of loads in flight
  for (int t = warp; t < kKcBlocks; t += kKcThreads / 32) {
    float mx[E], mn[E], su[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      mx[e] = -INFINITY;
      mn[e] = INFINITY;
      su[e] = 0.f;
    }
    if (t < nblk) {
      const T* base = K + (bh * n_cap + (long long)(jb + t) * kBlock) * D + S::chunk(lane) * E;
#pragma unroll
      for (int s0 = 0; s0 < SPB; s0 += 2) {
        uint4 u[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          u[i] = dec::ldg16(base + (long long)((s0 + (i >> 3)) * S::ROWS + S::row(i & 7, lane)) * D);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x[E];
          dec::Chunk<T>::cvt(u[i], x);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            mx[e] = fmaxf(mx[e], x[e]);
            mn[e] = fminf(mn[e], x[e]);
            su[e] += x[e];
          }
        }
      }
    }
#pragma unroll
    for (int o = S::LPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], o));
        mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], o));
        su[e] += __shfl_xor_sync(0xffffffffu, su[e], o);
      }
    if (lane < S::LPR) {
      // blocks past the range pool to 0 (finite), their outputs are dropped
      const bool live = t < nblk;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int f = lane * E + e;
        kbarT[f * kKcBlocks + t] = live ? mx[e] : 0.f;
        kbarT[(D + f) * kKcBlocks + t] = live ? mn[e] : 0.f;
        kbarT[(2 * D + f) * kKcBlocks + t] = live ? su[e] * (1.0f / kBlock) : 0.f;
      }
    }
  }

  // ---- projection: thread (o, group) accumulates BPG blocks in f32x2 pairs
  const int o = threadIdx.x % D, grp = threadIdx.x / D;
  uint64_t acc[BPG / 2];
#pragma unroll
  for (int b = 0; b < BPG / 2; ++b) acc[b] = 0ull;
  const float* W = Wk + (long long)g * D * 3 * D;
  // The 32-feature slices of Wk[g] go through registers one slice ahead, so
  // that a slice's loads are in flight while the previous one is multiplied.
  constexpr int PER = D * 32 / kKcThreads;  // elements of a slice per thread
  float wr[PER];
  auto load_slice = [&](int e0) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int x = threadIdx.x + i * kKcThreads, r = x >> 5, cc = x & 31;
      wr[i] = W[(long long)r * 3 * D + e0 + cc];
    }
  };
  load_slice(0);
  for (int e0 = 0; e0 < 3 * D; e0 += 32) {
    __syncthreads();  // kbarT complete / previous tile consumed
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int x = threadIdx.x + i * kKcThreads, r = x >> 5, cc = x & 31;
      wt[cc * WS + r] = wr[i];
    }
    __syncthreads();
    if (e0 + 32 < 3 * D) load_slice(e0 + 32);
#pragma unroll 4
    for (int ee = 0; ee < 32; ++ee) {
      const float w = wt[ee * WS + o];
      const uint64_t w2 = f32x2_pack(w, w);
      const float4* kb = reinterpret_cast<const float4*>(kbarT + (e0 + ee) * kKcBlocks + grp * BPG);
#pragma unroll
      for (int b4 = 0; b4 < BPG / 4; ++b4) {
        const float4 v = kb[b4];
        acc[2 * b4] = fma_f32x2(w2, f32x2_pack(v.x, v.y), acc[2 * b4]);
        acc[2 * b4 + 1] = fma_f32x2(w2, f32x2_pack(v.z, v.w), acc[2 * b4 + 1]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BPG / 2; ++b) {
    float lo, hi;
    f32x2_unpack(acc[b], lo, hi);
    const int t = grp * BPG + 2 * b;
    if (t < nblk) kt[(bh * nb_cap + jb + t) * D + o] = lo;
    if (t + 1 < nblk) kt[(bh * nb_cap + jb + t + 1) * D + o] = hi;
  }
}

// ------------------------------------------------------------ gate logits --
template <typename T, int D, int GT>
__global__ void __launch_bounds__(128) decode_logits_kernel(const T* __restrict__ q, const float* __restrict__ kt,
                                                            float* __restrict__ logits, int Hq, int Hkv, int nc,
                                                            int nb_cap, int rows_per_cta, int nch, float scale) {
  using S = dec::Slab<float, D>;
  constexpr int E = S::EPC;
  const int G = Hq / Hkv, nhg = G / GT;
  const int ch = (int)(blockIdx.x % nch);
  const long long grp = blockIdx.x / nch;  // (b * Hkv + g) * nhg + hg
  const int hg = (int)(grp % nhg);
  const long long bg = grp / nhg;
  const long long b = bg / Hkv;
  const int g = (int)(bg % Hkv);
  const long long row0 = b * Hq + (long long)g * G + hg * GT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float qv[GT][E];
#pragma unroll
  for (int h = 0; h < GT; ++h)
#pragma unroll
    for (int e = 0; e < E; ++e) qv[h][e] = dec::ld1(q, (row0 + h) * D + S::chunk(lane) * E + e) * scale;
  const float* kg = kt + bg * (long long)nb_cap * D + S::chunk(lane) * E;
  const int r_begin = ch * rows_per_cta, r_end = min(nc, r_begin + rows_per_cta);
  for (int r0 = r_begin + warp * S::ROWS; r0 < r_end; r0 += 4 * S::ROWS) {
    uint4 u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = r0 + S::row(i, lane);
      u[i] = r < r_end ? dec::ldg16(kg + (long long)r * D) : make_uint4(0u, 0u, 0u, 0u);
    }
    float v[8][GT];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float x[E];
      dec::Chunk<float>::cvt(u[i], x);
#pragma unroll
      for (int h = 0; h < GT; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) a = fmaf(x[e], qv[h][e], a);
        v[i][h] = a;
      }
    }
    const int ii = dec::reduce_rows<S::LPR, GT>(v, lane);
    const int r = r0 + S::row(ii, lane);
    if (dec::row_owner<S::LPR>(lane) && r < r_end) {
#pragma unroll
      for (int h = 0; h < GT; ++h) logits[(row0 + h) * nc + r] = v[0][h];
    }
  }
}

// ------------------------------------------------ streamed key-block ring --
// The attention and ground-truth kernels stream whole key blocks through a
// shared-memory ring filled by 1D bulk copies (TMA, no multicast): warp NS
// issues the copies, consumer warp w takes the CTA's blocks w, w + NS, ...
// from stage w, so every stage has one consumer and its own full/empty
// mbarrier pair.  About 96 KB of ring per CTA, two CTAs per SM.
template <int BLK_BYTES>
struct Ring {
  static constexpr int NS = (98304 / BLK_BYTES) < 2 ? 2 : ((98304 / BLK_BYTES) > 8 ? 8 : (98304 / BLK_BYTES));
  static constexpr int THREADS = 32 * (NS + 1);
  static constexpr uint32_t SMEM = (uint32_t)NS * BLK_BYTES;
};

// ------------------------------------------------------ decode attention --
struct DecAttnP {
  const void* q;
  const void* K;
  const void* V;
  const int32_t* counts;
  const int32_t* indices;
  int cap, Hq, Hkv, n_cap, seq_len, splits;
  float scale_log2;
  float* part;
  int32_t* ticket;
  void* O;
  float* lse;
  uint32_t* status;
  unsigned long long timeout_ns;
};

// The attention ring: NS stages of one key block (K then V); NC consumer
// warps share every block, warp w taking slabs w, w + NC, ... of it, so a
// stage is released after a quarter of a block's work instead of a whole one.
template <typename T, int D>
struct AttnRing : Ring<2 * kBlock * D * (int)sizeof(T)> {
  static constexpr uint32_t HALF = (uint32_t)kBlock * D * sizeof(T);  // K (then V) of a block
  static constexpr int NC = 4;                                          // consumer warps
  static constexpr int THREADS = 32 * (NC + 1);                         // + the copy warp
};

template <typename T, int D>
__global__ void __launch_bounds__(AttnRing<T, D>::THREADS, 2) decode_attn_kernel(const DecAttnP p) {
  using S = dec::Slab<T, D>;
  using R = AttnRing<T, D>;
  constexpr int E = S::EPC;
  constexpr int LPR = S::LPR;
  constexpr int NS = R::NS;
  constexpr int NC = R::NC;
  constexpr int SPB = kBlock / S::ROWS;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[NS], empty[NS];
  __shared__ int abort_flag, last;
  __shared__ float wm[NC], wl[NC], wo[NC][D];
  const long long row = blockIdx.x / p.splits;
  const int split = (int)(blockIdx.x % p.splits);
  const long long b = row / p.Hq;
  const int hq = (int)(row % p.Hq), g = hq / (p.Hq / p.Hkv);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = (p.seq_len - 1) / kBlock;
  const int tail = p.seq_len - c * kBlock;  // keys of the token's own block
  int cnt = p.counts[row];
  const int lim = min(p.cap, c);
  if (cnt < 0 || cnt > lim) {
    if (tid == 0 && split == 0) record_status(p.status, kDevBadIndex, (uint32_t)row);
    cnt = cnt < 0 ? 0 : lim;
  }
  // this CTA's range of the row's entries (the selected blocks, then block c)
  const int total = cnt + 1;
  const int per = (total + p.splits - 1) / p.splits;
  const int e0 = split * per, e1 = min(total, e0 + per);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NC);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_p = &abort_flag;
  const long long head0 = (b * p.Hkv + g) * (long long)p.n_cap * D;

  if (warp == NC) {
    // ------------------------------------------------------- producer ---
    if (lane == 0) {
      const T* Kh = reinterpret_cast<const T*>(p.K) + head0;
      const T* Vh = reinterpret_cast<const T*>(p.V) + head0;
      int it = 0;
      for (int e = e0; e < e1; ++e, ++it) {
        const int s = it % NS;
        if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, abort_p, p.status, p.timeout_ns)) break;
        int j = c, nk = tail;
        if (e < cnt) {
          j = p.indices[row * p.cap + e];
          if (j < 0 || j >= c) {
            record_status(p.status, kDevBadIndex, (uint32_t)row);
            j = j < 0 ? 0 : c - 1;
          }
          nk = kBlock;
        }
        const uint32_t bytes = (uint32_t)nk * D * sizeof(T);
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        bulk_load(ring + (size_t)s * 2 * R::HALF, Kh + (long long)j * kBlock * D, bytes, &full[s]);
        bulk_load(ring + (size_t)s * 2 * R::HALF + R::HALF, Vh + (long long)j * kBlock * D, bytes, &full[s]);
      }
      // every issued copy has landed before the CTA may exit
      for (int k = it > NS ? it - NS : 0; k < it; ++k)
        wait_landed(&full[k % NS], (k / NS) & 1);
    }
  } else {
    // ------------------------------------------------------ consumers ---
    const T* q = reinterpret_cast<const T*>(p.q);
    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = dec::ld1(q, row * D + S::chunk(lane) * E + e) * p.scale_log2;
    float m = -INFINITY, l = 0.f, o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.f;
    int k = 0;  // blocks taken so far (every consumer takes every block)
    for (int e = e0; e < e1; ++e, ++k) {
      const int st = k % NS;
      if (!mbar_wait(&full[st], (k / NS) & 1, abort_p, p.status, p.timeout_ns)) break;
      const int nk = e < cnt ? kBlock : tail;
      const uint8_t* Ks = ring + (size_t)st * 2 * R::HALF + S::chunk(lane) * 16;
      const uint8_t* Vs = Ks + R::HALF;
#pragma unroll
      for (int sb = warp; sb < SPB; sb += NC) {
        const int rbase = sb * S::ROWS;
        if (rbase >= nk) break;  // past the token (warp-uniform)
        uint4 ku[8], vu[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = rbase + S::row(i, lane);
          const bool ok = r < nk;
          ku[i] = ok ? *reinterpret_cast<const uint4*>(Ks + (size_t)r * D * sizeof(T)) : make_uint4(0u, 0u, 0u, 0u);
          vu[i] = ok ? *reinterpret_cast<const uint4*>(Vs + (size_t)r * D * sizeof(T)) : make_uint4(0u, 0u, 0u, 0u);
        }
        float v[8][1];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float x[E];
          dec::Chunk<T>::cvt(ku[i], x);
          float a = 0.f;
#pragma unroll
          for (int ee = 0; ee < E; ++ee) a = fmaf(x[ee], qv[ee], a);
          v[i][0] = a;
        }
        const int ii = dec::reduce_rows<LPR, 1>(v, lane);
        const float sc = rbase + S::row(ii, lane) < nk ? v[0][0] : -INFINITY;
        const float mn = fmaxf(m, warp_max(sc));  // finite: row rbase is a key
        const float alpha = exp2f(m - mn);
        const float pr = exp2f(sc - mn);
        l = l * alpha + (dec::row_owner<LPR>(lane) ? pr : 0.f);
#pragma unroll
        for (int ee = 0; ee < E; ++ee) o[ee] *= alpha;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float pi = __shfl_sync(0xffffffffu, pr, dec::holder<LPR>(i, lane));
          float x[E];
          dec::Chunk<T>::cvt(vu[i], x);
#pragma unroll
          for (int ee = 0; ee < E; ++ee) o[ee] = fmaf(pi, x[ee], o[ee]);
        }
        m = mn;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    l = warp_sum(l);
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
      for (int ee = 0; ee < E; ++ee) o[ee] += __shfl_xor_sync(0xffffffffu, o[ee], off);
    if (lane < LPR) {
#pragma unroll
      for (int ee = 0; ee < E; ++ee) wo[warp][lane * E + ee] = o[ee];
    }
    if (lane == 0) {
      wm[warp] = m;
      wl[warp] = l;
    }
  }
  __syncthreads();
  // ---- the CTA's partial (m, l, o)
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NC; ++w) M = fmaxf(M, wm[w]);
  float* pp = p.part + (row * p.splits + split) * (long long)(D + 2);
  for (int t = tid; t < D; t += R::THREADS) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < NC; ++w)
      if (wm[w] > -INFINITY) a += wo[w][t] * exp2f(wm[w] - M);
    pp[t] = a;
  }
  if (tid == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < NC; ++w)
      if (wm[w] > -INFINITY) L += wl[w] * exp2f(wm[w] - M);
    pp[D] = M;
    pp[D + 1] = L;
  }
  // ---- the row's last CTA merges the splits
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(p.ticket + row, 1) == p.splits - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* pr = p.part + row * p.splits * (long long)(D + 2);
  M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, __ldcg(pr + s * (D + 2) + D));
  float L = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const float ms = __ldcg(pr + s * (D + 2) + D);
    if (ms > -INFINITY) L += __ldcg(pr + s * (D + 2) + D + 1) * exp2f(ms - M);
  }
  const float invL = 1.0f / L;
  for (int t = tid; t < D; t += R::THREADS) {
    float a = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float ms = __ldcg(pr + s * (D + 2) + D);
      if (ms > -INFINITY) a += __ldcg(pr + s * (D + 2) + t) * exp2f(ms - M);
    }
    const float v = a * invL;
    if constexpr (sizeof(T) == 2)
      reinterpret_cast<__nv_bfloat16*>(p.O)[row * D + t] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<float*>(p.O)[row * D + t] = v;
  }
  if (tid == 0) {
    if (p.lse) p.lse[row] = (M + log2f(L)) * 0.6931471805599453f;
    p.ticket[row] = 0;
  }
}

// ------------------------------------------------------ 1D ground truth ---
struct DecGtP {
  const void* q;
  const void* K;
  int Hq, Hkv, n_cap, seq_len, bpc, nch;
  float scale_log2;
  float* gt;
  float* lse;
  float* stats;
  int32_t* ticket;
  uint32_t* status;
  unsigned long long timeout_ns;
};

template <typename T, int D>
struct GtRing : Ring<kBlock * D * (int)sizeof(T)> {
  static constexpr uint32_t BLK = (uint32_t)kBlock * D * sizeof(T);
};

template <typename T, int D, int GT>
__global__ void __launch_bounds__(GtRing<T, D>::THREADS, 2) decode_gt_kernel(const DecGtP p) {
  using S = dec::Slab<T, D>;
  using R = GtRing<T, D>;
  constexpr int E = S::EPC;
  constexpr int LPR = S::LPR;
  constexpr int NS = R::NS;
  constexpr int SPB = kBlock / S::ROWS;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[NS], empty[NS];
  __shared__ int abort_flag, last;
  __shared__ float wm[NS][GT], wl[NS][GT];
  __shared__ float lse2[GT];
  const int G = p.Hq / p.Hkv, nhg = G / GT;
  const int ch = (int)(blockIdx.x % p.nch);
  const long long grp = blockIdx.x / p.nch;  // (b * Hkv + g) * nhg + hg
  const int hg = (int)(grp % nhg);
  const long long bg = grp / nhg;
  const long long b = bg / p.Hkv;
  const int g = (int)(bg % p.Hkv);
  const long long row0 = b * p.Hq + (long long)g * G + hg * GT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = (p.seq_len - 1) / kBlock;
  const int nbc = c + 1;
  const int tail = p.seq_len - c * kBlock;
  const int jb = ch * p.bpc, je = min(nbc, jb + p.bpc);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_p = &abort_flag;

  if (warp == NS) {
    // ------------------------------------------------------- producer ---
    if (lane == 0) {
      const T* Kh = reinterpret_cast<const T*>(p.K) + bg * (long long)p.n_cap * D;
      int it = 0;
      for (int j = jb; j < je; ++j, ++it) {
        const int s = it % NS;
        if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, abort_p, p.status, p.timeout_ns)) break;
        const uint32_t bytes = (uint32_t)(j < c ? kBlock : tail) * D * sizeof(T);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load(ring + (size_t)s * R::BLK, Kh + (long long)j * kBlock * D, bytes, &full[s]);
      }
      for (int k = it > NS ? it - NS : 0; k < it; ++k)
        wait_landed(&full[k % NS], (k / NS) & 1);
    }
  } else {
    // ------------------------------------------------------ consumers ---
    const T* q = reinterpret_cast<const T*>(p.q);
    float qv[GT][E];
#pragma unroll
    for (int h = 0; h < GT; ++h)
#pragma unroll
      for (int e = 0; e < E; ++e) qv[h][e] = dec::ld1(q, (row0 + h) * D + S::chunk(lane) * E + e) * p.scale_log2;
    // per-lane online statistics over the lane's own rows
    float m[GT], l[GT];
#pragma unroll
    for (int h = 0; h < GT; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
    }
    const bool own = dec::row_owner<LPR>(lane);
    int k = 0;
    for (int j = jb + warp; j < je; j += NS, ++k) {
      if (!mbar_wait(&full[warp], k & 1, abort_p, p.status, p.timeout_ns)) break;
      const int nk = j < c ? kBlock : tail;
      const uint8_t* Ks = ring + (size_t)warp * R::BLK + S::chunk(lane) * 16;
      float bm[GT];
#pragma unroll
      for (int h = 0; h < GT; ++h) bm[h] = -INFINITY;
#pragma unroll
      for (int sb = 0; sb < SPB; ++sb) {
        const int rbase = sb * S::ROWS;
        if (rbase >= nk) break;  // warp-uniform
        uint4 ku[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = rbase + S::row(i, lane);
          ku[i] = r < nk ? *reinterpret_cast<const uint4*>(Ks + (size_t)r * D * sizeof(T)) : make_uint4(0u, 0u, 0u, 0u);
        }
        float v[8][GT];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float x[E];
          dec::Chunk<T>::cvt(ku[i], x);
#pragma unroll
          for (int h = 0; h < GT; ++h) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) a = fmaf(x[e], qv[h][e], a);
            v[i][h] = a;
          }
        }
        const int ii = dec::reduce_rows<LPR, GT>(v, lane);
        const bool ok = rbase + S::row(ii, lane) < nk;
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          if (ok) {
            const float sc = v[0][h];
            bm[h] = fmaxf(bm[h], sc);
            if (own) {
              const float mn = fmaxf(m[h], sc);
              l[h] = l[h] * exp2f(m[h] - mn) + exp2f(sc - mn);
              m[h] = mn;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[warp]);
#pragma unroll
      for (int h = 0; h < GT; ++h) bm[h] = warp_max(bm[h]);
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < GT; ++h) p.gt[(row0 + h) * nbc + j] = bm[h];  // raw, log2 units
      }
    }
    // the warp's statistics per head
#pragma unroll
    for (int h = 0; h < GT; ++h) {
      const float M = warp_max(m[h]);
      const float lw = warp_sum(m[h] > -INFINITY ? l[h] * exp2f(m[h] - M) : 0.f);
      if (lane == 0) {
        wm[warp][h] = M;
        wl[warp][h] = lw;
      }
    }
  }
  __syncthreads();
  if (tid < GT) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NS; ++w) M = fmaxf(M, wm[w][tid]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < NS; ++w)
      if (wm[w][tid] > -INFINITY) L += wl[w][tid] * exp2f(wm[w][tid] - M);
    float* st = p.stats + ((row0 + tid) * kGtMaxChunks + ch) * 2;
    st[0] = M;
    st[1] = L;
  }
  // ---- the group's last CTA: the rows' LSE, then maxima -> probabilities
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(p.ticket + grp, 1) == p.nch - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (tid < GT) {
    const float* st = p.stats + (row0 + tid) * kGtMaxChunks * 2;
    float M = -INFINITY;
    for (int k = 0; k < p.nch; ++k) M = fmaxf(M, __ldcg(st + 2 * k));
    float L = 0.f;
    for (int k = 0; k < p.nch; ++k) {
      const float mk = __ldcg(st + 2 * k);
      if (mk > -INFINITY) L += __ldcg(st + 2 * k + 1) * exp2f(mk - M);
    }
    lse2[tid] = M + log2f(L);
    if (p.lse) p.lse[row0 + tid] = lse2[tid] * 0.6931471805599453f;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < GT; ++h) {
    float* gr = p.gt + (row0 + h) * nbc;
    for (int j = tid; j < nbc; j += R::THREADS) gr[j] = exp2f(__ldcg(gr + j) - lse2[h]);
  }
  if (tid == 0) p.ticket[grp] = 0;
}

// ------------------------------------------------------------- launchers --
namespace {
int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n = v;
  }
  return n;
}

// largest of 4, 2, 1 that divides the group size
int head_tile(int G) { return G % 4 == 0 ? 4 : (G % 2 == 0 ? 2 : 1); }
}  // namespace

cudaError_t launch_kcache(const void* K, bool fp32, const float* Wk, float* kt, long long BHkv, int Hkv, int n_cap,
                          int d, int j0, int nnew, cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)kKcBlocks * 3 * d + 32 * (size_t)(d + 1));
  const long long grid = BHkv * ((nnew + kKcBlocks - 1) / kKcBlocks);
  if (fp32) {
    if (d == 64)
      kcache_kernel<float, 64><<<(unsigned)grid, kKcThreads, smem, st>>>((const float*)K, Wk, kt, Hkv, n_cap, j0, nnew);
    else
      kcache_kernel<float, 128><<<(unsigned)grid, kKcThreads, smem, st>>>((const float*)K, Wk, kt, Hkv, n_cap, j0,
                                                                          nnew);
  } else {
    if (d == 64)
      kcache_kernel<uint16_t, 64><<<(unsigned)grid, kKcThreads, smem, st>>>((const uint16_t*)K, Wk, kt, Hkv, n_cap,
                                                                            j0, nnew);
    else
      kcache_kernel<uint16_t, 128><<<(unsigned)grid, kKcThreads, smem, st>>>((const uint16_t*)K, Wk, kt, Hkv, n_cap,
                                                                             j0, nnew);
  }
  return cudaGetLastError();
}

template <typename T, int D>
static void logits_dispatch_gt(int GT, unsigned grid, const T* q, const float* kt, float* logits, int Hq, int Hkv,
                               int nc, int nb_cap, int rpc, int nch, float scale, cudaStream_t st) {
  if (GT == 4)
    decode_logits_kernel<T, D, 4><<<grid, 128, 0, st>>>(q, kt, logits, Hq, Hkv, nc, nb_cap, rpc, nch, scale);
  else if (GT == 2)
    decode_logits_kernel<T, D, 2><<<grid, 128, 0, st>>>(q, kt, logits, Hq, Hkv, nc, nb_cap, rpc, nch, scale);
  else
    decode_logits_kernel<T, D, 1><<<grid, 128, 0, st>>>(q, kt, logits, Hq, Hkv, nc, nb_cap, rpc, nch, scale);
}

cudaError_t launch_decode_logits(const void* q, bool fp32, const float* kt, float* logits, long long B, int Hq,
                                 int Hkv, int d, int nc, int nb_cap, float scale, cudaStream_t st) {
  const int GT = head_tile(Hq / Hkv);
  const long long groups = B * (long long)Hq / GT;
  // rows of a CTA: a multiple of the 4 warps' slabs, about 8 CTAs per SM
  const int unit = 4 * (d == 64 ? 16 : 8);
  long long rpc = (nc * groups + 8LL * sm_count() - 1) / (8LL * sm_count());
  rpc = ((rpc + unit - 1) / unit) * unit;
  if (rpc < unit) rpc = unit;
  const int nch = (int)((nc + rpc - 1) / rpc);
  const unsigned grid = (unsigned)(groups * nch);
  if (fp32) {
    if (d == 64)
      logits_dispatch_gt<float, 64>(GT, grid, (const float*)q, kt, logits, Hq, Hkv, nc, nb_cap, (int)rpc, nch, scale,
                                    st);
    else
      logits_dispatch_gt<float, 128>(GT, grid, (const float*)q, kt, logits, Hq, Hkv, nc, nb_cap, (int)rpc, nch, scale,
                                     st);
  } else {
    if (d == 64)
      logits_dispatch_gt<uint16_t, 64>(GT, grid, (const uint16_t*)q, kt, logits, Hq, Hkv, nc, nb_cap, (int)rpc, nch,
                                       scale, st);
    else
      logits_dispatch_gt<uint16_t, 128>(GT, grid, (const uint16_t*)q, kt, logits, Hq, Hkv, nc, nb_cap, (int)rpc, nch,
                                        scale, st);
  }
  return cudaGetLastError();
}

int decode_attn_splits(long long rows) {
  // two resident CTAs per SM over all rows
  const long long target = 2LL * sm_count();
  long long s = target / rows;
  return (int)(s < 1 ? 1 : (s > 64 ? 64 : s));
}

template <typename T, int D>
static cudaError_t attn_launch(const DecAttnP& p, unsigned grid, cudaStream_t st) {
  using R = AttnRing<T, D>;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)R::SMEM);
  if (e != cudaSuccess) return e;
  decode_attn_kernel<T, D><<<grid, R::THREADS, R::SMEM, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_attn(const DecodeAttnArgs& a, cudaStream_t st) {
  DecAttnP p{a.q,        a.K,          a.V,      a.counts, a.indices, a.cap, a.Hq,    a.Hkv,
             a.n_cap,    a.seq_len,    a.splits, a.scale_log2, a.part, a.ticket, a.O, a.lse,
             a.status,   a.timeout_ns};
  const unsigned grid = (unsigned)(a.rows * a.splits);
  if (a.fp32) return a.d == 64 ? attn_launch<float, 64>(p, grid, st) : attn_launch<float, 128>(p, grid, st);
  return a.d == 64 ? attn_launch<uint16_t, 64>(p, grid, st) : attn_launch<uint16_t, 128>(p, grid, st);
}

template <typename T, int D, int GT>
static cudaError_t gt_launch_one(const DecGtP& p, unsigned grid, cudaStream_t st) {
  using R = GtRing<T, D>;
  cudaError_t e = cudaFuncSetAttribute(decode_gt_kernel<T, D, GT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)R::SMEM);
  if (e != cudaSuccess) return e;
  decode_gt_kernel<T, D, GT><<<grid, R::THREADS, R::SMEM, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t gt_dispatch(int GT, unsigned grid, const DecGtP& p, cudaStream_t st) {
  if (GT == 4) return gt_launch_one<T, D, 4>(p, grid, st);
  if (GT == 2) return gt_launch_one<T, D, 2>(p, grid, st);
  return gt_launch_one<T, D, 1>(p, grid, st);
}

cudaError_t launch_decode_gt(const void* q, const void* K, bool fp32, long long B, int Hq, int Hkv, int d, int n_cap,
                             int seq_len, float scale_log2, float* gt, float* lse, float* stats, int32_t* ticket,
                             uint32_t* status, unsigned long long timeout_ns, cudaStream_t st) {
  const int GT = head_tile(Hq / Hkv);
  const long long groups = B * (long long)Hq / GT;
  const int nbc = (seq_len - 1) / kBlock + 1;
  // one wave of two CTAs per SM, at most kGtMaxChunks chunks a row
  long long nch = (2LL * sm_count()) / groups;
  if (nch > kGtMaxChunks) nch = kGtMaxChunks;
  if (nch > nbc) nch = nbc;
  if (nch < 1) nch = 1;
  const int bpc = (int)((nbc + nch - 1) / nch);
  nch = (nbc + bpc - 1) / bpc;
  DecGtP p{q, K, Hq, Hkv, n_cap, seq_len, bpc, (int)nch, scale_log2, gt, lse, stats, ticket, status, timeout_ns};
  const unsigned grid = (unsigned)(groups * nch);
  if (fp32) return d == 64 ? gt_dispatch<float, 64>(GT, grid, p, st) : gt_dispatch<float, 128>(GT, grid, p, st);
  return d == 64 ? gt_dispatch<uint16_t, 64>(GT, grid, p, st) : gt_dispatch<uint16_t, 128>(GT, grid, p, st);
}

}  // namespace seer
