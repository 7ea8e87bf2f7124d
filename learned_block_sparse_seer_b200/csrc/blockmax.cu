// blockmax.cu -- the max-pooled attention-probability map that SeerAttention's
// gate is distilled against, for sm_100a (B200).
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4, "Ground truth generation"
// (gt = MaxPool2D_{BxB}(softmax(Q K^T / sqrt(d)))) and "The customized
// training kernel" / Figure 10: a first pass over the key blocks forms the
// online-softmax statistics and keeps each row's raw maximum per key block,
// r_ij = rowmax(S_ij); a second pass rescales the kept maxima into
// probabilities a_ij = exp(r_ij - m_i) / l_i and takes the column maximum
// over the rows of the block.
//
// B200 design:
//  * A unit is one query head and two consecutive 64-row query blocks
//    (i0 = 2m, i1 = 2m+1): a 128-row tile, so every tcgen05 MMA is
//    M = 128 x N = 128 (two key blocks per step), both operands from 128-byte
//    swizzled shared memory loaded by TMA (no multicast), S in TMEM (three
//    buffers, so the MMA runs up to two steps ahead of the softmax).
//  * The work is bound by the exponentials (one per causal pair; the MMA is
//    half as long), so four softmax warpgroups share each step: warpgroup w
//    takes the 32 score columns of key block 2s + (w >> 1), half (w & 1).
//    Each thread owns one query row, keeps its own (max, sum) with a lazily
//    raised running max, uses packed f32x2 arithmetic and 3-input max trees,
//    and stores its per-half-block raw maximum to a per-CTA scratch slot
//    (L2-resident, rewritten by every unit).
//  * The second pass runs in the unit's epilogue: the four warpgroups'
//    statistics give each row's log-sum-exp; then each warpgroup takes every
//    fourth key block, reads both halves' kept maxima of each row, turns them
//    into probabilities, and a shuffle reduce-scatter takes the maximum over
//    the 64 rows of each query block.
//  * Warp roles (608 threads): warps 0..15 are the softmax warpgroups, warp
//    16 schedules units and loads Q, warp 17 loads K pairs, warp 18 issues
//    the MMAs (straight-line, unrolled groups).  All waits are bounded.
#include <cstdint>

#include "blockmax.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace seer {

namespace bmax {
constexpr int kThreads = 608;
constexpr int kWarpSched = 16, kWarpK = 17, kWarpMma = 18;
constexpr int kWG = 4;                  // softmax warpgroups
constexpr int kSoftmaxWarps = 4 * kWG;
constexpr int kNK = 4;                  // K pair ring
constexpr int kSBuf = 3;                // S buffers in TMEM (128 columns each)
constexpr uint32_t kTileBytes = 32768;  // 128 rows x 128 dims x bf16
constexpr uint32_t kOffQ = 0;           // 2 x 32 KB
constexpr uint32_t kOffK = 2 * kTileBytes;
constexpr uint32_t kSmemTiles = kOffK + kNK * kTileBytes;  // 192 KB
constexpr uint32_t kTmemCols = 512;                        // S x 3 (128 cols each)
constexpr float kRaise = 8.0f;

struct Ctrl {
  uint64_t unit_full[2], unit_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t s_full[kSBuf], s_free[kSBuf];
  uint64_t wg[kWG], all, fin;
  int unit_w[2];
  uint32_t tmem_base;
  int abort_flag;
  float m_part[kWG][128], l_part[kWG][128];
  float red[kWG][4][32];
};
constexpr uint32_t kSmemAlloc = kSmemTiles + (uint32_t)sizeof(Ctrl);
static_assert(kSmemAlloc <= 232448, "dynamic shared memory above the per-CTA limit");
}  // namespace bmax

namespace {

// A named group of warps meeting at an mbarrier (one arrival per warp).
struct Sync {
  uint64_t* bar;
  volatile int* abort;
  uint32_t* status;
  uint64_t tmo;
  uint32_t phase;
  __device__ __forceinline__ bool sync(int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase & 1, abort, status, tmo);
    ++phase;
    return ok;
  }
};

struct BUnit {
  int b, hq, g, m;
};

__device__ __forceinline__ BUnit decode(const BmaxParams& p, int w) {
  BUnit u;
  const int per_bg = p.npairs * p.G;
  const int bg = w / per_bg, rem = w % per_bg;
  u.b = bg / p.Hkv;
  u.g = bg % p.Hkv;
  u.m = p.npairs - 1 - rem / p.G;
  u.hq = u.g * p.G + rem % p.G;
  return u;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(bmax::kThreads, 1)
    blockmax_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const BmaxParams p) {
  using namespace bmax;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(p.status, kDevBadSchedule, smem_u32(smem));
    return;
  }
  Ctrl& C = *reinterpret_cast<Ctrl*>(smem + kSmemTiles);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  volatile int* abort_p = &C.abort_flag;
  const uint64_t tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    C.abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&C.unit_full[s], 1);
      mbar_init(&C.unit_empty[s], 2 + kSoftmaxWarps);  // K loader, MMA, softmax warps
      mbar_init(&C.q_full[s], 1);
      mbar_init(&C.q_empty[s], 1);
    }
    for (int s = 0; s < kSBuf; ++s) {
      mbar_init(&C.s_full[s], 1);
      mbar_init(&C.s_free[s], kSoftmaxWarps);
    }
    for (int s = 0; s < kWG; ++s) mbar_init(&C.wg[s], 4);
    for (int s = 0; s < kNK; ++s) {
      mbar_init(&C.k_full[s], 1);
      mbar_init(&C.k_empty[s], 1);
    }
    mbar_init(&C.all, kSoftmaxWarps);
    mbar_init(&C.fin, 1);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&C.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;
  constexpr int dpanels = D / 64;
  constexpr uint32_t tile_bytes = 128u * D * 2u;

  if (warp == kWarpSched) {
    // ------------------------------------------------ scheduler + Q loads --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      int u_idx = 0;
      for (;;) {
        const int slot = u_idx & 1;
        if (u_idx >= 2 && !mbar_wait(&C.unit_empty[slot], ((u_idx >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        int w = (int)atomicAdd(p.work_counter, 1u);
        if (w >= p.total_units || *abort_p) w = -1;
        C.unit_w[slot] = w;
        mbar_arrive(&C.unit_full[slot]);
        if (w < 0) break;
        const BUnit u = decode(p, w);
        if (u_idx >= 2 && !mbar_wait(&C.q_empty[slot], ((u_idx >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        mbar_arrive_expect_tx(&C.q_full[slot], tile_bytes);
        const int row = (int)(((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.m * 128);
        for (int pn = 0; pn < dpanels; ++pn)
          tma_load_2d(smem + kOffQ + slot * kTileBytes + pn * 16384, &tmQ, &C.q_full[slot], pn * 64, row);
        ++u_idx;
      }
      for (int k = 0; k < 2 && k < u_idx; ++k) {
        const int uu = u_idx - 1 - k;
        wait_landed(&C.q_full[uu & 1], (uu >> 1) & 1);
      }
    }
  } else if (warp == kWarpK) {
    // --------------------------------------------------------- K loads ---
    if (lane == 0) {
      prefetch_tmap(&tmK);
      int u_idx = 0, step = 0;
      bool ok = true;
      while (ok) {
        const int slot = u_idx & 1;
        if (!mbar_wait(&C.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
        const int w = C.unit_w[slot];
        mbar_arrive(&C.unit_empty[slot]);
        if (w < 0) break;
        ++u_idx;
        const BUnit u = decode(p, w);
        const long long row0 = ((long long)u.b * p.Hkv + u.g) * p.n;
        for (int s = 0; s <= u.m; ++s, ++step) {
          const int ks = step % kNK;
          if (step >= kNK && !mbar_wait(&C.k_empty[ks], ((step / kNK) - 1) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&C.k_full[ks], tile_bytes);
          for (int pn = 0; pn < dpanels; ++pn)
            tma_load_2d(smem + kOffK + ks * kTileBytes + pn * 16384, &tmK, &C.k_full[ks], pn * 64,
                        (int)(row0 + (long long)s * 128));
        }
      }
      for (int k = 0; k < kNK && k < step; ++k) {
        const int st = step - 1 - k;
        wait_landed(&C.k_full[st % kNK], (st / kNK) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA ----
    // Straight-line groups: descriptors are a per-step base plus constant
    // offsets (the start address field holds address >> 4).
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dQ0 = make_sw128_desc(sbase + kOffQ, 16, 1024);
      const uint64_t dK0 = make_sw128_desc(sbase + kOffK, 16, 1024);
      int u_idx = 0, g = 0, ks = 0, kph = 0, sb = 0, sph = 0;
      bool ok = true;
      while (ok) {
        const int slot = u_idx & 1;
        if (!mbar_wait(&C.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
        const int w = C.unit_w[slot];
        mbar_arrive(&C.unit_empty[slot]);
        if (w < 0) break;
        const BUnit u = decode(p, w);
        if (!mbar_wait(&C.q_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
        const uint64_t dq = dQ0 + ((uint64_t)(slot * kTileBytes) >> 4);
        for (int s = 0; s <= u.m; ++s, ++g) {
          if (!mbar_wait(&C.k_full[ks], kph, abort_p, p.status, tmo)) { ok = false; break; }
          // S buffer sb was last read by the softmax of step g - kSBuf
          if (g >= kSBuf && !mbar_wait(&C.s_free[sb], sph ^ 1, abort_p, p.status, tmo)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dk = dK0 + ((uint64_t)(ks * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) / 16);
            mma_bf16_ss(tmem + (uint32_t)sb * 128u, dq + off, dk + off, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&C.s_full[sb]);
          mma_commit(&C.k_empty[ks]);
          if (++ks == kNK) {
            ks = 0;
            kph ^= 1;
          }
          if (++sb == kSBuf) {
            sb = 0;
            sph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&C.q_empty[slot]);
        ++u_idx;
      }
      mma_commit(&C.fin);
      wait_landed(&C.fin, 0);
    }
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------ softmax WGs ---
    const int wgi = warp >> 2;          // warpgroup 0..3
    const int ww = warp & 3;            // TMEM sub-partition
    const int row = ww * 32 + lane;     // query row of the unit's tile, 0..127
    const int half = row >> 6, rloc = row & 63;
    const int jo = wgi >> 1, hh = wgi & 1;  // key block of the pair, column half
    const uint32_t lane_addr = tmem + ((uint32_t)(ww * 32) << 16) + (uint32_t)(jo * 64 + hh * 32);
    const float c = p.scale_log2;
    const uint64_t c2 = f32x2_pack(c, c);
    Sync wgs{&C.wg[wgi], abort_p, p.status, tmo, 0};
    Sync all{&C.all, abort_p, p.status, tmo, 0};
    // per-CTA scratch: [key block][column half][128 rows] raw maxima (log2)
    float* rslot = p.r + (long long)blockIdx.x * 256 * p.nb;
    int u_idx = 0, sb = 0, sph = 0;
    for (;;) {
      const int slot = u_idx & 1;
      if (!mbar_wait(&C.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
      const int w = C.unit_w[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.unit_empty[slot]);
      if (w < 0) break;
      ++u_idx;
      const BUnit u = decode(p, w);
      const int irow = 2 * u.m + half;  // query block of this row
      const bool row_valid = irow < p.nb;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int s = 0; s <= u.m; ++s) {
        const int j = 2 * s + jo;  // key block of these columns
        if (!mbar_wait(&C.s_full[sb], sph, abort_p, p.status, tmo)) { ok = false; break; }
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(lane_addr + (uint32_t)sb * 128u, r);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.s_free[sb]);
        if (++sb == kSBuf) {
          sb = 0;
          sph ^= 1;
        }
        if (j > irow || !row_valid) continue;  // key block entirely in the future
        float x[32];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          f32x2_unpack(mul_f32x2(f32x2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1])), c2),
                       x[2 * q], x[2 * q + 1]);
        if (j == irow) {
#pragma unroll
          for (int q = 0; q < 32; ++q) x[q] = hh * 32 + q > rloc ? -INFINITY : x[q];
        }
        float t[11];
#pragma unroll
        for (int q = 0; q < 10; ++q) t[q] = fmax3(x[3 * q], x[3 * q + 1], x[3 * q + 2]);
        t[10] = fmaxf(x[30], x[31]);
        const float mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]),
                               fmax3(fmax3(t[6], t[7], t[8]), t[9], t[10]));
        rslot[((long long)j * 2 + hh) * 128 + row] = mx;
        if (mx > m_run + kRaise) {
          l_run *= ex2_approx(m_run - mx);
          m_run = mx;
        }
        const uint64_t nm2 = f32x2_pack(-m_run, -m_run);
        uint64_t acc = 0ull;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float a, b;
          f32x2_unpack(add_f32x2(f32x2_pack(x[2 * q], x[2 * q + 1]), nm2), a, b);
          acc = add_f32x2(acc, f32x2_pack(ex2_approx(a), ex2_approx(b)));
        }
        float s0, s1;
        f32x2_unpack(acc, s0, s1);
        l_run += s0 + s1;
      }
      if (!ok) break;
      // ---- combine the four warpgroups' statistics into the row's lse (log2)
      C.m_part[wgi][row] = m_run;
      C.l_part[wgi][row] = l_run;
      if (!all.sync(lane)) break;
      float lse2;
      {
        float mm = C.m_part[0][row];
#pragma unroll
        for (int k = 1; k < kWG; ++k) mm = fmaxf(mm, C.m_part[k][row]);
        float l = 0.f;
#pragma unroll
        for (int k = 0; k < kWG; ++k) {
          const float mk = C.m_part[k][row];
          if (mk > -INFINITY) l += C.l_part[k][row] * ex2_approx(mk - mm);
        }
        lse2 = mm + log2f(l);
      }
      if (wgi == 0 && row_valid && p.lse)
        p.lse[((long long)u.b * p.Hq + u.hq) * p.n + (long long)irow * 64 + rloc] = lse2 * 0.6931471805599453f;
      // ---- second pass: probabilities of the kept maxima, max over rows ----
      // warpgroup wgi takes key blocks j = wgi, wgi + 4, ... of the unit
      const int nkb = 2 * (u.m + 1);
      for (int t0 = 0; 4 * t0 < nkb && ok; t0 += 32) {
        float v[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int j = 4 * (t0 + k) + wgi;
          v[k] = (j < nkb && j <= irow && row_valid)
                     ? ex2_approx(fmaxf(rslot[((long long)j * 2) * 128 + row], rslot[((long long)j * 2 + 1) * 128 + row]) -
                                  lse2)
                     : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const bool up = lane & 16;
          const float send = up ? v[k] : v[k + 16], keep = up ? v[k + 16] : v[k];
          v[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const bool up = lane & 8;
          const float send = up ? v[k] : v[k + 8], keep = up ? v[k + 8] : v[k];
          v[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 8));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const bool up = lane & 4;
          const float send = up ? v[k] : v[k + 4], keep = up ? v[k + 4] : v[k];
          v[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const bool up = lane & 2;
          const float send = up ? v[k] : v[k + 2], keep = up ? v[k + 2] : v[k];
          v[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 2));
        }
        {
          const bool up = lane & 1;
          const float send = up ? v[0] : v[1], keep = up ? v[1] : v[0];
          v[0] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 1));
        }
        // lane holds the max over this warp's 32 rows for key block 4(t0 + lane) + wgi
        C.red[wgi][ww][lane] = v[0];
        if (!wgs.sync(lane)) { ok = false; break; }
        if (ww == 0 || ww == 2) {
          const int hb = ww >> 1;  // 0: block i0 (warps 0,1), 1: block i1 (warps 2,3)
          const int ib = 2 * u.m + hb;
          const int j = 4 * (t0 + lane) + wgi;
          if (ib < p.nb && j < nkb && j <= ib) {
            const float val = fmaxf(C.red[wgi][ww][lane], C.red[wgi][ww + 1][lane]);
            p.map[(((long long)u.b * p.Hq + u.hq) * p.nb + ib) * p.nb + j] = val;
          }
        }
        if (!wgs.sync(lane)) { ok = false; break; }
      }
      if (!ok) break;
      // keep the statistics area until every warpgroup has read it
      if (!all.sync(lane)) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == bmax::kWarpMma) tmem_dealloc(tmem, bmax::kTmemCols);
}

cudaError_t launch_blockmax(const CUtensorMap& tmQ, const CUtensorMap& tmK, const BmaxParams& p,
                            int ctas, cudaStream_t st) {
  auto kern = p.d == 64 ? blockmax_kernel<64> : blockmax_kernel<128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bmax::kSmemAlloc);
  if (e != cudaSuccess) return e;
  // entries above the diagonal are 0; the kernel writes j <= i only
  e = cudaMemsetAsync(p.map, 0, sizeof(float) * (size_t)p.B * p.Hq * p.nb * p.nb, st);
  if (e != cudaSuccess) return e;
  long long grid = p.total_units < ctas ? p.total_units : ctas;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, bmax::kThreads, bmax::kSmemAlloc, st>>>(tmQ, tmK, p);
  return cudaGetLastError();
}

}  // namespace seer
