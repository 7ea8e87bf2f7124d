// fwd.cu -- dense causal attention forward that also forms the 2D-max-pooled
// probability map in the same pass (the gate's training forward), for
// sm_100a (B200).
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4, "The customized training kernel"
// (Figure 10): a FlashAttention forward that also keeps, for every row, the
// raw score maximum of each key block, and rescales those maxima with the
// row's final log-sum-exp into probabilities; "Ground truth generation":
// gt = MaxPool2D_{BxB}(softmax(Q K^T / sqrt(d))).
//
// B200 design:
//  * A unit is one query head and two consecutive 64-row query blocks
//    (2m, 2m+1): a 128-row tile.  Under the dense causal mask the two blocks
//    share every key block up to the first one's diagonal, so the tile walks
//    the key pairs s = 0..m and every MMA has M = 128 query rows: QK with
//    N = 128 keys, PV with N = d.
//  * Query-major products: S = Q K^T from 128-byte-swizzled shared memory
//    into tensor memory (TMEM, three buffers); the softmax writes P as bf16
//    back into the same TMEM buffer (tcgen05.st), and O += P V takes P
//    straight from TMEM as the A operand, V from shared memory.  P never
//    passes through shared memory.
//  * Softmax: four warpgroups share a step, warpgroup w the 32 keys
//    32w..32w+31 of the pair; every thread owns one query row (its TMEM
//    lane), so row statistics need no cross-thread reduction within a step.
//    The row maximum is fixed at the unit's first step (the exact maximum of
//    that pair, combined across the four warpgroups once): P of every step
//    is relative to it and O accumulates in TMEM without rescaling.  A score
//    more than 2^64 above it flags the unit; the exact fallback kernel then
//    recomputes it.  Below that bound nothing overflows (P <= 2^64 in bf16,
//    row sums and O in fp32).
//  * The map: each thread stores its row's raw score maximum per half key
//    block to a per-CTA scratch slot; at the unit's end they become
//    probabilities with the row's log-sum-exp, and each warpgroup takes the
//    maximum over the 64 rows of each query block for every fourth key
//    block (a shuffle reduce-scatter).
//  * Warp roles (640 threads): warps 0..15 softmax, warp 16 schedules units
//    and loads Q and K, warp 17 issues PV and owns TMEM, warp 18 issues QK,
//    warp 19 loads V.  Each MMA warp waits once per step.  Bulk copies use
//    no cluster multicast.  Every wait is bounded.
#include <cstdint>

#include "common.cuh"
#include "fwd.cuh"
#include "ptx.cuh"

namespace seer {

namespace fwd {
constexpr int kThreads = 640;
constexpr int kWarpLoadK = 16, kWarpPV = 17, kWarpQK = 18, kWarpLoadV = 19;
constexpr int kWG = 4;
constexpr int kSoftmaxWarps = 4 * kWG;
constexpr int kUnitReaders = 3 + kSoftmaxWarps;  // V loader, both MMA warps, softmax warps
constexpr uint32_t kTile = 32768;                // 128 rows x 128 dims bf16 (two 64-dim panels)
constexpr uint32_t kOffQ = 0;                    // 2 slots
constexpr uint32_t kOffK = 2 * kTile;            // 2 slots
constexpr uint32_t kOffV = 4 * kTile;            // 2 slots
constexpr uint32_t kSmemTiles = 6 * kTile;       // 192 KB
constexpr int kRing = 4;                         // step barriers
constexpr int kSBuf = 3;                         // S / P buffers in TMEM (128 columns each)
constexpr int kUnits = 4;                        // unit ring
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = kSBuf * 128;
constexpr float kFlagThreshold = 64.0f;
static_assert(kSBuf < kRing, "kfull(g) takes PV(g - kSBuf)'s completion");

struct Ctrl {
  uint64_t unit_full[kUnits], unit_empty[kUnits];
  uint64_t kfull[kRing];   // K(g) [+ the unit's Q] landed and PV(g-3) complete: the QK warp's one wait per step
  uint64_t s_full[kRing];  // QK(g) complete: S(g) readable, K slot of g free
  uint64_t go[kRing];      // V(g) landed and every softmax warp wrote its P(g): the PV warp's one wait per step
  uint64_t v_free[kRing];  // PV(g) complete: V slot of g free
  uint64_t q_free[2];      // the unit's last QK complete: its Q slot free
  uint64_t o_full;         // the unit's last PV complete: O readable
  uint64_t fin_qk, fin_pv;
  int unit_w[kUnits];
  uint32_t tmem_base;
  int abort_flag;
  int redo_unit;
  // teardown accounting after an abort
  int armed_k, armed_v, pv_steps;
  int sm_steps[kSoftmaxWarps];
  float m_part[kWG][128];
  float l_part[kWG][128];
  float red[kWG][4][32];
};
constexpr uint32_t kSmemAlloc = kSmemTiles + (uint32_t)sizeof(Ctrl);
static_assert(kSmemAlloc <= 232448, "dynamic shared memory above the per-CTA limit");
}  // namespace fwd

namespace {

struct FUnit {
  int b, hq, g, m;
};

// Unit w: KV-head-major, the longest units (last query pairs) first.
__device__ __forceinline__ FUnit fwd_decode(const FwdParams& p, int w) {
  FUnit u;
  const int per_bg = p.npairs * p.G;
  const int bg = w / per_bg, rem = w % per_bg;
  u.b = bg / p.Hkv;
  u.g = bg % p.Hkv;
  u.m = p.npairs - 1 - rem / p.G;
  u.hq = u.g * p.G + rem % p.G;
  return u;
}

__device__ __forceinline__ bool fwd_wait_teardown(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000u))
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  return true;
}

// Reads one unit ring entry (bounded); -2 when the wait gave up.
__device__ __forceinline__ int read_unit(fwd::Ctrl& C, int ur, volatile int* abort_p, const FwdParams& p) {
  const int slot = ur % fwd::kUnits;
  if (!mbar_wait(&C.unit_full[slot], (ur / fwd::kUnits) & 1, abort_p, p.status, p.timeout_ns)) return -2;
  return C.unit_w[slot];
}

}  // namespace

template <int D, bool MAP>
__global__ void __launch_bounds__(fwd::kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using namespace fwd;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (p.run_if && ((*p.run_if != 0u) != (p.run_if_value != 0u))) return;  // the sparse kernel takes this call
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(p.status, kDevBadSchedule, smem_u32(smem));
    return;
  }
  Ctrl& C = *reinterpret_cast<Ctrl*>(smem + kSmemTiles);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  volatile int* abort_p = &C.abort_flag;
  const uint64_t tmo = p.timeout_ns;
  constexpr uint32_t tile_bytes = 128u * D * 2u;

  if (threadIdx.x == 0) {
    C.abort_flag = 0;
    C.redo_unit = -1;
    C.armed_k = C.armed_v = C.pv_steps = 0;
    for (int s = 0; s < kUnits; ++s) {
      mbar_init(&C.unit_full[s], 1);
      mbar_init(&C.unit_empty[s], kUnitReaders);
    }
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&C.kfull[s], 2);  // the K loader's copies + PV(g-3)'s completion
      mbar_init(&C.s_full[s], 1);
      mbar_init(&C.go[s], 1 + kSoftmaxWarps);
      mbar_init(&C.v_free[s], 1);
    }
    // the first kSBuf steps' S buffers are free from the start
    for (int s = 0; s < kSBuf; ++s) mbar_arrive(&C.kfull[s]);
    for (int s = 0; s < 2; ++s) mbar_init(&C.q_free[s], 1);
    mbar_init(&C.o_full, 1);
    mbar_init(&C.fin_qk, 1);
    mbar_init(&C.fin_pv, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < kSoftmaxWarps) C.sm_steps[threadIdx.x] = 0;
  if (warp == kWarpPV) {
    tmem_alloc(&C.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;

  if (warp == kWarpLoadK) {
    // --------------------------------------- scheduler, Q and K loads ----
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      int u_idx = 0, g = 0;
      bool ok = true;
      while (ok) {
        const int slot = u_idx % kUnits;
        if (u_idx >= kUnits &&
            !mbar_wait(&C.unit_empty[slot], ((u_idx / kUnits) - 1) & 1, abort_p, p.status, tmo))
          break;
        int w = (int)atomicAdd(p.work_counter, 1u);
        if (w >= p.total_units || *abort_p) w = -1;
        C.unit_w[slot] = w;
        mbar_arrive(&C.unit_full[slot]);
        if (w < 0) break;  // the end marker is never released: nothing reuses its slot
        const int qs = u_idx & 1;
        if (u_idx >= 2 && !mbar_wait(&C.q_free[qs], ((u_idx >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        ++u_idx;
        const FUnit u = fwd_decode(p, w);
        const int qrow = (int)(((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.m * 128);
        const int krow0 = (int)(((long long)u.b * p.Hkv + u.g) * p.n);
        for (int s = 0; s <= u.m; ++s) {
          // K slot of g free once QK(g-2) is complete
          if (g >= 2 && !mbar_wait(&C.s_full[(g - 2) % kRing], ((g - 2) / kRing) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          uint64_t* kf = &C.kfull[g % kRing];
          mbar_arrive_expect_tx(kf, tile_bytes * (s == 0 ? 2u : 1u));
          if (s == 0) tma_load_3d(smem + kOffQ + qs * kTile, &tmQ, kf, 0, qrow, 0);
          tma_load_3d(smem + kOffK + (g & 1) * kTile, &tmK, kf, 0, krow0 + s * 128, 0);
          ++g;
        }
      }
      C.armed_k = g;
    }
  } else if (warp == kWarpLoadV) {
    // -------------------------------------------------------- V loads ----
    if (lane == 0) {
      prefetch_tmap(&tmV);
      int ur = 0, g = 0;
      bool ok = true;
      while (ok) {
        const int w = read_unit(C, ur, abort_p, p);
        if (w < 0) break;
        mbar_arrive(&C.unit_empty[ur % kUnits]);
        ++ur;
        const FUnit u = fwd_decode(p, w);
        const int vrow0 = (int)(((long long)u.b * p.Hkv + u.g) * p.n);
        for (int s = 0; s <= u.m; ++s) {
          // V slot of g free once PV(g-2) is complete
          if (g >= 2 && !mbar_wait(&C.v_free[(g - 2) % kRing], ((g - 2) / kRing) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          uint64_t* gb = &C.go[g % kRing];
          mbar_arrive_expect_tx(gb, tile_bytes);
          tma_load_3d(smem + kOffV + (g & 1) * kTile, &tmV, gb, 0, vrow0 + s * 128, 0);
          ++g;
        }
      }
      C.armed_v = g;
    }
  } else if (warp == kWarpQK) {
    // ------------------------------------------------------ QK issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);  // Q and K both K-major
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dQ0 = make_sw128_desc(sbase + kOffQ, 16, 1024);
      const uint64_t dK0 = make_sw128_desc(sbase + kOffK, 16, 1024);
      int ur = 0, g = 0;
      for (;;) {
        const int w = read_unit(C, ur, abort_p, p);
        if (w < 0) break;
        mbar_arrive(&C.unit_empty[ur % kUnits]);
        const int qs = ur & 1;
        ++ur;
        const FUnit u = fwd_decode(p, w);
        const uint64_t dq = dQ0 + ((uint64_t)(qs * kTile) >> 4);
        bool ok = true;
        for (int s = 0; s <= u.m; ++s) {
          if (!mbar_wait(&C.kfull[g % kRing], (g / kRing) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = dK0 + ((uint64_t)((g & 1) * kTile) >> 4);
          const uint32_t sc = tmem + (uint32_t)(g % kSBuf) * 128u;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_bf16_ss(sc, dq + off, dk + off, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&C.s_full[g % kRing]);
          if (s == u.m) mma_commit(&C.q_free[qs]);
          ++g;
        }
        if (!ok) break;
      }
      mma_commit(&C.fin_qk);
      fwd_wait_teardown(&C.fin_qk, 0, 20000000ull);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------ PV issuer ----
    if (lane == 0) {
      // A = P from TMEM (rows = lanes), B = V tile [128 keys x d], MN-major:
      // 64-dim panels 16 KB apart (LBO), 8-key groups 1 KB apart (SBO)
      constexpr uint32_t idesc = make_idesc_bf16(128, D, 0, 1);
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dV0 = make_sw128_desc(sbase + kOffV, 16384, 1024);
      int ur = 0, g = 0;
      for (;;) {
        const int w = read_unit(C, ur, abort_p, p);
        if (w < 0) break;
        mbar_arrive(&C.unit_empty[ur % kUnits]);
        ++ur;
        const FUnit u = fwd_decode(p, w);
        bool ok = true;
        for (int s = 0; s <= u.m; ++s) {
          if (!mbar_wait(&C.go[g % kRing], (g / kRing) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dv = dV0 + ((uint64_t)((g & 1) * kTile) >> 4);
          const uint32_t pa = tmem + (uint32_t)(g % kSBuf) * 128u;
          // key slice kk (16 keys) is warpgroup kk/2's P, columns 8 (kk % 2) on
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + kColO, pa + (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1)),
                        dv + (uint64_t)((kk * 2048) >> 4), idesc, (s > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&C.v_free[g % kRing]);
          mma_commit(&C.kfull[(g + kSBuf) % kRing]);  // S / P buffer of g free for QK(g+3)
          if (s == u.m) mma_commit(&C.o_full);
          ++g;
        }
        if (!ok) break;
      }
      C.pv_steps = g;
      mma_commit(&C.fin_pv);
      fwd_wait_teardown(&C.fin_pv, 0, 20000000ull);
    }
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------- softmax WGs ---
    // Named barriers: 1 joins all 512 softmax threads, 2 + w warpgroup w.
    // They have no timeout, so every thread reaches each of them; a failed
    // wait is ORed into the next one and the threads leave together.
    const int wgi = warp >> 2;       // keys 32*wgi .. of each pair
    const int ww = warp & 3;         // TMEM sub-partition
    const int row = ww * 32 + lane;  // query row of the tile
    const int half = row >> 6;
    const uint32_t lane_addr = tmem + ((uint32_t)(ww * 32) << 16);
    const float c = p.scale_log2;
    const uint64_t c2 = f32x2_pack(c, c);
    float* const rslot = MAP ? p.r + (long long)blockIdx.x * 256 * p.nb : nullptr;
    int ur = 0, g = 0, arrived = 0;
    bool dead = false;  // after a failed wait: no more barrier arrivals
    for (;;) {
      const int w = read_unit(C, ur, abort_p, p);
      if (bar_red_or(1, 512, w == -2 || dead)) break;
      if (w < 0) break;  // the end marker is never released
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.unit_empty[ur % kUnits]);
      ++ur;
      const FUnit u = fwd_decode(p, w);
      const int irow = 2 * u.m + half;  // query block of this row
      const bool row_valid = irow < p.nb;
      const int qpos = u.m * 128 + row;  // query position in the head
      float m0 = 0.f;
      uint64_t l2 = 0ull;  // row-sum partial, packed pair
      bool fail = false;
      for (int s = 0; s <= u.m; ++s, ++g) {
        const int sb = g % kSBuf;
        const bool okS = mbar_wait(&C.s_full[g % kRing], (g / kRing) & 1, abort_p, p.status, tmo);
        dead = dead || __any_sync(0xffffffffu, !okS);
        tc_fence_after();
        const uint32_t saddr = lane_addr + (uint32_t)sb * 128u + (uint32_t)(32 * wgi);
        uint32_t r[32];
        if (!dead) {
          tmem_ld32(saddr, r);
          tmem_wait_ld();
        }
        float x[32];
#pragma unroll
        for (int q = 0; q < 16; ++q)
          f32x2_unpack(mul_f32x2(f32x2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1])), c2),
                       x[2 * q], x[2 * q + 1]);
        const int kbase = s * 128 + 32 * wgi;  // key position of column 0
        if (!row_valid) {
#pragma unroll
          for (int q = 0; q < 32; ++q) x[q] = -INFINITY;
        } else if (kbase + 31 > qpos) {
#pragma unroll
          for (int q = 0; q < 32; ++q) x[q] = kbase + q > qpos ? -INFINITY : x[q];
        }
        float t[11];
#pragma unroll
        for (int q = 0; q < 10; ++q) t[q] = fmax3(x[3 * q], x[3 * q + 1], x[3 * q + 2]);
        t[10] = fmaxf(x[30], x[31]);
        const float mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]),
                               fmax3(fmax3(t[6], t[7], t[8]), t[9], t[10]));
        if constexpr (MAP) {
          const int j = 2 * s + (wgi >> 1);
          if (row_valid && j <= irow) rslot[((long long)j * 2 + (wgi & 1)) * 128 + row] = mx;
        }
        if (s == 0) {
          // the row's fixed maximum: the exact maximum of the unit's first pair
          C.m_part[wgi][row] = mx;
          if (bar_red_or(1, 512, dead)) {
            fail = true;
            break;
          }
          m0 = fmaxf(fmaxf(C.m_part[0][row], C.m_part[1][row]), fmaxf(C.m_part[2][row], C.m_part[3][row]));
          if (m0 == -INFINITY) m0 = 0.f;  // a row past the sequence: every P is 0
        }
        // far above the fixed maximum: the unit goes to the exact fallback
        if (__any_sync(0xffffffffu, mx - m0 > kFlagThreshold) && !dead && lane == 0 &&
            atomicExch(&C.redo_unit, w) != w) {
          for (int hb = 0; hb < 2; ++hb) {
            const int i = 2 * u.m + hb;
            if (i >= p.nb) continue;
            const int bg = u.b * p.Hkv + u.g;
            const int w64 = (bg * p.nb + (p.nb - 1 - i)) * p.G + (u.hq - u.g * p.G);
            const uint32_t e = atomicAdd(p.redo_count, 1u);
            if (e < (uint32_t)p.redo_cap) p.redo_list[e] = w64;
          }
        }
        const uint64_t nm2 = f32x2_pack(-m0, -m0);
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float a, b;
          f32x2_unpack(add_f32x2(f32x2_pack(x[2 * q], x[2 * q + 1]), nm2), a, b);
          a = ex2_approx(a);
          b = ex2_approx(b);
          l2 = add_f32x2(l2, f32x2_pack(a, b));
          pk[q] = pack_bf16x2(a, b);
        }
        if (!dead) {
          tmem_st16(saddr, pk);
          tmem_wait_st();
        }
        tc_fence_before();
        if (!dead) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&C.go[g % kRing]);
          ++arrived;
        }
      }
      if (fail) break;
      // ------------------------------------------------------ epilogue ---
      const bool okO = mbar_wait(&C.o_full, (ur - 1) & 1, abort_p, p.status, tmo);
      dead = dead || __any_sync(0xffffffffu, !okO);
      float la, lb;
      f32x2_unpack(l2, la, lb);
      C.l_part[wgi][row] = la + lb;
      if (bar_red_or(1, 512, dead)) break;
      const float ltot = (C.l_part[0][row] + C.l_part[1][row]) + (C.l_part[2][row] + C.l_part[3][row]);
      const float lse2 = m0 + lg2_approx(ltot);
      const long long orow = ((long long)u.b * p.Hq + u.hq) * p.n + qpos;
      if (wgi == 0 && row_valid && p.lse) p.lse[orow] = lse2 * 0.6931471805599453f;
      tc_fence_after();
      {
        constexpr int NC = D / 4;  // this warpgroup's output columns
        uint32_t o[32];
        if (NC == 32)
          tmem_ld32(lane_addr + kColO + (uint32_t)(NC * wgi), o);
        else
          tmem_ld16(lane_addr + kColO + (uint32_t)(NC * wgi), *reinterpret_cast<uint32_t(*)[16]>(o));
        tmem_wait_ld();
        if (row_valid) {
          const float inv = rcp_approx(ltot);  // ltot >= 1: the maximum's own term
          if (p.out_fp32) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.O) + orow * D + NC * wgi);
#pragma unroll
            for (int q = 0; q < NC; q += 4)
              dst[q / 4] = make_float4(__uint_as_float(o[q]) * inv, __uint_as_float(o[q + 1]) * inv,
                                       __uint_as_float(o[q + 2]) * inv, __uint_as_float(o[q + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.O) + orow * D + NC * wgi);
#pragma unroll
            for (int q = 0; q < NC; q += 8)
              dst[q / 8] = make_uint4(pack_bf16x2(__uint_as_float(o[q]) * inv, __uint_as_float(o[q + 1]) * inv),
                                      pack_bf16x2(__uint_as_float(o[q + 2]) * inv, __uint_as_float(o[q + 3]) * inv),
                                      pack_bf16x2(__uint_as_float(o[q + 4]) * inv, __uint_as_float(o[q + 5]) * inv),
                                      pack_bf16x2(__uint_as_float(o[q + 6]) * inv, __uint_as_float(o[q + 7]) * inv));
          }
        }
      }
      tc_fence_before();
      if constexpr (MAP) {
        // second pass: probabilities of the kept maxima, max over the rows of
        // each query block; warpgroup wgi takes key blocks wgi, wgi + 4, ...
        const int nkb = 2 * (u.m + 1);
        bool mfail = false;
        for (int t0 = 0; 4 * t0 < nkb; t0 += 32) {
          float v[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int j = 4 * (t0 + k) + wgi;
            v[k] = (j < nkb && j <= irow && row_valid)
                       ? ex2_approx(fmaxf(rslot[((long long)j * 2) * 128 + row],
                                          rslot[((long long)j * 2 + 1) * 128 + row]) - lse2)
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
          // lane: the max over this warp's 32 rows for key block 4(t0 + lane) + wgi
          C.red[wgi][ww][lane] = v[0];
          named_barrier_sync(2 + wgi, 128);
          if (ww == 0 || ww == 2) {
            const int ib = 2 * u.m + (ww >> 1);  // warps 0,1: block 2m; warps 2,3: block 2m+1
            const int j = 4 * (t0 + lane) + wgi;
            if (ib < p.nb && j < nkb && j <= ib)
              p.map[(((long long)u.b * p.Hq + u.hq) * p.nb + ib) * p.nb + j] =
                  fmaxf(C.red[wgi][ww][lane], C.red[wgi][ww + 1][lane]);
          }
          named_barrier_sync(2 + wgi, 128);
        }
        (void)mfail;
      }
    }
    if (lane == 0) C.sm_steps[warp] = arrived;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpPV) tmem_dealloc(tmem, kTmemCols);
  // After an abort, bulk copies may still be in flight.  Every warp has left
  // its loop, so each open phase's missing arrivals are known: kfull(g)
  // lacks PV(g-3)'s completion if PV stopped before g-3, go(g) lacks the P
  // arrivals of the softmax warps that stopped before g.  Make them; each
  // armed phase then completes exactly when its copies have landed.  A
  // loader arms step g only after step g-2's slot was released, so only the
  // last two phases of each can be open.
  if (threadIdx.x == 0 && *abort_p) {
    for (int g = C.armed_k - 2 > 0 ? C.armed_k - 2 : 0; g < C.armed_k; ++g) {
      if (g >= kSBuf && C.pv_steps <= g - kSBuf) mbar_arrive(&C.kfull[g % kRing]);
      fwd_wait_teardown(&C.kfull[g % kRing], (g / kRing) & 1, 20000000ull);
    }
    for (int g = C.armed_v - 2 > 0 ? C.armed_v - 2 : 0; g < C.armed_v; ++g) {
      for (int w2 = 0; w2 < kSoftmaxWarps; ++w2)
        if (C.sm_steps[w2] <= g) mbar_arrive(&C.go[g % kRing]);
      fwd_wait_teardown(&C.go[g % kRing], (g / kRing) & 1, 20000000ull);
    }
  }
}

cudaError_t launch_fwd(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const FwdParams& p,
                       int ctas, cudaStream_t st) {
  auto kern = p.map ? (p.d == 64 ? fwd_kernel<64, true> : fwd_kernel<128, true>)
                    : (p.d == 64 ? fwd_kernel<64, false> : fwd_kernel<128, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fwd::kSmemAlloc);
  if (e != cudaSuccess) return e;
  long long grid = p.total_units < ctas ? p.total_units : ctas;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, fwd::kThreads, fwd::kSmemAlloc, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace seer
