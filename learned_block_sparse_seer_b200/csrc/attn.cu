// attn.cu -- block-sparse causal attention forward for sm_100a (B200).
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4, "Block-sparse FlashAttention
// kernel": tiles are aligned with the gate's 64-token blocks; an inactive
// block costs no QK^T, no softmax, no PV and no K/V load; an active block is
// an ordinary online-softmax attention step.
//
// B200 design (not the pages' FlashAttention-2 kernel):
//  * A "unit" is one query head hq and one 64-row query block i.  Its active
//    key blocks are walked two at a time.  The products are formed
//    TRANSPOSED so that both tcgen05 MMAs have M = 128 rows without pairing
//    unrelated units:
//        S^T[128 keys x 64 queries]   = Kpair[128 x d]  . Q_i^T        (QK)
//        O^T[d x 64 queries]         += V_pair^T[d x 128] . P^T        (PV)
//    S^T and O^T live in tensor memory (TMEM); K/V/Q/P^T are 128-byte
//    swizzled shared-memory tiles.  K and V tiles are gathered by index with
//    TMA (no cluster multicast).
//  * Warp roles (256 threads): warp 0 schedules units and loads Q; warp 1
//    loads K pairs; warp 2 loads V pairs; warp 3 issues all MMAs from one
//    thread; warps 4..7 do the softmax, one key (TMEM lane) per thread.
//  * Online softmax with a lazily updated running maximum per query column:
//    the exact column maximum is formed on a unit's first step; afterwards a
//    warpgroup vote re-forms it only when some score exceeds the running
//    maximum by more than 2^8 (log2 domain), rescaling the row sums and O^T.
//  * Units are handed out by an atomic counter in KV-head-major order, query
//    blocks from the last (longest lists) to the first, so the K/V of one KV
//    head stay hot in L2 while its query heads are processed.
//  * Every mbarrier wait is bounded (%globaltimer); on expiry the kernel
//    records a timeout in the workspace status word and unwinds.
#include <cstdint>

#include "attn.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace seer {

namespace attn {
constexpr int kThreads = 256;
constexpr int kNK = 3;  // K-pair ring stages (32 KB each)
constexpr int kNV = 2;  // V-pair ring stages (32 KB each)
constexpr uint32_t kQBytes = 16384, kPairBytes = 32768, kPBytes = 16384;
constexpr uint32_t kOffQ = 0;                                  // 2 x 16 KB
constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;                // kNK x 32 KB
constexpr uint32_t kOffV = kOffK + kNK * kPairBytes;           // kNV x 32 KB
constexpr uint32_t kOffP = kOffV + kNV * kPairBytes;           // 2 x 16 KB
constexpr uint32_t kSmemBytes = kOffP + 2 * kPBytes;           // 224 KB of tiles
constexpr uint32_t kTmemCols = 256;  // S^T x 2 (64 cols each) + O^T (64 cols)
constexpr uint32_t kColS0 = 0, kColO = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t unit_full[2], unit_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t v_full[kNV], v_empty[kNV];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_free, fin, wg;
};
// Control block, placed in dynamic shared memory right after the tiles (the
// tiles need the whole 227 KB budget, so nothing is static).
struct Ctrl {
  Bars bars;
  int unit_w[2];
  uint32_t tmem_base;
  int abort_flag;
  int vote[2][4];
  float red[4 * 64];
  float m_sh[64], tmp_sh[64], l_sh[64];
};
constexpr uint32_t kSmemAlloc = kSmemBytes + (uint32_t)sizeof(Ctrl);
}  // namespace attn

struct UnitInfo {
  int b, hq, g, i, count;
  long long u;  // (b*Hq + hq)*nb + i
};

__device__ __forceinline__ UnitInfo decode_unit(const AttnParams& p, int w) {
  UnitInfo r;
  const int per_bg = p.nb * p.G;
  const int bg = w / per_bg, rem = w % per_bg;
  r.b = bg / p.Hkv;
  r.g = bg % p.Hkv;
  r.i = p.nb - 1 - rem / p.G;
  r.hq = r.g * p.G + rem % p.G;
  r.u = ((long long)r.b * p.Hq + r.hq) * p.nb + r.i;
  int c = p.counts[r.u];
  int lim = min(p.cap, r.i + 1);
  if (c < 0 || c > lim) {
    record_status(p.status, kDevBadIndex, (uint32_t)r.u);
    c = c < 0 ? 0 : lim;
  }
  r.count = c;
  return r;
}

// Entry m of a unit's list, checked: it must satisfy 0 <= j <= i and be larger
// than the previous entry.  A failing entry is recorded and replaced by a safe
// in-range block so that no load leaves the tensor.
__device__ __forceinline__ int list_entry(const AttnParams& p, const UnitInfo& u, int m) {
  int j = p.indices[u.u * p.cap + m];
  int prev = m > 0 ? p.indices[u.u * p.cap + m - 1] : -1;
  if (j < 0 || j > u.i || j <= prev) {
    record_status(p.status, kDevBadIndex, (uint32_t)u.u);
    j = j < 0 ? 0 : (j > u.i ? u.i : j);
  }
  return j;
}

// Warpgroup barrier of the 4 softmax warps built on an mbarrier (count 4),
// so that it can give up: bar.sync has no timeout.  `phase` counts the syncs
// this thread has done; every thread of the warpgroup performs the same
// sequence.  Returns false when the wait gave up.
struct WgSync {
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

// Column-wise (per query) max over the 128 keys held one per thread by the
// softmax warpgroup.  x[64] is destroyed.  Result goes to out[64] in smem.
__device__ __forceinline__ bool wg_colmax(float (&x)[64], float* red /*[4][64]*/, float* out,
                                          int wg_warp, int lane, int tl, WgSync& ws) {
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const bool up = lane & 16;
    const float send = up ? x[k] : x[k + 32], keep = up ? x[k + 32] : x[k];
    x[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const bool up = lane & 8;
    const float send = up ? x[k] : x[k + 16], keep = up ? x[k + 16] : x[k];
    x[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool up = lane & 4;
    const float send = up ? x[k] : x[k + 8], keep = up ? x[k + 8] : x[k];
    x[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool up = lane & 2;
    const float send = up ? x[k] : x[k + 4], keep = up ? x[k + 4] : x[k];
    x[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool up = lane & 1;
    const float send = up ? x[k] : x[k + 2], keep = up ? x[k + 2] : x[k];
    x[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 1));
  }
  // lane now holds columns 2*lane and 2*lane+1
  red[wg_warp * 64 + 2 * lane] = x[0];
  red[wg_warp * 64 + 2 * lane + 1] = x[1];
  if (!ws.sync(lane)) return false;
  if (tl < 64)
    out[tl] = fmaxf(fmaxf(red[tl], red[64 + tl]), fmaxf(red[128 + tl], red[192 + tl]));
  return ws.sync(lane);
}

// Same reduction with a sum (row sums l of the softmax), destroying x.
__device__ __forceinline__ bool wg_colsum(float (&x)[64], float* red, float* out, int wg_warp,
                                          int lane, int tl, WgSync& ws) {
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const bool up = lane & 16;
    const float send = up ? x[k] : x[k + 32], keep = up ? x[k + 32] : x[k];
    x[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const bool up = lane & 8;
    const float send = up ? x[k] : x[k + 16], keep = up ? x[k + 16] : x[k];
    x[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool up = lane & 4;
    const float send = up ? x[k] : x[k + 8], keep = up ? x[k + 8] : x[k];
    x[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool up = lane & 2;
    const float send = up ? x[k] : x[k + 4], keep = up ? x[k + 4] : x[k];
    x[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool up = lane & 1;
    const float send = up ? x[k] : x[k + 2], keep = up ? x[k + 2] : x[k];
    x[k] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
  red[wg_warp * 64 + 2 * lane] = x[0];
  red[wg_warp * 64 + 2 * lane + 1] = x[1];
  if (!ws.sync(lane)) return false;
  if (tl < 64) out[tl] = (red[tl] + red[64 + tl]) + (red[128 + tl] + red[192 + tl]);
  return ws.sync(lane);
}

// Loads this thread's S^T row (one key, 64 query columns) from TMEM, scaled to
// the log2 domain; keys that are absent or causally masked become -inf.
__device__ __forceinline__ void load_scores(uint32_t taddr, float (&x)[64], float c, bool valid,
                                            bool diag, int kl) {
  uint32_t r0[32], r1[32];
  tmem_ld32(taddr, r0);
  tmem_ld32(taddr + 32, r1);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    x[q] = __uint_as_float(r0[q]) * c;
    x[q + 32] = __uint_as_float(r1[q]) * c;
  }
  if (!valid) {
#pragma unroll
    for (int q = 0; q < 64; ++q) x[q] = -INFINITY;
  } else if (diag) {
#pragma unroll
    for (int q = 0; q < 64; ++q) x[q] = (q < kl) ? -INFINITY : x[q];
  }
}

__global__ void __launch_bounds__(attn::kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using namespace attn;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The 128-byte-swizzled tiles need a 1024-byte aligned base.  The dynamic
  // window starts after the reserved per-CTA area, which keeps it aligned;
  // if it ever were not, refuse to run rather than compute garbage.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(p.status, kDevBadSchedule, smem_u32(smem));
    return;
  }
  Ctrl& C = *reinterpret_cast<Ctrl*>(smem + kSmemBytes);
  Bars& bars = C.bars;
  int* unit_w = C.unit_w;
  uint32_t& tmem_base_sh = C.tmem_base;
  int& abort_flag = C.abort_flag;
  float* red = C.red;
  float* m_sh = C.m_sh;
  float* tmp_sh = C.tmp_sh;
  float* l_sh = C.l_sh;
  auto& vote = C.vote;

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  volatile int* abort_p = &abort_flag;
  const uint64_t tmo = p.timeout_ns;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.unit_full[s], 1);
      mbar_init(&bars.unit_empty[s], 7);  // K, V, MMA + 4 softmax warps
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.pv_done[s], 1);
    }
    for (int s = 0; s < kNK; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
    }
    for (int s = 0; s < kNV; ++s) {
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    mbar_init(&bars.o_free, 4);
    mbar_init(&bars.fin, 1);
    mbar_init(&bars.wg, 4);
    fence_barrier_init();
  }
  if (p.d == 64) {
    // V^T rows 64..127 of the PV product read the second 64-column panel of
    // each V stage; with d = 64 nothing is loaded there, so it is zeroed once.
    for (int s = 0; s < kNV; ++s) {
      uint4* z = reinterpret_cast<uint4*>(smem + kOffV + s * kPairBytes + 16384);
      for (int e = threadIdx.x; e < 16384 / 16; e += blockDim.x) z[e] = make_uint4(0, 0, 0, 0);
    }
    fence_async_shared();
  }
  if (warp == 3) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int dpanels = p.d / 64;

  if (warp == 0) {
    // ------------------------------------------------ scheduler + Q loads --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      int u_idx = 0, qn = 0;
      for (;;) {
        const int slot = u_idx & 1;
        if (u_idx >= 2 && !mbar_wait(&bars.unit_empty[slot], ((u_idx >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        int w = (int)atomicAdd(p.work_counter, 1u);
        if (w >= p.total_units || *abort_p) w = -1;
        unit_w[slot] = w;
        mbar_arrive(&bars.unit_full[slot]);
        if (w < 0) break;
        const UnitInfo u = decode_unit(p, w);
        ++u_idx;
        if (u.count == 0) continue;
        const int qs = qn & 1;
        if (qn >= 2 && !mbar_wait(&bars.q_empty[qs], ((qn >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        mbar_arrive_expect_tx(&bars.q_full[qs], 64u * p.d * 2u);
        const int row = (int)(((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64);
        for (int pn = 0; pn < dpanels; ++pn)
          tma_load_2d(smem + kOffQ + qs * kQBytes + pn * 8192, &tmQ, &bars.q_full[qs], pn * 64, row);
        ++qn;
      }
      // wait for Q loads still in flight before the CTA may exit
      for (int k = 0; k < 2 && k < qn; ++k) {
        const int qq = qn - 1 - k;
        mbar_wait(&bars.q_full[qq & 1], (qq >> 1) & 1, abort_p, nullptr, 20000000ull);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------- K / V pair loads ---
    if (lane == 0) {
      const bool isK = warp == 1;
      const CUtensorMap* tm = isK ? &tmK : &tmV;
      prefetch_tmap(tm);
      const int NS = isK ? kNK : kNV;
      uint64_t* full = isK ? bars.k_full : bars.v_full;
      uint64_t* empty = isK ? bars.k_empty : bars.v_empty;
      const uint32_t base = isK ? kOffK : kOffV;
      int u_idx = 0, step = 0;
      bool ok = true;
      while (ok) {
        const int slot = u_idx & 1;
        if (!mbar_wait(&bars.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
        const int w = unit_w[slot];
        mbar_arrive(&bars.unit_empty[slot]);
        if (w < 0) break;
        ++u_idx;
        const UnitInfo u = decode_unit(p, w);
        const long long kvrow0 = ((long long)u.b * p.Hkv + u.g) * p.n;
        for (int m = 0; m < u.count; m += 2, ++step) {
          const int s = step % NS;
          if (step >= NS && !mbar_wait(&empty[s], ((step / NS) - 1) & 1, abort_p, p.status, tmo)) {
            ok = false;
            break;
          }
          const int ntile = (m + 1 < u.count) ? 2 : 1;
          mbar_arrive_expect_tx(&full[s], (uint32_t)ntile * 64u * p.d * 2u);
          for (int h = 0; h < ntile; ++h) {
            const int j = list_entry(p, u, m + h);
            const int row = (int)(kvrow0 + (long long)j * 64);
            for (int pn = 0; pn < dpanels; ++pn)
              tma_load_2d(smem + base + s * kPairBytes + pn * 16384 + h * 8192, tm, &full[s], pn * 64, row);
          }
        }
      }
      // wait for loads still in flight before the CTA may exit
      for (int k = 0; k < NS && k < step; ++k) {
        const int st = step - 1 - k;
        mbar_wait(&full[st % NS], (st / NS) & 1, abort_p, nullptr, 20000000ull);
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_pv = make_idesc_bf16(128, 64, 1, 1);
      const uint32_t sbase = smem_u32(smem);
      int u_idx = 0, qn = 0, step = 0, units_done = 0;
      const int ksteps_qk = p.d / 16;
      bool ok = true;
      auto issue_pv = [&](int g, bool first, bool two) -> bool {
        if (!mbar_wait(&bars.p_full[g & 1], (g >> 1) & 1, abort_p, p.status, tmo)) return false;
        if (first && units_done > 0 && !mbar_wait(&bars.o_free, (units_done - 1) & 1, abort_p, p.status, tmo)) return false;
        const int vs = g % kNV;
        if (!mbar_wait(&bars.v_full[vs], (g / kNV) & 1, abort_p, p.status, tmo)) return false;
        tc_fence_after();
        const uint32_t va = sbase + kOffV + vs * kPairBytes;
        const uint32_t pa = sbase + kOffP + (g & 1) * kPBytes;
        const int nk = two ? 8 : 4;  // 16 keys per MMA
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t adesc = make_sw128_desc(va + kk * 2048, 16384, 1024);
          const uint64_t bdesc = make_sw128_desc(pa + kk * 2048, 16384, 1024);
          mma_bf16_ss(tmem + kColO, adesc, bdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&bars.pv_done[g & 1]);
        mma_commit(&bars.v_empty[vs]);
        return true;
      };
      while (ok) {
        const int slot = u_idx & 1;
        if (!mbar_wait(&bars.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
        const int w = unit_w[slot];
        mbar_arrive(&bars.unit_empty[slot]);
        if (w < 0) break;
        ++u_idx;
        const UnitInfo u = decode_unit(p, w);
        if (u.count == 0) continue;
        const int T = (u.count + 1) / 2;
        const int qs = qn & 1;
        if (!mbar_wait(&bars.q_full[qs], (qn >> 1) & 1, abort_p, p.status, tmo)) break;
        const uint32_t qa = sbase + kOffQ + qs * kQBytes;
        for (int t = 0; t < T && ok; ++t) {
          const int g = step + t;
          const int ks = g % kNK;
          if (!mbar_wait(&bars.k_full[ks], (g / kNK) & 1, abort_p, p.status, tmo)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ka = sbase + kOffK + ks * kPairBytes;
          for (int kk = 0; kk < ksteps_qk; ++kk) {
            const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kColS0 + (g & 1) * 64, make_sw128_desc(ka + koff, 16, 1024),
                        make_sw128_desc(qa + qoff, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[g & 1]);
          mma_commit(&bars.k_empty[ks]);
          if (t == T - 1) mma_commit(&bars.q_empty[qs]);
          if (t >= 1 && !issue_pv(g - 1, t - 1 == 0, 2 * (t - 1) + 1 < u.count)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(step + T - 1, T == 1, 2 * (T - 1) + 1 < u.count)) break;
        step += T;
        ++qn;
        ++units_done;
      }
      // all MMAs complete before TMEM is released
      mma_commit(&bars.fin);
      mbar_wait(&bars.fin, 0, abort_p, nullptr, 20000000ull);
    }
  } else {
    // -------------------------------------------------------- softmax WG --
    const int wg_warp = warp - 4;              // 0..3 == TMEM sub-partition
    const int tl = wg_warp * 32 + lane;        // TMEM lane == key in pair / dim of O^T
    const uint32_t lane_addr = tmem + ((uint32_t)(wg_warp * 32) << 16);
    const float c = p.scale_log2;
    int u_idx = 0, step = 0, units_done = 0;
    WgSync ws{&bars.wg, abort_p, p.status, tmo, 0};
    float lpart[64];
    for (;;) {
      const int slot = u_idx & 1;
      if (!mbar_wait(&bars.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
      const int w = unit_w[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.unit_empty[slot]);
      if (w < 0) break;
      ++u_idx;
      const UnitInfo u = decode_unit(p, w);
      const long long orow0 = ((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64;
      if (u.count == 0) {
        if (tl < p.d) {
          for (int q = 0; q < 64; ++q) {
            if (p.out_fp32)
              reinterpret_cast<float*>(p.O)[(orow0 + q) * p.d + tl] = 0.f;
            else
              reinterpret_cast<uint16_t*>(p.O)[(orow0 + q) * p.d + tl] = 0;
          }
        }
        if (tl < 64 && p.lse) p.lse[orow0 + tl] = -INFINITY;
        continue;
      }
      const int T = (u.count + 1) / 2;
      const int half = tl >> 6, kl = tl & 63;
#pragma unroll
      for (int q = 0; q < 64; ++q) lpart[q] = 0.f;
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const int g = step + t;
        const int mi = 2 * t + half;
        const bool valid = mi < u.count;
        const int j = valid ? p.indices[u.u * p.cap + mi] : -1;
        const bool diag = valid && j == u.i;
        if (!mbar_wait(&bars.s_full[g & 1], (g >> 1) & 1, abort_p, p.status, tmo)) { ok = false; break; }
        tc_fence_after();
        const uint32_t saddr = lane_addr + kColS0 + (g & 1) * 64;
        float x[64];
        if (t == 0) {
          load_scores(saddr, x, c, valid, diag, kl);
          if (!wg_colmax(x, red, m_sh, wg_warp, lane, tl, ws)) { ok = false; break; }
          load_scores(saddr, x, c, valid, diag, kl);
#pragma unroll
          for (int q = 0; q < 64; ++q) x[q] -= m_sh[q];
        } else {
          load_scores(saddr, x, c, valid, diag, kl);
          float dmax = -INFINITY;
#pragma unroll
          for (int q = 0; q < 64; ++q) {
            x[q] -= m_sh[q];
            dmax = fmaxf(dmax, x[q]);
          }
          const int any = __any_sync(0xffffffffu, dmax > kRescaleThreshold);
          if (lane == 0) vote[g & 1][wg_warp] = any;
          if (!ws.sync(lane)) { ok = false; break; }
          const bool slow = vote[g & 1][0] | vote[g & 1][1] | vote[g & 1][2] | vote[g & 1][3];
          if (slow) {
            // exact column maxima of this step, relative to the running max
            if (!wg_colmax(x, red, tmp_sh, wg_warp, lane, tl, ws)) { ok = false; break; }
            // tmp_sh[q] = max(0, colmax) = increase of the running max
            if (tl < 64) tmp_sh[tl] = fmaxf(tmp_sh[tl], 0.f);
            if (!ws.sync(lane)) { ok = false; break; }
#pragma unroll
            for (int q = 0; q < 64; ++q) lpart[q] *= ex2_approx(-tmp_sh[q]);
            // O^T columns are rescaled once the previous PV has landed
            const int gp = g - 1;
            if (!mbar_wait(&bars.pv_done[gp & 1], (gp >> 1) & 1, abort_p, p.status, tmo)) { ok = false; break; }
            tc_fence_after();
            {
              uint32_t o0[32], o1[32];
              tmem_ld32(lane_addr + kColO, o0);
              tmem_ld32(lane_addr + kColO + 32, o1);
              tmem_wait_ld();
              uint32_t w16[16];
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                  w16[q] = __float_as_uint(__uint_as_float(o0[h2 * 16 + q]) * ex2_approx(-tmp_sh[h2 * 16 + q]));
                tmem_st16(lane_addr + kColO + h2 * 16, w16);
              }
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                  w16[q] = __float_as_uint(__uint_as_float(o1[h2 * 16 + q]) * ex2_approx(-tmp_sh[32 + h2 * 16 + q]));
                tmem_st16(lane_addr + kColO + 32 + h2 * 16, w16);
              }
              tmem_wait_st();
            }
            if (tl < 64) m_sh[tl] += tmp_sh[tl];
            if (!ws.sync(lane)) { ok = false; break; }
            load_scores(saddr, x, c, valid, diag, kl);
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] -= m_sh[q];
          }
        }
        // probabilities, row-sum partials, bf16 P^T row
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 64; q += 2) {
          const float p0 = ex2_approx(x[q]), p1 = ex2_approx(x[q + 1]);
          lpart[q] += p0;
          lpart[q + 1] += p1;
          pk[q >> 1] = pack_bf16x2(p0, p1);
        }
        if (g >= 2 && !mbar_wait(&bars.pv_done[g & 1], ((g - 2) >> 1) & 1, abort_p, p.status, tmo)) { ok = false; break; }
        uint8_t* prow = smem + kOffP + (g & 1) * kPBytes + tl * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          *reinterpret_cast<uint4*>(prow + ((ch ^ (tl & 7)) << 4)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        fence_async_shared();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[g & 1]);
      }
      if (!ok) break;
      // ------------------------------------------------------- epilogue ---
      const int gl = step + T - 1;
      if (!mbar_wait(&bars.pv_done[gl & 1], (gl >> 1) & 1, abort_p, p.status, tmo)) break;
      tc_fence_after();
      if (!wg_colsum(lpart, red, l_sh, wg_warp, lane, tl, ws)) break;
      {
        uint32_t o0[32], o1[32];
        tmem_ld32(lane_addr + kColO, o0);
        tmem_ld32(lane_addr + kColO + 32, o1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.o_free);
        if (tl < p.d) {
#pragma unroll
          for (int q = 0; q < 64; ++q) {
            const float v = __uint_as_float(q < 32 ? o0[q] : o1[q - 32]) / l_sh[q];
            const long long idx = (orow0 + q) * p.d + tl;
            if (p.out_fp32)
              reinterpret_cast<float*>(p.O)[idx] = v;
            else
              reinterpret_cast<__nv_bfloat16*>(p.O)[idx] = __float2bfloat16_rn(v);
          }
        }
      }
      if (tl < 64 && p.lse) p.lse[orow0 + tl] = (m_sh[tl] + log2f(l_sh[tl])) * 0.6931471805599453f;
      if (!ws.sync(lane)) break;
      step += T;
      ++units_done;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 3) tmem_dealloc(tmem, kTmemCols);
}

cudaError_t launch_sparse_attn(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                               const AttnParams& p, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)attn::kSmemAlloc);
  if (e != cudaSuccess) return e;
  long long grid = p.total_units < num_sms ? p.total_units : num_sms;
  if (grid < 1) grid = 1;
  sparse_attn_kernel<<<(unsigned)grid, attn::kThreads, attn::kSmemAlloc, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace seer
