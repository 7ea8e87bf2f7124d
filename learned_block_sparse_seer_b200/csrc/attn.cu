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
//    key blocks are walked two at a time ("pair steps").  The products are
//    formed TRANSPOSED so that both tcgen05 MMAs have M = 128 rows without
//    pairing unrelated units:
//        S^T[128 keys x 64 queries]   = Kpair[128 x d]  . Q_i^T        (QK)
//        O^T[d x 64 queries]         += V_pair^T[d x 128] . P^T        (PV)
//    S^T and O^T live in tensor memory (TMEM); K/V/Q/P^T are 128-byte
//    swizzled shared-memory tiles.
//  * TMA on B200 costs about the same per instruction for any box up to
//    16 KB, so a gathered tile must arrive in as few instructions as
//    possible.  A re-layout pass (kv_tile_kernel) first writes every
//    (KV head, key block) as one contiguous record [K^T: d rows x 64 keys |
//    V: 64 keys x d in 64-column panels]; one 2*d-row TMA box (32 KB at
//    d = 128, no cluster multicast) then brings both K and V of a block into
//    the ring.  The ring has 3 pair stages of two records; K^T is read by the
//    QK MMA as an MN-major operand whose two 64-key halves are the stage's
//    two records (leading-byte offset = one record).
//  * Warp roles (576 threads): warps 0..15 are four softmax warpgroups, each
//    owning 16 of the 64 query columns (its own running max, row sums, vote
//    and epilogue), one key (TMEM lane) per thread -- a warp w reaches TMEM
//    lanes 32*(w%4)..+31; warp 16 schedules units and issues every TMA load
//    (Q and the gathered records); warp 17 issues all MMAs from one thread
//    and owns the TMEM allocation.  Four warps per SMSP work on the same
//    step, so their latency chains interleave.
//  * Online softmax with a lazily updated running maximum per query column:
//    the exact column maximum is formed on a unit's first step; afterwards a
//    warpgroup vote re-forms it only when some score exceeds the running
//    maximum by more than 2^8 (log2 domain), rescaling the row sums and O^T.
//    The vote is one hardware barrier-with-reduction per step, taken after
//    the exponentials (which are recomputed in the rare rescale case).
//  * P^T of a step is written into the K^T half of its own stage (dead once
//    the step's QK MMA is done), so P is buffered as deeply as the ring.
//  * Units are handed out by an atomic counter in KV-head-major order, query
//    blocks from the last (longest lists) to the first, so the K/V of one KV
//    head stay hot in L2 while its query heads are processed.
//  * Every mbarrier wait is bounded (%globaltimer); on expiry the kernel
//    records a timeout in the workspace status word and unwinds.
#include <cstddef>
#include <cstdint>

#include "attn.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace seer {

namespace attn {
constexpr int kThreads = 576;
constexpr int kStages = 3;  // pair stages: two K^T+V records each
constexpr uint32_t kRecBytes = 32768, kStageBytes = 2 * kRecBytes;
constexpr uint32_t kQBytes = 16384;
constexpr uint32_t kOffRing = 0;                               // 3 x 64 KB
constexpr uint32_t kOffQ = kOffRing + kStages * kStageBytes;   // 2 x 16 KB
constexpr uint32_t kSmemBytes = kOffQ + 2 * kQBytes;           // 224 KB of tiles
// P^T of a pair step is written into its stage: the K^T part of record h
// (dead once the step's QK MMA has completed) takes keys 64h .. 64h+63.
constexpr uint32_t kTmemCols = 256;  // S^T x 2 (64 cols each) + O^T (64 cols)
constexpr uint32_t kColS0 = 0, kColO = 128;
constexpr int kWG = 4;     // softmax warpgroups
constexpr int kCols = 16;  // query columns per warpgroup
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t unit_full[2], unit_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t st_full[kStages], st_empty[kStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_free, fin;
};
// Control block, placed in dynamic shared memory right after the tiles (the
// tiles need nearly the whole 227 KB budget, so nothing is static).
struct Ctrl {
  Bars bars;
  int unit_w[2];
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float red[kWG][2][4][kCols];  // read with 16-byte vector loads
#ifdef SEER_TRACE
  unsigned long long trace[24];
#endif
};
constexpr uint32_t kSmemAlloc = kSmemBytes + (uint32_t)sizeof(Ctrl);
static_assert(kSmemBytes % 16 == 0, "control block must start 16-byte aligned");
static_assert(offsetof(Ctrl, red) % 16 == 0, "red is read with float4 loads");
static_assert(offsetof(Ctrl, bars) % 8 == 0, "mbarriers need 8-byte alignment");
static_assert(kSmemAlloc <= 232448, "dynamic shared memory above the per-CTA limit");
}  // namespace attn

// Optional cycle accounting of the pipeline (build with -DSEER_TRACE): every
// wait and the softmax work are timed with clock64 and summed per CTA into
// the workspace header (trace words), to see which stage binds.
#ifdef SEER_TRACE
#define SEER_TRACE_ADD(k, v) atomicAdd(&C.trace[k], (unsigned long long)(v))
// segment k of the softmax step: time since the previous mark (lane 0 only)
#define SEER_MARK(k)                                   \
  do {                                                 \
    const long long tn_ = clock64();                   \
    if (lane == 0) SEER_TRACE_ADD(k, tn_ - tmark);     \
    tmark = tn_;                                       \
  } while (0)
#define SEER_TIMED(k, expr)                                  \
  [&]() {                                                    \
    const long long t0_ = clock64();                         \
    const auto r_ = (expr);                                  \
    SEER_TRACE_ADD(k, clock64() - t0_);                      \
    return r_;                                               \
  }()
#define SEER_TIMED_L0(k, expr)                               \
  [&]() {                                                    \
    const long long t0_ = clock64();                         \
    const auto r_ = (expr);                                  \
    if (lane == 0) SEER_TRACE_ADD(k, clock64() - t0_);       \
    return r_;                                               \
  }()
#else
#define SEER_TRACE_ADD(k, v) ((void)0)
#define SEER_MARK(k) ((void)0)
#define SEER_TIMED(k, expr) (expr)
#define SEER_TIMED_L0(k, expr) (expr)
#endif

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

// A list entry j, checked: it must satisfy 0 <= j <= i and be larger than the
// previous entry `prev` (as read, -1 before the first).  A failing entry is
// recorded and replaced by a safe in-range block so that no load leaves the
// tensor.
__device__ __forceinline__ int checked_entry(const AttnParams& p, const UnitInfo& u, int j, int prev) {
  if (j < 0 || j > u.i || j <= prev) {
    record_status(p.status, kDevBadIndex, (uint32_t)u.u);
    j = j < 0 ? 0 : (j > u.i ? u.i : j);
  }
  return j;
}

// Reduce-scatter of 16 column partials over the 32 lanes of a warp: first
// lanes l and l^16 combine all 16 values, then halving exchanges leave lane l
// with column (l & 15); lanes 0..15 store their column to out[0..15].  x is
// destroyed.  SUM selects sum (row sums) or max (column maxima).
template <bool SUM>
__device__ __forceinline__ void warp_reduce_scatter16(float (&x)[16], int lane, float* out) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float r = __shfl_xor_sync(0xffffffffu, x[k], 16);
    x[k] = SUM ? x[k] + r : fmaxf(x[k], r);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool up = lane & 8;
    const float send = up ? x[k] : x[k + 8], keep = up ? x[k + 8] : x[k];
    const float r = __shfl_xor_sync(0xffffffffu, send, 8);
    x[k] = SUM ? keep + r : fmaxf(keep, r);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool up = lane & 4;
    const float send = up ? x[k] : x[k + 4], keep = up ? x[k + 4] : x[k];
    const float r = __shfl_xor_sync(0xffffffffu, send, 4);
    x[k] = SUM ? keep + r : fmaxf(keep, r);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool up = lane & 2;
    const float send = up ? x[k] : x[k + 2], keep = up ? x[k + 2] : x[k];
    const float r = __shfl_xor_sync(0xffffffffu, send, 2);
    x[k] = SUM ? keep + r : fmaxf(keep, r);
  }
  const bool up = lane & 1;
  const float send = up ? x[0] : x[1], keep = up ? x[1] : x[0];
  const float r = __shfl_xor_sync(0xffffffffu, send, 1);
  if (lane < 16) out[lane] = SUM ? keep + r : fmaxf(keep, r);
}

// Combines the four warps' reduce-scatter results of a warpgroup (red is
// [4][kCols], each warp's row holding its column partials) into all kCols
// column results, for every thread.
template <bool SUM>
__device__ __forceinline__ void col_combine(const float* red, float (&out)[attn::kCols]) {
#pragma unroll
  for (int q = 0; q < attn::kCols; q += 4) {
    const float4 a = *reinterpret_cast<const float4*>(red + 0 * attn::kCols + q);
    const float4 b = *reinterpret_cast<const float4*>(red + 1 * attn::kCols + q);
    const float4 c = *reinterpret_cast<const float4*>(red + 2 * attn::kCols + q);
    const float4 d = *reinterpret_cast<const float4*>(red + 3 * attn::kCols + q);
    if (SUM) {
      out[q] = (a.x + b.x) + (c.x + d.x);
      out[q + 1] = (a.y + b.y) + (c.y + d.y);
      out[q + 2] = (a.z + b.z) + (c.z + d.z);
      out[q + 3] = (a.w + b.w) + (c.w + d.w);
    } else {
      out[q] = fmaxf(fmaxf(a.x, b.x), fmaxf(c.x, d.x));
      out[q + 1] = fmaxf(fmaxf(a.y, b.y), fmaxf(c.y, d.y));
      out[q + 2] = fmaxf(fmaxf(a.z, b.z), fmaxf(c.z, d.z));
      out[q + 3] = fmaxf(fmaxf(a.w, b.w), fmaxf(c.w, d.w));
    }
  }
}

__device__ __forceinline__ float exp2f_approx_sub(float a, float b) { return ex2_approx(a - b); }

// Loads this thread's kCols S^T columns (one key, kCols queries starting at
// column q0) from TMEM, scaled to the log2 domain; keys that are absent or
// causally masked (key position kl > query position) become -inf.
__device__ __forceinline__ void load_scores(uint32_t taddr, float (&x)[attn::kCols], float c,
                                            bool valid, bool diag, int kl, int q0) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < attn::kCols; ++q) x[q] = __uint_as_float(r[q]) * c;
  if (!valid) {
#pragma unroll
    for (int q = 0; q < attn::kCols; ++q) x[q] = -INFINITY;
  } else if (diag) {
#pragma unroll
    for (int q = 0; q < attn::kCols; ++q) x[q] = (q0 + q < kl) ? -INFINITY : x[q];
  }
}

// Issues the PV MMAs of pair step g: O^T (+)= V_pair^T . P^T, 16 keys per
// MMA (8 MMAs for two records, 4 for one).  Waits for the step's P^T and, on
// a unit's first step after an earlier unit, for that unit's epilogue to
// have read O^T.  Then releases the stage and signals pv_done.
__device__ __forceinline__ bool issue_pv(attn::Ctrl& C, const AttnParams& p, uint32_t tmem,
                                         uint32_t sbase, uint32_t vpart, int g, bool wait_o_free,
                                         bool first, bool two, int units_done) {
  using namespace attn;
  Bars& bars = C.bars;
  volatile int* abort_p = &C.abort_flag;
  const uint64_t tmo = p.timeout_ns;
  // p_full is double-buffered by step: the four softmax warpgroups are not
  // synchronised with each other, so one may already arrive for step g+1
  // while another is still on step g (never for g+2: S(g+2) needs PV(g)).
  if (!SEER_TIMED(3, mbar_wait(&bars.p_full[g & 1], (g >> 1) & 1, abort_p, p.status, tmo))) return false;
  if (wait_o_free && !SEER_TIMED(5, mbar_wait(&bars.o_free, (units_done - 1) & 1, abort_p, p.status, tmo)))
    return false;
  tc_fence_after();
  const uint32_t idesc_pv = make_idesc_bf16(128, 64, 1, 1);  // A = V^T, B = P^T (MN-major)
  const uint32_t stage = sbase + kOffRing + (g % kStages) * kStageBytes;
  const int nk = two ? 8 : 4;
  for (int kk = 0; kk < nk; ++kk) {
    const uint32_t rec = stage + (kk >> 2) * kRecBytes;  // keys 64*(kk/4) .. of the pair
    const uint32_t va = rec + vpart + (kk & 3) * 2048;
    const uint32_t pa = rec + (kk & 3) * 2048;           // P^T rows in the record's K^T part
    mma_bf16_ss(tmem + kColO, make_sw128_desc(va, 8192, 1024), make_sw128_desc(pa, 16384, 1024),
                idesc_pv, (first && kk == 0) ? 0u : 1u);
  }
  mma_commit(&bars.pv_done[g & 1]);
  mma_commit(&bars.st_empty[g % kStages]);
  return true;
}

__global__ void __launch_bounds__(attn::kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                       const AttnParams p) {
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
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  volatile int* abort_p = &C.abort_flag;
  const uint64_t tmo = p.timeout_ns;
  const uint32_t rec_rows = 2u * p.d;            // K^T rows + V rows of a record
  const uint32_t vpart = (uint32_t)p.d * 128u;   // byte offset of V inside a record

#ifdef SEER_TRACE
  const long long t_kernel0 = clock64();
  if (threadIdx.x < 24) C.trace[threadIdx.x] = 0;
#endif
  if (threadIdx.x == 0) {
    C.abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.unit_full[s], 1);
      mbar_init(&bars.unit_empty[s], 1 + 4 * kWG);  // MMA + softmax warps
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.pv_done[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(&bars.p_full[s], 4 * kWG);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.st_full[s], 1);
      mbar_init(&bars.st_empty[s], 1);
    }
    mbar_init(&bars.o_free, 4 * kWG);
    mbar_init(&bars.fin, 1);
    fence_barrier_init();
  }
  if (p.d == 64) {
    // With d = 64 a record is [K^T 64 rows | V 64 rows]; the PV product's
    // second 64-row panel of V^T (head dims 64..127) then reads the zeroed
    // third quarter of the record slot, which no load ever writes.
    for (int r = 0; r < 2 * kStages; ++r) {
      uint4* z = reinterpret_cast<uint4*>(smem + kOffRing + r * kRecBytes + 16384);
      for (int e = threadIdx.x; e < 8192 / 16; e += blockDim.x) z[e] = make_uint4(0, 0, 0, 0);
    }
    fence_async_shared();
  }
  if (warp == 17) {
    tmem_alloc(&C.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;
  const int dpanels = p.d / 64;

  if (warp == 16) {
    // ------------------------------- scheduler, Q loads, record gathers --
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKV);
      int u_idx = 0, qn = 0, g = 0;
      bool ok = true;
      while (ok) {
        const int slot = u_idx & 1;
        if (u_idx >= 2 && !mbar_wait(&bars.unit_empty[slot], ((u_idx >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        int w = (int)atomicAdd(p.work_counter, 1u);
        if (w >= p.total_units || *abort_p) w = -1;
        C.unit_w[slot] = w;
        mbar_arrive(&bars.unit_full[slot]);
        if (w < 0) break;
        ++u_idx;
        const UnitInfo u = decode_unit(p, w);
        if (u.count == 0) continue;
        const int qs = qn & 1;
        if (qn >= 2 && !mbar_wait(&bars.q_empty[qs], ((qn >> 1) - 1) & 1, abort_p, p.status, tmo)) break;
        mbar_arrive_expect_tx(&bars.q_full[qs], 64u * p.d * 2u);
        const int row = (int)(((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64);
        for (int pn = 0; pn < dpanels; ++pn)
          tma_load_2d(smem + kOffQ + qs * kQBytes + pn * 8192, &tmQ, &bars.q_full[qs], pn * 64, row);
        ++qn;
        const long long rec0 = ((long long)u.b * p.Hkv + u.g) * p.nb;
        // The list entries of the next pair step are loaded before this
        // step's wait for a free stage, so that their global-memory latency
        // is hidden behind it instead of delaying the gather.
        const int* lst = p.indices + u.u * p.cap;
        int jn0 = lst[0];
        int jn1 = u.count > 1 ? lst[1] : 0;
        int prev = -1;
        for (int m = 0; m < u.count; m += 2, ++g) {
          const int ntile = m + 1 < u.count ? 2 : 1;
          const int ja = jn0, jb = jn1;
          if (m + 2 < u.count) jn0 = lst[m + 2];
          if (m + 3 < u.count) jn1 = lst[m + 3];
          const int st = g % kStages;
          if (g >= kStages && !SEER_TIMED(0, mbar_wait(&bars.st_empty[st], ((g / kStages) - 1) & 1, abort_p, p.status, tmo))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars.st_full[st], (uint32_t)ntile * rec_rows * 128u);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h < ntile) {
              const int raw = h == 0 ? ja : jb;
              const int j = checked_entry(p, u, raw, prev);
              prev = raw;
              tma_load_2d(smem + kOffRing + st * kStageBytes + h * kRecBytes, &tmKV, &bars.st_full[st], 0,
                          (int)((rec0 + j) * rec_rows));
            }
          }
        }
      }
      // wait for loads still in flight before the CTA may exit
      for (int k = 0; k < 2 && k < qn; ++k) {
        const int qq = qn - 1 - k;
        mbar_wait(&bars.q_full[qq & 1], (qq >> 1) & 1, abort_p, nullptr, 20000000ull);
      }
      for (int k = 0; k < kStages && k < g; ++k) {
        const int gg = g - 1 - k;
        mbar_wait(&bars.st_full[gg % kStages], (gg / kStages) & 1, abort_p, nullptr, 20000000ull);
      }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(128, 64, 1, 0);  // A = K^T pair (MN-major)
      const uint32_t sbase = smem_u32(smem);
      int u_idx = 0, qn = 0, step = 0, units_done = 0;
      const int ksteps_qk = p.d / 16;
      bool ok = true;
      while (ok) {
        const int slot = u_idx & 1;
        if (!mbar_wait(&bars.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo)) break;
        const int w = C.unit_w[slot];
        mbar_arrive(&bars.unit_empty[slot]);
        if (w < 0) break;
        ++u_idx;
        const UnitInfo u = decode_unit(p, w);
        if (u.count == 0) continue;
        const int T = (u.count + 1) / 2;
        const int qs = qn & 1;
        if (!SEER_TIMED(4, mbar_wait(&bars.q_full[qs], (qn >> 1) & 1, abort_p, p.status, tmo))) break;
        const uint32_t qa = sbase + kOffQ + qs * kQBytes;
        for (int t = 0; t < T && ok; ++t) {
          const int g = step + t;
          const int st = g % kStages;
          if (!SEER_TIMED(2, mbar_wait(&bars.st_full[st], (g / kStages) & 1, abort_p, p.status, tmo))) { ok = false; break; }
          SEER_TRACE_ADD(12, 1);
          tc_fence_after();
          const uint32_t ka = sbase + kOffRing + st * kStageBytes;
          for (int kk = 0; kk < ksteps_qk; ++kk) {
            const uint32_t qoff = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kColS0 + (g & 1) * 64, make_sw128_desc(ka + kk * 2048, kRecBytes, 1024),
                        make_sw128_desc(qa + qoff, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars.s_full[g & 1]);
          if (t == T - 1) mma_commit(&bars.q_empty[qs]);
          if (t >= 1 && !issue_pv(C, p, tmem, sbase, vpart, g - 1, t - 1 == 0 && units_done > 0,
                                  t - 1 == 0, 2 * (t - 1) + 1 < u.count, units_done)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(C, p, tmem, sbase, vpart, step + T - 1, T == 1 && units_done > 0, T == 1,
                      2 * (T - 1) + 1 < u.count, units_done)) break;
        step += T;
        ++qn;
        ++units_done;
      }
      // all MMAs complete before TMEM is released
      mma_commit(&bars.fin);
      mbar_wait(&bars.fin, 0, abort_p, nullptr, 20000000ull);
    }
  } else if (warp < 16) {
    // ------------------------------------------------------- softmax WGs ---
    // The warpgroup synchronises with barrier.cta.red (hardware, no timeout),
    // so every one of its 128 threads must reach every barrier: a bounded wait
    // that gives up does not leave the loop on its own; its failure is ORed
    // into the next barrier and the whole warpgroup leaves together.
    const int wgi = warp >> 2;                 // warpgroup: query columns 32*wgi..
    const int ww = warp & 3;                   // TMEM sub-partition
    const int tl = ww * 32 + lane;             // TMEM lane == key in pair / dim of O^T
    const int q0 = wgi * kCols;
    const uint32_t bar_id = 1 + wgi;
    const uint32_t lane_addr = tmem + ((uint32_t)(ww * 32) << 16);
    const float c = p.scale_log2;
    const int half = tl >> 6, kl = tl & 63;
    int u_idx = 0, step = 0, red_use = 0;
    float lpart[kCols], m[kCols];
    for (;;) {
      const int slot = u_idx & 1;
      const bool okw = mbar_wait(&bars.unit_full[slot], (u_idx >> 1) & 1, abort_p, p.status, tmo);
      const int w = okw ? C.unit_w[slot] : -1;
      if (bar_red_or(bar_id, 128, !okw)) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.unit_empty[slot]);
      if (w < 0) break;
      ++u_idx;
      const UnitInfo u = decode_unit(p, w);
      const long long orow0 = ((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64 + q0;
      if (u.count == 0) {
        if (tl < p.d) {
          for (int q = 0; q < kCols; ++q) {
            if (p.out_fp32)
              reinterpret_cast<float*>(p.O)[(orow0 + q) * p.d + tl] = 0.f;
            else
              reinterpret_cast<uint16_t*>(p.O)[(orow0 + q) * p.d + tl] = 0;
          }
        }
        if (tl < kCols && p.lse) p.lse[orow0 + tl] = -INFINITY;
        continue;
      }
      const int T = (u.count + 1) / 2;
      // lists are ascending, so only the last entry can be the diagonal block
      const bool last_is_diag = p.indices[u.u * p.cap + u.count - 1] == u.i;
#pragma unroll
      for (int q = 0; q < kCols; ++q) lpart[q] = 0.f;
      bool fail = false;
      for (int t = 0; t < T; ++t) {
        const int g = step + t;
        const int mi = 2 * t + half;
        const bool valid = mi < u.count;
        const bool diag = valid && last_is_diag && mi == u.count - 1;
        const bool okS = SEER_TIMED_L0(6, mbar_wait(&bars.s_full[g & 1], (g >> 1) & 1, abort_p, p.status, tmo));
#ifdef SEER_TRACE
        const long long tstep0 = clock64();
        long long tmark = tstep0;
#endif
        tc_fence_after();
        const uint32_t saddr = lane_addr + kColS0 + (g & 1) * 64 + q0;
        float x[kCols];
        if (okS) load_scores(saddr, x, c, valid, diag, kl, q0);
        SEER_MARK(14);
        float* red = &C.red[wgi][red_use & 1][0][0];
        if (t == 0) {
          // exact column maxima of the unit's first step
          warp_reduce_scatter16<false>(x, lane, red + ww * kCols);
          ++red_use;
          if (bar_red_or(bar_id, 128, !okS)) { fail = true; break; }
          col_combine<false>(red, m);
          load_scores(saddr, x, c, valid, diag, kl, q0);
#pragma unroll
          for (int q = 0; q < kCols; ++q) x[q] = exp2f_approx_sub(x[q], m[q]);
        } else {
          float dmax = -INFINITY;
#pragma unroll
          for (int q = 0; q < kCols; ++q) {
            x[q] -= m[q];
            dmax = fmaxf(dmax, x[q]);
          }
          // probabilities with the running max; the barrier then tells
          // whether any score of the step exceeded it by more than 2^8
#pragma unroll
          for (int q = 0; q < kCols; ++q) x[q] = ex2_approx(x[q]);
          SEER_MARK(16);
          if (SEER_TIMED_L0(8, bar_red_or(bar_id, 128, !okS || dmax > kRescaleThreshold))) {
            if (*abort_p) { fail = true; break; }
            if (lane == 0) SEER_TRACE_ADD(13, 1);
            // exact column maxima of this step relative to the running max
            load_scores(saddr, x, c, valid, diag, kl, q0);
#pragma unroll
            for (int q = 0; q < kCols; ++q) x[q] -= m[q];
            warp_reduce_scatter16<false>(x, lane, red + ww * kCols);
            ++red_use;
            bar_red_or(bar_id, 128, false);
            col_combine<false>(red, x);
            float (&inc)[kCols] = x;  // increase of the running max per column
#pragma unroll
            for (int q = 0; q < kCols; ++q) {
              inc[q] = fmaxf(inc[q], 0.f);
              m[q] += inc[q];
              lpart[q] *= ex2_approx(-inc[q]);
            }
            // O^T columns are rescaled once the previous PV has landed
            const int gp = g - 1;
            const bool okPV = mbar_wait(&bars.pv_done[gp & 1], (gp >> 1) & 1, abort_p, p.status, tmo);
            if (okPV) {
              tc_fence_after();
              uint32_t o[16];
              tmem_ld16(lane_addr + kColO + q0, o);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 16; ++q)
                o[q] = __float_as_uint(__uint_as_float(o[q]) * ex2_approx(-inc[q]));
              tmem_st16(lane_addr + kColO + q0, o);
              tmem_wait_st();
            }
            if (bar_red_or(bar_id, 128, !okPV)) { fail = true; break; }
            load_scores(saddr, x, c, valid, diag, kl, q0);
#pragma unroll
            for (int q = 0; q < kCols; ++q) x[q] = exp2f_approx_sub(x[q], m[q]);
          }
          SEER_MARK(17);
        }
        // row-sum partials and this warpgroup's half of the bf16 P^T row
        uint32_t pk[kCols / 2];
#pragma unroll
        for (int q = 0; q < kCols; q += 2) {
          lpart[q] += x[q];
          lpart[q + 1] += x[q + 1];
          pk[q >> 1] = pack_bf16x2(x[q], x[q + 1]);
        }
        SEER_MARK(18);
        // P^T row `kl` of record `half` of the step's stage (its K^T part)
        uint8_t* prow = smem + kOffRing + (g % kStages) * kStageBytes + half * kRecBytes + kl * 128;
#pragma unroll
        for (int ch = 0; ch < kCols / 8; ++ch) {
          const int chunk = wgi * (kCols / 8) + ch;
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (kl & 7)) << 4)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        SEER_MARK(20);
        fence_async_shared();
        SEER_MARK(21);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[g & 1]);
        SEER_MARK(22);
#ifdef SEER_TRACE
        if (lane == 0) SEER_TRACE_ADD(9, clock64() - tstep0);
#endif
      }
      if (fail) break;
      // ------------------------------------------------------- epilogue ---
#ifdef SEER_TRACE
      const long long tep0 = clock64();
#endif
      const int gl = step + T - 1;
      const bool okPV = mbar_wait(&bars.pv_done[gl & 1], (gl >> 1) & 1, abort_p, p.status, tmo);
      float* red = &C.red[wgi][red_use & 1][0][0];
      warp_reduce_scatter16<true>(lpart, lane, red + ww * kCols);
      ++red_use;
      if (bar_red_or(bar_id, 128, !okPV)) break;
      float l[kCols];
      col_combine<true>(red, l);
      tc_fence_after();
      {
        uint32_t o[16];
        tmem_ld16(lane_addr + kColO + q0, o);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.o_free);
        if (tl < p.d) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float v = __uint_as_float(o[q]) * (1.0f / l[q]);
            const long long idx = (orow0 + q) * p.d + tl;
            if (p.out_fp32)
              reinterpret_cast<float*>(p.O)[idx] = v;
            else
              reinterpret_cast<__nv_bfloat16*>(p.O)[idx] = __float2bfloat16_rn(v);
          }
        }
      }
      if (tl < kCols && p.lse) {
        float mq = m[0], lq = l[0];
#pragma unroll
        for (int q = 1; q < kCols; ++q)
          if (q == tl) {
            mq = m[q];
            lq = l[q];
          }
        p.lse[orow0 + tl] = (mq + log2f(lq)) * 0.6931471805599453f;
      }
#ifdef SEER_TRACE
      if (lane == 0) SEER_TRACE_ADD(10, clock64() - tep0);
#endif
      step += T;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 17) tmem_dealloc(tmem, kTmemCols);
#ifdef SEER_TRACE
  if (threadIdx.x == 0) {
    C.trace[11] = clock64() - t_kernel0;
    for (int k = 0; k < 24; ++k) atomicAdd(p.trace + k, C.trace[k]);
  }
#endif
}

// ---------------------------------------------------------------- re-layout --
// Writes every (batch, KV head, key block j) as one contiguous record of
// 2*d rows x 64 bf16 (128-byte rows):
//   rows 0 .. d-1        K^T: row c holds K[64j + 0 .. 63][c]
//   rows d .. 2d-1       V in 64-column panels: row d + 64p + r holds
//                        V[64j + r][64p .. 64p + 63]
// so that one TMA box of 2*d rows gathers K and V of a block at once.
// fp32 inputs are rounded to bf16 here (round to nearest even).
template <typename T>
__global__ void __launch_bounds__(256) kv_tile_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                      __nv_bfloat16* __restrict__ out, int n, int d) {
  __shared__ __nv_bfloat16 sk[64][128 + 2];
  const int nb = n / kBlock;
  const long long rec = blockIdx.x;  // (b*Hkv + g)*nb + j
  const long long bg = rec / nb;
  const int j = (int)(rec % nb);
  const T* Kt = K + (bg * n + (long long)j * kBlock) * d;
  const T* Vt = V + (bg * n + (long long)j * kBlock) * d;
  __nv_bfloat16* o = out + rec * (2LL * d) * 64;
  for (int e = threadIdx.x; e < 64 * d; e += blockDim.x) {
    const int r = e / d, c = e % d;
    if constexpr (sizeof(T) == 2)
      sk[r][c] = reinterpret_cast<const __nv_bfloat16*>(Kt)[e];
    else
      sk[r][c] = __float2bfloat16_rn(reinterpret_cast<const float*>(Kt)[e]);
  }
  __syncthreads();
  // K^T: 8 keys (16 bytes) per store
  for (int e = threadIdx.x; e < d * 8; e += blockDim.x) {
    const int c = e / 8, k0 = (e % 8) * 8;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t lo = __bfloat16_as_ushort(sk[k0 + 2 * q][c]);
      const uint32_t hi = __bfloat16_as_ushort(sk[k0 + 2 * q + 1][c]);
      w[q] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(o + (long long)c * 64 + k0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  // V panels: 8 elements (16 bytes) per move
  for (int e = threadIdx.x; e < 64 * d / 8; e += blockDim.x) {
    const int r = e / (d / 8), c8 = (e % (d / 8)) * 8;
    const int pnl = c8 / 64, cc = c8 % 64;
    uint4 v;
    if constexpr (sizeof(T) == 2) {
      v = *reinterpret_cast<const uint4*>(Vt + (long long)r * d + c8);
    } else {
      const float* f = reinterpret_cast<const float*>(Vt) + (long long)r * d + c8;
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        w[q] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * q])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * q + 1])) << 16);
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(o + (long long)(d + pnl * 64 + r) * 64 + cc) = v;
  }
}

cudaError_t launch_kv_tiles(const void* K, const void* V, bool fp32, void* out, long long records,
                            int n, int d, cudaStream_t st) {
  if (fp32)
    kv_tile_kernel<float><<<(unsigned)records, 256, 0, st>>>((const float*)K, (const float*)V,
                                                             (__nv_bfloat16*)out, n, d);
  else
    kv_tile_kernel<uint16_t><<<(unsigned)records, 256, 0, st>>>((const uint16_t*)K, (const uint16_t*)V,
                                                                (__nv_bfloat16*)out, n, d);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKV, const AttnParams& p,
                               int num_sms, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)attn::kSmemAlloc);
  if (e != cudaSuccess) return e;
  long long grid = p.total_units < num_sms ? p.total_units : num_sms;
  if (grid < 1) grid = 1;
  sparse_attn_kernel<<<(unsigned)grid, attn::kThreads, attn::kSmemAlloc, st>>>(tmQ, tmKV, p);
  return cudaGetLastError();
}

}  // namespace seer
