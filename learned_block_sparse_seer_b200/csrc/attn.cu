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
//  * A re-layout pass (kt_tile_kernel) first writes K^T of every (KV head,
//    key block) as one contiguous record (d rows x 64 keys); one d-row TMA
//    box (16 KB at d = 128, no cluster multicast) brings it into shared
//    memory as the MN-major A operand of QK.  V is read in place through a
//    3-D map (64 dims x 64 keys x d/64 panels): one 16 KB box per block,
//    landing as 64-dim panels, the MN-major A operand of PV.
//  * The tensor pipe stalls for about 200 cycles whenever the thread that
//    issues MMAs synchronises (an mbarrier wait, a shared-memory read, a
//    barrier), so two warps issue them, each waiting once per pair step on
//    its own barrier: the QK warp on kfull(h) (K^T of step h landed, plus the
//    unit's Q tile on its first step, and the softmax has released the S^T
//    buffer of step h-3), the PV warp on go(g) (P^T and V of step g ready).
//    While one waits the other keeps the pipe fed.  The MMA groups are
//    straight-line code: fully unrolled, descriptors as a base plus constant
//    offsets, ring positions as counters.
//  * Separate rings keep each buffer only as long as it is needed: K^T pairs
//    (2 slots, free once their QK is done), V pairs (3 slots, free once their
//    PV is done), P^T tiles (3 slots), one Q tile, S^T in TMEM (3 buffers).
//    224 KB of shared memory in all.
//  * Warp roles (608 threads): warps 0..15 are four softmax warpgroups, each
//    owning 16 of the 64 query columns, one key (TMEM lane) per thread -- a
//    warp w reaches TMEM lanes 32*(w%4)..+31; warp 16 schedules units and
//    issues every TMA load; warp 17 issues the PV MMAs and owns the TMEM
//    allocation; warp 18 issues the QK MMAs.
//  * Softmax without a per-step barrier: each unit's column maxima are formed
//    exactly on its first step and then kept; later steps compute
//    exp2(score * scale - max) with packed f32x2 arithmetic.  Scores above
//    the kept maximum are harmless until P, a column sum or O would overflow
//    fp32 / bf16 (about 2^128); the unit's epilogue checks for that, flags
//    the unit, and sparse_attn_redo_kernel recomputes flagged units exactly.
//  * Units are handed out by an atomic counter in KV-head-major order, query
//    blocks from the last (longest lists) to the first, so the K/V of one KV
//    head stay hot in L2 while its query heads are processed.  Units with an
//    empty list never enter the ring (empty_rows_kernel writes their rows).
//  * Every mbarrier wait is bounded (%globaltimer); on expiry the kernel
//    records a timeout in the workspace status word and unwinds: the warps
//    stop making barrier arrivals, and before the CTA exits the teardown
//    completes each barrier phase the loader armed with exactly the
//    arrivals it lacks and waits until its bulk copies have landed.
#include <cstddef>
#include <cstdint>

#include "attn.cuh"
#include "common.cuh"
#include "ptx.cuh"


namespace seer {

namespace attn {
constexpr int kThreads = 608;
constexpr int kWarpLoad = 16, kWarpPV = 17, kWarpQK = 18;
constexpr uint32_t kHalf = 16384;              // one key block's K^T record or V (d = 128)
constexpr uint32_t kPair = 2 * kHalf;          // the K^T (or V) of a pair step
constexpr int kKSlots = 2, kVSlots = 3, kPSlots = 3, kQSlots = 1;
constexpr uint32_t kPBytes = 16384;            // P^T of a pair step: 2 x [64 keys x 64 queries]
constexpr uint32_t kQBytes = 16384;            // Q tile: 64 rows x d (two 64-column panels)
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kKSlots * kPair;       //  64 KB
constexpr uint32_t kOffP = kOffV + kVSlots * kPair;       // 160 KB
constexpr uint32_t kOffQ = kOffP + kPSlots * kPBytes;     // 208 KB
constexpr uint32_t kSmemBytes = kOffQ + kQSlots * kQBytes;  // 224 KB of tiles
constexpr int kRing = 4;   // kfull / go / qk_done / pv_done barriers, indexed by step
constexpr int kSBuf = 3;   // S^T buffers in TMEM (QK runs two steps ahead of PV)
constexpr int kUnits = 8;  // unit ring entries (the scheduler runs ahead of the consumers)
constexpr uint32_t kTmemCols = 256;            // S^T x 3 (64 columns each) + O^T (64)
constexpr uint32_t kColO = kSBuf * 64;
constexpr int kWG = 4;     // softmax warpgroups
constexpr int kCols = 16;  // query columns per warpgroup
constexpr int kSoftmaxWarps = 4 * kWG;
// readers of a unit ring entry: both MMA warps and every softmax warp
constexpr int kUnitReaders = 2 + kSoftmaxWarps;
static_assert(kSBuf < kRing, "kfull(h) takes softmax(h - kSBuf) arrivals");
static_assert(kVSlots < kRing && kPSlots < kRing && kKSlots < kRing, "slot reuse is tracked on the step rings");

struct Bars {
  uint64_t unit_full[kUnits], unit_empty[kUnits];
  uint64_t kfull[kRing];    // K^T(h) [+ Q] landed and softmax(h-3) done: the QK warp's one wait per step
  uint64_t go[kRing];       // P^T(g) and V(g) ready: the PV warp's one wait per step
  uint64_t qk_done[kRing];  // QK(g) complete: S^T(g) readable, K slot of g free
  uint64_t pv_done[kRing];  // PV(g) complete: V slot and P^T slot of g free
  uint64_t q_free[kQSlots];  // the last QK of the unit that used a Q slot is complete
  uint64_t fin_qk, fin_pv;
};
// What the scheduler publishes about each unit: the work index (-1 ends the
// work), its checked list length, whether its last entry is the diagonal
// block, and the flat unit index u = (b*Hq + hq)*nb + i (its 64 query rows
// start at row 64*u of Q and O).
struct UnitEntry {
  int w, count, diag, u;
};
// Control block, placed in dynamic shared memory right after the tiles (the
// tiles need nearly the whole 227 KB budget, so nothing is static).
struct Ctrl {
  Bars bars;
  UnitEntry unit[kUnits];
  uint32_t tmem_base;
  int abort_flag;
  int redo_unit;  // the last unit this CTA flagged for the exact fallback
  // Teardown accounting after an abort: the steps whose K^T (and Q) and V
  // copies the loader issued, and the steps for which each softmax warp made
  // its go / kfull arrivals.
  int armed_k, armed_v;
  int sm_steps[kSoftmaxWarps];
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

// Coordinates of unit w (no memory access): batch, query head, its KV head,
// query block and flat unit index.
__device__ __forceinline__ UnitInfo unit_coords(const AttnParams& p, int w) {
  UnitInfo r;
  const int per_bg = p.nb * p.G;
  const int bg = w / per_bg, rem = w % per_bg;
  r.b = bg / p.Hkv;
  r.g = bg % p.Hkv;
  r.i = p.nb - 1 - rem / p.G;
  r.hq = r.g * p.G + rem % p.G;
  r.u = ((long long)r.b * p.Hq + r.hq) * p.nb + r.i;
  r.count = 0;
  return r;
}

// unit_coords plus the unit's list length, read and checked: it must lie in
// [0, min(cap, i + 1)].  A failing count is recorded and clamped.
__device__ __forceinline__ UnitInfo decode_unit(const AttnParams& p, int w) {
  UnitInfo r = unit_coords(p, w);
  if (p.dense) {
    r.count = r.i + 1;
    return r;
  }
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

// A consumer's walk over the unit ring, one pair step at a time.  next()
// returns the step's info -- bit 0: two key blocks, bit 1: first step of its
// unit, bit 2: last step, bit 3: the unit's Q slot -- or -1 at the end (or on
// a timeout, which also clears ok).  A ring entry is released as soon as it
// has been read.
struct UnitCursor {
  int ur = 0, qn = 0, count = 0, rem = 0, t = 0, qslot = 0;
  bool end = false;
  __device__ __forceinline__ int next(attn::Ctrl& C, const AttnParams& p, volatile int* abort_p, bool& ok) {
    using namespace attn;
    while (rem == 0) {
      if (end) return -1;
      const int slot = ur % kUnits;
      if (!mbar_wait(&C.bars.unit_full[slot], (ur / kUnits) & 1, abort_p, p.status, p.timeout_ns)) {
        ok = false;
        end = true;
        return -1;
      }
      const int w = C.unit[slot].w, cnt = C.unit[slot].count;
      ++ur;
      if (w < 0) {  // the end marker is never released: nothing reuses its slot
        end = true;
        return -1;
      }
      mbar_arrive(&C.bars.unit_empty[slot]);
      count = cnt;
      rem = (cnt + 1) / 2;
      t = 0;
      qslot = qn % kQSlots;
      ++qn;
    }
    const int info = (2 * t + 1 < count ? 1 : 0) | (t == 0 ? 2 : 0) | (rem == 1 ? 4 : 0) | (qslot << 3);
    ++t;
    --rem;
    return info;
  }
};

// This thread's kCols S^T columns from TMEM as (score * c - m) in the log2
// domain, with packed pair arithmetic (nm2 holds -m); absent or causally
// masked keys become -inf.
__device__ __forceinline__ void scores_minus_max(uint32_t taddr, float (&x)[attn::kCols], uint64_t c2,
                                                 const uint64_t (&nm2)[attn::kCols / 2], bool valid, bool diag,
                                                 int kl, int q0) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int q = 0; q < attn::kCols / 2; ++q) {
    const uint64_t v = fma_f32x2(f32x2_pack(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1])), c2, nm2[q]);
    f32x2_unpack(v, x[2 * q], x[2 * q + 1]);
  }
  if (!valid) {
#pragma unroll
    for (int q = 0; q < attn::kCols; ++q) x[q] = -INFINITY;
  } else if (diag) {
#pragma unroll
    for (int q = 0; q < attn::kCols; ++q) x[q] = (q0 + q < kl) ? -INFINITY : x[q];
  }
}

// This warpgroup's 16 bf16 probabilities of key row kl into the step's P^T
// tile (128-byte rows, 16-byte chunks swizzled by the row index).
// off0/off1 are the row's two swizzled 16-byte chunk offsets.
__device__ __forceinline__ void store_p(uint8_t* prow, const float (&x)[attn::kCols], uint32_t off0, uint32_t off1) {
  static_assert(attn::kCols == 16, "two 16-byte chunks per row and warpgroup");
  uint32_t pk[attn::kCols / 2];
#pragma unroll
  for (int q = 0; q < attn::kCols; q += 2) pk[q >> 1] = pack_bf16x2(x[q], x[q + 1]);
  *reinterpret_cast<uint4*>(prow + off0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  *reinterpret_cast<uint4*>(prow + off1) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// Waits (bounded) until the phase of `bar` with the given parity has
// completed; used only at teardown, so it does not look at the abort flag.
__device__ __forceinline__ bool mbar_wait_teardown(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000u))
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(attn::kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKt,
                       const __grid_constant__ CUtensorMap tmV,
                       const AttnParams p) {
  using namespace attn;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (p.run_if && ((*p.run_if != 0u) != (p.run_if_value != 0u))) return;  // the dense kernel takes this call
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

#ifdef SEER_TRACE
  const long long t_kernel0 = clock64();
  if (threadIdx.x < 24) C.trace[threadIdx.x] = 0;
#endif
  if (threadIdx.x == 0) {
    C.abort_flag = 0;
    C.redo_unit = -1;
    C.armed_k = 0;
    C.armed_v = 0;
    for (int s = 0; s < kUnits; ++s) {
      mbar_init(&bars.unit_full[s], 1);
      mbar_init(&bars.unit_empty[s], kUnitReaders);  // released by every reader on reading
    }
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&bars.kfull[s], 1 + kSoftmaxWarps);  // K loader's K^T (+Q) part + softmax(h-3) done
      mbar_init(&bars.go[s], 1 + kSoftmaxWarps);     // V loader's V part + softmax's P^T(g)
      mbar_init(&bars.qk_done[s], 1);
      mbar_init(&bars.pv_done[s], 1);
    }
    // The first kSBuf steps' S^T buffers are free from the start: their
    // "softmax(h-3) done" arrivals are made here.
    for (int s = 0; s < kSBuf; ++s)
      for (int a = 0; a < kSoftmaxWarps; ++a) mbar_arrive(&bars.kfull[s]);
    for (int s = 0; s < kQSlots; ++s) mbar_init(&bars.q_free[s], 1);
    mbar_init(&bars.fin_qk, 1);
    mbar_init(&bars.fin_pv, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < kSoftmaxWarps) C.sm_steps[threadIdx.x] = 0;
  if (D == 64) {
    // With d = 64 a key block's V is one 8 KB panel; the PV product's second
    // 64-row panel of V^T (head dims 64..127) then reads the zeroed upper
    // half of each block's V slot, which no load ever writes.
    for (int r = 0; r < 2 * kVSlots; ++r) {
      uint4* z = reinterpret_cast<uint4*>(smem + kOffV + r * kHalf + 8192);
      for (int e = threadIdx.x; e < 8192 / 16; e += blockDim.x) z[e] = make_uint4(0, 0, 0, 0);
    }
    fence_async_shared();
  }
  if (warp == kWarpPV) {
    tmem_alloc(&C.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;
  constexpr uint32_t part_bytes = (uint32_t)D * 128u;  // a key block's K^T record, or its V

  if (warp == kWarpLoad) {
    // ------------------------------- scheduler, Q loads, record gathers --
    // Units are handed out by an atomic counter and published in the unit
    // ring.  Units with an empty list never enter the ring: their output
    // (O = 0, LSE = -inf) is written by empty_rows_kernel before this kernel.
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmKt);
      prefetch_tmap(&tmV);
      int u_idx = 0, qn = 0, hk = 0, hv = 0;  // units published, Q tiles, steps whose K^T / V copies are out
      bool ok = true;
      while (ok) {
        const int slot = u_idx % kUnits;
        if (u_idx >= kUnits &&
            !mbar_wait(&bars.unit_empty[slot], ((u_idx / kUnits) - 1) & 1, abort_p, p.status, tmo))
          break;
        int w;
        UnitInfo u{};
        for (;;) {
          w = (int)atomicAdd(p.work_counter, 1u);
          if (w >= p.total_units || *abort_p) {
            w = -1;
            break;
          }
          u = decode_unit(p, w);
          if (u.count > 0) break;
        }
        // lists are ascending, so only the last entry can be the diagonal block
        const int diag = w >= 0 ? (p.dense ? 1 : (p.indices[u.u * p.cap + u.count - 1] == u.i)) : 0;
        C.unit[slot].w = w;
        C.unit[slot].count = u.count;
        C.unit[slot].diag = diag;
        C.unit[slot].u = w >= 0 ? (int)u.u : 0;
        mbar_arrive(&bars.unit_full[slot]);
        ++u_idx;
        if (w < 0) break;  // the end marker is never released: nothing reuses its slot
        const int qs = qn % kQSlots;
        if (qn >= kQSlots && !mbar_wait(&bars.q_free[qs], ((qn / kQSlots) - 1) & 1, abort_p, p.status, tmo)) break;
        ++qn;
        const int qrow = (int)(((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64);
        const long long rec0 = ((long long)u.b * p.Hkv + u.g) * p.nb;  // this KV head's first block
        // The list entries of the next pair step are read one step early, so
        // that their global-memory latency hides behind this step's waits.
        const int* lst = p.indices + u.u * p.cap;
        auto entry = [&](int t) { return p.dense ? t : lst[t]; };
        int jn0 = entry(0);
        int jn1 = u.count > 1 ? entry(1) : 0;
        int prev = -1;
        for (int m = 0; m < u.count; m += 2) {
          const int h = hk;
          const int ntile = m + 1 < u.count ? 2 : 1;
          const int ra = jn0, rb = jn1;
          if (m + 2 < u.count) jn0 = entry(m + 2);
          if (m + 3 < u.count) jn1 = entry(m + 3);
          int jj[2];
          jj[0] = checked_entry(p, u, ra, prev);
          prev = ra;
          jj[1] = 0;
          if (ntile == 2) {
            jj[1] = checked_entry(p, u, rb, prev);
            prev = rb;
          }
          // K^T part: its slot is free once QK(h-2) is complete; it (and the
          // unit's Q tile on its first step) completes kfull(h).
          if (h >= kKSlots && !SEER_TIMED(0, mbar_wait(&bars.qk_done[(h - kKSlots) % kRing],
                                                        ((h - kKSlots) / kRing) & 1, abort_p, p.status, tmo))) {
            ok = false;
            break;
          }
          uint64_t* tk = &bars.kfull[h % kRing];
          mbar_arrive_expect_tx(tk, (uint32_t)ntile * part_bytes + (m == 0 ? 64u * D * 2u : 0u));
          if (m == 0) tma_load_3d(smem + kOffQ + qs * kQBytes, &tmQ, tk, 0, qrow, 0);
          for (int t = 0; t < ntile; ++t)
            tma_load_2d(smem + kOffK + (h % kKSlots) * kPair + t * kHalf, &tmKt, tk, 0, (int)((rec0 + jj[t]) * D));
          ++hk;
          // V part: its slot is free once PV(h-3) is complete; it completes go(h).
          if (h >= kVSlots &&
              !SEER_TIMED(1, mbar_wait(&bars.pv_done[(h - kVSlots) % kRing], ((h - kVSlots) / kRing) & 1, abort_p,
                                       p.status, tmo))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars.go[h % kRing], (uint32_t)ntile * part_bytes);
          for (int t = 0; t < ntile; ++t)
            tma_load_3d(smem + kOffV + (h % kVSlots) * kPair + t * kHalf, &tmV, &bars.go[h % kRing], 0,
                        (int)((rec0 + jj[t]) * 64), 0);
          ++hv;
        }
      }
      // steps whose copies were issued: the teardown drains them after an abort
      C.armed_k = hk;
      C.armed_v = hv;
    }
  } else if (warp == kWarpQK) {
    // ------------------------------------------------------ QK issuer ----
    // Two warps issue the MMAs, QK and PV, each waiting once per step on its
    // own barrier: while one waits, the other keeps the tensor pipe fed.
    // The issue code is straight-line (fully unrolled groups, descriptors as
    // a per-step base plus compile-time offsets, ring positions as counters):
    // per-MMA branches or address arithmetic measurably slow the pipe's intake.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, 64, 1, 0);  // A = K^T pair (MN-major)
      const uint32_t sbase = smem_u32(smem);
      // The start address field holds (address >> 4): a byte offset b inside
      // the 256 KB window is added as (b >> 4).
      const uint64_t dK0 = make_sw128_desc(sbase + kOffK, kHalf, 1024);
      const uint64_t dQ0 = make_sw128_desc(sbase + kOffQ, 16, 1024);
      UnitCursor cur;
      bool ok = true;
      int h = 0, kslot = 0, sbuf = 0, ring = 0;
      for (;;) {
        const int info = cur.next(C, p, abort_p, ok);
        if (info < 0) break;
        if (!SEER_TIMED(4, mbar_wait(&bars.kfull[ring], (h / kRing) & 1, abort_p, p.status, tmo))) break;
        tc_fence_after();
        const uint64_t dk = dK0 + ((uint64_t)(kslot * kPair) >> 4);
        const uint64_t dq = dQ0 + ((uint64_t)(((info >> 3) & 1) * kQBytes) >> 4);
        const uint32_t sc = tmem + (uint32_t)sbuf * 64u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(sc, dk + (uint64_t)(kk * 2048 / 16), dq + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) / 16),
                      idesc_qk, kk > 0 ? 1u : 0u);
        // (a test hook can leave out one step's completion signal, so that
        // the waits on it run into their limit)
        if (h != p.test_skip_qk_commit) mma_commit(&bars.qk_done[ring]);
        if (info & 4) mma_commit(&bars.q_free[(info >> 3) & 1]);
        ++h;
        kslot = kslot + 1 == kKSlots ? 0 : kslot + 1;
        sbuf = sbuf + 1 == kSBuf ? 0 : sbuf + 1;
        ring = ring + 1 == kRing ? 0 : ring + 1;
      }
      // this thread's MMAs complete before TMEM is released
      mma_commit(&bars.fin_qk);
      mbar_wait_teardown(&bars.fin_qk, 0, 20000000ull);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------ PV issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, 64, 1, 1);  // A = V^T, B = P^T (MN-major)
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dV0 = make_sw128_desc(sbase + kOffV, 8192, 1024);
      const uint64_t dP0 = make_sw128_desc(sbase + kOffP, 16384, 1024);
      UnitCursor cur;
      bool ok = true;
      int g = 0, vslot = 0, pslot = 0, ring = 0;
      for (;;) {
        const int info = cur.next(C, p, abort_p, ok);
        if (info < 0) break;
        if (!SEER_TIMED(3, mbar_wait(&bars.go[ring], (g / kRing) & 1, abort_p, p.status, tmo))) break;
        SEER_TRACE_ADD(12, 1);
        tc_fence_after();
        const uint64_t dv = dV0 + ((uint64_t)(vslot * kPair) >> 4);
        const uint64_t dp = dP0 + ((uint64_t)(pslot * kPBytes) >> 4);
        const uint32_t acc0 = (info & 2) ? 0u : 1u;
        if (info & 1) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem + kColO, dv + (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 2048) / 16),
                        dp + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 2048) / 16), idesc_pv, kk == 0 ? acc0 : 1u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + kColO, dv + (uint64_t)((kk * 2048) / 16), dp + (uint64_t)((kk * 2048) / 16), idesc_pv,
                        kk == 0 ? acc0 : 1u);
        }
        mma_commit(&bars.pv_done[ring]);
        ++g;
        vslot = vslot + 1 == kVSlots ? 0 : vslot + 1;
        pslot = pslot + 1 == kPSlots ? 0 : pslot + 1;
        ring = ring + 1 == kRing ? 0 : ring + 1;
      }
      mma_commit(&bars.fin_pv);
      mbar_wait_teardown(&bars.fin_pv, 0, 20000000ull);
    }
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------- softmax WGs ---
    // The warpgroup synchronises with barrier.cta.red (hardware, no timeout),
    // so every one of its 128 threads must reach every barrier: a bounded wait
    // that gives up does not leave the loop on its own; its failure is ORed
    // into the next barrier and the whole warpgroup leaves together.
    const int wgi = warp >> 2;                 // warpgroup: query columns 16*wgi..
    const int ww = warp & 3;                   // TMEM sub-partition
    const int tl = ww * 32 + lane;             // TMEM lane == key in pair / dim of O^T
    const int q0 = wgi * kCols;
    const uint32_t bar_id = 1 + wgi;
    const uint32_t lane_addr = tmem + ((uint32_t)(ww * 32) << 16);
    const float c = p.scale_log2;
    const int half = tl >> 6, kl = tl & 63;
    int u_idx = 0, step = 0, red_use = 0;
    int arrived = 0;  // steps whose go / kfull arrivals this warp has made
    // Set (warp-uniformly, for good) by the warp's first failed wait: from
    // then on it makes no barrier arrivals, so that every barrier phase is
    // only ever completed by real work and the teardown can account for the
    // arrivals that are missing.
    bool dead = false;
    // Per query column of this warpgroup, as packed pairs: the negated
    // running maximum (log2 domain) and this thread's row-sum partial.
    uint64_t nm2[kCols / 2], lp2[kCols / 2];
    const uint64_t c2 = f32x2_pack(c, c);
    // this thread's P^T row (key kl of half `half`) and its two swizzled
    // 16-byte chunks (this warpgroup's 16 query columns)
    uint8_t* const prow0 = smem + kOffP + half * 8192 + kl * 128;
    const uint32_t poff0 = (uint32_t)(((2 * wgi) ^ (kl & 7)) << 4);
    const uint32_t poff1 = (uint32_t)(((2 * wgi + 1) ^ (kl & 7)) << 4);
    // ring positions of the current step g: barrier ring slot and phase,
    // S^T buffer, P^T slot
    int rg = 0, rph = 0, sb = 0, ps = 0;
    for (;;) {
      const int slot = u_idx % kUnits;
      const bool okw = mbar_wait(&bars.unit_full[slot], (u_idx / kUnits) & 1, abort_p, p.status, tmo);
      const int w = okw ? C.unit[slot].w : -1;
      const int count = okw ? C.unit[slot].count : 0;
      const bool last_is_diag = okw && C.unit[slot].diag != 0;
      const int uu = okw ? C.unit[slot].u : 0;
      if (bar_red_or(bar_id, 128, !okw || dead)) break;
      if (w < 0) break;  // the end marker is never released: nothing reuses its slot
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.unit_empty[slot]);
      ++u_idx;
      const long long orow0 = (long long)uu * 64 + q0;
      const int T = (count + 1) / 2;
#pragma unroll
      for (int q = 0; q < kCols / 2; ++q) lp2[q] = 0ull;
      bool fail = false;
      for (int t = 0; t < T; ++t) {
        const int g = step + t;
        (void)g;
        const int mi = 2 * t + half;
        const bool valid = mi < count;
        const bool diag = valid && last_is_diag && mi == count - 1;
        const bool okS = SEER_TIMED_L0(6, mbar_wait(&bars.qk_done[rg], rph, abort_p, p.status, tmo));
        // P^T(g) goes to the slot of step g-kPSlots, free once that step's PV
        // is complete (long done in steady state); a failed wait joins the
        // unit's next barrier.
        static_assert(kPSlots <= kRing, "P^T slot reuse is tracked on the pv_done ring");
        const int pr = rg >= kPSlots ? rg - kPSlots : rg - kPSlots + kRing;
        const int pph = rg >= kPSlots ? rph : rph ^ 1;
        const bool okP = g < kPSlots || mbar_wait(&bars.pv_done[pr], pph, abort_p, p.status, tmo);
        dead = dead || __any_sync(0xffffffffu, !okS || !okP);
#ifdef SEER_TRACE
        const long long tstep0 = clock64();
        long long tmark = tstep0;
#endif
        tc_fence_after();
        const uint32_t saddr = lane_addr + (uint32_t)sb * 64u + q0;
        uint8_t* const prow = prow0 + ps * kPBytes;
        float x[kCols];
        if (t == 0) {
          // exact column maxima of the unit's first step
          if (okS) load_scores(saddr, x, c, valid, diag, kl, q0);
          float* red = &C.red[wgi][red_use & 1][0][0];
          warp_reduce_scatter16<false>(x, lane, red + ww * kCols);
          ++red_use;
          if (bar_red_or(bar_id, 128, dead)) { fail = true; break; }
          float mcol[kCols];
          col_combine<false>(red, mcol);
#pragma unroll
          for (int q = 0; q < kCols / 2; ++q) nm2[q] = f32x2_pack(-mcol[2 * q], -mcol[2 * q + 1]);
          scores_minus_max(saddr, x, c2, nm2, valid, diag, kl, q0);
#pragma unroll
          for (int q = 0; q < kCols; ++q) x[q] = ex2_approx(x[q]);
          store_p(prow, x, poff0, poff1);
        } else {
          if (okS) scores_minus_max(saddr, x, c2, nm2, valid, diag, kl, q0);
#pragma unroll
          for (int q = 0; q < kCols; ++q) x[q] = ex2_approx(x[q]);
          store_p(prow, x, poff0, poff1);
          SEER_MARK(17);
        }
        // row-sum partials
#pragma unroll
        for (int q = 0; q < kCols / 2; ++q) lp2[q] = add_f32x2(lp2[q], f32x2_pack(x[2 * q], x[2 * q + 1]));
        SEER_MARK(20);
        fence_async_shared();
        SEER_MARK(21);
        tc_fence_before();
        if (!dead) {
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bars.go[rg]);
            mbar_arrive(&bars.kfull[(rg + kSBuf) % kRing]);  // S^T(g)'s buffer is free for QK(g+3)
          }
          ++arrived;
        }
        if (++rg == kRing) {
          rg = 0;
          rph ^= 1;
        }
        sb = sb + 1 == kSBuf ? 0 : sb + 1;
        ps = ps + 1 == kPSlots ? 0 : ps + 1;
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
      // the unit's last step is the one before the current ring position
      const bool okPV = mbar_wait(&bars.pv_done[rg > 0 ? rg - 1 : kRing - 1], rg > 0 ? rph : rph ^ 1, abort_p,
                                  p.status, tmo);
      float* red = &C.red[wgi][red_use & 1][0][0];
      float lpart[kCols];
#pragma unroll
      for (int q = 0; q < kCols / 2; ++q) f32x2_unpack(lp2[q], lpart[2 * q], lpart[2 * q + 1]);
      warp_reduce_scatter16<true>(lpart, lane, red + ww * kCols);
      ++red_use;
      if (bar_red_or(bar_id, 128, !okPV || dead)) break;
      float l[kCols];
      col_combine<true>(red, l);
      tc_fence_after();
      {
        uint32_t o[16];
        tmem_ld16(lane_addr + kColO + q0, o);
        tmem_wait_ld();
        // The column maximum stays at the unit's first step's: no rescale, no
        // per-step barrier.  Scores far above it can overflow P, the column
        // sums or O; such a unit is recomputed exactly by the fallback kernel
        // (one list entry per unit: the first warp to see it appends it).
        bool bad = false;
#pragma unroll
        for (int q = 0; q < 16; ++q) bad = bad || !(fabsf(__uint_as_float(o[q])) <= 3.0e38f) || !(l[q] <= 3.0e38f);
        if (__any_sync(0xffffffffu, bad) && !dead && lane == 0 && atomicExch(&C.redo_unit, w) != w) {
          const uint32_t e = atomicAdd(p.redo_count, 1u);
          if (e < (uint32_t)p.redo_cap) p.redo_list[e] = w;
        }
        if (tl < p.d) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            // l >= 1: the column's maximum contributes exp2(0)
            const float v = __uint_as_float(o[q]) * rcp_approx(l[q]);
            const long long idx = (orow0 + q) * p.d + tl;
            if (p.out_fp32)
              reinterpret_cast<float*>(p.O)[idx] = v;
            else
              reinterpret_cast<__nv_bfloat16*>(p.O)[idx] = __float2bfloat16_rn(v);
          }
        }
      }
      if (tl < kCols && p.lse) {
        float m[kCols];
#pragma unroll
        for (int q = 0; q < kCols / 2; ++q) f32x2_unpack(nm2[q], m[2 * q], m[2 * q + 1]);
        float mq = -m[0], lq = l[0];
#pragma unroll
        for (int q = 1; q < kCols; ++q)
          if (q == tl) {
            mq = -m[q];
            lq = l[q];
          }
        p.lse[orow0 + tl] = (mq + lg2_approx(lq)) * 0.6931471805599453f;
      }
#ifdef SEER_TRACE
      if (lane == 0) SEER_TRACE_ADD(10, clock64() - tep0);
#endif
      step += T;
    }
    if (lane == 0) C.sm_steps[warp] = arrived;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpPV) tmem_dealloc(tmem, kTmemCols);
  // After an abort, bulk copies may still be in flight into shared memory.
  // Every warp has left its loop, so the arrivals each barrier still lacks
  // are known exactly: kfull(h) waits for the softmax warps' release of step
  // h-3, go(h) for their P^T of step h.  Make those arrivals here; each
  // phase the loaders armed then completes exactly when its copies have
  // landed, which the teardown waits for (bounded) before the CTA exits.
  // A loader arms kfull(h) only after QK(h-2) and go(h) only after PV(h-3),
  // so only the last two kfull and last three go phases can be open.
  if (threadIdx.x == 0 && *abort_p) {
    const int hk = C.armed_k, hv = C.armed_v;
    for (int h = hk - kKSlots > 0 ? hk - kKSlots : 0; h < hk; ++h) {
      if (h >= kSBuf)
        for (int w2 = 0; w2 < kSoftmaxWarps; ++w2)
          if (C.sm_steps[w2] <= h - kSBuf) mbar_arrive(&bars.kfull[h % kRing]);
      mbar_wait_teardown(&bars.kfull[h % kRing], (h / kRing) & 1, 20000000ull);
    }
    for (int h = hv - kVSlots > 0 ? hv - kVSlots : 0; h < hv; ++h) {
      for (int w2 = 0; w2 < kSoftmaxWarps; ++w2)
        if (C.sm_steps[w2] <= h) mbar_arrive(&bars.go[h % kRing]);
      mbar_wait_teardown(&bars.go[h % kRing], (h / kRing) & 1, 20000000ull);
    }
  }
#ifdef SEER_TRACE
  if (threadIdx.x == 0) {
    C.trace[11] = clock64() - t_kernel0;
    for (int k = 0; k < 24; ++k) atomicAdd(p.trace + k, C.trace[k]);
  }
#endif
}


// ---------------------------------------------------------------- re-layout --
// Writes K^T of every (batch, KV head, key block j) as one contiguous record
// of d rows x 64 bf16 (128-byte rows): row c holds K[64j + 0 .. 63][c].  The
// block is read with 16-byte loads into a padded shared tile, then written 8
// keys (16 bytes) per store.  fp32 inputs are rounded to bf16 here (round to
// nearest even).
template <typename T>
__global__ void __launch_bounds__(256) kt_tile_kernel(const T* __restrict__ K, __nv_bfloat16* __restrict__ out,
                                                      int n, int d, const uint32_t* __restrict__ run_if) {
  __shared__ uint16_t sk[64][128 + 2];  // [key][dim]; 260-byte rows keep the column reads spread over banks
  if (run_if && *run_if == 0u) return;  // the dense kernel takes this call
  const int nb = n / kBlock;
  const long long rec = blockIdx.x;  // (b*Hkv + g)*nb + j
  const long long bg = rec / nb;
  const int j = (int)(rec % nb);
  const T* Kt = K + (bg * n + (long long)j * kBlock) * d;
  __nv_bfloat16* o = out + rec * (long long)d * 64;
  constexpr int EPL = 16 / sizeof(T);  // elements per 16-byte load
  for (int e = threadIdx.x; e < 64 * d / EPL; e += blockDim.x) {
    const int r = e / (d / EPL), c = (e % (d / EPL)) * EPL;
    const uint4 v = *reinterpret_cast<const uint4*>(Kt + (long long)r * d + c);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&sk[r][c]);  // c even: 4-byte aligned
    if constexpr (sizeof(T) == 2) {
      dst[0] = v.x;
      dst[1] = v.y;
      dst[2] = v.z;
      dst[3] = v.w;
    } else {
      const float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w)};
      dst[0] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[0])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[1])) << 16);
      dst[1] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[3])) << 16);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < d * 8; e += blockDim.x) {
    const int c = e / 8, k0 = (e % 8) * 8;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = (uint32_t)sk[k0 + 2 * q][c] | ((uint32_t)sk[k0 + 2 * q + 1][c] << 16);
    *reinterpret_cast<uint4*>(o + (long long)c * 64 + k0) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Units whose list is empty (count <= 0) get O = 0 and LSE = -inf here; the
// attention kernel never schedules them.  One warp per unit.
__global__ void __launch_bounds__(256) empty_rows_kernel(const int32_t* __restrict__ counts, void* O, float* lse,
                                                         int out_fp32, long long units, int d) {
  const long long u = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (u >= units || counts[u] > 0) return;
  const long long elems = 64LL * d;  // the unit's 64 rows of O
  if (out_fp32) {
    float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(O) + u * elems);
    for (long long e = lane; e < elems / 4; e += 32) o[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(O) + u * elems);
    for (long long e = lane; e < elems / 8; e += 32) o[e] = make_uint4(0, 0, 0, 0);
  }
  if (lse) {
    lse[u * 64 + lane] = -INFINITY;
    lse[u * 64 + 32 + lane] = -INFINITY;
  }
}

// Exact recomputation of the units the attention kernel flagged: plain fp32
// online softmax that rescales at every key, one warp per query row, lanes
// splitting the head dimension.  It reads the same bf16 Q, K^T records and
// V as the attention kernel (so fp32 inputs see the same rounding), and the
// same checked list entries.  Slow by design: it only runs for units whose
// scores rise so far above the unit's first-step maximum that the attention
// kernel's fp32 / bf16 values overflowed (or, in the training forward,
// rose more than 2^64 above the row's first-step maximum).
template <int D, bool KT>
__global__ void __launch_bounds__(256) sparse_attn_redo_kernel(const __nv_bfloat16* __restrict__ Q16,
                                                               const __nv_bfloat16* __restrict__ Kt16,
                                                               const __nv_bfloat16* __restrict__ V16,
                                                               const AttnParams p) {
  constexpr int DL = D / 32;  // head dims per lane
  __shared__ float lse2s[64];  // the unit's row LSEs (log2), for the map
  if (p.run_if && ((*p.run_if != 0u) != (p.run_if_value != 0u))) return;  // the other path's fallback
  const uint32_t nredo = min(*reinterpret_cast<volatile uint32_t*>(p.redo_count), (uint32_t)p.redo_cap);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  for (uint32_t e = blockIdx.x; e < nredo; e += gridDim.x) {
    const int w = p.redo_list[e];
    const UnitInfo u = decode_unit(p, w);
    const int* lst = p.indices + u.u * p.cap;
    const long long rec0 = ((long long)u.b * p.Hkv + u.g) * p.nb;
    for (int r = warp; r < 64; r += 8) {
      const long long qrow = ((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64 + r;
      float q[DL], o[DL];
#pragma unroll
      for (int k = 0; k < DL; ++k) {
        q[k] = __bfloat162float(Q16[qrow * D + lane * DL + k]);
        o[k] = 0.f;
      }
      float m = -INFINITY, l = 0.f;
      int prev = -1;
      for (int t = 0; t < u.count; ++t) {
        const int raw = p.dense ? t : lst[t];
        const int j = checked_entry(p, u, raw, prev);
        prev = raw;
        const __nv_bfloat16* rec = Kt16 + (rec0 + j) * (D * 64LL);  // K^T: [dim][key], or K: [key][dim]
        const __nv_bfloat16* vb = V16 + (rec0 + j) * (64LL * D);    // V: [key][dim]
        const int kmax = j == u.i ? r : 63;  // causal inside the diagonal block
        for (int key = 0; key <= kmax; ++key) {
          float sdot = 0.f;
#pragma unroll
          for (int k = 0; k < DL; ++k)
            sdot += q[k] * __bfloat162float(KT ? rec[(lane * DL + k) * 64 + key] : rec[key * D + lane * DL + k]);
          const float sc = warp_sum(sdot) * p.scale_log2;
          const float mn = fmaxf(m, sc);
          const float a = exp2f(m - mn), pr = exp2f(sc - mn);
          l = l * a + pr;
#pragma unroll
          for (int k = 0; k < DL; ++k) {
            const int dim = lane * DL + k;
            const float v = __bfloat162float(vb[key * D + dim]);
            o[k] = o[k] * a + pr * v;
          }
          m = mn;
        }
      }
#pragma unroll
      for (int k = 0; k < DL; ++k) {
        const float v = o[k] / l;
        const long long idx = qrow * D + lane * DL + k;
        if (p.out_fp32)
          reinterpret_cast<float*>(p.O)[idx] = v;
        else
          reinterpret_cast<__nv_bfloat16*>(p.O)[idx] = __float2bfloat16_rn(v);
      }
      if (lane == 0 && p.lse) p.lse[qrow] = (m + log2f(l)) * 0.6931471805599453f;
      if (lane == 0) lse2s[r] = m + log2f(l);
    }
    if (p.map) {
      // the unit's map row, exactly: for each listed key block, the largest
      // probability exp2(score - lse2) over the 64 rows and the block's keys
      __syncthreads();
      for (int t = warp; t < u.count; t += 8) {
        int j = p.dense ? t : lst[t];
        j = j < 0 ? 0 : (j > u.i ? u.i : j);
        const __nv_bfloat16* rec = Kt16 + (rec0 + j) * (D * 64LL);
        float best = 0.f;
        for (int r = 0; r < 64; ++r) {
          const long long qrow = ((long long)u.b * p.Hq + u.hq) * p.n + (long long)u.i * 64 + r;
          float q[DL];
#pragma unroll
          for (int k = 0; k < DL; ++k) q[k] = __bfloat162float(Q16[qrow * D + lane * DL + k]);
          const int kmax = j == u.i ? r : 63;
          for (int key = 0; key <= kmax; ++key) {
            float sdot = 0.f;
#pragma unroll
            for (int k = 0; k < DL; ++k)
              sdot += q[k] * __bfloat162float(KT ? rec[(lane * DL + k) * 64 + key] : rec[key * D + lane * DL + k]);
            best = fmaxf(best, exp2f(warp_sum(sdot) * p.scale_log2 - lse2s[r]));
          }
        }
        if (lane == 0) p.map[u.u * p.nb + j] = best;
      }
      __syncthreads();
    }
  }
}

cudaError_t launch_sparse_attn_redo(const void* Q16, const void* Kt16, const void* V16, const AttnParams& p,
                                    cudaStream_t st) {
  const auto q = (const __nv_bfloat16*)Q16;
  const auto kt = (const __nv_bfloat16*)Kt16;
  const auto v = (const __nv_bfloat16*)V16;
  if (p.k_rows) {
    if (p.d == 64)
      sparse_attn_redo_kernel<64, false><<<148, 256, 0, st>>>(q, kt, v, p);
    else
      sparse_attn_redo_kernel<128, false><<<148, 256, 0, st>>>(q, kt, v, p);
  } else {
    if (p.d == 64)
      sparse_attn_redo_kernel<64, true><<<148, 256, 0, st>>>(q, kt, v, p);
    else
      sparse_attn_redo_kernel<128, true><<<148, 256, 0, st>>>(q, kt, v, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_empty_rows(const AttnParams& p, cudaStream_t st) {
  const long long blocks = (p.total_units + 7) / 8;
  empty_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(p.counts, p.O, p.lse, p.out_fp32, p.total_units, p.d);
  return cudaGetLastError();
}

__global__ void dense_check_kernel(const int32_t* __restrict__ counts, long long units, int nb,
                                   uint32_t* __restrict__ not_dense) {
  bool bad = false;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units; u += (long long)gridDim.x * blockDim.x)
    bad = bad || counts[u] != (int)(u % nb) + 1;
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) *not_dense = 1u;
}

cudaError_t launch_dense_check(const int32_t* counts, long long units, int nb, uint32_t* not_dense, cudaStream_t st) {
  long long blocks = (units + 255) / 256;
  if (blocks > 592) blocks = 592;
  dense_check_kernel<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, st>>>(counts, units, nb, not_dense);
  return cudaGetLastError();
}

cudaError_t launch_kt_tiles(const void* K, bool fp32, void* out, long long records, int n, int d, cudaStream_t st,
                            const uint32_t* run_if) {
  if (fp32)
    kt_tile_kernel<float><<<(unsigned)records, 256, 0, st>>>((const float*)K, (__nv_bfloat16*)out, n, d, run_if);
  else
    kt_tile_kernel<uint16_t><<<(unsigned)records, 256, 0, st>>>((const uint16_t*)K, (__nv_bfloat16*)out, n, d, run_if);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKt, const CUtensorMap& tmV, const AttnParams& p,
                               int num_sms, cudaStream_t st) {
  auto kern = p.d == 64 ? sparse_attn_kernel<64> : sparse_attn_kernel<128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)attn::kSmemAlloc);
  if (e != cudaSuccess) return e;
  long long grid = p.total_units < num_sms ? p.total_units : num_sms;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, attn::kThreads, attn::kSmemAlloc, st>>>(tmQ, tmKt, tmV, p);
  return cudaGetLastError();
}

}  // namespace seer
