// attn_tf32.cu -- block-sparse causal attention for fp32 Q/K/V on the tf32
// tensor cores (tcgen05 kind::tf32), for callers who want fp32 I/O without
// the bf16 rounding of the main kernel.
//
// Paper: "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs";
// paper-graph summary page, section 3.4, "Block-sparse FlashAttention kernel":
// for query block i only the listed key blocks take part, causal inside the
// diagonal block, online softmax, O and the row log-sum-exp.
//
// Design (one CTA per unit = (batch, query head, 64-row query block)):
//  * Operands come straight from the fp32 tensors by TMA (no conversion): a
//    3-D tensor map reads a [rows, d] tensor as 32-float panels, so one copy
//    brings a whole 64-row tile (d/32 panels of 64 rows x 128 bytes, 128-byte
//    swizzle); copies of 8 KB or less cost about as much per copy as 32 KB.
//  * S = Q K^T per key block: tcgen05 kind::tf32, M = 64 query rows, N = 64
//    keys, K = d (8 per instruction); A and B K-major.  With M = 64 the rows
//    sit in TMEM lanes 0-15 of each 32-lane sub-partition (row r at lane
//    r % 16 + 32 (r / 16)), so each softmax warp owns 16 rows, two threads
//    per row: the .16x32bx2 TMEM load gives each half-warp 32 of the 64 keys.
//  * P stays on chip: the softmax writes it (fp32 values, read by the tensor
//    core as tf32) over S in TMEM, and O += P V runs with A = P from TMEM
//    (M = 64, the layout of S) and B = V^T from shared memory (N = d, K = 64
//    keys, K-major: V is first transposed per 64-key block into the
//    workspace by vt_kernel, since kind::tf32 reads K-major operands only).
//  * O is a 64 x d accumulator in TMEM in the same row layout, so a row's
//    rescale (its running maximum is raised lazily, by more than 8 in log2
//    units) is done by the two threads that own the row, and the softmax
//    warps never wait for one another.
//  * Three S / P buffers in TMEM: QK of block t+1 and t+2 and PV of block t-1
//    can run while the softmax works on block t.
//  * Warp roles (256 threads): warps 0-3 softmax and epilogue (TMEM
//    sub-partitions 0-3), warp 4 loads Q and K (three K stages, freed by
//    QK), warp 5 issues the QK products, warp 6 loads V^T (three stages,
//    freed by PV), warp 7 issues the PV products.  With one issuer per
//    product, QK runs ahead into free S buffers while PV waits for the
//    softmax.  Every wait is bounded; a wait that gives up raises the CTA's abort
//    flag, so every other wait of the CTA gives up too.
#include <cmath>
#include <cstdint>

#include "attn_tf32.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "tf32mma.cuh"

namespace seer {

namespace tf32a {
constexpr int kThreads = 256;
constexpr int kWarpLoad = 4, kWarpQK = 5, kWarpLoadV = 6, kWarpPV = 7;
constexpr int kKS = 3, kVS = 3;  // K and V^T stages
constexpr int kSB = 3;           // S / P buffers in TMEM
constexpr uint32_t kPanel = 64u * 128u;  // 64 rows x 32 floats
constexpr uint32_t kTmemCols = 512;      // S / P x 3 (64 cols each), O (d cols from kColO)
constexpr uint32_t kColO = 256;
constexpr float kRaise = 8.0f;

template <int D>
struct Layout {
  static constexpr int P = D / 32;                  // 32-float panels per row
  static constexpr uint32_t kTile = P * kPanel;     // a 64-row tile of d floats
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kTile;                  // kKS K tiles
  static constexpr uint32_t kOffV = kOffK + kKS * kTile;     // kVS V^T tiles
  static constexpr uint32_t kSmem = kOffV + kVS * kTile;
  static constexpr uint32_t kVtPanel = (uint32_t)D * 128u;  // V^T: d rows x 32 keys
};

struct Ctrl {
  uint64_t q_full, k_full[kKS], k_empty[kKS], v_full[kVS], v_empty[kVS], s_full[kSB], p_full[kSB], pv_done[kSB];
  uint64_t fin_qk, fin_pv;
  uint32_t tmem_base;
  int abort_flag;
};

// The .16x32bx2 shape: threads 0-15 read TMEM lanes 0-15 of the warp's
// sub-partition at 32 consecutive columns from taddr's column, threads 16-31
// the same lanes at 32 columns from taddr's column + OFF.  (The layout of an
// M = 64 accumulator: its rows sit in lanes 0-15 of each sub-partition, so a
// warp covers 16 rows with all 32 threads, two threads per row.)
template <int OFF>
__device__ __forceinline__ void tmem_ld32_halves(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(OFF)
      : "memory");
}

// The store of the same shape and layout as tmem_ld32_halves.
template <int OFF>
__device__ __forceinline__ void tmem_st32_halves(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], %1, "
      "{%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
      "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33};" ::"r"(taddr),
      "n"(OFF), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// The thread's half of its O row in TMEM (row 16 w + l % 16 of warp w, lane
// l): columns (l / 16) d/2 .. + d/2, in two (d = 128) or one (d = 64)
// 32-column pieces.
template <int D>
__device__ __forceinline__ void o_load(uint32_t taddr, uint32_t (&a)[32], uint32_t (&b)[32]) {
  if constexpr (D == 128) {
    tmem_ld32_halves<64>(taddr, a);
    tmem_ld32_halves<64>(taddr + 32u, b);
  } else {
    tmem_ld32_halves<32>(taddr, a);
  }
}
template <int D>
__device__ __forceinline__ void o_store(uint32_t taddr, const uint32_t (&a)[32], const uint32_t (&b)[32]) {
  if constexpr (D == 128) {
    tmem_st32_halves<64>(taddr, a);
    tmem_st32_halves<64>(taddr + 32u, b);
  } else {
    tmem_st32_halves<32>(taddr, a);
  }
}

// The list entry t of a unit, checked: an entry outside 0..i is recorded
// and replaced by the diagonal block.
__device__ __forceinline__ int entry(const Tf32AttnParams& p, long long unit, int i, int t) {
  int j = p.indices[unit * p.cap + t];
  if (j < 0 || j > i) {
    record_status(p.status, kDevBadIndex, (uint32_t)unit);
    j = i;
  }
  return j;
}
}  // namespace tf32a

template <int D>
__global__ void __launch_bounds__(tf32a::kThreads, 1)
    attn_tf32_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Tf32AttnParams p) {
  using namespace tf32a;
  using L = Layout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(p.status, kDevBadSchedule, smem_u32(smem));
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long unit = blockIdx.x;  // (b * Hq + hq) * nb + i
  const int i = (int)(unit % p.nb);
  const long long bh = unit / p.nb;
  const long long b = bh / p.Hq;
  const int hq = (int)(bh % p.Hq), g = hq / (p.Hq / p.Hkv);
  const long long qrow0 = bh * p.n + (long long)i * kBlock;
  int cnt = p.counts[unit];
  const int lim = min(p.cap, i + 1);
  if (cnt < 0 || cnt > lim) {
    if (threadIdx.x == 0) record_status(p.status, kDevBadIndex, (uint32_t)unit);
    cnt = cnt < 0 ? 0 : lim;
  }
  Ctrl& C = *reinterpret_cast<Ctrl*>(smem + L::kSmem);
  float* O = p.O;
  if (cnt == 0) {  // no admissible key: O = 0, LSE = -inf
    for (int x = threadIdx.x; x < kBlock * D; x += kThreads) O[qrow0 * D + x] = 0.f;
    if (p.lse)
      for (int x = threadIdx.x; x < kBlock; x += kThreads) p.lse[qrow0 + x] = -INFINITY;
    return;
  }
  volatile int* abort_p = &C.abort_flag;
  const uint64_t tmo = p.timeout_ns;
  if (threadIdx.x == 0) {
    C.abort_flag = 0;
    mbar_init(&C.q_full, 1);
    for (int s = 0; s < kKS; ++s) {
      mbar_init(&C.k_full[s], 1);
      mbar_init(&C.k_empty[s], 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(&C.v_full[s], 1);
      mbar_init(&C.v_empty[s], 1);
    }
    for (int s = 0; s < kSB; ++s) {
      mbar_init(&C.s_full[s], 1);
      mbar_init(&C.p_full[s], 4);
      mbar_init(&C.pv_done[s], 1);
    }
    mbar_init(&C.fin_qk, 1);
    mbar_init(&C.fin_pv, 1);
    fence_barrier_init();
  }
  if (warp == kWarpQK) {
    tmem_alloc(&C.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;

  if (warp == kWarpLoad) {
    // ----------------------------------------------- producer: Q, K ---
    // K tiles free as soon as their QK is done, V^T tiles only after PV:
    // separate rings and separate producers, so a V^T slot never holds up K.
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      mbar_arrive_expect_tx(&C.q_full, L::kTile);
      tma_load_3d(smem + L::kOffQ, &tmQ, &C.q_full, 0, (int)qrow0, 0);
      const long long krow0 = (b * p.Hkv + g) * p.n;
      int t = 0;
      for (; t < cnt; ++t) {
        const int s = t % kKS;
        if (t >= kKS && !mbar_wait(&C.k_empty[s], ((t / kKS) - 1) & 1, abort_p, p.status, tmo)) break;
        const int j = tf32a::entry(p, unit, i, t);
        mbar_arrive_expect_tx(&C.k_full[s], L::kTile);
        tma_load_3d(smem + L::kOffK + (uint32_t)s * L::kTile, &tmK, &C.k_full[s], 0,
                    (int)(krow0 + (long long)j * kBlock), 0);
      }
      // copies in flight land before the CTA exits
      wait_landed(&C.q_full, 0);
      for (int k = t > kKS ? t - kKS : 0; k < t; ++k)
        wait_landed(&C.k_full[k % kKS], (k / kKS) & 1);
    }
  } else if (warp == kWarpLoadV) {
    // --------------------------------------------------- producer: V^T ---
    if (lane == 0) {
      prefetch_tmap(&tmV);
      int t = 0;
      for (; t < cnt; ++t) {
        const int s = t % kVS;
        if (t >= kVS && !mbar_wait(&C.v_empty[s], ((t / kVS) - 1) & 1, abort_p, p.status, tmo)) break;
        const int j = tf32a::entry(p, unit, i, t);
        // V^T block of this key block: d rows of 64 keys in the workspace
        mbar_arrive_expect_tx(&C.v_full[s], L::kTile);
        tma_load_3d(smem + L::kOffV + (uint32_t)s * L::kTile, &tmV, &C.v_full[s], 0,
                    (int)(((b * p.Hkv + g) * p.nb + j) * (long long)D), 0);
      }
      for (int k = t > kVS ? t - kVS : 0; k < t; ++k)
        wait_landed(&C.v_full[k % kVS], (k / kVS) & 1);
    }
  } else if (warp == kWarpQK) {
    // ----------------------------------------------------- QK issuer ---
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_tf32(64, 64, 0, 0);  // A = Q, B = K (both K-major)
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dQ = make_sw128_desc(sbase + L::kOffQ, 16, 1024);
      bool ok = mbar_wait(&C.q_full, 0, abort_p, p.status, tmo);
      for (int t = 0; ok && t < cnt; ++t) {
        const int sb = t % kSB, ks = t % kKS;
        if (!mbar_wait(&C.k_full[ks], (t / kKS) & 1, abort_p, p.status, tmo)) break;
        // S / P buffer sb held P(t - kSB): free once that block's PV is done
        if (t >= kSB && !mbar_wait(&C.pv_done[sb], ((t / kSB) - 1) & 1, abort_p, p.status, tmo)) break;
        tc_fence_after();
        const uint64_t dK = make_sw128_desc(sbase + L::kOffK + (uint32_t)ks * L::kTile, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 8; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kPanel + (kk & 3) * 32) >> 4);
          mma_tf32_ss(tmem + (uint32_t)sb * 64u, dQ + off, dK + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&C.s_full[sb]);
        mma_commit(&C.k_empty[ks]);
      }
      mma_commit(&C.fin_qk);
      wait_landed(&C.fin_qk, 0);
    }
  } else if (warp == kWarpPV) {
    // ----------------------------------------------------- PV issuer ---
    if (lane == 0) {
      constexpr uint32_t idesc_pv = make_idesc_tf32(64, D, 0, 0);  // A = P (TMEM), B = V^T (K-major)
      const uint32_t sbase = smem_u32(smem);
      for (int u = 0; u < cnt; ++u) {
        const int vs = u % kVS, ub = u % kSB;
        if (!mbar_wait(&C.v_full[vs], (u / kVS) & 1, abort_p, p.status, tmo)) break;
        if (!mbar_wait(&C.p_full[ub], (u / kSB) & 1, abort_p, p.status, tmo)) break;
        tc_fence_after();
        // V^T, K-major: d rows of 32 keys per panel, two panels; P: one
        // TMEM column per key
        const uint64_t dV = make_sw128_desc(sbase + L::kOffV + (uint32_t)vs * L::kTile, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32_ts(tmem + kColO, tmem + (uint32_t)ub * 64u + (uint32_t)(8 * kk),
                      dV + (uint64_t)(((kk >> 2) * L::kVtPanel + (kk & 3) * 32) >> 4), idesc_pv,
                      (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&C.pv_done[ub]);
        mma_commit(&C.v_empty[vs]);
      }
      mma_commit(&C.fin_pv);
      wait_landed(&C.fin_pv, 0);
    }
  } else {
    // ------------------------------------------- softmax and epilogue ---
    // Warp ww owns query rows 16 ww .. 16 ww + 15 (lanes 0-15 of its TMEM
    // sub-partition), two threads per row: thread l takes row 16 ww + l % 16
    // and keys 32 hf .. 32 hf + 31 of each block, hf = l / 16, and the
    // same half of the row's d columns of O.
    const int ww = warp;
    const bool row_thread = lane < 16;
    const int hf = lane >> 4;
    const int q = 16 * ww + (lane & 15);
    const uint32_t lane_base = tmem + ((uint32_t)(ww * 32) << 16);
    const float c = p.scale_log2;
    const uint64_t c2 = f32x2_pack(c, c);
    // m: the row's running maximum (the same in both threads of a row);
    // l: this thread's half of the row sum, scaled as m rises
    float m = -INFINITY, l = 0.f;
    // lists ascend with every entry <= i, so only the last can be the
    // diagonal block (a bad entry reads as the diagonal, as the producers do)
    const int last_j = tf32a::entry(p, unit, i, cnt - 1);
    bool ok = true;
    for (int t = 0; t < cnt; ++t) {
      const int s = t % kSB;
      const int j = t == cnt - 1 ? last_j : -1;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&C.s_full[s], (t / kSB) & 1, abort_p, p.status, tmo));
      uint32_t r0[32];
      if (ok) {
        tc_fence_after();
        tmem_ld32_halves<32>(lane_base + (uint32_t)s * 64u, r0);
        tmem_wait_ld();
      }
      // scores in log2 units, two at a time (packed f32x2)
      float x[32];
#pragma unroll
      for (int k = 0; k < 16; ++k)
        f32x2_unpack(mul_f32x2(f32x2_pack(__uint_as_float(r0[2 * k]), __uint_as_float(r0[2 * k + 1])), c2), x[2 * k],
                     x[2 * k + 1]);
      if (j == i) {  // causal rule inside the diagonal block
#pragma unroll
        for (int k = 0; k < 32; ++k) x[k] = 32 * hf + k > q ? -INFINITY : x[k];
      }
      // row maximum: a tree of 3-input maxima over this thread's 32 keys,
      // then the other half of the row
      float t1[11];
#pragma unroll
      for (int k = 0; k < 10; ++k) t1[k] = fmax3(x[3 * k], x[3 * k + 1], x[3 * k + 2]);
      t1[10] = fmaxf(x[30], x[31]);
      const float mh = fmaxf(fmax3(fmax3(t1[0], t1[1], t1[2]), fmax3(t1[3], t1[4], t1[5]), fmax3(t1[6], t1[7], t1[8])),
                             fmaxf(t1[9], t1[10]));
      const float mx = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));
      float alpha = 1.f;
      bool raise = false;
      if (mx > m + kRaise) {
        if (t > 0) {
          alpha = ex2_approx(m - mx);
          raise = true;
        }
        l *= alpha;
        m = mx;
      }
      // probabilities, and their sum by a tree of packed adds
      const uint64_t nm2 = f32x2_pack(-m, -m);
      uint64_t acc[8];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float a, bb;
        f32x2_unpack(add_f32x2(f32x2_pack(x[2 * k], x[2 * k + 1]), nm2), a, bb);
        x[2 * k] = ex2_approx(a);
        x[2 * k + 1] = ex2_approx(bb);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
        acc[k] = add_f32x2(f32x2_pack(x[4 * k], x[4 * k + 1]), f32x2_pack(x[4 * k + 2], x[4 * k + 3]));
#pragma unroll
      for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int k = 0; k < w2; ++k) acc[k] = add_f32x2(acc[k], acc[k + w2]);
      float s0, s1;
      f32x2_unpack(acc[0], s0, s1);
      l += s0 + s1;
      // a raised row rescales its O row, after every PV so far (PV(t-1) and
      // before) has landed; the warp's rows share the TMEM access
      if (__any_sync(0xffffffffu, raise)) {
        const int u = t - 1;  // raise implies t > 0
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&C.pv_done[u % kSB], (u / kSB) & 1, abort_p, p.status, tmo));
        if (ok) {
          tc_fence_after();
          uint32_t oa[32], ob[32];
          o_load<D>(lane_base + kColO, oa, ob);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            oa[k] = __float_as_uint(__uint_as_float(oa[k]) * alpha);
            if (D == 128) ob[k] = __float_as_uint(__uint_as_float(ob[k]) * alpha);
          }
          o_store<D>(lane_base + kColO, oa, ob);
        }
      }
      // P(t) over S(t): the A operand of PV(t)
      if (ok) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = __float_as_uint(x[k]);
        tmem_st32_halves<32>(lane_base + (uint32_t)s * 64u, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (!ok) break;
      if (lane == 0) mbar_arrive(&C.p_full[s]);
    }
    // ---- epilogue: O / l, LSE
    if (ok) {
      const int u = cnt - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&C.pv_done[u % kSB], (u / kSB) & 1, abort_p, p.status, tmo));
    }
    l += __shfl_xor_sync(0xffffffffu, l, 16);  // the row's two halves
    if (row_thread && p.lse) p.lse[qrow0 + q] = (m + log2f(l)) * 0.6931471805599453f;
    if (ok) {
      tc_fence_after();
      uint32_t oa[32], ob[32];
      o_load<D>(lane_base + kColO, oa, ob);
      tmem_wait_ld();
      const float linv = 1.0f / l;
      float* out = O + (qrow0 + q) * D + hf * (D / 2);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        reinterpret_cast<float4*>(out)[k] =
            make_float4(__uint_as_float(oa[4 * k]) * linv, __uint_as_float(oa[4 * k + 1]) * linv,
                        __uint_as_float(oa[4 * k + 2]) * linv, __uint_as_float(oa[4 * k + 3]) * linv);
        if (D == 128)
          reinterpret_cast<float4*>(out + 32)[k] =
              make_float4(__uint_as_float(ob[4 * k]) * linv, __uint_as_float(ob[4 * k + 1]) * linv,
                          __uint_as_float(ob[4 * k + 2]) * linv, __uint_as_float(ob[4 * k + 3]) * linv);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpQK) tmem_dealloc(tmem, kTmemCols);
}

// V^T per 64-key block: Vt[(bh * nb + j) * d + c][k] = V[bh][64 j + k][c].
__global__ void __launch_bounds__(256) vt_kernel(const float* __restrict__ V, float* __restrict__ Vt, int n, int d) {
  __shared__ float tile[64][129];
  const long long blk = blockIdx.x;  // bh * nb + j
  const int nb = n / kBlock;
  const long long bh = blk / nb;
  const int j = (int)(blk % nb);
  const float* src = V + (bh * n + (long long)j * kBlock) * d;
  for (int x = threadIdx.x; x < kBlock * d; x += 256) tile[x / d][x % d] = src[x];
  __syncthreads();
  float* dst = Vt + blk * (long long)d * kBlock;
  for (int x = threadIdx.x; x < kBlock * d; x += 256) dst[x] = tile[x % kBlock][x / kBlock];
}

cudaError_t launch_vt(const float* V, float* Vt, long long BHkv, int n, int d, cudaStream_t st) {
  vt_kernel<<<(unsigned)(BHkv * (n / kBlock)), 256, 0, st>>>(V, Vt, n, d);
  return cudaGetLastError();
}

cudaError_t launch_attn_tf32(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const Tf32AttnParams& p, cudaStream_t st) {
  auto kern = p.d == 64 ? attn_tf32_kernel<64> : attn_tf32_kernel<128>;
  const uint32_t smem =
      (p.d == 64 ? tf32a::Layout<64>::kSmem : tf32a::Layout<128>::kSmem) + (uint32_t)sizeof(tf32a::Ctrl);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)p.total_units, tf32a::kThreads, smem, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace seer
