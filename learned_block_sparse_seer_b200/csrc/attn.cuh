// attn.cuh -- parameters and launcher of the block-sparse attention kernel.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace seer {

struct AttnParams {
  int B, Hq, Hkv, n, d, nb, G, cap;
  long long total_units;     // B * Hq * nb
  const int32_t* counts;     // [B, Hq, nb]
  const int32_t* indices;    // [B, Hq, nb, cap]
  int dense;                 // exact fallback of the training forward: every causal block (count = i+1, entry t = t); lists not read
  void* O;                   // [B, Hq, n, d] bf16 or fp32
  float* lse;                // [B, Hq, n] or null
  int out_fp32;              // O element type
  float scale_log2;          // softmax scale * log2(e)
  uint32_t* status;          // workspace status word
  uint32_t* work_counter;    // workspace work counter (zeroed per call)
  unsigned long long timeout_ns;
  unsigned long long* trace;  // 16 cycle counters (only with -DSEER_TRACE)
  uint32_t* redo_count;       // units flagged for the exact fallback (workspace)
  int* redo_list;             // [redo_cap] flagged unit indices
  int redo_cap;
  float* map;          // exact fallback of the training forward: [B*Hq*nb, nb] map rows to rewrite, or null
  int test_skip_qk_commit;  // test hook: step whose QK completion is never signalled (-1: none)
  int k_rows;               // exact fallback only: K given as rows [B*Hkv*n, d] instead of K^T records
  // Device-side choice between this kernel and the 128-row dense kernel: when
  // run_if is non-null the launch does nothing unless (*run_if != 0) equals
  // run_if_value (the word is set by launch_dense_check).
  const uint32_t* run_if;
  uint32_t run_if_value;
};

// *not_dense = 1 unless every unit's count is i + 1 (with ascending entries
// in [0, i], a list of i + 1 entries is then exactly 0..i: the all-ones
// causal mask).  The word must be 0 before the launch.
cudaError_t launch_dense_check(const int32_t* counts, long long units, int nb, uint32_t* not_dense, cudaStream_t st);

// Re-layout of K into per-block K^T records of d rows x 64 bf16;
// `records` = B * Hkv * n/64.
// With run_if non-null the pass is skipped when *run_if == 0 (the dense path
// of launch_dense_check's choice needs no records).
cudaError_t launch_kt_tiles(const void* K, bool fp32, void* out, long long records, int n, int d, cudaStream_t st,
                            const uint32_t* run_if = nullptr);

// Exact fp32 recomputation of the units the attention kernel flagged (scores
// so far above the unit's first-step column maximum that its values
// overflowed; in the training forward, more than 2^64 above the row's);
// returns at once when none was.  Q16 is the bf16 Q the attention kernel
// read, Kt16 the K^T records (or, with p.k_rows, the bf16 K rows) and V16 the
// bf16 V [B*Hkv*n, d].  Launch after launch_sparse_attn (or launch_fwd).
cudaError_t launch_sparse_attn_redo(const void* Q16, const void* Kt16, const void* V16, const AttnParams& p,
                                    cudaStream_t st);

// O = 0 and LSE = -inf for every unit whose list is empty (count <= 0); the
// attention kernel skips those units.  Launch before launch_sparse_attn.
cudaError_t launch_empty_rows(const AttnParams& p, cudaStream_t st);

// Persistent launch: one CTA per SM (at most one per unit).  tmQ is a 3-D
// bf16 map over Q (64 dims, B*Hq*n rows, d/64 panels) with a 64 x 64 x d/64
// box; tmKt a 2-D bf16 map over the
// K^T records [records * d, 64] with a d-row box; tmV a 3-D bf16 map over V
// (64 dims, B*Hkv*n rows, d/64 panels) with a 64 x 64 x d/64 box; all
// 128-byte swizzled.
cudaError_t launch_sparse_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKt, const CUtensorMap& tmV,
                               const AttnParams& p, int num_sms, cudaStream_t st);

}  // namespace seer
