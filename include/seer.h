/*
 * seer.h -- C ABI of the B200 (sm_100a) SeerAttention prefill library.
 *
 * The library implements the prefill hot path of "SeerAttention: Learning
 * Intrinsic Sparse Attention in Your LLMs" (arXiv 2410.13276):
 *   seer_gate           AttnGate block scorer + binary block-mask generation
 *   seer_gate_select    the mask-generation step alone, on supplied scores
 *   seer_sparse_attn    block-sparse causal attention over the selected blocks
 *   seer_attn_blockmax  2D max-pooled attention-probability map (the gate's
 *                       self-distillation target)
 *   seer_attn_forward_map  the training forward: dense causal O, LSE and the
 *                       max-pooled map in one pass
 *   seer_gate_kl_backward  one distillation step: KL(gt || score) and the
 *                       gradients of the gate's two linear layers
 *   seer_gate_varlen    the gate over variable-length sequences packed along
 *                       the token axis (then seer_sparse_attn as usual)
 *   seer_sparse_attn_tf32  the attention for fp32 inputs on the tf32 tensor
 *                       cores
 *   seer_gate_noalloc   seer_gate without a workspace
 *   seer_prefill_host   gate + attention for inputs and outputs in host
 *                       memory, the copies overlapped with the compute
 *   seer_decode_*       the decode stage: compressed K cache, token gate,
 *                       block-sparse decode attention, 1D ground truth
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller (except the
 *    host tensors of seer_prefill_host, named hQ, hK, hV, hO, hLSE).  The library
 *    allocates no device memory; scratch comes from the caller's workspace,
 *    whose size the matching *_workspace_size() call returns.  Workspace
 *    pointers must be 256-byte aligned.
 *  - Layout: every tensor is contiguous [B, H, n, d], row-major ("head-major").
 *    Query head hq uses KV head hq / (Hq / Hkv) (grouped-query attention).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronises.  Arguments are validated on the
 *    host before anything is launched; on any error nothing is written.
 *  - Device-side failures (a bounded wait that gave up, an index that failed a
 *    bounds check) are recorded in a status word at the start of the
 *    workspace.  seer_workspace_status() synchronises `stream` and reads it.
 *  - The library keeps no global state (except the per-thread copy streams of
 *    seer_prefill_host, the fixed buffer of seer_gate_noalloc and the
 *    per-thread test hook seer_testing_attn_wait_fault) and is safe to call
 *    from several host threads on different streams (each call with its own
 *    workspace).
 *  - The block size is fixed at 64 tokens (the pages fix B = 64 in all
 *    experiments: summary page, section 3.4, "Key Configuration Summary").
 */
#ifndef SEER_H
#define SEER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SEER_API __attribute__((visibility("default")))
#else
#define SEER_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *seer_stream_t; /* == cudaStream_t */

typedef enum {
  SEER_OK = 0,
  SEER_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, T <= 0, k < 1, ... */
  SEER_ERR_UNSUPPORTED = 2,   /* block != 64, d not in {64,128}, dtype, ...    */
  SEER_ERR_CAPACITY = 3,      /* cap smaller than the largest possible count  */
  SEER_ERR_CUDA = 4,          /* a CUDA runtime call failed; see
                                 seer_last_cuda_error()                        */
  SEER_ERR_TIMEOUT = 5,       /* device status: a bounded wait gave up        */
  SEER_ERR_DEVICE_CHECK = 6,  /* device status: an index failed its check     */
  SEER_ERR_WORKSPACE = 7      /* workspace null, misaligned or too small      */
} seer_status;

typedef enum { SEER_BF16 = 0, SEER_FP32 = 1 } seer_dtype;

typedef enum {
  /* Thresholding: block j is active iff score[i][j] > T (strict).
     Summary page, section 3.4, "Method 2: Thresholding"; rebuttal 3.3. */
  SEER_SELECT_THRESHOLD = 0,
  /* TopK with a uniform k: the k_i = min(k, i+1) largest scores of row i.
     Summary page, section 3.4, "Method 1: TopK selection". */
  SEER_SELECT_TOPK_K = 1,
  /* TopK with a density rho: k_i = clamp(ceil(rho*(i+1)), 1, i+1), the product
     rounded in fp32.  Gives block sparsity ~ 1 - rho on every causal row. */
  SEER_SELECT_TOPK_DENSITY = 2,
  /* Flag, OR-ed into any of the modes above: the diagonal block i always
     joins row i's list (the list is the mode's selection plus i), so no row
     is empty.  A top-k row may then hold k_i + 1 blocks.  (The pages do not
     force the diagonal; the flag is an option, off unless given.)  For the
     decode gate it changes nothing: the token's own block is always
     attended there. */
  SEER_SELECT_FORCE_DIAGONAL = 0x100
} seer_select_mode;

/* Problem shape.  n must be a multiple of `block`; Hq a multiple of Hkv. */
typedef struct {
  int32_t B;     /* batch                                   */
  int32_t Hq;    /* query heads                             */
  int32_t Hkv;   /* key/value heads                         */
  int32_t n;     /* sequence length (tokens), multiple of 64 */
  int32_t d;     /* head dimension: 64 or 128               */
  int32_t block; /* block size: must be 64                  */
} seer_dims;

/* ------------------------------------------------------------------------ */
/* seer_gate -- the AttnGate of SeerAttention plus mask generation.
 *
 * Computes, per query head and query block i (summary page, section 3.4,
 * "AttnGate", Eq. 1; pooling per "Pooling Method Selection"):
 *   qbar_i = mean of Q over block i                       [d]
 *   kbar_j = [max | min | mean] of K over block j         [3d]
 *   q~_i   = Wq[hq] qbar_i,   k~_j = Wk[g] kbar_j        [h]  (no bias)
 *   optional block RoPE on q~, k~ at block positions with base rope_theta/64
 *     (summary page, "Block-Level RoPE"; rope_theta <= 0 disables it)
 *   score[i][j] = softmax_{j <= i}( q~_i . k~_j / sqrt(d) ), 0 for j > i
 * then the active key blocks of every row as an ascending index list
 * (rebuttal, section 3.3: "torch.topk ... indices [S/B, k]").
 *
 *   Q         [B, Hq, n, d]  bf16 or fp32 (dtype)
 *   K         [B, Hkv, n, d] same dtype
 *   Wq        [Hq, h, d]     fp32
 *   Wk        [Hkv, h, 3d]   fp32, input features ordered [max | min | avg]
 *   h         gate hidden size, 1..256, multiple of 4
 *   mode/T/k/density   selection (see seer_select_mode); T > 0 for
 *             THRESHOLD, k >= 1 for TOPK_K, 0 < density <= 1 for TOPK_DENSITY
 *   scores_out  optional [B, Hq, nb, nb] fp32 (nb = n/64): the scores the
 *             selection used; entries j > i are written as 0.  May be NULL.
 *   counts    [B, Hq, nb] int32: number of active blocks of each row
 *   indices   [B, Hq, nb, cap] int32: ascending active key blocks of each row;
 *             entries past counts[row] are left untouched
 *   cap       row capacity; must be >= seer_gate_required_cap(...)
 *   ws/ws_bytes  workspace of at least seer_gate_workspace_size(...) bytes
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_CAPACITY,
 *         SEER_ERR_WORKSPACE, SEER_ERR_CUDA.                               */
SEER_API seer_status seer_gate(const seer_dims *dims, const void *Q, const void *K, seer_dtype dtype,
                      const float *Wq, const float *Wk, int32_t h, float rope_theta,
                      seer_select_mode mode, float T, int32_t k, float density,
                      float *scores_out, int32_t *counts, int32_t *indices, int32_t cap,
                      void *ws, size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_gate_workspace_size(const seer_dims *dims, int32_t h);

/* Smallest `cap` that can hold every row's list for this selection:
 * nb for THRESHOLD, min(k, nb) for TOPK_K, the largest k_i for TOPK_DENSITY;
 * with SEER_SELECT_FORCE_DIAGONAL the top-k figures allow one more block
 * (never more than the row length).  Also valid for seer_gate_varlen.
 * Returns -1 on invalid arguments. */
SEER_API int32_t seer_gate_required_cap(const seer_dims *dims, seer_select_mode mode, int32_t k,
                               float density);

/* seer_gate_varlen -- seer_gate over variable-length sequences packed along
 * the token axis (rebuttal, batching: "variable-length inputs can be packed
 * along the sequence dimension").  dims->B must be 1 and dims->n is the
 * packed buffer's length (a multiple of 64).
 *   seq_start, seq_len  DEVICE int32 arrays [nseq]: sequence s occupies tokens
 *             seq_start[s] .. seq_start[s] + seq_len[s] - 1.  Each start is a
 *             multiple of 64 (so a block belongs to one sequence), the
 *             sequences ascend without overlap, and seq_len[s] >= 1.  Tokens
 *             of no sequence are padding; the gate never reads them.
 * Per sequence the gate is seer_gate's on that sequence alone: its last
 * block pools only its own tokens, row i's candidates are the sequence's
 * blocks f .. i (f its first block), k_i is taken at the local row i - f,
 * and block RoPE (if on) rotates by block position (scores depend only on
 * i - j, so packed and separate positions agree).  Lists hold global block
 * indices, so seer_sparse_attn runs on the packed Q/K/V unchanged: inside a
 * sequence's last block the causal rule already hides its padding keys from
 * its tokens.  For that call the padding tokens of K and V must hold finite
 * values (zero them), since a masked key still enters the PV product with
 * weight 0.  Rows of blocks outside every sequence get count 0; rows of the
 * padding positions of a last block are not meaningful.
 * A malformed seq_start/seq_len entry is recorded as SEER_ERR_DEVICE_CHECK
 * in the workspace status and its blocks are treated as padding.
 * Other arguments, outputs and errors as seer_gate.                        */
SEER_API seer_status seer_gate_varlen(const seer_dims *dims, const void *Q, const void *K, seer_dtype dtype,
                                     const float *Wq, const float *Wk, int32_t h, float rope_theta,
                                     const int32_t *seq_start, const int32_t *seq_len, int32_t nseq,
                                     seer_select_mode mode, float T, int32_t k, float density,
                                     float *scores_out, int32_t *counts, int32_t *indices, int32_t cap,
                                     void *ws, size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_gate_varlen_workspace_size(const seer_dims *dims, int32_t h);

/* seer_gate_kl_backward -- one distillation step of the AttnGate: its loss
 * and the gradients of the loss with respect to the gate's two linear layers
 * (summary page, section 3.4, "Loss function: KL-divergence": loss =
 * D_KL(gt || score); "Training data and hyperparameters": only the gate is
 * trained).
 *
 * Recomputes the gate forward exactly as seer_gate does (block RoPE off),
 * then, per causal row (b, hq, i) with g = gt row / sum_{j<=i} gt row:
 *   loss = mean over rows of sum_{j<=i, g_j>0} g_j (log g_j - log score_ij)
 *   dz_ij = (score_ij - g_ij) / rows          (gradient of loss wrt the logits)
 *   dq~_i = sum_j dz_ij k~_j / sqrt(d),   dk~_j = sum_{hq of g} sum_i dz_ij q~_i / sqrt(d)
 *   dWq[hq] = sum_{b,i} dq~_i qbar_i^T,   dWk[g] = sum_{b,j} dk~_j kbar_j^T
 *
 *   Q, K, dtype, Wq, Wk, h   as seer_gate
 *   gt        [B, Hq, nb, nb] fp32: the max-pooled map (seer_attn_blockmax's
 *             map_out); entries j > i are ignored; every row must have a
 *             positive causal sum
 *   loss      one fp32 on the device: the mean KL term (fixed summation
 *             order, deterministic)
 *   dWq       [Hq, h, d] fp32 and dWk [Hkv, h, 3d] fp32: overwritten
 *   ws/ws_bytes  workspace of at least seer_gate_kl_backward_workspace_size(...)
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA.                                                    */
SEER_API seer_status seer_gate_kl_backward(const seer_dims *dims, const void *Q, const void *K,
                                          seer_dtype dtype, const float *Wq, const float *Wk,
                                          int32_t h, const float *gt, float *loss, float *dWq,
                                          float *dWk, void *ws, size_t ws_bytes,
                                          seer_stream_t stream);

SEER_API size_t seer_gate_kl_backward_workspace_size(const seer_dims *dims, int32_t h);

/* seer_gate_select -- the mask-generation step alone on caller-supplied fp32
 * scores [B, Hq, nb, nb] (entries j > i are ignored).  Same selection rules
 * and outputs as seer_gate; used to check index lists bit-exactly against an
 * independent implementation fed the same scores.  No workspace. */
SEER_API seer_status seer_gate_select(const seer_dims *dims, const float *scores, seer_select_mode mode,
                             float T, int32_t k, float density, int32_t *counts,
                             int32_t *indices, int32_t cap, seer_stream_t stream);

/* ------------------------------------------------------------------------ */
/* seer_sparse_attn -- block-sparse causal attention forward (summary page,
 * section 3.4, "Block-sparse FlashAttention kernel"): for query block i of
 * head hq, only key blocks j in its list are used -- a skipped block costs no
 * QK^T, no softmax, no PV and no K/V load.  Inside the diagonal block the
 * causal rule (key position <= query position) applies.  Per query row t:
 *   O[t]   = sum_s softmax_s(scale * q_t . k_s) v_s
 *   lse[t] = ln sum_s exp(scale * q_t . k_s)
 * over the admissible keys s; a row with none gets O = 0 and lse = -inf.
 *
 *   Q [B,Hq,n,d], K/V [B,Hkv,n,d]: bf16 (fp32 is converted to bf16 in the
 *             workspace before the tensor-core pass)
 *   counts [B,Hq,nb], indices [B,Hq,nb,cap]: lists as written by seer_gate:
 *             ascending, unique, every j <= i.  The kernel checks every
 *             count (0 <= c <= min(cap, i+1)) and entry (in range, strictly
 *             ascending) before loading; a failing one is clamped into range
 *             and recorded as SEER_ERR_DEVICE_CHECK in the workspace status.
 *             With bf16 inputs, when every count is i + 1 (the all-ones
 *             causal mask: valid lists are then exactly 0..i) a device-side
 *             check hands the call to the dense 128-row-tile kernel and the
 *             entries are not read (nor checked).
 *   scale     softmax scale; 0 means 1/sqrt(d)
 *   O         [B,Hq,n,d] same dtype as Q;  lse [B,Hq,n] fp32 (may be NULL)
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA.                                                    */
SEER_API seer_status seer_sparse_attn(const seer_dims *dims, const void *Q, const void *K, const void *V,
                             seer_dtype dtype, const int32_t *counts, const int32_t *indices,
                             int32_t cap, float scale, void *O, float *lse, void *ws,
                             size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_sparse_attn_workspace_size(const seer_dims *dims, seer_dtype dtype);

/* seer_sparse_attn_tf32 -- seer_sparse_attn for fp32 Q/K/V/O on the tf32
 * tensor cores: the operands are read as fp32 (the tensor core uses their
 * top 19 bits, tf32) instead of being rounded to bf16 first, and P enters
 * the PV product as fp32 (tf32) too.  About 8x smaller rounding error than
 * the bf16 path, at half its tensor-core rate.  Same lists, scale, layouts
 * and outputs as seer_sparse_attn; O and lse are fp32.
 *   ws/ws_bytes  workspace of at least seer_sparse_attn_tf32_workspace_size
 *               (the status word and V transposed per 64-key block)
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA.                                                    */
SEER_API seer_status seer_sparse_attn_tf32(const seer_dims *dims, const float *Q, const float *K,
                                          const float *V, const int32_t *counts, const int32_t *indices,
                                          int32_t cap, float scale, float *O, float *lse, void *ws,
                                          size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_sparse_attn_tf32_workspace_size(const seer_dims *dims);

/* ------------------------------------------------------------------------ */
/* seer_attn_blockmax -- the ground truth of the gate's self-distillation
 * (summary page, section 3.4, "Ground truth generation" and "The customized
 * training kernel", Figure 10):
 *   map[i][j] = max over the 64x64 block (i, j) of softmax(scale * Q K^T)
 * with the causal softmax of every query row; map[i][j] = 0 for j > i.
 * Two passes: the first forms every row's log-sum-exp and each row's raw
 * maximum per key block; the second rescales those maxima into
 * probabilities and takes the column maximum over the rows of the block.
 *
 *   Q [B,Hq,n,d], K [B,Hkv,n,d]  bf16 (fp32 converted in the workspace)
 *   scale     0 means 1/sqrt(d)
 *   map_out   [B, Hq, nb, nb] fp32
 *   lse_out   optional [B, Hq, n] fp32 row log-sum-exp (may be NULL)
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA.                                                    */
SEER_API seer_status seer_attn_blockmax(const seer_dims *dims, const void *Q, const void *K,
                               seer_dtype dtype, float scale, float *map_out, float *lse_out,
                               void *ws, size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_blockmax_workspace_size(const seer_dims *dims, seer_dtype dtype);

/* ------------------------------------------------------------------------ */
/* seer_gate_noalloc -- seer_gate for callers that cannot allocate device
 * memory.  (The paper has no counterpart: this is an integration variant.)
 *
 * seer_gate's scratch (pooled Q/K, gate vectors, block logits) normally comes
 * from a caller-allocated workspace.  Callers that cannot allocate -- a plugin
 * inside a host framework that owns all device memory and hands out only its
 * own tensors, or a runtime that forbids device allocation after start-up --
 * call this instead: same inputs and outputs, no workspace argument, and no
 * allocation of any kind.  Its scratch is a static device buffer of
 * SEER_GATE_NOALLOC_MAX_SCRATCH bytes inside the library, which every GPU that
 * loads the library's device code keeps until the process exits.
 *  - Problems whose scratch (seer_gate_workspace_size) exceeds the buffer are
 *    rejected with SEER_ERR_WORKSPACE before anything is launched (for
 *    example the 8k-token, 32-head layer fits; 32k tokens do not).
 *  - The device that holds the tensors and the stream must be the current
 *    device when the call is made: the buffer used is the current device's.
 *  - The first call on each device resolves the buffer's device address
 *    (once, with that device current; again after a device reset); make that
 *    first call before any stream capture.  A failure there returns
 *    SEER_ERR_CUDA.
 *  - All calls on a device share the buffer: calls whose work may overlap on
 *    the GPU (different streams without ordering) race and must not be made.
 *  - Device status (seer_workspace_status) cannot be read for this entry
 *    point.  Instead, if a bounded wait inside the gate gives up, every count
 *    is set to -1 after the gate has run (indices and scores are then
 *    unspecified).  Results and errors are otherwise those of seer_gate.   */
#define SEER_GATE_NOALLOC_MAX_SCRATCH (32u << 20) /* bytes */

SEER_API seer_status seer_gate_noalloc(const seer_dims *dims, const void *Q, const void *K,
                                       seer_dtype dtype, const float *Wq, const float *Wk,
                                       int32_t h, float rope_theta, seer_select_mode mode, float T,
                                       int32_t k, float density, float *scores_out,
                                       int32_t *counts, int32_t *indices, int32_t cap,
                                       seer_stream_t stream);

/* ------------------------------------------------------------------------ */
/* seer_attn_forward_map -- the training forward of the summary page's
 * customized kernel ("The customized training kernel", Figure 10): dense
 * causal attention output O and row log-sum-exp, plus the 2D-max-pooled
 * probability map gt, in one pass.  A dense kernel walks 128-row query
 * tiles (two query blocks) over every causal key pair and also keeps each
 * row's score maximum over each 32-key half block; at the end of each tile
 * those maxima become probabilities with the row's log-sum-exp, and their
 * maximum over the 64 rows of a query block is the map entry.  Tiles that
 * need the exact fallback (a score more than 2^64 above the row's
 * first-step maximum) get their O, LSE and map rows recomputed exactly.
 *   Q [B,Hq,n,d], K, V [B,Hkv,n,d] (dtype); scale 0 means 1/sqrt(d)
 *   O [B,Hq,n,d] (dtype), lse [B,Hq,n] fp32 (may be NULL),
 *   map_out [B,Hq,nb,nb] fp32 (0 above the diagonal)
 *   ws/ws_bytes  workspace of at least seer_attn_forward_map_workspace_size(...)
 * Errors: as seer_sparse_attn.                                              */
SEER_API seer_status seer_attn_forward_map(const seer_dims *dims, const void *Q, const void *K, const void *V,
                                          seer_dtype dtype, float scale, void *O, float *lse, float *map_out,
                                          void *ws, size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_attn_forward_map_workspace_size(const seer_dims *dims, seer_dtype dtype);

/* ------------------------------------------------------------------------ */
/* Decode stage (the authors' OpenReview rebuttal, "decode-stage
 * evaluation"): one new token per (batch, query head) attends to a KV cache.
 * The gate keeps no Q-branch pooling or projection -- the token's own query
 * q scores the key blocks -- and reads only a compressed K cache, one
 * vector k~_j per complete 64-key block; attention then loads K/V only for
 * the selected blocks.  Readings of that passage:
 *  - the token sits at position seq_len - 1, in block c = (seq_len - 1) / 64;
 *    the candidates are the complete blocks j < c; block c (positions
 *    64c .. seq_len-1) is always attended and is never a candidate;
 *  - k~_j = Wk[g] [max | min | avg](K block j) (the prefill gate's K branch,
 *    applied to the cached keys as stored), so h = d and
 *    score_j = softmax_{j < c}(q . k~_j / sqrt(d));
 *  - the distillation target is the 1D max-pooling of the token's attention
 *    probabilities over each key block.
 * The KV cache is [B, Hkv, n, d] (dims->n = its capacity in tokens, a
 * multiple of 64); the query is [B, Hq, d].  Cache pointers (K, V, the
 * compressed cache) must be 16-byte aligned.
 */

/* seer_decode_kcache_update -- writes k~_j for key blocks
 * block_begin .. block_end-1 of every (batch, KV head): call it once a block
 * of the cache is complete (or once after a prefill, for all its blocks).
 *   Kcache    [B, Hkv, n, d] bf16 or fp32 (dtype)
 *   Wk        [Hkv, h, 3d] fp32, input features ordered [max | min | avg]
 *   h         must equal d (the query meets k~ directly)
 *   kt_cache  [B, Hkv, n/64, h] fp32; only the listed blocks are written
 * An empty range does nothing.  No workspace.
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_CUDA.       */
SEER_API seer_status seer_decode_kcache_update(const seer_dims *dims, const void *Kcache, seer_dtype dtype,
                                              const float *Wk, int32_t h, int32_t block_begin,
                                              int32_t block_end, float *kt_cache, seer_stream_t stream);

/* seer_decode_gate -- scores of the c = (seq_len-1)/64 candidate blocks and
 * the selected ones, by the prefill rules applied to a row of c candidates
 * (THRESHOLD: score > T; TOPK_K: min(k, c) largest; TOPK_DENSITY:
 * clamp(ceil(density*c), 1, c) largest, the product rounded in fp32).
 *   q         [B, Hq, d] bf16 or fp32 (dtype): the current token's query
 *   kt_cache  [B, Hkv, n/64, d] fp32 from seer_decode_kcache_update, valid
 *             for blocks 0 .. c-1
 *   seq_len   tokens in the cache including the current one, 1 .. n
 *   scores_out  optional [B, Hq, c] fp32 (NULL to skip)
 *   counts    [B, Hq] int32;  indices [B, Hq, cap] int32 ascending, entries
 *             past counts[row] untouched; c == 0 gives counts 0
 *   cap       >= seer_decode_gate_required_cap(...)
 *   ws/ws_bytes  workspace of at least seer_decode_gate_workspace_size(...)
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_CAPACITY,
 *         SEER_ERR_WORKSPACE, SEER_ERR_CUDA.                               */
SEER_API seer_status seer_decode_gate(const seer_dims *dims, const void *q, seer_dtype dtype,
                                     const float *kt_cache, int32_t seq_len, seer_select_mode mode, float T,
                                     int32_t k, float density, float *scores_out, int32_t *counts,
                                     int32_t *indices, int32_t cap, void *ws, size_t ws_bytes,
                                     seer_stream_t stream);

SEER_API size_t seer_decode_gate_workspace_size(const seer_dims *dims);

/* Smallest `cap` for seer_decode_gate at this seq_len (0 when c == 0);
 * -1 on invalid arguments. */
SEER_API int32_t seer_decode_gate_required_cap(const seer_dims *dims, int32_t seq_len, seer_select_mode mode,
                                              int32_t k, float density);

/* seer_sparse_decode_attn -- the token's attention over the keys of its
 * selected blocks and of its own block c (positions 64c .. seq_len-1):
 *   O   = sum_s softmax_s(scale * q . k_s) v_s,  lse = ln sum_s exp(...)
 * Split over the list (split-KV) with a log-sum-exp merge.
 *   q [B,Hq,d], Kcache/Vcache [B,Hkv,n,d]: bf16 or fp32 (dtype)
 *   counts [B,Hq], indices [B,Hq,cap]: lists as seer_decode_gate writes them
 *             (every entry < c); a count outside 0..min(cap, c) or an entry
 *             outside 0..c-1 is clamped and recorded as SEER_ERR_DEVICE_CHECK
 *   scale     0 means 1/sqrt(d)
 *   O [B,Hq,d] (dtype), lse [B,Hq] fp32 (may be NULL)
 *   ws/ws_bytes  workspace of at least seer_sparse_decode_attn_workspace_size
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA.                                                    */
SEER_API seer_status seer_sparse_decode_attn(const seer_dims *dims, const void *q, const void *Kcache,
                                            const void *Vcache, seer_dtype dtype, int32_t seq_len,
                                            const int32_t *counts, const int32_t *indices, int32_t cap,
                                            float scale, void *O, float *lse, void *ws, size_t ws_bytes,
                                            seer_stream_t stream);

SEER_API size_t seer_sparse_decode_attn_workspace_size(const seer_dims *dims);

/* seer_decode_blockmax -- the decode gate's distillation target: over the
 * token's full causal attention row (positions 0 .. seq_len-1),
 *   gt[j] = max over the keys of block j of softmax(scale * q . K^T)
 * for j = 0 .. c (block c partial), and the row's lse.  The query heads of a
 * KV head are scored together, so the K cache is read once per KV head.
 *   gt_out [B, Hq, c+1] fp32;  lse_out [B, Hq] fp32 (may be NULL)
 *   ws/ws_bytes  workspace of at least seer_decode_blockmax_workspace_size
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA.                                                    */
SEER_API seer_status seer_decode_blockmax(const seer_dims *dims, const void *q, const void *Kcache,
                                         seer_dtype dtype, int32_t seq_len, float scale, float *gt_out,
                                         float *lse_out, void *ws, size_t ws_bytes, seer_stream_t stream);

SEER_API size_t seer_decode_blockmax_workspace_size(const seer_dims *dims);

/* ------------------------------------------------------------------------ */
/* seer_prefill_host -- the whole prefill hot path (seer_gate, then
 * seer_sparse_attn) for inputs and outputs in host memory, with the
 * host-device copies overlapped with the compute.
 *
 * The layer is processed one KV head's group of query heads (b, g) at a
 * time: the group's Q, K, V are copied in on a copy stream, its gate and
 * attention run on `stream`, its O (and LSE) are copied out on a second copy
 * stream, through two device buffer slots, so that the copy in of group
 * i + 1 and the copy out of group i - 1 overlap the compute of group i.  The
 * results are those of seer_gate + seer_sparse_attn on the whole layer
 * (every step is per head and per query block).
 *
 *   hQ [B,Hq,n,d], hK/hV [B,Hkv,n,d]  host memory, dtype (page-locked memory
 *             gives the overlap; pageable memory works but serialises)
 *   Wq, Wk    device pointers, as for seer_gate;  h, rope_theta, mode, T, k,
 *             density as for seer_gate;  scale as for seer_sparse_attn
 *   hO [B,Hq,n,d] host, dtype;  hLSE [B,Hq,n] host fp32, or NULL
 *   dbuf      device buffer of at least seer_prefill_host_buffer_size(...)
 *             bytes, 256-byte aligned (two slots of one group's Q, K, V, O,
 *             LSE and lists, one gate and one attention workspace)
 * The call returns when the outputs are in host memory.  It checks every
 * group's device status words and returns SEER_ERR_TIMEOUT or
 * SEER_ERR_DEVICE_CHECK if one was set.  The two copy streams and their
 * events are made on the first call of each host thread on each device and
 * kept until the thread exits (this is the one piece of state the library
 * keeps between calls).
 * Errors: SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_WORKSPACE,
 *         SEER_ERR_CUDA, SEER_ERR_TIMEOUT, SEER_ERR_DEVICE_CHECK.            */
SEER_API seer_status seer_prefill_host(const seer_dims *dims, const void *hQ, const void *hK, const void *hV,
                                       seer_dtype dtype, const float *Wq, const float *Wk, int32_t h,
                                       float rope_theta, seer_select_mode mode, float T, int32_t k, float density,
                                       float scale, void *hO, float *hLSE, void *dbuf, size_t dbuf_bytes,
                                       seer_stream_t stream);

/* Device buffer bytes seer_prefill_host needs; 0 for invalid arguments. */
SEER_API size_t seer_prefill_host_buffer_size(const seer_dims *dims, seer_dtype dtype, int32_t h,
                                              seer_select_mode mode, int32_t k, float density);

/* Synchronises `stream`, reads the device status word at the start of a
 * workspace that a previous call used, and maps it: SEER_OK,
 * SEER_ERR_TIMEOUT or SEER_ERR_DEVICE_CHECK (SEER_ERR_CUDA if the read
 * fails).  Every call clears the word when it starts. */
SEER_API seer_status seer_workspace_status(const void *ws, seer_stream_t stream);

/* Human-readable name of a status code (static storage). */
SEER_API const char *seer_status_string(seer_status s);

/* The cudaError_t of the last SEER_ERR_CUDA returned on this host thread. */
SEER_API int32_t seer_last_cuda_error(void);

/* Library version, e.g. "0.1.0". */
SEER_API const char *seer_version(void);

/* seer_testing_attn_wait_fault -- a test hook for the failure path of the
 * attention kernels' bounded waits (no counterpart in the pages: it exists so
 * that the timeout path can be exercised without faulting or hanging a GPU).
 * After this call, seer_sparse_attn calls made on the same host thread leave
 * out the completion signal of QK step `step` (counted from 0 in every CTA of
 * the persistent kernel) and bound each of their waits by `wait_limit_ns`
 * (0 keeps the default of 2 s).  The waits that depend on the missing signal
 * then give up: the kernel unwinds (every bulk copy it issued lands before
 * it exits), SEER_ERR_TIMEOUT is recorded in the workspace status word, and
 * the device stays usable.  `step` < 0 turns the hook off (the default).
 * Outputs of a call made with the hook on are unspecified.               */
SEER_API void seer_testing_attn_wait_fault(int32_t step, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif
#endif /* SEER_H */
