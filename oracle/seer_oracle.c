/*
 * seer_oracle.c -- plain fp64 CPU oracle for the SeerAttention prefill path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code with the CUDA library.
 *
 * Every function computes a plain definition from "SeerAttention: Learning
 * Intrinsic Sparse Attention in Your LLMs" (arXiv 2410.13276), as summarised
 * on the paper-graph summary page, section 3.4, and the authors' OpenReview
 * rebuttal, section 3.3.  Arithmetic is fp64 throughout; inputs arrive as
 * fp32 arrays (bf16 inputs are upcast exactly before the call).  No blocking,
 * fusion or reordering beyond the definitions.
 *
 * Layout: every tensor is contiguous [B, H, n, d] (row-major).  Query head hq
 * uses KV head hq / (Hq / Hkv).  Block size is `blk` (64 in the method).
 *
 * Parity status: pooling, projection, gate softmax, selection, masked
 * attention and the max-pooled map are pinned by the CPU tests (library
 * routines, closed forms, invariants).  Block RoPE (orc_block_rope) is only
 * partly pinned: its rotation structure is checked, but the base reading
 * theta' = theta / B is "parity unpinned" (no worked example on the pages).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef int64_t i64;

/* ---------------------------------------------------------------------- */
/* AttnGate pooling (summary page, section 3.4 "Input and pooling" and
 * "Pooling Method Selection"): average pooling of Q with kernel = stride = B;
 * max, min and average pooling of K, concatenated along the feature axis in
 * the order [max | min | avg].                                             */

/* qbar[bh, i, c] = mean_{t in block i} Q[bh, t, c];  qbar is [BH, nb, d]. */
void orc_pool_q(const float *Q, i64 BH, i64 n, i64 d, i64 blk, double *qbar)
{
    i64 nb = n / blk;
#pragma omp parallel for collapse(2) schedule(static)
    for (i64 bh = 0; bh < BH; ++bh)
        for (i64 i = 0; i < nb; ++i)
            for (i64 c = 0; c < d; ++c) {
                double s = 0.0;
                for (i64 t = 0; t < blk; ++t)
                    s += (double)Q[(bh * n + i * blk + t) * d + c];
                qbar[(bh * nb + i) * d + c] = s / (double)blk;
            }
}

/* kbar[bh, i, :] = [max_t K | min_t K | mean_t K] over block i; [BH, nb, 3d]. */
void orc_pool_k(const float *K, i64 BH, i64 n, i64 d, i64 blk, double *kbar)
{
    i64 nb = n / blk;
#pragma omp parallel for collapse(2) schedule(static)
    for (i64 bh = 0; bh < BH; ++bh)
        for (i64 i = 0; i < nb; ++i)
            for (i64 c = 0; c < d; ++c) {
                double mx = -INFINITY, mn = INFINITY, s = 0.0;
                for (i64 t = 0; t < blk; ++t) {
                    double v = (double)K[(bh * n + i * blk + t) * d + c];
                    if (v > mx) mx = v;
                    if (v < mn) mn = v;
                    s += v;
                }
                double *o = kbar + (bh * nb + i) * 3 * d;
                o[c] = mx;
                o[d + c] = mn;
                o[2 * d + c] = s / (double)blk;
            }
}

/* ---------------------------------------------------------------------- */
/* Gate projections (summary page, section 3.4 "Linear transformation"):
 * y[b, hh, i, :] = W[hh] x[b, hh, i, :], W[hh] is [h, din]; no bias.       */
void orc_project(const double *x, const float *W, i64 B, i64 H, i64 nb,
                 i64 din, i64 h, double *y)
{
#pragma omp parallel for collapse(3) schedule(static)
    for (i64 b = 0; b < B; ++b)
        for (i64 hh = 0; hh < H; ++hh)
            for (i64 i = 0; i < nb; ++i) {
                const double *xv = x + ((b * H + hh) * nb + i) * din;
                const float *Wh = W + hh * h * din;
                double *yv = y + ((b * H + hh) * nb + i) * h;
                for (i64 r = 0; r < h; ++r) {
                    double s = 0.0;
                    for (i64 c = 0; c < din; ++c)
                        s += (double)Wh[r * din + c] * xv[c];
                    yv[r] = s;
                }
            }
}

/* Block-level RoPE (summary page, section 3.4 "Block-Level RoPE"): applied
 * to the projected gate vectors at block positions i, with the base divided
 * by the block size (theta' = theta / B, the formula as printed).  Pairs are
 * (c, c + h/2) ("rotate half"); frequency of pair c is base'^(-2c/h).
 * In place on x [BH, nb, h].  Parity unpinned for the base reading.        */
void orc_block_rope(double *x, i64 BH, i64 nb, i64 h, double theta, i64 blk)
{
    double base = theta / (double)blk;
    i64 half = h / 2;
#pragma omp parallel for collapse(2) schedule(static)
    for (i64 bh = 0; bh < BH; ++bh)
        for (i64 i = 0; i < nb; ++i) {
            double *v = x + (bh * nb + i) * h;
            for (i64 c = 0; c < half; ++c) {
                double freq = pow(base, -2.0 * (double)c / (double)h);
                double ang = (double)i * freq;
                double cs = cos(ang), sn = sin(ang);
                double a = v[c], bb = v[c + half];
                v[c] = a * cs - bb * sn;
                v[c + half] = bb * cs + a * sn;
            }
        }
}

/* ---------------------------------------------------------------------- */
/* Gate scores, Eq. 1 of the summary page (section 3.4 "Scoring via
 * multiplication"): score = softmax(q~ k~^T / sqrt(d)) per row.  Causal
 * prefill: row i is a softmax over the key blocks j <= i only; entries with
 * j > i are 0.  qt is [B, Hq, nb, h], kt is [B, Hkv, nb, h]; scores is
 * [B, Hq, nb, nb].  `scale` is 1/sqrt(d), d = head dimension.              */
void orc_gate_scores(const double *qt, const double *kt, i64 B, i64 Hq,
                     i64 Hkv, i64 nb, i64 h, double scale, double *scores)
{
    i64 G = Hq / Hkv;
#pragma omp parallel for collapse(3) schedule(dynamic, 4)
    for (i64 b = 0; b < B; ++b)
        for (i64 hq = 0; hq < Hq; ++hq)
            for (i64 i = 0; i < nb; ++i) {
                const double *q = qt + ((b * Hq + hq) * nb + i) * h;
                const double *kbase = kt + (b * Hkv + hq / G) * nb * h;
                double *row = scores + ((b * Hq + hq) * nb + i) * nb;
                double mx = -INFINITY;
                for (i64 j = 0; j <= i; ++j) {
                    double z = 0.0;
                    for (i64 c = 0; c < h; ++c) z += q[c] * kbase[j * h + c];
                    z *= scale;
                    row[j] = z;
                    if (z > mx) mx = z;
                }
                double sum = 0.0;
                for (i64 j = 0; j <= i; ++j) {
                    row[j] = exp(row[j] - mx);
                    sum += row[j];
                }
                for (i64 j = 0; j <= i; ++j) row[j] /= sum;
                for (i64 j = i + 1; j < nb; ++j) row[j] = 0.0;
            }
}


/* Eq. 1 for listed rows only: unit u = (b*Hq + hq)*nb + i; out is [nunits, nb]
 * (entries j > i are 0).  Same arithmetic as orc_gate_scores.              */
void orc_gate_scores_units(const double *qt, const double *kt, i64 B, i64 Hq,
                           i64 Hkv, i64 nb, i64 h, double scale,
                           const i64 *units, i64 nunits, double *out)
{
    (void)B;
    i64 G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (i64 u = 0; u < nunits; ++u) {
        i64 unit = units[u];
        i64 i = unit % nb, bhq = unit / nb;
        i64 b = bhq / Hq, hq = bhq % Hq;
        const double *q = qt + ((b * Hq + hq) * nb + i) * h;
        const double *kbase = kt + (b * Hkv + hq / G) * nb * h;
        double *row = out + u * nb;
        double mx = -INFINITY;
        for (i64 j = 0; j <= i; ++j) {
            double z = 0.0;
            for (i64 c = 0; c < h; ++c) z += q[c] * kbase[j * h + c];
            z *= scale;
            row[j] = z;
            if (z > mx) mx = z;
        }
        double sum = 0.0;
        for (i64 j = 0; j <= i; ++j) {
            row[j] = exp(row[j] - mx);
            sum += row[j];
        }
        for (i64 j = 0; j <= i; ++j) row[j] /= sum;
        for (i64 j = i + 1; j < nb; ++j) row[j] = 0.0;
    }
}

/* ---------------------------------------------------------------------- */
/* Binary mask generation (summary page, section 3.4 "Generating the binary
 * block mask"; rebuttal section 3.3).  The mask of row i is returned as the
 * ascending list of active key blocks j <= i.  rows = B*Hq*nb rows of
 * length nb; row r is query block i = r % nb, or row_i[r] when row_i is
 * not NULL.  idx is [rows, cap].
 * Return value: the largest count of any row (the caller checks it against
 * cap; rows whose count exceeds cap are truncated to cap entries).         */

/* Method 2, thresholding: active iff score > T (strict).  T is an fp32 value
 * so that supplied fp32 scores are compared exactly as an fp32 kernel does. */
i64 orc_select_threshold(const double *scores, i64 rows, i64 nb, float T,
                         int32_t *counts, int32_t *idx, i64 cap,
                         const i64 *row_i, int force_diag)
{
    i64 worst = 0;
#pragma omp parallel for schedule(static) reduction(max : worst)
    for (i64 r = 0; r < rows; ++r) {
        i64 i = row_i ? row_i[r] : r % nb, c = 0;
        const double *s = scores + r * nb;
        for (i64 j = 0; j <= i; ++j)
            if (s[j] > (double)T || (force_diag && j == i)) {
                if (c < cap) idx[r * cap + c] = (int32_t)j;
                ++c;
            }
        counts[r] = (int32_t)(c < cap ? c : cap);
        if (c > worst) worst = c;
    }
    return worst;
}

/* Per-row k for the top-k methods.  mode 1: uniform k, k_i = min(k, i+1)
 * (the pages' "k largest scores in row i"; a causal row has only i+1
 * candidates).  mode 2: density rho, k_i = clamp(ceil(rho*(i+1)), 1, i+1),
 * with the product rounded in fp32 so both sides take the same decision.  */
i64 orc_topk_count(i64 i, int mode, i64 k, float density)
{
    i64 ki;
    if (mode == 1) {
        ki = k;
    } else {
        volatile float prod = density * (float)(i + 1);
        ki = (i64)ceilf(prod);
        if (ki < 1) ki = 1;
    }
    if (ki > i + 1) ki = i + 1;
    return ki;
}

typedef struct { double s; i64 j; } cand_t;

static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->s > b->s) return -1;          /* larger score first        */
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j); /* ties: lower j first */
}

static int int_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Method 1, TopK: the k_i largest scores of row i (ties: lower j first),
 * returned in ascending j.                                                 */
i64 orc_select_topk(const double *scores, i64 rows, i64 nb, int mode, i64 k,
                    float density, int32_t *counts, int32_t *idx, i64 cap,
                    const i64 *row_i, int force_diag)
{
    i64 worst = 0;
#pragma omp parallel reduction(max : worst)
    {
        cand_t *buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)nb);
#pragma omp for schedule(static)
        for (i64 r = 0; r < rows; ++r) {
            i64 i = row_i ? row_i[r] : r % nb;
            const double *s = scores + r * nb;
            for (i64 j = 0; j <= i; ++j) { buf[j].s = s[j]; buf[j].j = j; }
            qsort(buf, (size_t)(i + 1), sizeof(cand_t), cand_cmp);
            i64 ki = orc_topk_count(i, mode, k, density);
            i64 c = ki < cap ? ki : cap;
            int has_diag = 0;
            for (i64 m = 0; m < c; ++m) {
                idx[r * cap + m] = (int32_t)buf[m].j;
                if (buf[m].j == i) has_diag = 1;
            }
            /* the optional forced diagonal joins the list when not chosen */
            i64 need = ki;
            if (force_diag && !has_diag) {
                need = ki + 1;
                if (c < cap) idx[r * cap + c++] = (int32_t)i;
            }
            qsort(idx + r * cap, (size_t)c, sizeof(int32_t), int_cmp);
            counts[r] = (int32_t)c;
            if (need > worst) worst = need;
        }
        free(buf);
    }
    return worst;
}

/* ---------------------------------------------------------------------- */
/* Block-sparse attention (summary page, section 3.4 "Block-sparse
 * FlashAttention kernel"): for query block i, only the key blocks in its
 * list take part; within them the causal rule s <= t holds.  For each query
 * row t:  p_s = softmax_s(q_t . k_s * scale),  o_t = sum_s p_s v_s,
 * lse_t = ln sum_s exp(q_t . k_s * scale).  A row with no key gets o = 0 and
 * lse = -inf.  Computed per unit u = (b*Hq + hq)*nb + i; O_out is
 * [nunits, blk, d], lse_out is [nunits, blk].                              */
static void attn_unit(const float *Q, const float *K, const float *V,
                      i64 Hq, i64 Hkv, i64 n, i64 d, i64 blk, i64 unit,
                      const int32_t *list, i64 count, double scale,
                      double *O_out, double *lse_out, double *z)
{
    i64 nb = n / blk, G = Hq / Hkv;
    i64 i = unit % nb, bhq = unit / nb;
    i64 b = bhq / Hq, hq = bhq % Hq;
    const float *Qh = Q + (b * Hq + hq) * n * d;
    const float *Kh = K + (b * Hkv + hq / G) * n * d;
    const float *Vh = V + (b * Hkv + hq / G) * n * d;
    for (i64 r = 0; r < blk; ++r) {
        i64 t = i * blk + r;
        const float *q = Qh + t * d;
        double *o = O_out + r * d;
        for (i64 c = 0; c < d; ++c) o[c] = 0.0;
        /* logits of every admissible key, in list order */
        i64 nk = 0;
        double mx = -INFINITY;
        for (i64 m = 0; m < count; ++m) {
            i64 j = list[m];
            for (i64 s = j * blk; s < (j + 1) * blk && s <= t; ++s) {
                const float *kk = Kh + s * d;
                double acc = 0.0;
                for (i64 c = 0; c < d; ++c) acc += (double)q[c] * (double)kk[c];
                acc *= scale;
                z[nk++] = acc;
                if (acc > mx) mx = acc;
            }
        }
        if (nk == 0) { lse_out[r] = -INFINITY; continue; }
        double l = 0.0;
        nk = 0;
        for (i64 m = 0; m < count; ++m) {
            i64 j = list[m];
            for (i64 s = j * blk; s < (j + 1) * blk && s <= t; ++s) {
                double p = exp(z[nk++] - mx);
                l += p;
                const float *vv = Vh + s * d;
                for (i64 c = 0; c < d; ++c) o[c] += p * (double)vv[c];
            }
        }
        for (i64 c = 0; c < d; ++c) o[c] /= l;
        lse_out[r] = mx + log(l);
    }
}

/* Units given explicitly (units[u] as above); counts/idx are the full
 * [B*Hq*nb] / [B*Hq*nb, cap] selection arrays.                            */
void orc_sparse_attn_units(const float *Q, const float *K, const float *V,
                           i64 B, i64 Hq, i64 Hkv, i64 n, i64 d, i64 blk,
                           const int32_t *counts, const int32_t *idx, i64 cap,
                           double scale, const i64 *units, i64 nunits,
                           double *O_out, double *lse_out)
{
    (void)B;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
        for (i64 u = 0; u < nunits; ++u) {
            i64 unit = units[u];
            attn_unit(Q, K, V, Hq, Hkv, n, d, blk, unit, idx + unit * cap,
                      counts[unit], scale, O_out + u * blk * d,
                      lse_out + u * blk, z);
        }
        free(z);
    }
}

/* All units: O is [B, Hq, n, d], lse is [B, Hq, n]. */
void orc_sparse_attn(const float *Q, const float *K, const float *V, i64 B,
                     i64 Hq, i64 Hkv, i64 n, i64 d, i64 blk,
                     const int32_t *counts, const int32_t *idx, i64 cap,
                     double scale, double *O, double *lse)
{
    i64 nunits = B * Hq * (n / blk);
    i64 *units = (i64 *)malloc(sizeof(i64) * (size_t)nunits);
    for (i64 u = 0; u < nunits; ++u) units[u] = u;
    /* unit u covers rows [i*blk, (i+1)*blk) of head (b,hq): contiguous in O */
    orc_sparse_attn_units(Q, K, V, B, Hq, Hkv, n, d, blk, counts, idx, cap,
                          scale, units, nunits, O, lse);
    free(units);
}

/* ---------------------------------------------------------------------- */
/* Ground truth of the gate's self-distillation (summary page, section 3.4
 * "Ground truth generation"): gt = MaxPool2D_{BxB, stride B}(softmax(Q K^T *
 * scale)) with the causal softmax of every query row over its keys s <= t.
 * Direct definition: every probability P[t, s] is formed and max-pooled; the
 * two-pass rescaling of the pages' training kernel is not used here.
 * For unit u = (b*Hq + hq)*nb + i it writes gt_out[u, 0..nb) (0 for j > i)
 * and lse_out[u, 0..blk) (row log-sum-exp).                               */
void orc_blockmax_units(const float *Q, const float *K, i64 B, i64 Hq,
                        i64 Hkv, i64 n, i64 d, i64 blk, double scale,
                        const i64 *units, i64 nunits, double *gt_out,
                        double *lse_out)
{
    (void)B;
    i64 nb = n / blk, G = Hq / Hkv;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
        for (i64 u = 0; u < nunits; ++u) {
            i64 unit = units[u];
            i64 i = unit % nb, bhq = unit / nb;
            i64 b = bhq / Hq, hq = bhq % Hq;
            const float *Qh = Q + (b * Hq + hq) * n * d;
            const float *Kh = K + (b * Hkv + hq / G) * n * d;
            double *gt = gt_out + u * nb;
            for (i64 j = 0; j < nb; ++j) gt[j] = 0.0;
            for (i64 r = 0; r < blk; ++r) {
                i64 t = i * blk + r;
                const float *q = Qh + t * d;
                double mx = -INFINITY;
                for (i64 s = 0; s <= t; ++s) {
                    double acc = 0.0;
                    for (i64 c = 0; c < d; ++c)
                        acc += (double)q[c] * (double)Kh[s * d + c];
                    z[s] = acc * scale;
                    if (z[s] > mx) mx = z[s];
                }
                double l = 0.0;
                for (i64 s = 0; s <= t; ++s) l += exp(z[s] - mx);
                for (i64 s = 0; s <= t; ++s) {
                    double p = exp(z[s] - mx) / l;
                    if (p > gt[s / blk]) gt[s / blk] = p;
                }
                lse_out[u * blk + r] = mx + log(l);
            }
        }
        free(z);
    }
}

/* All units: gt is [B, Hq, nb, nb], lse is [B, Hq, n]. */
void orc_blockmax(const float *Q, const float *K, i64 B, i64 Hq, i64 Hkv,
                  i64 n, i64 d, i64 blk, double scale, double *gt, double *lse)
{
    i64 nunits = B * Hq * (n / blk);
    i64 *units = (i64 *)malloc(sizeof(i64) * (size_t)nunits);
    for (i64 u = 0; u < nunits; ++u) units[u] = u;
    orc_blockmax_units(Q, K, B, Hq, Hkv, n, d, blk, scale, units, nunits, gt,
                       lse);
    free(units);
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int orc_num_threads(void)
{
    int t = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            t = omp_get_num_threads();
#endif
        }
    }
    return t;
}
