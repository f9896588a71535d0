/*
 * fp64 CPU oracle for the sparse Lightning Indexer KL-loss backward.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg may load this library. The CUDA product path never calls it.
 *
 * It is the plain definition written out, following the formulas of
 * aclnnSparseLightningIndexerKLLossGrad (section "计算公式"):
 *
 *   S_t   = q_t . K_topk(t)^T                  (per head h: S[h][j] = sum_d q[t,h,d] k[r_j,d])
 *   I_t   = W_t . ReLU(S_t)                    (I[j] = sum_h w[t,h] max(S[h][j], 0))
 *   y_t   = Softmax(I_t)                       (written to softmaxOut)
 *   dI_t  = Softmax(I_t) - p_t                 (p = attnSoftmaxL1Norm)
 *   dW_t  = dI_t . ReLU(S_t)^T
 *   dq_t  = dS_t . K_topk(t)
 *   dK_topk(t) = dS_t^T . q_t, scatter-added to the key rows named by sparseIndices
 *
 * dS is not printed on the page; it follows from I = W . ReLU(S) by the chain rule:
 *   dS[h][j] = dI[j] * w[t,h] * (S[h][j] > 0 ? 1 : 0).
 *
 * Invalid top-k slots (index -1) take no part in any sum (same section):
 * the softmax runs over the valid slots only, y = 0 and dI = 0 at invalid slots.
 * Valid indices are local to the query's batch (section "公共约束"): key row =
 * k_start[b] + index. A token with no valid slot gets y = 0 and zero gradients.
 *
 * The KL loss of the same section, L_t = sum_{valid j} p_j log(p_j / y_j) (with
 * 0 log 0 = 0), is returned per token for finite-difference checks.
 *
 * Used lengths (seqUsedQOptional / seqUsedKOptional of the same page, which fixes only
 * their type; read here as the rows of each batch in use): when given, query rows of
 * batch b at local position >= q_used[b] are padding (their indices are not read, all
 * their outputs are 0, they add nothing to dk) and a slot naming a key at local position
 * >= k_used[b] is invalid like -1.
 *
 * Everything is fp64. Tokens are independent and run in parallel (OpenMP); dk is
 * accumulated key row by key row, each row summing its references in ascending
 * (token, slot) order, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t B;                /* batches */
    int64_t T1, T2;           /* total query rows, total key rows */
    int64_t N1, D, K;         /* query heads, head dim, top-k */
    const int64_t *q_start;   /* [B+1] first query row of each batch (q_start[B] = T1) */
    const int64_t *k_start;   /* [B+1] first key row of each batch (k_start[B] = T2) */
    const int64_t *q_used;    /* [B] query rows of each batch in use, or NULL (all) */
    const int64_t *k_used;    /* [B] key rows of each batch in use, or NULL (all) */
} oracle_problem;

enum { ORACLE_OK = 0, ORACLE_BAD_SHAPE = 1, ORACLE_BAD_INDEX = 2, ORACLE_NO_MEMORY = 3 };

/* Batch of query row t (linear scan over the batch table: B is small). */
static int64_t batch_of(const oracle_problem *pr, int64_t t) {
    for (int64_t b = 0; b < pr->B; ++b)
        if (t < pr->q_start[b + 1]) return b;
    return pr->B - 1;
}

/* Is query row t in use (not a padding row past q_used of its batch)? */
static int row_in_use(const oracle_problem *pr, int64_t t) {
    if (!pr->q_used) return 1;
    int64_t b = batch_of(pr, t);
    return t - pr->q_start[b] < pr->q_used[b];
}

/* Key row of slot j of query row t, or -1 when the slot is invalid (index -1, a key past
 * k_used of the batch, or any slot of a padding row). */
static int64_t key_row(const oracle_problem *pr, const int32_t *idx, int64_t t, int64_t j) {
    if (!row_in_use(pr, t)) return -1;
    int32_t v = idx[t * pr->K + j];
    if (v < 0) return -1;
    int64_t b = batch_of(pr, t);
    if (pr->k_used && v >= pr->k_used[b]) return -1;
    return pr->k_start[b] + v;
}

/* Check the index contract on the rows in use: -1 or inside the batch's key range. */
int oracle_check_indices(const oracle_problem *pr, const int32_t *idx) {
    for (int64_t t = 0; t < pr->T1; ++t) {
        if (!row_in_use(pr, t)) continue;
        int64_t b = batch_of(pr, t);
        int64_t klen = pr->k_start[b + 1] - pr->k_start[b];
        for (int64_t j = 0; j < pr->K; ++j) {
            int32_t v = idx[t * pr->K + j];
            if (v < -1 || v >= klen) return ORACLE_BAD_INDEX;
        }
    }
    return ORACLE_OK;
}

/* S[h][j] = q_t[h,:] . k[r,:] */
static double score(const oracle_problem *pr, const double *q, const double *k,
                    int64_t t, int64_t h, int64_t r) {
    const double *qh = q + (t * pr->N1 + h) * pr->D;
    const double *kr = k + r * pr->D;
    double s = 0.0;
    for (int64_t d = 0; d < pr->D; ++d) s += qh[d] * kr[d];
    return s;
}

/*
 * Per-token part: S, I, y, dI, dw, dq and the KL loss of one query row t.
 * Writes y[t,:], dI[t,:], dw[t,:], dq[t,:,:] and loss[t].
 */
static void token_forward_backward(const oracle_problem *pr, const double *q, const double *k,
                                   const double *w, const double *p, const int32_t *idx,
                                   int64_t t, double *S, double *I, double *y, double *dI,
                                   double *dw, double *dq, double *loss) {
    const int64_t N1 = pr->N1, D = pr->D, K = pr->K;
    double *yt = y + t * K, *dIt = dI + t * K, *dwt = dw + t * N1, *dqt = dq + t * N1 * D;
    const double *pt = p + t * K, *wt = w + t * N1;

    /* S and I over the valid slots */
    int64_t nvalid = 0;
    double m = -INFINITY;
    for (int64_t j = 0; j < K; ++j) {
        int64_t r = key_row(pr, idx, t, j);
        if (r < 0) continue;
        ++nvalid;
        double Ij = 0.0;
        for (int64_t h = 0; h < N1; ++h) {
            double s = score(pr, q, k, t, h, r);
            S[h * K + j] = s;
            Ij += wt[h] * (s > 0.0 ? s : 0.0);
        }
        I[j] = Ij;
        if (Ij > m) m = Ij;
    }

    for (int64_t h = 0; h < N1; ++h) dwt[h] = 0.0;
    for (int64_t e = 0; e < N1 * D; ++e) dqt[e] = 0.0;
    if (nvalid == 0) {
        for (int64_t j = 0; j < K; ++j) { yt[j] = 0.0; dIt[j] = 0.0; }
        if (loss) loss[t] = 0.0;
        return;
    }

    /* y = Softmax(I) over the valid slots (max subtracted; identical in exact arithmetic) */
    double Z = 0.0;
    for (int64_t j = 0; j < K; ++j)
        if (key_row(pr, idx, t, j) >= 0) Z += exp(I[j] - m);
    double L = 0.0;
    for (int64_t j = 0; j < K; ++j) {
        if (key_row(pr, idx, t, j) < 0) { yt[j] = 0.0; dIt[j] = 0.0; continue; }
        yt[j] = exp(I[j] - m) / Z;
        dIt[j] = yt[j] - pt[j];                         /* dI = Softmax(I) - p */
        if (pt[j] > 0.0) L += pt[j] * log(pt[j] / yt[j]);
    }
    if (loss) loss[t] = L;

    /* dW = dI . ReLU(S)^T ; dq = dS . K_topk with dS = dI * w * 1[S > 0] */
    for (int64_t j = 0; j < K; ++j) {
        int64_t r = key_row(pr, idx, t, j);
        if (r < 0) continue;
        const double *kr = k + r * D;
        for (int64_t h = 0; h < N1; ++h) {
            double s = S[h * K + j];
            if (s > 0.0) {
                dwt[h] += dIt[j] * s;
                double ds = dIt[j] * wt[h];
                for (int64_t d = 0; d < D; ++d) dqt[h * D + d] += ds * kr[d];
            }
        }
    }
}

/*
 * Full oracle. Outputs (all fp64, caller-allocated):
 *   y [T1,K], dw [T1,N1], dq [T1,N1,D], dk [T2,D], loss [T1] (may be NULL).
 * tokens / ntokens: optional subset of query rows (NULL = all rows). Rows outside
 * the subset are left untouched in y/dw/dq/loss and contribute nothing to dk.
 * nthreads <= 0 lets OpenMP choose.
 */
int oracle_grad(const oracle_problem *pr, const double *q, const double *k, const double *w,
                const double *p, const int32_t *idx, const int64_t *tokens, int64_t ntokens,
                int nthreads, double *y, double *dw, double *dq, double *dk, double *loss) {
    const int64_t T1 = pr->T1, T2 = pr->T2, N1 = pr->N1, D = pr->D, K = pr->K;
    if (pr->B <= 0 || N1 <= 0 || D <= 0 || K <= 0 || T1 < 0 || T2 < 0) return ORACLE_BAD_SHAPE;
    if (pr->q_start[0] != 0 || pr->k_start[0] != 0 || pr->q_start[pr->B] != T1 ||
        pr->k_start[pr->B] != T2)
        return ORACLE_BAD_SHAPE;
    for (int64_t b = 0; b < pr->B; ++b) {
        if (pr->q_used && (pr->q_used[b] < 0 ||
                           pr->q_used[b] > pr->q_start[b + 1] - pr->q_start[b]))
            return ORACLE_BAD_SHAPE;
        if (pr->k_used && (pr->k_used[b] < 0 ||
                           pr->k_used[b] > pr->k_start[b + 1] - pr->k_start[b]))
            return ORACLE_BAD_SHAPE;
    }
    int rc = oracle_check_indices(pr, idx);
    if (rc != ORACLE_OK) return rc;

    int64_t nt = tokens ? ntokens : T1;
    double *dI = (double *)calloc((size_t)(T1 * K > 0 ? T1 * K : 1), sizeof(double));
    if (!dI) return ORACLE_NO_MEMORY;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif

    /* Phase 1: per-token outputs */
    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc((size_t)(N1 * K) * sizeof(double));
        double *I = (double *)malloc((size_t)K * sizeof(double));
        if (!S || !I) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < nt; ++i) {
                int64_t t = tokens ? tokens[i] : i;
                token_forward_backward(pr, q, k, w, p, idx, t, S, I, y, dI, dw, dq, loss);
            }
        }
        free(S);
        free(I);
    }
    if (failed) { free(dI); return ORACLE_NO_MEMORY; }

    /* Phase 2: dk[r,:] = sum over references (t, j) of row r, in ascending (t, j) order,
     * of sum_h dS[h][j] q[t,h,:]. The references of each key row are listed by a
     * counting pass over the selected tokens (their order is the token-list order). */
    int64_t *count = (int64_t *)calloc((size_t)T2 + 1, sizeof(int64_t));
    if (!count) { free(dI); return ORACLE_NO_MEMORY; }
    for (int64_t i = 0; i < nt; ++i) {
        int64_t t = tokens ? tokens[i] : i;
        for (int64_t j = 0; j < K; ++j) {
            int64_t r = key_row(pr, idx, t, j);
            if (r >= 0) count[r + 1] += 1;
        }
    }
    for (int64_t r = 0; r < T2; ++r) count[r + 1] += count[r];
    int64_t nref = count[T2];
    int64_t *ref_t = (int64_t *)malloc((size_t)(nref > 0 ? nref : 1) * sizeof(int64_t));
    int64_t *ref_j = (int64_t *)malloc((size_t)(nref > 0 ? nref : 1) * sizeof(int64_t));
    int64_t *fill = (int64_t *)malloc((size_t)(T2 > 0 ? T2 : 1) * sizeof(int64_t));
    if (!ref_t || !ref_j || !fill) {
        free(dI); free(count); free(ref_t); free(ref_j); free(fill);
        return ORACLE_NO_MEMORY;
    }
    for (int64_t r = 0; r < T2; ++r) fill[r] = count[r];
    for (int64_t i = 0; i < nt; ++i) {
        int64_t t = tokens ? tokens[i] : i;
        for (int64_t j = 0; j < K; ++j) {
            int64_t r = key_row(pr, idx, t, j);
            if (r < 0) continue;
            ref_t[fill[r]] = t;
            ref_j[fill[r]] = j;
            fill[r] += 1;
        }
    }

#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t r = 0; r < T2; ++r) {
        double *dkr = dk + r * D;
        for (int64_t d = 0; d < D; ++d) dkr[d] = 0.0;
        for (int64_t e = count[r]; e < count[r + 1]; ++e) {
            int64_t t = ref_t[e], j = ref_j[e];
            double dIj = dI[t * K + j];
            for (int64_t h = 0; h < N1; ++h) {
                double s = score(pr, q, k, t, h, r);          /* S[h][j] of token t */
                if (s > 0.0) {
                    double ds = dIj * w[t * N1 + h];           /* dS[h][j] */
                    const double *qh = q + (t * N1 + h) * D;
                    for (int64_t d = 0; d < D; ++d) dkr[d] += ds * qh[d];
                }
            }
        }
    }

    free(dI); free(count); free(ref_t); free(ref_j); free(fill);
    return ORACLE_OK;
}

/*
 * Work split of the merged B*S1 query rows over `cores` workers, as the metadata
 * generator of DenseLightningIndexerKLLossGradMetadata describes it (section
 * "功能定位" and "Metadata 输出布局"): former = ceil(total / cores) rows for the
 * first workers, remain = former - 1 for the rest, with usedCoreNum = min(cores, total)
 * workers in all. out[0..5] = totalSize, formerCoreSize, remainCoreSize, remainCoreNum,
 * usedCoreNum, maxSeqK; ranges[2c], ranges[2c+1] = [start, end) of worker c (empty
 * ranges for unused workers).
 */
void oracle_split_equal(int64_t total, int64_t cores, int64_t max_seq_k, int64_t *out,
                        int64_t *ranges) {
    int64_t former = total > 0 ? (total + cores - 1) / cores : 0;
    int64_t remain = former > 0 ? former - 1 : 0;
    int64_t used = total < cores ? total : cores;
    int64_t former_cores = total - used * remain;   /* workers that take `former` rows */
    int64_t remain_cores = used - former_cores;
    out[0] = total; out[1] = former; out[2] = remain; out[3] = remain_cores;
    out[4] = used;  out[5] = max_seq_k;
    int64_t start = 0;
    for (int64_t c = 0; c < cores; ++c) {
        int64_t n = c < former_cores ? former : (c < used ? remain : 0);
        ranges[2 * c] = start;
        ranges[2 * c + 1] = start + n;
        start += n;
    }
}

/*
 * Cost-weighted variant of the same split (this library's own refinement; the pages
 * split by row count only). cost(t) = 1 + the number of 128-slot tiles of row t that
 * hold at least one valid index (index >= 0). With P(t) the cost of rows [0, t) and
 * C = P(total), worker c starts at the first row t with P(t) * cores >= c * C.
 */
void oracle_split_weighted(const int32_t *idx, int64_t total, int64_t K, int64_t cores,
                           int64_t *ranges) {
    int64_t *P = (int64_t *)malloc((size_t)(total + 1) * sizeof(int64_t));
    P[0] = 0;
    for (int64_t t = 0; t < total; ++t) {
        int64_t tiles = 0;
        for (int64_t j0 = 0; j0 < K; j0 += 128) {
            int any = 0;
            for (int64_t j = j0; j < j0 + 128 && j < K; ++j)
                if (idx[t * K + j] >= 0) any = 1;
            tiles += any;
        }
        P[t + 1] = P[t] + 1 + tiles;
    }
    int64_t C = P[total];
    for (int64_t c = 0; c <= cores; ++c) {
        int64_t t = 0;
        while (t < total && P[t] * cores < c * C) ++t;
        if (c < cores) ranges[2 * c] = t;
        if (c > 0) ranges[2 * c - 1] = t;
    }
    free(P);
}
