/*
 * oracle.c -- plain fp64 CPU reference for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this code;
 * only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes is the plain definition that every page on FlashAttention
 * says the method reproduces exactly:
 *   - "FlashAttention: making attention fast by respecting the memory
 *     hierarchy", opening paragraph and the tiling paragraph: an exact
 *     algorithm, the same math reorganised;
 *   - "FlashAttention: Fast and Memory-Efficient Exact Attention with
 *     IO-Awareness", section "What FlashAttention targets": same outputs as
 *     the naive formulation;
 *   - "Flash Attention", sections "Definition" and "Common Confusions": exact,
 *     not approximate attention.
 * So the oracle is naive attention written out, in fp64, materialising every
 * score row:
 *     S_ij = scale * q_i . k_j          for allowed (i, j), else -inf
 *     P_ij = exp(S_ij - m_i) / l_i      m_i = max_j S_ij, l_i = sum_j exp(S_ij - m_i)
 *     O_i  = sum_j P_ij v_j,            LSE_i = m_i + ln l_i
 * The per-row LSE is the "softmax normalization statistics" that the summary
 * page's "Backward / recomputation" section says the forward stores.
 *
 * The backward is the calculus of that definition (the pages only say that
 * the backward recomputes from the stored statistics):
 *     dP_ij = dO_i . v_j,  D_i = sum_j P_ij dP_ij,  dS_ij = P_ij (dP_ij - D_i)
 *     dV_j = sum_i P_ij dO_i,  dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i
 *
 * Queries and keys may differ in number (Nq query rows, Nk key rows; the
 * square entry points are the case Nq = Nk = N).  Masks: none; causal,
 * aligned at the bottom right: key j visible to query i iff
 * j <= i + (Nk - Nq), so the last query sees every key and, for Nq = Nk, this
 * is j <= i (the pages do not treat Nq != Nk; this is the reading that keeps
 * a suffix of the queries' outputs equal to those of the full problem);
 * block (a [ceil(Nq/block) x ceil(Nk/block)] uint8 grid of block x block
 * tiles, 1 = keep).  A row with no allowed key has O_i = 0, LSE_i = -inf and
 * contributes no gradient.
 *
 * Inputs and outputs are fp64 host arrays: Q, O, dO, dQ [BH, Nq, d], K, V,
 * dK, dV [BH, Nk, d] (heads flattened), LSE and D [BH, Nq].  Work is split
 * over rows or key columns with OpenMP; every output element is written by
 * exactly one thread, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_MASK_NONE = 0, OR_MASK_CAUSAL = 1, OR_MASK_BLOCK = 2 };
enum { OR_OK = 0, OR_ERR_ARG = 1, OR_ERR_NOMEM = 2 };

typedef struct {
    int Nq, Nk, d, kind, block, nbk;  /* nbk: key blocks, the mask's row length */
    const uint8_t *bm;
    double scale;
} spec_t;

static int allowed(const spec_t *s, int i, int j)
{
    switch (s->kind) {
    case OR_MASK_NONE: return 1;
    case OR_MASK_CAUSAL: return j <= i + (s->Nk - s->Nq);
    default: return s->bm[(size_t)(i / s->block) * s->nbk + (j / s->block)] != 0;
    }
}

static double dot(const double *a, const double *b, int n)
{
    double acc = 0.0;
#pragma omp simd reduction(+ : acc)
    for (int k = 0; k < n; ++k) acc += a[k] * b[k];
    return acc;
}

static int check(const spec_t *s, int BH)
{
    if (BH <= 0 || s->Nq <= 0 || s->Nk <= 0 || s->d <= 0) return OR_ERR_ARG;
    if (s->kind < 0 || s->kind > 2) return OR_ERR_ARG;
    if (s->kind == OR_MASK_BLOCK && (s->bm == NULL || s->block <= 0)) return OR_ERR_ARG;
    return OR_OK;
}

static spec_t make_spec(int Nq, int Nk, int d, int kind, const uint8_t *bm, int block, double scale)
{
    spec_t s;
    s.Nq = Nq; s.Nk = Nk; s.d = d; s.kind = kind; s.bm = bm; s.scale = scale;
    s.block = block > 0 ? block : 1;
    s.nbk = (Nk + s.block - 1) / s.block;
    return s;
}

/* Score row i of one head into S[0..Nk), masked entries -inf; returns m_i. */
static double score_row(const spec_t *s, const double *Qh, const double *Kh, int i, double *S)
{
    const double *q = Qh + (size_t)i * s->d;
    double m = -INFINITY;
    for (int j = 0; j < s->Nk; ++j) {
        if (allowed(s, i, j)) {
            S[j] = s->scale * dot(q, Kh + (size_t)j * s->d, s->d);
            if (S[j] > m) m = S[j];
        } else {
            S[j] = -INFINITY;
        }
    }
    return m;
}

/* Turn a score row into probabilities in place; returns LSE_i (-inf if empty). */
static double softmax_row(const spec_t *s, double *S, double m)
{
    if (m == -INFINITY) {                       /* no allowed key */
        for (int j = 0; j < s->Nk; ++j) S[j] = 0.0;
        return -INFINITY;
    }
    double l = 0.0;
    for (int j = 0; j < s->Nk; ++j) {
        S[j] = (S[j] == -INFINITY) ? 0.0 : exp(S[j] - m);
        l += S[j];
    }
    for (int j = 0; j < s->Nk; ++j) S[j] /= l;
    return m + log(l);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Forward: O [BH,Nq,d], LSE [BH,Nq]. */
int oracle_fwd_qk(const double *Q, const double *K, const double *V, int BH, int Nq, int Nk, int d,
                  int kind, const uint8_t *block_mask, int block, double scale,
                  double *O, double *LSE)
{
    spec_t s = make_spec(Nq, Nk, d, kind, block_mask, block, scale);
    if (check(&s, BH) != OR_OK || !Q || !K || !V || !O || !LSE) return OR_ERR_ARG;
    int err = OR_OK;
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!P) {
#pragma omp atomic write
            err = OR_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 8) collapse(2)
        for (int h = 0; h < BH; ++h)
            for (int i = 0; i < Nq; ++i) {
                if (!P) continue;
                const size_t hq = (size_t)h * Nq * d, hk = (size_t)h * Nk * d;
                double m = score_row(&s, Q + hq, K + hk, i, P);
                LSE[(size_t)h * Nq + i] = softmax_row(&s, P, m);
                double *o = O + hq + (size_t)i * d;
                for (int k = 0; k < d; ++k) o[k] = 0.0;
                for (int j = 0; j < Nk; ++j) {
                    if (P[j] == 0.0) continue;          /* masked (or underflowed) */
                    const double *v = V + hk + (size_t)j * d;
                    for (int k = 0; k < d; ++k) o[k] += P[j] * v[k];
                }
            }
        free(P);
    }
    return err;
}

int oracle_fwd(const double *Q, const double *K, const double *V, int BH, int N, int d,
               int kind, const uint8_t *block_mask, int block, double scale,
               double *O, double *LSE)
{
    return oracle_fwd_qk(Q, K, V, BH, N, N, d, kind, block_mask, block, scale, O, LSE);
}

/* Backward, recomputing everything from Q, K, V and dO.
 * Outputs dQ [BH,Nq,d], dK, dV [BH,Nk,d]; optional O [BH,Nq,d], LSE [BH,Nq]
 * and D [BH,Nq] (pass NULL to skip).  Pass 1 goes row by row (P_i, D_i, dQ_i,
 * O_i, LSE_i); pass 2 goes key column by key column (dV_j, dK_j), rebuilding
 * P_ij as exp(S_ij - LSE_i), the same softmax value written through its
 * normaliser. */
int oracle_bwd_qk(const double *Q, const double *K, const double *V, const double *dO,
                  int BH, int Nq, int Nk, int d, int kind, const uint8_t *block_mask, int block,
                  double scale, double *dQ, double *dK, double *dV,
                  double *O, double *LSE, double *D)
{
    spec_t s = make_spec(Nq, Nk, d, kind, block_mask, block, scale);
    if (check(&s, BH) != OR_OK || !Q || !K || !V || !dO || !dQ || !dK || !dV) return OR_ERR_ARG;
    double *lse = (double *)malloc(sizeof(double) * (size_t)BH * Nq);
    double *Dv = (double *)malloc(sizeof(double) * (size_t)BH * Nq);
    if (!lse || !Dv) { free(lse); free(Dv); return OR_ERR_NOMEM; }
    int err = OR_OK;

    /* pass 1: rows */
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)Nk);
        double *dP = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!P || !dP) {
#pragma omp atomic write
            err = OR_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 8) collapse(2)
        for (int h = 0; h < BH; ++h)
            for (int i = 0; i < Nq; ++i) {
                if (!P || !dP) continue;
                const size_t hq = (size_t)h * Nq * d, hk = (size_t)h * Nk * d;
                const double *dq_o = dO + hq + (size_t)i * d;
                double m = score_row(&s, Q + hq, K + hk, i, P);
                double L = softmax_row(&s, P, m);
                double Di = 0.0;
                for (int j = 0; j < Nk; ++j) {
                    dP[j] = 0.0;
                    if (P[j] == 0.0) continue;
                    dP[j] = dot(dq_o, V + hk + (size_t)j * d, d);
                    Di += P[j] * dP[j];
                }
                double *dq = dQ + hq + (size_t)i * d;
                for (int k = 0; k < d; ++k) dq[k] = 0.0;
                for (int j = 0; j < Nk; ++j) {
                    if (P[j] == 0.0) continue;
                    double ds = P[j] * (dP[j] - Di);
                    const double *kj = K + hk + (size_t)j * d;
                    for (int k = 0; k < d; ++k) dq[k] += ds * kj[k];
                }
                for (int k = 0; k < d; ++k) dq[k] *= scale;
                if (O) {
                    double *o = O + hq + (size_t)i * d;
                    for (int k = 0; k < d; ++k) o[k] = 0.0;
                    for (int j = 0; j < Nk; ++j) {
                        if (P[j] == 0.0) continue;
                        const double *v = V + hk + (size_t)j * d;
                        for (int k = 0; k < d; ++k) o[k] += P[j] * v[k];
                    }
                }
                lse[(size_t)h * Nq + i] = L;
                Dv[(size_t)h * Nq + i] = Di;
            }
        free(P);
        free(dP);
    }

    /* pass 2: key columns */
    if (err == OR_OK) {
#pragma omp parallel for schedule(dynamic, 8) collapse(2)
        for (int h = 0; h < BH; ++h)
            for (int j = 0; j < Nk; ++j) {
                const size_t hq = (size_t)h * Nq * d, hk = (size_t)h * Nk * d;
                const double *kj = K + hk + (size_t)j * d;
                const double *vj = V + hk + (size_t)j * d;
                double *dk = dK + hk + (size_t)j * d;
                double *dv = dV + hk + (size_t)j * d;
                for (int k = 0; k < d; ++k) { dk[k] = 0.0; dv[k] = 0.0; }
                for (int i = 0; i < Nq; ++i) {
                    if (!allowed(&s, i, j)) continue;
                    const double L = lse[(size_t)h * Nq + i];
                    if (L == -INFINITY) continue;
                    const double *qi = Q + hq + (size_t)i * d;
                    const double *doi = dO + hq + (size_t)i * d;
                    double p = exp(s.scale * dot(qi, kj, d) - L);
                    double dp = dot(doi, vj, d);
                    double ds = p * (dp - Dv[(size_t)h * Nq + i]);
                    for (int k = 0; k < d; ++k) {
                        dv[k] += p * doi[k];
                        dk[k] += ds * qi[k];
                    }
                }
                for (int k = 0; k < d; ++k) dk[k] *= scale;
            }
    }
    if (LSE) memcpy(LSE, lse, sizeof(double) * (size_t)BH * Nq);
    if (D) memcpy(D, Dv, sizeof(double) * (size_t)BH * Nq);
    free(lse);
    free(Dv);
    return err;
}

int oracle_bwd(const double *Q, const double *K, const double *V, const double *dO,
               int BH, int N, int d, int kind, const uint8_t *block_mask, int block,
               double scale, double *dQ, double *dK, double *dV,
               double *O, double *LSE, double *D)
{
    return oracle_bwd_qk(Q, K, V, dO, BH, N, N, d, kind, block_mask, block, scale, dQ, dK, dV, O, LSE, D);
}

/* Selected rows: for each (head[r], row[r]) pair, O_r [d], LSE_r and, when dO
 * is given, dQ_r [d].  Everything here depends on that one query row only,
 * so the cost is O(N d) per row whatever the problem size. */
int oracle_rows_qk(const double *Q, const double *K, const double *V, const double *dO,
                   int BH, int Nq, int Nk, int d, int kind, const uint8_t *block_mask, int block,
                   double scale, const int *head, const int *row, int nrows,
                   double *O, double *LSE, double *dQ)
{
    spec_t s = make_spec(Nq, Nk, d, kind, block_mask, block, scale);
    if (check(&s, BH) != OR_OK || !Q || !K || !V || !head || !row || nrows < 0 || !O || !LSE)
        return OR_ERR_ARG;
    if (dQ && !dO) return OR_ERR_ARG;
    for (int r = 0; r < nrows; ++r)
        if (head[r] < 0 || head[r] >= BH || row[r] < 0 || row[r] >= Nq) return OR_ERR_ARG;
    int err = OR_OK;
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!P) {
#pragma omp atomic write
            err = OR_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            if (!P) continue;
            const size_t hq = (size_t)head[r] * Nq * d, hk = (size_t)head[r] * Nk * d;
            const int i = row[r];
            double m = score_row(&s, Q + hq, K + hk, i, P);
            LSE[r] = softmax_row(&s, P, m);
            double *o = O + (size_t)r * d;
            for (int k = 0; k < d; ++k) o[k] = 0.0;
            for (int j = 0; j < Nk; ++j) {
                if (P[j] == 0.0) continue;
                const double *v = V + hk + (size_t)j * d;
                for (int k = 0; k < d; ++k) o[k] += P[j] * v[k];
            }
            if (dQ) {
                const double *doi = dO + hq + (size_t)i * d;
                double Di = 0.0;
                for (int j = 0; j < Nk; ++j)
                    if (P[j] != 0.0) Di += P[j] * dot(doi, V + hk + (size_t)j * d, d);
                double *dq = dQ + (size_t)r * d;
                for (int k = 0; k < d; ++k) dq[k] = 0.0;
                for (int j = 0; j < Nk; ++j) {
                    if (P[j] == 0.0) continue;
                    double ds = P[j] * (dot(doi, V + hk + (size_t)j * d, d) - Di);
                    const double *kj = K + hk + (size_t)j * d;
                    for (int k = 0; k < d; ++k) dq[k] += ds * kj[k];
                }
                for (int k = 0; k < d; ++k) dq[k] *= scale;
            }
        }
        free(P);
    }
    return err;
}

int oracle_rows(const double *Q, const double *K, const double *V, const double *dO,
                int BH, int N, int d, int kind, const uint8_t *block_mask, int block,
                double scale, const int *head, const int *row, int nrows,
                double *O, double *LSE, double *dQ)
{
    return oracle_rows_qk(Q, K, V, dO, BH, N, N, d, kind, block_mask, block, scale, head, row, nrows, O, LSE, dQ);
}

/* Selected key columns: for each (head[c], col[c]) pair, dK_c [d] and
 * dV_c [d], the gradients of one key row.  They sum over the query rows that
 * see the key, and each such row enters through its normaliser LSE_i and its
 * D_i = sum_j P_ij dP_ij, which depend on the whole score row.  So the row
 * statistics of every head named in the list are computed first, row by row
 * from the definition; then each requested column is a plain loop over the
 * query rows:
 *     P_ij = exp(scale q_i . k_j - LSE_i),  dP_ij = dO_i . v_j,
 *     dS_ij = P_ij (dP_ij - D_i),
 *     dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i.
 * The cost is one forward over the named heads plus O(Nq d) per column. */
int oracle_cols_qk(const double *Q, const double *K, const double *V, const double *dO,
                   int BH, int Nq, int Nk, int d, int kind, const uint8_t *block_mask, int block,
                   double scale, const int *head, const int *col, int ncols,
                   double *dK, double *dV)
{
    spec_t s = make_spec(Nq, Nk, d, kind, block_mask, block, scale);
    if (check(&s, BH) != OR_OK || !Q || !K || !V || !dO || !head || !col || ncols < 0 || !dK || !dV)
        return OR_ERR_ARG;
    for (int c = 0; c < ncols; ++c)
        if (head[c] < 0 || head[c] >= BH || col[c] < 0 || col[c] >= Nk) return OR_ERR_ARG;
    unsigned char *need = (unsigned char *)calloc((size_t)BH, 1);
    double *lse = (double *)malloc(sizeof(double) * (size_t)BH * Nq);
    double *Dv = (double *)malloc(sizeof(double) * (size_t)BH * Nq);
    if (!need || !lse || !Dv) { free(need); free(lse); free(Dv); return OR_ERR_NOMEM; }
    for (int c = 0; c < ncols; ++c) need[head[c]] = 1;
    int err = OR_OK;

    /* row statistics of the named heads */
#pragma omp parallel
    {
        double *P = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!P) {
#pragma omp atomic write
            err = OR_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 8) collapse(2)
        for (int h = 0; h < BH; ++h)
            for (int i = 0; i < Nq; ++i) {
                if (!P || !need[h]) continue;
                const size_t hq = (size_t)h * Nq * d, hk = (size_t)h * Nk * d;
                const double *doi = dO + hq + (size_t)i * d;
                double m = score_row(&s, Q + hq, K + hk, i, P);
                double L = softmax_row(&s, P, m);
                double Di = 0.0;
                for (int j = 0; j < Nk; ++j)
                    if (P[j] != 0.0) Di += P[j] * dot(doi, V + hk + (size_t)j * d, d);
                lse[(size_t)h * Nq + i] = L;
                Dv[(size_t)h * Nq + i] = Di;
            }
        free(P);
    }

    /* one key column at a time */
    if (err == OR_OK) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int c = 0; c < ncols; ++c) {
            const int h = head[c], j = col[c];
            const size_t hq = (size_t)h * Nq * d, hk = (size_t)h * Nk * d;
            const double *kj = K + hk + (size_t)j * d;
            const double *vj = V + hk + (size_t)j * d;
            double *gk = dK + (size_t)c * d;
            double *gv = dV + (size_t)c * d;
            for (int k = 0; k < d; ++k) { gk[k] = 0.0; gv[k] = 0.0; }
            for (int i = 0; i < Nq; ++i) {
                if (!allowed(&s, i, j)) continue;
                const double L = lse[(size_t)h * Nq + i];
                if (L == -INFINITY) continue;
                const double *qi = Q + hq + (size_t)i * d;
                const double *doi = dO + hq + (size_t)i * d;
                const double pij = exp(s.scale * dot(qi, kj, d) - L);
                const double dpij = dot(doi, vj, d);
                const double dsij = pij * (dpij - Dv[(size_t)h * Nq + i]);
                for (int k = 0; k < d; ++k) {
                    gv[k] += pij * doi[k];
                    gk[k] += dsij * qi[k];
                }
            }
            for (int k = 0; k < d; ++k) gk[k] *= scale;
        }
    }
    free(need);
    free(lse);
    free(Dv);
    return err;
}

/* Full probability matrix P [BH,Nq,Nk] (small sizes only). */
int oracle_probs_qk(const double *Q, const double *K, int BH, int Nq, int Nk, int d, int kind,
                    const uint8_t *block_mask, int block, double scale, double *P)
{
    spec_t s = make_spec(Nq, Nk, d, kind, block_mask, block, scale);
    if (check(&s, BH) != OR_OK || !Q || !K || !P) return OR_ERR_ARG;
#pragma omp parallel for schedule(static) collapse(2)
    for (int h = 0; h < BH; ++h)
        for (int i = 0; i < Nq; ++i) {
            double *Prow = P + ((size_t)h * Nq + i) * Nk;
            double m = score_row(&s, Q + (size_t)h * Nq * d, K + (size_t)h * Nk * d, i, Prow);
            softmax_row(&s, Prow, m);
        }
    return OR_OK;
}

int oracle_probs(const double *Q, const double *K, int BH, int N, int d, int kind,
                 const uint8_t *block_mask, int block, double scale, double *P)
{
    return oracle_probs_qk(Q, K, BH, N, N, d, kind, block_mask, block, scale, P);
}
