/*
 * hstu_oracle.c -- plain, slow, fp64 CPU oracle for jagged HSTU attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (per sequence b, head h, query row i of that sequence):
 *
 *   s_ij  = alpha * <q_i, k_j> + rel[clamp(p(i)-p(j), 0, R-1)]
 *                              + tb[min(floor(log(|ts[p(i)]-ts[p(j)]| + 1) / div), NB-1)]
 *   A_ij  = valid(i,j) ? SiLU(s_ij) / N : 0                   SiLU(x) = x * sigmoid(x)
 *   Y_i   = sum_j A_ij V_j             (per head, heads concatenated to D = H*d_v)
 *   Zhat  = (Y_i - mean(Y_i)) / sqrt(var(Y_i) + eps)          (biased variance, no affine)
 *   O_i   = U_i (.) Zhat
 *
 * Sources, by page and section:
 *  - "HSTU tensor by tensor: SiLU aggregation, temporal bias and gating",
 *    section "Similar shape, different aggregation": the teaching equation
 *    A_ij = 1[j<=i] SiLU(q_i.k_j + b_ij)/N and o_i = W_o[U_i (.) Norm(sum_j A_ij V_j)] + x_i.
 *    This file stops at U (.) Norm(.): W_o and the residual are outside the path.
 *  - same page, "SiLU aggregation coefficients are not probabilities": SiLU = x*sigmoid(x).
 *  - same page, "Do not copy softmax masking mechanically": illegal coefficients are
 *    zeroed after the nonlinearity (never -inf before it).
 *  - same page, "Relative time adds information content similarity lacks" and
 *    "Temporal bias is not simply fixed forgetting": relative position and elapsed
 *    time bias the scores; units and bucketing matter.
 *  - "HSTU-MUSA: HSTU for Moore Threads (MUSA)", section "Mathematical Equivalence":
 *    the mask family (contextual bidirectional attention, candidate position clamping,
 *    target group masking, max attention length); section "Accuracy Alignment":
 *    scaling_seqlen = -1, i.e. N is the actual batch max_seqlen.
 *
 * Readings where the pages leave a step open (each is also listed in the design notes):
 *  - positions are local to the sequence, 0..L-1; c = num_contextuals, t = num_targets,
 *    E = L - t is the end of the history;
 *  - p(x) = x for x < E, else E-1 (candidate positions clamp to the last history
 *    position); if E == 0, p(x) = x;
 *  - valid(i,j):  j >= E            -> i == j          (a candidate key is seen by itself only)
 *                 else i < c        -> j < c           (contextual rows: bidirectional prefix)
 *                 else j < c        -> true            (contextual keys seen by every row)
 *                 else              -> j <= p(i) and (W <= 0 or p(i) - j <= W)
 *  - the rel index p(i)-p(j) is clamped into [0, R-1] (negative -> 0);
 *  - the time bucket uses natural log, div taken literally, |dt| in the caller's
 *    integer units, and is computed in fp64 as written here;
 *  - alpha multiplies q.k only, not the bias;
 *  - one rel table and one time table shared by all heads.
 *
 * Two variants of the mask family, as flags (both off by default):
 *  - ORACLE_CTX_SEES_HISTORY: contextual rows attend to every key before the candidates
 *    (the contextual prefix and the whole history), not only to the contextual prefix;
 *  - ORACLE_REL_ABS: the rel index is min(|p(i) - p(j)|, R-1) rather than clamp(p(i) - p(j),
 *    0, R-1), so bidirectional pairs with p(i) < p(j) index by their distance.
 *
 * All inputs are fp64 copies of the values the device sees (bf16 inputs are rounded
 * by the input generator and upcast exactly).  Layouts: q,k [T,H,dqk], v [T,H,dv],
 * u, out, y [T,H*dv], row-major; column index of (head h, element e) is h*dv+e.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- helpers */

static double oracle_silu(double x) { return x / (1.0 + exp(-x)); }

/* d/dx [x * sigmoid(x)] = sigmoid(x) * (1 + x * (1 - sigmoid(x))) */
static double oracle_silu_grad(double x)
{
    double sg = 1.0 / (1.0 + exp(-x));
    return sg * (1.0 + x * (1.0 - sg));
}

/* floor(log(|dt| + 1) / div), clamped to [0, NB-1]; evaluated in fp64 exactly as written. */
int64_t hstu_oracle_time_bucket(int64_t dt, double div, int64_t NB)
{
    if (NB <= 0) return 0;
    /* |dt| without overflow for INT64_MIN: go through unsigned. */
    uint64_t a = dt < 0 ? (uint64_t)0 - (uint64_t)dt : (uint64_t)dt;
    double x = log((double)a + 1.0) / div;
    double f = floor(x);
    if (f < 0.0) f = 0.0;
    if (f > (double)(NB - 1)) return NB - 1;
    return (int64_t)f;
}

#define ORACLE_CTX_SEES_HISTORY 1
#define ORACLE_REL_ABS 2

static int64_t clamped_pos(int64_t x, int64_t E)
{
    if (E <= 0) return x;
    return x < E ? x : E - 1;
}

/* The mask predicate of the reading above, for local positions i (query) and j (key). */
static int oracle_valid(int64_t i, int64_t j, int64_t L, int64_t c, int64_t t, int64_t W,
                        int64_t flags)
{
    int64_t E = L - t;
    if (j >= E) return i == j;
    if (i < c) return (flags & ORACLE_CTX_SEES_HISTORY) ? 1 : j < c;
    if (j < c) return 1;
    int64_t pi = clamped_pos(i, E);
    if (j > pi) return 0;
    if (W > 0 && pi - j > W) return 0;
    return 1;
}

/* Mask of one sequence as an L*L byte matrix (row i = query).  Returns the valid-pair count. */
int64_t hstu_oracle_mask_flags(int64_t L, int64_t c, int64_t t, int64_t W, int64_t flags,
                               uint8_t *mask)
{
    int64_t n = 0;
    for (int64_t i = 0; i < L; ++i)
        for (int64_t j = 0; j < L; ++j) {
            int v = oracle_valid(i, j, L, c, t, W, flags);
            if (mask) mask[i * L + j] = (uint8_t)v;
            n += v;
        }
    return n;
}

int64_t hstu_oracle_mask(int64_t L, int64_t c, int64_t t, int64_t W, uint8_t *mask)
{
    return hstu_oracle_mask_flags(L, c, t, W, 0, mask);
}

/* Rows [r0, r0+nrows) x keys [0, ncols) of the same mask, positions past the sequence's end
 * (>= L) counted invalid; row r - r0 of `mask` has ncols bytes.  Returns the valid count. */
int64_t hstu_oracle_mask_rows(int64_t L, int64_t c, int64_t t, int64_t W, int64_t flags,
                              int64_t r0, int64_t nrows, int64_t ncols, uint8_t *mask)
{
    int64_t n = 0;
    for (int64_t r = 0; r < nrows; ++r)
        for (int64_t j = 0; j < ncols; ++j) {
            int64_t i = r0 + r;
            int v = i < L && j < L && oracle_valid(i, j, L, c, t, W, flags);
            mask[r * ncols + j] = (uint8_t)v;
            n += v;
        }
    return n;
}

typedef struct {
    int64_t B, H, dqk, dv;
    const int64_t *offsets;
    const int32_t *ctx, *tgt;
    const int64_t *ts;
    const double *rel;
    int64_t R;
    const double *tb;
    int64_t NB;
    double div, alpha;
    int64_t W, N;
    int64_t flags;
} oracle_problem;

/* Bias b_ij for local positions i, j of a sequence starting at global row s0. */
static double oracle_bias(const oracle_problem *P, int64_t s0, int64_t E, int64_t i, int64_t j,
                          int64_t *rel_idx, int64_t *bucket)
{
    int64_t pi = clamped_pos(i, E), pj = clamped_pos(j, E);
    double b = 0.0;
    *rel_idx = -1;
    *bucket = -1;
    if (P->R > 0) {
        int64_t r = pi - pj;
        if (r < 0) r = (P->flags & ORACLE_REL_ABS) ? -r : 0;
        if (r > P->R - 1) r = P->R - 1;
        *rel_idx = r;
        b += P->rel[r];
    }
    if (P->NB > 0) {
        int64_t dt = P->ts[s0 + pi] - P->ts[s0 + pj];
        int64_t k = hstu_oracle_time_bucket(dt, P->div, P->NB);
        *bucket = k;
        b += P->tb[k];
    }
    return b;
}

static int oracle_seq(const oracle_problem *P, int64_t b, int64_t *s0, int64_t *L, int64_t *c,
                      int64_t *t)
{
    *s0 = P->offsets[b];
    *L = P->offsets[b + 1] - P->offsets[b];
    *c = P->ctx ? P->ctx[b] : 0;
    *t = P->tgt ? P->tgt[b] : 0;
    if (*L < 0 || *c < 0 || *t < 0 || *c + *t > *L) return -1;
    return 0;
}

/* ---------------------------------------------------------------- forward */

int hstu_oracle_fwd(int64_t B, int64_t H, int64_t dqk, int64_t dv, const int64_t *offsets,
                    const int32_t *ctx, const int32_t *tgt, const int64_t *ts, const double *q,
                    const double *k, const double *v, const double *u, const double *rel,
                    int64_t R, const double *tb, int64_t NB, double div, double alpha,
                    int64_t max_attn_len, int64_t N, double eps, int64_t flags, double *out,
                    double *y, double *mean, double *rstd)
{
    oracle_problem P = {B, H, dqk, dv, offsets, ctx, tgt, ts, rel, R, tb, NB, div, alpha,
                        max_attn_len, N, flags};
    const int64_t D = H * dv;
    int bad = 0;
    for (int64_t b = 0; b < B; ++b) {
        int64_t s0, L, c, t;
        if (oracle_seq(&P, b, &s0, &L, &c, &t)) bad = 1;
    }
    if (bad || N <= 0) return -1;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < B; ++b) {
        int64_t s0, L, c, t;
        oracle_seq(&P, b, &s0, &L, &c, &t);
        int64_t E = L - t;
        double *yrow = (double *)malloc(sizeof(double) * (size_t)(D > 0 ? D : 1));
        for (int64_t i = 0; i < L; ++i) {
            memset(yrow, 0, sizeof(double) * (size_t)D);
            for (int64_t h = 0; h < H; ++h) {
                const double *qi = q + ((s0 + i) * H + h) * dqk;
                for (int64_t j = 0; j < L; ++j) {
                    if (!oracle_valid(i, j, L, c, t, max_attn_len, flags)) continue;
                    const double *kj = k + ((s0 + j) * H + h) * dqk;
                    double dot = 0.0;
                    for (int64_t e = 0; e < dqk; ++e) dot += qi[e] * kj[e];
                    int64_t ri, bk;
                    double s = alpha * dot + oracle_bias(&P, s0, E, i, j, &ri, &bk);
                    double a = oracle_silu(s) / (double)N;
                    const double *vj = v + ((s0 + j) * H + h) * dv;
                    for (int64_t e = 0; e < dv; ++e) yrow[h * dv + e] += a * vj[e];
                }
            }
            /* LayerNorm over all H*dv features of the token, then U gating. */
            double mu = 0.0;
            for (int64_t e = 0; e < D; ++e) mu += yrow[e];
            mu /= (double)D;
            double var = 0.0;
            for (int64_t e = 0; e < D; ++e) var += (yrow[e] - mu) * (yrow[e] - mu);
            var /= (double)D;
            double rs = 1.0 / sqrt(var + eps);
            int64_t row = s0 + i;
            for (int64_t e = 0; e < D; ++e) {
                double z = (yrow[e] - mu) * rs;
                if (out) out[row * D + e] = u[row * D + e] * z;
                if (y) y[row * D + e] = yrow[e];
            }
            if (mean) mean[row] = mu;
            if (rstd) rstd[row] = rs;
        }
        free(yrow);
    }
    return 0;
}

/* ---------------------------------------------------------------- backward */

/*
 * Gradients of  loss = sum(dout (.) O)  with respect to q, k, v, u and both bias tables,
 * by the plain reverse pass of the forward above (chain rule, fp64).  All outputs are
 * overwritten.
 */
int hstu_oracle_bwd(int64_t B, int64_t H, int64_t dqk, int64_t dv, const int64_t *offsets,
                    const int32_t *ctx, const int32_t *tgt, const int64_t *ts, const double *q,
                    const double *k, const double *v, const double *u, const double *rel,
                    int64_t R, const double *tb, int64_t NB, double div, double alpha,
                    int64_t max_attn_len, int64_t N, double eps, int64_t flags,
                    const double *dout, double *dq, double *dk, double *dvv, double *du,
                    double *drel, double *dtb)
{
    oracle_problem P = {B, H, dqk, dv, offsets, ctx, tgt, ts, rel, R, tb, NB, div, alpha,
                        max_attn_len, N, flags};
    const int64_t D = H * dv;
    int64_t T = offsets[B];
    int bad = 0;
    for (int64_t b = 0; b < B; ++b) {
        int64_t s0, L, c, t;
        if (oracle_seq(&P, b, &s0, &L, &c, &t)) bad = 1;
    }
    if (bad || N <= 0) return -1;

    /* Forward again to get Y, mean and rstd. */
    double *y = (double *)malloc(sizeof(double) * (size_t)(T * D + 1));
    double *mean = (double *)malloc(sizeof(double) * (size_t)(T + 1));
    double *rstd = (double *)malloc(sizeof(double) * (size_t)(T + 1));
    double *dy = (double *)malloc(sizeof(double) * (size_t)(T * D + 1));
    hstu_oracle_fwd(B, H, dqk, dv, offsets, ctx, tgt, ts, q, k, v, u, rel, R, tb, NB, div, alpha,
                    max_attn_len, N, eps, flags, NULL, y, mean, rstd);

    /* O = U (.) Zhat, Zhat = (Y - mu) * rstd.  dU = dO (.) Zhat; dZhat = dO (.) U;
     * dY = rstd * (dZhat - mean(dZhat) - Zhat * mean(dZhat (.) Zhat)). */
    for (int64_t row = 0; row < T; ++row) {
        double m1 = 0.0, m2 = 0.0;
        for (int64_t e = 0; e < D; ++e) {
            double z = (y[row * D + e] - mean[row]) * rstd[row];
            double dz = dout[row * D + e] * u[row * D + e];
            du[row * D + e] = dout[row * D + e] * z;
            m1 += dz;
            m2 += dz * z;
        }
        m1 /= (double)D;
        m2 /= (double)D;
        for (int64_t e = 0; e < D; ++e) {
            double z = (y[row * D + e] - mean[row]) * rstd[row];
            double dz = dout[row * D + e] * u[row * D + e];
            dy[row * D + e] = rstd[row] * (dz - m1 - z * m2);
        }
    }

    memset(dq, 0, sizeof(double) * (size_t)(T * H * dqk));
    memset(dk, 0, sizeof(double) * (size_t)(T * H * dqk));
    memset(dvv, 0, sizeof(double) * (size_t)(T * H * dv));
    if (drel && R > 0) memset(drel, 0, sizeof(double) * (size_t)R);
    if (dtb && NB > 0) memset(dtb, 0, sizeof(double) * (size_t)NB);

#pragma omp parallel
    {
        double *lrel = (double *)calloc((size_t)(R > 0 ? R : 1), sizeof(double));
        double *ltb = (double *)calloc((size_t)(NB > 0 ? NB : 1), sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t b = 0; b < B; ++b) {
            int64_t s0, L, c, t;
            oracle_seq(&P, b, &s0, &L, &c, &t);
            int64_t E = L - t;
            for (int64_t h = 0; h < H; ++h)
                for (int64_t i = 0; i < L; ++i) {
                    const double *qi = q + ((s0 + i) * H + h) * dqk;
                    const double *dyi = dy + (s0 + i) * D + h * dv;
                    for (int64_t j = 0; j < L; ++j) {
                        if (!oracle_valid(i, j, L, c, t, max_attn_len, flags)) continue;
                        const double *kj = k + ((s0 + j) * H + h) * dqk;
                        const double *vj = v + ((s0 + j) * H + h) * dv;
                        double dot = 0.0;
                        for (int64_t e = 0; e < dqk; ++e) dot += qi[e] * kj[e];
                        int64_t ri, bk;
                        double s = alpha * dot + oracle_bias(&P, s0, E, i, j, &ri, &bk);
                        double a = oracle_silu(s) / (double)N;
                        /* dV_j += A_ij dY_i ; dA_ij = <dY_i, V_j> */
                        double da = 0.0;
                        double *dvj = dvv + ((s0 + j) * H + h) * dv;
                        for (int64_t e = 0; e < dv; ++e) {
                            dvj[e] += a * dyi[e];
                            da += dyi[e] * vj[e];
                        }
                        double ds = da * oracle_silu_grad(s) / (double)N;
                        double *dqi = dq + ((s0 + i) * H + h) * dqk;
                        double *dkj = dk + ((s0 + j) * H + h) * dqk;
                        for (int64_t e = 0; e < dqk; ++e) {
                            dqi[e] += alpha * ds * kj[e];
                            dkj[e] += alpha * ds * qi[e];
                        }
                        if (ri >= 0) lrel[ri] += ds;
                        if (bk >= 0) ltb[bk] += ds;
                    }
                }
        }
#pragma omp critical
        {
            if (drel)
                for (int64_t r = 0; r < R; ++r) drel[r] += lrel[r];
            if (dtb)
                for (int64_t r = 0; r < NB; ++r) dtb[r] += ltb[r];
        }
        free(lrel);
        free(ltb);
    }
    free(y);
    free(mean);
    free(rstd);
    free(dy);
    return 0;
}

/* Number of threads the OpenMP runtime will use (1 without OpenMP). */
int hstu_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
