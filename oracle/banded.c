/*
 * Float64 banded CPU oracle for blockwise, fixed-support, balanced log-domain Sinkhorn
 * attention.  TEST INFRASTRUCTURE ONLY: it is loaded by tests/ and by bench.py's CPU
 * baseline, never by the product library, and shares no code or headers with it.
 *
 * It computes exactly what oracle/eot_oracle.py computes (the same equations, the same
 * readings of the pages), but keeps S in band storage [L][2h+1] instead of a dense L x L
 * array, so that long sequences fit.  It is pinned to the dense oracle by tests.
 *
 * Source: "Blockwise Differentiable Sinkhorn Attention", technical summary
 * (gist.science 2605.08123):
 *   §2.1  fixed band support of width W, epsilon absorbed into S, T stopped balanced
 *         Sinkhorn steps, then an R-step differentiable tail;
 *   §2.2  exact tail adjoint through the staircase factors P(a,b);
 *   §2.3  dustbin token plus inactive fillers on an extended state space.
 * Equations (one unit = one (batch, head) pair; h = W / 2):
 *   S_ij = scale <q_i, k_j> on Omega = {i, j active, |i - j| <= h}, plus, with a dustbin
 *   D, (i, D), (D, j) for active real i, j and (D, D).
 *   u_i = log a_i - LSE_j (S_ij + v_j),   v_j = log b_j - LSE_i (S_ij + u_i)
 *   O = diag(1/a) exp(S + u(R) + v(R)) V
 * Inactive tokens get u = v = 0 and zero rows in O, dQ, dK, dV.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC banded.c -o libeot_banded.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int L, d, W, h, R;
    double scale;
    const double *q, *k, *v;   /* [L][d] */
    unsigned char *real;       /* [L] active real token */
    int D;                     /* dustbin index or -1 */
    int dself;                 /* (D, D) in the support */
    double *log_a;             /* [L], -inf inactive */
    int n_active;
    double *S;                 /* [L][2h+1], -inf outside Omega (dustbin links kept apart) */
    double *sDr;               /* [L]: S_iD (row i, dustbin column) */
    double *sDc;               /* [L]: S_Dj (dustbin row, column j) */
    double sDD;
} unit_t;

static inline int wid(const unit_t *U) { return 2 * U->h + 1; }

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += a[t] * b[t];
    return s;
}

/* Active set, uniform marginals and band scores for one unit (§2.1, §2.3). */
static int unit_init(unit_t *U, int L, int d, int W, int R, double scale, const double *q,
                     const double *k, const double *v, const unsigned char *mask_row,
                     int dustbin, int dustbin_index, double mass, int dself)
{
    U->L = L; U->d = d; U->W = W; U->h = W / 2; U->R = R; U->scale = scale;
    U->q = q; U->k = k; U->v = v; U->dself = dself;
    U->real = (unsigned char *)malloc((size_t)L);
    U->log_a = (double *)malloc(sizeof(double) * (size_t)L);
    U->S = (double *)malloc(sizeof(double) * (size_t)L * (size_t)wid(U));
    U->sDr = (double *)calloc((size_t)L, sizeof(double));
    U->sDc = (double *)calloc((size_t)L, sizeof(double));
    if (!U->real || !U->log_a || !U->S || !U->sDr || !U->sDc) return -1;
    int n_real = 0;
    for (int i = 0; i < L; ++i) {
        int r = mask_row ? (mask_row[i] != 0) : 1;
        if (dustbin && i >= dustbin_index) r = 0;
        U->real[i] = (unsigned char)r;
        n_real += r;
    }
    int use_db = dustbin && n_real > 0 && mass > 0.0;
    U->D = use_db ? dustbin_index : -1;
    double real_mass = use_db ? (1.0 - mass) : 1.0;
    for (int i = 0; i < L; ++i)
        U->log_a[i] = U->real[i] ? log(real_mass / n_real) : -INFINITY;
    if (use_db) U->log_a[U->D] = log(mass);
    U->n_active = n_real + (use_db ? 1 : 0);
    const int w = wid(U), h = U->h;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        double *row = U->S + (size_t)i * w;
        for (int o = 0; o < w; ++o) {
            int j = i - h + o;
            row[o] = (j >= 0 && j < L && U->real[i] && U->real[j])
                         ? scale * dot(q + (size_t)i * d, k + (size_t)j * d, d) : -INFINITY;
        }
        if (U->D >= 0 && U->real[i]) {
            U->sDr[i] = scale * dot(q + (size_t)i * d, k + (size_t)U->D * d, d);
            U->sDc[i] = scale * dot(q + (size_t)U->D * d, k + (size_t)i * d, d);
        }
    }
    U->sDD = (U->D >= 0) ? scale * dot(q + (size_t)U->D * d, k + (size_t)U->D * d, d) : 0.0;
    return 0;
}

static void unit_free(unit_t *U)
{
    free(U->real); free(U->log_a); free(U->S); free(U->sDr); free(U->sDc);
}

static inline int is_active(const unit_t *U, int i) { return U->real[i] || i == U->D; }

/* LSE over row i of (S_ij + x_j), band entries plus the dustbin column; max-shifted. */
static double row_lse(const unit_t *U, int i, const double *x)
{
    const int w = wid(U), h = U->h;
    const double *row = U->S + (size_t)i * w;
    double m = -INFINITY;
    if (i == U->D) {
        for (int j = 0; j < U->L; ++j)
            if (U->real[j]) { double t = U->sDc[j] + x[j]; if (t > m) m = t; }
        if (U->dself) { double t = U->sDD + x[i]; if (t > m) m = t; }
        if (!isfinite(m)) return -INFINITY;
        double s = 0.0;
        for (int j = 0; j < U->L; ++j)
            if (U->real[j]) s += exp(U->sDc[j] + x[j] - m);
        if (U->dself) s += exp(U->sDD + x[i] - m);
        return m + log(s);
    }
    for (int o = 0; o < w; ++o) {
        int j = i - h + o;
        if (row[o] > -INFINITY) { double t = row[o] + x[j]; if (t > m) m = t; }
    }
    if (U->D >= 0) { double t = U->sDr[i] + x[U->D]; if (t > m) m = t; }
    if (!isfinite(m)) return -INFINITY;
    double s = 0.0;
    for (int o = 0; o < w; ++o) {
        int j = i - h + o;
        if (row[o] > -INFINITY) s += exp(row[o] + x[j] - m);
    }
    if (U->D >= 0) s += exp(U->sDr[i] + x[U->D] - m);
    return m + log(s);
}

/* LSE over column j of (S_ij + y_i). */
static double col_lse(const unit_t *U, int j, const double *y)
{
    const int w = wid(U), h = U->h;
    double m = -INFINITY;
    if (j == U->D) {
        for (int i = 0; i < U->L; ++i)
            if (U->real[i]) { double t = U->sDr[i] + y[i]; if (t > m) m = t; }
        if (U->dself) { double t = U->sDD + y[j]; if (t > m) m = t; }
        if (!isfinite(m)) return -INFINITY;
        double s = 0.0;
        for (int i = 0; i < U->L; ++i)
            if (U->real[i]) s += exp(U->sDr[i] + y[i] - m);
        if (U->dself) s += exp(U->sDD + y[j] - m);
        return m + log(s);
    }
    for (int i = j - h; i <= j + h; ++i) {
        if (i < 0 || i >= U->L) continue;
        double sij = U->S[(size_t)i * w + (j - i + h)];
        if (sij > -INFINITY) { double t = sij + y[i]; if (t > m) m = t; }
    }
    if (U->D >= 0) { double t = U->sDc[j] + y[U->D]; if (t > m) m = t; }
    if (!isfinite(m)) return -INFINITY;
    double s = 0.0;
    for (int i = j - h; i <= j + h; ++i) {
        if (i < 0 || i >= U->L) continue;
        double sij = U->S[(size_t)i * w + (j - i + h)];
        if (sij > -INFINITY) s += exp(sij + y[i] - m);
    }
    if (U->D >= 0) s += exp(U->sDc[j] + y[U->D] - m);
    return m + log(s);
}

/* One balanced step (§2.1): u from v, then v from u.  Inactive entries become 0. */
static void sinkhorn_step(const unit_t *U, double *u, double *v)
{
    const int L = U->L;
    double *vm = (double *)malloc(sizeof(double) * (size_t)L);
    double *um = (double *)malloc(sizeof(double) * (size_t)L);
    for (int j = 0; j < L; ++j) vm[j] = is_active(U, j) ? v[j] : -INFINITY;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) u[i] = is_active(U, i) ? U->log_a[i] - row_lse(U, i, vm) : 0.0;
    for (int i = 0; i < L; ++i) um[i] = is_active(U, i) ? u[i] : -INFINITY;
#pragma omp parallel for schedule(static)
    for (int j = 0; j < L; ++j) v[j] = is_active(U, j) ? U->log_a[j] - col_lse(U, j, um) : 0.0;
    free(vm); free(um);
}

/* Visit every support entry (i, j, S_ij) of the unit, band and dustbin links alike. */
#define FOR_ROW_ENTRIES(U, i, j, sij, ...)                                           \
    do {                                                                             \
        const int w_ = wid(U), h_ = (U)->h;                                          \
        if ((i) == (U)->D) {                                                         \
            for (int j = 0; j < (U)->L; ++j)                                         \
                if ((U)->real[j]) { double sij = (U)->sDc[j]; __VA_ARGS__ }                 \
            if ((U)->dself) { int j = (U)->D; double sij = (U)->sDD; __VA_ARGS__ }          \
        } else if ((U)->real[i]) {                                                   \
            const double *row_ = (U)->S + (size_t)(i) * w_;                          \
            for (int o_ = 0; o_ < w_; ++o_) {                                        \
                if (row_[o_] == -INFINITY) continue;                                 \
                int j = (i) - h_ + o_; double sij = row_[o_]; __VA_ARGS__                 \
            }                                                                        \
            if ((U)->D >= 0) { int j = (U)->D; double sij = (U)->sDr[i]; __VA_ARGS__ }      \
        }                                                                            \
    } while (0)

/*
 * Forward for one unit.  u_tail/v_tail: [R+1][L]; O: [L][d].
 */
static void unit_forward(unit_t *U, int T, double *O, double *u_tail, double *v_tail)
{
    const int L = U->L, d = U->d, R = U->R;
    double *u = (double *)calloc((size_t)L, sizeof(double));
    double *v = (double *)calloc((size_t)L, sizeof(double));
    for (int t = 0; t < T; ++t) sinkhorn_step(U, u, v);            /* stopped base */
    memcpy(u_tail, u, sizeof(double) * (size_t)L);
    memcpy(v_tail, v, sizeof(double) * (size_t)L);
    for (int kk = 1; kk <= R; ++kk) {                                /* tail */
        sinkhorn_step(U, u, v);
        memcpy(u_tail + (size_t)kk * L, u, sizeof(double) * (size_t)L);
        memcpy(v_tail + (size_t)kk * L, v, sizeof(double) * (size_t)L);
    }
    const double *uR = u_tail + (size_t)R * L, *vR = v_tail + (size_t)R * L;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        double *o = O + (size_t)i * d;
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        if (!is_active(U, i)) continue;
        double inv_a = exp(-U->log_a[i]);
        FOR_ROW_ENTRIES(U, i, j, sij, {
            double p = exp(sij + uR[i] + vR[j]) * inv_a;
            const double *vj = U->v + (size_t)j * d;
            for (int t = 0; t < d; ++t) o[t] += p * vj[t];
        });
    }
    free(u); free(v);
}

/* Visit every support entry (i, j, S_ij) of column j: band rows plus the dustbin row. */
#define FOR_COL_ENTRIES(U, j, i, sij, ...)                                           \
    do {                                                                             \
        const int w_ = wid(U), h_ = (U)->h;                                          \
        if ((j) == (U)->D) {                                                         \
            for (int i = 0; i < (U)->L; ++i)                                         \
                if ((U)->real[i]) { double sij = (U)->sDr[i]; __VA_ARGS__ }          \
            if ((U)->dself) { int i = (U)->D; double sij = (U)->sDD; __VA_ARGS__ }   \
        } else if ((U)->real[j]) {                                                   \
            for (int i = (j) - h_; i <= (j) + h_; ++i) {                             \
                if (i < 0 || i >= (U)->L) continue;                                  \
                double sij = (U)->S[(size_t)i * w_ + ((j) - i + h_)];                \
                if (sij == -INFINITY) continue;                                      \
                __VA_ARGS__                                                          \
            }                                                                        \
            if ((U)->D >= 0) { int i = (U)->D; double sij = (U)->sDc[j]; __VA_ARGS__ } \
        }                                                                            \
    } while (0)

/*
 * Tail adjoint for one unit (§2.2), same chain as the dense oracle:
 *   dP_ij = <dO_i, V_j> / a_i, G = P(R,R) * dP
 *   beta_R = colsum G, alpha_R = rowsum G - P(R,R)(beta_R / b)
 *   beta_k = -P(k+1,k)^T (alpha_{k+1} / a), alpha_k = -P(k,k)(beta_k / b)
 *   dS = G - sum_k [P(k,k) (beta_k/b)_j + P(k,k-1) (alpha_k/a)_i]
 *   dQ = scale dS K, dK = scale dS^T Q, dV = P(R,R)^T (dO / a)
 * Row-owned sums loop over the row's support, column-owned sums over the column's
 * support, so every loop is parallel over its owner.
 */
static void unit_backward(unit_t *U, const double *u_tail, const double *v_tail, const double *dO,
                          double *dQ, double *dK, double *dV)
{
    const int L = U->L, d = U->d, R = U->R;
    const double sc = U->scale;
#define UT(k_, i_) u_tail[(size_t)(k_) * L + (i_)]
#define VT(k_, j_) v_tail[(size_t)(k_) * L + (j_)]
    double *inv_a = (double *)malloc(sizeof(double) * (size_t)L);
    for (int i = 0; i < L; ++i) inv_a[i] = is_active(U, i) ? exp(-U->log_a[i]) : 0.0;
    double *alpha = (double *)calloc((size_t)(R + 1) * L, sizeof(double));
    double *beta = (double *)calloc((size_t)(R + 1) * L, sizeof(double));
    memset(dQ, 0, sizeof(double) * (size_t)L * d);
    memset(dK, 0, sizeof(double) * (size_t)L * d);
    memset(dV, 0, sizeof(double) * (size_t)L * d);

    if (R > 0) {
        double *Rb = beta + (size_t)R * L, *Ra = alpha + (size_t)R * L;
#pragma omp parallel for schedule(dynamic, 64)
        for (int j = 0; j < L; ++j) {            /* beta_R = colsum G */
            if (!is_active(U, j)) continue;
            double acc = 0.0;
            FOR_COL_ENTRIES(U, j, i, sij, {
                acc += exp(sij + UT(R, i) + VT(R, j)) * dot(dO + (size_t)i * d, U->v + (size_t)j * d, d) * inv_a[i];
            });
            Rb[j] = acc;
        }
#pragma omp parallel for schedule(dynamic, 64)
        for (int i = 0; i < L; ++i) {            /* alpha_R = rowsum G - P(R,R)(beta_R/b) */
            if (!is_active(U, i)) continue;
            double acc = 0.0;
            const double *doi = dO + (size_t)i * d;
            FOR_ROW_ENTRIES(U, i, j, sij, {
                double p = exp(sij + UT(R, i) + VT(R, j));
                acc += p * (dot(doi, U->v + (size_t)j * d, d) * inv_a[i] - Rb[j] * inv_a[j]);
            });
            Ra[i] = acc;
        }
        for (int kk = R - 1; kk >= 1; --kk) {
            double *bk = beta + (size_t)kk * L, *ak = alpha + (size_t)kk * L;
            const double *a1 = alpha + (size_t)(kk + 1) * L;
#pragma omp parallel for schedule(dynamic, 64)
            for (int j = 0; j < L; ++j) {        /* beta_k = -P(k+1,k)^T (alpha_{k+1}/a) */
                if (!is_active(U, j)) continue;
                double acc = 0.0;
                FOR_COL_ENTRIES(U, j, i, sij, { acc += exp(sij + UT(kk + 1, i) + VT(kk, j)) * a1[i] * inv_a[i]; });
                bk[j] = -acc;
            }
#pragma omp parallel for schedule(dynamic, 64)
            for (int i = 0; i < L; ++i) {        /* alpha_k = -P(k,k)(beta_k/b) */
                if (!is_active(U, i)) continue;
                double acc = 0.0;
                FOR_ROW_ENTRIES(U, i, j, sij, { acc += exp(sij + UT(kk, i) + VT(kk, j)) * bk[j] * inv_a[j]; });
                ak[i] = -acc;
            }
        }
    }
    /* dS_ij; dQ by rows, dK and dV by columns. */
#define DS_ENTRY(i_, j_, sij_, p_, ds_)                                                        \
    double p_ = exp((sij_) + UT(R, i_) + VT(R, j_));                                           \
    double ds_ = p_ * dot(dO + (size_t)(i_) * d, U->v + (size_t)(j_) * d, d) * inv_a[i_];      \
    for (int kk = 1; kk <= R; ++kk) {                                                          \
        ds_ -= exp((sij_) + UT(kk, i_) + VT(kk, j_)) * beta[(size_t)kk * L + (j_)] * inv_a[j_]; \
        ds_ -= exp((sij_) + UT(kk, i_) + VT(kk - 1, j_)) * alpha[(size_t)kk * L + (i_)] * inv_a[i_]; \
    }
#pragma omp parallel for schedule(dynamic, 64)
    for (int i = 0; i < L; ++i) {
        if (!is_active(U, i)) continue;
        double *dqi = dQ + (size_t)i * d;
        FOR_ROW_ENTRIES(U, i, j, sij, {
            DS_ENTRY(i, j, sij, p, ds)
            (void)p;
            const double *kj = U->k + (size_t)j * d;
            for (int t = 0; t < d; ++t) dqi[t] += sc * ds * kj[t];
        });
    }
#pragma omp parallel for schedule(dynamic, 64)
    for (int j = 0; j < L; ++j) {
        if (!is_active(U, j)) continue;
        double *dkj = dK + (size_t)j * d, *dvj = dV + (size_t)j * d;
        FOR_COL_ENTRIES(U, j, i, sij, {
            DS_ENTRY(i, j, sij, p, ds)
            const double *qi = U->q + (size_t)i * d, *doi = dO + (size_t)i * d;
            for (int t = 0; t < d; ++t) {
                dkj[t] += sc * ds * qi[t];
                dvj[t] += p * doi[t] * inv_a[i];
            }
        });
    }
#undef DS_ENTRY
#undef UT
#undef VT
    free(inv_a); free(alpha); free(beta);
}

/*
 * Batched entry points over [B][H][L][d] double arrays; mask is [B][L] or NULL.
 * ``units``/``n_units`` optionally restrict the work to a list of flattened b*H+h indices
 * (NULL: all).  Returns 0 on success, -1 on allocation failure.
 */
int eot_banded_forward(int B, int H, int L, int d, int W, int T, int R, double scale,
                       const double *Q, const double *K, const double *V, const unsigned char *mask,
                       int dustbin, int dustbin_index, double mass, int dself,
                       const int *units, int n_units, double *O, double *u_tail, double *v_tail)
{
    int n = units ? n_units : B * H;
    for (int t = 0; t < n; ++t) {
        int bh = units ? units[t] : t;
        int b = bh / H;
        size_t off = (size_t)bh * L * d;
        unit_t U;
        if (unit_init(&U, L, d, W, R, scale, Q + off, K + off, V + off, mask ? mask + (size_t)b * L : NULL,
                      dustbin, dustbin_index, mass, dself)) { unit_free(&U); return -1; }
        unit_forward(&U, T, O + off, u_tail + (size_t)bh * (R + 1) * L, v_tail + (size_t)bh * (R + 1) * L);
        unit_free(&U);
    }
    return 0;
}

int eot_banded_backward(int B, int H, int L, int d, int W, int R, double scale,
                        const double *Q, const double *K, const double *V, const unsigned char *mask,
                        int dustbin, int dustbin_index, double mass, int dself,
                        const int *units, int n_units, const double *u_tail, const double *v_tail,
                        const double *dO, double *dQ, double *dK, double *dV)
{
    int n = units ? n_units : B * H;
    for (int t = 0; t < n; ++t) {
        int bh = units ? units[t] : t;
        int b = bh / H;
        size_t off = (size_t)bh * L * d;
        unit_t U;
        if (unit_init(&U, L, d, W, R, scale, Q + off, K + off, V + off, mask ? mask + (size_t)b * L : NULL,
                      dustbin, dustbin_index, mass, dself)) { unit_free(&U); return -1; }
        unit_backward(&U, u_tail + (size_t)bh * (R + 1) * L, v_tail + (size_t)bh * (R + 1) * L, dO + off,
                      dQ + off, dK + off, dV + off);
        unit_free(&U);
    }
    return 0;
}
