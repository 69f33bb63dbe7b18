/*
 * wildcat_oracle.c -- plain, slow, fp64 CPU oracle for the WildCat hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file.  It shares no code with
 * the CUDA path and includes no CUDA header.
 *
 * Every quantity is computed in double precision with sequential sums, in the
 * order the method states it.  Source: "WildCat: Near-Linear Attention in
 * Theory and Practice" (Schroeder & Mackey), Sec. 2.
 *
 *   exact attention    O = D^-1 A V, A = exp(beta Q K^T), D = diag(A 1_n)
 *                      (Sec. 2, opening paragraph; exponential kernel h)
 *   RPCholesky pivots  s ~ p, p proportional to the diagonal of the current
 *                      residual kernel h_res, starting from h(k_l, k_l)
 *                      (Sec. 2, "randomly pivoted Cholesky"; Alg. 1 RPNys)
 *   Nystrom weights    W = h(K_S,K_S)^+ h(K_S,K) applied to (V, 1_n) before
 *                      the queries (Sec. 2, plug-in estimator; Alg. 2
 *                      CompressKV: V_S = W V, w = W 1_n)
 *   plug-in output     O_hat = diag(U W 1)^-1 U W V, U = h(Q, K_S), each entry
 *                      clipped to [v_min j, v_max j] (Sec. 2; Alg. 3 WtdAttn)
 *   inverse route      the same W through h(K_S,K_S)^-1 grown by the rank-one
 *                      update of RPNys as each pivot joins (Sec. 2)
 *
 * Readings where the pages are silent (the text of Alg. 1 and of the update
 * formulas was lost in extraction):
 *   - pivot law p_l = h_res(k_l,k_l) / sum_j h_res(k_j,k_j);
 *   - residual diagonal recursion d_l <- d_l - F_li^2 (Schur complement);
 *   - W is formed through the partial Cholesky factor F (n x r'):
 *     W (V,1) = F_S^-T (F^T (V,1)), F_S = rows S of F (lower triangular);
 *   - the pseudo-inverse is realised by truncation: the factorisation stops
 *     at the first pivot whose residual g_s <= eps * max_l h(k_l,k_l);
 *   - uniforms come from Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11,
 *     "Parallel Random Numbers: As Easy as 1, 2, 3"), key = (seed_lo,
 *     seed_hi), counter = (step, instance, 0, 0); u = (x + 1) 2^-53 with x the
 *     top 53 bits of (x1:x0), so u lies in (0, 1];
 *   - pivot = first index l whose cumulative residual diagonal C_l reaches
 *     u * T, T = sum of the residual diagonal;
 *   - a single shift M_K = max_l |k_l|^2 turns h into c * h (c = exp(-beta
 *     M_K)), which leaves pivot law and W unchanged; the output step uses
 *     M_Q = max_i |q_i| * max_{l in S} |k_l|, which cancels in N / D.
 *
 * Compile-time ORACLE_MUTANT=k plants one deliberate mistake (used only by
 * the mutation test, which checks that the pins catch it).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (SC'11 paper, Sec. 4 "Philox": two 32x32->64 multiplies per */
/* round, Weyl-sequence key schedule, 10 rounds).                            */
/* ------------------------------------------------------------------------ */
static void philox_round(uint32_t c[4], const uint32_t k[2]) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k[0];
    const uint32_t n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k[0] += 0x9E3779B9u; /* golden ratio */
            k[1] += 0xBB67AE85u; /* sqrt(3) - 1 */
        }
        philox_round(c, k);
    }
    out[0] = c[0];
    out[1] = c[1];
    out[2] = c[2];
    out[3] = c[3];
}

/* Pivot uniform for (seed, step, instance), in (0, 1]. */
double oracle_pivot_uniform(uint64_t seed, int64_t step, int64_t inst) {
    const uint32_t ctr[4] = {(uint32_t)step, (uint32_t)inst, 0u, 0u};
#if ORACLE_MUTANT == 14 /* planted: the seed's words swapped in the key */
    const uint32_t key[2] = {(uint32_t)(seed >> 32), (uint32_t)(seed & 0xffffffffu)};
#else
    const uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
#endif
    uint32_t x[4];
    oracle_philox4x32_10(ctr, key, x);
    const uint64_t bits = (((uint64_t)x[1] << 32) | (uint64_t)x[0]) >> 11;
    return ((double)bits + 1.0) * 0x1.0p-53;
}

/* u[b * steps + i] for b < BH, i < steps. */
void oracle_pivot_uniforms(uint64_t seed, int64_t BH, int64_t steps, double* u) {
    for (int64_t b = 0; b < BH; ++b)
        for (int64_t i = 0; i < steps; ++i) u[b * steps + i] = oracle_pivot_uniform(seed, i, b);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* ------------------------------------------------------------------------ */
/* Exact softmax attention, O = D^-1 A V (plain definition, max-subtracted).  */
/* rows == NULL: all m query rows, O is [BH, m, d]; else O is [BH, nrows, d]  */
/* for the listed query rows of every instance.                              */
/* ------------------------------------------------------------------------ */
int oracle_exact_attention(const double* Q, const double* K, const double* V, int64_t BH,
                           int64_t m, int64_t n, int d, double beta, const int64_t* rows,
                           int64_t nrows, double* O) {
    const int64_t nr = rows ? nrows : m;
    int err = 0;
#pragma omp parallel
    {
        double* e = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        if (!e) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < BH * nr; ++t) {
            if (!e) continue;
            const int64_t b = t / nr, ii = t % nr;
            const int64_t i = rows ? rows[ii] : ii;
            const double* q = Q + (b * m + i) * d;
            const double* Kb = K + b * n * d;
            const double* Vb = V + b * n * d;
            double mx = -INFINITY;
            for (int64_t l = 0; l < n; ++l) {
                e[l] = beta * dot(q, Kb + l * d, d);
                if (e[l] > mx) mx = e[l];
            }
            double den = 0.0;
            for (int64_t l = 0; l < n; ++l) {
                e[l] = exp(e[l] - mx);
                den += e[l];
            }
            double* o = O + (b * nr + ii) * d;
            for (int c = 0; c < d; ++c) {
                double num = 0.0;
                for (int64_t l = 0; l < n; ++l) num += e[l] * Vb[l * d + c];
                o[c] = num / den;
            }
        }
        free(e);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* RPCholesky pivot selection with Nystrom factor, one instance.             */
/*   Kb   [n, d]   keys                                                      */
/*   Sfix [r]      fixed pivots (NULL: sample them)                          */
/*   S    [r]      chosen pivots in order, -1 past the rank                  */
/*   F    [r, n]   F[i*n + l] = F_li (column i of the factor, contiguous)    */
/*   hist [r+1, n] residual diagonal at the start of each step (or NULL)     */
/*   margin [r]    distance of u*T to the nearest edge of the chosen bucket, */
/*                 relative to T (or NULL)                                   */
/* returns the effective rank r'.                                            */
/* ------------------------------------------------------------------------ */
static int rpc_one(const double* Kb, int64_t n, int d, double beta, int r, uint64_t seed,
                   int64_t inst, double eps, int shift, const int32_t* Sfix, int32_t* S,
                   double* F, double* hist, double* margin, double* dg, double* g) {
    /* step 1: kernel kappa(x, y) = exp(beta (<x, y> - M_K)) */
    double MK = 0.0;
    for (int64_t l = 0; l < n; ++l) {
        const double sq = dot(Kb + l * d, Kb + l * d, d);
        dg[l] = sq;
        if (l == 0 || sq > MK) MK = sq;
    }
    if (!shift) MK = 0.0;
    /* step 2: residual diagonal starts at kappa(k_l, k_l) */
    double dmax = 0.0;
    for (int64_t l = 0; l < n; ++l) {
        dg[l] = exp(beta * (dg[l] - MK));
        if (dg[l] > dmax) dmax = dg[l];
    }
    memset(F, 0, sizeof(double) * (size_t)r * (size_t)n);
    for (int i = 0; i < r; ++i) S[i] = -1;
    if (margin)
        for (int i = 0; i < r; ++i) margin[i] = NAN;

    int i = 0;
    for (; i < r; ++i) {
        /* 3a: clamp rounding negatives */
        for (int64_t l = 0; l < n; ++l)
            if (dg[l] < 0.0) dg[l] = 0.0;
        if (hist) memcpy(hist + (int64_t)i * n, dg, sizeof(double) * (size_t)n);
        int64_t s = -1;
        if (Sfix) {
            s = Sfix[i];
            if (s < 0 || s >= n) break;
        } else {
            /* 3b: total residual mass */
            double T = 0.0;
            for (int64_t l = 0; l < n; ++l) T += dg[l];
            if (!(T > 0.0)) break;
            /* 3c-d: inverse-CDF draw, first index whose cumulative sum reaches u T */
            const double u = oracle_pivot_uniform(seed, i, inst);
            const double t = u * T;
            double C = 0.0, Cprev = 0.0;
            for (int64_t l = 0; l < n; ++l) {
                Cprev = C;
                C += dg[l];
                if (C >= t) { s = l; break; }
            }
#if ORACLE_MUTANT == 5 /* planted: greedy (largest residual) pivot instead of a draw */
            s = 0;
            for (int64_t l = 1; l < n; ++l)
                if (dg[l] > dg[s]) s = l;
            C = dg[s];
            Cprev = 0.0;
#endif
            if (s < 0) { /* t beyond the rounded total: last index with mass */
                for (int64_t l = n - 1; l >= 0; --l)
                    if (dg[l] > 0.0) { s = l; break; }
                Cprev = C - (s >= 0 ? dg[s] : 0.0);
            }
            if (s < 0) break;
            if (margin) {
                const double lo = t - Cprev, hi = C - t;
                margin[i] = (lo < hi ? lo : hi) / T;
            }
        }
        /* 3e: column of the residual kernel at the pivot,
         *     g_l = kappa(k_l, k_s) - F_l0 F_s0 - F_l1 F_s1 - ... (in that order;
         *     the loop over l is innermost only to walk F contiguously) */
        const double* ks = Kb + s * d;
        for (int64_t l = 0; l < n; ++l) g[l] = exp(beta * (dot(Kb + l * d, ks, d) - MK));
#if ORACLE_MUTANT != 1 /* planted (1): drop the subtraction of earlier columns */
        for (int j = 0; j < i; ++j) {
            const double* Fj = F + (int64_t)j * n;
            const double fs = Fj[s];
            for (int64_t l = 0; l < n; ++l) g[l] -= Fj[l] * fs;
        }
#endif
        /* 3f: truncation stands in for the pseudo-inverse */
        if (!(g[s] > eps * dmax)) break;
        /* 3g: new factor column */
        const double piv = sqrt(g[s]);
        double* Fi = F + (int64_t)i * n;
        for (int64_t l = 0; l < n; ++l) Fi[l] = g[l] / piv;
        S[i] = (int32_t)s;
        /* 3h: residual diagonal update */
        for (int64_t l = 0; l < n; ++l) {
#if ORACLE_MUTANT == 2 /* planted: wrong sign */
            dg[l] += Fi[l] * Fi[l];
#else
            dg[l] -= Fi[l] * Fi[l];
#endif
        }
        dg[s] = 0.0;
    }
    if (hist) {
        for (int64_t l = 0; l < n; ++l)
            if (dg[l] < 0.0) dg[l] = 0.0;
        memcpy(hist + (int64_t)i * n, dg, sizeof(double) * (size_t)n);
    }
    return i;
}

int oracle_rpcholesky(const double* K, int64_t BH, int64_t n, int d, double beta, int r,
                      uint64_t seed, double eps, int shift, const int32_t* S_fixed, int32_t* S,
                      double* F, int32_t* rank, double* hist, double* margin) {
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < BH; ++b) {
        double* dg = (double*)malloc(sizeof(double) * (size_t)n);
        double* g = (double*)malloc(sizeof(double) * (size_t)n);
        if (!dg || !g) {
#pragma omp atomic write
            err = 1;
        } else {
            rank[b] = rpc_one(K + b * n * d, n, d, beta, r, seed, b, eps, shift,
                              S_fixed ? S_fixed + b * r : NULL, S + b * r,
                              F + b * (int64_t)r * n, hist ? hist + b * (int64_t)(r + 1) * n : NULL,
                              margin ? margin + b * r : NULL, dg, g);
        }
        free(dg);
        free(g);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Nystrom weights applied to (V, 1_n), one instance:                       */
/*   Y = F^T (V, 1_n)  (r' x (d+1), sequential over l)                       */
/*   solve F_S^T X = Y by back substitution, F_S[a][j] = F_j(S_a), lower     */
/*   triangular; V_S = X[:, :d], w = X[:, d].  Rows >= r' are zero.          */
/* ------------------------------------------------------------------------ */
static void weights_one(const double* F, const int32_t* S, int rr, const double* Vb, int64_t n,
                        int d, int r, double* VS, double* w, double* Y) {
    const int dp = d + 1;
    for (int j = 0; j < rr; ++j) {
        const double* Fj = F + (int64_t)j * n;
        for (int c = 0; c < dp; ++c) Y[j * dp + c] = 0.0;
        for (int64_t l = 0; l < n; ++l) {
            const double f = Fj[l];
            for (int c = 0; c < d; ++c) Y[j * dp + c] += f * Vb[l * d + c];
            Y[j * dp + d] += f;
        }
    }
    /* back substitution, X overwrites Y */
    for (int a = rr - 1; a >= 0; --a) {
        const double diag = F[(int64_t)a * n + S[a]];
        for (int c = 0; c < dp; ++c) {
            double acc = Y[a * dp + c];
            for (int j = a + 1; j < rr; ++j) {
#if ORACLE_MUTANT == 3 /* planted: transposed operand */
                acc -= F[(int64_t)j * n + S[a]] * Y[j * dp + c];
#else
                acc -= F[(int64_t)a * n + S[j]] * Y[j * dp + c];
#endif
            }
            Y[a * dp + c] = acc / diag;
        }
    }
    for (int a = 0; a < r; ++a) {
        for (int c = 0; c < d; ++c) VS[(int64_t)a * d + c] = a < rr ? Y[a * dp + c] : 0.0;
        w[a] = a < rr ? Y[a * dp + d] : 0.0;
    }
}

int oracle_weights(const double* F, const int32_t* S, const int32_t* rank, const double* V,
                   int64_t BH, int64_t n, int d, int r, double* VS, double* w) {
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < BH; ++b) {
        double* Y = (double*)malloc(sizeof(double) * (size_t)r * (size_t)(d + 1));
        if (!Y) {
#pragma omp atomic write
            err = 1;
        } else {
            weights_one(F + b * (int64_t)r * n, S + b * r, rank[b], V + b * n * d, n, d, r,
                        VS + b * (int64_t)r * d, w + b * r, Y);
        }
        free(Y);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Nystrom weights through the maintained inverse (Sec. 2, the rank-one     */
/* update of RPNys): as pivot s_a joins S, with b = h(K_S, k_s) and         */
/* c = h(k_s, k_s), y = H_S^-1 b and the residual sc = c - b.y,             */
/*   H_S'^-1 = [[H_S^-1, 0], [0, 0]] + g g^T,  g = (y, -1) / sqrt(sc).      */
/* Then W (V, 1_n) = H_S^-1 h(K_S, K) (V, 1_n).  h carries the shift M_K of */
/* the factor route, which cancels in W.  Rows >= r' are zero.              */
/* ------------------------------------------------------------------------ */
static void weights_inverse_one(const double* Kb, const int32_t* S, int rr, const double* Vb,
                                int64_t n, int d, int r, double beta, double* VS, double* w,
                                double* inv, double* y, double* Z) {
    double MK = -INFINITY;
    for (int64_t l = 0; l < n; ++l) {
        const double q = dot(Kb + l * d, Kb + l * d, d);
        if (q > MK) MK = q;
    }
    /* the inverse, grown one pivot at a time (inv is rr x rr, row-major) */
    for (int a = 0; a < rr; ++a) {
        const double* ks = Kb + (int64_t)S[a] * d;
        for (int j = 0; j < a; ++j) {
            double acc = 0.0;
            for (int k = 0; k < a; ++k)
                acc += inv[j * rr + k] * exp(beta * (dot(Kb + (int64_t)S[k] * d, ks, d) - MK));
            y[j] = acc;
        }
        double sc = exp(beta * (dot(ks, ks, d) - MK));
        for (int j = 0; j < a; ++j) sc -= exp(beta * (dot(Kb + (int64_t)S[j] * d, ks, d) - MK)) * y[j];
        for (int j = 0; j < a; ++j)
            for (int k = 0; k < a; ++k)
#if ORACLE_MUTANT == 6 /* planted: wrong sign in the rank-one update */
                inv[j * rr + k] -= y[j] * y[k] / sc;
#else
                inv[j * rr + k] += y[j] * y[k] / sc;
#endif
        for (int j = 0; j < a; ++j) {
            inv[j * rr + a] = -y[j] / sc;
            inv[a * rr + j] = -y[j] / sc;
        }
        inv[a * rr + a] = 1.0 / sc;
    }
    /* Z = h(K_S, K) (V, 1_n), sequential over l */
    const int dp = d + 1;
    for (int a = 0; a < rr; ++a) {
        const double* ks = Kb + (int64_t)S[a] * d;
        for (int c = 0; c < dp; ++c) Z[a * dp + c] = 0.0;
        for (int64_t l = 0; l < n; ++l) {
            const double h = exp(beta * (dot(ks, Kb + l * d, d) - MK));
            for (int c = 0; c < d; ++c) Z[a * dp + c] += h * Vb[l * d + c];
            Z[a * dp + d] += h;
        }
    }
    for (int a = 0; a < r; ++a) {
        for (int c = 0; c < dp; ++c) {
            double acc = 0.0;
            if (a < rr)
                for (int k = 0; k < rr; ++k) acc += inv[a * rr + k] * Z[k * dp + c];
            if (c < d)
                VS[(int64_t)a * d + c] = acc;
            else
                w[a] = acc;
        }
    }
}

int oracle_weights_inverse(const double* K, const int32_t* S, const int32_t* rank, const double* V,
                           int64_t BH, int64_t n, int d, int r, double beta, double* VS, double* w) {
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < BH; ++b) {
        const int rr = rank[b];
        double* inv = (double*)calloc((size_t)rr * (size_t)rr + 1, sizeof(double));
        double* y = (double*)malloc(sizeof(double) * ((size_t)rr + 1));
        double* Z = (double*)malloc(sizeof(double) * ((size_t)rr + 1) * (size_t)(d + 1));
        if (!inv || !y || !Z) {
#pragma omp atomic write
            err = 1;
        } else {
            weights_inverse_one(K + b * n * d, S + b * r, rr, V + b * n * d, n, d, r, beta,
                                VS + b * (int64_t)r * d, w + b * r, inv, y, Z);
        }
        free(inv);
        free(y);
        free(Z);
    }
    return err;
}

/* Column-wise value range over all n value rows of each instance. */
void oracle_value_range(const double* V, int64_t BH, int64_t n, int d, double* vmin,
                        double* vmax) {
    for (int64_t b = 0; b < BH; ++b)
        for (int c = 0; c < d; ++c) {
            double lo = INFINITY, hi = -INFINITY;
#if ORACLE_MUTANT == 15 /* planted: the last row left out */
            for (int64_t l = 0; l + 1 < n; ++l) {
#else
            for (int64_t l = 0; l < n; ++l) {
#endif
                const double v = V[(b * n + l) * d + c];
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            vmin[b * d + c] = lo;
            vmax[b * d + c] = hi;
        }
}

/* K_S = rows S of K (zero rows past the rank). */
void oracle_gather(const double* K, const int32_t* S, const int32_t* rank, int64_t BH, int64_t n,
                   int d, int r, double* KS) {
    for (int64_t b = 0; b < BH; ++b)
        for (int a = 0; a < r; ++a)
            for (int c = 0; c < d; ++c)
                KS[(b * r + a) * d + c] = a < rank[b] ? K[(b * n + S[b * r + a]) * d + c] : 0.0;
}

/* ------------------------------------------------------------------------ */
/* Weighted-coreset plug-in output, one query row:                          */
/*   u_l = exp(beta <q, k_S_l> - beta M_Q); N = sum u_l V_S,l; D = sum u_l w_l */
/*   O_hat_j = fmin(fmax(N_j / D, v_min j), v_max j)                         */
/* ------------------------------------------------------------------------ */
static void attend_row(const double* q, const double* KS, const double* VS, const double* w,
                       int rr, const double* vmin, const double* vmax, int d, double beta,
                       double MQ, double* o, double* N) {
    double D = 0.0;
    for (int c = 0; c < d; ++c) N[c] = 0.0;
    for (int l = 0; l < rr; ++l) {
        const double u = exp(beta * dot(q, KS + (int64_t)l * d, d) - beta * MQ);
        for (int c = 0; c < d; ++c) N[c] += u * VS[(int64_t)l * d + c];
        D += u * w[l];
    }
    for (int c = 0; c < d; ++c) {
#if ORACLE_MUTANT == 4 /* planted: clip bounds swapped */
        o[c] = fmax(fmin(N[c] / D, vmin[c]), vmax[c]);
#else
        o[c] = fmin(fmax(N[c] / D, vmin[c]), vmax[c]);
#endif
    }
}

/* M_Q = max_i |q_i| * max_{l < r'} |k_S_l| of one instance. */
static double query_shift(const double* Qb, int64_t m, const double* KSb, int rr, int d) {
    double qn = 0.0, kn = 0.0;
    for (int64_t i = 0; i < m; ++i) {
        const double v = sqrt(dot(Qb + i * d, Qb + i * d, d));
        if (v > qn) qn = v;
    }
    for (int l = 0; l < rr; ++l) {
        const double v = sqrt(dot(KSb + (int64_t)l * d, KSb + (int64_t)l * d, d));
        if (v > kn) kn = v;
    }
    return qn * kn;
}

int oracle_attend(const double* Q, const double* KS, const double* VS, const double* w,
                  const int32_t* rank, const double* vmin, const double* vmax, int64_t BH,
                  int64_t m, int d, int r, double beta, const int64_t* rows, int64_t nrows,
                  double* O) {
    const int64_t nr = rows ? nrows : m;
    double* MQ = (double*)malloc(sizeof(double) * (size_t)(BH > 0 ? BH : 1));
    if (!MQ) return 1;
    for (int64_t b = 0; b < BH; ++b)
        MQ[b] = query_shift(Q + b * m * d, m, KS + b * (int64_t)r * d, rank[b], d);
    int err = 0;
#pragma omp parallel
    {
        double* N = (double*)malloc(sizeof(double) * (size_t)d);
        if (!N) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < BH * nr; ++t) {
            if (!N) continue;
            const int64_t b = t / nr, ii = t % nr;
            const int64_t i = rows ? rows[ii] : ii;
            attend_row(Q + (b * m + i) * d, KS + b * (int64_t)r * d, VS + b * (int64_t)r * d,
                       w + b * r, rank[b], vmin + b * d, vmax + b * d, d, beta, MQ[b],
                       O + (b * nr + ii) * d, N);
        }
        free(N);
    }
    free(MQ);
    return err;
}

/* ------------------------------------------------------------------------ */
/* The whole WildCat forward (select -> weights -> value range -> attend),   */
/* instance by instance, holding one instance's factor at a time.  S_fixed   */
/* (or NULL) switches to fixed pivots.  rows/nrows as in exact attention.     */
/* ------------------------------------------------------------------------ */
int oracle_wildcat_forward(const double* Q, const double* K, const double* V, int64_t BH,
                           int64_t m, int64_t n, int d, double beta, int r, uint64_t seed,
                           double eps, const int32_t* S_fixed, const int64_t* rows,
                           int64_t nrows, double* O, int32_t* S_out, int32_t* rank_out) {
    const int64_t nr = rows ? nrows : m;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < BH; ++b) {
        double* F = (double*)malloc(sizeof(double) * (size_t)r * (size_t)n);
        double* dg = (double*)malloc(sizeof(double) * (size_t)n);
        double* g = (double*)malloc(sizeof(double) * (size_t)n);
        double* Y = (double*)malloc(sizeof(double) * (size_t)r * (size_t)(d + 1));
        double* VS = (double*)malloc(sizeof(double) * (size_t)r * (size_t)d);
        double* w = (double*)malloc(sizeof(double) * (size_t)r);
        double* KS = (double*)malloc(sizeof(double) * (size_t)r * (size_t)d);
        double* vmin = (double*)malloc(sizeof(double) * (size_t)d);
        double* vmax = (double*)malloc(sizeof(double) * (size_t)d);
        double* N = (double*)malloc(sizeof(double) * (size_t)d);
        int32_t* S = S_out ? S_out + b * r : (int32_t*)malloc(sizeof(int32_t) * (size_t)r);
        if (!F || !dg || !g || !Y || !VS || !w || !KS || !vmin || !vmax || !N || !S) {
#pragma omp atomic write
            err = 1;
        } else {
            const double* Kb = K + b * n * d;
            const double* Vb = V + b * n * d;
            const int rr = rpc_one(Kb, n, d, beta, r, seed, b, eps, 1,
                                   S_fixed ? S_fixed + b * r : NULL, S, F, NULL, NULL, dg, g);
            if (rank_out) rank_out[b] = rr;
            weights_one(F, S, rr, Vb, n, d, r, VS, w, Y);
            int32_t rk = rr;
#if ORACLE_MUTANT == 12 /* planted: the value range of the pivots' rows only */
            for (int c = 0; c < d; ++c) {
                vmin[c] = INFINITY;
                vmax[c] = -INFINITY;
                for (int a = 0; a < rr; ++a) {
                    const double v = Vb[(int64_t)S[a] * d + c];
                    if (v < vmin[c]) vmin[c] = v;
                    if (v > vmax[c]) vmax[c] = v;
                }
            }
#else
            oracle_value_range(Vb, 1, n, d, vmin, vmax);
#endif
            oracle_gather(Kb, S, &rk, 1, n, d, r, KS);
            const double MQ = query_shift(Q + b * m * d, m, KS, rr, d);
            for (int64_t ii = 0; ii < nr; ++ii) {
                const int64_t i = rows ? rows[ii] : ii;
                attend_row(Q + (b * m + i) * d, KS, VS, w, rr, vmin, vmax, d, beta, MQ,
                           O + (b * nr + ii) * d, N);
            }
        }
        free(F); free(dg); free(g); free(Y); free(VS); free(w); free(KS);
        free(vmin); free(vmax); free(N);
        if (!S_out) free(S);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Divide and conquer (Sec. 2, binning), with the optional recentring and   */
/* temperature of Sec. 2: the n keys of an instance are cut                 */
/* into nbins contiguous bins of n / nbins keys; each bin gets its own      */
/* RPNys coreset of r / nbins pivots and its own Nystrom weights over its    */
/* own keys (the pivot draws of bin q of instance b use instance index      */
/* b * nbins + q); the coreset is the union and the weights are block       */
/* diagonal.  The plug-in output then attends over the union exactly as     */
/* without bins (rows past a bin's rank are zero and contribute nothing).   */
/*   S_fixed  [BH, r]  global key indices to use instead of draws (or NULL); */
/*            row q * (r / nbins) + a must lie in bin q, -1 ends the bin    */
/*   S_out    [BH, r]  global key index of every union row (-1 past a bin's */
/*            rank)                                                         */
/*   rank_out [BH, nbins] effective rank of every bin                       */
/* ------------------------------------------------------------------------ */
int oracle_wildcat_forward_binned(const double* Q, const double* K, const double* V, int64_t BH,
                                  int64_t m, int64_t n, int d, double beta, int r, int nbins,
                                  int recenter, double tau, uint64_t seed, double eps,
                                  const int32_t* S_fixed, const int64_t* rows, int64_t nrows,
                                  double* O, int32_t* S_out, int32_t* rank_out) {
    if (nbins < 1 || n % nbins || r % nbins || !(tau > 0.0)) return 2;
    /* Sec. 2: selection and weights use the recentred keys k_l - kbar and the
     * key kernel exp(beta <x, y> / tau^2) (keys K / tau, queries tau Q); the
     * output step uses the original keys and beta, which differs only by a
     * per-query factor that cancels in N / D. */
#if ORACLE_MUTANT == 10 /* planted: the temperature applied once instead of squared */
    const double beta_key = beta / tau;
#else
    const double beta_key = beta / (tau * tau);
#endif
    const int64_t nb = n / nbins;
    const int rb = r / nbins;
    const int64_t nr = rows ? nrows : m;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < BH; ++b) {
        double* F = (double*)malloc(sizeof(double) * (size_t)rb * (size_t)nb);
        double* dg = (double*)malloc(sizeof(double) * (size_t)nb);
        double* g = (double*)malloc(sizeof(double) * (size_t)nb);
        double* Y = (double*)malloc(sizeof(double) * (size_t)rb * (size_t)(d + 1));
        double* VS = (double*)malloc(sizeof(double) * (size_t)r * (size_t)d);
        double* w = (double*)malloc(sizeof(double) * (size_t)r);
        double* KS = (double*)malloc(sizeof(double) * (size_t)r * (size_t)d);
        double* vmin = (double*)malloc(sizeof(double) * (size_t)d);
        double* vmax = (double*)malloc(sizeof(double) * (size_t)d);
        double* N = (double*)malloc(sizeof(double) * (size_t)d);
        int32_t* Sb = (int32_t*)malloc(sizeof(int32_t) * (size_t)rb);
        int32_t* Sf = (int32_t*)malloc(sizeof(int32_t) * (size_t)rb);
        double* Kc = (double*)malloc(sizeof(double) * (size_t)n * (size_t)d);
        if (!F || !dg || !g || !Y || !VS || !w || !KS || !vmin || !vmax || !N || !Sb || !Sf || !Kc) {
#pragma omp atomic write
            err = 1;
        } else {
            const double* Kb = K + b * n * d;
            const double* Vb = V + b * n * d;
            for (int c = 0; c < d; ++c) {
                double mean = 0.0;
                if (recenter) {
#if ORACLE_MUTANT == 11 /* planted: the mean of the first bin's keys only */
                    for (int64_t l = 0; l < nb; ++l) mean += Kb[l * d + c];
                    mean /= (double)nb;
#else
                    for (int64_t l = 0; l < n; ++l) mean += Kb[l * d + c];
                    mean /= (double)n;
#endif
                }
                for (int64_t l = 0; l < n; ++l) Kc[l * d + c] = Kb[l * d + c] - mean;
            }
            for (int q = 0; q < nbins; ++q) {
                const double* Kq = Kb + (int64_t)q * nb * d;
                const double* Kcq = Kc + (int64_t)q * nb * d;
                const double* Vq = Vb + (int64_t)q * nb * d;
                if (S_fixed)
                    for (int a = 0; a < rb; ++a) {
                        const int32_t sg = S_fixed[b * r + q * rb + a];
                        Sf[a] = (sg >= q * nb && sg < (q + 1) * nb) ? (int32_t)(sg - q * nb) : -1;
                    }
#if ORACLE_MUTANT == 8 /* planted: every bin of an instance draws the instance's stream */
                const int64_t ctr = b;
#else
                const int64_t ctr = b * nbins + q;
#endif
                const int rr = rpc_one(Kcq, nb, d, beta_key, rb, seed, ctr, eps, 1,
                                       S_fixed ? Sf : NULL, Sb, F, NULL, NULL, dg, g);
                if (rank_out) rank_out[b * nbins + q] = rr;
                weights_one(F, Sb, rr, Vq, nb, d, rb, VS + (int64_t)q * rb * d, w + q * rb, Y);
                for (int a = 0; a < rb; ++a) {
                    const int row = q * rb + a;
                    if (S_out) S_out[b * r + row] = a < rr ? (int32_t)(q * nb + Sb[a]) : -1;
                    for (int c = 0; c < d; ++c)
                        KS[(int64_t)row * d + c] = a < rr ? Kq[(int64_t)Sb[a] * d + c] : 0.0;
                }
            }
#if ORACLE_MUTANT == 9 /* planted: the value range of the first bin only */
            oracle_value_range(Vb, 1, nb, d, vmin, vmax);
#else
            oracle_value_range(Vb, 1, n, d, vmin, vmax);
#endif
            const double MQ = query_shift(Q + b * m * d, m, KS, r, d);
            for (int64_t ii = 0; ii < nr; ++ii) {
                const int64_t i = rows ? rows[ii] : ii;
                attend_row(Q + (b * m + i) * d, KS, VS, w, r, vmin, vmax, d, beta, MQ,
                           O + (b * nr + ii) * d, N);
            }
        }
        free(F); free(dg); free(g); free(Y); free(VS); free(w); free(KS);
        free(vmin); free(vmax); free(N); free(Sb); free(Sf); free(Kc);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* KV-cache decode with new tokens (Sec. 2: after CompressKV, m new tokens  */
/* cost O(rmd + m^2 d) instead of O(nmd + m^2 d)).  New query i attends over */
/* the weighted coreset of the compressed cache and, exactly, over the new  */
/* tokens j <= i (causal):                                                  */
/*   N_i = sum_l u_il V_S,l + sum_{j<=i} e_ij v_j                           */
/*   D_i = sum_l u_il w_l   + sum_{j<=i} e_ij                               */
/*   u_il = exp(beta <q_i, k_S_l> - beta M), e_ij = exp(beta <q_i, k_j> - beta M) */
/* with one shift M = max_i |q_i| * max(max_l |k_S_l|, max_j |k_j|), and    */
/* O_i = clip(N_i / D_i) to the range of the old values (vmin, vmax of the  */
/* cache) and the new values together.                                      */
/*   Qn, Kn, Vn [BH, m, d] new tokens; KS, VS [BH, r, d], w [BH, r], rank   */
/*   [BH], vmin/vmax [BH, d] from the compressed cache; O [BH, m, d]        */
/* ------------------------------------------------------------------------ */
int oracle_decode_attend(const double* Qn, const double* Kn, const double* Vn, const double* KS,
                         const double* VS, const double* w, const int32_t* rank,
                         const double* vmin, const double* vmax, int64_t BH, int64_t m, int d,
                         int r, double beta, double* O) {
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < BH; ++b) {
        double* N = (double*)malloc(sizeof(double) * (size_t)d);
        double* lo = (double*)malloc(sizeof(double) * (size_t)d);
        double* hi = (double*)malloc(sizeof(double) * (size_t)d);
        if (!N || !lo || !hi) {
#pragma omp atomic write
            err = 1;
        } else {
            const double* Qb = Qn + b * m * d;
            const double* Kb = Kn + b * m * d;
            const double* Vb = Vn + b * m * d;
            const double* KSb = KS + b * (int64_t)r * d;
            const double* VSb = VS + b * (int64_t)r * d;
            const int rr = rank[b];
            double qn = 0.0, kn = 0.0;
            for (int64_t i = 0; i < m; ++i) {
                const double v = sqrt(dot(Qb + i * d, Qb + i * d, d));
                if (v > qn) qn = v;
                const double u = sqrt(dot(Kb + i * d, Kb + i * d, d));
                if (u > kn) kn = u;
            }
            for (int l = 0; l < rr; ++l) {
                const double v = sqrt(dot(KSb + (int64_t)l * d, KSb + (int64_t)l * d, d));
                if (v > kn) kn = v;
            }
            const double M = qn * kn;
            for (int c = 0; c < d; ++c) {
                lo[c] = vmin[b * d + c];
                hi[c] = vmax[b * d + c];
#if ORACLE_MUTANT == 13 /* planted: the range of the cache's values only */
                continue;
#endif
                for (int64_t j = 0; j < m; ++j) {
                    const double v = Vb[j * d + c];
                    if (v < lo[c]) lo[c] = v;
                    if (v > hi[c]) hi[c] = v;
                }
            }
            for (int64_t i = 0; i < m; ++i) {
                const double* q = Qb + i * d;
                double D = 0.0;
                for (int c = 0; c < d; ++c) N[c] = 0.0;
                for (int l = 0; l < rr; ++l) {
                    const double u = exp(beta * dot(q, KSb + (int64_t)l * d, d) - beta * M);
                    for (int c = 0; c < d; ++c) N[c] += u * VSb[(int64_t)l * d + c];
                    D += u * w[b * r + l];
                }
#if ORACLE_MUTANT == 7 /* planted: a new token does not see itself */
                for (int64_t j = 0; j < i; ++j) {
#else
                for (int64_t j = 0; j <= i; ++j) {
#endif
                    const double e = exp(beta * dot(q, Kb + j * d, d) - beta * M);
                    for (int c = 0; c < d; ++c) N[c] += e * Vb[j * d + c];
                    D += e;
                }
                for (int c = 0; c < d; ++c) O[(b * m + i) * d + c] = fmin(fmax(N[c] / D, lo[c]), hi[c]);
            }
        }
        free(N); free(lo); free(hi);
    }
    return err;
}
