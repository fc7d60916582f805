/*
 * Oracle for the block selected inverse -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU implementation in double precision of
 * what the GPU library computes.  Only the tests, the smoke check and the
 * bench's CPU-baseline / reference arm may load it; the product path never
 * does.  It shares no code, header or table with the CUDA library.
 *
 * Sources (gabp-sparse-inv 0.3.2, PyPI page):
 *   - "Implemented and tested kernels" -> Chain: block LDL^T factorisation of
 *     a block-tridiagonal SPD matrix followed by the Takahashi back-recursion,
 *     returning the diagonal blocks and the first sub-diagonal blocks of A^-1.
 *   - "Implemented and tested kernels" -> Tree: parent array, one edge block
 *     per non-root node with edge[v] = A_{parent(v), v}; collect from the
 *     leaves to the root, then distribute from the root to the leaves.
 *   - "Quickstart": inputs diag [L,b,b], lower [L-1,b,b]; G_diag[v] = (A^-1)_vv,
 *     G_edge[v] = (A^-1)_{parent(v),v}, root slot zero.
 *   - "Gaussian sampling" / "junction_logdet": log det A from the same
 *     LDL^T factorisation; "junction_solve": x = A^-1 r sharing that factor.
 * (sparsax, PyPI page, "Features": a matrix that is not positive definite is
 *  an error, reported here through info[] as the first failing block.)
 *
 * The recursion, in the pages' notation (S = Schur complement, B_i = lower[i]
 * = A_{i+1,i}):
 *   collect     S_0 = D_0,  S_{i+1} = D_{i+1} - B_i S_i^-1 B_i^T
 *   log-det     log|A| = sum_i log det S_i
 *   distribute  G_{L-1,L-1} = S_{L-1}^-1,
 *               G_{i+1,i} = -G_{i+1,i+1} B_i S_i^-1,
 *               G_ii      = S_i^-1 - S_i^-1 B_i^T G_{i+1,i}
 *   solve       y_0 = r_0, y_{i+1} = r_{i+1} - B_i S_i^-1 y_i,
 *               x_{L-1} = S_{L-1}^-1 y_{L-1}, x_i = S_i^-1 (y_i - B_i^T x_{i+1})
 * Each S_i^-1 is formed from a textbook Cholesky factor S = R R^T (R lower):
 * S^-1 = R^-T R^-1, and log det S = 2 sum_k log R_kk.
 *
 * Readings where the pages are silent: only the lower triangle of a diagonal
 * block is read (the upper one is taken as its mirror); the returned G_ii is
 * symmetrised as (G + G^T)/2 and the largest |G - G^T| before that is
 * reported; a non-positive (or NaN) Cholesky pivot in block i stops that
 * batch element with info = i (else info = -1).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------- small dense helpers (row-major b x b, naive loops) ---------- */

/* R := lower Cholesky factor of the symmetric matrix S (only S's lower
 * triangle is read).  Returns 0, or -1 if a pivot is not > 0. */
static int cholesky_lower(int b, const double *S, double *R)
{
    for (int i = 0; i < b * b; ++i) R[i] = 0.0;
    for (int j = 0; j < b; ++j) {
        double d = S[j * b + j];
        for (int k = 0; k < j; ++k) d -= R[j * b + k] * R[j * b + k];
        if (!(d > 0.0)) return -1;             /* also catches NaN */
        double rjj = sqrt(d);
        R[j * b + j] = rjj;
        for (int i = j + 1; i < b; ++i) {
            double s = S[i * b + j];
            for (int k = 0; k < j; ++k) s -= R[i * b + k] * R[j * b + k];
            R[i * b + j] = s / rjj;
        }
    }
    return 0;
}

/* Rinv := R^-1 for lower-triangular R (column-by-column forward substitution). */
static void lower_inverse(int b, const double *R, double *Rinv)
{
    for (int i = 0; i < b * b; ++i) Rinv[i] = 0.0;
    for (int j = 0; j < b; ++j) {
        Rinv[j * b + j] = 1.0 / R[j * b + j];
        for (int i = j + 1; i < b; ++i) {
            double s = 0.0;
            for (int k = j; k < i; ++k) s += R[i * b + k] * Rinv[k * b + j];
            Rinv[i * b + j] = -s / R[i * b + i];
        }
    }
}

/* C := op(A) * op(B), op = identity or transpose; all b x b. */
static void matmul(int b, const double *A, int ta, const double *B, int tb, double *C)
{
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            double s = 0.0;
            for (int k = 0; k < b; ++k) {
                double a = ta ? A[k * b + i] : A[i * b + k];
                double c = tb ? B[j * b + k] : B[k * b + j];
                s += a * c;
            }
            C[i * b + j] = s;
        }
}

/* y := op(A) x for a b x b matrix and a length-b vector. */
static void matvec(int b, const double *A, int ta, const double *x, double *y)
{
    for (int i = 0; i < b; ++i) {
        double s = 0.0;
        for (int k = 0; k < b; ++k) s += (ta ? A[k * b + i] : A[i * b + k]) * x[k];
        y[i] = s;
    }
}

/* Full symmetric copy of a block from its lower triangle. */
static void sym_from_lower(int b, const double *D, double *S)
{
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j)
            S[i * b + j] = (j <= i) ? D[i * b + j] : D[j * b + i];
}

/* Factor S, form S^-1 = R^-T R^-1, return log det S (2 sum log R_kk).
 * Returns 0 or -1 (not positive definite).  work holds 2 b*b doubles. */
static int spd_inverse_logdet(int b, const double *S, double *Sinv, double *logdet, double *work)
{
    double *R = work, *Rinv = work + (size_t)b * b;
    if (cholesky_lower(b, S, R) != 0) return -1;
    double ld = 0.0;
    for (int k = 0; k < b; ++k) ld += 2.0 * log(R[k * b + k]);
    *logdet = ld;
    lower_inverse(b, R, Rinv);
    matmul(b, Rinv, 1, Rinv, 0, Sinv);         /* R^-T R^-1 */
    return 0;
}

/* G := (G + G^T)/2, returning the largest |G - G^T| seen before. */
static double symmetrise(int b, double *G)
{
    double worst = 0.0;
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < i; ++j) {
            double d = fabs(G[i * b + j] - G[j * b + i]);
            if (d > worst) worst = d;
            double m = 0.5 * (G[i * b + j] + G[j * b + i]);
            G[i * b + j] = m;
            G[j * b + i] = m;
        }
    return worst;
}

/* ------------------------------- chain ---------------------------------- */

/* One block-tridiagonal chain.  Returns info (-1 ok, else failing block). */
static int chain_one(int64_t L, int b, const double *diag, const double *lower,
                     double *G_diag, double *G_lower, double *logdet_out,
                     const double *rhs, double *x, double *asym_out)
{
    const size_t bb = (size_t)b * b;
    double *Sinv = malloc(sizeof(double) * bb * (size_t)L);  /* S_i^-1, all i */
    double *S = malloc(sizeof(double) * bb);
    double *T1 = malloc(sizeof(double) * bb);
    double *T2 = malloc(sizeof(double) * bb);
    double *work = malloc(sizeof(double) * 2 * bb);
    double *y = rhs ? malloc(sizeof(double) * (size_t)b * (size_t)L) : NULL;
    double *v1 = malloc(sizeof(double) * (size_t)b);
    double *v2 = malloc(sizeof(double) * (size_t)b);
    int info = -1;
    double logdet = 0.0, asym = 0.0;

    /* collect: S_0 = D_0; S_{i+1} = D_{i+1} - B_i S_i^-1 B_i^T */
    sym_from_lower(b, diag, S);
    for (int64_t i = 0; i < L; ++i) {
        double ld;
        if (spd_inverse_logdet(b, S, Sinv + bb * i, &ld, work) != 0) { info = (int)i; goto done; }
        logdet += ld;
        if (i + 1 < L) {
            const double *Bi = lower + bb * i;
            matmul(b, Bi, 0, Sinv + bb * i, 0, T1);          /* B_i S_i^-1 */
            matmul(b, T1, 0, Bi, 1, T2);                      /* B_i S_i^-1 B_i^T */
            sym_from_lower(b, diag + bb * (i + 1), S);
            for (size_t k = 0; k < bb; ++k) S[k] -= T2[k];
        }
    }
    if (logdet_out) *logdet_out = logdet;

    /* distribute: G_{L-1} = S_{L-1}^-1, then the Takahashi back-recursion */
    if (G_diag) {
        memcpy(G_diag + bb * (L - 1), Sinv + bb * (L - 1), sizeof(double) * bb);
        double a = symmetrise(b, G_diag + bb * (L - 1));
        if (a > asym) asym = a;
        for (int64_t i = L - 2; i >= 0; --i) {
            const double *Bi = lower + bb * i;
            double *Gl = G_lower + bb * i;
            double *Gii = G_diag + bb * i;
            const double *Gn = G_diag + bb * (i + 1);
            /* G_{i+1,i} = -G_{i+1,i+1} B_i S_i^-1 */
            matmul(b, Gn, 0, Bi, 0, T1);
            matmul(b, T1, 0, Sinv + bb * i, 0, T2);
            for (size_t k = 0; k < bb; ++k) Gl[k] = -T2[k];
            /* G_ii = S_i^-1 - S_i^-1 B_i^T G_{i+1,i} */
            matmul(b, Sinv + bb * i, 0, Bi, 1, T1);
            matmul(b, T1, 0, Gl, 0, T2);
            for (size_t k = 0; k < bb; ++k) Gii[k] = Sinv[bb * i + k] - T2[k];
            a = symmetrise(b, Gii);
            if (a > asym) asym = a;
        }
    }

    /* solve with the same factor */
    if (rhs && x) {
        memcpy(y, rhs, sizeof(double) * (size_t)b);
        for (int64_t i = 0; i + 1 < L; ++i) {
            /* y_{i+1} = r_{i+1} - B_i S_i^-1 y_i */
            matvec(b, Sinv + bb * i, 0, y + b * i, v1);
            matvec(b, lower + bb * i, 0, v1, v2);
            for (int k = 0; k < b; ++k) y[b * (i + 1) + k] = rhs[b * (i + 1) + k] - v2[k];
        }
        matvec(b, Sinv + bb * (L - 1), 0, y + b * (L - 1), x + b * (L - 1));
        for (int64_t i = L - 2; i >= 0; --i) {
            /* x_i = S_i^-1 (y_i - B_i^T x_{i+1}) */
            matvec(b, lower + bb * i, 1, x + b * (i + 1), v1);
            for (int k = 0; k < b; ++k) v2[k] = y[b * i + k] - v1[k];
            matvec(b, Sinv + bb * i, 0, v2, x + b * i);
        }
    }
done:
    if (asym_out) *asym_out = asym;
    free(Sinv); free(S); free(T1); free(T2); free(work); free(y); free(v1); free(v2);
    return info;
}

/*
 * Batched chain.  diag [batch,L,b,b], lower [batch,L-1,b,b] (row-major,
 * contiguous).  Any of G_diag/G_lower (given together), logdet, rhs/x
 * (given together), asym may be NULL.  info [batch] is required.
 * Batch elements are independent; they are spread over OpenMP threads.
 */
int oracle_chain(const double *diag, const double *lower, int64_t batch, int64_t L, int b,
                 double *G_diag, double *G_lower, double *logdet,
                 const double *rhs, double *x, int32_t *info, double *asym)
{
    if (batch < 0 || L < 1 || b < 1 || !diag || !info || (L > 1 && !lower)) return 1;
    const size_t bb = (size_t)b * b;
    int64_t e;
#pragma omp parallel for schedule(dynamic, 1)
    for (e = 0; e < batch; ++e) {
        info[e] = chain_one(L, b, diag + bb * L * e, lower ? lower + bb * (L - 1) * e : NULL,
                            G_diag ? G_diag + bb * L * e : NULL,
                            G_lower ? G_lower + bb * (L - 1) * e : NULL,
                            logdet ? logdet + e : NULL,
                            rhs ? rhs + (size_t)b * L * e : NULL,
                            x ? x + (size_t)b * L * e : NULL,
                            asym ? asym + e : NULL);
    }
    return 0;
}

/* ------------------------------ sampling --------------------------------- */

/*
 * Gaussian draw with the same factor (sparsax, PyPI page, "Factor once, do
 * everything": sample_gaussian returns eta = A^-1 b + P^T L^-T z for the
 * Cholesky factor A = P^T L L^T P; gabp-sparse-inv, "Gaussian sampling":
 * x ~ N(0, A^-1) reusing the factorisation).  A chain is factorised in its
 * own block order, so P = I and L is the block lower-bidiagonal Cholesky
 * factor of A:
 *   L_ii = R_i  (S_i = R_i R_i^T, R_i lower),   L_{i+1,i} = B_i R_i^-T.
 * The draw w = L^-T z solves L^T w = z by block back substitution:
 *   w_{L-1} = R_{L-1}^-T z_{L-1},
 *   w_i     = R_i^-T (z_i - R_i^-1 B_i^T w_{i+1}).
 * eta = x + w with x = A^-1 r (the solve above), or eta = w without r.
 */
static int chain_sample_one(int64_t L, int b, const double *diag, const double *lower,
                            const double *rhs, const double *z, double *eta, double *logdet_out)
{
    const size_t bb = (size_t)b * b;
    double *Rinv = malloc(sizeof(double) * bb * (size_t)L);   /* R_i^-1, all i */
    double *S = malloc(sizeof(double) * bb);
    double *R = malloc(sizeof(double) * bb);
    double *Sinv = malloc(sizeof(double) * bb);
    double *BS = malloc(sizeof(double) * bb);
    double *BSB = malloc(sizeof(double) * bb);
    double *v1 = malloc(sizeof(double) * (size_t)b);
    double *v2 = malloc(sizeof(double) * (size_t)b);
    int info = -1;
    double logdet = 0.0;

    /* the Cholesky factors R_i of the Schur complements, in block order */
    sym_from_lower(b, diag, S);
    for (int64_t i = 0; i < L; ++i) {
        if (cholesky_lower(b, S, R) != 0) { info = (int)i; goto done; }
        for (int k = 0; k < b; ++k) logdet += 2.0 * log(R[k * (b + 1)]);
        lower_inverse(b, R, Rinv + bb * i);
        if (i + 1 < L) {
            const double *Bi = lower + bb * i;
            matmul(b, Rinv + bb * i, 1, Rinv + bb * i, 0, Sinv);    /* S_i^-1 = R^-T R^-1 */
            matmul(b, Bi, 0, Sinv, 0, BS);                           /* B_i S_i^-1 */
            matmul(b, BS, 0, Bi, 1, BSB);                            /* B_i S_i^-1 B_i^T */
            sym_from_lower(b, diag + bb * (i + 1), S);
            for (size_t k = 0; k < bb; ++k) S[k] = S[k] - BSB[k];
        }
    }
    if (logdet_out) *logdet_out = logdet;

    /* w = L^-T z, back substitution; R_i^-T v = (R_i^-1)^T v */
    matvec(b, Rinv + bb * (L - 1), 1, z + (size_t)b * (L - 1), eta + (size_t)b * (L - 1));
    for (int64_t i = L - 2; i >= 0; --i) {
        matvec(b, lower + bb * i, 1, eta + (size_t)b * (i + 1), v1);        /* B_i^T w_{i+1} */
        matvec(b, Rinv + bb * i, 0, v1, v2);                                /* R_i^-1 B_i^T w_{i+1} */
        for (int k = 0; k < b; ++k) v1[k] = z[(size_t)b * i + k] - v2[k];
        matvec(b, Rinv + bb * i, 1, v1, eta + (size_t)b * i);              /* R_i^-T (...) */
    }
done:
    free(Rinv); free(S); free(R); free(Sinv); free(BS); free(BSB); free(v1); free(v2);
    if (info == -1 && rhs) {                                               /* + A^-1 r */
        double *x = malloc(sizeof(double) * (size_t)b * (size_t)L);
        info = chain_one(L, b, diag, lower, NULL, NULL, NULL, rhs, x, NULL);
        for (size_t k = 0; k < (size_t)b * (size_t)L; ++k) eta[k] += x[k];
        free(x);
    }
    return info;
}

/* Batched draws: z [batch,L,b] (standard normals, supplied by the caller),
 * rhs [batch,L,b] or NULL, eta [batch,L,b] out, logdet [batch] or NULL. */
int oracle_chain_sample(const double *diag, const double *lower, int64_t batch, int64_t L, int b,
                        const double *rhs, const double *z, double *eta, double *logdet, int32_t *info)
{
    if (batch < 0 || L < 1 || b < 1 || !diag || !z || !eta || !info || (L > 1 && !lower)) return 1;
    const size_t bb = (size_t)b * b;
    int64_t e;
#pragma omp parallel for schedule(dynamic, 1)
    for (e = 0; e < batch; ++e) {
        info[e] = chain_sample_one(L, b, diag + bb * L * e, lower ? lower + bb * (L - 1) * e : NULL,
                                   rhs ? rhs + (size_t)b * L * e : NULL, z + (size_t)b * L * e,
                                   eta + (size_t)b * L * e, logdet ? logdet + e : NULL);
    }
    return 0;
}

/* ------------------------------- backward -------------------------------- */

/*
 * Cotangents of the chain's selected inverse (gabp-sparse-inv, "Differentiable
 * selected inverse": gradients of a loss over the selected blocks flow back to
 * the input blocks as on-pattern cotangents).  Written from the definition:
 * G = A^-1 gives dG = -G dA G, so for a loss with cotangents Gb_ii on G_ii and
 * Gb_{i+1,i} on G_{i+1,i} (and nothing on the blocks above the diagonal, which
 * are not outputs),
 *     Ab = -G^T Gbar G^T = -G Gbar G         (dense, N = L b),
 * and the inputs receive what the forward map reads:
 *     D_i: only its lower triangle, the upper one being its mirror, so
 *          Db_i[r][c] = Ab_ii[r][c] + Ab_ii[c][r] (r > c), Ab_ii[r][r] (r = c),
 *          0 (r < c);
 *     B_i: at block (i+1, i) and, transposed, at (i, i+1), so
 *          Bb_i = Ab_{i+1,i} + (Ab_{i,i+1})^T.
 * The dense inverse comes from the textbook Cholesky factor of A.  Returns
 * info (-1 ok, else the block holding the first failing pivot).
 */
/* Ab := -A^-1 Gbar A^-1 for a dense SPD A (N x N, lower triangle read) from
 * its textbook Cholesky factor.  Returns -1, or the row of the first pivot
 * that is not > 0 (A is then not positive definite). */
static int dense_cotangent(int N, const double *A, const double *Gbar, double *Ab)
{
    const size_t NN = (size_t)N * N;
    double *R = malloc(NN * sizeof(double)), *Ri = malloc(NN * sizeof(double));
    double *G = malloc(NN * sizeof(double)), *T = malloc(NN * sizeof(double));
    int fail = -1;
    if (cholesky_lower(N, A, R) != 0) {
        for (int j = 0; j < N && fail < 0; ++j) {    /* the failing pivot's row */
            double d = A[(size_t)j * N + j];
            for (int k = 0; k < j; ++k) d -= R[(size_t)j * N + k] * R[(size_t)j * N + k];
            if (!(d > 0.0)) fail = j;
        }
        if (fail < 0) fail = 0;
        goto done;
    }
    lower_inverse(N, R, Ri);
    matmul(N, Ri, 1, Ri, 0, G);                      /* A^-1 = R^-T R^-1 */
    matmul(N, G, 0, Gbar, 0, T);                     /* G Gbar */
    matmul(N, T, 0, G, 0, Ab);                       /* G Gbar G */
    for (size_t k = 0; k < NN; ++k) Ab[k] = -Ab[k];
done:
    free(R); free(Ri); free(G); free(T);
    return fail;
}

static int chain_backward_one(int64_t L, int b, const double *diag, const double *lower,
                              const double *Gb_diag, const double *Gb_lower, double *Db, double *Bb)
{
    const size_t bb = (size_t)b * b;
    const int N = (int)(L * b);
    const size_t NN = (size_t)N * N;
    double *A = calloc(NN, sizeof(double)), *Gbar = calloc(NN, sizeof(double));
    double *Ab = malloc(NN * sizeof(double));
    int info = -1;
    for (int64_t i = 0; i < L; ++i)
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t row = (size_t)(i * b + r), col = (size_t)(i * b + c);
                A[row * N + col] = (c <= r) ? diag[bb * i + r * b + c] : diag[bb * i + c * b + r];
                Gbar[row * N + col] = Gb_diag[bb * i + r * b + c];
                if (i + 1 < L) {
                    const size_t lrow = (size_t)((i + 1) * b + r);
                    A[lrow * N + col] = lower[bb * i + r * b + c];              /* A_{i+1,i} = B_i */
                    A[col * N + lrow] = lower[bb * i + r * b + c];              /* A_{i,i+1} = B_i^T */
                    Gbar[lrow * N + col] = Gb_lower[bb * i + r * b + c];
                }
            }
    const int fail = dense_cotangent(N, A, Gbar, Ab);
    if (fail >= 0) { info = fail / b; goto done; }
    for (int64_t i = 0; i < L; ++i)
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t row = (size_t)(i * b + r), col = (size_t)(i * b + c);
                double v = 0.0;
                if (c < r) v = Ab[row * N + col] + Ab[col * N + row];
                else if (c == r) v = Ab[row * N + col];
                Db[bb * i + r * b + c] = v;
                if (i + 1 < L) {
                    const size_t lrow = (size_t)((i + 1) * b + r);
                    Bb[bb * i + r * b + c] = Ab[lrow * N + col] + Ab[col * N + lrow];
                }
            }
done:
    free(A); free(Gbar); free(Ab);
    return info;
}

/* Batched backward: Gb_diag [batch,L,b,b], Gb_lower [batch,L-1,b,b] (NULL when
 * L = 1) -> Db [batch,L,b,b], Bb [batch,L-1,b,b]; info [batch]. */
int oracle_chain_backward(const double *diag, const double *lower, int64_t batch, int64_t L, int b,
                          const double *Gb_diag, const double *Gb_lower, double *Db, double *Bb,
                          int32_t *info)
{
    if (batch < 0 || L < 1 || b < 1 || !diag || !Gb_diag || !Db || !info) return 1;
    if (L > 1 && (!lower || !Gb_lower || !Bb)) return 1;
    const size_t bb = (size_t)b * b;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < batch; ++e)
        info[e] = chain_backward_one(L, b, diag + bb * L * e, L > 1 ? lower + bb * (L - 1) * e : NULL,
                                     Gb_diag + bb * L * e, L > 1 ? Gb_lower + bb * (L - 1) * e : NULL,
                                     Db + bb * L * e, L > 1 ? Bb + bb * (L - 1) * e : NULL);
    return 0;
}

/* ------------------------------ dense SPD -------------------------------- */

/* A^-1 and log det A of a dense SPD matrix (lower triangle read) from its
 * textbook Cholesky factor: the definition the general sparse case is read
 * against.  Returns 0, or 1 + the row of the first pivot that is not > 0. */
int oracle_spd_inverse(const double *A, int N, double *Ainv, double *logdet)
{
    const size_t NN = (size_t)N * N;
    double *R = malloc(NN * sizeof(double)), *Ri = malloc(NN * sizeof(double));
    int rc = 0;
    if (cholesky_lower(N, A, R) != 0) {
        for (int j = 0; j < N && rc == 0; ++j) {
            double d = A[(size_t)j * N + j];
            for (int k = 0; k < j; ++k) d -= R[(size_t)j * N + k] * R[(size_t)j * N + k];
            if (!(d > 0.0)) rc = 1 + j;
        }
        if (rc == 0) rc = 1;
    } else {
        double ld = 0.0;
        for (int k = 0; k < N; ++k) ld += 2.0 * log(R[(size_t)k * N + k]);
        *logdet = ld;
        lower_inverse(N, R, Ri);
        matmul(N, Ri, 1, Ri, 0, Ainv);
    }
    free(R); free(Ri);
    return rc;
}

/* ---------------------------- non-symmetric ------------------------------ */

/* Ainv := A^-1 for a general N x N matrix by Gauss-Jordan elimination with
 * partial pivoting (row exchanges on the augmented [A | I]).  Returns -1, or
 * the first column whose pivot is zero or not finite (A singular). */
static int general_inverse(int N, const double *A, double *Ainv)
{
    const size_t W = 2 * (size_t)N;
    double *aug = malloc(sizeof(double) * (size_t)N * W);
    int fail = -1;
    for (int r = 0; r < N; ++r)
        for (int c = 0; c < N; ++c) {
            aug[r * W + c] = A[(size_t)r * N + c];
            aug[r * W + N + c] = (r == c) ? 1.0 : 0.0;
        }
    for (int k = 0; k < N; ++k) {
        int piv = k;
        for (int r = k + 1; r < N; ++r)
            if (fabs(aug[r * W + k]) > fabs(aug[piv * W + k])) piv = r;
        const double d = aug[piv * W + k];
        if (!(fabs(d) > 0.0) || !isfinite(d)) { fail = k; break; }
        if (piv != k)
            for (size_t c = 0; c < W; ++c) {
                const double tmp = aug[k * W + c];
                aug[k * W + c] = aug[piv * W + c];
                aug[piv * W + c] = tmp;
            }
        for (size_t c = 0; c < W; ++c) aug[k * W + c] /= d;
        for (int r = 0; r < N; ++r) {
            if (r == k) continue;
            const double f = aug[r * W + k];
            if (f != 0.0)
                for (size_t c = 0; c < W; ++c) aug[r * W + c] -= f * aug[k * W + c];
        }
    }
    if (fail < 0)
        for (int r = 0; r < N; ++r)
            for (int c = 0; c < N; ++c) Ainv[(size_t)r * N + c] = aug[r * W + N + c];
    free(aug);
    return fail;
}

/*
 * Selected inverse of a block lower-bidiagonal matrix M (general blocks, no
 * symmetry): gabp-sparse-inv 0.3.2, "Implemented and tested kernels" ->
 * Non-symmetric chain and "Non-symmetric selected inverse": G_ii and G_{i+1,i}
 * on M's pattern.  Written from the definition: the dense M^-1 (Gauss-Jordan
 * with partial pivoting) and its blocks (i, i) and (i+1, i).  M is block
 * lower triangular, so det M = prod det M_ii: info = -1, or the first block
 * i whose M_ii meets a zero pivot in its own pivoted elimination (M is then
 * singular and nothing is written).
 */
static int bidiag_one(int64_t L, int b, const double *diag, const double *lower, double *G_diag,
                      double *G_lower)
{
    const size_t bb = (size_t)b * b;
    const int N = (int)(L * b);
    const size_t NN = (size_t)N * N;
    double *M = calloc(NN, sizeof(double)), *Mi = malloc(NN * sizeof(double));
    int info = -1;
    for (int64_t i = 0; i < L; ++i)
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t row = (size_t)(i * b + r), col = (size_t)(i * b + c);
                M[row * N + col] = diag[bb * i + r * b + c];
                if (i + 1 < L) M[(row + b) * N + col] = lower[bb * i + r * b + c];   /* M_{i+1,i} */
            }
    for (int64_t i = 0; i < L; ++i)
        if (general_inverse(b, diag + bb * i, Mi) >= 0) { info = (int)i; goto done; }
    if (general_inverse(N, M, Mi) >= 0) { info = 0; goto done; }   /* not reached: det M != 0 */
    for (int64_t i = 0; i < L; ++i)
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t row = (size_t)(i * b + r), col = (size_t)(i * b + c);
                G_diag[bb * i + r * b + c] = Mi[row * N + col];
                if (i + 1 < L) G_lower[bb * i + r * b + c] = Mi[(row + b) * N + col];
            }
done:
    free(M); free(Mi);
    return info;
}

/* Batched: diag [batch,L,b,b], lower [batch,L-1,b,b] -> G_diag, G_lower; info [batch]. */
int oracle_bidiag(const double *diag, const double *lower, int64_t batch, int64_t L, int b, double *G_diag,
                  double *G_lower, int32_t *info)
{
    if (batch < 0 || L < 1 || b < 1 || !diag || !G_diag || !info) return 1;
    if (L > 1 && (!lower || !G_lower)) return 1;
    const size_t bb = (size_t)b * b;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < batch; ++e)
        info[e] = bidiag_one(L, b, diag + bb * L * e, L > 1 ? lower + bb * (L - 1) * e : NULL,
                             G_diag + bb * L * e, L > 1 ? G_lower + bb * (L - 1) * e : NULL);
    return 0;
}

/*
 * Cotangents of the non-symmetric chain (gabp-sparse-inv: selinv_bidiag's
 * hand-written analytic backward).  From the definition: G = M^-1 gives
 * dG = -G dM G, so Mb = -G^T Gbar G^T (dense), with Gbar holding Gb_ii at
 * (i, i) and Gb_{i+1,i} at (i+1, i); every entry of M_ii and M_{i+1,i} is
 * an independent input, so Mb_ii and Mb_{i+1,i} are just those blocks of Mb.
 * Returns info like bidiag_one.
 */
static int bidiag_backward_one(int64_t L, int b, const double *diag, const double *lower,
                               const double *Gb_diag, const double *Gb_lower, double *Mb_diag,
                               double *Mb_lower)
{
    const size_t bb = (size_t)b * b;
    const int N = (int)(L * b);
    const size_t NN = (size_t)N * N;
    double *M = calloc(NN, sizeof(double)), *Mi = malloc(NN * sizeof(double));
    double *Gbar = calloc(NN, sizeof(double)), *T = malloc(NN * sizeof(double));
    double *Mb = malloc(NN * sizeof(double));
    int info = -1;
    for (int64_t i = 0; i < L; ++i)
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t row = (size_t)(i * b + r), col = (size_t)(i * b + c);
                const size_t k = bb * i + (size_t)r * b + c;       /* entry (r, c) of block i */
                M[row * N + col] = diag[k];
                Gbar[row * N + col] = Gb_diag[k];
                if (i + 1 < L) {
                    M[(row + b) * N + col] = lower[k];
                    Gbar[(row + b) * N + col] = Gb_lower[k];
                }
            }
    for (int64_t i = 0; i < L; ++i)
        if (general_inverse(b, diag + bb * i, Mi) >= 0) { info = (int)i; goto done; }
    if (general_inverse(N, M, Mi) >= 0) { info = 0; goto done; }
    matmul(N, Mi, 1, Gbar, 0, T);                    /* G^T Gbar */
    matmul(N, T, 0, Mi, 1, Mb);                      /* G^T Gbar G^T */
    for (int64_t i = 0; i < L; ++i)
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t row = (size_t)(i * b + r), col = (size_t)(i * b + c);
                Mb_diag[bb * i + r * b + c] = -Mb[row * N + col];
                if (i + 1 < L) Mb_lower[bb * i + r * b + c] = -Mb[(row + b) * N + col];
            }
done:
    free(M); free(Mi); free(Gbar); free(T); free(Mb);
    return info;
}

int oracle_bidiag_backward(const double *diag, const double *lower, int64_t batch, int64_t L, int b,
                           const double *Gb_diag, const double *Gb_lower, double *Mb_diag, double *Mb_lower,
                           int32_t *info)
{
    if (batch < 0 || L < 1 || b < 1 || !diag || !Gb_diag || !Mb_diag || !info) return 1;
    if (L > 1 && (!lower || !Gb_lower || !Mb_lower)) return 1;
    const size_t bb = (size_t)b * b;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < batch; ++e)
        info[e] = bidiag_backward_one(L, b, diag + bb * L * e, L > 1 ? lower + bb * (L - 1) * e : NULL,
                                      Gb_diag + bb * L * e, L > 1 ? Gb_lower + bb * (L - 1) * e : NULL,
                                      Mb_diag + bb * L * e, L > 1 ? Mb_lower + bb * (L - 1) * e : NULL);
    return 0;
}

/* -------------------------------- tree ---------------------------------- */

/* One rooted tree (parent[root] = -1).  Collect in reverse breadth-first
 * order (every child before its parent; children summed in ascending
 * index), distribute in breadth-first order.  Returns info, or -2 if the
 * parent array is not a single rooted tree. */
static int tree_one(int64_t n, int b, const int32_t *parent, const double *diag,
                    const double *edge, double *G_diag, double *G_edge, double *logdet_out)
{
    const size_t bb = (size_t)b * b;
    int info = -1;
    int64_t root = -1;
    for (int64_t v = 0; v < n; ++v) {
        if (parent[v] == -1) { if (root >= 0) return -2; root = v; }
        else if (parent[v] < 0 || parent[v] >= n || parent[v] == v) return -2;
    }
    if (root < 0) return -2;

    /* children lists (ascending, since v is visited in increasing order) */
    int64_t *count = calloc((size_t)n + 1, sizeof(int64_t));
    int64_t *child = malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    int64_t *order = malloc(sizeof(int64_t) * (size_t)n);
    for (int64_t v = 0; v < n; ++v) if (parent[v] >= 0) count[parent[v] + 1]++;
    for (int64_t v = 0; v < n; ++v) count[v + 1] += count[v];
    int64_t *fill = malloc(sizeof(int64_t) * (size_t)n);
    for (int64_t v = 0; v < n; ++v) fill[v] = count[v];
    for (int64_t v = 0; v < n; ++v) if (parent[v] >= 0) child[fill[parent[v]]++] = v;

    /* breadth-first order from the root; a cycle leaves nodes unreached */
    int64_t head = 0, tail = 0;
    order[tail++] = root;
    while (head < tail) {
        int64_t v = order[head++];
        for (int64_t k = count[v]; k < count[v + 1]; ++k) order[tail++] = child[k];
    }
    double *Sinv = NULL, *S = NULL, *T1 = NULL, *T2 = NULL, *work = NULL;
    if (tail != n) { info = -2; goto done; }

    Sinv = malloc(sizeof(double) * bb * (size_t)n);
    S = malloc(sizeof(double) * bb);
    T1 = malloc(sizeof(double) * bb);
    T2 = malloc(sizeof(double) * bb);
    work = malloc(sizeof(double) * 2 * bb);
    double logdet = 0.0;

    /* collect: S_v = D_v - sum_{c in ch(v)} E_c S_c^-1 E_c^T, E_c = edge[c] */
    for (int64_t t = n - 1; t >= 0; --t) {
        int64_t v = order[t];
        sym_from_lower(b, diag + bb * v, S);
        for (int64_t k = count[v]; k < count[v + 1]; ++k) {
            int64_t c = child[k];
            matmul(b, edge + bb * c, 0, Sinv + bb * c, 0, T1);
            matmul(b, T1, 0, edge + bb * c, 1, T2);
            for (size_t q = 0; q < bb; ++q) S[q] -= T2[q];
        }
        double ld;
        if (spd_inverse_logdet(b, S, Sinv + bb * v, &ld, work) != 0) { info = (int)v; goto done; }
        logdet += ld;
    }
    if (logdet_out) *logdet_out = logdet;

    /* distribute: G_root = S_root^-1; G_edge[v] = -G_p E_v S_v^-1;
     * G_vv = S_v^-1 - S_v^-1 E_v^T G_edge[v] */
    if (G_diag) {
        memcpy(G_diag + bb * root, Sinv + bb * root, sizeof(double) * bb);
        symmetrise(b, G_diag + bb * root);
        memset(G_edge + bb * root, 0, sizeof(double) * bb);
        for (int64_t t = 1; t < n; ++t) {
            int64_t v = order[t], p = parent[v];
            matmul(b, G_diag + bb * p, 0, edge + bb * v, 0, T1);
            matmul(b, T1, 0, Sinv + bb * v, 0, T2);
            for (size_t q = 0; q < bb; ++q) G_edge[bb * v + q] = -T2[q];
            matmul(b, Sinv + bb * v, 0, edge + bb * v, 1, T1);
            matmul(b, T1, 0, G_edge + bb * v, 0, T2);
            for (size_t q = 0; q < bb; ++q) G_diag[bb * v + q] = Sinv[bb * v + q] - T2[q];
            symmetrise(b, G_diag + bb * v);
        }
    }
done:
    free(count); free(child); free(order); free(fill);
    free(Sinv); free(S); free(T1); free(T2); free(work);
    return info;
}

/*
 * Gaussian draw on a tree (gabp-sparse-inv, "Gaussian sampling":
 * sample_gaussian_tree draws x ~ N(0, A^-1) reusing the factorisation; the
 * factor is the one sparsax's sample_gaussian names, A = P^T L L^T P, here
 * with the tree's own elimination order, children before parents).  The
 * Cholesky factor's blocks are L_vv = R_v (S_v = R_v R_v^T) and
 * L_{p(v),v} = E_v R_v^-T (E_v = edge[v] = A_{p(v),v}); w = L^-T z by back
 * substitution from the root:
 *   w_root = R_root^-T z_root,   w_v = R_v^-T (z_v - R_v^-1 E_v^T w_{p(v)}).
 * The sibling order does not change L (each S_v depends on v's subtree only).
 */
static int tree_sample_one(int64_t n, int b, const int32_t *parent, const double *diag,
                           const double *edge, const double *z, double *w, double *logdet_out)
{
    const size_t bb = (size_t)b * b;
    int64_t root = -1;
    for (int64_t u = 0; u < n; ++u) {
        if (parent[u] == -1) { if (root >= 0) return -2; root = u; }
        else if (parent[u] < 0 || parent[u] >= n || parent[u] == u) return -2;
    }
    if (root < 0) return -2;
    int64_t *first = calloc((size_t)n + 1, sizeof(int64_t));    /* children CSR */
    int64_t *kids = malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    int64_t *next = malloc(sizeof(int64_t) * (size_t)n);
    int64_t *bfs = malloc(sizeof(int64_t) * (size_t)n);
    for (int64_t u = 0; u < n; ++u) if (parent[u] >= 0) first[parent[u] + 1]++;
    for (int64_t u = 0; u < n; ++u) first[u + 1] += first[u];
    for (int64_t u = 0; u < n; ++u) next[u] = first[u];
    for (int64_t u = 0; u < n; ++u) if (parent[u] >= 0) kids[next[parent[u]]++] = u;
    int64_t qh = 0, qt = 0;
    bfs[qt++] = root;
    while (qh < qt) {
        int64_t u = bfs[qh++];
        for (int64_t k = first[u]; k < first[u + 1]; ++k) bfs[qt++] = kids[k];
    }
    int info = -1;
    double *Rinv = NULL, *Sc = NULL, *Rf = NULL, *Si = NULL, *ES = NULL, *ESE = NULL, *t1 = NULL, *t2 = NULL;
    if (qt != n) { info = -2; goto out; }
    Rinv = malloc(sizeof(double) * bb * (size_t)n);              /* R_v^-1, all v */
    Sc = malloc(sizeof(double) * bb);
    Rf = malloc(sizeof(double) * bb);
    Si = malloc(sizeof(double) * bb);
    ES = malloc(sizeof(double) * bb);
    ESE = malloc(sizeof(double) * bb);
    t1 = malloc(sizeof(double) * (size_t)b);
    t2 = malloc(sizeof(double) * (size_t)b);
    double logdet = 0.0;
    /* the factors R_v, leaves first: S_v = D_v - sum_c E_c S_c^-1 E_c^T */
    for (int64_t q = n - 1; q >= 0; --q) {
        int64_t u = bfs[q];
        sym_from_lower(b, diag + bb * u, Sc);
        for (int64_t k = first[u]; k < first[u + 1]; ++k) {
            const double *Ec = edge + bb * kids[k];
            matmul(b, Rinv + bb * kids[k], 1, Rinv + bb * kids[k], 0, Si);   /* S_c^-1 */
            matmul(b, Ec, 0, Si, 0, ES);
            matmul(b, ES, 0, Ec, 1, ESE);
            for (size_t e2 = 0; e2 < bb; ++e2) Sc[e2] = Sc[e2] - ESE[e2];
        }
        if (cholesky_lower(b, Sc, Rf) != 0) { info = (int)u; goto out; }
        for (int k = 0; k < b; ++k) logdet += 2.0 * log(Rf[k * (b + 1)]);
        lower_inverse(b, Rf, Rinv + bb * u);
    }
    if (logdet_out) *logdet_out = logdet;
    /* w = L^-T z, root first */
    matvec(b, Rinv + bb * root, 1, z + (size_t)b * root, w + (size_t)b * root);
    for (int64_t q = 1; q < n; ++q) {
        int64_t u = bfs[q], pu = parent[u];
        matvec(b, edge + bb * u, 1, w + (size_t)b * pu, t1);                 /* E_v^T w_p */
        matvec(b, Rinv + bb * u, 0, t1, t2);                                 /* R_v^-1 E_v^T w_p */
        for (int k = 0; k < b; ++k) t1[k] = z[(size_t)b * u + k] - t2[k];
        matvec(b, Rinv + bb * u, 1, t1, w + (size_t)b * u);                  /* R_v^-T (...) */
    }
out:
    free(first); free(kids); free(next); free(bfs);
    free(Rinv); free(Sc); free(Rf); free(Si); free(ES); free(ESE); free(t1); free(t2);
    return info;
}

/*
 * Cotangents of the tree selected inverse (gabp-sparse-inv, "Differentiable
 * selected inverse": selinv_tree's gradients reach diag and edge).  The same
 * dense definition as the chain's, Ab = -A^-1 Gbar A^-1, with Gbar holding
 * Gb_diag[v] at (v, v) and Gb_edge[v] at (p(v), v) (the block G_edge[v]
 * holds); D_v receives the lower-triangle projection of Ab_vv and edge[v],
 * which sits at (p, v) and transposed at (v, p), receives
 * Ab_{p,v} + (Ab_{v,p})^T; the root's edge slot receives 0.  Returns info:
 * -1 ok, -2 malformed parent array, else the node of the first failing pivot
 * in natural order (A is then not positive definite).
 */
static int tree_backward_one(int64_t n, int b, const int32_t *parent, const double *diag, const double *edge,
                             const double *Gb_diag, const double *Gb_edge, double *Db, double *Eb)
{
    const size_t bb = (size_t)b * b;
    int64_t root = -1;
    for (int64_t v = 0; v < n; ++v) {
        if (parent[v] == -1) { if (root >= 0) return -2; root = v; }
        else if (parent[v] < 0 || parent[v] >= n || parent[v] == v) return -2;
    }
    if (root < 0) return -2;
    for (int64_t v = 0; v < n; ++v) {                /* every node reaches the root */
        int64_t u = v, steps = 0;
        while (parent[u] >= 0 && steps <= n) { u = parent[u]; ++steps; }
        if (u != root) return -2;
    }
    const int N = (int)(n * b);
    const size_t NN = (size_t)N * N;
    double *A = calloc(NN, sizeof(double)), *Gbar = calloc(NN, sizeof(double));
    double *Ab = malloc(NN * sizeof(double));
    int info = -1;
    for (int64_t v = 0; v < n; ++v) {
        const int64_t p = parent[v];
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t vr = (size_t)(v * b + r), vc = (size_t)(v * b + c);
                A[vr * N + vc] = (c <= r) ? diag[bb * v + r * b + c] : diag[bb * v + c * b + r];
                Gbar[vr * N + vc] = Gb_diag[bb * v + r * b + c];
                if (p >= 0) {
                    const size_t pr = (size_t)(p * b + r);
                    A[pr * N + vc] = edge[bb * v + r * b + c];                  /* A_{p,v} = E_v */
                    A[vc * N + pr] = edge[bb * v + r * b + c];                  /* A_{v,p} = E_v^T */
                    Gbar[pr * N + vc] = Gb_edge[bb * v + r * b + c];
                }
            }
    }
    const int fail = dense_cotangent(N, A, Gbar, Ab);
    if (fail >= 0) { info = fail / b; goto done; }
    for (int64_t v = 0; v < n; ++v) {
        const int64_t p = parent[v];
        for (int r = 0; r < b; ++r)
            for (int c = 0; c < b; ++c) {
                const size_t vr = (size_t)(v * b + r), vc = (size_t)(v * b + c);
                const double lo = Ab[vr * N + vc], up = Ab[vc * N + vr];
                Db[bb * v + r * b + c] = c < r ? lo + up : (c == r ? lo : 0.0);
                if (p >= 0) {
                    const size_t pr = (size_t)(p * b + r);
                    Eb[bb * v + r * b + c] = Ab[pr * N + vc] + Ab[vc * N + pr];
                } else {
                    Eb[bb * v + r * b + c] = 0.0;
                }
            }
    }
done:
    free(A); free(Gbar); free(Ab);
    return info;
}

/* Batched tree backward: parent [trees,n]; diag, edge, Gb_diag, Gb_edge, Db,
 * Eb [trees,n,b,b]; info [trees]. */
int oracle_tree_backward(const int32_t *parent, int64_t trees, int64_t n, int b, const double *diag,
                         const double *edge, const double *Gb_diag, const double *Gb_edge, double *Db,
                         double *Eb, int32_t *info)
{
    if (trees < 0 || n < 1 || b < 1 || !parent || !diag || !edge || !Gb_diag || !Gb_edge || !Db || !Eb ||
        !info)
        return 1;
    const size_t bb = (size_t)b * b;
    int64_t t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < trees; ++t)
        info[t] = tree_backward_one(n, b, parent + n * t, diag + bb * n * t, edge + bb * n * t,
                                    Gb_diag + bb * n * t, Gb_edge + bb * n * t, Db + bb * n * t,
                                    Eb + bb * n * t);
    return 0;
}

/* Batched tree draws: z, w [trees,n,b]; logdet [trees] or NULL; info [trees]. */
int oracle_tree_sample(const int32_t *parent, int64_t trees, int64_t n, int b, const double *diag,
                       const double *edge, const double *z, double *w, double *logdet, int32_t *info)
{
    if (trees < 0 || n < 1 || b < 1 || !parent || !diag || !edge || !z || !w || !info) return 1;
    const size_t bb = (size_t)b * b;
    int64_t e;
#pragma omp parallel for schedule(dynamic, 1)
    for (e = 0; e < trees; ++e) {
        info[e] = tree_sample_one(n, b, parent + n * e, diag + bb * n * e, edge + bb * n * e,
                                  z + (size_t)b * n * e, w + (size_t)b * n * e, logdet ? logdet + e : NULL);
    }
    return 0;
}

/*
 * Batched trees: parent [trees,n] (int32, root = -1), diag/edge
 * [trees,n,b,b] (edge root slot ignored), outputs G_diag/G_edge
 * [trees,n,b,b] (G_edge root slot set to 0), logdet [trees], info [trees]
 * (-1 ok, node index of a failing pivot, or -2 for a malformed tree).
 */
int oracle_tree(const int32_t *parent, int64_t trees, int64_t n, int b,
                const double *diag, const double *edge,
                double *G_diag, double *G_edge, double *logdet, int32_t *info)
{
    if (trees < 0 || n < 1 || b < 1 || !parent || !diag || !edge || !info) return 1;
    const size_t bb = (size_t)b * b;
    int64_t t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < trees; ++t) {
        info[t] = tree_one(n, b, parent + n * t, diag + bb * n * t, edge + bb * n * t,
                           G_diag ? G_diag + bb * n * t : NULL,
                           G_edge ? G_edge + bb * n * t : NULL,
                           logdet ? logdet + t : NULL);
    }
    return 0;
}

/* Threads an OpenMP parallel region will use (for reporting core counts). */
int oracle_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
