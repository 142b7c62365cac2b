/*
 * ict_oracle.c -- plain CPU oracle for the integer-only (C,e) training hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the slow, obviously-correct reference that the
 * CUDA library is checked against, element by element.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark load it.  It shares no code,
 * header, table or helper with the CUDA library, and the library never calls it.
 *
 * Source: "Memory-Efficient Integer-Only Training of Deep Neural Networks"
 * (Shalby, Pittorino, Roveri).  The page prints the abstract, the Figure 1 caption and
 * Tables 1-11 but not the equations those cite (Eq. 1, 3, 5, 6, 19), so each routine
 * below states the passage it follows and the reading it takes where the page is silent.
 *
 * Arithmetic is integer only: int64 everywhere, __int128 where a two-term sum needs the
 * range.  No floating point is used anywhere in this file.
 *
 * Representation (Abstract: "signed integer mantissas paired with explicit power-of-two
 * exponents"; Figure 1 caption: every tensor is a (C,e) pair; Table 7: symmetric clip
 * bound q_max; Table 5: one exponent byte per group):
 *   value = C * 2^e,  C in [-127, 127],  e an int8 in [-127, 127],
 *   e = E_ZERO = -128 marks a group whose mantissas are all zero.
 *
 * Parity pins: every public routine is checked in tests/ against closed forms,
 * hand-derived examples, brute force on tiny inputs and library primitives (numpy
 * matmul / convolution on the aligned mantissas); see tests/test_oracle_*.py.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define E_ZERO (-128)
#define QMAX 127
/* Two-term sums whose exponents are further apart than this are reduced to a sticky
 * unit (see two_term below); below it they are exact in __int128. */
#define EXACT_SPAN 100

enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_LAYOUT = 2, ORC_ERR_EXP_RANGE = 8 };

typedef __int128 i128;
typedef unsigned __int128 u128;

/* A (C,e) matrix view: mantissas row-major with leading dimension ld; exponents on a
 * grid of groups of g_rows x g_cols elements, row-major, ceil(rows/g_rows) x
 * ceil(cols/g_cols) bytes.  Groups at the bottom/right edge may be short. */
typedef struct {
    int8_t *mant;
    int8_t *exp;
    int64_t rows, cols, ld;
    int32_t g_rows, g_cols;
} o_tensor;

typedef struct { int32_t n, h, w, c, k, r, s, stride, pad; } o_conv;
typedef struct { int32_t mom_mul, mom_shift, lr_mul, lr_shift; } o_sgd;

/* ------------------------------------------------------------------------------------ */
/* Group geometry                                                                        */
/* ------------------------------------------------------------------------------------ */

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
static int64_t n_grp_rows(const o_tensor *t) { return cdiv(t->rows, t->g_rows); }
static int64_t n_grp_cols(const o_tensor *t) { return cdiv(t->cols, t->g_cols); }

/* exponent of the group holding element (i, j) */
static int exp_at(const o_tensor *t, int64_t i, int64_t j) {
    return t->exp[(i / t->g_rows) * n_grp_cols(t) + (j / t->g_cols)];
}
static int mant_at(const o_tensor *t, int64_t i, int64_t j) { return t->mant[i * t->ld + j]; }

/* Checks the input invariants: |C| <= 127 and E_ZERO groups hold only zeros. */
static int check_input(const o_tensor *t) {
    if (!t || !t->mant || !t->exp || t->rows < 0 || t->cols < 0 || t->g_rows < 1 ||
        t->g_cols < 1 || t->ld < t->cols)
        return ORC_ERR_ARG;
    for (int64_t i = 0; i < t->rows; i++)
        for (int64_t j = 0; j < t->cols; j++) {
            int c = mant_at(t, i, j);
            if (c < -QMAX || c > QMAX) return ORC_ERR_ARG;
            if (exp_at(t, i, j) == E_ZERO && c != 0) return ORC_ERR_ARG;
        }
    return ORC_OK;
}
static int check_output(const o_tensor *t, int64_t rows, int64_t cols) {
    if (!t || !t->mant || !t->exp || t->g_rows < 1 || t->g_cols < 1) return ORC_ERR_ARG;
    if (t->rows != rows || t->cols != cols || t->ld < cols) return ORC_ERR_ARG;
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Rounding and exponent selection (the requantisation step that follows every Product)  */
/* ------------------------------------------------------------------------------------ */

/* RNE(x * 2^k): exact for k >= 0; for k < 0 a right shift by s = -k that rounds to the
 * nearest integer, ties to even.  Reading: the page prints no rounding rule, so
 * round-half-to-even is taken. */
static i128 rne_scale(i128 x, int k) {
    if (k >= 0) return x * ((i128)1 << k); /* callers keep |x| * 2^k far below 2^126 */
    int s = -k;
    if (s >= 126) return 0; /* |x| < 2^120 here, so |x| / 2^s < 1/2 */
    i128 p = (i128)1 << s;
    /* floor division by 2^s */
    i128 q = x / p;
    if (x % p != 0 && x < 0) q -= 1;
    i128 rem = x - q * p; /* 0 <= rem < 2^s */
    i128 twice = 2 * rem;
    if (twice > p || (twice == p && (q & 1))) q += 1;
    return q;
}

static int fits_at_q(i128 x, int r, int e, int qmax) {
    i128 q = rne_scale(x, r - e);
    return q >= -qmax && q <= qmax;
}

static int bitlen(i128 x) {
    u128 a = x < 0 ? (u128)(-x) : (u128)x;
    int b = 0;
    while (a) { a >>= 1; b++; }
    return b;
}

/* need(x, r): the smallest exponent e at which RNE(x * 2^(r-e)) fits in [-127, 127], for
 * x != 0.  Written as the definition: start where it surely does not fit (|x| scaled to
 * at least 128) and step up until it does.  Reading of the spec requant rule
 * "smallest exponent that fits the group maximum". */
static int need_q(i128 x, int r, int qmax) {
    int e = r + bitlen(x) - 8; /* here |x| * 2^(r-e) >= 2^7 > qmax: does not fit */
    while (!fits_at_q(x, r, e, qmax)) e++;
    return e;
}
static int need(i128 x, int r) { return need_q(x, r, QMAX); }

/* FIT of one group of n values x[i] at exponents r[i]: the group exponent is the max of
 * need over the nonzero members (E_ZERO when all are zero), clamped below at -127; each
 * mantissa is RNE(x[i] * 2^(r[i] - e)).  Returns the exponent, or a value > 127 when the
 * group cannot be represented (ORC_ERR_EXP_RANGE). */
/* (the same with a clip bound qmax below 127: the B-bit variants of Table 4) */
static int fit_group_q(int64_t n, const i128 *x, const int *r, int8_t *c_out, int qmax) {
    int have = 0, e = 0;
    for (int64_t i = 0; i < n; i++) {
        if (x[i] == 0) continue;
        int ni = need_q(x[i], r[i], qmax);
        if (!have || ni > e) e = ni;
        have = 1;
    }
    if (!have) {
        for (int64_t i = 0; i < n; i++) c_out[i] = 0;
        return E_ZERO;
    }
    if (e < -127) e = -127;
    if (e > 127) {
        for (int64_t i = 0; i < n; i++) c_out[i] = 0;
        return 1000;
    }
    for (int64_t i = 0; i < n; i++) {
        i128 q = x[i] == 0 ? 0 : rne_scale(x[i], r[i] - e);
        if (q < -qmax) q = -qmax; /* never taken: e fits every member */
        if (q > qmax) q = qmax;
        c_out[i] = (int8_t)q;
    }
    return e;
}
static int fit_group(int64_t n, const i128 *x, const int *r, int8_t *c_out) {
    return fit_group_q(n, x, r, c_out, QMAX);
}

/* FIT of a whole matrix of values (x at exponent r, element (i,j) at i*cols+j) into the
 * groups of `out`. */
static int fit_matrix_q(const i128 *x, const int *r, o_tensor *out, int qmax) {
    int64_t ngr = n_grp_rows(out), ngc = n_grp_cols(out);
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t gi = 0; gi < ngr; gi++) {
        int64_t i0 = gi * out->g_rows, i1 = i0 + out->g_rows;
        if (i1 > out->rows) i1 = out->rows;
        int64_t maxn = (int64_t)out->g_rows * out->g_cols;
        i128 *gx = malloc(sizeof(i128) * maxn);
        int *gr = malloc(sizeof(int) * maxn);
        int8_t *gc = malloc(maxn);
        for (int64_t gj = 0; gj < ngc; gj++) {
            int64_t j0 = gj * out->g_cols, j1 = j0 + out->g_cols;
            if (j1 > out->cols) j1 = out->cols;
            int64_t n = 0;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++) {
                    gx[n] = x[i * out->cols + j];
                    gr[n] = r[i * out->cols + j];
                    n++;
                }
            int e = fit_group_q(n, gx, gr, gc, qmax);
            if (e > 127) {
#pragma omp atomic write
                status = ORC_ERR_EXP_RANGE;
                e = 127;
            }
            out->exp[gi * ngc + gj] = (int8_t)e;
            n = 0;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++) out->mant[i * out->ld + j] = gc[n++];
        }
        free(gx);
        free(gr);
        free(gc);
    }
    return status;
}
static int fit_matrix(const i128 *x, const int *r, o_tensor *out) { return fit_matrix_q(x, r, out, QMAX); }

/* ------------------------------------------------------------------------------------ */
/* Sum primitive: exact sum of two (C,e) terms                                          */
/* ------------------------------------------------------------------------------------ */

/* a*2^pa + b*2^pb as one integer x at exponent r.  Exact (Table 6: "Sum", Eq. 6, read as
 * an exact integer sum at the smaller exponent) while the exponents are at most
 * EXACT_SPAN apart.  Beyond that the smaller term is replaced by a one-unit sticky,
 * sign(b) * 2^(e_hi - EXACT_SPAN): the requantisation of the sum is unchanged, because
 * its exponent is at least e_hi - 7, every rounding and fitting threshold it compares
 * against is a multiple of 2^(e_hi - 8), and both the true small term (|b| < 2^16,
 * so below 2^(e_hi - 84)) and the sticky lie strictly inside the same gap between two
 * such thresholds next to a * 2^e_hi.  tests/test_oracle_pins.py checks this against
 * unbounded Python integers. */
static void two_term(int64_t a, int pa, int64_t b, int pb, i128 *x, int *r) {
    if (a == 0 && b == 0) { *x = 0; *r = 0; return; }
    if (a == 0) { *x = b; *r = pb; return; }
    if (b == 0) { *x = a; *r = pa; return; }
    if (pa < pb) { int64_t t = a; a = b; b = t; int tp = pa; pa = pb; pb = tp; }
    /* now pa >= pb: a is the term with the larger exponent */
    int d = pa - pb;
    if (d <= EXACT_SPAN) {
        *x = (i128)a * ((i128)1 << d) + b;
        *r = pb;
    } else {
        *x = (i128)a * ((i128)1 << EXACT_SPAN) + (b > 0 ? 1 : -1);
        *r = pa - EXACT_SPAN;
    }
}

/* ------------------------------------------------------------------------------------ */
/* Public: requantisation                                                                */
/* ------------------------------------------------------------------------------------ */

/* FIT of int64 values x[i][j] whose exponent is base + row_exp[i] + col_exp[j]
 * (either vector may be NULL) into the caller-chosen groups of `out`.  This is the
 * requantisation that closes every Product (Table 6, Eqs. 5 and 3, read as: exact
 * integer product, exponent addition, then requant to INT8 per group). */
int oracle_requant(int64_t rows, int64_t cols, const int64_t *x, int64_t ldx, int32_t base_exp,
                   const int8_t *row_exp, const int8_t *col_exp, o_tensor *out) {
    if (!x || ldx < cols || check_output(out, rows, cols)) return ORC_ERR_ARG;
    i128 *v = malloc(sizeof(i128) * (rows * cols + 1));
    int *r = malloc(sizeof(int) * (rows * cols + 1));
    int status = ORC_OK;
    for (int64_t i = 0; i < rows; i++)
        for (int64_t j = 0; j < cols; j++) {
            int64_t val = x[i * ldx + j];
            int re = row_exp ? row_exp[i] : 0, ce = col_exp ? col_exp[j] : 0;
            if ((re == E_ZERO || ce == E_ZERO) && val != 0) status = ORC_ERR_ARG;
            v[i * cols + j] = val;
            r[i * cols + j] = base_exp + re + ce;
        }
    if (status == ORC_OK) status = fit_matrix(v, r, out);
    free(v);
    free(r);
    return status;
}

/* FIT with B-bit mantissas (Table 4 sweeps B = 4..8): the clip bound is
 * q_max = 2^(B-1) - 1 instead of 127 (Table 7's q_max); everything else as in
 * oracle_requant.  Mantissas are stored one per byte. */
int oracle_requant_bits(int64_t rows, int64_t cols, const int64_t *x, int64_t ldx, int32_t base_exp,
                        const int8_t *row_exp, const int8_t *col_exp, int32_t bits, o_tensor *out) {
    if (!x || ldx < cols || bits < 2 || bits > 8 || check_output(out, rows, cols)) return ORC_ERR_ARG;
    i128 *v = malloc(sizeof(i128) * (rows * cols + 1));
    int *r = malloc(sizeof(int) * (rows * cols + 1));
    int status = ORC_OK;
    for (int64_t i = 0; i < rows; i++)
        for (int64_t j = 0; j < cols; j++) {
            int64_t val = x[i * ldx + j];
            int re = row_exp ? row_exp[i] : 0, ce = col_exp ? col_exp[j] : 0;
            if ((re == E_ZERO || ce == E_ZERO) && val != 0) status = ORC_ERR_ARG;
            v[i * cols + j] = val;
            r[i * cols + j] = base_exp + re + ce;
        }
    if (status == ORC_OK) status = fit_matrix_q(v, r, out, (1 << (bits - 1)) - 1);
    free(v);
    free(r);
    return status;
}

/* ------------------------------------------------------------------------------------ */
/* Public: exponent alignment along the contracted index                                 */
/* ------------------------------------------------------------------------------------ */

/* ALIGN_MAX.  Before an integer contraction every operand whose exponent varies along
 * the contracted index is brought to one exponent per non-contracted index: the largest
 * of the group exponents it meets (E_ZERO groups ignored), each mantissa shifted right
 * to it with RNE.  Reading of the Sum primitive (Table 6, Eq. 6): integer terms are
 * added at a common exponent, the larger one, so the aligned mantissas stay INT8.
 *   axis = 1: contracted index runs along columns -> one exponent per row (rows entries)
 *   axis = 0: contracted index runs along rows    -> one exponent per column
 * out (ld_out) receives the aligned mantissas, transposed when `transpose` is set. */
int oracle_align(const o_tensor *in, int axis, int8_t *out, int64_t ld_out, int transpose,
                 int8_t *e_star) {
    int st = check_input(in);
    if (st) return st;
    if (!out || !e_star || (axis != 0 && axis != 1)) return ORC_ERR_ARG;
    int64_t n_keep = axis == 1 ? in->rows : in->cols;
    int64_t n_red = axis == 1 ? in->cols : in->rows;
    for (int64_t a = 0; a < n_keep; a++) {
        int have = 0, m = E_ZERO;
        for (int64_t b = 0; b < n_red; b++) {
            int64_t i = axis == 1 ? a : b, j = axis == 1 ? b : a;
            int e = exp_at(in, i, j);
            if (e == E_ZERO) continue;
            if (!have || e > m) m = e;
            have = 1;
        }
        e_star[a] = (int8_t)m;
        for (int64_t b = 0; b < n_red; b++) {
            int64_t i = axis == 1 ? a : b, j = axis == 1 ? b : a;
            int c = mant_at(in, i, j);
            int q = 0;
            if (c != 0) q = (int)rne_scale(c, exp_at(in, i, j) - m);
            if (transpose) out[j * ld_out + i] = (int8_t)q;
            else out[i * ld_out + j] = (int8_t)q;
        }
    }
    return ORC_OK;
}

/* ALIGN_MAX to targets fixed elsewhere.  When a batch is split across devices, the
 * exponent an operand is aligned to along the contracted (batch) index is the largest
 * group exponent over ALL the shards, not only the local one (reading of the Sum
 * primitive, Table 6 Eq. 6, applied to the whole batch: training on a split batch must
 * compute what one device computes on all of it).  e_target has one entry per
 * non-contracted index (rows for axis 1, cols for axis 0); every entry must be at least
 * every non-E_ZERO group exponent it covers.  Each mantissa becomes
 * RNE(C * 2^(e - target)); E_ZERO groups and zero mantissas give 0. */
int oracle_align_to(const o_tensor *in, int axis, const int8_t *e_target, int8_t *out,
                    int64_t ld_out, int transpose) {
    int st = check_input(in);
    if (st) return st;
    if (!out || !e_target || (axis != 0 && axis != 1)) return ORC_ERR_ARG;
    for (int64_t i = 0; i < in->rows; i++)
        for (int64_t j = 0; j < in->cols; j++) {
            int t = e_target[axis == 1 ? i : j];
            int e = exp_at(in, i, j), c = mant_at(in, i, j);
            if (e != E_ZERO && (t == E_ZERO || t < e)) return ORC_ERR_ARG;
            int q = (c == 0 || e == E_ZERO) ? 0 : (int)rne_scale(c, e - t);
            if (transpose) out[j * ld_out + i] = (int8_t)q;
            else out[i * ld_out + j] = (int8_t)q;
        }
    return ORC_OK;
}

/* dense aligned copy (rows x cols, ld = cols) + exponent vector */
static int align_dense(const o_tensor *t, int axis, int8_t **m, int8_t **e) {
    *m = malloc(t->rows * t->cols + 1);
    *e = malloc((axis == 1 ? t->rows : t->cols) + 1);
    return oracle_align(t, axis, *m, t->cols, 0, *e);
}

static int sum_exp(int a, int b) { return (a == E_ZERO || b == E_ZERO) ? 0 : a + b; }

/* ------------------------------------------------------------------------------------ */
/* Public: linear layer, three training directions                                      */
/* ------------------------------------------------------------------------------------ */

/* Pre-requant accumulators of the forward product Y = X * W^T (Figure 1a; Table 6:
 * "Linear / fully-connected: Product"): align X per row and W per row (both contract
 * along their columns), exact int64 dot products, exponents added. */
int oracle_linear_fwd_acc(const o_tensor *X, const o_tensor *W, int64_t *acc, int32_t *r) {
    int st;
    if ((st = check_input(X)) || (st = check_input(W))) return st;
    if (X->cols != W->cols) return ORC_ERR_ARG;
    int8_t *xa, *xe, *wa, *we;
    align_dense(X, 1, &xa, &xe);
    align_dense(W, 1, &wa, &we);
    int64_t M = X->rows, N = W->rows, K = X->cols;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; k++) s += (int64_t)xa[m * K + k] * wa[n * K + k];
            acc[m * N + n] = s;
            r[m * N + n] = sum_exp(xe[m], we[n]);
        }
    free(xa); free(xe); free(wa); free(we);
    return ORC_OK;
}

/* Pre-requant accumulators of dX = dY * W: dY aligned per row, W per column (its
 * contracted index, the output feature, runs along W's rows). */
int oracle_linear_bwd_data_acc(const o_tensor *dY, const o_tensor *W, int64_t *acc, int32_t *r) {
    int st;
    if ((st = check_input(dY)) || (st = check_input(W))) return st;
    if (dY->cols != W->rows) return ORC_ERR_ARG;
    int8_t *ya, *ye, *wa, *we;
    align_dense(dY, 1, &ya, &ye);
    align_dense(W, 0, &wa, &we);
    int64_t M = dY->rows, N = W->rows, K = W->cols;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t k = 0; k < K; k++) {
            int64_t s = 0;
            for (int64_t n = 0; n < N; n++) s += (int64_t)ya[m * N + n] * wa[n * K + k];
            acc[m * K + k] = s;
            r[m * K + k] = sum_exp(ye[m], we[k]);
        }
    free(ya); free(ye); free(wa); free(we);
    return ORC_OK;
}

/* Pre-requant accumulators of dW = dY^T * X: both aligned per column (the contracted
 * index, the token, runs along their rows). */
int oracle_linear_bwd_weight_acc(const o_tensor *dY, const o_tensor *X, int64_t *acc, int32_t *r) {
    int st;
    if ((st = check_input(dY)) || (st = check_input(X))) return st;
    if (dY->rows != X->rows) return ORC_ERR_ARG;
    int8_t *ya, *ye, *xa, *xe;
    align_dense(dY, 0, &ya, &ye);
    align_dense(X, 0, &xa, &xe);
    int64_t M = dY->rows, N = dY->cols, K = X->cols;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++)
        for (int64_t k = 0; k < K; k++) {
            int64_t s = 0;
            for (int64_t m = 0; m < M; m++) s += (int64_t)ya[m * N + n] * xa[m * K + k];
            acc[n * K + k] = s;
            r[n * K + k] = sum_exp(ye[n], xe[k]);
        }
    free(ya); free(ye); free(xa); free(xe);
    return ORC_OK;
}

static int fit_acc_q(const int64_t *acc, const int32_t *r, o_tensor *out, int qmax) {
    int64_t n = out->rows * out->cols;
    i128 *v = malloc(sizeof(i128) * (n + 1));
    int *rr = malloc(sizeof(int) * (n + 1));
    for (int64_t i = 0; i < n; i++) { v[i] = acc[i]; rr[i] = r[i]; }
    int st = fit_matrix_q(v, rr, out, qmax);
    free(v);
    free(rr);
    return st;
}

static int fit_acc(const int64_t *acc, const int32_t *r, o_tensor *out) { return fit_acc_q(acc, r, out, QMAX); }

typedef int (*acc_fn)(const o_tensor *, const o_tensor *, int64_t *, int32_t *);
static int product_q(acc_fn f, const o_tensor *a, const o_tensor *b, o_tensor *out,
                     int64_t rows, int64_t cols, int qmax) {
    if (check_output(out, rows, cols)) return ORC_ERR_ARG;
    int64_t *acc = malloc(sizeof(int64_t) * (rows * cols + 1));
    int32_t *r = malloc(sizeof(int32_t) * (rows * cols + 1));
    int st = f(a, b, acc, r);
    if (!st) st = fit_acc_q(acc, r, out, qmax);
    free(acc);
    free(r);
    return st;
}
static int product(acc_fn f, const o_tensor *a, const o_tensor *b, o_tensor *out, int64_t rows, int64_t cols) {
    return product_q(f, a, b, out, rows, cols, QMAX);
}

/* The three linear directions with B-bit outputs (Table 4: INT8 down to INT4): the same
 * alignment and exact contraction, the FIT clipping at q_max = 2^(B-1) - 1.
 * op 0: Y = X W^T (a = X, b = W); 1: dX = dY W (a = dY, b = W); 2: dW = dY^T X. */
int oracle_linear_bits(int op, const o_tensor *a, const o_tensor *b, o_tensor *out, int32_t bits) {
    if (bits < 2 || bits > 8 || !a || !b) return ORC_ERR_ARG;
    const int q = (1 << (bits - 1)) - 1;
    if (op == 0) return product_q(oracle_linear_fwd_acc, a, b, out, a->rows, b->rows, q);
    if (op == 1) return product_q(oracle_linear_bwd_data_acc, a, b, out, a->rows, b->cols, q);
    if (op == 2) return product_q(oracle_linear_bwd_weight_acc, a, b, out, a->cols, b->cols, q);
    return ORC_ERR_ARG;
}

int oracle_linear_fwd(const o_tensor *X, const o_tensor *W, o_tensor *Y) {
    return product(oracle_linear_fwd_acc, X, W, Y, X->rows, W->rows);
}
int oracle_linear_bwd_data(const o_tensor *dY, const o_tensor *W, o_tensor *dX) {
    return product(oracle_linear_bwd_data_acc, dY, W, dX, dY->rows, W->cols);
}
int oracle_linear_bwd_weight(const o_tensor *dY, const o_tensor *X, o_tensor *dW) {
    return product(oracle_linear_bwd_weight_acc, dY, X, dW, dY->cols, X->cols);
}

/* ------------------------------------------------------------------------------------ */
/* Public: convolution (Table 6: "Convolution (incl. 1x1, depthwise): Product")          */
/* ------------------------------------------------------------------------------------ */

/* NHWC activations viewed as [n*h*w][c] (C,e) matrices whose exponent groups span all
 * pixels (g_rows >= rows: one exponent per channel group, uniform over pixels);
 * KRSC weights viewed as [k][r*s*c].  Directions:
 *   dir 0 forward      a = X  [N*H*W][C], b = W [K][R*S*C], out = Y  [N*P*Q][K]
 *   dir 1 bwd-data     a = dY [N*P*Q][K], b = W [K][R*S*C], out = dX [N*H*W][C]
 *   dir 2 bwd-weight   a = dY [N*P*Q][K], b = X [N*H*W][C], out = dW [K][R*S*C]
 * with P = (H + 2 pad - R) / stride + 1, zero padding.  Alignment: fwd aligns the
 * activation to the largest channel-group exponent and W per output channel; bwd-data
 * aligns dY the same way and W per input channel c (max over k, r, s); bwd-weight
 * aligns dY and X per channel over all pixels. */
static int64_t out_dim(int64_t in, int pad, int ker, int stride) {
    return (in + 2 * pad - ker) / stride + 1;
}

int oracle_conv_acc(int dir, const o_conv *d, const o_tensor *a, const o_tensor *b, int64_t *acc,
                    int32_t *rexp) {
    int st;
    if (!d || d->stride < 1 || d->pad < 0 || d->r < 1 || d->s < 1) return ORC_ERR_ARG;
    if ((st = check_input(a)) || (st = check_input(b))) return st;
    int64_t N = d->n, H = d->h, Wd = d->w, C = d->c, K = d->k, R = d->r, S = d->s;
    int64_t P = out_dim(H, d->pad, R, d->stride), Q = out_dim(Wd, d->pad, S, d->stride);
    if (P < 1 || Q < 1) return ORC_ERR_ARG;
    int64_t npix_in = N * H * Wd, npix_out = N * P * Q, RSC = R * S * C;

    if (dir == 0 || dir == 1) {
        /* activation operand: X (fwd) or dY (bwd-data); exponent uniform over pixels */
        const o_tensor *act = a;
        int64_t act_rows = dir == 0 ? npix_in : npix_out, act_cols = dir == 0 ? C : K;
        if (act->rows != act_rows || act->cols != act_cols) return ORC_ERR_ARG;
        if (act->g_rows < act->rows) return ORC_ERR_LAYOUT;
        if (b->rows != K || b->cols != RSC) return ORC_ERR_ARG;
        int8_t *aa = malloc(act_rows * act_cols + 1), *ae = malloc(act_rows + 1);
        oracle_align(act, 1, aa, act_cols, 0, ae); /* every row gets the same e* */
        int ea = act_rows ? ae[0] : E_ZERO;
        int8_t *wa = malloc(K * RSC + 1);
        int8_t *we;
        if (dir == 0) {
            we = malloc(K + 1);
            oracle_align(b, 1, wa, RSC, 0, we); /* per output channel k */
        } else {
            /* per input channel c: max over k, r, s of the group exponent */
            we = malloc(C + 1);
            for (int64_t c = 0; c < C; c++) {
                int have = 0, m = E_ZERO;
                for (int64_t k = 0; k < K; k++)
                    for (int64_t rs = 0; rs < R * S; rs++) {
                        int e = exp_at(b, k, rs * C + c);
                        if (e == E_ZERO) continue;
                        if (!have || e > m) m = e;
                        have = 1;
                    }
                we[c] = (int8_t)m;
                for (int64_t k = 0; k < K; k++)
                    for (int64_t rs = 0; rs < R * S; rs++) {
                        int v = mant_at(b, k, rs * C + c);
                        wa[k * RSC + rs * C + c] =
                            v ? (int8_t)rne_scale(v, exp_at(b, k, rs * C + c) - m) : 0;
                    }
            }
        }
        if (dir == 0) {
#pragma omp parallel for schedule(static)
            for (int64_t op = 0; op < npix_out; op++) {
                int64_t n = op / (P * Q), p = (op / Q) % P, q = op % Q;
                for (int64_t k = 0; k < K; k++) {
                    int64_t s = 0;
                    for (int64_t r = 0; r < R; r++)
                        for (int64_t ss = 0; ss < S; ss++) {
                            int64_t h = p * d->stride + r - d->pad, w = q * d->stride + ss - d->pad;
                            if (h < 0 || h >= H || w < 0 || w >= Wd) continue;
                            const int8_t *xr = aa + ((n * H + h) * Wd + w) * C;
                            const int8_t *wr = wa + k * RSC + (r * S + ss) * C;
                            for (int64_t c = 0; c < C; c++) s += (int64_t)xr[c] * wr[c];
                        }
                    acc[op * K + k] = s;
                    rexp[op * K + k] = sum_exp(ea, we[k]);
                }
            }
        } else {
#pragma omp parallel for schedule(static)
            for (int64_t ip = 0; ip < npix_in; ip++) {
                int64_t n = ip / (H * Wd), h = (ip / Wd) % H, w = ip % Wd;
                for (int64_t c = 0; c < C; c++) {
                    int64_t s = 0;
                    for (int64_t r = 0; r < R; r++)
                        for (int64_t ss = 0; ss < S; ss++) {
                            int64_t ph = h + d->pad - r, qw = w + d->pad - ss;
                            if (ph < 0 || qw < 0 || ph % d->stride || qw % d->stride) continue;
                            int64_t p = ph / d->stride, q = qw / d->stride;
                            if (p >= P || q >= Q) continue;
                            const int8_t *yr = aa + ((n * P + p) * Q + q) * K;
                            for (int64_t k = 0; k < K; k++)
                                s += (int64_t)yr[k] * wa[k * RSC + (r * S + ss) * C + c];
                        }
                    acc[ip * C + c] = s;
                    rexp[ip * C + c] = sum_exp(ea, we[c]);
                }
            }
        }
        free(aa); free(ae); free(wa); free(we);
        return ORC_OK;
    }
    if (dir == 2) {
        if (a->rows != npix_out || a->cols != K || b->rows != npix_in || b->cols != C)
            return ORC_ERR_ARG;
        int8_t *ya, *ye, *xa, *xe;
        align_dense(a, 0, &ya, &ye); /* per output channel k, over all pixels */
        align_dense(b, 0, &xa, &xe); /* per input channel c, over all pixels */
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < K; k++)
            for (int64_t rs = 0; rs < R * S; rs++) {
                int64_t r = rs / S, ss = rs % S;
                for (int64_t c = 0; c < C; c++) {
                    int64_t s = 0;
                    for (int64_t n = 0; n < N; n++)
                        for (int64_t p = 0; p < P; p++)
                            for (int64_t q = 0; q < Q; q++) {
                                int64_t h = p * d->stride + r - d->pad, w = q * d->stride + ss - d->pad;
                                if (h < 0 || h >= H || w < 0 || w >= Wd) continue;
                                s += (int64_t)ya[((n * P + p) * Q + q) * K + k] *
                                     xa[((n * H + h) * Wd + w) * C + c];
                            }
                    acc[k * RSC + rs * C + c] = s;
                    rexp[k * RSC + rs * C + c] = sum_exp(ye[k], xe[c]);
                }
            }
        free(ya); free(ye); free(xa); free(xe);
        return ORC_OK;
    }
    return ORC_ERR_ARG;
}

int oracle_conv(int dir, const o_conv *d, const o_tensor *a, const o_tensor *b, o_tensor *out) {
    if (!d || d->stride < 1) return ORC_ERR_ARG;
    int64_t P = out_dim(d->h, d->pad, d->r, d->stride), Q = out_dim(d->w, d->pad, d->s, d->stride);
    int64_t rows, cols;
    if (dir == 0) { rows = (int64_t)d->n * P * Q; cols = d->k; }
    else if (dir == 1) { rows = (int64_t)d->n * d->h * d->w; cols = d->c; }
    else if (dir == 2) { rows = d->k; cols = (int64_t)d->r * d->s * d->c; }
    else return ORC_ERR_ARG;
    if (check_output(out, rows, cols)) return ORC_ERR_ARG;
    int64_t *acc = malloc(sizeof(int64_t) * (rows * cols + 1));
    int32_t *r = malloc(sizeof(int32_t) * (rows * cols + 1));
    int st = oracle_conv_acc(dir, d, a, b, acc, r);
    if (!st) st = fit_acc(acc, r, out);
    free(acc);
    free(r);
    return st;
}

/* ------------------------------------------------------------------------------------ */
/* Public: depthwise convolution (Table 6: "Convolution (incl. 1 x 1, depthwise)" ->      */
/* Product)                                                                               */
/* ------------------------------------------------------------------------------------ */

/* Depthwise convolution, one R x S filter per channel (MobileNetV2's 3x3 depthwise
 * layers; Table 3 trains MobileNetV2).  NHWC activations with exponents uniform over
 * pixels; W [C][R*S].  The contraction of output channel ch runs over (r, s) of that one
 * channel, so the activation keeps its per-channel exponent (no alignment across
 * channels); W is aligned per row (ALIGN_MAX along (r, s)).  Exact int64 sums, exponents
 * added:
 *   dir 0  Y [n*P*Q][C]   = sum_(r,s) X[pixel(p,q,r,s)][ch] * W[ch][r,s]
 *   dir 1  dX [n*h*w][C]  = sum over (p,q,r,s) reaching the pixel of dY[(p,q)][ch] * W[ch][r,s]
 *   dir 2  dW [C][R*S]    = sum_(p,q) dY[(p,q)][ch] * X[pixel(p,q,r,s)][ch]
 * d->k must equal d->c. */
int oracle_depthwise_acc(int dir, const o_conv *d, const o_tensor *a, const o_tensor *b, int64_t *acc,
                         int32_t *rexp) {
    int st;
    if (!d || d->stride < 1 || d->pad < 0 || d->r < 1 || d->s < 1 || d->k != d->c) return ORC_ERR_ARG;
    if ((st = check_input(a)) || (st = check_input(b))) return st;
    int64_t N = d->n, H = d->h, Wd = d->w, C = d->c, R = d->r, S = d->s, RS = R * S;
    int64_t P = out_dim(H, d->pad, R, d->stride), Q = out_dim(Wd, d->pad, S, d->stride);
    if (P < 1 || Q < 1) return ORC_ERR_ARG;
    int64_t npix_in = N * H * Wd, npix_out = N * P * Q;
    if (dir == 0 || dir == 1) {
        if (a->rows != (dir == 0 ? npix_in : npix_out) || a->cols != C) return ORC_ERR_ARG;
        if (a->g_rows < a->rows) return ORC_ERR_LAYOUT;
        if (b->rows != C || b->cols != RS) return ORC_ERR_ARG;
        int8_t *wa = malloc(C * RS + 1), *we = malloc(C + 1);
        oracle_align(b, 1, wa, RS, 0, we);
        if (dir == 0) {
            for (int64_t op = 0; op < npix_out; op++) {
                int64_t n = op / (P * Q), p = (op / Q) % P, q = op % Q;
                for (int64_t ch = 0; ch < C; ch++) {
                    int64_t sum = 0;
                    for (int64_t r = 0; r < R; r++)
                        for (int64_t ss = 0; ss < S; ss++) {
                            int64_t h = p * d->stride + r - d->pad, w = q * d->stride + ss - d->pad;
                            if (h < 0 || h >= H || w < 0 || w >= Wd) continue;
                            sum += (int64_t)mant_at(a, (n * H + h) * Wd + w, ch) * wa[ch * RS + r * S + ss];
                        }
                    acc[op * C + ch] = sum;
                    rexp[op * C + ch] = sum_exp(exp_at(a, 0, ch), we[ch]);
                }
            }
        } else {
            for (int64_t ip = 0; ip < npix_in; ip++) {
                int64_t n = ip / (H * Wd), h = (ip / Wd) % H, w = ip % Wd;
                for (int64_t ch = 0; ch < C; ch++) {
                    int64_t sum = 0;
                    for (int64_t r = 0; r < R; r++)
                        for (int64_t ss = 0; ss < S; ss++) {
                            int64_t ph = h + d->pad - r, qw = w + d->pad - ss;
                            if (ph < 0 || qw < 0 || ph % d->stride || qw % d->stride) continue;
                            int64_t p = ph / d->stride, q = qw / d->stride;
                            if (p >= P || q >= Q) continue;
                            sum += (int64_t)mant_at(a, (n * P + p) * Q + q, ch) * wa[ch * RS + r * S + ss];
                        }
                    acc[ip * C + ch] = sum;
                    rexp[ip * C + ch] = sum_exp(exp_at(a, 0, ch), we[ch]);
                }
            }
        }
        free(wa);
        free(we);
        return ORC_OK;
    }
    if (dir == 2) {
        if (a->rows != npix_out || a->cols != C || b->rows != npix_in || b->cols != C) return ORC_ERR_ARG;
        if (a->g_rows < a->rows || b->g_rows < b->rows) return ORC_ERR_LAYOUT;
        for (int64_t ch = 0; ch < C; ch++)
            for (int64_t r = 0; r < R; r++)
                for (int64_t ss = 0; ss < S; ss++) {
                    int64_t sum = 0;
                    for (int64_t op = 0; op < npix_out; op++) {
                        int64_t n = op / (P * Q), p = (op / Q) % P, q = op % Q;
                        int64_t h = p * d->stride + r - d->pad, w = q * d->stride + ss - d->pad;
                        if (h < 0 || h >= H || w < 0 || w >= Wd) continue;
                        sum += (int64_t)mant_at(a, op, ch) * mant_at(b, (n * H + h) * Wd + w, ch);
                    }
                    acc[ch * RS + r * S + ss] = sum;
                    rexp[ch * RS + r * S + ss] = sum_exp(exp_at(a, 0, ch), exp_at(b, 0, ch));
                }
        return ORC_OK;
    }
    return ORC_ERR_ARG;
}

int oracle_depthwise(int dir, const o_conv *d, const o_tensor *a, const o_tensor *b, o_tensor *out) {
    if (!d || d->stride < 1) return ORC_ERR_ARG;
    int64_t P = out_dim(d->h, d->pad, d->r, d->stride), Q = out_dim(d->w, d->pad, d->s, d->stride);
    int64_t rows, cols = d->c;
    if (dir == 0) rows = (int64_t)d->n * P * Q;
    else if (dir == 1) rows = (int64_t)d->n * d->h * d->w;
    else if (dir == 2) { rows = d->c; cols = (int64_t)d->r * d->s; }
    else return ORC_ERR_ARG;
    if (check_output(out, rows, cols)) return ORC_ERR_ARG;
    int64_t *acc = malloc(sizeof(int64_t) * (rows * cols + 1));
    int32_t *r = malloc(sizeof(int32_t) * (rows * cols + 1));
    int st = oracle_depthwise_acc(dir, d, a, b, acc, r);
    if (!st) st = fit_acc(acc, r, out);
    free(acc);
    free(r);
    return st;
}

/* ------------------------------------------------------------------------------------ */
/* Public: integer SGD with momentum and per-group velocity (Figure 1b)                  */
/* ------------------------------------------------------------------------------------ */

/* One step of SGD with momentum, every tensor a (C,e) pair with its own exponent per
 * group (Abstract: "per-group velocity mechanism with independent exponent tracking";
 * Figure 1b; Table 10: SGD with momentum beta = 0.9).  Reading: the usual form
 *     v <- beta * v + g ;   w <- w - lr * v
 * with beta = mom_mul * 2^-mom_shift and lr = lr_mul * 2^-lr_shift as integer
 * multiply-shifts, each right-hand side an exact two-term Sum requantised once by FIT
 * into the group (so both exponents are chosen afresh every step).  W, V and G share
 * one group partition; W and V are updated in place. */
static int sgd_step_q(o_tensor *W, o_tensor *V, const o_tensor *G, const o_sgd *p, int qmax) {
    int st;
    if (!p) return ORC_ERR_ARG;
    if ((st = check_input(W)) || (st = check_input(V)) || (st = check_input(G))) return st;
    if (W->rows != V->rows || W->rows != G->rows || W->cols != V->cols || W->cols != G->cols ||
        W->g_rows != V->g_rows || W->g_rows != G->g_rows || W->g_cols != V->g_cols ||
        W->g_cols != G->g_cols)
        return ORC_ERR_ARG;
    if (p->mom_shift < 0 || p->lr_shift < 0) return ORC_ERR_ARG;
    int64_t ngr = n_grp_rows(W), ngc = n_grp_cols(W);
    int status = ORC_OK;
#pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < ngr; gi++) {
        int64_t maxn = (int64_t)W->g_rows * W->g_cols;
        i128 *x = malloc(sizeof(i128) * maxn);
        int *r = malloc(sizeof(int) * maxn);
        int8_t *cv = malloc(maxn), *cw = malloc(maxn);
        for (int64_t gj = 0; gj < ngc; gj++) {
            int64_t i0 = gi * W->g_rows, i1 = i0 + W->g_rows, j0 = gj * W->g_cols,
                    j1 = j0 + W->g_cols;
            if (i1 > W->rows) i1 = W->rows;
            if (j1 > W->cols) j1 = W->cols;
            int64_t ge = gi * ngc + gj;
            int ev = V->exp[ge], eg = G->exp[ge], ew = W->exp[ge];
            /* velocity: mom_mul * Cv * 2^(ev - mom_shift) + Cg * 2^eg */
            int64_t n = 0;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++, n++)
                    two_term((int64_t)p->mom_mul * mant_at(V, i, j), ev - p->mom_shift,
                             mant_at(G, i, j), eg, &x[n], &r[n]);
            int ev2 = fit_group_q(n, x, r, cv, qmax);
            /* weight: Cw * 2^ew - lr_mul * Cv' * 2^(ev' - lr_shift) */
            n = 0;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++, n++)
                    two_term(mant_at(W, i, j), ew, -(int64_t)p->lr_mul * cv[n],
                             ev2 - p->lr_shift, &x[n], &r[n]);
            int ew2 = fit_group_q(n, x, r, cw, qmax);
            if (ev2 > 127 || ew2 > 127) {
#pragma omp atomic write
                status = ORC_ERR_EXP_RANGE;
                if (ev2 > 127) ev2 = 127;
                if (ew2 > 127) ew2 = 127;
            }
            V->exp[ge] = (int8_t)ev2;
            W->exp[ge] = (int8_t)ew2;
            n = 0;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++, n++) {
                    V->mant[i * V->ld + j] = cv[n];
                    W->mant[i * W->ld + j] = cw[n];
                }
        }
        free(x); free(r); free(cv); free(cw);
    }
    return status;
}
int oracle_sgd_step(o_tensor *W, o_tensor *V, const o_tensor *G, const o_sgd *p) {
    return sgd_step_q(W, V, G, p, QMAX);
}

/* The same update with B-bit mantissas (Table 4 trains with INT8 down to INT4): both
 * FITs clip at q_max = 2^(B-1) - 1 (Table 7's symmetric bound), 2 <= B <= 8; every other
 * step is unchanged. */
int oracle_sgd_step_bits(o_tensor *W, o_tensor *V, const o_tensor *G, const o_sgd *p, int32_t bits) {
    if (bits < 2 || bits > 8) return ORC_ERR_ARG;
    return sgd_step_q(W, V, G, p, (1 << (bits - 1)) - 1);
}

/* ------------------------------------------------------------------------------------ */
/* Public: integer GELU                                                                  */
/* ------------------------------------------------------------------------------------ */

/* C * 2^e >= 2, decided exactly */
static int at_least_two(int64_t c, int e) {
    if (e >= 1) return c >= 1;
    if (1 - e > 100) return 0;
    return (i128)c >= ((i128)1 << (1 - e));
}

/* Forward of the piecewise GELU h(x) = x * clip((x + 2) / 4, 0, 1) on (C,e), the
 * exponent carried through unchanged (Table 7 caption: pointwise activations act on the
 * mantissa and keep e).  Reading: the page's own GELU is a lookup table (Table 7, Eq. 19)
 * whose contents are not printed; this shift-friendly curve stands in for it.
 *   x <= -2: 0;  x >= 2: x;  otherwise x (x + 2) / 4 = C^2 2^(2e-2) + C 2^(e-1),
 * rounded RNE to the input exponent.  E_ZERO groups stay zero. */
int oracle_gelu_fwd(const o_tensor *H, o_tensor *out) {
    int st;
    if ((st = check_input(H))) return st;
    if (check_output(out, H->rows, H->cols) || out->g_rows != H->g_rows ||
        out->g_cols != H->g_cols)
        return ORC_ERR_ARG;
    int64_t ne = n_grp_rows(H) * n_grp_cols(H);
    memcpy(out->exp, H->exp, ne);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < H->rows; i++)
        for (int64_t j = 0; j < H->cols; j++) {
            int c = mant_at(H, i, j), e = exp_at(H, i, j);
            int o;
            if (c == 0 || e == E_ZERO) o = 0;
            else if (at_least_two(-c, e)) o = 0;
            else if (at_least_two(c, e)) o = c;
            else {
                i128 x;
                int r;
                two_term((int64_t)c * c, 2 * e - 2, c, e - 1, &x, &r);
                o = (int)rne_scale(x, r - e);
            }
            out->mant[i * out->ld + j] = (int8_t)o;
        }
    return ORC_OK;
}

/* Backward of the same curve: dH = dG * h'(x) with h'(x) = 0 for x <= -2, 1 for x >= 2
 * and (x + 1) / 2 in between, i.e. dG * x / 2 + dG / 2 as an exact two-term Sum, then
 * FIT into the groups of dH.  H and dG share one shape. */
int oracle_gelu_bwd(const o_tensor *H, const o_tensor *dG, o_tensor *dH) {
    int st;
    if ((st = check_input(H)) || (st = check_input(dG))) return st;
    if (H->rows != dG->rows || H->cols != dG->cols) return ORC_ERR_ARG;
    int64_t rows = H->rows, cols = H->cols;
    if (check_output(dH, rows, cols)) return ORC_ERR_ARG;
    i128 *x = malloc(sizeof(i128) * (rows * cols + 1));
    int *r = malloc(sizeof(int) * (rows * cols + 1));
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; i++)
        for (int64_t j = 0; j < cols; j++) {
            int ch = mant_at(H, i, j), eh = exp_at(H, i, j);
            int cd = mant_at(dG, i, j), ed = exp_at(dG, i, j);
            i128 v = 0;
            int rr = 0;
            if (cd != 0) {
                if (eh == E_ZERO) ch = 0;
                if (ch != 0 && at_least_two(-ch, eh)) { v = 0; }
                else if (ch != 0 && at_least_two(ch, eh)) { v = cd; rr = ed; }
                else two_term((int64_t)cd * ch, ed + eh - 1, cd, ed - 1, &v, &rr);
            }
            x[i * cols + j] = v;
            r[i * cols + j] = rr;
        }
    st = fit_matrix(x, r, dH);
    free(x);
    free(r);
    return st;
}

/* ------------------------------------------------------------------------------------ */
/* Public: Sum (residual add, gradient merge)                                            */
/* ------------------------------------------------------------------------------------ */

/* Z = FIT(X + Y).  Table 6 lists "Residual add, gradient merge" under the Sum primitive
 * (Eq. 6, whose text the page does not print).  Reading, the same as for the two-term
 * sums of the SGD step: every element's two terms x * 2^ex + y * 2^ey are added exactly,
 * then the result is requantised into Z's groups.  X, Y and Z share one shape; each has
 * its own group geometry.
 * The scaled form weighs each term by an integer multiply-shift, m * 2^-s (the way the
 * SGD step applies momentum and learning rate): Z = FIT(xm 2^-xs X + ym 2^-ys Y).  With
 * weights (1, 0) it is the plain Sum; the weight decay of SGD (Table 10: 1e-4) is the
 * Sum G + lambda W with lambda = ym 2^-ys. */
int oracle_sum_scaled(const o_tensor *X, int32_t xm, int32_t xs, const o_tensor *Y, int32_t ym, int32_t ys,
                      o_tensor *Z) {
    int st;
    if ((st = check_input(X)) || (st = check_input(Y))) return st;
    if (X->rows != Y->rows || X->cols != Y->cols) return ORC_ERR_ARG;
    if ((st = check_output(Z, X->rows, X->cols))) return st;
    if (xm < -512 || xm > 512 || ym < -512 || ym > 512 || xs < 0 || ys < 0 || xs > 64 || ys > 64)
        return ORC_ERR_ARG;
    int64_t n = X->rows * X->cols;
    i128 *v = malloc(sizeof(i128) * (n + 1));
    int *r = malloc(sizeof(int) * (n + 1));
    for (int64_t i = 0; i < X->rows; i++)
        for (int64_t j = 0; j < X->cols; j++)
            two_term((int64_t)xm * mant_at(X, i, j), exp_at(X, i, j) - xs, (int64_t)ym * mant_at(Y, i, j),
                     exp_at(Y, i, j) - ys, &v[i * X->cols + j], &r[i * X->cols + j]);
    st = fit_matrix(v, r, Z);
    free(v);
    free(r);
    return st;
}

int oracle_sum(const o_tensor *X, const o_tensor *Y, o_tensor *Z) {
    return oracle_sum_scaled(X, 1, 0, Y, 1, 0, Z);
}

/* ------------------------------------------------------------------------------------ */
/* Public: ReLU / ReLU6 (the Clip primitive)                                             */
/* ------------------------------------------------------------------------------------ */

/* Clip bound of ReLU6 in a group at exponent e (Table 7: c = min(6 >> e, q_max)): the
 * integer 6 shifted right by e, a left shift for negative e, then capped at q_max.
 * Read literally, a right shift truncates, so e = 2 gives 1 and e >= 3 gives 0. */
static int relu6_bound(int e) {
    if (e >= 0) return e >= 3 ? 0 : (6 >> e);
    if (-e >= 5) return QMAX; /* 6 << 5 = 192 already exceeds q_max */
    int c = 6 << (-e);
    return c > QMAX ? QMAX : c;
}

/* Forward ReLU (six = 0: max(C, 0)) or ReLU6 (six = 1: clip(C, 0, c)), Table 7: integer
 * operations on the mantissas, the exponent carried through unchanged.  Z has X's
 * shape and group geometry; its exponent grid is a copy of X's. */
int oracle_relu_fwd(const o_tensor *X, int six, o_tensor *Z) {
    int st;
    if ((st = check_input(X))) return st;
    if ((st = check_output(Z, X->rows, X->cols))) return st;
    if (Z->g_rows != X->g_rows || Z->g_cols != X->g_cols || (six != 0 && six != 1)) return ORC_ERR_ARG;
    for (int64_t i = 0; i < X->rows; i++)
        for (int64_t j = 0; j < X->cols; j++) {
            int c = mant_at(X, i, j), e = exp_at(X, i, j);
            int q = c > 0 ? c : 0;
            if (six && e != E_ZERO) {
                int b = relu6_bound(e);
                if (q > b) q = b;
            }
            Z->mant[i * Z->ld + j] = (int8_t)q;
        }
    memcpy(Z->exp, X->exp, (size_t)(n_grp_rows(X) * n_grp_cols(X)));
    return ORC_OK;
}

/* Backward ReLU / ReLU6 (Table 7): dX = dY * 1[C > 0] (ReLU) or dY * 1[0 < C < c]
 * (ReLU6), C the forward input's mantissa and c the bound of its group.  dX has dY's
 * shape and groups and dY's exponents (a mask changes no exponent). */
int oracle_relu_bwd(const o_tensor *X, const o_tensor *dY, int six, o_tensor *dX) {
    int st;
    if ((st = check_input(X)) || (st = check_input(dY))) return st;
    if (X->rows != dY->rows || X->cols != dY->cols || (six != 0 && six != 1)) return ORC_ERR_ARG;
    if ((st = check_output(dX, dY->rows, dY->cols))) return st;
    if (dX->g_rows != dY->g_rows || dX->g_cols != dY->g_cols) return ORC_ERR_ARG;
    for (int64_t i = 0; i < X->rows; i++)
        for (int64_t j = 0; j < X->cols; j++) {
            int c = mant_at(X, i, j), e = exp_at(X, i, j);
            int pass = c > 0 && (!six || c < relu6_bound(e));
            dX->mant[i * dX->ld + j] = pass ? (int8_t)mant_at(dY, i, j) : 0;
        }
    memcpy(dX->exp, dY->exp, (size_t)(n_grp_rows(dY) * n_grp_cols(dY)));
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Public: average pool (the Divide-by-constant primitive)                               */
/* ------------------------------------------------------------------------------------ */

/* RNE(x * 2^k / D) for D >= 1, exactly: the numerator and denominator as integers, then
 * floor division and a remainder test (ties to even). */
static i128 rne_div(i128 x, int k, int64_t D) {
    i128 num = x, den = D;
    if (k >= 0) num = x * ((i128)1 << k);
    else den = (i128)D << (-k);
    i128 q = num / den, rem = num % den;
    if (rem != 0 && num < 0) { q -= 1; rem += den; } /* floor division, 0 <= rem < den */
    if (2 * rem > den || (2 * rem == den && (q & 1))) q += 1;
    return q;
}

/* The smallest exponent at which RNE(x * 2^(r - e) / D) fits in [-127, 127] (x != 0). */
static int need_div(i128 x, int r, int64_t D) {
    int e = r + bitlen(x) - bitlen(D) - 8; /* |x| 2^(r-e) / D > 2^7 here: does not fit */
    for (;;) {
        i128 q = rne_div(x, r - e, D);
        if (q >= -QMAX && q <= QMAX) return e;
        e++;
    }
}

/* FIT of values x[i] * 2^r[i] / D into the groups of `out` (the divided counterpart of
 * fit_matrix: the group exponent is the largest need over its nonzero members, raised to
 * -127, E_ZERO for an all-zero group; each mantissa RNE(x 2^(r - e) / D)). */
static int fit_matrix_div(const i128 *x, const int *r, int64_t D, o_tensor *out) {
    int64_t ngc = n_grp_cols(out);
    int status = ORC_OK;
    for (int64_t gi = 0; gi < n_grp_rows(out); gi++)
        for (int64_t gj = 0; gj < ngc; gj++) {
            int64_t i0 = gi * out->g_rows, i1 = i0 + out->g_rows, j0 = gj * out->g_cols, j1 = j0 + out->g_cols;
            if (i1 > out->rows) i1 = out->rows;
            if (j1 > out->cols) j1 = out->cols;
            int have = 0, e = 0;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++) {
                    i128 v = x[i * out->cols + j];
                    if (v == 0) continue;
                    int ni = need_div(v, r[i * out->cols + j], D);
                    if (!have || ni > e) e = ni;
                    have = 1;
                }
            if (!have) e = E_ZERO;
            else if (e < -127) e = -127;
            if (e > 127) { status = ORC_ERR_EXP_RANGE; e = 127; }
            out->exp[gi * ngc + gj] = (int8_t)e;
            for (int64_t i = i0; i < i1; i++)
                for (int64_t j = j0; j < j1; j++) {
                    i128 v = x[i * out->cols + j];
                    i128 q = (v == 0 || e == E_ZERO) ? 0 : rne_div(v, r[i * out->cols + j] - e, D);
                    if (q < -QMAX) q = -QMAX;
                    if (q > QMAX) q = QMAX;
                    out->mant[i * out->ld + j] = (int8_t)q;
                }
        }
    return status;
}

/* Average pool K x K with stride K over NHWC activations X [n*h*w][c] (Table 6: "Average
 * pool (K x K)" -> Divide-by-constant, Eqs. 7-8, whose text the page does not print).
 * Reading: the exact integer sum S of the window's mantissas (one exponent e: activation
 * groups are uniform over pixels) divided by the constant D = K^2, the quotient S 2^e / D
 * rounded once by FIT into Y's groups.  h and w are multiples of K;
 * Y is [n*(h/K)*(w/K)][c]. */
int oracle_avgpool_fwd(const o_tensor *X, int n, int h, int w, int K, o_tensor *Y) {
    int st;
    if ((st = check_input(X))) return st;
    if (n < 1 || h < 1 || w < 1 || K < 1 || h % K || w % K || X->rows != (int64_t)n * h * w) return ORC_ERR_ARG;
    if (X->g_rows < X->rows) return ORC_ERR_LAYOUT; /* exponents uniform over pixels */
    int64_t P = h / K, Q = w / K, C = X->cols, rows = (int64_t)n * P * Q;
    if ((st = check_output(Y, rows, C))) return st;
    i128 *v = malloc(sizeof(i128) * (rows * C + 1));
    int *r = malloc(sizeof(int) * (rows * C + 1));
    for (int64_t img = 0; img < n; img++)
        for (int64_t p = 0; p < P; p++)
            for (int64_t q = 0; q < Q; q++)
                for (int64_t ch = 0; ch < C; ch++) {
                    i128 sum = 0;
                    for (int dy = 0; dy < K; dy++)
                        for (int dx = 0; dx < K; dx++)
                            sum += mant_at(X, (img * h + p * K + dy) * w + q * K + dx, ch);
                    int64_t o = ((img * P + p) * Q + q) * C + ch;
                    v[o] = sum;
                    r[o] = exp_at(X, 0, ch);
                }
    st = fit_matrix_div(v, r, (int64_t)K * K, Y);
    free(v);
    free(r);
    return st;
}

/* Backward of the K x K average pool: every input pixel of a window receives the window's
 * upstream gradient divided by D = K^2, dX = FIT(dY 2^e / D) into dX's groups.
 * dY [n*(h/K)*(w/K)][c] may have any group geometry; dX is [n*h*w][c]. */
int oracle_avgpool_bwd(const o_tensor *dY, int n, int h, int w, int K, o_tensor *dX) {
    int st;
    if ((st = check_input(dY))) return st;
    if (n < 1 || h < 1 || w < 1 || K < 1 || h % K || w % K) return ORC_ERR_ARG;
    int64_t P = h / K, Q = w / K, C = dY->cols;
    if (dY->rows != (int64_t)n * P * Q) return ORC_ERR_ARG;
    int64_t rows = (int64_t)n * h * w;
    if ((st = check_output(dX, rows, C))) return st;
    i128 *v = malloc(sizeof(i128) * (rows * C + 1));
    int *r = malloc(sizeof(int) * (rows * C + 1));
    for (int64_t img = 0; img < n; img++)
        for (int64_t y = 0; y < h; y++)
            for (int64_t x = 0; x < w; x++)
                for (int64_t ch = 0; ch < C; ch++) {
                    int64_t o = (img * P + y / K) * Q + x / K;
                    int64_t i = ((img * h + y) * w + x) * C + ch;
                    v[i] = mant_at(dY, o, ch);
                    r[i] = exp_at(dY, o, ch);
                }
    st = fit_matrix_div(v, r, (int64_t)K * K, dX);
    free(v);
    free(r);
    return st;
}

/* ------------------------------------------------------------------------------------ */
/* Introspection for the tests                                                           */
/* ------------------------------------------------------------------------------------ */

/* need() and RNE on int64 inputs, exported so the tests can pin them by brute force. */
/* ------------------------------------------------------------------------------------ */
/* Public: nonlinear-function primitive through lookup tables (Tables 7 and 8)          */
/* ------------------------------------------------------------------------------------ */

/* The tables are inputs (oracle/luts.py builds them from their defining formulas):
 *   lut_exp [30][256] uint8, [e - LUT_E_LO][k + 255] = round(exp(k 2^e) 2^7), k in [-255, 0]
 *   lut_log [256]     uint8, [p] = round(-log(p / 2^8) 2^5), p in [1, 254]
 *   lut_gelu_fwd / _bwd [30][256] int8, [e - LUT_E_LO][C + 128]
 * Rows cover e = -26 .. 3; every other exponent reads the nearest end row, which equals
 * the formula's value there (see oracle/luts.py). */
#define LUT_E_LO (-26)
#define LUT_E_HI 3
static int lut_row(int e) { return (e < LUT_E_LO ? LUT_E_LO : (e > LUT_E_HI ? LUT_E_HI : e)) - LUT_E_LO; }

/* Output head: softmax and cross-entropy of one target class per row (Table 8: LUT_exp
 * and LUT_log, B = 8).  Reading of the page's tables, step by step per row i:
 *   1. the row's logits to one exponent e_i (ALIGN_MAX along the row, as before any sum);
 *   2. k_j = C_j - max_j C_j, in [-254, 0];
 *   3. E_j = LUT_exp[e_i][k_j], about exp(z_j - z_max) 2^7;
 *   4. S = sum_j E_j (at least 128: the largest logit has k = 0);
 *   5. p_j = round(E_j 2^8 / S), the exact quotient rounded half to even (probability
 *      p_j / 2^8);
 *   6. loss_i = LUT_log[clamp(p_t, 1, 254)], the cross-entropy at scale 2^-5;
 *   7. gradient of the summed loss: g_j = p_j - 2^8 [j = t] at exponent -8, FIT into the
 *      groups of dZ.
 * loss[rows] receives the integers of step 6; target[i] must lie in [0, cols). */
int oracle_softmax_ce(const o_tensor *Z, const int32_t *target, const uint8_t *lut_exp,
                      const uint8_t *lut_log, int32_t *loss, o_tensor *dZ) {
    int st = check_input(Z);
    if (st) return st;
    if ((st = check_output(dZ, Z->rows, Z->cols))) return st;
    if (!target || !lut_exp || !lut_log || !loss) return ORC_ERR_ARG;
    const int64_t R = Z->rows, K = Z->cols;
    for (int64_t i = 0; i < R; i++)
        if (target[i] < 0 || target[i] >= K) return ORC_ERR_ARG;
    if (R == 0 || K == 0) return ORC_OK;
    int8_t *m, *e;
    if ((st = align_dense(Z, 1, &m, &e))) { free(m); free(e); return st; }
    i128 *x = malloc(sizeof(i128) * R * K);
    int *r = malloc(sizeof(int) * R * K);
    for (int64_t i = 0; i < R; i++) {
        const int8_t *c = m + i * K;
        int cmax = c[0];
        for (int64_t j = 1; j < K; j++) if (c[j] > cmax) cmax = c[j];
        const uint8_t *row = lut_exp + (int64_t)lut_row(e[i]) * 256;
        int64_t S = 0;
        for (int64_t j = 0; j < K; j++) S += row[c[j] - cmax + 255];
        int pt = 0;
        for (int64_t j = 0; j < K; j++) {
            int64_t num = (int64_t)row[c[j] - cmax + 255] << 8;
            int64_t q = num / S, rem = num - q * S;
            if (2 * rem > S || (2 * rem == S && (q & 1))) q++;
            if (j == target[i]) pt = (int)q;
            x[i * K + j] = q - (j == target[i] ? 256 : 0);
            r[i * K + j] = -8;
        }
        loss[i] = lut_log[pt < 1 ? 1 : (pt > 254 ? 254 : pt)];
    }
    st = fit_matrix(x, r, dZ);
    free(x); free(r); free(m); free(e);
    return st;
}

/* GELU forward through its table (Table 7): out = LUT_fwd[e][C] with the exponent of
 * every group carried unchanged (E_ZERO groups stay E_ZERO with zero mantissas).  out
 * must have H's shape and group partition. */
int oracle_gelu_lut_fwd(const o_tensor *H, const int8_t *lut_fwd, o_tensor *out) {
    int st = check_input(H);
    if (st) return st;
    if ((st = check_output(out, H->rows, H->cols))) return st;
    if (!lut_fwd || out->g_rows != H->g_rows || out->g_cols != H->g_cols) return ORC_ERR_ARG;
    for (int64_t i = 0; i < H->rows; i++)
        for (int64_t j = 0; j < H->cols; j++) {
            int e = exp_at(H, i, j), c = mant_at(H, i, j);
            out->mant[i * out->ld + j] = e == E_ZERO ? 0 : lut_fwd[lut_row(e) * 256 + c + 128];
        }
    memcpy(out->exp, H->exp, (size_t)(n_grp_rows(H) * n_grp_cols(H)));
    return ORC_OK;
}

/* GELU backward through its table (Table 7, "(dY * LUT_bwd[e, C]) >> B_G", B_G = 6):
 * read as the exact product dY * LUT_bwd[e_H][C_H] at exponent e_dY - 6, requantised by
 * FIT into the groups of dH like every other product. */
int oracle_gelu_lut_bwd(const o_tensor *H, const o_tensor *dY, const int8_t *lut_bwd, o_tensor *dH) {
    int st = check_input(H);
    if (st || (st = check_input(dY))) return st;
    if (dY->rows != H->rows || dY->cols != H->cols || !lut_bwd) return ORC_ERR_ARG;
    if ((st = check_output(dH, H->rows, H->cols))) return st;
    const int64_t n = H->rows * H->cols;
    i128 *x = malloc(sizeof(i128) * (n + 1));
    int *r = malloc(sizeof(int) * (n + 1));
    for (int64_t i = 0; i < H->rows; i++)
        for (int64_t j = 0; j < H->cols; j++) {
            int eh = exp_at(H, i, j), ch = mant_at(H, i, j);
            int ed = exp_at(dY, i, j), cd = mant_at(dY, i, j);
            int slope = lut_bwd[lut_row(eh == E_ZERO ? 0 : eh) * 256 + ch + 128];
            x[i * H->cols + j] = (i128)cd * slope;
            r[i * H->cols + j] = ed == E_ZERO ? 0 : ed - 6;
        }
    st = fit_matrix(x, r, dH);
    free(x); free(r);
    return st;
}

int oracle_need64(int64_t x, int32_t r) { return x == 0 ? E_ZERO : need(x, r); }
int64_t oracle_rne_shift64(int64_t x, int32_t k) { return (int64_t)rne_scale(x, k); }

/* FIT of one group of two-term values (a[i] * 2^pa[i] + b[i] * 2^pb[i]), exported so the
 * tests can compare the sticky reduction against unbounded integers. */
int oracle_fit_two_term(int64_t n, const int64_t *a, const int32_t *pa, const int64_t *b,
                        const int32_t *pb, int8_t *c_out) {
    i128 *x = malloc(sizeof(i128) * (n + 1));
    int *r = malloc(sizeof(int) * (n + 1));
    for (int64_t i = 0; i < n; i++) two_term(a[i], pa[i], b[i], pb[i], &x[i], &r[i]);
    int e = fit_group(n, x, r, c_out);
    free(x);
    free(r);
    return e;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
