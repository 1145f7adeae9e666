/*
 * lcla_oracle.c -- fp64 CPU oracle for block-causal ReLU linear attention.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header or table
 * with the CUDA library; both receive the same seeded inputs from the caller.
 *
 * What is computed (per batch entry b and head h; all arithmetic in double,
 * inputs widened exactly from bf16 bits or float32):
 *
 *   phi(x)     = ReLU(x) elementwise
 *                ("Implementing Block Causal Linear Attention for Long Video
 *                 Generation with Sana", section "The Linear Attention Kernel":
 *                 the kernel function is nn.ReLU, applied to Q and K only).
 *   R_n y      = rotary embedding of y at token n: for each pair p,
 *                (y_2p, y_2p+1) -> (y_2p c - y_2p+1 s, y_2p s + y_2p+1 c) with
 *                c = rope_cos[n][p], s = rope_sin[n][p]; applied to phi(q) and
 *                phi(k) right after the kernel (same page, section "Rotary
 *                Position Embeddings").
 *   blk(n)     = n / block_len; a token attends to every token of its own block
 *                and of all earlier blocks (same page, section "Chunk-Wise
 *                Causality": causality through prefix-sum ordering over chunks;
 *                "Block Causal Linear Attention" note, section "What SANA-Video
 *                Actually Uses": the carried state is cumulative over earlier
 *                blocks).  Inside a block the attention is bidirectional.
 *   out_i      = sum_{j: blk(j) <= blk(i)} v_j (R_j phi(k_j) . R_i phi(q_i))
 *                / ( sum_{same j} phi(k_j) . phi(q_i) + eps )
 *                (same page, "The Linear Attention Kernel": the normaliser uses
 *                the unrotated features, vk = v k_rotated^T, out = vk q_rotated,
 *                output = out * z).
 *   state      = (S, z) with S[c][e] = sum_j v_j[c] (R_j phi(k_j))[e] and
 *                z[e] = sum_j phi(k_j)[e], packed row-major as [d+1][d] with
 *                row d holding z ("[feat] LongSANA" PR: the causal linear
 *                attention KV cache carried across chunks).
 *
 * Three independent evaluation routes are provided:
 *   lcla_oracle_masked      the definition above, pair by pair (O(N^2 d)).
 *   lcla_oracle_recurrence  per-block local states, running inclusive sum.
 *   lcla_oracle_step        one block against a carried state, optional save.
 *
 * Element type code: 0 = bf16 bit patterns (uint16), 1 = float32.
 * Return value: 0 on success, -1 on an invalid argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double widen(const void *p, int dtype, size_t i)
{
    if (dtype == 0) {
        uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* ReLU that lets NaN through, as a comparison-based max does. */
static double relu(double x) { return x < 0.0 ? 0.0 : x; }

/* Load row (b, n, h) of a [B, N, H, d] tensor, widened to double. */
static void load_row(const void *t, int dtype, int N, int H, int d,
                     int b, long n, int h, double *dst)
{
    size_t base = (((size_t)b * N + (size_t)n) * H + h) * (size_t)d;
    for (int e = 0; e < d; ++e) dst[e] = widen(t, dtype, base + e);
}

static void apply_relu(double *x, int d)
{
    for (int e = 0; e < d; ++e) x[e] = relu(x[e]);
}

/* Rotary embedding of x at table row n, interleaved pairs. */
static void rotate(const double *x, const float *cs, const float *sn, long n,
                   int d, double *y)
{
    const float *c = cs + (size_t)n * (d / 2);
    const float *s = sn + (size_t)n * (d / 2);
    for (int p = 0; p < d / 2; ++p) {
        double a = x[2 * p], b = x[2 * p + 1];
        y[2 * p] = a * (double)c[p] - b * (double)s[p];
        y[2 * p + 1] = a * (double)s[p] + b * (double)c[p];
    }
}

static double dot(const double *a, const double *b, int d)
{
    double acc = 0.0;
    for (int e = 0; e < d; ++e) acc += a[e] * b[e];
    return acc;
}

static int check(const void *q, const void *k, const void *v, int dtype,
                 const float *cs, const float *sn, int B, int H, long N, int d,
                 long block_len)
{
    if (!q || !k || !v || !cs || !sn) return -1;
    if (dtype != 0 && dtype != 1) return -1;
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || (d & 1) || block_len <= 0) return -1;
    return 0;
}

void lcla_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int lcla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Masked form: the definition evaluated pair by pair.
 * rows: token indices to evaluate (each in [0, N)), or NULL for all tokens.
 * out:  [B, nrows, H, d] (nrows = N when rows is NULL).
 */
int lcla_oracle_masked(const void *q, const void *k, const void *v, int dtype,
                       const float *rope_cos, const float *rope_sin,
                       int B, int H, int N, int d, int block_len, double eps,
                       const int64_t *rows, int64_t nrows, double *out)
{
    if (check(q, k, v, dtype, rope_cos, rope_sin, B, H, N, d, block_len) || !out)
        return -1;
    if (d > 256) return -1;
    if (!rows) nrows = N;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;

    /* phi(k_j) and R_j phi(k_j) for one (b, h), shared by every row i. */
    double *kf = (double *)malloc(sizeof(double) * (size_t)N * d);
    double *kr = (double *)malloc(sizeof(double) * (size_t)N * d);
    if (!kf || !kr) { free(kf); free(kr); return -1; }

    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            #pragma omp parallel for schedule(static)
            for (long j = 0; j < N; ++j) {
                load_row(k, dtype, N, H, d, b, j, h, kf + (size_t)j * d);
                apply_relu(kf + (size_t)j * d, d);
                rotate(kf + (size_t)j * d, rope_cos, rope_sin, j, d, kr + (size_t)j * d);
            }
            #pragma omp parallel for schedule(dynamic, 16)
            for (int64_t r = 0; r < nrows; ++r) {
                long i = rows ? (long)rows[r] : (long)r;
                double qf[256], qr[256], num[256], vj[256];
                load_row(q, dtype, N, H, d, b, i, h, qf);
                apply_relu(qf, d);
                rotate(qf, rope_cos, rope_sin, i, d, qr);
                long last = ((long)(i / block_len) + 1) * (long)block_len; /* end of i's block */
                if (last > N) last = N;
                double den = 0.0;
                for (int c = 0; c < d; ++c) num[c] = 0.0;
                for (long j = 0; j < last; ++j) {
                    double a = dot(kr + (size_t)j * d, qr, d);
                    load_row(v, dtype, N, H, d, b, j, h, vj);
                    for (int c = 0; c < d; ++c) num[c] += vj[c] * a;
                    den += dot(kf + (size_t)j * d, qf, d);
                }
                double *o = out + (((size_t)b * nrows + (size_t)r) * H + h) * (size_t)d;
                for (int c = 0; c < d; ++c) o[c] = num[c] / (den + eps);
            }
        }
    free(kf);
    free(kr);
    return 0;
}

/* (token, output slot) pair: requested rows are visited in token order. */
typedef struct { int64_t tok, slot; } row_ref;

static int row_ref_cmp(const void *a, const void *b)
{
    const row_ref *x = (const row_ref *)a, *y = (const row_ref *)b;
    return (x->tok > y->tok) - (x->tok < y->tok);
}

/* out_i = (P S-part . R_i phi(q_i)) / (P z-part . phi(q_i) + eps) */
static void eval_row(const void *q, int dtype, const float *cs, const float *sn, int N, int H,
                     int d, int b, int h, long i, const double *P, double eps, double *o)
{
    double qf[256], qr[256];
    load_row(q, dtype, N, H, d, b, i, h, qf);
    apply_relu(qf, d);
    rotate(qf, cs, sn, i, d, qr);
    double den = dot(P + (size_t)d * d, qf, d) + eps;
    for (int c = 0; c < d; ++c) o[c] = dot(P + (size_t)c * d, qr, d) / den;
}

/*
 * Block-recurrence form.  For each (b, h): start from state_in (zero when
 * NULL), add each block's local state (S_blk, z_blk) in block order to the
 * running sum P, and right after block blk evaluate that block's requested
 * tokens against P (the inclusive sum through blk).
 *
 * state_in     [B, H, d+1, d] or NULL.
 * rows, nrows  as in the masked form; out [B, nrows, H, d] or NULL.
 * state_out    [B, H, d+1, d] or NULL: the running sum after the last block.
 * prefix       [B, H, nblocks, d+1, d] or NULL: every inclusive running sum.
 */
int lcla_oracle_recurrence(const void *q, const void *k, const void *v, int dtype,
                           const float *rope_cos, const float *rope_sin,
                           int B, int H, int N, int d, int block_len, double eps,
                           const double *state_in,
                           const int64_t *rows, int64_t nrows, double *out,
                           double *state_out, double *prefix)
{
    if (check(q, k, v, dtype, rope_cos, rope_sin, B, H, N, d, block_len)) return -1;
    if (d > 256) return -1;
    if (!rows) nrows = N;
    for (int64_t r = 0; rows && r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;
    const long nb = ((long)N + block_len - 1) / block_len;
    const size_t sz = (size_t)(d + 1) * d;
    row_ref *order = (row_ref *)malloc(sizeof(row_ref) * (size_t)(nrows > 0 ? nrows : 1));
    if (!order) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        order[r].tok = rows ? rows[r] : r;
        order[r].slot = r;
    }
    if (rows) qsort(order, (size_t)nrows, sizeof(row_ref), row_ref_cmp);
    int failed = 0;

    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *acc = (double *)calloc(sz, sizeof(double));
            if (!acc) { failed = 1; continue; }
            if (state_in) memcpy(acc, state_in + ((size_t)b * H + h) * sz, sz * sizeof(double));
            double kf[256], kr[256], vj[256];
            int64_t next = 0;    /* next entry of order[] to evaluate */
            for (long blk = 0; blk < nb; ++blk) {
                long j0 = blk * (long)block_len, j1 = j0 + block_len;
                if (j1 > N) j1 = N;
                for (long j = j0; j < j1; ++j) {
                    load_row(k, dtype, N, H, d, b, j, h, kf);
                    apply_relu(kf, d);
                    rotate(kf, rope_cos, rope_sin, j, d, kr);
                    load_row(v, dtype, N, H, d, b, j, h, vj);
                    for (int c = 0; c < d; ++c)
                        for (int e = 0; e < d; ++e) acc[(size_t)c * d + e] += vj[c] * kr[e];
                    for (int e = 0; e < d; ++e) acc[(size_t)d * d + e] += kf[e];
                }
                if (prefix)
                    memcpy(prefix + (((size_t)b * H + h) * nb + blk) * sz, acc, sz * sizeof(double));
                for (; out && next < nrows && order[next].tok < j1; ++next)
                    eval_row(q, dtype, rope_cos, rope_sin, N, H, d, b, h, (long)order[next].tok,
                             acc, eps,
                             out + (((size_t)b * nrows + (size_t)order[next].slot) * H + h) * (size_t)d);
            }
            if (state_out) memcpy(state_out + ((size_t)b * H + h) * sz, acc, sz * sizeof(double));
            free(acc);
        }
    free(order);
    return failed ? -1 : 0;
}

/*
 * Step form: one block of L tokens against the carried state.
 * q, k, v [B, L, H, d]; tables [L, d/2] at the block's absolute positions.
 * state [B, H, d+1, d] in/out: P = state + local(block); out_i uses P; when
 * save != 0 the state becomes P, otherwise it is left untouched.
 */
int lcla_oracle_step(const void *q, const void *k, const void *v, int dtype,
                     const float *rope_cos, const float *rope_sin,
                     int B, int H, int L, int d, double eps,
                     double *state, int save, double *out)
{
    if (check(q, k, v, dtype, rope_cos, rope_sin, B, H, L, d, L) || !state || !out)
        return -1;
    if (d > 256) return -1;
    const size_t sz = (size_t)(d + 1) * d;
    int failed = 0;

    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *st = state + ((size_t)b * H + h) * sz;
            double *S = (double *)calloc(sz, sizeof(double));     /* local block state */
            if (!S) { failed = 1; continue; }
            double kf[256], kr[256], vj[256], qf[256], qr[256];
            for (long j = 0; j < L; ++j) {
                load_row(k, dtype, L, H, d, b, j, h, kf);
                apply_relu(kf, d);
                rotate(kf, rope_cos, rope_sin, j, d, kr);
                load_row(v, dtype, L, H, d, b, j, h, vj);
                for (int c = 0; c < d; ++c)
                    for (int e = 0; e < d; ++e) S[(size_t)c * d + e] += vj[c] * kr[e];
                for (int e = 0; e < d; ++e) S[(size_t)d * d + e] += kf[e];
            }
            for (size_t x = 0; x < sz; ++x) S[x] += st[x];          /* P = state + local */
            for (long i = 0; i < L; ++i) {
                load_row(q, dtype, L, H, d, b, i, h, qf);
                apply_relu(qf, d);
                rotate(qf, rope_cos, rope_sin, i, d, qr);
                double den = dot(S + (size_t)d * d, qf, d) + eps;
                double *o = out + (((size_t)b * L + (size_t)i) * H + h) * (size_t)d;
                for (int c = 0; c < d; ++c) o[c] = dot(S + (size_t)c * d, qr, d) / den;
            }
            if (save) memcpy(st, S, sz * sizeof(double));
            free(S);
        }
    return failed ? -1 : 0;
}
