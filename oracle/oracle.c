/*
 * oracle.c -- plain CPU reference of the fine-grained-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links,
 * loads or calls this file; only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * What it computes (the definition; every function below cites the passage
 * it follows):
 *
 *   D[m,n] = bf16_rne( sum_{kb=0}^{KB-1}
 *                        ( sum_{k=128kb}^{128kb+127} dec(A[m,k]) * dec(B[n,k]) )
 *                        * sa[m,kb] * sb[n/128, kb] )
 *
 * A carries one FP32 scale per 1x128 row group, B one per 128x128 block
 * (the "fine-grained scaling" of DeepSeek-V3 that DeepGEMM supports: GeekNews
 * "DeepSeek, DeepGEMM 오픈소스 공개", topic body, first bullet), and each
 * 128-wide K-block partial is promoted to higher precision before it is
 * scaled and accumulated (same page, fifth bullet: CUDA-core promotion of
 * the imprecise FP8 tensor-core accumulation).  Here the promotion target is
 * FP64:
 *   - a K-block partial is a sum of 128 products of e4m3 values; each product
 *     has at most 8 significant bits and lies in [2^-18, 448^2], so the
 *     128-term sum is exact in double;
 *   - the partial is multiplied by (double)sa then (double)sb and added to a
 *     double running sum, in K-block order (no reassociation);
 *   - the result is returned unrounded (for tolerance checks) and rounded
 *     once to bf16, round-to-nearest-even (the "bf16" of the API name,
 *     flashmla.net "Quick Start Guide": m_grouped_gemm_fp8_fp8_bf16_nt_...).
 *
 * Layouts (the library's boundary layouts):
 *   A  [M,K] e4m3 codes, K contiguous          (NT: B is [N,K], K contiguous)
 *   sa [KB][ld_sa] float, sa[kb*ld_sa + m]     (masked: [G][KB][ld_sa])
 *   sb [NB][KB]   float, sb[nb*KB + kb]        (grouped: [G][NB][KB])
 *   D  [M,N]                                   (masked: [G][Mmax][N])
 * Grouped layouts (GeekNews page, "MoE 모델을 위한 그룹화 GEMM 성능"):
 *   contiguous: rows grouped along M with N, K shared; m_indices[r] gives the
 *     expert of 128-row block r, -1 = no expert (rows left unwritten);
 *   masked: only rows m < masked_m[g] of group g are computed; the rest are
 *     left unwritten.
 *
 * Compiled with -ffp-contract=off so that no multiply-add is fused and every
 * operation rounds exactly as written.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------
 * e4m3 decode -- OCP 8-bit floating point, E4M3 ("fn") encoding: sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
 * subnormals m * 2^-9; S.1111.111 is NaN; there are no infinities; the
 * largest finite value is S.1111.110 = 448.  The pages name the format
 * (flashmla.net, "FP8 Precision Meets Industrial Rigor": fp8_e4m3/fp8_e5m2).
 * ------------------------------------------------------------------------- */
double fp8o_e4m3_value(uint8_t code)
{
    int s = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* (m/8) * 2^(1-7) */
    else
        v = ldexp(8.0 + (double)m, e - 7 - 3);  /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* ---------------------------------------------------------------------------
 * bf16 round-to-nearest-even of a double, one rounding.  bf16 = sign, 8-bit
 * exponent (bias 127), 7 stored mantissa bits; subnormal quantum 2^-133.
 * Returns the 16-bit pattern.
 * ------------------------------------------------------------------------- */
uint16_t fp8o_bf16_rne(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    int E, e;
    double q, n;
    if (isnan(x))
        return 0x7FC0;
    if (isinf(x))
        return sign | 0x7F80;
    if (a == 0.0)
        return sign;
    (void)frexp(a, &E);          /* a = f * 2^E, f in [0.5, 1) */
    e = E - 1;                   /* a in [2^e, 2^(e+1)) */
    if (e < -126)
        e = -126;                /* subnormal range shares the quantum 2^-133 */
    q = ldexp(1.0, e - 7);
    n = nearbyint(a / q);        /* a/q is exact (power-of-two scaling); ties to even */
    if (n >= 256.0) {            /* mantissa carried into the exponent */
        n = 128.0;
        e += 1;
    }
    if (n < 128.0)               /* subnormal (only when e == -126) */
        return sign | (uint16_t)n;
    if (e + 127 >= 255)
        return sign | 0x7F80;    /* overflow rounds to infinity */
    return sign | (uint16_t)(((e + 127) << 7) | ((int)n - 128));
}

/* ---------------------------------------------------------------------------
 * One output row of the definition above.  a_row: K codes of A's row;
 * sa_col: the row's K-block scales, stride sa_stride floats apart;
 * B: [N,K] codes; sb: [NB][KB].  Writes N doubles and N bf16 patterns.
 * ------------------------------------------------------------------------- */
static void row_nt(const uint8_t *a_row, const float *sa_col, long sa_stride,
                   const uint8_t *B, const float *sb, int N, int K,
                   double *out_exact, uint16_t *out_bf16)
{
    int KB = K / 128;
    double adec[128];
    double *acc = (double *)calloc((size_t)N, sizeof(double));
    for (int kb = 0; kb < KB; ++kb) {
        double s_a = (double)sa_col[(long)kb * sa_stride];
        for (int j = 0; j < 128; ++j)
            adec[j] = fp8o_e4m3_value(a_row[kb * 128 + j]);
        for (int n = 0; n < N; ++n) {
            const uint8_t *b = B + (long)n * K + (long)kb * 128;
            double partial = 0.0;                      /* exact: see header */
            for (int j = 0; j < 128; ++j)
                partial += adec[j] * fp8o_e4m3_value(b[j]);
            double s_b = (double)sb[(long)(n / 128) * KB + kb];
            acc[n] += (partial * s_a) * s_b;
        }
    }
    for (int n = 0; n < N; ++n) {
        if (out_exact)
            out_exact[n] = acc[n];
        if (out_bf16)
            out_bf16[n] = fp8o_bf16_rne(acc[n]);
    }
    free(acc);
}

/* ---------------------------------------------------------------------------
 * A job = a list of output rows; each resolved to (A row, sa column, B, sb,
 * output slot).  Threads take rows round-robin.  Rows are independent, so
 * splitting them across threads changes no arithmetic.
 * ------------------------------------------------------------------------- */
typedef struct {
    const uint8_t *a_row;
    const float *sa_col;
    long sa_stride;
    const uint8_t *B;
    const float *sb;
    double *out_exact;
    uint16_t *out_bf16;
} row_task;

typedef struct {
    const row_task *tasks;
    int ntasks, N, K, tid, nthreads;
} worker_arg;

static void *worker(void *p)
{
    worker_arg *w = (worker_arg *)p;
    for (int i = w->tid; i < w->ntasks; i += w->nthreads) {
        const row_task *t = &w->tasks[i];
        row_nt(t->a_row, t->sa_col, t->sa_stride, t->B, t->sb, w->N, w->K,
               t->out_exact, t->out_bf16);
    }
    return NULL;
}

static void run_tasks(const row_task *tasks, int ntasks, int N, int K, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    pthread_t th[256];
    worker_arg args[256];
    for (int t = 0; t < nthreads; ++t) {
        args[t] = (worker_arg){tasks, ntasks, N, K, t, nthreads};
        if (t > 0)
            pthread_create(&th[t], NULL, worker, &args[t]);
    }
    worker(&args[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
}

/* ---------------------------------------------------------------------------
 * Dense NT GEMM (GeekNews page, "일반 GEMM 성능 (Dense 모델)").
 * rows: the output rows to compute (NULL = all M rows, in order); output
 * slot i of out_exact/out_bf16 ([nrows][N]) holds row rows[i].
 * Returns 0, or -1 on a bad argument.
 * ------------------------------------------------------------------------- */
int fp8o_gemm_nt(const uint8_t *A, const float *sa, int ld_sa,
                 const uint8_t *B, const float *sb,
                 int M, int N, int K, const int *rows, int nrows,
                 double *out_exact, uint16_t *out_bf16, int nthreads)
{
    if (K % 128 || M < 0 || N < 0 || ld_sa < M)
        return -1;
    if (!rows)
        nrows = M;
    row_task *tasks = (row_task *)malloc(sizeof(row_task) * (size_t)(nrows ? nrows : 1));
    for (int i = 0; i < nrows; ++i) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) {
            free(tasks);
            return -1;
        }
        tasks[i] = (row_task){A + (long)m * K, sa + m, ld_sa, B, sb,
                              out_exact ? out_exact + (long)i * N : NULL,
                              out_bf16 ? out_bf16 + (long)i * N : NULL};
    }
    run_tasks(tasks, nrows, N, K, nthreads);
    free(tasks);
    return 0;
}

/* ---------------------------------------------------------------------------
 * M-grouped contiguous (GeekNews page, "연속된(contiguous) 레이아웃"): the
 * experts' row segments are concatenated along M; 128-row block r uses expert
 * m_indices[r]'s B [N,K] and sb [NB][KB]; blocks with m_indices[r] < 0 are
 * skipped and their output rows are not written.
 * B: [G][N][K]; sb: [G][NB][KB]; out rows are indexed like `rows`.
 * ------------------------------------------------------------------------- */
int fp8o_m_grouped_contiguous(const uint8_t *A, const float *sa, int ld_sa,
                              const uint8_t *B, const float *sb, const int32_t *m_indices,
                              int M, int N, int K, int G, const int *rows, int nrows,
                              double *out_exact, uint16_t *out_bf16, int nthreads)
{
    if (K % 128 || M % 128 || N < 0 || G < 1 || ld_sa < M)
        return -1;
    int KB = K / 128, NB = (N + 127) / 128;
    if (!rows)
        nrows = M;
    row_task *tasks = (row_task *)malloc(sizeof(row_task) * (size_t)(nrows ? nrows : 1));
    int nt = 0;
    for (int i = 0; i < nrows; ++i) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) {
            free(tasks);
            return -1;
        }
        int g = m_indices[m / 128];
        if (g < 0)
            continue;                 /* skipped block: row not written */
        if (g >= G) {
            free(tasks);
            return -1;
        }
        tasks[nt++] = (row_task){A + (long)m * K, sa + m, ld_sa,
                                 B + (long)g * N * K, sb + (long)g * NB * KB,
                                 out_exact ? out_exact + (long)i * N : NULL,
                                 out_bf16 ? out_bf16 + (long)i * N : NULL};
    }
    run_tasks(tasks, nt, N, K, nthreads);
    free(tasks);
    return 0;
}

/* ---------------------------------------------------------------------------
 * M-grouped masked (GeekNews page, "마스킹(masked) 레이아웃": a mask input
 * says how many rows each expert really has, for CUDA-graph decode where the
 * host does not know the counts): A [G][Mmax][K], sa [G][KB][ld_sa],
 * B [G][N][K], sb [G][NB][KB], out [G][Mmax][N].  Group g computes rows
 * m < min(masked_m[g], Mmax); other rows are not written.
 * ------------------------------------------------------------------------- */
int fp8o_m_grouped_masked(const uint8_t *A, const float *sa, int ld_sa,
                          const uint8_t *B, const float *sb, const int32_t *masked_m,
                          int G, int Mmax, int N, int K,
                          double *out_exact, uint16_t *out_bf16, int nthreads)
{
    if (K % 128 || Mmax < 0 || N < 0 || G < 1 || ld_sa < Mmax)
        return -1;
    int KB = K / 128, NB = (N + 127) / 128;
    long total = 0;
    for (int g = 0; g < G; ++g) {
        int mg = masked_m[g] < 0 ? 0 : (masked_m[g] > Mmax ? Mmax : masked_m[g]);
        total += mg;
    }
    row_task *tasks = (row_task *)malloc(sizeof(row_task) * (size_t)(total ? total : 1));
    int nt = 0;
    for (int g = 0; g < G; ++g) {
        int mg = masked_m[g] < 0 ? 0 : (masked_m[g] > Mmax ? Mmax : masked_m[g]);
        for (int m = 0; m < mg; ++m) {
            long orow = (long)g * Mmax + m;
            tasks[nt++] = (row_task){A + orow * K, sa + (long)g * KB * ld_sa + m, ld_sa,
                                     B + (long)g * N * K, sb + (long)g * NB * KB,
                                     out_exact ? out_exact + orow * N : NULL,
                                     out_bf16 ? out_bf16 + orow * N : NULL};
        }
    }
    run_tasks(tasks, nt, N, K, nthreads);
    free(tasks);
    return 0;
}

/* ===========================================================================
 * FP8 quantisation of the GEMM's inputs.  The pages leave this step to the
 * user (kakushin.no, "Hvorfor FP8 og FP4 er interessant": inputs must be
 * converted to FP8 by the caller); the granularity is the one of the GEMM
 * above (one FP32 scale per 1x128 row group of A, per 128x128 block of B).
 * Readings, since the pages give no formula: scale = amax / 448 in FP32 (448
 * is the largest finite e4m3 value), scale = 1 for an all-zero group, and
 * code = e4m3_rne_satfinite(x / scale) with x / scale one IEEE FP32 division.
 * These functions work in FP32 because that is the precision in which the
 * scale and the quotient are defined; the e4m3 rounding itself is done
 * exactly (in double) from the format definition.
 * ======================================================================== */

/* e4m3 ("fn") code of a finite float: round to nearest, ties to even, values
 * beyond the largest finite magnitude (448) saturate to +-448; the sign of
 * zero is kept.  Normal codes: (1 + m/8) * 2^(e-7), e = 1..15 (e = 15 only up
 * to m = 6); subnormals: (m/8) * 2^-6.  */
uint8_t fp8o_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    int E, e;
    double q, steps;
    if (a == 0.0)
        return sign;
    (void)frexp(a, &E);        /* a = f * 2^E, f in [0.5, 1) */
    e = E - 1;                 /* a in [2^e, 2^(e+1)) */
    if (e < -6)
        e = -6;                /* subnormals share the quantum 2^-9 */
    q = ldexp(1.0, e - 3);     /* 3 mantissa bits */
    steps = nearbyint(a / q);  /* exact quotient; ties to even */
    if (steps >= 16.0) {       /* mantissa carried into the exponent */
        steps = 8.0;
        e += 1;
    }
    if (e > 8 || (e == 8 && steps > 14.0))
        return sign | 0x7E;    /* saturate to 448 = 1.75 * 2^8 */
    if (steps < 8.0)           /* subnormal (only at e == -6) */
        return sign | (uint8_t)steps;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)steps - 8));
}

static float scale_of_amax(float amax)
{
    return amax > 0.0f ? amax / 448.0f : 1.0f;
}

/* Activations: x [rows][K] (K % 128 == 0) -> q [rows][K] e4m3 codes and
 * sa [KB][ld_sa] (the GEMM's MN-major layout): one scale per 1x128 group of
 * a row.  Entries of sa past `rows` are not written.  Returns 0, or -1 on a
 * bad argument. */
int fp8o_quantize_1x128(const float *x, int rows, int K, uint8_t *q, float *sa, int ld_sa)
{
    if (K <= 0 || K % 128 || rows < 0 || ld_sa < rows)
        return -1;
    int KB = K / 128;
    for (long r = 0; r < rows; ++r) {
        for (int kb = 0; kb < KB; ++kb) {
            const float *g = x + r * K + (long)kb * 128;
            float amax = 0.0f;
            for (int j = 0; j < 128; ++j)
                if (fabsf(g[j]) > amax)
                    amax = fabsf(g[j]);
            float s = scale_of_amax(amax);
            for (int j = 0; j < 128; ++j)
                q[r * K + (long)kb * 128 + j] = fp8o_e4m3_encode(g[j] / s);
            sa[(long)kb * ld_sa + r] = s;
        }
    }
    return 0;
}

/* Weights: x [N][K] (K % 128 == 0) -> q [N][K] codes and sb [NB][KB]: one
 * scale per 128x128 block; the last block row holds the N % 128 remaining
 * rows when N is not a multiple of 128.  Returns 0, or -1 on a bad argument. */
int fp8o_quantize_128x128(const float *x, int N, int K, uint8_t *q, float *sb)
{
    if (K <= 0 || K % 128 || N < 0)
        return -1;
    int KB = K / 128, NB = (N + 127) / 128;
    for (int nb = 0; nb < NB; ++nb) {
        int r0 = nb * 128, r1 = r0 + 128 < N ? r0 + 128 : N;
        for (int kb = 0; kb < KB; ++kb) {
            float amax = 0.0f;
            for (long r = r0; r < r1; ++r)
                for (int j = 0; j < 128; ++j) {
                    float v = fabsf(x[r * K + (long)kb * 128 + j]);
                    if (v > amax)
                        amax = v;
                }
            float s = scale_of_amax(amax);
            for (long r = r0; r < r1; ++r)
                for (int j = 0; j < 128; ++j) {
                    long i = r * K + (long)kb * 128 + j;
                    q[i] = fp8o_e4m3_encode(x[i] / s);
                }
            sb[(long)nb * KB + kb] = s;
        }
    }
    return 0;
}

/* ===========================================================================
 * The expert pipeline on either side of the contiguous grouped GEMM (GeekNews
 * page, "MoE 모델을 위한 그룹화 GEMM 성능": the contiguous layout groups the
 * rows of A along M by expert, with N and K shared, one expert per 128-row
 * block).  The pages describe only the layout; the steps below are its
 * plainest construction (readings, since the pages give no algorithm):
 *
 *  dispatch: routed row r (r = t * topk + k: token t, slot k) goes to expert
 *    e[r].  Expert g's rows, in increasing r, fill a segment padded to a
 *    multiple of 128 rows; the segments follow each other in expert order
 *    (off[g] = sum over g' < g of the padded counts).  Row r lands at
 *    pos[r] = off[e[r]] + (number of r' < r with e[r'] == e[r]).  Block b of
 *    the padded layout has m_indices[b] = its expert, or -1 past the last
 *    segment (up to `blocks` entries).  Row pos[r] of A holds token t's
 *    activations quantised per 1x128 group (the quantiser above); padding
 *    rows hold zero codes and zero scales.
 *  combine: out[t, n] = bf16_rne(acc), acc = sum over k of w[t*topk + k] *
 *    D[pos[t*topk + k], n], accumulated in FP32 in slot order with one fused
 *    multiply-add per slot (acc = fmaf(w, d, acc), acc starting at 0); D is
 *    bf16.  w == NULL means every weight is 1.
 * ======================================================================== */

/* Layout only.  e [R] experts (0 <= e < G, -1 = row dropped: it gets
 * pos = -1 and no place); outputs cnt [G], off [G], pos [R], m_indices
 * [blocks].  Returns the number of 128-row blocks used, or -1 if they do not
 * fit in `blocks` or an argument is bad. */
int fp8o_moe_layout(const int32_t *e, int R, int G, int blocks,
                    int32_t *cnt, int32_t *off, int32_t *pos, int32_t *m_indices)
{
    if (R < 0 || G < 1 || blocks < 0)
        return -1;
    for (int g = 0; g < G; ++g)
        cnt[g] = 0;
    for (int r = 0; r < R; ++r) {
        if (e[r] >= G)
            return -1;
        if (e[r] >= 0)
            cnt[e[r]]++;
    }
    long used = 0;
    for (int g = 0; g < G; ++g) {
        off[g] = (int32_t)(used * 128);
        used += (cnt[g] + 127) / 128;
    }
    if (used > blocks)
        return -1;
    for (int b = 0; b < blocks; ++b)
        m_indices[b] = -1;
    for (int g = 0; g < G; ++g)
        for (int b = off[g] / 128; b < off[g] / 128 + (cnt[g] + 127) / 128; ++b)
            m_indices[b] = g;
    int32_t *seen = (int32_t *)calloc((size_t)G, sizeof(int32_t));
    for (int r = 0; r < R; ++r) {
        if (e[r] < 0) {
            pos[r] = -1;
            continue;
        }
        pos[r] = off[e[r]] + seen[e[r]]++;
    }
    free(seen);
    return (int)used;
}

/* Dispatch with quantisation: x [T][K] float (token activations), e [R]
 * with R = T * topk.  Writes A [blocks*128][K] codes, sa [KB][ld_sa]
 * (ld_sa >= blocks*128), pos [R], m_indices [blocks].  Rows of A in unused
 * blocks are left as they are.  Returns the number of blocks used, or -1. */
int fp8o_moe_dispatch(const float *x, int T, int K, const int32_t *e, int topk, int G, int blocks,
                      uint8_t *A, float *sa, int ld_sa, int32_t *pos, int32_t *m_indices)
{
    if (T < 0 || topk < 1 || K <= 0 || K % 128 || ld_sa < blocks * 128)
        return -1;
    int R = T * topk, KB = K / 128;
    int32_t *cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)G);
    int32_t *off = (int32_t *)malloc(sizeof(int32_t) * (size_t)G);
    int used = fp8o_moe_layout(e, R, G, blocks, cnt, off, pos, m_indices);
    if (used >= 0) {
        /* padding rows: zero codes, zero scales */
        for (int g = 0; g < G; ++g)
            for (long row = off[g] + cnt[g]; row < off[g] + (long)(cnt[g] + 127) / 128 * 128; ++row) {
                memset(A + row * K, 0, (size_t)K);
                for (int kb = 0; kb < KB; ++kb)
                    sa[(long)kb * ld_sa + row] = 0.0f;
            }
        /* routed rows: the token's row quantised per 1x128 group */
        float *rowsa = (float *)malloc(sizeof(float) * (size_t)KB);
        for (int r = 0; r < R; ++r) {
            if (pos[r] < 0)
                continue;
            fp8o_quantize_1x128(x + (long)(r / topk) * K, 1, K, A + (long)pos[r] * K, rowsa, 1);
            for (int kb = 0; kb < KB; ++kb)
                sa[(long)kb * ld_sa + pos[r]] = rowsa[kb];
        }
        free(rowsa);
    }
    free(cnt);
    free(off);
    return used;
}

/* Combine: D [rows][N] bf16 patterns, pos [T*topk], w [T*topk] or NULL ->
 * out [T][N] bf16 patterns.  Slots with pos < 0 are skipped.  Returns 0. */
int fp8o_moe_combine(const uint16_t *D, int N, const int32_t *pos, const float *w,
                     int T, int topk, uint16_t *out)
{
    for (long t = 0; t < T; ++t)
        for (int n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int k = 0; k < topk; ++k) {
                long r = t * topk + k;
                if (pos[r] < 0)
                    continue;
                uint32_t bits = (uint32_t)D[(long)pos[r] * N + n] << 16;
                float d;
                memcpy(&d, &bits, sizeof d);
                acc = fmaf(w ? w[r] : 1.0f, d, acc);
            }
            out[t * N + n] = fp8o_bf16_rne((double)acc);
        }
    return 0;
}

/* ===========================================================================
 * BF16 NT GEMM, the other input format the pages list for the library
 * (kakushin.no, "Hva gjør DeepGEMM?": FP8, FP4 and BF16 computations):
 *   D[m,n] = bf16_rne( sum_k A[m,k] * B[n,k] ),  A [M][K], B [N][K] bf16.
 * Each product of two bf16 values is exact in double (8 + 8 significant
 * bits); the K-term sum is accumulated in double in k order (relative error
 * far below the bf16 output's 2^-9) and rounded once to bf16.  Returns the
 * unrounded sums and their bf16 patterns for the rows listed (NULL = all).
 * ======================================================================== */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int fp8o_bf16_gemm_nt(const uint16_t *A, const uint16_t *B, int M, int N, int K,
                      const int *rows, int nrows, double *out_exact, uint16_t *out_bf16)
{
    if (M < 0 || N < 0 || K < 0)
        return -1;
    if (!rows)
        nrows = M;
    double *arow = (double *)malloc(sizeof(double) * (size_t)(K ? K : 1));
    for (int i = 0; i < nrows; ++i) {
        int m = rows ? rows[i] : i;
        if (m < 0 || m >= M) {
            free(arow);
            return -1;
        }
        for (int k = 0; k < K; ++k)
            arow[k] = bf16_value(A[(long)m * K + k]);
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += arow[k] * bf16_value(B[(long)n * K + k]);
            if (out_exact)
                out_exact[(long)i * N + n] = acc;
            if (out_bf16)
                out_bf16[(long)i * N + n] = fp8o_bf16_rne(acc);
        }
    }
    free(arow);
    return 0;
}

/* ===========================================================================
 * Power-of-two (UE8M0) scales: the scale format of the block-scaled FP8
 * tensor-core instructions that the SM100 generation the pages list adds
 * (kakushin.no, requirements list: SM90 and SM100; the power-of-two scale
 * format is the OCP microscaling E8M0 one).  A scale byte e stands for
 * 2^(e - 127); e = 255 is NaN.  Same granularity and definition as the FP32
 * scales above:
 *   D[m,n] = bf16_rne( sum_kb ( sum_{k in kb} A[m,k] B[n,k] )
 *                             * 2^(ea[kb][m] - 127) * 2^(eb[n/128][kb] - 127) )
 * sfa [KB][ld_sf] bytes (MN-major like sa), sfb [NB][KB] bytes.  The powers
 * of two are exact in float, so the FP32-scale definition is evaluated on
 * the decoded scales.
 * ======================================================================== */
double fp8o_ue8m0_value(uint8_t e)
{
    return e == 255 ? NAN : ldexp(1.0, (int)e - 127);
}

int fp8o_gemm_nt_ue8m0(const uint8_t *A, const uint8_t *sfa, int ld_sf, const uint8_t *B,
                       const uint8_t *sfb, int M, int N, int K, const int *rows, int nrows,
                       double *out_exact, uint16_t *out_bf16, int nthreads)
{
    if (K <= 0 || K % 128 || M < 0 || N < 0 || ld_sf < M)
        return -1;
    int KB = K / 128, NB = (N + 127) / 128;
    float *sa = (float *)malloc(sizeof(float) * (size_t)KB * (size_t)(ld_sf ? ld_sf : 1));
    float *sb = (float *)malloc(sizeof(float) * (size_t)NB * (size_t)KB + 1);
    for (long i = 0; i < (long)KB * ld_sf; ++i)
        sa[i] = (float)fp8o_ue8m0_value(sfa[i]);
    for (long i = 0; i < (long)NB * KB; ++i)
        sb[i] = (float)fp8o_ue8m0_value(sfb[i]);
    int rc = fp8o_gemm_nt(A, sa, ld_sf, B, sb, M, N, K, rows, nrows, out_exact, out_bf16, nthreads);
    free(sa);
    free(sb);
    return rc;
}
