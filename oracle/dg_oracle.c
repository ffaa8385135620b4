/*
 * CPU oracle for the FP8 (E4M3) block-scaled GEMM D = A * B^T, dense and
 * MoE M-grouped (contiguous and masked layouts).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; the two are compared,
 * never mixed.
 *
 * What it computes (plain definitions, written out):
 *
 *  - E4M3 bytes are decoded by a 256-entry table built from the format
 *    definition (sign, 4 exponent bits with bias 7, 3 mantissa bits, the
 *    "fn" variant: no infinities, S.1111.111 is NaN, max 448).  The pages
 *    call the operand format FP8 ("DeepSeek open-source week day 3: DeepGEMM",
 *    deepseek.csdn.net, part 1.2 "precision safeguards"; the same page quotes
 *    a +-240 range, which is the FNUZ variant and contradicts the 448 used by
 *    the quantiser, so the "fn" reading is taken).
 *  - Fine-grained scaling: A has one FP32 scale per row per 128-wide K block,
 *    B one per 128 x 128 block (same article, part 1.2, "fine-grained scaling
 *    factors"; the later project card "DeepGEMM: FP8/FP4 high-performance CUDA
 *    matrix core library", aiproducthub.cn, section "technical implementation",
 *    on the scale-factor layout).  A_hat[m,k] = dec(a[m,k]) * sfa[m, k/128];
 *    B_hat[n,k] = dec(b[n,k]) * sfb[n/128, k/128].
 *  - Accumulation: the pages promote tensor-core partial sums to FP32 (part
 *    1.2, "CUDA-core two-level accumulation").  The oracle accumulates the
 *    exact products in double, k ascending, then rounds ONCE to BF16 with
 *    round-to-nearest-even (no float intermediate, so no double rounding).
 *  - NT layout, D = A B^T with both operands K-major: the project card,
 *    section "quick start", names the call fp8_gemm_nt(a, b, c, a_sf, b_sf).
 *  - Contiguous grouped layout: tokens of all experts concatenated along M,
 *    N and K fixed, one B per expert, m_indices[row] = expert or -1 for a
 *    padding row, which is left untouched (project card, "technical
 *    implementation": M-axis grouping, N/K fixed, contiguous layout).
 *  - Masked grouped layout: A[G, max_m, K]; only rows m < masked_m[g] of
 *    group g are computed, the others are left untouched (release article,
 *    part 4.2, names m_grouped_gemm_fp8_masked; project card, "core
 *    features": grouped GEMM, contiguous and masked layouts).  masked_m is
 *    clamped to [0, max_m].
 *  - K-grouped layout (the weight gradient of the grouped forms in
 *    training): see oracle_k_grouped_tn below.
 *
 * BF16 GEMM (same three forms, BF16 operands, no scales): the project card,
 * section "core features", lists BF16 beside FP8 and FP4 in its unified
 * dense GEMM family, and grouped GEMMs in contiguous and masked layouts for
 * MoE.  The plainest reading, taken here: D = A B^T with A [M,K] and B [N,K]
 * BF16 (K-major), every product exact in double, the sum in double, k
 * ascending, one rounding to BF16; the grouped forms index rows and groups
 * exactly as the FP8 ones do.  BF16 operands are decoded from the format
 * definition (1 sign, 8 exponent bits with bias 127, 7 mantissa bits;
 * exponent 0 is subnormal, 255 infinity or NaN) through a 65536-entry table.
 *
 * Parallelism: OpenMP over output rows only; every element is computed by
 * the same sequential loop, so the result does not depend on the thread
 * count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK_K 128
#define ORACLE_BLOCK_N 128

/* ---- E4M3 ("fn") decoding ------------------------------------------------ */

double oracle_e4m3_decode(uint8_t byte)
{
    int sign = (byte >> 7) & 1;
    int expo = (byte >> 3) & 0xF;
    int mant = byte & 0x7;
    double mag;
    if (expo == 0xF && mant == 0x7)
        return NAN;                              /* S.1111.111: the only NaN */
    if (expo == 0)
        mag = ldexp((double)mant, -9);           /* subnormal: m/8 * 2^(1-7) */
    else
        mag = ldexp(1.0 + mant / 8.0, expo - 7); /* normal: 1.m * 2^(e-7)     */
    return sign ? -mag : mag;
}

void oracle_e4m3_table(double *table256)
{
    for (int i = 0; i < 256; ++i)
        table256[i] = oracle_e4m3_decode((uint8_t)i);
}

/* ---- one rounding from double to BF16 (round to nearest, ties to even) ---- */

/* BF16: 1 sign, 8 exponent (bias 127), 7 stored mantissa bits; normal
 * numbers 1.f * 2^E for E in [-126, 127], subnormals k * 2^-133. */
uint16_t oracle_bf16_from_double(double x)
{
    if (isnan(x))
        return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    if (ax == 0.0)
        return sign;
    if (isinf(ax))
        return sign | 0x7F80;
    int e;
    frexp(ax, &e);                   /* ax = f * 2^e, f in [0.5, 1)        */
    int E = e - 1;                   /* ax = (2f) * 2^E, 2f in [1, 2)       */
    int q_exp = (E < -126) ? -133 : E - 7;  /* quantum: one unit in the last place */
    double n = ldexp(ax, -q_exp);    /* exact: scaling by a power of two    */
    double r = nearbyint(n);         /* default rounding mode: ties to even */
    double v = ldexp(r, q_exp);      /* the rounded magnitude               */
    if (v > ldexp(255.0, 120))       /* above the largest finite BF16       */
        return sign | 0x7F80;
    /* v is a BF16 value, hence exactly a float; its low 16 bits are zero */
    float fv = (float)v;
    uint32_t bits;
    memcpy(&bits, &fv, sizeof bits);
    return sign | (uint16_t)(bits >> 16);
}

/* ---- the GEMM definitions ------------------------------------------------- */

/* acc = sum_k A_hat[m,k] * B_hat[n,k] for one output element, k ascending. */
static double dot_row_col(const double *tab,
                          const uint8_t *a_row, const float *sfa_row,
                          const uint8_t *b_row, const float *sfb_nblock_row,
                          int64_t K)
{
    double s = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double ah = tab[a_row[k]] * (double)sfa_row[k / ORACLE_BLOCK_K];
        double bh = tab[b_row[k]] * (double)sfb_nblock_row[k / ORACLE_BLOCK_K];
        s += ah * bh;
    }
    return s;
}

/* One output row: D[m, 0:N] against one B[N, K] with its scales. */
static void gemm_row(const double *tab,
                     const uint8_t *a_row, const float *sfa_row,
                     const uint8_t *b, const float *sfb,
                     int64_t N, int64_t K,
                     double *acc_row, uint16_t *d_row)
{
    int64_t KB = K / ORACLE_BLOCK_K;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *b_row = b + n * K;
        const float *sfb_row = sfb + (n / ORACLE_BLOCK_N) * KB;
        double s = dot_row_col(tab, a_row, sfa_row, b_row, sfb_row, K);
        if (acc_row)
            acc_row[n] = s;
        if (d_row)
            d_row[n] = oracle_bf16_from_double(s);
    }
}

/* Dense NT: a [M,K] bytes, sfa [M, K/128], b [N,K] bytes, sfb [ceil(N/128), K/128].
 * acc [M,N] (double, may be NULL), d [M,N] (BF16 bits, may be NULL).
 * Returns 0, or -1 if K is not a multiple of 128. */
int oracle_gemm_nt(const uint8_t *a, const float *sfa, const uint8_t *b, const float *sfb,
                   int64_t M, int64_t N, int64_t K, double *acc, uint16_t *d)
{
    if (K % ORACLE_BLOCK_K != 0 || M < 0 || N < 0)
        return -1;
    double tab[256];
    oracle_e4m3_table(tab);
    int64_t KB = K / ORACLE_BLOCK_K;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        gemm_row(tab, a + m * K, sfa + m * KB, b, sfb, N, K,
                 acc ? acc + m * N : NULL, d ? d + m * N : NULL);
    return 0;
}

/* Contiguous grouped: a [M_sum,K], sfa [M_sum,K/128], b [G,N,K],
 * sfb [G, ceil(N/128), K/128], m_indices [M_sum].  A row whose index is -1
 * (any negative value) is padding: its D and acc rows are not written.
 * Returns 0, or -1 on bad sizes, or -2 if some index is >= G. */
int oracle_grouped_contiguous(const uint8_t *a, const float *sfa, const uint8_t *b,
                              const float *sfb, const int32_t *m_indices,
                              int64_t M_sum, int64_t N, int64_t K, int64_t G,
                              double *acc, uint16_t *d)
{
    if (K % ORACLE_BLOCK_K != 0 || M_sum < 0 || N < 0 || G < 0)
        return -1;
    for (int64_t r = 0; r < M_sum; ++r)
        if (m_indices[r] >= G)
            return -2;
    double tab[256];
    oracle_e4m3_table(tab);
    int64_t KB = K / ORACLE_BLOCK_K;
    int64_t NB = (N + ORACLE_BLOCK_N - 1) / ORACLE_BLOCK_N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M_sum; ++r) {
        int32_t e = m_indices[r];
        if (e < 0)
            continue;
        gemm_row(tab, a + r * K, sfa + r * KB, b + e * N * K, sfb + e * NB * KB, N, K,
                 acc ? acc + r * N : NULL, d ? d + r * N : NULL);
    }
    return 0;
}

/* Masked grouped: a [G,max_m,K], sfa [G,max_m,K/128], b [G,N,K],
 * sfb [G, ceil(N/128), K/128], masked_m [G].  Rows m >= clamp(masked_m[g],
 * 0, max_m) of group g are not written.  Returns 0 or -1 on bad sizes. */
int oracle_grouped_masked(const uint8_t *a, const float *sfa, const uint8_t *b,
                          const float *sfb, const int32_t *masked_m,
                          int64_t G, int64_t max_m, int64_t N, int64_t K,
                          double *acc, uint16_t *d)
{
    if (K % ORACLE_BLOCK_K != 0 || G < 0 || max_m < 0 || N < 0)
        return -1;
    double tab[256];
    oracle_e4m3_table(tab);
    int64_t KB = K / ORACLE_BLOCK_K;
    int64_t NB = (N + ORACLE_BLOCK_N - 1) / ORACLE_BLOCK_N;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t m = 0; m < max_m; ++m) {
            int64_t valid = masked_m[g] < 0 ? 0 : (masked_m[g] > max_m ? max_m : masked_m[g]);
            if (m >= valid)
                continue;
            int64_t r = g * max_m + m;
            gemm_row(tab, a + r * K, sfa + r * KB, b + g * N * K, sfb + g * NB * KB, N, K,
                     acc ? acc + r * N : NULL, d ? d + r * N : NULL);
        }
    }
    return 0;
}

/* ---- K-grouped form (MoE weight gradient) -------------------------------- */

/* The training backward pass of an M-grouped GEMM (project card, section
 * "core features": the unified GEMM family serves training forward and
 * backward, with NT / TN / NN / TT layouts on SM100) needs, per expert g,
 * the gradient of its weights: a GEMM whose reduction runs over that
 * expert's tokens only.  The tokens of all experts are concatenated along
 * the reduction axis ("K grouped"):
 *
 *   acc[g, m, n] = C[g, m, n] + sum_{k in K_g} A_hat[k, m] * B_hat[k, n],
 *   K_g = [k_off[g], k_off[g] + ks[g]),  k_off[g] = ks[0] + ... + ks[g-1],
 *
 * with A stored [K_sum, M] (M-major: one row per token) and B [K_sum, N]
 * (N-major), A_hat[k, m] = dec(a[k, m]) * sfa[m, k/128] (one scale per output
 * row per 128 tokens) and B_hat[k, n] = dec(b[k, n]) * sfb[n/128, k/128]
 * (128 x 128 blocks): the scale conventions of the dense call, with k the
 * global token index.  Every ks[g] is a multiple of 128 (each expert's
 * segment is padded as in the contiguous forward), so no scale block spans
 * two experts.  The sum runs k ascending in double; C may be NULL (zero).
 * Returns 0, -1 on bad sizes, -2 if the ks do not tile [0, K_sum) in
 * multiples of 128. */
int oracle_k_grouped_tn(const uint8_t *a, const float *sfa, const uint8_t *b, const float *sfb,
                        const int32_t *ks, const float *c, int64_t G, int64_t M, int64_t N,
                        int64_t K_sum, double *acc)
{
    if (K_sum % ORACLE_BLOCK_K != 0 || G < 0 || M < 0 || N < 0)
        return -1;
    int64_t total = 0;
    for (int64_t g = 0; g < G; ++g) {
        if (ks[g] < 0 || ks[g] % ORACLE_BLOCK_K != 0)
            return -2;
        total += ks[g];
    }
    if (total != K_sum)
        return -2;
    double tab[256];
    oracle_e4m3_table(tab);
    int64_t KB = K_sum / ORACLE_BLOCK_K;
    int64_t *k_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(G + 1));
    if (!k_off)
        return -1;
    k_off[0] = 0;
    for (int64_t g = 0; g < G; ++g)
        k_off[g + 1] = k_off[g] + ks[g];
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t m = 0; m < M; ++m) {
            for (int64_t n = 0; n < N; ++n) {
                double s = 0.0;
                for (int64_t k = k_off[g]; k < k_off[g + 1]; ++k) {
                    double ah = tab[a[k * M + m]] * (double)sfa[m * KB + k / ORACLE_BLOCK_K];
                    double bh = tab[b[k * N + n]] *
                                (double)sfb[(n / ORACLE_BLOCK_N) * KB + k / ORACLE_BLOCK_K];
                    s += ah * bh;
                }
                int64_t o = (g * M + m) * N + n;
                acc[o] = (c ? (double)c[o] : 0.0) + s;
            }
        }
    }
    free(k_off);
    return 0;
}

/* ---- BF16 operands -------------------------------------------------------- */

double oracle_bf16_decode(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 7) & 0xFF;
    int mant = bits & 0x7F;
    double mag;
    if (expo == 0xFF)
        mag = mant ? NAN : INFINITY;
    else if (expo == 0)
        mag = ldexp((double)mant, -133);              /* subnormal: m/128 * 2^-126 */
    else
        mag = ldexp(1.0 + mant / 128.0, expo - 127);  /* normal: 1.m * 2^(e-127)   */
    return sign ? -mag : mag;
}

/* One output row of the BF16 GEMM: D[m, 0:N] = bf16(sum_k A[m,k] * B[n,k]). */
static void bf16_gemm_row(const double *tab, const uint16_t *a_row, const uint16_t *b,
                          int64_t N, int64_t K, double *acc_row, uint16_t *d_row)
{
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *b_row = b + n * K;
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k)
            s += tab[a_row[k]] * tab[b_row[k]];
        if (acc_row)
            acc_row[n] = s;
        if (d_row)
            d_row[n] = oracle_bf16_from_double(s);
    }
}

static double *bf16_table(void)
{
    double *tab = (double *)malloc(65536 * sizeof(double));
    if (tab)
        for (int i = 0; i < 65536; ++i)
            tab[i] = oracle_bf16_decode((uint16_t)i);
    return tab;
}

/* Dense NT with BF16 operands: a [M,K], b [N,K] (BF16 bits); acc [M,N]
 * (double, may be NULL), d [M,N] (BF16 bits, may be NULL).  Returns 0, -1 on
 * bad sizes, -3 if out of memory. */
int oracle_bf16_gemm_nt(const uint16_t *a, const uint16_t *b, int64_t M, int64_t N, int64_t K,
                        double *acc, uint16_t *d)
{
    if (M < 0 || N < 0 || K < 0)
        return -1;
    double *tab = bf16_table();
    if (!tab)
        return -3;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        bf16_gemm_row(tab, a + m * K, b, N, K, acc ? acc + m * N : NULL, d ? d + m * N : NULL);
    free(tab);
    return 0;
}

/* Contiguous grouped, BF16 operands: a [M_sum,K], b [G,N,K], m_indices
 * [M_sum]; a negative index marks a padding row, left unwritten.  Returns 0,
 * -1 on bad sizes, -2 if some index is >= G, -3 if out of memory. */
int oracle_bf16_grouped_contiguous(const uint16_t *a, const uint16_t *b, const int32_t *m_indices,
                                   int64_t M_sum, int64_t N, int64_t K, int64_t G,
                                   double *acc, uint16_t *d)
{
    if (M_sum < 0 || N < 0 || K < 0 || G < 0)
        return -1;
    for (int64_t r = 0; r < M_sum; ++r)
        if (m_indices[r] >= G)
            return -2;
    double *tab = bf16_table();
    if (!tab)
        return -3;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M_sum; ++r) {
        int32_t e = m_indices[r];
        if (e < 0)
            continue;
        bf16_gemm_row(tab, a + r * K, b + e * N * K, N, K,
                      acc ? acc + r * N : NULL, d ? d + r * N : NULL);
    }
    free(tab);
    return 0;
}

/* Masked grouped, BF16 operands: a [G,max_m,K], b [G,N,K], masked_m [G];
 * rows m >= clamp(masked_m[g], 0, max_m) of group g are not written.
 * Returns 0, -1 on bad sizes, -3 if out of memory. */
int oracle_bf16_grouped_masked(const uint16_t *a, const uint16_t *b, const int32_t *masked_m,
                               int64_t G, int64_t max_m, int64_t N, int64_t K,
                               double *acc, uint16_t *d)
{
    if (G < 0 || max_m < 0 || N < 0 || K < 0)
        return -1;
    double *tab = bf16_table();
    if (!tab)
        return -3;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t m = 0; m < max_m; ++m) {
            int64_t valid = masked_m[g] < 0 ? 0 : (masked_m[g] > max_m ? max_m : masked_m[g]);
            if (m >= valid)
                continue;
            int64_t r = g * max_m + m;
            bf16_gemm_row(tab, a + r * K, b + g * N * K, N, K,
                          acc ? acc + r * N : NULL, d ? d + r * N : NULL);
        }
    }
    free(tab);
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
