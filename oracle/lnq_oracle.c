/*
 * lnq_oracle.c -- plain, slow, obviously correct CPU oracle for the
 * fine-grained block-scaled FP8 linear D = A . B^T and its M-grouped
 * contiguous MoE variant.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes, and where the pages define it:
 *
 *   - Activation quantization, one scale per 128 consecutive inputs of a row
 *     ("each 128 inputs of a row to FP8 with a scale of their own"):
 *     Linnet "Backend plugins", DeepGEMM plugin source, module docstring and
 *     _BlockProduct.execute; deepgemm-rust README, "What's implemented",
 *     fp8_gemm_nt row (per-(1x128) activation scales).
 *   - Scales stored column by column with the row count padded to a multiple
 *     of four (the scale columns 16-byte aligned): Linnet plugin docstring and
 *     the `padded = ceil4(rows)` line of _BlockProduct.execute.
 *   - Weight blocks of 128 x 128, one FP32 scale each, scale tensor of shape
 *     (ceil(n/128), ceil(k/128)): Linnet plugin docstring; deepgemm-rust
 *     README, "Quick start" (sfb shape).
 *   - The product with per-128-K-block FP32 promotion and BF16 output:
 *     deepgemm-rust README, "What's implemented" (DeepSeek recipe, FP32
 *     promotion, BF16 out).  The Linnet plugin docstring states that this and
 *     the generated block-scaled product differ only in summation order, so
 *     the oracle is the plain definition: dequantize both operands and
 *     accumulate in FP64.
 *   - M-grouped contiguous layout: tokens of all experts concatenated, each
 *     group starting at a 128-aligned row, a per-row group-id array, weights
 *     (G*n, k) and weight scales (G*ceil(n/128), ceil(k/128)): deepgemm-rust
 *     README, "Grouped (contiguous) MoE GEMM" and "What's implemented";
 *     Triton_Grouped_GEMM README, "Example DeepGEMM layout creation".
 *   - M-grouped masked layout (the per-expert output of a token dispatch):
 *     group g owns rows g*M_max .. g*M_max + M_max - 1 of A and D, of which
 *     only the first masked_m[g] are real; the counts stay on the device:
 *     deepgemm-rust README, "What's implemented", m_grouped_fp8_gemm_nt_masked
 *     (masked_m scheduler, DeepEP-style dispatch output, zero CPU sync).  The
 *     weights and their scales are laid out as in the contiguous variant.
 *   - M-grouped contiguous layout described by prefix sums: psum[g] is the
 *     number of tokens of groups 0..g, and group g's tokens start at the row
 *     sum_{j<g} align_up(count_j, alignment) of the A arena (alignment 128 or
 *     256): deepgemm-rust README, "The mk_alignment knob (MoE tile width)"
 *     (each group's tokens start at an aligned row) and the psum-layout
 *     contiguous entry point of the device-level API.
 *   - SiLU.mul after a gate_up linear: deepgemm-rust README, "What's
 *     implemented", moe_fp8_layer (grouped GEMM -> SiLU.mul -> grouped GEMM);
 *     silu(x) = x / (1 + e^-x), the sigmoid-weighted linear unit.
 *   - The UE8M0 recipe: the same groups and blocks with power-of-two scales
 *     stored as 8-bit exponents (value 2^(e - 127)), consumed by the
 *     tensor core's block-scaled MMA: deepgemm-rust README, "Blackwell-native
 *     FP4/FP8 (SM100a, tcgen05)" (UE8M0 power-of-two scales, block-scaled
 *     MMA) and "What's implemented" (gran-128 recipe on either side; FP32
 *     scales transformed into packed UE8M0).
 *   - E4M3 round-to-nearest-even with saturation at 448, scale = amax/448:
 *     the benchmark spec's numerics (the pages never print 448; the encoder
 *     below is written from the OCP FP8 E4M3 format definition: bias 7,
 *     3 mantissa bits, largest finite 448 = 0x7E, 0x7F/0xFF NaN, no
 *     infinities, subnormals k * 2^-9 for k = 1..7).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - the quotient is the correctly rounded FP32 x/s, then one E4M3 RNE
 *     rounding;
 *   - an all-zero group has scale 0.0f and codes 0x00 (0x80 for -0.0); no
 *     division is performed;
 *   - a negative value that rounds to zero keeps its sign (0x80);
 *   - magnitudes above 448 saturate to +-448 (0x7E / 0xFE);
 *   - pad scale entries (rows M..M4-1) are written as 0.0f;
 *   - grouped rows whose group id is negative contribute nothing and their
 *     output row is left untouched;
 *   - UE8M0 scale of a group or block: the smallest power of two p with
 *     448 * p >= amax (so no code saturates), exponent clamped to [-127, 127];
 *     an all-zero group gets p = 1 (byte 127); codes are the E4M3 RNE of x / p;
 *   - SiLU.mul: the gate_up weight stacks the I gate rows over the I up rows,
 *     and h[m][j] = silu(D[m][j]) * D[m][I + j] is taken of the product itself
 *     (before any BF16 rounding of D).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * x86-64 evaluates float arithmetic in SSE single precision
 * (FLT_EVAL_METHOD == 0), so `amax / 448.0f` and `x / s` below are single,
 * correctly rounded IEEE divisions.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 128 /* 1x128 activation groups, 128x128 weight blocks */

/* ------------------------------------------------------------------ */
/* bfloat16 -> float: the 16 bits are the top half of an IEEE binary32. */
static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* OCP FP8 E4M3 decode: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 is subnormal: m/8 * 2^(1-7) = m * 2^-9.
 * Otherwise (1 + m/8) * 2^(e-7).  S.1111.111 is NaN; there is no infinity. */
double oracle_e4m3_value(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* E4M3 encode of a binary32 value: round to nearest, ties to the even code
 * (mantissa LSB 0), magnitudes above 448 saturate to 448.  All arithmetic is
 * exact in double (t has a 24-bit significand). */
uint8_t oracle_e4m3_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a = fabs((double)t);
    int E;
    double f, scaled;
    int code;

    if (isnan(t))
        return (uint8_t)(sign | 0x7F); /* out of contract: inputs are finite */
    if (a > 448.0)
        return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range (and zero): the grid is k * 2^-9, k = 0..8;
         * k == 8 is the smallest normal 2^-6 = code 0x08. */
        double k = nearbyint(a * 512.0); /* default mode: ties to even */
        return (uint8_t)(sign | (uint8_t)k);
    }
    /* normal range: a = mant * 2^E with mant in [1, 2) */
    (void)frexp(a, &E);
    E -= 1;
    scaled = ldexp(a, -E);             /* mant, exact */
    f = nearbyint((scaled - 1.0) * 8.0); /* 3-bit mantissa, ties to even */
    if (f == 8.0) {
        E += 1;
        f = 0.0;
    }
    code = ((E + 7) << 3) | (int)f;
    if (code > 0x7E) /* would be the NaN pattern: saturate */
        code = 0x7E;
    return (uint8_t)(sign | code);
}

void oracle_e4m3_encode_array(const float* t, int64_t n, uint8_t* out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; ++i)
        out[i] = oracle_e4m3_encode(t[i]);
}

void oracle_e4m3_value_array(const uint8_t* c, int64_t n, double* out)
{
    int64_t i;
    for (i = 0; i < n; ++i)
        out[i] = oracle_e4m3_value(c[i]);
}

/* The quantization of one value given its group scale: the correctly rounded
 * binary32 quotient x/s, then E4M3 RNE with saturation.  An all-zero group
 * (s == 0) performs no division; the code keeps the sign of the zero. */
static uint8_t quantize_one(float x, float s)
{
    float t;
    if (s == 0.0f)
        t = x;
    else
        t = x / s;
    return oracle_e4m3_encode(t);
}

/* ------------------------------------------------------------------ */
/* Activation quantization, 1 x 128 groups.
 *   x    bf16 [M][ld_x]  (first K columns used)
 *   q    E4M3 [M][ld_q]
 *   sfa  fp32 [K/128][M4], sfa[g*M4 + m]; entries m in [M, M4) are 0.0f.
 * Returns 0 on success, -1 on a shape it does not take. */
int oracle_quantize_fp8_groups(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x,
                               uint8_t* q, int64_t ld_q, float* sfa, int64_t M4)
{
    int64_t G, m;
    if (M < 0 || K <= 0 || K % ORACLE_GROUP != 0 || M4 < M || ld_x < K || ld_q < K)
        return -1;
    G = K / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M4; ++m) {
        int64_t g, k;
        for (g = 0; g < G; ++g) {
            float amax = 0.0f, s;
            if (m < M) {
                for (k = 0; k < ORACLE_GROUP; ++k) {
                    float v = fabsf(bf16_bits_to_float(x[m * ld_x + g * ORACLE_GROUP + k]));
                    if (v > amax)
                        amax = v;
                }
            }
            s = amax / 448.0f;
            sfa[g * M4 + m] = s;
            if (m < M) {
                for (k = 0; k < ORACLE_GROUP; ++k) {
                    int64_t col = g * ORACLE_GROUP + k;
                    q[m * ld_q + col] = quantize_one(bf16_bits_to_float(x[m * ld_x + col]), s);
                }
            }
        }
    }
    return 0;
}

/* Weight quantization, 128 x 128 blocks.
 *   w    bf16 [N][K] row-major
 *   q    E4M3 [N][K]
 *   sfb  fp32 [ceil(N/128)][K/128] row-major, sfb[nb*KB + kb].
 * A ragged last row-block takes its amax over the rows that exist. */
int oracle_quantize_fp8_blocks(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* sfb)
{
    int64_t NB, KB, blk;
    if (N <= 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
    KB = K / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (blk = 0; blk < NB * KB; ++blk) {
        int64_t nb = blk / KB, kb = blk % KB;
        int64_t n0 = nb * ORACLE_GROUP, n1 = n0 + ORACLE_GROUP;
        int64_t n, k;
        float amax = 0.0f, s;
        if (n1 > N)
            n1 = N;
        for (n = n0; n < n1; ++n)
            for (k = kb * ORACLE_GROUP; k < (kb + 1) * ORACLE_GROUP; ++k) {
                float v = fabsf(bf16_bits_to_float(w[n * K + k]));
                if (v > amax)
                    amax = v;
            }
        s = amax / 448.0f;
        sfb[nb * KB + kb] = s;
        for (n = n0; n < n1; ++n)
            for (k = kb * ORACLE_GROUP; k < (kb + 1) * ORACLE_GROUP; ++k)
                q[n * K + k] = quantize_one(bf16_bits_to_float(w[n * K + k]), s);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Dequantized operands in FP64.  Each product value(q) * scale is exact in
 * double (4-bit by 24-bit significands). */
static void dequant_a_row(const uint8_t* qa, const float* sfa, int64_t M4, int64_t K,
                          int64_t m, double* out)
{
    int64_t k;
    for (k = 0; k < K; ++k)
        out[k] = oracle_e4m3_value(qa[m * K + k]) * (double)sfa[(k / ORACLE_GROUP) * M4 + m];
}

/* Row `row` of a weight matrix whose scale row for this row is `sb_row`. */
static void dequant_b_row(const uint8_t* qb, const float* sfb, int64_t K, int64_t row,
                          int64_t sb_row, double* out)
{
    int64_t k, KB = K / ORACLE_GROUP;
    for (k = 0; k < K; ++k)
        out[k] = oracle_e4m3_value(qb[row * K + k]) * (double)sfb[sb_row * KB + k / ORACLE_GROUP];
}

static double dot(const double* a, const double* b, int64_t K)
{
    double acc = 0.0;
    int64_t k;
    for (k = 0; k < K; ++k)
        acc += a[k] * b[k];
    return acc;
}

/* D[m][n] = sum_k (value(qa[m,k]) * sfa[k/128][m]) * (value(qb[n,k]) * sfb[n/128][k/128])
 * in FP64, for m < M, n < N.  D is [M][N] row-major doubles. */
int oracle_gemm_nt(const uint8_t* qa, const float* sfa, int64_t M4, const uint8_t* qb,
                   const float* sfb, int64_t M, int64_t N, int64_t K, double* D)
{
    double* bd;
    int64_t n, m;
    if (M <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || M4 < M)
        return -1;
    bd = (double*)malloc(sizeof(double) * (size_t)N * (size_t)K);
    if (!bd)
        return -2;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n)
        dequant_b_row(qb, sfb, K, n, n / ORACLE_GROUP, bd + n * K);
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
        for (m = 0; m < M; ++m) {
            int64_t j;
            if (!ad)
                continue;
            dequant_a_row(qa, sfa, M4, K, m, ad);
            for (j = 0; j < N; ++j)
                D[m * N + j] = dot(ad, bd + j * K, K);
        }
        free(ad);
    }
    free(bd);
    return 0;
}

/* The same sum at `count` chosen points (rows[i], cols[i]); out[i] = D[rows[i]][cols[i]].
 * Used where the whole product is too large for the CPU. */
int oracle_gemm_nt_points(const uint8_t* qa, const float* sfa, int64_t M4, const uint8_t* qb,
                          const float* sfb, int64_t M, int64_t N, int64_t K,
                          const int64_t* rows, const int64_t* cols, int64_t count, double* out)
{
    int64_t i;
    int bad = 0;
    if (M <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || M4 < M)
        return -1;
    for (i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M || cols[i] < 0 || cols[i] >= N)
            bad = 1;
    if (bad)
        return -1;
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
        double* bd = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 16)
        for (i = 0; i < count; ++i) {
            if (!ad || !bd)
                continue;
            dequant_a_row(qa, sfa, M4, K, rows[i], ad);
            dequant_b_row(qb, sfb, K, cols[i], cols[i] / ORACLE_GROUP, bd);
            out[i] = dot(ad, bd, K);
        }
        free(ad);
        free(bd);
    }
    return 0;
}

/* M-grouped contiguous product.  Row m of A belongs to group g = m_indices[m];
 * for g >= 0, D[m][n] = sum_k A~[m,k] * B~_g[n,k] where B~_g is rows
 * g*N .. g*N+N-1 of the dequantized weights, whose scale rows are
 * g*ceil(N/128) + n/128.  Rows with g < 0 are left untouched.
 *   qa [M_total][K], sfa [K/128][M_total], qb [G*N][K],
 *   sfb [G*ceil(N/128)][K/128], D [M_total][N]. */
int oracle_m_grouped_gemm_contiguous(const uint8_t* qa, const float* sfa, const uint8_t* qb,
                                     const float* sfb, const int32_t* m_indices, int32_t G,
                                     int64_t M_total, int64_t N, int64_t K, double* D)
{
    int64_t m, NB;
    if (M_total <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || G <= 0)
        return -1;
    for (m = 0; m < M_total; ++m)
        if (m_indices[m] >= G)
            return -1;
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
        double* bd = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
        for (m = 0; m < M_total; ++m) {
            int64_t n, g = m_indices[m];
            if (g < 0 || !ad || !bd)
                continue;
            dequant_a_row(qa, sfa, M_total, K, m, ad);
            for (n = 0; n < N; ++n) {
                dequant_b_row(qb, sfb, K, g * N + n, g * NB + n / ORACLE_GROUP, bd);
                D[m * N + n] = dot(ad, bd, K);
            }
        }
        free(ad);
        free(bd);
    }
    return 0;
}

/* Grouped product at chosen points; a point on a row with a negative group
 * id yields NaN. */
int oracle_m_grouped_gemm_points(const uint8_t* qa, const float* sfa, const uint8_t* qb,
                                 const float* sfb, const int32_t* m_indices, int32_t G,
                                 int64_t M_total, int64_t N, int64_t K, const int64_t* rows,
                                 const int64_t* cols, int64_t count, double* out)
{
    int64_t i, NB;
    int bad = 0;
    if (M_total <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || G <= 0)
        return -1;
    for (i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M_total || cols[i] < 0 || cols[i] >= N ||
            m_indices[rows[i]] >= G)
            bad = 1;
    if (bad)
        return -1;
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
        double* bd = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 16)
        for (i = 0; i < count; ++i) {
            int64_t g = m_indices[rows[i]], n = cols[i];
            if (!ad || !bd)
                continue;
            if (g < 0) {
                out[i] = NAN;
                continue;
            }
            dequant_a_row(qa, sfa, M_total, K, rows[i], ad);
            dequant_b_row(qb, sfb, K, g * N + n, g * NB + n / ORACLE_GROUP, bd);
            out[i] = dot(ad, bd, K);
        }
        free(ad);
        free(bd);
    }
    return 0;
}

/* M-grouped masked product: for each group g and each of its first masked_m[g]
 * rows m, D[g*M_max + m][n] = sum_k (value(qa[row,k]) * sfa[k/128][row]) *
 * (value(qb[g*N + n, k]) * sfb[g*ceil(N/128) + n/128][k/128]), row = g*M_max + m,
 * in FP64.  qa is [G*M_max][K]; sfa is [K/128][M4] over those G*M_max rows (M4 >=
 * G*M_max).  Rows past masked_m[g] are not written.  Returns -1 if a count lies
 * outside [0, M_max]. */
int oracle_m_grouped_gemm_masked(const uint8_t* qa, const float* sfa, int64_t M4, const uint8_t* qb,
                                 const float* sfb, const int32_t* masked_m, int32_t G, int64_t M_max,
                                 int64_t N, int64_t K, double* D)
{
    int64_t g, NB, total;
    if (G <= 0 || M_max <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || M4 < G * M_max)
        return -1;
    for (g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > M_max)
            return -1;
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
    total = G * M_max;
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
        double* bd = (double*)malloc(sizeof(double) * (size_t)K);
        int64_t r;
#pragma omp for schedule(dynamic, 1)
        for (r = 0; r < total; ++r) {
            int64_t n, gr = r / M_max, m = r % M_max;
            if (m >= masked_m[gr] || !ad || !bd)
                continue;
            dequant_a_row(qa, sfa, M4, K, r, ad);
            for (n = 0; n < N; ++n) {
                dequant_b_row(qb, sfb, K, gr * N + n, gr * NB + n / ORACLE_GROUP, bd);
                D[r * N + n] = dot(ad, bd, K);
            }
        }
        free(ad);
        free(bd);
    }
    return 0;
}

/* The masked product at chosen points (rows index the G*M_max rows); a point on a
 * row past its group's count yields NaN. */
int oracle_m_grouped_gemm_masked_points(const uint8_t* qa, const float* sfa, int64_t M4,
                                        const uint8_t* qb, const float* sfb,
                                        const int32_t* masked_m, int32_t G, int64_t M_max,
                                        int64_t N, int64_t K, const int64_t* rows,
                                        const int64_t* cols, int64_t count, double* out)
{
    int64_t i, g, NB;
    int bad = 0;
    if (G <= 0 || M_max <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || M4 < G * M_max)
        return -1;
    for (g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > M_max)
            return -1;
    for (i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= G * M_max || cols[i] < 0 || cols[i] >= N)
            bad = 1;
    if (bad)
        return -1;
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
        double* bd = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 16)
        for (i = 0; i < count; ++i) {
            int64_t gr = rows[i] / M_max, m = rows[i] % M_max, n = cols[i];
            if (!ad || !bd)
                continue;
            if (m >= masked_m[gr]) {
                out[i] = NAN;
                continue;
            }
            dequant_a_row(qa, sfa, M4, K, rows[i], ad);
            dequant_b_row(qb, sfb, K, gr * N + n, gr * NB + n / ORACLE_GROUP, bd);
            out[i] = dot(ad, bd, K);
        }
        free(ad);
        free(bd);
    }
    return 0;
}

/* M-grouped contiguous product with the prefix-sum layout: group g has
 * count_g = psum[g] - psum[g-1] tokens (psum[-1] = 0) at rows start_g ..
 * start_g + count_g - 1 of the arena, start_0 = 0, start_{g+1} = start_g +
 * align_up(count_g, alignment).  Those rows of D get the product with group g's
 * weights; every other row of D is left untouched.  qa is [M_total][K], sfa is
 * [K/128][M_total].  Returns -1 if psum decreases or the groups overrun M_total. */
int oracle_m_grouped_gemm_psum(const uint8_t* qa, const float* sfa, const uint8_t* qb,
                               const float* sfb, const int32_t* psum, int32_t G,
                               int64_t alignment, int64_t M_total, int64_t N, int64_t K, double* D)
{
    int64_t g, NB, start = 0, prev = 0;
    int64_t* first = NULL;
    int64_t* count = NULL;
    if (G <= 0 || M_total <= 0 || N <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || alignment <= 0)
        return -1;
    first = (int64_t*)malloc(sizeof(int64_t) * (size_t)G);
    count = (int64_t*)malloc(sizeof(int64_t) * (size_t)G);
    if (!first || !count) {
        free(first);
        free(count);
        return -2;
    }
    for (g = 0; g < G; ++g) {
        const int64_t c = (int64_t)psum[g] - prev;
        if (c < 0) {
            free(first);
            free(count);
            return -1;
        }
        first[g] = start;
        count[g] = c;
        start += (c + alignment - 1) / alignment * alignment;
        prev = psum[g];
    }
    if (start > M_total) {
        free(first);
        free(count);
        return -1;
    }
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
    for (g = 0; g < G; ++g) {
        int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
        for (i = 0; i < count[g]; ++i) {
            int64_t n, row = first[g] + i;
            double* ad = (double*)malloc(sizeof(double) * (size_t)K);
            double* bd = (double*)malloc(sizeof(double) * (size_t)K);
            if (ad && bd) {
                dequant_a_row(qa, sfa, M_total, K, row, ad);
                for (n = 0; n < N; ++n) {
                    dequant_b_row(qb, sfb, K, g * N + n, g * NB + n / ORACLE_GROUP, bd);
                    D[row * N + n] = dot(ad, bd, K);
                }
            }
            free(ad);
            free(bd);
        }
    }
    free(first);
    free(count);
    return 0;
}

/* SiLU.mul of n gate/up pairs: h[i] = silu(g[i]) * u[i], silu(x) = x / (1 + e^-x)
 * in FP64.  For x below about -709, e^-x overflows to infinity and x / inf gives
 * -0.0, which is silu's limit there. */
void oracle_silu_mul(const double* g, const double* u, int64_t n, double* h)
{
    int64_t i;
    for (i = 0; i < n; ++i)
        h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
}

/* UE8M0 recipe: the exponent e of the smallest power of two with 448 * 2^e >= amax,
 * clamped to [-127, 127]; 0 for amax == 0.  Every comparison is exact in double. */
static int ue8m0_exponent(float amax)
{
    int e;
    if (!(amax > 0.0f))
        return 0;
    (void)frexp((double)amax, &e);     /* amax < 2^e, so 448 * 2^(e - 8) > amax */
    e -= 10;
    while (ldexp(448.0, e) < (double)amax)
        ++e;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* E4M3 code of x / 2^e (the division by a power of two is exact). */
static uint8_t quantize_pow2(float x, int e)
{
    return oracle_e4m3_encode((float)ldexp((double)x, -e));
}

/* UE8M0 activation quantization, 1 x 128 groups.
 *   x    bf16 [M][ld_x];  q  E4M3 [M][ld_q];
 *   sfe  uint8 [K/128][M], sfe[g*M + m] = e + 127 of row m's group g. */
int oracle_quantize_ue8m0_groups(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x,
                                 uint8_t* q, int64_t ld_q, uint8_t* sfe)
{
    int64_t G, m;
    if (M <= 0 || K <= 0 || K % ORACLE_GROUP != 0 || ld_x < K || ld_q < K)
        return -1;
    G = K / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (m = 0; m < M; ++m) {
        int64_t g, k;
        for (g = 0; g < G; ++g) {
            float amax = 0.0f;
            int e;
            for (k = 0; k < ORACLE_GROUP; ++k) {
                float v = fabsf(bf16_bits_to_float(x[m * ld_x + g * ORACLE_GROUP + k]));
                if (v > amax)
                    amax = v;
            }
            e = ue8m0_exponent(amax);
            sfe[g * M + m] = (uint8_t)(e + 127);
            for (k = 0; k < ORACLE_GROUP; ++k) {
                int64_t col = g * ORACLE_GROUP + k;
                q[m * ld_q + col] = quantize_pow2(bf16_bits_to_float(x[m * ld_x + col]), e);
            }
        }
    }
    return 0;
}

/* UE8M0 weight quantization, 128 x 128 blocks (a ragged last row block takes its
 * amax over the rows that exist).  sfe uint8 [ceil(N/128)][K/128]. */
int oracle_quantize_ue8m0_blocks(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, uint8_t* sfe)
{
    int64_t NB, KB, blk;
    if (N <= 0 || K <= 0 || K % ORACLE_GROUP != 0)
        return -1;
    NB = (N + ORACLE_GROUP - 1) / ORACLE_GROUP;
    KB = K / ORACLE_GROUP;
#pragma omp parallel for schedule(static)
    for (blk = 0; blk < NB * KB; ++blk) {
        int64_t nb = blk / KB, kb = blk % KB;
        int64_t n0 = nb * ORACLE_GROUP, n1 = n0 + ORACLE_GROUP;
        int64_t n, k;
        float amax = 0.0f;
        int e;
        if (n1 > N)
            n1 = N;
        for (n = n0; n < n1; ++n)
            for (k = kb * ORACLE_GROUP; k < (kb + 1) * ORACLE_GROUP; ++k) {
                float v = fabsf(bf16_bits_to_float(w[n * K + k]));
                if (v > amax)
                    amax = v;
            }
        e = ue8m0_exponent(amax);
        sfe[nb * KB + kb] = (uint8_t)(e + 127);
        for (n = n0; n < n1; ++n)
            for (k = kb * ORACLE_GROUP; k < (kb + 1) * ORACLE_GROUP; ++k)
                q[n * K + k] = quantize_pow2(bf16_bits_to_float(w[n * K + k]), e);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MXFP8 gran-32 (deepgemm-rust README, benchmark block "SM100 FP8: DeepSeek gran-128
 * recipe and MXFP8 gran-32"; kernel table, kind::mxf8f6f4): every row of an operand,
 * activations and weights alike, in 1 x 32 blocks along K, each block with its own
 * UE8M0 scale chosen by the rule of the gran-128 recipe above (the smallest power of two
 * p with 448 p >= amax; p = 1 for an all-zero block), codes the E4M3 RNE of x / p.
 *   x    bf16 [R][ld_x];  q  E4M3 [R][ld_q];
 *   sfe  uint8 [R][K/32], sfe[r*(K/32) + b] = e + 127 of row r's block b. */
#define ORACLE_MX_BLOCK 32

int oracle_quantize_mxfp8(const uint16_t* x, int64_t R, int64_t K, int64_t ld_x, uint8_t* q, int64_t ld_q,
                          uint8_t* sfe)
{
    int64_t B, r;
    if (R <= 0 || K <= 0 || K % ORACLE_MX_BLOCK != 0 || ld_x < K || ld_q < K)
        return -1;
    B = K / ORACLE_MX_BLOCK;
#pragma omp parallel for schedule(static)
    for (r = 0; r < R; ++r) {
        int64_t b, k;
        for (b = 0; b < B; ++b) {
            float amax = 0.0f;
            int e;
            for (k = 0; k < ORACLE_MX_BLOCK; ++k) {
                float v = fabsf(bf16_bits_to_float(x[r * ld_x + b * ORACLE_MX_BLOCK + k]));
                if (v > amax)
                    amax = v;
            }
            e = ue8m0_exponent(amax);
            sfe[r * B + b] = (uint8_t)(e + 127);
            for (k = 0; k < ORACLE_MX_BLOCK; ++k) {
                int64_t col = b * ORACLE_MX_BLOCK + k;
                q[r * ld_q + col] = quantize_pow2(bf16_bits_to_float(x[r * ld_x + col]), e);
            }
        }
    }
    return 0;
}

/* D[m][n] = sum_k (value(qa[m][k]) * 2^(ea[m][k/32] - 127)) * (value(qb[n][k]) * 2^(eb[n][k/32] - 127))
 * in FP64 (each term exact), for qa [M][K], ea [M][K/32], qb [N][K], eb [N][K/32]; D [M][N]. */
int oracle_gemm_nt_mx32(const uint8_t* qa, const uint8_t* ea, const uint8_t* qb, const uint8_t* eb, int64_t M,
                        int64_t N, int64_t K, double* D)
{
    double* bd;
    int64_t n, m, B;
    if (M <= 0 || N <= 0 || K <= 0 || K % ORACLE_MX_BLOCK != 0)
        return -1;
    B = K / ORACLE_MX_BLOCK;
    bd = (double*)malloc(sizeof(double) * (size_t)N * (size_t)K);
    if (!bd)
        return -2;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        int64_t k;
        for (k = 0; k < K; ++k)
            bd[n * K + k] = oracle_e4m3_value(qb[n * K + k]) * ldexp(1.0, (int)eb[n * B + k / ORACLE_MX_BLOCK] - 127);
    }
#pragma omp parallel
    {
        double* ad = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
        for (m = 0; m < M; ++m) {
            int64_t j, k;
            if (!ad)
                continue;
            for (k = 0; k < K; ++k)
                ad[k] = oracle_e4m3_value(qa[m * K + k]) * ldexp(1.0, (int)ea[m * B + k / ORACLE_MX_BLOCK] - 127);
            for (j = 0; j < N; ++j)
                D[m * N + j] = dot(ad, bd + j * K, K);
        }
        free(ad);
    }
    free(bd);
    return 0;
}
