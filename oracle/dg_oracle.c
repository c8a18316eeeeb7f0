/*
 * dg_oracle.c -- CPU oracle for the FP8 block-scaled NT GEMM (TEST INFRASTRUCTURE).
 *
 * This file is test infrastructure only.  It is compiled into liboracle.so and
 * loaded by the tests, by __graft_entry__.smoke() and by bench.py's CPU-baseline
 * leg.  The product path (include/dg.h, the CUDA library) never links, loads or
 * calls it, and it shares no code, header, table or constant with that path.
 *
 * What it computes.  The page "DeepGEMM项目介绍与本地部署指南" (DeepGEMM project
 * introduction and local deployment guide), section "接口" (Interface), fixes the
 * NT layout and the transposed LHS scales; the page "Deepseek DeepGEMM 技术原理的
 * 深入分析" (in-depth analysis of DeepGEMM's technical principles), section
 * "技术背景与核心原理" (technical background and core principles), fixes the
 * 1x128 activation / 128x128 weight scale granularity and the promotion
 * interval N_C = 128:
 *
 *   D[m,n] = bf16_rne( sum_kb  sa[m,kb] * sb[n/128,kb] * P_kb[m,n] )
 *   P_kb[m,n] = sum_{k = 128*kb}^{min(K,128*kb+128)-1}  A[m,k] * B[n,k]
 *
 * A is e4m3 [M,K] with K contiguous (LHS not transposed), B is e4m3 [N,K]
 * with K contiguous (RHS transposed), sa holds one FP32 scale per 1x128 row tile of A and is stored
 * transposed (column-major, sa[kb*sa_stride + m]), sb holds one FP32 scale per
 * 128x128 block of B (sb[nb*nkb + kb]).  D is bf16 [M,N] row-major.
 *
 * Arithmetic: every product and every 128-term block sum is done in IEEE
 * double.  A product of two e4m3 values is an integer multiple of 2^-18 with
 * magnitude <= 448^2 < 2^18, so a 128-term block sum is below 2^25 and needs
 * fewer than 43 significant bits: the FP64 block dot is EXACT.  The scales are
 * then applied in double, the blocks summed in double, and the result rounded
 * once, directly from double to bf16 with round-to-nearest-even.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - "FP8" is OCP E4M3FN: sign, 4 exponent bits with bias 7, 3 mantissa bits,
 *    no infinities, codes 0x7F/0xFF are NaN, largest finite value 448.
 *  - K % 128 != 0: the last K block is zero-extended and uses scale column
 *    ceil(K/128)-1.
 *  - N % 128 != 0: column n uses sb row floor(n/128); sb has ceil(N/128) rows.
 *  - Overflow rounds to +-Inf, NaN propagates.
 *  - Grouped contiguous (section "分组 GEMM（连续布局）"): m_indices[m] = g uses
 *    B[g], sb[g]; -1 marks a padding row, which is left untouched; any other
 *    value is invalid input.
 *  - Grouped masked (section "分组 GEMM（掩码布局）"): rows m < masked_m[g] of
 *    group g are computed, the rest are untouched; masked_m outside [0, Mmax]
 *    is invalid input.
 *
 * Alongside D the oracle can return D64 (the double value before rounding) and
 * MAG = sum_k |sa*sb*A[m,k]*B[n,k]|, the magnitude that scales the tolerance
 * |D_gpu - D_ref| <= 2^-7 |D_ref| + 1e-4 * MAG.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DGO_OK 0
#define DGO_BAD_ARG 1
#define DGO_BAD_INDEX 2

/* ---------------------------------------------------------------- e4m3 ---- */

/* Decode one OCP E4M3FN code from its bit fields.
 *   exponent field 0      : subnormal, value = mantissa * 2^-9  (= m/8 * 2^(1-7))
 *   exponent field 1..15  : value = (1 + m/8) * 2^(e-7)
 *   exponent 15, m = 7    : NaN (E4M3FN has no infinities)                  */
double dgo_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

static double g_e4m3[256];
static int g_e4m3_ready = 0;

static void e4m3_table_init(void) {
    if (g_e4m3_ready) return;
    for (int c = 0; c < 256; ++c) g_e4m3[c] = dgo_e4m3_decode((uint8_t)c);
    g_e4m3_ready = 1;
}

void dgo_e4m3_table(double* out256) {
    e4m3_table_init();
    memcpy(out256, g_e4m3, sizeof(g_e4m3));
}

/* ---------------------------------------------------------------- bf16 ---- */

/* Round a double to bf16 (1 sign, 8 exponent bits with bias 127, 7 stored
 * mantissa bits) with round-to-nearest, ties-to-even, in one step.
 * Normal bf16 values in [2^(e-1), 2^e) are spaced 2^(e-8); below 2^-126 the
 * spacing stays at the subnormal step 2^-133.  Values that round to 2^128 or
 * beyond become infinity.                                                    */
uint16_t dgo_bf16_rne(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    double ax = fabs(x);
    if (ax == 0.0) return sign;
    if (isinf(ax)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(ax, &e);                       /* ax in [2^(e-1), 2^e) */
    if (e > 129) return (uint16_t)(sign | 0x7F80u);
    int q = e - 8;                       /* exponent of the spacing */
    if (q < -133) q = -133;
    double s = ldexp(ax, -q);            /* exact: scaling by a power of two */
    double fl = floor(s);
    double frac = s - fl;                /* exact */
    double r;
    if (frac > 0.5)
        r = fl + 1.0;
    else if (frac < 0.5)
        r = fl;
    else
        r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double v = ldexp(r, q);
    if (v >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    /* v has at most 8 significant bits and lies in the float range, so it is
     * an exact float whose low 16 bits are zero: its top half is the bf16. */
    float f = (float)v;
    uint32_t bits;
    memcpy(&bits, &f, 4);
    return (uint16_t)(sign | (uint16_t)(bits >> 16));
}

double dgo_bf16_to_double(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

void dgo_bf16_rne_array(const double* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = dgo_bf16_rne(x[i]);
}

/* ---------------------------------------------------------- one row ------- */

/* One output row m of the scaled NT GEMM against one group's B and sb.
 *   a     : A row m (K codes)
 *   sa_m  : sa for row m, element kb at sa_m[kb * sa_stride]
 *   b     : B of the group, b[n*K + k]
 *   sb    : sb of the group, sb[nb*nkb + kb]
 * Writes D row (bf16 bits) and, when given, D64 and MAG rows.               */
static void gemm_row(const uint8_t* a, const float* sa_m, int64_t sa_stride,
                     const uint8_t* b, const float* sb, int N, int K,
                     uint16_t* d, double* d64, double* mag) {
    int nkb = (K + 127) / 128;
    for (int n = 0; n < N; ++n) {
        const uint8_t* bn = b + (int64_t)n * K;
        int nb = n / 128;
        double acc = 0.0, acc_mag = 0.0;
        for (int kb = 0; kb < nkb; ++kb) {
            int k0 = kb * 128;
            int k1 = k0 + 128 < K ? k0 + 128 : K;
            double p = 0.0, pmag = 0.0;
            for (int k = k0; k < k1; ++k) {
                double t = g_e4m3[a[k]] * g_e4m3[bn[k]];
                p += t;
                pmag += fabs(t);
            }
            double s = (double)sa_m[(int64_t)kb * sa_stride] * (double)sb[(int64_t)nb * nkb + kb];
            acc += s * p;
            acc_mag += fabs(s) * pmag;
        }
        d[n] = dgo_bf16_rne(acc);
        if (d64) d64[n] = acc;
        if (mag) mag[n] = acc_mag;
    }
}

/* ------------------------------------------------------------ dense ------- */

/* Dense D[M,N] = scaled A[M,K] . B[N,K]^T.
 *   rows/nrows : optional list of rows to compute (NULL: all M rows).  Only
 *                those rows of D/D64/MAG are written.
 *   d64, mag   : optional, same [M,N] layout as D.                          */
int dgo_gemm_nt(const uint8_t* A, const float* sa, int64_t sa_stride,
                const uint8_t* B, const float* sb,
                int M, int N, int K,
                const int64_t* rows, int64_t nrows,
                uint16_t* D, double* D64, double* MAG) {
    if (M < 0 || N < 0 || K < 0 || sa_stride < M) return DGO_BAD_ARG;
    e4m3_table_init();
    int64_t cnt = rows ? nrows : M;
    for (int64_t i = 0; i < cnt; ++i)
        if (rows && (rows[i] < 0 || rows[i] >= M)) return DGO_BAD_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < cnt; ++i) {
        int64_t m = rows ? rows[i] : i;
        gemm_row(A + m * K, sa + m, sa_stride, B, sb, N, K,
                 D + m * N, D64 ? D64 + m * N : NULL, MAG ? MAG + m * N : NULL);
    }
    return DGO_OK;
}

/* ------------------------------------------------ grouped, contiguous ----- */

/* Grouped GEMM with the contiguous layout: the rows of all groups are
 * concatenated along M; m_indices[m] names the group of row m (B[g] is
 * B + g*N*K, sb[g] is sb + g*ceil(N/128)*ceil(K/128)); -1 marks a padding row
 * that is left untouched.  Returns DGO_BAD_INDEX for any other value outside
 * [0, G).                                                                    */
int dgo_grouped_contiguous(const uint8_t* A, const float* sa, int64_t sa_stride,
                           const uint8_t* B, const float* sb,
                           const int32_t* m_indices, int M, int N, int K, int G,
                           const int64_t* rows, int64_t nrows,
                           uint16_t* D, double* D64, double* MAG) {
    if (M < 0 || N < 0 || K < 0 || G <= 0 || sa_stride < M) return DGO_BAD_ARG;
    e4m3_table_init();
    int64_t cnt = rows ? nrows : M;
    int nkb = (K + 127) / 128, nbn = (N + 127) / 128;
    for (int64_t i = 0; i < cnt; ++i) {
        int64_t m = rows ? rows[i] : i;
        if (m < 0 || m >= M) return DGO_BAD_ARG;
        if (m_indices[m] < -1 || m_indices[m] >= G) return DGO_BAD_INDEX;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < cnt; ++i) {
        int64_t m = rows ? rows[i] : i;
        int g = m_indices[m];
        if (g < 0) continue;
        gemm_row(A + m * K, sa + m, sa_stride,
                 B + (int64_t)g * N * K, sb + (int64_t)g * nbn * nkb, N, K,
                 D + m * N, D64 ? D64 + m * N : NULL, MAG ? MAG + m * N : NULL);
    }
    return DGO_OK;
}

/* --------------------------------------------------- grouped, masked ------ */

/* Grouped GEMM with the masked layout: A is [G, Mmax, K], D is [G, Mmax, N],
 * sa is [G][ceil(K/128)][sa_stride] (sa_stride >= Mmax), B and sb as above.
 * In group g only rows m < masked_m[g] are computed; the other rows of D are
 * left untouched.  masked_m outside [0, Mmax] returns DGO_BAD_INDEX.
 * rows/nrows, when given, list flat row indices g*Mmax + m to compute (rows
 * at or beyond masked_m[g] in that list are skipped).                       */
int dgo_grouped_masked(const uint8_t* A, const float* sa, int64_t sa_stride,
                       const uint8_t* B, const float* sb,
                       const int32_t* masked_m, int G, int Mmax, int N, int K,
                       const int64_t* rows, int64_t nrows,
                       uint16_t* D, double* D64, double* MAG) {
    if (G <= 0 || Mmax < 0 || N < 0 || K < 0 || sa_stride < Mmax) return DGO_BAD_ARG;
    e4m3_table_init();
    int nkb = (K + 127) / 128, nbn = (N + 127) / 128;
    for (int g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > Mmax) return DGO_BAD_INDEX;
    int64_t cnt = rows ? nrows : (int64_t)G * Mmax;
    for (int64_t i = 0; i < cnt; ++i)
        if (rows && (rows[i] < 0 || rows[i] >= (int64_t)G * Mmax)) return DGO_BAD_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < cnt; ++i) {
        int64_t flat = rows ? rows[i] : i;
        int g = (int)(flat / Mmax);
        int m = (int)(flat % Mmax);
        if (m >= masked_m[g]) continue;
        const uint8_t* a = A + flat * K;
        const float* sa_m = sa + (int64_t)g * nkb * sa_stride + m;
        gemm_row(a, sa_m, sa_stride, B + (int64_t)g * N * K, sb + (int64_t)g * nbn * nkb, N, K,
                 D + flat * N, D64 ? D64 + flat * N : NULL, MAG ? MAG + flat * N : NULL);
    }
    return DGO_OK;
}

/* Number of OpenMP threads the oracle's parallel loops use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int dgo_num_threads(void) { return omp_get_max_threads(); }
#else
int dgo_num_threads(void) { return 1; }
#endif

/* ------------------------------------------------------- FP8 cast ---- */
/*
 * The cast that produces the GEMM's FP8 operands and their scales.  The pages
 * leave it to the caller: "DeepGEMM项目介绍与本地部署指南", section "接口"
 * (Interface), asks for e4m3 inputs with transposed, TMA-aligned LHS scales;
 * the later-version article (yfxerp.com), section 4.1, calls a helper
 * to_fp8 that returns the FP8 tensor and its scale factors; the page "Deepseek
 * DeepGEMM 技术原理的深入分析", section "技术背景与核心原理", fixes one scale
 * per 1x128 activation tile and per 128x128 weight block.  Reading taken here,
 * every step in IEEE single precision (the kernel takes each decision in the
 * same precision, so the codes compare bit for bit):
 *
 *   amax = max(max over the tile of |x|, 1e-4)   (fmaxf: a NaN is skipped)
 *   s    = amax / 448            the stored scale (sa or sb)
 *   r    = 448 / amax
 *   q    = e4m3_rne_satfinite(x * r)
 *
 * so that s * decode(q) ~ x and the largest |x| of a tile maps to 448.  The
 * floor 1e-4 keeps an all-zero tile finite.  x is bf16.
 */

/* e4m3 code of a float: round to nearest, ties to even, from the bit layout
 * above.  |x| >= 448 (infinities included) saturates to +-448; NaN gives 0x7F.
 * Binade [2^E, 2^(E+1)) with E >= -6 is spaced 2^(E-3); below 2^-6 the
 * subnormal spacing 2^-9 applies.                                           */
uint8_t dgo_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E); /* a = f * 2^E, f in [0.5, 1): a in [2^(E-1), 2^E) */
    E -= 1;
    if (E < -6) E = -6;
    const double ulp = ldexp(1.0, E - 3);
    const double q = a / ulp; /* exact: division by a power of two */
    double f = floor(q);
    const double rem = q - f;
    if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) == 1.0)) f += 1.0;
    const double v = f * ulp; /* <= 448: every a < 448 rounds to at most 448 */
    if (v < ldexp(1.0, -6)) return sign | (uint8_t)(v / ldexp(1.0, -9)); /* subnormal */
    int E2;
    frexp(v, &E2);
    E2 -= 1; /* v may have rounded up into the next binade */
    const int mant = (int)((v / ldexp(1.0, E2) - 1.0) * 8.0);
    return sign | (uint8_t)(((E2 + 7) << 3) | mant);
}

static float bf16_bits_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* One tile: rows [r0, r1) x columns [c0, c0+128) of a row-major bf16 [.][K]. */
static void cast_tile(const uint16_t* X, int64_t K, int r0, int r1, int c0, uint8_t* Q, float* s_out) {
    float amax = 0.0f;
    for (int r = r0; r < r1; ++r)
        for (int k = c0; k < c0 + 128; ++k) amax = fmaxf(amax, fabsf(bf16_bits_to_float(X[r * K + k])));
    amax = fmaxf(amax, 1e-4f);
    const float s = amax / 448.0f;
    const float rcp = 448.0f / amax;
    *s_out = s;
    for (int r = r0; r < r1; ++r)
        for (int k = c0; k < c0 + 128; ++k) {
            const float y = bf16_bits_to_float(X[r * K + k]) * rcp;
            Q[r * K + k] = dgo_e4m3_encode(y);
        }
}

/* Activations: X bf16 [M][K] -> Q e4m3 [M][K], sa[kb*sa_stride + m] (the
 * GEMM's transposed layout).  K % 128 == 0, sa_stride >= M.                */
int dgo_cast_1x128(const uint16_t* X, int M, int K, uint8_t* Q, float* sa, int64_t sa_stride) {
    if (M < 0 || K <= 0 || K % 128 != 0 || sa_stride < M || !X || !Q || !sa) return DGO_BAD_ARG;
    const int nkb = K / 128;
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int kb = 0; kb < nkb; ++kb) cast_tile(X, K, m, m + 1, kb * 128, Q, sa + (int64_t)kb * sa_stride + m);
    return DGO_OK;
}

/* Weights: W bf16 [N][K] -> Q e4m3 [N][K], sb[nb*nkb + kb] with one scale per
 * 128x128 block (the last row block may be shorter).  K % 128 == 0.        */
int dgo_cast_128x128(const uint16_t* W, int N, int K, uint8_t* Q, float* sb) {
    if (N < 0 || K <= 0 || K % 128 != 0 || !W || !Q || !sb) return DGO_BAD_ARG;
    const int nkb = K / 128, nbn = (N + 127) / 128;
#pragma omp parallel for schedule(static)
    for (int nb = 0; nb < nbn; ++nb) {
        const int r1 = (nb + 1) * 128 < N ? (nb + 1) * 128 : N;
        for (int kb = 0; kb < nkb; ++kb) cast_tile(W, K, nb * 128, r1, kb * 128, Q, sb + (int64_t)nb * nkb + kb);
    }
    return DGO_OK;
}

void dgo_e4m3_encode_array(const float* x, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = dgo_e4m3_encode(x[i]);
}
