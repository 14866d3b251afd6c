/*
 * fp8q_oracle.c -- plain, slow CPU oracle for fine-grained FP8 quantisation and the
 * block-scaled FP8 GEMM of DeepSeek-V3's linear layers.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark may load this library.  It shares no code, header, table or helper with the
 * CUDA path, and the CUDA path never calls it.
 *
 * Sources (pages on the DeepSeek-V3 Technical Report, arXiv 2412.19437):
 *   [SUMMARY]  "DeepSeek-V3 Technical Report" summary page (xyznot.com), Key ideas, FP8
 *              mixed-precision bullet, and Questions, the answer on training FP8 without
 *              divergence: all tensors use E4M3; activations are scaled per 1x128 tile, weights
 *              per 128x128 block; every N_c = 128 elements the tensor-core partial sum is copied
 *              to FP32 registers on the CUDA cores.
 *   [REPOST]   DeepSeek-V3 report repost (why-be.co.kr board post): paragraph 1 (128 elements,
 *              i.e. 4 WGMMAs, is the promotion interval; weight gradients kept in higher
 *              precision), paragraph 2 (Fprop, Dgrad and Wgrad all run in FP8, Figure 6),
 *              paragraph 3 (gradients kept in FP32), paragraph 4 (per-group scaling factors
 *              along the inner dimension of the GEMM, dequantisation folded into the
 *              increased-precision accumulation, Figure 7(b)).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - E4M3 is the OCP E4M3FN format: bias 7, no infinities, largest finite 448 (0x7E),
 *     NaN 0x7F/0xFF, subnormals m * 2^-9.
 *   - Encoding rounds to nearest, ties to even, and saturates finite values above 448 to 448.
 *   - Scale of a group: a = max(max|x|, 2^-100); s = a / 448 (stored, the dequantisation
 *     multiplier); codes are E4M3(x * (448 / a)).  Both divisions and the multiply are single
 *     IEEE binary32 operations rounded to nearest.
 *   - The GEMM result is the exact dot product of the dequantised operands, accumulated here in
 *     binary64 (each dequantised value dec(q)*s is exact in binary64).
 *   - Power-of-two (UE8M0) scale variant, a separate mode that the pages do not describe (it is
 *     the scale format the block-scaled tensor-core MMA accepts): s is the smallest power of two
 *     not below the binary32 quotient a / 448, and codes are E4M3(x * (1 / s)), where 1 / s is an
 *     exact power of two.  The default mode is the one above.
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * No FMA contraction and no excess precision: every float operation below is one IEEE
 * binary32 operation.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------------------------ */
/* E4M3 codec                                                                                  */
/* ------------------------------------------------------------------------------------------ */

/* Encode one binary32 value as an E4M3FN byte: round to nearest even on the dropped significand
 * bits (integer arithmetic on the binary32 bit pattern, so there is exactly one rounding), and
 * saturate every finite magnitude above 448 to 448.  NaN maps to 0x7F with its sign. */
uint8_t oracle_e4m3_encode(float f)
{
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    const uint8_t sign = (bits >> 31) ? 0x80u : 0x00u;
    const uint32_t mag = bits & 0x7FFFFFFFu;

    if (mag > 0x7F800000u) return (uint8_t)(sign | 0x7Fu);   /* NaN */
    if (mag > 0x43E00000u) return (uint8_t)(sign | 0x7Eu);   /* |f| > 448 (and inf): saturate */

    /* |f| = sig * 2^(e - 23) with sig the 24-bit significand including the hidden bit. */
    int e = (int)(mag >> 23) - 127;
    uint32_t sig = mag & 0x7FFFFFu;
    if (e == -127) {
        e = -126;                       /* binary32 subnormal: no hidden bit */
    } else {
        sig |= 0x800000u;
    }

    if (e >= -6) {
        /* Normal E4M3 range: keep the hidden bit and 3 fraction bits (drop 20 bits). */
        uint32_t q = sig >> 20;                 /* in [8, 15] */
        const uint32_t rem = sig & 0xFFFFFu;
        const uint32_t half = 0x80000u;
        if (rem > half || (rem == half && (q & 1u))) q += 1u;
        if (q == 16u) {                         /* rounded up to the next binade */
            q = 8u;
            e += 1;
        }
        uint32_t code = ((uint32_t)(e + 7) << 3) | (q - 8u);
        if (code > 0x7Eu) code = 0x7Eu;         /* cannot trigger for |f| <= 448; kept as a guard */
        return (uint8_t)(sign | code);
    }

    /* Subnormal E4M3 range: the code is round(|f| / 2^-9) = round(sig * 2^(e - 14)). */
    const int shift = 14 - e;                   /* >= 21 here */
    uint32_t q;
    if (shift >= 26) {
        q = 0u;                                 /* sig < 2^24, so |f| / 2^-9 < 1/4: rounds to 0 */
    } else {
        q = sig >> shift;
        const uint32_t rem = sig & ((1u << shift) - 1u);
        const uint32_t half = 1u << (shift - 1);
        if (rem > half || (rem == half && (q & 1u))) q += 1u;
    }
    /* q == 8 is code 0x08, the smallest normal 2^-6: the encoding carries over correctly. */
    return (uint8_t)(sign | q);
}

/* Decode one E4M3FN byte to binary64 (exact). */
double oracle_e4m3_decode(uint8_t c)
{
    const int s = c >> 7;
    const int E = (c >> 3) & 0xF;
    const int m = c & 0x7;
    if (E == 15 && m == 7) return NAN;
    const double v = (E == 0) ? ldexp((double)m, -9)            /* m/8 * 2^-6 */
                              : ldexp((double)(8 + m), E - 10); /* (1 + m/8) * 2^(E-7) */
    return s ? -v : v;
}

/* Vectorised helpers over arrays, for the Python wrapper. */
void oracle_e4m3_encode_array(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_array(const uint8_t* c, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

/* ------------------------------------------------------------------------------------------ */
/* Group quantisation                                                                          */
/* ------------------------------------------------------------------------------------------ */

static float bf16_to_float(uint16_t h)
{
    const uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* The smallest amax a group is scaled by.  A group whose largest magnitude is below this floor
 * (an all-zero group, say) still gets a normal, finite scale and inverse. */
static const float AMAX_FLOOR = 0x1p-100f;
static const float E4M3_MAX = 448.0f;

/* Scale formats of the quantisers: the pages' max-abs scale, or its power-of-two variant. */
enum { SCALE_FP32 = 0, SCALE_UE8M0 = 1 };

/* Scale and inverse of one group from its largest magnitude. */
static void group_scale(float amax, float* s, float* inv, int fmt)
{
    const float a = amax > AMAX_FLOOR ? amax : AMAX_FLOOR;
    if (fmt == SCALE_UE8M0) {
        /* r = m * 2^e with m in [0.5, 1): the smallest power of two >= r is 2^(e-1) when r is
         * itself a power of two (m = 0.5), else 2^e.  r >= 2^-109 and r < 2^120, so both
         * 2^p and 2^-p are normal binary32 numbers. */
        const float r = a / E4M3_MAX;
        int e;
        const float m = frexpf(r, &e);
        const int p = (m == 0.5f) ? e - 1 : e;
        *s = ldexpf(1.0f, p);
        *inv = ldexpf(1.0f, -p);
        return;
    }
    *s = a / E4M3_MAX;        /* dequantisation multiplier, stored */
    *inv = E4M3_MAX / a;      /* quantisation multiplier */
}

/* 1x128 tile-wise quantisation of activations [SUMMARY, Key ideas, FP8 bullet]: one scale per row per
 * 128 consecutive columns.  x[M][K] bf16 bits -> q[M][K] codes, s[K/128][M] scales. */
void oracle_quant_1x128_fmt(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s, int fmt)
{
    const int64_t KB = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t kb = 0; kb < KB; ++kb) {
            float amax = 0.0f;
            for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
                const float v = fabsf(bf16_to_float(x[m * K + k]));
                if (v > amax) amax = v;
            }
            float sc, inv;
            group_scale(amax, &sc, &inv, fmt);
            s[kb * M + m] = sc;
            for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
                const float scaled = bf16_to_float(x[m * K + k]) * inv;
                q[m * K + k] = oracle_e4m3_encode(scaled);
            }
        }
    }
}

/* 128x1 quantisation along tokens with transposed output, the operand form Wgrad needs
 * because its inner dimension is the token dimension [REPOST, paragraph 4]:
 * x[T][C] bf16 bits -> qt[C][T] codes, s[T/128][C] scales (one per channel per 128 tokens). */
void oracle_quant_128x1_t_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* qt, float* s, int fmt)
{
    const int64_t TB = T / 128;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        for (int64_t tb = 0; tb < TB; ++tb) {
            float amax = 0.0f;
            for (int64_t t = tb * 128; t < tb * 128 + 128; ++t) {
                const float v = fabsf(bf16_to_float(x[t * C + c]));
                if (v > amax) amax = v;
            }
            float sc, inv;
            group_scale(amax, &sc, &inv, fmt);
            s[tb * C + c] = sc;
            for (int64_t t = tb * 128; t < tb * 128 + 128; ++t) {
                const float scaled = bf16_to_float(x[t * C + c]) * inv;
                qt[c * T + t] = oracle_e4m3_encode(scaled);
            }
        }
    }
}

/* 128x128 block-wise quantisation of weights [SUMMARY, Key ideas, FP8 bullet]: one scale per 128 output
 * rows x 128 input columns.  w[N][K] -> q[N][K], s[N/128][K/128]; qt[K][N] (optional, may be
 * NULL) receives the same codes transposed. */
void oracle_quant_128x128_fmt(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s,
                              uint8_t* qt, int fmt)
{
    const int64_t NB = N / 128, KB = K / 128;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t nb = 0; nb < NB; ++nb) {
        for (int64_t kb = 0; kb < KB; ++kb) {
            float amax = 0.0f;
            for (int64_t n = nb * 128; n < nb * 128 + 128; ++n)
                for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
                    const float v = fabsf(bf16_to_float(w[n * K + k]));
                    if (v > amax) amax = v;
                }
            float sc, inv;
            group_scale(amax, &sc, &inv, fmt);
            s[nb * KB + kb] = sc;
            for (int64_t n = nb * 128; n < nb * 128 + 128; ++n)
                for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
                    const uint8_t code = oracle_e4m3_encode(bf16_to_float(w[n * K + k]) * inv);
                    q[n * K + k] = code;
                    if (qt) qt[k * N + n] = code;
                }
        }
    }
}

/* The pages' scale format (fmt = SCALE_FP32). */
void oracle_quant_1x128(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s)
{
    oracle_quant_1x128_fmt(x, M, K, q, s, SCALE_FP32);
}

void oracle_quant_128x1_t(const uint16_t* x, int64_t T, int64_t C, uint8_t* qt, float* s)
{
    oracle_quant_128x1_t_fmt(x, T, C, qt, s, SCALE_FP32);
}

void oracle_quant_128x128(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s, uint8_t* qt)
{
    oracle_quant_128x128_fmt(w, N, K, q, s, qt, SCALE_FP32);
}

/* ------------------------------------------------------------------------------------------ */
/* Block-scaled GEMM, exact in binary64                                                        */
/* ------------------------------------------------------------------------------------------ */

enum { ORACLE_FPROP = 0, ORACLE_DGRAD = 1, ORACLE_WGRAD = 2 };

/* Dequantised A operand, all modes: A is [M][K] codes with 1x128 (or 128x1 transposed) scales
 * stored s[K/128][M]. */
static double a_hat(const uint8_t* A, const float* sA, int64_t M, int64_t K, int64_t m, int64_t k)
{
    return oracle_e4m3_decode(A[m * K + k]) * (double)sA[(k / 128) * M + m];
}

/* Dequantised B operand B(k, n) of D[m][n] = sum_k A(m,k) B(k,n), per mode:
 *   FPROP: B = W[N][K] codes, block scales s[N/128][K/128]     (Y = X W^T)
 *   DGRAD: B = W[K][N] codes (the same weight buffer, used transposed), s[K/128][N/128]
 *                                                              (dX = dY W)
 *   WGRAD: B = X^T[N][K] codes, per-row scales s[K/128][N]    (dW = dY^T X) */
static double b_hat(int mode, const uint8_t* B, const float* sB, int64_t N, int64_t K,
                    int64_t k, int64_t n)
{
    switch (mode) {
    case ORACLE_FPROP:
        return oracle_e4m3_decode(B[n * K + k]) * (double)sB[(n / 128) * (K / 128) + k / 128];
    case ORACLE_DGRAD:
        return oracle_e4m3_decode(B[k * N + n]) * (double)sB[(k / 128) * (N / 128) + n / 128];
    default:
        return oracle_e4m3_decode(B[n * K + k]) * (double)sB[(k / 128) * N + n];
    }
}

/* Full product: D[m][n] = sum_k a_hat(m,k) b_hat(k,n) and Sabs[m][n] = sum_k |a_hat b_hat|
 * (the magnitude the tolerance is relative to).  Dequantised operands are formed once (exact
 * in binary64) and the dot products run in k order. */
void oracle_gemm(int mode, const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                 int64_t M, int64_t N, int64_t K, double* D, double* Sabs,
                 double* work_a /* M*K */, double* work_b /* N*K */)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) work_a[m * K + k] = a_hat(A, sA, M, K, m, k);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) work_b[n * K + k] = b_hat(mode, B, sB, N, K, k, n);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        const double* a = work_a + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const double* b = work_b + n * K;
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const double p = a[k] * b[k];
                acc += p;
                mag += fabs(p);
            }
            D[m * N + n] = acc;
            if (Sabs) Sabs[m * N + n] = mag;
        }
    }
}

/* Selected entries only: out[i] = D[ms[i]][ns[i]], sabs[i] likewise.  Used at full problem
 * sizes, where the whole product is too slow on the CPU. */
void oracle_gemm_entries(int mode, const uint8_t* A, const float* sA, const uint8_t* B,
                         const float* sB, int64_t M, int64_t N, int64_t K, const int64_t* ms,
                         const int64_t* ns, int64_t count, double* out, double* sabs)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < count; ++i) {
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double p = a_hat(A, sA, M, K, ms[i], k) * b_hat(mode, B, sB, N, K, k, ns[i]);
            acc += p;
            mag += fabs(p);
        }
        out[i] = acc;
        if (sabs) sabs[i] = mag;
    }
}

/* Grouped (MoE expert) Fprop: rows [off[e], off[e+1]) of A belong to expert e and multiply
 * W_e = B + e*N*K with block scales sB + e*(N/128)*(K/128).  A's scales are s[K/128][Mtot].
 * Selected entries only (row ms[i], column ns[i]). */
void oracle_grouped_entries(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                            const int32_t* off, int32_t E, int64_t Mtot, int64_t N, int64_t K,
                            const int64_t* ms, const int64_t* ns, int64_t count, double* out,
                            double* sabs)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < count; ++i) {
        const int64_t m = ms[i];
        int32_t e = 0;
        while (e < E && !(off[e] <= m && m < off[e + 1])) ++e;   /* linear search: plain */
        const uint8_t* Be = B + (int64_t)e * N * K;
        const float* sBe = sB + (int64_t)e * (N / 128) * (K / 128);
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double p = a_hat(A, sA, Mtot, K, m, k) * b_hat(ORACLE_FPROP, Be, sBe, N, K, k, ns[i]);
            acc += p;
            mag += fabs(p);
        }
        out[i] = acc;
        if (sabs) sabs[i] = mag;
    }
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
