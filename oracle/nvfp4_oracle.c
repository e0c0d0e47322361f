/*
 * nvfp4_oracle.c -- plain CPU oracle for the NVFP4 verify GEMM.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct
 * reference that the GPU library is checked against. Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it; the product
 * path never does. It shares no code, header, table or constant with the GPU
 * library.
 *
 * What it computes (cited by page title and section):
 *   - Weight format: four bits a weight with one scale per 16 weights
 *     (TandemLLM docs v0.12.0, "What TandemLLM is", section 1.2). The bit
 *     level is the OCP formats: E2M1 codes {+-0, 0.5, 1, 1.5, 2, 3, 4, 6}
 *     packed two per byte, low nibble = even k; one E4M3 ("fn": no infinity,
 *     0x7F/0xFF are NaN, max 448) scale per 16-element K block; one FP32
 *     tensor scale that multiplies.
 *   - The verify GEMM: Y[M,N] = X[M,K] . dequant(W)[N,K]^T, one pass of the
 *     big model over all draft-tree rows (same page, section 1.2; the
 *     StairCut research page, "What it says").
 *   - Quantiser (round to nearest): g = fp32(absmax_tensor / (6*448));
 *     per 16-block s = E4M3_RNE_satfinite(absmax_block / 6 / g) in fp64;
 *     codes = E2M1_RNE(w / (dec(s)*g)) in fp64, ties to the even code, zero
 *     never encoded as -0.
 *
 * Every function is written from those definitions, in fp64, with loops in
 * definition order. Nothing is blocked, fused or reordered. OpenMP splits
 * independent output elements (rows n) only; each sum runs sequentially
 * over k, so results do not depend on the thread count.
 *
 * Parity status: every function below is pinned by tests/test_oracle_pins.py
 * (hand-worked bytes, library decoders, closed forms, brute force with exact
 * rationals, identity / one-hot / small-integer cases, M-invariance).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_ERR_INVALID 1
#define OR_ERR_NONFINITE 2

/* ---- element formats --------------------------------------------------- */

/* E2M1 magnitudes, indexed by the low three bits of the code (e1 e0 m). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double or_e2m1_decode(uint32_t code) {
    double v = E2M1_MAG[code & 7u];
    return (code & 8u) ? -v : v;
}

/* E4M3 ("fn") by its bit fields: sign s, exponent e (4 bits, bias 7), mantissa m (3 bits).
 * e == 0: m * 2^-9 (subnormal); e == 15 and m == 7: NaN; else (1 + m/8) * 2^(e-7). */
double or_e4m3_decode(uint32_t byte) {
    uint32_t s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
    double v;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -v : v;
}

/* bf16 bit pattern -> value (exact). */
static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Nearest E4M3 code to t >= 0 (round to nearest, ties to the even mantissa),
 * saturating to 448 (0x7E). Plain search over the 127 finite non-negative codes. */
uint32_t or_e4m3_encode(double t) {
    uint32_t best = 0;
    double best_d = INFINITY;
    if (!(t >= 0.0)) return 0xFFu; /* negative or NaN: not produced by the quantiser */
    if (t >= 448.0) return 0x7Eu;
    for (uint32_t b = 0; b <= 0x7Eu; ++b) {
        double d = fabs(t - or_e4m3_decode(b));
        if (d < best_d || (d == best_d && (b & 1u) == 0u)) {
            best_d = d;
            best = b;
        }
    }
    return best;
}

/* Nearest E2M1 code to q (round to nearest, ties to the even mantissa), |q| clamped to 6.
 * A result of magnitude zero is code 0 (never -0). */
uint32_t or_e2m1_encode(double q) {
    double a = fabs(q);
    uint32_t best = 0;
    double best_d = INFINITY;
    if (a > 6.0) a = 6.0;
    for (uint32_t c = 0; c < 8u; ++c) {
        double d = fabs(a - E2M1_MAG[c]);
        if (d < best_d || (d == best_d && (c & 1u) == 0u)) {
            best_d = d;
            best = c;
        }
    }
    if (best != 0u && q < 0.0) best |= 8u;
    return best;
}

/* ---- quantiser ----------------------------------------------------------- */

/* w: fp32 [N][K] row-major, K % 16 == 0.
 * codes: [N][K/2] bytes, byte j of a row = code(k=2j) | code(k=2j+1) << 4.
 * scales: [N][K/16] E4M3 bytes. g_out: the FP32 tensor scale. */
int or_quantize(const float* w, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales,
                float* g_out) {
    if (N < 0 || K < 0 || (K % 16) != 0) return OR_ERR_INVALID;
    float amax = 0.0f;
    for (int64_t i = 0; i < N * K; ++i) {
        if (!isfinite(w[i])) return OR_ERR_NONFINITE;
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
    }
    float g = (float)((double)amax / (6.0 * 448.0));
    *g_out = g;
    int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* wb = w + n * K + b * 16;
            double bmax = 0.0;
            for (int j = 0; j < 16; ++j) {
                double a = fabs((double)wb[j]);
                if (a > bmax) bmax = a;
            }
            uint32_t s = 0;
            if (g != 0.0f) s = or_e4m3_encode(bmax / 6.0 / (double)g);
            scales[n * nb + b] = (uint8_t)s;
            double denom = or_e4m3_decode(s) * (double)g;
            for (int j = 0; j < 16; j += 2) {
                uint32_t c0 = 0, c1 = 0;
                if (denom != 0.0) {
                    c0 = or_e2m1_encode((double)wb[j] / denom);
                    c1 = or_e2m1_encode((double)wb[j + 1] / denom);
                }
                codes[n * (K / 2) + b * 8 + j / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
    return OR_OK;
}

/* ---- decoder ------------------------------------------------------------- */

/* Unscaled product e2m1 * e4m3 of element (n, k): exact in fp64 (at most 6 significant bits). */
static double wq_elem(const uint8_t* codes, const uint8_t* scales, int64_t K, int64_t n, int64_t k) {
    uint8_t byte = codes[n * (K / 2) + k / 2];
    uint32_t code = (k & 1) ? (uint32_t)(byte >> 4) : (uint32_t)(byte & 15u);
    return or_e2m1_decode(code) * or_e4m3_decode(scales[n * (K / 16) + k / 16]);
}

/* Dequantised weights w32[n][k] = fp32_RN(e2m1 * e4m3 * g) (one rounding: the fp64 product is exact).
 * wq (optional): the unscaled products e2m1 * e4m3 in fp64. */
int or_dequant(const uint8_t* codes, const uint8_t* scales, float g, int64_t N, int64_t K,
               float* w32, double* wq) {
    if (N < 0 || K < 0 || (K % 16) != 0) return OR_ERR_INVALID;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double p = wq_elem(codes, scales, K, n, k);
            if (wq) wq[n * K + k] = p;
            if (w32) w32[n * K + k] = (float)(p * (double)g);
        }
    }
    return OR_OK;
}

/* ---- GEMM ---------------------------------------------------------------- */

/* One output element: y = (sum_k x[m,k] * (e2m1*e4m3)[n,k]) * g and a = sum_k |x * w|, in fp64. */
static void gemm_elem(const uint16_t* x, int64_t K, const uint8_t* codes, const uint8_t* scales,
                      float g, int64_t m, int64_t n, double* y, double* a) {
    double acc = 0.0, abs_acc = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double p = bf16_to_double(x[m * K + k]) * wq_elem(codes, scales, K, n, k);
        acc += p;
        abs_acc += fabs(p);
    }
    *y = acc * (double)g;
    *a = abs_acc * fabs((double)g);
}

/* x: bf16 bits [M][K]; y_ref, a_ref: fp64 [M][N]. */
int or_gemm(const uint16_t* x, int64_t M, const uint8_t* codes, const uint8_t* scales, float g,
            int64_t N, int64_t K, double* y_ref, double* a_ref) {
    if (M < 0 || N < 0 || K < 0 || (K % 16) != 0) return OR_ERR_INVALID;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m)
            gemm_elem(x, K, codes, scales, g, m, n, &y_ref[m * N + n], &a_ref[m * N + n]);
    return OR_OK;
}

/* Sampled outputs: element i is (m_idx[i], n_idx[i]). */
int or_gemm_sampled(const uint16_t* x, int64_t M, const uint8_t* codes, const uint8_t* scales,
                    float g, int64_t N, int64_t K, const int64_t* m_idx, const int64_t* n_idx,
                    int64_t count, double* y, double* a) {
    if (M < 0 || N < 0 || K < 0 || (K % 16) != 0) return OR_ERR_INVALID;
    for (int64_t i = 0; i < count; ++i)
        if (m_idx[i] < 0 || m_idx[i] >= M || n_idx[i] < 0 || n_idx[i] >= N) return OR_ERR_INVALID;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i)
        gemm_elem(x, K, codes, scales, g, m_idx[i], n_idx[i], &y[i], &a[i]);
    return OR_OK;
}

int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void or_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
