/*
 * CPU oracle for the RT-Lynx activation-sparse linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library.  The product path (the
 * CUDA library under activation_sparse_gemm_b200/) shares no code with it and
 * never calls it.
 *
 * What it computes (RT-Lynx, paper.rainbus.top summary of arXiv 2605.26632,
 * "four-step pipeline" paragraph, steps 1-2; the fugumt abstract page for the
 * same paper states the method's scope):
 *
 *   X~   = per token, keep 2 of every 4 consecutive channels (Top-K, 2 of 4)
 *   s    = ||X||_2 / (||X~||_2 + eps),  eps = 1e-8
 *   S(X) = s * X~
 *   Y_s  = S(X) W^T,   Y_r = X (L_A L_B)^T  (dense X, rank R),   Y = Y_s + Y_r
 *   dense-skip layers ("Selective Layer Skipping", step 3): Y = X W^T
 *   feed-forward block of two such layers: H = bf16(GELU(Y_up)), GELU in its
 *   erf form, then Y = layer_down(H)
 *
 * Readings where the page is silent (each is listed in the design notes):
 *   - Top-K ranks by magnitude |x|; equal magnitudes go to the lower index;
 *     -0 and +0 are equal.  An all-zero group keeps indices 0 and 1.
 *   - eps is added to the norm (not to its square), as printed.
 *   - s is a float32 per token: computed here in double, rounded once.
 *   - the stored sparse value is bf16_rne(s * x), from the exact product.
 *   - the LoRA branch sees the dense X; no alpha/r scale, no bias.
 *   - metadata nibble for a group = i0 | (i1 << 2) with i0 < i1 (the
 *     2:4 encoding of the sparse tensor-core instructions).
 *
 * All arithmetic on values is double; every GEMM is a plain triple loop with
 * no blocking or reordering; rows are independent and run under OpenMP.
 *
 * Layouts (row-major, little-endian, bf16 passed as uint16 bit patterns):
 *   X [M,K], W [N,K], L_A [N,R], L_B [R,K]
 *   meta [M, K/4] uint8 (one nibble per byte), vals [M, K/2] bf16, s [M] f32
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define RTLYNX_EPS 1e-8

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even, in one step (no detour
 * through float, so there is no double rounding).  bf16 has 8 significant
 * bits and float's exponent range; its subnormals are multiples of 2^-133. */
static uint16_t double_to_bf16_rne(double v)
{
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (a < 0x1p-126) {
        r = ldexp(nearbyint(ldexp(a, 133)), -133);
    } else {
        int e;
        double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);
    }
    float f = (float)r; /* exact, or +inf past the largest bf16 */
    if (v < 0 || (v == 0 && signbit(v))) f = -f;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

uint16_t oracle_bf16_from_double(double v) { return double_to_bf16_rne(v); }
double oracle_double_from_bf16(uint16_t b) { return bf16_to_double(b); }

/* Top-K (2 of 4) on one group: index i is kept iff fewer than two other
 * entries beat it, where j beats i when |x_j| > |x_i|, or |x_j| == |x_i|
 * and j < i.  Returns the kept indices in ascending order.  For finite
 * entries exactly two are kept; a NaN (out of contract) compares false and
 * could pass the test for more, so at most the first two are taken. */
static void keep_two_of_four(const double x[4], int *i0, int *i1)
{
    int kept[2] = {0, 1}, n = 0;
    for (int i = 0; i < 4 && n < 2; ++i) {
        int beaten = 0;
        for (int j = 0; j < 4; ++j) {
            if (j == i) continue;
            double aj = fabs(x[j]), ai = fabs(x[i]);
            if (aj > ai || (aj == ai && j < i)) ++beaten;
        }
        if (beaten < 2) kept[n++] = i;
    }
    *i0 = kept[0];
    *i1 = kept[1];
}

/* Step 1 for one token: mask, norms, s, and the rounded kept values.
 * Xrow [K] bf16 -> meta [K/4], vals [K/2] bf16, returns s; also writes the
 * dense S(X) row (double, zeros at dropped positions) when S != NULL. */
static float sparsify_row(const uint16_t *Xrow, int64_t K, uint8_t *meta,
                          uint16_t *vals, double *S)
{
    double nx = 0.0, nt = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double x = bf16_to_double(Xrow[k]);
        nx += x * x;
    }
    for (int64_t g = 0; g < K / 4; ++g) {
        double x[4];
        for (int i = 0; i < 4; ++i) x[i] = bf16_to_double(Xrow[4 * g + i]);
        int i0, i1;
        keep_two_of_four(x, &i0, &i1);
        nt += x[i0] * x[i0] + x[i1] * x[i1];
    }
    float s = (float)(sqrt(nx) / (sqrt(nt) + RTLYNX_EPS));
    for (int64_t g = 0; g < K / 4; ++g) {
        double x[4];
        for (int i = 0; i < 4; ++i) x[i] = bf16_to_double(Xrow[4 * g + i]);
        int i0, i1;
        keep_two_of_four(x, &i0, &i1);
        uint16_t v0 = double_to_bf16_rne((double)s * x[i0]);
        uint16_t v1 = double_to_bf16_rne((double)s * x[i1]);
        if (meta) meta[g] = (uint8_t)(i0 | (i1 << 2));
        if (vals) {
            vals[2 * g] = v0;
            vals[2 * g + 1] = v1;
        }
        if (S) {
            for (int i = 0; i < 4; ++i) S[4 * g + i] = 0.0;
            S[4 * g + i0] = bf16_to_double(v0);
            S[4 * g + i1] = bf16_to_double(v1);
        }
    }
    return s;
}

/* Mask, metadata, s and compressed values for every token. */
int oracle_sparsify(const uint16_t *X, int64_t M, int64_t K, uint8_t *meta,
                    uint16_t *vals, float *s)
{
    if (M < 0 || K <= 0 || K % 4) return 1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        float sm = sparsify_row(X + m * K, K, meta ? meta + m * (K / 4) : NULL,
                                vals ? vals + m * (K / 2) : NULL, NULL);
        if (s) s[m] = sm;
    }
    return 0;
}

/* Y rows (and optionally T rows) for the tokens listed in rows[0..nrows)
 * (rows == NULL means every token, nrows = M).
 *   mode 0 (sparse):     T = X L_B^T,  Y = S(X) W^T + T L_A^T
 *   mode 1 (dense-skip): Y = X W^T
 * Y [nrows, N] double, T [nrows, R] double (may be NULL). R == 0 or a NULL
 * L_A / L_B means no LoRA branch. */
int oracle_linear_rows(const uint16_t *X, const uint16_t *W, const uint16_t *L_A,
                       const uint16_t *L_B, int64_t M, int64_t K, int64_t N,
                       int64_t R, int mode, const int64_t *rows, int64_t nrows,
                       double *Y, double *T)
{
    if (M < 0 || K <= 0 || N <= 0 || R < 0 || (mode != 0 && mode != 1)) return 1;
    if (mode == 0 && K % 4) return 1;
    if (!rows) nrows = M;
    int use_lora = (mode == 0 && R > 0 && L_A && L_B);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        if (m < 0 || m >= M) {
            bad = 1;
            continue;
        }
        const uint16_t *Xrow = X + m * K;
        double *A = (double *)malloc(sizeof(double) * (size_t)K);
        double *Trow = (double *)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1));
        if (mode == 0) {
            sparsify_row(Xrow, K, NULL, NULL, A);
        } else {
            for (int64_t k = 0; k < K; ++k) A[k] = bf16_to_double(Xrow[k]);
        }
        if (use_lora) {
            for (int64_t r = 0; r < R; ++r) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += bf16_to_double(Xrow[k]) * bf16_to_double(L_B[r * K + k]);
                Trow[r] = acc;
            }
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += A[k] * bf16_to_double(W[n * K + k]);
            if (use_lora) {
                double lr = 0.0;
                for (int64_t r = 0; r < R; ++r) lr += Trow[r] * bf16_to_double(L_A[n * R + r]);
                acc += lr;
            }
            Y[i * N + n] = acc;
        }
        if (T && R > 0) {
            for (int64_t r = 0; r < R; ++r) T[i * R + r] = use_lora ? Trow[r] : 0.0;
        }
        free(A);
        free(Trow);
    }
    return bad ? 1 : 0;
}

/* The activation between the two layers of a DiT feed-forward block:
 * GELU in its erf form, gelu(y) = y * Phi(y) = y/2 * (1 + erf(y / sqrt 2)),
 * written as y/2 * erfc(-y / sqrt 2), the same function without the
 * cancellation of 1 + erf for negative y.  Evaluated in double on the exact
 * output of the first layer and rounded once to bf16 (nearest even): the
 * block's intermediate activation is a bf16 tensor like every activation the
 * layers exchange.  H [n] bf16 bits. */
double oracle_gelu(double y) { return 0.5 * y * erfc(-y / sqrt(2.0)); }

int oracle_gelu_bf16(const double *Y, int64_t n, uint16_t *H)
{
    if (n < 0) return 1;
    for (int64_t i = 0; i < n; ++i) H[i] = double_to_bf16_rne(oracle_gelu(Y[i]));
    return 0;
}

/* ------------------------------------------------------------------ FP8
 * The FP8 form of the layer (the pages name FP8 as future work that stacks
 * with the method and give no recipe; the reading, listed in the design
 * notes):
 *   - E4M3 is the OCP 8-bit float without infinities (NVIDIA's e4m3): sign,
 *     4 exponent bits with bias 7, 3 mantissa bits; largest finite magnitude
 *     448 = 1.75 * 2^8, smallest normal 2^-6, subnormals j * 2^-9 (j = 1..7);
 *     S.1111.111 is NaN.  Encoding rounds to nearest, ties to even, and
 *     saturates magnitudes past 448 to 448.
 *   - W is quantised once per output channel n: B_n = max_k |W[n,k]|,
 *     w8 = E4M3(W * r_n) with r_n = 448 / B_n, dequantisation scale
 *     q_w[n] = B_n / 448.
 *   - S(X) is quantised per token with q_x = max |S(X)| / 448.  s > 0 scales
 *     every entry of the token alike and the largest |x| is always kept, so
 *     the codes are E4M3(x~ * r) with r = 448 / A, A = max_k |x_k|, and
 *     q_x = s * A / 448.
 *   - The quantisation decisions (r, and the product that is rounded to a
 *     code) are taken in float32, as a kernel takes them; everything after
 *     the codes is double.
 *   - Y = q_x * q_w[n] * sum over kept k of x8 * w8 + T L_A^T, T = X L_B^T
 *     as in the bf16 form.  An all-zero token or channel has scale 0 and
 *     codes 0. */
static uint8_t e4m3_from_double(double v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < 0x1p-6) {
        /* subnormal range: j * 2^-9, j = 0..8 (j = 8 is 2^-6, code 0x08) */
        return sign | (uint8_t)nearbyint(ldexp(a, 9));
    }
    int e;
    double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1): unbiased exponent e - 1 */
    int q = (int)nearbyint(ldexp(m, 4)) - 8; /* 3 mantissa bits: 2m in [1, 2) -> 8 + q */
    int ex = e - 1;
    if (q == 8) {
        q = 0;
        ex += 1;
    }
    return sign | (uint8_t)(((ex + 7) << 3) | q);
}

static double e4m3_to_double(uint8_t c)
{
    int ex = (c >> 3) & 0xF, q = c & 7;
    double a = ex == 0 ? ldexp((double)q, -9) : ldexp(1.0 + q / 8.0, ex - 7);
    return (c & 0x80) ? -a : a;
}

uint8_t oracle_e4m3_from_float(float v) { return e4m3_from_double((double)v); }
double oracle_e4m3_to_double(uint8_t c) { return e4m3_to_double(c); }

/* Per-channel E4M3 weights: W [N,K] bf16 -> W8 [N,K] codes, qw [N] float. */
int oracle_quantize_weight_fp8(const uint16_t *W, int64_t N, int64_t K, uint8_t *W8, float *qw)
{
    if (N < 0 || K <= 0) return 1;
    for (int64_t n = 0; n < N; ++n) {
        float b = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = (float)fabs(bf16_to_double(W[n * K + k]));
            if (a > b) b = a;
        }
        float r = b > 0.0f ? 448.0f / b : 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float t = (float)bf16_to_double(W[n * K + k]) * r;
            W8[n * K + k] = e4m3_from_double((double)t);
        }
        qw[n] = b / 448.0f;
    }
    return 0;
}

/* Step 1 in FP8 for one token: metadata as the bf16 form, the kept entries'
 * codes x8 [K/2], s, and the token's dequantisation scale q_x (double). */
static float sparsify_row_fp8(const uint16_t *Xrow, int64_t K, uint8_t *meta, uint8_t *x8, double *qx)
{
    float s = sparsify_row(Xrow, K, NULL, NULL, NULL);
    float A = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = (float)fabs(bf16_to_double(Xrow[k]));
        if (a > A) A = a;
    }
    float r = A > 0.0f ? 448.0f / A : 0.0f;
    for (int64_t g = 0; g < K / 4; ++g) {
        double x[4];
        for (int i = 0; i < 4; ++i) x[i] = bf16_to_double(Xrow[4 * g + i]);
        int i0, i1;
        keep_two_of_four(x, &i0, &i1);
        if (meta) meta[g] = (uint8_t)((i1 << 2) | i0);
        x8[2 * g] = e4m3_from_double((double)((float)x[i0] * r));
        x8[2 * g + 1] = e4m3_from_double((double)((float)x[i1] * r));
    }
    *qx = (double)s * (double)A / 448.0;
    return s;
}

int oracle_sparsify_fp8(const uint16_t *X, int64_t M, int64_t K, uint8_t *meta, uint8_t *x8, float *s,
                        double *qx)
{
    if (M < 0 || K <= 0 || K % 4) return 1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        double q;
        float sm = sparsify_row_fp8(X + m * K, K, meta ? meta + m * (K / 4) : NULL, x8 + m * (K / 2), &q);
        if (s) s[m] = sm;
        if (qx) qx[m] = q;
    }
    return 0;
}

/* Y rows of the FP8 form for the listed tokens (rows == NULL: all):
 * Y = q_x q_w[n] sum_{kept k} x8 w8[n,k] + X L_B^T L_A^T.  W8 [N,K] codes,
 * qw [N] from oracle_quantize_weight_fp8. */
int oracle_linear_fp8_rows(const uint16_t *X, const uint8_t *W8, const float *qw, const uint16_t *L_A,
                           const uint16_t *L_B, int64_t M, int64_t K, int64_t N, int64_t R,
                           const int64_t *rows, int64_t nrows, double *Y)
{
    if (M < 0 || K <= 0 || K % 4 || N <= 0 || R < 0) return 1;
    if (!rows) nrows = M;
    int use_lora = R > 0 && L_A && L_B;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        if (m < 0 || m >= M) {
            bad = 1;
            continue;
        }
        const uint16_t *Xrow = X + m * K;
        uint8_t *meta = (uint8_t *)malloc((size_t)(K / 4));
        uint8_t *x8 = (uint8_t *)malloc((size_t)(K / 2));
        double *Trow = (double *)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1));
        double qx;
        sparsify_row_fp8(Xrow, K, meta, x8, &qx);
        if (use_lora) {
            for (int64_t r = 0; r < R; ++r) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += bf16_to_double(L_B[r * K + k]) * bf16_to_double(Xrow[k]);
                Trow[r] = acc;
            }
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t g = 0; g < K / 4; ++g) {
                int i0 = meta[g] & 3, i1 = meta[g] >> 2;
                acc += e4m3_to_double(x8[2 * g]) * e4m3_to_double(W8[n * K + 4 * g + i0]);
                acc += e4m3_to_double(x8[2 * g + 1]) * e4m3_to_double(W8[n * K + 4 * g + i1]);
            }
            double y = qx * (double)qw[n] * acc;
            if (use_lora) {
                double lr = 0.0;
                for (int64_t r = 0; r < R; ++r) lr += bf16_to_double(L_A[n * R + r]) * Trow[r];
                y += lr;
            }
            Y[i * N + n] = y;
        }
        free(meta);
        free(x8);
        free(Trow);
    }
    return bad ? 1 : 0;
}

/* Threads the OpenMP runtime will use (reported next to CPU timings). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
