/*
 * convrot_oracle.c -- plain, slow CPU oracle for the rotated W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA
 * library and is written to be checked against the pages by eye: dense
 * matrices, scalar loops, fp64 wherever the pages leave the precision open.
 *
 * What it computes (sources are the pages' titles and sections):
 *
 *  - H_n, the normalised regular Hadamard matrix of order n = 4^k.
 *    "convrot-mlx" README, "What is included": normalised regular-Hadamard
 *    rotation for groups of 64 and 256.  Comfy-Org/comfy-quants issue
 *    "convrot is exactly same as ... QuaRot Stage 1c", section 2 ("The
 *    equivalent Hadamard matrix"): the regular matrix is used for N_0 = 4^k.
 *    Reading: H_n = (J - 2I)^{(x)k} / sqrt(n), the k-th Kronecker power of the
 *    order-4 regular Hadamard J - 2I, normalised so that H H^T = I.
 *    Entry (i, j) is (-1)^{number of base-4 digit positions where i and j
 *    agree} / sqrt(n).  oracle_hadamard builds it from that digit rule;
 *    oracle_hadamard_kron builds it by literal repeated Kronecker products.
 *
 *  - The block rotation R = I_G (x) H_n.  Same issue, section 1 ("Both apply
 *    'group-wise' operator"): X R = [X_1 H, ..., X_G H], one Hadamard per
 *    K-group of n channels.  Written here as a dense fp64 mat-vec per group.
 *
 *  - Rowwise symmetric absmax INT4 in [-7, 7].  "convrot-mlx" README, "What is
 *    included".  One scale per row (per token for activations, per output
 *    channel for weights); the group size only affects the rotation.
 *    Readings (the pages leave these open): the decision is taken in fp32,
 *      a   = fp32(max_k |y_k|)         (y the fp64 rotated row)
 *      s   = a / 7                      (fp32, IEEE division; the stored scale)
 *      inv = 7 / a                      (fp32, IEEE division)
 *      v_k = fp32(y_k) * inv            (one fp32 multiply)
 *      q_k = clamp(round_half_away(v_k), -7, 7);  a == 0 gives s = 0, q = 0.
 *
 *  - Packing, two codes per byte, low nibble = even k, 4-bit two's complement.
 *    "convrot-mlx" README, "What is included" (N x packed-K layout); nibble
 *    order per "mlx-nf4" README, "What it provides" (low-first intake).
 *
 *  - The integer GEMM acc[m][n] = sum_k qx[m][k] * qw[n][k] in int64, and the
 *    epilogue y = bf16_rne(((float)acc * sx[m]) * sw[n] + (float)b[n]) in
 *    fp32 in that order.  "convrot-mlx" README, "Install and test": the
 *    complete path is rotation, activation quantisation, the integer product,
 *    scaling and bias.
 *
 *  - The W4A16 variant.  "convrot-mlx" README, "What is included" (a W4A16
 *    TensorOps path beside W4A4) and "Requirements" (BF16 x INT4 products).
 *    The pages give no formula; reading: the weights are the W4A4 ones
 *    (rotated, quantised, packed), the activations are rotated by the same
 *    R and each rotated value is rounded once to bf16 (the operand type),
 *    and y = bf16_rne(sum_k xr[m][k] q[n][k] * sw[n] + b[n]) with the sum,
 *    the scaling and the bias exact (fp64 here), rounded once at the end.
 *
 *  - The reversible weight repack (oracle_repack_weight / _unpack_weight).
 *    "convrot-mlx" README, "What is included" (lossless repacking) and
 *    "Install and test" (repack_nk_weight_for_mpp): the packed bytes in
 *    128-byte column blocks, block-major, and back.
 *
 *  - The NVFP4 variant (oracle_nvfp4_*).  "convrot-mlx" README, "Why this
 *    repository exists" (the official ConvRot targets NVFP4 on Blackwell);
 *    the format itself is not on the pages: E2M1 codes with one E4M3 scale
 *    per 16 values and one fp32 scale per row (reading in the function).
 *
 * Every function returns 0 on success or a negative number for bad
 * arguments.  Buffers are caller-owned, row-major and contiguous.
 * bf16 values travel as their raw 16-bit patterns (uint16_t).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ----------------------------------------------------------------------- */
/* bf16 <-> float, written out by hand.                                     */
/* ----------------------------------------------------------------------- */

/* A bf16 pattern is the top half of an IEEE binary32 pattern. */
static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a finite binary32 to bf16, nearest-even on the 16 dropped bits. */
static uint16_t float_to_bf16_bits_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u) {            /* inf / nan: keep */
        uint16_t h = (uint16_t)(u >> 16);
        if (u & 0x007FFFFFu) h |= 0x0040u;              /* quiet nan */
        return h;
    }
    uint32_t dropped = u & 0xFFFFu;
    uint32_t kept = u >> 16;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

int oracle_bf16_to_double(const uint16_t *in, int64_t count, double *out) {
    if (!in || !out || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) out[i] = bf16_bits_to_double(in[i]);
    return 0;
}

int oracle_float_to_bf16(const float *in, int64_t count, uint16_t *out) {
    if (!in || !out || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) out[i] = float_to_bf16_bits_rne(in[i]);
    return 0;
}

/* ----------------------------------------------------------------------- */
/* The regular Hadamard matrix.                                             */
/* ----------------------------------------------------------------------- */

/* k such that n == 4^k, or -1. */
static int log4_exact(int n) {
    int k = 0;
    if (n < 1) return -1;
    while (n > 1) {
        if (n % 4) return -1;
        n /= 4;
        ++k;
    }
    return k;
}

/* H[i*n + j] = (-1)^{#digits where i and j agree} / sqrt(n). */
int oracle_hadamard(int n, double *H) {
    int k = log4_exact(n);
    if (k < 0 || !H) return -1;
    double norm = 1.0 / sqrt((double)n);
    for (int i = 0; i < n; ++i) {
        for (int j = 0; j < n; ++j) {
            int agree = 0, a = i, b = j;
            for (int d = 0; d < k; ++d) {
                if (a % 4 == b % 4) ++agree;
                a /= 4;
                b /= 4;
            }
            H[(int64_t)i * n + j] = (agree % 2 ? -1.0 : 1.0) * norm;
        }
    }
    return 0;
}

/* The same matrix by literal Kronecker products: start from the 1x1 matrix
 * [1] and k times form P <- P (x) T with T = (J - 2I) / 2. */
int oracle_hadamard_kron(int n, double *H) {
    int k = log4_exact(n);
    if (k < 0 || !H) return -1;
    double T[4][4];
    for (int a = 0; a < 4; ++a)
        for (int b = 0; b < 4; ++b) T[a][b] = (a == b ? -1.0 : 1.0) / 2.0;
    double *P = (double *)malloc(sizeof(double) * (size_t)n * n);
    double *Q = (double *)malloc(sizeof(double) * (size_t)n * n);
    if (!P || !Q) { free(P); free(Q); return -2; }
    int m = 1;
    P[0] = 1.0;
    for (int step = 0; step < k; ++step) {
        int m4 = m * 4;
        /* (P (x) T)[r*4 + a][c*4 + b] = P[r][c] * T[a][b] */
        for (int r = 0; r < m; ++r)
            for (int c = 0; c < m; ++c)
                for (int a = 0; a < 4; ++a)
                    for (int b = 0; b < 4; ++b)
                        Q[(int64_t)(r * 4 + a) * m4 + (c * 4 + b)] = P[(int64_t)r * m + c] * T[a][b];
        double *t = P; P = Q; Q = t;
        m = m4;
    }
    memcpy(H, P, sizeof(double) * (size_t)n * n);
    free(P);
    free(Q);
    return 0;
}

/* ----------------------------------------------------------------------- */
/* Block rotation X -> X (I_G (x) H_n).                                      */
/* ----------------------------------------------------------------------- */

/* y[r][g*n + i] = sum_j x[r][g*n + j] * H[j][i], all in fp64.
 * x is bf16 (rows x K); K must be a multiple of n. */
int oracle_rotate(const uint16_t *x, int64_t rows, int64_t K, int n, double *y) {
    if (!x || !y || rows < 0 || K <= 0 || log4_exact(n) < 0 || K % n) return -1;
    double *H = (double *)malloc(sizeof(double) * (size_t)n * n);
    double *Ht = (double *)malloc(sizeof(double) * (size_t)n * n);
    if (!H || !Ht) { free(H); free(Ht); return -2; }
    oracle_hadamard(n, H);
    /* Ht[i][j] = H[j][i]: the same products in the same order, read row-wise */
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) Ht[(int64_t)i * n + j] = H[(int64_t)j * n + i];
    int64_t G = K / n;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        double *xg = (double *)malloc(sizeof(double) * (size_t)n);
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t *src = x + r * K + g * n;
            for (int j = 0; j < n; ++j) xg[j] = bf16_bits_to_double(src[j]);
            double *dst = y + r * K + g * n;
            for (int i = 0; i < n; ++i) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j) acc += xg[j] * Ht[(int64_t)i * n + j];
                dst[i] = acc;
            }
        }
        free(xg);
    }
    free(H);
    free(Ht);
    return 0;
}

/* ----------------------------------------------------------------------- */
/* Rowwise symmetric absmax quantisation to [-7, 7].                         */
/* ----------------------------------------------------------------------- */

/* Round half away from zero, written from its definition: the integer
 * nearest to v, and on an exact tie the one of larger magnitude. */
static int round_half_away(float v) {
    double a = fabs((double)v);
    double f = floor(a);
    double frac = a - f;                  /* exact in double */
    int mag = (int)f + (frac >= 0.5 ? 1 : 0);
    return v < 0.0f ? -mag : mag;
}

int oracle_quantize_rows(const double *y, int64_t rows, int64_t K, int8_t *q, float *s) {
    if (!y || !q || !s || rows < 0 || K <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *yr = y + r * K;
        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double t = fabs(yr[k]);
            if (t > amax) amax = t;
        }
        float a = (float)amax;
        if (a == 0.0f) {
            s[r] = 0.0f;
            memset(q + r * K, 0, (size_t)K);
            continue;
        }
        float sr = a / 7.0f;
        float inv = 7.0f / a;
        s[r] = sr;
        for (int64_t k = 0; k < K; ++k) {
            float v = (float)yr[k] * inv;
            int c = round_half_away(v);
            if (c > 7) c = 7;
            if (c < -7) c = -7;
            q[r * K + k] = (int8_t)c;
        }
    }
    return 0;
}

/* ----------------------------------------------------------------------- */
/* Nibble packing.                                                           */
/* ----------------------------------------------------------------------- */

/* byte[j] = (q[2j] & 0xF) | ((q[2j+1] & 0xF) << 4).  K must be even. */
int oracle_pack(const int8_t *q, int64_t rows, int64_t K, uint8_t *p) {
    if (!q || !p || rows < 0 || K <= 0 || K % 2) return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < K / 2; ++j) {
            uint8_t lo = (uint8_t)q[r * K + 2 * j] & 0x0Fu;
            uint8_t hi = (uint8_t)q[r * K + 2 * j + 1] & 0x0Fu;
            p[r * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
    return 0;
}

/* A 4-bit two's complement nibble back to a signed integer. */
static int nibble_to_int(unsigned v) {
    v &= 0x0Fu;
    return v >= 8u ? (int)v - 16 : (int)v;
}

int oracle_unpack(const uint8_t *p, int64_t rows, int64_t K, int8_t *q) {
    if (!p || !q || rows < 0 || K <= 0 || K % 2) return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < K / 2; ++j) {
            uint8_t b = p[r * (K / 2) + j];
            q[r * K + 2 * j] = (int8_t)nibble_to_int(b);
            q[r * K + 2 * j + 1] = (int8_t)nibble_to_int(b >> 4);
        }
    return 0;
}

/* ----------------------------------------------------------------------- */
/* Integer GEMM and epilogue.                                                */
/* ----------------------------------------------------------------------- */

/* acc[m][n] = sum_k qx[m][k] * qw[n][k]; both operands packed [rows][K/2]. */
int oracle_gemm(const uint8_t *qx, const uint8_t *qw, int64_t M, int64_t N, int64_t K,
                int64_t *acc) {
    if (!qx || !qw || !acc || M < 0 || N < 0 || K <= 0 || K % 2) return -1;
    int8_t *a = (int8_t *)malloc((size_t)M * (size_t)K + 1);
    int8_t *b = (int8_t *)malloc((size_t)N * (size_t)K + 1);
    if (!a || !b) { free(a); free(b); return -2; }
    oracle_unpack(qx, M, K, a);
    oracle_unpack(qw, N, K, b);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)a[m * K + k] * (int64_t)b[n * K + k];
            acc[m * N + n] = s;
        }
    }
    free(a);
    free(b);
    return 0;
}

/* y[m][n] = bf16_rne( ((float)acc * sx[m]) * sw[n] + (float)bias[n] ), fp32,
 * no fused multiply-add; bias may be NULL (zeros). */
int oracle_epilogue(const int64_t *acc, const float *sx, const float *sw, const uint16_t *bias,
                    int64_t M, int64_t N, uint16_t *y) {
    if (!acc || !sx || !sw || !y || M < 0 || N < 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float t = (float)acc[m * N + n];
            t = t * sx[m];
            t = t * sw[n];
            float b = bias ? (float)bf16_bits_to_double(bias[n]) : 0.0f;
            t = t + b;
            y[m * N + n] = float_to_bf16_bits_rne(t);
        }
    return 0;
}

/* ----------------------------------------------------------------------- */
/* Composite steps.                                                          */
/* ----------------------------------------------------------------------- */

/* Rotate, quantise and pack rows of a bf16 matrix: the per-row preparation
 * shared by weights (offline) and activations (per call). */
int oracle_prepare_rows(const uint16_t *x, int64_t rows, int64_t K, int n, uint8_t *packed,
                        float *scale) {
    if (!x || !packed || !scale || rows < 0 || K <= 0 || log4_exact(n) < 0 || K % n) return -1;
    if (rows == 0) return 0;
    double *y = (double *)malloc(sizeof(double) * (size_t)rows * (size_t)K);
    int8_t *q = (int8_t *)malloc((size_t)rows * (size_t)K);
    if (!y || !q) { free(y); free(q); return -2; }
    int rc = oracle_rotate(x, rows, K, n, y);
    if (!rc) rc = oracle_quantize_rows(y, rows, K, q, scale);
    if (!rc) rc = oracle_pack(q, rows, K, packed);
    free(y);
    free(q);
    return rc;
}

/* The whole layer on bf16 inputs: prepare x, take the prepared weights, run
 * the integer product and the epilogue. */
int oracle_linear_prepared_w(const uint16_t *x, const uint8_t *qw, const float *sw,
                             const uint16_t *bias, int64_t M, int64_t N, int64_t K, int n,
                             uint16_t *y) {
    if (!x || !qw || !sw || !y || M < 0 || N < 0 || K <= 0) return -1;
    if (M == 0 || N == 0) return 0;
    uint8_t *qx = (uint8_t *)malloc((size_t)M * (size_t)(K / 2));
    float *sx = (float *)malloc(sizeof(float) * (size_t)M);
    int64_t *acc = (int64_t *)malloc(sizeof(int64_t) * (size_t)M * (size_t)N);
    if (!qx || !sx || !acc) { free(qx); free(sx); free(acc); return -2; }
    int rc = oracle_prepare_rows(x, M, K, n, qx, sx);
    if (!rc) rc = oracle_gemm(qx, qw, M, N, K, acc);
    if (!rc) rc = oracle_epilogue(acc, sx, sw, bias, M, N, y);
    free(qx);
    free(sx);
    free(acc);
    return rc;
}

/* ----------------------------------------------------------------------- */
/* The W4A16 variant.                                                        */
/* ----------------------------------------------------------------------- */

/* Round a finite double to the nearest bf16 (8 significant bits), ties to
 * even, in one step: scale |v| by a power of two so that the bf16 spacing
 * becomes 1, round that to an integer, scale back.  (Going through fp32
 * first would round twice.)  Below the normal range the spacing is that of
 * the subnormals, 2^-133; above it the result overflows to infinity. */
static uint16_t double_to_bf16_bits_rne(double v) {
    if (v == 0.0) return signbit(v) ? (uint16_t)0x8000u : (uint16_t)0;
    if (!isfinite(v)) return float_to_bf16_bits_rne((float)v);
    double a = fabs(v);
    int e;
    frexp(a, &e);                        /* a = f 2^e, 0.5 <= f < 1 */
    int q = e - 8;                       /* spacing 2^(e-1) * 2^-7 */
    if (e - 1 < -126) q = -133;          /* subnormal spacing */
    double scaled = ldexp(a, -q);        /* exact */
    double f = floor(scaled);
    double frac = scaled - f;            /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;
    float rf = (float)ldexp(f, q);       /* exact: at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    uint16_t h = (uint16_t)(u >> 16);
    return v < 0.0 ? (uint16_t)(h | 0x8000u) : h;
}

int oracle_round_bf16(const double *in, int64_t count, uint16_t *out) {
    if (!in || !out || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) out[i] = double_to_bf16_bits_rne(in[i]);
    return 0;
}

/* xr = bf16_rne(x R): the fp64 rotation above, each value rounded once. */
int oracle_w4a16_rotate_act(const uint16_t *x, int64_t rows, int64_t K, int n, uint16_t *xr) {
    if (!x || !xr || rows < 0 || K <= 0 || log4_exact(n) < 0 || K % n) return -1;
    if (rows == 0) return 0;
    double *y = (double *)malloc(sizeof(double) * (size_t)rows * (size_t)K);
    if (!y) return -2;
    int rc = oracle_rotate(x, rows, K, n, y);
    if (!rc) rc = oracle_round_bf16(y, rows * K, xr);
    free(y);
    return rc;
}

/* acc[m][n] = sum_k xr[m][k] q[n][k] in fp64 (every product is exact; so is
 * the sum while the row's values span fewer than about 40 binades), and two
 * magnitudes that bound the rounding of any evaluation that adds the terms
 * in K order, 16 at a time:
 *   l1[m][n]  = sum_k |xr[m][k] q[n][k]|,
 *   p16[m][n] = sum_j |partial sum over k < min(16 j, K)|, j = 1 .. ceil(K/16).
 * l1 and p16 may be NULL. */
int oracle_w4a16_gemm(const uint16_t *xr, const uint8_t *qw, int64_t M, int64_t N, int64_t K,
                      double *acc, double *l1, double *p16) {
    if (!xr || !qw || !acc || M < 0 || N < 0 || K <= 0 || K % 2) return -1;
    int8_t *b = (int8_t *)malloc((size_t)N * (size_t)K + 1);
    double *a = (double *)malloc(sizeof(double) * ((size_t)M * (size_t)K + 1));
    if (!a || !b) { free(a); free(b); return -2; }
    oracle_unpack(qw, N, K, b);
    for (int64_t i = 0; i < M * K; ++i) a[i] = bf16_bits_to_double(xr[i]);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0, s1 = 0.0, sp = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double t = a[m * K + k] * (double)b[n * K + k];
                s += t;
                s1 += fabs(t);
                if (k % 16 == 15 || k == K - 1) sp += fabs(s);
            }
            acc[m * N + n] = s;
            if (l1) l1[m * N + n] = s1;
            if (p16) p16[m * N + n] = sp;
        }
    }
    free(a);
    free(b);
    return 0;
}

/* t[m][n] = acc[m][n] * sw[n] + b[n] in fp64 and y = bf16_rne(t); bias may
 * be NULL (zeros); t may be NULL. */
int oracle_w4a16_epilogue(const double *acc, const float *sw, const uint16_t *bias, int64_t M,
                          int64_t N, double *t, uint16_t *y) {
    if (!acc || !sw || !y || M < 0 || N < 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v = acc[m * N + n] * (double)sw[n];
            v += bias ? bf16_bits_to_double(bias[n]) : 0.0;
            if (t) t[m * N + n] = v;
            y[m * N + n] = double_to_bf16_bits_rne(v);
        }
    return 0;
}

/* The whole W4A16 layer on bf16 inputs, given the prepared weights. */
int oracle_w4a16_linear(const uint16_t *x, const uint8_t *qw, const float *sw,
                        const uint16_t *bias, int64_t M, int64_t N, int64_t K, int n,
                        uint16_t *y) {
    if (!x || !qw || !sw || !y || M < 0 || N < 0 || K <= 0) return -1;
    if (M == 0 || N == 0) return 0;
    uint16_t *xr = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)M * (size_t)K);
    double *acc = (double *)malloc(sizeof(double) * (size_t)M * (size_t)N);
    if (!xr || !acc) { free(xr); free(acc); return -2; }
    int rc = oracle_w4a16_rotate_act(x, M, K, n, xr);
    if (!rc) rc = oracle_w4a16_gemm(xr, qw, M, N, K, acc, NULL, NULL);
    if (!rc) rc = oracle_w4a16_epilogue(acc, sw, bias, M, N, NULL, y);
    free(xr);
    free(acc);
    return rc;
}

/* ----------------------------------------------------------------------- */
/* The reversible weight repack.                                            */
/* ----------------------------------------------------------------------- */

/* "convrot-mlx" README, "What is included" (lossless repacking of the
 * packed weights for the kernels that read them) and "Install and test"
 * (repack_nk_weight_for_mpp).  The pages repack for Apple's layout; the
 * reading taken here: the same bytes, reordered without loss into the order
 * the reading kernel streams them.  The canonical layout is N x packed-K
 * (row n holds bytes 0 .. K/2 - 1).  The repacked one cuts every row into
 * 128-byte column blocks (256 codes) and stores block b of all rows before
 * block b + 1:
 *     rep[(b * N + n) * 128 + j] = qw[n * (K/2) + b * 128 + j]
 * for b < ceil(K / 256), j < 128; bytes past the end of a row (K not a
 * multiple of 256) are zero. */
int oracle_repack_weight(const uint8_t *qw, int64_t N, int64_t K, uint8_t *rep) {
    if (!qw || !rep || N < 0 || K <= 0 || K % 2) return -1;
    const int64_t row = K / 2, nblk = (row + 127) / 128;
    for (int64_t b = 0; b < nblk; ++b)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < 128; ++j) {
                const int64_t c = b * 128 + j;
                rep[(b * N + n) * 128 + j] = c < row ? qw[n * row + c] : 0;
            }
    return 0;
}

/* The inverse: qw[n * (K/2) + c] = rep[((c / 128) * N + n) * 128 + c % 128]. */
int oracle_unpack_weight(const uint8_t *rep, int64_t N, int64_t K, uint8_t *qw) {
    if (!qw || !rep || N < 0 || K <= 0 || K % 2) return -1;
    const int64_t row = K / 2;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t c = 0; c < row; ++c)
            qw[n * row + c] = rep[((c / 128) * N + n) * 128 + c % 128];
    return 0;
}

/* ----------------------------------------------------------------------- */
/* The NVFP4 variant.                                                       */
/* ----------------------------------------------------------------------- */

/* E2M1 (4-bit float): bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa; codes 0..7 are the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_value(unsigned code) {
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[code & 7u];
    return (code & 8u) ? -v : v;
}

/* Nearest E2M1 value by search over the eight magnitudes, ties to the even
 * code (mantissa bit 0), magnitudes past 6 to 6 (saturation); the sign bit
 * of v is kept, so a negative value that rounds to zero gives code 8. */
static unsigned e2m1_round(float v) {
    double a = fabs((double)v), bd = INFINITY;
    unsigned best = 0;
    for (unsigned c = 0; c < 8; ++c) {
        double d = fabs(a - e2m1_value(c));
        if (d < bd || (d == bd && (c & 1u) == 0)) {
            best = c;
            bd = d;
        }
    }
    return (signbit(v) ? 8u : 0u) | best;
}

/* Unsigned E4M3 scale: bits 6..3 exponent (bias 7), bits 2..0 mantissa;
 * exponent 0 is subnormal (m 2^-9); code 127 is not a number (not used).
 * The largest value, code 126, is 448. */
static double e4m3_value(unsigned code) {
    unsigned e = (code >> 3) & 15u, m = code & 7u;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp((double)(8u + m), (int)e - 10);
}

/* Nearest E4M3 value of a non-negative v by search over codes 0..126, ties
 * to the even code, values past 448 to 448 (saturation). */
static unsigned e4m3_round(float v) {
    double a = (double)v, bd = INFINITY;
    unsigned best = 0;
    for (unsigned c = 0; c < 127; ++c) {
        double d = fabs(a - e4m3_value(c));
        if (d < bd || (d == bd && (c & 1u) == 0)) {
            best = c;
            bd = d;
        }
    }
    return best;
}

int oracle_e2m1_round(const float *v, int64_t count, uint8_t *codes) {
    if (!v || !codes || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) codes[i] = (uint8_t)e2m1_round(v[i]);
    return 0;
}

int oracle_e4m3_round(const float *v, int64_t count, uint8_t *codes) {
    if (!v || !codes || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) {
        if (!(v[i] >= 0.0f)) return -1;
        codes[i] = (uint8_t)e4m3_round(v[i]);
    }
    return 0;
}

int oracle_e2m1_value(const uint8_t *codes, int64_t count, double *v) {
    if (!v || !codes || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) v[i] = e2m1_value(codes[i]);
    return 0;
}

int oracle_e4m3_value(const uint8_t *codes, int64_t count, double *v) {
    if (!v || !codes || count < 0) return -1;
    for (int64_t i = 0; i < count; ++i) {
        if (codes[i] > 126) return -1;
        v[i] = e4m3_value(codes[i]);
    }
    return 0;
}

/* NVFP4 quantisation of rotated rows.  The NVFP4 format (E2M1 elements, one
 * E4M3 scale per 16 elements, one fp32 scale above it) is named by the pages
 * ("convrot-mlx" README, "Why this repository exists": the official
 * implementation targets NVFP4 on Blackwell) but not spelled out; the
 * plainest reading, with the row as the unit of the fp32 scale as in the
 * W4A4 quantiser, decided in fp32:
 *   a    = fp32(max_k |y_k|),  s = a / 2688 (6 x 448, so the block scales
 *          span E4M3 up to 448), r = 448 / a;  a == 0 gives s = r = 0;
 *   per block b of 16: a_b = fp32(max |y_k|), sf_b = e4m3(a_b * r),
 *   d_b  = fp32(value(sf_b) * s), inv_b = 1 / d_b (0 when d_b == 0),
 *   q_k  = e2m1(fp32(y_k) * inv_b).
 * Outputs: codes, one per byte [rows][K]; sf [rows][K/16] (E4M3 codes);
 * s [rows]. */
int oracle_nvfp4_quantize_rows(const double *y, int64_t rows, int64_t K, uint8_t *codes,
                               uint8_t *sf, float *s) {
    if (!y || !codes || !sf || !s || rows < 0 || K <= 0 || K % 16) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *yr = y + r * K;
        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k)
            if (fabs(yr[k]) > amax) amax = fabs(yr[k]);
        const float a = (float)amax;
        const float sr = a > 0.0f ? a / 2688.0f : 0.0f;
        const float rr = a > 0.0f ? 448.0f / a : 0.0f;
        s[r] = sr;
        for (int64_t b = 0; b < K / 16; ++b) {
            double bmax = 0.0;
            for (int64_t k = 16 * b; k < 16 * b + 16; ++k)
                if (fabs(yr[k]) > bmax) bmax = fabs(yr[k]);
            const float t = (float)bmax * rr;
            const unsigned c = e4m3_round(t);
            sf[r * (K / 16) + b] = (uint8_t)c;
            const float d = (float)e4m3_value(c) * sr;
            const float inv = d > 0.0f ? 1.0f / d : 0.0f;
            for (int64_t k = 16 * b; k < 16 * b + 16; ++k)
                codes[r * K + k] = (uint8_t)e2m1_round((float)yr[k] * inv);
        }
    }
    return 0;
}

/* Two E2M1 codes per byte, low nibble = even k (as the INT4 packing). */
int oracle_nvfp4_pack(const uint8_t *codes, int64_t rows, int64_t K, uint8_t *p) {
    if (!codes || !p || rows < 0 || K <= 0 || K % 2) return -1;
    for (int64_t i = 0; i < rows * (K / 2); ++i)
        p[i] = (uint8_t)((codes[2 * i] & 0xFu) | ((codes[2 * i + 1] & 0xFu) << 4));
    return 0;
}

/* The block-scale storage layout of the GPU boundary (include/convrot_nvfp4.h):
 * 512-byte atoms of 128 rows x 4 blocks, atom (row / 128, block / 4) at
 * ((row / 128) * (K / 64) + block / 4) * 512, and inside an atom row r,
 * block j at 16 (r mod 32) + 4 (r / 32 mod 4) + j.  rows are padded to a
 * multiple of 128 (padding bytes 0).  sf: [rows][K/16] row-major. */
int oracle_nvfp4_sf_layout(const uint8_t *sf, int64_t rows, int64_t K, uint8_t *out) {
    if (!sf || !out || rows < 0 || K <= 0 || K % 64) return -1;
    const int64_t tiles = (rows + 127) / 128, ka = K / 64;
    memset(out, 0, (size_t)(tiles * 128 * (K / 16)));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 16; ++b) {
            const int64_t atom = (r / 128) * ka + b / 4;
            const int64_t rr = r % 128;
            out[atom * 512 + 16 * (rr % 32) + 4 * (rr / 32) + b % 4] = sf[r * (K / 16) + b];
        }
    return 0;
}

/* acc[m][n] = sum over blocks b of value(sfx[m][b]) value(sfw[n][b])
 *             sum_{k in b} e2m1(qx[m][k]) e2m1(qw[n][k])    (fp64, exact:
 * every product has at most 12 significant bits and the sums stay far below
 * 2^53 of its spacing), plus l1 = the sum of the |terms| and p64 = the sum
 * of |running sums| at every 64th k, for the accumulation bound.  Packed
 * codes [rows][K/2], block scales row-major [rows][K/16]. */
int oracle_nvfp4_gemm(const uint8_t *qx, const uint8_t *sfx, const uint8_t *qw,
                      const uint8_t *sfw, int64_t M, int64_t N, int64_t K, double *acc,
                      double *l1, double *p64) {
    if (!qx || !sfx || !qw || !sfw || !acc || M < 0 || N < 0 || K <= 0 || K % 64) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0, a1 = 0.0, pr = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                const unsigned cx = (qx[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xFu;
                const unsigned cw = (qw[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xFu;
                const double t = e2m1_value(cx) * e2m1_value(cw) *
                                 e4m3_value(sfx[m * (K / 16) + k / 16]) *
                                 e4m3_value(sfw[n * (K / 16) + k / 16]);
                sum += t;
                a1 += fabs(t);
                if (k % 64 == 63) pr += fabs(sum);
            }
            acc[m * N + n] = sum;
            if (l1) l1[m * N + n] = a1;
            if (p64) p64[m * N + n] = pr;
        }
    return 0;
}

/* t = acc sx sw + b exactly (fp64) and y = bf16_rne(t). */
int oracle_nvfp4_epilogue(const double *acc, const float *sx, const float *sw,
                          const uint16_t *bias, int64_t M, int64_t N, double *t, uint16_t *y) {
    if (!acc || !sx || !sw || !y || M < 0 || N < 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v = acc[m * N + n] * (double)sx[m] * (double)sw[n];
            v += bias ? bf16_bits_to_double(bias[n]) : 0.0;
            if (t) t[m * N + n] = v;
            y[m * N + n] = double_to_bf16_bits_rne(v);
        }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int t) {
#ifdef _OPENMP
    if (t > 0) omp_set_num_threads(t);
#else
    (void)t;
#endif
}
