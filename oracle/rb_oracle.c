/*
 * rb_oracle.c -- plain, slow, obviously-correct CPU oracle for the residual
 * dual-scale binarized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA library.
 *
 * Method (RaBiT: Residual-Aware Binarization Training, "Residual binarization"
 * and "Core method" sections; Algorithm 2, forward pass):
 *   W ~= sum_{i=1..k} diag(g_i) B_i diag(h_i),  B_i in {-1,+1}^{N x K}
 *   R_0 = W;  B_i = sign(R_{i-1}) with sign(0) = +1;
 *   R_i = R_{i-1} - (g_i h_i^T) .* B_i
 *   Y = sum_i g_i .* (B_i (h_i .* X))      ("matmul-free" evaluation)
 *
 * Readings taken where the pages leave a step open (each is listed in the
 * design notes):
 *   - the residual update runs in IEEE fp32: t = fl(g_i[r]*h_i[c]) (one
 *     rounding), then R = fl(R - t) if B = +1 else fl(R + t); no fused
 *     multiply-add.  The fp32 scales given by the caller are used, not their
 *     fp16 copies.
 *   - sign(0) = +1 includes -0.0 (the test is R >= 0); this is the tie rule of
 *     the binary-codebook page (BTC-LLM, binary k-means M-step: a zero
 *     centroid entry becomes +1).
 *   - bit = 1 <=> B = +1; 32 consecutive input columns per uint32 word with
 *     column c at bit c % 32 ("32 columns packed into one uint32_t", RaBiT,
 *     technical novelty paragraph).
 *   - word order (this library's storage format; the pages fix only the
 *     32-columns-per-word packing): plane i is cut into S = ceil(K/256)
 *     column slices and Nt = ceil(N/32) tiles of 32 rows; each
 *     (plane, slice, tile) block has 256 words and
 *        word(i, s, r, w) = (((i*S + s)*Nt + r/32)*256)
 *                           + (w ^ ((r%32)/4))*32 + r%32
 *     holds columns 256*s + 32*w .. +31 of row r (w = 0..7).  Bits of
 *     columns >= K and words of rows >= N are zero.
 *   - stored scales are fp16, rounded to nearest-even from the fp32 inputs.
 *   - the greedy SVID initialiser (Greedy SVID, named in the technical
 *     novelty paragraph) takes, per plane, the rank-1 approximation of
 *     |R_{i-1}| by power iteration in float64: v0 = 1/sqrt(K), then `iters`
 *     rounds of u = A v / |A v|, v = A^T u / |A^T u|; sigma = u^T A v;
 *     g_i = fp32(sqrt(sigma) u), h_i = fp32(sqrt(sigma) v).
 *   - the iterative residual SVID (RaBiT, Algorithm 1, without the I/O
 *     channel preprocessing, i.e. the alpha = 0 form) starts from the greedy
 *     scales and the signs of the greedy recurrence, then runs `sweeps`
 *     Gauss-Seidel sweeps: for i = 1..k the target of plane i is
 *     T_i = W - sum_{j != i} diag(g_j) B_j diag(h_j) with the latest values of
 *     the other planes, B_i = sign(T_i) and (g_i, h_i) = the rank-1 of |T_i|
 *     by the same power iteration.  T_i is formed in float64: each term
 *     g_j[r]*h_j[c] is exact there and is subtracted in plane order j = 1..k.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math);
 * on x86-64 float arithmetic is SSE single precision, so every fp32 step
 * above rounds exactly once.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Number formats (IEEE 754 binary16, bfloat16), round-to-nearest-even */
/* ------------------------------------------------------------------ */

/* Round a double to a binary format with p significand bits (implicit bit
 * included), minimum normal exponent emin and maximum exponent emax.
 * Subnormals keep the fixed quantum 2^(emin-p+1); results that round to
 * 2^(emax+1) or above overflow to infinity. */
static double round_to_format(double v, int p, int emin, int emax)
{
    if (v != v || isinf(v) || v == 0.0) return v;
    double a = fabs(v);
    int e;
    frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1): floor(log2 a) = e-1 */
    int E = e - 1;
    if (E < emin) E = emin;
    double q = ldexp(1.0, E - p + 1);
    double r = rint(a / q) * q;          /* a/q is exact; rint rounds half to even */
    if (r >= ldexp(1.0, emax + 1)) r = INFINITY;
    return copysign(r, v);
}

static uint16_t encode_binary16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (v != v) return 0x7e00u;
    double r = round_to_format(v, 11, -14, 15);
    double a = fabs(r);
    if (isinf(a)) return sign | 0x7c00u;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14))                       /* subnormal: m * 2^-24 */
        return sign | (uint16_t)(a / ldexp(1.0, -24));
    int e;
    frexp(a, &e);
    int E = e - 1;
    uint32_t mant = (uint32_t)(a / ldexp(1.0, E - 10)) - 1024u;
    return sign | (uint16_t)(((uint32_t)(E + 15) << 10) | mant);
}

static double decode_binary16(uint16_t b)
{
    int sign = (b >> 15) & 1, ex = (b >> 10) & 31, m = b & 1023;
    double v;
    if (ex == 31) v = m ? NAN : INFINITY;
    else if (ex == 0) v = ldexp((double)m, -24);
    else v = ldexp((double)(1024 + m), ex - 25);
    return sign ? -v : v;
}

static uint16_t encode_bfloat16(double v)
{
    if (v != v) return 0x7fc0u;
    double r = round_to_format(v, 8, -126, 127);
    float f = (float)r;                 /* exact: every bfloat16 value is a float */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static double decode_bfloat16(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* OpenMP threads a parallel region of this library runs on (for reporting). */
int oracle_threads(void) { return omp_get_max_threads(); }

/* Thread count of later parallel regions started from the calling thread. */
void oracle_set_threads(int n) { if (n > 0) omp_set_num_threads(n); }

uint16_t oracle_f64_to_f16(double v) { return encode_binary16(v); }
double oracle_f16_to_f64(uint16_t b) { return decode_binary16(b); }
uint16_t oracle_f64_to_bf16(double v) { return encode_bfloat16(v); }
double oracle_bf16_to_f64(uint16_t b) { return decode_bfloat16(b); }

/* ------------------------------------------------------------------ */
/* Storage layout                                                       */
/* ------------------------------------------------------------------ */

int64_t oracle_plane_words(int64_t N, int64_t K, int k)
{
    int64_t S = (K + 255) / 256, Nt = (N + 31) / 32;
    return (int64_t)k * S * Nt * 256;
}

static int64_t word_index(int64_t N, int64_t K, int i, int64_t r, int64_t c)
{
    int64_t S = (K + 255) / 256, Nt = (N + 31) / 32;
    int64_t s = c / 256, w = (c % 256) / 32, rho = r % 32;
    int64_t block = ((int64_t)i * S + s) * Nt + r / 32;
    return block * 256 + (w ^ (rho / 4)) * 32 + rho;
}

/* ------------------------------------------------------------------ */
/* Derivation + packing (Algorithm 2 forward, fp32 recurrence)          */
/* ------------------------------------------------------------------ */

/* Return codes: 0 ok, -1 bad argument, 1 non-finite W/g/h, 2 a scale
 * overflows fp16. Outputs are written in all non-negative-error cases. */
static int check_args(int64_t N, int64_t K, int k)
{
    if (N < 1 || K < 32 || K % 32 != 0 || k < 1 || k > 8) return -1;
    return 0;
}

/* Derive and pack one row r (row-local residual, length K). bits_out gets
 * the k*K bits of the row in [i][c] order (1 = +1). */
static void derive_row(const float *Wr, const float *g, const float *h,
                       int64_t N, int64_t K, int k, int64_t r,
                       float *R, unsigned char *bits_out)
{
    for (int64_t c = 0; c < K; ++c) R[c] = Wr[c];
    for (int i = 0; i < k; ++i) {
        float gi = g[(int64_t)i * N + r];
        for (int64_t c = 0; c < K; ++c) {
            int b = (R[c] >= 0.0f);             /* sign(0) = +1, -0.0 included */
            float t = gi * h[(int64_t)i * K + c];   /* one fp32 rounding */
            R[c] = b ? (R[c] - t) : (R[c] + t);     /* a second, separate rounding */
            bits_out[(int64_t)i * K + c] = (unsigned char)b;
        }
    }
}

static int scan_inputs(const float *W, const float *g, const float *h,
                       int64_t N, int64_t K, int k, uint16_t *g16, uint16_t *h16)
{
    int st = 0;
    for (int64_t x = 0; x < N * K; ++x)
        if (!isfinite(W[x])) st = 1;
    for (int64_t x = 0; x < (int64_t)k * N; ++x) {
        if (!isfinite(g[x])) st = 1;
        uint16_t e = encode_binary16((double)g[x]);
        if (isfinite(g[x]) && (e & 0x7c00u) == 0x7c00u && st == 0) st = 2;
        if (g16) g16[x] = e;
    }
    for (int64_t x = 0; x < (int64_t)k * K; ++x) {
        if (!isfinite(h[x])) st = 1;
        uint16_t e = encode_binary16((double)h[x]);
        if (isfinite(h[x]) && (e & 0x7c00u) == 0x7c00u && st == 0) st = 2;
        if (h16) h16[x] = e;
    }
    return st;
}

/* Full pack. planes has oracle_plane_words(N,K,k) words. R_out (nullable,
 * [N][K]) receives the final residual R_k. */
int oracle_pack(const float *W, const float *g, const float *h,
                int64_t N, int64_t K, int k,
                uint32_t *planes, uint16_t *g16, uint16_t *h16, float *R_out)
{
    if (check_args(N, K, k)) return -1;
    int st = scan_inputs(W, g, h, N, K, k, g16, h16);
    memset(planes, 0, sizeof(uint32_t) * (size_t)oracle_plane_words(N, K, k));
    #pragma omp parallel
    {
        float *R = (float *)malloc(sizeof(float) * (size_t)K);
        unsigned char *bits = (unsigned char *)malloc((size_t)k * (size_t)K);
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < N; ++r) {
            derive_row(W + r * K, g, h, N, K, k, r, R, bits);
            for (int i = 0; i < k; ++i)
                for (int64_t c = 0; c < K; ++c)
                    if (bits[(int64_t)i * K + c])
                        planes[word_index(N, K, i, r, c)] |= (uint32_t)1u << (c % 32);
            if (R_out) memcpy(R_out + r * K, R, sizeof(float) * (size_t)K);
        }
        free(R);
        free(bits);
    }
    return st;
}

/* Pack only the listed rows (for sampled checks at full size). Output is
 * row-local: words_out[j][i][s][w] for the j-th listed row, S = ceil(K/256). */
int oracle_pack_rows(const float *W, const float *g, const float *h,
                     int64_t N, int64_t K, int k,
                     const int64_t *rows, int64_t nrows, uint32_t *words_out)
{
    if (check_args(N, K, k)) return -1;
    int64_t S = (K + 255) / 256;
    memset(words_out, 0, sizeof(uint32_t) * (size_t)(nrows * k * S * 8));
    float *R = (float *)malloc(sizeof(float) * (size_t)K);
    unsigned char *bits = (unsigned char *)malloc((size_t)k * (size_t)K);
    for (int64_t j = 0; j < nrows; ++j) {
        int64_t r = rows[j];
        derive_row(W + r * K, g, h, N, K, k, r, R, bits);
        for (int i = 0; i < k; ++i)
            for (int64_t c = 0; c < K; ++c)
                if (bits[(int64_t)i * K + c])
                    words_out[((j * k + i) * S + c / 256) * 8 + (c % 256) / 32] |=
                        (uint32_t)1u << (c % 32);
    }
    free(R);
    free(bits);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Application: dequantise the stored representation, then multiply      */
/* ------------------------------------------------------------------ */

/* Y[m][n] = sum_c X[m][c] * What[n][c] in float64 with
 * What[n][c] = sum_i f16(g16_i[n]) * (bit ? +1 : -1) * f16(h16_i[c]).
 * rows / toks (nullable) select the outputs; Y is [ntoks][nrows]. */
void oracle_apply(const uint32_t *planes, const uint16_t *g16, const uint16_t *h16,
                  int64_t N, int64_t K, int k,
                  const uint16_t *X, int64_t M,
                  const int64_t *rows, int64_t nrows,
                  const int64_t *toks, int64_t ntoks, double *Y)
{
    if (!rows) nrows = N;
    if (!toks) ntoks = M;
    double *hd = (double *)malloc(sizeof(double) * (size_t)(k * K));
    for (int64_t x = 0; x < (int64_t)k * K; ++x) hd[x] = decode_binary16(h16[x]);
    #pragma omp parallel
    {
        double *What = (double *)malloc(sizeof(double) * (size_t)K);
        #pragma omp for schedule(dynamic, 4)
        for (int64_t j = 0; j < nrows; ++j) {
            int64_t n = rows ? rows[j] : j;
            for (int64_t c = 0; c < K; ++c) What[c] = 0.0;
            for (int i = 0; i < k; ++i) {
                double gi = decode_binary16(g16[(int64_t)i * N + n]);
                for (int64_t c = 0; c < K; ++c) {
                    uint32_t word = planes[word_index(N, K, i, n, c)];
                    double s = ((word >> (c % 32)) & 1u) ? 1.0 : -1.0;
                    What[c] += gi * s * hd[(int64_t)i * K + c];
                }
            }
            for (int64_t t = 0; t < ntoks; ++t) {
                int64_t m = toks ? toks[t] : t;
                double acc = 0.0;
                for (int64_t c = 0; c < K; ++c)
                    acc += decode_bfloat16(X[m * K + c]) * What[c];
                Y[t * nrows + j] = acc;
            }
        }
        free(What);
    }
    free(hd);
}

/* ------------------------------------------------------------------ */
/* Transposed layer and the input gradient (backward data path)          */
/* ------------------------------------------------------------------ */

/* Sign planes of the transposed layer: bit (i, c, r) of the K x N layer
 * equals bit (i, r, c) of the N x K layer, written in the same storage
 * layout (with N and K exchanged).  The scales of the transposed layer are
 * the original ones exchanged, g' = h and h' = g, since
 * What^T[c][r] = sum_i h_i[c] * B_i[r][c] * g_i[r].  out must hold
 * oracle_plane_words(K, N, k) words and is cleared first. */
void oracle_transpose_planes(const uint32_t *planes, int64_t N, int64_t K, int k, uint32_t *out)
{
    int64_t nw = oracle_plane_words(K, N, k);
    for (int64_t x = 0; x < nw; ++x) out[x] = 0u;
    for (int i = 0; i < k; ++i)
        for (int64_t r = 0; r < N; ++r)
            for (int64_t c = 0; c < K; ++c) {
                uint32_t bit = (planes[word_index(N, K, i, r, c)] >> (c % 32)) & 1u;
                out[word_index(K, N, i, c, r)] |= bit << (r % 32);
            }
}

/* Input gradient of Y = X What^T (RaBiT, Algorithm 2 backward: the gradient
 * reaching the layer input): dX[m][c] = sum_n dY[m][n] * What[n][c] in
 * float64, What dequantised from the stored representation as in
 * oracle_apply.  dY is [M][N] bfloat16 bit patterns; dX is [M][K]. */
void oracle_apply_t(const uint32_t *planes, const uint16_t *g16, const uint16_t *h16,
                    int64_t N, int64_t K, int k,
                    const uint16_t *dY, int64_t M, double *dX)
{
    #pragma omp parallel
    {
        double *What = (double *)malloc(sizeof(double) * (size_t)N);
        #pragma omp for schedule(dynamic, 4)
        for (int64_t c = 0; c < K; ++c) {
            for (int64_t n = 0; n < N; ++n) What[n] = 0.0;
            for (int i = 0; i < k; ++i) {
                double hc = decode_binary16(h16[(int64_t)i * K + c]);
                for (int64_t n = 0; n < N; ++n) {
                    uint32_t word = planes[word_index(N, K, i, n, c)];
                    double s = ((word >> (c % 32)) & 1u) ? 1.0 : -1.0;
                    What[n] += decode_binary16(g16[(int64_t)i * N + n]) * s * hc;
                }
            }
            for (int64_t m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    acc += decode_bfloat16(dY[m * N + n]) * What[n];
                dX[m * K + c] = acc;
            }
        }
        free(What);
    }
}

/* ------------------------------------------------------------------ */
/* Coupled training: gradients of one layer (Algorithm 2 backward)       */
/* ------------------------------------------------------------------ */

/* Gradients of a loss L through Y = X What^T with What = sum_i diag(g_i) B_i
 * diag(h_i) (RaBiT, Algorithm 2: the signs B_i are derived on the fly from W
 * by the fp32 recurrence of oracle_pack and held constant in the backward
 * pass; the latent weight takes the effective-weight gradient).  Given
 * dY = dL/dY, in float64:
 *   G[n][c]  = sum_m dY[m][n] X[m][c]              (dL/dWhat = dY^T X)
 *   dW       = G
 *   dg_i[n]  = sum_c G[n][c] B_i[n][c] h_i[c]
 *   dh_i[c]  = sum_n G[n][c] g_i[n] B_i[n][c]
 *   dX[m][c] = sum_n dY[m][n] What[n][c]           (fp32 scales, as trained)
 * X [M][K] and dY [M][N] are bfloat16 bit patterns; dW [N][K] and dX [M][K]
 * are nullable; dg [k][N], dh [k][K].  Returns oracle_pack's status codes
 * (-1 bad arguments, 1 non-finite input; fp16 range is not checked here). */
int oracle_qat_backward(const float *W, const float *g, const float *h,
                        int64_t N, int64_t K, int k,
                        const uint16_t *X, const uint16_t *dY, int64_t M,
                        double *dW, double *dg, double *dh, double *dX)
{
    if (check_args(N, K, k) || M < 1) return -1;
    int st = scan_inputs(W, g, h, N, K, k, NULL, NULL) == 1 ? 1 : 0;
    unsigned char *B = (unsigned char *)malloc((size_t)k * (size_t)N * (size_t)K);
    double *G = (double *)malloc(sizeof(double) * (size_t)(N * K));
    #pragma omp parallel
    {
        float *R = (float *)malloc(sizeof(float) * (size_t)K);
        unsigned char *bits = (unsigned char *)malloc((size_t)k * (size_t)K);
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < N; ++r) {
            derive_row(W + r * K, g, h, N, K, k, r, R, bits);
            for (int i = 0; i < k; ++i)
                memcpy(B + ((int64_t)i * N + r) * K, bits + (int64_t)i * K, (size_t)K);
            for (int64_t c = 0; c < K; ++c) {
                double acc = 0.0;
                for (int64_t m = 0; m < M; ++m)
                    acc += decode_bfloat16(dY[m * N + r]) * decode_bfloat16(X[m * K + c]);
                G[r * K + c] = acc;
            }
        }
        free(R);
        free(bits);
    }
    if (dW) memcpy(dW, G, sizeof(double) * (size_t)(N * K));
    for (int i = 0; i < k; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t c = 0; c < K; ++c) {
                double s = B[((int64_t)i * N + n) * K + c] ? 1.0 : -1.0;
                acc += G[n * K + c] * s * (double)h[(int64_t)i * K + c];
            }
            dg[(int64_t)i * N + n] = acc;
        }
        for (int64_t c = 0; c < K; ++c) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double s = B[((int64_t)i * N + n) * K + c] ? 1.0 : -1.0;
                acc += G[n * K + c] * (double)g[(int64_t)i * N + n] * s;
            }
            dh[(int64_t)i * K + c] = acc;
        }
    }
    if (dX) {
        for (int64_t m = 0; m < M; ++m)
            for (int64_t c = 0; c < K; ++c) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double w = 0.0;
                    for (int i = 0; i < k; ++i) {
                        double s = B[((int64_t)i * N + n) * K + c] ? 1.0 : -1.0;
                        w += (double)g[(int64_t)i * N + n] * s * (double)h[(int64_t)i * K + c];
                    }
                    acc += decode_bfloat16(dY[m * N + n]) * w;
                }
                dX[m * K + c] = acc;
            }
    }
    free(G);
    free(B);
    return st;
}

/* Forward pass of the coupled-training layer (RaBiT, Algorithm 2 forward:
 * the signs are derived on the fly from the latent weight W by the fp32
 * recurrence, with the trainable fp32 scales):
 *   Y[m][n] = sum_c X[m][c] * sum_i g_i[n] B_i[n][c] h_i[c]    (float64)
 * X is bfloat16 bits [M][K].  rows / toks (nullable) select output rows n and
 * tokens m; Y is [nt][nr].  Returns the status codes of oracle_pack's input
 * scan (-1 bad arguments, 1 non-finite input). */
int oracle_qat_forward(const float *W, const float *g, const float *h, int64_t N, int64_t K, int k,
                       const uint16_t *X, int64_t M, const int64_t *rows, int64_t nr,
                       const int64_t *toks, int64_t nt, double *Y)
{
    if (check_args(N, K, k) || M < 1) return -1;
    int st = scan_inputs(W, g, h, N, K, k, NULL, NULL) == 1 ? 1 : 0;
    #pragma omp parallel
    {
        float *R = (float *)malloc(sizeof(float) * (size_t)K);
        unsigned char *bits = (unsigned char *)malloc((size_t)k * (size_t)K);
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        #pragma omp for schedule(static)
        for (int64_t a = 0; a < nr; ++a) {
            const int64_t r = rows ? rows[a] : a;
            derive_row(W + r * K, g, h, N, K, k, r, R, bits);
            for (int64_t c = 0; c < K; ++c) {        /* What[r][c] */
                double v = 0.0;
                for (int i = 0; i < k; ++i) {
                    double s = bits[(int64_t)i * K + c] ? 1.0 : -1.0;
                    v += (double)g[(int64_t)i * N + r] * s * (double)h[(int64_t)i * K + c];
                }
                w[c] = v;
            }
            for (int64_t b = 0; b < nt; ++b) {
                const int64_t m = toks ? toks[b] : b;
                double acc = 0.0;
                for (int64_t c = 0; c < K; ++c) acc += decode_bfloat16(X[m * K + c]) * w[c];
                Y[b * nr + a] = acc;
            }
        }
        free(R);
        free(bits);
        free(w);
    }
    return st;
}

/* ------------------------------------------------------------------ */
/* Greedy SVID scales (rank-1 of |R_{i-1}| per plane, power iteration)   */
/* ------------------------------------------------------------------ */

int oracle_svid_greedy(const float *W, int64_t N, int64_t K, int k, int iters,
                       float *g, float *h)
{
    if (check_args(N, K, k) || iters < 1) return -1;
    float *R = (float *)malloc(sizeof(float) * (size_t)(N * K));
    double *u = (double *)malloc(sizeof(double) * (size_t)N);
    double *v = (double *)malloc(sizeof(double) * (size_t)K);
    if (!R || !u || !v) { free(R); free(u); free(v); return -1; }
    memcpy(R, W, sizeof(float) * (size_t)(N * K));

    for (int i = 0; i < k; ++i) {
        for (int64_t c = 0; c < K; ++c) v[c] = 1.0 / sqrt((double)K);
        for (int t = 0; t < iters; ++t) {
            double nu = 0.0, nv = 0.0;
            #pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < N; ++r) {          /* u = A v */
                double acc = 0.0;
                for (int64_t c = 0; c < K; ++c) acc += fabs((double)R[r * K + c]) * v[c];
                u[r] = acc;
            }
            for (int64_t r = 0; r < N; ++r) nu += u[r] * u[r];
            nu = sqrt(nu);
            for (int64_t r = 0; r < N; ++r) u[r] = nu > 0.0 ? u[r] / nu : 0.0;
            #pragma omp parallel
            {                                          /* v = A^T u, rows in order */
                int nt = omp_get_num_threads(), tid = omp_get_thread_num();
                int64_t c0 = K * tid / nt, c1 = K * (tid + 1) / nt;
                for (int64_t c = c0; c < c1; ++c) v[c] = 0.0;
                for (int64_t r = 0; r < N; ++r) {
                    double ur = u[r];
                    for (int64_t c = c0; c < c1; ++c) v[c] += fabs((double)R[r * K + c]) * ur;
                }
            }
            for (int64_t c = 0; c < K; ++c) nv += v[c] * v[c];
            nv = sqrt(nv);
            for (int64_t c = 0; c < K; ++c) v[c] = nv > 0.0 ? v[c] / nv : 0.0;
        }
        double sigma = 0.0;                            /* sigma = u^T A v */
        for (int64_t r = 0; r < N; ++r) {
            double acc = 0.0;
            for (int64_t c = 0; c < K; ++c) acc += fabs((double)R[r * K + c]) * v[c];
            sigma += u[r] * acc;
        }
        double rs = sigma > 0.0 ? sqrt(sigma) : 0.0;
        for (int64_t r = 0; r < N; ++r) g[(int64_t)i * N + r] = (float)(rs * u[r]);
        for (int64_t c = 0; c < K; ++c) h[(int64_t)i * K + c] = (float)(rs * v[c]);
        /* R_i from R_{i-1}: same fp32 recurrence as the packer */
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < N; ++r) {
            float gi = g[(int64_t)i * N + r];
            for (int64_t c = 0; c < K; ++c) {
                float Rv = R[r * K + c];
                int b = (Rv >= 0.0f);
                float tt = gi * h[(int64_t)i * K + c];
                R[r * K + c] = b ? (Rv - tt) : (Rv + tt);
            }
        }
    }
    free(R);
    free(u);
    free(v);
    return 0;
}

/* Rank-1 of |T| (T float64 [N][K]) by the greedy rule's power iteration,
 * with the same summation orders; writes g_row[N], h_row[K]. */
static void rank1_abs_f64(const double *T, int64_t N, int64_t K, int iters, double *u, double *v,
                          float *g_row, float *h_row)
{
    for (int64_t c = 0; c < K; ++c) v[c] = 1.0 / sqrt((double)K);
    for (int t = 0; t < iters; ++t) {
        double nu = 0.0, nv = 0.0;
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < N; ++r) {          /* u = A v */
            double acc = 0.0;
            for (int64_t c = 0; c < K; ++c) acc += fabs(T[r * K + c]) * v[c];
            u[r] = acc;
        }
        for (int64_t r = 0; r < N; ++r) nu += u[r] * u[r];
        nu = sqrt(nu);
        for (int64_t r = 0; r < N; ++r) u[r] = nu > 0.0 ? u[r] / nu : 0.0;
        #pragma omp parallel
        {                                          /* v = A^T u, rows in order */
            int nt = omp_get_num_threads(), tid = omp_get_thread_num();
            int64_t c0 = K * tid / nt, c1 = K * (tid + 1) / nt;
            for (int64_t c = c0; c < c1; ++c) v[c] = 0.0;
            for (int64_t r = 0; r < N; ++r) {
                double ur = u[r];
                for (int64_t c = c0; c < c1; ++c) v[c] += fabs(T[r * K + c]) * ur;
            }
        }
        for (int64_t c = 0; c < K; ++c) nv += v[c] * v[c];
        nv = sqrt(nv);
        for (int64_t c = 0; c < K; ++c) v[c] = nv > 0.0 ? v[c] / nv : 0.0;
    }
    double sigma = 0.0;                            /* sigma = u^T A v */
    for (int64_t r = 0; r < N; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < K; ++c) acc += fabs(T[r * K + c]) * v[c];
        sigma += u[r] * acc;
    }
    double rs = sigma > 0.0 ? sqrt(sigma) : 0.0;
    for (int64_t r = 0; r < N; ++r) g_row[r] = (float)(rs * u[r]);
    for (int64_t c = 0; c < K; ++c) h_row[c] = (float)(rs * v[c]);
}

int oracle_svid_iterative(const float *W, int64_t N, int64_t K, int k, int sweeps, int iters,
                          float *g, float *h)
{
    if (check_args(N, K, k) || iters < 1 || sweeps < 0) return -1;
    if (oracle_svid_greedy(W, N, K, k, iters, g, h)) return -1;     /* sweep 0: the greedy pass */
    if (sweeps == 0) return 0;
    signed char *B = (signed char *)malloc((size_t)(k * N * K));
    double *T = (double *)malloc(sizeof(double) * (size_t)(N * K));
    double *u = (double *)malloc(sizeof(double) * (size_t)N);
    double *v = (double *)malloc(sizeof(double) * (size_t)K);
    if (!B || !T || !u || !v) { free(B); free(T); free(u); free(v); return -1; }
    /* signs of the greedy pass: the fp32 recurrence of the packer */
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < N; ++r) {
        for (int64_t c = 0; c < K; ++c) {
            float Rv = W[r * K + c];
            for (int i = 0; i < k; ++i) {
                int b = (Rv >= 0.0f);
                B[((int64_t)i * N + r) * K + c] = (signed char)(b ? 1 : -1);
                float tt = g[(int64_t)i * N + r] * h[(int64_t)i * K + c];
                Rv = b ? (Rv - tt) : (Rv + tt);
            }
        }
    }
    for (int t = 0; t < sweeps; ++t) {
        for (int i = 0; i < k; ++i) {
            /* T_i = W - sum_{j != i} g_j B_j h_j (float64, planes in order), B_i = sign(T_i) */
            #pragma omp parallel for schedule(static)
            for (int64_t r = 0; r < N; ++r) {
                for (int64_t c = 0; c < K; ++c) {
                    double x = (double)W[r * K + c];
                    for (int j = 0; j < k; ++j) {
                        if (j == i) continue;
                        double p = (double)g[(int64_t)j * N + r] * (double)h[(int64_t)j * K + c];
                        x = B[((int64_t)j * N + r) * K + c] > 0 ? x - p : x + p;
                    }
                    T[r * K + c] = x;
                    B[((int64_t)i * N + r) * K + c] = (signed char)(x >= 0.0 ? 1 : -1);
                }
            }
            rank1_abs_f64(T, N, K, iters, u, v, g + (int64_t)i * N, h + (int64_t)i * K);
        }
    }
    free(B);
    free(T);
    free(u);
    free(v);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Binary codebook and its LUT application (BTC-LLM: "Binary codebook",  */
/* 2.1.1 binary k-means and dynamic codebook size; 2.1.2 LUT-GEMM;       */
/* 3.2.1 index of ceil(log2 c) bits; 5.1 v = 16, c = 7132 for 7B)          */
/* ------------------------------------------------------------------ */

/* Readings (listed in the design notes):
 *   - the vectors clustered are the v = 16 column groups of one sign plane
 *     B_i; pattern bit q = 1 <=> B_i[r][16 j + q] = +1 (the planes' own bit
 *     order);
 *   - the codebook size is c = min(c_max, number of distinct patterns)
 *     (dynamic size); the c initial centroids are the c most frequent
 *     patterns, ties to the smaller pattern value, in that order;
 *   - one round = assignment of every vector to the centroid at the least
 *     Hamming distance popcount(u ^ C[p]) (ties to the smaller p), then each
 *     centroid that has members becomes the per-bit majority of its members,
 *     sign(0) = +1 (a member-less centroid is kept); `iters` rounds, then a
 *     final assignment gives the indices;
 *   - index j of row r (the j-th 16-column group) is stored in w = ceil(log2
 *     c_max) bits (at least 1), LSB-first in a per-row bit stream of
 *     ceil(K/16 * w / 32) words: bits [j w, j w + w) of the row's stream.   */

static int popcount16(uint32_t x) { return __builtin_popcount(x & 0xFFFFu); }

int oracle_btc_index_bits(int c_max)
{
    int w = 1;
    while ((1 << w) < c_max) ++w;
    return w;
}

int64_t oracle_btc_row_words(int64_t K, int w) { return (K / 16 * w + 31) / 32; }

/* 16-bit patterns [N][K/16] of plane i from the storage layout. */
void oracle_btc_patterns(const uint32_t *planes, int64_t N, int64_t K, int k, int i, uint16_t *pat)
{
    int64_t J = K / 16;
    for (int64_t r = 0; r < N; ++r)
        for (int64_t j = 0; j < J; ++j) {
            uint32_t word = planes[word_index(N, K, i, r, 16 * j)];
            pat[r * J + j] = (uint16_t)((word >> ((16 * j) % 32)) & 0xFFFFu);
        }
    (void)k;
}

/* Binary k-means over the patterns of plane i.  codebook gets c_max entries
 * (those past *c_out are 0), idx [N][K/16] the final assignment; objective
 * (nullable) iters + 1 values: sum over all vectors of the Hamming distance
 * to the assigned centroid after each assignment step.  Returns 0, or -1 for
 * bad arguments. */
int oracle_btc_encode(const uint32_t *planes, int64_t N, int64_t K, int k, int i, int c_max, int iters,
                      uint16_t *codebook, int *c_out, uint16_t *idx, double *objective)
{
    if (N < 1 || K < 32 || K % 32 != 0 || k < 1 || k > 8 || i < 0 || i >= k || c_max < 1 || c_max > 65536 ||
        iters < 0)
        return -1;
    int64_t J = K / 16, nv = N * J;
    uint16_t *pat = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)nv);
    uint64_t *hist = (uint64_t *)calloc(65536, sizeof(uint64_t));
    int32_t *assign = (int32_t *)malloc(sizeof(int32_t) * 65536);
    oracle_btc_patterns(planes, N, K, k, i, pat);
    for (int64_t x = 0; x < nv; ++x) hist[pat[x]]++;
    int U = 0;
    for (int u = 0; u < 65536; ++u) U += hist[u] > 0;
    int c = U < c_max ? U : c_max;
    /* initial centroids: the c most frequent patterns (count descending, then
     * pattern ascending), by repeated selection of the best remaining one */
    unsigned char *taken = (unsigned char *)calloc(65536, 1);
    for (int p = 0; p < c_max; ++p) codebook[p] = 0;
    for (int p = 0; p < c; ++p) {
        int best = -1;
        for (int u = 0; u < 65536; ++u) {
            if (taken[u] || hist[u] == 0) continue;
            if (best < 0 || hist[u] > hist[best]) best = u;
        }
        taken[best] = 1;
        codebook[p] = (uint16_t)best;
    }
    free(taken);
    for (int round = 0; round <= iters; ++round) {
        double obj = 0.0;
        #pragma omp parallel for schedule(dynamic, 256) reduction(+ : obj)
        for (int u = 0; u < 65536; ++u) {
            if (hist[u] == 0) { assign[u] = -1; continue; }
            int bp = 0, bd = 17;
            for (int p = 0; p < c; ++p) {
                int d = popcount16((uint32_t)u ^ codebook[p]);
                if (d < bd) { bd = d; bp = p; }
            }
            assign[u] = bp;
            obj += (double)hist[u] * bd;
        }
        if (objective) objective[round] = obj;
        if (round == iters) break;
        /* majority of the members, bit by bit: +1 when the +1 count is at least the -1 count */
        int64_t *sum = (int64_t *)calloc((size_t)c * 16, sizeof(int64_t));
        uint64_t *members = (uint64_t *)calloc((size_t)c, sizeof(uint64_t));
        for (int u = 0; u < 65536; ++u) {
            if (hist[u] == 0) continue;
            int p = assign[u];
            members[p] += hist[u];
            for (int q = 0; q < 16; ++q) sum[(int64_t)p * 16 + q] += ((u >> q) & 1) ? (int64_t)hist[u] : -(int64_t)hist[u];
        }
        for (int p = 0; p < c; ++p) {
            if (members[p] == 0) continue;
            uint32_t cw = 0;
            for (int q = 0; q < 16; ++q) cw |= (sum[(int64_t)p * 16 + q] >= 0 ? 1u : 0u) << q;
            codebook[p] = (uint16_t)cw;
        }
        free(sum);
        free(members);
    }
    for (int64_t x = 0; x < nv; ++x) idx[x] = (uint16_t)assign[pat[x]];
    *c_out = c;
    free(pat);
    free(hist);
    free(assign);
    return 0;
}

/* Index bit stream of one plane: [N][row_words], index j of row r at bits
 * [j w, j w + w) of the row's words, LSB-first; unused bits zero. */
void oracle_btc_pack_indices(const uint16_t *idx, int64_t N, int64_t K, int w, uint32_t *words)
{
    int64_t J = K / 16, rw = oracle_btc_row_words(K, w);
    for (int64_t x = 0; x < N * rw; ++x) words[x] = 0u;
    for (int64_t r = 0; r < N; ++r)
        for (int64_t j = 0; j < J; ++j)
            for (int b = 0; b < w; ++b)
                if ((idx[r * J + j] >> b) & 1u) {
                    int64_t bit = j * w + b;
                    words[r * rw + bit / 32] |= 1u << (bit % 32);
                }
}

/* Y[t][j] = sum_i g_i[n] sum_c Bhat_i[n][c] h_i[c] x_m[c] in float64, with
 * Bhat_i[n][16 jj + q] = +1 if bit q of codebook_i[idx_i[n][jj]] is set, else
 * -1: the dense product of the codebook-reconstructed layer.  codebooks
 * [k][c_max], idx [k][N][K/16] (plain indices). */
void oracle_btc_apply(const uint16_t *codebooks, int c_max, const uint16_t *idx, const uint16_t *g16,
                      const uint16_t *h16, int64_t N, int64_t K, int k, const uint16_t *X, int64_t M,
                      const int64_t *rows, int64_t nrows, double *Y)
{
    if (!rows) nrows = N;
    int64_t J = K / 16;
    #pragma omp parallel
    {
        double *What = (double *)malloc(sizeof(double) * (size_t)K);
        #pragma omp for schedule(dynamic, 4)
        for (int64_t jr = 0; jr < nrows; ++jr) {
            int64_t n = rows ? rows[jr] : jr;
            for (int64_t c = 0; c < K; ++c) What[c] = 0.0;
            for (int i = 0; i < k; ++i) {
                double gi = decode_binary16(g16[(int64_t)i * N + n]);
                for (int64_t jj = 0; jj < J; ++jj) {
                    uint32_t p = codebooks[(int64_t)i * c_max + idx[((int64_t)i * N + n) * J + jj]];
                    for (int q = 0; q < 16; ++q) {
                        int64_t c = 16 * jj + q;
                        double s = ((p >> q) & 1u) ? 1.0 : -1.0;
                        What[c] += gi * s * decode_binary16(h16[(int64_t)i * K + c]);
                    }
                }
            }
            for (int64_t m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int64_t c = 0; c < K; ++c) acc += decode_bfloat16(X[m * K + c]) * What[c];
                Y[m * nrows + jr] = acc;
            }
        }
        free(What);
    }
}
