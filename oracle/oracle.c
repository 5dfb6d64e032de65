/*
 * Reference oracle for the weight-quantized linear layer  Y = X * dequant(W)^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load this code.  It shares nothing with the CUDA
 * library (no headers, no helpers, no tables) and never imports it.
 *
 * Everything here is plain, slow and written from the format definitions, in
 * double precision (fp64), single pass, k ascending, with no blocking or
 * reordering beyond the definitions below.
 *
 * Formats and the passages that define them:
 *  - GPTQ INT4, symmetric, group size 128, act-order off, codes packed into
 *    int32 words ("Qwen3.8-27B GPTQ-Int4-sym-G128" model card, section
 *    "Quantization contract"; Eole Qwen3.8 recipe, section "Compressed-tensors
 *    INT4 layout": symmetric grouped W4A16, group size 32/64/128, reordered
 *    groups rejected).  Reading adopted: word (i, n) of qweight[K/8][N] holds
 *    the code of row k = 8i + j in bits [4j, 4j+3] (least significant nibble
 *    first); the zero point of a symmetric code is the implicit 8, so
 *    w[n][k] = (q - 8) * scale[k / G][n].
 *  - The compressed-tensors export of the same weights (Eole Qwen3.8 recipe,
 *    section "Compressed-tensors INT4 layout": symmetric grouped W4A16
 *    pack-quantized weights that its converter transposes into the GPTQ
 *    layout without re-quantizing).  Reading adopted: word (n, i) of
 *    weight_packed[N][K/8] holds the code of row k = 8i + j of column n in
 *    bits [4j, 4j+3], the same code values as GPTQ, and weight_scale[N][K/G]
 *    holds scale (n, k / G); w[n][k] = (q - 8) * weight_scale[n][k / G].
 *  - INT8 W8A16 vocabulary head (Eole Qwen3.8 recipe, section "Optional
 *    vocabulary-head quantization": symmetric group-wise round-to-nearest
 *    int8, group size 32, 64 or 128; the W4A16 LowLatency model card: the
 *    INT8 lm_head is RTN g128 in compressed-tensors form).  Reading adopted:
 *    the GPTQ packing with 8-bit codes, word (i, n) of qweight[K/4][N] holding
 *    the code of row k = 4i + j in bits [8j, 8j+7] (least significant byte
 *    first), the implicit zero point 128 of a symmetric 8-bit code, so
 *    w[n][k] = (q - 128) * scale[k / G][n] with fp16 scales.
 *  - Dense bf16 projections with few output columns (Eole Qwen3.8 recipe,
 *    section "Pack inference projections": the paired 48 x 5120 GDN A/B
 *    projections in bf16).  Reading adopted: W[N][K] row-major (the Linear
 *    out x in layout), Y[m][n] = sum_k X[m][k] * W[n][k].
 *  - fp16 scales (IEEE binary16) and bf16 activations (top half of an IEEE
 *    binary32); accumulation in fp32, output bf16 (Eole Qwen3.8 recipe,
 *    "INT4 weights / BF16 compute").
 *  - MXFP8 (OCP Microscaling): E4M3 element codes, one E8M0 shared scale per
 *    32-element block ("Qwen3.8-27B-MXFP8 AutoRound" model card, header and
 *    section 8 "License and attribution"; kernel constraints N >= 128 and
 *    K % 32 == 0 in its section 2).  E4M3 "fn" flavour: bias 7, subnormals at
 *    exponent field 0, S.1111.111 is NaN, no infinities.  E8M0: 2^(E - 127),
 *    E = 255 is NaN.  Reading adopted: codes Wq[N][K] row-major (K contiguous),
 *    scales Ws[N][K/32].
 *
 * Status: every exported function returns 0 on success and -1 on an invalid
 * argument or an input the formats leave undefined (NaN codes or scales).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ decoders */

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double mxo_decode_fp16(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* 0.f * 2^-14 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);     /* 1.f * 2^(e-15) */
    return s ? -v : v;
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
double mxo_decode_bf16(uint16_t b)
{
    int s = (b >> 15) & 1;
    int e = (b >> 7) & 0xFF;
    int f = b & 0x7F;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);                /* 0.f * 2^-126 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);     /* 1.f * 2^(e-127) */
    return s ? -v : v;
}

/* OCP E4M3 ("fn"): 1 sign, 4 exponent (bias 7), 3 fraction bits. */
double mxo_decode_e4m3(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int f = c & 0x7;
    double v;
    if (e == 15 && f == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)f, -9);                  /* 0.f * 2^-6 */
    else
        v = ldexp((double)(8 + f), e - 10);        /* 1.f * 2^(e-7) */
    return s ? -v : v;
}

/* OCP E8M0 shared scale: 2^(E - 127), E = 255 is NaN. */
double mxo_decode_e8m0(uint8_t e)
{
    if (e == 255)
        return NAN;
    return ldexp(1.0, (int)e - 127);
}

/* Round a real value (given exactly as a double) to the nearest bfloat16,
 * ties to even, and return its bit pattern.  Subnormal results keep the
 * fixed quantum 2^-133; magnitudes that round past the largest finite value
 * become infinity. */
uint16_t mxo_round_bf16(double x)
{
    if (isnan(x))
        return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return sign | 0x7F80;

    int e2;
    frexp(a, &e2);             /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;            /* binade exponent */
    if (E < -126)
        E = -126;              /* subnormal range shares the 2^-133 quantum */
    double quantum = ldexp(1.0, E - 7);
    double n = a / quantum;    /* exact: division by a power of two */
    double lo = floor(n);
    double frac = n - lo;
    double r;
    if (frac > 0.5)
        r = lo + 1.0;
    else if (frac < 0.5)
        r = lo;
    else
        r = (fmod(lo, 2.0) == 0.0) ? lo : lo + 1.0;   /* tie: to even */

    double v = r * quantum;    /* the rounded magnitude, exactly */
    if (v == 0.0)
        return sign;
    if (v < ldexp(1.0, -126))  /* subnormal: fraction = v / 2^-133 */
        return sign | (uint16_t)(v / ldexp(1.0, -133));
    int ev;
    frexp(v, &ev);
    int Ev = ev - 1;
    if (Ev > 127)
        return sign | 0x7F80;  /* overflow to infinity */
    uint16_t frac7 = (uint16_t)(v / ldexp(1.0, Ev - 7) - 128.0);
    return sign | (uint16_t)((Ev + 127) << 7) | frac7;
}

/* ------------------------------------------------------------- INT4 W4A16 */

static int w4a16_args_ok(int K, int N, int G)
{
    if (K <= 0 || N <= 0 || G <= 0)
        return 0;
    if (K % 8 != 0 || K % G != 0)
        return 0;
    return 1;
}

/* The 4-bit code of weight (n, k) from GPTQ words qweight[K/8][N]. */
static int w4a16_code(const int32_t *qweight, int N, int n, int k)
{
    uint32_t word = (uint32_t)qweight[(size_t)(k / 8) * N + n];
    return (int)((word >> (4 * (k % 8))) & 0xF);
}

/* The dequantized weight (q - 8) * scale[k / G][n], exactly. */
static double w4a16_weight(const int32_t *qweight, const uint16_t *scales,
                           int N, int G, int n, int k)
{
    int q = w4a16_code(qweight, N, n, k);
    double s = mxo_decode_fp16(scales[(size_t)(k / G) * N + n]);
    return (double)(q - 8) * s;
}

/* Unpack GPTQ words into codes[N][K] (may be NULL) and weights w[N][K]
 * (may be NULL). */
int mxo_w4a16_unpack(const int32_t *qweight, const uint16_t *scales,
                     int K, int N, int G, uint8_t *codes, double *w)
{
    if (!qweight || !w4a16_args_ok(K, N, G) || (w && !scales))
        return -1;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            if (codes)
                codes[(size_t)n * K + k] = (uint8_t)w4a16_code(qweight, N, n, k);
            if (w)
                w[(size_t)n * K + k] = w4a16_weight(qweight, scales, N, G, n, k);
        }
    return 0;
}

/* Unpack compressed-tensors words weight_packed[N][K/8] and scales
 * weight_scale[N][K/G] into codes[N][K] (may be NULL) and weights w[N][K]
 * (may be NULL), from the definition above (row n of the export is column n
 * of the layer). */
int mxo_w4a16_unpack_ct(const int32_t *weight_packed, const uint16_t *weight_scale,
                        int K, int N, int G, uint8_t *codes, double *w)
{
    if (!weight_packed || !w4a16_args_ok(K, N, G) || (w && !weight_scale))
        return -1;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            uint32_t word = (uint32_t)weight_packed[(size_t)n * (K / 8) + k / 8];
            int q = (int)(word >> (4 * (k & 7))) & 0xF;
            if (codes)
                codes[(size_t)n * K + k] = (uint8_t)q;
            if (w)
                w[(size_t)n * K + k] =
                    (double)(q - 8) * mxo_decode_fp16(weight_scale[(size_t)n * (K / G) + k / G]);
        }
    return 0;
}

/* Inverse of the unpack: codes[N][K] (values 0..15) into words qweight[K/8][N]. */
int mxo_w4a16_pack(const uint8_t *codes, int K, int N, int32_t *qweight)
{
    if (!codes || !qweight || K <= 0 || N <= 0 || K % 8 != 0)
        return -1;
    for (int i = 0; i < K / 8; ++i)
        for (int n = 0; n < N; ++n) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) {
                uint8_t q = codes[(size_t)n * K + 8 * i + j];
                if (q > 15)
                    return -1;
                word |= (uint32_t)q << (4 * j);
            }
            qweight[(size_t)i * N + n] = (int32_t)word;
        }
    return 0;
}

/* Y[M][N] = sum_k x[m][k] * w[n][k] in double, k ascending.
 * The column n of W is dequantized once into a scratch row, then each output
 * of that column is a plain dot product.  nthreads > 1 splits the columns
 * across OpenMP threads; the arithmetic of every element is unchanged. */
int mxo_w4a16_gemm(const uint16_t *X, const int32_t *qweight, const uint16_t *scales,
                   int M, int N, int K, int G, double *Y, int nthreads)
{
    if (!X || !qweight || !scales || !Y || M <= 0 || !w4a16_args_ok(K, N, G))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    int bad = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        double *x = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w || !x)
            bad = 1;
#pragma omp for schedule(static)
        for (int n = 0; n < N; ++n) {
            if (!w || !x)
                continue;
            for (int k = 0; k < K; ++k)
                w[k] = w4a16_weight(qweight, scales, N, G, n, k);
            for (int m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int k = 0; k < K; ++k) {
                    x[k] = mxo_decode_bf16(X[(size_t)m * K + k]);
                    acc += x[k] * w[k];
                }
                Y[(size_t)m * N + n] = acc;
            }
        }
        free(w);
        free(x);
    }
    return bad ? -1 : 0;
}

/* Selected outputs only: out[i] = Y[rows[i]][cols[i]], same definition. */
int mxo_w4a16_gemm_at(const uint16_t *X, const int32_t *qweight, const uint16_t *scales,
                      int M, int N, int K, int G,
                      const int64_t *rows, const int64_t *cols, int64_t count,
                      double *out, int nthreads)
{
    if (!X || !qweight || !scales || !rows || !cols || !out || M <= 0 ||
        !w4a16_args_ok(K, N, G) || count < 0)
        return -1;
    for (int64_t i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M || cols[i] < 0 || cols[i] >= N)
            return -1;
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int m = (int)rows[i], n = (int)cols[i];
        double acc = 0.0;
        for (int k = 0; k < K; ++k)
            acc += mxo_decode_bf16(X[(size_t)m * K + k]) *
                   w4a16_weight(qweight, scales, N, G, n, k);
        out[i] = acc;
    }
    return 0;
}

/* ------------------------------------------------------------------ MXFP8 */

static int mxfp8_args_ok(int K, int N)
{
    return K > 0 && N > 0 && K % 32 == 0;
}

static double mxfp8_weight(const uint8_t *Wq, const uint8_t *Ws, int K, int n, int k)
{
    double v = mxo_decode_e4m3(Wq[(size_t)n * K + k]);
    double s = mxo_decode_e8m0(Ws[(size_t)n * (K / 32) + k / 32]);
    return v * s;
}

static int mxfp8_has_nan(const uint8_t *Wq, const uint8_t *Ws, int N, int K)
{
    for (size_t i = 0; i < (size_t)N * K; ++i)
        if ((Wq[i] & 0x7F) == 0x7F)
            return 1;
    for (size_t i = 0; i < (size_t)N * (K / 32); ++i)
        if (Ws[i] == 0xFF)
            return 1;
    return 0;
}

/* w[N][K] = e4m3(Wq[n][k]) * 2^(Ws[n][k/32] - 127), exactly. */
int mxo_mxfp8_dequant(const uint8_t *Wq, const uint8_t *Ws, int N, int K, double *w)
{
    if (!Wq || !Ws || !w || !mxfp8_args_ok(K, N) || mxfp8_has_nan(Wq, Ws, N, K))
        return -1;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
            w[(size_t)n * K + k] = mxfp8_weight(Wq, Ws, K, n, k);
    return 0;
}

int mxo_mxfp8_gemm(const uint16_t *X, const uint8_t *Wq, const uint8_t *Ws,
                   int M, int N, int K, double *Y, int nthreads)
{
    if (!X || !Wq || !Ws || !Y || M <= 0 || !mxfp8_args_ok(K, N) ||
        mxfp8_has_nan(Wq, Ws, N, K))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    int bad = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w)
            bad = 1;
#pragma omp for schedule(static)
        for (int n = 0; n < N; ++n) {
            if (!w)
                continue;
            for (int k = 0; k < K; ++k)
                w[k] = mxfp8_weight(Wq, Ws, K, n, k);
            for (int m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int k = 0; k < K; ++k)
                    acc += mxo_decode_bf16(X[(size_t)m * K + k]) * w[k];
                Y[(size_t)m * N + n] = acc;
            }
        }
        free(w);
    }
    return bad ? -1 : 0;
}

int mxo_mxfp8_gemm_at(const uint16_t *X, const uint8_t *Wq, const uint8_t *Ws,
                      int M, int N, int K,
                      const int64_t *rows, const int64_t *cols, int64_t count,
                      double *out, int nthreads)
{
    if (!X || !Wq || !Ws || !rows || !cols || !out || M <= 0 ||
        !mxfp8_args_ok(K, N) || count < 0)
        return -1;
    for (int64_t i = 0; i < count; ++i)
        if (rows[i] < 0 || rows[i] >= M || cols[i] < 0 || cols[i] >= N)
            return -1;
    if (nthreads < 1)
        nthreads = 1;
    int bad = 0;
#pragma omp parallel for num_threads(nthreads) schedule(static) reduction(| : bad)
    for (int64_t i = 0; i < count; ++i) {
        int m = (int)rows[i], n = (int)cols[i];
        double acc = 0.0;
        for (int k = 0; k < K; ++k) {
            double w = mxfp8_weight(Wq, Ws, K, n, k);
            if (isnan(w))
                bad = 1;
            acc += mxo_decode_bf16(X[(size_t)m * K + k]) * w;
        }
        out[i] = acc;
    }
    return bad ? -1 : 0;
}

/* Threads an OpenMP region would use with the given request (1 without OpenMP). */
int mxo_threads(int requested)
{
#ifdef _OPENMP
    int used = 1;
#pragma omp parallel num_threads(requested < 1 ? 1 : requested)
    {
#pragma omp single
        used = omp_get_num_threads();
    }
    return used;
#else
    (void)requested;
    return 1;
#endif
}

/* Dense bf16 weights W[N][K]: Y[m][n] = sum over k ascending of
 * X[m][k] * W[n][k], in double precision (not rounded). */
int mxo_bf16_gemm(const uint16_t *X, const uint16_t *W, int M, int N, int K, double *Y)
{
    if (!X || !W || !Y || M <= 0 || N <= 0 || K <= 0)
        return -1;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += mxo_decode_bf16(X[(size_t)m * K + k]) * mxo_decode_bf16(W[(size_t)n * K + k]);
            Y[(size_t)m * N + n] = acc;
        }
    return 0;
}

/* INT8 code of (n, k): byte k % 4 of word (k / 4, n) of qweight[K/4][N]. */
static int w8a16_code(const int32_t *qweight, int N, int n, int k)
{
    uint32_t word = (uint32_t)qweight[(size_t)(k / 4) * N + n];
    return (int)((word >> (8 * (k % 4))) & 0xFFu);
}

static int w8a16_args_ok(int K, int N, int G)
{
    return K > 0 && N > 0 && G > 0 && K % 4 == 0 && K % G == 0;
}

/* Codes[N][K] (may be NULL) and exact weights (q - 128) * scale (may be NULL). */
int mxo_w8a16_unpack(const int32_t *qweight, const uint16_t *scales, int K, int N, int G,
                     uint8_t *codes, double *w)
{
    if (!qweight || !w8a16_args_ok(K, N, G) || (w && !scales))
        return -1;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            int q = w8a16_code(qweight, N, n, k);
            if (codes)
                codes[(size_t)n * K + k] = (uint8_t)q;
            if (w)
                w[(size_t)n * K + k] =
                    (double)(q - 128) * mxo_decode_fp16(scales[(size_t)N * (k / G) + n]);
        }
    return 0;
}

/* Y[M][N] = X * dequant(W)^T for INT8 W8A16 weights, fp64, k ascending. */
int mxo_w8a16_gemm(const uint16_t *X, const int32_t *qweight, const uint16_t *scales,
                   int M, int N, int K, int G, double *Y, int nthreads)
{
    if (!X || !qweight || !scales || !Y || M <= 0 || !w8a16_args_ok(K, N, G))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    int bad = 0;
#pragma omp parallel num_threads(nthreads) reduction(| : bad)
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w)
            bad = 1;
#pragma omp for schedule(static)
        for (int n = 0; n < N; ++n) {
            if (!w)
                continue;
            for (int k = 0; k < K; ++k)
                w[k] = (double)(w8a16_code(qweight, N, n, k) - 128) *
                       mxo_decode_fp16(scales[(size_t)N * (k / G) + n]);
            for (int m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int k = 0; k < K; ++k)
                    acc += mxo_decode_bf16(X[(size_t)m * K + k]) * w[k];
                Y[(size_t)m * N + n] = acc;
            }
        }
        free(w);
    }
    return bad ? -1 : 0;
}
