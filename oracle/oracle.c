/*
 * Oracle for the low-bit mixed-precision matmul  C[M,N] = A[M,K] . dequant(W[N,K])^T  ("nt").
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously-correct statement of
 * what the CUDA library computes. Only the tests, the smoke check and the benchmark's CPU
 * baseline may load it; the library never does, and it shares no code, header, table or
 * helper with the CUDA path. Floating point is evaluated in fp64 and integers in int64:
 * first dequantise every weight, then multiply with a plain ascending-k loop.
 *
 * Sources (page title, then the place on it):
 *  - microsoft/BitBLAS issue #252, "Default Backend Should be changed into tilelang":
 *    the benchmark configuration listing (op_configs and the MatmulConfig argument tuple)
 *    fixes the operand types fp16 x int4, int8 x int8 with int32 accumulation,
 *    int8 x int2 with int32 accumulation, fp16 x fp16, the "nt" layout, group_size
 *    (-1 = one group over K), with_scaling and with_zeros.
 *  - triton-lang/triton PR #3595, "Convert INT8 MMAV2 accumulator layout to dot_operand
 *    layout", the review discussion: an int8 dot product accumulates and returns int32.
 *  - hidet-org/hidet issue #364, "Multi-stage software pipelining and update parallel k
 *    rule", parallel-k discussion: the K reduction may be split into parts whose partial
 *    results are added; the sum over parts equals the full sum.
 *
 * Readings where the pages are silent (each is listed with its reason in the design notes):
 *  - int4 codes are unsigned 0..15, packed 8 per uint32 along K, element k at bits 4*(k%8);
 *  - int2 values are two's complement in {-2..1}, packed 16 per uint32, element k at bits
 *    2*(k%16);
 *  - dequantisation is w = (q - z) * s with s, z fp16 of shape [N, K/group_size]
 *    (row-major); without zeros z = 0;
 *  - group_size -1 (or 0) means one group spanning K.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_BAD_ARGS -1
#define ORC_NO_MEMORY -2

/* IEEE 754-2008 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    return sign ? -mag : mag;
}

void orc_decode_half(const uint16_t *h, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_half_to_double(h[i]);
}

/* ---- packing ---------------------------------------------------------------------------- */

/* packed[n, j] = sum_i (codes[n, 8j+i] & 0xF) << 4i */
int orc_pack_int4(const uint8_t *codes, uint32_t *packed, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 8) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 8; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i)
                word |= (uint32_t)(codes[n * K + 8 * j + i] & 0xF) << (4 * i);
            packed[n * (K / 8) + j] = word;
        }
    return ORC_OK;
}

static int int4_code(const uint32_t *packed, int64_t K, int64_t n, int64_t k)
{
    return (int)((packed[n * (K / 8) + k / 8] >> (4 * (k % 8))) & 0xF);
}

int orc_unpack_int4(const uint32_t *packed, uint8_t *codes, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 8) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            codes[n * K + k] = (uint8_t)int4_code(packed, K, n, k);
    return ORC_OK;
}

/*
 * Interleaved int4 packing (the pre-shuffled layout): inside each word, code k = 8j + e sits in
 * nibble ILV_POS[e] = (e % 2) * 4 + e / 2, i.e. nibbles 0..7 hold codes 0, 2, 4, 6, 1, 3, 5, 7 of
 * the word. Reading nibbles i and i + 4 of a word then gives two codes adjacent in k.
 */
static const int ILV_POS[8] = {0, 4, 1, 5, 2, 6, 3, 7};

int orc_pack_int4_interleaved(const uint8_t *codes, uint32_t *packed, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 8) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 8; ++j) {
            uint32_t word = 0;
            for (int e = 0; e < 8; ++e)
                word |= (uint32_t)(codes[n * K + 8 * j + e] & 0xF) << (4 * ILV_POS[e]);
            packed[n * (K / 8) + j] = word;
        }
    return ORC_OK;
}

int orc_unpack_int4_interleaved(const uint32_t *packed, uint8_t *codes, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 8) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            codes[n * K + k] =
                (uint8_t)((packed[n * (K / 8) + k / 8] >> (4 * ILV_POS[k % 8])) & 0xF);
    return ORC_OK;
}

/* packed[n, j] = sum_i (vals[n, 16j+i] & 3) << 2i   (two's-complement 2-bit fields) */
int orc_pack_int2(const int8_t *vals, uint32_t *packed, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 16) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 16; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 16; ++i)
                word |= (uint32_t)((uint8_t)vals[n * K + 16 * j + i] & 3u) << (2 * i);
            packed[n * (K / 16) + j] = word;
        }
    return ORC_OK;
}

/*
 * Interleaved int2 packing (the pre-shuffled layout): inside each word, value k = 16j + i sits in
 * 2-bit field ILV2_POS[i] = 8 * (i / 8) + 2 * (i % 4) + (i % 8) / 4, i.e. fields 0..15 hold values
 * 0, 4, 1, 5, 2, 6, 3, 7, 8, 12, 9, 13, 10, 14, 11, 15 of the word.
 */
static const int ILV2_POS[16] = {0, 2, 4, 6, 1, 3, 5, 7, 8, 10, 12, 14, 9, 11, 13, 15};

int orc_pack_int2_interleaved(const int8_t *vals, uint32_t *packed, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 16) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 16; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 16; ++i)
                word |= (uint32_t)((uint8_t)vals[n * K + 16 * j + i] & 3u) << (2 * ILV2_POS[i]);
            packed[n * (K / 16) + j] = word;
        }
    return ORC_OK;
}

int orc_unpack_int2_interleaved(const uint32_t *packed, int8_t *vals, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 16) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            const int u = (int)((packed[n * (K / 16) + k / 16] >> (2 * ILV2_POS[k % 16])) & 3u);
            vals[n * K + k] = (int8_t)(u - 4 * (u >> 1));
        }
    return ORC_OK;
}

/* field u in 0..3 read as a two's-complement 2-bit integer: u - 4 * (u >> 1) */
static int int2_value(const uint32_t *packed, int64_t K, int64_t n, int64_t k)
{
    int u = (int)((packed[n * (K / 16) + k / 16] >> (2 * (k % 16))) & 3u);
    return u - 4 * (u >> 1);
}

int orc_unpack_int2(const uint32_t *packed, int8_t *vals, int64_t N, int64_t K)
{
    if (N < 0 || K < 0 || K % 16) return ORC_BAD_ARGS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            vals[n * K + k] = (int8_t)int2_value(packed, K, n, k);
    return ORC_OK;
}

/* ---- W4A16: fp16 activations x group-quantised uint4 weights ----------------------------- */

static int w4_args_ok(int64_t M, int64_t N, int64_t K, int64_t group_size)
{
    int64_t gs = (group_size <= 0) ? K : group_size;
    return M >= 0 && N >= 0 && K > 0 && K % 8 == 0 && gs > 0 && K % gs == 0;
}

/* w[k] = (q[n,k] - z[n, k/gs]) * s[n, k/gs]  for one weight row n, in fp64 */
static void w4_dequant_row(const uint32_t *Wq, const uint16_t *S, const uint16_t *Z,
                           int64_t n, int64_t K, int64_t gs, int has_zero, double *w)
{
    int64_t G = K / gs;
    for (int64_t k = 0; k < K; ++k) {
        int64_t g = k / gs;
        double s = orc_half_to_double(S[n * G + g]);
        double z = has_zero ? orc_half_to_double(Z[n * G + g]) : 0.0;
        w[k] = ((double)int4_code(Wq, K, n, k) - z) * s;
    }
}

static double dot_f64(const double *a, const double *b, int64_t K)
{
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k)
        acc += a[k] * b[k];
    return acc;
}

/* C[m, n] = sum_k A[m, k] * w[n, k] for all m < M, n < N; C is [M, N] row-major fp64. */
int orc_w4a16(const uint16_t *A, const uint32_t *Wq, const uint16_t *S, const uint16_t *Z,
              int64_t M, int64_t N, int64_t K, int64_t group_size, int has_zero,
              double *C, int nthreads)
{
    if (!w4_args_ok(M, N, K, group_size) || (has_zero && !Z)) return ORC_BAD_ARGS;
    int64_t gs = (group_size <= 0) ? K : group_size;
    double *Ad = (double *)malloc(sizeof(double) * (size_t)(M * K + 1));
    if (!Ad) return ORC_NO_MEMORY;
    orc_decode_half(A, Ad, M * K);
    int failed = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t n = 0; n < N; ++n) {
                w4_dequant_row(Wq, S, Z, n, K, gs, has_zero, w);
                for (int64_t m = 0; m < M; ++m)
                    C[m * N + n] = dot_f64(Ad + m * K, w, K);
            }
            free(w);
        }
    }
    free(Ad);
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* out[i] = C[ms[i], ns[i]] for i < count (same definition, evaluated one element at a time). */
int orc_w4a16_at(const uint16_t *A, const uint32_t *Wq, const uint16_t *S, const uint16_t *Z,
                 int64_t M, int64_t N, int64_t K, int64_t group_size, int has_zero,
                 const int64_t *ms, const int64_t *ns, int64_t count, double *out, int nthreads)
{
    if (!w4_args_ok(M, N, K, group_size) || (has_zero && !Z)) return ORC_BAD_ARGS;
    for (int64_t i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_BAD_ARGS;
    int64_t gs = (group_size <= 0) ? K : group_size;
    int failed = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *buf = (double *)malloc(sizeof(double) * (size_t)(2 * K));
        if (!buf) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < count; ++i) {
                w4_dequant_row(Wq, S, Z, ns[i], K, gs, has_zero, buf);
                orc_decode_half(A + ms[i] * K, buf + K, K);
                out[i] = dot_f64(buf + K, buf, K);
            }
            free(buf);
        }
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ---- dense fp16 x fp16 (the in-library baseline GEMM) --------------------------------------- */

int orc_dense_f16(const uint16_t *A, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                  double *C, int nthreads)
{
    if (M < 0 || N < 0 || K <= 0) return ORC_BAD_ARGS;
    double *Ad = (double *)malloc(sizeof(double) * (size_t)(M * K + 1));
    if (!Ad) return ORC_NO_MEMORY;
    orc_decode_half(A, Ad, M * K);
    int failed = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t n = 0; n < N; ++n) {
                orc_decode_half(W + n * K, w, K);
                for (int64_t m = 0; m < M; ++m)
                    C[m * N + n] = dot_f64(Ad + m * K, w, K);
            }
            free(w);
        }
    }
    free(Ad);
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

int orc_dense_f16_at(const uint16_t *A, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                     const int64_t *ms, const int64_t *ns, int64_t count, double *out,
                     int nthreads)
{
    if (M < 0 || N < 0 || K <= 0) return ORC_BAD_ARGS;
    for (int64_t i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_BAD_ARGS;
    int failed = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *buf = (double *)malloc(sizeof(double) * (size_t)(2 * K));
        if (!buf) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < count; ++i) {
                orc_decode_half(W + ns[i] * K, buf, K);
                orc_decode_half(A + ms[i] * K, buf + K, K);
                out[i] = dot_f64(buf + K, buf, K);
            }
            free(buf);
        }
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

/* ---- integer paths: int8 x int8 -> int32, int8 x int2 -> int32 ------------------------------ */

static int64_t dot_i64(const int64_t *a, const int64_t *b, int64_t K)
{
    int64_t acc = 0;
    for (int64_t k = 0; k < K; ++k)
        acc += a[k] * b[k];
    return acc;
}

/* weight row n widened to int64: kind 8 = int8 [N,K]; kind 2 = packed int2 [N,K/16] */
static void int_weight_row(const void *W, int kind, int64_t n, int64_t K, int64_t *w)
{
    if (kind == 8) {
        const int8_t *W8 = (const int8_t *)W;
        for (int64_t k = 0; k < K; ++k)
            w[k] = W8[n * K + k];
    } else {
        for (int64_t k = 0; k < K; ++k)
            w[k] = int2_value((const uint32_t *)W, K, n, k);
    }
}

static int int_gemm(const int8_t *A, const void *W, int kind, int64_t M, int64_t N, int64_t K,
                    int64_t *C, int nthreads)
{
    if (M < 0 || N < 0 || K <= 0 || (kind == 2 && K % 16)) return ORC_BAD_ARGS;
    int64_t *Ai = (int64_t *)malloc(sizeof(int64_t) * (size_t)(M * K + 1));
    if (!Ai) return ORC_NO_MEMORY;
    for (int64_t i = 0; i < M * K; ++i)
        Ai[i] = A[i];
    int failed = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        int64_t *w = (int64_t *)malloc(sizeof(int64_t) * (size_t)K);
        if (!w) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t n = 0; n < N; ++n) {
                int_weight_row(W, kind, n, K, w);
                for (int64_t m = 0; m < M; ++m)
                    C[m * N + n] = dot_i64(Ai + m * K, w, K);
            }
            free(w);
        }
    }
    free(Ai);
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

static int int_gemm_at(const int8_t *A, const void *W, int kind, int64_t M, int64_t N,
                       int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                       int64_t *out, int nthreads)
{
    if (M < 0 || N < 0 || K <= 0 || (kind == 2 && K % 16)) return ORC_BAD_ARGS;
    for (int64_t i = 0; i < count; ++i)
        if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return ORC_BAD_ARGS;
    int failed = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        int64_t *buf = (int64_t *)malloc(sizeof(int64_t) * (size_t)(2 * K));
        if (!buf) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < count; ++i) {
                int_weight_row(W, kind, ns[i], K, buf);
                for (int64_t k = 0; k < K; ++k)
                    buf[K + k] = A[ms[i] * K + k];
                out[i] = dot_i64(buf + K, buf, K);
            }
            free(buf);
        }
    }
    return failed ? ORC_NO_MEMORY : ORC_OK;
}

int orc_w8a8(const int8_t *A, const int8_t *W, int64_t M, int64_t N, int64_t K, int64_t *C,
             int nthreads)
{
    return int_gemm(A, W, 8, M, N, K, C, nthreads);
}

int orc_w8a8_at(const int8_t *A, const int8_t *W, int64_t M, int64_t N, int64_t K,
                const int64_t *ms, const int64_t *ns, int64_t count, int64_t *out, int nthreads)
{
    return int_gemm_at(A, W, 8, M, N, K, ms, ns, count, out, nthreads);
}

int orc_w2a8(const int8_t *A, const uint32_t *Wq, int64_t M, int64_t N, int64_t K, int64_t *C,
             int nthreads)
{
    return int_gemm(A, Wq, 2, M, N, K, C, nthreads);
}

int orc_w2a8_at(const int8_t *A, const uint32_t *Wq, int64_t M, int64_t N, int64_t K,
                const int64_t *ms, const int64_t *ns, int64_t count, int64_t *out, int nthreads)
{
    return int_gemm_at(A, Wq, 2, M, N, K, ms, ns, count, out, nthreads);
}

/* IEEE 754 binary16 encoding of a binary32 value, round to nearest, ties to even; overflow
   to infinity, NaN to a quiet NaN. Built from the two formats' definitions: a float is
   m * 2^(E-23) with m the 24-bit significand; a half keeps 11 significant bits when
   E >= -14 and a fixed 2^-24 unit below that. */
uint16_t orc_float_to_half(float x)
{
    uint32_t b;
    memcpy(&b, &x, sizeof b);
    const uint16_t sign = (uint16_t)((b >> 16) & 0x8000u);
    const uint32_t e = (b >> 23) & 0xFFu, f = b & 0x7FFFFFu;
    if (e == 0xFFu) return (uint16_t)(sign | 0x7C00u | (f ? 0x200u : 0u));
    if (e == 0) return sign;                  /* below 2^-126: far under half a half-ulp */
    const int32_t E = (int32_t)e - 127;
    if (E > 15) return (uint16_t)(sign | 0x7C00u);
    const uint32_t m = 0x800000u | f;
    const int shift = E >= -14 ? 13 : 13 + (-14 - E);   /* significand bits that go */
    if (shift > 24) return sign;
    uint32_t q = m >> shift;
    const uint32_t rem = m & ((1u << shift) - 1u), halfway = 1u << (shift - 1);
    if (rem > halfway || (rem == halfway && (q & 1u))) ++q;
    if (E >= -14) {
        uint32_t he = (uint32_t)(E + 15);
        if (q == 2048u) {                      /* rounding carried into the exponent */
            q = 1024u;
            ++he;
        }
        if (he >= 31u) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | (he << 10) | (q & 0x3FFu));
    }
    return (uint16_t)(sign | q);               /* subnormal (q == 1024 encodes 2^-14) */
}

/* Round-to-nearest int4 quantisation of fp16 weights W [N, K] into codes [N, K] (0..15) and
   fp16 scales / zeros [N, K / group_size], such that w ~ (q - z) * s.
   Source: the torchao issue's workflow table names int4 weight-only quantisation
   (Int4WeightOnlyConfig) without a formula; the reading used here (design notes):
   asymmetric min-max per group with the range widened to include 0,
       lo = min(0, min w), hi = max(0, max w), s = fp16((hi - lo) / 15)  (1 if hi == lo;
       the smallest subnormal if it rounds to 0), z = clamp(rint(0 - lo / s), 0, 15),
       q = clamp(rint(w / s) + z, 0, 15),
   rint rounding half to even. The values that decide a code (hi - lo, the divisions, rint)
   are evaluated in binary32 because the kernels decide in binary32 too. */
int orc_rtn_int4(const uint16_t *W, int64_t N, int64_t K, int64_t group_size, uint8_t *codes,
                 uint16_t *S, uint16_t *Z)
{
    const int64_t gs = (group_size <= 0) ? K : group_size;
    if (N <= 0 || K <= 0 || gs <= 0 || K % gs) return ORC_BAD_ARGS;
    const int64_t G = K / gs;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t *w = W + n * K + g * gs;
            float lo = 0.0f, hi = 0.0f;
            for (int64_t k = 0; k < gs; ++k) {
                const float v = (float)orc_half_to_double(w[k]);   /* exact */
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            const float range = hi - lo;
            const float s32 = range > 0.0f ? range / 15.0f : 1.0f;
            uint16_t s16 = orc_float_to_half(s32);
            if ((s16 & 0x7FFFu) == 0) s16 = 0x0001u;
            const float s = (float)orc_half_to_double(s16);
            float z = rintf(0.0f - lo / s);    /* +0, not -0, when lo is 0 */
            if (z < 0.0f) z = 0.0f;
            if (z > 15.0f) z = 15.0f;
            S[n * G + g] = s16;
            Z[n * G + g] = orc_float_to_half(z);
            for (int64_t k = 0; k < gs; ++k) {
                const float v = (float)orc_half_to_double(w[k]);
                float q = rintf(v / s) + z;
                if (q < 0.0f) q = 0.0f;
                if (q > 15.0f) q = 15.0f;
                codes[n * K + g * gs + k] = (uint8_t)q;
            }
        }
    return ORC_OK;
}

/* W8A8 with int8 requantised output: C8[m, n] = clamp(rint(float(C[m, n]) * mult[n]), -128,
   127) with C the exact int32 product of orc_w8a8.
   Source: microsoft/BitBLAS issue #252, benchmark configuration listing: the int8 x int8
   configurations carry an int8 output type besides the int32 accumulator. The pages do not say
   how the accumulator becomes int8; the reading (design notes) is a per-output-channel binary32
   multiplier, round half to even, saturation. The conversion, the product and rint are binary32
   operations because the kernels decide in binary32 too. */
int orc_w8a8_requant(const int8_t *A, const int8_t *W, const float *mult, int64_t M, int64_t N,
                     int64_t K, int8_t *C8, int nthreads)
{
    if (M <= 0 || N <= 0 || K <= 0 || K > 131072) return ORC_BAD_ARGS;
    int64_t *acc = (int64_t *)malloc((size_t)(M * N) * sizeof(int64_t));
    if (!acc) return ORC_NO_MEMORY;
    const int rc = orc_w8a8(A, W, M, N, K, acc, nthreads);
    if (rc != ORC_OK) {
        free(acc);
        return rc;
    }
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const float x = (float)(int32_t)acc[m * N + n] * mult[n];
            float r = rintf(x);
            if (r < -128.0f) r = -128.0f;
            if (r > 127.0f) r = 127.0f;
            C8[m * N + n] = (int8_t)r;
        }
    free(acc);
    return ORC_OK;
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
