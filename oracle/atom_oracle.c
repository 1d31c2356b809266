/*
 * Atom W4A4 mixed-precision oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of what the Atom hot path
 * computes. Only the tests, the package's smoke check and the bench's CPU
 * baseline leg may load it. The product path never calls it, and it shares no
 * code, header or constant with the CUDA library.
 *
 * Sources (the Atom pages):
 *  - "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 *    arXiv abstract: 4-bit weight-activation quantization with a mixed-precision,
 *    fine-grained quantization process.
 *  - Same title, paper summary: weights grouped into small blocks with per-group
 *    scales; outliers captured by separate higher-precision channels; activations
 *    get a dedicated outlier path.
 *  - "Atom (mixed-precision block-outlier low-bit quantization for serving)",
 *    fields "Weight group size" (128), "Activation scheme" (outlier channels kept
 *    at higher precision, dense bulk 4-bit) and "notes" (every contiguous run of
 *    128 elements is one group quantized independently; high-precision channel
 *    size 128).
 *
 * Readings where the pages are silent (each one also listed in the design notes):
 *  S1 permutation: reordered position j < Kd = K-128 holds the j-th non-outlier
 *     channel in ascending order; positions Kd..K-1 hold the outlier list in
 *     list order.
 *  S2 scale: amax = max |x| over the group in fp32 (exact from fp16);
 *     scale = amax/qmax and inv = qmax/amax, each one correctly rounded fp32
 *     division; qmax = 7 for the INT4 groups, 127 for the INT8 outlier group;
 *     amax == 0 gives scale = inv = 0 and all-zero codes.
 *  S3 code: t = fl32(x * inv) (one rounded multiply, not fused), q = round
 *     half to even (t), clamped to [-qmax-1, qmax] (the clamp never binds).
 *  S4 packing: byte i of a row holds INT4 elements 2i (low nibble) and 2i+1
 *     (high nibble), 4-bit two's complement; INT8 codes are plain int8.
 *     Scales are stored group-major: scales[g*rows + r].
 *  S5 partials: P[g][m][n] = sum over the 128 k of group g of qa*qw, exact in
 *     int64, required to fit int32.
 *  S6 output: Y64[m][n] = sum_g (double)sa[g][m] * (double)sw[g][n] * P[g][m][n];
 *     Y32 is the same sum taken in fp32, in group order, for information.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * The OpenMP pragmas only split independent rows/columns across threads; the
 * arithmetic of every output element is the sequential loop written here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG (-1)
#define ORACLE_OVERFLOW (-2)

/* IEEE 754 binary16 -> binary32, from the format's definition (exact). */
float atom_oracle_f16_to_f32(uint16_t h)
{
    uint32_t sign = h >> 15, e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
    float mag;
    if (e == 0)
        mag = ldexpf((float)m, -24);                   /* subnormal: m * 2^-24 */
    else if (e == 31)
        mag = m ? NAN : INFINITY;
    else
        mag = ldexpf((float)(m | 0x400u), (int)e - 25); /* (1024+m) * 2^(e-25) */
    return sign ? -mag : mag;
}

/* binary32 -> binary16, round to nearest even (gcc's _Float16 conversion). */
uint16_t atom_oracle_f32_to_f16(float f)
{
    _Float16 h = (_Float16)f;
    uint16_t bits;
    memcpy(&bits, &h, sizeof bits);
    return bits;
}

/* S1: build the reorder permutation. perm[j] = source channel of position j.
 * Returns ORACLE_BAD_ARG when an index is out of range or repeated. */
int atom_oracle_permutation(int64_t K, const int32_t *outlier_idx, int32_t n_outlier,
                            int32_t *perm)
{
    if (K <= 0 || n_outlier <= 0 || n_outlier > K)
        return ORACLE_BAD_ARG;
    unsigned char *is_outlier = (unsigned char *)calloc((size_t)K, 1);
    if (!is_outlier)
        return ORACLE_BAD_ARG;
    for (int32_t i = 0; i < n_outlier; ++i) {
        int32_t c = outlier_idx[i];
        if (c < 0 || c >= K || is_outlier[c]) {
            free(is_outlier);
            return ORACLE_BAD_ARG;
        }
        is_outlier[c] = 1;
    }
    int64_t j = 0;
    for (int64_t c = 0; c < K; ++c)
        if (!is_outlier[c])
            perm[j++] = (int32_t)c;
    for (int32_t i = 0; i < n_outlier; ++i)
        perm[j++] = outlier_idx[i];
    free(is_outlier);
    return ORACLE_OK;
}

/* S2 + S3 for one group of `n` reordered values: writes the scale and codes. */
static void quantize_group(const float *v, int n, int qmax, float *scale_out, int *codes)
{
    float amax = 0.0f;
    for (int k = 0; k < n; ++k) {
        float a = fabsf(v[k]);
        if (a > amax)
            amax = a;
    }
    float scale = 0.0f, inv = 0.0f;
    if (amax > 0.0f) {
        scale = amax / (float)qmax;
        inv = (float)qmax / amax;
    }
    for (int k = 0; k < n; ++k) {
        float t = v[k] * inv;              /* one rounded fp32 multiply */
        float r = nearbyintf(t);           /* ties to even (default rounding mode) */
        int q = (int)r;
        if (q > qmax) q = qmax;
        if (q < -qmax - 1) q = -qmax - 1;
        codes[k] = q;
    }
    *scale_out = scale;
}

/* S1-S4 over `rows` rows of an fp16 matrix x (row stride ld elements).
 * q4: [rows][(K-128)/2] bytes, q8: [rows][128], scales: [K/128][rows]. */
int atom_oracle_quantize(const uint16_t *x, int64_t rows, int64_t K, int64_t ld,
                         const int32_t *outlier_idx, int32_t n_outlier, int32_t group,
                         uint8_t *q4, int8_t *q8, float *scales)
{
    if (group != 128 || n_outlier != 128 || K % 128 != 0 || K < 256 || rows < 0 || ld < K)
        return ORACLE_BAD_ARG;
    int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    if (!perm)
        return ORACLE_BAD_ARG;
    if (atom_oracle_permutation(K, outlier_idx, n_outlier, perm) != ORACLE_OK) {
        free(perm);
        return ORACLE_BAD_ARG;
    }
    const int64_t G = K / 128, Kd = K - 128, row_bytes = Kd / 2;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float v[128];
        int codes[128];
        for (int64_t g = 0; g < G; ++g) {
            for (int k = 0; k < 128; ++k)
                v[k] = atom_oracle_f16_to_f32(x[r * ld + perm[g * 128 + k]]);
            int qmax = (g < G - 1) ? 7 : 127;
            float s;
            quantize_group(v, 128, qmax, &s, codes);
            scales[g * rows + r] = s;
            if (g < G - 1) {
                for (int k = 0; k < 128; k += 2) {
                    unsigned lo = (unsigned)codes[k] & 0xFu, hi = (unsigned)codes[k + 1] & 0xFu;
                    q4[r * row_bytes + (g * 128 + k) / 2] = (uint8_t)(lo | (hi << 4));
                }
            } else {
                for (int k = 0; k < 128; ++k)
                    q8[r * 128 + k] = (int8_t)codes[k];
            }
        }
    }
    free(perm);
    return ORACLE_OK;
}

/* The signed code at reordered position k of one quantized row. */
static int code_at(const uint8_t *q4row, const int8_t *q8row, int64_t Kd, int64_t k)
{
    if (k < Kd) {
        unsigned byte = q4row[k / 2];
        unsigned nib = (k % 2 == 0) ? (byte & 0xFu) : (byte >> 4);
        return (nib & 0x8u) ? (int)nib - 16 : (int)nib;
    }
    return q8row[k - Kd];
}

/* Expand quantized rows into one signed code per reordered position. */
static void decode_rows(const uint8_t *q4, const int8_t *q8, int64_t rows, int64_t K, int8_t *out)
{
    const int64_t Kd = K - 128;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = (int8_t)code_at(q4 + r * (Kd / 2), q8 + r * 128, Kd, k);
}

/* S5: per-group integer partial sums P[g][m][n], int32 [K/128][M][N]. */
int atom_oracle_partials(const uint8_t *qa4, const int8_t *qa8, const uint8_t *qw4,
                         const int8_t *qw8, int64_t M, int64_t N, int64_t K, int32_t *P)
{
    if (K % 128 != 0 || K < 256 || M < 0 || N < 0)
        return ORACLE_BAD_ARG;
    const int64_t G = K / 128;
    int8_t *a = (int8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    int8_t *w = (int8_t *)malloc((size_t)(N * K > 0 ? N * K : 1));
    if (!a || !w) {
        free(a);
        free(w);
        return ORACLE_BAD_ARG;
    }
    decode_rows(qa4, qa8, M, K, a);
    decode_rows(qw4, qw8, N, K, w);
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t g = 0; g < G; ++g) {
                int64_t s = 0;
                for (int64_t k = g * 128; k < g * 128 + 128; ++k)
                    s += (int64_t)a[m * K + k] * (int64_t)w[n * K + k];
                if (s > INT32_MAX || s < INT32_MIN)
                    overflow = 1;
                P[(g * M + m) * N + n] = (int32_t)s;
            }
    free(a);
    free(w);
    return overflow ? ORACLE_OVERFLOW : ORACLE_OK;
}

/* S5 + S6 without materialising P: Y64 (and Y32 if non-null) [M][N].
 * sa: [K/128][M], sw: [K/128][N] (group-major, as the quantizer writes them). */
int atom_oracle_gemm(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                     const uint8_t *qw4, const int8_t *qw8, const float *sw,
                     int64_t M, int64_t N, int64_t K, double *Y64, float *Y32)
{
    if (K % 128 != 0 || K < 256 || M < 0 || N < 0)
        return ORACLE_BAD_ARG;
    const int64_t G = K / 128;
    int8_t *a = (int8_t *)malloc((size_t)(M * K > 0 ? M * K : 1));
    int8_t *w = (int8_t *)malloc((size_t)(N * K > 0 ? N * K : 1));
    if (!a || !w) {
        free(a);
        free(w);
        return ORACLE_BAD_ARG;
    }
    decode_rows(qa4, qa8, M, K, a);
    decode_rows(qw4, qw8, N, K, w);
    int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double y64 = 0.0;
            float y32 = 0.0f;
            for (int64_t g = 0; g < G; ++g) {
                int64_t s = 0;
                for (int64_t k = g * 128; k < g * 128 + 128; ++k)
                    s += (int64_t)a[m * K + k] * (int64_t)w[n * K + k];
                if (s > INT32_MAX || s < INT32_MIN)
                    overflow = 1;
                float sa_ = sa[g * M + m], sw_ = sw[g * N + n];
                y64 += (double)sa_ * (double)sw_ * (double)s;
                y32 += (sa_ * sw_) * (float)s;
            }
            Y64[m * N + n] = y64;
            if (Y32)
                Y32[m * N + n] = y32;
        }
    free(a);
    free(w);
    return overflow ? ORACLE_OVERFLOW : ORACLE_OK;
}

/* Dequantize rows to fp64: out[r][k] = code(r,k) * scale(group(k), r), reordered. */
int atom_oracle_dequantize(const uint8_t *q4, const int8_t *q8, const float *scales,
                           int64_t rows, int64_t K, double *out)
{
    if (K % 128 != 0 || K < 256 || rows < 0)
        return ORACLE_BAD_ARG;
    const int64_t Kd = K - 128;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = (double)code_at(q4 + r * (Kd / 2), q8 + r * 128, Kd, k) *
                             (double)scales[(k / 128) * rows + r];
    return ORACLE_OK;
}
