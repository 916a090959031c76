/*
 * hq_oracle.c -- plain, slow, obviously correct CPU oracle for the W4A4
 * rotated linear layer.  TEST INFRASTRUCTURE ONLY: it is built and called by
 * the test suite, by the smoke check and by the benchmark's CPU-baseline leg,
 * never by the product path.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (page title, section):
 *  [OffQ]  "OffQ: Taming Structured Outliers in LLM Quantization by
 *          Offsetting", Methodology 2 (absorption by a Hadamard rotation whose
 *          first row is all ones) and Methodology 3 (group-wise application).
 *  [SERQ]  "SERQ: Saliency-Aware Low-Rank Error Reconstruction for LLM
 *          Quantization", Technical summary section 1 (W4A4, activation
 *          outliers), section 2.2 (saliency-aware error reconstruction with
 *          one low-rank matrix R on the salient rows, residual path in 4 bit)
 *          and section 2.3 (offline permutation).
 *  [CMPQ]  "Adaptación a cualquier ancho de bits: Cuantización de precisión
 *          mixta por canal para LLMs", Methodology A (per-channel activation
 *          L2 norm as the saliency heuristic).
 *  [WaterSIC] "WaterSIC: information-theoretically (near) optimal linear
 *          layer quantization", Technical summary section 1 (a linear layer
 *          computes Y = W X).
 *  [DynamicPTQ] "DynamicPTQ", Methodology 2 (8-bit activations on the
 *          quantisation-sensitive layers, weights and everything else in 4
 *          bit); SERQ section 4 evaluates the same layer at W4A8.
 *  [OffQ-A] "OffQ ...", Methodology 2, last point (the constant offset the
 *          rotation creates is absorbed by the zero point of an asymmetric
 *          quantiser) and Methodology 3 (one scale and zero point per group).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes): H = diag(d) * Sylvester(g), d a +-1 vector with d[0] = +1; the
 * butterfly runs in fp32 over stages h = 1, 2, 4, ... in ascending order with
 * (a, b) -> (a + b, a - b); 1/sqrt(g) is folded into the activation scale;
 * activation codes are round-half-even(u * fl32(7 / amax)) in [-7, 7];
 * element 2j sits in the low nibble of byte j.
 *
 * Build: gcc -O2 -std=c99 -fPIC -shared -ffp-contract=off -fno-fast-math
 *        -fexcess-precision=standard -fopenmp  (see build_oracle.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar format conversions (IEEE 754 binary16 / bfloat16 <-> binary32).    */
/* ------------------------------------------------------------------------ */

static float bits_to_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

/* binary16 -> binary32, exact. */
float hqo_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu;
    uint32_t m = h & 0x3FFu;
    if (e == 0x1Fu) return bits_to_f32(sign | 0x7F800000u | (m << 13));
    if (e == 0) {
        /* zero or subnormal: m * 2^-24, exact in binary32 */
        float v = (float)m * 5.9604644775390625e-08f;
        return sign ? -v : v;
    }
    return bits_to_f32(sign | ((e + 112u) << 23) | (m << 13));
}

/* binary32 -> binary16, round to nearest, ties to even. */
uint16_t hqo_f32_to_f16(float f)
{
    uint32_t x = f32_to_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7FFFFFFFu;
    if (ax >= 0x7F800000u) /* inf / nan */
        return (uint16_t)(sign | 0x7C00u | (ax > 0x7F800000u ? 0x200u : 0u));
    if (ax >= 0x477FF000u) /* >= 65520 rounds to inf */
        return (uint16_t)(sign | 0x7C00u);
    if (ax < 0x38800000u) { /* below 2^-14: fp16 subnormal grid k * 2^-24 */
        float a = bits_to_f32(ax) * 16777216.0f; /* exact power-of-two scale */
        float k = rintf(a);                      /* ties to even */
        return (uint16_t)(sign | (uint16_t)k);
    }
    uint32_t mant = ax & 0x7FFFFFu;
    uint32_t e = (ax >> 23) - 127u + 15u;
    uint32_t h = (e << 10) | (mant >> 13);
    uint32_t rem = mant & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h++;
    return (uint16_t)(sign | h);
}

float hqo_bf16_to_f32(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

/* Input element types of the activation / weight buffers. */
enum { HQO_F16 = 0, HQO_BF16 = 1, HQO_F32 = 2 };

static float load_elem(const void* p, int dtype, int64_t i)
{
    if (dtype == HQO_F16) return hqo_f16_to_f32(((const uint16_t*)p)[i]);
    if (dtype == HQO_BF16) return hqo_bf16_to_f32(((const uint16_t*)p)[i]);
    return ((const float*)p)[i];
}

/* ------------------------------------------------------------------------ */
/* The Hadamard matrix [OffQ, Methodology 2].                                */
/* ------------------------------------------------------------------------ */

static int popcount32(uint32_t v)
{
    int c = 0;
    while (v) { c += (int)(v & 1u); v >>= 1; }
    return c;
}

/* Dense g x g matrix H[i][j] = d[i] * (-1)^popcount(i & j).  With d[0] = +1
 * the first row is all ones.  d == NULL means d = 1. */
void hqo_hadamard_dense(int32_t g, const int8_t* d, int8_t* H)
{
    for (int32_t i = 0; i < g; ++i)
        for (int32_t j = 0; j < g; ++j) {
            int s = (popcount32((uint32_t)(i & j)) & 1) ? -1 : 1;
            H[(int64_t)i * g + j] = (int8_t)(s * (d ? d[i] : 1));
        }
}

/* ------------------------------------------------------------------------ */
/* Grouped rotation u = (x .* d) * H_sylv per group, fp32 butterfly.         */
/* ------------------------------------------------------------------------ */

/* One group of g values, in place: sign flip, then stages h = 1, 2, ..., g/2
 * with u[i], u[i+h] <- u[i] + u[i+h], u[i] - u[i+h] for every i with i&h = 0.
 * This is x * diag(d) * H_sylv (row vector times matrix), unnormalised. */
static void fwht_group(float* u, int32_t g, const int8_t* d)
{
    if (d)
        for (int32_t i = 0; i < g; ++i)
            if (d[i] < 0) u[i] = -u[i];
    for (int32_t h = 1; h < g; h <<= 1)
        for (int32_t i = 0; i < g; ++i)
            if ((i & h) == 0) {
                float a = u[i], b = u[i + h];
                u[i] = a + b;
                u[i + h] = a - b;
            }
}

/* u[M][K] = rotated rows of X (unnormalised).  K % g == 0. */
void hqo_rotate_rows(const void* X, int dtype, int64_t M, int64_t K, int32_t g,
                     const int8_t* d, float* u)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float* row = u + m * K;
        for (int64_t k = 0; k < K; ++k) row[k] = load_elem(X, dtype, m * K + k);
        for (int64_t b = 0; b < K / g; ++b) fwht_group(row + b * g, g, d);
    }
}

/* The orthonormal rotation x * blockdiag(H)/sqrt(g), as used to fold the
 * rotation into the weights: out = fl32(u * fl32(1/sqrt(g))). */
void hqo_rotate_normalised(const void* W, int dtype, int64_t N, int64_t K, int32_t g,
                           const int8_t* d, float* out)
{
    float cg = (float)(1.0 / sqrt((double)g));
    hqo_rotate_rows(W, dtype, N, K, g, d, out);
    for (int64_t i = 0; i < N * K; ++i) out[i] = out[i] * cg;
}

/* Dense fp64 product x * blockdiag(H), the cross-check of the butterfly. */
void hqo_rotate_dense_f64(const void* X, int dtype, int64_t M, int64_t K, int32_t g,
                          const int8_t* d, double* out)
{
    int8_t* H = (int8_t*)malloc((size_t)g * (size_t)g);
    hqo_hadamard_dense(g, d, H);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t b = 0; b < K / g; ++b)
            for (int32_t j = 0; j < g; ++j) {
                double acc = 0.0;
                for (int32_t i = 0; i < g; ++i)
                    acc += (double)load_elem(X, dtype, m * K + b * g + i) * (double)H[(int64_t)i * g + j];
                out[m * K + b * g + j] = acc;
            }
    free(H);
}

/* ------------------------------------------------------------------------ */
/* Nibble packing: element 2j -> low nibble of byte j, 2j+1 -> high nibble.  */
/* ------------------------------------------------------------------------ */

static void put_nibble(uint8_t* row, int64_t k, int v)
{
    uint8_t nib = (uint8_t)(v & 0xF);
    if (k & 1) row[k >> 1] = (uint8_t)((row[k >> 1] & 0x0F) | (nib << 4));
    else       row[k >> 1] = (uint8_t)((row[k >> 1] & 0xF0) | nib);
}

static int get_nibble_s(const uint8_t* row, int64_t k) /* two's complement */
{
    int v = (row[k >> 1] >> ((k & 1) * 4)) & 0xF;
    return v >= 8 ? v - 16 : v;
}

static int get_nibble_u(const uint8_t* row, int64_t k) /* unsigned 0..15 */
{
    return (row[k >> 1] >> ((k & 1) * 4)) & 0xF;
}

void hqo_pack_s4(const int8_t* q, int64_t rows, int64_t cols, uint8_t* packed)
{
    int64_t ld = (cols + 1) / 2;
    memset(packed, 0, (size_t)(rows * ld));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) put_nibble(packed + r * ld, c, q[r * cols + c]);
}

void hqo_unpack_s4(const uint8_t* packed, int64_t rows, int64_t cols, int8_t* q)
{
    int64_t ld = (cols + 1) / 2;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) q[r * cols + c] = (int8_t)get_nibble_s(packed + r * ld, c);
}

void hqo_unpack_u4(const uint8_t* packed, int64_t rows, int64_t cols, int8_t* q)
{
    int64_t ld = (cols + 1) / 2;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) q[r * cols + c] = (int8_t)get_nibble_u(packed + r * ld, c);
}

/* ------------------------------------------------------------------------ */
/* Online activation path: rotate, per-token symmetric int4 [SERQ s1, OffQ]. */
/* ------------------------------------------------------------------------ */

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Per row m: u = rotated row; amax = max |u|; if amax == 0 the codes are 0
 * and sx = 0; else s = fl32(amax / 7), inv = fl32(7 / amax),
 * q = clamp(rint(fl32(u * inv)), -7, 7), sx = fl32(s * fl32(1/sqrt(g))).
 * Xq is [M][K/2] packed; sx is [M].  u_out (optional) receives u. */
void hqo_rotate_quant(const void* X, int dtype, int64_t M, int64_t K, int32_t g,
                      const int8_t* d, uint8_t* Xq, float* sx, float* u_out)
{
    float cg = (float)(1.0 / sqrt((double)g));
    float* u = u_out ? u_out : (float*)malloc((size_t)(M * K) * sizeof(float));
    hqo_rotate_rows(X, dtype, M, K, g, d, u);
    memset(Xq, 0, (size_t)(M * (K / 2)));
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const float* row = u + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(row[k]));
        uint8_t* qrow = Xq + m * (K / 2);
        if (amax == 0.0f) { sx[m] = 0.0f; continue; }
        float s = amax / 7.0f;
        float inv = 7.0f / amax;
        sx[m] = s * cg;
        for (int64_t k = 0; k < K; ++k) {
            float t = row[k] * inv;
            int q = (int)clampf(rintf(t), -7.0f, 7.0f);
            put_nibble(qrow, k, q);
        }
    }
    if (!u_out) free(u);
}

/* W4A8 activations [DynamicPTQ Methodology 2; SERQ s4]: the same rotation
 * and per-token symmetric quantiser with 8-bit codes.  Per row m: amax =
 * max |u|; if amax == 0 the codes are 0 and sx = 0; else
 * s = fl32(amax / 127), inv = fl32(127 / amax),
 * q = clamp(rint(fl32(u * inv)), -127, 127), sx = fl32(s * fl32(1/sqrt(g))).
 * Xq8 is [M][K] int8 (one code per byte); sx is [M]. */
void hqo_rotate_quant8(const void* X, int dtype, int64_t M, int64_t K, int32_t g,
                       const int8_t* d, int8_t* Xq8, float* sx)
{
    float cg = (float)(1.0 / sqrt((double)g));
    float* u = (float*)malloc((size_t)(M * K) * sizeof(float));
    hqo_rotate_rows(X, dtype, M, K, g, d, u);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const float* row = u + m * K;
        int8_t* qrow = Xq8 + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(row[k]));
        if (amax == 0.0f) {
            sx[m] = 0.0f;
            memset(qrow, 0, (size_t)K);
            continue;
        }
        float s = amax / 127.0f;
        float inv = 127.0f / amax;
        sx[m] = s * cg;
        for (int64_t k = 0; k < K; ++k) {
            float t = row[k] * inv;
            qrow[k] = (int8_t)(int)clampf(rintf(t), -127.0f, 127.0f);
        }
    }
    free(u);
}

/* The W4A8 integer GEMM: as hqo_accum with 8-bit activation codes
 * (Xq8 [M][K] int8): acc[m][n][b] = sum_{k in group b} qx[m][k] *
 * (qw[n][k] - z[b][n]), acc_c[m][n] = sum_{j<r} qx[m][S_j] * qr[n][j].
 * Plain triple loop in int64; returns 1 if any value does not fit in int32. */
int hqo_accum8(const int8_t* Xq8, int64_t M, int64_t K, const uint8_t* Wq, const uint16_t* zw,
               int64_t N, int32_t gw, const uint8_t* Rq, const int32_t* sal, int32_t r,
               int64_t* acc, int64_t* acc_c);

/* ------------------------------------------------------------------------ */
/* Weight quantiser w4_pack.                                                 */
/* ------------------------------------------------------------------------ */

/* gw == 0: per-output-channel symmetric.  s16 = fl16(fl32(amax/7)); if s16
 *   is zero the codes are 0; q = clamp(rint(fl32(w / s16)), -8, 7),
 *   two's complement nibbles; sw[n] = s16; zw untouched.
 * gw  > 0: per (channel, group of gw inputs) asymmetric with the grid
 *   spanning [min(mn,0), max(mx,0)]: s16 = fl16(fl32(fl32(hi - lo) / 15)), 1
 *   if that is zero; z = clamp(rint(fl32(-lo / s16)), 0, 15);
 *   q = clamp(rint(fl32(w / s16)) + z, 0, 15), unsigned nibbles;
 *   sw[b][n] = s16, zw[b][n] = fl16(z) (exact): group-major [K/gw][N].
 * The stored (rounded) scale is the one used to form the codes. */
void hqo_w4_pack(const void* W, int dtype, int64_t N, int64_t K, int32_t gw,
                 uint8_t* Wq, uint16_t* sw, uint16_t* zw)
{
    memset(Wq, 0, (size_t)(N * (K / 2)));
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        uint8_t* qrow = Wq + n * (K / 2);
        if (gw == 0) {
            float amax = 0.0f;
            for (int64_t k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(load_elem(W, dtype, n * K + k)));
            uint16_t s16 = hqo_f32_to_f16(amax / 7.0f);
            float s = hqo_f16_to_f32(s16);
            sw[n] = s16;
            for (int64_t k = 0; k < K; ++k) {
                int q = 0;
                if (s != 0.0f) q = (int)clampf(rintf(load_elem(W, dtype, n * K + k) / s), -8.0f, 7.0f);
                put_nibble(qrow, k, q);
            }
        } else {
            int64_t G = K / gw;
            for (int64_t b = 0; b < G; ++b) {
                float lo = 0.0f, hi = 0.0f;
                for (int64_t k = b * gw; k < (b + 1) * gw; ++k) {
                    float w = load_elem(W, dtype, n * K + k);
                    lo = fminf(lo, w);
                    hi = fmaxf(hi, w);
                }
                uint16_t s16 = hqo_f32_to_f16((hi - lo) / 15.0f);
                if (hqo_f16_to_f32(s16) == 0.0f) s16 = 0x3C00u; /* 1.0 */
                float s = hqo_f16_to_f32(s16);
                /* an integer in 0..15; the int round trip makes a zero +0 (never -0) */
                float z = (float)(int)clampf(rintf(-lo / s), 0.0f, 15.0f);
                sw[b * N + n] = s16;
                zw[b * N + n] = hqo_f32_to_f16(z);
                for (int64_t k = b * gw; k < (b + 1) * gw; ++k) {
                    float w = load_elem(W, dtype, n * K + k);
                    int q = (int)clampf(rintf(w / s) + z, 0.0f, 15.0f);
                    put_nibble(qrow, k, q);
                }
            }
        }
    }
}

/* Dequantised weight value of element (n, k), exact in fp32. */
static float w_dequant(const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw,
                       int64_t N, int64_t K, int32_t gw, int64_t n, int64_t k)
{
    const uint8_t* row = Wq + n * (K / 2);
    if (gw == 0) return (float)get_nibble_s(row, k) * hqo_f16_to_f32(sw[n]);
    int64_t b = k / gw;
    float z = hqo_f16_to_f32(zw[b * N + n]);
    return ((float)get_nibble_u(row, k) - z) * hqo_f16_to_f32(sw[b * N + n]);
}

void hqo_w4_dequant(const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw,
                    int64_t N, int64_t K, int32_t gw, float* What)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) What[n * K + k] = w_dequant(Wq, sw, zw, N, K, gw, n, k);
}

/* ------------------------------------------------------------------------ */
/* SERQ single low-rank error matrix on the salient inputs [SERQ s2.2].      */
/* ------------------------------------------------------------------------ */

/* E_S[n][j] = fl32(W_rot[n][S_j] - What[n][S_j]) for the r salient input
 * channels S; R is quantised per output row like a symmetric weight row:
 * sr[n] = fl16(fl32(amax_j |E_S[n][j]| / 7)), Rq codes in [-8, 7] packed
 * [N][ceil(r/2)].  e_out (optional) receives E_S as fp32 [N][r]. */
void hqo_serq_prepare(const float* Wrot, int64_t N, int64_t K, const uint8_t* Wq,
                      const uint16_t* sw, const uint16_t* zw, int32_t gw,
                      const int32_t* sal, int32_t r, uint8_t* Rq, uint16_t* sr, float* e_out)
{
    int64_t ld = (r + 1) / 2;
    memset(Rq, 0, (size_t)(N * ld));
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float* e = (float*)malloc((size_t)(r > 0 ? r : 1) * sizeof(float));   /* any r */
        float amax = 0.0f;
        for (int32_t j = 0; j < r; ++j) {
            int64_t k = sal[j];
            e[j] = Wrot[n * K + k] - w_dequant(Wq, sw, zw, N, K, gw, n, k);
            amax = fmaxf(amax, fabsf(e[j]));
            if (e_out) e_out[n * r + j] = e[j];
        }
        uint16_t s16 = hqo_f32_to_f16(amax / 7.0f);
        float s = hqo_f16_to_f32(s16);
        sr[n] = s16;
        for (int32_t j = 0; j < r; ++j) {
            int q = 0;
            if (s != 0.0f) q = (int)clampf(rintf(e[j] / s), -8.0f, 7.0f);
            put_nibble(Rq + n * ld, j, q);
        }
        free(e);
    }
}

/* ------------------------------------------------------------------------ */
/* Integer GEMM and epilogue [SERQ s2.2, s3; WaterSIC s1: Y = W X].          */
/* ------------------------------------------------------------------------ */

/* acc[m][n][b] = sum_{k in group b} qx[m][k] * (qw[n][k] - z[b][n]) in int64
 * (one group when gw == 0, with symmetric weight codes), and
 * acc_c[m][n] = sum_{j<r} qx[m][S_j] * qr[n][j].  Plain triple loop.
 * Returns 0, or 1 if any value does not fit in int32. */
int hqo_accum(const uint8_t* Xq, int64_t M, int64_t K, const uint8_t* Wq, const uint16_t* zw,
              int64_t N, int32_t gw, const uint8_t* Rq, const int32_t* sal, int32_t r,
              int64_t* acc, int64_t* acc_c)
{
    int64_t G = gw ? K / gw : 1;
    int64_t glen = gw ? gw : K;
    int64_t ldr = (r + 1) / 2;
    int overflow = 0;
    #pragma omp parallel for schedule(static) reduction(|:overflow)
    for (int64_t m = 0; m < M; ++m) {
        const uint8_t* xrow = Xq + m * (K / 2);
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wrow = Wq + n * (K / 2);
            for (int64_t b = 0; b < G; ++b) {
                int64_t s = 0;
                int z = gw ? (int)hqo_f16_to_f32(zw[b * N + n]) : 0;
                for (int64_t k = b * glen; k < (b + 1) * glen; ++k) {
                    int wv = gw ? get_nibble_u(wrow, k) - z : get_nibble_s(wrow, k);
                    s += (int64_t)get_nibble_s(xrow, k) * wv;
                }
                acc[(m * N + n) * G + b] = s;
                if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
            }
            int64_t c = 0;
            for (int32_t j = 0; j < r; ++j)
                c += (int64_t)get_nibble_s(xrow, sal[j]) * get_nibble_s(Rq + n * ldr, j);
            if (acc_c) acc_c[m * N + n] = c;
        }
    }
    return overflow;
}

int hqo_accum8(const int8_t* Xq8, int64_t M, int64_t K, const uint8_t* Wq, const uint16_t* zw,
               int64_t N, int32_t gw, const uint8_t* Rq, const int32_t* sal, int32_t r,
               int64_t* acc, int64_t* acc_c)
{
    int64_t G = gw ? K / gw : 1;
    int64_t glen = gw ? gw : K;
    int64_t ldr = (r + 1) / 2;
    int overflow = 0;
    #pragma omp parallel for schedule(static) reduction(|:overflow)
    for (int64_t m = 0; m < M; ++m) {
        const int8_t* xrow = Xq8 + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wrow = Wq + n * (K / 2);
            for (int64_t b = 0; b < G; ++b) {
                int64_t s = 0;
                int z = gw ? (int)hqo_f16_to_f32(zw[b * N + n]) : 0;
                for (int64_t k = b * glen; k < (b + 1) * glen; ++k) {
                    int wv = gw ? get_nibble_u(wrow, k) - z : get_nibble_s(wrow, k);
                    s += (int64_t)xrow[k] * wv;
                }
                acc[(m * N + n) * G + b] = s;
                if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
            }
            int64_t c = 0;
            for (int32_t j = 0; j < r; ++j)
                c += (int64_t)xrow[sal[j]] * get_nibble_s(Rq + n * ldr, j);
            if (acc_c) acc_c[m * N + n] = c;
        }
    }
    return overflow;
}

/* y64[m][n] = sx[m] * (sum_b sw[b][n] * acc[m][n][b] + sr[n] * acc_c[m][n]),
 * evaluated in fp64 from the exact integers: the ground truth of the
 * dequantising epilogue.  sr / acc_c may be NULL (no correction). */
void hqo_epilogue_f64(const int64_t* acc, const int64_t* acc_c, int64_t M, int64_t N, int64_t G,
                      const float* sx, const uint16_t* sw, const uint16_t* sr, double* y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double t = 0.0;
            for (int64_t b = 0; b < G; ++b)
                t += (double)hqo_f16_to_f32(sw[b * N + n]) * (double)acc[(m * N + n) * G + b];
            if (acc_c && sr) t += (double)hqo_f16_to_f32(sr[n]) * (double)acc_c[m * N + n];
            y[m * N + n] = (double)sx[m] * t;
        }
}

/* Full layer for selected rows only (sampling at large sizes): the same
 * definitions as hqo_accum + hqo_epilogue_f64, for rows rows[0..nr). */
void hqo_linear_rows_f64(const uint8_t* Xq, const float* sx, int64_t K, const uint8_t* Wq,
                         const uint16_t* sw, const uint16_t* zw, int64_t N, int32_t gw,
                         const uint8_t* Rq, const uint16_t* sr, const int32_t* sal, int32_t r,
                         const int64_t* rows, int64_t nr, double* y)
{
    int64_t G = gw ? K / gw : 1;
    int64_t glen = gw ? gw : K;
    int64_t ldr = (r + 1) / 2;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nr; ++i) {
        const uint8_t* xrow = Xq + rows[i] * (K / 2);
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wrow = Wq + n * (K / 2);
            double t = 0.0;
            for (int64_t b = 0; b < G; ++b) {
                int64_t s = 0;
                int z = gw ? (int)hqo_f16_to_f32(zw[b * N + n]) : 0;
                for (int64_t k = b * glen; k < (b + 1) * glen; ++k) {
                    int wv = gw ? get_nibble_u(wrow, k) - z : get_nibble_s(wrow, k);
                    s += (int64_t)get_nibble_s(xrow, k) * wv;
                }
                t += (double)hqo_f16_to_f32(sw[b * N + n]) * (double)s;
            }
            if (r > 0) {
                int64_t c = 0;
                for (int32_t j = 0; j < r; ++j)
                    c += (int64_t)get_nibble_s(xrow, sal[j]) * get_nibble_s(Rq + n * ldr, j);
                t += (double)hqo_f16_to_f32(sr[n]) * (double)c;
            }
            y[i * N + n] = (double)sx[rows[i]] * t;
        }
    }
}

/* Unquantised reference Y = X * W^T in fp64 (for reporting the quantisation
 * error only). */
void hqo_linear_fp64(const void* X, int xdtype, int64_t M, int64_t K, const void* W, int wdtype,
                     int64_t N, double* y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double t = 0.0;
            for (int64_t k = 0; k < K; ++k)
                t += (double)load_elem(X, xdtype, m * K + k) * (double)load_elem(W, wdtype, n * K + k);
            y[m * N + n] = t;
        }
}

/* ------------------------------------------------------------------------ */
/* Calibration: salient input channels [CMPQ Methodology A; SERQ s2.2].      */
/* ------------------------------------------------------------------------ */

/* norm2[k] = sum_m (X * blockdiag(H))[m][k]^2 in fp64 (dense product), then
 * the r largest, ties to the lower index, returned in ascending index order. */
void hqo_salient_channels(const void* X, int dtype, int64_t M, int64_t K, int32_t g,
                          const int8_t* d, int32_t r, double* norm2, int32_t* sal)
{
    double* rot = (double*)malloc((size_t)(M * K) * sizeof(double));
    hqo_rotate_dense_f64(X, dtype, M, K, g, d, rot);
    for (int64_t k = 0; k < K; ++k) {
        double s = 0.0;
        for (int64_t m = 0; m < M; ++m) s += rot[m * K + k] * rot[m * K + k];
        norm2[k] = s;
    }
    free(rot);
    char* taken = (char*)calloc((size_t)K, 1);
    for (int32_t j = 0; j < r; ++j) {
        int64_t best = -1;
        for (int64_t k = 0; k < K; ++k)
            if (!taken[k] && (best < 0 || norm2[k] > norm2[best])) best = k;
        if (best < 0) break; /* r > K: every channel is taken */
        taken[best] = 1;
    }
    int32_t c = 0;
    for (int64_t k = 0; k < K; ++k)
        if (taken[k]) sal[c++] = (int32_t)k;
    free(taken);
}

/* Array forms of the scalar conversions (used by the Python wrapper). */
void hqo_f32_to_f16_array(const float* in, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = hqo_f32_to_f16(in[i]);
}

void hqo_f16_to_f32_array(const uint16_t* in, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = hqo_f16_to_f32(in[i]);
}

/* ------------------------------------------------------------------------ */
/* OffQ per-group asymmetric activations [OffQ-A].                           */
/* ------------------------------------------------------------------------ */

/* Per row m and Hadamard group b (g channels): u = the rotated group;
 * lo = min u, hi = max u, dlt = fl32(hi - lo) (the group's own range: the
 * offset is not forced into it); a constant group takes dlt = |lo| (15 when
 * lo == 0), so it is reconstructed exactly.  s = fl32(dlt / 15),
 * inv = fl32(15 / dlt), z = rint(fl32(-lo * inv)) (an integer, not clamped:
 * an all-positive group has z < 0), q = clamp(rint(fl32(u * inv)) + z, 0, 15),
 * unsigned nibbles.  sx[m][b] = fl32(s * fl32(1/sqrt(g))), zx[m][b] = z.
 * Xq is [M][K/2] packed; sx, zx are [M][K/g]. */
void hqo_rotate_quant_asym(const void* X, int dtype, int64_t M, int64_t K, int32_t g,
                           const int8_t* d, uint8_t* Xq, float* sx, int32_t* zx)
{
    float cg = (float)(1.0 / sqrt((double)g));
    int64_t G = K / g;
    float* u = (float*)malloc((size_t)(M * K) * sizeof(float));
    hqo_rotate_rows(X, dtype, M, K, g, d, u);
    memset(Xq, 0, (size_t)(M * (K / 2)));
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        uint8_t* qrow = Xq + m * (K / 2);
        for (int64_t b = 0; b < G; ++b) {
            const float* gu = u + m * K + b * g;
            float lo = gu[0], hi = gu[0];
            for (int32_t k = 1; k < g; ++k) {
                lo = fminf(lo, gu[k]);
                hi = fmaxf(hi, gu[k]);
            }
            float dlt = hi - lo;
            if (dlt == 0.0f) dlt = lo != 0.0f ? fabsf(lo) : 15.0f;
            float s = dlt / 15.0f;
            float inv = 15.0f / dlt;
            float zf = rintf(-lo * inv);
            int32_t z = (int32_t)zf;
            sx[m * G + b] = s * cg;
            zx[m * G + b] = z;
            for (int32_t k = 0; k < g; ++k) {
                float t = gu[k] * inv;
                int q = (int)clampf(rintf(t) + zf, 0.0f, 15.0f);
                put_nibble(qrow, b * g + k, q);
            }
        }
    }
    free(u);
}

/* The integer GEMM with per-group asymmetric activations (activation groups
 * of g inputs, nested in the weight groups: gw == 0 or gw % g == 0):
 *   acc[m][n][b]   = sum_{k in group b} (qx[m][k] - zx[m][b]) * wv[n][k]
 *   acc_c[m][n][b] = sum_{j: S_j in group b} (qx[m][S_j] - zx[m][b]) * qr[n][j]
 * wv = qw - z_w (group weights) or the signed code (per channel).  Plain
 * loops in int64; returns 1 if any value does not fit in int32. */
int hqo_accum_asym(const uint8_t* Xq, const int32_t* zx, int64_t M, int64_t K, int32_t g,
                   const uint8_t* Wq, const uint16_t* zw, int64_t N, int32_t gw,
                   const uint8_t* Rq, const int32_t* sal, int32_t r, int64_t* acc, int64_t* acc_c)
{
    int64_t G = K / g;
    int64_t ldr = (r + 1) / 2;
    int overflow = 0;
    #pragma omp parallel for schedule(static) reduction(|:overflow)
    for (int64_t m = 0; m < M; ++m) {
        const uint8_t* xrow = Xq + m * (K / 2);
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* wrow = Wq + n * (K / 2);
            for (int64_t b = 0; b < G; ++b) {
                int64_t zb = zx[m * G + b];
                int64_t s = 0;
                for (int64_t k = b * g; k < (b + 1) * g; ++k) {
                    int wv = gw ? get_nibble_u(wrow, k) - (int)hqo_f16_to_f32(zw[(k / gw) * N + n])
                                : get_nibble_s(wrow, k);
                    s += ((int64_t)get_nibble_u(xrow, k) - zb) * wv;
                }
                acc[(m * N + n) * G + b] = s;
                if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
                if (acc_c) {
                    int64_t c = 0;
                    for (int32_t j = 0; j < r; ++j)
                        if (sal[j] / g == b)
                            c += ((int64_t)get_nibble_u(xrow, sal[j]) - zb) * get_nibble_s(Rq + n * ldr, j);
                    acc_c[(m * N + n) * G + b] = c;
                }
            }
        }
    }
    return overflow;
}

/* y64[m][n] = sum_b sx[m][b] * (sw[b'][n] * acc[m][n][b] + sr[n] * acc_c[m][n][b]),
 * b' = the weight group holding activation group b (b' = 0 per channel),
 * in fp64 from the exact integers.  sr / acc_c may be NULL. */
void hqo_epilogue_asym_f64(const int64_t* acc, const int64_t* acc_c, int64_t M, int64_t N, int64_t G,
                           int32_t g, int32_t gw, const float* sx, const uint16_t* sw, const uint16_t* sr,
                           double* y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double t = 0.0;
            for (int64_t b = 0; b < G; ++b) {
                int64_t bw = gw ? (b * g) / gw : 0;
                double part = (double)hqo_f16_to_f32(sw[bw * N + n]) * (double)acc[(m * N + n) * G + b];
                if (acc_c && sr) part += (double)hqo_f16_to_f32(sr[n]) * (double)acc_c[(m * N + n) * G + b];
                t += (double)sx[m * G + b] * part;
            }
            y[m * N + n] = t;
        }
}
