/*
 * CPU oracle for the W4A16 weight-only matmul.  TEST INFRASTRUCTURE ONLY:
 * the tests, the smoke check and the CPU-baseline leg of the benchmark call
 * this file; the library's product path never does.  It shares no code,
 * header, table or constant generator with the CUDA kernels.
 *
 * What it computes, in the order the method takes its steps:
 *
 *   1. quantize  -- "quantizes a 2D matrix from FP16 to INT4" in three
 *      modes, GLOBAL / ROWWISE / GROUPWISE(g)   (anaaaiva/llm-quantization,
 *      Objective 1 and its mode table).  The page prints no formula; the
 *      reading taken here is asymmetric min-max to uint4 with an integer
 *      zero point, w ~= (q - z) * s, fp16 s and z per group:
 *          s = fp16_rn((max - min) / 15)        (IEEE fp32 divide)
 *          if s == 0:  s = fp16_rn(max(|min|, 2^-14))   (degenerate group)
 *          z = clamp(rint(-min / s), 0, 15)
 *          q = clamp(rint(w / s) + z, 0, 15)
 *      every step in IEEE fp32, round-half-even, no contraction; clamps are
 *      taken with fmaxf/fminf so that a NaN lands on 0 on every platform.
 *      Two format flags, or-ed into the mode, give the variants with a
 *      fractional zero point and with bf16 metadata ("Re-write HQQ Fused
 *      Gemm Transpose": the HQQ fused GEMM, whose quantizer keeps a float
 *      zero point; fp16 or bf16 scales are both allowed):
 *        FLOAT_ZERO  z = meta_rn(-min / s), not rounded to an integer or
 *                    clamped to [0, 15] (only to the finite range of the
 *                    metadata type), and q = clamp(rint(w / s + z), 0, 15):
 *                    the sum is rounded, as round(w / s + z) reads;
 *        META_BF16   s and z are stored as bf16 instead of fp16: every
 *                    meta_rn above is a bf16 rounding, and the degenerate
 *                    group's s is bf16_rn(max(|min|, 2^-14)).
 *   2. pack      -- "packs the quantized matrix into INT8 or INT32": eight
 *      codes per uint32 along K, code i of word j at bits 4i..4i+3, which
 *      is byte-identical to two codes per byte with the low nibble first.
 *   3. dequant   -- w_hat = (q - z) * s   (exact in fp64; also in fp32 when
 *      z is an integer).
 *   4. matmul    -- Y = X_bf16 @ W_int4^T  (Objective 2), accumulated in
 *      fp64 over ascending k, plus an optional bias per output column
 *      (vLLM "Adding bias epilogue support for cutlass_scaled_mm": bias
 *      dtype equals the output dtype), rounded once to bf16.
 *   5. transposed matmul -- dX = dY @ w_hat from the same packed weights,
 *      scales and zeros ("Re-write HQQ Fused Gemm Transpose": pass
 *      transposed=True, no repacking, no reshaping of scales or zeros),
 *      accumulated in fp64 over ascending n.
 *
 * Layouts: W bf16 [N,K] row-major; codes uint8 [N,K]; packed uint32
 * [N,K/8]; scales and zeros fp16 (or bf16) bit patterns [N,G] row-major
 * with G = K/g (ROWWISE [N,1], GLOBAL [1,1]).  bf16 and fp16 values cross
 * this API as uint16 bit patterns.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared (no -ffast-math).
 * OpenMP runs over output rows or columns only; each output element is
 * summed by one thread in a fixed order, so results do not depend on the
 * thread count.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

#define MODE_GLOBAL 0
#define MODE_ROWWISE 1
#define MODE_GROUPWISE 2
#define MODE_BASE_MASK 0x0F
#define FLAG_FLOAT_ZERO 0x10   /* fractional zero point */
#define FLAG_META_BF16 0x20    /* s and z stored as bf16 */

/* Threads an OpenMP region of this library uses (for reporting). */
int oracle_num_threads(void) { return omp_get_max_threads(); }

/* ---------------------------------------------------------------- formats */

static float bf16_bits_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint16_t f16_to_bits(_Float16 h)
{
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

static _Float16 bits_to_f16(uint16_t b)
{
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return h;
}

/* Round a double to the nearest bf16 (ties to even), straight from fp64 so
 * that no intermediate fp32 rounding can intervene. */
uint16_t oracle_f64_to_bf16(double d)
{
    if (isnan(d)) return 0x7FC0;
    double a = fabs(d);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (a < 0x1p-126) {
        /* bf16 subnormals are multiples of 2^-133 */
        r = nearbyint(a * 0x1p133) * 0x1p-133;
    } else {
        int e;
        double m = frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1) */
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);   /* 8 significant bits */
    }
    float f;
    if (r >= 0x1p128) {
        f = INFINITY;
    } else {
        f = (float)r;                      /* exact: r has <= 8 bits */
    }
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    if (signbit(d)) b |= 0x8000;
    return b;
}

/* -------------------------------------------------------------- quantize */

/* The metadata type's value of a bit pattern, and the nearest pattern to an
 * fp32 value (ties to even; bf16 from the exact double of the value). */
static float meta_value(uint16_t b, int flags)
{
    return (flags & FLAG_META_BF16) ? bf16_bits_to_f32(b) : (float)bits_to_f16(b);
}

static uint16_t meta_rn(float v, int flags)
{
    return (flags & FLAG_META_BF16) ? oracle_f64_to_bf16((double)v) : f16_to_bits((_Float16)v);
}

/* One group of n weights (fp32 values of bf16 inputs) at stride 1.
 * Writes n codes and the bit patterns of s and z (fp16, or bf16 with
 * FLAG_META_BF16). */
static void quantize_group(const float *w, long n, uint8_t *q, uint16_t *s_bits,
                           uint16_t *z_bits, int flags)
{
    float mn = w[0], mx = w[0];
    for (long i = 1; i < n; ++i) {
        mn = fminf(mn, w[i]);
        mx = fmaxf(mx, w[i]);
    }
    float range = mx - mn;
    float s32 = range / 15.0f;
    uint16_t sb = meta_rn(s32, flags);
    if (meta_value(sb, flags) == 0.0f) sb = meta_rn(fmaxf(fabsf(mn), 0x1p-14f), flags);
    float sf = meta_value(sb, flags);
    if (flags & FLAG_FLOAT_ZERO) {
        /* z = -min / s, kept fractional; only kept finite in its type */
        const float zmax = (flags & FLAG_META_BF16) ? 0x1.FEp127f : 65504.0f;
        float z32 = fminf(fmaxf(-mn / sf, -zmax), zmax);
        uint16_t zb = meta_rn(z32, flags);
        float zf = meta_value(zb, flags);
        for (long i = 0; i < n; ++i) {
            float u = w[i] / sf + zf;
            float t = fminf(fmaxf(rintf(u), 0.0f), 15.0f);
            q[i] = (uint8_t)(int)t;
        }
        *s_bits = sb;
        *z_bits = zb;
        return;
    }
    float zf = fminf(fmaxf(rintf(-mn / sf), 0.0f), 15.0f);
    int zi = (int)zf;
    for (long i = 0; i < n; ++i) {
        float t = rintf(w[i] / sf) + (float)zi;
        t = fminf(fmaxf(t, 0.0f), 15.0f);
        q[i] = (uint8_t)(int)t;
    }
    *s_bits = sb;
    *z_bits = meta_rn((float)zi, flags);
}

/* Number of groups per row (G) for a mode; 0 on invalid arguments. */
long oracle_groups_per_row(long K, int mode, long g)
{
    mode &= MODE_BASE_MASK;
    if (K <= 0) return 0;
    if (mode == MODE_GLOBAL || mode == MODE_ROWWISE) return 1;
    if (mode != MODE_GROUPWISE || g <= 0 || K % g != 0) return 0;
    return K / g;
}

/* W: bf16 bits [N,K].  q: uint8 [N,K].  s, z: fp16 bits [N,G] (GROUPWISE),
 * [N,1] (ROWWISE) or [1,1] (GLOBAL).  Returns 0 on success, -1 on bad
 * arguments. */
int oracle_quantize(const uint16_t *W, long N, long K, int mode, long g, uint8_t *q,
                    uint16_t *s, uint16_t *z)
{
    const int flags = mode & ~MODE_BASE_MASK;
    mode &= MODE_BASE_MASK;
    if (flags & ~(FLAG_FLOAT_ZERO | FLAG_META_BF16)) return -1;
    long G = oracle_groups_per_row(K, mode, g);
    if (N <= 0 || G == 0) return -1;
    if (mode == MODE_GLOBAL) {
        /* one group over all N*K elements */
        long total = N * K;
        float mn = bf16_bits_to_f32(W[0]), mx = mn;
        for (long i = 1; i < total; ++i) {
            float v = bf16_bits_to_f32(W[i]);
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        }
        /* Reuse the per-group code on a two-element summary to get s, z,
         * then quantize every element with them. */
        float ends[2] = {mn, mx};
        uint8_t dummy[2];
        quantize_group(ends, 2, dummy, &s[0], &z[0], flags);
        float sf = meta_value(s[0], flags);
        float zf = meta_value(z[0], flags);
        const int fz = (flags & FLAG_FLOAT_ZERO) != 0;
#pragma omp parallel for schedule(static)
        for (long i = 0; i < total; ++i) {
            float w = bf16_bits_to_f32(W[i]);
            float t = fz ? rintf(w / sf + zf) : rintf(w / sf) + zf;
            t = fminf(fmaxf(t, 0.0f), 15.0f);
            q[i] = (uint8_t)(int)t;
        }
        return 0;
    }
    long gl = K / G;
#pragma omp parallel
    {
        float buf_small[256];
        float *buf = buf_small;
        float *heap = 0;
        if (gl > 256) {
            heap = (float *)__builtin_malloc(sizeof(float) * (size_t)gl);
            buf = heap;
        }
#pragma omp for schedule(static)
        for (long n = 0; n < N; ++n) {
            for (long gi = 0; gi < G; ++gi) {
                const uint16_t *src = W + n * K + gi * gl;
                for (long i = 0; i < gl; ++i) buf[i] = bf16_bits_to_f32(src[i]);
                quantize_group(buf, gl, q + n * K + gi * gl, &s[n * G + gi], &z[n * G + gi], flags);
            }
        }
        if (heap) __builtin_free(heap);
    }
    return 0;
}

/* ------------------------------------------------------------ pack/unpack */

void oracle_pack(const uint8_t *q, long N, long K, uint32_t *packed)
{
    long W8 = K / 8;
#pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n)
        for (long j = 0; j < W8; ++j) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) word |= (uint32_t)(q[n * K + 8 * j + i] & 0xF) << (4 * i);
            packed[n * W8 + j] = word;
        }
}

void oracle_unpack(const uint32_t *packed, long N, long K, uint8_t *q)
{
    long W8 = K / 8;
#pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n)
        for (long k = 0; k < K; ++k) q[n * K + k] = (uint8_t)((packed[n * W8 + k / 8] >> (4 * (k % 8))) & 0xF);
}

/* ---------------------------------------------------------------- dequant */

/* s and z of element (n, k) for the given mode. */
static void group_params(const uint16_t *s, const uint16_t *z, long n, long k, long K, int mode,
                         long g, double *sd, double *zd)
{
    const int flags = mode & ~MODE_BASE_MASK;
    long idx;
    mode &= MODE_BASE_MASK;
    if (mode == MODE_GLOBAL) idx = 0;
    else if (mode == MODE_ROWWISE) idx = n;
    else idx = n * (K / g) + k / g;
    *sd = (double)meta_value(s[idx], flags);
    *zd = (double)meta_value(z[idx], flags);
}

/* One dequantized row: out[k] = (q[n,k] - z) * s, for k in [0, K). */
static void dequant_row(const uint32_t *packed, const uint16_t *s, const uint16_t *z, long n,
                        long K, int mode, long g, double *out)
{
    long W8 = K / 8;
    for (long k = 0; k < K; ++k) {
        double sd, zd;
        group_params(s, z, n, k, K, mode, g, &sd, &zd);
        double qd = (double)((packed[n * W8 + k / 8] >> (4 * (k % 8))) & 0xF);
        out[k] = (qd - zd) * sd;
    }
}

/* Dequantize rows [0, N) into fp64 out [N,K]. */
void oracle_dequant(const uint32_t *packed, const uint16_t *s, const uint16_t *z, long N, long K,
                    int mode, long g, double *out)
{
#pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) dequant_row(packed, s, z, n, K, mode, g, out + n * K);
}

/* ----------------------------------------------------------------- matmul */

/* Forward: Y[m, n] = sum_k X[m,k] * w_hat[n,k] + bias[n], for the output
 * columns n = cols[0..ncols) (all N columns when cols is NULL, ncols = N).
 * X bf16 bits [M,K]; bias bf16 bits [N] or NULL.  Writes y64 [M,ncols]
 * (unrounded fp64) and ybf [M,ncols] (bf16 bits), either may be NULL. */
void oracle_linear(const uint16_t *X, long M, long K, const uint32_t *packed, const uint16_t *s,
                   const uint16_t *z, long N, int mode, long g, const uint16_t *bias,
                   const long *cols, long ncols, double *y64, uint16_t *ybf)
{
    (void)N;
#pragma omp parallel
    {
        double *wrow = (double *)__builtin_malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 4)
        for (long j = 0; j < ncols; ++j) {
            long n = cols ? cols[j] : j;
            dequant_row(packed, s, z, n, K, mode, g, wrow);
            double b = bias ? (double)bf16_bits_to_f32(bias[n]) : 0.0;
            for (long m = 0; m < M; ++m) {
                double acc = 0.0;
                const uint16_t *xr = X + m * K;
                for (long k = 0; k < K; ++k) acc += (double)bf16_bits_to_f32(xr[k]) * wrow[k];
                acc += b;
                if (y64) y64[m * ncols + j] = acc;
                if (ybf) ybf[m * ncols + j] = oracle_f64_to_bf16(acc);
            }
        }
        __builtin_free(wrow);
    }
}

/* Transposed: dX[m, k] = sum_n dY[m,n] * w_hat[n,k] + bias[k], for the
 * output columns k = cols[0..ncols) (all K when cols is NULL).  dY bf16
 * bits [M,N]; bias bf16 bits [K] or NULL.  Outputs [M,ncols]. */
void oracle_linear_t(const uint16_t *dY, long M, long N, const uint32_t *packed,
                     const uint16_t *s, const uint16_t *z, long K, int mode, long g,
                     const uint16_t *bias, const long *cols, long ncols, double *y64,
                     uint16_t *ybf)
{
    long W8 = K / 8;
#pragma omp parallel
    {
        double *wcol = (double *)__builtin_malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 4)
        for (long j = 0; j < ncols; ++j) {
            long k = cols ? cols[j] : j;
            /* column k of w_hat, all N rows */
            for (long n = 0; n < N; ++n) {
                double sd, zd;
                group_params(s, z, n, k, K, mode, g, &sd, &zd);
                double qd = (double)((packed[n * W8 + k / 8] >> (4 * (k % 8))) & 0xF);
                wcol[n] = (qd - zd) * sd;
            }
            double b = bias ? (double)bf16_bits_to_f32(bias[k]) : 0.0;
            for (long m = 0; m < M; ++m) {
                double acc = 0.0;
                const uint16_t *dyr = dY + m * N;
                for (long n = 0; n < N; ++n) acc += (double)bf16_bits_to_f32(dyr[n]) * wcol[n];
                double v = acc + b;
                if (y64) y64[m * ncols + j] = v;
                if (ybf) ybf[m * ncols + j] = oracle_f64_to_bf16(v);
            }
        }
        __builtin_free(wcol);
    }
}
