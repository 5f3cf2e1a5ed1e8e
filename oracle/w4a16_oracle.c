/*
 * w4a16_oracle.c -- plain, slow CPU oracle for the W4A16 pack + matmul path.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load this code.  It shares nothing with the CUDA library: its
 * own format tables, its own encoders, its own loops.  No blocking, fusion or
 * reordering beyond what the format definitions state; OpenMP only splits the
 * independent output rows across threads (every row is computed the same way
 * whatever the thread count).
 *
 * Floating-point rule: every step that decides a stored code (global scale,
 * block scale, element quotient, ROCmFP4 error sums) runs in IEEE binary32 with
 * round-to-nearest-even and no contraction (built with -ffp-contract=off, no
 * fast-math), because the CUDA packer takes the same decisions in binary32.
 * Dequantised weights and all matmul sums are binary64.
 *
 * Sources (web pages on the subject):
 *  - "EdgeRock-4B-NVFP4" model card, intro: NVFP4 W4A16 = E2M1 4-bit weights,
 *    one FP8 E4M3 scale per 16 values, one FP32 global scale per matrix.
 *  - "Nanbeige4.2-3B-NVFP4A16" card, Creation: data-free round-to-nearest,
 *    group 16.
 *  - "rocmwhy" ROCmFP4 page, sections 01-03 and the format table: Codebook10
 *    levels 0,+-1,+-2,+-3,+-4,+-6,+-8,+-10; two unsigned E4M3 scales, one per
 *    16-weight half (Dual, 18-byte blocks) or one per 32 (FAST, 17 bytes);
 *    scale chosen by exhaustive search over the finite UE4M3 candidates,
 *    scored by reconstruction MSE.
 *  - The global-scale formula absmax/(6*448) and block scale absmax/6/global
 *    are the library's stated NVFP4 recipe.
 *
 * Readings where the pages are silent (each is pinned by a test):
 *  - E2M1 is the OCP MX FP4 code: bit 3 sign, bits 2..1 exponent (bias 1),
 *    bit 0 mantissa; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6.
 *  - E4M3 is E4M3FN: bias 7, subnormals m*2^-9, 0x7F/0xFF NaN, max 448.
 *  - Conversions round to nearest, ties to the even code, and saturate to the
 *    largest finite magnitude.  NVFP4 codes keep the sign of the quotient
 *    (-0 and negatives that round to zero encode as 0x8).  A block whose
 *    decoded scale times the global scale is 0 encodes all-zero codes.
 *  - NVFP4 layout: codes[n][k/2], element 2i in the low nibble of byte i;
 *    scales[n][k/16]; one float global scale.
 *  - Codebook10 nibble: bit 3 sign, bits 2..0 index into {0,1,2,3,4,6,8,10};
 *    level 0 always encodes as 0x0.
 *  - ROCmFP4 block: Dual = [scale(0..15), scale(16..31), 16 code bytes],
 *    FAST = [scale, 16 code bytes]; code byte j = code[j] | code[j+16] << 4.
 *  - UE4M3 candidates are the bytes 0x00..0x7E (zero included), weights are
 *    level * scale (no tensor scale).  Error E(u) = sum_i fma(d_i, d_i, E) in
 *    element order with d_i = x_i - s*l_i; argmin, ties to the smallest code.
 *  - Importance weighting (the "rocmwhy" page, section 03: candidates scored by
 *    reconstruction error "with optional importance weighting"; its example
 *    gives an outlier low importance): one nonnegative weight per input channel
 *    k, E(u) = sum_i fma(w_k * d_i, d_i, E); with no weights w = 1, which gives
 *    exactly the unweighted sum.
 *  - NVFP4 scale by search (the same recipe applied to NVFP4 blocks, global
 *    scale g fixed by the abs-max rule): candidates are the E4M3 bytes
 *    0x00..0x7E; under candidate u, d = E4M3(u) * g, each code is the E2M1
 *    encoding of x / d exactly as in the abs-max packer, r = e2m1 * d (binary32),
 *    E(u) = sum_i fma(w_k * (x_i - r_i), x_i - r_i, E); argmin, ties to the
 *    smallest code.  The abs-max scale is one of the candidates.
 *  - Stock Q4_0, the pages' comparison format ("rocmwhy" format table and
 *    section 02: 32 weights, evenly spaced integer steps, one FP16 scale,
 *    18-byte blocks, "signed abs-max" reference scale; the lab's outlier 8.2
 *    gives the shared scale 1.025 = 8.2 / 8): m = the weight of largest
 *    magnitude (the first in k order on ties), d = FP16(m / -8) (binary32
 *    division, then round to nearest even with saturation at 65504), each code
 *    q = the nearest integer (ties to even) of x / d in binary32, clamped to
 *    [-8, 7], stored as q + 8; d == 0 gives codes 8.  Block = [d (FP16, little
 *    endian), 16 code bytes], code byte j = code[j] | code[j+16] << 4.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NONFINITE 5

/* ------------------------------------------------------------------------ */
/* Scalar formats                                                           */
/* ------------------------------------------------------------------------ */

static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* E2M1 value of a 4-bit code (OCP MX FP4). */
double orc_e2m1_decode(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3FN value of a byte: (1 + m/8) * 2^(e-7), subnormal m/8 * 2^-6. */
double orc_e4m3_decode(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7)
        return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    return s ? -mag : mag;
}

static const int CB10[8] = {0, 1, 2, 3, 4, 6, 8, 10};

/* Codebook10 value of a 4-bit code (sign bit 3, index bits 2..0). */
double orc_cb10_decode(int code)
{
    double mag = CB10[code & 7];
    return (code & 8) ? -mag : mag;
}

/*
 * Round a non-negative value onto a sorted grid q[0] < q[1] < ... < q[n-1]
 * whose consecutive entries have consecutive codes: nearest entry, ties to the
 * even index, saturating at q[n-1].  All comparisons are exact in binary64.
 */
static int round_to_grid(double a, const double *q, int n)
{
    if (a >= q[n - 1])
        return n - 1;
    int i = 0;
    while (q[i + 1] <= a)
        i++;
    if (a == q[i])
        return i;
    double mid = 0.5 * (q[i] + q[i + 1]);
    if (a < mid)
        return i;
    if (a > mid)
        return i + 1;
    return (i % 2 == 0) ? i : i + 1;
}

/* binary32 -> E2M1 code, round to nearest even, saturating, sign kept. */
int orc_e2m1_encode(float v)
{
    double q[8];
    for (int i = 0; i < 8; i++)
        q[i] = orc_e2m1_decode(i);
    int idx = round_to_grid(fabs((double)v), q, 8);
    return (signbit(v) ? 8 : 0) | idx;
}

/* binary32 -> E4M3FN byte, round to nearest even, saturating; NaN -> 0x7F. */
int orc_e4m3_encode(float v)
{
    if (isnan(v))
        return 0x7F;
    double q[127];
    for (int i = 0; i < 127; i++)
        q[i] = orc_e4m3_decode(i);
    int idx = round_to_grid(fabs((double)v), q, 127);
    return (signbit(v) ? 0x80 : 0) | idx;
}

/* Nearest Codebook10 index for magnitude a under scale s > 0 (ties even). */
int orc_cb10_index(float a, float s)
{
    double q[8];
    for (int i = 0; i < 8; i++)
        q[i] = (double)s * CB10[i];
    return round_to_grid((double)a, q, 8);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 pack / dequant                                                     */
/* ------------------------------------------------------------------------ */

/* Reconstruction error of 16 weights x under E4M3 scale code u and global
 * scale g, in binary32 (see the header); imp: 16 weights or NULL. */
float orc_nvfp4_error(const float *x, const float *imp, int u, float g)
{
    const float d = (float)orc_e4m3_decode(u) * g;
    float E = 0.0f;
    for (int i = 0; i < 16; i++) {
        int c = 0;
        if (d != 0.0f)
            c = orc_e2m1_encode(x[i] / d);
        const float r = (float)orc_e2m1_decode(c) * d;
        const float e = x[i] - r;
        const float t = imp ? imp[i] * e : e;
        E = fmaf(t, e, E);
    }
    return E;
}

/* Search over the 127 finite E4M3 codes; ties -> smallest code. */
int orc_nvfp4_search(const float *x, const float *imp, float g, float *best_err)
{
    int best_u = 0;
    float best = orc_nvfp4_error(x, imp, 0, g);
    for (int u = 1; u < 127; u++) {
        const float E = orc_nvfp4_error(x, imp, u, g);
        if (E < best) {
            best = E;
            best_u = u;
        }
    }
    if (best_err)
        *best_err = best;
    return best_u;
}

/* imp: NULL, or K weights that must be finite and >= 0. */
static int check_importance(const float *imp, int K)
{
    if (!imp)
        return ORC_OK;
    for (int k = 0; k < K; k++)
        if (!isfinite(imp[k]) || imp[k] < 0.0f)
            return ORC_ERR_NONFINITE;
    return ORC_OK;
}

/*
 * W: bf16 bit patterns, [N][K] (K contiguous).  K % 16 == 0.
 * codes: [N][K/2]; scales: [N][K/16]; *g_out: global scale.
 * mse = 0: block scale E4M3(absmax / 6 / g) (imp must be NULL);
 * mse = 1: block scale by the error search, imp = NULL or K channel weights.
 */
int orc_pack_nvfp4_ex(const uint16_t *W, int K, int N, int mse, const float *imp, uint8_t *codes,
                      uint8_t *scales, float *g_out)
{
    if (K <= 0 || N <= 0 || K % 16 != 0 || (mse != 0 && mse != 1) || (!mse && imp))
        return ORC_ERR_ARG;
    if (check_importance(imp, K) != ORC_OK)
        return ORC_ERR_NONFINITE;
    long long total = (long long)K * N;

    /* 1. tensor abs-max */
    float amax = 0.0f;
    int bad = 0;
    for (long long i = 0; i < total; i++) {
        float a = fabsf(bf16_to_float(W[i]));
        if (!isfinite(a))
            bad = 1;
        else if (a > amax)
            amax = a;
    }
    if (bad)
        return ORC_ERR_NONFINITE;

    /* 2. global scale = absmax / (6 * 448) */
    const float g = amax / 2688.0f;
    *g_out = g;

    /* 3. per 16-block: the scale, then code = E2M1(x / (scale * global)) */
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
        const uint16_t *row = W + (long long)n * K;
        for (int b = 0; b < K / 16; b++) {
            float x[16];
            float bamax = 0.0f;
            for (int j = 0; j < 16; j++) {
                x[j] = bf16_to_float(row[16 * b + j]);
                if (fabsf(x[j]) > bamax)
                    bamax = fabsf(x[j]);
            }
            int s = 0;
            if (mse) {
                s = orc_nvfp4_search(x, imp ? imp + 16 * b : NULL, g, NULL);
            } else if (g != 0.0f) {
                float sf = (bamax / 6.0f) / g;
                s = orc_e4m3_encode(sf);
            }
            scales[(long long)n * (K / 16) + b] = (uint8_t)s;
            float ds = (float)orc_e4m3_decode(s);
            float d = ds * g;
            for (int j = 0; j < 16; j += 2) {
                int c0 = 0, c1 = 0;
                if (d != 0.0f) {
                    float q0 = x[j] / d;
                    float q1 = x[j + 1] / d;
                    c0 = orc_e2m1_encode(q0);
                    c1 = orc_e2m1_encode(q1);
                }
                codes[(long long)n * (K / 2) + 8 * b + j / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    }
    return ORC_OK;
}

int orc_pack_nvfp4(const uint16_t *W, int K, int N, uint8_t *codes, uint8_t *scales, float *g_out)
{
    return orc_pack_nvfp4_ex(W, K, N, 0, NULL, codes, scales, g_out);
}

/* w_hat[r][k] for rows n0..n0+rows-1: e2m1 * E4M3(scale) * global, in binary64. */
void orc_dequant_nvfp4(const uint8_t *codes, const uint8_t *scales, float g, int K,
                       int n0, int rows, double *w_hat)
{
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++) {
        long long n = n0 + r;
        for (int k = 0; k < K; k++) {
            uint8_t byte = codes[n * (K / 2) + k / 2];
            int c = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
            double s = orc_e4m3_decode(scales[n * (K / 16) + k / 16]);
            w_hat[(long long)r * K + k] = orc_e2m1_decode(c) * s * (double)g;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* ROCmFP4 pack / dequant                                                   */
/* ------------------------------------------------------------------------ */

/* Reconstruction error of x[0..n-1] under UE4M3 code u, in binary32; imp:
 * n channel weights or NULL. */
float orc_rocm_error_w(const float *x, const float *imp, int n, int u)
{
    float s = (float)orc_e4m3_decode(u);
    float E = 0.0f;
    for (int i = 0; i < n; i++) {
        int idx = (s == 0.0f) ? 0 : orc_cb10_index(fabsf(x[i]), s);
        float r = s * (float)CB10[idx];          /* exact: <= 8 significant bits */
        float w = signbit(x[i]) ? -r : r;
        float d = x[i] - w;
        float t = imp ? imp[i] * d : d;
        E = fmaf(t, d, E);
    }
    return E;
}

float orc_rocm_error(const float *x, int n, int u)
{
    return orc_rocm_error_w(x, NULL, n, u);
}

/* Exhaustive scale search over the 127 finite UE4M3 codes; ties -> smallest code. */
int orc_rocm_search_w(const float *x, const float *imp, int n, float *best_err)
{
    int best_u = 0;
    float best = orc_rocm_error_w(x, imp, n, 0);
    for (int u = 1; u < 127; u++) {
        float E = orc_rocm_error_w(x, imp, n, u);
        if (E < best) {
            best = E;
            best_u = u;
        }
    }
    if (best_err)
        *best_err = best;
    return best_u;
}

int orc_rocm_search(const float *x, int n, float *best_err)
{
    return orc_rocm_search_w(x, NULL, n, best_err);
}

/* Codebook10 code of x under scale code u. */
static int rocm_code(float x, int u)
{
    float s = (float)orc_e4m3_decode(u);
    if (s == 0.0f)
        return 0;
    int idx = orc_cb10_index(fabsf(x), s);
    if (idx == 0)
        return 0;
    return (signbit(x) ? 8 : 0) | idx;
}

/*
 * fmt 2 = Dual (18-byte blocks), 3 = FAST (17-byte blocks).  W: bf16 [N][K],
 * K % 32 == 0.  imp: NULL or K channel weights (finite, >= 0).
 * blocks: [N][K/32][18|17].
 */
int orc_pack_rocmfp4_w(const uint16_t *W, int K, int N, int fmt, const float *imp, uint8_t *blocks)
{
    if (K <= 0 || N <= 0 || K % 32 != 0 || (fmt != 2 && fmt != 3))
        return ORC_ERR_ARG;
    if (check_importance(imp, K) != ORC_OK)
        return ORC_ERR_NONFINITE;
    long long total = (long long)K * N;
    for (long long i = 0; i < total; i++)
        if (!isfinite(bf16_to_float(W[i])))
            return ORC_ERR_NONFINITE;
    const int bb = (fmt == 2) ? 18 : 17;
    const int nb = K / 32;

    #pragma omp parallel for schedule(dynamic, 4)
    for (int n = 0; n < N; n++) {
        for (int b = 0; b < nb; b++) {
            float x[32];
            for (int j = 0; j < 32; j++)
                x[j] = bf16_to_float(W[(long long)n * K + 32 * b + j]);
            uint8_t *out = blocks + ((long long)n * nb + b) * bb;
            int code[32];
            const float *wb = imp ? imp + 32 * b : NULL;
            if (fmt == 2) {
                int u0 = orc_rocm_search_w(x, wb, 16, NULL);
                int u1 = orc_rocm_search_w(x + 16, wb ? wb + 16 : NULL, 16, NULL);
                out[0] = (uint8_t)u0;
                out[1] = (uint8_t)u1;
                for (int j = 0; j < 16; j++) {
                    code[j] = rocm_code(x[j], u0);
                    code[j + 16] = rocm_code(x[j + 16], u1);
                }
            } else {
                int u = orc_rocm_search_w(x, wb, 32, NULL);
                out[0] = (uint8_t)u;
                for (int j = 0; j < 32; j++)
                    code[j] = rocm_code(x[j], u);
            }
            uint8_t *cb = out + (fmt == 2 ? 2 : 1);
            for (int j = 0; j < 16; j++)
                cb[j] = (uint8_t)(code[j] | (code[j + 16] << 4));
        }
    }
    return ORC_OK;
}

int orc_pack_rocmfp4(const uint16_t *W, int K, int N, int fmt, uint8_t *blocks)
{
    return orc_pack_rocmfp4_w(W, K, N, fmt, NULL, blocks);
}

void orc_dequant_rocmfp4(const uint8_t *blocks, int fmt, int K, int n0, int rows, double *w_hat)
{
    const int bb = (fmt == 2) ? 18 : 17;
    const int nb = K / 32;
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++) {
        long long n = n0 + r;
        for (int b = 0; b < nb; b++) {
            const uint8_t *blk = blocks + (n * nb + b) * bb;
            const uint8_t *cb = blk + (fmt == 2 ? 2 : 1);
            for (int j = 0; j < 32; j++) {
                int u = (fmt == 2) ? blk[j < 16 ? 0 : 1] : blk[0];
                int c = (j < 16) ? (cb[j] & 15) : (cb[j - 16] >> 4);
                w_hat[(long long)r * K + 32 * b + j] = orc_cb10_decode(c) * orc_e4m3_decode(u);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Stock Q4_0 (comparison format) and reconstruction error                  */
/* ------------------------------------------------------------------------ */

/* binary16 value of bits h, exactly. */
double orc_fp16_decode(int h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -v : v;
}

/* Nearest binary16 (ties to even), saturating at +-65504; by exact search over
 * the finite non-negative codes (the magnitudes are increasing in the code). */
int orc_fp16_encode(float v)
{
    double a = fabs((double)v);
    int sign = signbit(v) ? 0x8000 : 0;
    if (a >= 65504.0)
        return sign | 0x7BFF;
    int lo = 0, hi = 0x7BFF;            /* largest code with value <= a */
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (orc_fp16_decode(mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    int c = lo;
    if (orc_fp16_decode(c) != a && c < 0x7BFF) {
        double d0 = a - orc_fp16_decode(c), d1 = orc_fp16_decode(c + 1) - a;
        if (d1 < d0 || (d1 == d0 && (c & 1)))
            c = c + 1;
    }
    return sign | c;
}

/* W: bf16 [N][K], K % 32 == 0.  blocks: [N][K/32][18]. */
int orc_pack_q4_0(const uint16_t *W, int K, int N, uint8_t *blocks)
{
    if (K <= 0 || N <= 0 || K % 32 != 0)
        return ORC_ERR_ARG;
    long long total = (long long)K * N;
    for (long long i = 0; i < total; i++)
        if (!isfinite(bf16_to_float(W[i])))
            return ORC_ERR_NONFINITE;
    const int nb = K / 32;
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
        for (int b = 0; b < nb; b++) {
            float x[32];
            int jm = 0;
            for (int j = 0; j < 32; j++) {
                x[j] = bf16_to_float(W[(long long)n * K + 32 * b + j]);
                if (fabsf(x[j]) > fabsf(x[jm]))
                    jm = j;
            }
            const int h = orc_fp16_encode(x[jm] / -8.0f);
            const float d = (float)orc_fp16_decode(h);
            uint8_t *out = blocks + ((long long)n * nb + b) * 18;
            out[0] = (uint8_t)(h & 0xFF);
            out[1] = (uint8_t)(h >> 8);
            int code[32];
            for (int j = 0; j < 32; j++) {
                int q = 0;
                if (d != 0.0f) {
                    float r = nearbyintf(x[j] / d);   /* round to nearest even */
                    q = r < -8.0f ? -8 : (r > 7.0f ? 7 : (int)r);
                }
                code[j] = q + 8;
            }
            for (int j = 0; j < 16; j++)
                out[2 + j] = (uint8_t)(code[j] | (code[j + 16] << 4));
        }
    }
    return ORC_OK;
}

void orc_dequant_q4_0(const uint8_t *blocks, int K, int n0, int rows, double *w_hat)
{
    const int nb = K / 32;
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++) {
        for (int b = 0; b < nb; b++) {
            const uint8_t *blk = blocks + ((long long)(n0 + r) * nb + b) * 18;
            const double d = orc_fp16_decode(blk[0] | (blk[1] << 8));
            for (int j = 0; j < 32; j++) {
                int c = (j < 16) ? (blk[2 + j] & 15) : (blk[2 + j - 16] >> 4);
                w_hat[(long long)r * K + 32 * b + j] = d * (double)(c - 8);
            }
        }
    }
}

/* out[0] = sum (W - w_hat)^2, out[1] = sum W^2 over rows x K, in binary64. */
void orc_reconstruction_sse(const uint16_t *W, const double *w_hat, long long count, double *out)
{
    double e = 0.0, q = 0.0;
    for (long long i = 0; i < count; i++) {
        const double w = (double)bf16_to_float(W[i]);
        const double d = w - w_hat[i];
        e += d * d;
        q += w * w;
    }
    out[0] = e;
    out[1] = q;
}

/* ------------------------------------------------------------------------ */
/* Matmul                                                                   */
/* ------------------------------------------------------------------------ */

/*
 * y[m][r] = sum_k x[m][k] * w_hat[r][k] and a[m][r] = sum_k |x[m][k] * w_hat[r][k]|,
 * binary64, k ascending.  x: bf16 [M][K]; w_hat: [R][K]; y, a: [M][R].
 */
void orc_matmul(const uint16_t *x, int M, int K, const double *w_hat, int R, double *y, double *a)
{
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < R; r++) {
        for (int m = 0; m < M; m++) {
            double acc = 0.0, mag = 0.0;
            for (int k = 0; k < K; k++) {
                double p = (double)bf16_to_float(x[(long long)m * K + k]) * w_hat[(long long)r * K + k];
                acc += p;
                mag += fabs(p);
            }
            y[(long long)m * R + r] = acc;
            a[(long long)m * R + r] = mag;
        }
    }
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Elementwise encoders over arrays (for checking other implementations). */
void orc_e4m3_encode_array(const float *v, long long n, uint8_t *out)
{
    #pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; i++)
        out[i] = (uint8_t)orc_e4m3_encode(v[i]);
}

void orc_e2m1_encode_array(const float *v, long long n, uint8_t *out)
{
    #pragma omp parallel for schedule(static)
    for (long long i = 0; i < n; i++)
        out[i] = (uint8_t)orc_e2m1_encode(v[i]);
}
