/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for NVFP4 quantization and the
 * W4A4 block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may link, load or call this file; only the tests,
 * the smoke check and the benchmark's CPU-baseline leg do.  It shares no code,
 * header, table or constant with the CUDA path.
 *
 * Sources of the definitions (web pages about NVFP4):
 *   [WIKI]  NVFP4 wiki page (newton.com.tw), section "技術原理":
 *           E2M1 element = 1 sign, 2 exponent, 1 mantissa bit, range about
 *           -6..6; the tensor is cut into 16-value microblocks, each with one
 *           E4M3 FP8 scale (non-power-of-two, fractional scales allowed), and
 *           a second-level FP32 scale covers the whole tensor; about 4.5 bits
 *           per value.
 *   [EDGE]  eefocus.com article on FP4 vs INT4 for edge LLMs, section
 *           "为什么FP4是更合适的压缩方案？": E2M1 is a non-linear grid, dense
 *           near zero and sparse far from it.
 *   [W4A4]  aixq.cc article on Unsloth Dynamic NVFP4, section
 *           "核心差异：W4A4 vs W4A16": weights and activations are both 4-bit
 *           and the FP4 tensor cores consume them directly, with no
 *           dequantize-to-16-bit step.
 *   [MX]    eefocus.com article, section "FP4被视为下一代AI计算的核心标准":
 *           the OCP MXFP4 format, 32 E2M1 elements sharing one 8-bit (usually
 *           E8M0) scale, about 4.25 bits per value (the MXFP4 section below,
 *           readings M1-M4).
 *
 * The pages fix the structure but not the scale arithmetic.  The readings
 * taken here (each is also a rule the CUDA path follows):
 *   R1  tensor scale  g = fl32(amax / 2688), 2688 = 6 * 448 (E2M1 max times
 *       E4M3 max), so the largest block lands on the largest E4M3 scale.
 *   R2  block scale   t = fl32(bamax / fl32(6 * g)); s = E4M3 RNE satfinite(t)
 *       (the OCP "fn" E4M3: bias 7, subnormals, max 448, no infinity).
 *       g == 0 gives t = 0.
 *   R3  element       d = fl32(dec(s) * g); r = fl32(1 / d);
 *       v = fl32(x * r); code = E2M1 RNE satfinite(v), ties to the even
 *       magnitude index, sign in bit 3 (a negative value that rounds to zero
 *       keeps its sign: 0x8).
 *   R4  zero-scale block: when d == 0 or 1/d overflows to infinity, every
 *       code of the block is 0x0.  (All its values dequantize to zero.)
 *   R5  packing: byte j of a row holds element 2j in the low nibble and
 *       element 2j+1 in the high nibble.
 *   R6  dequantize: y = fl32(fl32(e * dec(s)) * g); the inner product is exact.
 *   R7  GEMM: Y[m][n] = sum_k deqA[m][k] * deqB[n][k] in fp64, with
 *       deq = e * dec(s) * g formed in fp64 (exact).
 *
 * Every fp32 operation is one IEEE-754 binary32 operation, round to nearest
 * even; build with -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* E2M1 element ([WIKI], [EDGE]).                                            */
/* ------------------------------------------------------------------------ */

/* Magnitudes of the eight non-negative E2M1 codes, derived from the bit
 * layout: exponent field e (2 bits, bias 1), mantissa bit m.
 *   e == 0 : subnormal, value = m * 0.5
 *   e >  0 : value = 2^(e-1) * (1 + m/2)
 * giving 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1_value(unsigned code)
{
    unsigned sign = (code >> 3) & 1u;
    unsigned e = (code >> 1) & 3u;
    unsigned m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m
                          : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return sign ? -mag : mag;
}

/* Round v onto the E2M1 grid: nearest magnitude, ties to the even magnitude
 * index (index = code & 7), |v| beyond 6 saturates to 6.  The sign of v,
 * including the sign of a zero, goes to bit 3.  Brute force over the eight
 * magnitudes. */
unsigned oracle_e2m1_encode(float v)
{
    unsigned sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    unsigned best = 0;
    double best_err = INFINITY;
    for (unsigned i = 0; i < 8; ++i) {
        double err = fabs(a - oracle_e2m1_value(i));
        if (err < best_err || (err == best_err && (i & 1u) == 0u)) {
            best = i;
            best_err = err;
        }
    }
    return sign | best;
}

/* ------------------------------------------------------------------------ */
/* E4M3 block scale ([WIKI]).                                                */
/* ------------------------------------------------------------------------ */

/* OCP E4M3 "fn": sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 * field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity,
 * so the largest finite value is 1.75 * 2^8 = 448. */
double oracle_e4m3_value(unsigned byte)
{
    unsigned sign = (byte >> 7) & 1u;
    unsigned e = (byte >> 3) & 15u;
    unsigned m = byte & 7u;
    double mag;
    if (e == 15u && m == 7u)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return sign ? -mag : mag;
}

/* Round a non-negative t onto the E4M3 grid, nearest value, ties to the even
 * code, saturating at 448 (0x7E).  Brute force over the 127 non-negative
 * finite codes 0x00..0x7E, which are in increasing order of value. */
unsigned oracle_e4m3_encode(float t)
{
    double a = (double)t;
    unsigned best = 0;
    double best_err = INFINITY;
    if (!(a >= 0.0))
        return 0xFFu; /* negative or NaN: outside the domain of a scale */
    if (a >= 448.0)
        return 0x7Eu; /* satfinite */
    for (unsigned c = 0; c <= 0x7Eu; ++c) {
        double err = fabs(a - oracle_e4m3_value(c));
        if (err < best_err || (err == best_err && (c & 1u) == 0u)) {
            best = c;
            best_err = err;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
/* Quantizer (R1..R5).                                                       */
/* ------------------------------------------------------------------------ */

/* Tensor amax over the logical [rows][cols] window of a row-major matrix with
 * leading dimension ld (elements).  Max is exact. */
float oracle_amax(const float *x, int64_t rows, int64_t cols, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(x[r * ld + c]);
            if (a > amax)
                amax = a;
        }
    return amax;
}

/* R1 */
float oracle_tensor_scale(float amax)
{
    return amax / 2688.0f;
}

/* R2: scale byte of one 16-element block whose max |x| is bamax. */
unsigned oracle_block_scale(float bamax, float g)
{
    float t;
    if (g == 0.0f) {
        t = 0.0f;
    } else {
        float six_g = 6.0f * g;
        t = bamax / six_g;
    }
    return oracle_e4m3_encode(t);
}

/* R3/R4: the multiplier r applied to the elements of a block with scale byte
 * s; returns 0 and sets *zero_block when the block is a zero-scale block. */
float oracle_block_reciprocal(unsigned s, float g, int *zero_block)
{
    float d = (float)oracle_e4m3_value(s) * g;
    float r;
    *zero_block = 0;
    if (d == 0.0f) {
        *zero_block = 1;
        return 0.0f;
    }
    r = 1.0f / d;
    if (isinf(r)) {
        *zero_block = 1;
        return 0.0f;
    }
    return r;
}

/* Quantize the logical [rows][cols] window (cols % 16 == 0) of a row-major
 * fp32 matrix.  Outputs:
 *   codes  [rows][cols/2]   packed, element 2j in the low nibble of byte j
 *   scales [rows][cols/16]  row-major E4M3 bytes (the tests map them to the
 *                           tiled layout the tensor cores read)
 *   *g_out                  the fp32 tensor scale
 * Returns 0, or -1 on bad arguments or a non-finite input. */
int oracle_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld,
                    uint8_t *codes, uint8_t *scales, float *g_out)
{
    int64_t nblk = cols / 16;
    float amax, g;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            if (!isfinite(x[r * ld + c]))
                return -1;
    amax = oracle_amax(x, rows, cols, ld);
    g = oracle_tensor_scale(amax);
    *g_out = g;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const float *blk = x + r * ld + b * 16;
            float bamax = 0.0f;
            unsigned s;
            float rcp;
            int zero_block;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(blk[i]);
                if (a > bamax)
                    bamax = a;
            }
            s = oracle_block_scale(bamax, g);
            scales[r * nblk + b] = (uint8_t)s;
            rcp = oracle_block_reciprocal(s, g, &zero_block);
            for (int i = 0; i < 16; i += 2) {
                unsigned lo = 0, hi = 0;
                if (!zero_block) {
                    float v0 = blk[i] * rcp;
                    float v1 = blk[i + 1] * rcp;
                    lo = oracle_e2m1_encode(v0);
                    hi = oracle_e2m1_encode(v1);
                }
                codes[r * (cols / 2) + b * 8 + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return 0;
}

/* R6: fp32 dequantization of [rows][cols] into y (row-major, ld = cols). */
int oracle_dequantize(const uint8_t *codes, const uint8_t *scales, float g,
                      int64_t rows, int64_t cols, float *y)
{
    int64_t nblk = cols / 16;
    if (rows < 0 || cols < 0 || cols % 16 != 0)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            unsigned byte = codes[r * (cols / 2) + c / 2];
            unsigned code = (c & 1) ? (byte >> 4) : (byte & 15u);
            float e = (float)oracle_e2m1_value(code);
            float s = (float)oracle_e4m3_value(scales[r * nblk + c / 16]);
            float es = e * s;
            y[r * cols + c] = es * g;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* fp64 GEMM of dequantized operands (R7), Y = A * B^T with A [M][K] and     */
/* B [N][K] both quantized along K.                                          */
/* ------------------------------------------------------------------------ */

/* One dequantized element in fp64: e * dec(s) * g, exact. */
static double deq64(const uint8_t *codes, const uint8_t *scales, double g,
                    int64_t cols, int64_t r, int64_t c)
{
    unsigned byte = codes[r * (cols / 2) + c / 2];
    unsigned code = (c & 1) ? (byte >> 4) : (byte & 15u);
    return oracle_e2m1_value(code) * oracle_e4m3_value(scales[r * (cols / 16) + c / 16]) * g;
}

/* Fully dequantize an operand to fp64 [rows][cols]. */
int oracle_dequantize_f64(const uint8_t *codes, const uint8_t *scales, float g,
                          int64_t rows, int64_t cols, double *y)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            y[r * cols + c] = deq64(codes, scales, (double)g, cols, r, c);
    return 0;
}

struct gemm_job {
    const double *a, *b; /* dequantized [M][K], [N][K] */
    double *y;
    int64_t M, N, K;
    int64_t row0, row1;
};

static void *gemm_worker(void *p)
{
    struct gemm_job *j = (struct gemm_job *)p;
    for (int64_t m = j->row0; m < j->row1; ++m)
        for (int64_t n = 0; n < j->N; ++n) {
            const double *ar = j->a + m * j->K;
            const double *br = j->b + n * j->K;
            double acc = 0.0;
            for (int64_t k = 0; k < j->K; ++k)
                acc += ar[k] * br[k];
            j->y[m * j->N + n] = acc;
        }
    return NULL;
}

/* Y[m][n] = sum_k a[m][k] * b[n][k] over fp64 dequantized operands, rows of Y
 * split across nthreads plain threads (k summed in order). */
int oracle_gemm_f64(const double *a, const double *b, int64_t M, int64_t N,
                    int64_t K, double *y, int nthreads)
{
    pthread_t tid[256];
    struct gemm_job jobs[256];
    int nt = nthreads < 1 ? 1 : (nthreads > 256 ? 256 : nthreads);
    if (M < 0 || N < 0 || K < 0)
        return -1;
    if (nt > M)
        nt = M > 0 ? (int)M : 1;
    for (int t = 0; t < nt; ++t) {
        jobs[t].a = a;
        jobs[t].b = b;
        jobs[t].y = y;
        jobs[t].M = M;
        jobs[t].N = N;
        jobs[t].K = K;
        jobs[t].row0 = M * t / nt;
        jobs[t].row1 = M * (t + 1) / nt;
    }
    for (int t = 1; t < nt; ++t)
        pthread_create(&tid[t], NULL, gemm_worker, &jobs[t]);
    gemm_worker(&jobs[0]);
    for (int t = 1; t < nt; ++t)
        pthread_join(tid[t], NULL);
    return 0;
}

/* Selected entries of the same GEMM straight from the quantized operands:
 * out[i] = sum_k deqA[ms[i]][k] * deqB[ns[i]][k]; also the Euclidean norms of
 * the dequantized row of A and row of B (for the tolerance floor). */
int oracle_gemm_entries_f64(const uint8_t *a_codes, const uint8_t *a_scales, float ga,
                            const uint8_t *b_codes, const uint8_t *b_scales, float gb,
                            int64_t K, const int64_t *ms, const int64_t *ns,
                            int64_t count, double *out, double *a_norm, double *b_norm)
{
    if (K < 0 || K % 16 != 0)
        return -1;
    for (int64_t i = 0; i < count; ++i) {
        double acc = 0.0, na = 0.0, nb = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double av = deq64(a_codes, a_scales, (double)ga, K, ms[i], k);
            double bv = deq64(b_codes, b_scales, (double)gb, K, ns[i], k);
            acc += av * bv;
            na += av * av;
            nb += bv * bv;
        }
        out[i] = acc;
        if (a_norm)
            a_norm[i] = sqrt(na);
        if (b_norm)
            b_norm[i] = sqrt(nb);
    }
    return 0;
}

/* Fused-MLP middle step in fp64: h = SiLU(gate) * up, SiLU(z) = z / (1 + e^-z). */
void oracle_silu_mul_f64(const double *gate, const double *up, int64_t n, double *h)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = gate[i] / (1.0 + exp(-gate[i])) * up[i];
}

/* Storage of one quantized [rows][cols] tensor in bytes: packed codes, one
 * scale byte per 16 values, one fp32 tensor scale ([WIKI]: about 4.5 bits per
 * value). */
int64_t oracle_storage_bytes(int64_t rows, int64_t cols)
{
    return rows * cols / 2 + rows * cols / 16 + 4;
}

/* Element-wise array forms of the codecs, for tests that sweep many values. */
void oracle_e2m1_encode_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = (uint8_t)oracle_e2m1_encode(v[i]);
}

void oracle_e4m3_encode_array(const float *t, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = (uint8_t)oracle_e4m3_encode(t[i]);
}

void oracle_e4m3_value_array(const uint8_t *b, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_value(b[i]);
}

/* bf16 bit patterns widened to fp32 (exact: the 16 bits become the top half). */
void oracle_bf16_to_f32(const uint16_t *x, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits = (uint32_t)x[i] << 16;
        memcpy(&out[i], &bits, sizeof bits);
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4 ([MX]: eefocus.com article on FP4 vs INT4, section                  */
/* "FP4被视为下一代AI计算的核心标准": the OCP Microscaling format shares one */
/* 8-bit scale, usually E8M0, among 32 consecutive elements, each an E2M1    */
/* value; about 4.25 bits per value).  The page gives no rule for choosing   */
/* the scale.  Readings taken:                                               */
/*   M1  X = 2^e with e = ceil(log2(bamax / 6)): the smallest power of two   */
/*       that brings every element of the block into the E2M1 range, so no   */
/*       element saturates; e clamped to [-127, 127]; an all-zero block gets */
/*       the smallest scale, byte 0.                                         */
/*   M2  element code = E2M1 RNE(x / X) with R3's grid, tie and sign rules;  */
/*       x / X is exact (a power-of-two scaling).                            */
/*   M3  no second-level (tensor) scale.                                     */
/*   M4  packing as R5; the oracle keeps scales row-major [rows][cols/32].   */
/* ------------------------------------------------------------------------ */

/* E8M0: eight exponent bits, bias 127, no sign and no mantissa; 0xFF is NaN. */
double oracle_e8m0_value(unsigned byte)
{
    if ((byte & 0xFFu) == 0xFFu)
        return NAN;
    return ldexp(1.0, (int)(byte & 0xFFu) - 127);
}

/* M1.  bamax / 6 = f * 2^p with f in [0.5, 1) (frexp).  The quotient is a
 * power of two exactly when f == 0.5 (bamax = 6 * 2^k is exact in binary, and
 * any other fp32 bamax is at least 2^-24 away from it in relative terms, far
 * more than the fp64 rounding of the quotient), and then ceil(log2) = p - 1;
 * otherwise it is p. */
unsigned oracle_mx_block_scale(float bamax)
{
    int p, e;
    double f;
    if (!(bamax > 0.0f))
        return 0u;
    f = frexp((double)bamax / 6.0, &p);
    e = (f == 0.5) ? p - 1 : p;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return (unsigned)(e + 127);
}

/* Quantize the logical [rows][cols] window (cols % 32 == 0) of a row-major
 * fp32 matrix with leading dimension ld to MXFP4: packed codes
 * [rows][cols/2] and E8M0 scale bytes [rows][cols/32].  Returns 0, or -1 on
 * bad arguments or a non-finite input. */
int oracle_mx_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld,
                       uint8_t *codes, uint8_t *scales)
{
    int64_t nblk = cols / 32;
    if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            if (!isfinite(x[r * ld + c]))
                return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const float *blk = x + r * ld + b * 32;
            float bamax = 0.0f;
            unsigned s;
            double scale;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(blk[i]);
                if (a > bamax)
                    bamax = a;
            }
            s = oracle_mx_block_scale(bamax);
            scales[r * nblk + b] = (uint8_t)s;
            scale = oracle_e8m0_value(s);
            for (int i = 0; i < 32; i += 2) {
                /* exact quotients; a result below the fp32 normal range
                 * rounds to a signed value far below 0.25, code 0 either way */
                unsigned lo = oracle_e2m1_encode((float)((double)blk[i] / scale));
                unsigned hi = oracle_e2m1_encode((float)((double)blk[i + 1] / scale));
                codes[r * (cols / 2) + b * 16 + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return 0;
}

/* fp64 dequantization of an MXFP4 [rows][cols]: e * 2^(s - 127), exact.  (An
 * fp32 result would overflow for the largest codes at the top scales, so the
 * oracle keeps fp64.) */
int oracle_mx_dequantize_f64(const uint8_t *codes, const uint8_t *scales,
                             int64_t rows, int64_t cols, double *y)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            unsigned byte = codes[r * (cols / 2) + c / 2];
            unsigned code = (c & 1) ? (byte >> 4) : (byte & 15u);
            y[r * cols + c] = oracle_e2m1_value(code) *
                              oracle_e8m0_value(scales[r * (cols / 32) + c / 32]);
        }
    return 0;
}

/* Storage of one MXFP4 [rows][cols] tensor in bytes: packed codes and one
 * scale byte per 32 values ([MX]: about 4.25 bits per value). */
int64_t oracle_mx_storage_bytes(int64_t rows, int64_t cols)
{
    return rows * cols / 2 + rows * cols / 32;
}


/* ------------------------------------------------------------------------ */
/* MXFP8 activations for the W4A8 product ([EEF]: the Zhouyi X3 passage,    */
/* FP4 weights with activations quantized to FP8; on hardware whose native  */
/* mixed FP4 x FP8 product is block-scaled, both operands carry MX scales). */
/* Readings taken (the page gives no formula):                               */
/*   X1  block scale: 32 consecutive values share an E8M0 scale X = 2^e,     */
/*       e = ceil(log2(bamax / 448)): the smallest power of two that brings  */
/*       the block's largest magnitude into the E4M3 range (bamax <= 448 X), */
/*       clamped to [-127, 127]; an all-zero block gets byte 0 (M1 with      */
/*       E4M3's largest value in place of E2M1's).                           */
/*   X2  element: E4M3 RNE (ties to even, OCP "fn" grid) of x / X, which is  */
/*       exact; the sign is kept, also for values that round to zero.       */
/* ------------------------------------------------------------------------ */

/* X1.  bamax / 448 = f * 2^p with f in [0.5, 1); the quotient is a power of
 * two exactly when f == 0.5 (bamax = 448 * 2^k = 7 * 2^(k+6) is exact in
 * fp32, and any other fp32 bamax is relatively at least 2^-24 away from it,
 * far more than the fp64 rounding of the quotient), and then
 * ceil(log2) = p - 1; otherwise it is p. */
unsigned oracle_mx8_block_scale(float bamax)
{
    int p, e;
    double f;
    if (!(bamax > 0.0f))
        return 0u;
    f = frexp((double)bamax / 448.0, &p);
    e = (f == 0.5) ? p - 1 : p;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return (unsigned)(e + 127);
}

/* X2: signed E4M3 byte of v, |v| <= 448 by construction (satfinite beyond). */
unsigned oracle_e4m3_encode_signed(float v)
{
    unsigned mag = oracle_e4m3_encode(fabsf(v));
    return signbit(v) ? (mag | 0x80u) : mag;
}

/* Quantize the logical [rows][cols] window (cols % 32 == 0) of a row-major
 * fp32 matrix with leading dimension ld to MXFP8: E4M3 bytes [rows][cols]
 * and E8M0 scale bytes [rows][cols/32].  Returns 0, or -1 on bad arguments or
 * a non-finite input. */
int oracle_mx8_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld,
                        uint8_t *elems, uint8_t *scales)
{
    int64_t nblk = cols / 32;
    if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            if (!isfinite(x[r * ld + c]))
                return -1;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const float *blk = x + r * ld + b * 32;
            float bamax = 0.0f;
            unsigned s;
            double scale;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(blk[i]);
                if (a > bamax)
                    bamax = a;
            }
            s = oracle_mx8_block_scale(bamax);
            scales[r * nblk + b] = (uint8_t)s;
            scale = oracle_e8m0_value(s);
            for (int i = 0; i < 32; ++i)
                elems[r * cols + b * 32 + i] =
                    (uint8_t)oracle_e4m3_encode_signed((float)((double)blk[i] / scale));
        }
    }
    return 0;
}

/* fp64 dequantization of an MXFP8 [rows][cols]: e4m3 * 2^(s - 127), exact. */
int oracle_mx8_dequantize_f64(const uint8_t *elems, const uint8_t *scales,
                              int64_t rows, int64_t cols, double *y)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0)
        return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            y[r * cols + c] = oracle_e4m3_value(elems[r * cols + c]) *
                              oracle_e8m0_value(scales[r * (cols / 32) + c / 32]);
    return 0;
}
