/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for NVFP4 quantization and the
 * block-scaled FP4 matrix products.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator
 * with the CUDA library; the two meet only on seeded inputs.
 *
 * Sources (web pages, cited by title and section):
 *  [DiT]  "NVFP4-DiT: Efficient 4-Bit Audio-Guided Video Diffusion Transformers
 *          for Low-Cost Video Generation" (project README), Methodology,
 *          1. Theoretical foundations: Definition III.1 (the quantizer
 *          Q_FP4(v;s) = s * clip(round(v/s)_FP4, -6, 6)), the E2M1 bit split
 *          (1 sign, 2 exponent, 1 mantissa bit), Lemma III.2 (eps = 2^-3);
 *          3. Systems optimization (two FP4 values per byte, FP32 accumulation).
 *  [RFC]  "[RFC]: NVFP4 Quantization Support for Diffusion Models" (vllm-omni
 *          issue 1959), Motivation: two-level scaling, one FP8 micro-block
 *          scale per 16 values plus one FP32 tensor-level scale; Open
 *          Questions 1: weight-only (W4A16) versus W4A4.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - round() is round-to-nearest-even onto the E2M1 format; the magnitude set
 *    of a 1-2-1 float is {0, .5, 1, 1.5, 2, 3, 4, 6} (the page's list, which
 *    shows 0.75 and omits 0, is read as garbled: 16 codes cannot hold 17 values).
 *  - The FP32 tensor scale maps the tensor's amax onto 6 * 448, the largest
 *    magnitude an E2M1 element times an E4M3 block scale can express:
 *    g = amax / 2688 (IEEE single division).
 *  - The FP8 block scale is E4M3FN (bias 7, max 448, no infinities), rounded
 *    to nearest even with saturation: sf = E4M3(a_b / (6 g)); the element
 *    quotient uses the decoded scale s = dec(sf) * g, so quantize and
 *    dequantize use the same s.
 *  - All-zero block or s == 0: codes 0x0 and no division.  Elements keep the
 *    sign of x (a negative value that rounds to zero gives code 0x8).
 *  - Element 2j goes to the low nibble, 2j+1 to the high nibble.
 *  - The 16-value block runs along K (the reduction axis); scales are stored
 *    in the tensor-core scale-factor layout (128-row x 4-block atoms of 512
 *    bytes), rows padded to a multiple of 128 with zero bytes.
 *  - Fake quantization (QAT) returns the same value the dequantizer gives
 *    for the codes (e2m1 * dec(sf) * g, rounded once), so a trained model sees
 *    in its forward pass exactly what the W4A4 product will multiply.  The
 *    straight-through estimator passes the gradient unchanged; the optional
 *    clip mask marks elements with |x| > 6 s (clip's derivative is zero
 *    there), and a zero scale s clips nothing.
 *
 * Build: plain C99, no fast-math, no FMA contraction (see oracle/build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Rounding a non-negative real (given as a double holding an exact value) to
 * a binary floating-point format with `mant_bits` fraction bits and smallest
 * normal exponent `emin`, to nearest with ties to even, saturating at `maxval`
 * (maxval = INFINITY means: overflow to infinity above `maxfinite`).
 * m / ulp is a power-of-two scaling and therefore exact; nearbyint() rounds
 * ties to even in the default rounding mode.                                  */
static double round_to_format(double m, int mant_bits, int emin, double maxval)
{
    if (m == 0.0) return 0.0;
    if (m >= maxval) return maxval;
    int e;
    (void)frexp(m, &e);          /* m = f * 2^e, f in [0.5, 1): floor(log2 m) = e - 1 */
    int E = e - 1;
    if (E < emin) E = emin;      /* subnormal range keeps the smallest spacing */
    double ulp = ldexp(1.0, E - mant_bits);
    double r = nearbyint(m / ulp) * ulp;
    if (r > maxval) r = maxval;
    return r;
}

/* ---------------------------- E2M1 --------------------------------------- */
/* 1 sign, 2 exponent (bias 1), 1 mantissa bit [DiT, Definition III.1]. */
double oracle_e2m1_decode(unsigned code)
{
    unsigned e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, (int)e - 1);
    return (code & 8u) ? -mag : mag;
}

/* Round an FP32 quotient q = x / s onto E2M1 (RNE, clip to [-6, 6]) and return
 * the 4-bit code.  The sign bit is the sign of q.                             */
unsigned oracle_e2m1_encode(float q)
{
    double m = fabs((double)q);
    double r = round_to_format(m, 1, 0, 6.0);
    unsigned mag_code = 0;
    for (unsigned c = 0; c < 8; ++c)
        if (oracle_e2m1_decode(c) == r) { mag_code = c; break; }
    return (signbit(q) ? 8u : 0u) | mag_code;
}

/* ---------------------------- E4M3 (FN) ---------------------------------- */
/* 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 is NaN, there is no
 * infinity; largest finite 448, smallest subnormal 2^-9.                     */
double oracle_e4m3_decode(unsigned code)
{
    unsigned e = (code >> 3) & 15u, m = code & 7u;
    if (e == 15u && m == 7u) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, (int)e - 7);
    return (code & 0x80u) ? -mag : mag;
}

/* Encode a non-negative FP32 value as an unsigned E4M3 scale: RNE, saturating
 * at 448 (block scales are non-negative, so the sign bit is always 0).       */
unsigned oracle_e4m3_encode(float v)
{
    double r = round_to_format((double)v, 3, -6, 448.0);
    if (r == 0.0) return 0u;
    if (r < ldexp(1.0, -6))                     /* subnormal: m * 2^-9 */
        return (unsigned)(r / ldexp(1.0, -9));
    int e;
    double f = frexp(r, &e);                    /* r = f * 2^e, f in [0.5,1) */
    int E = e - 1;                              /* r = (2f) * 2^E, 2f in [1,2) */
    unsigned mant = (unsigned)((2.0 * f - 1.0) * 8.0);
    return ((unsigned)(E + 7) << 3) | mant;
}

/* ---------------------------- bf16 --------------------------------------- */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round an exact double to bf16 (8 significant bits, emin -126), ties to even,
 * overflow to infinity.                                                       */
uint16_t oracle_bf16_from_double(double v)
{
    double m = fabs(v);
    double r;
    const double maxfinite = ldexp(255.0 / 128.0, 127);
    if (isnan(v)) return 0x7FC0u;
    if (m == 0.0) r = 0.0;
    else {
        int e;
        (void)frexp(m, &e);
        int E = e - 1;
        if (E < -126) E = -126;
        double ulp = ldexp(1.0, E - 7);
        r = nearbyint(m / ulp) * ulp;
        if (r > maxfinite) r = INFINITY;
    }
    float f = (float)r;                          /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    u >>= 16;
    if (signbit(v)) u |= 0x8000u;
    return (uint16_t)u;
}

/* ---------------------- scale-factor layout ------------------------------ */
/* Bytes of the scale buffer for a [rows, k] tensor: rows padded to 128, one
 * byte per 16-value block.                                                   */
int64_t oracle_sf_bytes(int64_t rows, int64_t k)
{
    return ((rows + 127) / 128) * 128 * (k / 16);
}

/* Byte offset of the scale of (row r, block c) with kb = k/16 blocks per row
 * (kb a multiple of 4): 128 x 4 atoms of 512 bytes, atoms ordered block-column
 * fastest; inside an atom row r%32 picks a 16-byte line, (r%128)/32 a 4-byte
 * word in it, and c%4 the byte.                                              */
int64_t oracle_sf_offset(int64_t r, int64_t c, int64_t kb)
{
    int64_t atom = (r / 128) * (kb / 4) + c / 4;
    return atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* --------------------------- quantize ------------------------------------ */
/* Tensor scale: g = amax / (6 * 448), amax = max |x| over the whole tensor. */
float oracle_tensor_scale_f32(const float *x, int64_t rows, int64_t k, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float a = fabsf(x[r * ld + j]);
            if (a > amax) amax = a;
        }
    return amax / 2688.0f;
}

/* The same tensor scale over a bf16 tensor (bf16 -> fp32 is exact). */
float oracle_tensor_scale_bf16(const uint16_t *x, int64_t rows, int64_t k, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float a = fabsf(oracle_bf16_to_f32(x[r * ld + j]));
            if (a > amax) amax = a;
        }
    return amax / 2688.0f;
}

/* Two-level NVFP4 quantization of an FP32 tensor x[rows, k] (row stride ld):
 *   g  = amax / 2688 unless scale_given (then g = *g_io)        [RFC, Motivation]
 *   per row, per 16 consecutive values along k:
 *     a_b = max |x|;  d = 6 g;  sf = E4M3(a_b / d);  s = dec(sf) * g
 *   per element:  q = x / s;  code = RNE_E2M1(clip(q, -6, 6))  [DiT, Def. III.1]
 *   pack two codes per byte (element 2j low nibble)           [DiT, Systems opt.]
 * codes: rows * k/2 bytes, row stride k/2.  sf: oracle_sf_bytes(rows, k) bytes
 * in the tensor-core layout, padding rows zero.  k must be a multiple of 64.  */
void oracle_quantize_f32(const float *x, int64_t rows, int64_t k, int64_t ld,
                         int scale_given, float *g_io, uint8_t *codes, uint8_t *sf)
{
    float g = scale_given ? *g_io : oracle_tensor_scale_f32(x, rows, k, ld);
    if (!scale_given) *g_io = g;
    const int64_t kb = k / 16;
    memset(sf, 0, (size_t)oracle_sf_bytes(rows, k));
    memset(codes, 0, (size_t)(rows * (k / 2)));
    const float d = 6.0f * g;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < kb; ++c) {
            const float *blk = x + r * ld + c * 16;
            float ab = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(blk[i]);
                if (a > ab) ab = a;
            }
            unsigned sfc = 0u;
            if (d > 0.0f) {
                float ratio = ab / d;
                sfc = oracle_e4m3_encode(ratio);
            }
            sf[oracle_sf_offset(r, c, kb)] = (uint8_t)sfc;
            float sdec = (float)oracle_e4m3_decode(sfc);
            float s = sdec * g;
            for (int i = 0; i < 16; ++i) {
                unsigned code = 0u;
                if (s != 0.0f) {
                    float q = blk[i] / s;
                    code = oracle_e2m1_encode(q);
                }
                int64_t j = c * 16 + i;
                codes[r * (k / 2) + j / 2] |= (uint8_t)(code << (4 * (j & 1)));
            }
        }
    }
}

/* The same on a bf16 tensor (bf16 -> fp32 is exact). */
void oracle_quantize_bf16(const uint16_t *x, int64_t rows, int64_t k, int64_t ld,
                          int scale_given, float *g_io, uint8_t *codes, uint8_t *sf)
{
    float *xf = (float *)malloc((size_t)(rows * k) * sizeof(float));
    if (!xf) return;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j)
            xf[r * k + j] = oracle_bf16_to_f32(x[r * ld + j]);
    oracle_quantize_f32(xf, rows, k, k, scale_given, g_io, codes, sf);
    free(xf);
}

/* -------------------------- dequantize ----------------------------------- */
/* Element value before the tensor scale: e2m1(code) * dec(sf), exact.       */
static double deq_elem(const uint8_t *codes, const uint8_t *sf, int64_t r, int64_t j, int64_t k)
{
    uint8_t byte = codes[r * (k / 2) + j / 2];
    unsigned code = (j & 1) ? (byte >> 4) : (byte & 15u);
    double s = oracle_e4m3_decode(sf[oracle_sf_offset(r, j / 16, k / 16)]);
    return oracle_e2m1_decode(code) * s;
}

/* v = (e2m1(code) * dec(sf)) * g, exact in double (at most 6 + 24 significant
 * bits) [DiT, Def. III.1: the quantizer returns s * round(...)].             */
void oracle_dequantize_f64(const uint8_t *codes, const uint8_t *sf, float g,
                           int64_t rows, int64_t k, double *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j)
            out[r * k + j] = deq_elem(codes, sf, r, j, k) * (double)g;
}

/* Dequantize rounded once to FP32 (RNE) or bf16 (RNE). */
void oracle_dequantize_f32(const uint8_t *codes, const uint8_t *sf, float g,
                           int64_t rows, int64_t k, float *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j)
            out[r * k + j] = (float)(deq_elem(codes, sf, r, j, k) * (double)g);
}

void oracle_dequantize_bf16(const uint8_t *codes, const uint8_t *sf, float g,
                            int64_t rows, int64_t k, uint16_t *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j)
            out[r * k + j] = oracle_bf16_from_double(deq_elem(codes, sf, r, j, k) * (double)g);
}

/* ------------------------------ GEMM ------------------------------------- */
/* W4A4 [DiT, Systems optimization; RFC, Open Questions 1]:
 *   Y[m,n] = g_a * g_b * sum_k (a^[m,k] * b^[n,k]),  a^ = e2m1(code) * dec(sf)
 * in double.  A is [M,K] (activations), B is [N,K] (weights, nn.Linear
 * layout), Y = A B^T is [M,N].  Rows m0 .. m0+mrows-1 of Y are computed (so a
 * caller can evaluate a slice); y holds mrows * N doubles.                   */
void oracle_gemm_w4a4_rows(const uint8_t *a_codes, const uint8_t *a_sf, float g_a,
                           const uint8_t *b_codes, const uint8_t *b_sf, float g_b,
                           int64_t M, int64_t N, int64_t K, int64_t m0, int64_t mrows,
                           double *y)
{
    (void)M;
    double *bh = (double *)malloc((size_t)(N * K) * sizeof(double));
    double *ah = (double *)malloc((size_t)K * sizeof(double));
    if (!bh || !ah) { free(bh); free(ah); return; }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j)
            bh[n * K + j] = deq_elem(b_codes, b_sf, n, j, K);
    const double alpha = (double)g_a * (double)g_b;
    for (int64_t i = 0; i < mrows; ++i) {
        int64_t m = m0 + i;
        for (int64_t j = 0; j < K; ++j) ah[j] = deq_elem(a_codes, a_sf, m, j, K);
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            const double *bn = bh + n * K;
            for (int64_t j = 0; j < K; ++j) acc += ah[j] * bn[j];
            y[i * N + n] = alpha * acc;
        }
    }
    free(bh);
    free(ah);
}

void oracle_gemm_w4a4(const uint8_t *a_codes, const uint8_t *a_sf, float g_a,
                      const uint8_t *b_codes, const uint8_t *b_sf, float g_b,
                      int64_t M, int64_t N, int64_t K, double *y)
{
    oracle_gemm_w4a4_rows(a_codes, a_sf, g_a, b_codes, b_sf, g_b, M, N, K, 0, M, y);
}

/* One output element (for sampled checks at full size). */
double oracle_gemm_w4a4_at(const uint8_t *a_codes, const uint8_t *a_sf, float g_a,
                           const uint8_t *b_codes, const uint8_t *b_sf, float g_b,
                           int64_t K, int64_t m, int64_t n)
{
    double acc = 0.0;
    for (int64_t j = 0; j < K; ++j)
        acc += deq_elem(a_codes, a_sf, m, j, K) * deq_elem(b_codes, b_sf, n, j, K);
    return (double)g_a * (double)g_b * acc;
}

/* W4A16 [RFC, Open Questions 1; weights-only NVFP4]:
 *   Y[m,n] = g_w * sum_k x[m,k] * w^[n,k]   in double, x the bf16 activation. */
void oracle_gemm_w4a16_rows(const uint16_t *x, const uint8_t *w_codes, const uint8_t *w_sf,
                            float g_w, int64_t M, int64_t N, int64_t K,
                            int64_t m0, int64_t mrows, double *y)
{
    (void)M;
    double *wh = (double *)malloc((size_t)(N * K) * sizeof(double));
    if (!wh) return;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j)
            wh[n * K + j] = deq_elem(w_codes, w_sf, n, j, K);
    for (int64_t i = 0; i < mrows; ++i) {
        int64_t m = m0 + i;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j)
                acc += (double)oracle_bf16_to_f32(x[m * K + j]) * wh[n * K + j];
            y[i * N + n] = (double)g_w * acc;
        }
    }
    free(wh);
}

double oracle_gemm_w4a16_at(const uint16_t *x, const uint8_t *w_codes, const uint8_t *w_sf,
                            float g_w, int64_t K, int64_t m, int64_t n)
{
    double acc = 0.0;
    for (int64_t j = 0; j < K; ++j)
        acc += (double)oracle_bf16_to_f32(x[m * K + j]) * deq_elem(w_codes, w_sf, n, j, K);
    return (double)g_w * acc;
}

/* ----------------------- QAT fake quantization --------------------------- */
/* Fake quantization for quantization-aware training [DiT, Definition III.1;
 * Methodology 2: training uses a straight-through estimator across the
 * fake quantizer].  The forward value is the quantizer's output
 *   y = Q_FP4(x; s) = e2m1(code) * dec(sf) * g,  rounded once to bf16 or f32,
 * with the codes and scales oracle_quantize_bf16 makes (same tensor-scale
 * rule, g_io in/out), and the clip indicator that the estimator's backward
 * rule uses:
 *   clipped = s > 0 and |x| > 6 s      (exact comparison, s = fl32(dec(sf) * g))
 * i.e. the elements whose scaled value x / s lies outside clip's range
 * [-6, 6].  A block with s == 0 (all zero, or a zero tensor scale) has no
 * clipped element: its values flush to zero by rounding, not by clip.
 * y: rows * k values, row stride k; bf16 bits when out_f32 == 0, else float.
 * mask (nullable): rows * k/8 bytes, row stride k/8; element j of a row is
 * bit j % 8 of byte j / 8.                                                    */
void oracle_fake_quantize_bf16(const uint16_t *x, int64_t rows, int64_t k, int64_t ld,
                               int scale_given, float *g_io, int out_f32, void *y, uint8_t *mask)
{
    const int64_t kb = k / 16;
    uint8_t *codes = (uint8_t *)malloc((size_t)(rows * (k / 2)) + 1);
    uint8_t *sf = (uint8_t *)malloc((size_t)oracle_sf_bytes(rows, k) + 1);
    if (!codes || !sf) { free(codes); free(sf); return; }
    oracle_quantize_bf16(x, rows, k, ld, scale_given, g_io, codes, sf);
    const float g = *g_io;
    if (out_f32) oracle_dequantize_f32(codes, sf, g, rows, k, (float *)y);
    else oracle_dequantize_bf16(codes, sf, g, rows, k, (uint16_t *)y);
    if (mask) {
        memset(mask, 0, (size_t)(rows * (k / 8)));
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t j = 0; j < k; ++j) {
                float sdec = (float)oracle_e4m3_decode(sf[oracle_sf_offset(r, j / 16, kb)]);
                float s = sdec * g;                       /* the quantizer's s, as above */
                double a = fabs((double)oracle_bf16_to_f32(x[r * ld + j]));
                if (s > 0.0f && a > 6.0 * (double)s)      /* 6 s exact in double */
                    mask[r * (k / 8) + j / 8] |= (uint8_t)(1u << (j % 8));
            }
    }
    free(codes);
    free(sf);
}

/* Backward rule of the straight-through estimator with the clip indicator
 * [DiT, Methodology 2]: the gradient passes unchanged (the estimator treats
 * round() as the identity) except where clip() cut the value off, whose
 * derivative is zero there:
 *   grad_x = 0 where clipped, grad_y elsewhere        (masked elements: +0)
 * grad_y, grad_x: rows * k elements of elem_bytes bytes (2: bf16, 4: f32),
 * row stride k; mask as oracle_fake_quantize_bf16 writes it.                  */
void oracle_ste_backward(const void *grad_y, const uint8_t *mask, int64_t rows, int64_t k,
                         int elem_bytes, void *grad_x)
{
    const uint8_t *src = (const uint8_t *)grad_y;
    uint8_t *dst = (uint8_t *)grad_x;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            int64_t e = r * k + j;
            int clipped = (mask[r * (k / 8) + j / 8] >> (j % 8)) & 1;
            if (clipped) memset(dst + e * elem_bytes, 0, (size_t)elem_bytes);
            else memcpy(dst + e * elem_bytes, src + e * elem_bytes, (size_t)elem_bytes);
        }
}

/* ------------------------- epilogue activation --------------------------- */
/* GELU in its tanh form, 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), in
 * double.  The pages name no activation; this is the one the DiT family's
 * MLPs use (a reading), applied by the fused GEMM epilogue to alpha * acc.   */
double oracle_gelu_tanh(double v)
{
    const double c = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/* Elementwise over n doubles (in place allowed). */
void oracle_gelu_tanh_array(const double *in, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_gelu_tanh(in[i]);
}

/* ------------------------------ MXFP4 ------------------------------------ */
/* The MX variant ("[RFC]: NVFP4 Quantization Support for Diffusion Models",
 * Related: the MXFP4 RFC, a related format): E2M1 elements in blocks of 32
 * along k, one power-of-two scale per block stored as an unsigned E8M0 byte
 * (value 2^(byte - 127)), no tensor scale.  The pages give no rule for the
 * scale; the reading taken is the OCP Microscaling (MX) specification's:
 *   shared exponent  e = floor(log2(max|x|)) - 2      (2 = E2M1's largest exponent)
 *   clamped to [-127, 127]; an all-zero block takes e = -127 (byte 0);
 *   element code     RNE_E2M1(clip(x / 2^e, -6, 6)), sign of x kept.
 * x / 2^e is exact (a power-of-two scaling), so no quotient rounding arises.
 * Scales use the tensor-core scale layout with kb32 = k/32 blocks per row
 * (k a multiple of 128, so that a row's blocks fill whole 4-block words).   */
int64_t oracle_mx_sf_bytes(int64_t rows, int64_t k)
{
    return ((rows + 127) / 128) * 128 * (k / 32);
}

void oracle_mx_quantize_bf16(const uint16_t *x, int64_t rows, int64_t k, int64_t ld,
                             uint8_t *codes, uint8_t *sf)
{
    const int64_t kb = k / 32;
    memset(sf, 0, (size_t)oracle_mx_sf_bytes(rows, k));
    memset(codes, 0, (size_t)(rows * (k / 2)));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < kb; ++c) {
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)oracle_bf16_to_f32(x[r * ld + c * 32 + i]));
                if (a > amax) amax = a;
            }
            int e = -127;
            if (amax > 0.0) {
                int ex;
                (void)frexp(amax, &ex);          /* amax = f 2^ex, f in [0.5, 1) */
                e = (ex - 1) - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            sf[oracle_sf_offset(r, c, kb)] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i) {
                int64_t j = c * 32 + i;
                double q = ldexp((double)oracle_bf16_to_f32(x[r * ld + j]), -e);   /* exact */
                unsigned code = oracle_e2m1_encode((float)q);                     /* |q| < 8: exact in float */
                codes[r * (k / 2) + j / 2] |= (uint8_t)(code << (4 * (j & 1)));
            }
        }
}

/* v = e2m1(code) * 2^(sf - 127), exact in double. */
static double mx_deq_elem(const uint8_t *codes, const uint8_t *sf, int64_t r, int64_t j, int64_t k)
{
    uint8_t byte = codes[r * (k / 2) + j / 2];
    unsigned code = (j & 1) ? (byte >> 4) : (byte & 15u);
    int s = (int)sf[oracle_sf_offset(r, j / 32, k / 32)] - 127;
    return ldexp(oracle_e2m1_decode(code), s);
}

void oracle_mx_dequantize_f64(const uint8_t *codes, const uint8_t *sf, int64_t rows, int64_t k, double *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j)
            out[r * k + j] = mx_deq_elem(codes, sf, r, j, k);
}

/* MX x MX product in double: Y[m,n] = sum_k a^[m,k] b^[n,k], rows m0.. of Y. */
void oracle_mx_gemm_rows(const uint8_t *a_codes, const uint8_t *a_sf, const uint8_t *b_codes,
                         const uint8_t *b_sf, int64_t N, int64_t K, int64_t m0, int64_t mrows, double *y)
{
    double *bh = (double *)malloc((size_t)(N * K) * sizeof(double));
    double *ah = (double *)malloc((size_t)K * sizeof(double));
    if (!bh || !ah) { free(bh); free(ah); return; }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j)
            bh[n * K + j] = mx_deq_elem(b_codes, b_sf, n, j, K);
    for (int64_t i = 0; i < mrows; ++i) {
        for (int64_t j = 0; j < K; ++j) ah[j] = mx_deq_elem(a_codes, a_sf, m0 + i, j, K);
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < K; ++j) acc += ah[j] * bh[n * K + j];
            y[i * N + n] = acc;
        }
    }
    free(bh);
    free(ah);
}

/* ---------------------- adaptive block size (Alg. 1) ---------------------- */
/* Two-level NVFP4 quantization with a block of `block` values along k
 * [DiT, Algorithmic framework: Algorithm 1 / Eq. 9 choose the block size per
 * layer from {1, 2, 4, 8, 16, 32, 64}]: the same rule as oracle_quantize_f32
 * with the block maximum taken over `block` values,
 *   sf = E4M3(a_b / (6 g)),  s = dec(sf) * g,  code = E2M1(x / s).
 * For block >= 16 (a multiple of 16 dividing 64) the codes and scales are
 * written in the block-16 tensor-core layout, each block scale repeated in its
 * block/16 slots, so the block-16 GEMM multiplies them unchanged.           */
void oracle_quantize_block_bf16(const uint16_t *x, int64_t rows, int64_t k, int64_t ld, int block,
                                int scale_given, float *g_io, uint8_t *codes, uint8_t *sf)
{
    float g = scale_given ? *g_io : oracle_tensor_scale_bf16(x, rows, k, ld);
    if (!scale_given) *g_io = g;
    const int64_t kb = k / 16;
    memset(sf, 0, (size_t)oracle_sf_bytes(rows, k));
    memset(codes, 0, (size_t)(rows * (k / 2)));
    const float d = 6.0f * g;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k / block; ++c) {
            float ab = 0.0f;
            for (int i = 0; i < block; ++i) {
                float a = fabsf(oracle_bf16_to_f32(x[r * ld + c * block + i]));
                if (a > ab) ab = a;
            }
            unsigned sfc = (d > 0.0f) ? oracle_e4m3_encode(ab / d) : 0u;
            for (int t = 0; t < block / 16; ++t)
                sf[oracle_sf_offset(r, c * (block / 16) + t, kb)] = (uint8_t)sfc;
            float s = (float)oracle_e4m3_decode(sfc) * g;
            for (int i = 0; i < block; ++i) {
                int64_t j = c * block + i;
                unsigned code = 0u;
                if (s != 0.0f) code = oracle_e2m1_encode(oracle_bf16_to_f32(x[r * ld + j]) / s);
                codes[r * (k / 2) + j / 2] |= (uint8_t)(code << (4 * (j & 1)));
            }
        }
}

/* Error(l, b) of Eq. 9 for every candidate block size b = 2^i, i = 0..6: the
 * squared quantization error sum_j (x_j - Q_b(x)_j)^2, Q_b(x)_j =
 * e2m1(code_j) * dec(sf) * g with the rule above (any b dividing k), in
 * double; err[7] receives them and *sumsq = sum_j x_j^2.  The tensor scale
 * is g (the caller's, e.g. amax / 2688).                                     */
void oracle_block_size_errors(const uint16_t *x, int64_t rows, int64_t k, int64_t ld, float g,
                              double *err, double *sumsq)
{
    const float d = 6.0f * g;
    double ss = 0.0;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            double v = (double)oracle_bf16_to_f32(x[r * ld + j]);
            ss += v * v;
        }
    *sumsq = ss;
    for (int i = 0; i < 7; ++i) {
        const int b = 1 << i;
        double e = 0.0;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < k / b; ++c) {
                float ab = 0.0f;
                for (int t = 0; t < b; ++t) {
                    float a = fabsf(oracle_bf16_to_f32(x[r * ld + c * b + t]));
                    if (a > ab) ab = a;
                }
                unsigned sfc = (d > 0.0f) ? oracle_e4m3_encode(ab / d) : 0u;
                double sdec = oracle_e4m3_decode(sfc);
                float s = (float)sdec * g;
                for (int t = 0; t < b; ++t) {
                    float xv = oracle_bf16_to_f32(x[r * ld + c * b + t]);
                    double q = 0.0;
                    if (s != 0.0f) q = oracle_e2m1_decode(oracle_e2m1_encode(xv / s)) * sdec * (double)g;
                    double diff = (double)xv - q;
                    e += diff * diff;
                }
            }
        err[i] = e;
    }
}

/* Eq. 9: argmin over b of Error(b) + lambda * Memory(b) / Memory_max, with
 * Error(b) = err[b] / sumsq (relative squared error) and Memory(b) = 4 + 8/b
 * bits per value (E2M1 element + one E8-bit E4M3 scale per block; the tensor
 * scale's 32 bits are shared by the whole tensor and left out), so
 * Memory_max = Memory(1) = 12.  Returns the chosen b (the first minimum).    */
int oracle_select_block_size(const double *err, double sumsq, double lambda)
{
    int best = 1;
    double bestv = 0.0;
    for (int i = 0; i < 7; ++i) {
        const int b = 1 << i;
        double e = sumsq > 0.0 ? err[i] / sumsq : 0.0;
        double v = e + lambda * (4.0 + 8.0 / b) / 12.0;
        if (i == 0 || v < bestv) { bestv = v; best = b; }
    }
    return best;
}

/* ------------------------ attention over NVFP4 K / V ---------------------- */
/* Attention of one head over NVFP4 operands [DiT, Algorithmic framework,
 * Eq. 10: Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k) + log(s_head)) V, with
 * a learnable per-head scale s_head; Systems optimization: FP4-packed
 * attention].  Q [H*Lq, d], K and V [H*Lk, d] are NVFP4 tensors quantized
 * along d (blocks of 16, tensor scales g_q, g_k, g_v); head h owns rows
 * h*Lq .. and h*Lk .. .  In double, from the exact element values:
 *   z[i][j] = (q^_i . k^_j) / sqrt(d) + log(s_head[h])
 *   p[i][j] = exp(z[i][j] - max_j z[i][j]) / sum_j exp(...)
 *   O[i]    = sum_j p[i][j] v^_j
 * for query rows q0 .. q0+nq-1 of head h; out holds nq * d doubles.          */
void oracle_attention_rows(const uint8_t *q_codes, const uint8_t *q_sf, float g_q,
                           const uint8_t *k_codes, const uint8_t *k_sf, float g_k,
                           const uint8_t *v_codes, const uint8_t *v_sf, float g_v,
                           int64_t Lq, int64_t Lk, int64_t d, const double *s_head, int64_t h,
                           int64_t q0, int64_t nq, double *out)
{
    double *kh = (double *)malloc((size_t)(Lk * d) * sizeof(double));
    double *vh = (double *)malloc((size_t)(Lk * d) * sizeof(double));
    double *z = (double *)malloc((size_t)Lk * sizeof(double));
    double *qi = (double *)malloc((size_t)d * sizeof(double));
    if (!kh || !vh || !z || !qi) { free(kh); free(vh); free(z); free(qi); return; }
    for (int64_t j = 0; j < Lk; ++j)
        for (int64_t c = 0; c < d; ++c) {
            kh[j * d + c] = deq_elem(k_codes, k_sf, h * Lk + j, c, d) * (double)g_k;
            vh[j * d + c] = deq_elem(v_codes, v_sf, h * Lk + j, c, d) * (double)g_v;
        }
    const double bias = log(s_head[h]);
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int64_t t = 0; t < nq; ++t) {
        const int64_t i = q0 + t;
        for (int64_t c = 0; c < d; ++c) qi[c] = deq_elem(q_codes, q_sf, h * Lq + i, c, d) * (double)g_q;
        double zmax = -INFINITY;
        for (int64_t j = 0; j < Lk; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) acc += qi[c] * kh[j * d + c];
            z[j] = acc * inv_sqrt_d + bias;
            if (z[j] > zmax) zmax = z[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < Lk; ++j) { z[j] = exp(z[j] - zmax); l += z[j]; }
        for (int64_t c = 0; c < d; ++c) {
            double o = 0.0;
            for (int64_t j = 0; j < Lk; ++j) o += z[j] * vh[j * d + c];
            out[t * d + c] = o / l;
        }
    }
    free(kh); free(vh); free(z); free(qi);
}

/* ------------------------------ LayerNorm -------------------------------- */
/* The producer of a block's first projections.  The pages name LayerNorm
 * only as part of the DiT blocks whose linear layers run in FP4 and do not
 * define it; the reading taken is the DiT pre-norm: LayerNorm over the hidden
 * dimension without its own affine, followed by the adaLN modulation
 * x (1 + scale) + shift of each sample, which is a per-channel affine shared
 * by a group of rows.  Written out:
 *   S1 = sum_j x_j,  S2 = sum_j x_j^2          double, in index order
 *   mu = S1 / k,  var = max(S2 / k - mu^2, 0),  rstd = 1 / sqrt(var + eps)
 *                                              double, one rounding per op
 *   y_j = ((x_j - (float)mu) * (float)rstd) * gamma_j + beta_j
 *                                              FP32, one rounding per op
 * gamma, beta: FP32 [groups, k] (row r uses group r / rows_per_group), or
 * NULL for 1 and 0.  Every square of a bf16 value is exact in double, and so
 * are the sums wherever the row's values span fewer than about 45 binary
 * orders of magnitude; then any summation order gives these S1 and S2.
 * y: FP32 [rows, k] contiguous.                                              */
void oracle_layernorm_f32(const uint16_t *x, int64_t rows, int64_t k, int64_t ld, const float *gamma,
                          const float *beta, int64_t rows_per_group, double eps, float *y)
{
    for (int64_t r = 0; r < rows; ++r) {
        double s1 = 0.0, s2 = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            const double v = (double)oracle_bf16_to_f32(x[r * ld + j]);
            s1 += v;
            s2 += v * v;
        }
        const double mu = s1 / (double)k;
        double var = s2 / (double)k - mu * mu;
        if (var < 0.0) var = 0.0;
        const double rstd = 1.0 / sqrt(var + eps);
        const float mu32 = (float)mu, rstd32 = (float)rstd;
        const int64_t grp = rows_per_group > 0 ? r / rows_per_group : 0;
        for (int64_t j = 0; j < k; ++j) {
            const float xv = oracle_bf16_to_f32(x[r * ld + j]);
            float v = xv - mu32;
            v = v * rstd32;
            if (gamma) v = v * gamma[grp * k + j];
            if (beta) v = v + beta[grp * k + j];
            y[r * k + j] = v;
        }
    }
}
