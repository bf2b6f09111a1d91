/*
 * oracle.c -- plain, slow CPU reference for fine-grained block quantization
 * (FP8-E4M3 with fp32 or E8M0 block scales, NVFP4) and the block-scaled GEMM.
 *
 * THIS IS TEST INFRASTRUCTURE.  It is the yardstick the CUDA path is checked
 * against; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load it.  It shares no code, header, table or constant
 * generator with the CUDA library, and the CUDA library never calls it.
 *
 * Sources of what is computed (the pages are cited by title and section):
 *   - "fireworks-prequant 0.1.0" (PyPI page), "Formats" table: mxfp8 is
 *     1x32-block FP8 with E8M0 scales, nvfp4 is packed FP4 with FP8 block
 *     scales; "Quick start": the quantized weight is float8_e4m3fn and its
 *     scale tensor ("weight_scale_inv") is uint8 E8M0.
 *   - "FP8 в DeepSeek V3 ...", sections "Как FP8 встроен в DeepSeek V3"
 *     (online per-token-per-128-channel activation quantization) and
 *     "Почему обычное округление не подходит" (128x128 weight blocks with a
 *     scale inverse used for dequantization).
 *   - "DeepSeek R1 and V3 get quantization-aware fine-tuning on Fireworks",
 *     "Interpretation": the LoRA delta is merged into the base weight, the
 *     merged bf16 weight is converted to block-wise FP8, and the forward pass
 *     fake-quantizes merged weights and activations.
 *   - "DeepSeek-V3 Blog 5: Low-Precision Training", "Hardware Optimization":
 *     FP8 products, accumulation in higher precision (fp32 here).
 * The pages give no bit-level formats.  The element encodings follow the
 * public OCP Microscaling (MX) v1.0 definitions; the rounding convention is
 * round-to-nearest-even with saturation to +-448 for E4M3 and to +-6 for
 * E2M1, and the MXFP8 scale is E8M0 = 2^ceil(log2(amax/448)).
 *
 * Arithmetic discipline: every decode goes through fp64 (exact for all the
 * formats here); every encode is a nearest-value search over the format's
 * own table of values with an explicit tie rule; fp32 steps are written as
 * single fp32 operations (IEEE binary32, round-to-nearest, gradual underflow),
 * so the file must be built without fast-math and without FMA contraction.
 *
 * Layouts (row-major, dense, batch-major):
 *   bf16 input           x[b][r][c]            (uint16 bit patterns)
 *   e4m3 codes           q[b][r][c]            (uint8)
 *   e2m1 codes, packed   q[b][r][c/2]          (element 2i in bits 0..3,
 *                                               element 2i+1 in bits 4..7)
 *   MXFP8 scales         s[b][r][c/32]         (uint8 E8M0)
 *   1x128 scales         s[b][r][c/128]        (fp32, dequant multiplier)
 *   128x128 scales       s[b][ceil(r/128)][c/128]  (fp32, dequant multiplier)
 *   NVFP4 block scales   s[b][r][c/16]         (uint8 E4M3), g[b] fp32
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* bf16 / fp32 helpers                                                       */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the top half of an fp32 pattern, so decoding is exact. */
ORC_API double orc_bf16_decode(uint16_t b) { return (double)f32_from_bits((uint32_t)b << 16); }

/* Round an fp32 value to the nearest bf16, ties to the even pattern.
 * The two candidates are the bf16 values that bracket v (truncation toward
 * zero and the next pattern away from zero); both differences are exact in
 * fp64 because all three numbers are fp32 values. */
ORC_API uint16_t orc_bf16_encode(float v)
{
    uint32_t u = bits_from_f32(v);
    if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040u);   /* quiet NaN */
    if (isinf(v)) return (uint16_t)(u >> 16);
    uint16_t lo = (uint16_t)(u >> 16);                        /* toward zero */
    uint16_t hi = (uint16_t)(lo + 1);                         /* away from zero */
    double a = fabs((double)v);
    double vlo = fabs(orc_bf16_decode(lo));
    /* past the largest finite bf16 the next value is 2^128, as if the
     * exponent were unbounded (IEEE overflow rule); that pattern is inf */
    double vhi = ((hi & 0x7F80u) == 0x7F80u) ? ldexp(1.0, 128) : fabs(orc_bf16_decode(hi));
    if (a == vlo) return lo;
    double dlo = a - vlo, dhi = vhi - a;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1u) ? hi : lo;                               /* tie: even */
}

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP "E4M3", a.k.a. float8_e4m3fn): 1 sign, 4 exponent (bias 7),    */
/* 3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite 448.    */
/* ------------------------------------------------------------------------ */

ORC_API double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m / 8.0, -6)          /* subnormal */
                          : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Non-negative finite codes 0x00..0x7E, in increasing order of value (the
 * code order of a sign-magnitude float equals its value order). */
static double e4m3_pos[127];
static int e4m3_ready = 0;
static void e4m3_init(void)
{
    if (e4m3_ready) return;
    for (int c = 0; c < 127; ++c) e4m3_pos[c] = orc_e4m3_decode((uint8_t)c);
    e4m3_ready = 1;
}

/* Nearest E4M3 code to v: NaN -> 0x7F; |v| >= 448 (incl. inf) -> +-448;
 * otherwise the nearest finite code, a tie going to the even code (even
 * mantissa).  The sign is kept, so a negative value that rounds to zero
 * encodes as 0x80. */
ORC_API uint8_t orc_e4m3_encode(double v)
{
    e4m3_init();
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* largest code whose value is <= a (binary search over the table) */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (e4m3_pos[mid] <= a) lo = mid; else hi = mid - 1;
    }
    int c = lo;
    if (e4m3_pos[c] == a) return (uint8_t)(sign | c);
    double midpoint = (e4m3_pos[c] + e4m3_pos[c + 1]) / 2.0;   /* exact */
    int pick;
    if (a < midpoint) pick = c;
    else if (a > midpoint) pick = c + 1;
    else pick = (c % 2 == 0) ? c : c + 1;
    return (uint8_t)(sign | pick);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (OCP "E2M1"): 1 sign, 2 exponent (bias 1), 1 mantissa bit.           */
/* Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no NaN or infinity.                 */
/* ------------------------------------------------------------------------ */

ORC_API double orc_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 code (4 bits): |v| >= 6 -> +-6, ties to the even code; the
 * sign is kept (a negative value that rounds to zero gives 0x8). */
ORC_API uint8_t orc_e2m1_encode(double v)
{
    static const double pos[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs(v);
    if (isnan(v)) return 0x7;          /* outside the contract: no NaN code */
    if (a >= 6.0) return (uint8_t)(sign | 7);
    int c = 0;
    while (c < 7 && pos[c + 1] <= a) ++c;
    if (pos[c] == a) return (uint8_t)(sign | c);
    double midpoint = (pos[c] + pos[c + 1]) / 2.0;
    int pick;
    if (a < midpoint) pick = c;
    else if (a > midpoint) pick = c + 1;
    else pick = (c % 2 == 0) ? c : c + 1;
    return (uint8_t)(sign | pick);
}

/* ------------------------------------------------------------------------ */
/* E8M0 (OCP "E8M0"): an unsigned power of two 2^(c-127), c in 0..254;      */
/* c = 0xFF is NaN.                                                          */
/* ------------------------------------------------------------------------ */

ORC_API double orc_e8m0_decode(uint8_t c)
{
    if (c == 0xFF) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* The MXFP8 block exponent: e = ceil(log2(amax / 448)), i.e. the smallest
 * integer with 448 * 2^e >= amax (so no element of the block exceeds the
 * E4M3 range after division by 2^e), clamped to [-127, 127].  amax = 0 gives
 * -127 (the clamp of -infinity).  NaN amax returns 128 (code 0xFF). */
ORC_API int orc_mx_block_exponent(double amax)
{
    if (isnan(amax)) return 128;
    for (int e = -127; e <= 127; ++e)
        if (ldexp(448.0, e) >= amax) return e;
    return 127;
}

/* ------------------------------------------------------------------------ */
/* Block quantizers.  All return scales as dequantization multipliers: the   */
/* decoded element times its scale approximates the input ("scale inverse"). */
/* ------------------------------------------------------------------------ */

static double absmax_row_span(const uint16_t* x, int64_t n)
{
    double m = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double a = fabs(orc_bf16_decode(x[i]));
        if (isnan(a)) return NAN;
        if (a > m) m = a;
    }
    return m;
}

/* MXFP8: blocks of 32 consecutive elements of a row.  Per block:
 *   e = clamp(ceil(log2(amax/448)), -127, 127), scale code c = e + 127,
 *   q_i = E4M3(x_i * 2^-e), the product formed exactly in fp64. */
ORC_API void orc_quant_mxfp8(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                             uint8_t* q, uint8_t* scales)
{
    const int64_t nb = cols / 32;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t r = 0; r < rows; ++r) {
            const uint16_t* xr = x + (b * rows + r) * cols;
            uint8_t* qr = q + (b * rows + r) * cols;
            uint8_t* sr = scales + (b * rows + r) * nb;
            for (int64_t j = 0; j < nb; ++j) {
                double amax = absmax_row_span(xr + 32 * j, 32);
                int e = orc_mx_block_exponent(amax);
                sr[j] = (uint8_t)(e + 127);
                for (int i = 0; i < 32; ++i) {
                    double v = orc_bf16_decode(xr[32 * j + i]);
                    qr[32 * j + i] = (e == 128) ? 0x7F : orc_e4m3_encode(ldexp(v, -e));
                }
            }
        }
}

/* fp32 scale of one block: s = fp32(amax / 448), or 1 for an all-zero block.
 * q = E4M3(fp32(x / s)): a correctly rounded fp32 division, then the E4M3
 * rounding of that fp32 quotient. */
static float fp32_block_scale(double amax)
{
    if (amax == 0.0) return 1.0f;
    float a = (float)amax;             /* amax is a bf16 value: exact */
    return a / 448.0f;                 /* one IEEE binary32 division */
}

static uint8_t e4m3_of_quotient(uint16_t xb, float s)
{
    float xf = (float)orc_bf16_decode(xb);
    float t = xf / s;                  /* one IEEE binary32 division */
    return orc_e4m3_encode((double)t);
}

/* 1x128 tiles along each row (per-token, per-128-channel). */
ORC_API void orc_quant_fp8_1x128(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                                 uint8_t* q, float* scales)
{
    const int64_t nb = cols / 128;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t r = 0; r < rows; ++r) {
            const uint16_t* xr = x + (b * rows + r) * cols;
            uint8_t* qr = q + (b * rows + r) * cols;
            float* sr = scales + (b * rows + r) * nb;
            for (int64_t j = 0; j < nb; ++j) {
                float s = fp32_block_scale(absmax_row_span(xr + 128 * j, 128));
                sr[j] = s;
                for (int i = 0; i < 128; ++i) qr[128 * j + i] = e4m3_of_quotient(xr[128 * j + i], s);
            }
        }
}

/* 128x128 blocks: rows [128i, 128i+128) x cols [128j, 128j+128); the last
 * block row may be shorter when rows is not a multiple of 128. */
ORC_API void orc_quant_fp8_128x128(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                                   uint8_t* q, float* scales)
{
    const int64_t nbr = (rows + 127) / 128, nbc = cols / 128;
    for (int64_t b = 0; b < batch; ++b) {
        const uint16_t* xb = x + b * rows * cols;
        uint8_t* qb = q + b * rows * cols;
        float* sb = scales + b * nbr * nbc;
        for (int64_t bi = 0; bi < nbr; ++bi)
            for (int64_t bj = 0; bj < nbc; ++bj) {
                int64_t r0 = 128 * bi, r1 = r0 + 128 < rows ? r0 + 128 : rows;
                double amax = 0.0;
                for (int64_t r = r0; r < r1; ++r) {
                    double m = absmax_row_span(xb + r * cols + 128 * bj, 128);
                    if (isnan(m) || m > amax) amax = m;
                    if (isnan(amax)) break;
                }
                float s = fp32_block_scale(amax);
                sb[bi * nbc + bj] = s;
                for (int64_t r = r0; r < r1; ++r)
                    for (int i = 0; i < 128; ++i)
                        qb[r * cols + 128 * bj + i] = e4m3_of_quotient(xb[r * cols + 128 * bj + i], s);
            }
    }
}

/* NVFP4: two-level scaling.
 *   g   = fp32(amax_T / (6 * 448))  per tensor (1 for an all-zero tensor);
 *   s_b = E4M3(fp32(fp32(amax_b / 6) / g))  per 16 consecutive elements;
 *   S   = fp32(dec(s_b) * g)        the block's effective dequant scale;
 *   q_i = E2M1(fp32(x_i / S)), or 0 for every element when S = 0. */
ORC_API float orc_nvfp4_tensor_scale(const uint16_t* x, int64_t n)
{
    double amax = absmax_row_span(x, n);
    if (amax == 0.0) return 1.0f;
    return (float)amax / 2688.0f;
}

ORC_API void orc_quant_nvfp4(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                             uint8_t* q, uint8_t* scales, float* g_out)
{
    const int64_t nb = cols / 16;
    for (int64_t b = 0; b < batch; ++b) {
        const uint16_t* xb = x + b * rows * cols;
        float g = orc_nvfp4_tensor_scale(xb, rows * cols);
        g_out[b] = g;
        for (int64_t r = 0; r < rows; ++r) {
            const uint16_t* xr = xb + r * cols;
            uint8_t* qr = q + (b * rows + r) * (cols / 2);
            uint8_t* sr = scales + (b * rows + r) * nb;
            for (int64_t j = 0; j < nb; ++j) {
                float amax_b = (float)absmax_row_span(xr + 16 * j, 16);
                float t = amax_b / 6.0f;
                uint8_t sc = orc_e4m3_encode((double)(t / g));
                sr[j] = sc;
                float S = (float)(orc_e4m3_decode(sc) * (double)g);   /* exact product, one rounding */
                for (int i = 0; i < 16; i += 2) {
                    uint8_t c[2];
                    for (int h = 0; h < 2; ++h) {
                        float xf = (float)orc_bf16_decode(xr[16 * j + i + h]);
                        c[h] = (S == 0.0f) ? 0 : orc_e2m1_encode((double)(xf / S));
                    }
                    qr[(16 * j + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Dequantizers: out = bf16(fp32(dec(q) * s)).  The product of a decoded     */
/* element and an fp32 (or power-of-two) scale is exact in fp64; it is then  */
/* rounded once to fp32 and once more to bf16, as two explicit steps.        */
/* ------------------------------------------------------------------------ */

static uint16_t deq_elem(double d, double s)
{
    float p = (float)(d * s);
    return orc_bf16_encode(p);
}

ORC_API void orc_dequant_mxfp8(const uint8_t* q, const uint8_t* scales, int64_t batch,
                               int64_t rows, int64_t cols, uint16_t* out)
{
    const int64_t nb = cols / 32;
    for (int64_t br = 0; br < batch * rows; ++br)
        for (int64_t c = 0; c < cols; ++c)
            out[br * cols + c] = deq_elem(orc_e4m3_decode(q[br * cols + c]),
                                          orc_e8m0_decode(scales[br * nb + c / 32]));
}

ORC_API void orc_dequant_fp8_1x128(const uint8_t* q, const float* scales, int64_t batch,
                                   int64_t rows, int64_t cols, uint16_t* out)
{
    const int64_t nb = cols / 128;
    for (int64_t br = 0; br < batch * rows; ++br)
        for (int64_t c = 0; c < cols; ++c)
            out[br * cols + c] = deq_elem(orc_e4m3_decode(q[br * cols + c]),
                                          (double)scales[br * nb + c / 128]);
}

ORC_API void orc_dequant_fp8_128x128(const uint8_t* q, const float* scales, int64_t batch,
                                     int64_t rows, int64_t cols, uint16_t* out)
{
    const int64_t nbr = (rows + 127) / 128, nbc = cols / 128;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                int64_t i = (b * rows + r) * cols + c;
                out[i] = deq_elem(orc_e4m3_decode(q[i]),
                                  (double)scales[b * nbr * nbc + (r / 128) * nbc + c / 128]);
            }
}

ORC_API void orc_dequant_nvfp4(const uint8_t* q, const uint8_t* scales, const float* g,
                               int64_t batch, int64_t rows, int64_t cols, uint16_t* out)
{
    const int64_t nb = cols / 16;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                int64_t br = b * rows + r;
                float S = (float)(orc_e4m3_decode(scales[br * nb + c / 16]) * (double)g[b]);
                uint8_t byte = q[br * (cols / 2) + c / 2];
                uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                out[br * cols + c] = deq_elem(orc_e2m1_decode(code), (double)S);
            }
}

/* ------------------------------------------------------------------------ */
/* LoRA merge for the QAT forward:                                           */
/*   delta[n,k] = sum_{j=0}^{r-1} B[n,j] * A[j,k]   in fp32, one fused       */
/*                multiply-add per term, j ascending, starting from 0;       */
/*   W_eff[n,k] = bf16(fp32 fma(alpha_over_r, delta[n,k], W[n,k])).          */
/* W is [n, k] (output features x input features), A is [r, k], B is [n, r], */
/* all bf16.  The merged weight is then quantized with 128x128 blocks.       */
/* ------------------------------------------------------------------------ */

ORC_API void orc_lora_merge(const uint16_t* w, const uint16_t* lora_a, const uint16_t* lora_b,
                            int64_t n, int64_t k, int32_t r, float alpha_over_r, uint16_t* w_eff)
{
    for (int64_t i = 0; i < n; ++i)
        for (int64_t c = 0; c < k; ++c) {
            float delta = 0.0f;
            for (int32_t j = 0; j < r; ++j)
                delta = fmaf((float)orc_bf16_decode(lora_b[i * r + j]),
                             (float)orc_bf16_decode(lora_a[(int64_t)j * k + c]), delta);
            float merged = fmaf(alpha_over_r, delta, (float)orc_bf16_decode(w[i * k + c]));
            w_eff[i * k + c] = orc_bf16_encode(merged);
        }
}

/* ------------------------------------------------------------------------ */
/* GEMM reference: C[m,n] = sum_k deqA[m,k] * deqB[n,k] in fp64, k ascending,*/
/* where deq = dec(q) * s taken exactly (no rounding of the dequantized      */
/* operand).  A is [M, K], B is [N, K] (C = A * B^T).                         */
/* ------------------------------------------------------------------------ */

/* operand formats understood by the GEMM reference */
enum { ORC_FMT_1x128 = 0, ORC_FMT_128x128 = 1, ORC_FMT_MXFP8 = 2, ORC_FMT_NVFP4 = 3 };

/* exact dequantized value of element (row, col) of a quantized operand with
 * `rows` rows (the row count matters only for the 128x128 scale grid) */
static double deq_value(int fmt, const uint8_t* q, const void* s, const float* g,
                        int64_t rows, int64_t cols, int64_t row, int64_t col)
{
    switch (fmt) {
    case ORC_FMT_1x128:
        return orc_e4m3_decode(q[row * cols + col]) *
               (double)((const float*)s)[row * (cols / 128) + col / 128];
    case ORC_FMT_128x128:
        (void)rows;
        return orc_e4m3_decode(q[row * cols + col]) *
               (double)((const float*)s)[(row / 128) * (cols / 128) + col / 128];
    case ORC_FMT_MXFP8:
        return orc_e4m3_decode(q[row * cols + col]) *
               orc_e8m0_decode(((const uint8_t*)s)[row * (cols / 32) + col / 32]);
    case ORC_FMT_NVFP4: {
        uint8_t byte = q[row * (cols / 2) + col / 2];
        uint8_t code = (col % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        double sb = orc_e4m3_decode(((const uint8_t*)s)[row * (cols / 16) + col / 16]);
        return orc_e2m1_decode(code) * sb * (double)g[0];
    }
    }
    return NAN;
}

/* One output entry. */
ORC_API double orc_gemm_entry(int fmt_a, const uint8_t* aq, const void* as, const float* ag,
                              int fmt_b, const uint8_t* bq, const void* bs, const float* bg,
                              int64_t m, int64_t n, int64_t k, int64_t row, int64_t col)
{
    double acc = 0.0;
    for (int64_t kk = 0; kk < k; ++kk)
        acc += deq_value(fmt_a, aq, as, ag, m, k, row, kk) *
               deq_value(fmt_b, bq, bs, bg, n, k, col, kk);
    return acc;
}

/* A list of entries (row_idx[i], col_idx[i]). */
ORC_API void orc_gemm_entries(int fmt_a, const uint8_t* aq, const void* as, const float* ag,
                              int fmt_b, const uint8_t* bq, const void* bs, const float* bg,
                              int64_t m, int64_t n, int64_t k,
                              const int64_t* row_idx, const int64_t* col_idx, int64_t count,
                              double* out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = orc_gemm_entry(fmt_a, aq, as, ag, fmt_b, bq, bs, bg, m, n, k, row_idx[i], col_idx[i]);
}

/* The full M x N product. */
ORC_API void orc_gemm_full(int fmt_a, const uint8_t* aq, const void* as, const float* ag,
                           int fmt_b, const uint8_t* bq, const void* bs, const float* bg,
                           int64_t m, int64_t n, int64_t k, double* out)
{
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j)
            out[i * n + j] = orc_gemm_entry(fmt_a, aq, as, ag, fmt_b, bq, bs, bg, m, n, k, i, j);
}

/* Grouped (per-expert) product: rows [off[e], off[e+1]) of A use expert e's
 * weight B_e = B[e] ([N, K], scales [N, K/32] for MXFP8).  Entry version. */
ORC_API void orc_grouped_gemm_entries(int fmt, const uint8_t* aq, const void* as,
                                      const uint8_t* bq, const void* bs,
                                      const int32_t* offsets, int32_t groups,
                                      int64_t total_m, int64_t n, int64_t k,
                                      const int64_t* row_idx, const int64_t* col_idx, int64_t count,
                                      double* out)
{
    int64_t sbytes = (fmt == ORC_FMT_MXFP8) ? (int64_t)sizeof(uint8_t) * (k / 32)
                                            : (int64_t)sizeof(float) * (k / 128);
    for (int64_t i = 0; i < count; ++i) {
        int64_t row = row_idx[i];
        int32_t e = 0;
        while (e < groups && !(row >= offsets[e] && row < offsets[e + 1])) ++e;
        if (e == groups) { out[i] = NAN; continue; }
        const uint8_t* be = bq + (int64_t)e * n * k;
        const uint8_t* bse = (const uint8_t*)bs + (int64_t)e * n * sbytes;
        out[i] = orc_gemm_entry(fmt, aq, as, 0, fmt, be, bse, 0, total_m, n, k, row, col_idx[i]);
    }
}

/* ------------------------------------------------------------------------ */
/* QAT backward with the straight-through estimator ("DeepSeek R1 and V3 get */
/* quantization-aware fine-tuning on Fireworks", Synopsis and Interpretation: */
/* LoRA adapters trained through the FP8-quantized forward, base weight      */
/* frozen).  For y = fq(x) fq(W_eff)^T, W_eff = W + (alpha/r) B A, the        */
/* fake-quantizers pass gradients unchanged:                                  */
/*   dx = dy Wfq, dw = dy^T Xfq, da = (alpha/r) B^T bf16(dw),                 */
/*   db = (alpha/r) bf16(dw) A^T.                                             */
/* The building block is one product entry of bf16 operands, C[i][j] =       */
/* alpha * sum_t P[i][t] Q[j][t] (both operands row-major with the summed    */
/* index last), summed in fp64 with t ascending (every product of two bf16   */
/* values is exact in fp64).                                                  */
/* ------------------------------------------------------------------------ */

static double bf16_dot(const uint16_t* p, const uint16_t* q, int64_t k)
{
    double s = 0.0;
    for (int64_t t = 0; t < k; ++t) s += orc_bf16_decode(p[t]) * orc_bf16_decode(q[t]);
    return s;
}

ORC_API void orc_gemm_bf16_entries(const uint16_t* p, const uint16_t* q, int64_t k, double alpha,
                                   const int64_t* row_idx, const int64_t* col_idx, int64_t count, double* out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = alpha * bf16_dot(p + row_idx[i] * k, q + col_idx[i] * k, k);
}

ORC_API void orc_gemm_bf16_full(const uint16_t* p, const uint16_t* q, int64_t m, int64_t n, int64_t k,
                                double alpha, double* out)
{
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) out[i * n + j] = alpha * bf16_dot(p + i * k, q + j * k, k);
}

/* bf16 rounding (nearest, ties to even) of an fp64 value: the fp32 step is
 * exact for every value the products above can produce only up to fp32
 * precision, so the rounding is done from the two bf16 neighbours of the
 * fp64 value directly. */
ORC_API uint16_t orc_bf16_encode_f64(double v)
{
    if (isnan(v)) return 0x7FC0u;
    float f = (float)v;                                /* nearest fp32 */
    uint16_t c = orc_bf16_encode(f);
    if ((double)f == v || isinf(f)) return c;
    /* the fp32 rounding may have moved v onto a bf16 midpoint: decide the
     * two bf16 candidates around v in fp64 */
    uint32_t u = bits_from_f32(f);
    uint16_t lo = (uint16_t)(u >> 16), hi = (uint16_t)(lo + 1);
    double a = fabs(v), vlo = fabs(orc_bf16_decode(lo));
    if (vlo > a) { hi = lo; lo = (uint16_t)(lo - 1); vlo = fabs(orc_bf16_decode(lo)); }
    double vhi = ((hi & 0x7F80u) == 0x7F80u) ? ldexp(1.0, 128) : fabs(orc_bf16_decode(hi));
    double dlo = a - vlo, dhi = vhi - a;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo & 1u) ? hi : lo;
}

ORC_API void orc_bf16_encode_f64_array(const double* x, int64_t count, uint16_t* out)
{
    for (int64_t i = 0; i < count; ++i) out[i] = orc_bf16_encode_f64(x[i]);
}
