/*
 * q4_oracle.c -- plain, slow, scalar CPU oracle for 4-bit block-scaled
 * quantization, first-order Sigma-Delta requantization and the W4A4 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity reference that the CUDA
 * path is checked against.  Only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark load it.  The product library never links,
 * calls or falls back to it, and it shares no code, header, table or constant
 * generator with the CUDA sources.
 *
 * Arithmetic rules: every floating-point step is a single IEEE-754 binary32
 * operation in round-to-nearest-even, in the order written, compiled with
 * -ffp-contract=off and without fast-math (x86-64 SSE arithmetic).  The GEMM is
 * a triple loop in binary64 over exactly decoded operands.  Codecs are written
 * as brute-force searches over every code, so that "nearest" is checked by eye.
 *
 * Sources (web pages, cited by title and section):
 *  [LT]  "Looped Transformer quantization: error propagation, NVFP4 and
 *        Sigma-Delta modulation" (mer.dev/posts/loopquant-fp4):
 *        sec. 0.2 (NVFP4 precision split: E2M1 grid, two-level scaling),
 *        sec. 2.1 (first-order Sigma-Delta recursion), sec. 2.2 (residue bound,
 *        4/6 block scale rounded up, s_tensor = max|W|/(6*256)), sec. 2.5
 *        (implementation details: block_scale_46, x = W/s, r = 0, v = x + r,
 *        q = e2m1_round(v), r = v - q).
 *  [GDN] "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the
 *        Recurrent Half of a Hybrid 27B LLM", prerequisites "NVFP4 and W4A4
 *        quantization" (16-element blocks, E4M3 scale = block max / 6, FP32
 *        per-tensor scale, GEMM on native 4-bit tensor cores).
 *  [MQ]  "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision
 *        Weights and Activations", prerequisites "MXFP4 microscaling format"
 *        (B = 32, shared E8M0 power-of-two scale, E2M1 elements) and "basis
 *        transform quantization"; core method steps (i) per-channel balancing
 *        scale and (ii) block Hadamard rotation of size 32, y = [(x.t)B] W'^T.
 *
 * Readings where the pages are silent (each one listed in the design notes):
 *  R1 E2M1 rounding ties go to the code with an even mantissa bit; magnitudes
 *     above 6 (and +-inf) saturate to 6; the sign bit is the sign bit of the
 *     input, so a negative value that rounds to zero gives code 0x8.
 *  R2 NVFP4 block scale: sbf = amax / (6 * s_t), two binary32 operations in
 *     that order, then E4M3 with round-to-nearest-even (mode RN) or round-up
 *     (mode RU, the "rounded up" candidate of [LT] sec. 2.2), saturating at 448.
 *  R3 Elements are normalised as [LT] sec. 2.5 writes it, x = W / s: the
 *     block's decoded scale S = dec(sb) * s_t (one binary32 product), then one
 *     correctly rounded binary32 division v = x / S per element.  If S is 0,
 *     or its reciprocal 1 / S overflows binary32, or s_t is not a positive
 *     finite number, the block is degenerate and its normalised values are
 *     taken as +0.
 *  R4 MXFP4 shared exponent (mode RN): e = floor(log2(amax)) - 2, the OCP rule
 *     (emax of E2M1 is 2), clamped to [-127, 127]; mode RU takes the smallest e
 *     with amax <= 6 * 2^e, so that nothing saturates (needed by Sigma-Delta).
 *     amax = 0 gives byte 0x00.
 *  R5 Optional MXFP4 transforms in this order: y = x * c (binary32), then the
 *     unnormalised Walsh-Hadamard butterflies over each 32-block in Sylvester
 *     order (strides 1, 2, 4, 8, 16; (a, b) -> (a + b, a - b)), then a
 *     multiplication by binary32(1/sqrt(32)).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define Q4O_NVFP4 0
#define Q4O_MXFP4 1

/* ------------------------------------------------------------------------ */
/* E2M1 element code ([LT] sec. 0.2; [GDN] prerequisites; [MQ] MXFP4 format) */
/* 1 sign bit, 2 exponent bits, 1 mantissa bit.  Positive magnitudes, in code */
/* order 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.                                   */
/* ------------------------------------------------------------------------ */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double q4o_e2m1_decode(uint8_t code)
{
    double m = E2M1_MAG[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Nearest magnitude by exhaustive search (R1).  Two grid points can only tie
 * when they are neighbours, and neighbours differ in mantissa parity, so "on a
 * tie take the even code" picks the even-mantissa neighbour. */
uint8_t q4o_e2m1_encode(float v)
{
    int neg = signbit(v) ? 1 : 0;
    double a = fabs((double)v);
    int best = 0;
    if (!(a <= 6.0)) {            /* > 6, +inf: saturate */
        best = 7;
    } else {
        double bestd = a;
        for (int c = 1; c < 8; ++c) {
            double d = fabs(a - E2M1_MAG[c]);
            if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
        }
    }
    return (uint8_t)((neg << 3) | best);
}

/* ------------------------------------------------------------------------ */
/* E4M3 (finite-only "fn" variant): bias 7, no infinities, 0x7F/0xFF NaN,    */
/* largest finite 448, subnormals down to 2^-9.  Block-scale type of NVFP4.  */
/* ------------------------------------------------------------------------ */
double q4o_e4m3_decode(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);            /* m/8 * 2^-6 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Encode a non-negative binary32 scale (R2).  round_up = 0: nearest, ties to
 * even code; round_up = 1: smallest code whose value is >= v.  Both saturate
 * at 448 (code 0x7E); v <= 0 gives 0x00. */
uint8_t q4o_e4m3_encode(float v, int round_up)
{
    double a = (double)v;
    if (!(a > 0.0)) return 0x00;
    if (!(a < 448.0)) return 0x7E;
    int best = 0;
    if (round_up) {
        for (int c = 0; c <= 0x7E; ++c)
            if (q4o_e4m3_decode((uint8_t)c) >= a) { best = c; break; }
    } else {
        double bestd = a;
        for (int c = 1; c <= 0x7E; ++c) {
            double d = fabs(a - q4o_e4m3_decode((uint8_t)c));
            if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* E8M0: unsigned power-of-two scale, value 2^(byte - 127), 0xFF is NaN.     */
/* ([MQ] prerequisites, MXFP4 microscaling format.)                          */
/* ------------------------------------------------------------------------ */
double q4o_e8m0_decode(uint8_t b)
{
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* Shared exponent of a 32-block (R4).  Returns e; the stored byte is e+127. */
int q4o_mx_exponent(float amax, int round_up)
{
    if (!(amax > 0.0f)) return -127;
    int ex;
    (void)frexpf(amax, &ex);          /* amax = f * 2^ex, f in [0.5, 1) */
    int e = (ex - 1) - 2;             /* floor(log2 amax) - emax(E2M1)  */
    if (round_up && ldexp((double)amax, -e) > 6.0) e += 1;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* ------------------------------------------------------------------------ */
/* Tensor amax and per-tensor FP32 scale ([LT] sec. 2.2: s_tensor =         */
/* max|W| / (6*256) for looped weights; the activation recipe uses           */
/* amax / (6*448)).  denom is the product written as one binary32 constant.  */
/* ------------------------------------------------------------------------ */
float q4o_amax(const float* x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

float q4o_tensor_scale(float amax, float denom)
{
    return amax / denom;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 two-level block quantization ([LT] sec. 0.2; [GDN] prerequisites): */
/* 16 contiguous elements along a row share one E4M3 scale of about block    */
/* max / 6, under the FP32 tensor scale s_t.  Codes are packed two per byte, */
/* element 2i in the low nibble.  Scales are written row-major [rows, cols/16]. */
/* Returns 0, or -1 for an invalid shape.                                    */
/* ------------------------------------------------------------------------ */
static int block_is_degenerate(float S, float s_t)
{
    return !(s_t > 0.0f) || !isfinite(s_t) || S == 0.0f || !isfinite(1.0f / S);
}

int q4o_nvfp4_quantize(const float* x, int64_t rows, int64_t cols, float s_t,
                       int round_up, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0) return -1;
    const int64_t nb = cols / 16;
    for (int64_t i = 0; i < rows; ++i) {
        const float* xr = x + i * cols;
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = xr + b * 16;
            float amax = 0.0f;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(xb[j]);
                if (a > amax) amax = a;
            }
            uint8_t sb = 0;
            if (s_t > 0.0f && isfinite(s_t)) {
                float denom = 6.0f * s_t;              /* R2, first op  */
                float sbf = amax / denom;              /* R2, second op */
                sb = q4o_e4m3_encode(sbf, round_up);
            }
            float S = (float)q4o_e4m3_decode(sb) * s_t;  /* R3 */
            int degenerate = block_is_degenerate(S, s_t);
            scales[i * nb + b] = sb;
            for (int j = 0; j < 16; ++j) {
                float v = degenerate ? 0.0f : xb[j] / S;
                uint8_t c = q4o_e2m1_encode(v);
                int64_t k = b * 16 + j;
                uint8_t* dst = codes + i * (cols / 2) + k / 2;
                if ((k & 1) == 0) *dst = (uint8_t)((*dst & 0xF0u) | c);
                else *dst = (uint8_t)((*dst & 0x0Fu) | (uint8_t)(c << 4));
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 32-point Walsh-Hadamard transform, Sylvester order, unnormalised (R5).    */
/* ([MQ] basis transform quantization; step (ii) block Hadamard of size 32.) */
/* ------------------------------------------------------------------------ */
void q4o_fwht32(float* v)
{
    for (int h = 1; h < 32; h *= 2) {
        for (int i = 0; i < 32; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4 block quantization ([MQ] MXFP4 format; core method (i), (ii)):      */
/* per 32-block, optional per-channel multiplier c (t for activations, 1/t   */
/* for weights), optional block Hadamard, shared E8M0 exponent (R4), E2M1.   */
/* Scales row-major [rows, cols/32] as E8M0 bytes.                           */
/* ------------------------------------------------------------------------ */
/* Transform one 32-block before quantization (R5): y = x * c, then the
 * normalised block Hadamard.  chan points at the block's 32 multipliers or is
 * NULL; hadamard = 0 skips the rotation. */
void q4o_mx_transform(const float* x, const float* chan, int hadamard, float* y)
{
    const float inv_sqrt32 = (float)(1.0 / sqrt(32.0));   /* binary32 RN */
    for (int j = 0; j < 32; ++j) y[j] = chan ? x[j] * chan[j] : x[j];
    if (hadamard) {
        q4o_fwht32(y);
        for (int j = 0; j < 32; ++j) y[j] = y[j] * inv_sqrt32;
    }
}

int q4o_mxfp4_quantize(const float* x, int64_t rows, int64_t cols,
                       const float* chan, int hadamard, int round_up,
                       uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0) return -1;
    const int64_t nb = cols / 32;
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t b = 0; b < nb; ++b) {
            float y[32];
            q4o_mx_transform(x + i * cols + b * 32, chan ? chan + b * 32 : NULL, hadamard, y);
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                float a = fabsf(y[j]);
                if (a > amax) amax = a;
            }
            int e = q4o_mx_exponent(amax, round_up);
            scales[i * nb + b] = (uint8_t)(e + 127);
            float mult = ldexpf(1.0f, -e);        /* exact power of two */
            for (int j = 0; j < 32; ++j) {
                float v = y[j] * mult;
                uint8_t c = q4o_e2m1_encode(v);
                int64_t k = b * 32 + j;
                uint8_t* dst = codes + i * (cols / 2) + k / 2;
                if ((k & 1) == 0) *dst = (uint8_t)((*dst & 0xF0u) | c);
                else *dst = (uint8_t)((*dst & 0x0Fu) | (uint8_t)(c << 4));
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Tensor-core scale-factor layout.  Rows are padded to a multiple of 128    */
/* and scale columns to a multiple of 4.  The padded matrix is cut into      */
/* 128 x 4 atoms of 512 bytes, stored atom-row-major; inside an atom, scale  */
/* (r, c) sits at byte (r % 32) * 16 + (r / 32) * 4 + c.  Padding is zero.    */
/* ------------------------------------------------------------------------ */
int64_t q4o_tc_scale_bytes(int64_t rows, int64_t scols)
{
    int64_t rp = (rows + 127) / 128 * 128;
    int64_t cp = (scols + 3) / 4 * 4;
    return rp * cp;
}

int64_t q4o_tc_scale_offset(int64_t r, int64_t c, int64_t scols)
{
    int64_t catoms = (scols + 3) / 4;
    int64_t atom = (r / 128) * catoms + (c / 4);
    int64_t rr = r % 128, cc = c % 4;
    return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc;
}

void q4o_scales_to_tc(const uint8_t* rowmajor, int64_t rows, int64_t scols, uint8_t* out)
{
    memset(out, 0, (size_t)q4o_tc_scale_bytes(rows, scols));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < scols; ++c)
            out[q4o_tc_scale_offset(r, c, scols)] = rowmajor[r * scols + c];
}

void q4o_scales_from_tc(const uint8_t* tc, int64_t rows, int64_t scols, uint8_t* rowmajor)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < scols; ++c)
            rowmajor[r * scols + c] = tc[q4o_tc_scale_offset(r, c, scols)];
}

/* ------------------------------------------------------------------------ */
/* Decoded value of one element: code * block scale (* tensor scale).       */
/* ------------------------------------------------------------------------ */
static double block_scale_value(int format, uint8_t sb)
{
    return format == Q4O_NVFP4 ? q4o_e4m3_decode(sb) : q4o_e8m0_decode(sb);
}

static uint8_t code_at(const uint8_t* codes, int64_t cols, int64_t i, int64_t k)
{
    uint8_t byte = codes[i * (cols / 2) + k / 2];
    return (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0x0F);
}

/* Fake quantization ([GDN] quantize-then-dequantize): out = code * s_b * s_t
 * in binary64 (exact).  s_t is ignored for MXFP4. */
int q4o_dequantize(int format, const uint8_t* codes, const uint8_t* scales,
                   float s_t, int64_t rows, int64_t cols, double* out)
{
    int blk = format == Q4O_NVFP4 ? 16 : 32;
    if (cols % blk != 0) return -1;
    int64_t nb = cols / blk;
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t k = 0; k < cols; ++k) {
            double v = q4o_e2m1_decode(code_at(codes, cols, i, k))
                     * block_scale_value(format, scales[i * nb + k / blk]);
            if (format == Q4O_NVFP4) v *= (double)s_t;
            out[i * cols + k] = v;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* One loop visit of first-order Sigma-Delta requantization ([LT] sec. 2.1  */
/* and the code of sec. 2.5): with the block scale fixed, x = W / s,         */
/* v_k = x + r_{k-1}, q_k = Q(v_k) (nearest E2M1, saturating), r_k = v_k - q_k.*/
/* The caller zeroes r before the first visit (r_0 = 0).  x = w / S, one     */
/* binary32 division (R3).  Scales row-major; s_t ignored for MXFP4.         */
/* ------------------------------------------------------------------------ */
int q4o_sigma_delta_step(int format, const float* w, int64_t rows, int64_t cols,
                         const uint8_t* scales, float s_t, float* r, uint8_t* codes)
{
    int blk = format == Q4O_NVFP4 ? 16 : 32;
    if (cols % blk != 0) return -1;
    int64_t nb = cols / blk;
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t b = 0; b < nb; ++b) {
            uint8_t sb = scales[i * nb + b];
            float S;
            int degenerate;
            if (format == Q4O_NVFP4) {
                S = (float)q4o_e4m3_decode(sb) * s_t;
                degenerate = block_is_degenerate(S, s_t);
            } else {
                S = ldexpf(1.0f, (int)sb - 127);     /* 2^e, exact */
                degenerate = 0;
            }
            for (int j = 0; j < blk; ++j) {
                int64_t k = b * blk + j;
                int64_t idx = i * cols + k;
                float x = degenerate ? 0.0f : w[idx] / S;
                float v = x + r[idx];
                uint8_t c = q4o_e2m1_encode(v);
                r[idx] = v - (float)q4o_e2m1_decode(c);
                uint8_t* dst = codes + i * (cols / 2) + k / 2;
                if ((k & 1) == 0) *dst = (uint8_t)((*dst & 0xF0u) | c);
                else *dst = (uint8_t)((*dst & 0x0Fu) | (uint8_t)(c << 4));
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* W4A4 GEMM Y = X W^T over decoded operands ([GDN] prerequisites: W4A4 GEMM */
/* on 4-bit operands; [MQ] inference layer y = x_q W_q^T).  Triple loop in   */
/* binary64; alpha = s_tA * s_tB for NVFP4 and 1 for MXFP4.  If row_idx is   */
/* non-NULL only those n_rows rows of Y are computed (Y is n_rows x N).      */
/* ------------------------------------------------------------------------ */
int q4o_gemm(int format, int64_t M, int64_t N, int64_t K,
             const uint8_t* a_codes, const uint8_t* a_scales, float a_st,
             const uint8_t* b_codes, const uint8_t* b_scales, float b_st,
             const int64_t* row_idx, int64_t n_rows, double* y)
{
    int blk = format == Q4O_NVFP4 ? 16 : 32;
    if (K % blk != 0) return -1;
    int64_t nb = K / blk;
    double alpha = format == Q4O_NVFP4 ? (double)a_st * (double)b_st : 1.0;
    int64_t nr = row_idx ? n_rows : M;
    for (int64_t ii = 0; ii < nr; ++ii) {
        int64_t i = row_idx ? row_idx[ii] : ii;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double a = q4o_e2m1_decode(code_at(a_codes, K, i, k))
                         * block_scale_value(format, a_scales[i * nb + k / blk]);
                double b = q4o_e2m1_decode(code_at(b_codes, K, j, k))
                         * block_scale_value(format, b_scales[j * nb + k / blk]);
                acc += a * b;
            }
            y[ii * N + j] = alpha * acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* W4A16 GEMM Y = alpha * X dec(W)^T ([LT] introduction: weight            */
/* Sigma-Delta evaluated in frozen-weight W4A16 forward passes; sec. 0.2:    */
/* BF16 is the compute view of the weights).  X holds the activations as     */
/* binary32 values (exact copies of their bf16 values); W is quantized       */
/* (codes, row-major block scales); dec(W) = code * s_b and alpha = s_t for   */
/* NVFP4, dec(W) = code * 2^e and alpha = 1 for MXFP4.  Triple loop in        */
/* binary64.  If row_idx is non-NULL only those n_rows rows of Y are computed. */
/* ------------------------------------------------------------------------ */
int q4o_gemm_w4a16(int format, int64_t M, int64_t N, int64_t K, const float* x,
                   const uint8_t* b_codes, const uint8_t* b_scales, float b_st,
                   const int64_t* row_idx, int64_t n_rows, double* y)
{
    int blk = format == Q4O_NVFP4 ? 16 : 32;
    if (K % blk != 0) return -1;
    int64_t nb = K / blk;
    double alpha = format == Q4O_NVFP4 ? (double)b_st : 1.0;
    int64_t nr = row_idx ? n_rows : M;
    for (int64_t ii = 0; ii < nr; ++ii) {
        int64_t i = row_idx ? row_idx[ii] : ii;
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double b = q4o_e2m1_decode(code_at(b_codes, K, j, k))
                         * block_scale_value(format, b_scales[j * nb + k / blk]);
                acc += (double)x[i * K + k] * b;
            }
            y[ii * N + j] = alpha * acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and    */
/* Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC 2011): ten rounds  */
/* of two 32x32 -> 64-bit multiplies (multipliers 0xD2511F53, 0xCD9E8D57)     */
/* mixing the four counter words with the two key words, the key bumped by    */
/* the Weyl constants 0x9E3779B9, 0xBB67AE85 after every round.               */
/* ------------------------------------------------------------------------ */
void q4o_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        uint32_t n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Uniform u in [0, 1) of element e at visit `visit`: Philox4x32-10 with     */
/* counter (e/4 low word, e/4 high word, visit, 0) and key (seed low, seed    */
/* high); element e takes output word e % 4, whose top 24 bits give          */
/* u = (word >> 8) * 2^-24 (exact in binary32).                              */
static float sr_uniform(uint64_t seed, uint32_t visit, int64_t e)
{
    uint64_t g = (uint64_t)e >> 2;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), visit, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    q4o_philox4x32_10(ctr, key, out);
    return (float)(out[e & 3] >> 8) * 0x1p-24f;
}

/* Stochastic rounding onto the E2M1 grid ([LT] sec. 2.1: SR draws each code */
/* so that its conditional expectation equals the weight).  For |x| between   */
/* neighbouring magnitudes a <= |x| < b the magnitude is b when               */
/* u < (|x| - a) / (b - a), else a (both operations exact: Sterbenz and a     */
/* power-of-two gap); |x| >= 6 gives 6; the sign bit is x's (R1).            */
static uint8_t sr_e2m1(float x, float u)
{
    float m = fabsf(x);
    int idx;
    if (m >= 6.0f) {
        idx = 7;
    } else {
        int i = 0;
        while (i < 7 && (float)E2M1_MAG[i + 1] <= m) ++i;
        float a = (float)E2M1_MAG[i], b = (float)E2M1_MAG[i + 1];
        float p = (m - a) / (b - a);
        idx = u < p ? i + 1 : i;
    }
    return (uint8_t)((signbit(x) ? 0x8 : 0x0) | idx);
}

/* One stochastic-rounding requant of W at loop visit `visit` ([LT] sec. 2.1  */
/* and sec. 3: the SR baseline of the looped-weight experiments, a fixed       */
/* seed giving one weight trajectory): x = W / S with the fixed block scale    */
/* (R3, degenerate blocks give +0), code = SR(x).  Scales row-major.           */
int q4o_sr_requant(int format, const float* w, int64_t rows, int64_t cols, const uint8_t* scales, float s_t,
                   uint64_t seed, uint32_t visit, uint8_t* codes)
{
    int blk = format == Q4O_NVFP4 ? 16 : 32;
    if (cols % blk != 0) return -1;
    int64_t nb = cols / blk;
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t b = 0; b < nb; ++b) {
            uint8_t sb = scales[i * nb + b];
            float S;
            int degenerate;
            if (format == Q4O_NVFP4) {
                S = (float)q4o_e4m3_decode(sb) * s_t;
                degenerate = block_is_degenerate(S, s_t);
            } else {
                S = ldexpf(1.0f, (int)sb - 127);     /* 2^e, exact */
                degenerate = 0;
            }
            for (int j = 0; j < blk; ++j) {
                int64_t k = b * blk + j;
                int64_t e = i * cols + k;
                float x = degenerate ? 0.0f : w[e] / S;
                uint8_t c = sr_e2m1(x, sr_uniform(seed, visit, e));
                uint8_t* dst = codes + i * (cols / 2) + k / 2;
                if ((k & 1) == 0) *dst = (uint8_t)((*dst & 0xF0u) | c);
                else *dst = (uint8_t)((*dst & 0x0Fu) | (uint8_t)(c << 4));
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 4/6 block scaling ([LT] sec. 2.2 and the block_scale_46 call of sec. 2.5:  */
/* each block's E4M3 scale is a rounded-up candidate that maps the block      */
/* maximum to 6 or to 4; under s_t = max|W| / (6 * 256) either keeps |x| <= 6). */
/* The choice between the two is not given on the page (reading R10): the      */
/* candidate whose quantized block has the smaller sum of squared errors in   */
/* the input's units, err = sum_j (x_j - dec(code_j) * S)^2 accumulated in     */
/* binary64 in element order (x_j - dec * S is exact there); ties go to 6.     */
/* ------------------------------------------------------------------------ */
static void nv46_candidate(const float* xb, float amax, float s_t, float target, uint8_t* sb_out,
                           uint8_t codes_out[16], double* err_out)
{
    uint8_t sb = 0;
    if (s_t > 0.0f && isfinite(s_t)) {
        float denom = target * s_t;
        float sbf = amax / denom;
        sb = q4o_e4m3_encode(sbf, 1);
    }
    float S = (float)q4o_e4m3_decode(sb) * s_t;
    int degenerate = block_is_degenerate(S, s_t);
    double err = 0.0;
    for (int j = 0; j < 16; ++j) {
        float v = degenerate ? 0.0f : xb[j] / S;     /* R3 */
        uint8_t c = q4o_e2m1_encode(v);
        codes_out[j] = c;
        double d = (double)xb[j] - q4o_e2m1_decode(c) * (double)S;
        err = err + d * d;
    }
    *sb_out = sb;
    *err_out = err;
}

int q4o_nvfp4_quantize46(const float* x, int64_t rows, int64_t cols, float s_t, uint8_t* codes, uint8_t* scales)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0) return -1;
    const int64_t nb = cols / 16;
    for (int64_t i = 0; i < rows; ++i) {
        const float* xr = x + i * cols;
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = xr + b * 16;
            float amax = 0.0f;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(xb[j]);
                if (a > amax) amax = a;
            }
            uint8_t sb6, sb4, c6[16], c4[16];
            double e6, e4;
            nv46_candidate(xb, amax, s_t, 6.0f, &sb6, c6, &e6);
            nv46_candidate(xb, amax, s_t, 4.0f, &sb4, c4, &e4);
            const int four = e4 < e6;
            scales[i * nb + b] = four ? sb4 : sb6;
            for (int j = 0; j < 16; ++j) {
                uint8_t c = four ? c4[j] : c6[j];
                int64_t k = b * 16 + j;
                uint8_t* dst = codes + i * (cols / 2) + k / 2;
                if ((k & 1) == 0) *dst = (uint8_t)((*dst & 0xF0u) | c);
                else *dst = (uint8_t)((*dst & 0x0Fu) | (uint8_t)(c << 4));
            }
        }
    }
    return 0;
}
