/*
 * q4.h -- C ABI of libq4: 4-bit block-scaled quantization (NVFP4, MXFP4),
 * first-order Sigma-Delta requantization and the block-scaled W4A4 GEMM on
 * NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 *   - Pointers named d_* and every tensor argument are DEVICE pointers on the
 *     current CUDA device.  The caller owns all memory; the library allocates
 *     nothing persistent and keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it; nothing synchronises
 *     the host except q4_get_device_error().
 *   - Every tensor pointer must be 16-byte aligned.  Matrices are row-major.
 *   - Inputs must be finite (no NaN, no inf); results for non-finite inputs
 *     are unspecified.
 *   - Argument errors are detected on the host before any launch and
 *     returned as a q4_status; no launch happens then.  A CUDA launch error is
 *     returned as Q4_ERR_CUDA (q4_last_error() gives the CUDA message).
 *     Device-side faults of the library's own bounded waits are recorded in a
 *     device error word and reported by q4_get_device_error().
 *
 * Formats (element codes are E2M1: 1 sign, 2 exponent, 1 mantissa bit;
 * magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6):
 *   Q4_NVFP4: blocks of 16 consecutive elements along a row share an E4M3
 *             block scale of about block-max / 6, times one FP32 tensor scale
 *             s_t ("Looped Transformer quantization", sec. 0.2 "NVFP4
 *             precision split"; "Why Gated DeltaNet Survives 4-Bit
 *             Quantization", prerequisites "NVFP4 and W4A4 quantization").
 *   Q4_MXFP4: blocks of 32 share an E8M0 power-of-two scale, no tensor scale
 *             ("MACaQ", prerequisites "MXFP4 microscaling format").
 *
 * Packed codes: [rows, cols/2] bytes, element 2i in the low nibble of byte i
 * of its row, element 2i+1 in the high nibble.
 *
 * Scale layouts (flag bit Q4_LAYOUT_TC):
 *   row-major : [rows, cols/block] bytes.
 *   Q4_LAYOUT_TC (tensor-core layout): rows padded to a multiple of 128,
 *       scale columns to a multiple of 4; the padded matrix is cut into
 *       128 x 4 atoms of 512 bytes stored atom-row-major (all atoms of rows
 *       0..127 first); inside an atom scale (r, c) is byte
 *       (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).  Padding bytes are 0.
 *       This is the layout the GEMM reads.  q4_scale_bytes() gives the size.
 */
#ifndef Q4_H_
#define Q4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { Q4_NVFP4 = 0, Q4_MXFP4 = 1 } q4_format;
typedef enum { Q4_F32 = 0, Q4_BF16 = 1 } q4_dtype;

typedef enum {
    Q4_OK = 0,
    Q4_ERR_ARG = 1,          /* NULL pointer, bad enum, negative size        */
    Q4_ERR_ALIGN = 2,        /* pointer or row stride not 16-byte aligned     */
    Q4_ERR_SHAPE = 3,        /* size not a multiple the operation needs       */
    Q4_ERR_UNSUPPORTED = 4,  /* valid request this build does not implement   */
    Q4_ERR_CUDA = 5,         /* a CUDA call failed (see q4_last_error)        */
    Q4_ERR_TIMEOUT = 6,      /* a bounded device wait ran out                 */
    Q4_ERR_WORKSPACE = 7     /* workspace missing or too small                */
} q4_status;

/* Flag bits for quantize / dequantize / sigma-delta. */
enum {
    Q4_SCALE_RU = 1,     /* round block scales up (NVFP4: E4M3 toward +inf;
                            MXFP4: smallest exponent with block max <= 6*2^e) */
    Q4_LAYOUT_TC = 2,    /* scales in the tensor-core layout (else row-major) */
    Q4_HADAMARD32 = 4,   /* MXFP4 only: block Hadamard-32 before quantizing   */
    Q4_SCALE_46 = 8,     /* NVFP4 only: 4/6 block scaling (see q4_quantize)    */
    Q4_INJECT_STALL = 1 << 16  /* q4_quantize only, for failure-detection tests:
                            every CTA's first input tile is never loaded, so a
                            bounded wait inside the kernel runs out; the codes
                            are then not valid and q4_get_device_error
                            reports Q4_ERR_TIMEOUT (see q4_set_wait_limit)    */
};

/* Kinds of GEMM left operand. */
enum {
    Q4_A_QUANTIZED = 0,  /* a = packed codes [M, K/2], a_scales in TC layout  */
    Q4_A_BF16 = 1,       /* a = bf16 [M, K]; quantized inside the call with
                            the tensor scale *d_a_gscale (NVFP4 only)         */
    Q4_A_BF16_W4A16 = 2  /* a = bf16 [M, K] kept in bf16: W4A16, the weight is
                            dequantized (exactly, to bf16) on the fly         */
};

/* Library version: major * 10000 + minor * 100 + patch. */
Q4_API int q4_version(void);

/* Human-readable name of a status code (static string, never NULL). */
Q4_API const char* q4_status_string(q4_status s);

/* Message of the last CUDA error seen by this thread's calls (static, never NULL). */
Q4_API const char* q4_last_error(void);

/* Bytes of the scale array of a rows x cols tensor in `format` with the given
 * layout flags (only Q4_LAYOUT_TC matters).  0 for invalid sizes. */
Q4_API size_t q4_scale_bytes(q4_format format, int64_t rows, int64_t cols, int flags);

/*
 * q4_amax -- tensor maximum magnitude and FP32 tensor scale.
 *   Computes d_out[0] = max_i |x_i| (exact) and d_out[1] = d_out[0] / denom
 *   (one binary32 division, round-to-nearest).  denom = 6*448 = 2688 gives the
 *   activation tensor scale; 6*256 = 1536 the looped-weight scale of
 *   "Looped Transformer quantization", sec. 2.2 (s_tensor = max|W|/(6*256)).
 *   x: device, n elements of dtype dt, 16-byte aligned.  d_out: device, 2 floats.
 *   n = 0 gives 0 and 0.  denom must be finite and > 0.
 */
Q4_API q4_status q4_amax(q4_dtype dt, const void* x, int64_t n, float denom, float* d_out,
                  void* stream);

/*
 * q4_amax_quantize -- q4_amax followed by the NVFP4 q4_quantize, in one launch.
 *   d_out[0] = amax = max|x| over the rows x cols matrix, d_out[1] = s_t =
 *   amax / denom (one binary32 division), and codes/scales exactly as
 *   q4_quantize(Q4_NVFP4, 16, ...) with that s_t ("Why Gated DeltaNet Survives
 *   4-Bit Quantization", prerequisites: block scales under an FP32 per-tensor
 *   scale taken from the tensor's maximum).  The launch is cooperative: every
 *   CTA folds its share of |x| into out[0], waits (bounded) at a grid-wide
 *   barrier counted in d_out[2], then quantizes; X is read a second time
 *   while still largely in L2, so HBM sees it about once.
 *   d_out: device, 4 floats (the last two are the launch's own scratch and
 *   are cleared by it); 4-byte aligned.  flags: Q4_LAYOUT_TC, Q4_SCALE_RU.
 *   Other arguments and requirements as q4_quantize.  rows or cols = 0 gives
 *   d_out = {0, 0, 0, 0}.  A barrier wait that runs out is reported by
 *   q4_get_device_error as Q4_ERR_TIMEOUT (codes then not valid).
 */
Q4_API q4_status q4_amax_quantize(q4_dtype in_dt, const void* x, int64_t rows, int64_t cols, int64_t ld,
                                  float denom, float* d_out, uint8_t* codes, uint8_t* scales, int flags,
                                  void* stream);

/*
 * q4_quantize -- block quantization of a rows x cols matrix.
 *   NVFP4 ("Looped Transformer quantization", sec. 0.2; "Why Gated DeltaNet
 *   Survives 4-Bit Quantization", prerequisites): per 16-block,
 *     amax = max|x|,  s_b = E4M3(amax / (6 * s_t))   [RN, or RU with Q4_SCALE_RU],
 *     S = s_b * s_t,  code_i = E2M1(x_i / S)  (one correctly rounded binary32
 *     division, as "Looped Transformer quantization", sec. 2.5 writes x = W / s;
 *     E2M1 rounding to nearest, ties to
 *     even mantissa, saturating at +-6, sign kept for values that round to 0);
 *     a block whose S is 0 or whose reciprocal 1 / S overflows, and every block when s_t
 *     is not a positive finite number, gets code 0.
 *   MXFP4 ("MACaQ", prerequisites "MXFP4 microscaling format" and core method
 *   steps (i)-(ii), y = [(x . t) B]_MXFP4): per 32-block,
 *     y_j = x_j * c_j (if d_chan), then if Q4_HADAMARD32 the Sylvester-order
 *     Walsh-Hadamard butterflies (strides 1,2,4,8,16) times fp32(1/sqrt(32)),
 *     amax = max|y|,  e = floor(log2 amax) - 2 (RN) or the smallest e with
 *     amax <= 6 * 2^e (RU), clamped to [-127, 127];  byte = e + 127 (0 if
 *     amax = 0);  code_j = E2M1(y_j * 2^-e).
 *   block: 16 for NVFP4, 32 for MXFP4 (anything else -> Q4_ERR_UNSUPPORTED).
 *   in_dt: Q4_BF16 or Q4_F32.  x: device [rows, ld] elements, ld >= cols,
 *   ld * elem_size a multiple of 16.  cols % block == 0.
 *   d_gscale: device pointer to s_t (NVFP4, required); must be NULL for MXFP4.
 *   d_chan: device float[cols] multipliers c (MXFP4 only, optional, NULL = 1).
 *   codes: device [rows, cols/2] bytes.  scales: device, q4_scale_bytes() bytes.
 *   flags: Q4_SCALE_RU | Q4_LAYOUT_TC | Q4_HADAMARD32 | Q4_SCALE_46.
 *   Q4_SCALE_46 (NVFP4; "Looped Transformer quantization", sec. 2.2 and the
 *     block_scale_46 of sec. 2.5): each block's scale is one of two rounded-up
 *     candidates, E4M3_RU(amax / (6 * s_t)) or E4M3_RU(amax / (4 * s_t)); the
 *     page gives no rule for the choice, so the block takes the candidate whose
 *     codes have the smaller sum of squared errors sum_j (x_j - dec_j * S)^2,
 *     formed in binary64 in element order (ties: the 6 candidate).  With
 *     s_t = max|W| / (6 * 256) either candidate keeps |x| <= 6, as Sigma-Delta
 *     requires.  Q4_SCALE_RU is implied.
 */
Q4_API q4_status q4_quantize(q4_format format, int block, q4_dtype in_dt, const void* x,
                      int64_t rows, int64_t cols, int64_t ld,
                      const float* d_gscale, const float* d_chan,
                      uint8_t* codes, uint8_t* scales, int flags, void* stream);

/*
 * q4_dequantize -- fake quantization, the inverse map ("Why Gated DeltaNet
 *   Survives 4-Bit Quantization", quantize-then-dequantize probes):
 *   out = code * s_b * s_t (NVFP4) or code * 2^e (MXFP4), formed in binary32
 *   (one rounding) and, for Q4_BF16 output, then rounded to bf16.
 *   codes/scales as written by q4_quantize with the same flags (only
 *   Q4_LAYOUT_TC matters).  out: device [rows, cols] of out_dt.
 */
Q4_API q4_status q4_dequantize(q4_format format, int block, const uint8_t* codes,
                        const uint8_t* scales, const float* d_gscale,
                        int64_t rows, int64_t cols, int flags,
                        q4_dtype out_dt, void* out, void* stream);

/*
 * q4_sigma_delta_step -- one loop visit of first-order Sigma-Delta
 *   requantization ("Looped Transformer quantization", sec. 2.1, and the code
 *   of sec. 2.5): with the block scales fixed,
 *     x = w / S (one correctly rounded binary32 division; S = s_b*s_t per
 *     NVFP4 block, 2^e per MXFP4 block),
 *     v = x + r,  q = E2M1(v),  r <- v - q,  codes <- q.
 *   Start a chain by zeroing r (r_0 = 0).  Scales normally come from
 *   q4_quantize with Q4_SCALE_RU and s_t = max|W| / (6*256), which keeps
 *   |x| <= 6 and hence |r| <= 1 (sec. 2.2).
 *   w: device float [rows, cols] (dense).  scales: device, layout per flags
 *   (Q4_LAYOUT_TC or row-major).  d_gscale: s_t (NVFP4) or NULL (MXFP4).
 *   residue: device float [rows, cols], read and written.  codes: device
 *   [rows, cols/2].  cols % block == 0.
 */
Q4_API q4_status q4_sigma_delta_step(q4_format format, int block, const float* w,
                              int64_t rows, int64_t cols, const uint8_t* scales,
                              const float* d_gscale, float* residue, uint8_t* codes,
                              int flags, void* stream);

/*
 * q4_sr_requant -- one stochastic-rounding requant of a weight at a loop visit
 *   ("Looped Transformer quantization", sec. 2.1: the stochastic-rounding
 *   baseline draws every code so that its conditional expectation equals the
 *   weight; sec. 3: a fixed seed gives one weight trajectory shared by all
 *   inputs).  With the block scales fixed, x = w / S (as in
 *   q4_sigma_delta_step); for neighbouring E2M1 magnitudes a <= |x| < b the
 *   code's magnitude is b when u < (|x| - a) / (b - a), else a; |x| >= 6 gives
 *   6; the sign bit is x's.  u = (word >> 8) * 2^-24, where for element
 *   e = row * cols + col the word is output e % 4 of Philox4x32-10 (Salmon et
 *   al., SC 2011) with counter (e / 4 low, e / 4 high, visit, 0) and key
 *   (seed low, seed high) -- any host or device implementation of that
 *   generator reproduces the codes.
 *   w, scales, d_gscale, codes, flags as q4_sigma_delta_step (no residue).
 */
Q4_API q4_status q4_sr_requant(q4_format format, int block, const float* w, int64_t rows,
                        int64_t cols, const uint8_t* scales, const float* d_gscale,
                        uint64_t seed, uint32_t visit, uint8_t* codes, int flags, void* stream);

/*
 * q4_sigma_delta_codebanks -- the whole Sigma-Delta chain of `visits` loop
 *   visits from r_0 = 0 in one pass, stored as codebanks ("Looped Transformer
 *   quantization", sec. 2.3: for frozen-weight inference the last K visits
 *   restart a chain of length K and use its codes in reverse order, tail visit
 *   j taking the code of chain step K - j + 1; sec. 4: those K codes are
 *   pre-generated as K codebanks, one bank read per visit).
 *   Same arithmetic as `visits` calls of q4_sigma_delta_step on a zeroed
 *   residue, but w and its scales are read once and the residue stays in
 *   registers.  codes: device [visits, rows, cols/2]; bank k (0-based) holds
 *   the codes of chain step k + 1, so tail visit j (1-based) of the reverse
 *   schedule reads bank visits - j.  residue_out: NULL, or device float
 *   [rows, cols] receiving r_visits.  visits in 1..4096.  Other arguments as
 *   q4_sigma_delta_step.
 */
Q4_API q4_status q4_sigma_delta_codebanks(q4_format format, int block, const float* w,
                                   int64_t rows, int64_t cols, const uint8_t* scales,
                                   const float* d_gscale, int visits, uint8_t* codes,
                                   float* residue_out, int flags, void* stream);

/*
 * q4_gemm -- block-scaled FP4 GEMM  Y = alpha * dec(A) dec(B)^T  on the
 *   tcgen05 tensor cores ("Why Gated DeltaNet Survives 4-Bit Quantization",
 *   prerequisites: W4A4 runs the GEMM on native 4-bit tensor cores; "MACaQ",
 *   core method: y = x_q W_q^T).  FP32 accumulation; alpha = s_tA * s_tB for
 *   NVFP4 and 1 for MXFP4.
 *   A (M x K): a_kind = Q4_A_QUANTIZED: `a` = codes [M, K/2], a_scales in TC
 *     layout, d_a_gscale = s_tA (NVFP4) or NULL.  a_kind = Q4_A_BF16 (NVFP4
 *     only): `a` = bf16 [M, K]; the call quantizes A exactly as q4_quantize
 *     (RN scales) with s_t = *d_a_gscale; a_scales must be NULL.
 *   B (N x K, the weight W): b_codes [N, K/2], b_scales in TC layout,
 *     d_b_gscale = s_tB (NVFP4) or NULL.
 *   Y: device [M, N] row-major, out_dt Q4_BF16 or Q4_F32.
 *   K % 64 == 0 (K = 0 writes zeros); N % 8 == 0; M, N >= 0 arbitrary otherwise.
 *   workspace: device scratch of ws_bytes >= q4_gemm_workspace_size(...)
 *     (0 bytes for Q4_A_QUANTIZED); its contents on entry do not matter.
 *     Q4_A_BF16 with M <= 16 and 256 <= K (up to about 16k: the quantized
 *     activations stay resident in shared memory) runs the fused decode kernel
 *     and needs none; other shapes quantize A once into the workspace.
 */
Q4_API q4_status q4_gemm(q4_format format, int block, int64_t M, int64_t N, int64_t K,
                  int a_kind, const void* a, const uint8_t* a_scales,
                  const float* d_a_gscale,
                  const uint8_t* b_codes, const uint8_t* b_scales,
                  const float* d_b_gscale,
                  q4_dtype out_dt, void* y, void* workspace, size_t ws_bytes,
                  void* stream);

/*
 * a_kind = Q4_A_BF16_W4A16 ("Looped Transformer quantization", introduction
 *   and sec. 0.2: the looped core runs weight-only 4-bit, W4A16, with BF16 as
 *   the compute view):  Y = alpha * X dec(W)^T with X the bf16 activations
 *   [M, K] (not quantized), dec(W) = code * s_b (NVFP4, exact in bf16) or
 *   code * 2^e (MXFP4), alpha = s_tB (NVFP4) or 1; bf16 x bf16 products summed
 *   in FP32 on the tensor cores.  a_scales and d_a_gscale must be NULL; no
 *   workspace.  K % 64 == 0, N % 8 == 0.
 */

/*
 * q4_sigma_delta_gemm -- one loop visit with the Sigma-Delta code generation
 *   fused into the GEMM's weight producer ("Looped Transformer quantization",
 *   sec. 4: online code generation from the reference weight and the residue
 *   state at every visit): with the NVFP4 block scales fixed,
 *     q = E2M1(w / S + r),  r <- (w / S + r) - q   (as q4_sigma_delta_step)
 *     Y = s_t * X (q * s_b)^T                          (as the W4A16 q4_gemm)
 *   without writing the codes: each weight element and its residue are read
 *   once and the residue is written back.  Decode shapes: M <= 16 (else
 *   Q4_ERR_UNSUPPORTED).  NVFP4 only; scales must be in the tensor-core layout
 *   (flags = Q4_LAYOUT_TC).  x: bf16 [M, K]; w: float [N, K]; residue: float
 *   [N, K], read and written (zero = start of a chain); y: [M, N] of out_dt.
 *   K % 64 == 0, N % 8 == 0.
 */
Q4_API q4_status q4_sigma_delta_gemm(q4_format format, int block, int64_t M, int64_t N, int64_t K,
                              const void* x, const float* w, const uint8_t* scales,
                              const float* d_gscale, float* residue, q4_dtype out_dt, void* y,
                              int flags, void* stream);

/*
 * Grouped calls -- one launch over a list of matrices.  The looped core of
 * "Looped Transformer quantization" (sec. 2.1 and sec. 4) requantizes every
 * weight of the core at each loop visit; the core has many matrices of a few
 * million weights, where one launch per matrix costs more than the work.  Each
 * grouped call is exactly the matching single-matrix call applied to every
 * entry of `mats` (same arithmetic, same outputs byte for byte), in one kernel
 * launch.  `mats` is a HOST array of `count` entries (0 <= count <=
 * Q4_MAX_GROUP; 0 does nothing) read before the call returns; every pointer in
 * it is device memory.  Matrices are dense (row stride = cols).  No output
 * buffer of one entry may overlap any buffer of another entry.  format,
 * block, flags apply to every entry.  An invalid entry fails the whole call
 * before any launch (Q4_ERR_ARG / Q4_ERR_ALIGN / Q4_ERR_SHAPE).
 */
#define Q4_MAX_GROUP 32
typedef struct q4_matrix {
    const void* w;          /* weights [rows, cols]: float; q4_quantize_grouped: in_dt */
    int64_t rows, cols;
    uint8_t* scales;        /* block scales (layout per flags): read by the requant
                               calls, written by q4_quantize_grouped (q4_scale_bytes) */
    const float* d_gscale;  /* NVFP4 tensor scale s_t (one float); NULL for MXFP4 */
    float* residue;         /* q4_sigma_delta_step_grouped: r [rows, cols], in/out;
                               q4_sigma_delta_codebanks_grouped: NULL or r_visits out;
                               ignored by the other calls */
    uint8_t* codes;         /* codes [rows, cols/2]; codebanks: [visits, rows, cols/2] */
} q4_matrix;

/* q4_quantize on every entry (x = w, ld = cols, no channel multipliers). */
Q4_API q4_status q4_quantize_grouped(q4_format format, int block, q4_dtype in_dt,
                                     const q4_matrix* mats, int count, int flags, void* stream);
/* q4_sigma_delta_step on every entry. */
Q4_API q4_status q4_sigma_delta_step_grouped(q4_format format, int block, const q4_matrix* mats,
                                             int count, int flags, void* stream);
/* q4_sr_requant on every entry, all with the same seed and visit (each
   matrix's elements are numbered from 0, as in the single call). */
Q4_API q4_status q4_sr_requant_grouped(q4_format format, int block, const q4_matrix* mats,
                                       int count, uint64_t seed, uint32_t visit, int flags,
                                       void* stream);
/* q4_sigma_delta_codebanks on every entry (residue = residue_out). */
Q4_API q4_status q4_sigma_delta_codebanks_grouped(q4_format format, int block,
                                                  const q4_matrix* mats, int count, int visits,
                                                  int flags, void* stream);

/* One matrix of q4_sigma_delta_gemm_grouped (all pointers device memory). */
typedef struct q4_sd_gemm_entry {
    const void* x;          /* bf16 activations [M, K] this weight multiplies */
    const float* w;         /* FP32 master weight [N, K] */
    const uint8_t* scales;  /* its NVFP4 block scales, tensor-core layout */
    const float* d_gscale;  /* its tensor scale s_t (one float) */
    float* residue;         /* its Sigma-Delta residue [N, K], read and written */
    void* y;                /* output [M, N] of out_dt */
    int64_t N;
} q4_sd_gemm_entry;

/* q4_sigma_delta_gemm on every entry in one launch: one loop visit of a looped
   core whose matrices share M and K (sec. 4 of the looped page: the visit
   requantizes and applies every weight of the core).  format = Q4_NVFP4,
   flags = Q4_LAYOUT_TC, 1 <= M <= 16, K % 64 == 0, each N % 8 == 0;
   0 <= count <= Q4_MAX_GROUP.  No buffer of one entry may overlap an output
   (residue, y) of another. */
Q4_API q4_status q4_sigma_delta_gemm_grouped(q4_format format, int block, int64_t M, int64_t K,
                                             const q4_sd_gemm_entry* entries, int count,
                                             q4_dtype out_dt, int flags, void* stream);

/* One weight of q4_gemm_shared_a. */
typedef struct {
    const uint8_t* b_codes;   /* [N, K/2] packed codes                              */
    const uint8_t* b_scales;  /* tensor-core scale layout                           */
    const float* d_b_gscale;  /* NVFP4: device s_t of the weight; MXFP4: NULL       */
    void* y;                  /* [M, N] output of out_dt                            */
    int64_t N;                /* N % 8 == 0; 0 skips the entry                      */
} q4_gemm_weight;

#define Q4_MAX_SHARED_A 4

/*
 * q4_gemm_shared_a -- one quantized A times several weights, Y_w = alpha_w *
 *   dec(A) dec(B_w)^T for w < count, in one persistent launch: the output tiles
 *   of every weight form one list walked by the same grid, so the launch pays
 *   one ramp and one partial last wave instead of one per weight (the
 *   projections of one layer input, as the W4A4 linear layers of the "Why
 *   Gated DeltaNet Survives 4-Bit Quantization" page apply to a quantized
 *   activation).  Each Y_w is, bit for bit, what q4_gemm with a_kind =
 *   Q4_A_QUANTIZED gives for that weight.  a, a_scales, d_a_gscale, M, K and the
 *   requirements as q4_gemm; 1 <= count <= Q4_MAX_SHARED_A; no y may overlap
 *   another entry's y or any input.
 */
Q4_API q4_status q4_gemm_shared_a(q4_format format, int block, int64_t M, int64_t K, const uint8_t* a,
                                  const uint8_t* a_scales, const float* d_a_gscale,
                                  const q4_gemm_weight* weights, int count, q4_dtype out_dt, void* stream);

/* Scratch bytes q4_gemm needs for these arguments (0 when none). */
Q4_API size_t q4_gemm_workspace_size(q4_format format, int64_t M, int64_t N, int64_t K,
                              int a_kind);

/*
 * q4_gemm_a_bf16_noalloc -- the NVFP4 GEMM with bf16 activations
 *   (q4_gemm with a_kind = Q4_A_BF16) for callers that cannot allocate device
 *   memory when they call it: code embedded in an application that owns every
 *   device buffer through its own fixed pool, or that has to keep its device
 *   footprint constant after start-up, and so cannot pass q4_gemm the scratch
 *   workspace it needs for larger M.  No counterpart on the source pages: it is
 *   a packaging variant, not part of the method.
 *   Same arithmetic as q4_gemm: the activations are quantized exactly as
 *   q4_quantize (NVFP4, RN scales, tensor scale *d_a_gscale) and multiplied with
 *   the quantized weight on the tensor cores.  Allocates nothing: the quantized
 *   activations go to a fixed array of Q4_NOALLOC_SCRATCH_BYTES inside the
 *   library, which every GPU that loads the library keeps until the process
 *   exits.  Codes [M, K/2] (rounded up to 256 bytes) plus the tensor-core scales
 *   must fit in it (M * K / 2 + scales <= 32 MiB, e.g. M = 8192, K = 5120);
 *   larger sizes return Q4_ERR_WORKSPACE before any launch.
 *   All calls share that one array: calls whose work overlaps on the GPU (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.  Each call overwrites every part of the array it reads, so nothing
 *   has to be cleared between calls.  The first call on a device looks up the
 *   array's device address (once per device, with that device current); make
 *   that first call before any stream capture.  The address stays cached for
 *   the life of the process, so a cudaDeviceReset after the first call on a
 *   device is not supported.
 *   Arguments and results as q4_gemm with a_kind = Q4_A_BF16: a_bf16 bf16
 *   [M, K]; b_codes/b_scales/d_b_gscale the NVFP4 weight (tensor-core scale
 *   layout); y [M, N] of out_dt; K % 64 == 0, N % 8 == 0, K <= 2^30,
 *   M, N <= 2^31 (else Q4_ERR_SHAPE); K == 0 zero-fills y.  It always takes the
 *   quantize-then-GEMM route, also for M <= 16, where q4_gemm runs the fused
 *   decode kernel instead (same codes and products, another summation order).
 *   A CUDA failure returns Q4_ERR_CUDA with its text in q4_last_error().
 */
#define Q4_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
Q4_API q4_status q4_gemm_a_bf16_noalloc(int64_t M, int64_t N, int64_t K, const void* a_bf16,
                                        const float* d_a_gscale, const uint8_t* b_codes,
                                        const uint8_t* b_scales, const float* d_b_gscale,
                                        q4_dtype out_dt, void* y, void* stream);

/*
 * q4_set_wait_limit -- how long a bounded wait inside a kernel may spin before
 *   it gives up: `cycles` SM clock cycles, 1000 <= cycles <= 2^40, or 0 for
 *   the default Q4_DEFAULT_WAIT_CYCLES (about 1 s at B200 clocks).  A wait
 *   that runs out records Q4_ERR_TIMEOUT for q4_get_device_error and the
 *   kernel winds down (stops issuing, waits with the same limit for its own
 *   copies in flight, frees what it allocated, exits).  Applies to launches
 *   made after the call returns; the setting is per process and device and is
 *   written with a synchronous copy, so do not call it during stream capture.
 *   No counterpart on the source pages: failure detection of this library.
 */
#define Q4_DEFAULT_WAIT_CYCLES 2000000000ll
Q4_API q4_status q4_set_wait_limit(int64_t cycles);

/*
 * q4_get_device_error -- synchronises `stream`, then reads and clears the
 *   library's device error word.  Returns Q4_ERR_TIMEOUT if a bounded wait
 *   inside a GEMM kernel gave up since the last call, Q4_ERR_CUDA if the
 *   synchronisation itself failed, else Q4_OK.
 */
Q4_API q4_status q4_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H_ */
