// q4_codec.cuh -- device-side number formats: E2M1 element codes, E4M3 and
// E8M0 block scales, and the per-block scale rules of NVFP4 and MXFP4.
//
// Every floating-point step uses an explicitly rounded intrinsic (_rn) so the
// compiler cannot contract or reorder it; the sequences follow the operation
// order documented in q4.h.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace q4 {

// Eight E2M1 codes from eight floats: round to nearest, ties to even
// mantissa, saturating at +-6, keeping the sign bit of values that round to
// zero (-0.1 -> 0x8).  Element 0 lands in the low nibble.
__device__ __forceinline__ uint32_t e2m1_pack8(const float (&v)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// Four E2M1 codes (element 0 in the low nibble) of four floats.
__device__ __forceinline__ uint32_t e2m1_pack4(float a, float b, float c, float d) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "mov.b32 %0, {b0, b1, 0, 0};\n\t}"
        : "=r"(out) : "f"(a), "f"(b), "f"(c), "f"(d));
    return out;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Eight E2M1 codes (element 0 in the low nibble) -> four packed bf16 pairs of
// their values (element 2i in the low half of word i) with byte permutes
// only, no conversion instructions (those run on a narrow pipe): the low and
// high bytes of the bf16 patterns of the 8 magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6
// are two 8-byte tables indexed by the code's low three bits, and each sign bit
// is moved to bit 15 / 31 by a sign-replicating permute.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, uint32_t (&o)[4]) {
    constexpr uint32_t LO0 = 0xC0800000u, LO1 = 0xC0804000u;   // low bytes: 0 0 80 C0 | 0 40 80 C0
    constexpr uint32_t HI0 = 0x3F3F3F00u, HI1 = 0x40404040u;   // high bytes: 0 3F 3F 3F | 40 40 40 40
    const uint32_t sel = w & 0x77777777u;
    const uint32_t lo_a = prmt(LO0, LO1, sel), hi_a = prmt(HI0, HI1, sel);
    const uint32_t lo_b = prmt(LO0, LO1, sel >> 16), hi_b = prmt(HI0, HI1, sel >> 16);
    const uint32_t sg = w & 0x88888888u, sg4 = sg << 4;
    o[0] = prmt(lo_a, hi_a, 0x5140u) | (prmt(sg4, sg, 0xC080u) & 0x80008000u);
    o[1] = prmt(lo_a, hi_a, 0x7362u) | (prmt(sg4, sg, 0xD090u) & 0x80008000u);
    o[2] = prmt(lo_b, hi_b, 0x5140u) | (prmt(sg4, sg, 0xE0A0u) & 0x80008000u);
    o[3] = prmt(lo_b, hi_b, 0x7362u) | (prmt(sg4, sg, 0xF0B0u) & 0x80008000u);
}

// Magnitude of an E2M1 code (low three bits) as float: 0, .5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
    // twice the magnitudes, one nibble each: 0,1,2,3,4,6,8,12
    const uint32_t twice = 0xC8643210u;
    float m = (float)((twice >> (4 * (code & 7u))) & 0xFu) * 0.5f;
    return (code & 8u) ? -m : m;
}

// E4M3 (finite variant) byte -> value, for non-negative codes 0x00..0x7E.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
    uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return (float)m * 0.001953125f;             // m * 2^-9, exact
    return __uint_as_float(((e + 120u) << 23) | (m << 20));  // (1 + m/8) * 2^(e-7)
}

// Non-negative float -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rn(float v) {
    v = fminf(v, 448.0f);
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;
}

// Smallest E4M3 byte whose value is >= v (v >= 0), saturating at 448.
__device__ __forceinline__ uint32_t e4m3_ru(float v) {
    uint32_t b = e4m3_rn(v);
    if (b < 0x7Eu && e4m3_value(b) < v) b += 1;
    return b;
}

// Shared MXFP4 exponent of a block with maximum magnitude amax >= 0:
// floor(log2 amax) - 2, or with round_up the smallest e with amax <= 6 * 2^e,
// clamped to [-127, 127]; amax = 0 gives -127.
__device__ __forceinline__ int mx_exponent(float amax, bool round_up) {
    uint32_t bits = __float_as_uint(amax);
    if (bits == 0) return -127;
    int fl;
    uint32_t m23;
    uint32_t biased = bits >> 23;
    if (biased != 0) {
        fl = (int)biased - 127;
        m23 = bits & 0x7FFFFFu;
    } else {
        int p = 31 - __clz(bits);          // leading bit of the subnormal mantissa
        fl = p - 149;
        m23 = (bits << (23 - p)) & 0x7FFFFFu;
    }
    int e = fl - 2;
    if (round_up && m23 > 0x400000u) e += 1;  // significand above 1.5: 4*sig > 6
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^k as a float for k in [-127, 127] (exact; 2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int k) {
    if (k >= -126) return __uint_as_float((uint32_t)(k + 127) << 23);
    return __uint_as_float(0x00400000u);
}

// Per-block normalisation of NVFP4 (see q4.h): elements are divided by the
// block's decoded scale S = dec(s_b) * s_t, one correctly rounded binary32
// division per element ("Looped Transformer quantization", sec. 2.5: x = W / s).
// y = RN(1 / S) feeds the quotient helpers below; it is NaN for a degenerate
// block (S = 0, a reciprocal that overflows, or an unusable s_t: every
// normalised value is +0) and 0 when S lies outside [2^-96, 2^29], where the
// helpers take the correctly rounded division itself.
struct NvScale {
    uint32_t byte;
    float S, y;
    bool degenerate;
};

__device__ __forceinline__ bool st_valid(float s_t) {
    return s_t > 0.0f && isfinite(s_t);
}

// y = RN(1 / S) for a scale S inside the correction step's range [2^-96, 2^29]
// (see quot_fast below), 0 outside it (the quotient helpers then divide).
__device__ __forceinline__ float quot_recip(float S) {
    return (S >= 0x1p-96f && S <= 0x1p29f) ? __frcp_rn(S) : 0.0f;
}

__device__ __forceinline__ NvScale nv_scale_of(uint32_t byte, float s_t) {
    NvScale r;
    r.byte = byte;
    r.S = __fmul_rn(e4m3_value(byte), s_t);
    r.degenerate = !st_valid(s_t) || r.S == 0.0f || !isfinite(__frcp_rn(r.S));
    r.y = r.degenerate ? __uint_as_float(0x7FC00000u) : quot_recip(r.S);
    return r;
}

__device__ __forceinline__ NvScale nv_scale_from_amax(float amax, float s_t, bool round_up) {
    uint32_t byte = 0;
    if (st_valid(s_t)) {
        float denom = __fmul_rn(6.0f, s_t);
        float sbf = __fdiv_rn(amax, denom);
        byte = round_up ? e4m3_ru(sbf) : e4m3_rn(sbf);
    }
    return nv_scale_of(byte, s_t);
}

__device__ __forceinline__ NvScale nv_scale_from_byte(uint32_t byte, float s_t) { return nv_scale_of(byte, s_t); }

// ---- pairs of binary32 values on the f32x2 ALU: each lane is rounded to
// nearest exactly as the scalar __fmul_rn / __fadd_rn / __fsub_rn.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// Two scalar products rounded to nearest, for a product that feeds an add:
// ptxas fuses a paired multiply into the paired add that consumes it,
// rounding modifier or not, while a scalar mul.rn is never contracted.
__device__ __forceinline__ float2 mul2_sep_rn(float2 a, float2 b) {
    return make_float2(__fmul_rn(a.x, b.x), __fmul_rn(a.y, b.y));
}
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
        "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// ---- the correctly rounded quotient RN(w / S) from y = RN(1 / S)
// One Markstein correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop. 34(1),
// 1990): q0 = RN(w * y) is within one unit in the last place of w / S, so the
// remainder r = w - q0 * S is a binary32 number that one fused multiply-add
// forms exactly, and RN(q0 + r * y) is the correctly rounded quotient.  For
// significands of w and S in [1, 2) the sequence was compared with the
// correctly rounded division on every one of the 2^46 pairs; scaling w and S
// by powers of two scales every step exactly while w, q0 and r stay on the
// binary32 grid without overflow, which holds for S in [2^-96, 2^29] (y > 0)
// and 2^-96 <= |w| <= 2^24 (then 2^-125 <= |q0| <= 2^120).
__device__ __forceinline__ float quot_fast(float w, float S, float y) {
    const float q0 = __fmul_rn(w, y);
    const float r = __fmaf_rn(-q0, S, w);
    return __fmaf_rn(r, y, q0);
}

__device__ __forceinline__ bool quot_domain(float w) { return fabsf(w) >= 0x1p-96f && fabsf(w) <= 0x1p24f; }

// The correctly rounded division, out of line: taken only for values outside
// the correction step's domain (zeros, subnormal-range or huge weights) or
// scales outside its range.
static __device__ __noinline__ float4 quot4_div(float4 w, float S) {
    return make_float4(__fdiv_rn(w.x, S), __fdiv_rn(w.y, S), __fdiv_rn(w.z, S), __fdiv_rn(w.w, S));
}

// RN(w_j / S) for four finite values (S > 0 with its NvScale y, y not NaN):
// the correction step on f32x2 pairs (the negated scale nS = -S is passed in,
// so no operand needs negating), or the correctly rounded division for all
// four when any of them lies outside the step's domain or y = 0.
__device__ __forceinline__ float4 quot4_rn(float4 w, float S, float nS, float y) {
    const float2 yy = make_float2(y, y), nn = make_float2(nS, nS);
    const float2 wa = make_float2(w.x, w.y), wb = make_float2(w.z, w.w);
    const float2 qa = mul2_rn(wa, yy), qb = mul2_rn(wb, yy);
    const float2 ra = fma2_rn(qa, nn, wa), rb = fma2_rn(qb, nn, wb);
    const float2 xa = fma2_rn(ra, yy, qa), xb = fma2_rn(rb, yy, qb);
    const bool ok = y > 0.0f && quot_domain(w.x) && quot_domain(w.y) && quot_domain(w.z) && quot_domain(w.w);
    if (__builtin_expect(!ok, 0)) return quot4_div(w, S);
    return make_float4(xa.x, xa.y, xb.x, xb.y);
}

// RN(w / S) for one finite value, as quot4_rn.
__device__ __forceinline__ float quot_rn(float w, float S, float y) {
    if (y > 0.0f && quot_domain(w)) return quot_fast(w, S, y);
    return __fdiv_rn(w, S);
}

// The code-decision form for a whole block whose guard `quot_block_fast`
// holds: for every element whose quotient reaches 2^-3, |w| >= 2^-3 S >= 2^-99
// keeps the remainder's bits above 2^-149 and q0 <= amax y <= 2^96, so the
// quotient there is exact; smaller quotients may be off by a few units but stay
// below 2^-3 with the sign of w, which is all the E2M1 code of such a value
// (magnitude 0) depends on.
__device__ __forceinline__ bool quot_block_fast(float amax, float y) {
    return y > 0.0f && __fmul_rn(amax, y) <= 0x1p96f;
}

// E4M3 byte (round to nearest even, saturating) of the binary32 quotient
// RN(amax / denom), for amax >= 0 and denom > 0, given rden = RN(1 / denom)
// normal and finite.  q0 = RN(amax * rden) carries two roundings of relative
// size <= 2^-24 each, so RN(amax / denom) lies within two units in the last
// place of q0 (four bit-pattern steps below a power of two).  E4M3 rounding
// is monotone, so when the bytes of q0 -/+ four steps agree that byte is the
// answer; otherwise (next to an E4M3 rounding boundary) the quotient is
// formed by the correctly rounded division.
// The fast half: true (byte set) when the bytes of q0 -/+ four steps agree.
__device__ __forceinline__ bool e4m3_rn_of_quotient_fast(float amax, float rden, uint32_t& byte) {
    const uint32_t b = __float_as_uint(__fmul_rn(amax, rden));
    const float lo = __uint_as_float(b >= 4u ? b - 4u : 0u);
    const float hi = __uint_as_float(b + 4u);
    uint16_t pr;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(fminf(hi, 448.0f)), "f"(fminf(lo, 448.0f)));
    byte = pr & 0xFFu;
    return byte == (uint32_t)(pr >> 8);
}
__device__ __forceinline__ uint32_t e4m3_rn_of_quotient(float amax, float denom, float rden) {
    uint32_t byte;
    if (e4m3_rn_of_quotient_fast(amax, rden, byte)) return byte;
    return e4m3_rn(__fdiv_rn(amax, denom));
}

// Largest magnitude of N values (0 if there is none that is not NaN) as a
// balanced tree of maxima: depth log2 N instead of a chain of N; the maximum
// does not depend on the order it is taken in.
template <int N>
__device__ __forceinline__ float amax_tree(const float* v) {
    float m[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) m[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
#pragma unroll
    for (int w = N / 4; w >= 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
    }
    return fmaxf(0.0f, m[0]);
}

// Values of the two E2M1 codes in one byte (element 0 = low nibble -> .x),
// through the hardware E2M1 -> f16 conversion (every E2M1 value is exact in
// f16 and in binary32).
__device__ __forceinline__ float2 e2m1x2_value(uint32_t byte) {
    uint32_t h;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(byte));
    float lo, hi;
    asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h));
    return make_float2(lo, hi);
}

// NVFP4 per-launch context: the tensor scale, 6 * s_t and its reciprocal,
// whether the fast RN scale path applies, and the shared-memory table of
// (S, y) = (dec(s_b) * s_t, RN(1 / S)) for every E4M3 byte 0..127, y as in
// NvScale (NaN: degenerate; 0: S outside the correction step's range).
struct NvCtx {
    float s_t, denom, rden;
    bool st_ok, fast;
    const float2* tab;
};

__device__ __forceinline__ NvCtx nv_ctx(float s_t, const float2* tab) {
    NvCtx c;
    c.s_t = s_t;
    c.st_ok = st_valid(s_t);
    c.denom = __fmul_rn(6.0f, s_t);
    c.rden = __frcp_rn(c.denom);
    c.fast = c.st_ok && isfinite(c.rden) && c.rden >= 0x1p-126f && c.denom >= 0x1p-126f;
    c.tab = tab;
    return c;
}

__device__ __forceinline__ void nv_fill_table(float s_t, float2* tab, int tid, int nthreads) {
    for (int b = tid; b < 128; b += nthreads) {
        const NvScale r = nv_scale_of((uint32_t)b, s_t);
        tab[b] = make_float2(r.S, r.y);
    }
}

// E2M1 codes of the 16 values of a block divided by S (y = RN(1 / S) from the
// table, amax the block's largest magnitude): 0 for a degenerate scale (y
// NaN), the correction step on f32x2 pairs when the block guard holds, the
// correctly rounded division otherwise.
__device__ __forceinline__ void nv_codes16(const float (&v)[16], float2 sy, float amax, uint32_t (&w)[2]) {
    const float S = sy.x, y = sy.y;
    if (y != y) {
        w[0] = w[1] = 0u;
    } else if (quot_block_fast(amax, y)) {
        const float2 yy = make_float2(y, y), SS = make_float2(S, S);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float q[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 x = make_float2(v[8 * g + 2 * i], v[8 * g + 2 * i + 1]);
                const float2 q0 = mul2_rn(x, yy);
                const float2 t = fma2_rn(q0, SS, make_float2(-x.x, -x.y));
                const float2 q1 = fma2_rn(make_float2(-t.x, -t.y), yy, q0);
                q[2 * i] = q1.x;
                q[2 * i + 1] = q1.y;
            }
            w[g] = e2m1_pack8(q);
        }
    } else {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float q[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(v[8 * g + i], S);
            w[g] = e2m1_pack8(q);
        }
    }
}

// N NVFP4 blocks at once: amax, E4M3 scale byte (RN or RU of amax / (6 s_t)),
// codes of x / S (all zero for a degenerate scale).  Each step runs over all
// N blocks before the next, with no branch that is not uniform across the
// warp in between, so the blocks' dependency chains interleave.
template <bool RU, int N>
__device__ __forceinline__ void nv_blocks(const float (&v)[N][16], const NvCtx& c, uint32_t (&byte)[N],
                                          uint32_t (&w)[N][2]) {
    float amax[N];
#pragma unroll
    for (int k = 0; k < N; ++k) amax[k] = amax_tree<16>(v[k]);
    if (!c.st_ok) {
#pragma unroll
        for (int k = 0; k < N; ++k) byte[k] = 0;
    } else if (!RU && c.fast) {
        bool ok[N];
#pragma unroll
        for (int k = 0; k < N; ++k) ok[k] = e4m3_rn_of_quotient_fast(amax[k], c.rden, byte[k]);
        // next to an E4M3 rounding boundary: the correctly rounded division
#pragma unroll
        for (int k = 0; k < N; ++k)
            if (!ok[k]) byte[k] = e4m3_rn(__fdiv_rn(amax[k], c.denom));
    } else {
#pragma unroll
        for (int k = 0; k < N; ++k)
            byte[k] = RU ? e4m3_ru(__fdiv_rn(amax[k], c.denom)) : e4m3_rn(__fdiv_rn(amax[k], c.denom));
    }
    float2 sy[N];
#pragma unroll
    for (int k = 0; k < N; ++k) sy[k] = c.tab[byte[k]];
#pragma unroll
    for (int k = 0; k < N; ++k) nv_codes16(v[k], sy[k], amax[k], w[k]);
}

template <bool RU>
__device__ __forceinline__ void nv_block(const float (&v)[16], const NvCtx& c, uint32_t& byte, uint32_t (&w)[2]) {
    uint32_t b[1], ww[1][2];
    nv_blocks<RU, 1>(reinterpret_cast<const float(&)[1][16]>(v), c, b, ww);
    byte = b[0];
    w[0] = ww[0][0];
    w[1] = ww[0][1];
}

// Offset of scale (r, c) in the tensor-core scale layout (see q4.h).
__host__ __device__ __forceinline__ int64_t tc_scale_offset(int64_t r, int64_t c, int64_t catoms) {
    return ((r >> 7) * catoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

}  // namespace q4
