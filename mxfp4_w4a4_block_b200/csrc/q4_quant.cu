// q4_quant.cu -- memory-bound kernels of the path: tensor amax, NVFP4 / MXFP4
// block quantization (with the optional per-channel scale and block
// Hadamard-32 of MACaQ fused in), dequantization and the first-order
// Sigma-Delta step of "Looped Transformer quantization", sec. 2.1.
//
// The quantizer gives each thread whole blocks (the scale rule, the Hadamard
// rotation and the code packing stay in registers) and each CTA one scale
// atom's worth of blocks, so the scales leave as 512 contiguous bytes.  The
// Sigma-Delta step only reads scales and is a plain elementwise stream.
#include <cstdint>
#include <cuda_runtime.h>

#include "q4_codec.cuh"
#include "q4_internal.h"

namespace q4 {

// ------------------------------------------------------------------ amax
__global__ void __launch_bounds__(256) amax_kernel(const void* __restrict__ x, int64_t n, int bf16,
                                                   unsigned int* __restrict__ out) {
    float m = 0.0f;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    if (bf16) {
        const uint4* v = reinterpret_cast<const uint4*>(x);
        const int64_t nv = n / 8;
        for (int64_t i = tid; i < nv; i += nthreads) {
            uint4 w = __ldcs(v + i);
            uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(ws[j])), fabsf(bf16_hi(ws[j]))));
        }
        const uint16_t* s = reinterpret_cast<const uint16_t*>(x);
        for (int64_t i = nv * 8 + tid; i < n; i += nthreads)
            m = fmaxf(m, fabsf(__uint_as_float((uint32_t)s[i] << 16)));
    } else {
        const float4* v = reinterpret_cast<const float4*>(x);
        const int64_t nv = n / 4;
        for (int64_t i = tid; i < nv; i += nthreads) {
            float4 w = __ldcs(v + i);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(w.x), fabsf(w.y)), fmaxf(fabsf(w.z), fabsf(w.w))));
        }
        const float* s = reinterpret_cast<const float*>(x);
        for (int64_t i = nv * 4 + tid; i < n; i += nthreads) m = fmaxf(m, fabsf(s[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < 8 ? red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        // magnitudes are non-negative, so their bit patterns order like integers
        if (threadIdx.x == 0) atomicMax(out, __float_as_uint(m));
    }
}

__global__ void amax_finalize_kernel(float* out, float denom) {
    out[1] = __fdiv_rn(out[0], denom);
}

cudaError_t launch_amax(const void* x, int64_t n, bool bf16, float denom, float* d_out,
                        cudaStream_t st, int num_sms) {
    cudaError_t e = cudaMemsetAsync(d_out, 0, 2 * sizeof(float), st);
    if (e != cudaSuccess) return e;
    if (n > 0) {
        int64_t vec = bf16 ? n / 8 : n / 4;
        int64_t blocks = (vec + 255) / 256;
        int grid = (int)(blocks < (int64_t)num_sms * 8 ? (blocks > 0 ? blocks : 1) : (int64_t)num_sms * 8);
        amax_kernel<<<grid, 256, 0, st>>>(x, n, bf16 ? 1 : 0, reinterpret_cast<unsigned int*>(d_out));
    }
    amax_finalize_kernel<<<1, 1, 0, st>>>(d_out, denom);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ helpers
// Load one 16-byte chunk: 8 bf16 or 4 fp32 values (two chunks make 8 fp32).
__device__ __forceinline__ void load_bf16x8(const void* src, float* v) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
    v[0] = bf16_lo(raw.x); v[1] = bf16_hi(raw.x); v[2] = bf16_lo(raw.y); v[3] = bf16_hi(raw.y);
    v[4] = bf16_lo(raw.z); v[5] = bf16_hi(raw.z); v[6] = bf16_lo(raw.w); v[7] = bf16_hi(raw.w);
}
__device__ __forceinline__ void load_f32x4(const void* src, float* v) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(src));
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

// Sylvester-order Walsh-Hadamard butterflies over 32 values held by one
// thread (strides 1, 2, 4, 8, 16; (a, b) -> (a + b, a - b)), unnormalised.
__device__ __forceinline__ void fwht32_reg(float (&v)[32]) {
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
}

// ------------------------------------------------------------------ quantize
// One thread per block.  A CTA of 256 threads owns a tile of 128 rows x 4
// blocks -- exactly one 512-byte atom of the tensor-core scale layout -- so
// each thread quantizes 2 blocks per tile.  Lanes 4k..4k+3 of a warp take the
// 4 consecutive blocks of one row, so a warp's loads cover 8 whole row
// segments (128 or 256 bytes each of bf16); the first 16-byte load of a block
// brings its lines into L1 for the rest.  All loads of a tile are issued
// before any arithmetic.
template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool CHAN>
__global__ void __launch_bounds__(256) quantize_kernel(QuantParams p) {
    constexpr int TILE_C = 4 * BLK;          // columns per tile (one scale atom)
    constexpr int BPT = 2;                   // blocks per thread per tile
    constexpr int ESZ = BF16 ? 2 : 4;
    constexpr int LOADS = BLK * ESZ / 16;    // 16-byte loads per block
    constexpr int PER_LOAD = 16 / ESZ;       // values per load
    __shared__ __align__(16) uint8_t sf_atom[512];

    const int tid = threadIdx.x;
    const int64_t tiles_c = (p.cols + TILE_C - 1) / TILE_C;
    const int64_t tiles = ((p.rows + 127) / 128) * tiles_c;
    const float s_t = (BLK == 16) ? *p.gscale : 0.0f;
    const float inv_sqrt32 = 0x1.6a09e6p-3f;   // binary32 nearest to 1/sqrt(32)
    const char* xb = reinterpret_cast<const char*>(p.x);

    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t tr = t / tiles_c, tc = t % tiles_c;
        const int64_t row0 = tr * 128, col0 = tc * TILE_C;

        float v[BPT][BLK];
        bool valid[BPT];
#pragma unroll
        for (int it = 0; it < BPT; ++it) {
            const int bt = it * 256 + tid;            // block inside the tile
            const int64_t row = row0 + (bt >> 2);
            const int64_t col = col0 + (bt & 3) * BLK;
            valid[it] = row < p.rows && col < p.cols;
            if (valid[it]) {
                const char* src = xb + (row * p.ld + col) * ESZ;
#pragma unroll
                for (int l = 0; l < LOADS; ++l) {
                    if (BF16) load_bf16x8(src + 16 * l, &v[it][PER_LOAD * l]);
                    else load_f32x4(src + 16 * l, &v[it][PER_LOAD * l]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < BLK; ++i) v[it][i] = 0.0f;
            }
        }
#pragma unroll
        for (int it = 0; it < BPT; ++it) {
            const int bt = it * 256 + tid;
            const int rt = bt >> 2, cb = bt & 3;
            const int64_t row = row0 + rt;
            const int64_t col = col0 + cb * BLK;
            if (CHAN && valid[it]) {
                const float4* cp = reinterpret_cast<const float4*>(p.chan + col);
#pragma unroll
                for (int q = 0; q < BLK / 4; ++q) {
                    const float4 c = __ldg(cp + q);
                    v[it][4 * q] = __fmul_rn(v[it][4 * q], c.x);
                    v[it][4 * q + 1] = __fmul_rn(v[it][4 * q + 1], c.y);
                    v[it][4 * q + 2] = __fmul_rn(v[it][4 * q + 2], c.z);
                    v[it][4 * q + 3] = __fmul_rn(v[it][4 * q + 3], c.w);
                }
            }
            if constexpr (HAD) {
                fwht32_reg(*reinterpret_cast<float(*)[32]>(&v[it][0]));
#pragma unroll
                for (int i = 0; i < BLK; ++i) v[it][i] = __fmul_rn(v[it][i], inv_sqrt32);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < BLK; ++i) amax = fmaxf(amax, fabsf(v[it][i]));
            uint32_t byte;
            if constexpr (BLK == 16) {
                const NvScale sc = nv_scale_from_amax(amax, s_t, RU);
                byte = sc.byte;
#pragma unroll
                for (int i = 0; i < BLK; ++i) v[it][i] = sc.degenerate ? 0.0f : __fmul_rn(v[it][i], sc.inv);
            } else {
                const int e = mx_exponent(amax, RU);
                byte = (uint32_t)(e + 127);
                const float mult = exp2_int(-e);
#pragma unroll
                for (int i = 0; i < BLK; ++i) v[it][i] = __fmul_rn(v[it][i], mult);
            }
            uint32_t w[BLK / 8];
#pragma unroll
            for (int g = 0; g < BLK / 8; ++g) w[g] = e2m1_pack8(*reinterpret_cast<float(*)[8]>(&v[it][8 * g]));
            if (valid[it]) {
                uint8_t* dst = p.codes + row * (p.cols / 2) + col / 2;
                if constexpr (BLK == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (TC) sf_atom[(rt & 31) * 16 + (rt >> 5) * 4 + cb] = (uint8_t)byte;
            else if (valid[it]) p.scales[row * p.scols + tc * 4 + cb] = (uint8_t)byte;
        }
        if (TC) {
            __syncthreads();
            if (tid < 32) {
                const uint4 a = reinterpret_cast<const uint4*>(sf_atom)[tid];
                reinterpret_cast<uint4*>(p.scales + (tr * p.catoms + tc) * 512)[tid] = a;
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------ sigma-delta
// Elementwise over 8-weight chunks (grid-stride, two chunks per thread in
// flight): it reads the fixed block scales and streams w, r in, r out, codes.
template <int BLK, bool TC>
__device__ __forceinline__ void sigma_delta_chunk(const SigmaDeltaParams& p, float s_t, int64_t row, int64_t col,
                                                  const float4& w0, const float4& w1, const float4& r0,
                                                  const float4& r1, uint32_t sb) {
    float inv;
    bool degenerate;
    if (BLK == 16) {
        const NvScale s = nv_scale_from_byte(sb, s_t);
        inv = s.inv;
        degenerate = s.degenerate;
    } else {
        inv = exp2_int(127 - (int)sb);
        degenerate = false;
    }
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float x = degenerate ? 0.0f : __fmul_rn(wv[i], inv);
        v[i] = __fadd_rn(x, rv[i]);
    }
    const uint32_t codes = e2m1_pack8(v);
#pragma unroll
    for (int i = 0; i < 8; ++i) rv[i] = __fsub_rn(v[i], e2m1_value((codes >> (4 * i)) & 15u));
    const int64_t off = row * p.cols + col;
    float4* rp = reinterpret_cast<float4*>(p.residue + off);
    rp[0] = make_float4(rv[0], rv[1], rv[2], rv[3]);
    rp[1] = make_float4(rv[4], rv[5], rv[6], rv[7]);
    *reinterpret_cast<uint32_t*>(p.codes + row * (p.cols / 2) + col / 2) = codes;
}

template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sigma_delta_kernel(SigmaDeltaParams p) {
    const int64_t cpr = p.cols / 8;
    const int64_t total = p.rows * cpr;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const float s_t = (BLK == 16) ? *p.gscale : 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += 2 * stride) {
        const int64_t j = i + stride;
        const bool has2 = j < total;
        const int64_t row_a = i / cpr, col_a = (i % cpr) * 8;
        const int64_t row_b = has2 ? j / cpr : row_a, col_b = has2 ? (j % cpr) * 8 : col_a;
        const float4* wa = reinterpret_cast<const float4*>(p.w + row_a * p.cols + col_a);
        const float4* ra = reinterpret_cast<const float4*>(p.residue + row_a * p.cols + col_a);
        const float4* wb = reinterpret_cast<const float4*>(p.w + row_b * p.cols + col_b);
        const float4* rb = reinterpret_cast<const float4*>(p.residue + row_b * p.cols + col_b);
        const float4 wa0 = __ldcs(wa), wa1 = __ldcs(wa + 1), ra0 = __ldcs(ra), ra1 = __ldcs(ra + 1);
        float4 wb0 = wa0, wb1 = wa1, rb0 = ra0, rb1 = ra1;
        if (has2) { wb0 = __ldcs(wb); wb1 = __ldcs(wb + 1); rb0 = __ldcs(rb); rb1 = __ldcs(rb + 1); }
        const int64_t ca = col_a / BLK, cbk = col_b / BLK;
        const uint32_t sa = TC ? p.scales[tc_scale_offset(row_a, ca, p.catoms)] : p.scales[row_a * p.scols + ca];
        const uint32_t sbb = TC ? p.scales[tc_scale_offset(row_b, cbk, p.catoms)] : p.scales[row_b * p.scols + cbk];
        sigma_delta_chunk<BLK, TC>(p, s_t, row_a, col_a, wa0, wa1, ra0, ra1, sa);
        if (has2) sigma_delta_chunk<BLK, TC>(p, s_t, row_b, col_b, wb0, wb1, rb0, rb1, sbb);
    }
}

// ------------------------------------------------------------------ dequantize
template <int BLK, bool TC, bool OUT_BF16>
__global__ void __launch_bounds__(256) dequantize_kernel(DequantParams p) {
    const int64_t chunks_per_row = p.cols / 8;
    const int64_t total = p.rows * chunks_per_row;
    const float s_t = (BLK == 16) ? *p.gscale : 1.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / chunks_per_row;
        const int64_t col = (i % chunks_per_row) * 8;
        const uint32_t codes = *reinterpret_cast<const uint32_t*>(p.codes + row * (p.cols / 2) + col / 2);
        const int64_t c = col / BLK;
        const uint32_t byte = TC ? p.scales[tc_scale_offset(row, c, p.catoms)] : p.scales[row * p.scols + c];
        float sc;
        if (BLK == 16) sc = __fmul_rn(e4m3_value(byte), s_t);
        else sc = exp2_int((int)byte - 127);
        float o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float cv = e2m1_value((codes >> (4 * j)) & 15u);
            // (code * s_b) is exact; one rounding for the tensor scale
            o[j] = (BLK == 16) ? __fmul_rn(__fmul_rn(cv, e4m3_value(byte)), s_t) : __fmul_rn(cv, sc);
        }
        if (OUT_BF16) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * j], o[2 * j + 1]);
                w[j] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + row * p.cols + col) =
                make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            float4* op = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + row * p.cols + col);
            op[0] = make_float4(o[0], o[1], o[2], o[3]);
            op[1] = make_float4(o[4], o[5], o[6], o[7]);
        }
    }
}

// ------------------------------------------------------------------ launchers
static int grid_for(int64_t tiles, int num_sms, int per_sm) {
    int64_t cap = (int64_t)num_sms * per_sm;
    if (tiles < 1) return 1;
    return (int)(tiles < cap ? tiles : cap);
}

// Grid of exactly the CTAs that fit on the GPU at once (a persistent
// grid-stride launch), so the last wave is never partial.
template <typename K>
static int resident_grid(K kernel, int64_t tiles, int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1)
        per_sm = 4;
    return grid_for(tiles, num_sms, per_sm);
}

template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool CHAN>
static void launch_quant_one(const QuantParams& p, int64_t tiles, int num_sms, cudaStream_t st) {
    auto k = quantize_kernel<BLK, BF16, TC, RU, HAD, CHAN>;
    k<<<resident_grid(k, tiles, num_sms), 256, 0, st>>>(p);
}

template <int BLK, bool BF16, bool TC, bool RU>
static void launch_quant_mx_variants(const QuantParams& p, bool had, bool chan, int64_t tiles, int num_sms,
                                     cudaStream_t st) {
    if (had && chan) launch_quant_one<BLK, BF16, TC, RU, true, true>(p, tiles, num_sms, st);
    else if (had) launch_quant_one<BLK, BF16, TC, RU, true, false>(p, tiles, num_sms, st);
    else if (chan) launch_quant_one<BLK, BF16, TC, RU, false, true>(p, tiles, num_sms, st);
    else launch_quant_one<BLK, BF16, TC, RU, false, false>(p, tiles, num_sms, st);
}

template <int BLK, bool BF16, bool TC>
static void launch_quant_ru(const QuantParams& p, bool ru, bool had, bool chan, int64_t tiles, int num_sms,
                            cudaStream_t st) {
    if constexpr (BLK == 16) {
        if (ru) launch_quant_one<BLK, BF16, TC, true, false, false>(p, tiles, num_sms, st);
        else launch_quant_one<BLK, BF16, TC, false, false, false>(p, tiles, num_sms, st);
    } else {
        if (ru) launch_quant_mx_variants<BLK, BF16, TC, true>(p, had, chan, tiles, num_sms, st);
        else launch_quant_mx_variants<BLK, BF16, TC, false>(p, had, chan, tiles, num_sms, st);
    }
}

template <int BLK>
static void launch_quant_blk(const QuantParams& p, bool bf16, bool tc, bool ru, bool had, bool chan,
                             int64_t tiles, int num_sms, cudaStream_t st) {
    if (bf16) {
        if (tc) launch_quant_ru<BLK, true, true>(p, ru, had, chan, tiles, num_sms, st);
        else launch_quant_ru<BLK, true, false>(p, ru, had, chan, tiles, num_sms, st);
    } else {
        if (tc) launch_quant_ru<BLK, false, true>(p, ru, had, chan, tiles, num_sms, st);
        else launch_quant_ru<BLK, false, false>(p, ru, had, chan, tiles, num_sms, st);
    }
}

cudaError_t launch_quantize(const QuantParams& p, int blk, bool bf16, bool tc, bool ru, bool had,
                            bool chan, cudaStream_t st, int num_sms) {
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    const int64_t tile_c = 4 * blk;
    const int64_t tiles = ((p.rows + 127) / 128) * ((p.cols + tile_c - 1) / tile_c);
    if (blk == 16) launch_quant_blk<16>(p, bf16, tc, ru, had, chan, tiles, num_sms, st);
    else launch_quant_blk<32>(p, bf16, tc, ru, had, chan, tiles, num_sms, st);
    return cudaGetLastError();
}

cudaError_t launch_sigma_delta(const SigmaDeltaParams& p, int blk, bool tc, cudaStream_t st, int num_sms) {
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    const int64_t tiles = (p.rows * (p.cols / 8) + 511) / 512;   // CTAs of 256 threads, 2 chunks each
#define Q4_SD(B, T) { auto k = sigma_delta_kernel<B, T>; k<<<resident_grid(k, tiles, num_sms), 256, 0, st>>>(p); }
    if (blk == 16) {
        if (tc) Q4_SD(16, true) else Q4_SD(16, false)
    } else {
        if (tc) Q4_SD(32, true) else Q4_SD(32, false)
    }
#undef Q4_SD
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const DequantParams& p, int blk, bool tc, bool out_bf16, cudaStream_t st,
                              int num_sms) {
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    const int64_t chunks = p.rows * (p.cols / 8);
    const int grid = grid_for((chunks + 255) / 256, num_sms, 8);
#define Q4_DQ(B, T, O) dequantize_kernel<B, T, O><<<grid, 256, 0, st>>>(p)
    if (blk == 16) {
        if (tc) { if (out_bf16) Q4_DQ(16, true, true); else Q4_DQ(16, true, false); }
        else { if (out_bf16) Q4_DQ(16, false, true); else Q4_DQ(16, false, false); }
    } else {
        if (tc) { if (out_bf16) Q4_DQ(32, true, true); else Q4_DQ(32, true, false); }
        else { if (out_bf16) Q4_DQ(32, false, true); else Q4_DQ(32, false, false); }
    }
#undef Q4_DQ
    return cudaGetLastError();
}

}  // namespace q4
