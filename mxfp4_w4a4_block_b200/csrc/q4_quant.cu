// q4_quant.cu -- memory-bound kernels of the path: tensor amax, NVFP4 / MXFP4
// block quantization (with the optional per-channel scale and block
// Hadamard-32 of MACaQ fused in), dequantization and the first-order
// Sigma-Delta step of "Looped Transformer quantization", sec. 2.1.
//
// Work decomposition shared by quantize and Sigma-Delta: a CTA of 256 threads
// owns a tile of 128 rows x (4 * block) columns, i.e. exactly one 512-byte
// atom of the tensor-core scale layout.  Each thread owns 8 consecutive
// elements of a row (one 16-byte bf16 load, two for fp32); the 2 (NVFP4) or 4
// (MXFP4) threads of a block are neighbouring lanes and combine their amax
// (and the Hadamard stages 8 and 16) with warp shuffles.  A warp reads whole
// 128- or 256-byte row segments, so loads are fully coalesced; codes leave as
// one 32-bit store per thread (32 contiguous bytes per row per 8 lanes) and
// the scale atom is staged in shared memory and written as 512 contiguous
// bytes.  All loads of a tile are issued before any arithmetic.
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
// Eight inputs of one chunk as floats.
template <bool BF16>
struct Chunk;

template <>
struct Chunk<true> {
    uint4 raw;
    __device__ __forceinline__ void load(const void* base) { raw = __ldcs(reinterpret_cast<const uint4*>(base)); }
    __device__ __forceinline__ void zero() { raw = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void to_float(float (&v)[8]) const {
        v[0] = bf16_lo(raw.x); v[1] = bf16_hi(raw.x); v[2] = bf16_lo(raw.y); v[3] = bf16_hi(raw.y);
        v[4] = bf16_lo(raw.z); v[5] = bf16_hi(raw.z); v[6] = bf16_lo(raw.w); v[7] = bf16_hi(raw.w);
    }
};

template <>
struct Chunk<false> {
    float4 a, b;
    __device__ __forceinline__ void load(const void* base) {
        const float4* p = reinterpret_cast<const float4*>(base);
        a = __ldcs(p);
        b = __ldcs(p + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void to_float(float (&v)[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// In-register stages (strides 1, 2, 4) of the Sylvester Walsh-Hadamard
// transform over 8 consecutive elements, then the cross-lane stages 8 and 16
// with the partner lanes of the same 32-block.  `lib` is the lane's index
// inside its block (0..3).  All lanes of the warp must call this.
__device__ __forceinline__ void fwht32_warp(float (&v)[8], int lib) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int lm = 1; lm <= 2; lm <<= 1) {
        const bool upper = (lib & lm) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float p = __shfl_xor_sync(0xffffffffu, v[i], lm);
            // lower element: a + b (a = own value); upper element: a - b with
            // a = the lower partner's value and b = own value
            v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
        }
    }
}

// ------------------------------------------------------------------ quantize
template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool CHAN>
__global__ void __launch_bounds__(256) quantize_kernel(QuantParams p) {
    constexpr int TILE_C = 4 * BLK;          // columns per tile (one scale atom)
    constexpr int CPR = TILE_C / 8;          // 8-element chunks per tile row
    constexpr int ITER = 128 * CPR / 256;    // chunks per thread per tile
    constexpr int TPB = BLK / 8;             // threads per block
    constexpr int ESZ = BF16 ? 2 : 4;
    __shared__ __align__(16) uint8_t sf_atom[512];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int lib = lane & (TPB - 1);
    const int64_t tiles_c = (p.cols + TILE_C - 1) / TILE_C;
    const int64_t tiles = ((p.rows + 127) / 128) * tiles_c;
    const float s_t = (BLK == 16) ? *p.gscale : 0.0f;
    const float inv_sqrt32 = 0x1.6a09e6p-3f;   // binary32 nearest to 1/sqrt(32)
    const char* xb = reinterpret_cast<const char*>(p.x);

    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t tr = t / tiles_c, tc = t % tiles_c;
        const int64_t row0 = tr * 128, col0 = tc * TILE_C;

        Chunk<BF16> ch[ITER];
        bool valid[ITER];
#pragma unroll
        for (int it = 0; it < ITER; ++it) {
            const int q = it * 256 + tid;
            const int64_t row = row0 + q / CPR;
            const int64_t col = col0 + (q % CPR) * 8;
            valid[it] = row < p.rows && col < p.cols;
            if (valid[it]) ch[it].load(xb + (row * p.ld + col) * ESZ);
            else ch[it].zero();
        }
#pragma unroll
        for (int it = 0; it < ITER; ++it) {
            const int q = it * 256 + tid;
            const int rt = q / CPR;                   // row inside the tile
            const int cq = q % CPR;                   // chunk inside the row
            const int64_t row = row0 + rt;
            const int64_t col = col0 + cq * 8;
            float v[8];
            ch[it].to_float(v);
            if (CHAN) {
                float c[8];
                if (valid[it]) {
                    const float4* cp = reinterpret_cast<const float4*>(p.chan + col);
                    float4 c0 = __ldg(cp), c1 = __ldg(cp + 1);
                    c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w;
                    c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) c[i] = 0.0f;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], c[i]);
            }
            if (HAD) {
                fwht32_warp(v, lib);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], inv_sqrt32);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
            for (int o = 1; o < TPB; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));

            uint32_t byte;
            if (BLK == 16) {
                NvScale s = nv_scale_from_amax(amax, s_t, RU);
                byte = s.byte;
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = s.degenerate ? 0.0f : __fmul_rn(v[i], s.inv);
            } else {
                int e = mx_exponent(amax, RU);
                byte = (uint32_t)(e + 127);
                float mult = exp2_int(-e);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], mult);
            }
            uint32_t codes = e2m1_pack8(v);
            if (valid[it])
                *reinterpret_cast<uint32_t*>(p.codes + row * (p.cols / 2) + col / 2) = codes;
            if (lib == 0) {
                const int cb = cq / TPB;              // block inside the tile (0..3)
                if (TC) sf_atom[(rt & 31) * 16 + (rt >> 5) * 4 + cb] = (uint8_t)byte;
                else if (valid[it]) p.scales[row * p.scols + tc * 4 + cb] = (uint8_t)byte;
            }
        }
        if (TC) {
            __syncthreads();
            if (tid < 32) {
                uint4 w = reinterpret_cast<const uint4*>(sf_atom)[tid];
                reinterpret_cast<uint4*>(p.scales + (tr * p.catoms + tc) * 512)[tid] = w;
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------------ sigma-delta
template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sigma_delta_kernel(SigmaDeltaParams p) {
    constexpr int TILE_C = 4 * BLK;
    constexpr int CPR = TILE_C / 8;
    constexpr int ITER = 128 * CPR / 256;
    const int tid = threadIdx.x;
    const int64_t tiles_c = (p.cols + TILE_C - 1) / TILE_C;
    const int64_t tiles = ((p.rows + 127) / 128) * tiles_c;
    const float s_t = (BLK == 16) ? *p.gscale : 0.0f;

    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t tr = t / tiles_c, tc = t % tiles_c;
        const int64_t row0 = tr * 128, col0 = tc * TILE_C;
        float4 w[ITER][2], r[ITER][2];
        uint32_t sb[ITER];
        bool valid[ITER];
#pragma unroll
        for (int it = 0; it < ITER; ++it) {
            const int q = it * 256 + tid;
            const int64_t row = row0 + q / CPR;
            const int64_t col = col0 + (q % CPR) * 8;
            valid[it] = row < p.rows && col < p.cols;
            if (valid[it]) {
                const int64_t off = row * p.cols + col;
                const float4* wp = reinterpret_cast<const float4*>(p.w + off);
                const float4* rp = reinterpret_cast<const float4*>(p.residue + off);
                w[it][0] = __ldcs(wp); w[it][1] = __ldcs(wp + 1);
                r[it][0] = __ldcs(rp); r[it][1] = __ldcs(rp + 1);
                const int64_t c = col / BLK;
                sb[it] = TC ? p.scales[tc_scale_offset(row, c, p.catoms)] : p.scales[row * p.scols + c];
            }
        }
#pragma unroll
        for (int it = 0; it < ITER; ++it) {
            if (!valid[it]) continue;
            const int q = it * 256 + tid;
            const int64_t row = row0 + q / CPR;
            const int64_t col = col0 + (q % CPR) * 8;
            float inv;
            bool degenerate;
            if (BLK == 16) {
                NvScale s = nv_scale_from_byte(sb[it], s_t);
                inv = s.inv;
                degenerate = s.degenerate;
            } else {
                inv = exp2_int(127 - (int)sb[it]);
                degenerate = false;
            }
            float wv[8] = {w[it][0].x, w[it][0].y, w[it][0].z, w[it][0].w,
                           w[it][1].x, w[it][1].y, w[it][1].z, w[it][1].w};
            float rv[8] = {r[it][0].x, r[it][0].y, r[it][0].z, r[it][0].w,
                           r[it][1].x, r[it][1].y, r[it][1].z, r[it][1].w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float x = degenerate ? 0.0f : __fmul_rn(wv[i], inv);
                v[i] = __fadd_rn(x, rv[i]);
            }
            uint32_t codes = e2m1_pack8(v);
#pragma unroll
            for (int i = 0; i < 8; ++i) rv[i] = __fsub_rn(v[i], e2m1_value((codes >> (4 * i)) & 15u));
            const int64_t off = row * p.cols + col;
            float4* rp = reinterpret_cast<float4*>(p.residue + off);
            rp[0] = make_float4(rv[0], rv[1], rv[2], rv[3]);
            rp[1] = make_float4(rv[4], rv[5], rv[6], rv[7]);
            *reinterpret_cast<uint32_t*>(p.codes + row * (p.cols / 2) + col / 2) = codes;
        }
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
    const int64_t tile_c = 4 * blk;
    const int64_t tiles = ((p.rows + 127) / 128) * ((p.cols + tile_c - 1) / tile_c);
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
