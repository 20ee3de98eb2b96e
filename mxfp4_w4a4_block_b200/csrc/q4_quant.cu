// q4_quant.cu -- memory-bound kernels of the path: tensor amax, NVFP4 / MXFP4
// block quantization (with the optional per-channel scale and block
// Hadamard-32 of MACaQ fused in, and 4/6 block scaling), dequantization, the
// first-order Sigma-Delta step of "Looped Transformer quantization", sec. 2.1,
// its K-visit codebanks (sec. 2.3, 4) and the stochastic-rounding requant.
//
// The quantizer and the Sigma-Delta step are persistent producer/consumer
// kernels: one thread streams tiles into shared memory by TMA, sixteen warps
// compute, and the results leave by TMA stores (see each kernel).  amax,
// dequantize, the codebanks and SR are grid-stride streams, and the grouped
// launches walk the work units of a list of matrices grid-stride.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "q4_codec.cuh"
#include "q4_internal.h"
#include "q4_ptx.cuh"

namespace q4 {

// ------------------------------------------------------------------ amax
// out[0] = max |x_i|; out[1] = out[0] / denom, written by the last CTA to
// finish (out[1] counts the finished CTAs until then; both start at 0).
__global__ void __launch_bounds__(256) amax_kernel(const void* __restrict__ x, int64_t n, int bf16, float denom,
                                                   unsigned int* __restrict__ out) {
    float m = 0.0f;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    if (bf16) {
        const uint4* v = reinterpret_cast<const uint4*>(x);
        const int64_t nv = n / 8;
        int64_t i = tid;
        // four independent 16-byte loads in flight per thread
        for (; i + 3 * nthreads < nv; i += 4 * nthreads) {
            uint4 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) w[u] = __ldg(v + i + u * nthreads);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(ws[j])), fabsf(bf16_hi(ws[j]))));
            }
        }
        for (; i < nv; i += nthreads) {
            uint4 w = __ldg(v + i);
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
        int64_t i = tid;
        for (; i + 3 * nthreads < nv; i += 4 * nthreads) {
            float4 w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) w[u] = __ldg(v + i + u * nthreads);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                m = fmaxf(m, fmaxf(fmaxf(fabsf(w[u].x), fabsf(w[u].y)), fmaxf(fabsf(w[u].z), fabsf(w[u].w))));
        }
        for (; i < nv; i += nthreads) {
            float4 w = __ldg(v + i);
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
        if (threadIdx.x == 0) {
            atomicMax(out, __float_as_uint(m));
            __threadfence();
            if (atomicAdd(out + 1, 1u) == gridDim.x - 1) {
                // every other CTA's maximum is in out[0]
                __threadfence();
                const float amax = __uint_as_float(atomicOr(out, 0u));
                reinterpret_cast<float*>(out)[1] = __fdiv_rn(amax, denom);
            }
        }
    }
}

cudaError_t launch_amax(const void* x, int64_t n, bool bf16, float denom, float* d_out,
                        cudaStream_t st, int num_sms) {
    cudaError_t e = cudaMemsetAsync(d_out, 0, 2 * sizeof(float), st);
    if (e != cudaSuccess) return e;
    if (n > 0) {
        int64_t vec = bf16 ? n / 8 : n / 4;
        int64_t blocks = (vec + 255) / 256;
        int grid = (int)(blocks < (int64_t)num_sms * 8 ? (blocks > 0 ? blocks : 1) : (int64_t)num_sms * 8);
        amax_kernel<<<grid, 256, 0, st>>>(x, n, bf16 ? 1 : 0, denom, reinterpret_cast<unsigned int*>(d_out));
    }
    // n = 0: both outputs stay 0 (= 0 / denom)
    return cudaGetLastError();
}

// ------------------------------------------------------------------ helpers
// ------------------------------------------------------------------ quantize
// Persistent, one CTA per SM.  A tile is ROWS rows x one scale-atom column
// (4 blocks along the row), so the tile's scales are whole 512-byte atoms of
// the tensor-core layout.  One producer thread streams tiles into a ring of
// shared-memory stages with TMA (128-byte-wide boxes, 128-byte swizzle, zero
// fill outside the tensor); 16 consumer warps give each thread whole blocks
// (the scale rule, the Hadamard rotation and the code packing stay in
// registers), a warp taking 32 consecutive rows of one block column so its
// swizzled shared-memory reads are conflict-free.  Codes and scale atoms are
// staged in shared memory (three staging buffers) and a store warp sends them
// out by TMA / bulk stores; the consumer warps hand a finished buffer to it
// through an mbarrier and go straight on to the next tile, so no consumer
// ever waits on a CTA-wide barrier or on a store.
namespace qz {
constexpr int CONSUMER_WARPS = 16;
constexpr int CONSUMERS = 32 * CONSUMER_WARPS;
constexpr int THREADS = CONSUMERS + 64;          // + the producer warp and the store warp
constexpr int IN_BYTES = 160 * 1024;             // input stages
constexpr int NBUF = 3;                          // output staging buffers
}  // namespace qz

template <int BLK, bool BF16>
struct QzGeom {
    static constexpr int ESZ = BF16 ? 2 : 4;
    static constexpr int ACOL = 4 * BLK * ESZ;                 // input bytes of one atom column per row
    static constexpr int NBOX = ACOL / 128;                    // 128-byte TMA boxes per row
    static constexpr int ROWS = (32768 / ACOL) < 128 ? 128 : 32768 / ACOL;
    static constexpr int STAGE = ROWS * ACOL;
    static constexpr int NSTAGE = qz::IN_BYTES / STAGE;
    static constexpr int CODE_TILE = ROWS * 2 * BLK;            // codes of a tile, [ROWS][2*BLK] bytes
    static constexpr int SF_TILE = ROWS * 4;                    // ROWS/128 scale atoms
    static constexpr int BPT = ROWS * 4 / qz::CONSUMERS;        // blocks per consumer thread
    static constexpr int CHUNKS = BLK * ESZ / 16;               // 16-byte chunks per block
    static constexpr int PER = 16 / ESZ;                        // values per chunk
    static constexpr int TAB_OFF = NSTAGE * STAGE + qz::NBUF * (CODE_TILE + SF_TILE);
    static constexpr int BAR_OFF = TAB_OFF + 1024;              // after the 128-entry (S, 1/S) table
    static constexpr int SMEM = BAR_OFF + 256 + 1024;           // + barriers, alignment slack
    static_assert(BPT >= 1 && ROWS % 128 == 0 && ROWS <= 256, "tile geometry");
};

// One candidate of 4/6 block scaling: the rounded-up E4M3 scale mapping the
// block max to `target` (6 or 4), its table entry (S, y) with S = dec(s_b) *
// s_t in binary32 (y NaN: a degenerate scale, every code +0), and the block's
// codes of x / S.
struct Nv46Cand {
    uint32_t byte, w[2];
    float S, y;
};

__device__ __forceinline__ Nv46Cand nv46_candidate(const float (&v)[16], const NvCtx& c, float amax, float target) {
    Nv46Cand k;
    k.byte = c.st_ok ? e4m3_ru(__fdiv_rn(amax, __fmul_rn(target, c.s_t))) : 0u;
    const float2 sy = c.tab[k.byte];
    k.S = sy.x;
    k.y = sy.y;
    nv_codes16(v, sy, amax, k.w);
    return k;
}

// The candidate's sum of squared errors sum_j (x_j - dec_j * S)^2 in the
// input's units, accumulated in binary64 in element order (x - dec * S is
// exact there), explicitly rounded so that no fused multiply-add changes it;
// a degenerate scale gives sum_j x_j^2.
__device__ __forceinline__ double nv46_sse_f64(const float (&v)[16], const Nv46Cand& k) {
    double err = 0.0;
    if (k.y != k.y) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const double d = (double)v[i];
            err = __dadd_rn(err, __dmul_rn(d, d));
        }
        return err;
    }
    const double S = (double)k.S;
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double d = __dsub_rn((double)v[8 * g + i], __dmul_rn((double)e2m1_value((k.w[g] >> (4 * i)) & 15u), S));
            err = __dadd_rn(err, __dmul_rn(d, d));
        }
    return err;
}

// The same sum estimated in binary32: e_j = fma(-dec_j, S, x_j) is x_j -
// dec_j * S correctly rounded, each square is added by one fma into one of
// two partial sums.  While everything stays in the normal range the estimate
// is within 20 * 2^-24 < 2^-19.6 of the exact sum, relatively (the square of
// e_j adds at most 2^-23, each of the <= 9 additions into a partial sum and
// the final one at most 2^-24 of what they add).  A non-finite scale gives a
// NaN estimate.
__device__ __forceinline__ float nv46_sse_f32(const float (&v)[16], const Nv46Cand& k) {
    const float S = k.y != k.y ? 0.0f : k.S;
    float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        uint32_t o[4];
        e2m1x8_to_bf16(k.w[g], o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float d0 = __uint_as_float(o[i] << 16), d1 = __uint_as_float(o[i] & 0xFFFF0000u);
            const float e0 = __fmaf_rn(-d0, S, v[8 * g + 2 * i]);
            const float e1 = __fmaf_rn(-d1, S, v[8 * g + 2 * i + 1]);
            acc0 = __fmaf_rn(e0, e0, acc0);
            acc1 = __fmaf_rn(e1, e1, acc1);
        }
    }
    return __fadd_rn(acc0, acc1);
}

// 4/6 block scaling of one NVFP4 block: the candidate with the smaller
// binary64 squared error (ties: the 6 candidate).  Equal scale bytes give
// equal codes, hence a tie.  Otherwise the binary32 estimates decide when
// they differ by more than 2^-16 of their sum and both lie in [2^-100, inf):
// each is within 2^-19.6 of its exact sum (the 2^-100 floor keeps the
// subnormal parts of the squares below 2^-45 of the sum), so the exact sums,
// and the binary64 sums (within 2^-48 of them), are ordered the same way.
// Every other block takes the binary64 sums.
__device__ __forceinline__ void nv_block46(const float (&v)[16], const NvCtx& c, uint32_t& byte, uint32_t (&w)[2]) {
    const float amax = amax_tree<16>(v);
    const Nv46Cand k6 = nv46_candidate(v, c, amax, 6.0f);
    const Nv46Cand k4 = nv46_candidate(v, c, amax, 4.0f);
    bool four = false;
    if (k6.byte != k4.byte) {
        const float e6 = nv46_sse_f32(v, k6), e4 = nv46_sse_f32(v, k4);
        const float lo = fminf(e6, e4), hi = fmaxf(e6, e4);
        const bool sure = e6 == e6 && e4 == e4 && hi < INFINITY && lo >= 0x1p-100f &&
                          __fsub_rn(hi, lo) > __fmul_rn(0x1p-16f, __fadd_rn(hi, lo));
        four = sure ? e4 < e6 : nv46_sse_f64(v, k4) < nv46_sse_f64(v, k6);
    }
    byte = four ? k4.byte : k6.byte;
    w[0] = four ? k4.w[0] : k6.w[0];
    w[1] = four ? k4.w[1] : k6.w[1];
}

// One MXFP4 block of 32 with the optional per-column multiplier and block
// Hadamard-32.  Values are held as pairs P_j = (v_j, v_{j+16}), so the
// butterflies of strides 1, 2, 4 and 8 (pairs j, j+h with both j, j+h < 16)
// are packed f32x2 operations; stride 16 pairs the two halves of each P_j.
// Channel factors come preloaded in `cw` (PRE) or are read from `chan`
// (nullptr: none).
template <bool RU, bool HAD, bool CHAN, bool PRE>
__device__ __forceinline__ void mx_block(const float (&v)[32], const float4 (&cw)[8], const float* chan, uint32_t& byte,
                                         uint32_t (&w)[4]) {
    float2 P[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) P[j] = make_float2(v[j], v[j + 16]);
    if (CHAN && (PRE || chan != nullptr)) {
        const float4* cp = reinterpret_cast<const float4*>(chan);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            // the products feed the butterfly adds: scalar, never fused
            const float4 lo = PRE ? cw[q] : __ldg(cp + q), hi = PRE ? cw[4 + q] : __ldg(cp + 4 + q);
            P[4 * q] = mul2_sep_rn(P[4 * q], make_float2(lo.x, hi.x));
            P[4 * q + 1] = mul2_sep_rn(P[4 * q + 1], make_float2(lo.y, hi.y));
            P[4 * q + 2] = mul2_sep_rn(P[4 * q + 2], make_float2(lo.z, hi.z));
            P[4 * q + 3] = mul2_sep_rn(P[4 * q + 3], make_float2(lo.w, hi.w));
        }
    }
    if constexpr (HAD) {
#pragma unroll
        for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if ((j & h) == 0) {
                    const float2 a = P[j], b = P[j + h];
                    P[j] = add2_rn(a, b);
                    P[j + h] = sub2_rn(a, b);
                }
            }
        }
        const float2 isq = make_float2(0x1.6a09e6p-3f, 0x1.6a09e6p-3f);   // binary32 nearest to 1/sqrt(32)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float a = P[j].x, b = P[j].y;
            P[j] = mul2_rn(make_float2(__fadd_rn(a, b), __fsub_rn(a, b)), isq);
        }
    }
    const float amax = amax_tree<32>(reinterpret_cast<const float*>(P));
    const int e = mx_exponent(amax, RU);
    byte = (uint32_t)(e + 127);
    const float m = exp2_int(-e);
    const float2 mm = make_float2(m, m);
#pragma unroll
    for (int j = 0; j < 16; ++j) P[j] = mul2_rn(P[j], mm);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        // codes of elements 8g..8g+7: P[8g..8g+7].x for g < 2, P[8(g-2)..].y otherwise
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = g < 2 ? P[8 * g + i].x : P[8 * (g - 2) + i].y;
        w[g] = e2m1_pack8(q);
    }
}

template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool CHAN, bool S46 = false, bool AMAX = false>
__global__ void __launch_bounds__(qz::THREADS, 1)
    quantize_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC, QuantParams p,
                    int codes_tma) {
    using G = QzGeom<BLK, BF16>;
    using namespace qz;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* cbuf = smem + G::NSTAGE * G::STAGE;
    uint8_t* sbuf = cbuf + NBUF * G::CODE_TILE;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::BAR_OFF);
    uint64_t* empty = full + G::NSTAGE;
    uint64_t* cfull = empty + G::NSTAGE;     // staging buffer written by every consumer warp
    uint64_t* cfree = cfull + NBUF;          // staging buffer read out by its stores
    float2* nv_tab = reinterpret_cast<float2*>(smem + G::TAB_OFF);  // NVFP4: (S, 1/S) per scale byte

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < G::NSTAGE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CONSUMER_WARPS);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&cfull[b], CONSUMER_WARPS);
            mbar_init(&cfree[b], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int64_t tiles_c = p.catoms;
    const int64_t tiles = ((p.rows + G::ROWS - 1) / G::ROWS) * tiles_c;
    // This CTA's tiles are blockIdx.x + i * gridDim.x, i < n_my.  With AMAX the
    // launch makes two passes over them: the first only folds |x| into the
    // tensor maximum, the second quantizes, in reverse order, so that the tiles
    // read last (the likeliest to be still in L2) come first.
    const int64_t n_my = tiles > blockIdx.x ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    auto quant_tile = [&](int64_t i) -> int64_t {
        return (int64_t)blockIdx.x + (AMAX ? (n_my - 1 - i) : i) * (int64_t)gridDim.x;
    };

    if (warp == CONSUMER_WARPS) {
        // ---- producer
        if (lane == 0) {
            tma_prefetch_desc(&tmX);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_phase[G::NSTAGE];
            bool issued[G::NSTAGE];
            for (int s = 0; s < G::NSTAGE; ++s) issued[s] = false, last_phase[s] = 0;
            // the loads need no tensor scale, so with AMAX they run straight on
            // from the first pass into the second while the grid meets
            const int64_t iters = (AMAX ? 2 : 1) * n_my;
            for (int64_t it = 0; it < iters; ++it) {
                const int64_t t = (AMAX && it < n_my) ? (int64_t)blockIdx.x + it * (int64_t)gridDim.x
                                                      : quant_tile(AMAX ? it - n_my : it);
                // on time-out stop issuing: the consumers then time out on `full`
                if (!mbar_wait(&empty[stage], phase ^ 1)) break;
                // failure-detection test (Q4_INJECT_STALL): the first tile's stage
                // is never filled, so the consumers' bounded wait on it runs out
                if (!(p.inject_stall && it == 0)) {
                    mbar_arrive_expect_tx(&full[stage], G::STAGE);
                    const int64_t tr = t / tiles_c, tc = t % tiles_c;
                    uint8_t* dst = smem + stage * G::STAGE;
#pragma unroll
                    for (int b = 0; b < G::NBOX; ++b)
                        tma_load_2d(dst + b * (G::ROWS * 128), &tmX, &full[stage],
                                    (int32_t)(tc * 4 * BLK + b * (128 / G::ESZ)), (int32_t)(tr * G::ROWS));
                    issued[stage] = true;
                    last_phase[stage] = phase;
                }
                if (++stage == G::NSTAGE) { stage = 0; phase ^= 1; }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int s = 0; s < G::NSTAGE; ++s)
                if (issued[s]) mbar_wait(&full[s], last_phase[s]);
        }
        return;
    }
    if (warp == CONSUMER_WARPS + 1) {
        // ---- store warp: sends each finished tile's codes and scale atoms
        if (lane == 0) {
            if (codes_tma) tma_prefetch_desc(&tmC);
            const int64_t bands = (p.rows + 127) / 128;
            int buf = 0;
            uint32_t bphase = 0;
            for (int64_t i = 0; i < n_my; ++i) {
                const int64_t t = quant_tile(i);
                // on time-out stop: nothing of this tile is complete
                if (!mbar_wait(&cfull[buf], bphase)) break;
                const int64_t tr = t / tiles_c, tc = t % tiles_c;
                const int64_t row0 = tr * G::ROWS, col0 = tc * 4 * BLK;
                uint8_t* cb = cbuf + buf * G::CODE_TILE;
                uint8_t* fb = sbuf + buf * G::SF_TILE;
                if (codes_tma) tma_store_2d(&tmC, cb, (int32_t)(col0 / 2), (int32_t)row0);
                if (TC) {
#pragma unroll
                    for (int a = 0; a < G::ROWS / 128; ++a) {
                        const int64_t band = row0 / 128 + a;
                        if (band < bands) bulk_store(p.scales + (band * p.catoms + tc) * 512, fb + a * 512, 512u);
                    }
                }
                bulk_commit_group();
                // the consumers may overwrite the buffer once its stores have read it
                bulk_wait_read_all();
                mbar_arrive(&cfree[buf]);
                if (++buf == NBUF) { buf = 0; bphase ^= 1; }
            }
            bulk_wait_all();
        }
        return;
    }

    // ---- consumers
    int stage = 0, buf = 0;
    uint32_t phase = 0, bphase = 0;
    // this thread's BPT blocks of a landed stage: the raw 16-byte chunks
    // (shared-memory loads), then as floats
    using Raw = uint4[G::BPT][G::CHUNKS];
    auto load_raw = [&](const uint8_t* sb, Raw& raw) {
#pragma unroll
        for (int k = 0; k < G::BPT; ++k) {
            const int b = tid + k * CONSUMERS;
            const int j = b / G::ROWS, r = b % G::ROWS;
            const int jo = j * BLK * G::ESZ;
            const uint8_t* rowp = sb + (jo >> 7) * (G::ROWS * 128) + r * 128;
            const int o16 = (jo & 127) >> 4;
#pragma unroll
            for (int c = 0; c < G::CHUNKS; ++c)
                raw[k][c] = *reinterpret_cast<const uint4*>(rowp + (((o16 + c) ^ (r & 7)) << 4));
        }
    };
    auto unpack = [&](const Raw& raw, float (&v)[G::BPT][BLK]) {
#pragma unroll
        for (int k = 0; k < G::BPT; ++k)
#pragma unroll
            for (int c = 0; c < G::CHUNKS; ++c) {
                const uint4 w = raw[k][c];
                float* d = &v[k][c * G::PER];
                if (BF16) {
                    d[0] = bf16_lo(w.x); d[1] = bf16_hi(w.x); d[2] = bf16_lo(w.y); d[3] = bf16_hi(w.y);
                    d[4] = bf16_lo(w.z); d[5] = bf16_hi(w.z); d[6] = bf16_lo(w.w); d[7] = bf16_hi(w.w);
                } else {
                    d[0] = __uint_as_float(w.x); d[1] = __uint_as_float(w.y);
                    d[2] = __uint_as_float(w.z); d[3] = __uint_as_float(w.w);
                }
            }
    };
    auto read_blocks = [&](const uint8_t* sb, float (&v)[G::BPT][BLK]) {
        Raw raw;
        load_raw(sb, raw);
        unpack(raw, v);
    };

    // With AMAX the tensor scale comes first: the first pass folds every
    // landed tile's |x| into this thread's maximum (zero-filled parts outside
    // the tensor add nothing), each CTA adds its maximum to out[0] (non-negative
    // floats order like their bit patterns) and arrives on out[2]; once all
    // CTAs have arrived (a bounded wait: the launch is cooperative, so all are
    // resident) each computes s_t = amax / denom itself and CTA 0 stores it in
    // out[1].  The producer keeps the ring full meanwhile.
    float s_t_dyn = 0.0f;
    if constexpr (AMAX) {
        __shared__ float red[CONSUMER_WARPS];
        __shared__ float s_shared;
        __shared__ int go;
        float m = 0.0f;
        bool ok = true;
        for (int64_t i = 0; i < n_my; ++i) {
            if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
            float v[G::BPT][BLK];
            read_blocks(smem + stage * G::STAGE, v);
#pragma unroll
            for (int k = 0; k < G::BPT; ++k) m = fmaxf(m, amax_tree<BLK>(v[k]));
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == G::NSTAGE) { stage = 0; phase ^= 1; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp] = ok ? m : -1.0f;
        named_barrier(1, CONSUMERS);
        if (tid == 0) {
            float b = 0.0f;
            bool all = true;
            for (int w = 0; w < CONSUMER_WARPS; ++w) {
                all = all && red[w] >= 0.0f;
                b = fmaxf(b, red[w]);
            }
            if (all) {
                atomicMax(p.amax_out, __float_as_uint(b));
                __threadfence();
                atomicAdd(p.amax_out + 2, 1u);
                const long long t0 = clock64(), limit = g_wait_limit;
                while (ld_acquire_gpu(p.amax_out + 2) < gridDim.x) {
                    if (clock64() - t0 > limit) {
                        atomicOr(&g_device_error, kErrTimeout);
                        all = false;
                        break;
                    }
                }
            }
            if (all) {
                const float amax = __uint_as_float(ld_acquire_gpu(p.amax_out));
                s_shared = __fdiv_rn(amax, p.denom);
                if (blockIdx.x == 0) reinterpret_cast<float*>(p.amax_out)[1] = s_shared;
            }
            go = all ? 1 : 0;
        }
        named_barrier(1, CONSUMERS);
        // without a tensor scale the consumers stop; the producer and the store
        // warp then run out their bounded waits and leave
        if (!go) return;
        s_t_dyn = s_shared;
    }

    NvCtx sc;
    if constexpr (BLK == 16) {
        const float s_t = AMAX ? s_t_dyn : *p.gscale;
        sc = nv_ctx(s_t, nv_tab);
        nv_fill_table(s_t, nv_tab, tid, CONSUMERS);
        named_barrier(1, CONSUMERS);
    }
    const int64_t crow = p.cols / 2;           // bytes of codes per row
    // a consumer warp whose wait times out stops; every other role then
    // times out in turn on the barriers that warp no longer arrives on
    for (int64_t i = 0; i < n_my; ++i) {
        const int64_t t = quant_tile(i);
        const int64_t tr = t / tiles_c, tc = t % tiles_c;
        const int64_t row0 = tr * G::ROWS, col0 = tc * 4 * BLK;
        // MXFP4 channel factors of this thread's blocks (1 outside the
        // tensor); for bf16 input they are loaded before the tile lands so
        // their latency overlaps the wait (fp32 input has no registers to
        // spare: there they are read inside the block step)
        constexpr bool PRE = BLK == 32 && CHAN && BF16;
        float4 cw[G::BPT][8];
        if constexpr (PRE) {
#pragma unroll
            for (int k = 0; k < G::BPT; ++k) {
                const int64_t col = col0 + ((tid + k * CONSUMERS) / G::ROWS) * BLK;
                const float4* cp = reinterpret_cast<const float4*>(p.chan + col);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    cw[k][q] = col < p.cols ? __ldg(cp + q) : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
            }
        }
        if (!mbar_wait(&full[stage], phase)) break;
        float v[G::BPT][BLK];
        read_blocks(smem + stage * G::STAGE, v);
        // the stage is handed back only once its values have been used (below):
        // a lane's shared-memory loads may still be in flight after __syncwarp,
        // and the refill must not overtake them
        const int read_stage = stage;
        if (++stage == G::NSTAGE) { stage = 0; phase ^= 1; }
        if (!mbar_wait(&cfree[buf], bphase ^ 1)) break;

        uint8_t* cb = cbuf + buf * G::CODE_TILE;
        uint8_t* fb = sbuf + buf * G::SF_TILE;
        // NVFP4 (RN / RU): all of this thread's blocks at once
        uint32_t nbyte[G::BPT], nw[G::BPT][2];
        if constexpr (BLK == 16 && !S46) nv_blocks<RU, G::BPT>(reinterpret_cast<const float(&)[G::BPT][16]>(v), sc,
                                                                 nbyte, nw);
#pragma unroll
        for (int k = 0; k < G::BPT; ++k) {
            const int b = tid + k * CONSUMERS;
            const int j = b / G::ROWS, r = b % G::ROWS;
            const int64_t row = row0 + r, col = col0 + j * BLK;
            uint32_t byte;
            uint32_t w[BLK / 8];
            if constexpr (BLK == 16) {
                if constexpr (S46) {
                    nv_block46(v[k], sc, byte, w);
                } else {
                    byte = nbyte[k];
                    w[0] = nw[k][0];
                    w[1] = nw[k][1];
                }
            } else {
                const float* chan = (CHAN && col < p.cols) ? p.chan + col : nullptr;
                mx_block<RU, HAD, CHAN, PRE>(v[k], cw[k], chan, byte, w);
            }
            const bool inside = row < p.rows && col < p.cols;
            if (codes_tma) {
                uint8_t* dst = cb + r * (2 * BLK) + j * (BLK / 2);
                if constexpr (BLK == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            } else if (inside) {
                uint8_t* dst = p.codes + row * crow + col / 2;
                if constexpr (BLK == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
                else *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (TC) fb[(r >> 7) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + j] = (uint8_t)byte;
            else if (inside) p.scales[row * p.scols + tc * 4 + j] = (uint8_t)byte;
        }
        // this warp's part of the staging buffer goes to the store warp, and the
        // input stage (every value of it now used) back to the producer
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&empty[read_stage]);
            mbar_arrive(&cfull[buf]);
        }
        if (++buf == NBUF) { buf = 0; bphase ^= 1; }
    }
}

// ------------------------------------------------------------------ sigma-delta
// Persistent, one CTA per SM, the same producer / consumer split as the
// quantizer.  A tile is 32 rows x 128 weights; TMA brings the tile of w and of
// the residue r into one shared-memory stage, together with the tile's scale
// atoms when the scales are in the tensor-core layout (a bulk copy, so no
// consumer waits on a global load), each consumer thread updates 4 weights
// per row it owns (a warp covers one 512-byte row: conflict-free), writes the
// new residue over the old one in the stage and its 4 codes into a staging
// buffer, and one thread sends both tiles back with TMA stores.  The stage is
// handed back to the producer once its residue store has read it.
namespace sdk {
constexpr int CONSUMER_WARPS = 16;
constexpr int CONSUMERS = 32 * CONSUMER_WARPS;
constexpr int THREADS = CONSUMERS + 32;
constexpr int ROWS = 32;
constexpr int COLS = 128;
constexpr int HALF = ROWS * COLS * 4;            // w (or r) of one tile, 16 KB
constexpr int SF_BYTES = 1024;                   // up to two scale atoms (tensor-core layout)
constexpr int STAGE = 2 * HALF + SF_BYTES;
constexpr int NSTAGE = 5;
constexpr int CODE_TILE = ROWS * COLS / 2;       // 2 KB
constexpr int NBUF = 3;
constexpr int TAB_OFF = NSTAGE * STAGE + NBUF * CODE_TILE;   // 256-entry (S, 1/S) table
constexpr int BAR_OFF = TAB_OFF + 2048;
constexpr int SMEM = BAR_OFF + 256 + 1024;
constexpr int GPT = ROWS * COLS / 4 / CONSUMERS; // 4-weight groups per thread per tile
}  // namespace sdk

template <int BLK, bool TC>
__global__ void __launch_bounds__(sdk::THREADS, 1)
    sigma_delta_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmR,
                       const __grid_constant__ CUtensorMap tmC, SigmaDeltaParams p, int codes_tma) {
    using namespace sdk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* cbuf = smem + NSTAGE * STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
    uint64_t* empty = full + NSTAGE;
    // consumer abort flags, indexed by tile-iteration parity: written before the
    // per-tile consumer barrier, read after it, so every consumer takes the
    // same decision
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NSTAGE);
    float2* sc_tab = reinterpret_cast<float2*>(smem + TAB_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        abort_flag[0] = 0;
        abort_flag[1] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int64_t tiles_c = (p.cols + COLS - 1) / COLS;
    const int64_t tiles = ((p.rows + ROWS - 1) / ROWS) * tiles_c;

    if (warp == CONSUMER_WARPS) {
        if (lane == 0) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmR);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_phase[NSTAGE];
            bool issued[NSTAGE];
            for (int s = 0; s < NSTAGE; ++s) issued[s] = false, last_phase[s] = 0;
            constexpr int ATOMS = COLS / BLK / 4;          // atom columns per tile: 2 (NVFP4) or 1 (MXFP4)
            for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
                if (!mbar_wait(&empty[stage], phase ^ 1)) break;
                const int64_t tc = t % tiles_c, tr = t / tiles_c;
                const int32_t c0 = (int32_t)(tc * COLS), r0 = (int32_t)(tr * ROWS);
                int64_t na = 0;
                if (TC) {
                    na = p.catoms - tc * ATOMS;
                    na = na < ATOMS ? na : ATOMS;
                }
                mbar_arrive_expect_tx(&full[stage], 2 * HALF + (uint32_t)na * 512u);
                tma_load_2d(smem + stage * STAGE, &tmW, &full[stage], c0, r0);
                tma_load_2d(smem + stage * STAGE + HALF, &tmR, &full[stage], c0, r0);
                if (TC)
                    bulk_load(smem + stage * STAGE + 2 * HALF,
                              p.scales + (((int64_t)r0 >> 7) * p.catoms + tc * ATOMS) * 512, (uint32_t)na * 512u,
                              &full[stage]);
                issued[stage] = true;
                last_phase[stage] = phase;
                if (++stage == NSTAGE) { stage = 0; phase ^= 1; }
            }
            for (int s = 0; s < NSTAGE; ++s)
                if (issued[s]) mbar_wait(&full[s], last_phase[s]);
        }
        return;
    }

    // per scale byte: (S, y) of NvScale (NVFP4; y NaN marks a degenerate scale,
    // whose weights normalise to +0), or (2^e, 2^-e) (MXFP4: dividing by 2^e is
    // the exact multiplication by 2^-e)
    for (int bb = tid; bb < 256; bb += CONSUMERS) {
        if (BLK == 16) {
            const NvScale r = nv_scale_of((uint32_t)(bb & 0x7F), *p.gscale);
            sc_tab[bb] = make_float2(r.S, r.y);
        } else {
            sc_tab[bb] = make_float2(exp2_int(bb - 127), exp2_int(127 - bb));
        }
    }
    named_barrier(1, CONSUMERS);
    const int64_t crow = p.cols / 2;
    int stage = 0, buf = 0, prev_stage = 0;
    uint32_t phase = 0, it = 0;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
        const int64_t row0 = (t / tiles_c) * ROWS, col0 = (t % tiles_c) * COLS;
        if (!mbar_wait(&full[stage], phase)) abort_flag[it & 1] = 1;
        uint8_t* sw = smem + stage * STAGE;
        uint8_t* cb = cbuf + buf * CODE_TILE;
#pragma unroll
        for (int k = 0; k < GPT; ++k) {
            const int g = tid + k * CONSUMERS;
            const int r = g >> 5, q = g & 31;
            const int64_t row = row0 + r, col = col0 + 4 * q;
            const bool inside = row < p.rows && col < p.cols;
            const float4 w4 = *reinterpret_cast<const float4*>(sw + r * 512 + q * 16);
            float4* rp = reinterpret_cast<float4*>(sw + HALF + r * 512 + q * 16);
            const float4 r4 = *rp;
            uint32_t sb = 0;
            if (inside) {
                if (TC) {
                    // atom q / (4 * BLK / 16) of the tile, byte (r0 + r) % 32 * 16 + (r0 / 32) % 4 * 4 + c % 4
                    const int c = (4 * q) / BLK;
                    sb = sw[2 * HALF + (c >> 2) * 512 + (int)(row & 31) * 16 + (int)((row >> 5) & 3) * 4 + (c & 3)];
                } else {
                    sb = __ldg(p.scales + row * p.scols + col / BLK);
                }
            }
            const float2 sy = sc_tab[sb];
            float2 x01, x23;
            if (BLK == 32) {
                x01 = mul2_sep_rn(make_float2(w4.x, w4.y), make_float2(sy.y, sy.y));   // feeds an add
                x23 = mul2_sep_rn(make_float2(w4.z, w4.w), make_float2(sy.y, sy.y));
            } else if (sy.y != sy.y) {
                x01 = make_float2(0.0f, 0.0f);
                x23 = x01;
            } else {
                const float4 x = quot4_rn(w4, sy.x, -sy.x, sy.y);
                x01 = make_float2(x.x, x.y);
                x23 = make_float2(x.z, x.w);
            }
            const float2 v01 = add2_rn(x01, make_float2(r4.x, r4.y));
            const float2 v23 = add2_rn(x23, make_float2(r4.z, r4.w));
            const uint32_t codes = e2m1_pack4(v01.x, v01.y, v23.x, v23.y);
            const float2 r01 = sub2_rn(v01, e2m1x2_value(codes & 0xFFu));
            const float2 r23 = sub2_rn(v23, e2m1x2_value(codes >> 8));
            *rp = make_float4(r01.x, r01.y, r23.x, r23.y);
            if (codes_tma) *reinterpret_cast<uint16_t*>(cb + r * (COLS / 2) + q * 2) = (uint16_t)codes;
            else if (inside) *reinterpret_cast<uint16_t*>(p.codes + row * crow + col / 2) = (uint16_t)codes;
        }
        fence_proxy_async_smem();
        named_barrier(1, CONSUMERS);
        if (tid == 0) {
            tma_store_2d(&tmR, sw + HALF, (int32_t)col0, (int32_t)row0);
            if (codes_tma) tma_store_2d(&tmC, cb, (int32_t)(col0 / 2), (int32_t)row0);
            bulk_commit_group();
            bulk_wait_read_1();
            // the previous tile's residue store has read its stage: refill it
            if (it > 0) mbar_arrive(&empty[prev_stage]);
            prev_stage = stage;
        }
        if (abort_flag[it & 1]) break;
        if (++stage == NSTAGE) { stage = 0; phase ^= 1; }
        if (++buf == NBUF) buf = 0;
    }
    if (tid == 0) bulk_wait_all();
}

// ------------------------------------------------------------------ sigma-delta codebanks
// The K-visit Sigma-Delta chain from r_0 = 0 in one pass ("Looped Transformer
// quantization", sec. 2.3: the tail visits restart a chain of length K and
// use its codes in reverse order; sec. 4: the codes are stored as K
// codebanks).  Each thread owns 8 consecutive weights: it reads them and their
// block scale once, runs the K visits with the residue in registers, and
// writes visit k's 4 code bytes into bank k (a warp writes 128 contiguous
// bytes per bank).  Optionally the final residue r_K is stored.
// Per-unit steps below are shared by the single-matrix and the grouped
// launches.  A unit is 8 consecutive weights of a row: u = row * (cols / 8) +
// col / 8.  Each step is split into the unit's loads (`load8`) and its
// arithmetic and stores (`*_finish`), so that a grouped launch can issue the
// next unit's loads before the current unit's arithmetic.  P is
// SigmaDeltaParams or GroupItem.
struct In8 {
    float4 w0, w1, r0, r1;   // weights; residue (Sigma-Delta step only)
    uint32_t sb;             // the unit's block scale byte
};

template <int BLK, bool TC, bool RES, class P>
__device__ __forceinline__ void load8(const P& p, int64_t u, In8& in) {
    const int64_t cpr = p.cols / 8;
    const int64_t row = u / cpr, col = (u % cpr) * 8;
    const float4* wp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.w) + row * p.cols + col);
    in.w0 = __ldcs(wp);
    in.w1 = __ldcs(wp + 1);
    if constexpr (RES) {
        const float4* rp = reinterpret_cast<const float4*>(p.residue + row * p.cols + col);
        in.r0 = __ldcs(rp);
        in.r1 = __ldcs(rp + 1);
    }
    const int64_t c = col / BLK;
    in.sb = TC ? p.scales[tc_scale_offset(row, c, p.catoms)] : p.scales[row * p.scols + c];
}

// The unit's 8 weights divided by their block scale, as pairs: x = w / S with
// S = dec(s_b) s_t (NVFP4; all +0 for a degenerate scale), or w * 2^-e
// (MXFP4, the exact quotient by 2^e).
template <int BLK>
__device__ __forceinline__ void scaled8(const In8& in, float s_t, float2 (&x)[4]) {
    const float wv[8] = {in.w0.x, in.w0.y, in.w0.z, in.w0.w, in.w1.x, in.w1.y, in.w1.z, in.w1.w};
    if (BLK == 16) {
        const NvScale sc = nv_scale_of(in.sb, s_t);
        if (sc.degenerate) {
#pragma unroll
            for (int j = 0; j < 4; ++j) x[j] = make_float2(0.0f, 0.0f);
        } else {
            const float4 a = quot4_rn(in.w0, sc.S, -sc.S, sc.y), b = quot4_rn(in.w1, sc.S, -sc.S, sc.y);
            x[0] = make_float2(a.x, a.y);
            x[1] = make_float2(a.z, a.w);
            x[2] = make_float2(b.x, b.y);
            x[3] = make_float2(b.z, b.w);
        }
    } else {
        const float m = exp2_int(127 - (int)in.sb);
        const float2 mm = make_float2(m, m);
        // the products feed adds: scalar, never fused
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = mul2_sep_rn(make_float2(wv[2 * j], wv[2 * j + 1]), mm);
    }
}

template <int BLK, class P>
__device__ __forceinline__ void banks_finish(const P& p, int64_t u, const In8& in, float s_t, int visits,
                                             int64_t bank_bytes, float* r_out) {
    const int64_t cpr = p.cols / 8;
    const int64_t row = u / cpr, col = (u % cpr) * 8;
    float2 x[4];
    scaled8<BLK>(in, s_t, x);
    float2 r[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                   make_float2(0.0f, 0.0f)};
    uint8_t* dst = p.codes + row * (p.cols / 2) + col / 2;
    for (int k = 0; k < visits; ++k) {
        float2 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = add2_rn(x[j], r[j]);
        const uint32_t codes = e2m1_pack4(v[0].x, v[0].y, v[1].x, v[1].y) |
                               (e2m1_pack4(v[2].x, v[2].y, v[3].x, v[3].y) << 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) r[j] = sub2_rn(v[j], e2m1x2_value((codes >> (8 * j)) & 0xFFu));
        __stcs(reinterpret_cast<unsigned int*>(dst + (int64_t)k * bank_bytes), codes);
    }
    if (r_out != nullptr) {
        float4* rp = reinterpret_cast<float4*>(r_out + row * p.cols + col);
        rp[0] = make_float4(r[0].x, r[0].y, r[1].x, r[1].y);
        rp[1] = make_float4(r[2].x, r[2].y, r[3].x, r[3].y);
    }
}

template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sigma_delta_banks_kernel(SigmaDeltaParams p, int visits, int64_t bank_bytes,
                                                                float* r_out) {
    const int64_t total = p.rows * (p.cols / 8);
    const float s_t = (BLK == 16) ? *p.gscale : 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        In8 in;
        load8<BLK, TC, false>(p, i, in);
        banks_finish<BLK>(p, i, in, s_t, visits, bank_bytes, r_out);
    }
}

// ------------------------------------------------------------------ stochastic-rounding requant
// Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC 2011): ten rounds of two 32 x 32 -> 64-bit multiplies
// mixing the four counter words with the two key words; the key is bumped by
// the Weyl constants after every round.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        // each 32 x 32 -> 64-bit product in one wide multiply
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x, p1 = (uint64_t)0xCD9E8D57u * c.z;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
        k.x += 0x9E3779B9u;
        k.y += 0xBB67AE85u;
    }
    return c;
}

// Stochastic rounding of a normalised value onto the E2M1 grid with the
// uniform u in [0, 1): between neighbouring magnitudes a <= |x| < b the
// magnitude is b when u < (|x| - a) / (b - a), else a; |x| >= 6 gives 6; the
// sign bit is x's.  The gap b - a is 0.5 below 2, 1 from 2 to 4 and 2 from 4
// to 6, so with s = |x| / gap (exact: a power-of-two scaling) the lower
// neighbour is floor(s) * gap and (|x| - a) / (b - a) = s - floor(s), both
// exact; a's grid index is floor(s) + 0, 2 or 4 in the three ranges.
__device__ __forceinline__ uint32_t sr_e2m1(float x, float u) {
    const float m = fabsf(x);
    // NaN takes the first range and index 0, as the rule's comparisons give it
    const bool lo = !(m >= 2.0f), mid = !(m >= 4.0f);
    const float sgap = lo ? 2.0f : (mid ? 1.0f : 0.5f);
    const float sv = __fmul_rn(m, sgap);
    const float fl = floorf(sv);
    const uint32_t i = (uint32_t)fl + (lo ? 0u : (mid ? 2u : 4u));
    uint32_t idx = (u < __fsub_rn(sv, fl)) ? i + 1 : i;
    if (m >= 6.0f) idx = 7;                 // also NaN-free saturation: |x| >= 6 takes 6
    return (signbit(x) ? 8u : 0u) | idx;
}

// One stochastic-rounding requant at a loop visit of one unit: the 8
// weights e0 .. e0 + 7 (e0 = row * cols + col, a multiple of 8) take the two
// Philox blocks of counters (e0/4 + {0, 1}, visit), key = seed.
template <int BLK, class P>
__device__ __forceinline__ void sr_finish(const P& p, int64_t u, const In8& in, float s_t, uint2 key,
                                          uint32_t visit) {
    const int64_t cpr = p.cols / 8;
    const int64_t row = u / cpr, col = (u % cpr) * 8;
    float2 xs[4];
    scaled8<BLK>(in, s_t, xs);
    const uint64_t g = (uint64_t)(row * p.cols + col) >> 2;
    const uint4 r0 = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)(g >> 32), visit, 0u), key);
    const uint4 r1 = philox4x32_10(make_uint4((uint32_t)(g + 1), (uint32_t)((g + 1) >> 32), visit, 0u), key);
    const uint32_t rw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    uint32_t codes = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float x = (j & 1) ? xs[j >> 1].y : xs[j >> 1].x;
        const float uu = (float)(rw[j] >> 8) * 0x1p-24f;
        codes |= sr_e2m1(x, uu) << (4 * j);
    }
    *reinterpret_cast<uint32_t*>(p.codes + row * (p.cols / 2) + col / 2) = codes;
}

template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sr_requant_kernel(SigmaDeltaParams p, uint64_t seed, uint32_t visit) {
    const int64_t total = p.rows * (p.cols / 8);
    const float s_t = (BLK == 16) ? *p.gscale : 0.0f;
    const uint2 key = make_uint2((uint32_t)seed, (uint32_t)(seed >> 32));
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        In8 in;
        load8<BLK, TC, false>(p, i, in);
        sr_finish<BLK>(p, i, in, s_t, key, visit);
    }
}

// One Sigma-Delta step of one unit (as the tiled kernel above): x = w / S,
// v = x + r, q = E2M1(v), r <- v - q.
template <int BLK, class P>
__device__ __forceinline__ void sd_finish(const P& p, int64_t u, const In8& in, float s_t) {
    const int64_t cpr = p.cols / 8;
    const int64_t row = u / cpr, col = (u % cpr) * 8;
    float2 x[4];
    scaled8<BLK>(in, s_t, x);
    const float2 r[4] = {make_float2(in.r0.x, in.r0.y), make_float2(in.r0.z, in.r0.w),
                         make_float2(in.r1.x, in.r1.y), make_float2(in.r1.z, in.r1.w)};
    float2 v[4], n[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = add2_rn(x[j], r[j]);
    const uint32_t codes = e2m1_pack4(v[0].x, v[0].y, v[1].x, v[1].y) |
                           (e2m1_pack4(v[2].x, v[2].y, v[3].x, v[3].y) << 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) n[j] = sub2_rn(v[j], e2m1x2_value((codes >> (8 * j)) & 0xFFu));
    float4* rp = reinterpret_cast<float4*>(p.residue + row * p.cols + col);
    __stcs(rp, make_float4(n[0].x, n[0].y, n[1].x, n[1].y));
    __stcs(rp + 1, make_float4(n[2].x, n[2].y, n[3].x, n[3].y));
    __stcs(reinterpret_cast<unsigned int*>(p.codes + row * (p.cols / 2) + col / 2), codes);
}

// ------------------------------------------------------------------ dequantize
// Eight elements from one word of codes: code * s_b (NVFP4) or code * 2^e
// (MXFP4), exact, then one rounding for the NVFP4 tensor scale.  The code
// values come from byte permutes (exact bf16 patterns, no conversions).
template <int BLK>
__device__ __forceinline__ void dq8(uint32_t codes, float sb, float s_t, float (&o)[8]) {
    uint32_t q[4];
    e2m1x8_to_bf16(codes, q);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float2 v = mul2_rn(make_float2(__uint_as_float(q[j] << 16), __uint_as_float(q[j] & 0xFFFF0000u)),
                           make_float2(sb, sb));
        if (BLK == 16) v = mul2_rn(v, make_float2(s_t, s_t));
        o[2 * j] = v.x;
        o[2 * j + 1] = v.y;
    }
}

__device__ __forceinline__ uint4 bf16x8(const float (&o)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * j], o[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Two layouts of the work, each the faster one measured for its output type:
// bf16 output: a thread owns whole blocks (its codes, BLK/2 bytes, and scale
//   byte in one load each), and loads the next block before converting and
//   storing the current one;
// fp32 output: a unit is 8 elements (4 code bytes, two 16-byte stores); a warp
//   takes 4 x 32 consecutive units, lane l the units l, l + 32, l + 64, l + 96,
//   so every load and store instruction covers one contiguous range, and a
//   thread issues its four units' loads before any of their arithmetic.
template <int BLK, bool TC, bool OUT_BF16>
__global__ void __launch_bounds__(256) dequantize_kernel(DequantParams p) {
    const float s_t = (BLK == 16) ? *p.gscale : 1.0f;
    if constexpr (OUT_BF16) {
        const int64_t total = p.rows * p.scols;
        const int64_t stride = (int64_t)gridDim.x * blockDim.x;
        int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        auto load = [&](int64_t u, uint32_t (&w)[BLK / 8], uint32_t& sb) {
            const int64_t row = u / p.scols, b = u % p.scols;
            const uint8_t* cp = p.codes + row * (p.cols / 2) + b * (BLK / 2);
            if constexpr (BLK == 16) {
                const uint2 c = __ldcs(reinterpret_cast<const uint2*>(cp));
                w[0] = c.x; w[1] = c.y;
            } else {
                const uint4 c = __ldcs(reinterpret_cast<const uint4*>(cp));
                w[0] = c.x; w[1] = c.y; w[2] = c.z; w[3] = c.w;
            }
            sb = TC ? p.scales[tc_scale_offset(row, b, p.catoms)] : p.scales[row * p.scols + b];
        };
        if (i >= total) return;
        uint32_t w[BLK / 8], sb;
        load(i, w, sb);
        for (;;) {
            const int64_t n = i + stride;
            uint32_t wn[BLK / 8], sbn = 0;
            if (n < total) load(n, wn, sbn);
            const int64_t row = i / p.scols, b = i % p.scols;
            const float sv = (BLK == 16) ? e4m3_value(sb) : exp2_int((int)sb - 127);
#pragma unroll
            for (int g = 0; g < BLK / 8; ++g) {
                float o[8];
                dq8<BLK>(w[g], sv, s_t, o);
                __stcs(reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + row * p.cols + b * BLK + g * 8),
                       bf16x8(o));
            }
            if (n >= total) break;
            i = n;
            sb = sbn;
#pragma unroll
            for (int g = 0; g < BLK / 8; ++g) w[g] = wn[g];
        }
    } else {
        constexpr int U = 4;
        const int64_t cpr = p.cols / 8;
        const int64_t total = p.rows * cpr;
        const int lane = threadIdx.x & 31;
        const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
        const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
        for (int64_t base = wid * 32 * U; base < total; base += nw * 32 * U) {
            uint32_t codes[U], byte[U];
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int64_t u = base + k * 32 + lane;
                if (u < total) {
                    const int64_t row = u / cpr, col = (u % cpr) * 8;
                    codes[k] = __ldcs(reinterpret_cast<const unsigned int*>(p.codes + row * (p.cols / 2) + col / 2));
                    const int64_t c = col / BLK;
                    byte[k] = TC ? p.scales[tc_scale_offset(row, c, p.catoms)] : p.scales[row * p.scols + c];
                }
            }
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int64_t u = base + k * 32 + lane;
                if (u >= total) break;
                const int64_t row = u / cpr, col = (u % cpr) * 8;
                float o[8];
                dq8<BLK>(codes[k], (BLK == 16) ? e4m3_value(byte[k]) : exp2_int((int)byte[k] - 127), s_t, o);
                float4* op = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + row * p.cols + col);
                __stcs(op, make_float4(o[0], o[1], o[2], o[3]));
                __stcs(op + 1, make_float4(o[4], o[5], o[6], o[7]));
            }
        }
    }
}

// ------------------------------------------------------------------ launchers
static int grid_for(int64_t tiles, int num_sms, int per_sm) {
    int64_t cap = (int64_t)num_sms * per_sm;
    if (tiles < 1) return 1;
    return (int)(tiles < cap ? tiles : cap);
}

// CTAs of `threads` threads of `kernel` resident on one SM at once (>= 1): a
// grid-stride kernel gets no more than that many per SM, since a partial
// second wave would leave most SMs idle at the end.
template <class K>
static int resident_per_sm(K kernel, int threads) {
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) != cudaSuccess || occ < 1) occ = 1;
    return occ;
}

struct QuantMaps {
    CUtensorMap x, codes;
    int codes_tma;
};

template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool CHAN, bool S46 = false>
static cudaError_t launch_quant_one(const QuantParams& p, const QuantMaps& m, int num_sms, cudaStream_t st) {
    using G = QzGeom<BLK, BF16>;
    auto k = quantize_kernel<BLK, BF16, TC, RU, HAD, CHAN, S46>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((p.rows + G::ROWS - 1) / G::ROWS) * p.catoms;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    k<<<grid, qz::THREADS, G::SMEM, st>>>(m.x, m.codes, p, m.codes_tma);
    return cudaGetLastError();
}

template <int BLK, bool BF16, bool TC, bool RU>
static cudaError_t launch_quant_mx_variants(const QuantParams& p, const QuantMaps& m, bool had, bool chan,
                                            int num_sms, cudaStream_t st) {
    if (had && chan) return launch_quant_one<BLK, BF16, TC, RU, true, true>(p, m, num_sms, st);
    if (had) return launch_quant_one<BLK, BF16, TC, RU, true, false>(p, m, num_sms, st);
    if (chan) return launch_quant_one<BLK, BF16, TC, RU, false, true>(p, m, num_sms, st);
    return launch_quant_one<BLK, BF16, TC, RU, false, false>(p, m, num_sms, st);
}

template <int BLK, bool BF16, bool TC>
static cudaError_t launch_quant_ru(const QuantParams& p, const QuantMaps& m, bool ru, bool had, bool chan,
                                   bool s46, int num_sms, cudaStream_t st) {
    if constexpr (BLK == 16) {
        if (s46) return launch_quant_one<BLK, BF16, TC, true, false, false, true>(p, m, num_sms, st);
        if (ru) return launch_quant_one<BLK, BF16, TC, true, false, false>(p, m, num_sms, st);
        return launch_quant_one<BLK, BF16, TC, false, false, false>(p, m, num_sms, st);
    } else {
        if (ru) return launch_quant_mx_variants<BLK, BF16, TC, true>(p, m, had, chan, num_sms, st);
        return launch_quant_mx_variants<BLK, BF16, TC, false>(p, m, had, chan, num_sms, st);
    }
}

template <int BLK>
static cudaError_t launch_quant_blk(const QuantParams& p, bool bf16, bool tc, bool ru, bool had, bool chan,
                                    bool s46, int num_sms, cudaStream_t st) {
    QuantMaps m;
    std::memset(&m, 0, sizeof(m));
    const int esz = bf16 ? 2 : 4;
    const int rows_tile = bf16 ? QzGeom<BLK, true>::ROWS : QzGeom<BLK, false>::ROWS;
    if (!encode_map_2d(&m.x, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.x,
                       (uint64_t)p.cols, (uint64_t)p.rows, (uint64_t)(p.ld * esz), (uint32_t)(128 / esz),
                       (uint32_t)rows_tile, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // codes leave by TMA when their row pitch allows it (a multiple of 16 bytes)
    m.codes_tma = ((p.cols / 2) % 16 == 0) ? 1 : 0;
    if (m.codes_tma &&
        !encode_map_2d(&m.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.codes, (uint64_t)(p.cols / 2), (uint64_t)p.rows,
                       (uint64_t)(p.cols / 2), (uint32_t)(2 * BLK), (uint32_t)rows_tile, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (bf16) {
        if (tc) return launch_quant_ru<BLK, true, true>(p, m, ru, had, chan, s46, num_sms, st);
        return launch_quant_ru<BLK, true, false>(p, m, ru, had, chan, s46, num_sms, st);
    }
    if (tc) return launch_quant_ru<BLK, false, true>(p, m, ru, had, chan, s46, num_sms, st);
    return launch_quant_ru<BLK, false, false>(p, m, ru, had, chan, s46, num_sms, st);
}

cudaError_t launch_quantize(const QuantParams& p, int blk, bool bf16, bool tc, bool ru, bool had,
                            bool chan, bool s46, cudaStream_t st, int num_sms) {
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    if (blk == 16) return launch_quant_blk<16>(p, bf16, tc, ru, had, chan, s46, num_sms, st);
    return launch_quant_blk<32>(p, bf16, tc, ru, had, chan, false, num_sms, st);
}

template <bool BF16, bool TC, bool RU>
static cudaError_t launch_amax_quant_one(const QuantParams& p, const QuantMaps& m, int num_sms, cudaStream_t st) {
    using G = QzGeom<16, BF16>;
    auto k = quantize_kernel<16, BF16, TC, RU, false, false, false, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, qz::THREADS, G::SMEM);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorCooperativeLaunchTooLarge;
    const int64_t tiles = ((p.rows + G::ROWS - 1) / G::ROWS) * p.catoms;
    // every CTA must be resident at once for the grid-wide wait
    const int64_t cap = (int64_t)num_sms * occ;
    const int grid = (int)(tiles < num_sms ? tiles : (num_sms < cap ? num_sms : cap));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(qz::THREADS);
    cfg.dynamicSmemBytes = G::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k, m.x, m.codes, p, m.codes_tma);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_amax_quantize(const QuantParams& p, bool bf16, bool tc, bool ru, cudaStream_t st, int num_sms) {
    cudaError_t e = cudaMemsetAsync(p.amax_out, 0, 4 * sizeof(unsigned int), st);
    if (e != cudaSuccess || p.rows == 0 || p.cols == 0) return e;
    QuantMaps m;
    std::memset(&m, 0, sizeof(m));
    const int esz = bf16 ? 2 : 4;
    const int rows_tile = bf16 ? QzGeom<16, true>::ROWS : QzGeom<16, false>::ROWS;
    if (!encode_map_2d(&m.x, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.x,
                       (uint64_t)p.cols, (uint64_t)p.rows, (uint64_t)(p.ld * esz), (uint32_t)(128 / esz),
                       (uint32_t)rows_tile, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    m.codes_tma = ((p.cols / 2) % 16 == 0) ? 1 : 0;
    if (m.codes_tma &&
        !encode_map_2d(&m.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.codes, (uint64_t)(p.cols / 2), (uint64_t)p.rows,
                       (uint64_t)(p.cols / 2), 32u, (uint32_t)rows_tile, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
#define Q4_AQ(B, T, R) return launch_amax_quant_one<B, T, R>(p, m, num_sms, st)
    if (bf16) {
        if (tc) { if (ru) Q4_AQ(true, true, true); Q4_AQ(true, true, false); }
        if (ru) Q4_AQ(true, false, true);
        Q4_AQ(true, false, false);
    }
    if (tc) { if (ru) Q4_AQ(false, true, true); Q4_AQ(false, true, false); }
    if (ru) Q4_AQ(false, false, true);
    Q4_AQ(false, false, false);
#undef Q4_AQ
}

cudaError_t read_clear_quant_error(unsigned int* word) { return read_clear_module_error(word); }
cudaError_t set_quant_wait_limit(long long cycles) { return set_module_wait_limit(cycles); }

cudaError_t launch_sigma_delta(const SigmaDeltaParams& p, int blk, bool tc, cudaStream_t st, int num_sms) {
    using namespace sdk;
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    CUtensorMap mw, mr, mc;
    std::memset(&mc, 0, sizeof(mc));
    if (!encode_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.w, (uint64_t)p.cols, (uint64_t)p.rows,
                       (uint64_t)p.cols * 4, COLS, ROWS, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_map_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.residue, (uint64_t)p.cols, (uint64_t)p.rows,
                       (uint64_t)p.cols * 4, COLS, ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int codes_tma = ((p.cols / 2) % 16 == 0) ? 1 : 0;
    if (codes_tma && !encode_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.codes, (uint64_t)(p.cols / 2),
                                    (uint64_t)p.rows, (uint64_t)(p.cols / 2), COLS / 2, ROWS,
                                    CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int64_t tiles = ((p.rows + ROWS - 1) / ROWS) * ((p.cols + COLS - 1) / COLS);
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
#define Q4_SD(B, T)                                                                                  \
    {                                                                                                \
        auto k = sigma_delta_kernel<B, T>;                                                           \
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM); \
        if (e != cudaSuccess) return e;                                                              \
        k<<<grid, THREADS, SMEM, st>>>(mw, mr, mc, p, codes_tma);                                    \
    }
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
    const int64_t units = p.rows * (p.cols / 8);
    // as many CTAs as are resident at once (a second partial wave would idle most SMs)
    // bf16 output: one block per thread-step; fp32: 4 units of 8 elements per thread-step
    const int64_t steps = out_bf16 ? p.rows * p.scols : (units + 3) / 4;
    auto launch = [&](auto kernel) {
        const int grid = grid_for((steps + 255) / 256, num_sms, resident_per_sm(kernel, 256));
        kernel<<<grid, 256, 0, st>>>(p);
    };
#define Q4_DQ(B, T, O) launch(dequantize_kernel<B, T, O>)
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

cudaError_t launch_sigma_delta_banks(const SigmaDeltaParams& p, int blk, bool tc, int visits, float* r_out,
                                     cudaStream_t st, int num_sms) {
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    const int64_t chunks = p.rows * (p.cols / 8);
    const int64_t bank = p.rows * (p.cols / 2);
#define Q4_SDB(B, T)                                                                                          \
    sigma_delta_banks_kernel<B, T><<<grid_for((chunks + 255) / 256, num_sms,                                   \
                                              resident_per_sm(sigma_delta_banks_kernel<B, T>, 256)),             \
                                     256, 0, st>>>(p, visits, bank, r_out)
    if (blk == 16) {
        if (tc) Q4_SDB(16, true); else Q4_SDB(16, false);
    } else {
        if (tc) Q4_SDB(32, true); else Q4_SDB(32, false);
    }
#undef Q4_SDB
    return cudaGetLastError();
}

cudaError_t launch_sr_requant(const SigmaDeltaParams& p, int blk, bool tc, uint64_t seed, uint32_t visit,
                              cudaStream_t st, int num_sms) {
    if (p.rows == 0 || p.cols == 0) return cudaSuccess;
    const int64_t chunks = p.rows * (p.cols / 8);
#define Q4_SR(B, T)                                                                                           \
    sr_requant_kernel<B, T><<<grid_for((chunks + 255) / 256, num_sms, resident_per_sm(sr_requant_kernel<B, T>, 256)), \
                              256, 0, st>>>(p, seed, visit)
    if (blk == 16) {
        if (tc) Q4_SR(16, true); else Q4_SR(16, false);
    } else {
        if (tc) Q4_SR(32, true); else Q4_SR(32, false);
    }
#undef Q4_SR
    return cudaGetLastError();
}

// ------------------------------------------------------------------ grouped launches
// One launch over a list of matrices (the looped core requantizes all of its
// weights at every loop visit; a matrix of a few million weights is too small
// to amortise a launch of its own).  The units of all entries form one range
// that the grid walks grid-stride; a unit's entry is the last one whose
// `start` it has reached, and because entries are in unit order a thread's
// entry index only moves forward along its walk.  Each unit runs exactly the
// per-unit step of the single-matrix launch.
__device__ __forceinline__ int group_entry(const GroupParams& g, int e, int64_t i) {
    while (e + 1 < g.count && i >= g.m[e + 1].start) ++e;
    return e;
}

// The grid-stride walk over a grouped launch's units.  With PIPE the loads of
// a thread's next unit are issued before the arithmetic of its current one,
// so every thread keeps one unit's loads in flight while it computes.
template <bool PIPE, class In, class Load, class Finish>
__device__ __forceinline__ void group_walk(const GroupParams& g, Load load, Finish finish) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= g.total) return;
    int e = group_entry(g, 0, i);
    if constexpr (!PIPE) {
        for (; i < g.total; i += stride) {
            e = group_entry(g, e, i);
            In in;
            load(e, i - g.m[e].start, in);
            finish(e, i - g.m[e].start, in);
        }
    } else {
        In cur;
        load(e, i - g.m[e].start, cur);
        for (;;) {
            const int64_t n = i + stride;
            const bool more = n < g.total;
            int en = e;
            In nxt;
            if (more) {
                en = group_entry(g, e, n);
                load(en, n - g.m[en].start, nxt);
            }
            finish(e, i - g.m[e].start, cur);
            if (!more) break;
            i = n;
            e = en;
            cur = nxt;
        }
    }
}

// Each entry's tensor scale s_t (NVFP4), read once per CTA.
template <int BLK>
__device__ __forceinline__ void group_scales(const GroupParams& g, float* s_ts) {
    if (BLK == 16)
        for (int k = threadIdx.x; k < g.count; k += blockDim.x) s_ts[k] = *g.m[k].gscale;
    __syncthreads();
}

template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sigma_delta_grouped_kernel(const __grid_constant__ GroupParams g) {
    __shared__ float s_ts[kMaxGroup];
    group_scales<BLK>(g, s_ts);
    group_walk<true, In8>(
        g, [&](int e, int64_t u, In8& in) { load8<BLK, TC, true>(g.m[e], u, in); },
        [&](int e, int64_t u, const In8& in) { sd_finish<BLK>(g.m[e], u, in, BLK == 16 ? s_ts[e] : 0.0f); });
}

template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sr_requant_grouped_kernel(const __grid_constant__ GroupParams g, uint64_t seed,
                                                                 uint32_t visit) {
    __shared__ float s_ts[kMaxGroup];
    group_scales<BLK>(g, s_ts);
    const uint2 key = make_uint2((uint32_t)seed, (uint32_t)(seed >> 32));
    group_walk<true, In8>(
        g, [&](int e, int64_t u, In8& in) { load8<BLK, TC, false>(g.m[e], u, in); },
        [&](int e, int64_t u, const In8& in) {
            sr_finish<BLK>(g.m[e], u, in, BLK == 16 ? s_ts[e] : 0.0f, key, visit);
        });
}

template <int BLK, bool TC>
__global__ void __launch_bounds__(256) sigma_delta_banks_grouped_kernel(const __grid_constant__ GroupParams g,
                                                                        int visits) {
    __shared__ float s_ts[kMaxGroup];
    group_scales<BLK>(g, s_ts);
    group_walk<true, In8>(
        g, [&](int e, int64_t u, In8& in) { load8<BLK, TC, false>(g.m[e], u, in); },
        [&](int e, int64_t u, const In8& in) {
            const GroupItem& it = g.m[e];
            banks_finish<BLK>(it, u, in, BLK == 16 ? s_ts[e] : 0.0f, visits, it.rows * (it.cols / 2), it.residue);
        });
}

// Quantizer unit: one block, over the padded block grid in the tensor-core
// layout (rows to a multiple of 128, blocks to a multiple of 4) so that the
// padding scale bytes are written (0) as the tiled quantizer writes them.
template <int BLK, bool BF16>
struct QzIn {
    uint4 raw[BLK * (BF16 ? 2 : 4) / 16];   // the block's input bytes
    bool inside;
};

template <int BLK, bool BF16, bool TC>
__device__ __forceinline__ void qz_load(const GroupItem& p, int64_t u, QzIn<BLK, BF16>& in) {
    const int64_t spad = TC ? p.catoms * 4 : p.scols;
    const int64_t row = u / spad, b = u % spad;
    in.inside = row < p.rows && b < p.scols;
    if (!in.inside) return;
    const uint4* xp = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(p.w) +
                                                     (row * p.cols + b * BLK) * (BF16 ? 2 : 4));
#pragma unroll
    for (int c = 0; c < BLK * (BF16 ? 2 : 4) / 16; ++c) in.raw[c] = __ldcs(xp + c);
}

template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool S46>
__device__ __forceinline__ void qz_finish(const GroupItem& p, int64_t u, const QzIn<BLK, BF16>& in,
                                          const NvCtx& sc) {
    const int64_t spad = TC ? p.catoms * 4 : p.scols;
    const int64_t row = u / spad, b = u % spad;
    if (!in.inside) {
        if (TC) p.scales[tc_scale_offset(row, b, p.catoms)] = 0;
        return;
    }
    float v[BLK];
#pragma unroll
    for (int c = 0; c < BLK * (BF16 ? 2 : 4) / 16; ++c) {
        const uint4 raw = in.raw[c];
        if constexpr (BF16) {
            float* d = v + 8 * c;
            d[0] = bf16_lo(raw.x); d[1] = bf16_hi(raw.x); d[2] = bf16_lo(raw.y); d[3] = bf16_hi(raw.y);
            d[4] = bf16_lo(raw.z); d[5] = bf16_hi(raw.z); d[6] = bf16_lo(raw.w); d[7] = bf16_hi(raw.w);
        } else {
            v[4 * c] = __uint_as_float(raw.x); v[4 * c + 1] = __uint_as_float(raw.y);
            v[4 * c + 2] = __uint_as_float(raw.z); v[4 * c + 3] = __uint_as_float(raw.w);
        }
    }
    uint32_t byte;
    uint8_t* dst = p.codes + row * (p.cols / 2) + b * (BLK / 2);
    if constexpr (BLK == 16) {
        uint32_t w[2];
        if constexpr (S46) {
            nv_block46(v, sc, byte, w);
        } else {
            uint32_t bb[1], ww[1][2];
            nv_blocks<RU, 1>(reinterpret_cast<const float(&)[1][16]>(v), sc, bb, ww);
            byte = bb[0];
            w[0] = ww[0][0];
            w[1] = ww[0][1];
        }
        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    } else {
        uint32_t w[4];
        const float4 cw[8] = {};
        mx_block<RU, HAD, false, false>(v, cw, nullptr, byte, w);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (TC) p.scales[tc_scale_offset(row, b, p.catoms)] = (uint8_t)byte;
    else p.scales[row * p.scols + b] = (uint8_t)byte;
}

template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool S46>
__global__ void __launch_bounds__(256) quantize_grouped_kernel(const __grid_constant__ GroupParams g) {
    // NVFP4: each entry's 128-entry table of (S, 1/S), as the tiled quantizer's
    __shared__ float2 tabs[BLK == 16 ? kMaxGroup * 128 : 1];
    __shared__ float s_ts[kMaxGroup];
    if constexpr (BLK == 16) {
        for (int k = threadIdx.x; k < g.count * 128; k += blockDim.x) {
            const NvScale r = nv_scale_of((uint32_t)(k & 127), *g.m[k >> 7].gscale);
            tabs[k] = make_float2(r.S, r.y);
        }
        for (int k = threadIdx.x; k < g.count; k += blockDim.x) s_ts[k] = *g.m[k].gscale;
        __syncthreads();
    }
    // a unit's loads in flight ahead of the current unit's arithmetic while that
    // stays within 64 bytes (MXFP4 fp32 blocks are read just in time)
    constexpr bool PIPE = BLK * (BF16 ? 2 : 4) <= 64;
    group_walk<PIPE, QzIn<BLK, BF16>>(
        g, [&](int e, int64_t u, QzIn<BLK, BF16>& in) { qz_load<BLK, BF16, TC>(g.m[e], u, in); },
        [&](int e, int64_t u, const QzIn<BLK, BF16>& in) {
            NvCtx sc;
            if constexpr (BLK == 16) sc = nv_ctx(s_ts[e], tabs + e * 128);
            qz_finish<BLK, BF16, TC, RU, HAD, S46>(g.m[e], u, in, sc);
        });
}

// Entries' unit ranges; the grid is as many CTAs of 256 threads as are
// resident on the GPU at once (persistent), fewer for a small launch.
template <class K>
static int fill_group(GroupParams& g, K kernel, int64_t (*units)(const GroupItem&), int num_sms) {
    int64_t acc = 0;
    for (int i = 0; i < g.count; ++i) {
        g.m[i].start = acc;
        acc += units(g.m[i]);
    }
    g.total = acc;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, 256, 0) != cudaSuccess || occ < 1) occ = 1;
    return grid_for((acc + 255) / 256, num_sms, occ);
}

static int64_t units8(const GroupItem& m) { return m.rows * (m.cols / 8); }
static int64_t units_blocks_tc(const GroupItem& m) { return ((m.rows + 127) / 128) * 128 * m.catoms * 4; }
static int64_t units_blocks_rm(const GroupItem& m) { return m.rows * m.scols; }

template <int BLK, bool BF16, bool TC, bool RU, bool HAD, bool S46>
static cudaError_t launch_qg(GroupParams& g, cudaStream_t st, int num_sms) {
    auto k = quantize_grouped_kernel<BLK, BF16, TC, RU, HAD, S46>;
    const int grid = fill_group(g, k, TC ? units_blocks_tc : units_blocks_rm, num_sms);
    if (g.total == 0) return cudaSuccess;
    k<<<grid, 256, 0, st>>>(g);
    return cudaGetLastError();
}

template <int BLK, bool BF16, bool TC>
static cudaError_t launch_qg_flags(GroupParams& g, bool ru, bool had, bool s46, cudaStream_t st, int num_sms) {
    if constexpr (BLK == 16) {
        if (s46) return launch_qg<16, BF16, TC, true, false, true>(g, st, num_sms);
        if (ru) return launch_qg<16, BF16, TC, true, false, false>(g, st, num_sms);
        return launch_qg<16, BF16, TC, false, false, false>(g, st, num_sms);
    } else {
        if (had) {
            if (ru) return launch_qg<32, BF16, TC, true, true, false>(g, st, num_sms);
            return launch_qg<32, BF16, TC, false, true, false>(g, st, num_sms);
        }
        if (ru) return launch_qg<32, BF16, TC, true, false, false>(g, st, num_sms);
        return launch_qg<32, BF16, TC, false, false, false>(g, st, num_sms);
    }
}

template <int BLK>
static cudaError_t launch_qg_blk(GroupParams& g, bool bf16, bool tc, bool ru, bool had, bool s46, cudaStream_t st,
                                 int num_sms) {
    if (bf16) {
        if (tc) return launch_qg_flags<BLK, true, true>(g, ru, had, s46, st, num_sms);
        return launch_qg_flags<BLK, true, false>(g, ru, had, s46, st, num_sms);
    }
    if (tc) return launch_qg_flags<BLK, false, true>(g, ru, had, s46, st, num_sms);
    return launch_qg_flags<BLK, false, false>(g, ru, had, s46, st, num_sms);
}

cudaError_t launch_quantize_grouped(GroupParams& g, int blk, bool bf16, bool tc, bool ru, bool had, bool s46,
                                    cudaStream_t st, int num_sms) {
    if (blk == 16) return launch_qg_blk<16>(g, bf16, tc, ru, had, s46, st, num_sms);
    return launch_qg_blk<32>(g, bf16, tc, ru, had, s46, st, num_sms);
}

#define Q4_GROUP_LAUNCH(KERNEL, ...)                                  \
    do {                                                              \
        auto k = KERNEL;                                              \
        const int grid = fill_group(g, k, units8, num_sms);           \
        if (g.total == 0) return cudaSuccess;                         \
        k<<<grid, 256, 0, st>>>(g __VA_OPT__(,) __VA_ARGS__);         \
        return cudaGetLastError();                                    \
    } while (0)

cudaError_t launch_sigma_delta_grouped(GroupParams& g, int blk, bool tc, cudaStream_t st, int num_sms) {
    if (blk == 16) {
        if (tc) Q4_GROUP_LAUNCH((sigma_delta_grouped_kernel<16, true>));
        Q4_GROUP_LAUNCH((sigma_delta_grouped_kernel<16, false>));
    }
    if (tc) Q4_GROUP_LAUNCH((sigma_delta_grouped_kernel<32, true>));
    Q4_GROUP_LAUNCH((sigma_delta_grouped_kernel<32, false>));
}

cudaError_t launch_sr_requant_grouped(GroupParams& g, int blk, bool tc, uint64_t seed, uint32_t visit,
                                      cudaStream_t st, int num_sms) {
    if (blk == 16) {
        if (tc) Q4_GROUP_LAUNCH((sr_requant_grouped_kernel<16, true>), seed, visit);
        Q4_GROUP_LAUNCH((sr_requant_grouped_kernel<16, false>), seed, visit);
    }
    if (tc) Q4_GROUP_LAUNCH((sr_requant_grouped_kernel<32, true>), seed, visit);
    Q4_GROUP_LAUNCH((sr_requant_grouped_kernel<32, false>), seed, visit);
}

cudaError_t launch_sigma_delta_banks_grouped(GroupParams& g, int blk, bool tc, int visits, cudaStream_t st,
                                             int num_sms) {
    if (blk == 16) {
        if (tc) Q4_GROUP_LAUNCH((sigma_delta_banks_grouped_kernel<16, true>), visits);
        Q4_GROUP_LAUNCH((sigma_delta_banks_grouped_kernel<16, false>), visits);
    }
    if (tc) Q4_GROUP_LAUNCH((sigma_delta_banks_grouped_kernel<32, true>), visits);
    Q4_GROUP_LAUNCH((sigma_delta_banks_grouped_kernel<32, false>), visits);
}
#undef Q4_GROUP_LAUNCH

}  // namespace q4
