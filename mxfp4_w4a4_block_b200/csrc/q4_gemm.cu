// q4_gemm.cu -- the GEMM kernels of the path, all on the sm_100a tensor cores
// (tcgen05.mma, accumulators in TMEM), persistent and warp specialised.
//
// gemm_kernel: block-scaled FP4 W4A4  Y = alpha * dec(A) dec(B)^T
// (kind::mxf4nvf4, block16 NVFP4 / block32 MXFP4):
//   warp 0      TMA producer: A and B code tiles (128-byte swizzle) by tiled
//               tensor copies, scale atoms by contiguous bulk copies, into a
//               STAGES-deep ring guarded by full/empty mbarriers;
//   warp 1      allocates TMEM; one lane issues each k-block's block-scaled
//               MMAs into the FP32 accumulator from an unrolled loop over
//               precomputed descriptors;
//   warps 2..5  scale warps: copy each k-block's A and B scale atoms from
//               shared memory into one of SF_NBUF TMEM scale buffers with
//               tcgen05.st (each warp its TMEM lane quarter), off the tensor
//               pipe that runs the MMAs, handed over through mbarriers;
//   warps 6..13 epilogue: two warps per TMEM lane quarter drain 128
//               accumulator columns each into registers (tcgen05.ld), release
//               the accumulator to the next tile's MMAs, then scale, convert
//               and store Y by TMA through a swizzled shared-memory buffer.
// CTA tile 128 x 256, k-block 256 elements (128 bytes of codes per row).
//
// w4a16_gemm_kernel: bf16 activations times the 4-bit weight dequantized
// exactly to bf16 in shared memory by converter warps (kind::f16).
// sd_gemm_decode_kernel / sd_gemm_grouped_kernel: the Sigma-Delta step fused
// into that weight producer for decode shapes, K split over a cluster.
// fused_decode_kernel: the W4A4 GEMM for M <= 16 with the activation
// quantization fused into its producer.
// Every mbarrier wait is bounded; on time-out the kernel records an error and
// winds down, waiting (bounded) for its own copies and MMAs before freeing TMEM.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "q4_codec.cuh"
#include "q4_internal.h"
#include "q4_ptx.cuh"

namespace q4 {

namespace gemm {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KB_BYTES = 128;            // bytes of codes per row per k-block
constexpr int KB_ELEMS = 256;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * KB_BYTES;   // 16 KB
constexpr int B_STAGE = BN * KB_BYTES;   // 32 KB
constexpr int SFA_STAGE = 4 * 512;       // up to 4 scale atoms
constexpr int SFB_STAGE = 2 * 4 * 512;   // 2 row bands of 128
constexpr int OFF_B = STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_EPI = OFF_SFB + STAGES * SFB_STAGE;   // 8 KB: one warp's 32 x 128 bf16 block
constexpr int EPI_BYTES = 8192;
constexpr int OFF_BAR = OFF_EPI + EPI_BYTES;
constexpr int BAR_BYTES = 512;
constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;   // + alignment slack
constexpr int SF_WARPS = 4;             // warps 2..5 stage scales, one per TMEM lane quarter
constexpr int EPI_WARPS = 8;
constexpr int FIRST_EPI_WARP = 2 + SF_WARPS;
constexpr int THREADS = 32 * FIRST_EPI_WARP + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;          // 256 fp32 columns
constexpr uint32_t SF_COL = 256;         // SF_NBUF buffers of 48 columns, one per k-block in flight
constexpr int SF_NBUF = 4;
constexpr uint32_t SF_BUF = 48;          // per buffer: SFA 4 atoms x 4 columns, then SFB 4 atoms x 8
constexpr uint32_t SFB_OFF = 16;
constexpr int MAX_W = 4;                 // weights that share one A in a launch
}  // namespace gemm

// One A [M, K] times up to MAX_W weights B_w [N_w, K] into Y_w [M, N_w]: the
// tiles of all weights form one list (weight w's tiles from tile_start[w]),
// walked by the persistent CTAs as one grid.
struct GemmDev {
    int64_t M, K;
    int nw;
    int64_t N[gemm::MAX_W];
    int64_t tile_start[gemm::MAX_W + 1];
    const uint8_t* a_scales;
    const uint8_t* b_scales[gemm::MAX_W];
    const float* a_gscale;
    const float* b_gscale[gemm::MAX_W];
    void* y[gemm::MAX_W];
    int64_t catoms;      // scale atom-columns per 128-row band (same for A and B)
    int out_bf16;
};

// The launch's tensor maps: A, and each weight's B and (bf16 output) Y.
struct GemmMaps {
    CUtensorMap a;
    CUtensorMap b[gemm::MAX_W];
    CUtensorMap y[gemm::MAX_W];
};

// Weight of tile t: the last w whose tiles start at or before t.
__device__ __forceinline__ int gemm_weight_of(const GemmDev& p, int64_t t) {
    int w = 0;
#pragma unroll
    for (int i = 1; i < gemm::MAX_W; ++i) w += (i < p.nw && t >= p.tile_start[i]) ? 1 : 0;
    return w;
}

// Store 32 consecutive fp32 results of one output row (columns col0..col0+31,
// only those < N), scaled by alpha.
__device__ __forceinline__ void store_row32(void* y, int64_t N, int64_t row, int64_t col0, const uint32_t (&r)[32],
                                            float alpha, bool out_bf16) {
    if (out_bf16) {
        uint16_t* yp = reinterpret_cast<uint16_t*>(y) + row * N + col0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (col0 + g * 8 >= N) break;
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[g * 8 + 2 * j]) * alpha,
                                                         __uint_as_float(r[g * 8 + 2 * j + 1]) * alpha);
                w[j] = *reinterpret_cast<uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(yp + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        float* yp = reinterpret_cast<float*>(y) + row * N + col0;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            if (col0 + g * 4 >= N) break;
            *reinterpret_cast<float4*>(yp + g * 4) =
                make_float4(__uint_as_float(r[g * 4]) * alpha, __uint_as_float(r[g * 4 + 1]) * alpha,
                            __uint_as_float(r[g * 4 + 2]) * alpha, __uint_as_float(r[g * 4 + 3]) * alpha);
        }
    }
}

// Scale atoms of one k-block from shared memory into TMEM by tcgen05.st.
// Called by the four scale warps; warp w writes its TMEM lane quarter w % 4,
// and every quarter receives the whole atom (the layout the block-scaled MMA
// reads: lane 32q + r, column j of an atom holds row 32j + r's four scales).
// Staging through registers keeps these writes out of the tensor pipe that
// executes the MMAs (a tcgen05.cp would serialise with them).
__device__ __forceinline__ void stage_scales(uint32_t quarter_taddr, const uint8_t* sfa_smem, const uint8_t* sfb_smem,
                                             int na, int lane) {
    for (int a = 0; a < na; ++a) {
        const uint4 va = *reinterpret_cast<const uint4*>(sfa_smem + a * 512 + lane * 16);
        const uint4 vb0 = *reinterpret_cast<const uint4*>(sfb_smem + a * 512 + lane * 16);
        const uint4 vb1 = *reinterpret_cast<const uint4*>(sfb_smem + 2048 + a * 512 + lane * 16);
        tmem_st4(quarter_taddr + a * 4, va.x, va.y, va.z, va.w);
        tmem_st4(quarter_taddr + 16 + a * 8, vb0.x, vb0.y, vb0.z, vb0.w);
        tmem_st4(quarter_taddr + 16 + a * 8 + 4, vb1.x, vb1.y, vb1.z, vb1.w);
    }
}

// Store 64 bf16 results (already scaled and packed in pairs) of one row,
// columns col0..col0+63 that are < N.
__device__ __forceinline__ void store_row32_bf16(void* y, int64_t N, int64_t row, int64_t col0, const uint32_t (&a)[32],
                                                 const uint32_t (&b)[32]) {
    uint16_t* yp = reinterpret_cast<uint16_t*>(y) + row * N + col0;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        if (col0 + g * 8 >= N) break;
        const uint32_t* src = g < 4 ? &a[4 * g] : &b[4 * (g - 4)];
        *reinterpret_cast<uint4*>(yp + g * 8) = make_uint4(src[0], src[1], src[2], src[3]);
    }
}

template <bool MX>
__global__ void __launch_bounds__(gemm::THREADS, 1)
    gemm_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmDev p) {
    using namespace gemm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* mma_done = tmem_empty + 1;
    uint64_t* sf_ready = mma_done + 1;       // [SF_NBUF] a k-block's scales are in TMEM buffer b
    uint64_t* sf_free = sf_ready + SF_NBUF;  // [SF_NBUF] the MMAs reading scale buffer b are done
    uint64_t* epi_turn = sf_free + SF_NBUF;  // [EPI_WARPS] whose turn it is to use the store buffer
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(epi_turn + EPI_WARPS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, EPI_WARPS);               // one arrival per epilogue warp
        mbar_init(mma_done, 1);
        for (int b = 0; b < SF_NBUF; ++b) { mbar_init(&sf_ready[b], SF_WARPS); mbar_init(&sf_free[b], 1); }
        for (int w = 0; w < EPI_WARPS; ++w) mbar_init(&epi_turn[w], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&maps.a);
        for (int w = 0; w < p.nw; ++w) {
            tma_prefetch_desc(&maps.b[w]);
            if (p.out_bf16) tma_prefetch_desc(&maps.y[w]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int64_t tiles_m = (p.M + BM - 1) / BM;
    const int64_t tiles = p.tile_start[p.nw];
    const int nkb = (int)((p.K + KB_ELEMS - 1) / KB_ELEMS);
    const int mma_per_atom = MX ? 2 : 1;
    const int atoms_per_kb = 4 / mma_per_atom;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_phase[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, last_phase[s] = 0;
            for (int64_t t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
                const int w = gemm_weight_of(p, t);
                const int64_t lt = t - p.tile_start[w];
                const int64_t mt = lt % tiles_m, nt = lt / tiles_m;
                const int64_t bands_n = (p.N[w] + 127) / 128;
                const int nbands = (nt * 2 + 1 < bands_n) ? 2 : 1;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { *abort_flag = 1; break; }
                    const int64_t krem = p.K - (int64_t)kb * KB_ELEMS;
                    const int kel = krem < KB_ELEMS ? (int)krem : KB_ELEMS;
                    const int nmma = kel / 64;
                    const int na = (nmma + mma_per_atom - 1) / mma_per_atom;
                    const uint32_t bytes = A_STAGE + B_STAGE + (uint32_t)na * 512u * (1u + (uint32_t)nbands);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + stage * A_STAGE, &maps.a, &full[stage], kb * KB_BYTES, (int32_t)(mt * BM));
                    tma_load_2d(smem + OFF_B + stage * B_STAGE, &maps.b[w], &full[stage], kb * KB_BYTES,
                                (int32_t)(nt * BN));
                    const int64_t acol = (int64_t)kb * atoms_per_kb;
                    bulk_load(smem + OFF_SFA + stage * SFA_STAGE, p.a_scales + (mt * p.catoms + acol) * 512,
                              (uint32_t)na * 512u, &full[stage]);
                    for (int b = 0; b < nbands; ++b)
                        bulk_load(smem + OFF_SFB + stage * SFB_STAGE + b * 2048,
                                  p.b_scales[w] + ((nt * 2 + b) * p.catoms + acol) * 512, (uint32_t)na * 512u,
                                  &full[stage]);
                    issued[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            // never leave a copy in flight into shared memory we are about to release
            for (int s = 0; s < STAGES; ++s)
                if (issued[s]) mbar_wait(&full[s], last_phase[s]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc0 = idesc_mxf4(BM, BN, MX);
            const uint32_t idesc_hi = idesc_with_sf_id(idesc0, 2, 2);   // MXFP4: second MMA of an atom
            const uint64_t adesc0 = smem_desc(smem_u32(smem), 16, 1024, 2);
            const uint64_t bdesc0 = smem_desc(smem_u32(smem + OFF_B), 16, 1024, 2);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0, kpar = 0, kcount = 0;
            for (int64_t t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
                if (!mbar_wait(tmem_empty, acc_phase ^ 1)) { *abort_flag = 1; break; }
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full[stage], phase)) { *abort_flag = 1; break; }
                    if (!mbar_wait(&sf_ready[kpar], (kcount / SF_NBUF) & 1)) { *abort_flag = 1; break; }
                    tc_fence_after();
                    const int64_t krem = p.K - (int64_t)kb * KB_ELEMS;
                    const int nmma = krem < KB_ELEMS ? (int)(krem / 64) : 4;
                    const uint64_t ad = adesc0 + (uint64_t)(stage * (A_STAGE >> 4));
                    const uint64_t bd = bdesc0 + (uint64_t)(stage * (B_STAGE >> 4));
                    const uint32_t sfa = tmem + SF_COL + kpar * SF_BUF;
                    const uint32_t sfb = sfa + SFB_OFF;
                    uint32_t accf = kb > 0 ? 1u : 0u;
                    if (nmma == 4) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const int atom = MX ? kk / 2 : kk;
                            if (MX)
                                mma_mxf4(tmem + ACC_COL, ad + 2 * kk, bd + 2 * kk, (kk & 1) ? idesc_hi : idesc0,
                                         sfa + atom * 4, sfb + atom * 8, accf);
                            else
                                mma_nvf4(tmem + ACC_COL, ad + 2 * kk, bd + 2 * kk, idesc0, sfa + atom * 4,
                                         sfb + atom * 8, accf);
                            accf = 1u;
                        }
                    } else {
                        for (int kk = 0; kk < nmma; ++kk) {
                            const int atom = MX ? kk / 2 : kk;
                            if (MX)
                                mma_mxf4(tmem + ACC_COL, ad + 2 * kk, bd + 2 * kk, (kk & 1) ? idesc_hi : idesc0,
                                         sfa + atom * 4, sfb + atom * 8, accf);
                            else
                                mma_nvf4(tmem + ACC_COL, ad + 2 * kk, bd + 2 * kk, idesc0, sfa + atom * 4,
                                         sfb + atom * 8, accf);
                            accf = 1u;
                        }
                    }
                    tc_commit(&empty[stage]);
                    tc_commit(&sf_free[kpar]);
                    ++kcount;
                    kpar = kcount % SF_NBUF;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (*abort_flag) break;
                tc_commit(tmem_full);
                acc_phase ^= 1;
            }
            // all MMAs of this thread are complete before TMEM is released
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (warp < FIRST_EPI_WARP) {
        // scale warps: stage each k-block's scale atoms into a TMEM buffer
        const uint32_t quarter = (uint32_t)(warp & 3) * 32u;
        int stage = 0;
        uint32_t phase = 0, kpar = 0, kcount = 0;
        for (int64_t t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&full[stage], phase)) { *abort_flag = 1; break; }
                // the MMAs that read this buffer two k-blocks ago are done
                if (!mbar_wait(&sf_free[kpar], ((kcount / SF_NBUF) & 1) ^ 1)) { *abort_flag = 1; break; }
                tc_fence_after();
                const int64_t krem = p.K - (int64_t)kb * KB_ELEMS;
                const int nmma = krem < KB_ELEMS ? (int)(krem / 64) : 4;
                const int na = (nmma + mma_per_atom - 1) / mma_per_atom;
                stage_scales(tmem + (quarter << 16) + SF_COL + kpar * SF_BUF, smem + OFF_SFA + stage * SFA_STAGE,
                             smem + OFF_SFB + stage * SFB_STAGE, na, lane);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[kpar]);
                ++kcount;
                kpar = kcount % SF_NBUF;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else {
        const int quad = warp & 3;                 // TMEM lane quarter this warp may access
        const int half = (warp - FIRST_EPI_WARP) >> 2;   // which 128 accumulator columns
        const int row_in_tile = quad * 32 + lane;
        const float a_st = MX ? 1.0f : *p.a_gscale;
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + half * 128;
        const bool out_bf16 = p.out_bf16 != 0;
        const int order = warp - FIRST_EPI_WARP;          // position in the store-buffer turn chain
        uint8_t* buf = smem + OFF_EPI;
        uint32_t acc_phase = 0, iter = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++iter) {
            if (!mbar_wait(tmem_full, acc_phase)) { *abort_flag = 1; break; }
            tc_fence_after();
            const int w = gemm_weight_of(p, t);
            const int64_t lt = t - p.tile_start[w];
            const int64_t mt = lt % tiles_m, nt = lt / tiles_m;
            const int64_t row = mt * BM + row_in_tile;
            const int64_t col_base = nt * BN + half * 128;
            const float alpha = MX ? 1.0f : __fmul_rn(a_st, *p.b_gscale[w]);
            uint32_t pk[2][32];          // bf16 pairs: [0] columns 0..63, [1] columns 64..127
#pragma unroll
            for (int round = 0; round < 4; ++round) {
                uint32_t r[32];
                tmem_ld32(taddr + round * 32, r);
                tmem_ld_wait();
                if (round == 3) {
                    // the whole accumulator slice is in registers: let the next tile's MMAs start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tmem_empty);
                }
                if (out_bf16) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * j]) * alpha,
                                                                 __uint_as_float(r[2 * j + 1]) * alpha);
                        pk[round >> 1][(round & 1) * 16 + j] = *reinterpret_cast<uint32_t*>(&h);
                    }
                } else if (row < p.M) {
                    store_row32(p.y[w], p.N[w], row, col_base + round * 32, r, alpha, false);
                }
            }
            if (out_bf16) {
                // Turn in the chain of epilogue warps sharing the 8 KB buffer: the
                // warp's 32 rows x 128 columns go out as two 32 x 64 TMA boxes in
                // the 128-byte-swizzled layout (conflict-free writes, coalesced
                // stores; rows and columns outside Y are clipped by the TMA).
                const bool first = order == 0;
                if (!mbar_wait(&epi_turn[order], first ? ((iter & 1) ^ 1) : (iter & 1))) { *abort_flag = 1; break; }
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4*>(buf + b * 4096 + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                            make_uint4(pk[b][4 * c], pk[b][4 * c + 1], pk[b][4 * c + 2], pk[b][4 * c + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int32_t r0 = (int32_t)(mt * BM + quad * 32);
                    tma_store_2d(&maps.y[w], buf, (int32_t)col_base, r0);
                    tma_store_2d(&maps.y[w], buf + 4096, (int32_t)(col_base + 64), r0);
                    bulk_commit_group();
                    bulk_wait_read_all();
                    mbar_arrive(&epi_turn[(order + 1) % EPI_WARPS]);
                }
                __syncwarp();
            }
            acc_phase ^= 1;
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D byte tensor [rows, row_bytes] with a box of 128 bytes x box_rows and
// 128-byte swizzle (the operand layout the MMA descriptors describe).
static bool make_code_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output Y [M, N] bf16 for TMA stores of 32-row x 64-column boxes, 128-byte swizzle.
static bool make_out_map(CUtensorMap* map, void* y, int64_t M, int64_t N) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(N * 2)};
    cuuint32_t box[2] = {64u, 32u};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


// One quantized A times nw weights in one persistent launch (nw = 1: q4_gemm).
cudaError_t launch_gemm_multi(const GemmParams* ps, int nw, cudaStream_t st, int num_sms) {
    using namespace gemm;
    if (nw < 1 || nw > MAX_W) return cudaErrorInvalidValue;
    const GemmParams& p0 = ps[0];
    if (p0.M == 0) return cudaSuccess;
    GemmMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    GemmDev d;
    std::memset(&d, 0, sizeof(d));
    if (!make_code_map(&maps.a, p0.a_codes, p0.M, p0.K / 2, BM)) return cudaErrorInvalidValue;
    d.M = p0.M; d.K = p0.K;
    d.a_scales = p0.a_scales; d.a_gscale = p0.a_gscale;
    const int blk = p0.mxfp4 ? 32 : 16;
    d.catoms = ((p0.K / blk) + 3) / 4;
    d.out_bf16 = p0.out_bf16 ? 1 : 0;
    const int64_t tiles_m = (p0.M + BM - 1) / BM;
    int n = 0;
    int64_t tiles = 0;
    for (int i = 0; i < nw; ++i) {
        const GemmParams& p = ps[i];
        if (p.N == 0) continue;               // nothing to compute for this weight
        if (!make_code_map(&maps.b[n], p.b_codes, p.N, p.K / 2, BN)) return cudaErrorInvalidValue;
        if (p.out_bf16 && !make_out_map(&maps.y[n], p.y, p.M, p.N)) return cudaErrorInvalidValue;
        d.N[n] = p.N;
        d.b_scales[n] = p.b_scales;
        d.b_gscale[n] = p.b_gscale;
        d.y[n] = p.y;
        d.tile_start[n] = tiles;
        tiles += tiles_m * ((p.N + BN - 1) / BN);
        ++n;
    }
    if (n == 0) return cudaSuccess;
    d.nw = n;
    for (int i = n; i <= MAX_W; ++i) d.tile_start[i] = tiles;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    cudaError_t e;
    if (p0.mxfp4) {
        e = cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        gemm_kernel<true><<<grid, THREADS, SMEM_BYTES, st>>>(maps, d);
    } else {
        e = cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        gemm_kernel<false><<<grid, THREADS, SMEM_BYTES, st>>>(maps, d);
    }
    return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p, cudaStream_t st, int num_sms) {
    if (p.M == 0 || p.N == 0) return cudaSuccess;
    return launch_gemm_multi(&p, 1, st, num_sms);
}

// ------------------------------------------------------------------ W4A16 GEMM
// Y = alpha * X dec(W)^T with bf16 activations X [M, K] and a 4-bit weight W
// [N, K] (codes + tensor-core scale atoms): the weight is dequantized in
// shared memory to bf16 -- code * block scale is exact in bf16 (at most 6
// significant bits, exponent in range) -- and multiplied on the tcgen05 tensor
// cores (kind::f16, bf16 x bf16 -> fp32).  alpha = s_t (NVFP4) or 1 (MXFP4) is
// applied in the epilogue.  Persistent CTAs over 128 x 256 output tiles:
//   warp 0       TMA producer: per k-stage of 64 elements, the X tile
//                (128 rows x 128 B, 128-byte swizzle), the weight code tile
//                (256 rows x 32 B) and the two scale atoms of its row bands,
//                into a 5-deep ring (a stage is free once the converters have
//                read its codes and the MMAs its X tile);
//   warp 1       TMEM owner (two 256-column accumulators) and MMA issuer:
//                four 128 x 256 x 16 MMAs per k-stage;
//   warps 2..9   converters: thread r dequantizes weight row r of the stage
//                (64 codes) into one of two bf16 operand tiles, in the
//                swizzled K-major layout the MMA descriptors describe;
//   warps 10..13 epilogue: drain an accumulator (one warp per TMEM lane
//                quarter, 256 columns in two halves), release it to the MMAs
//                of the next-but-one tile, scale, convert and store Y.
namespace w16 {
constexpr int BM = 128;                  // X rows of one MMA / one TMEM accumulator
constexpr int SUBS = 2;                  // at most this many X row blocks per tile: every
                                         // converted weight tile feeds one MMA per block
constexpr int BN = 256;
constexpr int KS = 64;                   // k elements per stage
constexpr int A_STAGE = BM * 128;        // one bf16 X row block
constexpr int C_STAGE = BN * 32;         // weight codes
constexpr int S_STAGE = 1024;            // two scale atoms
// A stage holds `subs` X row blocks, the codes and the scale atoms (25 or 41 KB,
// multiples of 1024); the ring is 5 stages deep with one block, 3 with two.
constexpr int MAX_STAGES = 5;
__host__ __device__ constexpr int stage_bytes(int subs) { return subs * A_STAGE + C_STAGE + S_STAGE; }
__host__ __device__ constexpr int ring_stages(int subs) { return subs == 1 ? 5 : 3; }
static_assert(stage_bytes(1) % 1024 == 0 && stage_bytes(2) % 1024 == 0, "stage alignment");
constexpr int BSLOTS = 2;                // converted bf16 weight tiles
constexpr int B_SLOT = BN * 128;
constexpr int OFF_B = ring_stages(1) * stage_bytes(1) > ring_stages(2) * stage_bytes(2)
                          ? ring_stages(1) * stage_bytes(1) : ring_stages(2) * stage_bytes(2);
constexpr int OFF_EPI = OFF_B + BSLOTS * B_SLOT;
constexpr int EPI_WARPS = 4;
constexpr int EPI_BYTES = 8192;          // per epilogue warp: 32 rows x 128 bf16
constexpr int OFF_BAR = OFF_EPI + EPI_WARPS * EPI_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
constexpr int CONV_WARPS = 8;
constexpr int FIRST_CONV = 2;
constexpr int FIRST_EPI = FIRST_CONV + CONV_WARPS;
constexpr int THREADS = 32 * (FIRST_EPI + EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;      // SUBS accumulators of BN columns
static_assert(SUBS * BN <= (int)TMEM_COLS && SMEM_BYTES <= 232448, "W4A16 tile resources");
}  // namespace w16

// Instruction descriptor of tcgen05.mma kind::f16: fp32 D (bits 4-5 = 1),
// bf16 A and B (bits 7-9 and 10-12 = 1), both K-major, N >> 3 at bit 17,
// M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// Two E2M1 codes (one byte, element 0 low) times a block scale, as a packed
// bf16 pair, through the hardware E2M1 -> f16 conversion (the conversion
// pipe; the byte-permute form above uses the integer pipe).
__device__ __forceinline__ uint32_t dequant2_bf16(uint32_t byte, float2 s) {
    const float2 v = mul2_rn(e2m1x2_value(byte), s);
    uint32_t out;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(out) : "f"(v.x), "f"(v.y));
    return out;
}

// a * b on packed bf16 pairs (exact here: code value times a block scale has
// at most 6 significant bits).
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

struct W16Dev {
    int64_t M, N, K;
    const uint8_t* w_scales;
    const float* b_gscale;
    void* y;
    int64_t catoms;
    int out_bf16;
    int subs;                // X row blocks per tile (1 or 2)
};

template <bool MX>
__global__ void __launch_bounds__(w16::THREADS, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmY, W16Dev p) {
    using namespace w16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);    // [stages] X, codes, scales landed
    uint64_t* empty = full + MAX_STAGES;                             // [stages] converters read it, MMAs done
    uint64_t* b_full = empty + MAX_STAGES;                           // [BSLOTS] weight tile converted
    uint64_t* b_empty = b_full + BSLOTS;                             // [BSLOTS] its MMAs are done
    uint64_t* tmem_full = b_empty + BSLOTS;                          // [2]
    uint64_t* tmem_empty = tmem_full + 2;                            // [2]
    uint64_t* mma_done = tmem_empty + 2;
    uint64_t* cfull = mma_done + 1;                                  // [stages] codes, scales landed
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(cfull + MAX_STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int subs = p.subs;
    const int STAGES = ring_stages(subs), STAGE = stage_bytes(subs);
    const int OFF_C = subs * A_STAGE, OFF_S = OFF_C + C_STAGE;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&cfull[s], 1);
            mbar_init(&empty[s], CONV_WARPS + 1);        // every converter warp + the MMA commit
        }
        for (int b = 0; b < BSLOTS; ++b) { mbar_init(&b_full[b], CONV_WARPS); mbar_init(&b_empty[b], 1); }
        for (int b = 0; b < SUBS; ++b) { mbar_init(&tmem_full[b], 1); mbar_init(&tmem_empty[b], EPI_WARPS); }
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_holder, TMEM_COLS); tmem_relinquish(); }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmC);
        if (p.out_bf16) tma_prefetch_desc(&tmY);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int64_t tiles_m = (p.M + subs * BM - 1) / (subs * BM);
    const int64_t tiles = tiles_m * ((p.N + BN - 1) / BN);
    const int nks = (int)(p.K / KS);
    const int64_t bands = (p.N + 127) / 128;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_phase[MAX_STAGES];
            bool issued[MAX_STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, last_phase[s] = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int64_t mt = t % tiles_m, nt = t / tiles_m;
                const int nb = (nt * 2 + 1 < bands) ? 2 : 1;
                for (int ks = 0; ks < nks; ++ks) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
                    uint8_t* st = smem + stage * STAGE;
                    // the weight codes and scale atoms first, on their own barrier: the
                    // converters start while the X row blocks are still landing
                    mbar_arrive_expect_tx(&cfull[stage], (uint32_t)(C_STAGE + nb * 512));
                    tma_load_2d(st + OFF_C, &tmC, &cfull[stage], ks * (KS / 2), (int32_t)(nt * BN));
                    // scale atom column of this stage: 64 elements = 4 NVFP4 blocks = one
                    // atom column; 2 MXFP4 blocks = half of one
                    const int64_t acol = MX ? ks / 2 : ks;
                    for (int b = 0; b < nb; ++b)
                        bulk_load(st + OFF_S + b * 512, p.w_scales + ((nt * 2 + b) * p.catoms + acol) * 512, 512u,
                                  &cfull[stage]);
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)(subs * A_STAGE));
                    // every X row block of the tile (rows past M read as zeros)
                    for (int sb = 0; sb < subs; ++sb)
                        tma_load_2d(st + sb * A_STAGE, &tmX, &full[stage], ks * KS,
                                    (int32_t)(mt * subs * BM + sb * BM));
                    issued[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            for (int s = 0; s < STAGES; ++s)
                if (issued[s]) {
                    mbar_wait(&cfull[s], last_phase[s]);
                    mbar_wait(&full[s], last_phase[s]);
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, BN);
            int stage = 0, bs = 0;
            uint32_t phase = 0, bphase = 0;
            uint32_t uses[SUBS] = {};            // tiles each accumulator has served
            bool ok = true;
            for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int64_t mt = t % tiles_m;
                // X row blocks of this tile that hold rows of X (a partial last tile skips the rest)
                const int nsub = (int)min((int64_t)subs, (p.M - mt * subs * BM + BM - 1) / BM);
                for (int ks = 0; ks < nks && ok; ++ks) {
                    if (!mbar_wait(&full[stage], phase) || !mbar_wait(&b_full[bs], bphase)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t bd = smem_desc(smem_u32(smem + OFF_B + bs * B_SLOT), 16, 1024, 2);
                    for (int sb = 0; sb < nsub; ++sb) {
                        if (ks == 0) {
                            // accumulator sb drained by the epilogue of its previous tile
                            if (!mbar_wait(&tmem_empty[sb], (uses[sb] & 1) ^ 1)) { ok = false; break; }
                            tc_fence_after();
                        }
                        const uint64_t ad = smem_desc(smem_u32(smem + stage * STAGE + sb * A_STAGE), 16, 1024, 2);
                        const uint32_t acc = tmem + sb * BN;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16(acc, ad + 2 * kk, bd + 2 * kk, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                        if (ks == nks - 1) tc_commit(&tmem_full[sb]);
                    }
                    if (!ok) break;
                    tc_commit(&empty[stage]);
                    tc_commit(&b_empty[bs]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    if (++bs == BSLOTS) { bs = 0; bphase ^= 1; }
                }
                for (int sb = 0; sb < nsub; ++sb) ++uses[sb];
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (warp < FIRST_EPI) {
        // ---- converters: thread r owns weight row r of every stage
        const int r = threadIdx.x - 32 * FIRST_CONV;
        int stage = 0, bs = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const int64_t nt = t / tiles_m;
            const bool row_ok = nt * BN + r < p.N;
            for (int ks = 0; ks < nks; ++ks) {
                if (!mbar_wait(&cfull[stage], phase) || !mbar_wait(&b_empty[bs], bphase ^ 1)) { ok = false; break; }
                uint8_t* st = smem + stage * STAGE;
                const uint4 c0 = *reinterpret_cast<const uint4*>(st + OFF_C + r * 32);
                const uint4 c1 = *reinterpret_cast<const uint4*>(st + OFF_C + r * 32 + 16);
                // the row's 4 scale bytes of this atom column: byte j = scale column j
                const uint32_t sw = *reinterpret_cast<const uint32_t*>(st + OFF_S + (r >> 7) * 512 + (r & 31) * 16 +
                                                                       ((r >> 5) & 3) * 4);
                // block scales as packed bf16 pairs (exact: E4M3 has 4 significant
                // bits, E8M0 is a power of two): sp[j] for elements 16j .. 16j + 15
                uint32_t sp[4];
                if (MX) {
                    const int j0 = (ks & 1) * 2;
                    const uint32_t a = __float_as_uint(exp2_int((int)((sw >> (8 * j0)) & 0xFFu) - 127)) >> 16;
                    const uint32_t b = __float_as_uint(exp2_int((int)((sw >> (8 * (j0 + 1))) & 0xFFu) - 127)) >> 16;
                    sp[0] = sp[1] = a | (a << 16);
                    sp[2] = sp[3] = b | (b << 16);
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t h = __float_as_uint(e4m3_value((sw >> (8 * j)) & 0xFFu)) >> 16;
                        sp[j] = h | (h << 16);
                    }
                }
                const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint8_t* brow = smem + OFF_B + bs * B_SLOT + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {          // 16-byte chunk c: elements 8c .. 8c + 7
                    const uint32_t sc = sp[c >> 1];
                    uint4 v;
                    if (c & 1) {
                        // odd chunks through the conversion pipe, even ones through the
                        // integer pipe: neither pipe alone sets the pace
                        const float f = __uint_as_float(sc << 16);
                        const float2 f2 = make_float2(f, f);
                        v = make_uint4(dequant2_bf16(cw[c] & 0xFFu, f2), dequant2_bf16((cw[c] >> 8) & 0xFFu, f2),
                                       dequant2_bf16((cw[c] >> 16) & 0xFFu, f2), dequant2_bf16(cw[c] >> 24, f2));
                    } else {
                        uint32_t o[4];
                        e2m1x8_to_bf16(cw[c], o);
                        v = make_uint4(mul_bf16x2(o[0], sc), mul_bf16x2(o[1], sc), mul_bf16x2(o[2], sc),
                                       mul_bf16x2(o[3], sc));
                    }
                    if (!row_ok) v = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4*>(brow + ((c ^ (r & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                // every code and scale of the stage has been used, so no lane's
                // shared-memory load of it is still in flight: it may be refilled
                if (lane == 0) {
                    mbar_arrive(&empty[stage]);
                    mbar_arrive(&b_full[bs]);
                }
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
                if (++bs == BSLOTS) { bs = 0; bphase ^= 1; }
            }
        }
    } else {
        // ---- epilogue: one warp per TMEM lane quarter, 256 columns in two halves,
        // each half through the warp's own 8 KB buffer and two TMA stores
        const int e = warp - FIRST_EPI;
        const int quad = warp & 3;
        const float alpha = MX ? 1.0f : *p.b_gscale;
        const bool out_bf16 = p.out_bf16 != 0;
        uint8_t* buf = smem + OFF_EPI + e * EPI_BYTES;
        uint32_t uses[SUBS] = {};
        bool ok = true;
        for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
          const int64_t mt = t % tiles_m, nt = t / tiles_m;
          const int nsub = (int)min((int64_t)subs, (p.M - mt * subs * BM + BM - 1) / BM);
          for (int ab = 0; ab < nsub; ++ab) {
            if (!mbar_wait(&tmem_full[ab], uses[ab] & 1)) { ok = false; break; }
            ++uses[ab];
            tc_fence_after();
            const int64_t row0 = mt * subs * BM + ab * BM;
            const int64_t row = row0 + quad * 32 + lane;
            for (int half = 0; half < 2; ++half) {
                const int64_t col_base = nt * BN + half * 128;
                const uint32_t taddr = tmem + ab * BN + ((uint32_t)(quad * 32) << 16) + half * 128;
                if (out_bf16) {
                    // the previous stores from this buffer have finished reading it
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                }
#pragma unroll
                for (int round = 0; round < 4; ++round) {
                    uint32_t v[32];
                    tmem_ld32(taddr + round * 32, v);
                    tmem_ld_wait();
                    if (half == 1 && round == 3) {
                        // the accumulator is drained: the next tile's MMAs may use it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tmem_empty[ab]);
                    }
                    if (out_bf16) {
                        // columns 32*round .. +31 of this half: 16-byte chunks 4*(round&1) .. +3
                        // of the 32 x 64 box round / 2, 128-byte swizzled
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * alpha,
                                                                     __uint_as_float(v[2 * j + 1]) * alpha);
                            pk[j] = *reinterpret_cast<uint32_t*>(&h);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int c = (round & 1) * 4 + q;
                            *reinterpret_cast<uint4*>(buf + (round >> 1) * 4096 + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                        }
                    } else if (row < p.M) {
                        store_row32(p.y, p.N, row, col_base + round * 32, v, alpha, false);
                    }
                }
                if (out_bf16) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int32_t r0 = (int32_t)(row0 + quad * 32);
                        tma_store_2d(&tmY, buf, (int32_t)col_base, r0);
                        tma_store_2d(&tmY, buf + 4096, (int32_t)(col_base + 64), r0);
                        bulk_commit_group();
                    }
                    __syncwarp();
                }
            }
          }
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

cudaError_t launch_w4a16(const W4A16Params& p, cudaStream_t st, int num_sms) {
    using namespace w16;
    if (p.M == 0 || p.N == 0) return cudaSuccess;
    CUtensorMap mx, mc, my;
    std::memset(&my, 0, sizeof(my));
    if (!encode_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, (uint64_t)p.K, (uint64_t)p.M, (uint64_t)p.K * 2,
                       64u, (uint32_t)BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.b_codes, (uint64_t)(p.K / 2), (uint64_t)p.N,
                       (uint64_t)(p.K / 2), 32u, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (p.out_bf16 && !make_out_map(&my, p.y, p.M, p.N)) return cudaErrorInvalidValue;
    W16Dev d;
    d.M = p.M; d.N = p.N; d.K = p.K;
    d.w_scales = p.b_scales; d.b_gscale = p.b_gscale; d.y = p.y;
    d.catoms = ((p.K / (p.mxfp4 ? 32 : 16)) + 3) / 4;
    d.out_bf16 = p.out_bf16 ? 1 : 0;
    d.subs = 1;
    // two X row blocks per tile (each converted weight tile feeds two MMAs) when
    // the tiles still cover every SM, else one (more tiles, a deeper ring)
    const int64_t tiles_n = (p.N + BN - 1) / BN;
    d.subs = ((p.M + 2 * BM - 1) / (2 * BM)) * tiles_n >= num_sms ? 2 : 1;
    const int64_t tiles = ((p.M + d.subs * BM - 1) / (d.subs * BM)) * tiles_n;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    cudaError_t e;
    if (p.mxfp4) {
        e = cudaFuncSetAttribute(w4a16_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        w4a16_gemm_kernel<true><<<grid, THREADS, SMEM_BYTES, st>>>(mx, mc, my, d);
    } else {
        e = cudaFuncSetAttribute(w4a16_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        w4a16_gemm_kernel<false><<<grid, THREADS, SMEM_BYTES, st>>>(mx, mc, my, d);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------ Sigma-Delta fused into the GEMM producer
// One loop visit of the looped core with the code generation moved into the
// GEMM ("Looped Transformer quantization", sec. 4: codes generated online from
// the reference weight and the residue state at every visit): for a small
// batch X (M <= 16 bf16 rows) and the FP32 master weight W [N, K] with fixed
// NVFP4 block scales,
//     q = E2M1(W / S + r),  r <- (W / S + r) - q,  Y = s_t * X (q * s_b)^T,
// where the codes q never leave the chip: each weight element is read once
// with its residue, the new residue is written back, and the dequantized
// weight q * s_b (exact in bf16) is the tensor-core operand.  The product is
// W4A16-style (bf16 activations) and operands are swapped so the weight fills
// the MMA's 128-row side (tcgen05 kind::f16, 128 x 16 x 16).
// A CTA owns 128 weight rows and one slice of K; the KS slices of a row band
// form a thread-block cluster whose partial outputs are summed through
// distributed shared memory by the cluster's first CTA.  A CTA holds one
// 85 KB stage, so two CTAs share an SM and one's set-up, first loads and
// reduction overlap the other's stream:
//   warp 0      TMA producer: per k-stage of 64 the W and r tiles (two
//               128-row x 128-byte boxes each, 128-byte swizzle), the block
//               scale atom and the X tile (np rows x 128 bytes, swizzled);
//   warp 1      TMEM owner and MMA issuer;
//   warps 2..5  Sigma-Delta: thread = weight row; the new residue replaces the
//               old one in the stage (then one TMA store per box) and the
//               dequantized bf16 row goes to the swizzled A operand tile;
//   warps 6..9  epilogue: accumulator -> shared memory, cluster reduction,
//               Y = s_t * sum by the cluster's first CTA.
namespace sdg {
constexpr int BM = 128;
constexpr int KSTAGE = 64;
constexpr int STAGES = 1;                // per CTA; two CTAs share an SM
constexpr int OFF_W = 0;                 // 2 boxes x 16 KB fp32
constexpr int OFF_R = 32768;             // 2 boxes x 16 KB fp32
constexpr int OFF_A = 65536;             // 128 x 128 B bf16 operand
constexpr int OFF_X = 81920;             // 16 x 128 B bf16 operand
constexpr int OFF_SF = OFF_X + 2048;     // one scale atom
constexpr int STAGE = 85 * 1024;
constexpr int OFF_RED = STAGES * STAGE;  // fp32 partial tile [128][16]
constexpr int OFF_BAR = OFF_RED + BM * 16 * 4;
constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024 + 1024;   // barriers, (S, 1/S) table, alignment
constexpr int CONV_WARPS = 8;            // two threads per weight row, one per 32-element box
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (2 + CONV_WARPS + EPI_WARPS);
constexpr uint32_t TMEM_COLS = 32;
constexpr int MAX_KS = 8;
static_assert((32 * CONV_WARPS) % BM == 0 && 32 * CONV_WARPS / BM <= 2, "converter threads per weight row");
}  // namespace sdg

struct SdgDev {
    int64_t M, N, K;
    const uint8_t* scales;   // tensor-core layout
    const float* gscale;
    void* y;
    int64_t catoms;
    int kslice;              // K elements per CTA (a multiple of 64)
    int out_bf16;
};

__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
    return v;
}

// One CTA of the fused step + GEMM: K slice `rank` of the 128-row band `band`
// of the entry described by (tmW, tmR, tmX, p).
__device__ __forceinline__ void sd_gemm_cta(const CUtensorMap& tmW, const CUtensorMap& tmR, const CUtensorMap& tmX,
                                            const SdgDev& p, int64_t band) {
    using namespace sdg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);   // [STAGES] W, r, X, scales landed
    uint64_t* conv = full + STAGES;                                 // [STAGES] residue + operand written
    uint64_t* empty = conv + STAGES;                                // [STAGES] MMAs done + residue stored
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* mma_done = tmem_full + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    float2* nv_tab = reinterpret_cast<float2*>(smem + OFF_BAR + 512);   // 128 (S, 1/S) entries
    float* red = reinterpret_cast<float*>(smem + OFF_RED);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();                        // K slice of this CTA
    const int64_t row0 = band * BM;
    const int64_t k_begin = (int64_t)rank * p.kslice;
    const int nst = p.kslice / KSTAGE;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], CONV_WARPS);
            mbar_init(&empty[s], 2);                                // MMA commit + residue-store release
        }
        mbar_init(tmem_full, 1);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_holder, TMEM_COLS); tmem_relinquish(); }
    if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmR); tma_prefetch_desc(&tmX); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t phase = 0;
            int stage = 0;
            uint32_t last_phase[STAGES];
            bool issued[STAGES] = {};
            for (int i = 0; i < nst; ++i) {
                if (!mbar_wait(&empty[stage], phase ^ 1)) break;
                uint8_t* st = smem + stage * STAGE;
                const int32_t k0 = (int32_t)(k_begin + (int64_t)i * KSTAGE);
                mbar_arrive_expect_tx(&full[stage], 2 * 2 * 16384 + 2048 + 512);
                for (int b = 0; b < 2; ++b) {
                    tma_load_2d(st + OFF_W + b * 16384, &tmW, &full[stage], k0 + 32 * b, (int32_t)row0);
                    tma_load_2d(st + OFF_R + b * 16384, &tmR, &full[stage], k0 + 32 * b, (int32_t)row0);
                }
                tma_load_2d(st + OFF_X, &tmX, &full[stage], k0, 0);
                bulk_load(st + OFF_SF, p.scales + (band * p.catoms + k0 / 64) * 512, 512u, &full[stage]);
                issued[stage] = true;
                last_phase[stage] = phase;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            for (int s = 0; s < STAGES; ++s)
                if (issued[s]) mbar_wait(&full[s], last_phase[s]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, 16);
            uint32_t phase = 0;
            int stage = 0;
            bool ok = true;
            for (int i = 0; i < nst; ++i) {
                if (!mbar_wait(&full[stage], phase) || !mbar_wait(&conv[stage], phase)) { ok = false; break; }
                tc_fence_after();
                uint8_t* st = smem + stage * STAGE;
                const uint64_t ad = smem_desc(smem_u32(st + OFF_A), 16, 1024, 2);
                const uint64_t bd = smem_desc(smem_u32(st + OFF_X), 16, 1024, 2);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&empty[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (ok) tc_commit(tmem_full);
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (warp < 2 + CONV_WARPS) {
        // ---- Sigma-Delta on weight row rr of each stage, box(es) hb, hb + BPR, ...
        const int ct = threadIdx.x - 64;
        constexpr int CT = 32 * CONV_WARPS;
        constexpr int BPR = CT / BM;                 // threads per weight row
        const int rr = ct % BM, hb = ct / BM;
        const float s_t = *p.gscale;
        nv_fill_table(s_t, nv_tab, ct, CT);
        named_barrier(1, CT);
        const bool row_ok = row0 + rr < p.N;
        uint32_t phase = 0;
        int stage = 0;
        for (int i = 0; i < nst; ++i) {
            const bool got = mbar_wait(&full[stage], phase);
            uint8_t* st = smem + stage * STAGE;
            const uint32_t sw = *reinterpret_cast<const uint32_t*>(st + OFF_SF + (rr & 31) * 16 + ((rr >> 5) & 3) * 4);
            uint8_t* arow = st + OFF_A + (rr >> 3) * 1024 + (rr & 7) * 128;
#pragma unroll
            for (int b = hb; b < 2; b += BPR) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    // elements e = 32b + 4c .. +3 of the stage, block j = e / 16
                    const int j = 2 * b + (c >> 2);
                    const uint32_t sb = (sw >> (8 * j)) & 0xFFu;
                    const float2 sy = nv_tab[sb & 0x7Fu];
                    const uint32_t off = (uint32_t)(b * 16384 + rr * 128 + ((c ^ (rr & 7)) << 4));
                    const float4 w4 = *reinterpret_cast<const float4*>(st + OFF_W + off);
                    float4* rp = reinterpret_cast<float4*>(st + OFF_R + off);
                    const float4 r4 = *rp;
                    float2 x01, x23;
                    if (sy.y != sy.y) {
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
                    const float2 q01 = e2m1x2_value(codes & 0xFFu), q23 = e2m1x2_value(codes >> 8);
                    const float2 n01 = sub2_rn(v01, q01), n23 = sub2_rn(v23, q23);
                    *rp = make_float4(n01.x, n01.y, n23.x, n23.y);
                    // dequantized weight q * s_b (exact in bf16), 4 elements = 8 bytes
                    const float sv = e4m3_value(sb & 0x7Fu);
                    uint32_t d0, d1;
                    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(d0) : "f"(q01.x * sv), "f"(q01.y * sv));
                    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(d1) : "f"(q23.x * sv), "f"(q23.y * sv));
                    if (!row_ok) d0 = d1 = 0u;
                    const int e2 = 64 * b + 8 * c;        // byte offset of the 4 bf16 in the 128-byte row
                    *reinterpret_cast<uint2*>(arow + ((((e2 >> 4) ^ (rr & 7)) & 7) << 4) + (e2 & 15)) =
                        make_uint2(d0, d1);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[stage]);
            // every row is done: store the new residue tile, release the stage once it is read
            named_barrier(1, CT);
            if (ct == 0) {
                if (got) {
                    const int32_t k0 = (int32_t)(k_begin + (int64_t)i * KSTAGE);
                    for (int b = 0; b < 2; ++b) tma_store_2d(&tmR, st + OFF_R + b * 16384, k0 + 32 * b, (int32_t)row0);
                    bulk_commit_group();
                    bulk_wait_read_all();
                }
                mbar_arrive(&empty[stage]);
            }
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ct == 0) bulk_wait_all();
    } else {
        // ---- epilogue: partial tile to shared memory, cluster reduction
        const int quad = warp & 3;
        const int rr = quad * 32 + lane;
        const bool ok = mbar_wait(tmem_full, 0);
        tc_fence_after();
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16), v);
        tmem_ld_wait();
#pragma unroll
        for (int m = 0; m < 16; ++m) red[rr * 16 + m] = ok ? __uint_as_float(v[m]) : 0.0f;
    }
    // every CTA's partial tile is in its shared memory
    __syncthreads();
    cluster_sync();
    if (warp >= 2 + CONV_WARPS && rank == 0) {
        const int quad = warp & 3;
        const int rr = quad * 32 + lane;
        const int64_t n = row0 + rr;
        const float s_t = *p.gscale;
        const uint32_t ks = (uint32_t)(p.K / p.kslice);
        // this row's 16 partial sums, then each peer's 16 added in rank order;
        // a peer's row comes as four independent 16-byte loads, not a chain of
        // dependent scalar loads
        float acc[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) acc[m] = red[rr * 16 + m];
        const uint32_t row_addr = smem_u32(&red[rr * 16]);
        for (uint32_t q = 1; q < ks; ++q) {
            const uint32_t peer = mapa_shared(row_addr, q);
            float4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = ld_shared_cluster_v4(peer + 16u * c);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                acc[4 * c] += v[c].x;
                acc[4 * c + 1] += v[c].y;
                acc[4 * c + 2] += v[c].z;
                acc[4 * c + 3] += v[c].w;
            }
        }
        if (n < p.N) {
            for (int m = 0; m < p.M; ++m) {
                const float val = acc[m] * s_t;
                if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[(int64_t)m * p.N + n] = __float2bfloat16_rn(val);
                else reinterpret_cast<float*>(p.y)[(int64_t)m * p.N + n] = val;
            }
        }
    }
    // the first CTA has read every partial tile before any CTA leaves
    __syncthreads();
    cluster_sync();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

__global__ void __launch_bounds__(sdg::THREADS, 2)
    sd_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmR,
                          const __grid_constant__ CUtensorMap tmX, SdgDev p) {
    sd_gemm_cta(tmW, tmR, tmX, p, (int64_t)blockIdx.y);
}

// Grouped: the row bands of all entries are the grid's y range, entry e
// owning bands [band_start[e], band_start[e + 1]); every entry has the same K
// and the same K split (the cluster shape is one per launch).
struct SdgItem {
    CUtensorMap w, r, x;
    SdgDev d;
};
struct SdgGroup {
    int count;
    int band_start[kMaxGroup + 1];
    SdgItem m[kMaxGroup];
};
static_assert(sizeof(SdgGroup) <= 32764, "kernel parameter space");

__global__ void __launch_bounds__(sdg::THREADS, 2) sd_gemm_grouped_kernel(const __grid_constant__ SdgGroup g) {
    int e = 0;
    while (e + 1 < g.count && (int)blockIdx.y >= g.band_start[e + 1]) ++e;
    const SdgItem& it = g.m[e];
    sd_gemm_cta(it.w, it.r, it.x, it.d, (int64_t)blockIdx.y - g.band_start[e]);
}

bool sd_gemm_supported(int64_t M, int64_t K) { return M >= 1 && M <= 16 && K % 64 == 0 && K > 0; }

// K slices per row band (the cluster size, 1 to 8, dividing K into 64-element
// stages) for `bands` row bands on `num_sms` SMs (two CTAs per SM at a time):
// the one with the least estimated time waves * (T0 + stages per CTA * TS),
// T0 ~ 8 us the fixed cost of a CTA (set-up, first loads, cluster reduction)
// and TS ~ 1.9 us a 64-element stage, both measured on the looped-core shapes
// with one two-stage CTA per SM (K = 1024: splits 1 / 2 / 4 / 8 took 118 /
// 120 / 155 / 261 us for 320 bands).  One single-stage CTA beside another on
// the same SM overlaps one CTA's set-up and reduction with the other's stream.
static int choose_ksplit(int64_t bands, int64_t K, int num_sms) {
    constexpr double T0 = 8.0, TS = 1.9;
    int best_ks = 1;
    double best_t = 1e300;
    for (int ks = 1; ks <= sdg::MAX_KS; ks *= 2) {
        if (K % (64 * ks)) break;
        const double waves = std::ceil((double)(bands * ks) / (2 * num_sms));
        const double t = waves * (T0 + (double)(K / ks / 64) * TS);
        if (t < best_t) { best_t = t; best_ks = ks; }
    }
    return best_ks;
}

cudaError_t launch_sd_gemm(const SdGemmParams& p, cudaStream_t st, int num_sms) {
    using namespace sdg;
    if (p.M == 0 || p.N == 0) return cudaSuccess;
    const int64_t tiles = (p.N + BM - 1) / BM;
    const int ks = choose_ksplit(tiles, p.K, num_sms);
    CUtensorMap mw, mr, mx;
    if (!encode_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.w, (uint64_t)p.K, (uint64_t)p.N, (uint64_t)p.K * 4, 32u,
                       (uint32_t)BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_2d(&mr, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.residue, (uint64_t)p.K, (uint64_t)p.N,
                       (uint64_t)p.K * 4, 32u, (uint32_t)BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, (uint64_t)p.K, (uint64_t)p.M, (uint64_t)p.K * 2, 64u,
                       16u, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    SdgDev d;
    d.M = p.M; d.N = p.N; d.K = p.K; d.scales = p.scales; d.gscale = p.gscale; d.y = p.y;
    d.catoms = ((p.K / 16) + 3) / 4;
    d.kslice = (int)(p.K / ks);
    d.out_bf16 = p.out_bf16 ? 1 : 0;
    cudaError_t e = cudaFuncSetAttribute(sd_gemm_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ks, (unsigned)tiles, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, sd_gemm_decode_kernel, mw, mr, mx, d);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Grouped launch: every entry has the same M, K and output type; the K split
// comes from the same estimate over all entries' bands.
cudaError_t launch_sd_gemm_grouped(const SdGemmParams* items, int count, cudaStream_t st, int num_sms) {
    using namespace sdg;
    if (count <= 0) return cudaSuccess;
    SdgGroup g;                         // the kernel parameter, staged on the host (14 KB)
    std::memset(&g, 0, sizeof(g));
    g.count = count;
    int bands = 0;
    for (int i = 0; i < count; ++i) {
        g.band_start[i] = bands;
        bands += (int)((items[i].N + BM - 1) / BM);
    }
    g.band_start[count] = bands;
    const int ks = choose_ksplit(bands, items[0].K, num_sms);
    for (int i = 0; i < count; ++i) {
        const SdGemmParams& p = items[i];
        SdgItem& it = g.m[i];
        if (!encode_map_2d(&it.w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.w, (uint64_t)p.K, (uint64_t)p.N,
                           (uint64_t)p.K * 4, 32u, (uint32_t)BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_map_2d(&it.r, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.residue, (uint64_t)p.K, (uint64_t)p.N,
                           (uint64_t)p.K * 4, 32u, (uint32_t)BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_map_2d(&it.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.x, (uint64_t)p.K, (uint64_t)p.M,
                           (uint64_t)p.K * 2, 64u, 16u, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        SdgDev& d = it.d;
        d.M = p.M; d.N = p.N; d.K = p.K; d.scales = p.scales; d.gscale = p.gscale; d.y = p.y;
        d.catoms = ((p.K / 16) + 3) / 4;
        d.kslice = (int)(p.K / ks);
        d.out_bf16 = p.out_bf16 ? 1 : 0;
    }
    cudaError_t e = cudaFuncSetAttribute(sd_gemm_grouped_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ks, (unsigned)bands, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, sd_gemm_grouped_kernel, g);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ fused decode
// Small-M GEMM (M <= 16) with the activation quantization inside the kernel:
// no bf16 activation round trip and no workspace.  Operands are swapped so the
// weight fills the MMA's 128-row side: D^T[n, m] = sum_k W[n, k] X[m, k], with
// MMA N = np (M rounded up to 16).  Persistent CTAs over 128-row weight tiles:
//   warp 0      TMA producer: per k-block of 256, the weight code tile
//               (128 rows x 128 B, 128-byte swizzle) and its 4 scale atoms
//               into a deep ring (the weight stream is the kernel's HBM
//               traffic);
//   warp 1      TMEM owner and MMA issuer: per k-block up to four
//               128 x np x 64 block-scaled MMAs into four accumulators;
//   warp 2      TMA producer of the bf16 activations: one 2-D tile of M rows
//               x 256 elements per k-block into a ring of its own, as deep as
//               shared memory allows, so their loads never queue behind one
//               another (a register-staged load a few k-blocks ahead waited
//               out the latency of the weight stream in flight at each step);
//   warps 3..10 quantize the landed activation tiles once per CTA into a
//               resident buffer (codes in the swizzled K-major operand layout,
//               scales packed per k-block) while the weight tiles stream in;
//   warps 11-14 stage each k-block's weight and activation scale atoms into
//               TMEM (tcgen05.st, off the MMA thread: a tcgen05.cp there would
//               queue with the MMAs), then run the epilogue: the summed
//               accumulator lanes (= output columns), times alpha, to Y.
namespace dec {
constexpr int QWARPS = 8;
constexpr int EWARPS = 4;
constexpr int XWARP = 2;                 // TMA producer of the bf16 activation tiles
constexpr int FIRST_Q = 3;
constexpr int FIRST_E = FIRST_Q + QWARPS;
constexpr int THREADS = 32 * (FIRST_E + EWARPS);
constexpr int W_STAGE = 128 * 128;       // weight codes of one k-block
constexpr int SFW_STAGE = 4 * 512;       // their scale atoms
// The activations are quantized once per CTA into a resident buffer (codes in
// the swizzled K-major operand layout, one 16-row x 128-byte tile per k-block,
// and the block scales packed per k-block), so the activation path never waits
// on the MMAs and CTAs with more than one weight tile reuse it.  The bf16 tiles
// it is made from land by TMA in a ring of XS stages; the rest of shared memory
// is the weight ring.
constexpr int MAX_M = 16;
constexpr int X_ROW = 512;               // bytes of one activation row of a k-block (256 bf16)
constexpr int X_STAGE = MAX_M * X_ROW;   // one k-block of activations
constexpr int MAX_XS = 8;
constexpr int MAX_STAGES = 12;
constexpr uint32_t TMEM_COLS = 256;
constexpr int NACC = 4;                  // independent accumulators (MMA kk of a k-block -> accumulator kk)
constexpr uint32_t ACC_COL = 0;          // NACC x np fp32 columns (np <= 32)
constexpr uint32_t SF_COL = 128;         // SF_NBUF scale buffers of SF_BUF columns:
constexpr uint32_t SF_BUF = 32;          //   weight atoms x 4 columns, then activation atoms x 4
constexpr int SF_NBUF = 4;
constexpr int MAX_SMEM = 232448;         // 227 KB opt-in limit per CTA
constexpr int FIXED_BARS = 56;           // weight ring 2 x 12, scale buffers 2 x 4, TMEM and done 3,
                                         // the TMEM holder's slot, activation ring 2 x 8 (<= 56)
}  // namespace dec

struct DecodeDev {
    int64_t M, N, K;
    const float* a_gscale;
    const uint8_t* w_scales;
    const float* b_gscale;
    void* y;
    int64_t catoms;
    int np;           // MMA N: M rounded up to 16
    int nkb;          // k-blocks of 256
    int stages;       // weight ring depth
    int xs;           // activation ring depth
    int out_bf16;
};

__device__ __forceinline__ uint32_t sw128_offset(int row, int byte_in_row) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((byte_in_row >> 4) ^ (row & 7)) & 7) << 4) +
                      (byte_in_row & 15));
}

struct DecodeLayout {
    int off_w, off_sfw, off_xq, off_x, off_xs, off_bar, off_tab, total;
};

// Weight ring (S stages of codes and scale atoms), the resident activation codes
// (nkb tiles of np x 128 bytes), the activation ring (XS bf16 tiles), the
// resident activation scales (nkb x 4 atoms x np rows x 4 bytes), the barriers
// (the fixed ones, then one per k-block of activations) and the 128-entry
// (S, 1/S) table.
__host__ __device__ inline DecodeLayout decode_layout(int np, int nkb, int stages, int xs) {
    DecodeLayout L;
    L.off_w = 0;
    L.off_sfw = L.off_w + stages * dec::W_STAGE;
    L.off_xq = L.off_sfw + stages * dec::SFW_STAGE;        // 1024-aligned: both stage sizes are
    L.off_x = L.off_xq + nkb * np * 128;                   // 1024-aligned: np * 128 = 2048
    L.off_xs = L.off_x + xs * dec::X_STAGE;
    L.off_bar = L.off_xs + nkb * 16 * np;
    L.off_tab = (L.off_bar + 8 * (dec::FIXED_BARS + nkb) + 15) / 16 * 16;
    L.total = L.off_tab + 128 * 8 + 1024;                   // + alignment slack
    return L;
}

__global__ void __launch_bounds__(dec::THREADS, 1)
    fused_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                        DecodeDev p) {
    using namespace dec;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int np = p.np, nkb = p.nkb, S = p.stages, XS = p.xs;
    const DecodeLayout L = decode_layout(np, nkb, S, XS);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.off_bar);   // [S] weight tile landed
    uint64_t* empty = full + MAX_STAGES;                               // [S] its MMAs are done
    uint64_t* sf_ready = empty + MAX_STAGES;                           // [SF_NBUF] scales staged in TMEM buffer
    uint64_t* sf_free = sf_ready + SF_NBUF;                            // [SF_NBUF] its MMAs are done
    uint64_t* tmem_full = sf_free + SF_NBUF;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* mma_done = tmem_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    uint64_t* xfull = mma_done + 2;                                    // [XS] activation tile landed
    uint64_t* xempty = xfull + MAX_XS;                                 // [XS] its values are quantized
    uint64_t* xres = reinterpret_cast<uint64_t*>(smem + L.off_bar) + FIXED_BARS;   // [nkb] activations ready
    float2* nv_tab = reinterpret_cast<float2*>(smem + L.off_tab);      // 128 (S, 1/S) entries
    const uint8_t* xs_res = smem + L.off_xs;                           // packed activation scales

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int kb = 0; kb < nkb; ++kb) mbar_init(&xres[kb], QWARPS);
        for (int s = 0; s < XS; ++s) { mbar_init(&xfull[s], 1); mbar_init(&xempty[s], QWARPS); }
        for (int b = 0; b < SF_NBUF; ++b) { mbar_init(&sf_ready[b], EWARPS); mbar_init(&sf_free[b], 1); }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, EWARPS);
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) { tmem_alloc(tmem_holder, TMEM_COLS); tmem_relinquish(); }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&tmW);
    if (warp == XWARP && lane == 0) tma_prefetch_desc(&tmX);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int64_t tiles = (p.N + 127) / 128;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t last_phase[MAX_STAGES];
            bool issued[MAX_STAGES];
            for (int s = 0; s < MAX_STAGES; ++s) issued[s] = false, last_phase[s] = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
                    const int64_t krem = p.K - (int64_t)kb * 256;
                    const int nmma = (krem < 256 ? (int)krem : 256) / 64;
                    mbar_arrive_expect_tx(&full[stage], W_STAGE + nmma * 512);
                    tma_load_2d(smem + L.off_w + stage * W_STAGE, &tmW, &full[stage], kb * 128, (int32_t)(t * 128));
                    bulk_load(smem + L.off_sfw + stage * SFW_STAGE, p.w_scales + (t * p.catoms + (int64_t)kb * 4) * 512,
                              (uint32_t)nmma * 512u, &full[stage]);
                    issued[stage] = true;
                    last_phase[stage] = phase;
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int s = 0; s < S; ++s)
                if (issued[s]) mbar_wait(&full[s], last_phase[s]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_mxf4(128, np, false);
            int stage = 0, b = 0;
            uint32_t phase = 0, bphase = 0, acc_phase = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                if (!mbar_wait(tmem_empty, acc_phase ^ 1)) { ok = false; break; }
                tc_fence_after();
                uint32_t started = 0;                    // bit j: accumulator j holds a partial sum
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full[stage], phase) || !mbar_wait(&xres[kb], 0) ||
                        !mbar_wait(&sf_ready[b], bphase)) { ok = false; break; }
                    tc_fence_after();
                    const int64_t krem = p.K - (int64_t)kb * 256;
                    const int nmma = (krem < 256 ? (int)krem : 256) / 64;
                    const uint32_t sfa = tmem + SF_COL + b * SF_BUF, sfb = sfa + 16;
                    const uint64_t adesc = smem_desc(smem_u32(smem + L.off_w + stage * W_STAGE), 16, 1024, 2);
                    const uint64_t bdesc = smem_desc(smem_u32(smem + L.off_xq + kb * np * 128), 16, 1024, 2);
                    // four independent accumulation chains: tiny-N MMAs into one
                    // accumulator would serialise on their latency
                    for (int kk = 0; kk < nmma; ++kk) {
                        mma_nvf4(tmem + ACC_COL + kk * np, adesc + 2 * kk, bdesc + 2 * kk, idesc, sfa + kk * 4,
                                 sfb + kk * 4, (started >> kk) & 1u);
                        started |= 1u << kk;
                    }
                    tc_commit(&empty[stage]);
                    tc_commit(&sf_free[b]);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                    if (++b == SF_NBUF) { b = 0; bphase ^= 1; }
                }
                if (!ok) break;
                tc_commit(tmem_full);
                acc_phase ^= 1;
            }
            // all MMAs of this thread are complete before TMEM is released
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (warp == XWARP) {
        // ---- activation tiles (M rows x 256 bf16 per k-block), once per CTA
        if (lane == 0) {
            const uint32_t xbytes = (uint32_t)p.M * (uint32_t)X_ROW;   // the box: M rows x 256 elements
            int s = 0;
            uint32_t ph = 0;
            uint32_t last_phase[MAX_XS];
            bool issued[MAX_XS];
            for (int i = 0; i < MAX_XS; ++i) issued[i] = false, last_phase[i] = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&xempty[s], ph ^ 1)) break;
                mbar_arrive_expect_tx(&xfull[s], xbytes);
                tma_load_2d(smem + L.off_x + s * X_STAGE, &tmX, &xfull[s], kb * 256, 0);
                issued[s] = true;
                last_phase[s] = ph;
                if (++s == XS) { s = 0; ph ^= 1; }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int i = 0; i < XS; ++i)
                if (issued[i]) mbar_wait(&xfull[i], last_phase[i]);
        }
    } else if (warp < FIRST_E) {
        // ---- quantize the activations (warps 3..10), once per CTA
        const int qt = threadIdx.x - 32 * FIRST_Q;
        constexpr int QT = 32 * QWARPS;
        const NvCtx sc = nv_ctx(*p.a_gscale, nv_tab);
        nv_fill_table(*p.a_gscale, nv_tab, qt, QT);
        named_barrier(1, QT);
        // Thread qt owns block (row m = qt / 16, block j = qt % 16) of every
        // k-block (np * 16 <= QT blocks per k-block): its 32 bytes of the landed
        // tile (rows at or beyond M and columns beyond K are zero) are quantized
        // into the resident codes and scales; the tile goes back to the producer
        // once every warp has used what it read (and the k-block is ready).
        const int m = qt >> 4, j = qt & 15;
        const bool active = qt < np * 16;
        uint8_t* xq_res = smem + L.off_xq;
        uint8_t* xs_w = smem + L.off_xs;
        int s = 0;
        uint32_t ph = 0;
        for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&xfull[s], ph)) break;
            if (active) {
                uint4 c0 = make_uint4(0u, 0u, 0u, 0u), c1 = c0;
                if (m < p.M) {
                    const uint8_t* src = smem + L.off_x + s * X_STAGE + m * X_ROW + j * 32;
                    c0 = *reinterpret_cast<const uint4*>(src);
                    c1 = *reinterpret_cast<const uint4*>(src + 16);
                }
                const float v[16] = {bf16_lo(c0.x), bf16_hi(c0.x), bf16_lo(c0.y), bf16_hi(c0.y),
                                     bf16_lo(c0.z), bf16_hi(c0.z), bf16_lo(c0.w), bf16_hi(c0.w),
                                     bf16_lo(c1.x), bf16_hi(c1.x), bf16_lo(c1.y), bf16_hi(c1.y),
                                     bf16_lo(c1.z), bf16_hi(c1.z), bf16_lo(c1.w), bf16_hi(c1.w)};
                uint32_t byte, w[2];
                nv_block<false>(v, sc, byte, w);
                *reinterpret_cast<uint2*>(xq_res + kb * np * 128 + sw128_offset(m, j * 8)) = make_uint2(w[0], w[1]);
                xs_w[((kb * 4 + (j >> 2)) * np + m) * 4 + (j & 3)] = (uint8_t)byte;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&xempty[s]);
                mbar_arrive(&xres[kb]);
            }
            if (++s == XS) { s = 0; ph ^= 1; }
        }
    } else {
        // ---- epilogue (warps 11..14): thread = one weight row = one output column
        const int quad = warp & 3;
        const float alpha = __fmul_rn(*p.a_gscale, *p.b_gscale);
        const int nacc = p.K / 64 < NACC ? (int)(p.K / 64) : NACC;   // accumulators that received an MMA
        const uint32_t qaddr = tmem + ((uint32_t)(quad * 32) << 16);
        uint32_t acc_phase = 0;
        int stage = 0, b = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            // Stage every k-block's weight and activation scale atoms into a TMEM
            // scale buffer with tcgen05.st (each warp fills its lane quarter
            // with the whole atom), keeping these copies off the MMA thread.
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&full[stage], phase) || !mbar_wait(&xres[kb], 0) ||
                    !mbar_wait(&sf_free[b], bphase ^ 1)) { ok = false; break; }
                tc_fence_after();
                const int64_t krem = p.K - (int64_t)kb * 256;
                const int nmma = (krem < 256 ? (int)krem : 256) / 64;
                const uint8_t* wf = smem + L.off_sfw + stage * SFW_STAGE;
                const uint32_t dst = qaddr + SF_COL + b * SF_BUF;
                for (int a = 0; a < nmma; ++a) {
                    // the activation atom in the tensor-core layout: lane l holds rows
                    // l, l + 32, l + 64, l + 96, of which only row l < np exists
                    const uint4 va = *reinterpret_cast<const uint4*>(wf + a * 512 + lane * 16);
                    const uint32_t xb =
                        lane < np ? *reinterpret_cast<const uint32_t*>(xs_res + ((kb * 4 + a) * np + lane) * 4) : 0u;
                    tmem_st4(dst + a * 4, va.x, va.y, va.z, va.w);
                    tmem_st4(dst + 16 + a * 4, xb, 0u, 0u, 0u);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[b]);
                if (++stage == S) { stage = 0; phase ^= 1; }
                if (++b == SF_NBUF) { b = 0; bphase ^= 1; }
            }
            if (!ok) break;
            if (!mbar_wait(tmem_full, acc_phase)) break;
            tc_fence_after();
            const int64_t n = t * 128 + quad * 32 + lane;
            for (int c0 = 0; c0 < np; c0 += 16) {
                float acc[16];
                for (int a = 0; a < nacc; ++a) {
                    uint32_t r[16];
                    tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + a * np + c0, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[j] = a == 0 ? __uint_as_float(r[j]) : __fadd_rn(acc[j], __uint_as_float(r[j]));
                }
                if (n < p.N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t m = c0 + j;
                        if (m < p.M) {
                            const float val = acc[j] * alpha;
                            if (p.out_bf16)
                                reinterpret_cast<__nv_bfloat16*>(p.y)[m * p.N + n] = __float2bfloat16_rn(val);
                            else
                                reinterpret_cast<float*>(p.y)[m * p.N + n] = val;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tmem_empty);
            acc_phase ^= 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// Ring depths that fit beside the resident activations: the deepest activation
// ring of 8, 4 or 2 tiles that leaves at least 4 (8) or 3 (4, 2) weight stages,
// with as many weight stages as then fit.  False: the shape is not taken by the
// fused kernel (K below one k-block of 256, M above 16, or K so long that the
// resident activations leave no room).
static bool decode_config(int64_t M, int64_t K, int* stages, int* xs) {
    if (M <= 0 || M > dec::MAX_M || K < 256 || K > (1 << 20)) return false;
    const int np = (int)((M + 15) / 16 * 16);
    const int nkb = (int)((K + 255) / 256);
    const int cand[3][2] = {{8, 4}, {4, 3}, {2, 3}};
    for (const auto& c : cand) {
        int st = dec::MAX_STAGES;
        while (st >= c[1] && decode_layout(np, nkb, st, c[0]).total > dec::MAX_SMEM) --st;
        if (st >= c[1]) {
            *stages = st;
            *xs = c[0];
            return true;
        }
    }
    return false;
}

bool fused_decode_supported(int64_t M, int64_t K) {
    int st, xs;
    return decode_config(M, K, &st, &xs);
}

// bf16 activations [M, K] for TMA tiles of M rows x 256 elements (no swizzle).
static bool make_act_map(CUtensorMap* map, const void* x, int64_t M, int64_t K) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(K * 2)};
    cuuint32_t box[2] = {256u, (cuuint32_t)M};
    cuuint32_t es[2] = {1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_fused_decode(const FusedDecodeParams& p, cudaStream_t st, int num_sms) {
    using namespace dec;
    if (p.M == 0 || p.N == 0) return cudaSuccess;
    const int np = (int)((p.M + 15) / 16 * 16);
    const int nkb = (int)((p.K + 255) / 256);
    int stages = 0, xs = 0;
    if (!decode_config(p.M, p.K, &stages, &xs)) return cudaErrorNotSupported;
    CUtensorMap mw, mx;
    if (!make_code_map(&mw, p.b_codes, p.N, p.K / 2, 128)) return cudaErrorInvalidValue;
    if (!make_act_map(&mx, p.a_bf16, p.M, p.K)) return cudaErrorInvalidValue;
    DecodeDev d;
    d.M = p.M; d.N = p.N; d.K = p.K; d.a_gscale = p.a_gscale;
    d.w_scales = p.b_scales; d.b_gscale = p.b_gscale; d.y = p.y;
    d.catoms = ((p.K / 16) + 3) / 4;
    d.np = np; d.nkb = nkb; d.stages = stages; d.xs = xs; d.out_bf16 = p.out_bf16 ? 1 : 0;
    const int smem = decode_layout(np, nkb, stages, xs).total;
    cudaError_t e = cudaFuncSetAttribute(fused_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (p.N + 127) / 128;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    fused_decode_kernel<<<grid, THREADS, smem, st>>>(mw, mx, d);
    return cudaGetLastError();
}

cudaError_t set_wait_limit(long long cycles) {
    cudaError_t e = set_module_wait_limit(cycles);
    if (e == cudaSuccess) e = set_quant_wait_limit(cycles);
    return e;
}

cudaError_t read_clear_device_error(unsigned int* word) {
    unsigned int a = 0, b = 0;
    cudaError_t e = read_clear_module_error(&a);
    if (e == cudaSuccess) e = read_clear_quant_error(&b);
    *word = a | b;
    return e;
}

}  // namespace q4
