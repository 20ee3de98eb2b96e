// e2m1_sweep.cu -- test kernel: the library's E2M1 conversions (e2m1_pack8 and
// e2m1_pack4 of q4_codec.cuh, the cvt.rn.satfinite.e2m1x2 path every quantizer
// ends in) on every binary32 bit pattern (sign << 31) | u, u in [0, hi],
// against a run-length table of expected codes (run k: u >= starts[k], code
// codes[k]) made on the host from the oracle.  Built by
// tests/test_gpu_e2m1_sweep.py.
#include <cstdint>
#include <cuda_runtime.h>

#include "q4_codec.cuh"

using namespace q4;

// Thread t converts u = 8t .. 8t + 7 (those <= hi) with both helpers and
// counts nibbles that differ from the table; the first mismatch seen is kept
// in first[0] (u), first[1] (got), first[2] (want), first[3] = 1 once set.
__global__ void sweep_kernel(uint32_t sign, uint32_t hi, const uint32_t* starts, const uint8_t* codes, int nruns,
                             unsigned long long* bad, uint32_t* first) {
    const uint64_t u0 = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8u;
    if (u0 > hi) return;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t u = u0 + i;
        v[i] = u <= hi ? __uint_as_float((sign << 31) | (uint32_t)u) : 0.0f;
    }
    const uint32_t w8 = e2m1_pack8(v);
    const uint32_t w4 = e2m1_pack4(v[0], v[1], v[2], v[3]) | (e2m1_pack4(v[4], v[5], v[6], v[7]) << 16);
    int k = 0;
    while (k + 1 < nruns && starts[k + 1] <= u0) ++k;
    unsigned long long nbad = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t u = u0 + i;
        if (u > hi) break;
        while (k + 1 < nruns && starts[k + 1] <= u) ++k;
        const uint32_t want = codes[k];
        const uint32_t g8 = (w8 >> (4 * i)) & 15u, g4 = (w4 >> (4 * i)) & 15u;
        if (g8 != want || g4 != want) {
            ++nbad;
            if (atomicCAS(first + 3, 0u, 1u) == 0u) {
                first[0] = (uint32_t)u;
                first[1] = g8 != want ? g8 : g4;
                first[2] = want;
            }
        }
    }
    if (nbad) atomicAdd(bad, nbad);
}

extern "C" __attribute__((visibility("default"))) int e2m1_sweep(uint32_t sign, uint32_t hi, const uint32_t* starts,
                                                                 const uint8_t* codes, int nruns,
                                                                 unsigned long long* bad, uint32_t* first) {
    if (sign > 1 || nruns < 1 || hi >= 0x7F800000u) return 1;
    const uint64_t threads = ((uint64_t)hi + 8u) / 8u;
    const unsigned blocks = (unsigned)((threads + 255u) / 256u);
    sweep_kernel<<<blocks, 256>>>(sign, hi, starts, codes, nruns, bad, first);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
