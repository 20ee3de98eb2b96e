// quotient_check.cu -- test kernels for the library's binary32 quotient
// helpers (q4_codec.cuh): the Markstein correction step quot_fast, the guarded
// quot_rn and the block-level code form, each compared with CUDA's correctly
// rounded division __fdiv_rn.  Built by tests/test_gpu_quotient.py.
#include <cstdint>
#include <cuda_runtime.h>

#include "q4_codec.cuh"

using namespace q4;

// Significand pairs: w = 1.a and S = 1.b (a, b 23-bit fields).  Thread t takes
// b = b_lo + t and walks a = a_off, a_off + a_step, ... below 2^23, counting
// pairs where quot_fast(w, S, RN(1/S)) and __fdiv_rn(w, S) differ in any bit;
// the first mismatch seen is kept in first[0..1] (first[2] = 1 once set).
__global__ void pairs_kernel(uint32_t b_lo, uint32_t b_count, uint32_t a_off, uint32_t a_step,
                             unsigned long long* count, uint32_t* first) {
    const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= b_count) return;
    const uint32_t b = b_lo + t;
    const float S = __uint_as_float(0x3F800000u | b);
    const float y = __frcp_rn(S);
    unsigned long long bad = 0;
    for (uint32_t a = a_off; a < (1u << 23); a += a_step) {
        const float w = __uint_as_float(0x3F800000u | a);
        const float q = quot_fast(w, S, y);
        const float d = __fdiv_rn(w, S);
        if (__float_as_uint(q) != __float_as_uint(d)) {
            ++bad;
            if (atomicCAS(first + 2, 0u, 1u) == 0u) {
                first[0] = a;
                first[1] = b;
            }
        }
    }
    if (bad) atomicAdd(count, bad);
}

// Elementwise: out_rn[i] = quot_rn(w[i], S[i], y), out_div[i] = __fdiv_rn(w[i], S[i]),
// with y the library's reciprocal of S (0 outside the fast range).
__global__ void elems_kernel(const float* w, const float* S, int64_t n, float* out_rn, float* out_div) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float s = S[i];
    const float y = quot_recip(s);            // the library's rule: 0 outside the fast range
    out_rn[i] = quot_rn(w[i], s, y);
    out_div[i] = __fdiv_rn(w[i], s);
}

// Blocks of 16: codes of nv_codes16 (the quantizer's block form) against the
// E2M1 codes of __fdiv_rn, for blocks with the given S.
__global__ void codes_kernel(const float* x, const float* S, int64_t nblocks, uint32_t* got, uint32_t* want) {
    const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (blk >= nblocks) return;
    float v[16];
    for (int j = 0; j < 16; ++j) v[j] = x[blk * 16 + j];
    const float s = S[blk];
    const float y = quot_recip(s);
    const float amax = amax_tree<16>(v);
    uint32_t w[2];
    nv_codes16(v, make_float2(s, y), amax, w);
    got[2 * blk] = w[0];
    got[2 * blk + 1] = w[1];
    for (int g = 0; g < 2; ++g) {
        float q[8];
        for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(v[8 * g + i], s);
        want[2 * blk + g] = e2m1_pack8(q);
    }
}

#define QC_EXPORT __attribute__((visibility("default")))
extern "C" {

QC_EXPORT int qc_pairs(uint32_t b_lo, uint32_t b_count, uint32_t a_off, uint32_t a_step, unsigned long long* count,
             uint32_t* first) {
    if (b_lo + (uint64_t)b_count > (1u << 23) || a_step == 0) return 1;
    pairs_kernel<<<(b_count + 255) / 256, 256>>>(b_lo, b_count, a_off, a_step, count, first);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

QC_EXPORT int qc_elems(const float* w, const float* S, int64_t n, float* out_rn, float* out_div) {
    if (n <= 0) return 0;
    elems_kernel<<<(unsigned)((n + 255) / 256), 256>>>(w, S, n, out_rn, out_div);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

QC_EXPORT int qc_codes(const float* x, const float* S, int64_t nblocks, uint32_t* got, uint32_t* want) {
    if (nblocks <= 0) return 0;
    codes_kernel<<<(unsigned)((nblocks + 127) / 128), 128>>>(x, S, nblocks, got, want);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
}
