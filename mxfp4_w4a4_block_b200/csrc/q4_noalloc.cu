// q4_noalloc.cu -- q4_gemm_a_bf16_noalloc: the bf16-activation W4A4 GEMM for
// callers that cannot allocate device memory at the point of the call (for
// example code embedded in a host application that owns every device buffer
// through its own fixed pool, or that must keep its device footprint constant
// after start-up, and therefore cannot hand q4_gemm the scratch workspace it
// asks for).  The activation codes and scales live in a fixed array inside this
// library instead of a caller workspace.
//
// The array below is allocated when the library's device code is loaded on a
// GPU and stays resident on every GPU that loaded it until the process exits.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/q4.h"
#include "q4_internal.h"

namespace {

// Library-owned scratch: activation codes [M, K/2] (rounded up to 256 bytes),
// then their tensor-core scale atoms.
static __device__ __align__(256) uint8_t g_noalloc_scratch[Q4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
uint8_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached for the life of the
// process: a cudaDeviceReset after the first call on a device is not supported
// (the module may be loaded again elsewhere and the cached address goes stale).
cudaError_t scratch_on_current_device(uint8_t** out, int* dev_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_scratch_ptr[dev];
    *dev_out = dev;
    return cudaSuccess;
}

q4_status status_of(cudaError_t e) { return (q4_status)q4::status_of_cuda(e); }

}  // namespace

extern "C" Q4_API q4_status q4_gemm_a_bf16_noalloc(int64_t M, int64_t N, int64_t K, const void* a_bf16,
                                                   const float* d_a_gscale, const uint8_t* b_codes,
                                                   const uint8_t* b_scales, const float* d_b_gscale,
                                                   q4_dtype out_dt, void* y, void* stream) {
    if (M < 0 || N < 0 || K < 0 || (out_dt != Q4_F32 && out_dt != Q4_BF16)) return Q4_ERR_ARG;
    if (!d_a_gscale || !d_b_gscale) return Q4_ERR_ARG;
    if (K % 64 || N % 8) return Q4_ERR_SHAPE;
    if (K > ((int64_t)1 << 30) || M > ((int64_t)1 << 31) || N > ((int64_t)1 << 31)) return Q4_ERR_SHAPE;
    if (M == 0 || N == 0) return Q4_OK;
    if (!y) return Q4_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(y) & 15u) return Q4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    // K = 0: an empty sum, as q4_gemm gives it
    if (K == 0) return status_of(cudaMemsetAsync(y, 0, (size_t)M * (size_t)N * (out_dt == Q4_BF16 ? 2 : 4), st));
    if (!a_bf16 || !b_codes || !b_scales) return Q4_ERR_ARG;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(a_bf16) | reinterpret_cast<uintptr_t>(b_codes) |
                          reinterpret_cast<uintptr_t>(b_scales);
    if (mis & 15u) return Q4_ERR_ALIGN;
    // the activation codes and scales must fit in the fixed array
    const size_t codes = (size_t)M * (size_t)(K / 2);
    const size_t codes_al = (codes + 255) / 256 * 256;
    const size_t scales = q4_scale_bytes(Q4_NVFP4, M, K, Q4_LAYOUT_TC);
    if (codes_al + scales > (size_t)Q4_NOALLOC_SCRATCH_BYTES) return Q4_ERR_WORKSPACE;

    uint8_t* scratch = nullptr;
    int dev = 0, sms = 148;
    cudaError_t e = scratch_on_current_device(&scratch, &dev);
    if (e != cudaSuccess) return status_of(e);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;

    // Every code byte the GEMM reads and every scale atom (padding included)
    // is written by the quantize launch, so nothing left from an earlier call
    // needs clearing.
    q4::QuantParams qp;
    qp.x = a_bf16; qp.rows = M; qp.cols = K; qp.ld = K; qp.gscale = d_a_gscale; qp.chan = nullptr;
    qp.codes = scratch; qp.scales = scratch + codes_al; qp.scols = K / 16; qp.catoms = ((K / 16) + 3) / 4;
    e = q4::launch_quantize(qp, 16, true, true, false, false, false, false, st, sms);
    if (e != cudaSuccess) return status_of(e);

    q4::GemmParams p;
    p.M = M; p.N = N; p.K = K;
    p.a_codes = scratch; p.a_scales = scratch + codes_al; p.a_gscale = d_a_gscale;
    p.b_codes = b_codes; p.b_scales = b_scales; p.b_gscale = d_b_gscale;
    p.y = y; p.out_bf16 = out_dt == Q4_BF16; p.mxfp4 = false;
    return status_of(q4::launch_gemm(p, st, sms));
}
