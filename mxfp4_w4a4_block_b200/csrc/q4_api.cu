// q4_api.cu -- the extern "C" entry points declared in include/q4.h: argument
// validation on the host, then one or more kernel launches on the caller's
// stream.  No entry point allocates device memory.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/q4.h"
#include "q4_internal.h"


namespace {

thread_local char g_last_error[256] = "no error";

q4_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return Q4_OK;
    std::strncpy(g_last_error, cudaGetErrorString(e), sizeof(g_last_error) - 1);
    g_last_error[sizeof(g_last_error) - 1] = '\0';
    return Q4_ERR_CUDA;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int block_of(q4_format f) { return f == Q4_NVFP4 ? 16 : 32; }

bool valid_format(int f) { return f == Q4_NVFP4 || f == Q4_MXFP4; }
bool valid_dtype(int d) { return d == Q4_F32 || d == Q4_BF16; }

int64_t catoms_of(int64_t cols, int blk) { return ((cols / blk) + 3) / 4; }

// Per-entry checks of a grouped call (the single-matrix call's checks) and
// the launch table; entries with no elements are dropped.  need_res: the
// residue must be present; res_io: a present residue must be aligned.
q4_status group_from(q4_format format, int block, const q4_matrix* mats, int count, int flags, int allowed,
                     bool need_res, bool res_io, bool scales_aligned, q4::GroupParams& g) {
    if (!valid_format(format)) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (flags & ~allowed) return Q4_ERR_ARG;
    if (count < 0 || count > Q4_MAX_GROUP || (count > 0 && !mats)) return Q4_ERR_ARG;
    g.count = 0;
    g.total = 0;
    for (int i = 0; i < count; ++i) {
        const q4_matrix& m = mats[i];
        if (m.rows < 0 || m.cols < 0) return Q4_ERR_ARG;
        if (format == Q4_NVFP4 && !m.d_gscale) return Q4_ERR_ARG;
        if (format == Q4_MXFP4 && m.d_gscale) return Q4_ERR_ARG;
        if (m.cols % block) return Q4_ERR_SHAPE;
        if (m.rows == 0 || m.cols == 0) continue;
        if (!m.w || !m.scales || !m.codes || (need_res && !m.residue)) return Q4_ERR_ARG;
        if (!aligned16(m.w) || !aligned16(m.codes) || (res_io && m.residue && !aligned16(m.residue)) ||
            (scales_aligned && !aligned16(m.scales)))
            return Q4_ERR_ALIGN;
        q4::GroupItem& it = g.m[g.count++];
        it.w = m.w; it.rows = m.rows; it.cols = m.cols; it.scales = m.scales; it.gscale = m.d_gscale;
        it.residue = res_io ? m.residue : nullptr; it.codes = m.codes;
        it.scols = m.cols / block; it.catoms = catoms_of(m.cols, block); it.start = 0;
    }
    return Q4_OK;
}

}  // namespace

namespace q4 {
int status_of_cuda(cudaError_t e) { return (int)cuda_status(e); }
}  // namespace q4

extern "C" {

int q4_version(void) { return 100; }

const char* q4_status_string(q4_status s) {
    switch (s) {
        case Q4_OK: return "ok";
        case Q4_ERR_ARG: return "invalid argument";
        case Q4_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
        case Q4_ERR_SHAPE: return "unsupported shape";
        case Q4_ERR_UNSUPPORTED: return "unsupported request";
        case Q4_ERR_CUDA: return "CUDA error";
        case Q4_ERR_TIMEOUT: return "device wait timed out";
        case Q4_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char* q4_last_error(void) { return g_last_error; }

size_t q4_scale_bytes(q4_format format, int64_t rows, int64_t cols, int flags) {
    if (!valid_format(format) || rows < 0 || cols < 0) return 0;
    const int blk = block_of(format);
    if (cols % blk) return 0;
    const int64_t scols = cols / blk;
    if (flags & Q4_LAYOUT_TC) return (size_t)(((rows + 127) / 128) * 128 * ((scols + 3) / 4) * 4);
    return (size_t)(rows * scols);
}

q4_status q4_amax(q4_dtype dt, const void* x, int64_t n, float denom, float* d_out, void* stream) {
    if (!valid_dtype(dt) || n < 0 || !d_out || (n > 0 && !x)) return Q4_ERR_ARG;
    if (!(denom > 0.0f) || !(denom < 3.0e38f)) return Q4_ERR_ARG;
    if ((x && !aligned16(x)) || (reinterpret_cast<uintptr_t>(d_out) & 3u)) return Q4_ERR_ALIGN;
    return cuda_status(q4::launch_amax(x, n, dt == Q4_BF16, denom, d_out, (cudaStream_t)stream, num_sms()));
}

q4_status q4_amax_quantize(q4_dtype in_dt, const void* x, int64_t rows, int64_t cols, int64_t ld, float denom,
                           float* d_out, uint8_t* codes, uint8_t* scales, int flags, void* stream) {
    if (!valid_dtype(in_dt) || rows < 0 || cols < 0 || ld < cols || !d_out) return Q4_ERR_ARG;
    if (!(denom > 0.0f) || !(denom < 3.0e38f)) return Q4_ERR_ARG;
    if (flags & ~(Q4_SCALE_RU | Q4_LAYOUT_TC)) return Q4_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(d_out) & 3u) return Q4_ERR_ALIGN;
    if (cols % 16) return Q4_ERR_SHAPE;
    const int esz = in_dt == Q4_BF16 ? 2 : 4;
    if (rows > 0 && cols > 0) {
        if (!x || !codes || !scales) return Q4_ERR_ARG;
        if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (ld * esz) % 16) return Q4_ERR_ALIGN;
    }
    q4::QuantParams p;
    p.x = x; p.rows = rows; p.cols = cols; p.ld = ld;
    p.gscale = nullptr; p.chan = nullptr; p.codes = codes; p.scales = scales;
    p.scols = cols / 16; p.catoms = catoms_of(cols, 16);
    p.amax_out = reinterpret_cast<unsigned int*>(d_out);
    p.denom = denom;
    return cuda_status(q4::launch_amax_quantize(p, in_dt == Q4_BF16, (flags & Q4_LAYOUT_TC) != 0,
                                                (flags & Q4_SCALE_RU) != 0, (cudaStream_t)stream, num_sms()));
}

q4_status q4_quantize(q4_format format, int block, q4_dtype in_dt, const void* x, int64_t rows, int64_t cols,
                      int64_t ld, const float* d_gscale, const float* d_chan, uint8_t* codes, uint8_t* scales,
                      int flags, void* stream) {
    if (!valid_format(format) || !valid_dtype(in_dt) || rows < 0 || cols < 0 || ld < cols) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (flags & ~(Q4_SCALE_RU | Q4_LAYOUT_TC | Q4_HADAMARD32 | Q4_SCALE_46 | Q4_INJECT_STALL)) return Q4_ERR_ARG;
    if (format == Q4_NVFP4 && ((flags & Q4_HADAMARD32) || d_chan)) return Q4_ERR_UNSUPPORTED;
    if (format == Q4_MXFP4 && (flags & Q4_SCALE_46)) return Q4_ERR_UNSUPPORTED;
    if (format == Q4_NVFP4 && !d_gscale) return Q4_ERR_ARG;
    if (format == Q4_MXFP4 && d_gscale) return Q4_ERR_ARG;
    if (cols % block) return Q4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return Q4_OK;
    if (!x || !codes || !scales) return Q4_ERR_ARG;
    const int esz = in_dt == Q4_BF16 ? 2 : 4;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (ld * esz) % 16) return Q4_ERR_ALIGN;
    if (d_chan && !aligned16(d_chan)) return Q4_ERR_ALIGN;
    q4::QuantParams p;
    p.x = x; p.rows = rows; p.cols = cols; p.ld = ld;
    p.gscale = d_gscale; p.chan = d_chan; p.codes = codes; p.scales = scales;
    p.scols = cols / block; p.catoms = catoms_of(cols, block);
    p.inject_stall = (flags & Q4_INJECT_STALL) ? 1 : 0;
    return cuda_status(q4::launch_quantize(p, block, in_dt == Q4_BF16, (flags & Q4_LAYOUT_TC) != 0,
                                           (flags & Q4_SCALE_RU) != 0, (flags & Q4_HADAMARD32) != 0,
                                           d_chan != nullptr, (flags & Q4_SCALE_46) != 0, (cudaStream_t)stream,
                                           num_sms()));
}

q4_status q4_dequantize(q4_format format, int block, const uint8_t* codes, const uint8_t* scales,
                        const float* d_gscale, int64_t rows, int64_t cols, int flags, q4_dtype out_dt, void* out,
                        void* stream) {
    if (!valid_format(format) || !valid_dtype(out_dt) || rows < 0 || cols < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (format == Q4_NVFP4 && !d_gscale) return Q4_ERR_ARG;
    if (cols % block) return Q4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return Q4_OK;
    if (!codes || !scales || !out) return Q4_ERR_ARG;
    if (!aligned16(codes) || !aligned16(out)) return Q4_ERR_ALIGN;
    q4::DequantParams p;
    p.codes = codes; p.scales = scales; p.gscale = d_gscale; p.rows = rows; p.cols = cols; p.out = out;
    p.scols = cols / block; p.catoms = catoms_of(cols, block);
    return cuda_status(q4::launch_dequantize(p, block, (flags & Q4_LAYOUT_TC) != 0, out_dt == Q4_BF16,
                                             (cudaStream_t)stream, num_sms()));
}

q4_status q4_sigma_delta_codebanks(q4_format format, int block, const float* w, int64_t rows, int64_t cols,
                                   const uint8_t* scales, const float* d_gscale, int visits, uint8_t* codes,
                                   float* residue_out, int flags, void* stream) {
    if (!valid_format(format) || rows < 0 || cols < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (flags & ~(Q4_LAYOUT_TC)) return Q4_ERR_ARG;
    if (visits < 1 || visits > 4096) return Q4_ERR_ARG;
    if (format == Q4_NVFP4 && !d_gscale) return Q4_ERR_ARG;
    if (format == Q4_MXFP4 && d_gscale) return Q4_ERR_ARG;
    if (cols % block) return Q4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return Q4_OK;
    if (!w || !scales || !codes) return Q4_ERR_ARG;
    if (!aligned16(w) || !aligned16(codes) || (residue_out && !aligned16(residue_out))) return Q4_ERR_ALIGN;
    q4::SigmaDeltaParams p;
    p.w = w; p.rows = rows; p.cols = cols; p.scales = scales; p.gscale = d_gscale;
    p.residue = nullptr; p.codes = codes; p.scols = cols / block; p.catoms = catoms_of(cols, block);
    return cuda_status(q4::launch_sigma_delta_banks(p, block, (flags & Q4_LAYOUT_TC) != 0, visits, residue_out,
                                                    (cudaStream_t)stream, num_sms()));
}

q4_status q4_sr_requant(q4_format format, int block, const float* w, int64_t rows, int64_t cols,
                        const uint8_t* scales, const float* d_gscale, uint64_t seed, uint32_t visit, uint8_t* codes,
                        int flags, void* stream) {
    if (!valid_format(format) || rows < 0 || cols < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (flags & ~(Q4_LAYOUT_TC)) return Q4_ERR_ARG;
    if (format == Q4_NVFP4 && !d_gscale) return Q4_ERR_ARG;
    if (format == Q4_MXFP4 && d_gscale) return Q4_ERR_ARG;
    if (cols % block) return Q4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return Q4_OK;
    if (!w || !scales || !codes) return Q4_ERR_ARG;
    if (!aligned16(w) || !aligned16(codes)) return Q4_ERR_ALIGN;
    q4::SigmaDeltaParams p;
    p.w = w; p.rows = rows; p.cols = cols; p.scales = scales; p.gscale = d_gscale;
    p.residue = nullptr; p.codes = codes; p.scols = cols / block; p.catoms = catoms_of(cols, block);
    return cuda_status(q4::launch_sr_requant(p, block, (flags & Q4_LAYOUT_TC) != 0, seed, visit,
                                             (cudaStream_t)stream, num_sms()));
}

q4_status q4_sigma_delta_step(q4_format format, int block, const float* w, int64_t rows, int64_t cols,
                              const uint8_t* scales, const float* d_gscale, float* residue, uint8_t* codes,
                              int flags, void* stream) {
    if (!valid_format(format) || rows < 0 || cols < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (flags & ~(Q4_LAYOUT_TC)) return Q4_ERR_ARG;
    if (format == Q4_NVFP4 && !d_gscale) return Q4_ERR_ARG;
    if (format == Q4_MXFP4 && d_gscale) return Q4_ERR_ARG;
    if (cols % block) return Q4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return Q4_OK;
    if (!w || !scales || !residue || !codes) return Q4_ERR_ARG;
    if (!aligned16(w) || !aligned16(residue) || !aligned16(codes)) return Q4_ERR_ALIGN;
    q4::SigmaDeltaParams p;
    p.w = w; p.rows = rows; p.cols = cols; p.scales = scales; p.gscale = d_gscale;
    p.residue = residue; p.codes = codes; p.scols = cols / block; p.catoms = catoms_of(cols, block);
    return cuda_status(q4::launch_sigma_delta(p, block, (flags & Q4_LAYOUT_TC) != 0, (cudaStream_t)stream,
                                              num_sms()));
}

q4_status q4_sigma_delta_gemm(q4_format format, int block, int64_t M, int64_t N, int64_t K, const void* x,
                              const float* w, const uint8_t* scales, const float* d_gscale, float* residue,
                              q4_dtype out_dt, void* y, int flags, void* stream) {
    if (!valid_format(format) || !valid_dtype(out_dt) || M < 0 || N < 0 || K < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (format != Q4_NVFP4 || !(flags & Q4_LAYOUT_TC) || (flags & ~Q4_LAYOUT_TC)) return Q4_ERR_UNSUPPORTED;
    if (!d_gscale) return Q4_ERR_ARG;
    if (K % 64 || N % 8) return Q4_ERR_SHAPE;
    if (M == 0 || N == 0 || K == 0) return M == 0 || N == 0 ? Q4_OK : Q4_ERR_SHAPE;
    if (!q4::sd_gemm_supported(M, K)) return Q4_ERR_UNSUPPORTED;
    if (!x || !w || !scales || !residue || !y) return Q4_ERR_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(scales) || !aligned16(residue) || !aligned16(y))
        return Q4_ERR_ALIGN;
    q4::SdGemmParams p;
    p.M = M; p.N = N; p.K = K; p.x = x; p.w = w; p.scales = scales; p.gscale = d_gscale; p.residue = residue;
    p.y = y; p.out_bf16 = out_dt == Q4_BF16;
    return cuda_status(q4::launch_sd_gemm(p, (cudaStream_t)stream, num_sms()));
}

q4_status q4_quantize_grouped(q4_format format, int block, q4_dtype in_dt, const q4_matrix* mats, int count,
                              int flags, void* stream) {
    if (!valid_dtype(in_dt)) return Q4_ERR_ARG;
    if (format == Q4_NVFP4 && (flags & Q4_HADAMARD32)) return Q4_ERR_UNSUPPORTED;
    if (format == Q4_MXFP4 && (flags & Q4_SCALE_46)) return Q4_ERR_UNSUPPORTED;
    q4::GroupParams g;
    const q4_status s = group_from(format, block, mats, count, flags,
                                   Q4_SCALE_RU | Q4_LAYOUT_TC | Q4_HADAMARD32 | Q4_SCALE_46, false, false, true, g);
    if (s != Q4_OK || g.count == 0) return s;
    return cuda_status(q4::launch_quantize_grouped(g, block, in_dt == Q4_BF16, (flags & Q4_LAYOUT_TC) != 0,
                                                   (flags & Q4_SCALE_RU) != 0, (flags & Q4_HADAMARD32) != 0,
                                                   (flags & Q4_SCALE_46) != 0, (cudaStream_t)stream, num_sms()));
}

q4_status q4_sigma_delta_step_grouped(q4_format format, int block, const q4_matrix* mats, int count, int flags,
                                      void* stream) {
    q4::GroupParams g;
    const q4_status s = group_from(format, block, mats, count, flags, Q4_LAYOUT_TC, true, true, false, g);
    if (s != Q4_OK || g.count == 0) return s;
    return cuda_status(q4::launch_sigma_delta_grouped(g, block, (flags & Q4_LAYOUT_TC) != 0, (cudaStream_t)stream,
                                                      num_sms()));
}

q4_status q4_sr_requant_grouped(q4_format format, int block, const q4_matrix* mats, int count, uint64_t seed,
                                uint32_t visit, int flags, void* stream) {
    q4::GroupParams g;
    const q4_status s = group_from(format, block, mats, count, flags, Q4_LAYOUT_TC, false, false, false, g);
    if (s != Q4_OK || g.count == 0) return s;
    return cuda_status(q4::launch_sr_requant_grouped(g, block, (flags & Q4_LAYOUT_TC) != 0, seed, visit,
                                                     (cudaStream_t)stream, num_sms()));
}

q4_status q4_sigma_delta_codebanks_grouped(q4_format format, int block, const q4_matrix* mats, int count,
                                           int visits, int flags, void* stream) {
    if (visits < 1 || visits > 4096) return Q4_ERR_ARG;
    q4::GroupParams g;
    const q4_status s = group_from(format, block, mats, count, flags, Q4_LAYOUT_TC, false, true, false, g);
    if (s != Q4_OK || g.count == 0) return s;
    return cuda_status(q4::launch_sigma_delta_banks_grouped(g, block, (flags & Q4_LAYOUT_TC) != 0, visits,
                                                            (cudaStream_t)stream, num_sms()));
}

q4_status q4_sigma_delta_gemm_grouped(q4_format format, int block, int64_t M, int64_t K,
                                      const q4_sd_gemm_entry* entries, int count, q4_dtype out_dt, int flags,
                                      void* stream) {
    if (!valid_format(format) || !valid_dtype(out_dt) || M < 0 || K < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (format != Q4_NVFP4 || !(flags & Q4_LAYOUT_TC) || (flags & ~Q4_LAYOUT_TC)) return Q4_ERR_UNSUPPORTED;
    if (count < 0 || count > Q4_MAX_GROUP || (count > 0 && !entries)) return Q4_ERR_ARG;
    if (K % 64) return Q4_ERR_SHAPE;
    if (count == 0 || M == 0) return Q4_OK;
    if (K == 0) return Q4_ERR_SHAPE;
    if (!q4::sd_gemm_supported(M, K)) return Q4_ERR_UNSUPPORTED;
    q4::SdGemmParams items[Q4_MAX_GROUP];
    int n = 0;
    for (int i = 0; i < count; ++i) {
        const q4_sd_gemm_entry& e = entries[i];
        if (e.N < 0) return Q4_ERR_ARG;
        if (e.N % 8) return Q4_ERR_SHAPE;
        if (e.N == 0) continue;
        if (!e.x || !e.w || !e.scales || !e.d_gscale || !e.residue || !e.y) return Q4_ERR_ARG;
        if (!aligned16(e.x) || !aligned16(e.w) || !aligned16(e.scales) || !aligned16(e.residue) || !aligned16(e.y))
            return Q4_ERR_ALIGN;
        q4::SdGemmParams& p = items[n++];
        p.M = M; p.N = e.N; p.K = K; p.x = e.x; p.w = e.w; p.scales = e.scales; p.gscale = e.d_gscale;
        p.residue = e.residue; p.y = e.y; p.out_bf16 = out_dt == Q4_BF16;
    }
    return cuda_status(q4::launch_sd_gemm_grouped(items, n, (cudaStream_t)stream, num_sms()));
}

size_t q4_gemm_workspace_size(q4_format format, int64_t M, int64_t N, int64_t K, int a_kind) {
    (void)N;
    if (a_kind != Q4_A_BF16 || format != Q4_NVFP4 || M <= 0 || K <= 0 || K % 64) return 0;
    if (q4::fused_decode_supported(M, K)) return 0;
    // quantize-once: codes [M, K/2] then tensor-core scales, 256-byte aligned
    const size_t codes = (size_t)M * (size_t)(K / 2);
    const size_t codes_al = (codes + 255) / 256 * 256;
    return codes_al + q4_scale_bytes(Q4_NVFP4, M, K, Q4_LAYOUT_TC);
}

q4_status q4_gemm(q4_format format, int block, int64_t M, int64_t N, int64_t K, int a_kind, const void* a,
                  const uint8_t* a_scales, const float* d_a_gscale, const uint8_t* b_codes,
                  const uint8_t* b_scales, const float* d_b_gscale, q4_dtype out_dt, void* y, void* workspace,
                  size_t ws_bytes, void* stream) {
    if (!valid_format(format) || !valid_dtype(out_dt) || M < 0 || N < 0 || K < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (a_kind != Q4_A_QUANTIZED && a_kind != Q4_A_BF16 && a_kind != Q4_A_BF16_W4A16) return Q4_ERR_ARG;
    if (a_kind == Q4_A_BF16 && format != Q4_NVFP4) return Q4_ERR_UNSUPPORTED;
    const bool w4a16 = a_kind == Q4_A_BF16_W4A16;
    if (format == Q4_NVFP4 && ((!w4a16 && !d_a_gscale) || !d_b_gscale)) return Q4_ERR_ARG;
    if (format == Q4_MXFP4 && (d_a_gscale || d_b_gscale)) return Q4_ERR_ARG;
    if (w4a16 && d_a_gscale) return Q4_ERR_ARG;
    if (a_kind != Q4_A_QUANTIZED && a_scales) return Q4_ERR_ARG;
    if (K % 64 || N % 8) return Q4_ERR_SHAPE;
    if (K > ((int64_t)1 << 30) || M > ((int64_t)1 << 31) || N > ((int64_t)1 << 31)) return Q4_ERR_SHAPE;
    if (M == 0 || N == 0) return Q4_OK;
    if (!y) return Q4_ERR_ARG;
    if (!aligned16(y)) return Q4_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t ysz = (size_t)M * (size_t)N * (out_dt == Q4_BF16 ? 2 : 4);
    if (K == 0) return cuda_status(cudaMemsetAsync(y, 0, ysz, st));
    if (!a || !b_codes || !b_scales || (a_kind == Q4_A_QUANTIZED && !a_scales)) return Q4_ERR_ARG;
    if (!aligned16(a) || !aligned16(b_codes) || !aligned16(b_scales) || (a_scales && !aligned16(a_scales)))
        return Q4_ERR_ALIGN;

    if (w4a16) {
        q4::W4A16Params w;
        w.M = M; w.N = N; w.K = K; w.x = a; w.b_codes = b_codes; w.b_scales = b_scales;
        w.b_gscale = d_b_gscale; w.y = y; w.out_bf16 = out_dt == Q4_BF16; w.mxfp4 = format == Q4_MXFP4;
        return cuda_status(q4::launch_w4a16(w, st, num_sms()));
    }
    const uint8_t* a_codes = static_cast<const uint8_t*>(a);
    if (a_kind == Q4_A_BF16) {
        if (q4::fused_decode_supported(M, K)) {
            q4::FusedDecodeParams f;
            f.M = M; f.N = N; f.K = K; f.a_bf16 = static_cast<const uint16_t*>(a); f.a_gscale = d_a_gscale;
            f.b_codes = b_codes; f.b_scales = b_scales; f.b_gscale = d_b_gscale; f.y = y;
            f.out_bf16 = out_dt == Q4_BF16;
            return cuda_status(q4::launch_fused_decode(f, st, num_sms()));
        }
        // larger M: quantize the activations once into the workspace, then the GEMM
        const size_t need = q4_gemm_workspace_size(format, M, N, K, a_kind);
        if (!workspace || ws_bytes < need) return Q4_ERR_WORKSPACE;
        if (!aligned16(workspace)) return Q4_ERR_ALIGN;
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        const size_t codes_al = ((size_t)M * (size_t)(K / 2) + 255) / 256 * 256;
        q4::QuantParams qp;
        qp.x = a; qp.rows = M; qp.cols = K; qp.ld = K; qp.gscale = d_a_gscale; qp.chan = nullptr;
        qp.codes = ws; qp.scales = ws + codes_al; qp.scols = K / 16; qp.catoms = catoms_of(K, 16);
        cudaError_t e = q4::launch_quantize(qp, 16, true, true, false, false, false, false, st, num_sms());
        if (e != cudaSuccess) return cuda_status(e);
        a_codes = ws;
        a_scales = ws + codes_al;
    }
    q4::GemmParams p;
    p.M = M; p.N = N; p.K = K;
    p.a_codes = a_codes; p.a_scales = a_scales; p.a_gscale = d_a_gscale;
    p.b_codes = b_codes; p.b_scales = b_scales; p.b_gscale = d_b_gscale;
    p.y = y; p.out_bf16 = out_dt == Q4_BF16; p.mxfp4 = format == Q4_MXFP4;
    return cuda_status(q4::launch_gemm(p, st, num_sms()));
}

q4_status q4_set_wait_limit(int64_t cycles) {
    if (cycles == 0) cycles = Q4_DEFAULT_WAIT_CYCLES;
    if (cycles < 1000 || cycles > ((int64_t)1 << 40)) return Q4_ERR_ARG;
    return cuda_status(q4::set_wait_limit((long long)cycles));
}

q4_status q4_gemm_shared_a(q4_format format, int block, int64_t M, int64_t K, const uint8_t* a,
                           const uint8_t* a_scales, const float* d_a_gscale, const q4_gemm_weight* weights,
                           int count, q4_dtype out_dt, void* stream) {
    if (!valid_format(format) || !valid_dtype(out_dt) || M < 0 || K < 0) return Q4_ERR_ARG;
    if (block != block_of(format)) return Q4_ERR_UNSUPPORTED;
    if (count < 1 || count > Q4_MAX_SHARED_A || !weights) return Q4_ERR_ARG;
    if (format == Q4_NVFP4 && !d_a_gscale) return Q4_ERR_ARG;
    if (format == Q4_MXFP4 && d_a_gscale) return Q4_ERR_ARG;
    if (K % 64) return Q4_ERR_SHAPE;
    if (K > ((int64_t)1 << 30) || M > ((int64_t)1 << 31)) return Q4_ERR_SHAPE;
    for (int i = 0; i < count; ++i) {
        const q4_gemm_weight& w = weights[i];
        if (w.N < 0) return Q4_ERR_ARG;
        if (w.N % 8 || w.N > ((int64_t)1 << 31)) return Q4_ERR_SHAPE;
        if (format == Q4_NVFP4 && !w.d_b_gscale) return Q4_ERR_ARG;
        if (format == Q4_MXFP4 && w.d_b_gscale) return Q4_ERR_ARG;
        if (M == 0 || w.N == 0) continue;
        if (!w.y) return Q4_ERR_ARG;
        if (!aligned16(w.y)) return Q4_ERR_ALIGN;
        if (K == 0) continue;
        if (!w.b_codes || !w.b_scales) return Q4_ERR_ARG;
        if (!aligned16(w.b_codes) || !aligned16(w.b_scales)) return Q4_ERR_ALIGN;
    }
    if (M == 0) return Q4_OK;
    cudaStream_t st = (cudaStream_t)stream;
    if (K == 0) {
        for (int i = 0; i < count; ++i)
            if (weights[i].N > 0) {
                const size_t ysz = (size_t)M * (size_t)weights[i].N * (out_dt == Q4_BF16 ? 2 : 4);
                const q4_status s = cuda_status(cudaMemsetAsync(weights[i].y, 0, ysz, st));
                if (s != Q4_OK) return s;
            }
        return Q4_OK;
    }
    if (!a || !a_scales) return Q4_ERR_ARG;
    if (!aligned16(a) || !aligned16(a_scales)) return Q4_ERR_ALIGN;
    q4::GemmParams ps[Q4_MAX_SHARED_A];
    for (int i = 0; i < count; ++i) {
        q4::GemmParams& p = ps[i];
        const q4_gemm_weight& w = weights[i];
        p.M = M; p.N = w.N; p.K = K;
        p.a_codes = a; p.a_scales = a_scales; p.a_gscale = d_a_gscale;
        p.b_codes = w.b_codes; p.b_scales = w.b_scales; p.b_gscale = w.d_b_gscale;
        p.y = w.y; p.out_bf16 = out_dt == Q4_BF16; p.mxfp4 = format == Q4_MXFP4;
    }
    return cuda_status(q4::launch_gemm_multi(ps, count, st, num_sms()));
}

q4_status q4_get_device_error(void* stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e);
    unsigned int word = 0;
    e = q4::read_clear_device_error(&word);
    if (e != cudaSuccess) return cuda_status(e);
    return word ? Q4_ERR_TIMEOUT : Q4_OK;
}

}  // extern "C"
