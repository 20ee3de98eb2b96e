// q4_internal.h -- parameter blocks and launcher declarations shared by the
// kernel files and the C-ABI layer.  Not part of the public interface.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace q4 {

struct QuantParams {
    const void* x;        // [rows, ld] bf16 or fp32
    int64_t rows, cols, ld;
    const float* gscale;  // NVFP4 tensor scale (device), else unused
    const float* chan;    // MXFP4 per-column multiplier or nullptr
    uint8_t* codes;       // [rows, cols/2]
    uint8_t* scales;      // tensor-core layout or row-major
    int64_t scols;        // cols / block
    int64_t catoms;       // ceil(scols / 4)
    int inject_stall = 0; // failure-detection test: the tiled kernel loads nothing for its first tile
    // amax + quantize in one launch: out[0] = amax, out[1] = amax / denom (the
    // tensor scale used), out[2] = the grid barrier's arrival count (zeroed
    // by the launcher)
    unsigned int* amax_out = nullptr;
    float denom = 0.0f;
};

struct SigmaDeltaParams {
    const float* w;       // [rows, cols]
    int64_t rows, cols;
    const uint8_t* scales;
    const float* gscale;
    float* residue;       // [rows, cols], in/out
    uint8_t* codes;       // [rows, cols/2]
    int64_t scols, catoms;
};

// One matrix of a grouped launch, and the launch's table of them (passed
// by value as a kernel parameter).  A work unit is 8 weights of a row for the
// requant kernels and one block (padded grid in the tensor-core layout) for
// the quantizer; `start` is the entry's first unit in the launch.
constexpr int kMaxGroup = 32;
struct GroupItem {
    const void* w;        // [rows, cols], dense
    int64_t rows, cols;
    uint8_t* scales;
    const float* gscale;
    float* residue;
    uint8_t* codes;
    int64_t scols, catoms;
    int64_t start;
};
struct GroupParams {
    int count;
    int64_t total;        // units over all entries
    GroupItem m[kMaxGroup];
};
static_assert(sizeof(GroupParams) <= 4096, "a grouped launch's table must fit the kernel parameter space");

struct DequantParams {
    const uint8_t* codes;
    const uint8_t* scales;
    const float* gscale;
    int64_t rows, cols;
    void* out;
    int64_t scols, catoms;
};

struct GemmParams {
    int64_t M, N, K;
    const uint8_t* a_codes;   // [M, K/2]
    const uint8_t* a_scales;  // tensor-core layout
    const float* a_gscale;    // NVFP4 s_tA or nullptr
    const uint8_t* b_codes;   // [N, K/2]
    const uint8_t* b_scales;
    const float* b_gscale;
    void* y;                  // [M, N]
    bool out_bf16;
    bool mxfp4;
};

struct FusedDecodeParams {
    int64_t M, N, K;
    const uint16_t* a_bf16;   // [M, K] bf16 activations
    const float* a_gscale;    // activation tensor scale
    const uint8_t* b_codes;
    const uint8_t* b_scales;
    const float* b_gscale;
    void* y;
    bool out_bf16;
};

struct W4A16Params {
    int64_t M, N, K;
    const void* x;            // [M, K] bf16 activations
    const uint8_t* b_codes;   // [N, K/2]
    const uint8_t* b_scales;  // tensor-core layout
    const float* b_gscale;    // NVFP4 s_t or nullptr
    void* y;                  // [M, N]
    bool out_bf16;
    bool mxfp4;
};

cudaError_t launch_w4a16(const W4A16Params& p, cudaStream_t st, int num_sms);

struct SdGemmParams {
    int64_t M, N, K;
    const void* x;            // [M, K] bf16 activations, M <= 16
    const float* w;           // [N, K] fp32 master weight
    const uint8_t* scales;    // NVFP4 block scales, tensor-core layout
    const float* gscale;      // s_t
    float* residue;           // [N, K] fp32, read and written
    void* y;                  // [M, N]
    bool out_bf16;
};

bool sd_gemm_supported(int64_t M, int64_t K);
cudaError_t launch_sd_gemm(const SdGemmParams& p, cudaStream_t st, int num_sms);
// Every entry as launch_sd_gemm, in one launch (entries share M, K, out_bf16;
// count <= kMaxGroup).
cudaError_t launch_sd_gemm_grouped(const SdGemmParams* items, int count, cudaStream_t st, int num_sms);
cudaError_t launch_amax(const void* x, int64_t n, bool bf16, float denom, float* d_out,
                        cudaStream_t st, int num_sms);
cudaError_t launch_quantize(const QuantParams& p, int blk, bool bf16, bool tc, bool ru, bool had,
                            bool chan, bool s46, cudaStream_t st, int num_sms);
// NVFP4 tensor amax, tensor scale and block quantize in one cooperative launch.
cudaError_t launch_amax_quantize(const QuantParams& p, bool bf16, bool tc, bool ru, cudaStream_t st, int num_sms);
cudaError_t launch_sigma_delta(const SigmaDeltaParams& p, int blk, bool tc, cudaStream_t st, int num_sms);
cudaError_t launch_sigma_delta_banks(const SigmaDeltaParams& p, int blk, bool tc, int visits, float* r_out,
                                     cudaStream_t st, int num_sms);
cudaError_t launch_sr_requant(const SigmaDeltaParams& p, int blk, bool tc, uint64_t seed, uint32_t visit,
                              cudaStream_t st, int num_sms);
cudaError_t launch_dequantize(const DequantParams& p, int blk, bool tc, bool out_bf16, cudaStream_t st,
                              int num_sms);
// Grouped launches: every entry of g as the single-matrix launch above
// (g.m[i].start and g.total are filled in by the launcher).
cudaError_t launch_quantize_grouped(GroupParams& g, int blk, bool bf16, bool tc, bool ru, bool had, bool s46,
                                    cudaStream_t st, int num_sms);
cudaError_t launch_sigma_delta_grouped(GroupParams& g, int blk, bool tc, cudaStream_t st, int num_sms);
cudaError_t launch_sr_requant_grouped(GroupParams& g, int blk, bool tc, uint64_t seed, uint32_t visit,
                                      cudaStream_t st, int num_sms);
cudaError_t launch_sigma_delta_banks_grouped(GroupParams& g, int blk, bool tc, int visits, cudaStream_t st,
                                             int num_sms);
cudaError_t launch_gemm(const GemmParams& p, cudaStream_t st, int num_sms);
// One quantized A (ps[i].M, K, a_* equal for all i) times 1..4 weights in one launch.
cudaError_t launch_gemm_multi(const GemmParams* ps, int nw, cudaStream_t st, int num_sms);
cudaError_t launch_fused_decode(const FusedDecodeParams& p, cudaStream_t st, int num_sms);

// Reads and clears the device error words of all kernel files (bit 0: a
// bounded wait ran out); read_clear_quant_error covers the quantize file only.
cudaError_t read_clear_device_error(unsigned int* word);
cudaError_t read_clear_quant_error(unsigned int* word);

// Sets the bounded-wait limit (SM clock cycles) of all kernel files.
cudaError_t set_wait_limit(long long cycles);
cudaError_t set_quant_wait_limit(long long cycles);

// 2-D tiled tensor map over a row-major [outer, inner] array of `dt`
// elements with rows `row_bytes` apart; out-of-range box parts read as zero
// and are not written by stores.  False if the encoder rejects it.
bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// Whether the fused-activation small-M GEMM takes this shape (M <= 128 and
// the quantized activations fit in shared memory next to >= 2 weight stages).
bool fused_decode_supported(int64_t M, int64_t K);

// Q4_OK for cudaSuccess; otherwise records the error's text for q4_last_error()
// (per host thread) and returns Q4_ERR_CUDA (the value as an int: q4.h is not
// included here).
int status_of_cuda(cudaError_t e);

}  // namespace q4
