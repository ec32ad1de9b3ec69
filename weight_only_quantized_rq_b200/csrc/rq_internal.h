// rq_internal.h -- host-side interfaces between librq's C ABI layer
// (rq_api.cu) and its kernel files. Not installed; not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace rq {

// Device status bit of a Cholesky pivot that was not positive (the other
// bits, all bounded-wait timeouts, are listed with the device helpers).
constexpr unsigned kStatusNotSpd = 1u << 5;

constexpr int kFmtW4G64 = 1;
constexpr int kFmtW8G16 = 2;
constexpr int kFmtW4SB32 = 3;
constexpr int kFmtW5SB32 = 4;
constexpr int kFmtW6SB32 = 5;
constexpr int kFmtW8G64 = 6;
constexpr int kFmtW6G16 = 7;

// int8 codes (one byte per weight; group 16 or 64).
__host__ __device__ constexpr bool is_w8(int fmt) { return fmt == kFmtW8G16 || fmt == kFmtW8G64; }
// Weights per fp16 scale of the symmetric formats.
__host__ __device__ constexpr int sym_group(int fmt) { return fmt == kFmtW4G64 || fmt == kFmtW8G64 ? 64 : 16; }

// The asymmetric superblock formats: bits per code and bytes per record of
// 256 weights (16-byte header, 128 bytes of low nibbles, high-bit plane).
__host__ __device__ constexpr bool is_sb(int fmt) { return fmt >= kFmtW4SB32 && fmt <= kFmtW6SB32; }
__host__ __device__ constexpr int sb_bits(int fmt) { return fmt - kFmtW4SB32 + 4; }
__host__ __device__ constexpr int sb_record(int fmt) { return 16 + 128 + (sb_bits(fmt) - 4) * 32; }

// Bytes per row of the codes plane (records plane for the superblock formats)
// and of the scales plane.
// 6-bit symmetric codes: 48 bytes per 64 weights (32 bytes of low nibbles,
// then 16 bytes of the codes' bits 4..5).
inline size_t code_row_bytes(int fmt, int K) {
    return fmt == kFmtW4G64 ? (size_t)K / 2
         : is_w8(fmt)       ? (size_t)K
         : fmt == kFmtW6G16 ? (size_t)K / 64 * 48
                            : (size_t)K / 256 * sb_record(fmt);
}
inline size_t scale_row_bytes(int fmt, int K) {
    return is_sb(fmt) ? 0 : (size_t)K / sym_group(fmt) * 2;
}
__host__ __device__ inline size_t round16(size_t v) { return (v + 15) & ~(size_t)15; }

struct PackArgs {
    int fmt, K, N;
    const float* W;
    const float* act_sq;
    int n_cand;
    float t_lo, t_hi;
    void* codes;
    void* scales;
    size_t scales_bytes;   // padded plane size (padding is zeroed)
};

cudaError_t launch_quantize_pack(const PackArgs& a, cudaStream_t st);

// GPTQ on the preset's grid (every format): the input Hessian, the upper
// Cholesky factor U of its damped inverse, and the column loop.
struct GptqArgs {
    int fmt, K, N;
    const float* W;
    const double* U;
    const uint8_t* dead;
    const float* act_sq;
    int n_cand;
    float t_lo, t_hi;
    void* codes;
    void* scales;
    size_t scales_bytes;
};
cudaError_t launch_hessian(const void* x, int R, int K, double* H, cudaStream_t st);
cudaError_t launch_gptq_prepare(const double* H, int K, double damp, double* U, uint8_t* dead, cudaStream_t st);
cudaError_t launch_gptq_pack(const GptqArgs& a, cudaStream_t st);
int gptq_rows_per_block(int fmt, int K);   // 0 when one row does not fit in shared memory
cudaError_t launch_dequant(int fmt, int K, int N, const void* codes, const void* scales, float* out,
                           cudaStream_t st);

struct WgemmArgs {
    int fmt, M, K, N;
    const void* x;         // bf16 [M][K]
    const void* codes;
    const void* scales;
    void* y;               // fp32 [M][N], or bf16 [M][N] when ybf16
    int ybf16;             // 1: y is rounded once to bf16 (round to nearest even)
};

// Memory-bound path (few activation rows): dequantize in registers, fp32
// accumulate. `count` independent products of one format and one M share a
// launch (1 <= count <= kMaxBatch).
constexpr int kMaxBatch = 160;
cudaError_t launch_gemv(const WgemmArgs* a, int count, cudaStream_t st);

// Tensor-core path (kTcMinM <= M <= 128; every M for the 5- and 6-bit
// formats): bf16 tiles dequantized into tensor memory, tcgen05.mma against x
// in shared memory.
// `count` independent products of one format and one M share a launch.
constexpr int kTcMinM = 3;
bool tc_supported(int fmt, int M);
cudaError_t launch_tc(const WgemmArgs* a, int count, cudaStream_t st);

// Per-channel sums of squares of bf16 activations (adds into sum_sq) and
// their finalization into fp32 E[x^2].
cudaError_t launch_act_sumsq(const void* x, int R, int K, double* sum_sq, cudaStream_t st);
cudaError_t launch_act_finalize(const double* sum_sq, int K, long long rows, float* act_sq, cudaStream_t st);

// Read and clear the device status word of each kernel file (synchronizes st).
cudaError_t status_pack(cudaStream_t st, unsigned* word);
cudaError_t status_gptq(cudaStream_t st, unsigned* word);
cudaError_t status_gemv(cudaStream_t st, unsigned* word);
cudaError_t status_tc(cudaStream_t st, unsigned* word);

int sm_count();   // multiprocessors of the current device

// Bound of every device wait that a launch passes to its kernel (2 s unless
// rq_test_hooks set another), and the testing flags rq_test_hooks set
// (bit 0: the threads that issue weight copies issue none, so the waits for
// them run out).
unsigned long long wait_limit_ns();
int test_flags();
constexpr int kTestNoCopies = 1;

}  // namespace rq
