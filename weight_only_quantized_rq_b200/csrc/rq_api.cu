// rq_api.cu -- the C ABI of librq (declared in include/rq.h): argument
// validation on the host, then dispatch to the kernels. Validation happens
// before any CUDA runtime call, so a rejected call launches nothing and needs
// no GPU.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/rq.h"
#include "rq_internal.h"

namespace {

thread_local int t_last_cuda = 0;

bool fmt_ok(int fmt) {
    return fmt == rq::kFmtW4G64 || rq::is_w8(fmt) || fmt == rq::kFmtW6G16 || rq::is_sb(fmt);
}

// RQ_OK, or the status for an unsupported (fmt, K, N).
int shape_status(int fmt, int K, int N) {
    if (!fmt_ok(fmt)) return RQ_ERR_INVALID_ARG;
    if (N < 1 || N > (1 << 24) || K < 64 || K > 32768) return RQ_ERR_INVALID_ARG;
    if (K % 64 != 0) return RQ_ERR_UNSUPPORTED_SHAPE;
    if (rq::is_sb(fmt) && K % 256 != 0) return RQ_ERR_UNSUPPORTED_SHAPE;
    return RQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_packed(const rq_packed* w, int K, int N) {
    if (!w) return RQ_ERR_INVALID_ARG;
    int s = shape_status(w->fmt, w->K, w->N);
    if (s != RQ_OK) return s;
    if (w->K != K || w->N != N || w->reserved != 0) return RQ_ERR_FORMAT_MISMATCH;
    if (!w->codes) return RQ_ERR_INVALID_ARG;
    if (rq::is_sb(w->fmt)) {
        if (w->scales) return RQ_ERR_FORMAT_MISMATCH;
    } else if (!w->scales) {
        return RQ_ERR_INVALID_ARG;
    }
    if (!aligned16(w->codes) || (w->scales && !aligned16(w->scales))) return RQ_ERR_MISALIGNED;
    return RQ_OK;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return RQ_OK;
    t_last_cuda = (int)e;
    return RQ_ERR_CUDA;
}

}  // namespace

namespace rq {

namespace {
unsigned long long g_wait_ns = 2000000000ull;
int g_test_flags = 0;
}  // namespace

unsigned long long wait_limit_ns() { return __atomic_load_n(&g_wait_ns, __ATOMIC_RELAXED); }
int test_flags() { return __atomic_load_n(&g_test_flags, __ATOMIC_RELAXED); }

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    int v = __atomic_load_n(&cache[dev & 63], __ATOMIC_RELAXED);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        __atomic_store_n(&cache[dev & 63], v, __ATOMIC_RELAXED);
    }
    return v;
}

}  // namespace rq

extern "C" {

size_t rq_packed_size(int fmt, int K, int N, size_t* codes_bytes, size_t* scales_bytes) {
    if (shape_status(fmt, K, N) != RQ_OK) return 0;
    const size_t cb = rq::code_row_bytes(fmt, K) * (size_t)N;
    const size_t sb = rq::round16(rq::scale_row_bytes(fmt, K) * (size_t)N);
    if (codes_bytes) *codes_bytes = cb;
    if (scales_bytes) *scales_bytes = sb;
    return cb + sb;
}

int rq_quantize_pack(const float* W, int K, int N, const float* act_sq, const rq_search* search,
                     const rq_packed* out, void* stream) {
    if (!W || !out) return RQ_ERR_INVALID_ARG;
    int s = check_packed(out, K, N);
    if (s != RQ_OK) return s;
    rq_search sr = {64, 0.7f, 1.0f};
    if (search) sr = *search;
    if (sr.n_cand < 1 || sr.n_cand > 256 || !std::isfinite(sr.t_lo) || !std::isfinite(sr.t_hi) ||
        !(sr.t_lo > 0.0f) || sr.t_lo > sr.t_hi || sr.t_hi > 4.0f)
        return RQ_ERR_INVALID_ARG;
    if (!aligned16(W) || (act_sq && !aligned16(act_sq))) return RQ_ERR_MISALIGNED;
    size_t sbytes = 0;
    rq_packed_size(out->fmt, K, N, nullptr, &sbytes);
    rq::PackArgs a = {out->fmt, K, N, W, act_sq, sr.n_cand, sr.t_lo, sr.t_hi, out->codes, out->scales, sbytes};
    return cuda_status(rq::launch_quantize_pack(a, static_cast<cudaStream_t>(stream)));
}

int rq_hessian_accum(const void* x, int R, int K, double* H, void* stream) {
    if (!x || !H) return RQ_ERR_INVALID_ARG;
    if (R < 1 || R > (1 << 24) || K < 1 || K > 32768) return RQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(H)) return RQ_ERR_MISALIGNED;
    return cuda_status(rq::launch_hessian(x, R, K, H, static_cast<cudaStream_t>(stream)));
}

int rq_gptq_prepare(const double* H, int K, double damp, double* U, unsigned char* dead, void* stream) {
    if (!H || !U || !dead) return RQ_ERR_INVALID_ARG;
    if (K < 1 || K > 16384 || !std::isfinite(damp) || damp < 0.0) return RQ_ERR_INVALID_ARG;
    const uintptr_t h0 = reinterpret_cast<uintptr_t>(H), u0 = reinterpret_cast<uintptr_t>(U);
    const uintptr_t bytes = (uintptr_t)K * (uintptr_t)K * sizeof(double);
    if (h0 < u0 + bytes && u0 < h0 + bytes) return RQ_ERR_INVALID_ARG;      // H and U must not overlap
    if (!aligned16(H) || !aligned16(U)) return RQ_ERR_MISALIGNED;
    return cuda_status(rq::launch_gptq_prepare(H, K, damp, U, dead, static_cast<cudaStream_t>(stream)));
}

int rq_gptq_quantize_pack(const float* W, int K, int N, const double* U, const unsigned char* dead,
                          const float* act_sq, const rq_search* search, const rq_packed* out, void* stream) {
    if (!W || !U || !dead || !out) return RQ_ERR_INVALID_ARG;
    int s = check_packed(out, K, N);
    if (s != RQ_OK) return s;
    if (K > 16384 || rq::gptq_rows_per_block(out->fmt, K) == 0) return RQ_ERR_UNSUPPORTED_SHAPE;
    rq_search sr = {64, 0.7f, 1.0f};
    if (search) sr = *search;
    if (sr.n_cand < 1 || sr.n_cand > 256 || !std::isfinite(sr.t_lo) || !std::isfinite(sr.t_hi) ||
        !(sr.t_lo > 0.0f) || sr.t_lo > sr.t_hi || sr.t_hi > 4.0f)
        return RQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(U) || (act_sq && !aligned16(act_sq))) return RQ_ERR_MISALIGNED;
    size_t sbytes = 0;
    rq_packed_size(out->fmt, K, N, nullptr, &sbytes);
    rq::GptqArgs a = {out->fmt, K, N, W, U, dead, act_sq, sr.n_cand, sr.t_lo, sr.t_hi, out->codes, out->scales,
                      sbytes};
    return cuda_status(rq::launch_gptq_pack(a, static_cast<cudaStream_t>(stream)));
}

int rq_wgemm_out(const void* x, int M, int K, int N, const rq_packed* w, void* y, int out_type, void* stream) {
    if (!x || !y || !w) return RQ_ERR_INVALID_ARG;
    if (M < 1 || M > 128) return RQ_ERR_INVALID_ARG;
    if (out_type != RQ_OUT_F32 && out_type != RQ_OUT_BF16) return RQ_ERR_INVALID_ARG;
    int s = check_packed(w, K, N);
    if (s != RQ_OK) return s;
    if (!aligned16(x) || !aligned16(y)) return RQ_ERR_MISALIGNED;
    rq::WgemmArgs a = {w->fmt, M, K, N, x, w->codes, w->scales, y, out_type == RQ_OUT_BF16 ? 1 : 0};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rq::tc_supported(w->fmt, M)) return cuda_status(rq::launch_tc(&a, 1, st));
    return cuda_status(rq::launch_gemv(&a, 1, st));
}

int rq_wgemm(const void* x, int M, int K, int N, const rq_packed* w, float* y, void* stream) {
    return rq_wgemm_out(x, M, K, N, w, y, RQ_OUT_F32, stream);
}

int rq_wgemm_batch_out(const rq_wgemm_item* items, int count, int M, int out_type, void* stream) {
    if (!items || count < 1 || count > rq::kMaxBatch) return RQ_ERR_INVALID_ARG;
    if (M < 1 || M > 128) return RQ_ERR_INVALID_ARG;
    if (out_type != RQ_OUT_F32 && out_type != RQ_OUT_BF16) return RQ_ERR_INVALID_ARG;
    rq::WgemmArgs a[rq::kMaxBatch];
    for (int i = 0; i < count; ++i) {
        const rq_wgemm_item& it = items[i];
        if (!it.x || !it.y || !it.w) return RQ_ERR_INVALID_ARG;
        int s = check_packed(it.w, it.w->K, it.w->N);
        if (s != RQ_OK) return s;
        if (it.w->fmt != items[0].w->fmt) return RQ_ERR_FORMAT_MISMATCH;
        if (!aligned16(it.x) || !aligned16(it.y)) return RQ_ERR_MISALIGNED;
        a[i] = {it.w->fmt, M, it.w->K, it.w->N, it.x, it.w->codes, it.w->scales, it.y, out_type == RQ_OUT_BF16 ? 1 : 0};
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (rq::tc_supported(a[0].fmt, M)) return cuda_status(rq::launch_tc(a, count, st));
    return cuda_status(rq::launch_gemv(a, count, st));
}

int rq_wgemm_batch(const rq_wgemm_item* items, int count, int M, void* stream) {
    return rq_wgemm_batch_out(items, count, M, RQ_OUT_F32, stream);
}

int rq_dequant(const rq_packed* w, float* W_out, void* stream) {
    if (!w || !W_out) return RQ_ERR_INVALID_ARG;
    int s = check_packed(w, w->K, w->N);
    if (s != RQ_OK) return s;
    if (!aligned16(W_out)) return RQ_ERR_MISALIGNED;
    return cuda_status(rq::launch_dequant(w->fmt, w->K, w->N, w->codes, w->scales, W_out,
                                          static_cast<cudaStream_t>(stream)));
}

int rq_act_sumsq(const void* x, int R, int K, double* sum_sq, void* stream) {
    if (!x || !sum_sq) return RQ_ERR_INVALID_ARG;
    if (R < 1 || R > (1 << 24) || K < 1 || K > (1 << 20)) return RQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(sum_sq)) return RQ_ERR_MISALIGNED;
    return cuda_status(rq::launch_act_sumsq(x, R, K, sum_sq, static_cast<cudaStream_t>(stream)));
}

int rq_act_finalize(const double* sum_sq, int K, long long rows, float* act_sq, void* stream) {
    if (!sum_sq || !act_sq) return RQ_ERR_INVALID_ARG;
    if (K < 1 || K > (1 << 20) || rows < 1) return RQ_ERR_INVALID_ARG;
    if (!aligned16(sum_sq) || !aligned16(act_sq)) return RQ_ERR_MISALIGNED;
    return cuda_status(rq::launch_act_finalize(sum_sq, K, rows, act_sq, static_cast<cudaStream_t>(stream)));
}

const char* rq_status_string(int status) {
    switch (status) {
        case RQ_OK: return "ok";
        case RQ_ERR_INVALID_ARG: return "invalid argument (NULL pointer, or M/K/N/search out of range)";
        case RQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (K must be a multiple of 64; of 256 for the superblock formats)";
        case RQ_ERR_FORMAT_MISMATCH: return "packed descriptor does not match the call (format, K or N)";
        case RQ_ERR_MISALIGNED: return "a device pointer is not 16-byte aligned";
        case RQ_ERR_CUDA: return "CUDA runtime error (see rq_last_cuda_error)";
        case RQ_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
        case RQ_ERR_NOT_POSITIVE_DEFINITE: return "a GPTQ Hessian was not positive definite after damping";
        default: return "unknown status";
    }
}

int rq_last_cuda_error(void) { return t_last_cuda; }

int rq_device_status(void* stream, int* word) {
    if (!word) return RQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned a = 0, b = 0, c = 0, d = 0;
    int s = cuda_status(rq::status_pack(st, &a));
    if (s == RQ_OK) s = cuda_status(rq::status_gemv(st, &b));
    if (s == RQ_OK) s = cuda_status(rq::status_tc(st, &c));
    if (s == RQ_OK) s = cuda_status(rq::status_gptq(st, &d));
    const unsigned w = a | b | c | d;
    *word = (int)w;
    if (s != RQ_OK) return s;
    if (w & ~(unsigned)rq::kStatusNotSpd) return RQ_ERR_DEVICE_TIMEOUT;
    return w ? RQ_ERR_NOT_POSITIVE_DEFINITE : RQ_OK;
}

int rq_test_hooks(long long wait_ns, int flags) {
    if (wait_ns < 0 || wait_ns > 60000000000ll || (flags & ~rq::kTestNoCopies) != 0) return RQ_ERR_INVALID_ARG;
    __atomic_store_n(&rq::g_wait_ns, wait_ns == 0 ? 2000000000ull : (unsigned long long)wait_ns, __ATOMIC_RELAXED);
    __atomic_store_n(&rq::g_test_flags, flags, __ATOMIC_RELAXED);
    return RQ_OK;
}

int rq_version(void) { return 200; }

}  // extern "C"
