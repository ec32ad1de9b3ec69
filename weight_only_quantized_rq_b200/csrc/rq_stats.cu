// rq_stats.cu -- per-channel E[x^2] of calibration activations on the device:
// the weights a_k of the E[x^2]-weighted scale search, computed where the
// activations already are and fed to rq_quantize_pack with no host round trip.
//
// Sources: rwkv-quant article, "Two presets and six sizes" (each group's
// scale and shift search weights input channel k by E[x_k^2]);
// rwkv_quant_nv project description, "Operator Optimization Details" (the
// activation statistic of the FP8 path, amax, is computed on the device in a
// prep kernel).
//
// Design: a CTA of 256 threads covers 64 channels of a contiguous range of
// rows. Thread t reads 8 channels (one 16-byte load: eight lanes cover one
// 128-byte line of a row) of rows r0 + t / 8, r0 + t / 8 + 32, ..., eight
// loads in flight per thread (32 KB per CTA, about 100 KB per SM), so the
// activations stream at HBM speed. Each thread adds its rows' squares in
// ascending order into eight fp64 sums; the 32 row phases are then added in
// phase order through shared memory, and a thread-block cluster of up to 8
// CTAs (consecutive row ranges of the same channels) adds its CTAs' totals in
// cluster-rank order through distributed shared memory and adds the result
// to the running sum. The order is fixed, so the result is reproducible run
// to run; it differs from a single ascending sum per channel only by fp64
// rounding (squares of bf16 values are exact in fp64, and every partial sum
// of values that are multiples of a common power of two with few significant
// bits is exact, so for such inputs the two agree bit for bit). No global
// workspace and no atomics.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kThreads = 256;
constexpr int kChan = 64;                    // channels per CTA
constexpr int kLanesPerRow = kChan / 8;      // threads sharing one row (8 channels each)
constexpr int kPhases = kThreads / kLanesPerRow;   // rows read per CTA step
constexpr int kAhead = 8;                    // loads in flight per thread
constexpr int kMaxCluster = 8;

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldg_u16(const uint16_t* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
// a + v^2 for the bf16 value in the low / high half of w (exact square in fp64)
__device__ __forceinline__ double add_sq_lo(double a, uint32_t w) {
    const double f = (double)__uint_as_float(w << 16);
    return __fma_rn(f, f, a);
}
__device__ __forceinline__ double add_sq_hi(double a, uint32_t w) {
    const double f = (double)__uint_as_float(w & 0xffff0000u);
    return __fma_rn(f, f, a);
}
__device__ __forceinline__ void add_sq8(double (&a)[8], const uint4 v) {
    a[0] = add_sq_lo(a[0], v.x); a[1] = add_sq_hi(a[1], v.x);
    a[2] = add_sq_lo(a[2], v.y); a[3] = add_sq_hi(a[3], v.y);
    a[4] = add_sq_lo(a[4], v.z); a[5] = add_sq_hi(a[5], v.z);
    a[6] = add_sq_lo(a[6], v.w); a[7] = add_sq_hi(a[7], v.w);
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ double ld_dsmem_f64(const void* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(a) : "memory");
    return v;
}

// Grid: (channel blocks) x (row ranges), clusters of `split` CTAs along the
// row ranges; CTA j of a cluster takes rows [R j / split, R (j + 1) / split).
__global__ void __launch_bounds__(kThreads) act_sumsq_kernel(const uint16_t* __restrict__ x, int R, int K,
                                                               double* __restrict__ sum_sq) {
    __shared__ double part[kPhases][kChan];
    __shared__ double tot[kChan];
    const int t = threadIdx.x, lr = t % kLanesPerRow, ph = t / kLanesPerRow;
    const uint32_t j = cluster_rank(), split = cluster_size();
    const int cb = (int)(blockIdx.x / split);
    const int k0 = cb * kChan + 8 * lr;                       // this thread's first channel
    const int ra = (int)((long long)R * j / split), rb = (int)((long long)R * (j + 1) / split);
    double a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = 0.0;
    if ((K & 7) == 0) {                                       // 16-byte rows of 8 channels
        if (k0 < K) {
            const uint16_t* p = x + (size_t)(ra + ph) * K + k0;
            const size_t step = (size_t)kPhases * K;
            int r = ra + ph;
            for (; r + (kAhead - 1) * kPhases < rb; r += kAhead * kPhases) {
                uint4 v[kAhead];
#pragma unroll
                for (int i = 0; i < kAhead; ++i) v[i] = ldg_stream(p + (size_t)i * step);
                p += (size_t)kAhead * step;
#pragma unroll
                for (int i = 0; i < kAhead; ++i) add_sq8(a, v[i]);   // ascending rows
            }
            for (; r < rb; r += kPhases, p += step) add_sq8(a, ldg_stream(p));
        }
    } else {                                                  // any K: one value at a time
        for (int r = ra + ph; r < rb; r += kPhases) {
            const uint16_t* row = x + (size_t)r * K;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (k0 + i < K) a[i] = add_sq_lo(a[i], ldg_u16(row + k0 + i));
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) part[ph][8 * lr + i] = a[i];
    __syncthreads();
    if (t < kChan) {                                          // row phases in order
        double s = 0.0;
        for (int q = 0; q < kPhases; ++q) s += part[q][t];
        tot[t] = s;
    }
    cluster_sync();                                           // every CTA total of the cluster is in place
    if (j == 0 && t < kChan) {
        const int k = cb * kChan + t;
        if (k < K) {
            double s = 0.0;
            for (uint32_t q = 0; q < split; ++q) s += ld_dsmem_f64(&tot[t], q);   // row ranges in order
            sum_sq[k] = sum_sq[k] + s;
        }
    }
    cluster_sync();                                           // peers' shared memory stays until rank 0 has read it
}

__global__ void act_finalize_kernel(const double* __restrict__ sum_sq, int K, double rows, float* __restrict__ out) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < K) out[k] = (float)(sum_sq[k] / rows);
}

}  // namespace

cudaError_t launch_act_sumsq(const void* x, int R, int K, double* sum_sq, cudaStream_t st) {
    // Row ranges per channel block: enough CTAs for about four per SM, at
    // least one CTA step of rows each, at most one cluster.
    const int cblocks = (K + kChan - 1) / kChan;
    int split = (4 * sm_count() + cblocks - 1) / cblocks;
    split = split > kMaxCluster ? kMaxCluster : split;
    while (split > 1 && R / split < kPhases) --split;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(cblocks * split));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, act_sumsq_kernel, static_cast<const uint16_t*>(x), R, K, sum_sq);
}

cudaError_t launch_act_finalize(const double* sum_sq, int K, long long rows, float* act_sq, cudaStream_t st) {
    act_finalize_kernel<<<(K + 255) / 256, 256, 0, st>>>(sum_sq, K, (double)rows, act_sq);
    return cudaGetLastError();
}

}  // namespace rq
