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
// Design: the rows are cut into 64 contiguous chunks. A thread-block cluster
// of 8 CTAs covers 64 channels: warp w of cluster rank j sums chunk 8 j + w
// (rows ascending) for the cluster's channels, two channels per lane so that
// a warp reads one 128-byte line per row, with eight loads in flight ahead of
// the in-order additions. Rank 0 then adds the 64 chunk sums in chunk order,
// reading its peers' partials through distributed shared memory, and adds
// the total to the running sum. Squares of bf16 values are exact in fp64 and
// every sum is an fp64 addition in this fixed order, so the result is
// bit-reproducible; no global workspace and no atomics.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kWarps = 8;        // warps (row chunks) per CTA
constexpr int kCluster = 8;      // CTAs per cluster (one channel block)
constexpr int kChunks = kWarps * kCluster;   // row chunks per call
constexpr int kChan = 64;        // channels per cluster
constexpr int kAhead = 8;        // loads in flight per thread

__device__ __forceinline__ double sq_lo(uint32_t v) {
    const double f = (double)__uint_as_float(v << 16);
    return f * f;
}
__device__ __forceinline__ double sq_hi(uint32_t v) {
    const double f = (double)__uint_as_float(v & 0xffff0000u);
    return f * f;
}
__device__ __forceinline__ uint32_t ldg_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldg_u16(const uint16_t* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
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

__global__ void __launch_bounds__(kWarps * 32) act_sumsq_kernel(const uint16_t* __restrict__ x, int R, int K,
                                                                 double* __restrict__ sum_sq) {
    __shared__ double part[kWarps][kChan];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t j = cluster_rank();
    const int c = (int)j * kWarps + w;                      // this warp's row chunk
    const int k = (int)(blockIdx.x / kCluster) * kChan + 2 * lane;   // this lane's channels k, k + 1
    const int rc = (R + kChunks - 1) / kChunks;
    const int r0 = c * rc < R ? c * rc : R, r1 = r0 + rc < R ? r0 + rc : R;
    double a0 = 0.0, a1 = 0.0;
    if ((K & 1) == 0 && k + 1 < K) {                          // both channels, one 4-byte load per row
        const size_t step = (size_t)K / 2;
        const uint32_t* p = reinterpret_cast<const uint32_t*>(x + (size_t)r0 * K + k);
        int r = r0;
        for (; r + kAhead <= r1; r += kAhead) {
            uint32_t v[kAhead];
#pragma unroll
            for (int i = 0; i < kAhead; ++i) v[i] = ldg_u32(p + (size_t)i * step);
            p += (size_t)kAhead * step;
#pragma unroll
            for (int i = 0; i < kAhead; ++i) {                // ascending rows
                a0 += sq_lo(v[i]);
                a1 += sq_hi(v[i]);
            }
        }
        for (; r < r1; ++r, p += step) {
            const uint32_t v = ldg_u32(p);
            a0 += sq_lo(v);
            a1 += sq_hi(v);
        }
    } else {                                                  // odd K or the last channel: one value at a time
        for (int r = r0; r < r1; ++r) {
            const uint16_t* row = x + (size_t)r * K;
            if (k < K) a0 += sq_lo(ldg_u16(row + k));
            if (k + 1 < K) a1 += sq_lo(ldg_u16(row + k + 1));
        }
    }
    part[w][2 * lane] = a0;
    part[w][2 * lane + 1] = a1;
    cluster_sync();                                          // every chunk sum of the cluster is in place
    if (j == 0 && threadIdx.x < kChan) {
        const int kk = (int)(blockIdx.x / kCluster) * kChan + threadIdx.x;
        if (kk < K) {
            double t = 0.0;
            for (uint32_t rk = 0; rk < (uint32_t)kCluster; ++rk)      // chunks ascending
#pragma unroll
                for (int ww = 0; ww < kWarps; ++ww) t += ld_dsmem_f64(&part[ww][threadIdx.x], rk);
            sum_sq[kk] = sum_sq[kk] + t;
        }
    }
    cluster_sync();                                          // peers' shared memory stays until rank 0 has read it
}

__global__ void act_finalize_kernel(const double* __restrict__ sum_sq, int K, double rows, float* __restrict__ out) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < K) out[k] = (float)(sum_sq[k] / rows);
}

}  // namespace

cudaError_t launch_act_sumsq(const void* x, int R, int K, double* sum_sq, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(((K + kChan - 1) / kChan) * kCluster));
    cfg.blockDim = dim3(kWarps * 32);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
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
