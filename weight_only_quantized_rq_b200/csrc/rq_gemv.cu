// rq_gemv.cu -- the memory-bound product y = x * w_hat^T for a few activation
// rows (decode), with w_hat formed in registers.
//
// Source: RWKV-7 G1 1.5B int4 model card, summary paragraph: decode is served
// by a hand-written int4 GEMV / small-M GEMM family and the kernel output is
// bit-identical to the offline dequantization; rwkv-quant article, "Two
// presets and six sizes": the int8 group-16 and int4 superblock formats.
//
// Design (B200):
//  * One producer warp streams whole row tiles (R rows x K, codes and scales
//    are contiguous in HBM) into a ring of shared-memory stages with
//    untiled bulk-async copies completed on mbarriers; the copies are issued
//    before griddepcontrol.wait, so with programmatic dependent launch the
//    next matrix's weights are already in flight while the previous kernel
//    drains.
//  * x is staged once per CTA as fp32 in shared memory, in the order the
//    unpack produces weights, interleaved by 16-byte quads so that lanes
//    reading consecutive half-chunks hit consecutive banks; the sum of x over
//    each 32-weight half-chunk is stored beside it.
//  * A team of T lanes (a power of two dividing K/32) owns RW rows of a tile;
//    lane i of the team takes half-chunks i, i+T, ... of those rows. Codes are
//    unpacked to fp32 values 128 + u (or q for int8) with byte permutes and
//    multiplied into fp32 accumulators; the per-group scale and the code
//    offset are applied once per half-chunk:
//        sum_k (u_k - 8) x_k s = s * (sum_k (128 + u_k) x_k - 136 sum_k x_k).
//  * Team partial sums are reduced with warp shuffles and written once.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;

struct GemvParams {
    const uint16_t* x;     // bf16 bits [M][K]
    const uint8_t* codes;
    const uint8_t* scales;
    float* y;
    int K, N;
    int m0, mrows;         // activation rows [m0, m0 + mrows) handled here
    int T, HJ, RW, R;      // team lanes, half-chunks per lane, rows per team, rows per tile
    int stages, tiles;
    uint32_t crb, srb;     // code / scale bytes per row
    uint32_t stage_bytes, scale_off;
    uint32_t x_off, bar_off;
};

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int FMT, int MT, int RW>
__global__ void __launch_bounds__(kGemvThreads)
gemv_kernel(const GemvParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hcpr = p.K >> 5;                       // half-chunks (32 weights) per row
    float* xs = reinterpret_cast<float*>(smem + p.x_off);   // [MT][8][hcpr] float4
    float* xsum = xs + (size_t)MT * p.K;                    // [MT][hcpr]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + p.stages;

    const int my_tiles = (int)blockIdx.x < p.tiles ? (p.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    grid_dep_launch();

    if (warp == kConsumerWarps) {                    // producer warp
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            for (int i = 0; i < my_tiles; ++i) {
                const int s = i % p.stages;
                if (i >= p.stages && !mbar_wait_bounded(&empty[s], ((i / p.stages) - 1) & 1, kStatusSlotWait))
                    break;
                const int n0 = ((int)blockIdx.x + i * (int)gridDim.x) * p.R;
                const int rows = min(p.R, p.N - n0);
                const uint32_t cb = (uint32_t)rows * p.crb;
                const uint32_t sb = p.srb ? (((uint32_t)rows * p.srb + 15u) & ~15u) : 0u;
                uint8_t* st = smem + (size_t)s * p.stage_bytes;
                mbar_arrive_expect_tx(&full[s], cb + sb);
                bulk_g2s(st, p.codes + (size_t)n0 * p.crb, cb, &full[s], pol);
                if (sb) bulk_g2s(st + p.scale_off, p.scales + (size_t)n0 * p.srb, sb, &full[s], pol);
            }
        }
        return;
    }

    // ---- consumers: stage x (it is written by the previous kernel) --------
    grid_dep_wait();
    for (int i = tid; i < MT * hcpr; i += kConsumerWarps * 32) {
        const int m = i / hcpr, h = i - m * hcpr;
        uint4 v[4] = {};
        if (m < p.mrows) {
            const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)(p.m0 + m) * p.K + (size_t)h * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = __ldg(src + j);
        }
        const uint32_t* w = reinterpret_cast<const uint32_t*>(v);  // 16 words = 32 bf16, natural order
        float4* dst = reinterpret_cast<float4*>(xs) + (size_t)m * 8 * hcpr + h;
        float sum = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float4 f;
            if (FMT == kFmtW8G16) {          // natural order: weights 4q..4q+3
                f = make_float4(bf_lo(w[2 * q]), bf_hi(w[2 * q]), bf_lo(w[2 * q + 1]), bf_hi(w[2 * q + 1]));
            } else {                          // int4 slot order: word q/2, even (q even) or odd weights
                const uint32_t* ww = w + 4 * (q >> 1);
                f = (q & 1) ? make_float4(bf_hi(ww[0]), bf_hi(ww[1]), bf_hi(ww[2]), bf_hi(ww[3]))
                            : make_float4(bf_lo(ww[0]), bf_lo(ww[1]), bf_lo(ww[2]), bf_lo(ww[3]));
            }
            dst[(size_t)q * hcpr] = f;
            sum += (f.x + f.y) + (f.z + f.w);
        }
        xsum[(size_t)m * hcpr + h] = sum;
    }
    asm volatile("bar.sync 1, %0;" :: "n"(kConsumerWarps * 32) : "memory");

    const int T = p.T;
    const int team = lane / T, li = lane - team * T;
    const int rbase = (warp * (32 / T) + team) * RW;
    bool ok = true;

    for (int it = 0; it < my_tiles; ++it) {
        const int s = it % p.stages;
        if (!mbar_wait_bounded(&full[s], (it / p.stages) & 1, kStatusTmaWait)) { ok = false; break; }
        const int n0 = ((int)blockIdx.x + it * (int)gridDim.x) * p.R;
        const int rows = min(p.R, p.N - n0);
        const uint8_t* st = smem + (size_t)s * p.stage_bytes;
        const uint8_t* ssc = st + p.scale_off;

        float yacc[RW][MT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) yacc[r][m] = 0.0f;

        for (int hj = 0; hj < p.HJ; ++hj) {
            const int h = li + T * hj;
            float xsm[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) xsm[m] = xsum[(size_t)m * hcpr + h];
            const float4* xq = reinterpret_cast<const float4*>(xs) + h;

            if (FMT == kFmtW8G16) {
                // 32 bytes per row: two uint4, words 0..3 = group 2h, 4..7 = group 2h+1
                uint4 c0[RW], c1[RW];
                float s0[RW], s1[RW];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const int rr = rbase + r;
                    if (rr < rows) {
                        const uint8_t* rowp = st + (size_t)rr * p.crb + (size_t)h * 32;
                        c0[r] = lds128(rowp);
                        c1[r] = lds128(rowp + 16);
                        const uint32_t sp = *reinterpret_cast<const uint32_t*>(ssc + (size_t)rr * p.srb + (size_t)h * 4);
                        s0[r] = __half2float(__ushort_as_half((unsigned short)(sp & 0xffffu)));
                        s1[r] = __half2float(__ushort_as_half((unsigned short)(sp >> 16)));
                    } else {
                        c0[r] = make_uint4(0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u);
                        c1[r] = c0[r];
                        s0[r] = s1[r] = 0.0f;
                    }
                }
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float acc[RW][MT];
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float4 xv[MT];
#pragma unroll
                        for (int m = 0; m < MT; ++m) xv[m] = xq[((size_t)m * 8 + g * 4 + i) * hcpr];
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            const uint4 c = g ? c1[r] : c0[r];
                            const uint32_t wd = i == 0 ? c.x : i == 1 ? c.y : i == 2 ? c.z : c.w;
                            float f[4];
                            unpack_w8(wd, f);
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                acc[r][m] = fmaf(f[0], xv[m].x, acc[r][m]);
                                acc[r][m] = fmaf(f[1], xv[m].y, acc[r][m]);
                                acc[r][m] = fmaf(f[2], xv[m].z, acc[r][m]);
                                acc[r][m] = fmaf(f[3], xv[m].w, acc[r][m]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int m = 0; m < MT; ++m) yacc[r][m] = fmaf(g ? s1[r] : s0[r], acc[r][m], yacc[r][m]);
                }
            } else {
                // int4: 16 bytes (32 nibbles) per row and half-chunk
                uint4 c[RW];
                float sA[RW], sB[RW];   // W4G64: (scale, -136 offset); SB32: (S, M)
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const int rr = rbase + r;
                    if (rr < rows) {
                        if (FMT == kFmtW4G64) {
                            c[r] = lds128(st + (size_t)rr * p.crb + (size_t)h * 16);
                            const uint16_t sc = *reinterpret_cast<const uint16_t*>(ssc + (size_t)rr * p.srb + (size_t)(h >> 1) * 2);
                            sA[r] = __half2float(__ushort_as_half(sc));
                            sB[r] = 0.0f;
                        } else {
                            const uint8_t* rec = st + (size_t)rr * p.crb + (size_t)(h >> 3) * 144;
                            const uint4 hd = lds128(rec);
                            c[r] = lds128(rec + 16 + (h & 7) * 16);
                            const int j = h & 7;
                            const float d = __half2float(__ushort_as_half((unsigned short)(hd.x & 0xffffu)));
                            const float dm = __half2float(__ushort_as_half((unsigned short)(hd.x >> 16)));
                            sA[r] = __fmul_rn(d, (float)sb_field(hd.y, hd.z, hd.w, 0, j));
                            sB[r] = __fmul_rn(dm, (float)sb_field(hd.y, hd.z, hd.w, 1, j));
                        }
                    } else {
                        c[r] = make_uint4(0u, 0u, 0u, 0u);
                        sA[r] = sB[r] = 0.0f;
                    }
                }
                float acc[RW][MT];
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float4 xa[MT], xb[MT];
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        xa[m] = xq[((size_t)m * 8 + 2 * i) * hcpr];
                        xb[m] = xq[((size_t)m * 8 + 2 * i + 1) * hcpr];
                    }
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        const uint32_t wd = i == 0 ? c[r].x : i == 1 ? c[r].y : i == 2 ? c[r].z : c[r].w;
                        float f[8];
                        unpack_w4(wd, f);
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            float a = acc[r][m];
                            a = fmaf(f[0], xa[m].x, a);
                            a = fmaf(f[1], xa[m].y, a);
                            a = fmaf(f[2], xa[m].z, a);
                            a = fmaf(f[3], xa[m].w, a);
                            a = fmaf(f[4], xb[m].x, a);
                            a = fmaf(f[5], xb[m].y, a);
                            a = fmaf(f[6], xb[m].z, a);
                            a = fmaf(f[7], xb[m].w, a);
                            acc[r][m] = a;
                        }
                    }
                }
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (FMT == kFmtW4G64) {
                            // s * (sum (128+u) x - 136 sum x) = s * sum q x
                            yacc[r][m] = fmaf(sA[r], fmaf(-136.0f, xsm[m], acc[r][m]), yacc[r][m]);
                        } else {
                            // S * (sum (128+q) x - 128 sum x) - M sum x
                            yacc[r][m] = fmaf(sA[r], fmaf(-128.0f, xsm[m], acc[r][m]), yacc[r][m]);
                            yacc[r][m] = fmaf(-sB[r], xsm[m], yacc[r][m]);
                        }
                    }
            }
        }
        // stage consumed: release it to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        // team reduction and store
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float v = yacc[r][m];
                for (int o = T >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                yacc[r][m] = v;
            }
        if (li == 0) {
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int rr = rbase + r;
                if (rr < rows)
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < p.mrows) p.y[(size_t)(p.m0 + m) * p.N + n0 + rr] = yacc[r][m];
            }
        }
    }
    (void)ok;
}

template <int FMT, int MT, int RW>
cudaError_t launch_one(const GemvParams& prm, size_t smem, int grid, cudaStream_t st) {
    auto kern = gemv_kernel<FMT, MT, RW>;
    // The attribute is per device; set it once per device (a race between
    // host threads only repeats the same idempotent call).
    static unsigned long long attr_done = 0ull;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_done, bit, __ATOMIC_RELEASE);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int FMT, int MT>
cudaError_t launch_rw(const GemvParams& prm, size_t smem, int grid, cudaStream_t st) {
    return prm.RW == 2 ? launch_one<FMT, MT, 2>(prm, smem, grid, st) : launch_one<FMT, MT, 1>(prm, smem, grid, st);
}

template <int FMT>
cudaError_t launch_mt(int MT, const GemvParams& prm, size_t smem, int grid, cudaStream_t st) {
    switch (MT) {
        case 4: return launch_rw<FMT, 4>(prm, smem, grid, st);
        case 2: return launch_rw<FMT, 2>(prm, smem, grid, st);
        default: return launch_rw<FMT, 1>(prm, smem, grid, st);
    }
}

constexpr size_t kSmemBudget = 220 * 1024;

}  // namespace

cudaError_t status_gemv(cudaStream_t st, unsigned* word) {
    unsigned v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *word = v;
    return e;
}

cudaError_t launch_gemv(const WgemmArgs& a, cudaStream_t st) {
    const int K = a.K, N = a.N;
    const int hcpr = K / 32;
    int T = 32;
    while (T > 1 && (hcpr % T) != 0) T >>= 1;
    const int teams = kConsumerWarps * (32 / T);
    const size_t crb = code_row_bytes(a.fmt, K), srb = scale_row_bytes(a.fmt, K);

    auto stage_bytes = [&](int R) { return round16((size_t)R * crb) + round16((size_t)R * srb); };
    const int RW = stage_bytes(teams * 2) <= 24 * 1024 ? 2 : 1;
    const int R = teams * RW;
    const size_t sb = stage_bytes(R);

    int MT = a.M >= 4 ? 4 : (a.M >= 2 ? 2 : 1);
    auto x_bytes = [&](int mt) { return (size_t)mt * K * 4 + (size_t)mt * hcpr * 4; };
    while (MT > 1 && x_bytes(MT) + 2 * sb > kSmemBudget) MT >>= 1;
    const size_t xb = x_bytes(MT);
    if (xb + 2 * sb + 64 > kSmemBudget) return cudaErrorInvalidValue;
    int stages = (int)((kSmemBudget - xb - 64) / sb);
    stages = stages > 4 ? 4 : stages;

    GemvParams p = {};
    p.x = static_cast<const uint16_t*>(a.x);
    p.codes = static_cast<const uint8_t*>(a.codes);
    p.scales = static_cast<const uint8_t*>(a.scales);
    p.y = a.y;
    p.K = K;
    p.N = N;
    p.T = T;
    p.HJ = hcpr / T;
    p.RW = RW;
    p.R = R;
    p.stages = stages;
    p.tiles = (N + R - 1) / R;
    p.crb = (uint32_t)crb;
    p.srb = (uint32_t)srb;
    p.stage_bytes = (uint32_t)sb;
    p.scale_off = (uint32_t)round16((size_t)R * crb);
    p.x_off = (uint32_t)(stages * sb);
    p.bar_off = (uint32_t)(p.x_off + xb);
    const size_t smem = p.bar_off + 2 * stages * sizeof(uint64_t);

    // CTAs resident per SM for this footprint (smem and threads), then one
    // wave of CTAs that loop over the tiles.
    int per_sm = (int)(228 * 1024 / (smem + 1024));
    per_sm = per_sm < 1 ? 1 : (per_sm > 2048 / kGemvThreads ? 2048 / kGemvThreads : per_sm);
    int grid = sm_count() * per_sm;
    if (grid > p.tiles) grid = p.tiles;

    for (int m0 = 0; m0 < a.M; m0 += MT) {
        p.m0 = m0;
        p.mrows = a.M - m0 < MT ? a.M - m0 : MT;
        cudaError_t e;
        switch (a.fmt) {
            case kFmtW4G64: e = launch_mt<kFmtW4G64>(MT, p, smem, grid, st); break;
            case kFmtW8G16: e = launch_mt<kFmtW8G16>(MT, p, smem, grid, st); break;
            default: e = launch_mt<kFmtW4SB32>(MT, p, smem, grid, st); break;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace rq
