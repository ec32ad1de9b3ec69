// rq_gemv.cu -- the memory-bound product y = x * w_hat^T for a few activation
// rows (decode), with w_hat formed in registers; one launch may carry a batch
// of independent products (e.g. the r, k, v projections of a layer).
//
// Sources: RWKV-7 G1 1.5B int4 model card, summary paragraph: decode is
// served by a hand-written int4 GEMV / small-M GEMM family and the kernel
// output is bit-identical to the offline dequantization. rwkv-quant article,
// "Two presets and six sizes": the int8 group-16 and int4 superblock formats.
// rwkv_quant_nv project description, "Operator Optimization Details": the
// r/k/v projections computed in a single kernel.
//
// Design (B200):
//  * The products of a launch are laid end to end on one axis of packed
//    bytes; CTA c (one per SM) owns a contiguous, balanced stretch of it, i.e.
//    contiguous row ranges of one or a few products. Codes and scales of
//    consecutive rows are contiguous in HBM, so a group of rows is one
//    untiled bulk-async copy per plane into a shared-memory stage, completed
//    on an mbarrier. A producer warp keeps the ring full, starting before
//    griddepcontrol.wait: with programmatic dependent launch the weights
//    stream in while the previous kernel finishes.
//  * After the wait, each product's x is staged in shared memory, interleaved
//    by 16-byte quads so that lanes reading consecutive half-chunks (32
//    weights) hit consecutive banks. For int4, x is held as fp16 under a
//    power-of-two scale per half-chunk, with the half-chunk's offset sums.
//  * A team of T lanes (a power of two dividing K/32) owns RW rows of a group;
//    lane i takes half-chunks i, i+T, ... of those rows; long rows are split
//    over KS warps whose partial sums meet in shared memory.
//    int4: a lop3 with mask and exponent pattern turns two nibbles into an
//    fp16 pair ((1024 + u), or (1024 + 16 u) for the upper nibble of a byte),
//    one shift and four lop3 per eight weights, multiplied by the fp16 x with
//    fp32-accumulating fma.rn.f32.f16; scale and code offset are applied once
//    per half-chunk:  sum_k (u_k - 8) x_k s = s f (lo + hi / 16 - z).
//    int8: a byte permute places each code under an fp32 exponent (32768 + u),
//    one subtraction gives q exactly, fp32 fma with fp32 x.
//  * Team partial sums are reduced with warp shuffles; one store per output.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_device.cuh"
#include "rq_internal.h"

// Phase marks for external profiling builds; no code in this library.
#ifndef RQ_PHASE_MARK
#define RQ_PHASE_MARK(i)
#endif

namespace rq {
namespace {

#ifndef RQ_GEMV_WARPS
#define RQ_GEMV_WARPS 8
#endif
constexpr int kConsumerWarps = RQ_GEMV_WARPS;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

struct Item {                  // one product of a launch
    const uint16_t* x;         // bf16 bits [M][K]
    const uint8_t* codes;
    const uint8_t* scales;
    float* y;                  // fp32 [M][N]
    long long cost0;           // packed bytes of the items before this one
    long long cost1;           // cost0 + this item's packed bytes
    int K, N;
    int T, HJ;                 // team lanes, half-chunks per lane and warp
    int KS;                    // warps sharing a row (each takes HJ * T consecutive half-chunk slots)
    int RW, Rg;                // rows per team, rows per group (a multiple of rho)
    int rho;                   // rows per unit; a unit is the grain of the CTA split
    uint32_t crb, srb;         // code / scale bytes per row
    uint32_t ucost;            // bytes of one unit (rho rows of both planes)
};

template <int MAXI>
struct Batch {
    int count, m0, mrows;      // items; activation rows [m0, m0 + mrows) of every item
    int stages;
    long long total;           // packed bytes of all items
    uint32_t stage_bytes, x_off, xmeta_off, red_off, red_bytes, bar_off;
    Item it[MAXI];
};

// Units [ua, ub) of item `it` that start inside the cost range [lo, hi).
__device__ __forceinline__ void item_units(const Item& it, long long lo, long long hi, int& ua, int& ub) {
    const long long U = (it.N + it.rho - 1) / it.rho;
    auto first_at_or_after = [&](long long c) -> long long {
        const long long d = c - it.cost0;
        if (d <= 0) return 0;
        const long long u = (d + it.ucost - 1) / it.ucost;
        return u < U ? u : U;
    };
    ua = (int)first_at_or_after(lo);
    ub = (int)first_at_or_after(hi);
}

// Bytes of the x metadata of the int4 formats for K and MT activation rows:
// per row m and half-chunk h a float2 {z, sx}, then the per-row factors f[m],
// then a word per consumer warp and row for the max reduction.
__host__ __device__ constexpr size_t xmeta_bytes(int K, int MT) {
    return (size_t)MT * (K / 32) * 8 + 16 + (size_t)kConsumerWarps * MT * 4;
}

// Staged x for one product and activation rows [m0, m0 + MT).
//  int4 formats: fp16 quads in natural order (quad q = x[8q .. 8q+7]); row m
//  scaled by the power of two 2^e_m that puts its largest |x| in [2^14, 2^15)
//  (exact for every value no more than 2^32 times smaller than the largest),
//  with f[m] = 2^-e_m and per half-chunk h: sx = the sum of the scaled values,
//  z = the code offsets' share (g64: 1032 * sum over even k + 72 * sum over
//  odd k; sb32: 1024 / 64), both summed from the fp16 values the products use.
//  int8 format: fp32 quads (quad q = x[4q .. 4q+3]).
// Called by all consumer threads; contains consumer barriers.
template <int FMT, int MT>
__device__ __forceinline__ void stage_x(const Item& it, int m0, int mrows, uint8_t* xbuf, uint8_t* xmeta, int tid) {
    constexpr bool kW4 = FMT != kFmtW8G16;
    constexpr int kT = kConsumerWarps * 32;
    const int hcpr = it.K >> 5;
    auto load = [&](int m, int h, uint4 (&v)[4]) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = make_uint4(0u, 0u, 0u, 0u);
        if (m < mrows) {
            const uint4* src = reinterpret_cast<const uint4*>(it.x + (size_t)(m0 + m) * it.K + (size_t)h * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = __ldg(src + j);
        }
    };
    if constexpr (kW4) {
        float2* zx = reinterpret_cast<float2*>(xmeta);
        float* fm = reinterpret_cast<float*>(xmeta + (size_t)MT * hcpr * 8);
        uint32_t* wmax = reinterpret_cast<uint32_t*>(xmeta + (size_t)MT * hcpr * 8 + 16);
        // largest |x| bit pattern of each row (bf16 magnitudes order as integers)
        uint32_t mb[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) mb[m] = 0u;
        for (int i = tid; i < MT * hcpr; i += kT) {
            const int m = i / hcpr, h = i - m * hcpr;
            uint4 v[4];
            load(m, h, v);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(v);
            uint32_t t = 0u;
#pragma unroll
            for (int j = 0; j < 16; ++j) t = max(t, max(w[j] & 0x7fffu, (w[j] >> 16) & 0x7fffu));
#pragma unroll
            for (int mm = 0; mm < MT; ++mm)
                if (mm == m) mb[mm] = max(mb[mm], t);
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint32_t r = __reduce_max_sync(0xffffffffu, mb[m]);
            if ((tid & 31) == 0) wmax[(tid >> 5) * MT + m] = r;
        }
        asm volatile("bar.sync 1, %0;" :: "n"(kT) : "memory");
        float up[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            uint32_t r = 0u;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) r = max(r, wmax[w * MT + m]);
            const int e = r != 0u ? min(126, max(-126, 14 - ((int)(r >> 7) - 127))) : 0;
            up[m] = __int_as_float((e + 127) << 23);
            if (tid == 0) fm[m] = __int_as_float((127 - e) << 23);
        }
        for (int i = tid; i < MT * hcpr; i += kT) {
            const int m = i / hcpr, h = i - m * hcpr;
            uint4 v[4];
            load(m, h, v);
            uint32_t* w = reinterpret_cast<uint32_t*>(v);
            float u = up[0];
#pragma unroll
            for (int mm = 1; mm < MT; ++mm)
                if (mm == m) u = up[mm];
            float se = 0.0f, so = 0.0f;                  // even-k and odd-k sums
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const __half a = __float2half_rn(__fmul_rn(bf16lo_f32(w[j]), u));
                const __half b = __float2half_rn(__fmul_rn(bf16hi_f32(w[j]), u));
                se = __fadd_rn(se, __half2float(a));
                so = __fadd_rn(so, __half2float(b));
                w[j] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
            }
            uint4* dst = reinterpret_cast<uint4*>(xbuf) + (size_t)m * 4 * hcpr + h;
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[(size_t)q * hcpr] = v[q];
            const float z = FMT == kFmtW4G64 ? __fmaf_rn(1032.0f, se, __fmul_rn(72.0f, so))
                                             : __fmaf_rn(1024.0f, se, __fmul_rn(64.0f, so));
            zx[(size_t)m * hcpr + h] = make_float2(z, __fadd_rn(se, so));
        }
    } else {
        for (int i = tid; i < MT * hcpr; i += kT) {
            const int m = i / hcpr, h = i - m * hcpr;
            uint4 v[4];
            load(m, h, v);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(v);
            float4* dst = reinterpret_cast<float4*>(xbuf) + (size_t)m * 8 * hcpr + h;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[(size_t)q * hcpr] = make_float4(bf16lo_f32(w[2 * q]), bf16hi_f32(w[2 * q]),
                                                    bf16lo_f32(w[2 * q + 1]), bf16hi_f32(w[2 * q + 1]));
        }
    }
}

__device__ __forceinline__ uint32_t word_of(const uint4& c, int i) {
    return i == 0 ? c.x : i == 1 ? c.y : i == 2 ? c.z : c.w;
}

// One group of rows of item `it` in the stage at shared address st_s: this
// team's rows rbase .. rbase + RW - 1 of the group; writes their outputs.
// Rows past rg (the group's last rows) lie inside the stage buffer, which
// always has room for Rg rows; they hold stale bytes whose results are never
// stored.
template <int FMT, int MT, int RW>
__device__ __forceinline__ void gemv_group(const Item& it, uint32_t st_s, int g0, int rg, uint32_t x_s,
                                           uint32_t xmeta_s, int m0, int mrows, int lane, int rbase, int slice,
                                           float* red) {
    constexpr bool kW4 = FMT != kFmtW8G16;
    constexpr int U = RW == 1 ? 2 : 1;                   // half-chunks per iteration
    const int hcpr = it.K >> 5, T = it.T, HJ = it.HJ;
    const int li = lane & (T - 1);
    const int hoff = slice * HJ;                         // this warp's k-slice of the row
    const uint32_t crb = it.crb, srb = it.srb;
    const uint32_t ssc_s = st_s + (uint32_t)round16((size_t)it.Rg * crb);
    // x quads: (m * Q + q) * hcpr + h, Q = 4 (bf16) or 8 (fp32) quads per half-chunk
    const uint32_t xstride = (uint32_t)hcpr * 16u;
    const uint32_t xa0 = x_s + (uint32_t)li * 16u;
    const uint32_t xm0 = xmeta_s + (uint32_t)li * 8u;
    float yacc[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[r][m] = 0.0f;

    if (kW4) {
        // W4G64: codes at row * crb + h * 16, scale at (h / 2) * 2.
        // W4SB32: record at row * crb + (h / 8) * 144; T is a multiple of 8
        // (K % 256 == 0), so a lane always sees the same group j = li % 8.
        const int j = li & 7;
        uint32_t ca[RW], sa[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            if (FMT == kFmtW4G64) {
                ca[r] = st_s + (uint32_t)(rbase + r) * crb + (uint32_t)li * 16u;
                sa[r] = ssc_s + (uint32_t)(rbase + r) * srb + (uint32_t)(li >> 1) * 2u;
            } else {
                ca[r] = st_s + (uint32_t)(rbase + r) * crb + (uint32_t)(li >> 3) * 144u;
                sa[r] = 0u;
            }
        }
        for (int hj = 0; hj < HJ; hj += U) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (u > 0 && hj + u >= HJ) break;
                const uint32_t dh = (uint32_t)(hoff + hj + u) * (uint32_t)T;
                float2 xm[MT];                           // {z, sx}
#pragma unroll
                for (int m = 0; m < MT; ++m) xm[m] = lds64f_a(xm0 + ((uint32_t)m * (uint32_t)hcpr + dh) * 8u);
                uint4 c[RW];
                float sA[RW], sB[RW];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    if (FMT == kFmtW4G64) {
                        c[r] = lds128_a(ca[r] + dh * 16u);
                        sA[r] = __half2float(__ushort_as_half((unsigned short)lds16_a(sa[r] + dh)));
                        sB[r] = 0.0f;
                    } else {
                        const uint32_t rec = ca[r] + (dh >> 3) * 144u;
                        const uint4 hd = lds128_a(rec);
                        c[r] = lds128_a(rec + 16u + (uint32_t)j * 16u);
                        const float d = __half2float(__ushort_as_half((unsigned short)(hd.x & 0xffffu)));
                        const float dm = __half2float(__ushort_as_half((unsigned short)(hd.x >> 16)));
                        sA[r] = __fmul_rn(d, (float)sb_field(hd.y, hd.z, hd.w, 0, j));
                        sB[r] = __fmul_rn(dm, (float)sb_field(hd.y, hd.z, hd.w, 1, j));
                    }
                }
                // one accumulator for even k ((1024 + u) x), started at -z, and
                // one for odd k ((1024 + 16 u) x) per row and m, whatever the
                // launch shape, so a row's sums do not depend on RW or batching
                float lo[RW][MT], hi[RW][MT];
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        lo[r][m] = -xm[m].x;
                        hi[r][m] = 0.0f;
                    }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint4 X = lds128_a(xa0 + dh * 16u + (uint32_t)(m * 4 + i) * xstride);
#pragma unroll
                        for (int r = 0; r < RW; ++r) dot8_w4_f16(word_of(c[r], i), X, lo[r][m], hi[r][m]);
                    }
                }
                // sum_k q_k x'_k (g64) or sum_k u_k x'_k (sb32) = lo + hi / 16
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float a = __fmaf_rn(hi[r][m], 0.0625f, lo[r][m]);
                        yacc[r][m] = __fmaf_rn(sA[r], a, yacc[r][m]);
                        if (FMT == kFmtW4SB32) yacc[r][m] = __fmaf_rn(-sB[r], xm[m].y, yacc[r][m]);
                    }
            }
        }
        // back from the scaled x domain: y = f[m] * sum
        const uint32_t f_s = xmeta_s + (uint32_t)(MT * hcpr * 8);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float f = ldsf_a(f_s + (uint32_t)m * 4u);
#pragma unroll
            for (int r = 0; r < RW; ++r) yacc[r][m] = __fmul_rn(yacc[r][m], f);
        }
    } else {
        // int8 group 16: 32 code bytes per row and half-chunk = groups 2h, 2h+1;
        // x as fp32 quads, 8 per half-chunk
        uint32_t ca[RW], sa[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            ca[r] = st_s + (uint32_t)(rbase + r) * crb + (uint32_t)li * 32u;
            sa[r] = ssc_s + (uint32_t)(rbase + r) * srb + (uint32_t)li * 4u;
        }
        for (int hj = 0; hj < HJ; hj += U) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (u > 0 && hj + u >= HJ) break;
                const uint32_t dh = (uint32_t)(hoff + hj + u) * (uint32_t)T;
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const uint4 c0 = lds128_a(ca[r] + dh * 32u);
                    const uint4 c1 = lds128_a(ca[r] + dh * 32u + 16u);
                    const uint32_t sp = lds32_a(sa[r] + dh * 4u);
                    const float s0 = __half2float(__ushort_as_half((unsigned short)(sp & 0xffffu)));
                    const float s1 = __half2float(__ushort_as_half((unsigned short)(sp >> 16)));
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float a[MT];
#pragma unroll
                        for (int m = 0; m < MT; ++m) a[m] = 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            float f[4];
                            unpack_w8(word_of(g ? c1 : c0, i), f);
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                const float4 xv = lds128f_a(xa0 + dh * 16u + (uint32_t)(m * 8 + g * 4 + i) * xstride);
                                a[m] = fmaf(f[0], xv.x, a[m]);
                                a[m] = fmaf(f[1], xv.y, a[m]);
                                a[m] = fmaf(f[2], xv.z, a[m]);
                                a[m] = fmaf(f[3], xv.w, a[m]);
                            }
                        }
#pragma unroll
                        for (int m = 0; m < MT; ++m) yacc[r][m] = fmaf(g ? s1 : s0, a[m], yacc[r][m]);
                    }
                }
            }
        }
    }
    if (T == 32 && RW == 4) {
        // Recursive halving over the warp: after the offset-16 step lanes 0-15
        // hold rows {0,1} and lanes 16-31 rows {2,3}; after offset 8 each lane
        // holds one row (lane bits 4..3); three more steps finish the sum, so
        // lane 8r holds row r.
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const bool up16 = (lane & 16) != 0;
            float a0 = up16 ? yacc[2 % RW][m] : yacc[0][m], a1 = up16 ? yacc[3 % RW][m] : yacc[1 % RW][m];
            const float give0 = up16 ? yacc[0][m] : yacc[2 % RW][m], give1 = up16 ? yacc[1 % RW][m] : yacc[3 % RW][m];
            a0 += __shfl_xor_sync(0xffffffffu, give0, 16);
            a1 += __shfl_xor_sync(0xffffffffu, give1, 16);
            const bool up8 = (lane & 8) != 0;
            float v = up8 ? a1 : a0;
            v += __shfl_xor_sync(0xffffffffu, up8 ? a0 : a1, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            const int r = lane >> 3;                     // row of this lane's sum
            const int rr = rbase + r;
            if ((lane & 7) == 0 && rr < rg) {
                if (it.KS > 1) red[((size_t)rr * MT + m) * it.KS + slice] = v;
                else if (m < mrows) it.y[(size_t)(m0 + m) * it.N + g0 + rr] = v;
            }
        }
        return;
    }
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
            if (rr < rg)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (it.KS > 1) red[((size_t)rr * MT + m) * it.KS + slice] = yacc[r][m];
                    else if (m < mrows) it.y[(size_t)(m0 + m) * it.N + g0 + rr] = yacc[r][m];
                }
        }
    }
}

// Resident CTAs per SM the register budget is sized for.
constexpr int min_blocks(int mt) {
    return kConsumerWarps <= 8 ? (mt == 1 ? 3 : 2) : (kConsumerWarps <= 12 ? 2 : 1);
}

template <int FMT, int MT, int MAXI>
__global__ void __launch_bounds__(kThreads, min_blocks(MT))
gemv_kernel(const Batch<MAXI> p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + p.stages;
    uint8_t* xbuf = smem + p.x_off;
    uint8_t* xmeta = smem + p.xmeta_off;
    const long long lo = (long long)blockIdx.x * p.total / gridDim.x;
    const long long hi = (long long)(blockIdx.x + 1) * p.total / gridDim.x;

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    grid_dep_launch();
    RQ_PHASE_MARK(0);

    if (warp == kConsumerWarps) {                        // producer warp
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            int gi = 0;
            bool ok = true;
            for (int i = 0; i < p.count && ok; ++i) {
                const Item& it = p.it[i];
                if (it.cost0 >= hi) break;               // items are in cost order
                if (it.cost1 <= lo) continue;            // no overlap: skip without dividing
                int ua, ub;
                item_units(it, lo, hi, ua, ub);
                const int ra = ua * it.rho, rb = min(ub * it.rho, it.N);
                for (int g0 = ra; g0 < rb; g0 += it.Rg, ++gi) {
                    const int s = gi % p.stages;
                    if (gi >= p.stages && !mbar_wait_bounded(&empty[s], ((gi / p.stages) - 1) & 1, kStatusSlotWait)) {
                        ok = false;
                        break;
                    }
                    const int rg = min(it.Rg, rb - g0);
                    const uint32_t cb = (uint32_t)rg * it.crb;
                    const uint32_t sb = it.srb ? (((uint32_t)rg * it.srb + 15u) & ~15u) : 0u;
                    uint8_t* st = smem + (size_t)s * p.stage_bytes;
                    mbar_arrive_expect_tx(&full[s], cb + sb);
                    bulk_g2s(st, it.codes + (size_t)g0 * it.crb, cb, &full[s], pol);
                    if (sb)
                        bulk_g2s(st + round16((size_t)it.Rg * it.crb), it.scales + (size_t)g0 * it.srb, sb, &full[s], pol);
                }
            }
        }
        return;
    }

    // ---- consumers ---------------------------------------------------------
    const uint32_t smem_s = smem_u32(smem);
    grid_dep_wait();                                     // x is written by the previous kernel
    RQ_PHASE_MARK(1);
    int gi = 0;
    bool first = true;
    for (int i = 0; i < p.count; ++i) {
        const Item& it = p.it[i];
        if (it.cost0 >= hi) break;                       // items are in cost order
        if (it.cost1 <= lo) continue;                    // no overlap: skip without dividing
        int ua, ub;
        item_units(it, lo, hi, ua, ub);
        const int ra = ua * it.rho, rb = min(ub * it.rho, it.N);
        if (ra >= rb) continue;
        if (!first) asm volatile("bar.sync 1, %0;" :: "n"(kConsumerWarps * 32) : "memory");
        first = false;
        stage_x<FMT, MT>(it, p.m0, p.mrows, xbuf, xmeta, tid);
        asm volatile("bar.sync 1, %0;" :: "n"(kConsumerWarps * 32) : "memory");
        RQ_PHASE_MARK(2);
        const int T = it.T, RW = it.RW, KS = it.KS;
        const int slice = warp % KS;                     // k-slice of this warp (KS > 1 only when T == 32)
        const int wteam = (warp / KS) * (32 / T);         // first team of this warp
        const int rbase = (wteam + lane / T) * RW;        // first row of this team in a group
        const int wfirst = wteam * RW;                    // first row of this warp in a group
        for (int g0 = ra; g0 < rb; g0 += it.Rg, ++gi) {
            const int s = gi % p.stages;
            if (!mbar_wait_bounded(&full[s], (gi / p.stages) & 1, kStatusTmaWait)) return;
            RQ_PHASE_MARK(3);
            const int rg = min(it.Rg, rb - g0);
            float* red = reinterpret_cast<float*>(smem + p.red_off + (gi & 1) * p.red_bytes);
            if (wfirst < rg) {                           // warp-uniform
                const uint32_t st_s = smem_s + (uint32_t)s * p.stage_bytes;
                if (RW == 4)
                    gemv_group<FMT, MT, 4>(it, st_s, g0, rg, smem_s + p.x_off, smem_s + p.xmeta_off, p.m0, p.mrows,
                                           lane, rbase, slice, red);
                else if (RW == 2)
                    gemv_group<FMT, MT, 2>(it, st_s, g0, rg, smem_s + p.x_off, smem_s + p.xmeta_off, p.m0, p.mrows,
                                           lane, rbase, slice, red);
                else
                    gemv_group<FMT, MT, 1>(it, st_s, g0, rg, smem_s + p.x_off, smem_s + p.xmeta_off, p.m0, p.mrows,
                                           lane, rbase, slice, red);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);       // stage consumed
            if (KS > 1) {                                // combine the k-slices of each row
                asm volatile("bar.sync 1, %0;" :: "n"(kConsumerWarps * 32) : "memory");
                for (int t = tid; t < rg * MT; t += kConsumerWarps * 32) {
                    const int rr = t / MT, m = t - rr * MT;
                    float v = 0.0f;
                    for (int k = 0; k < KS; ++k) v += red[(size_t)t * KS + k];
                    if (m < p.mrows) it.y[(size_t)(p.m0 + m) * it.N + g0 + rr] = v;
                }
            }
        }
    }
    RQ_PHASE_MARK(4);
}

// Shared-memory target per CTA for single products: three CTAs (three kernels
// of a dependent chain) fit on one SM. Batches run two CTAs per SM.
#ifndef RQ_GEMV_SINGLE_CTAS_PER_SM
#define RQ_GEMV_SINGLE_CTAS_PER_SM 1
#endif
#ifndef RQ_GEMV_BATCH_CTAS_PER_SM
#define RQ_GEMV_BATCH_CTAS_PER_SM 2
#endif
constexpr size_t kSmemTarget = 72 * 1024;
#ifndef RQ_GEMV_SMEM_BATCH_KB
#define RQ_GEMV_SMEM_BATCH_KB 100
#endif
constexpr size_t kSmemBatch = RQ_GEMV_SMEM_BATCH_KB * 1024;
constexpr size_t kSmemLimit = 220 * 1024;
constexpr size_t kSmemAttr = kSmemLimit + 1024;

template <int FMT, int MT, int MAXI>
cudaError_t launch_one(const Batch<MAXI>& prm, size_t smem, int grid, cudaStream_t st) {
    auto kern = gemv_kernel<FMT, MT, MAXI>;
    // The attribute is per device; set it once per device (a race between
    // host threads only repeats the same idempotent call).
    static unsigned long long attr_done = 0ull;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAttr);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_done, bit, __ATOMIC_RELEASE);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

// Lane and warp layout of a product's rows: T lanes per team (a power of two
// dividing K/32), KS warps per row (when T == 32, long rows are split so that
// each warp covers about two half-chunks per lane), HJ half-chunks per lane.
struct Layout { int T, KS, HJ, teams; };
Layout layout_of(int K) {
    const int hcpr = K / 32;
    Layout l;
    l.T = 32;
    while (l.T > 1 && (hcpr % l.T) != 0) l.T >>= 1;
    const int hj_all = hcpr / l.T;
    l.KS = 1;
    while (l.T == 32 && kConsumerWarps % (l.KS * 2) == 0 && hj_all % (l.KS * 2) == 0 && hj_all / (l.KS * 2) >= 2)
        l.KS *= 2;
    l.HJ = hj_all / l.KS;
    l.teams = (kConsumerWarps / l.KS) * (32 / l.T);
    return l;
}

// Rows per team for a product: the largest of 4, 2, 1 whose group of
// teams * RW rows stays within 48 KB.
int rw_allowed(int fmt, int K) {
    const Layout l = layout_of(K);
    auto sb = [&](size_t R) { return round16(R * code_row_bytes(fmt, K)) + round16(R * scale_row_bytes(fmt, K)); };
    if (sb((size_t)l.teams * 4) <= 48 * 1024) return 4;
    return sb((size_t)l.teams * 2) <= 48 * 1024 ? 2 : 1;
}

// Per-item launch geometry for rows-per-team RW; false for a shape that does
// not fit.
bool plan_item(int fmt, int K, int N, int MT, int RW, Item& it, size_t& stage_b, size_t& x_b) {
    const bool w4 = fmt != kFmtW8G16;
    const Layout l = layout_of(K);
    const size_t crb = code_row_bytes(fmt, K), srb = scale_row_bytes(fmt, K);
    int rho = 1;
    while (((size_t)rho * srb) % 16 != 0) rho <<= 1;     // srb is even, so rho <= 8
    auto stage_bytes = [&](int R) { return round16((size_t)R * crb) + round16((size_t)R * srb); };
    x_b = (size_t)MT * K * (w4 ? 2 : 4) + (w4 ? round16(xmeta_bytes(K, MT)) : 0);
    int Rg = l.teams * RW;
    while (Rg > rho && Rg > RW && x_b + 2 * stage_bytes(Rg) + 64 > kSmemLimit) Rg >>= 1;
    if (Rg % rho != 0 || x_b + stage_bytes(Rg) + 64 > kSmemLimit) return false;
    it.K = K;
    it.N = N;
    it.T = l.T;
    it.HJ = l.HJ;
    it.KS = l.KS;
    it.RW = RW;
    it.Rg = Rg;
    it.rho = rho;
    it.crb = (uint32_t)crb;
    it.srb = (uint32_t)srb;
    it.ucost = (uint32_t)((size_t)rho * (crb + srb));
    stage_b = stage_bytes(Rg);
    return true;
}

template <int FMT, int MAXI>
cudaError_t launch_batch(const WgemmArgs* a, int count, cudaStream_t st) {
    const int M = a[0].M;
    const int MT = M >= 2 ? 2 : 1;
    Batch<MAXI> p = {};
    p.count = count;
    size_t sb = 0, xq = 0, xs = 0, red = 0;
    long long total = 0, units_min = -1;
    for (int i = 0; i < count; ++i) {
        Item& it = p.it[i];
        size_t s1, x1;
        if (!plan_item(FMT, a[i].K, a[i].N, MT, rw_allowed(FMT, a[i].K), it, s1, x1)) return cudaErrorInvalidValue;
        it.x = static_cast<const uint16_t*>(a[i].x);
        it.codes = static_cast<const uint8_t*>(a[i].codes);
        it.scales = static_cast<const uint8_t*>(a[i].scales);
        it.y = a[i].y;
        it.cost0 = total;
        const long long U = (it.N + it.rho - 1) / it.rho;
        total += U * it.ucost;
        it.cost1 = total;
        units_min = units_min < 0 || U < units_min ? U : units_min;
        sb = s1 > sb ? s1 : sb;
        const size_t q = (size_t)MT * a[i].K * (FMT != kFmtW8G16 ? 2 : 4);
        xq = q > xq ? q : xq;
        if constexpr (FMT != kFmtW8G16) {                // x metadata, int4 formats
            const size_t s = round16(xmeta_bytes(a[i].K, MT));
            xs = s > xs ? s : xs;
        }
        const size_t rd = it.KS > 1 ? round16((size_t)it.Rg * MT * it.KS * 4) : 0;
        red = rd > red ? rd : red;
    }
    p.total = total;
    int grid = sm_count() * (count > 1 ? RQ_GEMV_BATCH_CTAS_PER_SM : RQ_GEMV_SINGLE_CTAS_PER_SM);
    if (count == 1 && grid > units_min) grid = (int)units_min;
    const size_t fixed = xq + xs + 2 * red + 64;
    const size_t want = count > 1 ? kSmemBatch : kSmemTarget;
    const size_t budget = fixed + 2 * sb <= want ? want : kSmemLimit;
    int stages = (int)((budget - fixed) / sb);
    if (stages > 6) stages = 6;
    if (count == 1) {   // a single product needs no more stages than its largest CTA has groups
        const Item& it = p.it[0];
        const long long per = (units_min + grid - 1) / grid * it.rho;
        const int gmax = (int)((per + it.Rg - 1) / it.Rg);
        if (stages > gmax) stages = gmax;
    }
    if (stages < 1) return cudaErrorInvalidValue;
    p.stages = stages;
    p.stage_bytes = (uint32_t)sb;
    p.x_off = (uint32_t)(stages * sb);
    p.xmeta_off = (uint32_t)(p.x_off + xq);
    p.red_off = (uint32_t)round16(p.xmeta_off + xs);
    p.red_bytes = (uint32_t)red;
    p.bar_off = (uint32_t)round16(p.red_off + 2 * red);
    const size_t smem = p.bar_off + 2 * stages * sizeof(uint64_t);
    if (smem > kSmemAttr) return cudaErrorInvalidValue;

    for (int m0 = 0; m0 < M; m0 += MT) {
        p.m0 = m0;
        p.mrows = M - m0 < MT ? M - m0 : MT;
        const cudaError_t e = MT == 2 ? launch_one<FMT, 2, MAXI>(p, smem, grid, st)
                                      : launch_one<FMT, 1, MAXI>(p, smem, grid, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int FMT>
cudaError_t launch_fmt(const WgemmArgs* a, int count, cudaStream_t st) {
    return count == 1 ? launch_batch<FMT, 1>(a, count, st) : launch_batch<FMT, kMaxBatch>(a, count, st);
}

}  // namespace

cudaError_t status_gemv(cudaStream_t st, unsigned* word) {
    unsigned v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *word = v;
    return e;
}

cudaError_t launch_gemv(const WgemmArgs* a, int count, cudaStream_t st) {
    switch (a[0].fmt) {
        case kFmtW4G64: return launch_fmt<kFmtW4G64>(a, count, st);
        case kFmtW8G16: return launch_fmt<kFmtW8G16>(a, count, st);
        default: return launch_fmt<kFmtW4SB32>(a, count, st);
    }
}

}  // namespace rq
