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

namespace rq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kProducerWarp = kConsumerWarps;         // issues the weight copies
constexpr int kStagerWarp = kConsumerWarps + 1;       // stages x
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr unsigned kProducerNapNs = 256;                  // poll interval of the producer's slot waits
constexpr unsigned kStagerNapNs = 512;                   // and of the x stager's buffer waits

struct Item {                  // one product of a launch
    const uint16_t* x;         // bf16 bits [M][K]
    const uint8_t* codes;
    const uint8_t* scales;
    void* y;                   // fp32 [M][N], or bf16 (the kernel's YB)
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
    int nxb;                   // staged-x buffers (2, or 1 when two do not fit)
    long long total;           // packed bytes of all items
    uint32_t stage_bytes;      // weight ring: stages * stage_bytes at offset 0
    uint32_t x_off, x_bytes;   // nxb staged-x buffers (x, then its metadata)
    uint32_t red_off, red_bytes;  // per stage: k-slice partial sums
    uint32_t bar_off;          // full[stages], empty[stages], xfull[2], xempty[2]
    unsigned long long wait_ns;  // bound of every device wait
    int test_flags;            // kTestNoCopies: the producer issues no copies (tests the waits)
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

// Bytes of one staged-x buffer for K and MT activation rows: the values
// (fp16 for the int4 formats, fp32 for int8), then for the int4 formats a
// metadata record per row m and half-chunk h (g64: float2, sb32: float4).
__host__ __device__ constexpr size_t xvals_bytes(int fmt, int K, int MT) {
    return (size_t)MT * K * (!is_w8(fmt) ? 2 : 4);
}
__host__ __device__ constexpr size_t xbuf_bytes(int fmt, int K, int MT) {
    return xvals_bytes(fmt, K, MT) + (size_t)MT * (fmt == kFmtW4G64 ? (K / 64) * 8 : fmt == kFmtW4SB32 ? (K / 32) * 16 : 0);
}

// Stages x for one product and activation rows [m0, m0 + MT); the calling
// threads split it, thread `first` of `stride` taking units first,
// first + stride, ... (a unit is 64 values for g64, 32 otherwise).
//  int4 formats: fp16 quads in natural order (quad q = x[8q .. 8q+7]), each
//  half-chunk h (32 values) scaled by the power of two 2^e_h that puts its
//  largest |x| in [2^14, 2^15) (exact for every value no more than 2^32 times
//  smaller than the largest), and per half-chunk f = 2^-e_h and
//  z = the code offsets' share (g64: 1032 * sum over even k + 72 * sum over
//  odd k; sb32: 1024 / 64), summed from the fp16 values the products use;
//  g64 keeps {z, f}, sb32 {z, f * sum, f, 0}.
//  int8 format: fp32 quads (quad q = x[4q .. 4q+3]).
// First item whose cost range ends after lo (binary search: items are in
// cost order), or count.
template <int MAXI>
__device__ __forceinline__ int item_after(const Batch<MAXI>& p, long long lo) {
    int a = 0, b = p.count;
    while (a < b) {
        const int c = (a + b) >> 1;
        if (p.it[c].cost1 <= lo) a = c + 1;
        else b = c;
    }
    return a;
}

// Index of the first item with rows in the cost range [lo, hi), or -1.
template <int MAXI>
__device__ __forceinline__ int first_item(const Batch<MAXI>& p, long long lo, long long hi) {
    for (int i = item_after(p, lo); i < p.count; ++i) {
        const Item& it = p.it[i];
        if (it.cost0 >= hi) break;
        int ua, ub;
        item_units(it, lo, hi, ua, ub);
        if (ua * it.rho < min(ub * it.rho, it.N)) return i;
    }
    return -1;
}

// Named barriers: 1 .. kConsumerWarps (k-slice teams), kCoopBarrier (the
// consumers and the stager after staging a CTA's first item).
constexpr int kCoopBarrier = 15;

// g64 unit sums: the even-k and odd-k fp32 sums of a 64-value unit are formed
// in one fixed order whichever threads stage it -- each 8-value chunk summed
// in k order, then the chunk sums as the tree ((c0 + c1) + (c2 + c3)) +
// ((c4 + c5) + (c6 + c7)) -- so the staged records, and the products, do
// not depend on how a launch splits the staging.
__device__ __forceinline__ float tree8(const float (&c)[8]) {
    return __fadd_rn(__fadd_rn(__fadd_rn(c[0], c[1]), __fadd_rn(c[2], c[3])),
                     __fadd_rn(__fadd_rn(c[4], c[5]), __fadd_rn(c[6], c[7])));
}

// g64 staging with eight threads per unit (one 16-byte chunk each): for a
// CTA's first item, staged by all nthreads (a multiple of 32) threads right
// after the dependency wait, where the latency of the x loads and of one
// thread's pass over 64 values is on the critical path of a dependent launch.
// Rounds are uniform over the threads, so every shuffle has all lanes.
template <int MT>
__device__ __forceinline__ void stage_x_g64_wide(const Item& it, int m0, int mrows, uint8_t* xb, int t, int nthreads) {
    const int G = it.K >> 6, nu = MT * G;
    uint8_t* meta = xb + xvals_bytes(kFmtW4G64, it.K, MT);
    const int grp = t >> 3, sub = t & 7, ngrp = nthreads >> 3;
    for (int base = 0; base < nu; base += ngrp) {
        const int i = base + grp;
        const bool act = i < nu;
        const int m = act ? i / G : 0, g = act ? i - m * G : 0;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (act && m < mrows)
            v = __ldg(reinterpret_cast<const uint4*>(it.x + (size_t)(m0 + m) * it.K + (size_t)g * 64) + sub);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t mb = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) mb = max(mb, max(w[j] & 0x7fffu, (w[j] >> 16) & 0x7fffu));
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        const int e = mb != 0u ? min(126, max(-126, 14 - ((int)(mb >> 7) - 127))) : 0;
        const float up = __int_as_float((e + 127) << 23), f = __int_as_float((127 - e) << 23);
        float se = 0.0f, so = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half a = __float2half_rn(__fmul_rn(bf16lo_f32(w[j]), up));
            const __half b = __float2half_rn(__fmul_rn(bf16hi_f32(w[j]), up));
            se = __fadd_rn(se, __half2float(a));
            so = __fadd_rn(so, __half2float(b));
            w[j] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {                // the tree of tree8, one level per step
            se = __fadd_rn(se, __shfl_xor_sync(0xffffffffu, se, o));
            so = __fadd_rn(so, __shfl_xor_sync(0xffffffffu, so, o));
        }
        if (act) {
            reinterpret_cast<uint4*>(xb)[((size_t)m * 8 + sub) * G + g] = make_uint4(w[0], w[1], w[2], w[3]);
            if (sub == 0)
                reinterpret_cast<float2*>(meta)[(size_t)m * G + g] =
                    make_float2(__fmaf_rn(1032.0f, se, __fmul_rn(72.0f, so)), f);
        }
    }
}

template <int FMT, int MT>
__device__ __forceinline__ void stage_x(const Item& it, int m0, int mrows, uint8_t* xb, int first, int stride) {
    constexpr bool kW4 = !is_w8(FMT);
    const int hcpr = it.K >> 5, n = MT * hcpr;
    uint8_t* meta = xb + xvals_bytes(FMT, it.K, MT);
    if constexpr (FMT == kFmtW4G64) {
        // g64: one 64-value unit (a quantization group) per lane at a time;
        // quad q of unit g of row m at (m * 8 + q) * G + g, record {z, f} at
        // m * G + g, with z = 1032 * sum over even k + 72 * sum over odd k.
        const int G = it.K >> 6, nu = MT * G;
        for (int i = first; i < nu; i += stride) {
            const int m = i / G, g = i - m * G;
            uint4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = make_uint4(0u, 0u, 0u, 0u);
            if (m < mrows) {
                const uint4* src = reinterpret_cast<const uint4*>(it.x + (size_t)(m0 + m) * it.K + (size_t)g * 64);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = __ldg(src + j);
            }
            uint32_t* w = reinterpret_cast<uint32_t*>(v);
            uint32_t mb = 0u;
#pragma unroll
            for (int j = 0; j < 32; ++j) mb = max(mb, max(w[j] & 0x7fffu, (w[j] >> 16) & 0x7fffu));
            const int e = mb != 0u ? min(126, max(-126, 14 - ((int)(mb >> 7) - 127))) : 0;
            const float up = __int_as_float((e + 127) << 23), f = __int_as_float((127 - e) << 23);
            float ce[8], co[8];                          // per 8-value chunk, in k order
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                ce[q] = 0.0f;
                co[q] = 0.0f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = 4 * q + jj;
                    const __half a = __float2half_rn(__fmul_rn(bf16lo_f32(w[j]), up));
                    const __half b = __float2half_rn(__fmul_rn(bf16hi_f32(w[j]), up));
                    ce[q] = __fadd_rn(ce[q], __half2float(a));
                    co[q] = __fadd_rn(co[q], __half2float(b));
                    w[j] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
                }
            }
            const float se = tree8(ce), so = tree8(co);
            uint4* dst = reinterpret_cast<uint4*>(xb) + (size_t)m * 8 * G + g;
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[(size_t)q * G] = v[q];
            reinterpret_cast<float2*>(meta)[(size_t)m * G + g] =
                make_float2(__fmaf_rn(1032.0f, se, __fmul_rn(72.0f, so)), f);
        }
    } else {
        for (int i0 = first; i0 < n; i0 += 2 * stride) {
            uint4 v[2][4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {               // both loads in flight before use
                const int i = i0 + stride * u, m = i / hcpr, h = i - m * hcpr;
#pragma unroll
                for (int j = 0; j < 4; ++j) v[u][j] = make_uint4(0u, 0u, 0u, 0u);
                if (i < n && m < mrows) {
                    const uint4* src = reinterpret_cast<const uint4*>(it.x + (size_t)(m0 + m) * it.K + (size_t)h * 32);
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[u][j] = __ldg(src + j);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = i0 + stride * u, m = i / hcpr, h = i - m * hcpr;
                if (i >= n) break;
                uint32_t* w = reinterpret_cast<uint32_t*>(v[u]);
                if constexpr (kW4) {
                    uint32_t mb = 0u;
#pragma unroll
                    for (int j = 0; j < 16; ++j) mb = max(mb, max(w[j] & 0x7fffu, (w[j] >> 16) & 0x7fffu));
                    const int e = mb != 0u ? min(126, max(-126, 14 - ((int)(mb >> 7) - 127))) : 0;
                    const float up = __int_as_float((e + 127) << 23), f = __int_as_float((127 - e) << 23);
                    float se = 0.0f, so = 0.0f;              // even-k and odd-k sums
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const __half a = __float2half_rn(__fmul_rn(bf16lo_f32(w[j]), up));
                        const __half b = __float2half_rn(__fmul_rn(bf16hi_f32(w[j]), up));
                        se = __fadd_rn(se, __half2float(a));
                        so = __fadd_rn(so, __half2float(b));
                        w[j] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(xb) + (size_t)m * 4 * hcpr + h;
#pragma unroll
                    for (int q = 0; q < 4; ++q) dst[(size_t)q * hcpr] = v[u][q];
                    const float z = __fmaf_rn(1024.0f, se, __fmul_rn(64.0f, so));   // sb32
                    reinterpret_cast<float4*>(meta)[(size_t)m * hcpr + h] =
                        make_float4(z, __fmul_rn(f, __fadd_rn(se, so)), f, 0.0f);
                } else {
                    float4* dst = reinterpret_cast<float4*>(xb) + (size_t)m * 8 * hcpr + h;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dst[(size_t)q * hcpr] = make_float4(bf16lo_f32(w[2 * q]), bf16hi_f32(w[2 * q]),
                                                            bf16lo_f32(w[2 * q + 1]), bf16hi_f32(w[2 * q + 1]));
                }
            }
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
template <int FMT, int MT, int RW, int TT, int YB>
__device__ __forceinline__ void gemv_group(const Item& it, uint32_t st_s, int g0, int rg, uint32_t x_s, int m0, int mrows, int lane, int rbase, int slice,
                                           float* red) {
    constexpr bool kW4 = !is_w8(FMT);
    constexpr int U = RW == 1 ? 2 : 1;                   // half-chunks per iteration
    const int hcpr = it.K >> 5, T = TT ? TT : it.T, HJ = it.HJ;   // TT: team lanes fixed at compile time
    const int li = lane & (T - 1);
    const int hoff = slice * HJ;                         // this warp's k-slice of the row
    const uint32_t crb = it.crb, srb = it.srb;
    const uint32_t ssc_s = st_s + (uint32_t)round16((size_t)it.Rg * crb);
    // x quads: (m * Q + q) * hcpr + h, Q = 4 (bf16) or 8 (fp32) quads per half-chunk
    const uint32_t xstride = (uint32_t)hcpr * 16u;
    const uint32_t xa0 = x_s + (uint32_t)li * 16u;
    const uint32_t xm0 = x_s + (uint32_t)xvals_bytes(FMT, it.K, MT) + (uint32_t)li * 16u;   // sb32 records
    float yacc[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[r][m] = 0.0f;

    if constexpr (FMT == kFmtW4G64) {
        // One 64-weight group (unit) per lane and row: 32 code bytes at
        // row * crb + unit * 32, its scale at unit * 2; x as 8 quads per unit
        // (quad q of unit g at (m * 8 + q) * G + g) and a record {z, f}.
        const int G = it.K >> 6;
        const uint32_t gstride = (uint32_t)G * 16u;
        const uint32_t xmg0 = x_s + (uint32_t)xvals_bytes(FMT, it.K, MT) + (uint32_t)li * 8u;
        uint32_t ca[RW], sa[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            ca[r] = st_s + (uint32_t)(rbase + r) * crb + (uint32_t)li * 32u;
            sa[r] = ssc_s + (uint32_t)(rbase + r) * srb + (uint32_t)li * 2u;
        }
        for (int hj = 0; hj < HJ; ++hj) {
            const uint32_t du = (uint32_t)(hoff + hj) * (uint32_t)T;   // first unit of this step
            float2 xm[MT];                               // {z, f}
#pragma unroll
            for (int m = 0; m < MT; ++m) xm[m] = lds64f_a(xmg0 + ((uint32_t)m * (uint32_t)G + du) * 8u);
            uint4 c0[RW], c1[RW];
            float sA[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                c0[r] = lds128_a(ca[r] + du * 32u);
                c1[r] = lds128_a(ca[r] + du * 32u + 16u);
                sA[r] = __half2float(__ushort_as_half((unsigned short)lds16_a(sa[r] + du * 2u)));
            }
            // one accumulator for even k ((1024 + u) x), started at -z, and one
            // for odd k ((1024 + 16 u) x) per row and m, whatever the launch
            // shape, so a row's sums do not depend on RW or batching
            float lo[RW][MT], hi[RW][MT];
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    lo[r][m] = -xm[m].x;
                    hi[r][m] = 0.0f;
                }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const uint4 X = lds128_a(xa0 + du * 16u + (uint32_t)(m * 8 + q) * gstride);
#pragma unroll
                    for (int r = 0; r < RW; ++r)
                        dot8_w4_f16(word_of(q < 4 ? c0[r] : c1[r], q & 3), X, lo[r][m], hi[r][m]);
                }
            }
            // sum_k q_k x'_k = lo + hi / 16, back to x's scale with f = 2^-e_g
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    yacc[r][m] = __fmaf_rn(__fmul_rn(sA[r], xm[m].y), __fmaf_rn(hi[r][m], 0.0625f, lo[r][m]),
                                           yacc[r][m]);
        }
    } else if constexpr (kW4) {
        // W4SB32: record at row * crb + (h / 8) * 144; T is a multiple of 8
        // (K % 256 == 0), so a lane always sees the same group j = li % 8.
        const int j = li & 7;
        uint32_t ca[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) ca[r] = st_s + (uint32_t)(rbase + r) * crb + (uint32_t)(li >> 3) * 144u;
        for (int hj = 0; hj < HJ; hj += U) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (u > 0 && hj + u >= HJ) break;
                const uint32_t dh = (uint32_t)(hoff + hj + u) * (uint32_t)T;
                float4 xm[MT];                           // {z, f * sum, f}
#pragma unroll
                for (int m = 0; m < MT; ++m) xm[m] = lds128f_a(xm0 + ((uint32_t)m * (uint32_t)hcpr + dh) * 16u);
                uint4 c[RW];
                float sA[RW], sB[RW];
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const uint32_t rec = ca[r] + (dh >> 3) * 144u;
                    const uint4 hd = lds128_a(rec);
                    c[r] = lds128_a(rec + 16u + (uint32_t)j * 16u);
                    const float d = __half2float(__ushort_as_half((unsigned short)(hd.x & 0xffffu)));
                    const float dm = __half2float(__ushort_as_half((unsigned short)(hd.x >> 16)));
                    sA[r] = __fmul_rn(d, (float)sb_field(hd.y, hd.z, hd.w, 0, j));
                    sB[r] = __fmul_rn(dm, (float)sb_field(hd.y, hd.z, hd.w, 1, j));
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
                // sum_k u_k x'_k = lo + hi / 16;
                // back to x's scale with f = 2^-e_h
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float a = __fmaf_rn(hi[r][m], 0.0625f, lo[r][m]);
                        yacc[r][m] = __fmaf_rn(__fmul_rn(sA[r], xm[m].z), a, yacc[r][m]);
                        yacc[r][m] = __fmaf_rn(-sB[r], xm[m].y, yacc[r][m]);
                    }
            }
        }
    } else {
        // int8: 32 code bytes per row and half-chunk h = groups 2h, 2h+1 of
        // 16 (two scales) or half of group h/2 of 64 (one scale); x as fp32
        // quads, 8 per half-chunk. Rows are taken two at a time, so each x
        // quad loaded from shared memory serves two rows (halving the x
        // traffic, which is what limits two activation rows) within the
        // register budget.
        constexpr int RB = MT == 1 || RW < 2 ? 1 : 2;
        constexpr int UW = MT == 1 ? U : 1;              // two half-chunks per iteration spill at MT = 2
        uint32_t ca[RW], sa[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            ca[r] = st_s + (uint32_t)(rbase + r) * crb + (uint32_t)li * 32u;
            sa[r] = ssc_s + (uint32_t)(rbase + r) * srb;
        }
        for (int hj = 0; hj < HJ; hj += UW) {
#pragma unroll
          for (int u = 0; u < UW; ++u) {
            if (u > 0 && hj + u >= HJ) break;
            const uint32_t dh = (uint32_t)(hoff + hj + u) * (uint32_t)T;
            const uint32_t hc = dh + (uint32_t)li;           // this lane's half-chunk of the row
#pragma unroll
            for (int r0 = 0; r0 < RW; r0 += RB) {
                uint32_t sp[RB];
#pragma unroll
                for (int r = 0; r < RB; ++r)
                    sp[r] = FMT == kFmtW8G64 ? lds16_a(sa[r0 + r] + ((hc >> 1) << 1)) * 0x10001u
                                             : lds32_a(sa[r0 + r] + hc * 4u);
#pragma unroll
                for (int g = 0; g < 2; ++g) {                // 16-weight halves of the half-chunk
                    uint4 c[RB];
#pragma unroll
                    for (int r = 0; r < RB; ++r) c[r] = lds128_a(ca[r0 + r] + dh * 32u + 16u * (uint32_t)g);
                    float a[RB][MT];
#pragma unroll
                    for (int r = 0; r < RB; ++r)
#pragma unroll
                        for (int m = 0; m < MT; ++m) a[r][m] = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float f[RB][4];
#pragma unroll
                        for (int r = 0; r < RB; ++r) unpack_w8(word_of(c[r], i), f[r]);
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            const float4 xv = lds128f_a(xa0 + dh * 16u + (uint32_t)(m * 8 + g * 4 + i) * xstride);
#pragma unroll
                            for (int r = 0; r < RB; ++r) {
                                a[r][m] = fmaf(f[r][0], xv.x, a[r][m]);
                                a[r][m] = fmaf(f[r][1], xv.y, a[r][m]);
                                a[r][m] = fmaf(f[r][2], xv.z, a[r][m]);
                                a[r][m] = fmaf(f[r][3], xv.w, a[r][m]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < RB; ++r) {
                        const float sg = __half2float(__ushort_as_half((unsigned short)(g ? sp[r] >> 16 : sp[r] & 0xffffu)));
#pragma unroll
                        for (int m = 0; m < MT; ++m) yacc[r0 + r][m] = fmaf(sg, a[r][m], yacc[r0 + r][m]);
                    }
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
                else if (m < mrows) store_y(it.y, (size_t)(m0 + m) * it.N + g0 + rr, v, YB);
            }
        }
    } else {                                             // shuffle tree per row, lane 0 of each team stores
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
                        else if (m < mrows) store_y(it.y, (size_t)(m0 + m) * it.N + g0 + rr, yacc[r][m], YB);
                    }
            }
        }
    }
}

// Consumer view of the weight ring (one copy per warp, in registers).
struct Ring {
    uint64_t* full;
    uint64_t* empty;
    uint8_t* red;              // per-stage k-slice partial sums
    uint32_t base;             // shared address of stage 0
    uint32_t stage_bytes, red_bytes;
    int stages;
    int s;                     // stage of the next group
    uint32_t ph;               // its phase parity
    unsigned long long lim;    // wait bound
};

// All groups of rows [ra, rb) of item `it` for this warp: waits for each
// stage, computes its team's rows, stores the outputs (with KS > 1: the
// team's slice-0 warp adds the k-slices after a team barrier) and releases
// the stage. The launch shape (RW, TT) is fixed per item, so the per-item
// setup stays outside the group loop. False if a bounded wait gave up.
template <int FMT, int MT, int RW, int TT, int YB>
__device__ __forceinline__ bool gemv_item(const Item& it, int ra, int rb, Ring& ring, uint32_t x_s, int m0,
                                          int mrows, int warp, int lane, int& g_fail) {
    const int T = TT ? TT : it.T, KS = it.KS, Rg = it.Rg;
    const int slice = warp % KS;                         // k-slice of this warp (KS > 1 only when T == 32)
    const int team = warp / KS;                          // warps team*KS .. team*KS+KS-1 share rows
    const int wteam = team * (32 / T);                   // first lane team of this warp
    const int rbase = (wteam + lane / T) * RW;           // first row of this lane team in a group
    const int wfirst = wteam * RW;                       // first row of this warp in a group
    for (int g0 = ra; g0 < rb; g0 += Rg) {
        const int s = ring.s;
        const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&ring.full[s], ring.ph, kStatusTmaWait, 0u, ring.lim));
        if (++ring.s == ring.stages) {                   // next stage and its phase parity
            ring.s = 0;
            ring.ph ^= 1u;
        }
        const int rg = min(Rg, rb - g0);
        bool all = got;
        if (wfirst < rg) {                               // warp-uniform
            float* red = reinterpret_cast<float*>(ring.red + (size_t)s * ring.red_bytes);
            if (got)
                gemv_group<FMT, MT, RW, TT, YB>(it, ring.base + (uint32_t)s * ring.stage_bytes, g0, rg, x_s, m0,
                                                mrows, lane, rbase, slice, red);
            if (KS > 1) {
                // the k-slices of a team meet here; a slice whose wait gave up
                // still arrives, after raising the CTA's give-up flag, and the
                // whole team leaves together (no warp is left at the barrier)
                asm volatile("bar.sync %0, %1;" :: "r"(1 + team), "r"(KS * 32) : "memory");
                if (all && slice == 0 && lane < RW * MT) {
                    const int r = lane / MT, m = lane - r * MT, rr = wfirst + r;
                    if (rr < rg && m < mrows) {
                        const float* q = red + ((size_t)rr * MT + m) * KS;
                        float v = 0.0f;
                        for (int k = 0; k < KS; ++k) v += q[k];
                        store_y(it.y, (size_t)(m0 + m) * it.N + g0 + rr, v, YB);
                    }
                }
            }
        }
        if (!all) {
            g_fail = g0;                                 // this group's barrier was met; the rest are not
            return false;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring.empty[s]);     // stage consumed
    }
    return true;
}

// After a bounded wait gave up in the group at row g_fail of item i0, a
// consumer warp still owes its team its part in every later k-slice barrier
// that its teammates, which may still be computing, will reach: it takes
// each of them in turn (a barrier instance must complete before the warp
// counts toward the next), then leaves. Never taken unless a wait ran out.
template <int MAXI>
__device__ __noinline__ void gemv_give_up(const Batch<MAXI>& p, int i0, int g_fail, long long lo, long long hi,
                                          int warp) {
    for (int i = i0; i < p.count; ++i) {
        const Item& it = p.it[i];
        if (it.cost0 >= hi) break;
        if (it.cost1 <= lo) continue;
        int ua, ub;
        item_units(it, lo, hi, ua, ub);
        const int ra = ua * it.rho, rb = min(ub * it.rho, it.N);
        if (ra >= rb || it.KS <= 1) continue;
        const int team = warp / it.KS, wfirst = team * (32 / it.T) * it.RW;
        for (int g0 = (i == i0 ? g_fail + it.Rg : ra); g0 < rb; g0 += it.Rg)
            if (wfirst < min(it.Rg, rb - g0))
                asm volatile("bar.sync %0, %1;" :: "r"(1 + team), "r"(it.KS * 32) : "memory");
    }
}

// Resident CTAs per SM the register budget is sized for.
constexpr int min_blocks(int) { return kConsumerWarps <= 12 ? 2 : 1; }

// YB: outputs rounded once to bf16 (1) or fp32 (0), fixed per launch.
template <int FMT, int MT, int MAXI, int YB>
__global__ void __launch_bounds__(kThreads, min_blocks(MT))
gemv_kernel(const __grid_constant__ Batch<MAXI> p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + p.stages;
    uint64_t* xfull = empty + p.stages;                  // staged x buffer b ready (32 stager lanes)
    uint64_t* xempty = xfull + 2;                        // staged x buffer b released (consumer warps)
    const long long lo = (long long)blockIdx.x * p.total / gridDim.x;
    const long long hi = (long long)(blockIdx.x + 1) * p.total / gridDim.x;

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&xfull[b], 32);
            mbar_init(&xempty[b], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    grid_dep_launch();

    if (warp == kProducerWarp) {                         // weight copies into the ring
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            int gi = 0, armed = 0;
            bool ok = true;
            for (int i = item_after(p, lo); i < p.count && ok; ++i) {
                const Item& it = p.it[i];
                if (it.cost0 >= hi) break;               // items are in cost order
                if (it.cost1 <= lo) continue;            // no overlap: skip without dividing
                int ua, ub;
                item_units(it, lo, hi, ua, ub);
                const int ra = ua * it.rho, rb = min(ub * it.rho, it.N);
                for (int g0 = ra; g0 < rb; g0 += it.Rg, ++gi) {
                    const int s = gi % p.stages;
                    if (gi >= p.stages &&
                        !mbar_wait_bounded(&empty[s], ((gi / p.stages) - 1) & 1, kStatusSlotWait, kProducerNapNs,
                                           p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (p.test_flags & kTestNoCopies) continue;
                    const int rg = min(it.Rg, rb - g0);
                    const uint32_t cb = (uint32_t)rg * it.crb;
                    const uint32_t sb = it.srb ? (((uint32_t)rg * it.srb + 15u) & ~15u) : 0u;
                    uint8_t* st = smem + (size_t)s * p.stage_bytes;
                    mbar_arrive_expect_tx(&full[s], cb + sb);
                    bulk_g2s(st, it.codes + (size_t)g0 * it.crb, cb, &full[s], pol);
                    if (sb)
                        bulk_g2s(st + round16((size_t)it.Rg * it.crb), it.scales + (size_t)g0 * it.srb, sb, &full[s], pol);
                    armed = gi + 1;
                }
            }
            // Copies still in flight (consumers that gave up) land before the CTA
            // leaves: wait for the last phase armed on every stage.
            for (int s = 0; s < p.stages && s < armed; ++s) {
                const int uses = armed / p.stages + (s < armed % p.stages ? 1 : 0);
                mbar_wait_bounded(&full[s], (uint32_t)(uses - 1) & 1u, kStatusTmaWait, kProducerNapNs, p.wait_ns);
            }
        }
        return;
    }

    // A CTA's first item is staged by the consumer warps and the stager
    // together (it is on the critical path of a dependent launch); the
    // stager alone stages the later ones while the consumers compute.
    const int i_first = first_item(p, lo, hi);
    constexpr int kCoop = (kConsumerWarps + 1) * 32;
    if (warp == kStagerWarp) {                           // x of each item into alternating buffers
        grid_dep_wait();                                 // x is written by the previous kernel
        if (i_first < 0) return;
        if constexpr (FMT == kFmtW4G64)
            stage_x_g64_wide<MT>(p.it[i_first], p.m0, p.mrows, smem + p.x_off, kConsumerWarps * 32 + lane, kCoop);
        else
            stage_x<FMT, MT>(p.it[i_first], p.m0, p.mrows, smem + p.x_off, kConsumerWarps * 32 + lane, kCoop);
        asm volatile("bar.sync %0, %1;" :: "n"(kCoopBarrier), "n"(kCoop) : "memory");
        mbar_arrive(&xfull[0]);
        int xi = 1;
        for (int i = i_first + 1; i < p.count; ++i) {
            const Item& it = p.it[i];
            if (it.cost0 >= hi) break;
            if (it.cost1 <= lo) continue;
            int ua, ub;
            item_units(it, lo, hi, ua, ub);
            if (ua * it.rho >= min(ub * it.rho, it.N)) continue;
            const int b = xi % p.nxb;
            if (xi >= p.nxb &&
                !mbar_wait_bounded(&xempty[b], ((xi / p.nxb) - 1) & 1, kStatusXWait, kStagerNapNs, p.wait_ns))
                break;
            stage_x<FMT, MT>(it, p.m0, p.mrows, smem + p.x_off + (size_t)b * p.x_bytes, lane, 32);
            mbar_arrive(&xfull[b]);                      // each lane: its stores are released
            ++xi;
        }
        return;
    }

    // ---- consumers ---------------------------------------------------------
    const uint32_t smem_s = smem_u32(smem);
    grid_dep_wait();                                     // x is written by the previous kernel
    if (i_first >= 0) {
        if constexpr (FMT == kFmtW4G64)
            stage_x_g64_wide<MT>(p.it[i_first], p.m0, p.mrows, smem + p.x_off, tid, kCoop);
        else
            stage_x<FMT, MT>(p.it[i_first], p.m0, p.mrows, smem + p.x_off, tid, kCoop);
        asm volatile("bar.sync %0, %1;" :: "n"(kCoopBarrier), "n"(kCoop) : "memory");
    }
    Ring ring;
    ring.full = full;
    ring.empty = empty;
    ring.red = smem + p.red_off;
    ring.base = smem_s;
    ring.stage_bytes = p.stage_bytes;
    ring.red_bytes = p.red_bytes;
    ring.stages = p.stages;
    ring.s = 0;
    ring.ph = 0u;
    ring.lim = p.wait_ns;
    int xi = 0;                                          // items done
    for (int i = i_first < 0 ? p.count : i_first; i < p.count; ++i) {
        const Item it = p.it[i];                         // this item's fields in registers
        if (it.cost0 >= hi) break;                       // items are in cost order
        if (it.cost1 <= lo) continue;                    // no overlap: skip without dividing
        int ua, ub;
        item_units(it, lo, hi, ua, ub);
        const int ra = ua * it.rho, rb = min(ub * it.rho, it.N);
        if (ra >= rb) continue;
        const int b = xi % p.nxb;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&xfull[b], (xi / p.nxb) & 1, kStatusXWait, 0u, p.wait_ns))) {
            gemv_give_up(p, i, ra - it.Rg, lo, hi, warp);  // owes every barrier of this item and the later ones
            return;
        }
        const uint32_t x_s = smem_s + p.x_off + (uint32_t)b * p.x_bytes;
        bool ok;
        int g_fail = 0;
        // int8 at two activation rows keeps at most two rows per lane team (four
        // would not fit the register budget); that case is never planned
        constexpr int RW4 = is_w8(FMT) && MT == 2 ? 2 : 4;
        if (it.T == 32) {                                // whole-warp teams: the common case
            ok = it.RW == 4   ? gemv_item<FMT, MT, RW4, 32, YB>(it, ra, rb, ring, x_s, p.m0, p.mrows, warp, lane, g_fail)
                 : it.RW == 2 ? gemv_item<FMT, MT, 2, 32, YB>(it, ra, rb, ring, x_s, p.m0, p.mrows, warp, lane, g_fail)
                              : gemv_item<FMT, MT, 1, 32, YB>(it, ra, rb, ring, x_s, p.m0, p.mrows, warp, lane, g_fail);
        } else {
            ok = it.RW == 4   ? gemv_item<FMT, MT, RW4, 0, YB>(it, ra, rb, ring, x_s, p.m0, p.mrows, warp, lane, g_fail)
                 : it.RW == 2 ? gemv_item<FMT, MT, 2, 0, YB>(it, ra, rb, ring, x_s, p.m0, p.mrows, warp, lane, g_fail)
                              : gemv_item<FMT, MT, 1, 0, YB>(it, ra, rb, ring, x_s, p.m0, p.mrows, warp, lane, g_fail);
        }
        if (!ok) {
            gemv_give_up(p, i, g_fail, lo, hi, warp);
            return;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&xempty[b]);          // staged x released
        ++xi;
    }
}

// Shared-memory target per CTA for single products: three CTAs (three kernels
// of a dependent chain) fit on one SM. Batches run two CTAs per SM.
constexpr int kSingleCtasPerSm = 1;
constexpr int kBatchCtasPerSm = 2;
constexpr size_t kSmemTarget = 72 * 1024;
constexpr long long kWideBytes = 32ll << 20;          // single products from this size run as batches do
constexpr size_t kSmemBatch = 112 * 1024;
constexpr size_t kSmemLimit = 220 * 1024;
constexpr size_t kSmemAttr = kSmemLimit + 1024;

template <int FMT, int MT, int MAXI, int YB>
cudaError_t launch_one(const Batch<MAXI>& prm, size_t smem, int grid, cudaStream_t st) {
    auto kern = gemv_kernel<FMT, MT, MAXI, YB>;
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

// Lane and warp layout of a product's rows. A lane's unit of a row is one
// 64-weight group for g64 and a 32-weight half-chunk otherwise; T lanes per
// team (a power of two dividing the units per row), KS warps per row (when
// T == 32, long rows are split so that each warp keeps at least 128 weights
// per lane and row), HJ units per lane and warp.
struct Layout { int T, KS, HJ, teams; };
Layout layout_of(int fmt, int K) {
    const int units = fmt == kFmtW4G64 ? K / 64 : K / 32;
    const int min_hj = fmt == kFmtW4G64 ? 1 : 2;
    Layout l;
    l.T = 32;
    while (l.T > 1 && (units % l.T) != 0) l.T >>= 1;
    const int hj_all = units / l.T;
    l.KS = 1;
    while (l.T == 32 && kConsumerWarps % (l.KS * 2) == 0 && hj_all % (l.KS * 2) == 0 &&
           hj_all / (l.KS * 2) >= min_hj)
        l.KS *= 2;
    l.HJ = hj_all / l.KS;
    l.teams = (kConsumerWarps / l.KS) * (32 / l.T);
    return l;
}

// Rows per team for a product: the largest of 4, 2, 1 whose group of
// teams * RW rows stays within 48 KB.
int rw_allowed(int fmt, int K) {
    const Layout l = layout_of(fmt, K);
    auto sb = [&](size_t R) { return round16(R * code_row_bytes(fmt, K)) + round16(R * scale_row_bytes(fmt, K)); };
    if (sb((size_t)l.teams * 4) <= 48 * 1024) return 4;
    return sb((size_t)l.teams * 2) <= 48 * 1024 ? 2 : 1;
}

// Per-item launch geometry for rows-per-team RW; false for a shape that does
// not fit even with one staged-x buffer.
bool plan_item(int fmt, int K, int N, int MT, int RW, Item& it, size_t& stage_b) {
    const Layout l = layout_of(fmt, K);
    const size_t crb = code_row_bytes(fmt, K), srb = scale_row_bytes(fmt, K);
    int rho = 1;
    while (((size_t)rho * srb) % 16 != 0) rho <<= 1;     // srb is even, so rho <= 8
    auto stage_bytes = [&](int R) { return round16((size_t)R * crb) + round16((size_t)R * srb); };
    auto red_bytes = [&](int R) { return l.KS > 1 ? round16((size_t)R * MT * l.KS * 4) : (size_t)0; };
    const size_t x1 = round16(xbuf_bytes(fmt, K, MT)) + 256;   // one x buffer, counters, barriers
    int Rg = l.teams * RW;
    while (Rg > rho && Rg > RW && x1 + 2 * (stage_bytes(Rg) + red_bytes(Rg)) > kSmemLimit) Rg >>= 1;
    if (Rg % rho != 0 || x1 + stage_bytes(Rg) + red_bytes(Rg) > kSmemLimit) return false;
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

// Shared-memory plan of a launch: ring of `stages` stages, nxb staged-x
// buffers, per-stage k-slice partials, barriers. Prefers two
// x buffers and a size that lets two CTAs share an SM (`want`).
struct SmemPlan { int stages, nxb; size_t smem; };
bool plan_smem(size_t sb, size_t xbb, size_t red, size_t want, int max_stages, SmemPlan& o) {
    auto fixed = [&](int nxb, int st) { return (size_t)nxb * xbb + (size_t)(2 * st + 4) * 8; };
    auto fits = [&](int nxb, int st, size_t cap) { return st * (sb + red) + fixed(nxb, st) <= cap; };
    for (size_t cap : {want, kSmemLimit})
        for (int nxb = 2; nxb >= 1; --nxb) {
            if (!fits(nxb, cap == want ? 2 : 1, cap)) continue;
            int st = 1;
            while (st < max_stages && fits(nxb, st + 1, cap)) ++st;
            o.stages = st;
            o.nxb = nxb;
            o.smem = st * (sb + red) + fixed(nxb, st);
            return true;
        }
    return false;
}

template <int FMT, int MAXI>
cudaError_t launch_batch(const WgemmArgs* a, int count, cudaStream_t st) {
    const int M = a[0].M;
    for (int MT = M >= 2 ? 2 : 1; MT >= 1; --MT) {
        Batch<MAXI> p = {};
        p.count = count;
        size_t sb = 0, xbb = 0, red = 0;
        long long total = 0, units_min = -1;
        bool ok = true;
        for (int i = 0; i < count && ok; ++i) {
            Item& it = p.it[i];
            size_t s1;
            int rw = rw_allowed(FMT, a[i].K);
            if (is_w8(FMT) && MT == 2 && rw > 2) rw = 2;   // the register budget (see the kernel's dispatch)
            if (!plan_item(FMT, a[i].K, a[i].N, MT, rw, it, s1)) {
                ok = false;
                break;
            }
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
            const size_t xq = round16(xbuf_bytes(FMT, a[i].K, MT));
            xbb = xq > xbb ? xq : xbb;
            const size_t rd = it.KS > 1 ? round16((size_t)it.Rg * MT * it.KS * 4) : 0;
            red = rd > red ? rd : red;
        }
        // A large single product (the 7.2B head: 302 MB) runs like a batch, two
        // CTAs per SM with deeper rings; a small one keeps room for the next
        // kernels of a dependent chain on the same SM.
        const bool wide = count > 1 || total >= kWideBytes;
        SmemPlan sp;
        if (!ok || !plan_smem(sb, xbb, red, wide ? kSmemBatch : kSmemTarget, 6, sp)) {
            if (MT == 2) continue;                       // retry one activation row per launch
            return cudaErrorInvalidValue;
        }
        p.total = total;
        p.wait_ns = wait_limit_ns();
        p.test_flags = test_flags();
        int grid = sm_count() * (wide ? kBatchCtasPerSm : kSingleCtasPerSm);
        if (count == 1 && grid > units_min) grid = (int)units_min;
        int stages = sp.stages;
        if (count == 1) {   // a single product needs no more stages than its largest CTA has groups
            const Item& it = p.it[0];
            const long long per = (units_min + grid - 1) / grid * it.rho;
            const int gmax = (int)((per + it.Rg - 1) / it.Rg);
            if (stages > gmax) stages = gmax;
        }
        p.stages = stages;
        p.nxb = sp.nxb;
        p.stage_bytes = (uint32_t)sb;
        p.x_off = (uint32_t)(stages * sb);
        p.x_bytes = (uint32_t)xbb;
        p.red_off = (uint32_t)(p.x_off + sp.nxb * xbb);
        p.red_bytes = (uint32_t)red;
        p.bar_off = (uint32_t)(p.red_off + stages * red);
        const size_t smem = p.bar_off + (size_t)(2 * stages + 4) * sizeof(uint64_t);
        if (smem > kSmemAttr) return cudaErrorInvalidValue;

        for (int m0 = 0; m0 < M; m0 += MT) {
            p.m0 = m0;
            p.mrows = M - m0 < MT ? M - m0 : MT;
            const bool yb = a[0].ybf16 != 0;
            const cudaError_t e = MT == 2 ? (yb ? launch_one<FMT, 2, MAXI, 1>(p, smem, grid, st)
                                                : launch_one<FMT, 2, MAXI, 0>(p, smem, grid, st))
                                          : (yb ? launch_one<FMT, 1, MAXI, 1>(p, smem, grid, st)
                                                : launch_one<FMT, 1, MAXI, 0>(p, smem, grid, st));
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    return cudaErrorInvalidValue;
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
        case kFmtW8G64: return launch_fmt<kFmtW8G64>(a, count, st);
        case kFmtW4SB32: return launch_fmt<kFmtW4SB32>(a, count, st);
        default: return cudaErrorNotSupported;            // 5- and 6-bit codes run on the tensor-core kernel
    }
}

}  // namespace rq
