// rq_prefill.cu -- y = x * w_hat^T for prefill-sized activation blocks
// (33 <= M <= 128) on the 5th-generation tensor cores: packed weights are
// dequantized to bf16 into shared-memory tiles, x is copied beside them, and
// one thread issues tcgen05.mma into an fp32 accumulator in tensor memory.
//
// Sources: RWKV-7 G1 1.5B int4 model card, summary paragraph (a tensor-core
// GEMM beside the int4 GEMV and small-M kernels, output bit-identical to the
// offline dequantization in the GEMV); rwkv_quant_nv project description,
// "Operator Optimization Details" (the 4096-wide shapes and a 1 x 128 prefill).
//
// Design (B200):
//  * CTA tile: 128 weight rows (the MMA's M) x all activation rows (the MMA's
//    N = M rounded up to 16) x a K range; D[128][Mpad] fp32 lives in TMEM.
//  * K advances in stages of 64 (one 128-byte swizzle row of bf16): A = the
//    dequantized weight tile [128][64], B = x [Mpad][64], both K-major with the
//    128-byte swizzle (16-byte chunk c of row r stored at chunk c ^ (r % 8) of
//    its 128-byte row, 8-row groups 1024 bytes apart).
//  * Eight producer warps, two threads per weight row: cp.async brings the raw
//    codes, a 16-byte window of the scale row and x (zero-filled past M) into
//    a per-stage raw area two stages ahead; the dequantization writes A. int4:
//    a lop3 places a nibble pair in fp16 mantissas ((1024 + u), (1024 + 16 u));
//    fma.rn.f32.f16 against the fp16 scale gives q * s exactly; a cvt rounds
//    each pair of weights to bf16 (one rounding). int8: a byte permute gives
//    fp16 (1024 + u), the same FMA gives q * s.
//  * Warp 0 allocates TMEM; its lane 0 issues four MMAs (K = 16) per stage and
//    commits each stage to that stage's `empty` barrier and the last one to
//    `accfull`. The producer warps then read D back with tcgen05.ld and store
//    y (fp32, coalesced along N for each activation row).
//  * Every wait is bounded; on a timeout a status bit is set, the MMA thread
//    still commits `accfull` and TMEM is always released.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kPfRowsT = 128;                 // weight rows per tile (MMA M)
constexpr int kPfK = 64;                      // K per stage
constexpr int kPfStages = 4;
constexpr int kPfLook = 2;                    // stages of raw data in flight ahead of the dequantization
constexpr int kPfProdWarps = 8;
constexpr int kPfProd = kPfProdWarps * 32;    // producer threads: two per weight row
constexpr int kPfThreads = kPfProd + 32;      // + warp 0 (TMEM, MMA issue)
constexpr uint32_t kPfATile = kPfRowsT * 128; // 16 KB

struct PfArgs {
    const uint16_t* x;          // bf16 [M][K]
    const uint8_t* codes;
    const uint8_t* scales;
    float* y;                   // fp32 [M][N]
    int M, K, N, Mpad, T;       // T = K / 64 stages
    uint32_t crb, srb;          // code / scale bytes per row
    uint32_t stage_bytes;       // A + B + raw codes + raw scales
    uint32_t b_off, rc_off, rs_off;   // offsets inside a stage
    uint32_t bar_off;           // full[S], empty[S], accfull, TMEM slot
    uint32_t tmem_cols;
};

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused (16),
// descriptor version 1, base offset 0 (tiles are 1024-byte aligned).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, both K-major,
// N = n, M = 128.
__device__ __forceinline__ uint32_t mma_idesc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kPfRowsT >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
        :: "r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}

// fp32 pair -> bf16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// c + a.half(AH) * b (fp16 operands, fp32 accumulate; the product is exact).
template <int AH>
__device__ __forceinline__ float fma_h(uint32_t a, uint16_t b, float c) {
    float d;
    if (AH == 0)
        asm("{ .reg .b16 a0, a1; mov.b32 {a0, a1}, %1; fma.rn.f32.f16 %0, a0, %2, %3; }"
            : "=f"(d) : "r"(a), "h"(b), "f"(c));
    else
        asm("{ .reg .b16 a0, a1; mov.b32 {a0, a1}, %1; fma.rn.f32.f16 %0, a1, %2, %3; }"
            : "=f"(d) : "r"(a), "h"(b), "f"(c));
    return d;
}

// Byte offset of 16-byte chunk c of row r in a K-major 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
    return (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u + ((uint32_t)(c ^ (r & 7)) << 4);
}


// Raw bytes of one stage for thread (r, h): the codes of its half row and
// (h == 0) the 16-byte window of the scale row holding the stage's scales.
template <int FMT>
__device__ __forceinline__ void pf_issue(const PfArgs& p, int t, uint32_t st, int r, int h, int n0, int pt) {
    const int n = n0 + r;
    const bool in = n < p.N;
    // x: Mpad rows x 8 chunks, zero past M
    for (int q = pt; q < p.Mpad * 8; q += kPfProd) {
        const int m = q >> 3, c = q & 7;
        const bool ok = m < p.M;
        const uint16_t* src = ok ? p.x + (size_t)m * p.K + (size_t)t * kPfK + c * 8 : p.x;
        cp_async16(st + p.b_off + sw128_off(m, c), src, ok ? 16u : 0u);
    }
    if (FMT == kFmtW4G64) {            // 32 code bytes per row and stage
        const uint8_t* src = in ? p.codes + (size_t)n * p.crb + (size_t)t * 32 + h * 16 : p.codes;
        cp_async16(st + p.rc_off + (uint32_t)r * 32u + (uint32_t)h * 16u, src, in ? 16u : 0u);
    } else {                           // 64 code bytes per row and stage
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint8_t* src = in ? p.codes + (size_t)n * p.crb + (size_t)t * 64 + h * 32 + j * 16 : p.codes;
            cp_async16(st + p.rc_off + (uint32_t)r * 64u + (uint32_t)h * 32u + (uint32_t)j * 16u, src, in ? 16u : 0u);
        }
    }
    if (h == 0) {
        const size_t so = (size_t)n * p.srb + (size_t)t * (FMT == kFmtW4G64 ? 2 : 8);
        const uint8_t* src = in ? p.scales + (so & ~(size_t)15) : p.scales;
        cp_async16(st + p.rs_off + (uint32_t)r * 16u, src, in ? 16u : 0u);
    }
    cp_async_commit();
}

// Dequantizes thread (r, h)'s 32 weights of one stage into the A tile.
template <int FMT>
__device__ __forceinline__ void pf_dequant(const PfArgs& p, int t, uint8_t* st, int r, int h, int n0) {
    const size_t so = (size_t)(n0 + r) * p.srb + (size_t)t * (FMT == kFmtW4G64 ? 2 : 8);
    const uint8_t* sw = st + p.rs_off + (size_t)r * 16 + (so & 15);
    uint8_t* a = st;
    if (FMT == kFmtW4G64) {
        const uint4 c = *reinterpret_cast<const uint4*>(st + p.rc_off + (size_t)r * 32 + h * 16);
        const uint16_t sb = *reinterpret_cast<const uint16_t*>(sw);
        const float sf = __half2float(__ushort_as_half(sb));
        const float ce = __fmul_rn(-1032.0f, sf), co = __fmul_rn(-1152.0f, sf);   // exact
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t v = w[i] >> 8;
            const uint32_t p0 = lop_or_mask(w[i], 0x000F000Fu), p1 = lop_or_mask(w[i], 0x00F000F0u);
            const uint32_t p2 = lop_or_mask(v, 0x000F000Fu), p3 = lop_or_mask(v, 0x00F000F0u);
            // even k: (1024 + u) s - 1032 s = q s; odd k: (1024 + 16 u) s - 1152 s = 16 q s
            const float d0 = fma_h<0>(p0, sb, ce), d4 = fma_h<1>(p0, sb, ce);
            const float d2 = fma_h<0>(p2, sb, ce), d6 = fma_h<1>(p2, sb, ce);
            const float d1 = __fmul_rn(fma_h<0>(p1, sb, co), 0.0625f), d5 = __fmul_rn(fma_h<1>(p1, sb, co), 0.0625f);
            const float d3 = __fmul_rn(fma_h<0>(p3, sb, co), 0.0625f), d7 = __fmul_rn(fma_h<1>(p3, sb, co), 0.0625f);
            const uint4 o = make_uint4(pack_bf16(d0, d1), pack_bf16(d2, d3), pack_bf16(d4, d5), pack_bf16(d6, d7));
            *reinterpret_cast<uint4*>(a + sw128_off(r, 4 * h + i)) = o;
        }
    } else {
        const uint4 c0 = *reinterpret_cast<const uint4*>(st + p.rc_off + (size_t)r * 64 + h * 32);
        const uint4 c1 = *reinterpret_cast<const uint4*>(st + p.rc_off + (size_t)r * 64 + h * 32 + 16);
        const uint32_t sp = *reinterpret_cast<const uint32_t*>(sw + h * 4);     // groups 2h, 2h + 1
        const uint16_t sb0 = (uint16_t)(sp & 0xffffu), sb1 = (uint16_t)(sp >> 16);
        const float cf0 = __fmul_rn(-1152.0f, __half2float(__ushort_as_half(sb0)));
        const float cf1 = __fmul_rn(-1152.0f, __half2float(__ushort_as_half(sb1)));
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t ow[16];                             // bf16 pairs in k order
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint16_t sb = i < 4 ? sb0 : sb1;
            const float cf = i < 4 ? cf0 : cf1;
            // bytes -> fp16 (1024 + u); (1024 + u) s - 1152 s = q s with u = q + 128
            const uint32_t e0 = prmt(w[i], 0x6464u, 0x4140u), e1 = prmt(w[i], 0x6464u, 0x4342u);
            ow[2 * i] = pack_bf16(fma_h<0>(e0, sb, cf), fma_h<1>(e0, sb, cf));
            ow[2 * i + 1] = pack_bf16(fma_h<0>(e1, sb, cf), fma_h<1>(e1, sb, cf));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(a + sw128_off(r, 4 * h + j)) =
                make_uint4(ow[4 * j], ow[4 * j + 1], ow[4 * j + 2], ow[4 * j + 3]);
    }
}

template <int FMT>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const PfArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);   // 1024-byte aligned base
    const uint32_t base = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + kPfStages;
    uint64_t* accfull = empty + kPfStages;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(accfull + 1);
    const int n0 = blockIdx.x * kPfRowsT;

    if (tid == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&full[s], kPfProd);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tslot)), "r"(p.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_launch();

    if (warp == 0) {
        if (lane == 0) {                                 // MMA issue
            const uint32_t idesc = mma_idesc(p.Mpad);
            for (int t = 0; t < p.T; ++t) {
                const int s = t % kPfStages;
                if (!mbar_wait_bounded(&full[s], (uint32_t)(t / kPfStages) & 1u, kStatusTmaWait)) break;
                tc_fence_after();
                const uint32_t sa = base + (uint32_t)s * p.stage_bytes;
                const uint64_t da = sw128_desc(sa), db = sw128_desc(sa + p.b_off);
#pragma unroll
                for (int j = 0; j < kPfK / 16; ++j)      // K = 16 per MMA: +32 bytes along the row
                    mma_bf16(tmem, da + (uint64_t)(2 * j), db + (uint64_t)(2 * j), idesc, (t | j) != 0 ? 1u : 0u);
                mma_commit(&empty[s]);
            }
            mma_commit(accfull);                         // always: the epilogue and teardown wait on it
        }
        __syncwarp();
    } else {
        // ---- producers: two threads per weight row -----------------------
        const int pt = tid - 32, r = pt >> 1, h = pt & 1;
        grid_dep_wait();                                 // x (and possibly the planes) come from earlier kernels
        bool ok = true;
        auto issue = [&](int t) -> bool {
            const int s = t % kPfStages;
            if (t >= kPfStages &&
                !mbar_wait_bounded(&empty[s], (uint32_t)(t / kPfStages - 1) & 1u, kStatusSlotWait))
                return false;
            pf_issue<FMT>(p, t, base + (uint32_t)s * p.stage_bytes, r, h, n0, pt);
            return true;
        };
        for (int t = 0; t < kPfLook && t < p.T && ok; ++t) ok = issue(t);
        for (int t = 0; t < p.T && ok; ++t) {
            if (t + kPfLook < p.T) ok = issue(t + kPfLook);
            if (!ok) break;
            const int ahead = min(kPfLook, p.T - 1 - t);     // groups issued after stage t
            if (ahead >= 2) cp_async_wait<2>();
            else if (ahead == 1) cp_async_wait<1>();
            else cp_async_wait<0>();
            __syncwarp();                                // the pair's scale window
            const int s = t % kPfStages;
            pf_dequant<FMT>(p, t, smem + (size_t)s * p.stage_bytes, r, h, n0);
            fence_proxy_async();                         // generic-proxy smem writes -> tensor core reads
            mbar_arrive(&full[s]);
        }
        cp_async_wait<0>();
        // ---- epilogue: D[128][Mpad] -> y ---------------------------------
        const bool acc_ok = mbar_wait_bounded(accfull, 0u, kStatusMmaWait);
        if (__all_sync(0xffffffffu, acc_ok)) {           // tcgen05.ld is warp-collective
            tc_fence_after();
            const int q = warp & 3, half = (warp - 1) >> 2;
            const int cw = p.Mpad >> 1;
            const int n = n0 + 32 * q + lane;
            for (int col = half * cw; col < (half + 1) * cw; col += 8) {
                float v[8];
                tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)col, v);
                if (n < p.N) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (col + j < p.M) p.y[(size_t)(col + j) * p.N + n] = v[j];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(p.tmem_cols) : "memory");
    }
}

template <int FMT>
cudaError_t launch_fmt_pf(const WgemmArgs& a, cudaStream_t st) {
    PfArgs p = {};
    p.x = static_cast<const uint16_t*>(a.x);
    p.codes = static_cast<const uint8_t*>(a.codes);
    p.scales = static_cast<const uint8_t*>(a.scales);
    p.y = a.y;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.Mpad = (a.M + 15) & ~15;
    p.T = a.K / kPfK;
    p.crb = (uint32_t)code_row_bytes(FMT, a.K);
    p.srb = (uint32_t)scale_row_bytes(FMT, a.K);
    const uint32_t b_bytes = (uint32_t)p.Mpad * 128u;               // multiple of 2048
    const uint32_t rc_bytes = kPfRowsT * (FMT == kFmtW4G64 ? 32u : 64u);
    p.b_off = kPfATile;
    p.rc_off = p.b_off + b_bytes;
    p.rs_off = p.rc_off + rc_bytes;
    p.stage_bytes = (p.rs_off + kPfRowsT * 16u + 1023u) & ~1023u;     // next stage 1024-byte aligned
    p.bar_off = kPfStages * p.stage_bytes;
    p.tmem_cols = p.Mpad <= 64 ? 64u : 128u;
    const size_t smem = p.bar_off + (2 * kPfStages + 1) * 8 + 16 + 1024;   // + alignment slack
    auto kern = prefill_kernel<FMT>;
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
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((a.N + kPfRowsT - 1) / kPfRowsT));
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

bool prefill_supported(int fmt, int M) { return M >= kPrefillMinM && (fmt == kFmtW4G64 || fmt == kFmtW8G16); }

cudaError_t launch_prefill(const WgemmArgs& a, cudaStream_t st) {
    return a.fmt == kFmtW4G64 ? launch_fmt_pf<kFmtW4G64>(a, st) : launch_fmt_pf<kFmtW8G16>(a, st);
}

cudaError_t status_prefill(cudaStream_t st, unsigned* word) {
    unsigned v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *word = v;
    return e;
}

}  // namespace rq
