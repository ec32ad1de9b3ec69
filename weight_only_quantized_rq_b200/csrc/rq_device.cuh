// rq_device.cuh -- device-side building blocks shared by librq's kernels:
// inline-PTX wrappers (mbarrier, bulk async copy, programmatic dependent
// launch), bounded waits, and the in-register unpack of packed codes.
//
// Each unpack below turns stored codes into exact numbers (128 + u, 1024 + u,
// q); the kernels then apply the scales in their own arithmetic: rq_dequant
// forms w_hat = q * s exactly (the offline dequantization, RWKV-7 G1 1.5B
// int4 model card, summary paragraph), the products fold the scale into fp32
// sums, and agree with x * w_hat^T within the library's stated tolerance.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace rq {

// ---------------------------------------------------------------- status ---
// Bit flags of the device status word (one per device, read and cleared by
// rq_device_status). A bounded wait that gives up ORs its bit in and returns.
enum : unsigned {
    kStatusTmaWait = 1u << 0,    // waited too long for an async copy
    kStatusSlotWait = 1u << 1,   // waited too long for a ring slot to free
    kStatusMmaWait = 1u << 2,    // waited too long for a tensor-core commit
    kStatusTmem = 1u << 3,       // TMEM allocation did not succeed
    kStatusXWait = 1u << 4,      // waited too long for a staged activation buffer
    // 1u << 5: kStatusNotSpd (rq_internal.h), a Cholesky pivot that was not positive
};

// Output element idx of y: fp32, or rounded once to bf16 (nearest even).
__device__ __forceinline__ void store_y(void* y, size_t idx, float v, int bf16) {
    if (bf16) static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
    else static_cast<float*>(y)[idx] = v;
}

// One word per translation unit (internal linkage, so no device linking is
// needed); each kernel file exports a host accessor that reads and clears it.
static __device__ unsigned g_status = 0u;

// Default wall-clock bound of a device spin-wait, in nanoseconds (launches
// pass the bound they were given, which is this unless a test changed it).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// -------------------------------------------------------------- mbarrier ---
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// As mbar_try_wait, but a thread whose phase is not complete may be
// suspended for up to `hint_ns` (or until the phase completes) instead of the
// system-dependent default, so waiting warps leave the issue slots to the
// warps that compute.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete. Gives up after
// kWaitLimitNs, ORs `flag` into the device status word and returns false.
// With nap_ns > 0 the warp sleeps that long between polls: for waits off the
// critical path (a producer waiting for a free slot), so that polling does
// not take issue slots from the warps that compute.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned flag,
                                                  unsigned nap_ns = 0u,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (nap_ns) __nanosleep(nap_ns);
        if (mbar_try_wait_sleep(bar, parity, 1000u)) return true;
        if ((it & 15u) == 0u && globaltimer_ns() - t0 > limit_ns) {
            atomicOr(&g_status, flag);
            return false;
        }
    }
}

// ------------------------------------------------------ bulk async copy ---
// One contiguous global -> shared copy completed on an mbarrier (the untiled
// TMA form). dst, src and bytes must be multiples of 16. Loads with an L2
// evict-first policy: the packed weights are streamed once per call.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// -------------------------------------------- programmatic dependent launch
// The packed weights never depend on the previous kernel, so kernels prefetch
// them before grid_dep_wait(); x and y are touched only after it.
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------- loads ------
// Loads from 32-bit shared-memory addresses (no generic-to-shared conversion
// per access). Volatile keeps them after the barrier waits that guard them.
__device__ __forceinline__ uint4 lds128_a(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 lds128f_a(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float2 lds64f_a(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32_a(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16_a(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
// --------------------------------------------------------------- unpack ---
// int4 codes. A 32-bit word holds eight nibbles; nibble p (bits 4p..4p+3)
// is the code of weight k = 8i + p of that word (byte j: k = 2j low, 2j+1
// high). unpack_w4 turns the word into eight fp32 values 128 + u exactly:
// each nibble is placed in bits 16..19 under the exponent byte 0x43 (fp32
// 128.0, whose mantissa bit 16 weighs 1), one byte permute per value.
// Output order: f[0..3] = nibbles 0, 2, 4, 6 (low nibble of bytes 0..3),
//               f[4..7] = nibbles 1, 3, 5, 7 (high nibble of bytes 0..3).
constexpr uint32_t kW4Magic = 0x43000000u;  // 128.0f

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ void unpack_w4(uint32_t w, float f[8]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
    // prmt selector nibbles pick bytes of {b = magic (bytes 4..7), a (bytes 0..3)}:
    // result byte3 = 0x43 (selector 7), byte2 = a.byte_k, bytes1..0 = 0x00 (selector 4)
    f[0] = __uint_as_float(prmt(lo, kW4Magic, 0x7044u));
    f[1] = __uint_as_float(prmt(lo, kW4Magic, 0x7144u));
    f[2] = __uint_as_float(prmt(lo, kW4Magic, 0x7244u));
    f[3] = __uint_as_float(prmt(lo, kW4Magic, 0x7344u));
    f[4] = __uint_as_float(prmt(hi, kW4Magic, 0x7044u));
    f[5] = __uint_as_float(prmt(hi, kW4Magic, 0x7144u));
    f[6] = __uint_as_float(prmt(hi, kW4Magic, 0x7244u));
    f[7] = __uint_as_float(prmt(hi, kW4Magic, 0x7344u));
}
// int4 codes as bf16 pairs (the GEMV and dequant unpack). Pair j (0..3) of a
// word holds nibble j in its low half and nibble j+4 in its high half, each
// as the bf16 value 128 + u: the nibble lands in mantissa bits 0..3 under the
// exponent pattern 0x43 (bf16 128.0, mantissa bit 0 weighs 1). One shift and
// one three-input logic op per two weights.
constexpr uint32_t kW4PairMagic = 0x43004300u;

template <int J>
__device__ __forceinline__ uint32_t w4_pair(uint32_t w) {
    uint32_t d;
    const uint32_t v = J ? (w >> (4 * J)) : w;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v), "r"(0x000F000Fu), "r"(kW4PairMagic));  // (v & m) | c
    return d;
}

// fp32 value of the low / high bf16 half of a 32-bit word (exact).
__device__ __forceinline__ float bf16lo_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_f32(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// The eight values 128 + u_k of one code word, in natural k order, widened
// exactly from the bf16 pairs the GEMV multiplies (rq_dequant's unpack).
__device__ __forceinline__ void w4_word_values(uint32_t w, float o[8]) {
    const uint32_t r0 = w4_pair<0>(w), r1 = w4_pair<1>(w), r2 = w4_pair<2>(w), r3 = w4_pair<3>(w);
    o[0] = bf16lo_f32(r0); o[4] = bf16hi_f32(r0);
    o[1] = bf16lo_f32(r1); o[5] = bf16hi_f32(r1);
    o[2] = bf16lo_f32(r2); o[6] = bf16hi_f32(r2);
    o[3] = bf16lo_f32(r3); o[7] = bf16hi_f32(r3);
}

// int4 codes as fp16 pairs (the GEMV unpack). An fp16 mantissa has ten bits,
// so both nibbles of a byte fit under the exponent pattern 0x64 (fp16 1024.0,
// mantissa bit 0 weighs 1): masking nibble positions 0 and 4 of each 16-bit
// half gives (1024 + u), positions 1 and 5 give (1024 + 16 u). Pairs of word
// w: P0 = (k0, k4), P1 = (k1, k5) from w; P2 = (k2, k6), P3 = (k3, k7) from
// w >> 8. One shift and four three-input logic ops per eight weights.
constexpr uint32_t kW4HalfMagic = 0x64006400u;

__device__ __forceinline__ uint32_t lop_or_mask(uint32_t v, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v), "r"(m), "r"(kW4HalfMagic));  // (v & m) | c
    return d;
}

// c + a.half(AH) * b.half(BH) with fp16 operands and an fp32 accumulator; the
// product of two fp16 values is exact in fp32 (one rounding, in the add).
template <int AH, int BH>
__device__ __forceinline__ float fma_f16(uint32_t a, uint32_t b, float c) {
    float d;
    if (AH == 0 && BH == 0)
        asm("{ .reg .b16 a0, a1, b0, b1; mov.b32 {a0, a1}, %1; mov.b32 {b0, b1}, %2;"
            " fma.rn.f32.f16 %0, a0, b0, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else if (AH == 1 && BH == 0)
        asm("{ .reg .b16 a0, a1, b0, b1; mov.b32 {a0, a1}, %1; mov.b32 {b0, b1}, %2;"
            " fma.rn.f32.f16 %0, a1, b0, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else if (AH == 0 && BH == 1)
        asm("{ .reg .b16 a0, a1, b0, b1; mov.b32 {a0, a1}, %1; mov.b32 {b0, b1}, %2;"
            " fma.rn.f32.f16 %0, a0, b1, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else
        asm("{ .reg .b16 a0, a1, b0, b1; mov.b32 {a0, a1}, %1; mov.b32 {b0, b1}, %2;"
            " fma.rn.f32.f16 %0, a1, b1, %3; }" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}

// One code word against x_0..x_7 (fp16, natural-order pairs X.x = (x0, x1),
// X.y = (x2, x3), X.z = (x4, x5), X.w = (x6, x7)): lo += (1024 + u_k) x_k over
// even k, hi += (1024 + 16 u_k) x_k over odd k.
__device__ __forceinline__ void dot8_w4_f16(uint32_t w, uint4 X, float& lo, float& hi) {
    const uint32_t v = w >> 8;
    const uint32_t p0 = lop_or_mask(w, 0x000F000Fu), p1 = lop_or_mask(w, 0x00F000F0u);
    const uint32_t p2 = lop_or_mask(v, 0x000F000Fu), p3 = lop_or_mask(v, 0x00F000F0u);
    lo = fma_f16<0, 0>(p0, X.x, lo);   // k0
    hi = fma_f16<0, 1>(p1, X.x, hi);   // k1
    lo = fma_f16<0, 0>(p2, X.y, lo);   // k2
    hi = fma_f16<0, 1>(p3, X.y, hi);   // k3
    lo = fma_f16<1, 0>(p0, X.z, lo);   // k4
    hi = fma_f16<1, 1>(p1, X.z, hi);   // k5
    lo = fma_f16<1, 0>(p2, X.w, lo);   // k6
    hi = fma_f16<1, 1>(p3, X.w, hi);   // k7
}

// int8 codes. Byte k of a word is the code u = q + 128 of weight k. Each byte
// is placed in bits 8..15 under exponent byte 0x47 (fp32 32768.0, mantissa
// bit 8 weighs 1), giving 32768 + u; subtracting 32896 gives q exactly.
constexpr uint32_t kW8Magic = 0x47000000u;  // 32768.0f

__device__ __forceinline__ void unpack_w8(uint32_t w, float f[4]) {
    f[0] = __fsub_rn(__uint_as_float(prmt(w, kW8Magic, 0x7404u)), 32896.0f);
    f[1] = __fsub_rn(__uint_as_float(prmt(w, kW8Magic, 0x7414u)), 32896.0f);
    f[2] = __fsub_rn(__uint_as_float(prmt(w, kW8Magic, 0x7424u)), 32896.0f);
    f[3] = __fsub_rn(__uint_as_float(prmt(w, kW8Magic, 0x7434u)), 32896.0f);
}

// Superblock header: 6-bit field of group j (which = 0: scale, 1: min) from
// the 96-bit string held in words b0 (bits 0..31), b1 (32..63), b2 (64..95).
__device__ __forceinline__ uint32_t sb_field(uint32_t b0, uint32_t b1, uint32_t b2, int which, int j) {
    const int s = 48 * which + 6 * j;
    const uint32_t lo = s < 32 ? b0 : (s < 64 ? b1 : b2);
    const uint32_t hi = s < 32 ? b1 : (s < 64 ? b2 : 0u);
    return __funnelshift_r(lo, hi, s & 31) & 63u;
}

}  // namespace rq
