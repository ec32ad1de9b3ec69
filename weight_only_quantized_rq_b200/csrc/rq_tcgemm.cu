// rq_tcgemm.cu -- y = x * w_hat^T on the 5th-generation tensor cores, for
// activation blocks of 3 <= M <= 128 rows (small-M decode batches and
// prefill), for all three formats: int4 group-64, int8 group-16 and the int4
// asymmetric superblock (144-byte records of 8 groups of 32).
//
// Sources: RWKV-7 G1 1.5B int4 model card, summary paragraph (a tensor-core
// GEMM beside the int4 GEMV and small-M kernels; output bit-identical to the
// offline dequantization in the GEMV); rwkv_quant_nv project description,
// "Operator Optimization Details" (4096-wide decode shapes, 1 x 128 prefill,
// r/k/v projections in one kernel).
//
// Why tensor cores from M = 3: the int4 GEMV spends about 2.5 instructions
// per weight at M = 1; every further activation row adds at least one FMA per
// weight, so on the CUDA cores the product becomes ALU-bound long before the
// weight stream saturates HBM. With tcgen05.mma the per-weight cost is the
// dequantization alone, whatever M is.
//
// Design (B200):
//  * Tile: 128 weight rows (the MMA's M) x all activation rows (the MMA's N =
//    M rounded up to 16) x a K range, in stages of KS = 128 or 256 K. D =
//    [128][Mpad] fp32 accumulates in tensor memory (two buffers, so the
//    epilogue of one tile overlaps the main loop of the next).
//  * Dequantized weights never touch shared memory: the dequantizing threads
//    write the bf16 tile with tcgen05.st straight into a ring of A slots in
//    tensor memory, and tcgen05.mma takes A from there (the ".kind::f16 [d],
//    [a], b-desc" form). Shared memory carries only the codes and x (the B
//    operand, K-major with the 128-byte swizzle).
//  * One thread streams each stage with two tensor copies: the codes tile
//    ([128 rows][KS/2 or KS bytes], swizzled so that 32 threads reading the
//    same chunk of 32 rows hit distinct bank groups) and x (a 3-D box holding
//    all KS/64 atoms of the stage). Boxes have 128-byte rows wherever the
//    shape allows: the copy engine's cost grows with the number of box rows,
//    and rows of 64 bytes or less cannot keep HBM busy.
//  * Scales bypass shared memory: each dequantizing thread keeps the scales
//    of its row for the next few stages in registers, loaded ahead of use
//    through a cursor that follows the CTA's sequence of tiles.
//  * Warp roles (23 warps): warps 0 and 1 issue the MMAs (the whole warp
//    runs the loop with warp-uniform operands; one elected lane issues the
//    four MMAs of a 64-K atom). A single issuing thread cannot keep up with
//    MMAs of small N, so for M <= 64 the two warps take alternate atoms into
//    two accumulators that the epilogue adds in a fixed order. Warp 0 also
//    allocates tensor memory. Warp 2 issues the tensor copies; warps 3-18
//    dequantize (warp w owns tensor-memory lanes 32 (w % 4) .. +31, i.e. one
//    weight row per thread); warps 19-22 read D back with tcgen05.ld and
//    store y.
//  * Dequantizing groups: where the A ring has room (3 or more slots; 5 or
//    more at 128-K stages), the sixteen dequantizing warps form 2 (or 4)
//    groups that take the stages in turn, each warp writing 2 (or 4) K
//    quarters of its group's stage. When all sixteen warps shared every
//    stage, they met every barrier together and the SM sub-partitions sat
//    idle between stages (traced: about 1.8 thousand cycles per 256-K stage,
//    half of them outside the arithmetic); with groups out of phase one
//    group's waits overlap another's arithmetic, and a warp meets fewer
//    barriers per weight. Where the ring is smaller (M > 32 at 256-K stages,
//    M > 64 at 128-K stages) all sixteen share each stage, a quarter each.
//  * int4: a lop3 with mask and exponent pattern places nibble pairs in fp16
//    mantissas: (1024 + u) for the low nibble of a byte, (64 + u) for the high
//    nibble; fma.rn.f32.f16 against the fp16 scale and an exact fp32 offset
//    gives q * s exactly; cvt.rn.bf16x2.f32 rounds each pair to bf16 in natural
//    k order (one rounding per weight). int8: a byte permute gives fp16
//    (1024 + u), the same FMA gives q * s. Superblock: each 256-K stage holds
//    one 144-byte record per row (box rows of 144 bytes, unswizzled: the row
//    stride of nine 16-byte chunks keeps 8 consecutive rows on distinct bank
//    groups); a thread reads the record header and its two 32-weight groups,
//    forms S = d * sc and M = dmin * m in fp32, places nibbles under an fp32
//    exponent (128 + u) with a byte permute and evaluates S u - M with one FFMA
//    before the bf16 rounding.
//  * Work: a persistent CTA per SM walks the tiles of all products of the
//    launch (largest K first). A single product with fewer tiles than about
//    half the SMs is split along K over a thread-block cluster; the partial
//    tiles are summed through distributed shared memory in cluster-rank order
//    (deterministic; no global workspace).
//  * Every mbarrier wait is bounded; on a timeout a status bit is set, the
//    role leaves its loop, and tensor memory is always released.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kTcRows = 128;        // weight rows per tile (MMA M)
constexpr int kTcMaxStages = 16;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxAS = 8;           // A slots at most (the accumulators take the first columns)
constexpr int kDqThreads = 512;     // warps 3-18
constexpr int kEpiThreads = 128;    // warps 19-22
constexpr int kTcThreads = 736;
constexpr int kScaleAhead = 2;      // stages of scales held in registers ahead of use
constexpr size_t kTcSmemMax = 227 * 1024;


struct __align__(64) TcItem {       // one product of a launch
    CUtensorMap cmap;               // codes plane: uint8 [N][crb], box [128 rows][RB bytes], swizzled
    CUtensorMap xmap;               // x: bf16 [M][K] viewed as [K/64][M][64], box [KS/64][xrows][64]
    const uint8_t* scales;          // fp16 [N][K / G]
    void* y;                        // fp32 [M][N], or bf16 when ybf16
    int ybf16;
    int K, N, T;                    // T = stages = ceil(K / KS)
    int unit0;                      // index of this product's first tile
    uint32_t srb;                   // scale bytes per row
};

// Products per launch (the tensor maps travel in the kernel parameters, which
// hold at most 32 KB); larger batches take several launches.
constexpr int kTcMaxItems = 96;

template <int MAXI>
struct TcArgs {
    TcItem it[MAXI];
    int count, units, M, Mpad, split, R;
    int niss;                       // MMA-issuing warps (two accumulators when Mpad <= 64)
    int AS;                         // A slots in tensor memory
    uint32_t A0;                    // first tensor-memory column of the A slots (after 2 * niss accumulators)
    int ng;                         // groups of dequantizing warps that take the stages in turn (1, 2 or 4)
    uint32_t stage_bytes, x_atom, codes_off, bar_off, tx_bytes;
    unsigned long long wait_ns;     // bound of every device wait
    int test_flags;                 // kTestNoCopies: the copy thread issues nothing (tests the waits)
};

// ------------------------------------------------------------ PTX wrappers
// Tensor copies global -> shared, completed on an mbarrier.
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(dst), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart, descriptor version 1, base offset 0 (atoms are
// 1024-byte aligned).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, both K-major,
// N = n, M = 128.
__device__ __forceinline__ uint32_t mma_idesc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);
}

// D[tmem d] (+)= A[tmem a] * B[smem desc b]^T for the four MMAs (K = 16
// each) of one 64-K atom, issued by one elected lane of a converged warp (the
// operands are warp-uniform, so they stay in uniform registers and the MMAs
// issue back to back): A columns a, a+8, a+16, a+24; B 32 bytes
// further along the swizzled rows each time (+2 in the descriptor's address
// field, which stays below 2^14 for any shared-memory address). The first
// overwrites D when acc is 0.
__device__ __forceinline__ void mma_atom(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p, q, t;\n .reg .b64 b1, b2, b3;\n .reg .b32 a1, a2, a3;\n"
        " elect.sync _|q, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.eq.u32 t, 0, 0;\n"
        " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
        " add.u32 a1, %1, 8;\n add.u32 a2, %1, 16;\n add.u32 a3, %1, 24;\n"
        " @q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
        " @q tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, t;\n"
        " @q tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, t;\n"
        " @q tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, t;\n}"
        :: "r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

// The mbarrier receives one arrival when all earlier MMAs of the elected lane
// have completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "{\n .reg .pred q;\n elect.sync _|q, 0xffffffff;\n"
        " @q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}"
        :: "r"(smem_u32(bar)) : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
           "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
           "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
           "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
// 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16};"
        :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
           "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t saddr, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(saddr), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
    return v;
}

// Read-only global loads of scale words (the planes are not written while a
// product runs).
__device__ __forceinline__ uint32_t ldg_nc_u16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ldg_nc_u64(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
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

// (v & m) | c in one three-input logic op.
__device__ __forceinline__ uint32_t lop_mask_or(uint32_t v, uint32_t m, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(v), "r"(m), "r"(c));
    return d;
}

// Byte position of 16-byte chunk c of code row r in a stage, as the tensor
// copy's swizzle lays it out: rows of 128 bytes use the 128-byte pattern
// (chunk c ^ (r % 8)), rows of 64 bytes the 64-byte pattern (c ^ (r / 2 % 4)).
template <int RB>
__device__ __forceinline__ uint32_t code_pos(int r, int c) {
    return RB == 128 ? (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4))
         : RB == 64 ? (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4))
                    : (uint32_t)(r * RB + (c << 4));                       // superblock records: unswizzled
}

// 8 NW int4 weights (NW code words, one fp16 scale) -> 4 NW bf16 pairs in
// natural k order.
template <int NW>
__device__ __forceinline__ void dq_w4(const uint32_t (&w)[NW], uint16_t sb, uint32_t (&o)[4 * NW]) {
    const float sf = __half2float(__ushort_as_half(sb));
    const float ce = __fmul_rn(-1032.0f, sf), co = __fmul_rn(-72.0f, sf);   // exact
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        const uint32_t v = w[i] >> 8;
        // low nibbles of bytes 0 and 2 (k0, k4) as 1024 + u; high nibbles (k1, k5) as 64 + u
        const uint32_t p0 = lop_mask_or(w[i], 0x000F000Fu, 0x64006400u);
        const uint32_t p1 = lop_mask_or(w[i], 0x00F000F0u, 0x54005400u);
        const uint32_t p2 = lop_mask_or(v, 0x000F000Fu, 0x64006400u);   // k2, k6
        const uint32_t p3 = lop_mask_or(v, 0x00F000F0u, 0x54005400u);   // k3, k7
        const float d0 = fma_h<0>(p0, sb, ce), d4 = fma_h<1>(p0, sb, ce);
        const float d1 = fma_h<0>(p1, sb, co), d5 = fma_h<1>(p1, sb, co);
        const float d2 = fma_h<0>(p2, sb, ce), d6 = fma_h<1>(p2, sb, ce);
        const float d3 = fma_h<0>(p3, sb, co), d7 = fma_h<1>(p3, sb, co);
        o[4 * i + 0] = pack_bf16(d0, d1);
        o[4 * i + 1] = pack_bf16(d2, d3);
        o[4 * i + 2] = pack_bf16(d4, d5);
        o[4 * i + 3] = pack_bf16(d6, d7);
    }
}

// 32 int8 weights (32 code bytes, two fp16 scales, one per 16 weights) -> 16
// bf16 pairs.
__device__ __forceinline__ void dq_w8(const uint4 (&c)[2], uint32_t sc, uint32_t (&o)[16]) {
    const uint16_t s16[2] = {(uint16_t)(sc & 0xffffu), (uint16_t)(sc >> 16)};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const uint16_t sb = s16[g];
        const float cf = __fmul_rn(-1152.0f, __half2float(__ushort_as_half(sb)));   // exact
        const uint32_t w[4] = {c[g].x, c[g].y, c[g].z, c[g].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // bytes -> fp16 (1024 + u); (1024 + u) s - 1152 s = q s with u = q + 128
            const uint32_t e0 = prmt(w[i], 0x6464u, 0x4140u), e1 = prmt(w[i], 0x6464u, 0x4342u);
            o[8 * g + 2 * i] = pack_bf16(fma_h<0>(e0, sb, cf), fma_h<1>(e0, sb, cf));
            o[8 * g + 2 * i + 1] = pack_bf16(fma_h<0>(e1, sb, cf), fma_h<1>(e1, sb, cf));
        }
    }
}

// 64 superblock weights: groups 2h and 2h+1 of a 144-byte record (header
// hd = fp16 d, fp16 dmin, 96-bit string of 6-bit sc_j / m_j; c0, c1 = the
// groups' 16 code bytes each) -> 32 bf16 pairs. w = S u - M with S = d sc_j,
// M = dmin m_j (both exact in fp32); u from the nibble under the fp32 exponent
// of 128: (128 + u) S + (-128 S - M), then one rounding to bf16.
__device__ __forceinline__ void dq_sb32(const uint4 hd, const uint4 c0, const uint4 c1, int h, uint32_t (&o)[32]) {
    const float d = __half2float(__ushort_as_half((uint16_t)(hd.x & 0xffffu)));
    const float dmin = __half2float(__ushort_as_half((uint16_t)(hd.x >> 16)));
#pragma unroll
    for (int gl = 0; gl < 2; ++gl) {
        const int j = 2 * h + gl;
        const float S = __fmul_rn(d, (float)sb_field(hd.y, hd.z, hd.w, 0, j));
        const float Mv = __fmul_rn(dmin, (float)sb_field(hd.y, hd.z, hd.w, 1, j));
        const float c = __fsub_rn(__fmul_rn(-128.0f, S), Mv);
        const uint4 cw = gl == 0 ? c0 : c1;
        const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float f[8];
            unpack_w4(w[i], f);            // f[0..3]: k = 0, 2, 4, 6; f[4..7]: k = 1, 3, 5, 7 (128 + u)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[16 * gl + 4 * i + e] = pack_bf16(__fmaf_rn(f[e], S, c), __fmaf_rn(f[4 + e], S, c));
        }
    }
}

// 5- and 6-bit superblock codes: the high-bit plane of one 32-bit word of low
// nibbles (eight weights k = 0..7) becomes two words whose byte m holds the
// high bits of weight 2m (hl) or 2m + 1 (hh) at bit 4 and up, so that OR-ing
// them into the unpacked nibbles gives bytes 0..63 that the fp32 magic turns
// into 128 + q exactly.
// 5 bits: pw is the plane byte, bit k for weight k. The multiply moves bit 2m
// to bit 8m + 4; the other partial products land elsewhere (and collide only
// at bits 10, 16, 22, whose carries stop at 11, 17, 23), so the mask keeps
// exactly the wanted bits.
// 6 bits: pw holds 16 plane bits, bits 2k..2k+1 for weight k. After masking,
// nibble m of e holds the pair of weight 2m; the byte permute places nibble m
// in the high half of byte m (the low halves are masked off where used).
template <int BITS>
__device__ __forceinline__ void sb_high(uint32_t pw, uint32_t& hl, uint32_t& hh) {
    if (BITS == 5) {
        hl = ((pw & 0x55u) * 0x00410410u) & 0x10101010u;
        hh = (((pw >> 1) & 0x55u) * 0x00410410u) & 0x10101010u;
    } else {
        const uint32_t e = pw & 0x3333u, o = (pw >> 2) & 0x3333u;
        hl = prmt(e << 4, e, 0x5140u);
        hh = prmt(o << 4, o, 0x5140u);
    }
}

// (a & 0x0F0F0F0F) | (b & 0xF0F0F0F0)
__device__ __forceinline__ uint32_t merge_nib(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(0x0F0F0F0Fu));
    return d;
}

// 64 weights of a 5- or 6-bit record (groups 2h, 2h + 1): as dq_sb32, with
// the high bits of each code from the plane words pl (two per group for 6
// bits: words 2gl, 2gl + 1 of pl; one byte per code word for 5 bits).
template <int BITS>
__device__ __forceinline__ void dq_sbw(const uint4 hd, const uint4 c0, const uint4 c1, const uint32_t (&pl)[4], int h,
                                       uint32_t (&o)[32]) {
    const float d = __half2float(__ushort_as_half((uint16_t)(hd.x & 0xffffu)));
    const float dmin = __half2float(__ushort_as_half((uint16_t)(hd.x >> 16)));
#pragma unroll
    for (int gl = 0; gl < 2; ++gl) {
        const int j = 2 * h + gl;
        const float S = __fmul_rn(d, (float)sb_field(hd.y, hd.z, hd.w, 0, j));
        const float Mv = __fmul_rn(dmin, (float)sb_field(hd.y, hd.z, hd.w, 1, j));
        const float c = __fsub_rn(__fmul_rn(-128.0f, S), Mv);
        const uint4 cw = gl == 0 ? c0 : c1;
        const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t pw = BITS == 5 ? (pl[gl] >> (8 * i)) & 0xffu : (pl[2 * gl + (i >> 1)] >> (16 * (i & 1))) & 0xffffu;
            uint32_t hl, hh;
            sb_high<BITS>(pw, hl, hh);
            const uint32_t lo = merge_nib(w[i], hl), hi = merge_nib(w[i] >> 4, hh);
            float f[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                f[e] = __uint_as_float(prmt(lo, kW4Magic, 0x7044u + 0x100u * e));
                f[4 + e] = __uint_as_float(prmt(hi, kW4Magic, 0x7044u + 0x100u * e));
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[16 * gl + 4 * i + e] = pack_bf16(__fmaf_rn(f[e], S, c), __fmaf_rn(f[4 + e], S, c));
        }
    }
}

// 32 6-bit symmetric weights (half of a 64-weight chunk: 16 low-nibble bytes
// c, 8 plane bytes pl; two fp16 scales, one per 16 weights) -> 16 bf16 pairs.
// Each code byte u = q + 32 (low nibble plus plane bits 4..5 merged as for
// the wider superblock codes) goes under the fp16 exponent of 1024:
// (1024 + u) s - 1056 s = q s, exact in fp32, then one rounding to bf16.
__device__ __forceinline__ void dq_w6(const uint4 c, const uint2 pl, uint32_t sc, uint32_t (&o)[16]) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    const uint32_t pw[2] = {pl.x, pl.y};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const uint16_t sb = (uint16_t)(g ? sc >> 16 : sc & 0xffffu);
        const float cf = __fmul_rn(-1056.0f, __half2float(__ushort_as_half(sb)));   // exact
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
            const int i = 2 * g + ii;
            uint32_t hl, hh;
            sb_high<6>((pw[i >> 1] >> (16 * (i & 1))) & 0xffffu, hl, hh);
            const uint32_t lo = merge_nib(w[i], hl), hi = merge_nib(w[i] >> 4, hh);   // u of weights 0,2,4,6 / 1,3,5,7
            const uint32_t e0 = lop_mask_or(lo, 0x00FF00FFu, 0x64006400u);        // weights 0, 4
            const uint32_t e1 = lop_mask_or(lo >> 8, 0x00FF00FFu, 0x64006400u);   // weights 2, 6
            const uint32_t d0 = lop_mask_or(hi, 0x00FF00FFu, 0x64006400u);        // weights 1, 5
            const uint32_t d1 = lop_mask_or(hi >> 8, 0x00FF00FFu, 0x64006400u);   // weights 3, 7
            const float v0 = fma_h<0>(e0, sb, cf), v4 = fma_h<1>(e0, sb, cf);
            const float v2 = fma_h<0>(e1, sb, cf), v6 = fma_h<1>(e1, sb, cf);
            const float v1 = fma_h<0>(d0, sb, cf), v5 = fma_h<1>(d0, sb, cf);
            const float v3 = fma_h<0>(d1, sb, cf), v7 = fma_h<1>(d1, sb, cf);
            o[4 * i + 0] = pack_bf16(v0, v1);
            o[4 * i + 1] = pack_bf16(v2, v3);
            o[4 * i + 2] = pack_bf16(v4, v5);
            o[4 * i + 3] = pack_bf16(v6, v7);
        }
    }
}

// ------------------------------------------------------------ work units
struct Unit { int item, n0, t0, t1; };

template <class P>
__device__ __forceinline__ bool get_unit(const P& p, int i, Unit& u) {
    if (p.split > 1) {                       // one tile, one K range per CTA of the cluster
        if (i > 0) return false;
        const int tile = (int)blockIdx.x / p.split, j = (int)cluster_rank();
        const int T = p.it[0].T;
        u.item = 0;
        u.n0 = tile * kTcRows;
        u.t0 = (int)((long long)T * j / p.split);
        u.t1 = (int)((long long)T * (j + 1) / p.split);
        return true;
    }
    const int g = (int)blockIdx.x + i * (int)gridDim.x;
    if (g >= p.units) return false;
    int lo = 0, hi = p.count - 1;            // last product whose first tile is <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.it[mid].unit0 <= g) lo = mid;
        else hi = mid - 1;
    }
    u.item = lo;
    u.n0 = (g - p.it[lo].unit0) * kTcRows;
    u.t0 = 0;
    u.t1 = p.it[lo].T;
    return true;
}

// The scales one dequantizing thread needs at each stage, read from global
// memory kScaleAhead stages before use. The cursor walks the same (tile,
// stage) sequence as every role of the CTA. Per stage a thread takes a
// quarter of the stage's K: int4 one scale (64 weights at 256-K stages, 32 at
// 128-K stages), int8 two (32 weights).
template <int FMT, int KS, class P>
struct ScaleCursor {
    const P* p;
    int ui, t;
    Unit u;
    bool valid;
    const uint8_t* row;      // this thread's scale row in the current tile (nullptr past N)
    const uint8_t* spare;    // a valid address to load from when there is no scale
    int groups;              // groups per row (K / G)
    int r, h;                // weight row in the tile, quarter of the stage

    __device__ __forceinline__ void enter() {
        if (!valid) return;
        const TcItem& it = p->it[u.item];
        const int n = u.n0 + r;
        row = n < it.N ? it.scales + (size_t)n * it.srb : nullptr;
        groups = it.K / sym_group(FMT);
        t = u.t0;
    }
    __device__ __forceinline__ void start(const P* prm, int rr, int hh) {
        p = prm;
        r = rr;
        h = hh;
        spare = prm->it[0].scales;
        ui = 0;
        valid = get_unit(*p, 0, u);
        enter();
    }
    // Issues the load of the current stage's scale word(s) into v (from a
    // harmless address when there is none, with mask 0), then advances one
    // stage. The value is only combined with the mask where it is used, so
    // nothing waits for the load here.
    __device__ __forceinline__ void next(uint32_t& v, uint32_t& mask) {
        const uint8_t* a = spare;
        bool in = false;
        if (valid && row) {
            const int gi = sym_group(FMT) == 64 ? (KS == 128 ? 2 * t + (h >> 1) : 4 * t + h) : 8 * t + 2 * h;
            in = gi < groups;
            if (in) a = row + 2 * gi;
        }
        if (is_sb(FMT)) v = 0u;                           // scales travel inside the records
        else if (sym_group(FMT) == 64) v = ldg_nc_u16(a);
        else v = ldg_nc_u32(a);
        mask = in ? 0xffffffffu : 0u;
        if (valid && ++t >= u.t1) {
            ++ui;
            valid = get_unit(*p, ui, u);
            enter();
        }
    }
};

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity, sleeping about nap_ns between
// tests. A blocking try_wait keeps its warp issuing while it polls, and with
// 23 warps per CTA most of them wait most of the time: sleeping waiters leave
// the issue slots to the warps that dequantize. Gives up after kWaitLimitNs,
// ORs `flag` into the status word and returns false.
__device__ __forceinline__ bool nap_wait(uint64_t* bar, uint32_t parity, unsigned flag, unsigned nap_ns,
                                         unsigned long long lim) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(nap_ns);
        if (mbar_test(bar, parity)) return true;
        if ((it & 63u) == 0u && globaltimer_ns() - t0 > lim) {
            atomicOr(&g_status, flag);
            return false;
        }
    }
}

// Bounded wait by every lane of a warp; true only if all lanes saw the phase.
// nap_ns == 0: waits on the critical path (dequantizing warps, MMA issue) use
// the suspending try_wait, which measured faster there than sleeping between
// tests; the long waits (epilogue, drains) sleep.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned flag, unsigned nap_ns,
                                          unsigned long long lim) {
    const bool ok = nap_ns ? nap_wait(bar, parity, flag, nap_ns, lim) : mbar_wait_bounded(bar, parity, flag, 0u, lim);
    return __all_sync(0xffffffffu, ok);
}

// Sleep between phase tests, by waiter (ns; 0 = suspending try_wait).
constexpr unsigned kNapCritical = 0, kNapLoader = 64, kNapEpilogue = 512, kNapDrain = 256;

// Dequantizing warps in NG groups (2 or 4) that take the CTA's stages in
// turn: in its group's stage, warp (q, h) writes rows 32q .. 32q+31 of the
// NG consecutive K quarters from (h mod 4/NG) NG on (64 weights per quarter
// at 256-K int4 stages, 32 otherwise). Compared with all sixteen warps
// sharing every stage, a warp meets 1/NG as many barriers per weight, and
// the groups run out of phase, so one group's waits overlap another's
// arithmetic. Needs more than NG A slots. A wait that runs out ends the role
// (its status bit is set).
template <int FMT, int KS, int NG, int MAXI>
__device__ __forceinline__ void dequant_groups(const TcArgs<MAXI>& p, const uint8_t* smem, uint32_t tmem,
                                               uint64_t* full, uint64_t* afull, uint64_t* aempty, int warp,
                                               int lane) {
    constexpr int RB = FMT == kFmtW4G64 ? KS / 2 : is_w8(FMT) ? KS : FMT == kFmtW6G16 ? KS / 64 * 48
                                                                   : sb_record(FMT);   // code bytes per row and stage
    constexpr uint32_t QCOLS = KS / 8;                       // tensor-memory columns per K quarter
    constexpr int SUBS = 4 / NG;                             // warps of a group per lane quarter
    const int q = warp & 3, hh = (warp - 3) >> 2, grp = hh / SUBS, h0 = (hh % SUBS) * NG;
    const int r = 32 * q + lane;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    const int R = p.R, AS = p.AS;
    Unit u;
    int ui = 0, t = 0, slot = 0, wrap = 0, aslot = 0, awrap = 0;
    bool live = get_unit(p, 0, u);
    if (live) t = u.t0;
    auto step = [&]() {                                      // to the CTA's next stage
        if (++slot == R) { slot = 0; ++wrap; }
        if (++aslot == AS) { aslot = 0; ++awrap; }
        if (++t >= u.t1) {
            live = get_unit(p, ++ui, u);
            if (live) t = u.t0;
        }
    };
    // Scale words of this thread's row for quarters h0 .. h0 + NG - 1 at the
    // current stage, loaded together: group-16 formats two fp16 scales per
    // quarter (8 bytes per pair of quarters); int4 g64 at 256-K stages one per
    // quarter (NG = 2: one 4-byte load); g64 at 128-K stages one per two
    // quarters. The superblock formats carry theirs in the records. Rows past
    // N and groups past K get zero (and nothing is read there).
    constexpr int NW = is_sb(FMT) ? 1 : sym_group(FMT) == 16 ? NG : 1;
    auto load_scales = [&](uint32_t (&w)[NW]) {
#pragma unroll
        for (int k = 0; k < NW; ++k) w[k] = 0u;
        if constexpr (!is_sb(FMT)) {
            const TcItem& it = p.it[u.item];
            const int n = u.n0 + r;
            if (n >= it.N) return;
            const int groups = it.K / sym_group(FMT);
            const uint8_t* row = it.scales + (size_t)n * it.srb;
            if constexpr (sym_group(FMT) == 16) {            // K % 64 == 0: pairs of quarters are whole or absent
#pragma unroll
                for (int k = 0; k < NG; k += 2) {
                    const int gi = 8 * t + 2 * (h0 + k);
                    if (gi < groups) {
                        const uint2 v = ldg_nc_u64(row + 2 * gi);
                        w[k] = v.x;
                        w[k + 1] = v.y;
                    }
                }
            } else if constexpr (KS == 256) {                // K % 256 == 0: both groups exist
                w[0] = ldg_nc_u32(row + 2 * (4 * t + h0));
            } else {
                const int gi = 2 * t + (h0 >> 1);
                if (NG == 4 && gi + 1 < groups && (it.srb & 3u) == 0u) w[0] = ldg_nc_u32(row + 2 * gi);
                else if (gi < groups)
                    w[0] = ldg_nc_u16(row + 2 * gi) | (NG == 4 && gi + 1 < groups ? ldg_nc_u16(row + 2 * gi + 2) << 16 : 0u);
            }
        }
    };
    auto scale_at = [](const uint32_t (&w)[NW], int j) -> uint32_t {
        if constexpr (is_sb(FMT)) return 0u;
        else if constexpr (sym_group(FMT) == 16) return w[j];
        else if constexpr (KS == 256) return j & 1 ? w[0] >> 16 : w[0] & 0xffffu;
        else return NG == 4 && j >= 2 ? w[0] >> 16 : w[0] & 0xffffu;
    };
    for (int k = 0; k < grp && live; ++k) step();
    uint32_t sw[NW];
    if (live) load_scales(sw);
    while (live) {
        if (!warp_wait(&full[slot], (uint32_t)wrap & 1u, kStatusTmaWait, kNapCritical, p.wait_ns)) return;
        const int a = aslot;
        if (awrap && !warp_wait(&aempty[a], (uint32_t)(awrap - 1) & 1u, kStatusMmaWait, kNapCritical, p.wait_ns))
            return;
        const uint8_t* cs = smem + (size_t)slot * p.stage_bytes + p.codes_off;
        const uint32_t ta0 = tmem + tl + p.A0 + (uint32_t)a * (KS / 2);
        // the stage's code loads first, so that their latency overlaps the
        // bookkeeping below (a tensor-memory store would order later
        // shared-memory loads after it)
        uint4 hd = make_uint4(0u, 0u, 0u, 0u), c[NG][2];
        uint32_t pl[NG][4];
#pragma unroll
        for (int j = 0; j < NG; ++j) {
            const int hq = h0 + j;
            if constexpr (is_sb(FMT)) {                      // 64 weights: groups 2hq, 2hq+1 of the record
                if (j == 0) hd = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, 0));
                c[j][0] = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, 1 + 2 * hq));
                c[j][1] = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, 2 + 2 * hq));
                const uint32_t pp = code_pos<RB>(r, 0) + 144u + (FMT == kFmtW6SB32 ? 16u : 8u) * (uint32_t)hq;
                if constexpr (FMT == kFmtW6SB32) {
                    const uint4 v = *reinterpret_cast<const uint4*>(cs + pp);
                    pl[j][0] = v.x; pl[j][1] = v.y; pl[j][2] = v.z; pl[j][3] = v.w;
                } else if constexpr (FMT == kFmtW5SB32) {
                    const uint2 v = *reinterpret_cast<const uint2*>(cs + pp);
                    pl[j][0] = v.x; pl[j][1] = v.y; pl[j][2] = 0u; pl[j][3] = 0u;
                }
            } else if constexpr (FMT == kFmtW4G64 && KS == 128) {   // 32 weights: chunk hq, half a group
                c[j][0] = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, hq));
            } else if constexpr (FMT == kFmtW6G16) {          // 32 weights: two groups of 16
                c[j][0] = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, 3 * (hq >> 1) + (hq & 1)));
                const uint2 v = *reinterpret_cast<const uint2*>(cs + code_pos<RB>(r, 3 * (hq >> 1) + 2) +
                                                                8u * (uint32_t)(hq & 1));
                pl[j][0] = v.x; pl[j][1] = v.y;
            } else {                                          // int4 at 256-K stages (64 weights) or int8 (32):
                c[j][0] = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, 2 * hq));   // chunks 2hq, 2hq+1
                c[j][1] = *reinterpret_cast<const uint4*>(cs + code_pos<RB>(r, 2 * hq + 1));
            }
        }
        uint32_t sc[NG];
#pragma unroll
        for (int j = 0; j < NG; ++j) sc[j] = scale_at(sw, j);
#pragma unroll
        for (int k = 0; k < NG; ++k)                         // to this group's next stage
            if (live) step();
        if (live) load_scales(sw);                           // loads while this stage is dequantized
#pragma unroll
        for (int j = 0; j < NG; ++j) {
            const int hq = h0 + j;
            const uint32_t ta = ta0 + (uint32_t)hq * QCOLS;
            if constexpr (is_sb(FMT)) {
                uint32_t o[32];
                if constexpr (FMT == kFmtW4SB32) dq_sb32(hd, c[j][0], c[j][1], hq, o);
                else dq_sbw<FMT == kFmtW6SB32 ? 6 : 5>(hd, c[j][0], c[j][1], pl[j], hq, o);
                tmem_st32(ta, o);
            } else if constexpr (FMT == kFmtW4G64 && KS == 256) {
                const uint32_t wv[8] = {c[j][0].x, c[j][0].y, c[j][0].z, c[j][0].w,
                                        c[j][1].x, c[j][1].y, c[j][1].z, c[j][1].w};
                uint32_t o[32];
                dq_w4<8>(wv, (uint16_t)sc[j], o);
                tmem_st32(ta, o);
            } else if constexpr (FMT == kFmtW4G64) {
                const uint32_t wv[4] = {c[j][0].x, c[j][0].y, c[j][0].z, c[j][0].w};
                uint32_t o[16];
                dq_w4<4>(wv, (uint16_t)sc[j], o);
                tmem_st16(ta, o);
            } else if constexpr (FMT == kFmtW6G16) {
                uint32_t o[16];
                dq_w6(c[j][0], make_uint2(pl[j][0], pl[j][1]), sc[j], o);
                tmem_st16(ta, o);
            } else {
                uint32_t o[16];
                dq_w8(c[j], FMT == kFmtW8G64 ? sc[j] * 0x10001u : sc[j], o);   // g64: one scale for both halves
                tmem_st16(ta, o);
            }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&afull[a]);
    }
}

template <int FMT, int KS, int MAXI>
__global__ void __launch_bounds__(kTcThreads, 1) tc_kernel(const __grid_constant__ TcArgs<MAXI> p) {
    constexpr int RB = FMT == kFmtW4G64 ? KS / 2 : is_w8(FMT) ? KS : FMT == kFmtW6G16 ? KS / 64 * 48
                                                                   : sb_record(FMT);   // code bytes per row and stage
    const int AS = p.AS;                                     // A slots (KS / 2 columns each)
    constexpr uint32_t ACOLS = KS / 2;
    constexpr uint32_t QCOLS = ACOLS / 4;                    // columns one dequantizing thread writes per stage
    constexpr int NAT = KS / 64;                             // 64-K atoms per stage
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);   // 1024-byte aligned base
    const uint32_t base = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = p.R, niss = p.niss;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint64_t* empty = full + kTcMaxStages;
    uint64_t* afull = empty + kTcMaxStages;
    uint64_t* aempty = afull + kMaxAS;
    uint64_t* dfull = aempty + kMaxAS;
    uint64_t* dempty = dfull + 2;
    uint64_t* mmadone = dempty + 2;                          // one per issuer
    uint32_t* tslot = reinterpret_cast<uint32_t*>(mmadone + 2);
    const int Mpad = p.Mpad;

    if (tid == 0) {
        for (int s = 0; s < R; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], (uint32_t)niss);
        }
        for (int a = 0; a < AS; ++a) {
            mbar_init(&afull[a], (uint32_t)(kDqThreads / p.ng));
            mbar_init(&aempty[a], (uint32_t)niss);
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(&dfull[d], (uint32_t)niss);
            mbar_init(&dempty[d], kEpiThreads);
        }
        mbar_init(&mmadone[0], 1);
        mbar_init(&mmadone[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_u32(tslot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    grid_dep_launch();

    if (warp < 2) {
        // ------------------------------------------------------ MMA issue
        // Issuer w (warps 0 and 1; only warp 0 when niss == 1) takes atoms
        // w, w + niss, ... of every stage into its own accumulator; the whole
        // warp runs the loop and one elected lane issues.
        const int w = warp;
        if (w < niss) {
            const uint32_t idesc = mma_idesc(Mpad);
            bool ok = true;
            uint32_t g = 0;
            int slot = 0, aslot = 0, awrap = 0;
            Unit u;
            for (int ui = 0; ok && get_unit(p, ui, u); ++ui) {
                const int d = ui & 1;
                if (ui >= 2 && !warp_wait(&dempty[d], (uint32_t)((ui >> 1) - 1) & 1u, kStatusMmaWait, kNapDrain, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + (uint32_t)((d * niss + w) * Mpad);
                for (int t = u.t0; t < u.t1; ++t, ++g) {
                    const int a = aslot;
                    if (!warp_wait(&afull[a], (uint32_t)awrap & 1u, kStatusTmaWait, kNapCritical, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xs = base + (uint32_t)slot * p.stage_bytes;
                    const uint32_t acol = tmem + p.A0 + (uint32_t)a * ACOLS;
                    const uint64_t bd = sw128_desc(xs);
                    const uint64_t xstep = (uint64_t)(p.x_atom >> 4);
                    for (int at = w; at < NAT; at += niss)
                        mma_atom(dcol, acol + 32u * (uint32_t)at, bd + xstep * (uint64_t)at, idesc,
                                 (t != u.t0 || at != w) ? 1u : 0u);
                    mma_commit(&empty[slot]);
                    mma_commit(&aempty[a]);
                    if (++slot == R) slot = 0;
                    if (++aslot == AS) { aslot = 0; ++awrap; }
                }
                if (ok) mma_commit(&dfull[d]);
            }
            mma_commit(&mmadone[w]);
            warp_wait(&mmadone[w], 0u, kStatusMmaWait, kNapDrain, p.wait_ns);      // no MMA in flight at teardown
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ tensor copies (one thread)
        if (lane == 0) {
            grid_dep_wait();                                 // x comes from earlier kernels
            int slot = 0, wrap = 0, issued = 0;
            Unit u;
            bool ok = true;
            for (int ui = 0; ok && get_unit(p, ui, u); ++ui) {
                const TcItem& it = p.it[u.item];
                asm volatile("prefetch.tensormap [%0];" :: "l"(&it.cmap) : "memory");
                asm volatile("prefetch.tensormap [%0];" :: "l"(&it.xmap) : "memory");
                for (int t = u.t0; t < u.t1; ++t) {
                    if (wrap && !nap_wait(&empty[slot], (uint32_t)(wrap - 1) & 1u, kStatusSlotWait, kNapLoader, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (!(p.test_flags & kTestNoCopies)) {
                        const uint32_t st = base + (uint32_t)slot * p.stage_bytes;
                        mbar_arrive_expect_tx(&full[slot], p.tx_bytes);
                        tma_2d(st + p.codes_off, &it.cmap, t * RB, u.n0, &full[slot]);
                        tma_3d(st, &it.xmap, 0, 0, t * NAT, &full[slot]);
                        ++issued;
                    }
                    if (++slot == R) { slot = 0; ++wrap; }
                }
            }
            // Copies still in flight (consumers that gave up) land before the CTA leaves.
            for (int s = 0; s < R && s < issued; ++s) {
                const int uses = issued / R + (s < issued % R ? 1 : 0);
                nap_wait(&full[s], (uint32_t)(uses - 1) & 1u, kStatusTmaWait, kNapDrain, p.wait_ns);
            }
        }
        __syncwarp();
    } else if (KS == 128 && warp <= 18 && p.ng == 4) {             // 256-K stages have at most 3 A slots
        dequant_groups<FMT, KS, KS == 128 ? 4 : 2>(p, smem, tmem, full, afull, aempty, warp, lane);
    } else if (warp <= 18 && p.ng == 2) {
        dequant_groups<FMT, KS, 2>(p, smem, tmem, full, afull, aempty, warp, lane);
    } else if (warp <= 18) {
        // ------------------------------------------------------ dequantize into tensor memory
        const int q = warp & 3, h = (warp - 3) >> 2;           // lane quarter, quarter of the stage's K
        const int r = 32 * q + lane;
        const uint32_t tl = (uint32_t)(32 * q) << 16;         // this warp's lane quarter
        ScaleCursor<FMT, KS, TcArgs<MAXI>> sc;
        sc.start(&p, r, h);
        // scale FIFO: slot i is written and read at the same unrolled position,
        // so no register holding an in-flight load is ever copied
        uint32_t sq[kScaleAhead], sm[kScaleAhead];
#pragma unroll
        for (int i = 0; i < kScaleAhead; ++i) sc.next(sq[i], sm[i]);
        Unit u;
        int ui = 0, t = 0;
        bool live = get_unit(p, 0, u);
        if (live) t = u.t0;
        // this thread's code chunks within a stage's codes tile
        const uint32_t cp0 = code_pos<RB>(r, is_sb(FMT) ? 1 + 2 * h : FMT == kFmtW4G64 && KS == 128 ? h : 2 * h);
        const uint32_t cp1 = code_pos<RB>(r, is_sb(FMT) ? 2 + 2 * h : 2 * h + 1);
        const uint32_t cph = code_pos<RB>(r, 0);               // superblock record header
        // high-bit plane of groups 2h, 2h + 1: 8 bytes (5 bits) or 16 (6 bits) at 144 + 8h or 144 + 16h
        const uint32_t cpp = code_pos<RB>(r, 0) + 144u + (FMT == kFmtW6SB32 ? 16u : 8u) * (uint32_t)h;
        // 6-bit symmetric: quarter h is half h & 1 of 48-byte chunk h >> 1 (16 nibble bytes, 8 plane bytes)
        const uint32_t cw6 = code_pos<RB>(r, 3 * (h >> 1) + (h & 1));
        const uint32_t cp6 = code_pos<RB>(r, 3 * (h >> 1) + 2) + 8u * (uint32_t)(h & 1);
        uint32_t g = 0;
        int slot = 0, wrap = 0, aslot = 0, awrap = 0;
        bool ok = true;
        while (ok && live) {
#pragma unroll
            for (int i = 0; i < kScaleAhead; ++i) {
                if (!live) break;
                const uint32_t s = sq[i] & sm[i];
                sc.next(sq[i], sm[i]);
                if (!warp_wait(&full[slot], (uint32_t)wrap & 1u, kStatusTmaWait, kNapCritical, p.wait_ns)) { ok = false; break; }
                const int a = aslot;
                if (awrap && !warp_wait(&aempty[a], (uint32_t)(awrap - 1) & 1u, kStatusMmaWait, kNapCritical, p.wait_ns)) { ok = false; break; }
                const uint8_t* cs = smem + (size_t)slot * p.stage_bytes + p.codes_off;
                const uint32_t ta = tmem + tl + p.A0 + (uint32_t)a * ACOLS + (uint32_t)h * QCOLS;
                if (FMT == kFmtW4SB32) {                      // 64 weights: groups 2h, 2h+1 of the record
                    const uint4 hd = *reinterpret_cast<const uint4*>(cs + cph);
                    const uint4 c0 = *reinterpret_cast<const uint4*>(cs + cp0);
                    const uint4 c1 = *reinterpret_cast<const uint4*>(cs + cp1);
                    uint32_t o[32];
                    dq_sb32(hd, c0, c1, h, o);
                    tmem_st32(ta, o);
                } else if (is_sb(FMT)) {                      // the same with the high-bit plane
                    const uint4 hd = *reinterpret_cast<const uint4*>(cs + cph);
                    const uint4 c0 = *reinterpret_cast<const uint4*>(cs + cp0);
                    const uint4 c1 = *reinterpret_cast<const uint4*>(cs + cp1);
                    uint32_t pl[4];
                    if (FMT == kFmtW6SB32) {
                        const uint4 v = *reinterpret_cast<const uint4*>(cs + cpp);
                        pl[0] = v.x; pl[1] = v.y; pl[2] = v.z; pl[3] = v.w;
                    } else {
                        const uint2 v = *reinterpret_cast<const uint2*>(cs + cpp);
                        pl[0] = v.x; pl[1] = v.y; pl[2] = 0u; pl[3] = 0u;
                    }
                    uint32_t o[32];
                    dq_sbw<FMT == kFmtW6SB32 ? 6 : 5>(hd, c0, c1, pl, h, o);
                    tmem_st32(ta, o);
                } else if (FMT == kFmtW4G64 && KS == 256) {   // 64 weights: chunks 2h, 2h+1, one group
                    const uint4 c0 = *reinterpret_cast<const uint4*>(cs + cp0);
                    const uint4 c1 = *reinterpret_cast<const uint4*>(cs + cp1);
                    const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                    uint32_t o[32];
                    dq_w4<8>(wv, (uint16_t)s, o);
                    tmem_st32(ta, o);
                } else if (FMT == kFmtW4G64) {                // 32 weights: chunk h, half a group
                    const uint4 c0 = *reinterpret_cast<const uint4*>(cs + cp0);
                    const uint32_t wv[4] = {c0.x, c0.y, c0.z, c0.w};
                    uint32_t o[16];
                    dq_w4<4>(wv, (uint16_t)s, o);
                    tmem_st16(ta, o);
                } else if (FMT == kFmtW6G16) {               // 32 weights: two groups of 16
                    const uint4 c0 = *reinterpret_cast<const uint4*>(cs + cw6);
                    const uint2 pl = *reinterpret_cast<const uint2*>(cs + cp6);
                    uint32_t o[16];
                    dq_w6(c0, pl, s, o);
                    tmem_st16(ta, o);
                } else {                                      // int8, 32 weights: chunks 2h, 2h+1
                    uint4 c[2];
                    c[0] = *reinterpret_cast<const uint4*>(cs + cp0);
                    c[1] = *reinterpret_cast<const uint4*>(cs + cp1);
                    uint32_t o[16];
                    dq_w8(c, FMT == kFmtW8G64 ? s * 0x10001u : s, o);   // g64: one scale for both halves
                    tmem_st16(ta, o);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&afull[a]);
                if (++slot == R) { slot = 0; ++wrap; }
                if (++aslot == AS) { aslot = 0; ++awrap; }
                ++g;
                if (++t >= u.t1) {
                    live = get_unit(p, ++ui, u);
                    if (live) t = u.t0;
                }
            }
        }
    } else {
        // ------------------------------------------------------ epilogue (warps 19-22)
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t tl = (uint32_t)(32 * q) << 16;
        const int M = p.M;
        grid_dep_wait();                                     // y may be read by earlier kernels
        Unit u;
        for (int ui = 0; get_unit(p, ui, u); ++ui) {
            const int d = ui & 1;
            if (!warp_wait(&dfull[d], (uint32_t)(ui >> 1) & 1u, kStatusMmaWait, kNapEpilogue, p.wait_ns)) break;
            tc_fence_after();
            const TcItem& it = p.it[u.item];
            const int N = it.N, n = u.n0 + r;
            void* y = it.y;
            const uint32_t dc = tmem + tl + (uint32_t)(d * niss * Mpad);
            for (int c0 = 0; c0 < Mpad; c0 += 16) {
                float v[16];
                tmem_ld16(dc + (uint32_t)c0, v);
                if (niss == 2) {                             // second issuer's accumulator, fixed order
                    float v2[16];
                    tmem_ld16(dc + (uint32_t)(Mpad + c0), v2);
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] += v2[j];
                }
                if (p.split > 1) {                           // partial tile -> own shared memory [m][128]
                    float* red = reinterpret_cast<float*>(smem);
#pragma unroll
                    for (int j = 0; j < 16; ++j) red[(c0 + j) * kTcRows + r] = v[j];
                } else if (n < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < M) store_y(y, (size_t)(c0 + j) * N + n, v[j], it.ybf16);
                }
            }
            tc_fence_before();
            mbar_arrive(&dempty[d]);
        }
    }

    __syncwarp();
    if (p.split > 1) {
        // partial tiles of the cluster's CTAs are summed in rank order; rank j
        // writes activation rows m = j, j + split, ...
        cluster_sync();
        const uint32_t j = cluster_rank();
        const TcItem& it = p.it[0];
        const int N = it.N, M = p.M;
        const int n0 = ((int)blockIdx.x / p.split) * kTcRows;
        const int mine = (M - (int)j + p.split - 1) / p.split;      // rows m of this rank
        for (int e = tid; e < mine * 32; e += kTcThreads) {
            const int m = (int)j + (e >> 5) * p.split, r4 = (e & 31) * 4;
            const uint32_t off = base + (uint32_t)(m * kTcRows + r4) * 4u;
            float4 s = ld_dsmem_f4(off, 0);
            for (int k = 1; k < p.split; ++k) {
                const float4 v = ld_dsmem_f4(off, (uint32_t)k);
                s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
            }
            const int n = n0 + r4;
            const size_t row = (size_t)m * N;
            if ((N & 3) == 0 && n + 3 < N) {
                if (it.ybf16) {
                    const __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
                    uint2 u;
                    u.x = *reinterpret_cast<const uint32_t*>(&lo);
                    u.y = *reinterpret_cast<const uint32_t*>(&hi);
                    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(it.y) + row + n) = u;
                } else {
                    *reinterpret_cast<float4*>(static_cast<float*>(it.y) + row + n) = s;
                }
            } else {
                if (n < N) store_y(it.y, row + n, s.x, it.ybf16);
                if (n + 1 < N) store_y(it.y, row + n + 1, s.y, it.ybf16);
                if (n + 2 < N) store_y(it.y, row + n + 2, s.z, it.ybf16);
                if (n + 3 < N) store_y(it.y, row + n + 3, s.w, it.ybf16);
            }
        }
        cluster_sync();                                     // peers have finished reading this CTA
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------ host side
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on the driver library).
EncodeTiled encoder() {
    static EncodeTiled fn = nullptr;
    static int tried = 0;
    if (!__atomic_load_n(&tried, __ATOMIC_ACQUIRE)) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(f);
        __atomic_store_n(&tried, 1, __ATOMIC_RELEASE);
    }
    return fn;
}

// Tensor map over `rank` dimensions (innermost first; strides in bytes for
// dimensions 1..rank-1); out-of-range elements read as zero.
bool encode(EncodeTiled enc, CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* ptr, const uint64_t* dims,
            const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
    cuuint64_t d[3], s[2];
    cuuint32_t b[3], e[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
    for (int i = 0; i + 1 < rank; ++i) s[i] = strides[i];
    return enc(m, dt, (cuuint32_t)rank, const_cast<void*>(ptr), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int KS, int MAXI>
cudaError_t launch_fmt_tc(const WgemmArgs* a, int count, cudaStream_t st) {
    constexpr uint32_t RB = FMT == kFmtW4G64 ? KS / 2 : is_w8(FMT) ? KS : FMT == kFmtW6G16 ? KS / 64 * 48
                                                                        : sb_record(FMT);
    const EncodeTiled enc = encoder();
    if (!enc) return cudaErrorNotSupported;
    TcArgs<MAXI> p = {};
    const int M = a[0].M;
    p.count = count;
    p.M = M;
    p.Mpad = (M + 15) & ~15;
    const int xrows = (M + 7) & ~7;                          // x rows copied; MMA rows past M are never stored
    // products in decreasing K (longest tiles first in the persistent order)
    int order[kTcMaxItems];
    for (int i = 0; i < count; ++i) order[i] = i;
    for (int i = 1; i < count; ++i) {                        // stable insertion sort
        const int v = order[i];
        int j = i - 1;
        while (j >= 0 && a[order[j]].K < a[v].K) { order[j + 1] = order[j]; --j; }
        order[j + 1] = v;
    }
    int units = 0;
    for (int i = 0; i < count; ++i) {
        const WgemmArgs& w = a[order[i]];
        TcItem& it = p.it[i];
        const uint64_t crb = code_row_bytes(FMT, w.K);
        const uint64_t cd[2] = {crb, (uint64_t)w.N}, cs[1] = {crb};
        const uint32_t cb[2] = {RB, (uint32_t)kTcRows};
        // x [M][K] as [K/64 atoms][M rows][64]: one box holds the stage's KS/64 atoms
        const uint64_t xd[3] = {64, (uint64_t)M, (uint64_t)(w.K / 64)}, xs[2] = {(uint64_t)w.K * 2, 128};
        const uint32_t xb[3] = {64, (uint32_t)xrows, (uint32_t)(KS / 64)};
        if (!encode(enc, &it.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w.codes, cd, cs, cb,
                    RB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : RB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                                    : CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !encode(enc, &it.xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w.x, xd, xs, xb, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        it.scales = static_cast<const uint8_t*>(w.scales);
        it.y = w.y;
        it.ybf16 = w.ybf16;
        it.K = w.K;
        it.N = w.N;
        it.T = (w.K + KS - 1) / KS;
        it.unit0 = units;
        it.srb = (uint32_t)scale_row_bytes(FMT, w.K);
        units += (w.N + kTcRows - 1) / kTcRows;
    }
    p.units = units;
    p.niss = p.Mpad <= 64 ? 2 : 1;
    p.A0 = (uint32_t)(2 * p.niss * p.Mpad + 31) & ~31u;       // accumulator columns, then the A ring
    p.AS = (int)((kTmemCols - p.A0) / (KS / 2));
    if (p.AS > kMaxAS) p.AS = kMaxAS;
    if (p.AS < 2) return cudaErrorInvalidValue;
    // dequantizing groups: as many as the A slots allow (each group holds one
    // slot while it works, the MMA at least one more)
    p.ng = KS == 128 && p.AS >= 5 ? 4 : p.AS >= 3 ? 2 : 1;
    const int sms = sm_count();
    p.split = 1;
    if (count == 1 && units < sms / 2) {                     // too few tiles: split K over a cluster
        int s = (sms - sms / 8) / units;                     // leave room for whole clusters per GPC
        s = s < 1 ? 1 : (s > 8 ? 8 : s);
        const int T = p.it[0].T;
        while (s > 1 && T / s < 2) --s;
        p.split = s;
    }
    // shared-memory stage: x (KS/64 atoms of xrows rows), then the codes tile
    p.x_atom = (uint32_t)xrows * 128u;
    const uint32_t x_b = (uint32_t)(KS / 64) * p.x_atom;
    p.codes_off = (x_b + 1023u) & ~1023u;
    const uint32_t codes_b = kTcRows * RB;
    p.stage_bytes = (p.codes_off + codes_b + 1023u) & ~1023u;
    p.tx_bytes = x_b + codes_b;                              // tensor-copy bytes per stage (boxes incl. zero fill)
    const size_t bars = (2 * kTcMaxStages + 2 * kMaxAS + 6) * 8 + 16;
    const size_t avail = kTcSmemMax - 1024 - bars;
    int R = (int)(avail / p.stage_bytes);
    R = R > kTcMaxStages ? kTcMaxStages : R;
    if (R < 2) return cudaErrorInvalidValue;
    const uint32_t red_b = (uint32_t)p.Mpad * kTcRows * 4u;   // cluster partial tile (reuses the ring)
    if (p.split > 1 && (size_t)R * p.stage_bytes < red_b) return cudaErrorInvalidValue;
    p.R = R;
    p.bar_off = (uint32_t)R * p.stage_bytes;
    const size_t smem = p.bar_off + bars + 1024;             // + alignment slack
    p.wait_ns = wait_limit_ns();
    p.test_flags = test_flags();

    auto kern = tc_kernel<FMT, KS, MAXI>;
    static unsigned long long attr_done = 0ull;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmemMax);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_done, bit, __ATOMIC_RELEASE);
    }
    cudaLaunchConfig_t cfg = {};
    const int grid = p.split > 1 ? units * p.split : (units < sms ? units : sms);
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)p.split;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.split > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// int4 runs 256-K stages (128-byte code rows) when x leaves room for them and
// K allows; int8 rows are 128 bytes at 128-K stages already.
template <int FMT>
cudaError_t launch_chunk(const WgemmArgs* a, int count, cudaStream_t st) {
    if constexpr (is_sb(FMT)) {                             // K % 256 == 0: one record per row and stage
        return count == 1 ? launch_fmt_tc<FMT, 256, 1>(a, 1, st) : launch_fmt_tc<FMT, 256, kTcMaxItems>(a, count, st);
    } else {
        if constexpr (FMT == kFmtW4G64) {
            bool wide = a[0].M <= 64;
            for (int i = 0; i < count; ++i) wide = wide && (a[i].K % 256 == 0);
            if (wide)
                return count == 1 ? launch_fmt_tc<FMT, 256, 1>(a, 1, st)
                                  : launch_fmt_tc<FMT, 256, kTcMaxItems>(a, count, st);
        }
        return count == 1 ? launch_fmt_tc<FMT, 128, 1>(a, 1, st) : launch_fmt_tc<FMT, 128, kTcMaxItems>(a, count, st);
    }
}

template <int FMT>
cudaError_t launch_chunks(const WgemmArgs* a, int count, cudaStream_t st) {
    for (int i = 0; i < count; i += kTcMaxItems) {
        const int c = count - i < kTcMaxItems ? count - i : kTcMaxItems;
        const cudaError_t e = launch_chunk<FMT>(a + i, c, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

// The 5- and 6-bit formats have no register-path kernel: their products run
// here at every M (x rows past M are zero-filled by the copy).
bool tc_supported(int fmt, int M) {
    if (fmt == kFmtW5SB32 || fmt == kFmtW6SB32 || fmt == kFmtW6G16) return M >= 1;
    return M >= kTcMinM && (fmt == kFmtW4G64 || is_w8(fmt) || fmt == kFmtW4SB32);
}

cudaError_t launch_tc(const WgemmArgs* a, int count, cudaStream_t st) {
    if (a[0].fmt == kFmtW4G64) return launch_chunks<kFmtW4G64>(a, count, st);
    if (a[0].fmt == kFmtW8G16) return launch_chunks<kFmtW8G16>(a, count, st);
    if (a[0].fmt == kFmtW8G64) return launch_chunks<kFmtW8G64>(a, count, st);
    if (a[0].fmt == kFmtW6G16) return launch_chunks<kFmtW6G16>(a, count, st);
    if (a[0].fmt == kFmtW4SB32) return launch_chunks<kFmtW4SB32>(a, count, st);
    if (a[0].fmt == kFmtW5SB32) return launch_chunks<kFmtW5SB32>(a, count, st);
    return launch_chunks<kFmtW6SB32>(a, count, st);
}

cudaError_t status_tc(cudaStream_t st, unsigned* word) {
    unsigned v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *word = v;
    return e;
}

}  // namespace rq
