// rq_pack.cu -- quantize-pack (RTN / E[x^2]-weighted grid search) and the
// dequant export, for the three packed formats.
//
// Sources: rwkv-quant article ("rwkv-quant: keeping one matrix in bf16 removes
// 39% of RWKV-7 2.9B's quantization loss", section "Two presets and six
// sizes"): symmetric int8 group 16 (REDUCTION), asymmetric int4 superblock
// group 32 (COMPRESSION), each group's scale and shift found by a search
// weighted by E[x^2] of the input channel. RWKV-7 G1 1.5B int4 model card
// ("Format & loading"): symmetric int4 group 64 as codes plus scales.
//
// Determinism: every fp32 / fp64 operation on the search path is an explicit
// round-to-nearest intrinsic (never contracted into an FMA), each candidate's
// loss is summed sequentially in ascending k by one thread, and the argmin
// keeps the lowest index among equal losses. The output bytes therefore do
// not depend on the launch shape.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

// Candidate t_i = fp32(lo + (hi - lo) * i / (n - 1)) in fp64; n = 1 -> hi.
__device__ __forceinline__ float cand_t(int i, int n, float t_lo, float t_hi) {
    if (n == 1) return t_hi;
    const double lo = (double)t_lo, hi = (double)t_hi;
    double step = __dmul_rn(__dsub_rn(hi, lo), (double)i);
    step = __ddiv_rn(step, (double)(n - 1));
    return __double2float_rn(__dadd_rn(lo, step));
}

__device__ __forceinline__ float clampf(float v, float lo, float hi) {
    return v < lo ? lo : (v > hi ? hi : v);
}

// Symmetric code for scale sf: clamp(rint(w / sf), -qmax, qmax); 0 if sf == 0.
__device__ __forceinline__ int sym_code(float w, float sf, float qmax) {
    if (sf == 0.0f) return 0;
    return (int)rintf(clampf(__fdiv_rn(w, sf), -qmax, qmax));
}

// Asymmetric code: clamp(rint((w + M) / S), 0, L), L = 2^bits - 1; 0 if S == 0.
__device__ __forceinline__ int asym_code(float w, float S, float M, float L) {
    if (S == 0.0f) return 0;
    return (int)rintf(clampf(__fdiv_rn(__fadd_rn(w, M), S), 0.0f, L));
}

// (loss, index) pair reduction over a warp: smallest loss, then smallest index.
__device__ __forceinline__ void warp_argmin(double& L, int& idx) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double L2 = __shfl_xor_sync(0xffffffffu, L, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
        if (L2 < L || (L2 == L && i2 < idx)) { L = L2; idx = i2; }
    }
}

constexpr int kPackWarps = 8;
constexpr int kGptqWarps = 8;      // most rows per block of the GPTQ kernel

// Shared memory of one GPTQ row: the row in fp64, its codes, the group's
// fp32 weights and loss weights.
__host__ __device__ constexpr size_t gptq_warp_bytes(int K, int G) {
    return (size_t)K * 8 + (size_t)K + (size_t)G * 8;
}
// Superblock formats: the record (208 bytes at most), 32 scale/min floats,
// the superblock's 256 weights and loss weights, the row in fp64.
__host__ __device__ constexpr size_t gptq_sb_warp_bytes(int K) {
    return 208 + 32 * 4 + 512 * 4 + (size_t)K * 8;
}
constexpr double kInf = __builtin_huge_val();

// The E[x^2]-weighted search of one symmetric group of G weights held in
// shared memory by the calling warp (w, and the weights a of the loss):
// absmax, base = absmax / qmax, candidate i's scale fp16(t_i * base), loss
// sum_k a_k (w_k - q_k s_i)^2 in fp64 in ascending k, the lowest index with
// the least loss. Lane l evaluates candidates l, l + 32, ...; every lane
// returns the chosen scale.
template <int G>
__device__ __forceinline__ __half sym_search(const float* w, const float* a, float qmax, int n_cand, float t_lo,
                                             float t_hi, int lane) {
    float amax = 0.0f;
    for (int k = lane; k < G; k += 32) amax = fmaxf(amax, fabsf(w[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float base = __fdiv_rn(amax, qmax);
    if (n_cand == 1) return __float2half_rn(__fmul_rn(cand_t(0, 1, t_lo, t_hi), base));
    double bestL = kInf;   // lanes without a candidate never win
    int bestI = 0x7fffffff;
    for (int i = lane; i < n_cand; i += 32) {
        const float sf = __half2float(__float2half_rn(__fmul_rn(cand_t(i, n_cand, t_lo, t_hi), base)));
        double L = 0.0;
        for (int k = 0; k < G; ++k) {
            const float wk = w[k];
            const float wq = __fmul_rn((float)sym_code(wk, sf, qmax), sf);
            const double d = __dsub_rn((double)wk, (double)wq);
            L = __dadd_rn(L, __dmul_rn((double)a[k], __dmul_rn(d, d)));
        }
        if (bestI == 0x7fffffff || L < bestL) { bestL = L; bestI = i; }
    }
    warp_argmin(bestL, bestI);
    return __float2half_rn(__fmul_rn(cand_t(bestI, n_cand, t_lo, t_hi), base));
}

// One warp per symmetric group of G weights: int4 (G = 64, qmax 7), int8
// (G = 16 or 64, qmax 127), 6-bit (G = 16, qmax 31).
template <int G, int QMAX>
__global__ void __launch_bounds__(kPackWarps * 32)
qpack_sym_kernel(const float* __restrict__ W, int K, int N, const float* __restrict__ act_sq,
                 int n_cand, float t_lo, float t_hi, uint8_t* __restrict__ codes,
                 uint16_t* __restrict__ scales) {
    __shared__ float s_w[kPackWarps][G];
    __shared__ float s_a[kPackWarps][G];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ng = K / G;
    const long long total = (long long)N * ng;
    const long long gid = (long long)blockIdx.x * kPackWarps + warp;
    if (gid >= total) return;
    const int n = (int)(gid / ng), g = (int)(gid % ng);
    const float* w = W + (size_t)n * K + (size_t)g * G;
    for (int k = lane; k < G; k += 32) {
        s_w[warp][k] = w[k];
        s_a[warp][k] = act_sq ? act_sq[(size_t)g * G + k] : 1.0f;
    }
    __syncwarp();
    const float qmax = (float)QMAX;
    const __half best_s = sym_search<G>(s_w[warp], s_a[warp], qmax, n_cand, t_lo, t_hi, lane);
    const float sf = __half2float(best_s);
    if (QMAX == 7) {
        // lane l writes byte l of the group: k = 2l (low nibble), 2l+1 (high)
        const int q0 = sym_code(s_w[warp][2 * lane], sf, qmax);
        const int q1 = sym_code(s_w[warp][2 * lane + 1], sf, qmax);
        codes[(size_t)n * (K / 2) + (size_t)g * 32 + lane] = (uint8_t)((q0 + 8) | ((q1 + 8) << 4));
    } else if (QMAX == 127) {
        for (int k = lane; k < G; k += 32) {
            const int q = sym_code(s_w[warp][k], sf, qmax);
            codes[(size_t)n * K + (size_t)g * G + k] = (uint8_t)(q + 128);
        }
    } else {
        // 6 bits, u = q + 32: group g is weights j0 .. j0 + 15 of the 64-weight
        // chunk g / 4 (j0 = 16 (g % 4)); lanes 0..7 write its low-nibble bytes
        // (weights j0 + 2l, j0 + 2l + 1), lanes 8..11 its plane bytes (bits 4..5
        // of weights j0 + 4i .. j0 + 4i + 3)
        uint8_t* chunk = codes + (size_t)n * (K / 64 * 48) + (size_t)(g >> 2) * 48;
        const int j0 = 16 * (g & 3);
        if (lane < 8) {
            const int u0 = sym_code(s_w[warp][2 * lane], sf, qmax) + 32;
            const int u1 = sym_code(s_w[warp][2 * lane + 1], sf, qmax) + 32;
            chunk[j0 / 2 + lane] = (uint8_t)((u0 & 15) | ((u1 & 15) << 4));
        } else if (lane < 12) {
            const int i = lane - 8;
            uint32_t v = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) v |= (uint32_t)((sym_code(s_w[warp][4 * i + e], sf, qmax) + 32) >> 4) << (2 * e);
            chunk[32 + j0 / 4 + i] = (uint8_t)v;
        }
    }
    if (lane == 0) scales[(size_t)n * ng + g] = __half_as_ushort(best_s);
}

// GPTQ on the preset's grid for a symmetric format (GPTQ, Frantar et al.
// 2022; rwkv-quant article, "Calibration leakage and honest measurements"):
// one warp per row, the row held in fp64 in shared memory. Columns in order;
// at each group's first column the group's scale is the preset's search on
// fp32 of the current weights; then per column k:
//   q_k = clamp(rint(fp32(w_k) / s), -qmax, qmax),
//   err = (w_k - q_k s) / U[k][k],  w_j = w_j - err * U[k][j] for j > k
// (fp64, one rounding per operation, lanes over j; the updates of each w_j
// arrive in ascending k). Dead columns start at 0. The codes are emitted at
// the end in the format's layout.
template <int G, int QMAX>
__global__ void __launch_bounds__(kGptqWarps * 32)
gptq_sym_kernel(const float* __restrict__ W, int K, int N, const double* __restrict__ U,
                const uint8_t* __restrict__ dead, const float* __restrict__ act_sq, int n_cand, float t_lo,
                float t_hi, uint8_t* __restrict__ codes, uint16_t* __restrict__ scales) {
    extern __shared__ __align__(16) uint8_t g_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * (int)(blockDim.x >> 5) + warp;
    if (n >= N) return;
    const size_t per = gptq_warp_bytes(K, G);
    double* w = reinterpret_cast<double*>(g_smem + (size_t)warp * per);
    int8_t* q = reinterpret_cast<int8_t*>(w + K);
    float* wg = reinterpret_cast<float*>(q + K);          // K % 64 == 0: 4-byte aligned
    float* ag = wg + G;
    for (int k = lane; k < K; k += 32) w[k] = dead[k] ? 0.0 : (double)W[(size_t)n * K + k];
    __syncwarp();
    const float qmax = (float)QMAX;
    const int ng = K / G;
    for (int g = 0; g < ng; ++g) {
        const int k0 = g * G;
        for (int i = lane; i < G; i += 32) {
            wg[i] = __double2float_rn(w[k0 + i]);
            ag[i] = act_sq ? act_sq[k0 + i] : 1.0f;
        }
        __syncwarp();
        const __half sh = sym_search<G>(wg, ag, qmax, n_cand, t_lo, t_hi, lane);
        if (lane == 0) scales[(size_t)n * ng + g] = __half_as_ushort(sh);
        const float sf = __half2float(sh);
        for (int i = 0; i < G; ++i) {
            const int k = k0 + i;
            const double wk = w[k];
            const int qk = sym_code(__double2float_rn(wk), sf, qmax);
            if (lane == 0) q[k] = (int8_t)qk;
            const double err = __ddiv_rn(__dsub_rn(wk, (double)__fmul_rn((float)qk, sf)), U[(size_t)k * K + k]);
            const double* Uk = U + (size_t)k * K;
            for (int j = k + 1 + lane; j < K; j += 32) w[j] = __dsub_rn(w[j], __dmul_rn(err, Uk[j]));
            __syncwarp();
        }
    }
    __syncwarp();
    if (QMAX == 7) {
        for (int t = lane; t < K / 2; t += 32)
            codes[(size_t)n * (K / 2) + t] = (uint8_t)((q[2 * t] + 8) | ((q[2 * t + 1] + 8) << 4));
    } else if (QMAX == 127) {
        for (int k = lane; k < K; k += 32) codes[(size_t)n * K + k] = (uint8_t)(q[k] + 128);
    } else {
        // 6 bits: per 64-weight chunk, bytes 0..31 low nibbles, 32..47 bits 4..5
        uint8_t* row = codes + (size_t)n * (K / 64 * 48);
        for (int b = lane; b < K / 64 * 48; b += 32) {
            const int c = b / 48, o = b - c * 48, j0 = 64 * c;
            uint32_t v = 0;
            if (o < 32) {
                v = (uint32_t)((q[j0 + 2 * o] + 32) & 15) | ((uint32_t)((q[j0 + 2 * o + 1] + 32) & 15) << 4);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) v |= (uint32_t)((q[j0 + 4 * (o - 32) + e] + 32) >> 4) << (2 * e);
            }
            row[b] = (uint8_t)v;
        }
    }
}

// The preset's search for one asymmetric group of 32 weights held in shared
// memory by the calling warp (w, and the loss weights a): lo = min(0, min w),
// hi = max(0, max w); candidate i shrinks [lo, hi] about its midpoint by t_i
// (r = t_i (hi - lo) / 2, S = 2 r / (2^b - 1), M = max(0, r - mid)); loss as
// for the symmetric search; lowest index with the least loss. Every lane
// returns the chosen (S*, M*).
template <int BITS>
__device__ __forceinline__ void asym_search(const float* w, const float* a, int n_cand, float t_lo, float t_hi,
                                            int lane, float& S_out, float& M_out) {
    constexpr float kTop = (float)((1 << BITS) - 1);        // highest code
    float lo = w[lane] < 0.0f ? w[lane] : 0.0f;
    float hi = w[lane] > 0.0f ? w[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const float h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
    }
    const float half = __fmul_rn(__fsub_rn(hi, lo), 0.5f);
    const float mid = __fmul_rn(__fadd_rn(hi, lo), 0.5f);
    double bestL = kInf;
    int bestI = 0x7fffffff;
    for (int i = lane; i < n_cand; i += 32) {
        const float r = __fmul_rn(cand_t(i, n_cand, t_lo, t_hi), half);
        const float S = __fdiv_rn(__fmul_rn(2.0f, r), kTop);
        const float loi = __fsub_rn(mid, r);
        const float M = loi < 0.0f ? -loi : 0.0f;
        double loss = 0.0;
        if (n_cand > 1) {
            for (int k = 0; k < 32; ++k) {
                const float wk = w[k];
                const float wq = __fsub_rn(__fmul_rn((float)asym_code(wk, S, M, kTop), S), M);
                const double d = __dsub_rn((double)wk, (double)wq);
                loss = __dadd_rn(loss, __dmul_rn((double)a[k], __dmul_rn(d, d)));
            }
        }
        if (bestI == 0x7fffffff || loss < bestL) { bestL = loss; bestI = i; }
    }
    warp_argmin(bestL, bestI);
    const float r = __fmul_rn(cand_t(bestI, n_cand, t_lo, t_hi), half);
    const float loi = __fsub_rn(mid, r);
    S_out = __fdiv_rn(__fmul_rn(2.0f, r), kTop);
    M_out = loi < 0.0f ? -loi : 0.0f;
}

// A record's header from the eight groups' (S*, M*) (shared memory s_S,
// s_M), by one warp: d = fp16(max S* / 63), dmin = fp16(max M* / 63), 6-bit
// sc_j = rint(S*_j / d), m_j = rint(M*_j / dmin) (0 when d or dmin is 0),
// the stored S_j = d sc_j, M_j = dmin m_j into s_Sq, s_Mq, and the 16 header
// bytes (fp16 d, fp16 dmin, the 96-bit field string) into s_blk.
__device__ __forceinline__ void sb_header(const float* s_S, const float* s_M, int lane, float* s_Sq, float* s_Mq,
                                          uint8_t* s_blk) {
    float mS = 0.0f, mM = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        mS = s_S[j] > mS ? s_S[j] : mS;
        mM = s_M[j] > mM ? s_M[j] : mM;
    }
    const __half dh = __float2half_rn(__fdiv_rn(mS, 63.0f));
    const __half mh = __float2half_rn(__fdiv_rn(mM, 63.0f));
    const float d = __half2float(dh), dm = __half2float(mh);
    uint32_t field = 0;   // lanes 0..7: sc_j, lanes 8..15: m_j
    if (lane < 16) {
        const int j = lane & 7;
        const float num = lane < 8 ? s_S[j] : s_M[j];
        const float den = lane < 8 ? d : dm;
        field = den == 0.0f ? 0u : (uint32_t)(int)rintf(clampf(__fdiv_rn(num, den), 0.0f, 63.0f));
        if (lane < 8) s_Sq[j] = __fmul_rn(d, (float)field);
        else s_Mq[j] = __fmul_rn(dm, (float)field);
    }
    // assemble the 96-bit string: field f (0..15) at bit 6f
    uint32_t words[3] = {0u, 0u, 0u};
#pragma unroll
    for (int f = 0; f < 16; ++f) {
        const uint64_t v = (uint64_t)__shfl_sync(0xffffffffu, field, f);
        const int bit = 6 * f;
        const int wi = bit >> 5, sh = bit & 31;
        const uint64_t placed = v << sh;
        words[wi] |= (uint32_t)placed;
        if (wi + 1 < 3) words[wi + 1] |= (uint32_t)(placed >> 32);
    }
    if (lane == 0) {
        uint32_t* hdr = reinterpret_cast<uint32_t*>(s_blk);
        hdr[0] = (uint32_t)__half_as_ushort(dh) | ((uint32_t)__half_as_ushort(mh) << 16);
        hdr[1] = words[0];
        hdr[2] = words[1];
        hdr[3] = words[2];
    }
}

// One block per superblock of 256 weights with BITS-bit codes (4, 5, 6):
// warp j searches group j (32 weights), then warp 0 forms d, dmin, the 6-bit
// fields, and the block the codes' low nibbles and (5, 6 bits) the high-bit
// plane.
template <int BITS>
__global__ void __launch_bounds__(256)
qpack_sb_kernel(const float* __restrict__ W, int K, int N, const float* __restrict__ act_sq,
                int n_cand, float t_lo, float t_hi, uint8_t* __restrict__ blocks) {
    constexpr int RS = 16 + 128 + (BITS - 4) * 32;          // record bytes
    constexpr float kTop = (float)((1 << BITS) - 1);        // highest code
    __shared__ float s_w[256];
    __shared__ float s_a[256];
    __shared__ float s_S[8], s_M[8];     // searched S*_j, M*_j
    __shared__ float s_Sq[8], s_Mq[8];   // stored S_j = d sc_j, M_j = dmin m_j
    __shared__ uint8_t s_q[256];         // final codes
    __shared__ __align__(16) uint8_t s_blk[RS];
    const int nb = K / 256;
    const long long sb = blockIdx.x;
    const int n = (int)(sb / nb), b = (int)(sb % nb);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const size_t k0 = (size_t)b * 256;
    s_w[t] = W[(size_t)n * K + k0 + t];
    s_a[t] = act_sq ? act_sq[k0 + t] : 1.0f;
    __syncthreads();
    {   // group search (warp = group j)
        float S, M;
        asym_search<BITS>(s_w + 32 * warp, s_a + 32 * warp, n_cand, t_lo, t_hi, lane, S, M);
        if (lane == 0) {
            s_S[warp] = S;
            s_M[warp] = M;
        }
    }
    __syncthreads();
    if (warp == 0) sb_header(s_S, s_M, lane, s_Sq, s_Mq, s_blk);
    __syncthreads();
    s_q[t] = (uint8_t)asym_code(s_w[t], s_Sq[t >> 5], s_Mq[t >> 5], kTop);   // code of weight t
    __syncthreads();
    if (t < 128) {   // low-nibble byte t: k = 2t (low nibble), 2t+1 (high)
        s_blk[16 + t] = (uint8_t)((s_q[2 * t] & 15) | ((s_q[2 * t + 1] & 15) << 4));
    } else if (BITS == 5 && t < 160) {   // plane byte i: bit 4 of codes 8i .. 8i+7
        const int i = t - 128;
        uint32_t v = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) v |= (uint32_t)((s_q[8 * i + e] >> 4) & 1) << e;
        s_blk[144 + i] = (uint8_t)v;
    } else if (BITS == 6 && t < 192) {   // plane byte i: bits 4..5 of codes 4i .. 4i+3
        const int i = t - 128;
        uint32_t v = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) v |= (uint32_t)((s_q[4 * i + e] >> 4) & 3) << (2 * e);
        s_blk[144 + i] = (uint8_t)v;
    }
    __syncthreads();
    if (t < RS / 16) {
        uint4* dst = reinterpret_cast<uint4*>(blocks + ((size_t)n * nb + b) * RS);
        dst[t] = reinterpret_cast<const uint4*>(s_blk)[t];
    }
}

// GPTQ into the asymmetric superblock formats: one warp per row, the row in
// fp64 in shared memory. At each superblock's first column: the eight group
// searches on fp32 of the current weights and the record's header (the same
// helpers as qpack_sb_kernel); then the superblock's 256 columns in order:
//   q = asym_code(fp32(w_k), S_j, M_j), w_hat = fp32(S_j q) - M_j,
//   err = (w_k - w_hat) / U[k][k],  w_j = w_j - err * U[k][j] for j > k.
template <int BITS>
__global__ void __launch_bounds__(kGptqWarps * 32)
gptq_sb_kernel(const float* __restrict__ W, int K, int N, const double* __restrict__ U,
               const uint8_t* __restrict__ dead, const float* __restrict__ act_sq, int n_cand, float t_lo,
               float t_hi, uint8_t* __restrict__ blocks) {
    constexpr int RS = 16 + 128 + (BITS - 4) * 32;
    constexpr float kTop = (float)((1 << BITS) - 1);
    extern __shared__ __align__(16) uint8_t g_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * (int)(blockDim.x >> 5) + warp;
    if (n >= N) return;
    uint8_t* base = g_smem + (size_t)warp * gptq_sb_warp_bytes(K);
    uint8_t* blk = base;                                           // RS bytes (16-byte aligned)
    float* S = reinterpret_cast<float*>(base + 208);               // S*[8], M*[8], Sq[8], Mq[8]
    float* M = S + 8;
    float* Sq = S + 16;
    float* Mq = S + 24;
    float* wsb = S + 32;                                           // 256 fp32 weights
    float* asb = wsb + 256;                                        // 256 loss weights
    double* w = reinterpret_cast<double*>(asb + 256);              // the row
    for (int k = lane; k < K; k += 32) w[k] = dead[k] ? 0.0 : (double)W[(size_t)n * K + k];
    __syncwarp();
    const int nb = K / 256;
    for (int b = 0; b < nb; ++b) {
        const int k0 = 256 * b;
        for (int i = lane; i < 256; i += 32) {
            wsb[i] = __double2float_rn(w[k0 + i]);
            asb[i] = act_sq ? act_sq[k0 + i] : 1.0f;
        }
        __syncwarp();
        for (int j = 0; j < 8; ++j) {
            float Sj, Mj;
            asym_search<BITS>(wsb + 32 * j, asb + 32 * j, n_cand, t_lo, t_hi, lane, Sj, Mj);
            if (lane == 0) {
                S[j] = Sj;
                M[j] = Mj;
            }
        }
        __syncwarp();
        sb_header(S, M, lane, Sq, Mq, blk);
        for (int i = 16 + lane; i < RS; i += 32) blk[i] = 0;
        __syncwarp();
        for (int i = 0; i < 256; ++i) {
            const int k = k0 + i, j = i >> 5;
            const double wk = w[k];
            const int q = asym_code(__double2float_rn(wk), Sq[j], Mq[j], kTop);
            if (lane == 0) {                                       // low nibble, then the plane bits
                if ((i & 1) == 0) blk[16 + i / 2] = (uint8_t)(q & 15);
                else blk[16 + i / 2] |= (uint8_t)((q & 15) << 4);
                if (BITS == 5) blk[144 + i / 8] |= (uint8_t)((q >> 4) << (i % 8));
                if (BITS == 6) blk[144 + i / 4] |= (uint8_t)((q >> 4) << (2 * (i % 4)));
            }
            const float wq = __fsub_rn(__fmul_rn((float)q, Sq[j]), Mq[j]);
            const double err = __ddiv_rn(__dsub_rn(wk, (double)wq), U[(size_t)k * K + k]);
            const double* Uk = U + (size_t)k * K;
            for (int j2 = k + 1 + lane; j2 < K; j2 += 32) w[j2] = __dsub_rn(w[j2], __dmul_rn(err, Uk[j2]));
            __syncwarp();
        }
        uint4* dst = reinterpret_cast<uint4*>(blocks + ((size_t)n * nb + b) * RS);
        if (lane < RS / 16) dst[lane] = reinterpret_cast<const uint4*>(blk)[lane];
        __syncwarp();
    }
}

__global__ void zero_bytes_kernel(uint8_t* p, int n) {
    if ((int)threadIdx.x < n) p[threadIdx.x] = 0;
}

// An empty kernel launched with ordinary stream ordering after the packing
// kernels. rq_wgemm's kernels may start (and read the packed planes) while the
// kernel launched just before them is still running; putting this one in
// between guarantees that the packing grid has completed first.
__global__ void pack_done_kernel() {}

// ---------------------------------------------------------------- dequant --
// One thread per 32-bit word of codes; writes fp32 w_hat in natural k order.
__global__ void dequant_w4_kernel(const uint32_t* __restrict__ codes, const __half* __restrict__ scales,
                                  int K, long long words, float* __restrict__ out) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= words) return;
    const long long wpr = K / 8;
    const long long n = i / wpr;
    const int k0 = (int)(i % wpr) * 8;
    const float s = __half2float(scales[n * (K / 64) + k0 / 64]);
    float o[8];
    w4_word_values(codes[i], o);
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = __fmul_rn(__fsub_rn(o[j], 136.0f), s);
    float4* dst = reinterpret_cast<float4*>(out + n * K + k0);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

template <int G>
__global__ void dequant_w8_kernel(const uint32_t* __restrict__ codes, const __half* __restrict__ scales,
                                  int K, long long words, float* __restrict__ out) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= words) return;
    const long long wpr = K / 4;
    const long long n = i / wpr;
    const int k0 = (int)(i % wpr) * 4;
    const float s = __half2float(scales[n * (K / G) + k0 / G]);
    float f[4];
    unpack_w8(codes[i], f);
    *reinterpret_cast<float4*>(out + n * K + k0) =
        make_float4(__fmul_rn(f[0], s), __fmul_rn(f[1], s), __fmul_rn(f[2], s), __fmul_rn(f[3], s));
}

// 6-bit symmetric codes: one thread per 8 weights (word w of a 64-weight
// chunk: low-nibble bytes 4w .. 4w + 3, plane bytes 32 + 2w, 33 + 2w).
__global__ void dequant_w6_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ scales,
                                  int K, long long units, float* __restrict__ out) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= units) return;
    const long long upr = K / 8;
    const long long n = i / upr;
    const int k0 = (int)(i % upr) * 8;
    const uint8_t* chunk = codes + n * (K / 64 * 48) + (k0 / 64) * 48;
    const int w = (k0 % 64) / 8;
    const float s = __half2float(scales[n * (K / 16) + k0 / 16]);
    const uint32_t lo = *reinterpret_cast<const uint32_t*>(chunk + 4 * w);
    const uint32_t hi = (uint32_t)chunk[32 + 2 * w] | ((uint32_t)chunk[33 + 2 * w] << 8);
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int u = (int)(((lo >> (4 * e)) & 15u) | (((hi >> (2 * e)) & 3u) << 4));
        o[e] = __fmul_rn((float)(u - 32), s);
    }
    float4* dst = reinterpret_cast<float4*>(out + n * K + k0);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

// One thread per 32-bit word of a superblock's low nibbles (32 words, 8
// weights each, per record); the high-bit plane adds bits 4 (5-bit codes)
// or 4..5 (6-bit codes).
template <int BITS>
__global__ void dequant_sb_kernel(const uint8_t* __restrict__ blocks, int K, long long words,
                                  float* __restrict__ out) {
    constexpr int RS = 16 + 128 + (BITS - 4) * 32;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= words) return;
    const long long rec = i / 32;
    const int wi = (int)(i % 32);
    const int nb = K / 256;
    const long long n = rec / nb;
    const int b = (int)(rec % nb);
    const uint8_t* rb = blocks + rec * RS;
    const uint32_t* r = reinterpret_cast<const uint32_t*>(rb);
    const uint32_t h0 = r[0];
    const float d = __half2float(__ushort_as_half((unsigned short)(h0 & 0xffffu)));
    const float dm = __half2float(__ushort_as_half((unsigned short)(h0 >> 16)));
    const int j = wi / 4;   // 4 words (32 weights) per group
    const float S = __fmul_rn(d, (float)sb_field(r[1], r[2], r[3], 0, j));
    const float M = __fmul_rn(dm, (float)sb_field(r[1], r[2], r[3], 1, j));
    float o[8];
    w4_word_values(r[4 + wi], o);
    const uint32_t hb = BITS == 5 ? (uint32_t)rb[144 + wi]
                      : BITS == 6 ? (uint32_t)rb[144 + 2 * wi] | ((uint32_t)rb[145 + 2 * wi] << 8) : 0u;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const float up = BITS == 5 ? (float)((hb >> s) & 1u) : BITS == 6 ? (float)((hb >> (2 * s)) & 3u) : 0.0f;
        const float q = __fadd_rn(__fsub_rn(o[s], 128.0f), __fmul_rn(16.0f, up));   // exact small integer
        o[s] = __fmaf_rn(S, q, -M);
    }
    float4* dst = reinterpret_cast<float4*>(out + n * K + (size_t)b * 256 + wi * 8);
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
}

}  // namespace

cudaError_t launch_quantize_pack(const PackArgs& a, cudaStream_t st) {
    const long long N = a.N;
    if (is_sb(a.fmt)) {
        const long long blocksN = N * (a.K / 256);
        auto kern = a.fmt == kFmtW4SB32 ? qpack_sb_kernel<4> : a.fmt == kFmtW5SB32 ? qpack_sb_kernel<5>
                                                                                : qpack_sb_kernel<6>;
        kern<<<(unsigned)blocksN, 256, 0, st>>>(a.W, a.K, a.N, a.act_sq, a.n_cand, a.t_lo, a.t_hi,
                                                static_cast<uint8_t*>(a.codes));
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        pack_done_kernel<<<1, 32, 0, st>>>();
        return cudaGetLastError();
    }
    const int G = sym_group(a.fmt);
    const long long groups = N * (a.K / G);
    const unsigned grid = (unsigned)((groups + kPackWarps - 1) / kPackWarps);
    auto kern = a.fmt == kFmtW4G64 ? qpack_sym_kernel<64, 7>
              : a.fmt == kFmtW8G16 ? qpack_sym_kernel<16, 127>
              : a.fmt == kFmtW8G64 ? qpack_sym_kernel<64, 127>
                                   : qpack_sym_kernel<16, 31>;
    kern<<<grid, kPackWarps * 32, 0, st>>>(a.W, a.K, a.N, a.act_sq, a.n_cand, a.t_lo, a.t_hi,
                                           static_cast<uint8_t*>(a.codes), static_cast<uint16_t*>(a.scales));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t used = (size_t)groups * 2;
    if (a.scales_bytes > used) {
        zero_bytes_kernel<<<1, 32, 0, st>>>(static_cast<uint8_t*>(a.scales) + used, (int)(a.scales_bytes - used));
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    pack_done_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError();
}

// Rows per block: as many as fit in 200 KB of shared memory (at most 8).
int gptq_rows_per_block(int fmt, int K) {
    const size_t per = is_sb(fmt) ? gptq_sb_warp_bytes(K) : gptq_warp_bytes(K, sym_group(fmt));
    int w = kGptqWarps;
    while (w > 1 && (size_t)w * per > 200 * 1024) --w;
    return (size_t)w * per <= 200 * 1024 ? w : 0;
}

cudaError_t launch_gptq_pack(const GptqArgs& a, cudaStream_t st) {
    const int rows = gptq_rows_per_block(a.fmt, a.K);
    if (rows == 0) return cudaErrorInvalidValue;
    if (is_sb(a.fmt)) {
        auto kern = a.fmt == kFmtW4SB32 ? gptq_sb_kernel<4> : a.fmt == kFmtW5SB32 ? gptq_sb_kernel<5>
                                                                               : gptq_sb_kernel<6>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)((a.N + rows - 1) / rows), rows * 32, (size_t)rows * gptq_sb_warp_bytes(a.K), st>>>(
            a.W, a.K, a.N, a.U, a.dead, a.act_sq, a.n_cand, a.t_lo, a.t_hi, static_cast<uint8_t*>(a.codes));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        pack_done_kernel<<<1, 32, 0, st>>>();
        return cudaGetLastError();
    }
    const int G = sym_group(a.fmt);
    auto kern = a.fmt == kFmtW4G64 ? gptq_sym_kernel<64, 7>
              : a.fmt == kFmtW8G16 ? gptq_sym_kernel<16, 127>
              : a.fmt == kFmtW8G64 ? gptq_sym_kernel<64, 127>
                                   : gptq_sym_kernel<16, 31>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)rows * gptq_warp_bytes(a.K, G);
    kern<<<(unsigned)((a.N + rows - 1) / rows), rows * 32, smem, st>>>(
        a.W, a.K, a.N, a.U, a.dead, a.act_sq, a.n_cand, a.t_lo, a.t_hi, static_cast<uint8_t*>(a.codes),
        static_cast<uint16_t*>(a.scales));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t used = (size_t)a.N * (a.K / G) * 2;
    if (a.scales_bytes > used) {
        zero_bytes_kernel<<<1, 32, 0, st>>>(static_cast<uint8_t*>(a.scales) + used, (int)(a.scales_bytes - used));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    pack_done_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError();
}

cudaError_t launch_dequant(int fmt, int K, int N, const void* codes, const void* scales, float* out,
                           cudaStream_t st) {
    const int threads = 256;
    if (fmt == kFmtW4G64) {
        const long long words = (long long)N * K / 8;
        dequant_w4_kernel<<<(unsigned)((words + threads - 1) / threads), threads, 0, st>>>(
            static_cast<const uint32_t*>(codes), static_cast<const __half*>(scales), K, words, out);
    } else if (is_w8(fmt)) {
        const long long words = (long long)N * K / 4;
        auto kern = fmt == kFmtW8G16 ? dequant_w8_kernel<16> : dequant_w8_kernel<64>;
        kern<<<(unsigned)((words + threads - 1) / threads), threads, 0, st>>>(
            static_cast<const uint32_t*>(codes), static_cast<const __half*>(scales), K, words, out);
    } else if (fmt == kFmtW6G16) {
        const long long units = (long long)N * K / 8;
        dequant_w6_kernel<<<(unsigned)((units + threads - 1) / threads), threads, 0, st>>>(
            static_cast<const uint8_t*>(codes), static_cast<const __half*>(scales), K, units, out);
    } else {
        const long long words = (long long)N * (K / 256) * 32;
        auto kern = fmt == kFmtW4SB32 ? dequant_sb_kernel<4> : fmt == kFmtW5SB32 ? dequant_sb_kernel<5>
                                                                              : dequant_sb_kernel<6>;
        kern<<<(unsigned)((words + threads - 1) / threads), threads, 0, st>>>(static_cast<const uint8_t*>(codes), K,
                                                                             words, out);
    }
    return cudaGetLastError();
}

cudaError_t status_pack(cudaStream_t st, unsigned* word) {
    unsigned v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *word = v;
    return e;
}

}  // namespace rq
