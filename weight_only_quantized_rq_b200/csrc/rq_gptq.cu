// rq_gptq.cu -- the two preparatory steps of GPTQ on the preset's grid: the
// running Hessian of a layer's inputs and the factor the column loop uses.
//
// Sources: rwkv-quant article, "Calibration leakage and honest measurements"
// (GPTQ on the preset's grid without changing the format, the kernels or the
// file size); RWKV-7 G1 1.5B int4 model card (symmetric int4 group 64,
// GPTQ-calibrated). The method is GPTQ (Frantar et al., 2022): with H the
// input Hessian, quantize the columns in order and move the not yet quantized
// columns by each error times a row of U, the upper Cholesky factor of the
// damped H^-1.
//
// U without an explicit inverse of H: if J reverses the index order and
// J H J = M M^T (lower Cholesky), then H = V V^T with V = J M J upper, so
// H^-1 = V^-T V^-1 and U = V^-1 = J M^-1 J (upper, positive diagonal): one
// Cholesky and one triangular inverse. All of it runs in the caller's U
// buffer:
//   1. U := J (H + lambda I) J (dead diagonal entries set to 1 first);
//   2. lower Cholesky in place, in blocks of 32 columns: one CTA factors the
//      32 x 32 diagonal block (the sums over the columns left of the block
//      first, by all its warps, then the block's columns in order) and keeps
//      each pivot in the strictly upper triangle (free until step 3); then
//      one warp per row below the block forms the row's 32 entries (its sums
//      over the left columns against the block's rows, staged 32 columns at
//      a time in shared memory, then a forward solve with the block). Two
//      launches per 32 columns instead of one per column; a last launch
//      moves the pivots onto the diagonal;
//   3. M^-1 by one forward substitution per column (a warp each), reading
//      the lower triangle and writing column j of M^-1 transposed into row j
//      of the strictly upper triangle, which no solve reads;
//   4. U[a][b] = M^-1[K-1-a][K-1-b]: an anti-transpose of the upper triangle,
//      the reciprocal of the reversed diagonal, zeros below.
// The Hessian is bit-reproducible: every element is a sum of exact fp64
// products in ascending row order.
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_device.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kHT = 64;           // Hessian tile (rows and columns)
constexpr int kHR = 32;           // activation rows per staged chunk
constexpr int kWarps = 8;         // warps per block in the factor kernels

__device__ __forceinline__ double bf16_f64(uint16_t b) {
    return (double)__uint_as_float((uint32_t)b << 16);
}

// H[i][j] += sum_r x[r][i] x[r][j], tile 64 x 64 per block, 4 x 4 per thread.
__global__ void __launch_bounds__(256) hessian_kernel(const uint16_t* __restrict__ x, int R, int K,
                                                      double* __restrict__ H) {
    __shared__ double xi[kHR][kHT];
    __shared__ double xj[kHR][kHT];
    const int i0 = blockIdx.y * kHT, j0 = blockIdx.x * kHT;
    const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
    double acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
    for (int r0 = 0; r0 < R; r0 += kHR) {
        for (int e = tid; e < kHR * kHT; e += 256) {
            const int rr = e / kHT, c = e - rr * kHT, r = r0 + rr;
            xi[rr][c] = (r < R && i0 + c < K) ? bf16_f64(x[(size_t)r * K + i0 + c]) : 0.0;
            xj[rr][c] = (r < R && j0 + c < K) ? bf16_f64(x[(size_t)r * K + j0 + c]) : 0.0;
        }
        __syncthreads();
        const int rn = R - r0 < kHR ? R - r0 : kHR;
        for (int rr = 0; rr < rn; ++rr) {            // ascending rows
            double a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = xi[rr][4 * ti + u];
                b[u] = xj[rr][4 * tj + u];
            }
            // the product of two bf16 values is exact in fp64, so the fused
            // form rounds exactly like a product followed by a sum
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = __fma_rn(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = i0 + 4 * ti + u, j = j0 + 4 * tj + v;
            if (i < K && j < K) H[(size_t)i * K + j] = __dadd_rn(H[(size_t)i * K + j], acc[u][v]);
        }
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Step 1: A = J (H + lambda I) J with dead diagonal entries set to 1 first;
// lambda = damp * mean of that diagonal. Block a writes row a; block 0 also
// writes the dead flags.
__global__ void __launch_bounds__(256) gptq_reverse_kernel(const double* __restrict__ H, int K, double damp,
                                                           double* __restrict__ A, uint8_t* __restrict__ dead) {
    __shared__ double red[256];
    double part = 0.0;
    for (int k = threadIdx.x; k < K; k += 256) {
        const double h = H[(size_t)k * K + k];
        part += h == 0.0 ? 1.0 : h;
    }
    red[threadIdx.x] = part;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    const double lambda = damp * (red[0] / (double)K);
    const int a = blockIdx.x, ra = K - 1 - a;
    for (int b = threadIdx.x; b < K; b += 256) {
        const int rb = K - 1 - b;
        double v = H[(size_t)ra * K + rb];
        if (ra == rb) v = (v == 0.0 ? 1.0 : v) + lambda;
        A[(size_t)a * K + b] = v;
    }
    if (a == 0)
        for (int k = threadIdx.x; k < K; k += 256) dead[k] = H[(size_t)k * K + k] == 0.0 ? 1 : 0;
}

constexpr int kNB = 32;           // Cholesky block (columns)
constexpr int kCh = 128;          // left columns staged per round
constexpr int kDiagThreads = 1024;

// A pivot that is not positive: NaN, and the status bit (no fault).
__device__ __forceinline__ double chol_root(double d) {
    if (d > 0.0) return sqrt(d);
    atomicOr(&g_status, kStatusNotSpd);
    return __longlong_as_double(0x7ff8000000000000ll);
}

// Step 2a: the diagonal block [j0, j0 + nb) of the lower Cholesky factor (one
// CTA). G[r][c] (r >= c) = sum over p < j0 of L[j0+r][p] L[j0+c][p], thread
// (r, c) over the block's rows staged kCh columns at a time (in p order);
// then column by column: the pivot d_c from row c, and rows r > c of column
// c. G's lower part is overwritten by the block's L entries as they are
// formed. Writes the block's strictly lower entries into A, and d_c into
// A[j0+c][j0+c+1] (the strictly upper triangle is not read before step 3
// overwrites it), or onto the diagonal for the last row of A.
__global__ void __launch_bounds__(kDiagThreads) chol_block_diag_kernel(double* __restrict__ A, int K, int j0, int nb) {
    __shared__ double T[kNB][kCh + 1];
    __shared__ double G[kNB][kNB + 1];
    __shared__ double piv;
    const int tr = (int)threadIdx.x >> 5, tc = (int)threadIdx.x & 31;
    double g = 0.0;
    for (int p0 = 0; p0 < j0; p0 += kCh) {
        __syncthreads();
        for (int e = threadIdx.x; e < nb * kCh; e += kDiagThreads) {
            const int rr = e / kCh, l = e - rr * kCh;
            T[rr][l] = p0 + l < j0 ? A[(size_t)(j0 + rr) * K + p0 + l] : 0.0;
        }
        __syncthreads();
        if (tr < nb && tc <= tr)
            for (int l = 0; l < kCh; ++l) g = __fma_rn(T[tr][l], T[tc][l], g);
    }
    if (tr < nb && tc <= tr) G[tr][tc] = g;
    __syncthreads();
    for (int c = 0; c < nb; ++c) {
        if (threadIdx.x == 0) {
            double s = G[c][c];
            for (int q = 0; q < c; ++q) s = __fma_rn(G[c][q], G[c][q], s);
            const double d = chol_root(A[(size_t)(j0 + c) * K + j0 + c] - s);
            piv = d;
            if (j0 + c < K - 1) A[(size_t)(j0 + c) * K + j0 + c + 1] = d;
            else A[(size_t)(j0 + c) * K + j0 + c] = d;
        }
        __syncthreads();
        const int r = c + 1 + (int)threadIdx.x;
        if (r < nb) {
            double s = G[r][c];
            for (int q = 0; q < c; ++q) s = __fma_rn(G[r][q], G[c][q], s);
            const double v = (A[(size_t)(j0 + r) * K + j0 + c] - s) / piv;
            G[r][c] = v;
            A[(size_t)(j0 + r) * K + j0 + c] = v;
        }
        __syncthreads();
    }
}

// Step 2b: rows i >= j0 + nb of the block's columns, one warp per row: the
// sums over p < j0 of L[i][p] L[j0+c][p] for all c at once (the block's rows
// staged kCh columns at a time in shared memory; lane l takes p = l, l + 32,
// ... in order), then the forward solve with the block's lower triangle and
// pivots.
__global__ void __launch_bounds__(kWarps * 32) chol_block_panel_kernel(double* __restrict__ A, int K, int j0, int nb) {
    __shared__ double T[kNB][kCh + 1];                // T[c][l] = L[j0+c][p0+l]
    __shared__ double D[kNB][kNB + 1];                // the block: strict lower L, pivots on the diagonal
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = j0 + nb + (int)blockIdx.x * kWarps + warp;
    const bool act = i < K;
    for (int e = threadIdx.x; e < nb * nb; e += kWarps * 32) {
        const int r = e / nb, c = e - r * nb;
        if (r > c) D[r][c] = A[(size_t)(j0 + r) * K + j0 + c];
        else if (r == c) D[r][r] = A[(size_t)(j0 + r) * K + j0 + r + 1];   // j0 + r < K - 1 here
    }
    const double* Li = A + (size_t)(act ? i : j0) * K;
    double acc[kNB];
#pragma unroll
    for (int c = 0; c < kNB; ++c) acc[c] = 0.0;
    for (int p0 = 0; p0 < j0; p0 += kCh) {
        double li[kCh / 32];
#pragma unroll
        for (int k = 0; k < kCh / 32; ++k) {
            const int p = p0 + 32 * k + lane;
            li[k] = act && p < j0 ? Li[p] : 0.0;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nb * kCh; e += kWarps * 32) {
            const int c = e / kCh, l = e - c * kCh;
            T[c][l] = p0 + l < j0 ? A[(size_t)(j0 + c) * K + p0 + l] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kCh / 32; ++k)
#pragma unroll
            for (int c = 0; c < kNB; ++c)
                if (c < nb) acc[c] = __fma_rn(li[k], T[c][32 * k + lane], acc[c]);
    }
    __syncthreads();                                   // D is complete (also when j0 == 0)
    if (!act) return;
#pragma unroll
    for (int c = 0; c < kNB; ++c) acc[c] = warp_sum(acc[c]);
    double lr[kNB];                                    // L[i][j0 + c], the same in every lane
#pragma unroll
    for (int c = 0; c < kNB; ++c) {
        if (c < nb) {
            double s = acc[c];
#pragma unroll
            for (int q = 0; q < c; ++q) s = __fma_rn(lr[q], D[c][q], s);
            lr[c] = (Li[j0 + c] - s) / D[c][c];
        }
    }
    if (lane < nb) {
        double v = 0.0;
#pragma unroll
        for (int c = 0; c < kNB; ++c)
            if (c == lane) v = lr[c];
        A[(size_t)i * K + j0 + lane] = v;
    }
}

// Step 2c: the pivots onto the diagonal (the last row's is there already).
__global__ void chol_pivots_kernel(double* __restrict__ A, int K) {
    const int j = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    if (j < K - 1) A[(size_t)j * K + j] = A[(size_t)j * K + j + 1];
}

// Step 3: column j of M^-1 by forward substitution (M x = e_j): x_j = 1/M_jj,
// x_i = -(sum_{p=j}^{i-1} M_ip x_p) / M_ii for i > j, x in shared memory;
// x_i (i > j) goes to A[j][i]. One warp per column.
__global__ void __launch_bounds__(kWarps * 32) trinv_kernel(double* __restrict__ A, int K) {
    extern __shared__ double xs[];                    // one column of K values per warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x * (int)(blockDim.x >> 5) + warp;
    if (j >= K) return;
    double* x = xs + (size_t)warp * K;
    if (lane == 0) x[j] = 1.0 / A[(size_t)j * K + j];
    __syncwarp();
    for (int i = j + 1; i < K; ++i) {
        const double* Mi = A + (size_t)i * K;
        double s = 0.0;
        for (int p = j + lane; p < i; p += 32) s = __fma_rn(Mi[p], x[p], s);
        s = warp_sum(s);
        const double xi = -s / Mi[i];
        if (lane == 0) {
            x[i] = xi;
            A[(size_t)j * K + i] = xi;
        }
        __syncwarp();
    }
}

// Step 4: U[a][b] = Minv[K-1-a][K-1-b]. Minv[i][j] (i > j) sits at A[j][i],
// so U[a][b] (a < b) = A[K-1-b][K-1-a]: swap each strictly-upper pair across
// the anti-diagonal; U[a][a] = 1 / A[K-1-a][K-1-a]. One thread per element
// (r, c) with r <= c and r + c <= K - 1 (each pair once).
__global__ void gptq_finish_kernel(double* __restrict__ A, int K) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (long long)K * K) return;
    const int r = (int)(e / K), c = (int)(e % K);
    if (r > c || r + c > K - 1) return;
    const int r2 = K - 1 - c, c2 = K - 1 - r;             // partner (same element on the anti-diagonal)
    if (r == c) {                                      // diagonal pair (r, K-1-r)
        const double a = A[(size_t)r * K + r], b = A[(size_t)c2 * K + c2];
        A[(size_t)r * K + r] = 1.0 / b;
        if (c2 != r) A[(size_t)c2 * K + c2] = 1.0 / a;
        return;
    }
    const double v = A[(size_t)r * K + c], w = A[(size_t)r2 * K + c2];
    A[(size_t)r * K + c] = w;
    A[(size_t)r2 * K + c2] = v;
}

// Step 4, then: zeros strictly below the diagonal.
__global__ void gptq_lower_zero_kernel(double* __restrict__ A, int K) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (long long)K * K) return;
    const int r = (int)(e / K), c = (int)(e % K);
    if (r > c) A[(size_t)r * K + c] = 0.0;
}

}  // namespace

cudaError_t launch_hessian(const void* x, int R, int K, double* H, cudaStream_t st) {
    const dim3 grid((unsigned)((K + kHT - 1) / kHT), (unsigned)((K + kHT - 1) / kHT));
    hessian_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), R, K, H);
    return cudaGetLastError();
}

cudaError_t launch_gptq_prepare(const double* H, int K, double damp, double* U, uint8_t* dead, cudaStream_t st) {
    gptq_reverse_kernel<<<(unsigned)K, 256, 0, st>>>(H, K, damp, U, dead);
    cudaError_t e = cudaGetLastError();
    for (int j0 = 0; j0 < K && e == cudaSuccess; j0 += kNB) {
        const int nb = K - j0 < kNB ? K - j0 : kNB;
        chol_block_diag_kernel<<<1, kDiagThreads, 0, st>>>(U, K, j0, nb);
        e = cudaGetLastError();
        const int rows = K - j0 - nb;
        if (e == cudaSuccess && rows > 0) {
            chol_block_panel_kernel<<<(unsigned)((rows + kWarps - 1) / kWarps), kWarps * 32, 0, st>>>(U, K, j0, nb);
            e = cudaGetLastError();
        }
    }
    if (e != cudaSuccess) return e;
    chol_pivots_kernel<<<(unsigned)((K + 255) / 256), 256, 0, st>>>(U, K);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // forward substitutions: one column of K doubles in shared memory per warp; fewer warps per block
    // for wide K
    const size_t per = (size_t)K * sizeof(double);
    int w = kWarps;
    while (w > 1 && (size_t)w * per > 200 * 1024) w >>= 1;
    if ((size_t)w * per > 200 * 1024) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(trinv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    trinv_kernel<<<(unsigned)((K + w - 1) / w), w * 32, (size_t)w * per, st>>>(U, K);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long n = (long long)K * K;
    gptq_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(U, K);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gptq_lower_zero_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(U, K);
    return cudaGetLastError();
}

cudaError_t status_gptq(cudaStream_t st, unsigned* word) {
    unsigned v = 0, z = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &z, sizeof(z), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *word = v;
    return e;
}

}  // namespace rq
