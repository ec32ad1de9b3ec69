/*
 * rq.h -- C ABI of librq: weight-only group-quantized matrix products for
 * RWKV-7 decode and short prefill on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [ART]  "rwkv-quant: keeping one matrix in bf16 removes 39% of RWKV-7 2.9B's
 *          quantization loss", section "Two presets and six sizes": the
 *          REDUCTION preset keeps projections in 8 bits, symmetric, group 16;
 *          COMPRESSION keeps them in 4 bits with an asymmetric superblock
 *          layout and group 32; in both, each group's scale and shift are
 *          found by a search weighted by the input channel's E[x^2].
 *   [CARD] "RWKV-7 G1 1.5B -- int4 GPTQ for rwkv-sglang", section "Format &
 *          loading": symmetric int4 weights with group 64, stored as a code
 *          tensor plus a scale tensor; summary paragraph: the kernels' output
 *          is bit-identical to the offline dequantization, and an int4 GEMV /
 *          small-M GEMM / tensor-core GEMM family serves batches up to 32.
 *   [rwkv_quant_nv] "rwkv_quant_nv" project description, section "Operator
 *          Optimization Details": decode tile shapes for the 4096x4096,
 *          16384x4096 and 4096x16384 projections; r/k/v fused in one kernel;
 *          the activation statistic of its path computed on the device.
 *
 * Conventions shared by every call:
 *   - W is stored [N][K] row-major (row n = output feature, K = input
 *     features); groups run along K. x is bf16 [M][K], y is fp32 [M][N]
 *     (or bf16 with rq_wgemm_out / rq_wgemm_batch_out).
 *   - Every pointer named "device" is CUDA device memory that the CALLER
 *     allocated and owns; the library allocates nothing and keeps no state
 *     between calls. Every such pointer must be 16-byte aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as a
 *     plain pointer; NULL is the legacy default stream) and never
 *     synchronizes. Arguments are validated on the host before anything is
 *     launched; a failed validation launches nothing.
 *   - A launch that CUDA rejects returns RQ_ERR_CUDA; rq_last_cuda_error()
 *     then gives the cudaError_t value (per host thread).
 *   - Non-finite values in W, act_sq or x are outside the contract: the codes
 *     and outputs they produce are unspecified (but every access stays in
 *     bounds).
 *   - Calls made from several host threads on different streams are safe.
 */
#ifndef RQ_H
#define RQ_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rq_status {
    RQ_OK = 0,
    RQ_ERR_INVALID_ARG = 1,        /* NULL pointer, M/K/N or search outside range */
    RQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K not a multiple of the format's block size */
    RQ_ERR_FORMAT_MISMATCH = 3,    /* descriptor's fmt/K/N differ from the call's */
    RQ_ERR_MISALIGNED = 4,         /* a device pointer is not 16-byte aligned */
    RQ_ERR_CUDA = 5,               /* a CUDA runtime call failed */
    RQ_ERR_DEVICE_TIMEOUT = 6,     /* a bounded device wait gave up (see rq_device_status) */
    RQ_ERR_NOT_POSITIVE_DEFINITE = 7  /* a GPTQ factorization met a non-positive pivot (rq_device_status) */
} rq_status;

/* Packed formats.
 *
 * RQ_W4_SYM_G64 ([CARD] "Format & loading"): symmetric int4, group 64.
 *   codes  [N][K/2] bytes: byte j of row n holds k = 2j in its low nibble
 *          and k = 2j+1 in its high nibble; nibble = q + 8, q in [-7, 7].
 *   scales [N][K/64] fp16 (IEEE binary16, little-endian).
 *   w_hat = q * scale (exact in fp32). 4.25 bits per weight.
 *
 * RQ_W8_SYM_G16 ([ART], REDUCTION projections): symmetric int8, group 16.
 *   codes  [N][K] bytes, byte = q + 128, q in [-127, 127].
 *   scales [N][K/16] fp16.   w_hat = q * scale. 9 bits per weight.
 *
 * RQ_W8_SYM_G64 ([CARD] "Accuracy warning": the int8 w8g64 tier it recommends
 *   for reasoning-heavy use): RQ_W8_SYM_G16 with groups of 64: scales
 *   [N][K/64] fp16. 8.25 bits per weight.
 *
 * RQ_W6_SYM_G16 ([ART], the REDUCTION preset's channel-mix in 6 bits):
 *   symmetric, group 16, q in [-31, 31], u = q + 32 in [1, 63].
 *   codes  [N][K/64 * 48] bytes, one 48-byte chunk per 64 weights j = 0..63:
 *          [0:32]  low 4 bits of u_j: byte j/2, low nibble for even j
 *          [32:48] bits 4..5 of u_j in bits 2 (j % 4) .. +1 of byte 32 + j/4
 *   scales [N][K/16] fp16.   w_hat = q * scale. 7 bits per weight.
 *
 * RQ_W4_ASYM_SB32 ([ART], COMPRESSION projections): asymmetric int4 in
 *   superblocks of 256 weights = 8 groups of 32 along K; one 144-byte record
 *   per superblock, records [N][K/256]:
 *     [0:2]    fp16 d      superblock scale
 *     [2:4]    fp16 dmin   superblock min
 *     [4:16]   96-bit little-endian bit string; bits 6j..6j+5 = sc_j,
 *              bits 48+6j..48+6j+5 = m_j (6-bit, j = 0..7)
 *     [16:144] 128 code bytes, nibble order as RQ_W4_SYM_G64, code = q in [0, 15]
 *   Group j: S_j = d * sc_j, M_j = dmin * m_j; w_hat = S_j * q - M_j
 *   (S_j * q exact, one fp32 rounding). 4.5 bits per weight; scales = NULL.
 *
 * RQ_W5_ASYM_SB32, RQ_W6_ASYM_SB32 ([ART], the COMPRESSION preset's wider
 *   matrices; +1 and +2 bits per weight, the o_proj file-size deltas the
 *   article quotes): the RQ_W4_ASYM_SB32 record with the codes' low 4 bits in
 *   [16:144] and a high-bit plane appended; q in [0, 31] or [0, 63]:
 *     5 bits, 176-byte records: [144:176] bit 4 of code k in bit k % 8 of
 *             byte 144 + k / 8
 *     6 bits, 208-byte records: [144:208] bits 4..5 of code k in bits
 *             2 (k % 4) .. 2 (k % 4) + 1 of byte 144 + k / 4
 *   The group search spans 2^b - 1 steps (S = 2 r / (2^b - 1)); the rest is
 *   as RQ_W4_ASYM_SB32. 5.5 and 6.5 bits per weight; scales = NULL.
 */
typedef enum rq_format {
    RQ_W4_SYM_G64 = 1,
    RQ_W8_SYM_G16 = 2,
    RQ_W4_ASYM_SB32 = 3,
    RQ_W5_ASYM_SB32 = 4,
    RQ_W6_ASYM_SB32 = 5,
    RQ_W8_SYM_G64 = 6,
    RQ_W6_SYM_G16 = 7
} rq_format;

/* Candidate grid of the E[x^2]-weighted search ([ART]): n_cand points
 * t_i = fp32(t_lo + (t_hi - t_lo) * i / (n_cand - 1)) computed in fp64
 * (n_cand = 1 gives the single point t_hi). {1, 1.0, 1.0} is plain RTN;
 * the default (search == NULL) is {64, 0.7, 1.0}.
 * Limits: 1 <= n_cand <= 256, 0 < t_lo <= t_hi <= 4. */
typedef struct rq_search {
    int n_cand;
    float t_lo;
    float t_hi;
} rq_search;

/* Descriptor of one packed matrix. A host struct holding device pointers;
 * the caller fills it and owns both planes. scales is NULL for the
 * superblock formats (RQ_W4/W5/W6_ASYM_SB32). */
typedef struct rq_packed {
    int fmt;        /* rq_format */
    int K;          /* input features */
    int N;          /* output features */
    int reserved;   /* must be 0 */
    void *codes;    /* device, rq_packed_size(...) codes_bytes */
    void *scales;   /* device, rq_packed_size(...) scales_bytes, or NULL */
} rq_packed;

/* Shape limits: 1 <= N <= 2^24; 64 <= K <= 32768 with K % 64 == 0
 * (K % 256 == 0 for the superblock formats); 1 <= M <= 128. */

/* Bytes of the two planes of a packed [N][K] matrix; the scales plane is
 * rounded up to a multiple of 16 bytes (the padding is written as zero by
 * rq_quantize_pack). Returns the total, or 0 for an unknown format or an
 * unsupported shape. Either out-pointer may be NULL. Host only; no CUDA call. */
size_t rq_packed_size(int fmt, int K, int N, size_t *codes_bytes, size_t *scales_bytes);

/* Quantize and pack W.  ([ART] "Two presets and six sizes"; [CARD])
 *   W      device fp32 [N][K]
 *   act_sq device fp32 [K], E[x_k^2] of the input channels, the weights of
 *          the search's loss; NULL means every a_k = 1 (plain MSE search).
 *   search candidate grid; NULL means {64, 0.7, 1.0}.
 *   out    descriptor whose fmt/K/N must equal the call's and whose planes
 *          receive the codes and scales.
 * For each symmetric group: absmax = max|w|, base = absmax / qmax (fp32,
 * qmax = 7, 31 or 127); candidate i has scale s_i = fp16(t_i * base); its loss is
 * sum_k a_k (w_k - q_k s_i)^2 with q_k = clamp(rint(w_k / s_i), -qmax, qmax),
 * evaluated in fp64 in ascending k; the lowest index attaining the minimum
 * wins. For each asymmetric group of 32: lo = min(0, min w),
 * hi = max(0, max w), candidate i shrinks [lo, hi] about its midpoint by t_i
 * (S_i = 2 r_i / L, M_i = max(0, r_i - mid), r_i = t_i (hi - lo) / 2,
 * L = 2^b - 1 = 15, 31 or 63 for b-bit codes),
 * codes q = clamp(rint((w + M_i) / S_i), 0, L), the same loss and tie rule;
 * then d = fp16(max_j S_j / 63), dmin = fp16(max_j M_j / 63), 6-bit
 * sc_j = rint(S_j / d), m_j = rint(M_j / dmin), and the final codes use the
 * stored S_j = d sc_j, M_j = dmin m_j. The output is byte-for-byte
 * deterministic. */
int rq_quantize_pack(const float *W, int K, int N, const float *act_sq,
                     const rq_search *search, const rq_packed *out, void *stream);

/* y = x * w_hat^T.  ([CARD] summary: an int4 GEMV / small-M GEMM /
 * tensor-core GEMM family serving batches of 1..32; [ART]: the same product
 * over the REDUCTION and COMPRESSION projection formats)
 *   x   device bf16 [M][K] (raw bf16 bit patterns, row-major)
 *   M   activation rows, 1..128
 *   K,N must equal the descriptor's
 *   w   packed matrix
 *   y   device fp32 [M][N], overwritten (not accumulated into)
 * w_hat is formed in registers (M <= 2: CUDA-core GEMV, exact fp32 w_hat) or
 * in tensor memory (M >= 3, and every M for the 5- and 6-bit formats
 * RQ_W5/W6_ASYM_SB32 and RQ_W6_SYM_G16: tensor-core kernel, w_hat rounded
 * once to bf16)
 * and never written out; the products accumulate in fp32. Kernels are launched with programmatic
 * dependent launch allowed: they read the packed weights while the kernel
 * launched just before them on the stream may still be running, and read x
 * and write y only after it has completed. So the packed planes must not be
 * written by the kernel launched immediately before rq_wgemm on the same
 * stream (rq_quantize_pack already ends with a kernel that makes this hold;
 * after writing the planes with your own kernel, synchronize or launch any
 * other kernel in between). Copies (cudaMemcpy*) are ordered as usual. */
int rq_wgemm(const void *x, int M, int K, int N, const rq_packed *w, float *y, void *stream);

/* One product of a batch: y = x * w_hat^T. */
typedef struct rq_wgemm_item {
    const void *x;          /* device bf16 [M][K] */
    const rq_packed *w;     /* packed matrix (host descriptor) */
    void *y;                /* device [M][N], overwritten: fp32 (rq_wgemm_batch,
                               RQ_OUT_F32) or bf16 (RQ_OUT_BF16) */
} rq_wgemm_item;

/* `count` independent products in ONE launch, e.g. the r, k and v
 * projections of a layer ([rwkv_quant_nv] "Operator Optimization Details":
 * r/k/v computed in a single kernel). Every item has the same format and the
 * same M; shapes may differ. The result equals `count` rq_wgemm calls. The
 * launch's CTAs split the items' work evenly (packed bytes for M <= 2,
 * 128-row tiles for M >= 3), so small matrices share the GPU instead of
 * leaving it idle between launches; above 96 items the tensor-core path
 * takes one launch per 96 items.
 *   items  host array of `count` items, 1 <= count <= 160
 *   M      activation rows of every item, 1..128
 * No y may overlap another item's y or any x. Same validation, status codes
 * and ordering rules as rq_wgemm (the packed planes must not be written by
 * the kernel launched just before this call on the stream). */
int rq_wgemm_batch(const rq_wgemm_item *items, int count, int M, void *stream);

/* Output element types of rq_wgemm_out / rq_wgemm_batch_out. */
typedef enum rq_out_type {
    RQ_OUT_F32 = 0,         /* fp32, as rq_wgemm */
    RQ_OUT_BF16 = 1         /* the fp32 result rounded once to bf16 (nearest even) */
} rq_out_type;

/* rq_wgemm / rq_wgemm_batch with the output element type chosen: y is fp32
 * [M][N] (RQ_OUT_F32) or bf16 [M][N] (RQ_OUT_BF16). The bf16 result is
 * exactly the RQ_OUT_F32 result rounded to nearest even, written by the same
 * launch (no second pass over y), so a batched r/k/v launch
 * ([rwkv_quant_nv] "Operator Optimization Details": r/k/v in one kernel) can
 * hand its outputs on in the bf16 that every product here takes as x (the
 * pages give no output type; this one is this library's choice). Same
 * validation and ordering rules as rq_wgemm; any other out_type is
 * RQ_ERR_INVALID_ARG. */
int rq_wgemm_out(const void *x, int M, int K, int N, const rq_packed *w, void *y, int out_type, void *stream);
int rq_wgemm_batch_out(const rq_wgemm_item *items, int count, int M, int out_type, void *stream);

/* Export w_hat as fp32 [N][K] into W_out (device).  ([CARD] summary: the
 * kernel output is bit-identical to the offline dequantization.) Bit-exact:
 * q * scale for the symmetric formats, fp32(S_j * q - M_j) for the
 * superblock formats, the values the oracle's dequantization gives. The
 * products do not go through this export: rq_wgemm unpacks the same codes
 * with its own in-register arithmetic (see there for its rounding), so its
 * outputs agree with x * (this w_hat)^T within the stated tolerance, and
 * exactly whenever every partial sum is exact (integer-valued cases). */
int rq_dequant(const rq_packed *w, float *W_out, void *stream);

/* Accumulate the statistic of the E[x^2]-weighted search on the device.
 * ([ART] "Two presets and six sizes": the search weights input channel k by
 * E[x_k^2]; [rwkv_quant_nv] "Operator Optimization Details": the activation
 * statistic is computed on the device.)
 *   x       device bf16 [R][K], calibration activations (raw bf16 bits)
 *   sum_sq  device fp64 [K], caller-owned running sums: the call adds
 *           sum_r x[r][k]^2 to sum_sq[k]. Zero it before the first batch;
 *           call once per batch of rows.
 * The statistic is the mean of x_k^2 over all calibration rows; the pages fix
 * no summation order. Squares of bf16 values are exact in fp64, so the result
 * differs from one ascending fp64 sum over the rows only by the rounding of
 * the additions: |difference| <= 2 (R + 1) 2^-53 sum_sq[k] (and none at all
 * when every partial sum is exact, e.g. for activations that are small
 * multiples of a common power of two). The device order is fixed (each CTA
 * sums interleaved rows ascending, then its row phases and the CTAs of a
 * cluster in order), so repeated calls give the same bits.
 * Limits: 1 <= R <= 2^24, 1 <= K <= 2^20. Non-finite x: unspecified. */
int rq_act_sumsq(const void *x, int R, int K, double *sum_sq, void *stream);

/* act_sq[k] = fp32(sum_sq[k] / rows) (one fp64 division, one rounding to
 * fp32), the E[x^2] that rq_quantize_pack takes.
 *   sum_sq  device fp64 [K] from rq_act_sumsq; act_sq device fp32 [K];
 *   rows    total calibration rows summed, >= 1. */
int rq_act_finalize(const double *sum_sq, int K, long long rows, float *act_sq, void *stream);

/* GPTQ on the preset's grid ([ART] "Calibration leakage and honest
 * measurements": GPTQ on the preset's grid without changing the format, the
 * kernels or the file size; [CARD]: symmetric int4 group 64, GPTQ-calibrated).
 * The method is GPTQ (Frantar et al., 2022), in three calls:
 *
 * rq_hessian_accum: H += x^T x for the layer's calibration inputs.
 *   x  device bf16 [R][K] (raw bits), H device fp64 [K][K], caller-owned,
 *   zeroed before the first batch. Each element is summed in fp64 in
 *   ascending row order from 0 and then added to H (products of bf16 values
 *   are exact in fp64, so the result is bit-reproducible). GPTQ's factor
 *   2/rows is left out: it scales H uniformly and the damping is relative.
 *   Limits: 1 <= R <= 2^24, 1 <= K <= 32768. */
int rq_hessian_accum(const void *x, int R, int K, double *H, void *stream);

/* rq_gptq_prepare: the factor of the column loop.
 *   H     device fp64 [K][K] (read only)
 *   damp  relative damping (GPTQ's usual value: 0.01), finite, >= 0
 *   U     device fp64 [K][K], out: the upper Cholesky factor of the inverse of
 *         H' = H with zero diagonal entries set to 1, plus damp * mean(diag)
 *         on the diagonal (H'^-1 = U^T U; zeros below the diagonal). U is the
 *         workspace too; it must not overlap H.
 *   dead  device [K] bytes, out: 1 where H's diagonal entry was 0.
 * Computed as J inv(chol(J H' J)) J (J reverses the index order): one
 * Cholesky (two launches per block of 32 columns) and one triangular inverse
 * (a warp per column).
 * A non-positive pivot sets bit 5 of the device status word (see
 * rq_device_status) and leaves NaNs in U. Limits: 1 <= K <= 16384. */
int rq_gptq_prepare(const double *H, int K, double damp, double *U, unsigned char *dead, void *stream);

/* rq_gptq_quantize_pack: quantize W into `out` (any format; the same
 * planes as rq_quantize_pack). Per row, in fp64, columns in order; dead
 * columns start at 0.
 *   Symmetric formats: at each group's first column the group's scale is
 *   rq_quantize_pack's search (act_sq, search as there) on the group's
 *   current weights rounded to fp32; then q_k = clamp(rint(fp32(w_k) / s),
 *   +-qmax) and w_hat_k = q_k s.
 *   Superblock formats: at each superblock's first column its eight groups
 *   are searched and its header (d, dmin, 6-bit fields) formed as
 *   rq_quantize_pack does, on the current weights rounded to fp32; then
 *   q_k = clamp(rint((fp32(w_k) + M_j) / S_j), 0, 2^b - 1) with the stored
 *   S_j, M_j and w_hat_k = fp32(S_j q_k) - M_j.
 * In both: err = (w_k - w_hat_k) / U[k][k] and w_j -= err * U[k][j] for j > k.
 *   W device fp32 [N][K]; U, dead from rq_gptq_prepare. K <= 16384.
 * Same ordering rules as rq_quantize_pack. */
int rq_gptq_quantize_pack(const float *W, int K, int N, const double *U, const unsigned char *dead,
                          const float *act_sq, const rq_search *search, const rq_packed *out, void *stream);

/* Static description of a status code. Never NULL. */
const char *rq_status_string(int status);

/* cudaError_t of the last RQ_ERR_CUDA returned on this host thread (0 if none). */
int rq_last_cuda_error(void);

/* Reads and clears the device status word that bounded waits inside the
 * kernels set when they give up, and that rq_gptq_prepare sets for a
 * non-positive pivot (bit 5). Synchronizes `stream`. Writes the word to *word
 * (0 = nothing since the last read) and returns RQ_OK,
 * RQ_ERR_DEVICE_TIMEOUT if a wait bit was set, RQ_ERR_NOT_POSITIVE_DEFINITE
 * if only the pivot bit was, or RQ_ERR_CUDA. */
int rq_device_status(void *stream, int *word);

/* Testing hook for the bounded device waits (the pages have no counterpart;
 * this exists so that the give-up paths can be exercised without a fault).
 * Every later launch from any host thread uses:
 *   wait_ns  the bound of each device wait, in nanoseconds; 0 restores the
 *            default of 2 s. At most 60 s.
 *   flags    bit 0 (1): the threads that issue the weight copies of the
 *            products issue none, so every wait for a copy runs out after
 *            wait_ns; the call then completes with unspecified y and
 *            rq_device_status reports RQ_ERR_DEVICE_TIMEOUT. 0 = normal.
 * Returns RQ_ERR_INVALID_ARG for other values. Not for production use: set
 * it back with rq_test_hooks(0, 0). */
int rq_test_hooks(long long wait_ns, int flags);

/* Library version, major * 10000 + minor * 100 + patch. */
int rq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RQ_H */
