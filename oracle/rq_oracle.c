/*
 * rq_oracle.c -- the CPU oracle for weight-only group quantization.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load this file's library. The product (the CUDA library)
 * shares no code, header, table or constant with it, and never calls it.
 *
 * What it computes, step by step, in plain loops:
 *   - symmetric group quantization (RTN, or a grid search weighted by the
 *     per-channel mean square of the input activation, E[x^2]) into the int4
 *     group-64, int8 group-16 / group-64 and 6-bit group-16 formats;
 *   - the asymmetric 4-, 5- and 6-bit superblock formats (groups of 32, eight
 *     groups per superblock, 6-bit group scale and min against fp16
 *     superblock scale/min);
 *   - exact fp32 dequantization of every format;
 *   - the product y[m][n] = sum_k x[m][k] * w_hat[n][k], summed in fp64 in
 *     ascending k;
 *   - the activation statistic E[x^2] in a fixed fp64 summation order;
 *   - GPTQ on the preset's grid: the input Hessian and the column loop with
 *     error feedback into every format (the factor U of the damped inverse
 *     Hessian is computed in oracle/__init__.py with numpy's LAPACK steps).
 *
 * Sources (web pages; cited by title and section):
 *   [ART]  "rwkv-quant: keeping one matrix in bf16 removes 39% of RWKV-7 2.9B's
 *          quantization loss", section "Two presets and six sizes": REDUCTION
 *          projections are 8-bit symmetric with a group of 16; COMPRESSION
 *          projections are 4-bit with an asymmetric superblock layout and a
 *          group of 32; in both presets every group's scale and shift come from
 *          a search weighted by E[x^2] of the input channel.
 *   [CARD] "RWKV-7 G1 1.5B -- int4 GPTQ for rwkv-sglang" (model card), section
 *          "Format & loading": group-wise (group 64) symmetric int4 weights
 *          stored as a code tensor plus a scale tensor; summary paragraph:
 *          kernel output is bit-identical to the offline dequantization, and
 *          calibration-free RTN is the baseline; section "Accuracy warning":
 *          the int8 w8g64 tier.
 *
 * Where the pages leave a step open the plainest reading is taken; every such
 * reading is listed in the design notes and restated at the function below.
 *
 * Floating point: every fp32 and fp64 operation here is a single IEEE
 * round-to-nearest-even operation. The file must be built with
 * -ffp-contract=off and without fast-math (x86-64 SSE, FLT_EVAL_METHOD 0), so
 * that no multiply-add is fused and no sum is reassociated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must not be built with fast-math"
#endif

#define ORC_W4G64 1
#define ORC_W8G16 2
#define ORC_W4SB32 3
#define ORC_W5SB32 4
#define ORC_W6SB32 5
#define ORC_W8G64 6
#define ORC_W6G16 7

/* Bits per code and group size of the symmetric formats. */
static int sym_bits(int fmt) { return fmt == ORC_W4G64 ? 4 : (fmt == ORC_W6G16 ? 6 : 8); }
static int sym_gsize(int fmt) { return (fmt == ORC_W4G64 || fmt == ORC_W8G64) ? 64 : 16; }

/* Bits per code and record bytes of the superblock formats (4, 5, 6 bits:
 * 144, 176, 208 bytes per 256 weights). */
static int sb_bits(int fmt) { return fmt == ORC_W6SB32 ? 6 : (fmt == ORC_W5SB32 ? 5 : 4); }
static int sb_bytes(int bits) { return 16 + 128 + (bits - 4) * 32; }

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* IEEE binary16 from binary32, round to nearest, ties to even, with
 * subnormals, overflow to infinity, and NaN kept quiet. Written from the
 * IEEE 754 definition: keep 11 significant bits for normals, a fixed ulp of
 * 2^-24 below 2^-14. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t x = f2u(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);
    if (ax == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);
    int be = (int)(ax >> 23);
    uint32_t sig = (ax & 0x7fffffu) | (be ? 0x800000u : 0u); /* 24-bit significand */
    int ue = be ? be - 127 : -126;            /* exponent of significand bit 23 */
    if (ue > 15) return (uint16_t)(sign | 0x7c00u);
    int shift = (ue >= -14) ? 13 : 13 + (-14 - ue);
    if (shift > 24) return sign;               /* below 2^-25: rounds to zero */
    uint32_t kept = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t halfway = 1u << (shift - 1);
    if (rem > halfway || (rem == halfway && (kept & 1u))) kept++;
    if (ue >= -14) {
        int he = ue + 15;
        if (kept == 0x800u) { kept = 0x400u; he++; }
        if (he >= 31) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | ((uint32_t)he << 10) | (kept & 0x3ffu));
    }
    return (uint16_t)(sign | kept);            /* subnormal (0x400 = min normal) */
}

float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    int he = (h >> 10) & 0x1f;
    uint32_t m = h & 0x3ffu;
    if (he == 0) {
        float v = (float)m * 5.9604644775390625e-08f; /* m * 2^-24, exact */
        return sign ? -v : v;
    }
    if (he == 31) return u2f(sign | 0x7f800000u | (m << 13));
    return u2f(sign | ((uint32_t)(he - 15 + 127) << 23) | (m << 13));
}

float orc_bf16_to_f32(uint16_t b) { return u2f((uint32_t)b << 16); }

void orc_f32_to_f16_n(const float *in, uint16_t *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_f32_to_f16(in[i]);
}

void orc_f16_to_f32_n(const uint16_t *in, float *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_f16_to_f32(in[i]);
}

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ------------------------------------------------------------------------ */
/* Candidate grid                                                           */
/* ------------------------------------------------------------------------ */

/* [ART] says only that the group scale is found by a search. The grid is the
 * plainest reading of "64 candidates in [0.7, 1.0] * absmax / qmax": n points
 * uniformly spaced and including both ends, each computed in fp64 and rounded
 * once to fp32:  t_i = fl32(lo + (hi - lo) * i / (n - 1)).  n = 1 gives the
 * single point hi (RTN when hi = 1). */
void orc_grid(int n, float t_lo, float t_hi, float *t)
{
    if (n == 1) { t[0] = t_hi; return; }
    double lo = (double)t_lo, hi = (double)t_hi;
    for (int i = 0; i < n; i++) {
        double step = (hi - lo) * (double)i;
        step = step / (double)(n - 1);
        t[i] = (float)(lo + step);
    }
}

/* ------------------------------------------------------------------------ */
/* Symmetric group: search and codes                                        */
/* ------------------------------------------------------------------------ */

/* Codes of one symmetric group for the fp32 scale sf:
 *   q_k = clamp(rint(w_k / sf), -qmax, qmax),  and q_k = 0 when sf == 0.
 * Symmetric codes ([ART], [CARD]) use qmax = 2^(b-1) - 1, so -2^(b-1) is never
 * emitted. rint rounds half to even. */
static int sym_code(float w, float sf, int qmax)
{
    if (sf == 0.0f) return 0;
    float v = w / sf;
    float r = rintf(clampf(v, -(float)qmax, (float)qmax));
    return (int)r;
}

/* Weighted squared error of one candidate:
 *   L = sum_k a_k * (w_k - q_k * sf)^2
 * with q_k * sf in fp32 (exact: |q| < 2^7, sf has 11 significant bits), the
 * difference, square, product and sum in fp64, in ascending k. */
static double sym_loss(const float *w, const float *a, int G, float sf, int qmax)
{
    double L = 0.0;
    for (int k = 0; k < G; k++) {
        float wq = (float)sym_code(w[k], sf, qmax) * sf;
        double d = (double)w[k] - (double)wq;
        double e = d * d;
        double ak = a ? (double)a[k] : 1.0;
        L = L + ak * e;
    }
    return L;
}

/* One symmetric group: the E[x^2]-weighted search of [ART].
 *   absmax = max_k |w_k|;  base = absmax / qmax  (fp32 division)
 *   candidate i: s_i = fp16(t_i * base);  sf_i = fp32(s_i)
 *   pick the first i whose loss is strictly below every earlier loss, so the
 *   lowest index wins ties.
 * The loss is evaluated on the stored (fp16) scale: the search optimises what
 * is kept. Returns the chosen index; writes the fp16 scale bits, the codes and,
 * if losses != NULL, every candidate's loss. */
int orc_sym_group(const float *w, const float *a, int G, int qmax,
                  const float *t, int n, uint16_t *s_out, int8_t *q_out, double *losses)
{
    float absmax = 0.0f;
    for (int k = 0; k < G; k++) {
        float v = fabsf(w[k]);
        if (v > absmax) absmax = v;
    }
    float base = absmax / (float)qmax;
    int best = 0;
    double bestL = 0.0;
    uint16_t bests = 0;
    for (int i = 0; i < n; i++) {
        float prod = t[i] * base;
        uint16_t sh = orc_f32_to_f16(prod);
        float sf = orc_f16_to_f32(sh);
        double L = sym_loss(w, a, G, sf, qmax);
        if (losses) losses[i] = L;
        if (i == 0 || L < bestL) { best = i; bestL = L; bests = sh; }
    }
    float sf = orc_f16_to_f32(bests);
    for (int k = 0; k < G; k++) q_out[k] = (int8_t)sym_code(w[k], sf, qmax);
    *s_out = bests;
    return best;
}

/* Pack a whole [N][K] fp32 matrix (row n = output feature, groups along K)
 * into a symmetric format.
 *   int4 group 64: codes [N][K/2] bytes, byte j of a row holds k = 2j in its
 *                  low nibble and k = 2j+1 in its high nibble, nibble = q + 8;
 *                  scales [N][K/64] fp16.                         ([CARD])
 *   int8 group 16: codes [N][K] bytes, byte = q + 128; scales [N][K/16] fp16.
 *                                                                   ([ART])
 *   int8 group 64: the int8 codes with scales [N][K/64] fp16 (the int8 w8g64
 *                  tier that [CARD] "Accuracy warning" recommends).
 *   6-bit group 16 (REDUCTION preset's channel-mix, [ART]): qmax = 31,
 *                  u = q + 32 in [1, 63]; codes [N][K/64 * 48] bytes, one
 *                  48-byte chunk per 64 weights j = 0..63 of a row:
 *                    bytes [0:32]  low 4 bits of u_j: byte j/2, low nibble for
 *                                  even j, high nibble for odd j
 *                    bytes [32:48] bits 4..5 of u_j in bits 2 (j % 4) .. +1
 *                                  of byte 32 + j/4
 *                  scales [N][K/16] fp16. 7 bits per weight. The layout is
 *                  this project's own (the pages give only the bit width).
 * a == NULL means every a_k = 1 (plain MSE search). */
/* Write the codes of row n (qrow[k], k = 0..K-1) in the format's layout. */
static void emit_sym_row(uint8_t *codes, int bits, int K, int n, const int8_t *qrow)
{
    for (size_t kk = 0; kk < (size_t)K; kk++) {
        int qk = qrow[kk];
        if (bits == 8) {
            codes[(size_t)n * K + kk] = (uint8_t)(qk + 128);
        } else if (bits == 6) {
            int u = qk + 32;
            uint8_t *chunk = codes + (size_t)n * (K / 64 * 48) + (kk / 64) * 48;
            size_t j = kk % 64;
            if ((j & 1) == 0) chunk[j / 2] = (uint8_t)(u & 15);
            else chunk[j / 2] = (uint8_t)(chunk[j / 2] | ((u & 15) << 4));
            if (j % 4 == 0) chunk[32 + j / 4] = 0;
            chunk[32 + j / 4] |= (uint8_t)((u >> 4) << (2 * (j % 4)));
        } else {
            uint8_t u = (uint8_t)(qk + 8);
            uint8_t *byte = codes + (size_t)n * (K / 2) + kk / 2;
            if ((kk & 1) == 0) *byte = u;
            else *byte = (uint8_t)(*byte | (u << 4));
        }
    }
}

void orc_pack_sym(const float *W, int K, int N, const float *a, int fmt,
                  int n_cand, float t_lo, float t_hi, uint8_t *codes, uint16_t *scales)
{
    int bits = sym_bits(fmt);
    int G = sym_gsize(fmt);
    int qmax = (1 << (bits - 1)) - 1;
    int ng = K / G;
    float *t = (float *)malloc(sizeof(float) * (size_t)n_cand);
    orc_grid(n_cand, t_lo, t_hi, t);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < N; n++) {
        int8_t *qrow = (int8_t *)malloc((size_t)K);
        const float *row = W + (size_t)n * K;
        for (int g = 0; g < ng; g++) {
            uint16_t s;
            orc_sym_group(row + (size_t)g * G, a ? a + (size_t)g * G : NULL, G, qmax,
                          t, n_cand, &s, qrow + (size_t)g * G, NULL);
            scales[(size_t)n * ng + g] = s;
        }
        emit_sym_row(codes, bits, K, n, qrow);
        free(qrow);
    }
    free(t);
}

/* ------------------------------------------------------------------------ */
/* GPTQ on the preset's grid (symmetric formats)                            */
/* ------------------------------------------------------------------------ */

/* Running Hessian of the layer's input: H[i][j] += sum_r x[r][i] * x[r][j]
 * over the R bf16 rows of this call (row-major [R][K]), every element summed
 * in fp64 in ascending r starting from 0, then added to H. Products of two
 * bf16 values are exact in fp64. GPTQ's factor 2/R scales H uniformly and
 * changes nothing below (the damping is relative), so it is left out. */
void orc_hessian_accum(const uint16_t *x, int R, int K, double *H)
{
#pragma omp parallel for schedule(static)
    for (int i = 0; i < K; i++) {
        for (int j = 0; j < K; j++) {
            double acc = 0.0;
            for (int r = 0; r < R; r++) {
                double xi = (double)orc_bf16_to_f32(x[(size_t)r * K + i]);
                double xj = (double)orc_bf16_to_f32(x[(size_t)r * K + j]);
                acc = acc + xi * xj;
            }
            H[(size_t)i * K + j] = H[(size_t)i * K + j] + acc;
        }
    }
}

/* GPTQ (Frantar et al., "GPTQ: Accurate Post-Training Quantization for
 * Generative Pre-trained Transformers", 2022), restated for the preset's
 * symmetric formats; [ART] "Calibration leakage and honest measurements": GPTQ
 * on the preset's grid without changing the format, the kernels or the file size;
 * [CARD]: symmetric int4 group 64, GPTQ-calibrated.
 *   U       fp64 [K][K], the upper Cholesky factor of the damped inverse
 *           Hessian (H^-1 = U^T U; only the upper triangle is read)
 *   dead    [K], 1 where the Hessian's diagonal was 0: those columns of W
 *           are set to 0 before quantization
 * Per row, columns k = 0..K-1 in order, w the row in fp64:
 *   at the first column of each group: the group's scale is the preset's
 *   E[x^2]-weighted search (orc_sym_group) on fp32(w) of the group's current
 *   weights;
 *   q_k = clamp(rint(fp32(w_k) / s), -qmax, qmax);
 *   err = (w_k - q_k s) / U[k][k];  w_j = w_j - err * U[k][j] for j > k
 *   (fp64, one rounding per operation, the updates of w_j in ascending k).
 * The codes and scales land in the same planes as orc_pack_sym's. */
void orc_gptq_pack_sym(const float *W, int K, int N, const double *U, const uint8_t *dead,
                       const float *a, int fmt, int n_cand, float t_lo, float t_hi,
                       uint8_t *codes, uint16_t *scales)
{
    int bits = sym_bits(fmt);
    int G = sym_gsize(fmt);
    int qmax = (1 << (bits - 1)) - 1;
    int ng = K / G;
    float *t = (float *)malloc(sizeof(float) * (size_t)n_cand);
    orc_grid(n_cand, t_lo, t_hi, t);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < N; n++) {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        int8_t *qrow = (int8_t *)malloc((size_t)K);
        for (int k = 0; k < K; k++) w[k] = dead[k] ? 0.0 : (double)W[(size_t)n * K + k];
        for (int g = 0; g < ng; g++) {
            int k0 = g * G;
            float wg[64];
            int8_t qg[64];
            uint16_t s;
            for (int i = 0; i < G; i++) wg[i] = (float)w[k0 + i];
            orc_sym_group(wg, a ? a + k0 : NULL, G, qmax, t, n_cand, &s, qg, NULL);
            scales[(size_t)n * ng + g] = s;
            float sf = orc_f16_to_f32(s);
            for (int i = 0; i < G; i++) {
                int k = k0 + i;
                int q = sym_code((float)w[k], sf, qmax);
                qrow[k] = (int8_t)q;
                double d = w[k] - (double)((float)q * sf);
                double err = d / U[(size_t)k * K + k];
                for (int j = k + 1; j < K; j++) w[j] = w[j] - err * U[(size_t)k * K + j];
            }
        }
        emit_sym_row(codes, bits, K, n, qrow);
        free(w);
        free(qrow);
    }
    free(t);
}

/* ------------------------------------------------------------------------ */
/* Asymmetric superblock: group search, superblock scales, codes           */
/* ------------------------------------------------------------------------ */

/* Codes of one asymmetric group with scale S and min offset M (w_hat = S*q - M):
 *   q = clamp(rint((w + M) / S), 0, L),  L = 2^bits - 1,  and q = 0 when S == 0. */
static int asym_code(float w, float S, float M, int L)
{
    if (S == 0.0f) return 0;
    float v = (w + M) / S;
    return (int)rintf(clampf(v, 0.0f, (float)L));
}

static float asym_deq(int q, float S, float M)
{
    float p = (float)q * S;
    return p - M;
}

/* One asymmetric group of G (= 32) weights with codes of `bits` bits: the
 * E[x^2]-weighted scale/shift search of [ART] applied to the COMPRESSION
 * preset's asymmetric layout (4 bits for projections; 5 and 6 bits for the
 * channel-mix key, head, embedding and LoRA weights of that preset).
 * The pages name the search but not its candidates; the reading taken here:
 *   lo = min(0, min w), hi = max(0, max w), levels = 2^bits - 1
 *   candidate i shrinks [lo, hi] about its midpoint by t_i:
 *     half = (hi - lo) * 0.5,  mid = (hi + lo) * 0.5,  r = t_i * half
 *     S_i = (2r) / levels,  M_i = max(0, -(mid - r))
 *   w_hat = S_i * q - M_i (fp32 multiply, then fp32 subtract), loss as in the
 *   symmetric case, lowest index on ties.
 * Returns the chosen index; writes the fp32 (S*, M*) of the winner. */
int orc_asym_group(const float *w, const float *a, int G, const float *t, int n, int bits,
                   float *S_out, float *M_out, double *losses)
{
    const int levels = (1 << bits) - 1;
    float lo = 0.0f, hi = 0.0f;
    for (int k = 0; k < G; k++) {
        if (w[k] < lo) lo = w[k];
        if (w[k] > hi) hi = w[k];
    }
    float half = (hi - lo) * 0.5f;
    float mid = (hi + lo) * 0.5f;
    int best = 0;
    double bestL = 0.0;
    float bS = 0.0f, bM = 0.0f;
    for (int i = 0; i < n; i++) {
        float r = t[i] * half;
        float S = (2.0f * r) / (float)levels;
        float lo_i = mid - r;
        float M = (lo_i < 0.0f) ? -lo_i : 0.0f;
        double L = 0.0;
        for (int k = 0; k < G; k++) {
            float wq = asym_deq(asym_code(w[k], S, M, levels), S, M);
            double d = (double)w[k] - (double)wq;
            double e = d * d;
            double ak = a ? (double)a[k] : 1.0;
            L = L + ak * e;
        }
        if (losses) losses[i] = L;
        if (i == 0 || L < bestL) { best = i; bestL = L; bS = S; bM = M; }
    }
    *S_out = bS;
    *M_out = bM;
    return best;
}

/* Finish one superblock of 8 groups x 32 weights into its record (144, 176
 * or 208 bytes for 4-, 5- or 6-bit codes). The layout is this project's own
 * (the pages give only "asymmetric superblock, group 32"; the 6-bit
 * scale/min against an fp16 superblock scale/min is the stated
 * configuration; 5 and 6 bits add exactly 1 and 2 bits per weight, the
 * file-size deltas [ART] quotes for o_proj):
 *   [0:2]    fp16 d      = fp16(max_j S*_j / 63)
 *   [2:4]    fp16 dmin   = fp16(max_j M*_j / 63)
 *   [4:16]   96-bit little-endian bit string: bits 6j..6j+5 hold sc_j,
 *            bits 48+6j..48+6j+5 hold m_j (j = 0..7)
 *            sc_j = clamp(rint(S*_j / d), 0, 63), 0 when d == 0; m_j likewise
 *   [16:144] 128 bytes of the codes' low 4 bits: low nibble k = 2t, high
 *            nibble k = 2t+1
 *   5 bits:  [144:176] bit 4 of code k in bit k % 8 of byte 144 + k / 8
 *   6 bits:  [144:208] bits 4..5 of code k in bits 2 (k % 4) .. +1 of byte
 *            144 + k / 4
 * The final codes use the stored values S_j = d * sc_j and M_j = dmin * m_j
 * (both exact fp32 products); there is no second search after the 6-bit
 * rounding. */
/* Put code q of weight kk (0..255) into a record whose code area starts
 * zeroed: the low 4 bits in the nibble bytes, bits 4.. in the plane. */
static void sb_put_code(uint8_t *blk, int kk, int q, int bits)
{
    int lo4 = q & 15, up = q >> 4;
    if ((kk & 1) == 0) blk[16 + kk / 2] = (uint8_t)lo4;
    else blk[16 + kk / 2] |= (uint8_t)(lo4 << 4);
    if (bits == 5) blk[144 + kk / 8] |= (uint8_t)(up << (kk % 8));
    if (bits == 6) blk[144 + kk / 4] |= (uint8_t)(up << (2 * (kk % 4)));
}

void orc_sb_finish(const float *w, const float *S_star, const float *M_star, int bits, uint8_t *blk)
{
    const int levels = (1 << bits) - 1;
    float mS = 0.0f, mM = 0.0f;
    for (int j = 0; j < 8; j++) {
        if (S_star[j] > mS) mS = S_star[j];
        if (M_star[j] > mM) mM = M_star[j];
    }
    uint16_t dh = orc_f32_to_f16(mS / 63.0f);
    uint16_t mh = orc_f32_to_f16(mM / 63.0f);
    float d = orc_f16_to_f32(dh), dm = orc_f16_to_f32(mh);
    int sc[8], mc[8];
    for (int j = 0; j < 8; j++) {
        sc[j] = (d == 0.0f) ? 0 : (int)rintf(clampf(S_star[j] / d, 0.0f, 63.0f));
        mc[j] = (dm == 0.0f) ? 0 : (int)rintf(clampf(M_star[j] / dm, 0.0f, 63.0f));
    }
    memset(blk, 0, (size_t)sb_bytes(bits));
    blk[0] = (uint8_t)(dh & 0xff); blk[1] = (uint8_t)(dh >> 8);
    blk[2] = (uint8_t)(mh & 0xff); blk[3] = (uint8_t)(mh >> 8);
    for (int j = 0; j < 8; j++) {
        for (int b = 0; b < 6; b++) {
            int bs = 6 * j + b, bm = 48 + 6 * j + b;
            if ((sc[j] >> b) & 1) blk[4 + bs / 8] |= (uint8_t)(1u << (bs % 8));
            if ((mc[j] >> b) & 1) blk[4 + bm / 8] |= (uint8_t)(1u << (bm % 8));
        }
    }
    for (int j = 0; j < 8; j++) {
        float S = d * (float)sc[j];
        float M = dm * (float)mc[j];
        for (int k = 0; k < 32; k++) {
            int kk = 32 * j + k;
            sb_put_code(blk, kk, asym_code(w[kk], S, M, levels), bits);
        }
    }
}

/* Pack a whole [N][K] matrix (K % 256 == 0) into [N][K/256] superblocks of
 * `bits`-bit codes. */
int orc_sb_field(const uint8_t *blk, int which, int j);

/* GPTQ into the asymmetric superblock formats (the COMPRESSION preset's
 * grid): at each superblock's first column the eight groups' (S*, M*) come
 * from the preset's search (orc_asym_group) on fp32 of the current weights and
 * the record's header is formed as orc_sb_finish forms it; the stored
 * S_j = d sc_j, M_j = dmin m_j are then fixed and the superblock's 256 columns
 * are quantized in order with GPTQ's error feedback:
 *   q = asym_code(fp32(w_k), S_j, M_j),  w_hat = fp32(S_j q) - M_j,
 *   err = (w_k - w_hat) / U[k][k],  w_j -= err * U[k][j] for j > k (fp64).
 * U and dead as for orc_gptq_pack_sym. */
void orc_gptq_pack_sb(const float *W, int K, int N, const double *U, const uint8_t *dead, const float *a,
                      int n_cand, float t_lo, float t_hi, int bits, uint8_t *blocks)
{
    int nb = K / 256;
    int levels = (1 << bits) - 1;
    size_t rs = (size_t)sb_bytes(bits);
    float *t = (float *)malloc(sizeof(float) * (size_t)n_cand);
    orc_grid(n_cand, t_lo, t_hi, t);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < N; n++) {
        double *w = (double *)malloc(sizeof(double) * (size_t)K);
        for (int k = 0; k < K; k++) w[k] = dead[k] ? 0.0 : (double)W[(size_t)n * K + k];
        for (int b = 0; b < nb; b++) {
            int k0 = b * 256;
            float wsb[256], S[8], M[8];
            for (int i = 0; i < 256; i++) wsb[i] = (float)w[k0 + i];
            for (int j = 0; j < 8; j++)
                orc_asym_group(wsb + 32 * j, a ? a + k0 + 32 * j : NULL, 32, t, n_cand, bits, &S[j], &M[j], NULL);
            uint8_t *blk = blocks + ((size_t)n * nb + b) * rs;
            orc_sb_finish(wsb, S, M, bits, blk);
            memset(blk + 16, 0, rs - 16);
            float d = orc_f16_to_f32((uint16_t)(blk[0] | (blk[1] << 8)));
            float dm = orc_f16_to_f32((uint16_t)(blk[2] | (blk[3] << 8)));
            for (int i = 0; i < 256; i++) {
                int k = k0 + i;
                float Sj = d * (float)orc_sb_field(blk, 0, i / 32);
                float Mj = dm * (float)orc_sb_field(blk, 1, i / 32);
                int q = asym_code((float)w[k], Sj, Mj, levels);
                sb_put_code(blk, i, q, bits);
                double err = (w[k] - (double)asym_deq(q, Sj, Mj)) / U[(size_t)k * K + k];
                for (int j = k + 1; j < K; j++) w[j] = w[j] - err * U[(size_t)k * K + j];
            }
        }
        free(w);
    }
    free(t);
}

void orc_pack_sb32(const float *W, int K, int N, const float *a, int n_cand,
                   float t_lo, float t_hi, int bits, uint8_t *blocks)
{
    int nb = K / 256;
    size_t rs = (size_t)sb_bytes(bits);
    float *t = (float *)malloc(sizeof(float) * (size_t)n_cand);
    orc_grid(n_cand, t_lo, t_hi, t);
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < N; n++) {
        const float *row = W + (size_t)n * K;
        for (int b = 0; b < nb; b++) {
            float S[8], M[8];
            for (int j = 0; j < 8; j++) {
                size_t k0 = (size_t)b * 256 + (size_t)j * 32;
                orc_asym_group(row + k0, a ? a + k0 : NULL, 32, t, n_cand, bits, &S[j], &M[j], NULL);
            }
            orc_sb_finish(row + (size_t)b * 256, S, M, bits, blocks + ((size_t)n * nb + b) * rs);
        }
    }
    free(t);
}

/* Decode the 6-bit scale (which = 0) or min (which = 1) of group j from a
 * superblock record. */
int orc_sb_field(const uint8_t *blk, int which, int j)
{
    int v = 0;
    for (int b = 0; b < 6; b++) {
        int bit = 48 * which + 6 * j + b;
        v |= ((blk[4 + bit / 8] >> (bit % 8)) & 1) << b;
    }
    return v;
}

/* ------------------------------------------------------------------------ */
/* Dequantization and the product                                           */
/* ------------------------------------------------------------------------ */

/* Exact fp32 dequantization of row n into out[K]:
 *   symmetric:  w_hat = q * s          (exact: 8 + 11 significant bits)
 *   superblock: w_hat = S_j * q - M_j  (S_j * q exact, one rounding) */
static void deq_row(int fmt, int K, const uint8_t *codes, const uint16_t *scales,
                    int n, float *out)
{
    if (fmt == ORC_W4SB32 || fmt == ORC_W5SB32 || fmt == ORC_W6SB32) {
        int nb = K / 256, bits = sb_bits(fmt);
        size_t rs = (size_t)sb_bytes(bits);
        for (int b = 0; b < nb; b++) {
            const uint8_t *blk = codes + ((size_t)n * nb + b) * rs;
            float d = orc_f16_to_f32((uint16_t)(blk[0] | (blk[1] << 8)));
            float dm = orc_f16_to_f32((uint16_t)(blk[2] | (blk[3] << 8)));
            for (int j = 0; j < 8; j++) {
                float S = d * (float)orc_sb_field(blk, 0, j);
                float M = dm * (float)orc_sb_field(blk, 1, j);
                for (int k = 0; k < 32; k++) {
                    int kk = 32 * j + k;
                    int q = (blk[16 + kk / 2] >> (4 * (kk & 1))) & 0xf;
                    if (bits == 5) q |= ((blk[144 + kk / 8] >> (kk % 8)) & 1) << 4;
                    if (bits == 6) q |= ((blk[144 + kk / 4] >> (2 * (kk % 4))) & 3) << 4;
                    out[(size_t)b * 256 + kk] = asym_deq(q, S, M);
                }
            }
        }
        return;
    }
    int G = sym_gsize(fmt);
    int ng = K / G;
    for (int k = 0; k < K; k++) {
        int q;
        if (fmt == ORC_W4G64) {
            q = ((codes[(size_t)n * (K / 2) + k / 2] >> (4 * (k & 1))) & 0xf) - 8;
        } else if (fmt == ORC_W6G16) {
            const uint8_t *chunk = codes + (size_t)n * (K / 64 * 48) + (k / 64) * 48;
            int j = k % 64;
            int u = (chunk[j / 2] >> (4 * (j & 1))) & 0xf;
            u |= ((chunk[32 + j / 4] >> (2 * (j % 4))) & 3) << 4;
            q = u - 32;
        } else {
            q = (int)codes[(size_t)n * K + k] - 128;
        }
        float s = orc_f16_to_f32(scales[(size_t)n * ng + k / G]);
        out[k] = (float)q * s;
    }
}

void orc_dequant(int fmt, int K, int N, const uint8_t *codes, const uint16_t *scales, float *W_out)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) deq_row(fmt, K, codes, scales, n, W_out + (size_t)n * K);
}

/* y[m][r] = sum_k x[m][k] * w_hat[rows[r]][k], in fp64, ascending k.
 * x is bf16 [M][K]; rows == NULL means every row 0..N-1 (then nrows = N).
 * Every product of a bf16 and an fp32 value is exact in fp64. */
void orc_wgemm(int fmt, const uint16_t *x, int M, int K, int N, const uint8_t *codes,
               const uint16_t *scales, const int *rows, int nrows, double *y)
{
    if (!rows) nrows = N;
    double *xd = (double *)malloc(sizeof(double) * (size_t)M * K);
    for (size_t i = 0; i < (size_t)M * K; i++) xd[i] = (double)orc_bf16_to_f32(x[i]);
#pragma omp parallel
    {
        float *wrow = (float *)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < nrows; r++) {
            int n = rows ? rows[r] : r;
            deq_row(fmt, K, codes, scales, n, wrow);
            for (int m = 0; m < M; m++) {
                const double *xm = xd + (size_t)m * K;
                double acc = 0.0;
                for (int k = 0; k < K; k++) acc = acc + xm[k] * (double)wrow[k];
                y[(size_t)m * nrows + r] = acc;
            }
        }
        free(wrow);
    }
    free(xd);
}

/* ------------------------------------------------------------------------ */
/* Activation statistic E[x^2]                                              */
/* ------------------------------------------------------------------------ */

/* [ART] "Two presets and six sizes": the search weights input channel k by
 * E[x_k^2], the mean over the calibration rows of the squared activation.
 * Written as that definition: for each channel the square of every row is
 * added to the channel's running sum, one row at a time in ascending row
 * order, in fp64 (x[r][k]^2 of a bf16 value is exact in fp64). A batch of
 * rows continues the sum of the batches before it. */
void orc_act_sumsq(const uint16_t *x, int R, int K, double *sum_sq)
{
    for (int k = 0; k < K; k++) {
        double s = sum_sq[k];
        for (int r = 0; r < R; r++) {
            double v = (double)orc_bf16_to_f32(x[(size_t)r * K + k]);
            s = s + v * v;
        }
        sum_sq[k] = s;
    }
}

/* E[x_k^2] = fp32(sum_sq[k] / rows): one fp64 division, one rounding. */
void orc_act_finalize(const double *sum_sq, int K, long long rows, float *act_sq)
{
    for (int k = 0; k < K; k++) act_sq[k] = (float)(sum_sq[k] / (double)rows);
}

/* Number of OpenMP threads a parallel region would use (0 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int orc_threads(void) { return omp_get_max_threads(); }
void orc_set_threads(int n) { omp_set_num_threads(n); }
#else
int orc_threads(void) { return 1; }
void orc_set_threads(int n) { (void)n; }
#endif
