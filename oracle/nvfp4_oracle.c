/*
 * nvfp4_oracle.c - plain CPU oracle for the NVFP4 W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA product library
 * shares no code, header, table or helper with it, and never calls it.
 *
 * What is computed, and where it is defined (the pages are web write-ups of
 * arXiv 2609.04098, "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4
 * W4A4 for the Recurrent Half of a Hybrid 27B LLM"):
 *
 *   - NVFP4 storage: 4-bit E2M1 element codes, one E4M3 scale per block of 16
 *     elements chosen from the block's largest magnitude divided by 6, and one
 *     FP32 scale per tensor. [picx.dev summary of the paper, "Background"]
 *   - 16-element E4M3 blocks (as opposed to 32-element power-of-two MX
 *     blocks). [anthology record LIT-800, "Standing in the anthology"]
 *   - W4A4 GEMM: both operands in NVFP4, FP32 output scaled back to real
 *     units. [picx.dev summary, "Background": native 4-bit tensor-core GEMMs]
 *   - Fused projections: several projection weights, each calibrated with its
 *     own global scale, concatenated along the output dimension of one GEMM;
 *     every output segment must be rescaled by its own weight scale.
 *     [anthology record LIT-800, "Standing in the anthology"; cctest.ai
 *     article, "Main findings"; podcast abstract]
 *
 * Readings taken where the pages are silent, each one a choice, numbered
 * R1-R7 here; the same numbers label them wherever the library, its tests and
 * its documentation refer to them:
 *   R1  E2M1 is the OCP FP4 layout: bit 3 sign, bits 2..1 exponent (bias 1),
 *       bit 0 mantissa; magnitudes {0,0.5,1,1.5,2,3,4,6}.
 *   R2  E4M3 is OCP FP8 E4M3FN: bias 7, largest finite 448, no infinity,
 *       0x7F/0xFF are NaN, subnormal step 2^-9.
 *   R3  Both encodings round to nearest, ties to an even mantissa, and
 *       saturate to the largest finite magnitude. The sign of the input is
 *       kept, so a negative value that rounds to zero gives negative zero.
 *   R4  The global scale g multiplies on encode and divides on decode:
 *       value = e2m1(code) * e4m3(scale) / g.  Default calibration
 *       g = 448*6/amax(tensor) puts the largest block scale at 448.
 *   R5  The block scale is computed in FP32 as t = (amax_b / 6) * g, two
 *       correctly rounded operations in that order, s = E4M3(t).  If s is 0
 *       every code of the block is a signed zero.  Otherwise r = g / e4m3(s)
 *       (one FP32 division) and code_i = E2M1(x_i * r) (one FP32 multiply).
 *   R6  Packing: element 2j of a row sits in the low nibble of byte j.
 *   R7  The GEMM is the FP64 dot product of the dequantized operands.
 *
 * Build: plain C11, -O2 -ffp-contract=off, no fast-math (x86-64 SSE float
 * arithmetic is IEEE single precision with round-to-nearest-even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* threads (rows are independent; this changes no arithmetic)          */
/* ------------------------------------------------------------------ */

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* E2M1 (reading R1, R3)                                               */
/* ------------------------------------------------------------------ */

/* Value of a 4-bit E2M1 code (only the low 4 bits are used). */
double orc_e2m1_decode(uint8_t code) {
    int sign = (code >> 3) & 1;
    int exp = (code >> 1) & 3;
    int man = code & 1;
    double mag;
    if (exp == 0)
        mag = 0.5 * man;                                /* subnormal: 0 or 0.5 */
    else
        mag = ldexp(1.0 + 0.5 * man, exp - 1);          /* 1,1.5,2,3,4,6 */
    return sign ? -mag : mag;
}

/* Nearest E2M1 code to v: ties go to the code with an even mantissa bit,
 * magnitudes at or above 6 saturate to 6, the sign bit copies v's sign.
 * Codes 0..7 are ordered by value, so the neighbours of |v| are found by a
 * scan; both distances are exact in double (|v| lies between lo and 2*lo or
 * lo is 0, see the Sterbenz lemma). */
uint8_t orc_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs((double)v);
    if (a >= 6.0) return sign | 0x7;
    int lo = 0;
    for (int c = 0; c < 7; ++c)
        if (orc_e2m1_decode((uint8_t)c) <= a) lo = c;
    double dlo = a - orc_e2m1_decode((uint8_t)lo);
    double dhi = orc_e2m1_decode((uint8_t)(lo + 1)) - a;
    int code;
    if (dlo < dhi) code = lo;
    else if (dhi < dlo) code = lo + 1;
    else code = (lo & 1) ? lo + 1 : lo;                 /* tie: even mantissa */
    return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------ */
/* E4M3 (reading R2, R3)                                               */
/* ------------------------------------------------------------------ */

/* Value of an E4M3FN byte; NaN for 0x7F and 0xFF. */
double orc_e4m3_decode(uint8_t code) {
    int sign = (code >> 7) & 1;
    int exp = (code >> 3) & 15;
    int man = code & 7;
    double mag;
    if (exp == 15 && man == 7) return NAN;
    if (exp == 0)
        mag = ldexp((double)man, -9);                   /* subnormal: man * 2^-9 */
    else
        mag = ldexp(1.0 + man / 8.0, exp - 7);
    return sign ? -mag : mag;
}

/* Nearest E4M3FN byte to t, ties to even mantissa, saturating at 448, sign
 * copied from t.  Codes 0x00..0x7E are ordered by value. */
uint8_t orc_e4m3_encode(float t) {
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a = fabs((double)t);
    if (isnan(t)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0;
    for (int c = 0; c < 126; ++c)
        if (orc_e4m3_decode((uint8_t)c) <= a) lo = c;
    double dlo = a - orc_e4m3_decode((uint8_t)lo);
    double dhi = orc_e4m3_decode((uint8_t)(lo + 1)) - a;
    int code;
    if (dlo < dhi) code = lo;
    else if (dhi < dlo) code = lo + 1;
    else code = (lo & 1) ? lo + 1 : lo;
    return sign | (uint8_t)code;
}

void orc_e2m1_encode_array(const float* v, uint8_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float* v, uint8_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------ */
/* Per-tensor amax and the default global scale (reading R4)           */
/* ------------------------------------------------------------------ */

float orc_amax(const float* x, int64_t n) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

/* g = (448 * 6) / amax in FP32, so the block holding the tensor's largest
 * magnitude gets scale 448.  An all-zero tensor gets g = 1. */
float orc_global_scale(float amax) {
    if (!(amax > 0.0f)) return 1.0f;
    return 2688.0f / amax;
}

/* ------------------------------------------------------------------ */
/* Quantize (readings R5, R6)                                          */
/* ------------------------------------------------------------------ */

/* x: [M, K] FP32 row-major, K a multiple of 16.
 * codes: [M, K/2] bytes, element 2j of a row in the low nibble of byte j.
 * scales: [M, K/16] E4M3 bytes, row-major. */
void orc_quantize(const float* x, int64_t M, int64_t K, float g,
                  uint8_t* codes, uint8_t* scales) {
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + m * K + b * 16;
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            float q = amax / 6.0f;
            float t = q * g;
            uint8_t s = orc_e4m3_encode(t);
            scales[m * nb + b] = s;
            uint8_t c[16];
            if (s == 0) {
                for (int i = 0; i < 16; ++i) c[i] = signbit(xb[i]) ? 0x8 : 0x0;
            } else {
                float sf = (float)orc_e4m3_decode(s);
                float r = g / sf;
                for (int i = 0; i < 16; ++i) {
                    float y = xb[i] * r;
                    c[i] = orc_e2m1_encode(y);
                }
            }
            uint8_t* cb = codes + m * (K / 2) + b * 8;
            for (int j = 0; j < 8; ++j)
                cb[j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
    }
}

/* Dequantized FP64 values: out[m,k] = e2m1(code) * e4m3(scale) / g. */
void orc_dequantize(const uint8_t* codes, const uint8_t* scales, float g,
                    int64_t M, int64_t K, double* out) {
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[m * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);
            double s = orc_e4m3_decode(scales[m * nb + k / 16]);
            out[m * K + k] = orc_e2m1_decode(code) * s / (double)g;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Tensor-core scale-factor layout (a storage order, not arithmetic)   */
/* ------------------------------------------------------------------ */

/* The block-scaled tensor-core MMA reads scales from 512-byte chunks, each
 * covering 128 rows x 4 consecutive scales (64 K-elements) of one operand.
 * Inside a chunk, the 4 scales of row r sit at byte
 *     (r % 32) * 16 + ((r / 32) % 4) * 4 + (scale index % 4).
 * Chunks are ordered by row block, then by K: chunk (r/128, j/4) starts at
 * ((r/128) * ceil(K/64) + j/4) * 512.  Rows are padded to a multiple of 128
 * and scale columns to a multiple of 4; padding bytes are zero.
 * Sizes: out has ceil(R/128)*128 * ceil(K/64)*4 bytes. */
int64_t orc_tc_scale_bytes(int64_t R, int64_t K) {
    int64_t rb = (R + 127) / 128, kc = (K + 63) / 64;
    return rb * kc * 512;
}

void orc_scales_to_tc(const uint8_t* rowmajor, int64_t R, int64_t K, uint8_t* out) {
    const int64_t nb = K / 16, kc = (K + 63) / 64;
    memset(out, 0, (size_t)orc_tc_scale_bytes(R, K));
    for (int64_t r = 0; r < R; ++r)
        for (int64_t j = 0; j < nb; ++j) {
            int64_t chunk = (r / 128) * kc + j / 4;
            int64_t off = chunk * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);
            out[off] = rowmajor[r * nb + j];
        }
}

void orc_scales_from_tc(const uint8_t* tc, int64_t R, int64_t K, uint8_t* rowmajor) {
    const int64_t nb = K / 16, kc = (K + 63) / 64;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t j = 0; j < nb; ++j) {
            int64_t chunk = (r / 128) * kc + j / 4;
            int64_t off = chunk * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);
            rowmajor[r * nb + j] = tc[off];
        }
}

/* ------------------------------------------------------------------ */
/* GEMM and fused projection (reading R7)                              */
/* ------------------------------------------------------------------ */

/* Shared body: column n of W uses global scale w_gs[seg_of[n]]. */
static void gemm_segments(const uint8_t* a_codes, const uint8_t* a_scales, float a_gs,
                          const uint8_t* w_codes, const uint8_t* w_scales,
                          const float* w_gs_per_col,
                          int64_t M, int64_t N, int64_t K, double* out) {
    double* da = (double*)malloc(sizeof(double) * (size_t)(M * K));
    orc_dequantize(a_codes, a_scales, a_gs, M, K, da);
    const int64_t nb = K / 16;
#pragma omp parallel
    {
        double* dw = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            /* dequantize row n of W */
            for (int64_t k = 0; k < K; ++k) {
                uint8_t byte = w_codes[n * (K / 2) + k / 2];
                uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);
                double s = orc_e4m3_decode(w_scales[n * nb + k / 16]);
                dw[k] = orc_e2m1_decode(code) * s / (double)w_gs_per_col[n];
            }
            for (int64_t m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += da[m * K + k] * dw[k];
                out[m * N + n] = acc;
            }
        }
        free(dw);
    }
    free(da);
}

/* out[m,n] = sum_k deqA[m,k] * deqW[n,k] in FP64.
 * A: codes [M,K/2], scales [M,K/16] row-major; W: codes [N,K/2], scales
 * [N,K/16] row-major (W stored like a linear layer's weight, [out, in]). */
void orc_gemm(const uint8_t* a_codes, const uint8_t* a_scales, float a_gs,
              const uint8_t* w_codes, const uint8_t* w_scales, float w_gs,
              int64_t M, int64_t N, int64_t K, double* out) {
    float* g = (float*)malloc(sizeof(float) * (size_t)N);
    for (int64_t n = 0; n < N; ++n) g[n] = w_gs;
    gemm_segments(a_codes, a_scales, a_gs, w_codes, w_scales, g, M, N, K, out);
    free(g);
}

/* Fused projection: W is the row-wise concatenation of n_seg weights; rows
 * [seg_offsets[i], seg_offsets[i+1]) belong to segment i and are dequantized
 * with that segment's own global scale seg_gs[i].  The activation is
 * quantized once, with one global scale. */
void orc_fused_proj(const uint8_t* a_codes, const uint8_t* a_scales, float a_gs,
                    const uint8_t* w_codes, const uint8_t* w_scales,
                    const int64_t* seg_offsets, const float* seg_gs, int n_seg,
                    int64_t M, int64_t K, double* out) {
    int64_t N = seg_offsets[n_seg];
    float* g = (float*)malloc(sizeof(float) * (size_t)N);
    for (int i = 0; i < n_seg; ++i)
        for (int64_t n = seg_offsets[i]; n < seg_offsets[i + 1]; ++n) g[n] = seg_gs[i];
    gemm_segments(a_codes, a_scales, a_gs, w_codes, w_scales, g, M, N, K, out);
    free(g);
}

/* Exact integer form of the same sum, used to pin the FP64 GEMM.
 * 2*e2m1 is an integer in [-12,12] and 512*e4m3 an integer in [0,229376],
 * so   sum_k e2m1(a)e4m3(sa) e2m1(w)e4m3(sw)  =  S * 2^-20  with S integer:
 *   S[m,n] = sum_b (512 sa_b)(512 sw_b) * sum_{k in b} (2 a_k)(2 w_k).
 * |S| < 2^63 for K up to about 10^5.  The real result is S*2^-20/(gA*gW). */
static int64_t twice_e2m1(uint8_t code) {
    static const int mag2[8] = {0, 1, 2, 3, 4, 6, 8, 12};
    int v = mag2[code & 7];
    return (code & 8) ? -v : v;
}

static int64_t e4m3_times_512(uint8_t code) {
    int exp = (code >> 3) & 15, man = code & 7;
    if (exp == 0) return man;                           /* man * 2^-9 * 2^9 */
    return (int64_t)(8 + man) << (exp - 1);             /* (1+man/8)*2^(exp-7)*2^9 */
}

void orc_gemm_exact(const uint8_t* a_codes, const uint8_t* a_scales,
                    const uint8_t* w_codes, const uint8_t* w_scales,
                    int64_t M, int64_t N, int64_t K, int64_t* S) {
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t b = 0; b < nb; ++b) {
                int64_t blk = 0;
                for (int64_t k = b * 16; k < b * 16 + 16; ++k) {
                    uint8_t ab = a_codes[m * (K / 2) + k / 2];
                    uint8_t wb = w_codes[n * (K / 2) + k / 2];
                    uint8_t ac = (k & 1) ? (ab >> 4) : (ab & 0xF);
                    uint8_t wc = (k & 1) ? (wb >> 4) : (wb & 0xF);
                    blk += twice_e2m1(ac) * twice_e2m1(wc);
                }
                acc += blk * e4m3_times_512(a_scales[m * nb + b]) *
                       e4m3_times_512(w_scales[n * nb + b]);
            }
            S[m * N + n] = acc;
        }
}

/* ------------------------------------------------------------------ */
/* Static calibration: how much a fixed global scale clips (R15)       */
/* ------------------------------------------------------------------ */

/* A global scale calibrated on other data can be too large for a new input:
 * a block's scale target t = (amax_b / 6) * g then exceeds 448 and the E4M3
 * scale saturates, after which x * r can exceed 6 and the E2M1 code
 * saturates too.  [anthology record LIT-800, "Key takeaways": the recipe is
 * calibration-only, on a fixed set of sequences; cctest.ai article,
 * "Introduction"]  The arithmetic is that of orc_quantize, step for step.
 *   counts[0] = blocks with t > 448 (scale clipped)
 *   counts[1] = elements with |x * r| > 6 (code clipped)
 *   counts[2] = blocks whose scale rounded to zero while amax_b > 0 */
void orc_saturation(const float* x, int64_t M, int64_t K, float g, int64_t* counts) {
    const int64_t nb = K / 16;
    int64_t c0 = 0, c1 = 0, c2 = 0;
#pragma omp parallel for schedule(static) reduction(+ : c0, c1, c2)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + m * K + b * 16;
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            float q = amax / 6.0f;
            float t = q * g;
            if (t > 448.0f) c0 += 1;
            uint8_t s = orc_e4m3_encode(t);
            if ((s & 0x7F) == 0) {
                if (amax > 0.0f) c2 += 1;
                continue;
            }
            float r = g / (float)orc_e4m3_decode(s);
            for (int i = 0; i < 16; ++i) {
                float y = xb[i] * r;
                if (fabsf(y) > 6.0f) c1 += 1;
            }
        }
    }
    counts[0] = c0;
    counts[1] = c1;
    counts[2] = c2;
}

/* ------------------------------------------------------------------ */
/* Offline global-scale harmonisation of a fused weight (R14)          */
/* ------------------------------------------------------------------ */

/* A fused projection weight stacks row segments [offs[i], offs[i+1]), each
 * quantized with its own global scale gs[i].  A kernel that applies one
 * scale to the whole GEMM needs the checkpoint rewritten to a common scale g
 * first ("pre-harmonized") [cctest.ai article, "Main findings"; anthology
 * record LIT-800, "Standing in the anthology"].  The element codes are kept;
 * every block scale s of segment i becomes
 *     s' = E4M3(e4m3(s) * q_i),   q_i = g / gs[i]
 * with q_i rounded to FP32 once per segment and one FP32 multiply per scale,
 * so that e2m1 * e4m3(s') / g approximates e2m1 * e4m3(s) / gs[i].
 * scales and out are [R, K/16] row-major; rows outside every segment are
 * copied unchanged. */
void orc_harmonize_scales(const uint8_t* scales, int64_t R, int64_t K, const int64_t* offs,
                          const float* gs, int nseg, float g, uint8_t* out) {
    const int64_t nb = K / 16;
    memcpy(out, scales, (size_t)(R * nb));
    for (int i = 0; i < nseg; ++i) {
        float qi = g / gs[i];
        for (int64_t r = offs[i]; r < offs[i + 1] && r < R; ++r)
            for (int64_t j = 0; j < nb; ++j) {
                float sv = (float)orc_e4m3_decode(scales[r * nb + j]);
                float y = sv * qi;
                out[r * nb + j] = orc_e4m3_encode(y);
            }
    }
}

/* ------------------------------------------------------------------ */
/* MXFP4, the contrast format (readings R16, R17)                      */
/* ------------------------------------------------------------------ */

/* The pages set NVFP4 against the MX format: blocks of 32 elements sharing
 * one power-of-two scale, where NVFP4 uses 16 elements and an E4M3 scale
 * [anthology record LIT-800, "Standing in the anthology"].  The conversion
 * below is the published OCP Microscaling v1.0 rule for MXFP4, in the
 * spec's order: per block of 32 along K,
 *     E = floor(log2(max |x|)) - 2        (2: exponent of E2M1's largest
 *                                           normal, 6 = 1.5 * 2^2)
 * clamped to the E8M0 range [-127, 127]; the scale byte is E + 127 and
 * every element is E2M1(x * 2^-E), nearest even, saturating at 6 (the
 * quotient is exact: a power-of-two scaling of a float).  An all-zero
 * block gets E = -127 (byte 0).  Value = e2m1(code) * 2^(byte - 127).
 * There is no per-tensor scale.  Byte 255 (NaN) is never produced. */

double orc_e8m0_decode(uint8_t b) {
    return ldexp(1.0, (int)b - 127);
}

uint8_t orc_mx_scale(float amax) {
    if (!(amax > 0.0f)) return 0;
    int e2;
    (void)frexp((double)amax, &e2);       /* amax = f * 2^e2, f in [0.5, 1) */
    int E = (e2 - 1) - 2;                 /* floor(log2(amax)) - 2 */
    if (E < -127) E = -127;
    if (E > 127) E = 127;
    return (uint8_t)(E + 127);
}

/* x: [M, K] FP32, K a multiple of 32.  codes: [M, K/2] (element 2j in the
 * low nibble of byte j); scales: [M, K/32] E8M0 bytes, row-major. */
void orc_mx_quantize(const float* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* scales) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + m * K + b * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            uint8_t s = orc_mx_scale(amax);
            scales[m * nb + b] = s;
            int E = (int)s - 127;
            uint8_t c[32];
            for (int i = 0; i < 32; ++i) {
                float y = (float)ldexp((double)xb[i], -E);
                c[i] = orc_e2m1_encode(y);
            }
            uint8_t* cb = codes + m * (K / 2) + b * 16;
            for (int j = 0; j < 16; ++j)
                cb[j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
        }
    }
}

void orc_mx_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t M, int64_t K, double* out) {
    const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[m * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);
            out[m * K + k] = orc_e2m1_decode(code) * orc_e8m0_decode(scales[m * nb + k / 32]);
        }
}

/* out[m,n] = sum_k deqA[m,k] * deqW[n,k] in FP64, MXFP4 operands. */
void orc_mx_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                 const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, double* out) {
    double* da = (double*)malloc(sizeof(double) * (size_t)(M * K));
    double* dw = (double*)malloc(sizeof(double) * (size_t)(N * K));
    orc_mx_dequantize(a_codes, a_scales, M, K, da);
    orc_mx_dequantize(w_codes, w_scales, N, K, dw);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += da[m * K + k] * dw[n * K + k];
            out[m * N + n] = acc;
        }
    free(da);
    free(dw);
}
