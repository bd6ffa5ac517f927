/*
 * W4A4 oracle (test infrastructure only; see oracle.h for the contract and
 * the passages followed).  Plain C, single thread, no blocking or fusion:
 * every function is the rule it implements, written out step by step.
 */
#include "oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ======================================================================== */
/* Scalar encodings                                                         */
/* ======================================================================== */

/* E2M1 magnitudes by code 0..7 (sign is bit 3). */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

float orc_e2m1_decode(uint8_t code) {
    float m = kE2M1[code & 7];
    return (code & 8) ? -m : m;
}

/* Round |v| to the E2M1 grid.  Within a binade the representable values are
 * the integer multiples of the binade's quantum (0.5 below 2, then 1, then
 * 2), so "nearest, ties to even code" is rint() of |v|/quantum: the parity of
 * the multiple is the parity of the code's mantissa bit.  Values at or above
 * 6 saturate to 6 (the format has no infinities). */
uint8_t orc_e2m1_encode(float v) {
    int neg = signbit(v) ? 1 : 0;
    float m = fabsf(v);
    float val;
    if (!(m < 6.0f)) {
        val = 6.0f;
    } else {
        float q = (m < 2.0f) ? 0.5f : (m < 4.0f ? 1.0f : 2.0f);
        val = rintf(m / q) * q;           /* exact: q is a power of two */
        if (val > 6.0f) val = 6.0f;
    }
    uint8_t code = 0;
    for (uint8_t c = 0; c < 8; ++c)
        if (kE2M1[c] == val) code = c;
    return (uint8_t)(code | (neg << 3));
}

/* E4M3 ("FN" variant): bias 7, normals (1+M/8)*2^(E-7) for E=1..15 except
 * the all-ones pattern (NaN), subnormals M*2^-9, largest finite 448. */
float orc_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    float v;
    if ((code & 0x7F) == 0x7F) return NAN;
    if (e == 0) v = ldexpf((float)m, -9);
    else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -v : v;
}

/* Non-negative input; nearest representable E4M3 value, ties to even
 * mantissa, values at or above 448 (and +inf) saturate to 448. */
uint8_t orc_e4m3_encode(float v) {
    if (!(v > 0.0f)) return 0;                    /* +0, -0 (and NaN) -> 0 */
    if (v >= 448.0f) return 0x7E;                 /* 448 = E15 M6 */
    double q;                                     /* quantum of v's binade */
    if (v < ldexpf(1.0f, -6)) {
        q = ldexp(1.0, -9);
    } else {
        int e;
        frexp((double)v, &e);                     /* v = f * 2^e, f in [0.5,1) */
        q = ldexp(1.0, (e - 1) - 3);
    }
    double val = rint((double)v / q) * q;        /* exact power-of-two scaling */
    if (val > 448.0) val = 448.0;
    if (val == 0.0) return 0;
    if (val < ldexp(1.0, -6)) return (uint8_t)(val / ldexp(1.0, -9));
    int e;
    double f = frexp(val, &e);                    /* val = f*2^e */
    int E = (e - 1) + 7;
    int Mnt = (int)((f * 2.0 - 1.0) * 8.0);       /* exact */
    return (uint8_t)((E << 3) | Mnt);
}

float orc_e8m0_decode(uint8_t code) { return ldexpf(1.0f, (int)code - 127); }

int orc_floor_log2(float a) {
    int e;
    frexpf(a, &e);                                /* a = f * 2^e, f in [0.5,1) */
    return e - 1;
}

/* Round a double to bf16 (8 significant bits, exponent range of binary32),
 * nearest even, in one step. */
uint16_t orc_f64_to_bf16(double v) {
    uint32_t u;
    float f;
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else if (a < ldexp(1.0, -126)) {
        r = rint(a * ldexp(1.0, 133)) * ldexp(1.0, -133);   /* subnormal quantum 2^-133 */
    } else {
        int e;
        frexp(a, &e);                                        /* a in [2^(e-1), 2^e) */
        double q = ldexp(1.0, (e - 1) - 7);
        r = rint(a / q) * q;
    }
    /* largest finite bf16 is (2 - 2^-7) * 2^127; beyond half an ulp above it -> inf */
    if (r > ldexp(2.0 - ldexp(1.0, -7), 127)) r = INFINITY;
    f = (float)r;                                            /* exact */
    if (signbit(v)) f = -f;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ======================================================================== */
/* NVFP4                                                                    */
/* ======================================================================== */

/* Second-level (FP32) scale from an amax: the amax maps onto the largest
 * block scale times the largest element, 448 * 6 = 2688.  A zero amax, or a
 * quotient that is not a positive normal float, gives scale 1. */
float orc_nvfp4_s2_from_amax(float amax) {
    float s2 = amax / 2688.0f;
    if (!(amax > 0.0f) || !(s2 >= FLT_MIN)) s2 = 1.0f;
    return s2;
}

/* One 16-element block: E4M3 block scale against s2, then E2M1 codes of
 * x / (scale * s2).  A zero block scale gives all-zero codes. */
static void nvfp4_block(const float* x, float s2, uint8_t* codes4 /* 8 bytes */,
                        uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    float t = (amax / 6.0f) / s2;
    uint8_t sb = orc_e4m3_encode(t);
    float d = orc_e4m3_decode(sb) * s2;
    uint8_t q[16];
    for (int i = 0; i < 16; ++i) q[i] = (sb == 0) ? 0 : orc_e2m1_encode(x[i] / d);
    for (int j = 0; j < 8; ++j) codes4[j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
    *scale = sb;
}

int orc_quant_nvfp4(const uint16_t* X, int M, int K, int ldx, int mode,
                    const float* static_s2, uint8_t* codes, uint8_t* scales,
                    float* s2) {
    if (M < 0 || K % 16 || ldx < K || (mode != 0 && mode != 1)) return -1;
    float* row = (float*)malloc(sizeof(float) * (size_t)(K > 0 ? K : 1));
    float tensor_s2 = 1.0f;
    if (mode == 0) {
        if (static_s2) {
            tensor_s2 = static_s2[0];
        } else {
            float amax = 0.0f;
            for (int m = 0; m < M; ++m)
                for (int k = 0; k < K; ++k)
                    amax = fmaxf(amax, fabsf(orc_bf16_to_f32(X[(size_t)m * ldx + k])));
            tensor_s2 = orc_nvfp4_s2_from_amax(amax);
        }
        s2[0] = tensor_s2;
    }
    for (int m = 0; m < M; ++m) {
        for (int k = 0; k < K; ++k) row[k] = orc_bf16_to_f32(X[(size_t)m * ldx + k]);
        float rs2 = tensor_s2;
        if (mode == 1) {
            if (static_s2) {
                rs2 = static_s2[m];
            } else {
                float amax = 0.0f;
                for (int k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(row[k]));
                rs2 = orc_nvfp4_s2_from_amax(amax);
            }
            s2[m] = rs2;
        }
        for (int b = 0; b < K / 16; ++b)
            nvfp4_block(row + 16 * b, rs2, codes + (size_t)m * (K / 2) + 8 * b,
                        scales + (size_t)m * (K / 16) + b);
    }
    free(row);
    return 0;
}

void orc_dequant_nvfp4(const uint8_t* codes, const uint8_t* scales,
                       const float* s2, int mode, int M, int K, double* out) {
    for (int m = 0; m < M; ++m) {
        float rs2 = (mode == 1) ? s2[m] : s2[0];
        for (int k = 0; k < K; ++k) {
            uint8_t byte = codes[(size_t)m * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            uint8_t sb = scales[(size_t)m * (K / 16) + k / 16];
            /* exact real value e * scale * s2 (at most 31 significant bits) */
            out[(size_t)m * K + k] =
                (double)orc_e2m1_decode(c) * (double)orc_e4m3_decode(sb) * (double)rs2;
        }
    }
}

/* ======================================================================== */
/* MXFP4                                                                    */
/* ======================================================================== */

/* One 32-element block: shared exponent c = floor(log2(amax)) - 2 + 127
 * (2 = the exponent of E2M1's largest value, 6 = 1.5 * 2^2), clamped to
 * [0, 254]; elements are E2M1(x * 2^-(c-127)).  An all-zero block gets c = 0
 * and zero codes. */
static void mxfp4_block(const float* x, uint8_t* codes16 /* 16 bytes */, uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    uint8_t q[32];
    int c = 0;
    if (amax > 0.0f) {
        c = orc_floor_log2(amax) - 2 + 127;
        if (c < 0) c = 0;
        if (c > 254) c = 254;
        float inv = ldexpf(1.0f, 127 - c);          /* 2^-(c-127) */
        for (int i = 0; i < 32; ++i) q[i] = orc_e2m1_encode(x[i] * inv);
    } else {
        for (int i = 0; i < 32; ++i) q[i] = 0;
    }
    for (int j = 0; j < 16; ++j) codes16[j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
    *scale = (uint8_t)c;
}

/* Fused modules ("Daily Papers", para 4): each row segment is quantized as
 * its own NVFP4 tensor (the tensor rule over the segment's rows), and every
 * row records its segment's second-level scale. */
int orc_quant_nvfp4_segments(const uint16_t* X, int M, int K, int ldx,
                             const int32_t* seg, int nseg, uint8_t* codes,
                             uint8_t* scales, float* s2_rows) {
    if (nseg < 1 || seg[0] != 0 || seg[nseg] != M || K % 16) return -1;
    for (int i = 0; i < nseg; ++i) {
        const int r0 = seg[i], r1 = seg[i + 1];
        if (r1 < r0) return -1;
        float s2 = 1.0f;
        if (orc_quant_nvfp4(X + (size_t)r0 * ldx, r1 - r0, K, ldx, 0, NULL, codes + (size_t)r0 * (K / 2),
                            scales + (size_t)r0 * (K / 16), &s2))
            return -1;
        for (int r = r0; r < r1; ++r) s2_rows[r] = s2;
    }
    return 0;
}

int orc_quant_mxfp4(const uint16_t* X, int M, int K, int ldx, uint8_t* codes, uint8_t* scales) {
    if (M < 0 || K % 32 || ldx < K) return -1;
    float x[32];
    for (int m = 0; m < M; ++m)
        for (int b = 0; b < K / 32; ++b) {
            for (int i = 0; i < 32; ++i) x[i] = orc_bf16_to_f32(X[(size_t)m * ldx + 32 * b + i]);
            mxfp4_block(x, codes + (size_t)m * (K / 2) + 16 * b, scales + (size_t)m * (K / 32) + b);
        }
    return 0;
}

/* Multi-pass MXFP4 decomposition ("APEX4: Efficient Pure W4A4 LLM Inference
 * via Intra-SM Compute Rebalancing" page, para 1, MSD: the activation becomes
 * a sum of low-precision components, each multiplied with the quantized
 * weights).  Per 32-element block: pass 0 quantizes x by the MXFP4 rule;
 * pass p quantizes the residual x - (sum of the earlier passes' values), again
 * by the MXFP4 rule with its own shared exponent.  The residual is formed in
 * FP32 and is exact: it is x minus x rounded to a grid at least as coarse as
 * x's own, so it keeps at most 8 significant bits and is a bf16 value (the
 * function returns -2 if that ever failed, which would break this reading).
 * Pass p fills columns [p*K, (p+1)*K): codes [M][passes*K/2], scales
 * [M][passes*K/32]. */
int orc_quant_mxfp4_msd(const uint16_t* X, int M, int K, int ldx, int passes, uint8_t* codes,
                        uint8_t* scales) {
    if (M < 0 || K % 32 || ldx < K || passes < 1) return -1;
    const size_t cb = (size_t)passes * (K / 2), sb = (size_t)passes * (K / 32);
    float x[32];
    for (int m = 0; m < M; ++m)
        for (int b = 0; b < K / 32; ++b) {
            for (int i = 0; i < 32; ++i) x[i] = orc_bf16_to_f32(X[(size_t)m * ldx + 32 * b + i]);
            for (int p = 0; p < passes; ++p) {
                uint8_t* c16 = codes + (size_t)m * cb + (size_t)p * (K / 2) + 16 * b;
                uint8_t* sc = scales + (size_t)m * sb + (size_t)p * (K / 32) + b;
                mxfp4_block(x, c16, sc);
                if (p + 1 == passes) break;
                const float unit = orc_e8m0_decode(*sc);
                for (int i = 0; i < 32; ++i) {
                    const uint8_t q = (i & 1) ? (c16[i / 2] >> 4) : (c16[i / 2] & 15);
                    const float v = orc_e2m1_decode(q) * unit; /* exact: 3 significant bits */
                    const float r = x[i] - v;
                    if ((double)r != (double)x[i] - (double)v) return -2;
                    uint32_t u;
                    memcpy(&u, &r, 4);
                    if (u & 0xFFFFu) return -2; /* not a bf16 value */
                    x[i] = r;
                }
            }
        }
    return 0;
}

void orc_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int M, int K, double* out) {
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) {
            uint8_t byte = codes[(size_t)m * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            out[(size_t)m * K + k] = (double)orc_e2m1_decode(c) *
                                     (double)orc_e8m0_decode(scales[(size_t)m * (K / 32) + k / 32]);
        }
}

/* ======================================================================== */
/* Block-local Walsh-Hadamard rotation                                      */
/* ======================================================================== */

/* In-place fast Walsh-Hadamard transform of n = 2^k FP32 values (Sylvester
 * order, H[i][j] = (-1)^popcount(i & j)): stages h = 1, 2, 4, ..., n/2, each
 * replacing every pair (v[j], v[j+h]) with j & h == 0 by (v[j] + v[j+h],
 * v[j] - v[j+h]), rounded to FP32. */
static void fwht_f32(float* v, int n) {
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                const float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* Rotation of each n-element block along K of X (bf16) before quantization
 * (the block-local form of the Hadamard rotation the "Depth Registers Unlock
 * W4A4 on SwiGLU" (mlsanity) abstract names as QuaRot; block-local so that
 * block isolation, which the "APEX4..." page, para 2 (ARCQuant) says full
 * rotations compromise, is kept).  act_side = 1 multiplies the transform by
 * 1/n (an exact power of two), act_side = 0 leaves it unscaled, so that
 * (X H/n)(W H)^T = X W^T.  out: FP32 [M][K]. */
int orc_rotate_blocks(const uint16_t* X, int M, int K, int ldx, int n, int act_side, float* out) {
    if (M < 0 || n < 2 || (n & (n - 1)) || K % n || ldx < K) return -1;
    const float inv = 1.0f / (float)n;
    for (int m = 0; m < M; ++m)
        for (int b = 0; b < K / n; ++b) {
            float* v = out + (size_t)m * K + (size_t)b * n;
            for (int i = 0; i < n; ++i) v[i] = orc_bf16_to_f32(X[(size_t)m * ldx + (size_t)b * n + i]);
            fwht_f32(v, n);
            if (act_side)
                for (int i = 0; i < n; ++i) v[i] = v[i] * inv;
        }
    return 0;
}

/* The quantizers on FP32 input (rotated values are not bf16): the same block
 * rules as orc_quant_nvfp4 / orc_quant_mxfp4 / orc_quant_int4. */
int orc_quant_nvfp4_f32(const float* X, int M, int K, int mode, uint8_t* codes, uint8_t* scales, float* s2) {
    if (M < 0 || K % 16 || (mode != 0 && mode != 1)) return -1;
    float tensor_s2 = 1.0f;
    if (mode == 0) {
        float amax = 0.0f;
        for (size_t i = 0; i < (size_t)M * K; ++i) amax = fmaxf(amax, fabsf(X[i]));
        tensor_s2 = orc_nvfp4_s2_from_amax(amax);
        s2[0] = tensor_s2;
    }
    for (int m = 0; m < M; ++m) {
        const float* row = X + (size_t)m * K;
        float rs2 = tensor_s2;
        if (mode == 1) {
            float amax = 0.0f;
            for (int k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(row[k]));
            rs2 = orc_nvfp4_s2_from_amax(amax);
            s2[m] = rs2;
        }
        for (int b = 0; b < K / 16; ++b)
            nvfp4_block(row + 16 * b, rs2, codes + (size_t)m * (K / 2) + 8 * b, scales + (size_t)m * (K / 16) + b);
    }
    return 0;
}

int orc_quant_mxfp4_f32(const float* X, int M, int K, uint8_t* codes, uint8_t* scales) {
    if (M < 0 || K % 32) return -1;
    for (int m = 0; m < M; ++m)
        for (int b = 0; b < K / 32; ++b)
            mxfp4_block(X + (size_t)m * K + 32 * b, codes + (size_t)m * (K / 2) + 16 * b,
                        scales + (size_t)m * (K / 32) + b);
    return 0;
}

/* ======================================================================== */
/* INT4, group 128, symmetric round-to-nearest                              */
/* ======================================================================== */

/* One 128-element group: s = amax / 7 (FP32); q = clamp(rint(x / s), -8, 7),
 * ties to even; a zero group stores s = 0 and zero codes.  Codes are 4-bit
 * two's complement. */
static void int4_group(const float* x, uint8_t* codes64 /* 64 bytes */, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(x[i]));
    float s = amax / 7.0f;
    int q[128];
    for (int i = 0; i < 128; ++i) {
        if (s == 0.0f) { q[i] = 0; continue; }
        float r = rintf(x[i] / s);
        if (r > 7.0f) r = 7.0f;
        if (r < -8.0f) r = -8.0f;
        q[i] = (int)r;
    }
    for (int j = 0; j < 64; ++j)
        codes64[j] = (uint8_t)((q[2 * j] & 15) | ((q[2 * j + 1] & 15) << 4));
    *scale = s;
}

/* The INT4 rule over a group of G elements (G a multiple of 128): the same
 * steps as int4_group with the group's own amax.  Coarser groups are the
 * granularity knob of the "Depth Registers..." thelatestinai page, para 2
 * (APEX4: rho-aware granularity adaptation, mixed-granularity mode). */
static void int4_group_n(const float* x, int G, uint8_t* codes, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < G; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const float s = amax / 7.0f;
    for (int j = 0; j < G / 2; ++j) {
        int q[2];
        for (int h = 0; h < 2; ++h) {
            q[h] = 0;
            if (s == 0.0f) continue;
            float r = rintf(x[2 * j + h] / s);
            if (r > 7.0f) r = 7.0f;
            if (r < -8.0f) r = -8.0f;
            q[h] = (int)r;
        }
        codes[j] = (uint8_t)((q[0] & 15) | ((q[1] & 15) << 4));
    }
    *scale = s;
}

int orc_quant_int4_g(const uint16_t* X, int M, int K, int ldx, int G, uint8_t* codes, float* scales) {
    if (M < 0 || G < 128 || G % 128 || K % G || ldx < K) return -1;
    float* x = (float*)malloc(sizeof(float) * (size_t)G);
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / G; ++g) {
            for (int i = 0; i < G; ++i) x[i] = orc_bf16_to_f32(X[(size_t)m * ldx + (size_t)G * g + i]);
            int4_group_n(x, G, codes + (size_t)m * (K / 2) + (size_t)(G / 2) * g, scales + (size_t)m * (K / G) + g);
        }
    free(x);
    return 0;
}

int orc_quant_int4_f32_g(const float* X, int M, int K, int G, uint8_t* codes, float* scales) {
    if (M < 0 || G < 128 || G % 128 || K % G) return -1;
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / G; ++g)
            int4_group_n(X + (size_t)m * K + (size_t)G * g, G, codes + (size_t)m * (K / 2) + (size_t)(G / 2) * g,
                         scales + (size_t)m * (K / G) + g);
    return 0;
}

int orc_quant_int4_f32(const float* X, int M, int K, uint8_t* codes, float* scales) {
    if (M < 0 || K % 128) return -1;
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / 128; ++g)
            int4_group(X + (size_t)m * K + 128 * g, codes + (size_t)m * (K / 2) + 64 * g,
                       scales + (size_t)m * (K / 128) + g);
    return 0;
}

int orc_quant_int4(const uint16_t* X, int M, int K, int ldx, uint8_t* codes, float* scales) {
    if (M < 0 || K % 128 || ldx < K) return -1;
    float x[128];
    for (int m = 0; m < M; ++m)
        for (int g = 0; g < K / 128; ++g) {
            for (int i = 0; i < 128; ++i) x[i] = orc_bf16_to_f32(X[(size_t)m * ldx + 128 * g + i]);
            int4_group(x, codes + (size_t)m * (K / 2) + 64 * g, scales + (size_t)m * (K / 128) + g);
        }
    return 0;
}

static int int4_value(uint8_t nib) { return (nib & 8) ? (int)nib - 16 : (int)nib; }

void orc_dequant_int4(const uint8_t* codes, const float* scales, int M, int K, double* out) {
    for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) {
            uint8_t byte = codes[(size_t)m * (K / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            out[(size_t)m * K + k] = (double)int4_value(c) * (double)scales[(size_t)m * (K / 128) + k / 128];
        }
}

/* ======================================================================== */
/* GEMM references                                                          */
/* ======================================================================== */

static uint8_t nib(const uint8_t* codes, size_t row_bytes, int r, int k) {
    uint8_t byte = codes[(size_t)r * row_bytes + k / 2];
    return (k & 1) ? (byte >> 4) : (byte & 15);
}

/* Twice an E2M1 value is an integer in [-12, 12]. */
static int e2m1_x2(uint8_t c) {
    static const int mag2[8] = {0, 1, 2, 3, 4, 6, 8, 12};
    int v = mag2[c & 7];
    return (c & 8) ? -v : v;
}

/* Block-scaled NVFP4 product, exact: every E4M3 scale is an integer times
 * 2^-9 and every E2M1 value an integer times 2^-1, so
 *   sum_k a^ w^ = 2^-20 * sum_b (512 sa_b)(512 sw_b) sum_{k in b} (2 ea)(2 ew)
 * is an integer times 2^-20; it is summed in 128-bit integers and multiplied
 * by alpha = s2a * s2w in fp64 before the single bf16 rounding. */
int orc_gemm_nvfp4(const uint8_t* ca, const uint8_t* sa, const float* s2a, int a_mode,
                   const uint8_t* cw, const uint8_t* sw, const float* s2w,
                   int M, int N, int K, uint16_t* Y, double* yref, double* absdot) {
    return orc_gemm_nvfp4_wrows(ca, sa, s2a, a_mode, cw, sw, s2w, 0, M, N, K, Y, yref, absdot);
}

int orc_gemm_nvfp4_wrows(const uint8_t* ca, const uint8_t* sa, const float* s2a, int a_mode,
                         const uint8_t* cw, const uint8_t* sw, const float* s2w, int w_mode,
                         int M, int N, int K, uint16_t* Y, double* yref, double* absdot) {
    if (K % 16) return -1;
    const int KB = K / 16;
    for (int m = 0; m < M; ++m) {
        double s2m = (double)(a_mode == 1 ? s2a[m] : s2a[0]);
        for (int n = 0; n < N; ++n) {
            double alpha = s2m * (double)(w_mode == 1 ? s2w[n] : s2w[0]);
            __int128 acc = 0, aacc = 0;
            for (int b = 0; b < KB; ++b) {
                long long p = 0, ap = 0;
                for (int k = 16 * b; k < 16 * b + 16; ++k) {
                    int t = e2m1_x2(nib(ca, K / 2, m, k)) * e2m1_x2(nib(cw, K / 2, n, k));
                    p += t;
                    ap += t < 0 ? -t : t;
                }
                long long sab = (long long)ldexp((double)orc_e4m3_decode(sa[(size_t)m * KB + b]), 9);
                long long swb = (long long)ldexp((double)orc_e4m3_decode(sw[(size_t)n * KB + b]), 9);
                acc += (__int128)p * sab * swb;
                aacc += (__int128)ap * sab * swb;
            }
            double exact = ldexp((double)acc, -20) * alpha;
            if (Y) Y[(size_t)m * N + n] = orc_f64_to_bf16(exact);
            if (yref) yref[(size_t)m * N + n] = exact;
            if (absdot) absdot[(size_t)m * N + n] = ldexp((double)aacc, -20) * fabs(alpha);
        }
    }
    return 0;
}

/* MXFP4: per 32-block integer sum of (2ea)(2ew), times the two power-of-two
 * block scales, accumulated in fp64. */
int orc_gemm_mxfp4(const uint8_t* ca, const uint8_t* sa, const uint8_t* cw, const uint8_t* sw,
                   int M, int N, int K, uint16_t* Y, double* yref, double* absdot) {
    if (K % 32) return -1;
    const int KB = K / 32;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int b = 0; b < KB; ++b) {
                long long p = 0, ap = 0;
                for (int k = 32 * b; k < 32 * b + 32; ++k) {
                    int t = e2m1_x2(nib(ca, K / 2, m, k)) * e2m1_x2(nib(cw, K / 2, n, k));
                    p += t;
                    ap += t < 0 ? -t : t;
                }
                double sc = 0.25 * (double)orc_e8m0_decode(sa[(size_t)m * KB + b]) *
                            (double)orc_e8m0_decode(sw[(size_t)n * KB + b]);
                acc += (double)p * sc;
                aacc += (double)ap * sc;
            }
            if (Y) Y[(size_t)m * N + n] = orc_f64_to_bf16(acc);
            if (yref) yref[(size_t)m * N + n] = acc;
            if (absdot) absdot[(size_t)m * N + n] = aacc;
        }
    return 0;
}

/* INT4-g128: exact integer partial sum per group, rescaled by the product of
 * the two FP32 group scales, accumulated in fp64. */
int orc_gemm_int4(const uint8_t* ca, const float* sa, const uint8_t* cw, const float* sw,
                  int M, int N, int K, uint16_t* Y, double* yref, double* absdot) {
    if (K % 128) return -1;
    const int G = K / 128;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int g = 0; g < G; ++g) {
                long long p = 0, ap = 0;
                for (int k = 128 * g; k < 128 * g + 128; ++k) {
                    int t = int4_value(nib(ca, K / 2, m, k)) * int4_value(nib(cw, K / 2, n, k));
                    p += t;
                    ap += t < 0 ? -t : t;
                }
                double sc = (double)sa[(size_t)m * G + g] * (double)sw[(size_t)n * G + g];
                acc += (double)p * sc;
                aacc += (double)ap * fabs(sc);
            }
            if (Y) Y[(size_t)m * N + n] = orc_f64_to_bf16(acc);
            if (yref) yref[(size_t)m * N + n] = acc;
            if (absdot) absdot[(size_t)m * N + n] = aacc;
        }
    return 0;
}

/* INT4 product with groups of G elements: exact integer partial sum per
 * group, scaled by sa[m,g] * sw[n,g] (fp64), summed. */
int orc_gemm_int4_g(const uint8_t* ca, const float* sa, const uint8_t* cw, const float* sw,
                    int M, int N, int K, int G, uint16_t* Y, double* yref, double* absdot) {
    if (G < 128 || G % 128 || K % G) return -1;
    const int NG = K / G;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int g = 0; g < NG; ++g) {
                long long p = 0, ap = 0;
                for (int k = G * g; k < G * g + G; ++k) {
                    int t = int4_value(nib(ca, K / 2, m, k)) * int4_value(nib(cw, K / 2, n, k));
                    p += t;
                    ap += t < 0 ? -t : t;
                }
                double sc = (double)sa[(size_t)m * NG + g] * (double)sw[(size_t)n * NG + g];
                acc += (double)p * sc;
                aacc += (double)ap * fabs(sc);
            }
            if (Y) Y[(size_t)m * N + n] = orc_f64_to_bf16(acc);
            if (yref) yref[(size_t)m * N + n] = acc;
            if (absdot) absdot[(size_t)m * N + n] = aacc;
        }
    return 0;
}

/* ======================================================================== */
/* Dual-stage residual augmentation                                         */
/* ======================================================================== */

int orc_augment_nvfp4(const uint16_t* X, int M, int K, int ldx,
                      const int32_t* S, int nS,
                      const uint8_t* codes, const uint8_t* scales,
                      const float* s2, int mode,
                      uint8_t* rcodes, uint8_t* rscales) {
    if (nS % 16 || K % 16 || ldx < K) return -1;
    for (int j = 0; j < nS; ++j)
        if (S[j] < 0 || S[j] >= K) return -1; /* any order: column K + j holds channel S[j] */
    float* r = (float*)malloc(sizeof(float) * (size_t)(nS > 0 ? nS : 1));
    for (int m = 0; m < M; ++m) {
        float rs2 = (mode == 1) ? s2[m] : s2[0];
        for (int j = 0; j < nS; ++j) {
            int k = S[j];
            float x = orc_bf16_to_f32(X[(size_t)m * ldx + k]);
            uint8_t c = nib(codes, K / 2, m, k);
            uint8_t sb = scales[(size_t)m * (K / 16) + k / 16];
            /* first-stage dequantized value e * scale * s2, rounded to FP32 */
            float xhat = (float)((double)orc_e2m1_decode(c) * (double)orc_e4m3_decode(sb) * (double)rs2);
            r[j] = x - xhat;
        }
        for (int b = 0; b < nS / 16; ++b)
            nvfp4_block(r + 16 * b, rs2, rcodes + (size_t)m * (nS / 2) + 8 * b,
                        rscales + (size_t)m * (nS / 16) + b);
    }
    free(r);
    return 0;
}

int orc_select_channels(const uint16_t* Xcal, int Mc, int K, int nS, int32_t* S) {
    if (nS < 0 || nS > K) return -1;
    float* amax = (float*)calloc((size_t)K, sizeof(float));
    char* taken = (char*)calloc((size_t)K, 1);
    for (int m = 0; m < Mc; ++m)
        for (int k = 0; k < K; ++k)
            amax[k] = fmaxf(amax[k], fabsf(orc_bf16_to_f32(Xcal[(size_t)m * K + k])));
    for (int j = 0; j < nS; ++j) {         /* pick the largest remaining, lowest index on ties */
        int best = -1;
        for (int k = 0; k < K; ++k)
            if (!taken[k] && (best < 0 || amax[k] > amax[best])) best = k;
        taken[best] = 1;
    }
    int j = 0;
    for (int k = 0; k < K; ++k)
        if (taken[k]) S[j++] = k;
    free(amax);
    free(taken);
    return 0;
}
