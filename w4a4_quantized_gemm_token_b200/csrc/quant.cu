// Activation / weight quantizers (NVFP4, MXFP4, INT4-g128), the tensor-amax
// pass, the residual-channel second stage and channel selection.
//
// Row-per-CTA design: a CTA owns one row, every thread owns J chunks of 16
// consecutive elements (two 16-byte loads each).  All loads of a row are
// issued before any arithmetic, so each SM keeps tens of KB in flight; block
// amaxes reduce over 1 (NVFP4), 2 (MXFP4) or 8 (INT4) neighbouring lanes with
// xor-shuffles, the per-token amax over the CTA.  Codes leave as 8-byte
// stores (a warp writes 256 contiguous bytes), NVFP4/MXFP4 scales as 4-byte
// words gathered by shuffles into the MMA's 128x4 scale atoms.
#include <cstdint>
#include <cuda_bf16.h>
#include <type_traits>
#include <cuda_fp8.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

__constant__ float kE2M1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// max |x| of the 16 bf16 elements held in w[8]: packed bf16x2 maxima of the
// magnitudes (exact; the xorsign result sign is discarded), then the halves.
__device__ __forceinline__ float bmax16(const uint32_t* w) {
    uint32_t m[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[e]) : "r"(w[e]), "r"(w[e + 4]));
    asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m[0]) : "r"(m[2]));
    asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m[1]) : "r"(m[3]));
    asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m[0]) : "r"(m[1]));
    const uint32_t a = m[0] & 0x7FFF7FFFu;
    return fmaxf(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u));
}

// E2M1 codes of 8 floats packed into one word, element i in nibble i (round
// to nearest even, saturating at 6).  The conversion keeps the input's sign
// bit, so a negative value that rounds to zero (and -0) encodes as 0x8.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// E2M1 codes of two values in one byte, lo in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2_byte(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.u32.u8 %0, b0;\n\t}"
        : "=r"(out)
        : "f"(lo), "f"(hi));
    return out & 0xFFu;
}

// Correctly rounded quotient x/d from a correctly rounded reciprocal
// y = RN(1/d): q = RN(x*y) is within an ulp of x/d, the residual x - q*d is
// exact in one FMA, and one more FMA rounds q + residual*y to RN(x/d).  This
// is Markstein's correction theorem for FMA-based division (P. Markstein,
// IBM J. Res. Dev. 34(1), 1990; restated in Muller et al., Handbook of
// Floating-Point Arithmetic, the section on Newton-Raphson division).  This
// holds whenever the quotient is a normal float; the callers keep operands in
// that range (or their results do not depend on it: quotients below the
// normal range encode to zero anyway) and fall back to IEEE division outside.
// d > 0, so the quotient carries x's sign; restoring it keeps -0 for x = -0
// (the residual step would otherwise return +0).
__device__ __forceinline__ float div_refined(float x, float d, float y) {
    const float q = __fmul_rn(x, y);
    return copysignf(__fmaf_rn(__fmaf_rn(-q, d, x), y, q), x);
}

// Two correctly rounded quotients at once with sm_100's packed FP32 pipe.
// Inputs are the NEGATED dividends nx = -x (the bf16 unpack yields them at no
// cost) and ny = -y.  q = nx*ny = x*y, R = q*d + nx = q*d - x (exact), and
// q' = R*ny + q = q - R*y, the same refinement as div_refined; written this
// way a dividend of -0 keeps its sign (q = -0, R = +0, q' = -0 + -0 = -0).
__device__ __forceinline__ void div2_refined(uint32_t nx0, uint32_t nx1, uint64_t ny2, uint64_t d2, float& q0,
                                             float& q1) {
    asm("{\n\t.reg .b64 x, q, r;\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mul.rn.f32x2 q, x, %4;\n\t"
        "fma.rn.f32x2 r, q, %5, x;\n\t"
        "fma.rn.f32x2 q, r, %4, q;\n\t"
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(q0), "=f"(q1)
        : "r"(nx0), "r"(nx1), "l"(ny2), "l"(d2));
}
__device__ __forceinline__ uint64_t pack2(float v) {
    const uint32_t u = __float_as_uint(v);
    return ((uint64_t)u << 32) | u;
}

// Negated dividends of the 16 bf16 elements held in w[8] (element 2e in the
// low half of w[e]): -x = float bits of the bf16 with the sign flipped.
__device__ __forceinline__ uint32_t neg_lo(uint32_t w) { return (w << 16) ^ 0x80000000u; }
__device__ __forceinline__ uint32_t neg_hi(uint32_t w) { return (w & 0xFFFF0000u) ^ 0x80000000u; }

// E2M1 codes of x/d for the 8 elements held in w[0..3], quotients correctly
// rounded by the refined division (divisor and quotients in normal range),
// on sm_100's packed FP32 operations.  ny2 holds ny = -RN(1/d) (both
// halves), d2 holds d.  With the dividend x as it is: q = RN(x * ny) is
// within an ulp of -x/d, R = q*d + x is exact, and q' = RN(R * ny + q) is
// the correctly rounded -x/d (the same correction step as div_refined).
// The codes of -x/d are those of x/d with the sign bit flipped (the E2M1
// grid and its rounding are symmetric), so one XOR per 8 codes restores
// them; a dividend of +0 or -0 gives the opposite zero, so the flip keeps
// the sign of zero too.
__device__ __forceinline__ uint32_t e2m1x8_fast(const uint32_t* w, uint64_t ny2, uint64_t d2) {
    const float2 ny = make_float2(__uint_as_float((uint32_t)ny2), __uint_as_float((uint32_t)ny2));
    const float2 d = make_float2(__uint_as_float((uint32_t)d2), __uint_as_float((uint32_t)d2));
    float q[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 x = make_float2(bf16lo(w[e]), bf16hi(w[e]));
        const float2 q0 = __fmul2_rn(x, ny);
        const float2 r = __ffma2_rn(q0, d, x);
        const float2 q1 = __ffma2_rn(r, ny, q0);
        q[2 * e] = q1.x;
        q[2 * e + 1] = q1.y;
    }
    return e2m1x8(q) ^ 0x88888888u;
}
// The same with IEEE division (any operands).
__device__ __forceinline__ uint32_t e2m1x8_exact(uint4 v, float d) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float q[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        q[2 * e] = __fdiv_rn(bf16lo(w[e]), d);
        q[2 * e + 1] = __fdiv_rn(bf16hi(w[e]), d);
    }
    return e2m1x8(q);
}

// 4-bit two's-complement codes of clamp(rint(x/s), -8, 7) for the 8 elements
// held in w[0..3].  Rounding to the nearest integer, ties to even, is an
// addition of 1.5 * 2^23: the low bits of the sum are rint(q) in two's
// complement.  On the refined path |x/s| <= 7(1 + 2^-24), so no clamp.
__device__ __forceinline__ uint32_t int4x8_fast(const uint32_t* w, uint64_t ny2, uint64_t d2) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    uint32_t out = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float q0, q1;
        div2_refined(neg_lo(w[e]), neg_hi(w[e]), ny2, d2, q0, q1);
        const uint32_t n0 = __float_as_uint(__fadd_rn(q0, kMagic)) & 15u;
        const uint32_t n1 = __float_as_uint(__fadd_rn(q1, kMagic)) & 15u;
        out |= (n0 | (n1 << 4)) << (8 * e);
    }
    return out;
}
__device__ __forceinline__ uint32_t int4x8_exact(uint4 v, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int n0 = min(max(__float2int_rn(__fdiv_rn(bf16lo(w[e]), s)), -8), 7);
        const int n1 = min(max(__float2int_rn(__fdiv_rn(bf16hi(w[e]), s)), -8), 7);
        out |= (uint32_t)((n0 & 15) | ((n1 & 15) << 4)) << (8 * e);
    }
    return out;
}

// The same encoders on FP32 inputs (rotated values): negated dividends are the
// inputs with the sign bit flipped.
__device__ __forceinline__ uint32_t neg_f(float v) { return __float_as_uint(v) ^ 0x80000000u; }
__device__ __forceinline__ uint32_t e2m1x8_fast_f(const float* v, uint64_t ny2, uint64_t d2) {
    float q[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) div2_refined(neg_f(v[2 * e]), neg_f(v[2 * e + 1]), ny2, d2, q[2 * e], q[2 * e + 1]);
    return e2m1x8(q);
}
__device__ __forceinline__ uint32_t e2m1x8_exact_f(const float* v, float d) {
    float q[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = __fdiv_rn(v[e], d);
    return e2m1x8(q);
}
__device__ __forceinline__ uint32_t int4x8_fast_f(const float* v, uint64_t ny2, uint64_t d2) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    uint32_t out = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float q0, q1;
        div2_refined(neg_f(v[2 * e]), neg_f(v[2 * e + 1]), ny2, d2, q0, q1);
        const uint32_t n0 = __float_as_uint(__fadd_rn(q0, kMagic)) & 15u;
        const uint32_t n1 = __float_as_uint(__fadd_rn(q1, kMagic)) & 15u;
        out |= (n0 | (n1 << 4)) << (8 * e);
    }
    return out;
}
__device__ __forceinline__ uint32_t int4x8_exact_f(const float* v, float s) {
    uint32_t out = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int n0 = min(max(__float2int_rn(__fdiv_rn(v[2 * e], s)), -8), 7);
        const int n1 = min(max(__float2int_rn(__fdiv_rn(v[2 * e + 1], s)), -8), 7);
        out |= (uint32_t)((n0 & 15) | ((n1 & 15) << 4)) << (8 * e);
    }
    return out;
}

// Block-local Walsh-Hadamard rotation of one item (16 consecutive elements of
// an N-element block; the block's items sit on N/16 consecutive lanes, the
// item's place in its block is c mod N/16).  Fast Walsh-Hadamard butterflies
// in FP32, stages h = 1, 2, ..., N/2, (a, b) -> (a + b, a - b): stages below
// 16 inside the thread, the others with the lane holding the partner items.
// The activation side then multiplies by 1/N (exact), the weight side keeps
// the transform unscaled, so (X H/N)(W H)^T = X W^T.  Every lane of the warp
// must call it (the shuffles use the full mask).
template <int N>
__device__ __forceinline__ void rotate_item(const uint32_t* w, float* v, int c, bool act) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        v[2 * e] = bf16lo(w[e]);
        v[2 * e + 1] = bf16hi(w[e]);
    }
#pragma unroll
    for (int h = 1; h < 16; h *= 2)
#pragma unroll
        for (int e = 0; e < 16; ++e)
            if (!(e & h)) {
                const float x = v[e], y = v[e + h];
                v[e] = __fadd_rn(x, y);
                v[e + h] = __fsub_rn(x, y);
            }
#pragma unroll
    for (int st = 0; (16 << st) < N; ++st) {
        const bool upper = (c >> st) & 1;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float p = __shfl_xor_sync(0xffffffffu, v[e], 1 << st);
            v[e] = upper ? __fsub_rn(p, v[e]) : __fadd_rn(v[e], p);
        }
    }
    if (act) {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = __fmul_rn(v[e], 1.0f / N);
    }
}
__device__ __forceinline__ float absmax16(const float* v) {
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
    return m;
}

__device__ __forceinline__ uint8_t e4m3_rn_sat(float t) {
    return (uint8_t)__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_value(uint8_t c) {
    __nv_fp8_e4m3 f;
    f.__x = c;
    return static_cast<float>(f);
}

// Second-level NVFP4 scale from an amax: amax/2688, or 1 when that is not a
// positive normal float (zero amax included).
__device__ __forceinline__ float nvfp4_s2(float amax) {
    float s2 = __fdiv_rn(amax, 2688.0f);
    return (amax > 0.0f && s2 >= 1.17549435e-38f) ? s2 : 1.0f;
}

// Byte offset of scale (row r, block c) in the MMA scale layout.
__device__ __forceinline__ size_t sf_offset(int r, int c, int col_atoms) {
    return ((size_t)(r >> 7) * col_atoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// MXFP4 shared-exponent code of a block with amax a > 0: floor(log2 a) - 2,
// biased by 127 and clamped to E8M0's range (subnormal amaxes included).
__device__ __forceinline__ uint32_t mx_code(float a) {
    const uint32_t u = __float_as_uint(a);
    const int E = (int)(u >> 23);
    const int e = (E != 0) ? E - 127 : (31 - __clz((int)(u & 0x7FFFFF))) - 149;
    return (uint32_t)min(max(e + 125, 0), 254);
}
// 2^(code - 127), the unit of an E8M0 code (code 0 is the subnormal 2^-127).
__device__ __forceinline__ float mx_unit(uint32_t code) {
    return code ? __uint_as_float(code << 23) : __uint_as_float(0x00400000u);
}
// Value of an E2M1 code (bit 3 the sign): m/2 for exponent field 0, else
// (1 + m/2) * 2^(e-1); built as float bits.
__device__ __forceinline__ float e2m1_decode(uint32_t nib) {
    const uint32_t e = (nib >> 1) & 3u, m = nib & 1u;
    const uint32_t mag = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
    return __uint_as_float(mag | ((nib & 8u) << 28));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// The same maximum for values that are >= 0 or NaN, in one warp reduction:
// the bit patterns of non-negative floats order as their values.  A NaN lane
// counts as 0 (fmaxf ignores NaN operands); only an all-NaN warp differs (0
// instead of NaN), and a row amax of 0 or NaN gives the same s2 (1).
__device__ __forceinline__ float warp_max_nonneg(float v) {
    return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(v, 0.0f))));
}

// ---------------------------------------------------------------------------
// Quantize rows.  A CTA owns `rows_per_cta` consecutive rows: one bulk copy
// per row brings the bf16 row into shared memory (several CTAs per SM keep
// tens of KB in flight), a first pass takes per-token amaxes (NVFP4 TOKEN),
// a second quantizes.  Work item = (row, chunk of 16 elements), flattened so
// that every thread is busy whatever K is; since K/16 is a multiple of 8,
// the groups of 2 (MXFP4) and 8 (INT4, scale packing) consecutive items that
// the shuffles combine never straddle two rows.  Rows >= M only write zero
// scales (padding of the 128-row scale atoms).
// ---------------------------------------------------------------------------
// Per-row constants of the NVFP4 block rule, kept in shared memory.
struct RowConsts {
    float s2;    // second-level scale
    float rinv;  // RN(1/s2)
    int fast;    // s2 in the range where refined division is exact
    int pad;
};

// MULTI (MXFP4 only): the multi-pass decomposition, a.passes passes.  ROT:
// every block rotated first (rotate_item; a.rot 1 = activation side, 2 =
// weight side).
template <int FMT, bool GATHER, bool MULTI = false, bool ROT = false>
__global__ void __launch_bounds__(256, 4) quant_rows_kernel(QuantArgs a, int rows_per_cta, int nbuf) {
    constexpr int NB = FMT == FMT_NVFP4 ? 16 : FMT == FMT_MXFP4 ? 32 : 128;  // block (rotation) size
    pdl_launch_dependents();
    pdl_wait();  // X and the words to clear may belong to the preceding launch
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.zero_count; i += blockDim.x) a.zero_words[i] = 0;
    extern __shared__ __align__(16) uint8_t qsm[];
    const int row_bytes = a.K_src * 2;                        // bf16 source row in shared memory
    const size_t buf_bytes = (size_t)rows_per_cta * row_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(qsm + nbuf * buf_bytes);
    float* rmax = reinterpret_cast<float*>(bars + nbuf);      // [rows_per_cta] per-token amax
    RowConsts* rc = reinterpret_cast<RowConsts*>(rmax + rows_per_cta);
    float* bm = reinterpret_cast<float*>(rc + rows_per_cta);  // per-item block max (NVFP4 token mode)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bm + (FMT == FMT_NVFP4 ? rows_per_cta * (a.K / 16) : 0));
    const int t = threadIdx.x, T = blockDim.x;
    const int nchunk = a.K / 16;
    const int nblocks = (a.rows_pad + rows_per_cta - 1) / rows_per_cta;

    // live rows of row block bi (rows >= M are scale padding, never loaded)
    auto live_rows = [&](int bi) { return max(0, min(rows_per_cta, a.M - bi * rows_per_cta)); };
    auto issue_load = [&](int bi, int buf) {
        const int nl = live_rows(bi);
        if (nl == 0) return;
        mbar_arrive_expect_tx(&bars[buf], (uint32_t)(nl * row_bytes));
        for (int i = 0; i < nl; ++i)
            bulk_load(qsm + buf * buf_bytes + (size_t)i * row_bytes,
                      a.X + (size_t)(bi * rows_per_cta + i) * a.ldx, row_bytes, &bars[buf]);
    };

    if (t == 0) {
        for (int b = 0; b < nbuf; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (t == 0)
        for (int k = 0; k < nbuf; ++k) {
            const int bi = blockIdx.x + k * gridDim.x;
            if (bi < nblocks) issue_load(bi, k);
        }

    int li = 0;
    for (int bi = blockIdx.x; bi < nblocks; bi += gridDim.x, ++li) {
    const int buf = li % nbuf;
    const uint8_t* rows = qsm + buf * buf_bytes;
    const int r0 = bi * rows_per_cta;
    const int nrows = min(rows_per_cta, a.rows_pad - r0);
    const int nlive = live_rows(bi);
    if (t < rows_per_cta) rmax[t] = 0.0f;
    if (nlive > 0 && !mbar_wait(&bars[buf], (li / nbuf) & 1, 2000000000ull, abort_flag, 20000)) break;
    __syncthreads();

    const bool token = FMT == FMT_NVFP4 && a.mode == 1 && !a.static_s2;
    const int items = nrows * nchunk;
    if (token) {
        for (int it = t; it < items; it += T) {
            const int i = it / nchunk, c = it - i * nchunk;
            if (i >= nlive) break;
            const uint4* p = reinterpret_cast<const uint4*>(rows + (size_t)i * row_bytes) + 2 * c;
            const uint4 v0 = p[0], v1 = p[1];
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float m;
            if constexpr (ROT) {  // NVFP4 blocks are single items: no lane exchange here
                float v[16];
                rotate_item<16>(w, v, c, a.rot == 1);
                m = absmax16(v);
            } else {
                m = bmax16(w);
            }
            bm[it] = m;  // reused by the quantization pass
            // items of one row are consecutive: reduce over the 8-lane group first
            m = fmaxf(m, __shfl_xor_sync(__activemask(), m, 1));
            m = fmaxf(m, __shfl_xor_sync(__activemask(), m, 2));
            m = fmaxf(m, __shfl_xor_sync(__activemask(), m, 4));
            if ((c & 7) == 0) atomicMax(reinterpret_cast<unsigned int*>(rmax + i), __float_as_uint(m));  // m >= 0
        }
        __syncthreads();
    }
    if constexpr (FMT == FMT_NVFP4) {
        const float tensor_s2 = a.mode == 0 ? (a.static_s2 ? a.static_s2[0] : nvfp4_s2(*a.tensor_amax)) : 1.0f;
        if (a.mode == 0 && bi == 0 && t == 0 && a.s2_out) a.s2_out[0] = tensor_s2;
        if (t < nrows) {
            float s2 = tensor_s2;
            if (a.mode == 1) s2 = t < nlive ? (a.static_s2 ? a.static_s2[r0 + t] : nvfp4_s2(rmax[t])) : 1.0f;
            if (a.mode == 1 && t < nlive) a.s2_out[r0 + t] = s2;
            RowConsts k;
            k.s2 = s2;
            k.rinv = __frcp_rn(s2);
            k.fast = (s2 >= 0x1p-100f && s2 <= 0x1p100f) ? 1 : 0;
            k.pad = 0;
            rc[t] = k;
        }
        __syncthreads();
    }

    const int iters = (items + T - 1) / T;
    // (row, chunk) of item t + T*j, advanced without a division per item
    const int di = T / nchunk, dc = T - di * nchunk;
    int i = t / nchunk, c = t - i * nchunk;
    for (int j = 0; j < iters; ++j) {
        const int it = t + T * j;
        const bool valid = it < items;           // uniform per group of 8 lanes
        const int r = r0 + i;
        const bool live = valid && i < nlive;
        uint32_t w[8];  // 16 bf16 elements, element 2e in the low half of w[e]
        if (live) {
            const uint8_t* row = rows + (size_t)i * row_bytes;
            if (!GATHER || 16 * c + 16 <= a.K_src) {
                const uint4* p = reinterpret_cast<const uint4*>(row) + 2 * c;
                const uint4 v0 = p[0], v1 = p[1];
                w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
                w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
            } else {
                // augmented weight columns: element k >= K_src is column S[k - K_src]
                const uint16_t* rw = reinterpret_cast<const uint16_t*>(row);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[e] = (uint32_t)rw[checked_channel(a.S, 16 * c + 2 * e - a.K_src, a.K_src)] |
                           ((uint32_t)rw[checked_channel(a.S, 16 * c + 2 * e + 1 - a.K_src, a.K_src)] << 16);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = 0;
        }
        float v[16];  // ROT: the rotated values of the item
        if constexpr (ROT) rotate_item<NB>(w, v, c, a.rot == 1);
        float bmax;
        if constexpr (ROT) bmax = (token && live) ? bm[it] : absmax16(v);
        else bmax = (token && live) ? bm[it] : bmax16(w);

        uint32_t w0 = 0, w1 = 0;  // 16 codes
        bool stored = false;      // INT4 codes already written widened
        if constexpr (FMT == FMT_NVFP4) {
            const RowConsts k = rc[i < nrows ? i : 0];
            // block scale E4M3(RN(RN(bmax/6)/s2)) and quotients x/(scale*s2), by refined
            // division on the hot path; operands outside its range go to IEEE division
            const float u = div_refined(bmax, 6.0f, 0x1.555556p-3f);  // RN(1/6)
            const uint8_t sb = live ? e4m3_rn_sat(div_refined(u, k.s2, k.rinv)) : 0;
            const float d = sb ? __fmul_rn(e4m3_value(sb), k.s2) : 1.0f;
            const float y = __frcp_rn(d);
            if constexpr (ROT) {
                w0 = e2m1x8_fast_f(v, pack2(-y), pack2(d));
                w1 = e2m1x8_fast_f(v + 8, pack2(-y), pack2(d));
            } else {
                w0 = e2m1x8_fast(w, pack2(-y), pack2(d));
                w1 = e2m1x8_fast(w + 4, pack2(-y), pack2(d));
            }
            const bool slow = live && !(k.fast && bmax >= 0x1p-100f && d >= 0x1p-100f && d <= 0x1p100f &&
                                        __fmul_rn(bmax, y) <= 0x1p60f);
            uint8_t sbf = sb;
            if (__any_sync(0xffffffffu, slow)) {
                if (slow) {
                    sbf = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), k.s2));
                    const float de = __fmul_rn(e4m3_value(sbf), k.s2);
                    if constexpr (ROT) {
                        w0 = sbf ? e2m1x8_exact_f(v, de) : 0u;
                        w1 = sbf ? e2m1x8_exact_f(v + 8, de) : 0u;
                    } else {
                        w0 = sbf ? e2m1x8_exact(make_uint4(w[0], w[1], w[2], w[3]), de) : 0u;
                        w1 = sbf ? e2m1x8_exact(make_uint4(w[4], w[5], w[6], w[7]), de) : 0u;
                    }
                }
            }
            if (sbf == 0) {
                w0 = 0;
                w1 = 0;
            }
            // gather 4 consecutive block scales (lanes l..l+3) into one word
            const uint32_t b = sbf;
            const uint32_t b1 = __shfl_down_sync(0xffffffffu, b, 1);
            const uint32_t b2 = __shfl_down_sync(0xffffffffu, b, 2);
            const uint32_t b3 = __shfl_down_sync(0xffffffffu, b, 3);
            if (valid && (c & 3) == 0)
                *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, c, a.sf_col_atoms)) =
                    b | (b1 << 8) | (b2 << 16) | (b3 << 24);
        } else if constexpr (FMT == FMT_MXFP4) {
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));  // 32-element block = 2 items
            uint32_t code = 0;
            if (live && bmax > 0.0f) {
                code = mx_code(bmax);
                const float inv = __uint_as_float((254u - code) << 23);  // 2^(127 - code)
                float q0[8], q1[8];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    if constexpr (ROT) {
                        q0[2 * e2] = __fmul_rn(v[2 * e2], inv);
                        q0[2 * e2 + 1] = __fmul_rn(v[2 * e2 + 1], inv);
                        q1[2 * e2] = __fmul_rn(v[8 + 2 * e2], inv);
                        q1[2 * e2 + 1] = __fmul_rn(v[9 + 2 * e2], inv);
                        continue;
                    }
                    q0[2 * e2] = __fmul_rn(bf16lo(w[e2]), inv);
                    q0[2 * e2 + 1] = __fmul_rn(bf16hi(w[e2]), inv);
                    q1[2 * e2] = __fmul_rn(bf16lo(w[4 + e2]), inv);
                    q1[2 * e2 + 1] = __fmul_rn(bf16hi(w[4 + e2]), inv);
                }
                w0 = e2m1x8(q0);
                w1 = e2m1x8(q1);
            }
            const uint32_t b1 = __shfl_down_sync(0xffffffffu, code, 2);
            const uint32_t b2 = __shfl_down_sync(0xffffffffu, code, 4);
            const uint32_t b3 = __shfl_down_sync(0xffffffffu, code, 6);
            if (valid && (c & 7) == 0)
                *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, c >> 1, a.sf_col_atoms)) =
                    code | (b1 << 8) | (b2 << 16) | (b3 << 24);
            if constexpr (MULTI) {
                // Multi-pass decomposition ("APEX4: Efficient Pure W4A4..." page,
                // para 1, MSD): pass p quantizes, by the same rule, the residual
                // x - (values of passes 0..p-1), formed in FP32 (exact: a bf16 value).
                float res[16];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) {
                    res[e2] = (e2 & 1) ? bf16hi(w[e2 >> 1]) : bf16lo(w[e2 >> 1]);
                    res[8 + e2] = (e2 & 1) ? bf16hi(w[4 + (e2 >> 1)]) : bf16lo(w[4 + (e2 >> 1)]);
                }
                uint32_t pc = code, p0 = w0, p1 = w1;
                for (int p = 1; p < a.passes; ++p) {
                    const float unit = mx_unit(pc);
                    float rmax = 0.0f;
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const uint32_t nib = ((e2 < 8 ? p0 : p1) >> (4 * (e2 & 7))) & 15u;
                        res[e2] = __fsub_rn(res[e2], __fmul_rn(e2m1_decode(nib), unit));
                        rmax = fmaxf(rmax, fabsf(res[e2]));
                    }
                    rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 1));
                    pc = 0;
                    p0 = p1 = 0;
                    if (live && rmax > 0.0f) {
                        pc = mx_code(rmax);
                        const float inv = __uint_as_float((254u - pc) << 23);
                        float q0[8], q1[8];
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2) {
                            q0[e2] = __fmul_rn(res[e2], inv);
                            q1[e2] = __fmul_rn(res[8 + e2], inv);
                        }
                        p0 = e2m1x8(q0);
                        p1 = e2m1x8(q1);
                    }
                    const uint32_t c1 = __shfl_down_sync(0xffffffffu, pc, 2);
                    const uint32_t c2 = __shfl_down_sync(0xffffffffu, pc, 4);
                    const uint32_t c3 = __shfl_down_sync(0xffffffffu, pc, 6);
                    if (valid && (c & 7) == 0)
                        *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, p * (a.K >> 5) + (c >> 1), a.sf_col_atoms)) =
                            pc | (c1 << 8) | (c2 << 16) | (c3 << 24);
                    if (live)
                        *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + (size_t)p * (a.K >> 1) + 8 * c) =
                            make_uint2(p0, p1);
                }
            }
        } else {  // INT4, a group of a.group elements = R8 items on consecutive lanes
            const int R8 = a.group >> 4;  // 8, 16 or 32
            for (int o = 1; o < R8; o <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
            const bool fast = bmax >= 0x1p-100f && bmax <= 0x1p100f;
            float sc = live ? div_refined(bmax, 7.0f, 0x1.24924ap-3f) : 0.0f;  // RN(1/7)
            const float y = __frcp_rn(sc > 0.0f ? sc : 1.0f);
            if constexpr (ROT) {
                w0 = int4x8_fast_f(v, pack2(-y), pack2(sc));
                w1 = int4x8_fast_f(v + 8, pack2(-y), pack2(sc));
            } else {
                w0 = int4x8_fast(w, pack2(-y), pack2(sc));
                w1 = int4x8_fast(w + 4, pack2(-y), pack2(sc));
            }
            const bool slow = live && !fast;
            if (__any_sync(0xffffffffu, slow)) {
                if (slow) {
                    sc = __fdiv_rn(bmax, 7.0f);
                    if constexpr (ROT) {
                        w0 = sc != 0.0f ? int4x8_exact_f(v, sc) : 0u;
                        w1 = sc != 0.0f ? int4x8_exact_f(v + 8, sc) : 0u;
                    } else {
                        w0 = sc != 0.0f ? int4x8_exact(make_uint4(w[0], w[1], w[2], w[3]), sc) : 0u;
                        w1 = sc != 0.0f ? int4x8_exact(make_uint4(w[4], w[5], w[6], w[7]), sc) : 0u;
                    }
                }
            }
            if (sc == 0.0f) {
                w0 = 0;
                w1 = 0;
            }
            if (valid && (c & (R8 - 1)) == 0) a.sfi[(size_t)(c / R8) * a.sfi_ld + r] = sc;
            if (a.int8_codes) {  // already widened for the GEMM: 16 bytes of 16 * q
                if (live) {
                    uint32_t o[4];
                    widen8_x16(w0, o[0], o[1]);
                    widen8_x16(w1, o[2], o[3]);
                    *reinterpret_cast<uint4*>(a.codes + (size_t)r * a.ldc + 16 * c) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                stored = true;
            }
        }
        if (live && !stored) *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + 8 * c) = make_uint2(w0, w1);
        i += di;
        c += dc;
        if (c >= nchunk) {
            c -= nchunk;
            ++i;
        }
    }
    __syncthreads();  // every thread is done with this buffer and with rmax/rc
    if (t == 0) {
        const int nb = bi + nbuf * gridDim.x;
        if (nb < nblocks) issue_load(nb, buf);
    }
    }
    if (*abort_flag && t == 0)  // wait for the loads still in flight
        for (int b = 0; b < nbuf; ++b) mbar_wait_drain(&bars[b], 0, 100000000ull);
}

// ---------------------------------------------------------------------------
// Tensor amax: max |x| over X[M, K] into *out (as float bits; *out must start
// at 0).  Flat index i over the 16-byte vectors of the rows (row i / (K/8));
// each thread has four vectors in flight per step (a grid stride apart, so a
// warp's loads stay contiguous).  WIDE: 64-bit indices for tensors of 2^31 or
// more vectors.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float absmax8(uint4 q) {
    return fmaxf(fmaxf(fmaxf(fabsf(bf16lo(q.x)), fabsf(bf16hi(q.x))), fmaxf(fabsf(bf16lo(q.y)), fabsf(bf16hi(q.y)))),
                 fmaxf(fmaxf(fabsf(bf16lo(q.z)), fabsf(bf16hi(q.z))), fmaxf(fabsf(bf16lo(q.w)), fabsf(bf16hi(q.w)))));
}

template <bool WIDE>
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* X, int M, int K, int ldx, float* out) {
    pdl_launch_dependents();
    using I = typename std::conditional<WIDE, unsigned long long, unsigned>::type;
    const I vpr = (I)(K / 8);
    const I total = (I)M * vpr;
    const I S = (I)gridDim.x * blockDim.x;
    float m = 0.0f;
    for (I i0 = (I)blockIdx.x * blockDim.x + threadIdx.x; i0 < total; i0 += 4 * S) {
        uint4 q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const I i = i0 + (I)u * S;
            q[u] = make_uint4(0, 0, 0, 0);
            if (i < total) {
                const I r = i / vpr;
                q[u] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)r * ldx) + (i - r * vpr));
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) m = fmaxf(m, absmax8(q[u]));
    }
    m = warp_max(m);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float v = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v = fmaxf(v, red[w]);
        atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(v));  // v >= 0: bit order = value order
    }
}

// The tensor amax of the rotated NVFP4 tensor (16-element blocks rotated by
// rotate_item, act: times 1/16): grid-stride over 16-element chunks.
__global__ void __launch_bounds__(256) amax_rot_kernel(const uint16_t* X, int M, int K, int ldx, int act, float* out) {
    pdl_launch_dependents();
    const int chunks = K / 16;
    const long long total = (long long)M * chunks;
    float m = 0.0f;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long r = i / chunks;
        const int c = (int)(i - r * chunks);
        const uint4* p = reinterpret_cast<const uint4*>(X + r * ldx) + 2 * c;
        const uint4 v0 = __ldg(p), v1 = __ldg(p + 1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float v[16];
        rotate_item<16>(w, v, c, act != 0);  // one item per block: no lane exchange
        m = fmaxf(m, absmax16(v));
    }
    m = warp_max(m);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float v = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v = fmaxf(v, red[w]);
        atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(v));
    }
}

// NVFP4 codes (w0: elements 0..7, w1: 8..15) and E4M3 scale of one 16-element
// block of second-stage residuals R with the row's scale s2: the same rule as
// the first stage (block scale E4M3(RN(RN(amax / 6) / s2)), codes E2M1 of the
// correctly rounded quotients), by IEEE division for the scale and by refined
// division for the codes wherever that is exact.
__device__ __forceinline__ uint8_t residual_block(const float* R, float s2, uint32_t& w0, uint32_t& w1) {
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(R[i]));
    const uint8_t sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), s2));
    w0 = 0;
    w1 = 0;
    if (sb != 0) {
        const float d = __fmul_rn(e4m3_value(sb), s2);
        const float y = __frcp_rn(d);
        const bool exact = !(d >= 0x1p-100f && d <= 0x1p100f && __fmul_rn(bmax, y) <= 0x1p60f);
        float q0[8], q1[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            q0[e] = exact ? __fdiv_rn(R[e], d) : div_refined(R[e], d, y);
            q1[e] = exact ? __fdiv_rn(R[8 + e], d) : div_refined(R[8 + e], d, y);
        }
        w0 = e2m1x8(q0);
        w1 = e2m1x8(q1);
    }
    return sb;
}

// ---------------------------------------------------------------------------
// Residual second stage: thread = (row, 16-block of the nS residual channels).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) residual_kernel(ResidualArgs a) {
    pdl_launch_dependents();
    const int nb = a.nS / 16;
    const long long idx = blockIdx.x * 128LL + threadIdx.x;
    if (idx >= (long long)a.rows_pad * nb) return;
    const int r = (int)(idx / nb);
    const int b = (int)(idx % nb);
    const int cblk = a.K / 16 + b;  // block index of the residual block in the augmented row
    uint8_t sb = 0;
    uint32_t w0 = 0, w1 = 0;
    if (r < a.M) {
        const float s2 = a.s2[a.mode == 1 ? r : 0];
        float R[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int k = checked_channel(a.S, 16 * b + i, a.K);
            const float x = __uint_as_float((uint32_t)a.X[(size_t)r * a.ldx + k] << 16);
            const uint8_t byte = a.codes[(size_t)r * a.ldc + (k >> 1)];
            const uint32_t code = (k & 1) ? (byte >> 4) : (byte & 15);
            const float mags[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
            const float ev = (code & 8u) ? -mags[code & 7] : mags[code & 7];
            const float sv = e4m3_value(a.sf[sf_offset(r, k >> 4, a.sf_col_atoms)]);
            const float xhat = __fmul_rn(__fmul_rn(ev, sv), s2);  // ev*sv is exact
            R[i] = __fsub_rn(x, xhat);
        }
        sb = residual_block(R, s2, w0, w1);
        *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + (a.K >> 1) + 8 * b) = make_uint2(w0, w1);
    }
    a.sf[sf_offset(r, cblk, a.sf_col_atoms)] = sb;
}

// ---------------------------------------------------------------------------
// Channel selection: column amax, rank (ties to the lower index), compaction.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) colmax_kernel(const uint16_t* X, int Mc, int K, int ldx, float* amax) {
    const int k = blockIdx.x * 256 + threadIdx.x;
    if (k >= K) return;
    float m = 0.0f;
    for (int r = blockIdx.y; r < Mc; r += gridDim.y)
        m = fmaxf(m, fabsf(__uint_as_float((uint32_t)X[(size_t)r * ldx + k] << 16)));
    atomicMax(reinterpret_cast<unsigned int*>(amax + k), __float_as_uint(m));
}

__global__ void __launch_bounds__(256) rank_kernel(const float* amax, int K, int nS, int* selected) {
    const int k = blockIdx.x * 256 + threadIdx.x;
    __shared__ float tile[256];
    const float mine = (k < K) ? amax[k] : 0.0f;
    int rank = 0;
    for (int base = 0; base < K; base += 256) {
        __syncthreads();
        tile[threadIdx.x] = (base + threadIdx.x < K) ? amax[base + threadIdx.x] : -1.0f;
        __syncthreads();
        const int lim = min(256, K - base);
        for (int i = 0; i < lim; ++i) {
            const float o = tile[i];
            rank += (o > mine) || (o == mine && base + i < k);
        }
    }
    if (k < K) selected[k] = rank < nS;
}

__global__ void __launch_bounds__(1024) compact_kernel(const int* selected, int K, int32_t* S) {
    // one CTA: each thread counts a contiguous slice, a block scan gives offsets
    __shared__ int counts[1024];
    const int t = threadIdx.x;
    const int per = (K + 1023) / 1024;
    const int k0 = min(K, t * per), k1 = min(K, k0 + per);
    int c = 0;
    for (int k = k0; k < k1; ++k) c += selected[k];
    counts[t] = c;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        int v = (t >= o) ? counts[t - o] : 0;
        __syncthreads();
        counts[t] += v;
        __syncthreads();
    }
    int pos = counts[t] - c;
    for (int k = k0; k < k1; ++k)
        if (selected[k]) S[pos++] = k;
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
// Second stage of one row in the per-token kernel (RES): residual channel e
// (e < res_n, in S order) of the row is R = x - x^, with x from the row
// buffer xs, and its first-stage code and block scale from cb / sbs
// (x^ = code value * block scale * s2).  Sixteen channels form a residual
// block; EPL consecutive channels per lane, so 16 / EPL lanes share a block:
// block maximum by lane exchange, block scale E4M3(RN(RN(max / 6) / s2)) and
// codes E2M1(RN(R / d)), the rule of residual_block.  The lane holding a
// block's first channel writes its 8 code bytes to crow + 8 * block and its
// scale at block column c0 + block.  Every lane of the CTA calls this (the
// loop bounds are CTA-uniform; T is a multiple of 32, res_n of 16).
template <int EPL>
__device__ __forceinline__ void residual_stage(const uint16_t* xs, const uint8_t* cb, const uint8_t* sbs,
                                               const int32_t* sS, int res_n, float s2, float rinv, bool fast,
                                               uint8_t* crow, uint8_t* sf, int r, int c0, int sf_col_atoms) {
    constexpr int LPB = 16 / EPL;  // lanes per residual block
    constexpr int LPW = 8 / EPL;   // lanes per 32-bit word of codes
    const int t = threadIdx.x, T = blockDim.x;
    for (int e0 = 0; e0 < res_n; e0 += EPL * T) {
        const int e = e0 + EPL * t;  // this lane's first channel
        const bool live = e < res_n;  // the same for the lanes of a block
        float R[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) R[j] = 0.0f;
        if (live) {
            int k[EPL];
            if constexpr (EPL == 4) {
                const int4 v = *reinterpret_cast<const int4*>(sS + e);
                k[0] = v.x; k[1] = v.y; k[2] = v.z; k[3] = v.w;
            } else if constexpr (EPL == 2) {
                const int2 v = *reinterpret_cast<const int2*>(sS + e);
                k[0] = v.x; k[1] = v.y;
            } else {
                k[0] = sS[e];
            }
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const float x = __uint_as_float((uint32_t)xs[k[j]] << 16);
                const uint32_t nib = (cb[k[j] >> 1] >> (4 * (k[j] & 1))) & 15u;
                // the first product is exact
                R[j] = __fsub_rn(x, __fmul_rn(__fmul_rn(e2m1_decode(nib), e4m3_value(sbs[k[j] >> 4])), s2));
            }
        }
        float bmax = fabsf(R[0]);
#pragma unroll
        for (int j = 1; j < EPL; ++j) bmax = fmaxf(bmax, fabsf(R[j]));
#pragma unroll
        for (int o = LPB / 2; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
        // block scale by refined divisions in the range where they are exact,
        // as for the first stage (R is finite for finite x, so bmax is too)
        uint8_t sbr;
        if (fast) {
            const float u0 = __fmul_rn(bmax, 0x1.555556p-3f);  // RN(1/6)
            const float u = __fmaf_rn(__fmaf_rn(-u0, 6.0f, bmax), 0x1.555556p-3f, u0);
            const float v0 = __fmul_rn(u, rinv);
            sbr = e4m3_rn_sat(__fmaf_rn(__fmaf_rn(-v0, s2, u), rinv, v0));
        } else {
            sbr = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), s2));
        }
        uint32_t h = 0;  // this lane's 4 * EPL bits of codes, channel e + j in nibble j
        if (sbr != 0) {
            const float d = __fmul_rn(e4m3_value(sbr), s2);
            const float y = __frcp_rn(d);
            const bool exact = !(d >= 0x1p-100f && d <= 0x1p100f && __fmul_rn(bmax, y) <= 0x1p60f);
            float q[EPL];
#pragma unroll
            for (int j = 0; j < EPL; ++j) q[j] = exact ? __fdiv_rn(R[j], d) : div_refined(R[j], d, y);
            if constexpr (EPL == 4) h = e2m1x2_byte(q[0], q[1]) | (e2m1x2_byte(q[2], q[3]) << 8);
            else if constexpr (EPL == 2) h = e2m1x2_byte(q[0], q[1]);
            else h = e2m1x2_byte(q[0], 0.0f) & 15u;
        }
        uint32_t word = h << (4 * EPL * (t % LPW));
#pragma unroll
        for (int o = LPW / 2; o > 0; o >>= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
        const uint32_t hi = __shfl_down_sync(0xffffffffu, word, LPW);
        if (live && t % LPB == 0) {
            *reinterpret_cast<uint2*>(crow + 8 * (e >> 4)) = make_uint2(word, hi);
            sf[sf_offset(r, c0 + (e >> 4), sf_col_atoms)] = sbr;
        }
    }
}

// ---------------------------------------------------------------------------
// NVFP4 with a dynamic per-token scale (the activation hot path), or with the
// dynamic tensor scale of an amax pass (TENSOR mode).  Persistent
// CTAs walk rows r = blockIdx.x, +gridDim.x, ...; thread 0 keeps the next
// NB-1 rows in flight as bulk copies into a ring of shared-memory row
// buffers, so each SM has its loads outstanding while it computes.  For the
// current row every thread takes J chunks of 16 elements (items t, t+T, ...)
// into registers and the CTA reduces the row amax: the only CTA barrier of a
// row (the per-warp maxima alternate between two buffers, so no barrier is
// needed before the next row rewrites them).  Each item is then quantized
// from registers: block scale by two refined divisions, codes by refined
// division with RN(1/d) of its own divisor d = E4M3(scale) * s2.  The refined
// division is exact here whenever
// s2 >= 2^-100 (the block quotients are then either below 2^-10, which
// encodes to zero either way, or normal and at most about 12); a row below
// that takes IEEE division throughout (a CTA-uniform branch).  Rows
// M .. rows_pad-1 write the zero scales of the 128-row atoms' padding.
// ---------------------------------------------------------------------------
// ROT: every 16-element block rotated first (rotate_item; a block is one
// item, so no lane exchange; a.rot 1 = activation side, 2 = weight side).
// TENSOR: one s2 for the whole tensor (see below) instead of one per row.
// RES: also the residual-channel second stage ("APEX4..." page, para 2:
// ARCQuant) of every row, written at columns K .. K + res_n.  Each thread
// keeps its blocks' codes and scales in shared memory as well; after a CTA
// barrier, residual channel e = S[e] of the row (still in its ring buffer,
// which is refilled only once the next row has started) gives
// R = x - x^ with x^ = code value * block scale * s2 (residual_stage: EPL
// channels per lane, 16 / EPL lanes per residual block; EPL = 0 is the
// kernel without the second stage).  S is cached per CTA; an index outside
// [0, K) is recorded in the error word and channel 0 taken.
template <int J, bool ROT, bool TENSOR, int EPL>
__global__ void __launch_bounds__(J <= 2 ? 1024 : 768) quant_nvfp4_token_kernel(QuantArgs a, int nb) {
    constexpr bool RES = EPL > 0;
    pdl_launch_dependents();
    pdl_wait();  // X and the words to clear may belong to the preceding launch
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < a.zero_count; i += blockDim.x) a.zero_words[i] = 0;
    extern __shared__ __align__(128) uint8_t qring[];
    __shared__ float wmax[2][32];  // per-warp row maxima, alternating rows
    const int t = threadIdx.x, T = blockDim.x;
    const int lane = t & 31, warp = t >> 5, nwarps = T >> 5;
    const int items = a.K / 16;
    const int row_bytes = a.K * 2;
    uint64_t* bars = reinterpret_cast<uint64_t*>(qring + (size_t)nb * row_bytes);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + nb);
    // RES: the residual channels S, and the current row's codes and block scales
    // (16-byte aligned: four channels are read at a time)
    int32_t* sS = reinterpret_cast<int32_t*>((reinterpret_cast<uintptr_t>(bars + nb + 2) + 15) & ~uintptr_t(15));
    uint2* scodes = reinterpret_cast<uint2*>(sS + (RES ? a.res_n : 0));
    uint8_t* sbs = reinterpret_cast<uint8_t*>(scodes + (RES ? items : 0));
    const int G = gridDim.x;
    // rows of this CTA that are loaded: blockIdx.x + i*G < M
    const int nlive = a.M > (int)blockIdx.x ? (a.M - 1 - (int)blockIdx.x) / G + 1 : 0;
    // TENSOR mode: one s2 from the amax pass that precedes this launch; every
    // block amax is at most that amax, so the quotients keep the ranges the
    // refined division needs, as with a row's own s2
    const float ts2 = TENSOR ? nvfp4_s2(*a.tensor_amax) : 1.0f;
    if (TENSOR && blockIdx.x == 0 && threadIdx.x == 0) a.s2_out[0] = ts2;
    auto issue = [&](int i) {
        const int b = i % nb, r = blockIdx.x + i * G;
        mbar_arrive_expect_tx(&bars[b], (uint32_t)row_bytes);
        bulk_load(qring + (size_t)b * row_bytes, a.X + (size_t)r * a.ldx, row_bytes, &bars[b]);
    };
    if (t == 0) {
        for (int b = 0; b < nb; ++b) mbar_init(&bars[b], 1);
        *abort_flag = 0;
        fence_mbar_init();
        for (int i = 0; i < nb && i < nlive; ++i) issue(i);
    }
    if constexpr (RES)
        for (int k = t; k < a.res_n; k += T) sS[k] = checked_channel(a.res_S, k, a.K);
    __syncthreads();
    for (int i = 0; i < nlive; ++i) {
        const int b = i % nb, r = blockIdx.x + i * G;
        if (!mbar_wait(&bars[b], (i / nb) & 1, 2000000000ull, abort_flag)) break;
        const uint4* xr = reinterpret_cast<const uint4*>(qring + (size_t)b * row_bytes);
        uint32_t w[J][8];
        float vr[ROT ? J : 1][16];  // ROT: the rotated values of each item
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int it = t + T * j;
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
            if (it < items) {
                v0 = xr[2 * it];
                v1 = xr[2 * it + 1];
            }
            w[j][0] = v0.x; w[j][1] = v0.y; w[j][2] = v0.z; w[j][3] = v0.w;
            w[j][4] = v1.x; w[j][5] = v1.y; w[j][6] = v1.z; w[j][7] = v1.w;
        }
        float bm[J], m = 0.0f;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            if constexpr (ROT) {
                rotate_item<16>(w[j], vr[j], 0, a.rot == 1);
                bm[j] = absmax16(vr[j]);
            } else {
                bm[j] = bmax16(w[j]);
            }
            m = fmaxf(m, bm[j]);
        }
        if constexpr (!TENSOR) {
            m = warp_max_nonneg(m);
            if (lane == 0) wmax[i & 1][warp] = m;
        }
        __syncthreads();  // (also: every thread has its row data in registers)
        // the buffer is free again: this row's (RES: the previous row's, whose
        // second stage read it until this barrier)
        if constexpr (RES) {
            if (t == 0 && i >= 1 && i - 1 + nb < nlive) issue(i - 1 + nb);
        } else {
            if (t == 0 && i + nb < nlive) issue(i + nb);
        }
        float s2 = ts2;
        if constexpr (!TENSOR) {
            s2 = nvfp4_s2(warp_max_nonneg(lane < nwarps ? wmax[i & 1][lane] : 0.0f));
            if (t == 0) a.s2_out[r] = s2;
        }
        const bool fast = s2 >= 0x1p-100f;  // the same for the whole CTA
        const float rinv = __frcp_rn(s2);
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int it = t + T * j;
            uint32_t sb, w0, w1;
            if (fast) {
                // RN(RN(bm / 6) / s2) by the refined division; both operands are
                // non-negative, so no sign fix-up is needed
                const float u0 = __fmul_rn(bm[j], 0x1.555556p-3f);  // RN(1/6)
                const float u = __fmaf_rn(__fmaf_rn(-u0, 6.0f, bm[j]), 0x1.555556p-3f, u0);
                const float v0 = __fmul_rn(u, rinv);
                sb = e4m3_rn_sat(__fmaf_rn(__fmaf_rn(-v0, s2, u), rinv, v0));
                const float d = sb ? __fmul_rn(e4m3_value((uint8_t)sb), s2) : 1.0f;
                const float y = __frcp_rn(d);
                if constexpr (ROT) {
                    w0 = e2m1x8_fast_f(vr[j], pack2(-y), pack2(d));
                    w1 = e2m1x8_fast_f(vr[j] + 8, pack2(-y), pack2(d));
                } else {
                    w0 = e2m1x8_fast(w[j], pack2(-y), pack2(d));
                    w1 = e2m1x8_fast(w[j] + 4, pack2(-y), pack2(d));
                }
            } else {
                sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bm[j], 6.0f), s2));
                const float d = sb ? __fmul_rn(e4m3_value((uint8_t)sb), s2) : 1.0f;
                if constexpr (ROT) {
                    w0 = e2m1x8_exact_f(vr[j], d);
                    w1 = e2m1x8_exact_f(vr[j] + 8, d);
                } else {
                    w0 = e2m1x8_exact(make_uint4(w[j][0], w[j][1], w[j][2], w[j][3]), d);
                    w1 = e2m1x8_exact(make_uint4(w[j][4], w[j][5], w[j][6], w[j][7]), d);
                }
            }
            if (sb == 0) {
                w0 = 0;
                w1 = 0;
            }
            if constexpr (RES) {
                if (it < items) {
                    scodes[it] = make_uint2(w0, w1);
                    sbs[it] = (uint8_t)sb;
                }
            }
            // one byte per scale: the warp's stores still fill whole 4-byte
            // groups (items l .. l+3 sit on consecutive lanes), without lane
            // exchanges to assemble them
            if (it < items) {
                a.sf[sf_offset(r, it, a.sf_col_atoms)] = (uint8_t)sb;
                *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + 8 * it) = make_uint2(w0, w1);
            }
        }
        if constexpr (RES) {
            // the second stage of this row (the next row rewrites the codes and
            // scales in shared memory only after its own barrier)
            __syncthreads();
            residual_stage<EPL>(reinterpret_cast<const uint16_t*>(xr), reinterpret_cast<const uint8_t*>(scodes),
                                sbs, sS, a.res_n, s2, rinv, fast, a.codes + (size_t)r * a.ldc + (a.K >> 1), a.sf, r,
                                a.K >> 4, a.sf_col_atoms);
        }
    }
    if (*abort_flag && t == 0)  // wait for the copies still in flight
        for (int b = 0; b < nb; ++b) mbar_wait_drain(&bars[b], 0, 100000000ull);
    // padding rows of the 128-row scale atoms: zero scales
    for (int r = a.M + (int)blockIdx.x; r < a.rows_pad; r += G)
        for (int c4 = t; c4 < items / 4; c4 += T)
            *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, 4 * c4, a.sf_col_atoms)) = 0u;
}

// NVFP4 TENSOR mode in one pass, for activations that fit in shared memory
// across the grid: one CTA per SM, launched cooperatively so that every CTA
// is resident.  Each CTA brings its rows r = blockIdx.x, +G, ... into shared
// memory and folds their amax into the tensor amax (atomicMax on s2[1]). It
// then counts itself in on s2[2] and waits, bounded, until every CTA has.
// Last it quantizes its rows from shared memory with s2 = amax/2688.  The
// codes, block scales and s2 are those of the amax pass followed by
// quant_nvfp4_token_kernel<TENSOR>: the same block maxima, refined divisions
// and E2M1 conversions.  s2[1] and s2[2] are zero at launch.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__global__ void __launch_bounds__(1024) quant_nvfp4_tensor_onepass_kernel(QuantArgs a, unsigned* arrive) {
    pdl_launch_dependents();
    pdl_wait();  // X and the words to clear may belong to the preceding launch
    const int t = threadIdx.x, T = blockDim.x, lane = t & 31, warp = t >> 5, nwarps = T >> 5;
    if (blockIdx.x == 0)
        for (int i = t; i < a.zero_count; i += T) a.zero_words[i] = 0;
    extern __shared__ __align__(128) uint8_t rows[];
    __shared__ uint64_t bar;
    __shared__ float red[32];
    __shared__ float s2_sh;
    __shared__ int abort_sh;
    volatile int* abort_flag = &abort_sh;
    const int G = gridDim.x;
    const int items = a.K / 16, row_bytes = a.K * 2;
    const int nlive = a.M > (int)blockIdx.x ? (a.M - 1 - (int)blockIdx.x) / G + 1 : 0;
    if (t == 0) {
        mbar_init(&bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (nlive > 0) {
            mbar_arrive_expect_tx(&bar, (uint32_t)(nlive * row_bytes));
            for (int i = 0; i < nlive; ++i)
                bulk_load(rows + (size_t)i * row_bytes, a.X + (size_t)(blockIdx.x + i * G) * a.ldx, row_bytes, &bar);
        }
    }
    __syncthreads();
    if (nlive > 0) mbar_wait(&bar, 0, 2000000000ull, abort_flag);
    // the CTA's amax (block maxima as in the token kernel; NaN ignored)
    const int total = nlive * items;
    // item f = t + k T of the CTA's rows is (row i, item it); both advance by
    // (T / items, T % items) per step, so no division inside the loops
    const int di = T / items, dit = T - di * items, i0 = t / items, it0 = t - i0 * items;
    float m = 0.0f;
    if (!*abort_flag)
        for (int f = t, i = i0, it = it0; f < total; f += T) {
            const uint4* p = reinterpret_cast<const uint4*>(rows + (size_t)i * row_bytes) + 2 * it;
            const uint4 v0 = p[0], v1 = p[1];
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            m = fmaxf(m, bmax16(w));
            i += di;
            it += dit;
            if (it >= items) {
                it -= items;
                ++i;
            }
        }
    m = warp_max_nonneg(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (t == 0) {
        float v = 0.0f;
        for (int k = 0; k < nwarps; ++k) v = fmaxf(v, red[k]);
        unsigned* amax = reinterpret_cast<unsigned*>(const_cast<float*>(a.tensor_amax));
        atomicMax(amax, __float_as_uint(v));  // v >= 0: bit order = value order
        __threadfence();                      // the maximum is visible before the count
        atomicAdd(arrive, 1u);
        // every CTA is resident (cooperative launch): wait for all, bounded
        const uint64_t t0 = globaltimer();
        while (ld_acquire_u32(arrive) < (unsigned)G) {
            if (globaltimer() - t0 > 2000000000ull) {
                report_error(kErrTimeout);
                *abort_flag = 1;
                break;
            }
            __nanosleep(100);
        }
        s2_sh = nvfp4_s2(__uint_as_float(ld_acquire_u32(amax)));
        if (blockIdx.x == 0 && !*abort_flag) a.s2_out[0] = s2_sh;
    }
    __syncthreads();
    if (*abort_flag) {  // (the outputs are undefined; the error word says so)
        if (t == 0 && nlive > 0) mbar_wait_drain(&bar, 0, 100000000ull);  // copies still in flight
        return;
    }
    const float s2 = s2_sh;
    const float rinv = __frcp_rn(s2);
    const bool fast = s2 >= 0x1p-100f;  // the same for the whole grid
    const int iters = (total + T - 1) / T;
    for (int k = 0, fi = i0, fit = it0; k < iters; ++k) {
        const int f = t + k * T;
        const bool valid = f < total;
        const int i = valid ? fi : 0, it = valid ? fit : 0;
        fi += di;
        fit += dit;
        if (fit >= items) {
            fit -= items;
            ++fi;
        }
        const int r = (int)blockIdx.x + i * G;
        uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (valid) {
            const uint4* p = reinterpret_cast<const uint4*>(rows + (size_t)i * row_bytes) + 2 * it;
            const uint4 v0 = p[0], v1 = p[1];
            w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
            w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
        }
        const float bm = bmax16(w);
        uint32_t sb, w0, w1;
        if (fast) {
            const float u = div_refined(bm, 6.0f, 0x1.555556p-3f);  // RN(1/6)
            sb = e4m3_rn_sat(div_refined(u, s2, rinv));
            const float d = sb ? __fmul_rn(e4m3_value((uint8_t)sb), s2) : 1.0f;
            const float y = __frcp_rn(d);
            w0 = e2m1x8_fast(w, pack2(-y), pack2(d));
            w1 = e2m1x8_fast(w + 4, pack2(-y), pack2(d));
        } else {
            sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bm, 6.0f), s2));
            const float d = sb ? __fmul_rn(e4m3_value((uint8_t)sb), s2) : 1.0f;
            w0 = e2m1x8_exact(make_uint4(w[0], w[1], w[2], w[3]), d);
            w1 = e2m1x8_exact(make_uint4(w[4], w[5], w[6], w[7]), d);
        }
        if (sb == 0) {
            w0 = 0;
            w1 = 0;
        }
        if (valid) {  // one byte per scale (as in the per-token kernel)
            a.sf[sf_offset(r, it, a.sf_col_atoms)] = (uint8_t)sb;
            *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + 8 * it) = make_uint2(w0, w1);
        }
    }
    // padding rows of the 128-row scale atoms: zero scales
    for (int r = a.M + (int)blockIdx.x; r < a.rows_pad; r += G)
        for (int c4 = t; c4 < items / 4; c4 += T)
            *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, 4 * c4, a.sf_col_atoms)) = 0u;
}

// Shared memory the one-pass kernel may hold per CTA.
constexpr size_t kOnepassSmem = 200 * 1024;

bool nvfp4_tensor_onepass_fits(int M, int K, int num_sms) {
    if (M <= 0 || num_sms <= 0) return false;
    const size_t rows = (size_t)((M + num_sms - 1) / num_sms);
    return rows * (size_t)K * 2 <= kOnepassSmem;
}

cudaError_t launch_nvfp4_tensor_onepass(const QuantArgs& a, int rows_pad, int num_sms, unsigned* arrive, bool pdl,
                                        cudaStream_t st) {
    static SmemAttrCache smem_attr;
    const void* kern = reinterpret_cast<const void*>(quant_nvfp4_tensor_onepass_kernel);
    cudaError_t e = ensure_dynamic_smem(kern, kOnepassSmem, smem_attr);
    if (e != cudaSuccess) return e;
    QuantArgs b = a;
    b.rows_pad = rows_pad;
    const size_t smem = (size_t)((a.M + num_sms - 1) / num_sms) * (size_t)a.K * 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(1024);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    // cooperative (every CTA resident: the grid-wide amax wait), and with pdl
    // a programmatic dependent of the preceding launch where the runtime
    // allows both; the kernel waits for that launch before touching memory
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    static std::atomic<int> pdl_refused{0};
    if (pdl && !pdl_refused.load(std::memory_order_relaxed)) {
        e = cudaLaunchKernelEx(&cfg, quant_nvfp4_tensor_onepass_kernel, b, arrive);
        if (e == cudaSuccess || e == cudaErrorCooperativeLaunchTooLarge) return e;
        cudaGetLastError();  // the combination refused: plain cooperative launches from now on
        pdl_refused.store(1, std::memory_order_relaxed);
    }
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quant_nvfp4_tensor_onepass_kernel, b, arrive);
}

// Launch as a programmatic dependent of the preceding launch (the kernels wait
// for it before touching memory it may write).
template <typename... Args>
static cudaError_t launch_dep(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int J, bool ROT, int EPL>
static const void* tok_kernel_e(bool tensor) {
    return tensor ? reinterpret_cast<const void*>(quant_nvfp4_token_kernel<J, ROT, true, EPL>)
                  : reinterpret_cast<const void*>(quant_nvfp4_token_kernel<J, ROT, false, EPL>);
}
template <int J, bool ROT>
static const void* tok_kernel(bool tensor, int epl) {
    if constexpr (!ROT) {
        if (epl == 4) return tok_kernel_e<J, false, 4>(tensor);
        if (epl == 2) return tok_kernel_e<J, false, 2>(tensor);
        if (epl == 1) return tok_kernel_e<J, false, 1>(tensor);
    }
    return tok_kernel_e<J, ROT, 0>(tensor);
}

template <int J, bool ROT, bool TENSOR, int EPL>
static cudaError_t launch_tok_mode(const QuantArgs& b, int grid, int T, size_t smem, int nb, cudaStream_t st) {
    static SmemAttrCache smem_attr;
    auto kern = quant_nvfp4_token_kernel<J, ROT, TENSOR, EPL>;
    const cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem, smem_attr);
    if (e != cudaSuccess) return e;
    return launch_dep(kern, dim3(grid), dim3(T), smem, st, b, nb);
}
template <int J, bool ROT, int EPL>
static cudaError_t launch_tok_e(const QuantArgs& b, int grid, int T, size_t smem, int nb, cudaStream_t st) {
    return b.mode == 0 ? launch_tok_mode<J, ROT, true, EPL>(b, grid, T, smem, nb, st)
                       : launch_tok_mode<J, ROT, false, EPL>(b, grid, T, smem, nb, st);
}
template <int J, bool ROT>
static cudaError_t launch_tok(const QuantArgs& b, int epl, int grid, int T, size_t smem, int nb, cudaStream_t st) {
    if constexpr (!ROT) {
        if (epl == 4) return launch_tok_e<J, false, 4>(b, grid, T, smem, nb, st);
        if (epl == 2) return launch_tok_e<J, false, 2>(b, grid, T, smem, nb, st);
        if (epl == 1) return launch_tok_e<J, false, 1>(b, grid, T, smem, nb, st);
    }
    return launch_tok_e<J, ROT, 0>(b, grid, T, smem, nb, st);
}

bool nvfp4_token_fuses_residual(int K, int res_n) {
    return res_n > 0 && res_n % 16 == 0 && res_n <= 1024 && K / 16 <= 2048;
}

static cudaError_t launch_nvfp4_token(const QuantArgs& a, int rows_pad, int num_sms, cudaStream_t st) {
    // J items (32 J bytes of the row) per thread: two, so that the resident
    // CTAs bring enough warps to hide the per-item latency (at most 1024
    // threads; four for the longest rows)
    const int items = a.K / 16;
    const int J = items < 64 ? 1 : items <= 2048 ? 2 : 4;
    int T = (items + J - 1) / J;
    T = (T + 31) / 32 * 32;
    // resident CTAs per SM from the kernel's registers (allocated per warp in
    // units of 256) and from a ring of at least three row buffers each (two
    // rows in flight while one is computed), within about 200 KB of shared
    // memory per SM
    const int row_bytes = a.K * 2;
    const bool tensor = a.mode == 0;
    const bool res = a.res_n > 0;
    if (res && (a.rot || !nvfp4_token_fuses_residual(a.K, a.res_n))) return cudaErrorInvalidValue;
    // second stage: four residual channels per lane where every thread has at
    // least four, else fewer, so that more warps share a short stage
    const int epl = !res ? 0 : 4 * T <= a.res_n ? 4 : 2 * T <= a.res_n ? 2 : 1;
    const void* kern = J == 1 ? (a.rot ? tok_kernel<1, true>(tensor, 0) : tok_kernel<1, false>(tensor, epl))
                     : J == 2 ? (a.rot ? tok_kernel<2, true>(tensor, 0) : tok_kernel<2, false>(tensor, epl))
                              : tok_kernel<4, false>(tensor, epl);
    // [J 1/2/4][rot][tensor][res]: registers per thread
    static std::atomic<int> regs_seen[3][2][2][4];  // [J][rot][tensor][EPL 0, 1, 2, 4]
    std::atomic<int>& rs = regs_seen[J == 1 ? 0 : J == 2 ? 1 : 2][a.rot ? 1 : 0][tensor ? 1 : 0][epl == 4 ? 3 : epl];
    int regs = rs.load(std::memory_order_relaxed);
    if (!regs) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs <= 0) return cudaErrorInvalidValue;
        regs = fa.numRegs;
        rs.store(regs, std::memory_order_relaxed);
    }
    const int warp_regs = (regs * 32 + 255) / 256 * 256;
    int per_sm = 65536 / ((T / 32) * warp_regs);
    // the residual stage's shared arrays: S, and one row's codes and block scales
    const int res_bytes = res ? (4 * a.res_n + 9 * items + 15) / 16 * 16 + 16 : 0;  // + alignment of S
    const int by_smem = (200 * 1024) / (3 * row_bytes + res_bytes);
    per_sm = per_sm < by_smem ? per_sm : by_smem;
    per_sm = per_sm < 1 ? 1 : (per_sm > 16 ? 16 : per_sm);
    int nb = ((200 * 1024) / per_sm - res_bytes) / row_bytes;
    nb = nb < 2 ? 2 : (nb > 8 ? 8 : nb);
    const size_t smem = (size_t)nb * row_bytes + 8 * nb + 16 + res_bytes;
    if (smem > 220 * 1024) return cudaErrorInvalidValue;
    int grid = num_sms * per_sm;
    if (grid > rows_pad) grid = rows_pad;
    // a few tokens (decode): as many CTAs as rows (they also write the zero
    // scales of the padding rows), so that the few SMs they take are all the
    // next launch has to wait for before it can start streaming its weights
    if (a.M <= 16 && grid > (a.M > 4 ? a.M : 4)) grid = a.M > 4 ? a.M : 4;
    QuantArgs b = a;
    b.rows_pad = rows_pad;
    cudaError_t e;
    if (J == 1)
        e = a.rot ? launch_tok<1, true>(b, 0, grid, T, smem, nb, st) : launch_tok<1, false>(b, epl, grid, T, smem, nb, st);
    else if (J == 2)
        e = a.rot ? launch_tok<2, true>(b, 0, grid, T, smem, nb, st) : launch_tok<2, false>(b, epl, grid, T, smem, nb, st);
    else
        e = launch_tok<4, false>(b, epl, grid, T, smem, nb, st);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <int FMT, bool GATHER, bool MULTI = false, bool ROT = false>
static cudaError_t launch_quant_fmt(const QuantArgs& a, int rows_pad, int num_sms, cudaStream_t st) {
    const int row_bytes = a.K_src * 2;
    // One row block per CTA (about 32 KB of rows, several CTAs resident per
    // SM): many warps in flight hide the latency of the per-item arithmetic.
    int rpc = 32768 / row_bytes;
    rpc = rpc < 1 ? 1 : (rpc > 64 ? 64 : rpc);
    const size_t buf = (size_t)rpc * row_bytes;
    const int nbuf = 1;
    const size_t smem = nbuf * buf + 8 * nbuf + 4 * rpc + sizeof(RowConsts) * rpc +
                        (FMT == FMT_NVFP4 ? 4 * (size_t)rpc * (a.K / 16) : 0) + 16;
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    auto kern = quant_rows_kernel<FMT, GATHER, MULTI, ROT>;
    static SmemAttrCache smem_attr;
    const cudaError_t e0 = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem, smem_attr);
    if (e0 != cudaSuccess) return e0;
    const int items = rpc * (a.K / 16);
    const int T = items < 256 ? (items + 31) / 32 * 32 : 256;
    const int nblocks = (rows_pad + rpc - 1) / rpc;
    int grid = nblocks;
    // a few tokens (decode): few CTAs, which also write the padding rows' zero
    // scales (the kernel walks row blocks blockIdx.x, +gridDim.x, ...)
    if (a.M <= 16) {
        const int live = (a.M + rpc - 1) / rpc;
        const int want = live > 4 ? live : 4;
        if (grid > want) grid = want;
    }
    (void)num_sms;
    QuantArgs b = a;
    b.rows_pad = rows_pad;
    return launch_dep(kern, dim3(grid), dim3(T), smem, st, b, rpc, nbuf);
}

cudaError_t launch_quant(int fmt, bool gather, const QuantArgs& a, int rows_pad, int num_sms, cudaStream_t st) {
    if (a.rot) {  // block-local rotation (no gather, one pass)
        if (gather || a.passes > 1) return cudaErrorInvalidValue;
        if (fmt == FMT_NVFP4 && (a.mode == 1 || a.tensor_amax) && !a.static_s2 && a.K == a.K_src && a.K <= 32768 &&
            !a.int8_codes)
            return launch_nvfp4_token(a, rows_pad, num_sms, st);
        if (fmt == FMT_NVFP4) return launch_quant_fmt<FMT_NVFP4, false, false, true>(a, rows_pad, num_sms, st);
        if (fmt == FMT_MXFP4) return launch_quant_fmt<FMT_MXFP4, false, false, true>(a, rows_pad, num_sms, st);
        return launch_quant_fmt<FMT_INT4, false, false, true>(a, rows_pad, num_sms, st);
    }
    if (fmt == FMT_NVFP4 && !gather && (a.mode == 1 || a.tensor_amax) && !a.static_s2 && a.K == a.K_src &&
        a.K <= 49152)
        return launch_nvfp4_token(a, rows_pad, num_sms, st);
    if (fmt == FMT_NVFP4) return gather ? launch_quant_fmt<FMT_NVFP4, true>(a, rows_pad, num_sms, st)
                                        : launch_quant_fmt<FMT_NVFP4, false>(a, rows_pad, num_sms, st);
    if (fmt == FMT_MXFP4 && a.passes > 1)
        return gather ? cudaErrorInvalidValue : launch_quant_fmt<FMT_MXFP4, false, true>(a, rows_pad, num_sms, st);
    if (fmt == FMT_MXFP4) return gather ? launch_quant_fmt<FMT_MXFP4, true>(a, rows_pad, num_sms, st)
                                        : launch_quant_fmt<FMT_MXFP4, false>(a, rows_pad, num_sms, st);
    return gather ? launch_quant_fmt<FMT_INT4, true>(a, rows_pad, num_sms, st)
                  : launch_quant_fmt<FMT_INT4, false>(a, rows_pad, num_sms, st);
}

cudaError_t launch_amax(const uint16_t* X, int M, int K, int ldx, float* out, int num_sms, cudaStream_t st, int rot) {
    long long vecs = (long long)M * (K / 8);
    long long blocks = (vecs + 255) / 256;
    int grid = (int)(blocks < (long long)num_sms * 8 ? blocks : (long long)num_sms * 8);
    if (grid < 1) grid = 1;
    if (rot) amax_rot_kernel<<<grid, 256, 0, st>>>(X, M, K, ldx, rot == 1, out);
    else if ((long long)M * (K / 8) < (1LL << 31)) amax_kernel<false><<<grid, 256, 0, st>>>(X, M, K, ldx, out);
    else amax_kernel<true><<<grid, 256, 0, st>>>(X, M, K, ldx, out);
    return cudaGetLastError();
}

// Zeroes the tensor amax and the one-pass arrival count of an NVFP4 TENSOR
// activation (p[0], p[1]: s2[1], s2[2]), as a programmatic dependent of the
// preceding launch, so that the quantizer after it can be one too.
__global__ void clear_tensor_amax_kernel(float* p) {
    pdl_launch_dependents();
    pdl_wait();  // the preceding launch may still read these words
    if (threadIdx.x < 2) p[threadIdx.x] = 0.0f;
}

// p[1 .. n) = p[0]: spreads a segment's tensor scale over its rows.
__global__ void spread_first_kernel(float* p, int n) {
    const float v = p[0];
    for (int i = 1 + blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}

cudaError_t launch_clear_tensor_amax(float* p, cudaStream_t st) {
    const cudaError_t e = launch_dep(clear_tensor_amax_kernel, dim3(1), dim3(32), 0, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_spread_first(float* p, int n, cudaStream_t st) {
    if (n <= 1) return cudaSuccess;
    const int grid = (n + 255) / 256 < 64 ? (n + 255) / 256 : 64;
    spread_first_kernel<<<grid, 256, 0, st>>>(p, n);
    return cudaGetLastError();
}

cudaError_t launch_residual(const ResidualArgs& a, cudaStream_t st) {
    long long n = (long long)a.rows_pad * (a.nS / 16);
    residual_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_select(const uint16_t* X, int Mc, int K, int ldx, int nS, int32_t* S, float* amax, int* sel,
                          cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * K, st);
    if (e != cudaSuccess) return e;
    dim3 g1((K + 255) / 256, Mc < 64 ? (Mc > 0 ? Mc : 1) : 64);
    colmax_kernel<<<g1, 256, 0, st>>>(X, Mc, K, ldx, amax);
    rank_kernel<<<(K + 255) / 256, 256, 0, st>>>(amax, K, nS, sel);
    compact_kernel<<<1, 1024, 0, st>>>(sel, K, S);
    return cudaGetLastError();
}

}  // namespace w4a4
