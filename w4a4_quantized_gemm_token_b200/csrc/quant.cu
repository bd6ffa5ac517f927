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
#include <cuda_fp8.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

__constant__ float kE2M1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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

// Bracketing multipliers for a divisor d: with r = RN(1/d),
// rlo = RN(r * (1 - 2^-21)) and rhi = RN(r * (1 + 2^-21)) satisfy, for every x
// whose quotient is a normal float, |x*rlo| < |RN(x/d)| < |x*rhi| (the three
// roundings contribute at most 3 * 2^-24 relative error, less than 2^-21).
// Any function of the quotient that is monotone in its magnitude (E2M1
// conversion, rint) therefore gives RN(x/d)'s result whenever it gives the
// same result at both brackets; otherwise the exact division decides.
// Quotients below the normal range convert to zero at both brackets.
struct Bracket {
    float lo, hi;
    bool ok;  // false: 1/d is not finite, always divide
};
__device__ __forceinline__ Bracket make_bracket(float d) {
    const float r = __frcp_rn(d);
    Bracket b;
    b.lo = __fmul_rn(r, 1.0f - 0x1p-21f);
    b.hi = __fmul_rn(r, 1.0f + 0x1p-21f);
    b.ok = fabsf(r) <= 3.0e38f;
    return b;
}

// E2M1 codes of x[i] / d for 8 values, bit-exact with the correctly rounded quotient.
__device__ __forceinline__ uint32_t e2m1x8_div(const float* x, float d, const Bracket& br) {
    if (br.ok) {
        float lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lo[i] = __fmul_rn(x[i], br.lo);
            hi[i] = __fmul_rn(x[i], br.hi);
        }
        const uint32_t clo = e2m1x8(lo), chi = e2m1x8(hi);
        if (clo == chi) return clo;
    }
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(x[i], d);
    return e2m1x8(q);
}

// 4-bit two's-complement codes of clamp(rint(x[i] / s), -8, 7) for 8 values,
// bit-exact with the correctly rounded quotient (same bracketing).
__device__ __forceinline__ uint32_t int4x8_div(const float* x, float s, const Bracket& br) {
    int q[8];
    bool same = br.ok;
    if (br.ok) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int a = __float2int_rn(__fmul_rn(x[i], br.lo));
            const int b = __float2int_rn(__fmul_rn(x[i], br.hi));
            q[i] = a;
            same &= (a == b);
        }
    }
    if (!same) {
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __float2int_rn(__fdiv_rn(x[i], s));
    }
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) w |= (uint32_t)(min(max(q[i], -8), 7) & 15) << (4 * i);
    return w;
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

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
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
template <int FMT, bool GATHER>
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantArgs a, int rows_per_cta) {
    pdl_launch_dependents();
    extern __shared__ __align__(16) uint8_t qsm[];
    const int row_bytes = a.K_src * 2;                        // bf16 source row in shared memory
    uint64_t* bar = reinterpret_cast<uint64_t*>(qsm + (size_t)rows_per_cta * row_bytes);
    float* rmax = reinterpret_cast<float*>(bar + 1);          // [rows_per_cta] per-token amax
    volatile int* abort_flag = reinterpret_cast<volatile int*>(rmax + rows_per_cta);
    const int t = threadIdx.x, T = blockDim.x;
    const int r0 = blockIdx.x * rows_per_cta;
    const int nrows = min(rows_per_cta, a.rows_pad - r0);
    const int nlive = max(0, min(nrows, a.M - r0));
    const int nchunk = a.K / 16;

    if (t == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (t < rows_per_cta) rmax[t] = 0.0f;
    __syncthreads();
    if (t == 0 && nlive > 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(nlive * row_bytes));
        for (int i = 0; i < nlive; ++i)
            bulk_load(qsm + (size_t)i * row_bytes, a.X + (size_t)(r0 + i) * a.ldx, row_bytes, bar);
    }
    bool ok = true;
    if (nlive > 0) ok = mbar_wait(bar, 0, 2000000000ull, abort_flag);
    if (!ok) {
        if (t == 0) mbar_wait(bar, 0, 100000000ull, abort_flag);  // drain (abort already set: returns)
        return;
    }

    const bool token = FMT == FMT_NVFP4 && a.mode == 1 && !a.static_s2;
    const int items = nrows * nchunk;
    if (token) {
        for (int it = t; it < items; it += T) {
            const int i = it / nchunk, c = it - i * nchunk;
            if (i >= nlive) break;
            const uint4* p = reinterpret_cast<const uint4*>(qsm + (size_t)i * row_bytes) + 2 * c;
            // the augmented weight columns never take this path (weights use TENSOR)
            const uint4 v0 = p[0], v1 = p[1];
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float m = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[e])), fabsf(bf16hi(w[e]))));
            atomicMax(reinterpret_cast<unsigned int*>(rmax + i), __float_as_uint(m));  // m >= 0
        }
        __syncthreads();
    }
    float tensor_s2 = 1.0f;
    if constexpr (FMT == FMT_NVFP4) {
        if (a.mode == 0) tensor_s2 = a.static_s2 ? a.static_s2[0] : nvfp4_s2(*a.tensor_amax);
        if (a.mode == 0 && blockIdx.x == 0 && t == 0 && a.s2_out) a.s2_out[0] = tensor_s2;
        if (a.mode == 1 && t < nlive) a.s2_out[r0 + t] = a.static_s2 ? a.static_s2[r0 + t] : nvfp4_s2(rmax[t]);
    }

    const int iters = (items + T - 1) / T;
    for (int j = 0; j < iters; ++j) {
        const int it = t + T * j;
        const bool valid = it < items;           // uniform per group of 8 lanes
        const int i = valid ? it / nchunk : 0;
        const int c = valid ? it - i * nchunk : 0;
        const int r = r0 + i;
        const bool live = valid && i < nlive;
        float x[16];
        if (live) {
            const uint8_t* row = qsm + (size_t)i * row_bytes;
            if (!GATHER || 16 * c + 16 <= a.K_src) {
                const uint4* p = reinterpret_cast<const uint4*>(row) + 2 * c;
                const uint4 v0 = p[0], v1 = p[1];
                const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[2 * e] = bf16lo(w[e]);
                    x[2 * e + 1] = bf16hi(w[e]);
                }
            } else {
                // augmented weight columns: element k >= K_src is column S[k - K_src]
                const uint16_t* rw = reinterpret_cast<const uint16_t*>(row);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    x[e] = __uint_as_float((uint32_t)rw[checked_channel(a.S, 16 * c + e - a.K_src, a.K_src)] << 16);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = 0.0f;
        }
        float bmax = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) bmax = fmaxf(bmax, fabsf(x[e]));

        uint32_t w0 = 0, w1 = 0;  // 16 codes
        if constexpr (FMT == FMT_NVFP4) {
            uint8_t sb = 0;
            if (live) {
                const float s2 = a.mode == 1 ? (a.static_s2 ? a.static_s2[r] : nvfp4_s2(rmax[i])) : tensor_s2;
                sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), s2));
                if (sb != 0) {
                    const float d = __fmul_rn(e4m3_value(sb), s2);
                    const Bracket br = make_bracket(d);
                    w0 = e2m1x8_div(x, d, br);
                    w1 = e2m1x8_div(x + 8, d, br);
                }
            }
            // gather 4 consecutive block scales (lanes l..l+3) into one word
            const uint32_t b = sb;
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
                const uint32_t u = __float_as_uint(bmax);
                const int E = (int)(u >> 23);
                const int e = (E != 0) ? E - 127 : (31 - __clz((int)(u & 0x7FFFFF))) - 149;
                code = (uint32_t)min(max(e + 125, 0), 254);
                const float inv = __uint_as_float((254u - code) << 23);  // 2^(127 - code)
                float q0[8], q1[8];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) {
                    q0[e2] = __fmul_rn(x[e2], inv);
                    q1[e2] = __fmul_rn(x[8 + e2], inv);
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
        } else {  // INT4, 128-element group = 8 items
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 4));
            const float sc = live ? __fdiv_rn(bmax, 7.0f) : 0.0f;
            if (sc != 0.0f) {
                const Bracket br = make_bracket(sc);
                w0 = int4x8_div(x, sc, br);
                w1 = int4x8_div(x + 8, sc, br);
            }
            if (valid && (c & 7) == 0) a.sfi[(size_t)(c >> 3) * a.sfi_ld + r] = sc;
        }
        if (live) *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + 8 * c) = make_uint2(w0, w1);
    }
}

// ---------------------------------------------------------------------------
// Tensor amax: max |x| over X[M, K] into *out (as float bits; *out must start
// at 0).  Grid-stride over 16-byte vectors of each row.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* X, int M, int K, int ldx, float* out) {
    pdl_launch_dependents();
    const int vec_per_row = K / 8;
    const long long total = (long long)M * vec_per_row;
    float m = 0.0f;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long r = i / vec_per_row;
        const int v = (int)(i - r * vec_per_row);
        uint4 q = __ldg(reinterpret_cast<const uint4*>(X + r * ldx) + v);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(q.x)), fabsf(bf16hi(q.x))), fmaxf(fabsf(bf16lo(q.y)), fabsf(bf16hi(q.y)))));
        m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(q.z)), fabsf(bf16hi(q.z))), fmaxf(fabsf(bf16lo(q.w)), fabsf(bf16hi(q.w)))));
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
        float bmax = 0.0f;
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
            bmax = fmaxf(bmax, fabsf(R[i]));
        }
        sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), s2));
        if (sb != 0) {
            const float d = __fmul_rn(e4m3_value(sb), s2);
            const Bracket br = make_bracket(d);
            w0 = e2m1x8_div(R, d, br);
            w1 = e2m1x8_div(R + 8, d, br);
        }
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
template <int FMT, bool GATHER>
static cudaError_t launch_quant_fmt(const QuantArgs& a, int rows_pad, cudaStream_t st) {
    const int row_bytes = a.K_src * 2;
    int rpc = 32768 / row_bytes;                 // about 32 KB of rows per CTA
    rpc = rpc < 1 ? 1 : (rpc > 64 ? 64 : rpc);
    const size_t smem = (size_t)rpc * row_bytes + 16 + 4 * rpc + 16;
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    auto kern = quant_rows_kernel<FMT, GATHER>;
    static size_t attr = 0;
    if (smem > 48 * 1024 && smem > attr) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = smem;
    }
    const int items = rpc * (a.K / 16);
    int T = items < 256 ? (items + 31) / 32 * 32 : 256;
    QuantArgs b = a;
    b.rows_pad = rows_pad;
    kern<<<(rows_pad + rpc - 1) / rpc, T, smem, st>>>(b, rpc);
    return cudaGetLastError();
}

cudaError_t launch_quant(int fmt, bool gather, const QuantArgs& a, int rows_pad, cudaStream_t st) {
    if (fmt == FMT_NVFP4) return gather ? launch_quant_fmt<FMT_NVFP4, true>(a, rows_pad, st)
                                        : launch_quant_fmt<FMT_NVFP4, false>(a, rows_pad, st);
    if (fmt == FMT_MXFP4) return gather ? launch_quant_fmt<FMT_MXFP4, true>(a, rows_pad, st)
                                        : launch_quant_fmt<FMT_MXFP4, false>(a, rows_pad, st);
    return gather ? launch_quant_fmt<FMT_INT4, true>(a, rows_pad, st) : launch_quant_fmt<FMT_INT4, false>(a, rows_pad, st);
}

cudaError_t launch_amax(const uint16_t* X, int M, int K, int ldx, float* out, int num_sms, cudaStream_t st) {
    long long vecs = (long long)M * (K / 8);
    long long blocks = (vecs + 255) / 256;
    int grid = (int)(blocks < (long long)num_sms * 8 ? blocks : (long long)num_sms * 8);
    if (grid < 1) grid = 1;
    amax_kernel<<<grid, 256, 0, st>>>(X, M, K, ldx, out);
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
