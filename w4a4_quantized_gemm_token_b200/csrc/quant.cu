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

// E2M1 codes of 8 floats packed into one word, element i in nibble i; the sign
// bit of each nibble is the sign bit of its input (so a negative value that
// rounds to zero encodes as 0x8), independent of how cvt treats -0.
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
    uint32_t sgn = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) sgn |= (__float_as_uint(v[i]) >> 31) << (4 * i + 3);
    return out | sgn;
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
// Quantize rows.  Grid: one CTA per row r in [0, rows_pad); rows >= M only
// write zero scales (padding of the 128-row scale atoms).
// ---------------------------------------------------------------------------
template <int FMT, int J, bool GATHER>
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantArgs a) {
    pdl_launch_dependents();
    const int r = blockIdx.x;
    const int T = blockDim.x;
    const int t = threadIdx.x;
    const int nchunk = a.K / 16;           // chunks of the quantized columns
    const bool live = r < a.M;
    const int lane = t & 31;

    uint32_t raw[J][8];
    float amax_thread = 0.0f;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = t + T * j;
        if (live && c < nchunk) {
            if (!GATHER || 16 * c + 16 <= a.K_src) {
                const uint4* p = reinterpret_cast<const uint4*>(a.X + (size_t)r * a.ldx + 16 * c);
                uint4 v0 = __ldg(p), v1 = __ldg(p + 1);
                raw[j][0] = v0.x; raw[j][1] = v0.y; raw[j][2] = v0.z; raw[j][3] = v0.w;
                raw[j][4] = v1.x; raw[j][5] = v1.y; raw[j][6] = v1.z; raw[j][7] = v1.w;
            } else {
                // augmented weight columns: element k >= K_src is column S[k - K_src]
                const uint16_t* row = a.X + (size_t)r * a.ldx;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    int k0 = 16 * c + 2 * i - a.K_src;
                    uint32_t lo = row[checked_channel(a.S, k0, a.K_src)];
                    uint32_t hi = row[checked_channel(a.S, k0 + 1, a.K_src)];
                    raw[j][i] = lo | (hi << 16);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) raw[j][i] = 0;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
            amax_thread = fmaxf(amax_thread, fmaxf(fabsf(bf16lo(raw[j][i])), fabsf(bf16hi(raw[j][i]))));
    }

    // ---- NVFP4 second-level scale of this row ----
    float s2 = 1.0f;
    if constexpr (FMT == FMT_NVFP4) {
        if (a.mode == 1) {  // per token
            if (a.static_s2) {
                s2 = live ? a.static_s2[r] : 1.0f;
            } else {
                __shared__ float red[32];
                float w = warp_max(amax_thread);
                if (lane == 0) red[t >> 5] = w;
                __syncthreads();
                if (t < 32) {
                    float v = (t < (T >> 5)) ? red[t] : 0.0f;
                    v = warp_max(v);
                    if (t == 0) red[0] = v;
                }
                __syncthreads();
                s2 = nvfp4_s2(red[0]);
            }
            if (live && t == 0) a.s2_out[r] = s2;
        } else {  // one scale for the tensor
            if (a.static_s2) {
                s2 = a.static_s2[0];
            } else {
                s2 = nvfp4_s2(*a.tensor_amax);
            }
            if (r == 0 && t == 0 && a.s2_out) a.s2_out[0] = s2;
        }
    }

#pragma unroll
    for (int j = 0; j < J; ++j) {
        const int c = t + T * j;
        // every lane takes part in the shuffles below; `valid` is uniform per
        // group of 8 lanes because nchunk % 8 == 0 and T % 32 == 0
        const bool valid = c < nchunk;
        float x[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            x[2 * i] = bf16lo(raw[j][i]);
            x[2 * i + 1] = bf16hi(raw[j][i]);
        }
        float bmax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(x[i]));

        uint32_t w0 = 0, w1 = 0;  // 16 codes
        if constexpr (FMT == FMT_NVFP4) {
            uint8_t sb = 0;
            if (live && valid) {
                sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(bmax, 6.0f), s2));
                if (sb != 0) {
                    const float d = __fmul_rn(e4m3_value(sb), s2);
                    float q0[8], q1[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        q0[i] = __fdiv_rn(x[i], d);
                        q1[i] = __fdiv_rn(x[8 + i], d);
                    }
                    w0 = e2m1x8(q0);
                    w1 = e2m1x8(q1);
                }
            }
            // gather 4 consecutive block scales (lanes l..l+3) into one word
            uint32_t b = sb;
            uint32_t b1 = __shfl_down_sync(0xffffffffu, b, 1);
            uint32_t b2 = __shfl_down_sync(0xffffffffu, b, 2);
            uint32_t b3 = __shfl_down_sync(0xffffffffu, b, 3);
            if (valid && (c & 3) == 0)
                *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, c, a.sf_col_atoms)) =
                    b | (b1 << 8) | (b2 << 16) | (b3 << 24);
        } else if constexpr (FMT == FMT_MXFP4) {
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));  // 32-element block = 2 lanes
            uint32_t code = 0;
            if (live && valid && bmax > 0.0f) {
                const uint32_t u = __float_as_uint(bmax);
                const int E = (int)(u >> 23);
                const int e = (E != 0) ? E - 127 : (31 - __clz((int)(u & 0x7FFFFF))) - 149;
                code = (uint32_t)min(max(e + 125, 0), 254);
                const float inv = __uint_as_float((254u - code) << 23);  // 2^(127 - code)
                float q0[8], q1[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    q0[i] = __fmul_rn(x[i], inv);
                    q1[i] = __fmul_rn(x[8 + i], inv);
                }
                w0 = e2m1x8(q0);
                w1 = e2m1x8(q1);
            }
            uint32_t b1 = __shfl_down_sync(0xffffffffu, code, 2);
            uint32_t b2 = __shfl_down_sync(0xffffffffu, code, 4);
            uint32_t b3 = __shfl_down_sync(0xffffffffu, code, 6);
            if (valid && (c & 7) == 0)
                *reinterpret_cast<uint32_t*>(a.sf + sf_offset(r, c >> 1, a.sf_col_atoms)) =
                    code | (b1 << 8) | (b2 << 16) | (b3 << 24);
        } else {  // INT4, 128-element group = 8 lanes
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
            bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 4));
            const float s = (live && valid) ? __fdiv_rn(bmax, 7.0f) : 0.0f;
            if (s != 0.0f) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    int q = __float2int_rn(__fdiv_rn(x[i], s));
                    q = min(max(q, -8), 7);
                    w0 |= (uint32_t)(q & 15) << (4 * i);
                    int p = __float2int_rn(__fdiv_rn(x[8 + i], s));
                    p = min(max(p, -8), 7);
                    w1 |= (uint32_t)(p & 15) << (4 * i);
                }
            }
            if (valid && (c & 7) == 0) a.sfi[(size_t)(c >> 3) * a.sfi_ld + r] = s;
        }
        if (live && valid) *reinterpret_cast<uint2*>(a.codes + (size_t)r * a.ldc + 8 * c) = make_uint2(w0, w1);
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
            float q0[8], q1[8];
            for (int i = 0; i < 8; ++i) {
                q0[i] = __fdiv_rn(R[i], d);
                q1[i] = __fdiv_rn(R[8 + i], d);
            }
            w0 = e2m1x8(q0);
            w1 = e2m1x8(q1);
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
    const int nchunk = a.K / 16;
    int J = 1;
    while (J < 16 && (nchunk + J - 1) / J > 256) J <<= 1;
    int T = (nchunk + J - 1) / J;
    T = (T + 31) / 32 * 32;
    if (T > 256) return cudaErrorInvalidValue;
    dim3 grid(rows_pad), block(T);
    switch (J) {
        case 1: quant_rows_kernel<FMT, 1, GATHER><<<grid, block, 0, st>>>(a); break;
        case 2: quant_rows_kernel<FMT, 2, GATHER><<<grid, block, 0, st>>>(a); break;
        case 4: quant_rows_kernel<FMT, 4, GATHER><<<grid, block, 0, st>>>(a); break;
        case 8: quant_rows_kernel<FMT, 8, GATHER><<<grid, block, 0, st>>>(a); break;
        default: quant_rows_kernel<FMT, 16, GATHER><<<grid, block, 0, st>>>(a); break;
    }
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
