// INT4-g128 W4A4 GEMM on the sm_100a 8-bit integer MMA (tcgen05.mma kind::i8).
//
// sm_100's tensor cores have no 4-bit integer kind, so the packed nibbles are
// widened to int8 in shared memory (as 16 * q, see widen8_x16).  Per scale
// group g (GS = 128, 256 or 512 elements of K) the MMAs produce the exact
// int32 partial sum P_g[m,n] = sum_{k in g} qa qw into one of two TMEM
// buffers (GS/128 shared-memory stages of 128 elements accumulate into it);
// CUDA-core warps rescale it,
//     acc[m,n] += float(P_g[m,n]) * (sa[m,g] * sw[n,g])    (FP32),
// and at the end round acc to bf16.  This per-group rescale on the CUDA cores
// is the cost the APEX4 paragraph ("Depth Registers..." thelatestinai page,
// para 2) analyses through the tensor-core / CUDA-core throughput ratio; the
// coarser groups are its rho-aware granularity: GS/128 times fewer rescales.
//
// Persistent (one CTA per SM, 128 x 128 output tiles in turn), 14 warps; the
// MMA and unpack warps run ahead into the next tile while the rescale warps
// finish and store the previous one:
//   warp 0 lane 0   TMA producer: packed codes of A and B (64-byte rows); with
//                   A8 the activations arrive already widened (int8 16 * q,
//                   written so by the quantizer of the fused linear) straight
//                   into the swizzled layout the MMA reads, and only B is unpacked.
//   warp 1          TMEM owner; lane 0 issues 4 MMAs (K=32) per group.
//   warps 2..5      unpack: nibbles -> int8, written in the 128-byte swizzled
//                   K-major layout the MMA reads.
//   warps 6..13     rescale + epilogue: warp w reads TMEM lane quarter w%4,
//                   columns [64*((w-6)/4), +64).
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

namespace i4 {
constexpr int STAGES = 4;
constexpr int PK_BYTES = 128 * 64;      // packed 128 rows x 128 nibbles
constexpr int UN_BYTES = 128 * 128;     // unpacked 128 rows x 128 int8
constexpr int STAGE = 2 * UN_BYTES + 2 * PK_BYTES;  // unpacked A, B, then packed A, B
// Scale ring: the A and B scales of one scale group (128 + 128 floats, 512
// contiguous bytes each in the group-major layout) are staged by the
// producer when the group's first stage loads, SR groups ahead of the
// rescale warps, so no global-memory latency sits on the rescale path.
constexpr int SR = 8;
constexpr int SC_BYTES = 2 * 128 * 4;
constexpr int SC_OFF = STAGES * STAGE;
constexpr int BAR_OFF = SC_OFF + SR * SC_BYTES;
constexpr int SMEM = BAR_OFF + 512 + 1024;
constexpr int THREADS = 14 * 32;
constexpr int TMEM_COLS = 256;                      // two int32 buffers of 128 columns
}  // namespace i4

__device__ __forceinline__ uint64_t pack2(float v) {
    const uint32_t u = __float_as_uint(v);
    return ((uint64_t)u << 32) | u;
}

// (a0, a1) += (float(p0), float(p1)) * (sa * b0, sa * b1) with sm_100's packed
// FP32 operations; every lane is the IEEE result of the scalar sequence
// (product of the scales, rounded; then one fused multiply-add).
__device__ __forceinline__ void rescale2(float& a0, float& a1, uint32_t p0, uint32_t p1, uint64_t sa2, float b0,
                                         float b1) {
    const float f0 = __int2float_rn((int)p0), f1 = __int2float_rn((int)p1);
    asm("{\n\t.reg .b64 b, s, f, a;\n\t"
        "mov.b64 b, {%2, %3};\n\t"
        "mul.rn.f32x2 s, %4, b;\n\t"
        "mov.b64 f, {%5, %6};\n\t"
        "mov.b64 a, {%0, %1};\n\t"
        "fma.rn.f32x2 a, f, s, a;\n\t"
        "mov.b64 {%0, %1}, a;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(b0), "f"(b1), "l"(sa2), "f"(f0), "f"(f1));
}

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

template <bool A8>
__global__ void __launch_bounds__(i4::THREADS, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs g) {
    using namespace i4;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const float* sc_smem = reinterpret_cast<const float*>(smem + SC_OFF);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
    uint64_t* conv = full + STAGES;
    uint64_t* empty = conv + STAGES;
    uint64_t* accf = empty + STAGES;    // [2]
    uint64_t* tfree = accf + 2;         // [2]
    uint64_t* drain = tfree + 2;
    uint64_t* scfull = drain + 1;       // [SR] scales of a group landed
    uint64_t* scfree = scfull + SR;     // [SR] the rescale warps are done with a slot
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(scfree + SR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = g.K / 128;               // shared-memory stages (128 elements of K) per tile
    const int R = g.int4_group / 128;       // stages per scale group
    const int NG = g.K / g.int4_group;      // scale groups per tile
    const uint64_t limit = g.wait_limit_ns;
    // persistent: tiles t = blockIdx.x, +gridDim.x, ...; grouped raster over (m tile, n tile)
    const int num_m = (g.M + 127) / 128, num_n = (g.N + kBN_I4 - 1) / kBN_I4;
    const int ntiles = num_m * num_n;
    auto coords = [&](int t, int& m_tile, int& n_tile) {
        const int GR = 8, per_group = GR * num_n;
        const int grp = t / per_group, first = grp * GR, gsz = min(GR, num_m - first);
        const int in = t - grp * per_group;
        m_tile = first + in % gsz;
        n_tile = in / gsz;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&tfree[b], 8);
        }
        mbar_init(drain, 1);
        for (int i = 0; i < SR; ++i) {
            mbar_init(&scfull[i], 1);
            mbar_init(&scfree[i], 8);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_wait();

    // gi counts the groups of every tile this CTA processes, in order
    if (warp == 0) {
        if (lane == 0) {
            int gi = 0, gg = 0;  // stages and scale groups issued
            bool stop = false;
            const float* sfa = reinterpret_cast<const float*>(g.sfa);
            const float* sfb = reinterpret_cast<const float*>(g.sfb);
            for (int t = blockIdx.x; t < ntiles && !stop; t += gridDim.x) {
                int m_tile, n_tile;
                coords(t, m_tile, n_tile);
                for (int k = 0; k < KT; ++k, ++gi) {
                    const int s = gi % STAGES, n = gi / STAGES;
                    if (gi >= STAGES && !mbar_wait(&empty[s], (n - 1) & 1, limit, abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (k % R == 0) {  // this group's scales, into its ring slot
                        const int slot = gg % SR;
                        if (gg >= SR && !mbar_wait(&scfree[slot], ((gg / SR) - 1) & 1, limit, abort_flag)) {
                            stop = true;
                            break;
                        }
                        uint8_t* dst = smem + SC_OFF + slot * SC_BYTES;
                        mbar_arrive_expect_tx(&scfull[slot], SC_BYTES);
                        bulk_load(dst, sfa + (size_t)(k / R) * g.sfa_ld + m_tile * 128, 512, &scfull[slot]);
                        bulk_load(dst + 512, sfb + (size_t)(k / R) * g.sfb_ld + n_tile * kBN_I4, 512, &scfull[slot]);
                        ++gg;
                    }
                    if (k == g.skip_k_tile) continue;
                    uint8_t* st = smem + s * STAGE;
                    if constexpr (A8) {
                        mbar_arrive_expect_tx(&full[s], UN_BYTES + PK_BYTES);
                        tma_load_2d(st, &tmA, k * 128, m_tile * 128, &full[s]);
                    } else {
                        mbar_arrive_expect_tx(&full[s], 2 * PK_BYTES);
                        tma_load_2d(st + 2 * UN_BYTES, &tmA, k * 64, m_tile * 128, &full[s]);
                    }
                    tma_load_2d(st + 2 * UN_BYTES + PK_BYTES, &tmB, k * 64, n_tile * kBN_I4, &full[s]);
                }
            }
            if (*abort_flag) {
                for (int j = max(0, gi - STAGES); j < gi; ++j) mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, 100000000ull);
                for (int j = max(0, gg - SR); j < gg; ++j) mbar_wait_drain(&scfull[j % SR], (j / SR) & 1, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = true;
            int gi = 0, sg = 0;  // stages and scale groups of every tile, in order
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                for (int k = 0; k < KT; ++k, ++gi) {
                    const int s = gi % STAGES, n = gi / STAGES, buf = sg & 1, sub = k % R;
                    if (!mbar_wait(&conv[s], n & 1, limit, abort_flag)) { ok = false; break; }
                    if (sub == 0 && sg >= 2 && !mbar_wait(&tfree[buf], ((sg >> 1) - 1) & 1, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sA = smem_u32(smem + s * STAGE), sB = sA + UN_BYTES;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_i8(tmem + buf * 128, desc_kmajor_sw128(sA + 32 * j), desc_kmajor_sw128(sB + 32 * j),
                               idesc_i8(128, kBN_I4), (sub > 0 || j > 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                    if (sub == R - 1) {
                        tc_commit(&accf[buf]);
                        ++sg;
                    }
                }
            }
            if (!ok) {
                tc_commit(drain);
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (warp < 6) {
        // ------------------------------ unpack ------------------------------
        const int uw = warp - 2;  // 0..3
        const int total = ((ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x) * KT;
        for (int gi = 0; gi < total; ++gi) {
            const int s = gi % STAGES, n = gi / STAGES;
            if (!mbar_wait(&full[s], n & 1, limit, abort_flag)) break;
            uint8_t* st = smem + s * STAGE;
            // each warp pass: 8 rows x 64 packed bytes; lane -> row r0 + lane/4, segment lane%4
#pragma unroll
            for (int op = A8 ? 1 : 0; op < 2; ++op) {  // A (unless it arrived widened), then B
                const uint8_t* pk = st + 2 * UN_BYTES + op * PK_BYTES;
                uint8_t* un = st + op * UN_BYTES;
#pragma unroll
                for (int pass = 0; pass < 4; ++pass) {
                    const int row = (uw * 4 + pass) * 8 + (lane >> 2);
                    const int seg = lane & 3;
                    const uint4 w = *reinterpret_cast<const uint4*>(pk + row * 64 + seg * 16);
                    uint32_t o[8];
                    widen8_x16(w.x, o[0], o[1]);
                    widen8_x16(w.y, o[2], o[3]);
                    widen8_x16(w.z, o[4], o[5]);
                    widen8_x16(w.w, o[6], o[7]);
                    // 16-byte chunk c of the 128-byte row lands at chunk c ^ (row % 8)
                    const int c0 = 2 * seg, c1 = 2 * seg + 1;
                    *reinterpret_cast<uint4*>(un + row * 128 + ((c0 ^ (row & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(un + row * 128 + ((c1 ^ (row & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
            fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[s]);
        }
    } else {
        // ------------------------------ rescale + epilogue ------------------------------
        const int q = warp & 3, half = (warp - 6) >> 2;
        const int row = q * 32 + lane;
        // the MMA sums 16 qa * 16 qw = 256 P, and scaling sa by 2^-8 (exact)
        // gives float(256 P) * RN(2^-8 sa * sw) = float(P) * RN(sa * sw)
        // After a failed wait the loop keeps running without waiting or
        // reading TMEM.
        bool ok = true;
        int gi = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            int m_tile, n_tile;
            coords(t, m_tile, n_tile);
            const int m = m_tile * 128 + row;
            const int ncol0 = n_tile * kBN_I4 + 64 * half;
            float acc[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
            for (int k = 0; k < NG; ++k, ++gi) {  // gi: scale groups of every tile, in order
                const int buf = gi & 1, slot = gi % SR;
                if (ok) ok = mbar_wait(&scfull[slot], (gi / SR) & 1, limit, abort_flag);
                if (ok) ok = mbar_wait(&accf[buf], (gi >> 1) & 1, limit, abort_flag);
                if (!ok) continue;
                tc_fence_after();
                const float* sc = sc_smem + slot * (SC_BYTES / 4);
                const uint64_t sa2 = pack2(sc[row] * 0.00390625f);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + buf * 128 + 64 * half + 32 * ch, r);
                    tmem_ld_wait();
                    const float4* sb4 = reinterpret_cast<const float4*>(sc + 128 + 64 * half + 32 * ch);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 b = sb4[i];
                        // acc += float(P) * (sa * sb), two columns per packed FP32 operation
                        rescale2(acc[32 * ch + 4 * i], acc[32 * ch + 4 * i + 1], r[4 * i], r[4 * i + 1], sa2, b.x, b.y);
                        rescale2(acc[32 * ch + 4 * i + 2], acc[32 * ch + 4 * i + 3], r[4 * i + 2], r[4 * i + 3], sa2,
                                 b.z, b.w);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&tfree[buf]);
                    mbar_arrive(&scfree[slot]);
                }
            }
            if (ok && m < g.M && ncol0 < g.N) {
                uint16_t* dst = g.Y + (size_t)m * g.ldy + ncol0;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(acc[8 * v + 2 * e], acc[8 * v + 2 * e + 1]);
                        pk[e] = *reinterpret_cast<uint32_t*>(&h);
                    }
                    *reinterpret_cast<uint4*>(dst + 8 * v) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, i4::TMEM_COLS);
    }
}

cudaError_t launch_gemm_int4(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g, int num_sms,
                             bool pdl, cudaStream_t st, bool a8) {
    auto kern = a8 ? gemm_int4_kernel<true> : gemm_int4_kernel<false>;
    static SmemAttrCache smem_attr[2];
    const cudaError_t e0 = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), i4::SMEM, smem_attr[a8]);
    if (e0 != cudaSuccess) return e0;
    const int tiles = ((g.M + 127) / 128) * ((g.N + kBN_I4 - 1) / kBN_I4);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles < num_sms ? tiles : num_sms);  // persistent: one CTA per SM
    cfg.blockDim = dim3(i4::THREADS);
    cfg.dynamicSmemBytes = i4::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, g);
}

}  // namespace w4a4
