// Block-scaled FP4 GEMM on sm_100a tensor cores (tcgen05.mma kind::mxf4nvf4).
//
// Y[m,n] = alpha_mn * sum_b sa[m,b] sb[n,b] sum_{k in b} ea[m,k] eb[n,k]: the
// MMA applies the E4M3 (NVFP4, 16-element blocks) or E8M0 (MXFP4, 32-element
// blocks) scales itself and accumulates in FP32 in tensor memory, so no
// dequantization runs on the CUDA cores ("APEX4..." page, para 1 (MSD) and
// "Depth Registers..." thelatestinai page, para 2 (APEX4) both locate the
// cost of W4A4 in that dequantization).
//
// One CTA computes one 128 x BN output tile.  Warp roles:
//   warp 0, lane 0  TMA producer: codes of A and B (128-byte swizzled K-major
//                   tiles of 256 elements), scale atoms by bulk copy, into a
//                   STAGES-deep shared-memory ring (full/empty mbarriers).
//   warp 1          owns the tensor memory; lane 0 issues tcgen05.cp (scales
//                   -> TMEM) and 4 MMAs (K=64 each) per stage, then commits
//                   the stage back to the producer.
//   warps 2..5      epilogue: TMEM -> registers (each warp its 32-lane
//                   quarter), x alpha, bf16, 16-byte stores.
// Every wait is bounded; on expiry the kernel records a timeout, drains its
// own in-flight copies and MMAs, frees TMEM and returns.
//
// The decode variant (DECODE = true) swaps the operands: 128 weight rows take
// the MMA's M side, the (<= 16) tokens its N side, and K is split across
// CTAs; FP32 partial sums are reduced by a second kernel.
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

__device__ int g_error_word = 0;

template <int BN, int STAGES>
struct Fp4Layout {
    static constexpr int A_BYTES = kBM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SF_ATOM = 512;
    static constexpr int SFA_BYTES = 4 * SF_ATOM;                  // <= 4 atoms per stage
    static constexpr int SFB_HALVES = BN >= 128 ? BN / 128 : 1;    // 128-row scale atoms per B tile
    static constexpr int SFB_BYTES = SFB_HALVES * 4 * SF_ATOM;
    static constexpr int STAGE = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int BAR_OFF = STAGES * STAGE;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;              // barriers + alignment slack
    // TMEM columns: accumulator, then one scale-factor region per pipeline stage
    // (SFA 16 columns, SFB 16 per 128 rows), so that copying the next stage's
    // scales never waits for the MMAs still reading the previous ones.
    static constexpr int SF_COLS = 16 + 16 * SFB_HALVES;
    static constexpr int SFA_COL = BN;
    static constexpr int SFB_COL = BN + 16;
    static constexpr int TMEM_USED = BN + STAGES * SF_COLS;
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                     : TMEM_USED <= 256 ? 256 : 512;
    static_assert(STAGE % 1024 == 0, "stage must keep 1024-byte alignment of the swizzled tiles");
    static_assert(TMEM_USED <= 512, "tensor memory holds 512 columns");
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

template <bool NV, int BN, int STAGES, bool DECODE>
__global__ void __launch_bounds__(192, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs g) {
    using L = Fp4Layout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* drain = accf + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = (g.K + kBK_FP4 - 1) / kBK_FP4;
    // A side = rows of the MMA's M (activations, or weights when DECODE)
    const int a_rows = DECODE ? g.N : g.M;
    const int b_rows = DECODE ? g.M : g.N;
    int a_tile, b_tile, kt_begin, kt_end, split = 0;
    if constexpr (!DECODE) {
        // grouped raster: 8 consecutive A tiles share each B tile within a wave
        const int num_a = (a_rows + kBM - 1) / kBM, num_b = (b_rows + BN - 1) / BN;
        const int G = 8;
        const int per_group = G * num_b;
        const int grp = blockIdx.x / per_group, first = grp * G;
        const int gsz = min(G, num_a - first);
        const int in = blockIdx.x - grp * per_group;
        a_tile = first + in % gsz;
        b_tile = in / gsz;
        kt_begin = 0;
        kt_end = KT;
    } else {
        a_tile = blockIdx.x;
        b_tile = 0;
        split = blockIdx.y;
        kt_begin = split * g.k_tiles_per_split;
        kt_end = min(KT, kt_begin + g.k_tiles_per_split);
    }
    const uint8_t* sfa_g = DECODE ? g.sfb : g.sfa;
    const uint8_t* sfb_g = DECODE ? g.sfa : g.sfb;
    const uint64_t limit = g.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_wait();  // operands written by the preceding kernel are visible from here on

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------ producer ------------------------------
            int i = 0;
            for (int kt = kt_begin; kt < kt_end; ++kt, ++i) {
                const int s = i % STAGES, n = i / STAGES;
                if (i >= STAGES && !mbar_wait(&empty[s], (n - 1) & 1, limit, abort_flag)) break;
                if (kt == g.skip_k_tile) continue;  // test hook: this stage never fills
                uint8_t* st = smem + s * L::STAGE;
                const int nk = min(4, (g.K - kt * kBK_FP4) / 64);              // MMAs in this stage
                const int atoms = NV ? nk : (nk + 1) / 2;                      // scale atoms per 128 rows
                const int atom_k0 = NV ? kt * 4 : kt * 2;
                const uint32_t sf_bytes = atoms * L::SF_ATOM;
                int halves = 0;
#pragma unroll
                for (int h = 0; h < L::SFB_HALVES; ++h)
                    if ((b_tile * L::SFB_HALVES + h) * 128 < max(b_rows, 1)) ++halves;
                mbar_arrive_expect_tx(&full[s], L::A_BYTES + L::B_BYTES + sf_bytes * (1 + halves));
                tma_load_2d(st, &tmA, kt * 128, a_tile * kBM, &full[s]);
                tma_load_2d(st + L::A_BYTES, &tmB, kt * 128, b_tile * BN, &full[s]);
                bulk_load(st + L::A_BYTES + L::B_BYTES,
                          sfa_g + ((size_t)a_tile * g.sf_col_atoms + atom_k0) * L::SF_ATOM, sf_bytes, &full[s]);
                for (int h = 0; h < halves; ++h)
                    bulk_load(st + L::A_BYTES + L::B_BYTES + L::SFA_BYTES + h * 4 * L::SF_ATOM,
                              sfb_g + ((size_t)(b_tile * L::SFB_HALVES + h) * g.sf_col_atoms + atom_k0) * L::SF_ATOM,
                              sf_bytes, &full[s]);
            }
            if (*abort_flag) {
                // wait for the copies this thread still has in flight
                const int issued = i;
                for (int j = max(0, issued - STAGES); j < issued; ++j)
                    if (kt_begin + j != g.skip_k_tile)
                        mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            const uint32_t acc = tmem;
            constexpr int MMA_N = BN;
            int i = 0;
            bool ok = true;
            for (int kt = kt_begin; kt < kt_end; ++kt, ++i) {
                const int s = i % STAGES, n = i / STAGES;
                if (!mbar_wait(&full[s], n & 1, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* st = smem + s * L::STAGE;
                const uint32_t sfa_t = tmem + L::SFA_COL + s * L::SF_COLS;
                const uint32_t sfb_t = tmem + L::SFB_COL + s * L::SF_COLS;
                const uint32_t sA = smem_u32(st), sB = smem_u32(st + L::A_BYTES);
                const uint32_t sSFA = smem_u32(st + L::A_BYTES + L::B_BYTES);
                const uint32_t sSFB = sSFA + L::SFA_BYTES;
                const int nk = min(4, (g.K - kt * kBK_FP4) / 64);
                const int atoms = NV ? nk : (nk + 1) / 2;
                for (int j = 0; j < atoms; ++j) {
                    tc_cp_32x128b_x4(sfa_t + 4 * j, desc_sf_32x16(sSFA + j * L::SF_ATOM));
#pragma unroll
                    for (int h = 0; h < L::SFB_HALVES; ++h)
                        tc_cp_32x128b_x4(sfb_t + 4 * L::SFB_HALVES * j + 4 * h,
                                         desc_sf_32x16(sSFB + h * 4 * L::SF_ATOM + j * L::SF_ATOM));
                }
                for (int j = 0; j < nk; ++j) {
                    const uint64_t ad = desc_kmajor_sw128(sA + 32 * j);
                    const uint64_t bd = desc_kmajor_sw128(sB + 32 * j);
                    const int atom = NV ? j : j >> 1;
                    const int sfid = NV ? 0 : (j & 1) * 2;
                    const uint32_t ta = (sfa_t + 4 * atom) | ((uint32_t)sfid << 30);
                    const uint32_t tb = (sfb_t + 4 * L::SFB_HALVES * atom) | ((uint32_t)sfid << 30);
                    mma_fp4<NV>(acc, ad, bd, idesc_fp4(kBM, MMA_N, !NV, sfid, sfid), ta, tb,
                                (kt > kt_begin || j > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            if (ok) {
                tc_commit(accf);
            } else {
                tc_commit(drain);  // let every MMA already issued finish before TMEM is freed
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const bool ok = mbar_wait(accf, 0, limit, abort_flag);
        tc_fence_after();
        const int row = q * 32 + lane;
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
        if (ok) {
            if constexpr (!DECODE) {
                const int m = a_tile * kBM + row;
                float alpha = 1.0f;
                if (NV && m < g.M) alpha = __fmul_rn(g.s2a[g.s2a_per_row ? m : 0], g.s2b[0]);
#pragma unroll 1
                for (int ch = 0; ch < BN / 32; ++ch) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + 32 * ch, r);
                    tmem_ld_wait();
                    const int n0 = b_tile * BN + 32 * ch;
                    if (m < g.M && n0 < g.N) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * e]), alpha),
                                                                     __fmul_rn(__uint_as_float(r[2 * e + 1]), alpha));
                            pk[e] = *reinterpret_cast<uint32_t*>(&h);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(g.Y + (size_t)m * g.ldy + n0);
#pragma unroll
                        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
            } else {
                const int n = a_tile * kBM + row;  // weight row = output column
                uint32_t r[16];
                tmem_ld_32x32b_x16(taddr, r);
                tmem_ld_wait();
                if (n < g.N) {
                    float* out = g.partial + (size_t)split * g.M * g.N + n;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (j < g.M) out[(size_t)j * g.N] = __uint_as_float(r[j]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// Sum the split-K partials, apply alpha, round to bf16.
template <bool NV>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(GemmArgs g) {
    const long long idx = blockIdx.x * 256LL + threadIdx.x;
    const long long total = (long long)g.M * g.N;
    if (idx >= total) return;
    const int m = (int)(idx / g.N), n = (int)(idx % g.N);
    float acc = 0.0f;
    for (int s = 0; s < g.splits; ++s) acc += g.partial[(size_t)s * total + idx];
    float alpha = NV ? __fmul_rn(g.s2a[g.s2a_per_row ? m : 0], g.s2b[0]) : 1.0f;
    __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(acc, alpha));
    g.Y[(size_t)m * g.ldy + n] = *reinterpret_cast<uint16_t*>(&h);
}

template <typename Kern>
static cudaError_t launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, bool pdl, cudaStream_t st,
                             const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& g) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, a, b, g);
}

template <bool NV>
static cudaError_t launch_dec_t(const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& g, bool pdl,
                                cudaStream_t st) {
    constexpr int STAGES = 8;
    using L = Fp4Layout<kBN_DEC, STAGES>;
    auto kern = gemm_fp4_kernel<NV, kBN_DEC, STAGES, true>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid((g.N + kBM - 1) / kBM, g.splits);
    cudaError_t e = launch_ex(kern, grid, dim3(192), L::SMEM, pdl, st, tmW, tmX, g);
    if (e != cudaSuccess) return e;
    const long long total = (long long)g.M * g.N;
    splitk_reduce_kernel<NV><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(g);
    return cudaGetLastError();
}

cudaError_t launch_gemm_fp4_decode(bool nvfp4, const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& g,
                                   bool pdl, cudaStream_t st) {
    return nvfp4 ? launch_dec_t<true>(tmW, tmX, g, pdl, st) : launch_dec_t<false>(tmW, tmX, g, pdl, st);
}

}  // namespace w4a4
