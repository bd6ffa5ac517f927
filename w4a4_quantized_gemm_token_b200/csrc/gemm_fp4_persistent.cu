// Persistent block-scaled FP4 GEMM for large M (tcgen05.mma kind::mxf4nvf4).
//
// Y[m,n] = alpha_mn * sum_b sa[m,b] sb[n,b] sum_{k in b} ea[m,k] eb[n,k]:
// the tensor cores apply the E4M3 (NVFP4, blocks of 16) or E8M0 (MXFP4,
// blocks of 32) scales and accumulate in FP32 in tensor memory, so no
// dequantization runs on the CUDA cores ("APEX4..." page, para 1 (MSD) and
// "Depth Registers..." thelatestinai page, para 2 (APEX4) both place the cost
// of W4A4 in that dequantization).
//
// One CTA per SM loops over 128 x 256 output tiles (grouped raster).  The
// tensor pipe executes the MMAs and the scale-factor copies (tcgen05.cp,
// shared memory -> tensor memory) in one stream, and the MMA-issuing thread
// blocks on each tcgen05 instruction for about its execution time; so the
// copies of a stage are issued by their own warp, and the MMA thread does
// nothing but wait for a stage's scales to land and issue its 4 MMAs.  An
// NVFP4 stage (K = 256) copies 12 atoms of 128 rows x 4 scales (A: 4, B: 8),
// an MXFP4 stage 6; each copy replicates its 32 x 16-byte source into the
// four 32-lane sub-partitions, where the MMA reads row r's scales from
// column base + r/32.
// Warp roles (640 threads):
//   warp 0 lane 0   TMA producer: A/B codes (128-byte swizzled K-major tiles of
//                   256 elements) and compact scale atoms, 4-stage ring.
//   warp 1          TMEM owner; lane 0 issues 4 MMAs (K = 64) per stage.
//   warp 2 lane 0   scale-factor copies into a per-stage TMEM region.
//   warps 4..19     epilogue: TMEM -> registers (lane quarter = warp % 4,
//                   64-column slice (warp - 4) / 4), x alpha, bf16; the
//                   accumulator is released as soon as it is in registers,
//                   the stores (transposed in groups of four lanes, whole
//                   128-byte lines of Y) overlap the next tile.
// Every wait is bounded; on expiry the kernel records a timeout, drains what
// it has in flight, frees TMEM and returns.
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

namespace pf {
constexpr int BN = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = kBM * 128;            // 16 KB of codes
constexpr int B_BYTES = BN * 128;             // 32 KB of codes
constexpr int ATOM = 512;                     // 128 rows x 4 scales
constexpr int SFA_C = 4 * ATOM;               // compact A scales of one stage
constexpr int SFB_C = 2 * 4 * ATOM;           // compact B scales: 2 row halves
constexpr int STAGE = A_BYTES + B_BYTES + SFA_C + SFB_C;
constexpr int BAR_OFF = STAGES * STAGE;
constexpr int SMEM = BAR_OFF + 256 + 1024;
constexpr int SF_COLS = 48;                   // TMEM per stage: A up to 16 + B 32 columns
constexpr int SF_COL0 = BN;                   // after the accumulator
constexpr int TMEM_COLS = 512;
constexpr int EPI_WARPS = 16;                 // four per TMEM lane quarter, 64 columns each
constexpr int THREADS = (4 + EPI_WARPS) * 32;
static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "tensor memory holds 512 columns");
static_assert(SMEM <= 232448, "shared memory per block");
}  // namespace pf

// PB: B (the weights) carries one second-level scale per row (per output
// column of Y), as NVFP4 weights of fused modules quantized per segment do.
template <bool NV, bool PB>
__global__ void __launch_bounds__(pf::THREADS, 1)
    gemm_fp4_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                               GemmArgs g) {
    using namespace pf;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* sfull = empty + STAGES;
    uint64_t* accf = sfull + STAGES;
    uint64_t* acce = accf + 1;
    uint64_t* drain = acce + 1;
    uint64_t* drain2 = drain + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain2 + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = (g.K + kBK_FP4 - 1) / kBK_FP4;
    const int num_a = (g.M + kBM - 1) / kBM, num_b = (g.N + BN - 1) / BN;
    const int ntiles = num_a * num_b;
    const uint64_t limit = g.wait_limit_ns;
    // grouped raster: 8 consecutive A tiles share each B tile
    auto coords = [&](int t, int& at, int& bt) {
        const int GR = 8, per_group = GR * num_b;
        const int grp = t / per_group, first = grp * GR, gsz = min(GR, num_a - first);
        const int in = t - grp * per_group;
        at = first + in % gsz;
        bt = in / gsz;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfull[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, pf::EPI_WARPS);
        mbar_init(drain, 1);
        mbar_init(drain2, 1);
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
    pdl_launch_dependents();  // the next launch may be placed as this grid's CTAs finish
    pdl_wait();  // operands written by the preceding kernel are visible from here on

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------ producer ------------------------------
            int it = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
                int at, bt;
                coords(t, at, bt);
                int halves = 0;
                for (int h = 0; h < 2; ++h)
                    if ((bt * 2 + h) * 128 < g.N) ++halves;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES, n = it / STAGES;
                    if (it >= STAGES && !mbar_wait(&empty[s], (n - 1) & 1, limit, abort_flag)) break;
                    if (kt == g.skip_k_tile) continue;  // test hook: this stage never fills
                    uint8_t* st = smem + s * STAGE;
                    const int nk = min(4, (g.K - kt * kBK_FP4) / 64);
                    const int atoms = NV ? nk : (nk + 1) / 2;
                    const int atom_k0 = NV ? kt * 4 : kt * 2;
                    const uint32_t sfb = atoms * ATOM;
                    mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES + sfb * (1 + halves));
                    tma_load_2d(st, &tmA, kt * 128, at * kBM, &full[s]);
                    tma_load_2d(st + A_BYTES, &tmB, kt * 128, bt * BN, &full[s]);
                    bulk_load(st + A_BYTES + B_BYTES, g.sfa + ((size_t)at * g.sf_col_atoms + atom_k0) * ATOM, sfb,
                              &full[s]);
                    for (int h = 0; h < halves; ++h)
                        bulk_load(st + A_BYTES + B_BYTES + SFA_C + h * 4 * ATOM,
                                  g.sfb + ((size_t)(bt * 2 + h) * g.sf_col_atoms + atom_k0) * ATOM, sfb, &full[s]);
                }
                if (*abort_flag) break;
            }
            if (*abort_flag)  // wait for the copies still in flight
                for (int j = max(0, it - STAGES); j < it; ++j)
                    mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, 100000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            bool ok = true;
            int it = 0, ti = 0;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++ti) {
                if (ti > 0 && !mbar_wait(acce, (ti - 1) & 1, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES, n = it / STAGES;
                    if (!mbar_wait(sfull + s, n & 1, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sA = smem_u32(smem + s * STAGE), sB = sA + A_BYTES;
                    const uint32_t sfa_t = tmem + SF_COL0 + s * SF_COLS, sfb_t = sfa_t + 16;
                    const int nk = min(4, (g.K - kt * kBK_FP4) / 64);
                    for (int j = 0; j < nk; ++j) {
                        const int sfid = NV ? 0 : (j & 1) * 2;
                        const int aj = NV ? j : (j >> 1);  // A scale atom of this MMA
                        const uint32_t ta = (sfa_t + 4 * aj) | ((uint32_t)sfid << 30);
                        const uint32_t tb = (NV ? sfb_t + 8 * j : sfb_t + 8 * (j >> 1)) | ((uint32_t)sfid << 30);
                        mma_fp4<NV>(tmem, desc_kmajor_sw128(sA + 32 * j), desc_kmajor_sw128(sB + 32 * j),
                                    idesc_fp4(kBM, BN, !NV, sfid, sfid), ta, tb, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok) break;
                tc_commit(accf);
            }
            if (!ok) {
                tc_commit(drain);  // every MMA already issued finishes before TMEM is freed
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            // ------------------------- scale-factor copies -------------------------
            bool ok = true;
            int it = 0;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % STAGES, n = it / STAGES;
                    if (!mbar_wait(&full[s], n & 1, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ca = smem_u32(smem + s * STAGE + A_BYTES + B_BYTES), cb = ca + SFA_C;
                    const uint32_t sfa_t = tmem + SF_COL0 + s * SF_COLS, sfb_t = sfa_t + 16;
                    const int nk = min(4, (g.K - kt * kBK_FP4) / 64);
                    const int atoms = NV ? nk : (nk + 1) / 2;
                    for (int j = 0; j < atoms; ++j) {
                        tc_cp_32x128b_x4(sfa_t + 4 * j, desc_sf_32x16(ca + j * ATOM));
                        tc_cp_32x128b_x4(sfb_t + 8 * j, desc_sf_32x16(cb + j * ATOM));
                        tc_cp_32x128b_x4(sfb_t + 8 * j + 4, desc_sf_32x16(cb + 4 * ATOM + j * ATOM));
                    }
                    tc_commit(sfull + s);
                }
            }
            if (!ok) {
                tc_commit(drain2);
                mbar_wait_drain(drain2, 0, 100000000ull);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3, slice = (warp - 4) >> 2;
        const bool y32 = (reinterpret_cast<uintptr_t>(g.Y) & 31) == 0 && (g.ldy & 15) == 0;
        const int j = lane & 3;  // place in the lane's group of four
        int ti = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++ti) {
            int at, bt;
            coords(t, at, bt);
            const int n0 = bt * BN + slice * 64;
            // per-row B scales of the slice's 64 columns, lane l holding column
            // 32 * ch + l, fetched before the accumulator is ready (N is a
            // multiple of 128: a slice is wholly inside N or wholly past it)
            float sbl[2];
            if constexpr (PB) {
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) sbl[ch] = g.s2b[min(n0, g.N - 64) + 32 * ch + lane];
            }
            if (!mbar_wait(accf, ti & 1, limit, abort_flag, 100000)) break;
            tc_fence_after();
            const int m0 = at * kBM + q * 32;
            const int m = m0 + lane;
            float alpha = 1.0f, sa = 0.0f;
            if (NV && m < g.M) {
                sa = g.s2a[g.s2a_per_row ? m : 0];
                alpha = __fmul_rn(sa, g.s2b[0]);
            }
            uint32_t pk[32];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + slice * 64 + 32 * ch, r);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float a0 = alpha, a1 = alpha;
                    if constexpr (PB) {
                        a0 = __fmul_rn(sa, __shfl_sync(0xffffffffu, sbl[ch], 2 * e));
                        a1 = __fmul_rn(sa, __shfl_sync(0xffffffffu, sbl[ch], 2 * e + 1));
                    }
                    __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * e]), a0),
                                                             __fmul_rn(__uint_as_float(r[2 * e + 1]), a1));
                    pk[16 * ch + e] = *reinterpret_cast<uint32_t*>(&h);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);  // accumulator may be overwritten now
            if (n0 >= g.N) continue;
            // 4 x 4 transpose of 32-byte units inside each group of four lanes:
            // lane 4i + j then holds unit j of rows 4i .. 4i + 3
#pragma unroll
            for (int sft = 2; sft >= 1; sft >>= 1) {
#pragma unroll
                for (int u0 = 0; u0 < 4; ++u0) {
                    if (u0 & sft) continue;
                    const int u1 = u0 | sft;
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        const uint32_t snd = (j & sft) ? pk[8 * u0 + w] : pk[8 * u1 + w];
                        const uint32_t rcv = __shfl_xor_sync(0xffffffffu, snd, sft);
                        if (j & sft) pk[8 * u0 + w] = rcv;
                        else pk[8 * u1 + w] = rcv;
                    }
                }
            }
            const int rg = m0 + (lane & ~3);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (rg + r >= g.M) break;
                uint16_t* dst = g.Y + (size_t)(rg + r) * g.ldy + n0 + 16 * j;
                if (y32) {
                    st_global_v8(dst, pk + 8 * r);
                } else {
                    uint4* d4 = reinterpret_cast<uint4*>(dst);
                    d4[0] = make_uint4(pk[8 * r], pk[8 * r + 1], pk[8 * r + 2], pk[8 * r + 3]);
                    d4[1] = make_uint4(pk[8 * r + 4], pk[8 * r + 5], pk[8 * r + 6], pk[8 * r + 7]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_gemm_fp4(bool nvfp4, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                            int num_sms, bool pdl, cudaStream_t st) {
    // variants: MXFP4, NVFP4 with one B scale, NVFP4 with per-row B scales
    const int v = !nvfp4 ? 0 : g.s2b_per_row ? 2 : 1;
    auto kern = v == 0 ? gemm_fp4_persistent_kernel<false, false>
                       : v == 1 ? gemm_fp4_persistent_kernel<true, false> : gemm_fp4_persistent_kernel<true, true>;
    static SmemAttrCache smem_attr[3];
    const cudaError_t e0 = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), pf::SMEM, smem_attr[v]);
    if (e0 != cudaSuccess) return e0;
    const int tiles = ((g.M + kBM - 1) / kBM) * ((g.N + pf::BN - 1) / pf::BN);
    const int grid = tiles < num_sms ? tiles : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(pf::THREADS);
    cfg.dynamicSmemBytes = pf::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, g);
}

}  // namespace w4a4
