// Persistent block-scaled FP4 GEMM on CTA pairs, for large M.
//
// Same product as the one-CTA kernel (Y = alpha * block-scaled E2M1 x E2M1,
// FP32 accumulation in tensor memory, bf16 out; "APEX4..." page, para 1
// (MSD) and "Depth Registers..." thelatestinai page, para 2 (APEX4) place
// the cost of W4A4 in dequantization, which the block-scaled MMA removes),
// but each output tile is 256 x 256 and is computed by a cluster of two CTAs
// on two SMs with tcgen05 cta_group::2:
//   - each CTA stages its own 128 rows of A and its own 128 rows of B, so the
//     B tile crosses each SM's shared memory only once per pair (half the
//     per-SM shared-memory traffic of a 128 x 256 one-CTA tile);
//   - one thread of the even CTA issues the pair MMA (256 x 256 x 64), whose
//     accumulator rows 0..127 live in the even CTA's tensor memory and rows
//     128..255 in the odd CTA's;
//   - one pair scale-factor copy fills both CTAs' tensor memory, each from
//     its own shared memory: A's scales are per CTA, B's (all 256 rows) are
//     staged by both.  The MMA reads row r's scales from TMEM lane r, column
//     base + r/32, so every lane quarter needs the whole 32 x 16-byte atom:
//     the atoms arrive already repeated four times (a TMA box over a
//     zero-stride dimension), and one 128 x 256-bit copy then fills the
//     columns of two atoms -- 6 copies per 256-wide K stage instead of 12
//     replicating 32 x 128-bit ones.
//   - a warp of its own issues each stage's copies and signals the MMA warp
//     through a per-stage barrier (one thread's tcgen05 operations block for
//     about their execution time; those of two threads overlap in part).
// All loads are tiled TMA copies without multicast; the odd CTA's copies
// count their bytes on the even CTA's stage barrier (cta_group::2 form),
// whose expected byte count covers both CTAs.  Out-of-range row tiles and K
// tails are zero-filled by the copies.
// Warp roles (384 threads per CTA):
//   warp 0 lane 0   TMA producer (both CTAs), 4-stage (NVFP4) / 5-stage (MXFP4) ring;
//                   each stage (56 KB NVFP4) is near the rate at which TMA fills
//                   shared memory (~64 B per cycle per SM), the bound of this kernel
//   warp 1          TMEM allocation (both CTAs, together); even CTA lane 0
//                   issues the MMAs
//   warp 2          even CTA lane 0 issues the scale-factor copies
//   warps 4..11     epilogue (both CTAs): TMEM -> registers -> bf16 stores,
//                   two warps per lane quarter so the accumulator drains fast
// Every wait is bounded; on expiry the kernel records a timeout, drains its
// copies and MMAs, frees TMEM and returns.
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

namespace pp {
constexpr int BM = 256;                       // pair tile rows of A (128 per CTA)
constexpr int BN = 256;                       // pair tile rows of B
constexpr int HALF = 128;                     // rows of A and of B staged by one CTA
constexpr int A_BYTES = HALF * 128;           // 16 KB of A codes (K = 256 per stage)
constexpr int B_BYTES = HALF * 128;           // 16 KB of B codes
constexpr int ATOM = 512;                     // 128 rows x 4 scales
constexpr int REP = 4;                        // each atom staged 4 times (the TMEM lane quarters)
constexpr int SF_COLS = 48;                   // TMEM per stage: A 16 + B 32 columns
constexpr int SF_COL0 = BN;                   // after the accumulator
constexpr int TMEM_COLS = 512;
constexpr int THREADS = 384;
constexpr int EPI_WARPS = 8;                  // two per TMEM lane quarter, 128 columns each
// Per format: NVFP4 stages 4 scale atoms per 128 rows and K-stage, MXFP4 2.
template <bool NV>
struct Cfg {
    static constexpr int ATOMS = NV ? 4 : 2;
    static constexpr int SFA_C = ATOMS * REP * ATOM;      // this CTA's A scale atoms of a stage
    static constexpr int SFB_C = 2 * ATOMS * REP * ATOM;  // B scale atoms of both row halves
    static constexpr int STAGE = A_BYTES + B_BYTES + SFA_C + SFB_C;
    static constexpr int STAGES = NV ? 4 : 5;
    static constexpr int BAR_OFF = STAGES * STAGE;
    static constexpr int SMEM = BAR_OFF + 256 + 1024;
    static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
    static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "tensor memory holds 512 columns");
    static_assert(SMEM <= 232448, "shared memory per block");
};
}  // namespace pp

// PB: B (the weights) carries one second-level scale per row (per output
// column of Y), as NVFP4 weights of fused modules quantized per segment do.
template <bool NV, bool PB>
__global__ void __launch_bounds__(pp::THREADS, 1)
    gemm_fp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                         GemmArgs g) {
    using namespace pp;
    using C = Cfg<NV>;
    constexpr int STAGES = C::STAGES, STAGE = C::STAGE, SFA_C = C::SFA_C, BAR_OFF = C::BAR_OFF;
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
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int KT = (g.K + kBK_FP4 - 1) / kBK_FP4;
    const int num_a = (g.M + BM - 1) / BM, num_b = (g.N + BN - 1) / BN;
    const int ntiles = num_a * num_b;
    const uint64_t limit = g.wait_limit_ns;
    constexpr int atoms_ps = C::ATOMS;  // scale atoms per 256-wide K stage and 128 rows
    // grouped raster: a group of A tiles (about 40 MB of A codes and scales, so
    // it stays in L2) is swept against every B tile, so B is read from HBM once
    // per group
    const int GR = max(1, min(num_a, (int)(40000000LL / (144LL * g.K))));
    auto coords = [&](int t, int& at, int& bt) {
        const int per_group = GR * num_b;
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
        mbar_init(acce, 2 * EPI_WARPS);  // the epilogue warps of both CTAs
        mbar_init(drain, 1);
        mbar_init(drain2, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers and tensor memory exist from here on
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // the next launch (the next linear's quantizer) may be placed on SMs as
    // this grid's CTAs finish; it waits for this grid before touching memory
    pdl_launch_dependents();
    const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
    const uint32_t acce_leader = mapa_shared(smem_u32(acce), 0);
    // operands written by the preceding kernel (A, its scales, s2a) are visible
    // after this wait; the producer waits only before its first A load, so the
    // weights of the first stages stream in while the quantizer finishes
    if (!(warp == 0 && lane == 0)) pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------ producer ------------------------------
            const uint32_t stage_tx = 2u * (A_BYTES + B_BYTES + 3u * atoms_ps * REP * ATOM);
            auto load_b = [&](int s, int bt, int kt) {  // weights: independent of the preceding kernel
                uint8_t* st = smem + s * STAGE;
                const uint32_t bar = full_leader + 8u * s;
                if (leader) mbar_arrive_expect_tx(&full[s], stage_tx);
                tma_load_2d_pair(st + A_BYTES, &tmB, kt * 128, bt * BN + (int)rank * HALF, bar);
                tma_load_5d_pair(st + A_BYTES + B_BYTES + SFA_C, &tmSB, 0, 0, 0, kt * atoms_ps, bt * 2, bar);
            };
            auto load_a = [&](int s, int at, int kt) {
                uint8_t* st = smem + s * STAGE;
                const uint32_t bar = full_leader + 8u * s;
                tma_load_2d_pair(st, &tmA, kt * 128, at * BM + (int)rank * HALF, bar);
                tma_load_5d_pair(st + A_BYTES + B_BYTES, &tmSA, 0, 0, 0, kt * atoms_ps, at * 2 + (int)rank, bar);
            };
            // the first stages' weights before the wait for the preceding kernel
            int pre = 0;
            if (pair < ntiles) {
                int at, bt;
                coords(pair, at, bt);
                for (; pre < STAGES && pre < KT; ++pre)
                    if (pre != g.skip_k_tile) load_b(pre, bt, pre);
                pdl_wait();
                for (int j = 0; j < pre; ++j)
                    if (j != g.skip_k_tile) load_a(j, at, j);
            } else {
                pdl_wait();
            }
            int it = 0;
            for (int t = pair; t < ntiles && !*abort_flag; t += npairs) {
                int at, bt;
                coords(t, at, bt);
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    if (it < pre) continue;  // loaded above
                    const int s = it % STAGES, n = it / STAGES;
                    if (it >= STAGES && !mbar_wait(&empty[s], (n - 1) & 1, limit, abort_flag)) break;
                    if (kt == g.skip_k_tile) continue;  // test hook: this stage never fills
                    load_b(s, bt, kt);
                    load_a(s, at, kt);
                }
                if (*abort_flag) break;
            }
            if (*abort_flag && leader)  // the stage barriers count both CTAs' copies
                for (int j = max(0, it - STAGES); j < it; ++j)
                    mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, 100000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------ MMA issuer ------------------------------
            bool ok = true;
            int it = 0, ti = 0;
            for (int t = pair; t < ntiles && ok; t += npairs, ++ti) {
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
                        const int aj = NV ? j : (j >> 1);  // scale atom of this MMA
                        const uint32_t ta = (sfa_t + 4 * aj) | ((uint32_t)sfid << 30);
                        const uint32_t tb = (sfb_t + 8 * aj) | ((uint32_t)sfid << 30);
                        mma_fp4_pair<NV>(tmem, desc_kmajor_sw128(sA + 32 * j), desc_kmajor_sw128(sB + 32 * j),
                                         idesc_fp4(BM, BN, !NV, sfid, sfid), ta, tb, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit_pair_mc(&empty[s], 3);
                }
                if (!ok) break;
                tc_commit_pair_mc(accf, 3);
            }
            if (!ok) {
                tc_commit_pair(drain);  // every MMA already issued finishes before TMEM is freed
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (warp == 2) {
        if (lane == 0 && leader) {
            // ------------------------- scale-factor copies -------------------------
            // From another thread than the MMAs (a thread's tcgen05 instructions
            // block for about their execution time, and the pipe overlaps copies
            // with MMAs of other threads).  A: atoms 2p, 2p+1 (4 repeats each, 2 KB
            // apart) -> columns 8p .. 8p+7; B: atom j of row halves 0 and 1 -> 8j .. 8j+7.
            bool ok = true;
            int it = 0;
            for (int t = pair; t < ntiles && ok; t += npairs) {
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
                    for (int pa = 0; pa < (atoms + 1) / 2; ++pa)
                        tc_cp_pair_128x256b(sfa_t + 8 * pa, smem_desc(ca + pa * 2 * REP * ATOM, REP * ATOM, 128, 0));
                    for (int j = 0; j < atoms; ++j)
                        tc_cp_pair_128x256b(sfb_t + 8 * j,
                                            smem_desc(cb + j * REP * ATOM, atoms_ps * REP * ATOM, 128, 0));
                    tc_commit_pair(sfull + s);
                }
            }
            if (!ok) {
                tc_commit_pair(drain2);
                mbar_wait_drain(drain2, 0, 100000000ull);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------ epilogue ------------------------------
        // warp w reads TMEM lane quarter w % 4 (rows q*32..) and column half
        // (w - 4) / 4 (128 accumulator columns = 128 outputs of its row)
        const int q = warp & 3, half = (warp - 4) >> 2;
        // rows of Y start on 32-byte boundaries: whole-sector stores
        const bool y32 = (reinterpret_cast<uintptr_t>(g.Y) & 31) == 0 && (g.ldy & 15) == 0;
        int ti = 0;
        for (int t = pair; t < ntiles; t += npairs, ++ti) {
            int at, bt;
            coords(t, at, bt);
            // per-row B scales of these 128 columns, lane l holding column
            // 32 * ch + l, fetched before the accumulator is ready (N is a
            // multiple of 128: a half tile is wholly inside N or wholly past it)
            float sbl[4];
            if constexpr (PB) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) sbl[ch] = g.s2b[min(bt * BN + half * 128, g.N - 128) + 32 * ch + lane];
            }
            if (!mbar_wait(accf, ti & 1, limit, abort_flag, 100000)) break;
            tc_fence_after();
            const int m = at * BM + (int)rank * HALF + q * 32 + lane;
            float alpha = 1.0f, sa = 0.0f;
            if (NV && m < g.M) {
                sa = g.s2a[g.s2a_per_row ? m : 0];
                alpha = __fmul_rn(sa, g.s2b[0]);
            }
            uint32_t pk[64];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + half * 128 + 32 * ch, r);
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
            if (lane == 0) mbar_arrive_cluster(acce_leader);  // this part of the accumulator is free
            if (m < g.M) {
                const int n0 = bt * BN + half * 128;
                const int nv = max(0, min(128, g.N - n0)) / 8;  // 16-byte vectors in range
                uint16_t* row = g.Y + (size_t)m * g.ldy + n0;
                if (y32 && nv == 16) {
                    // whole sectors: 32 bytes per lane and store (each lane writes
                    // its own row, so 16-byte stores would write half sectors and
                    // hold up the next tile's loads for microseconds; measured
                    // faster overall than transposing into whole lines first)
#pragma unroll
                    for (int v = 0; v < 8; ++v) st_global_v8(row + 16 * v, pk + 8 * v);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(row);
#pragma unroll
                    for (int v = 0; v < 16; ++v)
                        if (v < nv) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA frees tensor memory the pair's MMAs may still write
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

cudaError_t launch_gemm_fp4_pair(bool nvfp4, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmSA,
                                 const CUtensorMap& tmSB, const GemmArgs& g, int num_sms, bool pdl, cudaStream_t st) {
    // variants: MXFP4, NVFP4 with one B scale, NVFP4 with per-row B scales
    const int v = !nvfp4 ? 0 : g.s2b_per_row ? 2 : 1;
    auto kern = v == 0 ? gemm_fp4_pair_kernel<false, false>
                       : v == 1 ? gemm_fp4_pair_kernel<true, false> : gemm_fp4_pair_kernel<true, true>;
    static SmemAttrCache smem_attr[3];
    cudaError_t e0 = ensure_dynamic_smem(reinterpret_cast<const void*>(kern),
                                         nvfp4 ? pp::Cfg<true>::SMEM : pp::Cfg<false>::SMEM, smem_attr[v]);
    if (e0 != cudaSuccess) return e0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kAttrDevices) return cudaErrorInvalidDevice;
    const int tiles = ((g.M + pp::BM - 1) / pp::BM) * ((g.N + pp::BN - 1) / pp::BN);
    // as many pairs as can be resident at once (a persistent grid must not queue)
    static std::atomic<int> resident[kAttrDevices][3];  // per device (zero-initialised)
    if (!resident[dev][v].load(std::memory_order_acquire)) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(2 * (num_sms / 2));
        q.blockDim = dim3(pp::THREADS);
        q.dynamicSmemBytes = nvfp4 ? pp::Cfg<true>::SMEM : pp::Cfg<false>::SMEM;
        cudaLaunchAttribute ca[1];
        ca[0].id = cudaLaunchAttributeClusterDimension;
        ca[0].val.clusterDim.x = 2;
        ca[0].val.clusterDim.y = 1;
        ca[0].val.clusterDim.z = 1;
        q.attrs = ca;
        q.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = num_sms / 2;
        }
        resident[dev][v].store(n, std::memory_order_release);
    }
    int pairs = tiles < num_sms / 2 ? tiles : num_sms / 2;
    const int res = resident[dev][v].load(std::memory_order_acquire);
    if (pairs > res) pairs = res;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(pp::THREADS);
    cfg.dynamicSmemBytes = nvfp4 ? pp::Cfg<true>::SMEM : pp::Cfg<false>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmSA, tmSB, g);
}

}  // namespace w4a4
