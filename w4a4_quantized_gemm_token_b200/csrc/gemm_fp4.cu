// Small-M ("decode") block-scaled FP4 GEMM: Y[M,N] = X[M,K] W[N,K]^T for
// M <= 128, bound by streaming the 4-bit weights from HBM.
//
// The weights take the MMA's M side (128 rows per tile) and the tokens its N
// side (BN = 16, 32, 64 or 128: the smallest that holds M), so one
// tcgen05.mma kind::mxf4nvf4 covers 128 x BN x 64.  A work
// unit is a weight tile and KB consecutive K-stages of 256; the units are
// split into equal contiguous ranges, one per SM (stream-K), so every SM
// streams the same number of weight bytes whatever N and K are.  With KB = 2
// the weights arrive as 3-D boxes (128-byte K-block, row, K-block): each row
// contributes 256 contiguous bytes per copy instead of 128, which HBM serves
// much faster, and the box still lands as standard 128-byte-swizzled tiles.
// A CTA accumulates in TMEM while its range stays in one weight tile and
// writes an FP32 partial sum per tile segment (double-buffered accumulators
// up to BN = 128, one of 256 columns for BN = 256); the CTA that writes a
// tile's last segment adds the tile's
// segments in a fixed order (deterministic), applies alpha and rounds to
// bf16.  Launched as a
// programmatic dependent, the kernel starts streaming weights while the
// activation quantizer still runs and waits only before its first activation
// load.
// Warp roles (256 threads): warp 0 lane 0 TMA producer, warp 1 TMEM owner +
// MMA issuer, warp 2 lane 0 scale-factor copies, warps 4..7 epilogue (TMEM
// lane quarter = warp % 4).
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace w4a4 {

__device__ int g_error_word = 0;

// K-stages per work unit: two when the weights' K-block count is exact (the
// 3-D box view needs K % 256 == 0), else one (2-D boxes).
__host__ __device__ __forceinline__ int decode_kb(int K) { return K % kBK_FP4 == 0 ? 2 : 1; }

template <int KB, int BN_>
struct Dec {
    static constexpr int BN = BN_;                     // tokens per MMA (the MMA's N)
    static constexpr int TOK_TILES = BN > 128 ? 2 : 1; // 128-row tiles of the token scale atoms
    static constexpr int ACC_BUFS = BN > 128 ? 1 : 2;  // accumulators of BN columns
    static constexpr int A_BYTES = KB * kBM * 128;     // weight tiles [kb][128 rows][128 B]
    static constexpr int B_BYTES = KB * BN * 128;      // token tiles [kb][BN rows][128 B]
    static constexpr int ATOM = 512;
    static constexpr int SFA_C = KB * 4 * ATOM;        // weight scale atoms of a unit
    static constexpr int SFB_T = KB * 4 * ATOM;        // token scale atoms of a unit, per 128-row tile
    static constexpr int SFB_C = TOK_TILES * SFB_T;
    static constexpr int STAGE = A_BYTES + B_BYTES + SFA_C + SFB_C;
    static constexpr int SF_COLS = KB * 16 * (1 + TOK_TILES);  // per stage: weights, then tokens
    static constexpr int SF_COL0 = ACC_BUFS * BN;              // after the accumulators
    static constexpr int TMEM_COLS = 512;
    static constexpr int SMEM_MAX = 232448 - 512 - 1024;
    // as many stages as shared and tensor memory hold (at most 10)
    static constexpr int S_SMEM = SMEM_MAX / STAGE, S_TMEM = (TMEM_COLS - SF_COL0) / SF_COLS;
    static constexpr int STAGES = S_SMEM < S_TMEM ? (S_SMEM < 10 ? S_SMEM : 10) : (S_TMEM < 10 ? S_TMEM : 10);
    static constexpr int BAR_OFF = STAGES * STAGE;
    static constexpr int SMEM = BAR_OFF + 512 + 1024;
    static constexpr int THREADS = 256;
    static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
    static_assert(STAGES >= 2, "at least two stages");
    static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
    static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "tensor memory holds 512 columns");
    static_assert(SMEM <= 232448, "shared memory per block");
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// First unit of CTA c when U units are split into G equal contiguous ranges.
__host__ __device__ __forceinline__ long long unit_begin(int c, long long U, int G) { return (long long)c * U / G; }

// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long u, long long U, int G) {
    int c = (int)(u * G / U);
    while (c + 1 < G && unit_begin(c + 1, U, G) <= u) ++c;
    while (c > 0 && unit_begin(c, U, G) > u) --c;
    return c;
}

template <bool NV, int KB, int BN_>
__global__ void __launch_bounds__(Dec<KB, BN_>::THREADS, 1)
    gemm_fp4_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           GemmArgs g) {
    using D = Dec<KB, BN_>;
    constexpr int STAGES = D::STAGES, A_BYTES = D::A_BYTES, B_BYTES = D::B_BYTES, ATOM = D::ATOM;
    constexpr int BN = D::BN, TT = D::TOK_TILES, NBUF = D::ACC_BUFS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + D::BAR_OFF);
    uint64_t* empty = full + STAGES;
    uint64_t* sfull = empty + STAGES;
    uint64_t* accf = sfull + STAGES;  // [2]
    uint64_t* acce = accf + 2;        // [2]
    uint64_t* drain = acce + 2;
    uint64_t* drain2 = drain + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain2 + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = (g.K + kBK_FP4 - 1) / kBK_FP4;
    const int KG = (KT + KB - 1) / KB;  // units per weight tile
    const int ntiles = (g.N + kBM - 1) / kBM;
    const long long U = (long long)ntiles * KG;
    const int G = gridDim.x;
    const long long u0 = unit_begin(blockIdx.x, U, G), u1 = unit_begin(blockIdx.x + 1, U, G);
    const int nunits = (int)(u1 - u0);
    const uint64_t limit = g.wait_limit_ns;
    // weights are the MMA's A side, tokens its B side
    const uint8_t* sfw = g.sfb;
    const uint8_t* sfx = g.sfa;
    // K-chunks of 64 and scale atoms of unit u (K tails have fewer)
    auto unit_chunks = [&](long long u, int& nk, int& atoms, int& atom_k0) {
        const int kt0 = (int)(u % KG) * KB;
        nk = min(4 * KB, (g.K - kt0 * kBK_FP4) / 64);
        atoms = NV ? nk : (nk + 1) / 2;
        atom_k0 = NV ? kt0 * 4 : kt0 * 2;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfull[s], 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 4);
        }
        mbar_init(drain, 1);
        mbar_init(drain2, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, D::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_launch_dependents();  // the next launch may be scheduled; it waits for this grid

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------ producer ------------------------------
            auto load_w = [&](long long u, int s) {
                const int nt = (int)(u / KG), kt0 = (int)(u % KG) * KB;
                int nk, atoms, k0;
                unit_chunks(u, nk, atoms, k0);
                uint8_t* st = smem + s * D::STAGE;
                // full boxes (K-blocks past K are zero-filled) + the scale atoms in range
                mbar_arrive_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES + (1 + TT) * atoms * ATOM));
                if (KB == 1)
                    tma_load_2d(st, &tmW, kt0 * 128, nt * kBM, &full[s]);
                else
                    tma_load_3d(st, &tmW, 0, nt * kBM, kt0, &full[s]);
                bulk_load(st + A_BYTES + B_BYTES, sfw + ((size_t)nt * g.sf_col_atoms + k0) * ATOM, atoms * ATOM,
                          &full[s]);
            };
            auto load_x = [&](long long u, int s) {
                const int kt0 = (int)(u % KG) * KB;
                int nk, atoms, k0;
                unit_chunks(u, nk, atoms, k0);
                uint8_t* st = smem + s * D::STAGE;
                if (KB == 1)
                    tma_load_2d(st + A_BYTES, &tmX, kt0 * 128, 0, &full[s]);
                else
                    tma_load_3d(st + A_BYTES, &tmX, 0, 0, kt0, &full[s]);
                // the token scale atoms of each 128-row tile (rows past M are zero padding)
#pragma unroll
                for (int h = 0; h < TT; ++h)
                    bulk_load(st + A_BYTES + B_BYTES + D::SFA_C + h * D::SFB_T,
                              sfx + ((size_t)h * g.sf_col_atoms + k0) * ATOM, atoms * ATOM, &full[s]);
            };
            // stream the first weight units before the activations are known to be ready
            const int pre = min(STAGES, nunits);
            int it = 0;
            for (; it < pre; ++it)
                if (it != g.skip_k_tile) load_w(u0 + it, it);
            pdl_wait();
            for (int j = 0; j < pre; ++j)
                if (j != g.skip_k_tile) load_x(u0 + j, j);
            for (; it < nunits; ++it) {
                const int s = it % STAGES, n = it / STAGES;
                if (!mbar_wait(&empty[s], (n - 1) & 1, limit, abort_flag)) break;
                if (it == g.skip_k_tile) continue;  // test hook: this stage never fills
                load_w(u0 + it, s);
                load_x(u0 + it, s);
            }
            if (*abort_flag)
                for (int j = max(0, it - STAGES); j < it; ++j)
                    mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, 100000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------ MMA issuer ------------------------------
            bool ok = true;
            int it = 0, seg = 0;
            long long u = u0;
            while (u < u1 && ok) {
                const int nt = (int)(u / KG);
                const long long sbeg = u, send = min(u1, (long long)(nt + 1) * KG);
                const int buf = NBUF == 2 ? (seg & 1) : 0;
                const int use = NBUF == 2 ? (seg >> 1) : seg;  // earlier uses of this accumulator
                if (use >= 1 && !mbar_wait(&acce[buf], (use - 1) & 1, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (; u < send; ++u, ++it) {
                    const int s = it % STAGES, n = it / STAGES;
                    if (!mbar_wait(&sfull[s], n & 1, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    int nk, atoms, k0;
                    unit_chunks(u, nk, atoms, k0);
                    const uint32_t sA = smem_u32(smem + s * D::STAGE), sB = sA + A_BYTES;
                    const uint32_t sfa_t = tmem + D::SF_COL0 + s * D::SF_COLS, sfb_t = sfa_t + 16 * KB;
                    for (int j = 0; j < nk; ++j) {
                        const int kb = j >> 2, jj = j & 3;  // K-block of the unit, chunk within it
                        const int sfid = NV ? 0 : (j & 1) * 2;
                        const int aj = NV ? j : (j >> 1);
                        // token scales: 4 columns per atom and 128-row tile (tile 1 of
                        // BN = 256 at +4, where the MMA reads rows 128..255)
                        mma_fp4<NV>(tmem + buf * BN, desc_kmajor_sw128(sA + kb * (kBM * 128) + 32 * jj),
                                    desc_kmajor_sw128(sB + kb * (BN * 128) + 32 * jj),
                                    idesc_fp4(kBM, BN, !NV, sfid, sfid), (sfa_t + 4 * aj) | ((uint32_t)sfid << 30),
                                    (sfb_t + 4 * TT * aj) | ((uint32_t)sfid << 30), (u > sbeg || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok) break;
                tc_commit(&accf[buf]);
                ++seg;
            }
            if (!ok) {
                tc_commit(drain);
                mbar_wait_drain(drain, 0, 100000000ull);
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            // ------------------------- scale-factor copies -------------------------
            bool ok = true;
            for (int it = 0; it < nunits; ++it) {
                const int s = it % STAGES, n = it / STAGES;
                if (!mbar_wait(&full[s], n & 1, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                int nk, atoms, k0;
                unit_chunks(u0 + it, nk, atoms, k0);
                const uint32_t ca = smem_u32(smem + s * D::STAGE + A_BYTES + B_BYTES), cb = ca + D::SFA_C;
                const uint32_t sfa_t = tmem + D::SF_COL0 + s * D::SF_COLS, sfb_t = sfa_t + 16 * KB;
                for (int j = 0; j < atoms; ++j) {
                    tc_cp_32x128b_x4(sfa_t + 4 * j, desc_sf_32x16(ca + j * ATOM));
#pragma unroll
                    for (int h = 0; h < TT; ++h)
                        tc_cp_32x128b_x4(sfb_t + 4 * TT * j + 4 * h, desc_sf_32x16(cb + h * D::SFB_T + j * ATOM));
                }
                tc_commit(sfull + s);
            }
            if (!ok) {
                tc_commit(drain2);
                mbar_wait_drain(drain2, 0, 100000000ull);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------ epilogue ------------------------------
        // Segment partial sums -> workspace slot (tile, owner offset) [BN tokens][128
        // rows] FP32.  The CTA whose segment completes a tile (a per-tile counter)
        // adds all the tile's slots in owner order -- the same order whichever CTA
        // arrives last -- applies alpha, writes Y and clears the counter.
        const int q = warp & 3;
        const int row = q * 32 + lane;
        __shared__ int last_flag;
        // Every epilogue warp runs the same segments and named barriers; after a
        // failed (timed-out) wait a warp only skips its TMEM read and stores.
        int seg = 0;
        long long u = u0;
        bool waited = false, ok = true;
        while (u < u1) {
            const int nt = (int)(u / KG);
            const long long send = min(u1, (long long)(nt + 1) * KG);
            const int buf = NBUF == 2 ? (seg & 1) : 0;
            const int use = NBUF == 2 ? (seg >> 1) : seg;
            const int first = unit_owner((long long)nt * KG, U, G);
            const int last = unit_owner((long long)(nt + 1) * KG - 1, U, G);
            float* tile = g.partial + (size_t)nt * g.splits * (BN * kBM);
            if (ok) ok = mbar_wait(&accf[buf], use & 1, limit, abort_flag, 20000);
            if (ok) {
                tc_fence_after();
                float* slot = tile + (size_t)(blockIdx.x - first) * (BN * kBM);
                const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * BN;
                if constexpr (BN == 16) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(taddr, r);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce[buf]);
#pragma unroll
                    for (int t = 0; t < BN; ++t) slot[t * kBM + row] = __uint_as_float(r[t]);
                } else {
                    // 32 tokens at a time: read, then store while the next chunk is read
#pragma unroll 1
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(taddr + 32 * c, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 32; ++t) slot[(32 * c + t) * kBM + row] = __uint_as_float(r[t]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce[buf]);
                }
            }
            __threadfence();
            named_bar_sync(1, 128);  // the four epilogue warps wrote their rows
            if (threadIdx.x == 128) {
                if (!waited) pdl_wait();  // the counters were cleared by the preceding launch
                waited = true;
                last_flag = !*abort_flag && atomicAdd(&g.tile_count[nt], 1) == last - first;
            }
            named_bar_sync(1, 128);
            if (last_flag) {
                __threadfence();
                // thread e of the 128 takes positions (token, 4 rows) p = e, e+128, ...,
                // four at a time: the float4 loads of four positions and all their
                // segments are issued before any addition
                const int owners = last - first + 1, e = threadIdx.x - 128;
                constexpr int PMAX = BN * kBM / 4 / 128, PG = PMAX < 4 ? PMAX : 4, OMAX = 4;
#pragma unroll 1
                for (int p0 = 0; p0 < PMAX; p0 += PG) {
                    float4 v[PG][OMAX];
#pragma unroll
                    for (int pi = 0; pi < PG; ++pi) {
                        const int p = e + 128 * (p0 + pi), t = p >> 5, r4 = (p & 31) * 4;
                        const float4* src = reinterpret_cast<const float4*>(tile + t * kBM + r4);
#pragma unroll
                        for (int c = 0; c < OMAX; ++c)
                            if (t < g.M && c < owners) v[pi][c] = src[(size_t)c * (BN * kBM / 4)];
                    }
#pragma unroll
                    for (int pi = 0; pi < PG; ++pi) {
                        const int p = e + 128 * (p0 + pi), t = p >> 5, r4 = (p & 31) * 4;
                        if (t >= g.M) continue;
                        const float4* src = reinterpret_cast<const float4*>(tile + t * kBM + r4);
                        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        // fixed order: owner offset 0, 1, ...
#pragma unroll
                        for (int c = 0; c < OMAX; ++c)
                            if (c < owners) {
                                acc.x += v[pi][c].x;
                                acc.y += v[pi][c].y;
                                acc.z += v[pi][c].z;
                                acc.w += v[pi][c].w;
                            }
                        for (int c = OMAX; c < owners; ++c) {
                            const float4 w = src[(size_t)c * (BN * kBM / 4)];
                            acc.x += w.x;
                            acc.y += w.y;
                            acc.z += w.z;
                            acc.w += w.w;
                        }
                        const int n = nt * kBM + r4;
                        // alpha per output column: s2 of token t times s2 of weight row n
                        // (one weight scale, or one per row for per-segment weights)
                        float4 al = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
                        if (NV) {
                            const float sa = g.s2a[g.s2a_per_row ? t : 0];
                            const float4 sb = g.s2b_per_row
                                                  ? *reinterpret_cast<const float4*>(g.s2b + min(n, g.N - 4))
                                                  : make_float4(g.s2b[0], g.s2b[0], g.s2b[0], g.s2b[0]);
                            al = make_float4(__fmul_rn(sa, sb.x), __fmul_rn(sa, sb.y), __fmul_rn(sa, sb.z),
                                             __fmul_rn(sa, sb.w));
                        }
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(__fmul_rn(acc.x, al.x), __fmul_rn(acc.y, al.y));
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(__fmul_rn(acc.z, al.z), __fmul_rn(acc.w, al.w));
                        if (n < g.N)
                            *reinterpret_cast<uint2*>(g.Y + (size_t)t * g.ldy + n) =
                                make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
                    }
                }
                if (threadIdx.x == 128) g.tile_count[nt] = 0;  // ready for the next call
            }
            named_bar_sync(1, 128);  // last_flag is rewritten for the next segment
            u = send;
            ++seg;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, D::TMEM_COLS);
    }
}

static cudaError_t launch_pdl(const void* kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, void** args) {
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
    return cudaLaunchKernelExC(&cfg, kern, args);
}

static long long decode_units(int N, int K) {
    const int KT = (K + kBK_FP4 - 1) / kBK_FP4, kb = decode_kb(K);
    return (long long)((N + kBM - 1) / kBM) * ((KT + kb - 1) / kb);
}

int decode_grid(int N, int K, int num_sms) {
    const long long U = decode_units(N, K);
    return (int)(U < num_sms ? U : num_sms);
}

int decode_max_owners(int N, int K, int num_sms) {
    const int KT = (K + kBK_FP4 - 1) / kBK_FP4, kb = decode_kb(K);
    const int KG = (KT + kb - 1) / kb;
    const long long U = decode_units(N, K);
    const int G = decode_grid(N, K, num_sms);
    const long long per = U / G;  // every range holds per or per + 1 units
    return (int)((KG + per - 1) / per) + 1;
}

template <bool NV, int KB, int BN>
static cudaError_t launch_dec_t(const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& g0, int num_sms,
                                cudaStream_t st) {
    using D = Dec<KB, BN>;
    auto kern = gemm_fp4_decode_kernel<NV, KB, BN>;
    static SmemAttrCache attr;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), D::SMEM, attr);
    if (e != cudaSuccess) return e;
    GemmArgs g = g0;
    const int G = decode_grid(g.N, g.K, num_sms);
    g.splits = decode_max_owners(g.N, g.K, num_sms);  // slots per weight tile in the workspace
    CUtensorMap a = tmW, b = tmX;
    void* args[] = {&a, &b, &g};
    return launch_pdl(reinterpret_cast<const void*>(kern), dim3(G), dim3(D::THREADS), D::SMEM, st, args);
}

int decode_k_blocks(int K) { return decode_kb(K); }

int decode_token_tile(int M, int K) {
    if (M <= 16) return kBN_DEC;
    if (M > 128 || decode_kb(K) != 2) return 0;
    return M <= 32 ? 32 : M <= 64 ? 64 : 128;
}

template <bool NV>
static cudaError_t launch_dec_nv(const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& g, int num_sms,
                                 cudaStream_t st) {
    switch (decode_token_tile(g.M, g.K)) {
        case 16: return decode_kb(g.K) == 2 ? launch_dec_t<NV, 2, 16>(tmW, tmX, g, num_sms, st)
                                            : launch_dec_t<NV, 1, 16>(tmW, tmX, g, num_sms, st);
        case 32: return launch_dec_t<NV, 2, 32>(tmW, tmX, g, num_sms, st);
        case 64: return launch_dec_t<NV, 2, 64>(tmW, tmX, g, num_sms, st);
        case 128: return launch_dec_t<NV, 2, 128>(tmW, tmX, g, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_fp4_decode(bool nvfp4, const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& g,
                                   int num_sms, cudaStream_t st) {
    return nvfp4 ? launch_dec_nv<true>(tmW, tmX, g, num_sms, st) : launch_dec_nv<false>(tmW, tmX, g, num_sms, st);
}

}  // namespace w4a4
