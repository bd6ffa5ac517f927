// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace w4a4 {

// Per-device record that a kernel's dynamic shared-memory limit has been
// raised (cudaFuncSetAttribute acts on the current device); safe to share
// between host threads.
constexpr int kAttrDevices = 64;
struct SmemAttrCache {
    std::atomic<size_t> bytes[kAttrDevices] = {};
};
inline cudaError_t ensure_dynamic_smem(const void* func, size_t bytes, SmemAttrCache& c) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kAttrDevices) return cudaErrorInvalidDevice;
    if (bytes <= 48 * 1024 || c.bytes[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    size_t cur = c.bytes[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !c.bytes[dev].compare_exchange_weak(cur, bytes, std::memory_order_release)) {
    }
    return cudaSuccess;
}

enum { FMT_NVFP4 = 0, FMT_MXFP4 = 1, FMT_INT4 = 2 };

struct QuantArgs {
    const uint16_t* X;       // bf16 [rows][ldx]
    int M;                   // live rows
    int K;                   // columns to quantize (chunks of 16)
    int K_src;               // gather: columns >= K_src come from S (weights only)
    int ldx;
    const int32_t* S;        // gather map (weights only)
    uint8_t* codes;          // [M][ldc]
    int ldc;                 // bytes per codes row (= cols/2)
    uint8_t* sf;             // NVFP4/MXFP4 scales, MMA layout
    int sf_col_atoms;        // (cols / group) / 4
    float* sfi;              // INT4 scales [cols/128][sfi_ld]
    int sfi_ld;              // pad128(rows)
    int mode;                // NVFP4: 0 tensor, 1 token
    const float* static_s2;  // nullable
    float* s2_out;           // NVFP4 s2 ([1] or [M])
    const float* tensor_amax;  // NVFP4 tensor mode without static s2
    int rows_pad;              // pad128(M): rows of the scale atoms (set by the launcher)
    int* zero_words;           // nullable: words the first CTA clears (a later kernel's counters)
    int zero_count;
    int passes;                // MXFP4: 1, or more for the multi-pass decomposition (pass p
                               // in columns [p*K, (p+1)*K) of codes and scales)
    int group;                 // INT4: elements per scale group (128, 256 or 512)
    int int8_codes;            // INT4: write codes as int8 16 * q ([M][ldc] bytes, ldc >= K)
    int rot;                   // block-local Walsh-Hadamard rotation: 0 none, 1 activation
                               // side (times 1/block), 2 weight side (unscaled)
    const int32_t* res_S;      // NVFP4 per-token activations: the residual channels of the
    int res_n;                 // second stage, written at columns K .. K + res_n (0 = none)
};

// Whether the per-token NVFP4 quantizer can also compute the residual-channel
// second stage of a row (res_n channels of a K-column row) in the same launch.
bool nvfp4_token_fuses_residual(int K, int res_n);

struct ResidualArgs {
    const uint16_t* X;
    int M, K, ldx, rows_pad;
    const int32_t* S;
    int nS;
    uint8_t* codes;  // augmented codes [M][ldc]
    int ldc;
    uint8_t* sf;     // augmented scales, MMA layout
    int sf_col_atoms;
    const float* s2;
    int mode;
};

struct GemmArgs {
    int M, N, K;               // K = quantized columns (augmented included)
    const uint8_t* sfa;        // FP4 scales of A (MMA layout) / INT4: float [K/128][lda_s]
    const uint8_t* sfb;
    int sf_col_atoms;          // FP4: (K/group)/4
    int sfa_ld, sfb_ld;        // INT4: pad128(M), pad128(N)
    const float* s2a;          // NVFP4 alpha parts (nullable for MXFP4)
    int s2a_per_row;
    const float* s2b;          // NVFP4: [1], or [N] (16-byte aligned) when s2b_per_row
    int s2b_per_row;
    uint16_t* Y;
    int ldy;
    float* partial;            // split-K partial sums (decode variant)
    int* tile_count;           // decode variant: per weight tile, segments written so far (start at 0)
    int splits;                // split-K factor (decode variant)
    int k_tiles_per_split;
    int int4_group;            // INT4: elements per scale group (128, 256 or 512)
    int skip_k_tile;           // debug: never load this k-tile (-1 = off)
    unsigned long long wait_limit_ns;
};

cudaError_t launch_quant(int fmt, bool gather, const QuantArgs& a, int rows_pad, int num_sms, cudaStream_t st);
// NVFP4 TENSOR mode (dynamic scale, no gather, no rotation) in one
// cooperative launch of num_sms CTAs that hold all rows in shared memory:
// whether M x K fits, and the launch (a.tensor_amax and *arrive zero).
bool nvfp4_tensor_onepass_fits(int M, int K, int num_sms);
cudaError_t launch_nvfp4_tensor_onepass(const QuantArgs& a, int rows_pad, int num_sms, unsigned* arrive, bool pdl,
                                        cudaStream_t st);
// rot: 0 plain amax; 1 / 2 amax of the rotated 16-element blocks (activation / weight side)
cudaError_t launch_amax(const uint16_t* X, int M, int K, int ldx, float* out, int num_sms, cudaStream_t st,
                        int rot = 0);
cudaError_t launch_residual(const ResidualArgs& a, cudaStream_t st);
// p[1 .. n) = p[0] (device floats)
cudaError_t launch_spread_first(float* p, int n, cudaStream_t st);
cudaError_t launch_clear_tensor_amax(float* p, cudaStream_t st);
cudaError_t launch_select(const uint16_t* X, int Mc, int K, int ldx, int nS, int32_t* S, float* amax, int* sel,
                          cudaStream_t st);

// FP4 block-scaled GEMM (NVFP4 when nvfp4, else MXFP4).  tmA/tmB: byte tensor
// maps of the codes with a 128-byte swizzle and boxes of 128 x 128 (A) and
// 128 x bn (B) bytes.  pdl: launched as a programmatic dependent.
cudaError_t launch_gemm_fp4(bool nvfp4, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g,
                            int num_sms, bool pdl, cudaStream_t st);
// The same product on clusters of two CTAs (tcgen05 cta_group::2), 256 x 256
// output tiles: tmA/tmB boxes of 128 x 128 bytes (each CTA stages its half of
// A and of B), tmSA/tmSB 5-D maps over the scale atoms that repeat each atom
// four times (boxes of one stage's atoms for 1 (A) and 2 (B) row tiles).
cudaError_t launch_gemm_fp4_pair(bool nvfp4, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmSA,
                                 const CUtensorMap& tmSB, const GemmArgs& g, int num_sms, bool pdl, cudaStream_t st);
// Small-M variant (M <= 128): weights take the MMA's M side (128 rows per
// tile), the tokens its N side (decode_token_tile(M, K) rows); the (tile,
// K-stage) units are split evenly over the SMs, FP32 segment partials go to
// g.partial ([tiles][owners][token tile][128]) and the CTA that writes a
// tile's last segment adds them into Y (g.tile_count[N/128] must be zero on
// entry and is zero again on exit).  A programmatic dependent of the
// preceding launch.
cudaError_t launch_gemm_fp4_decode(bool nvfp4, const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& g,
                                   int num_sms, cudaStream_t st);
// Token tile (the MMA's N) of the small-M variant for M tokens and K
// columns: 16 for M <= 16; 32, 64 or 128 for 16 < M <= 128 when K is a
// multiple of 256; 0 when the variant does not apply.
int decode_token_tile(int M, int K);
// Partial-sum slots per weight tile of the small-M variant on `num_sms` SMs.
int decode_max_owners(int N, int K, int num_sms);
// K-stages of 256 per work unit of the small-M variant: 2 (weights and tokens
// read as 3-D boxes of two K-blocks) when K % 256 == 0, else 1 (2-D boxes).
int decode_k_blocks(int K);
// INT4-g128 GEMM on the 8-bit integer MMA with per-group FP32 rescaling.
// a8: A's codes are int8 (16 * q, row-major [M][K] bytes; tmA a 128-byte
// swizzled map with 128 x 128-byte boxes) instead of packed nibbles.
cudaError_t launch_gemm_int4(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& g, int num_sms,
                             bool pdl, cudaStream_t st, bool a8 = false);

// Tile shapes (shared with the host-side tensor-map set-up).
constexpr int kBM = 128;          // rows of A per tile
constexpr int kBN = 256;          // rows of B per tile (FP4)
constexpr int kBK_FP4 = 256;      // K elements per pipeline stage (128 bytes of codes)
constexpr int kBN_DEC = 16;       // token tile of the decode variant
constexpr int kBN_I4 = 128;       // rows of B per tile (INT4)
constexpr int kBK_I4 = 128;       // K elements per stage (one INT4 group)

}  // namespace w4a4
