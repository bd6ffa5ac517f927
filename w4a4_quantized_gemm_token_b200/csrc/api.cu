// C-ABI of the W4A4 library: argument checks, tensor-map set-up and dispatch
// to the kernels.  The library allocates no device memory; its only state is
// a per-device property cache, the driver entry point of the tensor-map
// encoder and the debug settings of w4a4_debug_set().
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/w4a4.h"
#include "kernels.h"
#include "ptx.cuh"

using namespace w4a4;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxK = 65536;
constexpr int kMaxPasses = 4;  // multi-pass MXFP4 decomposition
// Internal only (workspace tensors of w4a4_linear, never accepted from a
// caller): INT4 codes stored as int8 16 * q, [rows][cols] bytes, the layout
// the INT4 GEMM's MMA reads, so that its unpack warps widen only the weights.
constexpr int kFlagInt8Codes = 1 << 30;

struct DevInfo {
    bool init = false;
    bool ok = false;
    int num_sms = 0;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int g_skip_k_tile = -1;
unsigned long long g_wait_limit_ns = 2000000000ull;

int device_check(int* num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W4A4_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& d = g_dev[dev];
    if (!d.init) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return W4A4_ERR_CUDA;
        d.ok = (major == 10 && minor == 0);
        d.num_sms = sms;
        d.init = true;
    }
    if (!d.ok) return W4A4_ERR_ARCH;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return W4A4_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (num_sms) *num_sms = d.num_sms;
    return W4A4_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline int pad128(int x) { return (x + 127) / 128 * 128; }
inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int group_of(int fmt) { return fmt == W4A4_NVFP4 ? 16 : fmt == W4A4_MXFP4 ? 32 : fmt == W4A4_INT4 ? 128 : -1; }
// Group sizes a format accepts: its own, and for INT4 also 256 and 512 (the
// coarser scale groups of the rho-aware granularity).
bool group_ok(int fmt, int group) {
    return group == group_of(fmt) || (fmt == W4A4_INT4 && (group == 256 || group == 512));
}

// 2-D byte tensor map over codes[rows][row_bytes] with a box of box_x bytes x box_y rows.
int make_map(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_x, int box_y, bool swizzle128) {
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_y};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

// 3-D byte tensor map over codes[rows][row_bytes] (row_bytes a multiple of 128)
// seen as (128-byte K-block, row, K-block): a box of box_rows rows x box_kb
// consecutive K-blocks lands as box_kb 128-byte-swizzled [box_rows][128] tiles.
int make_map_kblocks(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_rows, int box_kb) {
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)(row_bytes / 128)};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, 128};
    cuuint32_t box[3] = {128, (cuuint32_t)box_rows, (cuuint32_t)box_kb};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

// 5-D byte tensor map over scale atoms [row_tiles][col_atoms][512 bytes] that
// repeats every atom 4 times: (256-byte half, half, repeat [stride 0], atom,
// row tile).  A box of box_atoms atoms x box_tiles row tiles lands as
// [tile][atom][repeat][512].
int make_map_sf_rep(CUtensorMap* map, const void* base, int row_tiles, int col_atoms, int box_atoms, int box_tiles) {
    cuuint64_t dims[5] = {256, 2, 4, (cuuint64_t)col_atoms, (cuuint64_t)row_tiles};
    cuuint64_t strides[4] = {256, 0, 512, (cuuint64_t)col_atoms * 512};
    cuuint32_t box[5] = {256, 2, 4, (cuuint32_t)box_atoms, (cuuint32_t)box_tiles};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W4A4_OK : W4A4_ERR_CUDA;
}

int check_qtensor(const w4a4_qtensor* q) {
    if (!q || !q->codes || !q->scales) return W4A4_ERR_INVALID_ARG;
    if (q->format < 0 || q->format > 2 || !group_ok(q->format, q->group) || (q->flags & ~W4A4_FLAG_HADAMARD))
        return W4A4_ERR_INVALID_ARG;
    if (q->rows < 0 || q->cols < 128 || q->cols % 128 || q->cols > kMaxPasses * kMaxK) return W4A4_ERR_INVALID_ARG;
    if (q->format == W4A4_INT4 && q->cols % q->group) return W4A4_ERR_INVALID_ARG;
    if (q->format == W4A4_NVFP4) {
        if (!q->s2) return W4A4_ERR_INVALID_ARG;
        if (q->scale_mode != W4A4_SCALE_TENSOR && q->scale_mode != W4A4_SCALE_TOKEN) return W4A4_ERR_INVALID_ARG;
    }
    if (!aligned16(q->codes) || !aligned16(q->scales) || (q->s2 && (reinterpret_cast<uintptr_t>(q->s2) & 3)))
        return W4A4_ERR_MISALIGNED;
    return W4A4_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA; }

// Quantize rows [0, M) of X into the first K columns of q (q->cols >= K).
// pad_scales: also write the zero scales of the padding rows [M, pad128(M))
// of the 128-row scale atoms (the public layout); the fused linear's
// workspace skips them, since every GEMM masks rows past M.
// res_S / res_n (NVFP4 activations with residual channels): when the
// per-token quantizer runs, it also writes the second stage into columns
// K .. K + res_n and *res_done is set; otherwise the caller runs it.
int quantize_rows(const uint16_t* X, int M, int K, int ldx, const int32_t* S, int K_src, const float* static_s2,
                  w4a4_qtensor* q, int num_sms, cudaStream_t st, int* zero_words = nullptr, int zero_count = 0,
                  int passes = 1, bool weight_side = false, bool pad_scales = true, const int32_t* res_S = nullptr,
                  int res_n = 0, bool* res_done = nullptr, bool chained = false) {
    const int rows_pad = pad_scales ? pad128(M) : M;
    if (res_done) *res_done = false;
    QuantArgs a{};
    a.passes = passes;
    a.rot = (q->flags & W4A4_FLAG_HADAMARD) ? (weight_side ? 2 : 1) : 0;
    a.zero_words = zero_words;
    a.zero_count = zero_count;
    a.X = X;
    a.M = M;
    a.K = K;
    a.K_src = K_src;
    a.ldx = ldx;
    a.S = S;
    a.codes = static_cast<uint8_t*>(q->codes);
    a.int8_codes = (q->flags & kFlagInt8Codes) ? 1 : 0;
    a.ldc = a.int8_codes ? q->cols : q->cols / 2;
    a.sf = static_cast<uint8_t*>(q->scales);
    a.sf_col_atoms = q->cols / q->group / 4;
    a.group = q->group;
    a.sfi = static_cast<float*>(q->scales);
    a.sfi_ld = pad128(q->rows);
    a.mode = q->scale_mode;
    a.static_s2 = static_s2;
    a.s2_out = q->s2;
    a.tensor_amax = nullptr;
    if (q->format == W4A4_NVFP4 && q->scale_mode == W4A4_SCALE_TENSOR && !static_s2) {
        // dynamic tensor scale: s2[1] collects the amax (s2[2] counts the CTAs
        // of the one-pass kernel); one cooperative pass when all rows fit in
        // shared memory, else an amax pass and the quantizer
        // Inside the fused linear (chained: a GEMM follows) the two words are
        // cleared by a kernel that is a programmatic dependent of the
        // preceding launch, and the one-pass quantizer is one too, so their
        // launches overlap the preceding GEMM's tail (SwiGLU layer 145 -> 141
        // us); alone, a memset and a plain cooperative launch cost less.
        cudaError_t e = chained ? launch_clear_tensor_amax(q->s2 + 1, st)
                                : cudaMemsetAsync(q->s2 + 1, 0, 2 * sizeof(float), st);
        if (e != cudaSuccess) return W4A4_ERR_CUDA;
        a.tensor_amax = q->s2 + 1;
        if (!S && K == K_src && !a.rot && passes == 1 && !a.int8_codes && nvfp4_tensor_onepass_fits(M, K, num_sms)) {
            e = launch_nvfp4_tensor_onepass(a, rows_pad, num_sms, reinterpret_cast<unsigned*>(q->s2 + 2), chained, st);
            if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_status(e);
            cudaGetLastError();  // fewer SMs available than reported: two passes
        }
        e = launch_amax(X, M, K_src, ldx, q->s2 + 1, num_sms, st, a.rot);
        if (e != cudaSuccess) return W4A4_ERR_CUDA;
    }
    // the per-token kernel (the path launch_quant takes for these arguments)
    // can fuse the residual-channel stage
    if (res_n && q->format == W4A4_NVFP4 && !S && !static_s2 && !a.rot && passes == 1 && !a.int8_codes &&
        K == K_src && K <= 49152 && nvfp4_token_fuses_residual(K, res_n)) {
        a.res_S = res_S;
        a.res_n = res_n;
        if (res_done) *res_done = true;
    }
    return cuda_status(launch_quant(q->format, S != nullptr, a, rows_pad, num_sms, st));
}

// NVFP4 weights with one s2 per row (per-segment scales): the GEMM epilogues
// read four consecutive row scales at a time.
int check_weight_s2(const w4a4_qtensor* B) {
    if (B->format == W4A4_NVFP4 && B->scale_mode == W4A4_SCALE_TOKEN && !aligned16(B->s2)) return W4A4_ERR_MISALIGNED;
    return W4A4_OK;
}

int check_S_args(const int32_t* S, int nS, int K) {
    if (nS < 0 || (nS > 0 && (!S || nS % 128 || nS > K))) return W4A4_ERR_INVALID_ARG;
    if (nS == 0 && S) return W4A4_ERR_INVALID_ARG;
    return W4A4_OK;
}

// The split-K small-M kernel (weights on the MMA's M side, every SM streaming
// its share of the weights) or the tiled kernels (tokens on the M side, one
// 128/256-row token tile against 256-row weight tiles), by the crossover
// measured on the Llama-2-70B layer: the small-M kernel for M <= 16; for
// 16 < M <= 64 unless N / 256 weight tiles already occupy every SM; for
// 64 < M <= 128 only where the tiled kernel would run at most 32 long tiles
// (K >= 16384) on as many SMs.  The small-M kernel pays an FP32 partial sum
// per tile segment, which outweighs its parallelism beyond that.
bool use_small_m(int fmt, int M, int N, int cols, int num_sms) {
    if (fmt == W4A4_INT4 || decode_token_tile(M, cols) == 0) return false;
    if (M <= 16) return true;
    const int tiles = (N + kBN - 1) / kBN;
    if (M <= 64) return tiles < num_sms / 2;
    if (M <= 128) return tiles <= 32 && cols >= 16384;
    return false;
}

struct GemmSetup {
    CUtensorMap ta, tb, tsa, tsb;  // codes of A and B; scale atoms (pair kernel)
    GemmArgs g;
};

// Large-M FP4 products run on CTA pairs (256 x 256 tiles); up to 128 rows of A
// the one-CTA kernel (128 x 256 tiles) wastes no MMA rows.
inline bool use_pair(const w4a4_qtensor* A) { return A->format != W4A4_INT4 && A->rows > kBM; }

// Fill tensor maps and arguments for A (activations) x B (weights).
int setup_gemm(const w4a4_qtensor* A, const w4a4_qtensor* B, uint16_t* Y, int ldy, bool decode, GemmSetup* s) {
    GemmArgs& g = s->g;
    std::memset(&g, 0, sizeof(g));
    g.M = A->rows;
    g.N = B->rows;
    g.K = A->cols;
    g.sfa = static_cast<const uint8_t*>(A->scales);
    g.sfb = static_cast<const uint8_t*>(B->scales);
    g.sf_col_atoms = A->format == W4A4_INT4 ? 0 : A->cols / A->group / 4;
    g.int4_group = A->group;
    g.sfa_ld = pad128(A->rows);
    g.sfb_ld = pad128(B->rows);
    g.s2a = A->s2;
    g.s2a_per_row = A->scale_mode == W4A4_SCALE_TOKEN ? 1 : 0;
    g.s2b = B->s2;
    g.s2b_per_row = B->format == W4A4_NVFP4 && B->scale_mode == W4A4_SCALE_TOKEN ? 1 : 0;
    g.Y = Y;
    g.ldy = ldy;
    g.skip_k_tile = g_skip_k_tile;
    g.wait_limit_ns = g_wait_limit_ns;
    const int row_bytes = A->cols / 2;
    int rc;
    if (A->format == W4A4_INT4) {
        if (A->flags & kFlagInt8Codes)
            rc = make_map(&s->ta, A->codes, A->rows, A->cols, 128, 128, true);
        else
            rc = make_map(&s->ta, A->codes, A->rows, row_bytes, 64, 128, false);
        if (rc == W4A4_OK) rc = make_map(&s->tb, B->codes, B->rows, row_bytes, 64, kBN_I4, false);
    } else if (!decode && use_pair(A)) {
        // each CTA of a pair stages 128 rows of A and 128 rows of B
        const int atoms_ps = A->format == W4A4_NVFP4 ? 4 : 2;
        rc = make_map(&s->ta, A->codes, A->rows, row_bytes, 128, kBM, true);
        if (rc == W4A4_OK) rc = make_map(&s->tb, B->codes, B->rows, row_bytes, 128, kBM, true);
        if (rc == W4A4_OK)
            rc = make_map_sf_rep(&s->tsa, A->scales, pad128(A->rows) / 128, g.sf_col_atoms, atoms_ps, 1);
        if (rc == W4A4_OK)
            rc = make_map_sf_rep(&s->tsb, B->scales, pad128(B->rows) / 128, g.sf_col_atoms, atoms_ps, 2);
    } else if (!decode) {
        rc = make_map(&s->ta, A->codes, A->rows, row_bytes, 128, kBM, true);
        if (rc == W4A4_OK) rc = make_map(&s->tb, B->codes, B->rows, row_bytes, 128, kBN, true);
    } else if (decode_k_blocks(A->cols) == 2) {
        // weights take the MMA's M side (128 rows), tokens its N side (the token
        // tile's rows); both read as boxes of two consecutive 128-byte K-blocks per row
        rc = make_map_kblocks(&s->ta, B->codes, B->rows, row_bytes, kBM, 2);
        if (rc == W4A4_OK)
            rc = make_map_kblocks(&s->tb, A->codes, A->rows, row_bytes, decode_token_tile(A->rows, A->cols), 2);
    } else {
        // weights take the MMA's M side (box of 128 rows), tokens its N side (16 rows)
        rc = make_map(&s->ta, B->codes, B->rows, row_bytes, 128, kBM, true);
        if (rc == W4A4_OK) rc = make_map(&s->tb, A->codes, A->rows, row_bytes, 128, kBN_DEC, true);
    }
    return rc;
}

int run_gemm(const w4a4_qtensor* A, const w4a4_qtensor* B, uint16_t* Y, int ldy, float* partial, int num_sms,
             bool pdl, cudaStream_t st, int* tile_count = nullptr) {
    const bool decode = A->format != W4A4_INT4 && partial != nullptr;
    GemmSetup s;
    int rc = setup_gemm(A, B, Y, ldy, decode, &s);
    if (rc != W4A4_OK) return rc;
    cudaError_t e;
    if (A->format == W4A4_INT4) {
        e = launch_gemm_int4(s.ta, s.tb, s.g, num_sms, pdl, st, (A->flags & kFlagInt8Codes) != 0);
    } else if (decode) {
        s.g.partial = partial;
        s.g.tile_count = tile_count;
        e = launch_gemm_fp4_decode(A->format == W4A4_NVFP4, s.ta, s.tb, s.g, num_sms, st);
    } else if (use_pair(A)) {
        e = launch_gemm_fp4_pair(A->format == W4A4_NVFP4, s.ta, s.tb, s.tsa, s.tsb, s.g, num_sms, pdl, st);
    } else {
        e = launch_gemm_fp4(A->format == W4A4_NVFP4, s.ta, s.tb, s.g, num_sms, pdl, st);
    }
    return cuda_status(e);
}

// Workspace layout of w4a4_linear: quantized activation (codes, scales, s2),
// then the split-K partial sums of the small-M variant.
struct WsLayout {
    size_t codes, scales, s2, partial, counters, total;
};

WsLayout ws_layout(int M, int N, int K, int fmt, int nS) {
    WsLayout w{};
    const int cols = K + nS;
    size_t cb = 0, sb = 0, s2b = 0;
    w4a4_qtensor_bytes(fmt, M, cols, W4A4_SCALE_TOKEN, &cb, &sb, &s2b);
    if (fmt == W4A4_INT4) cb *= 2;  // the linear keeps INT4 activations widened to int8
    if (s2b < 8) s2b = 8;
    w.codes = 0;
    w.scales = align256(cb);
    w.s2 = w.scales + align256(sb);
    w.partial = w.s2 + align256(s2b);
    size_t pb = 0;
    // sized for the small-M variant whenever it can be chosen (on any SM count)
    const bool small_m = use_small_m(fmt, M, N, cols, 1 << 20);
    if (small_m) {
        // FP32 segment partials of the small-M variant: [tiles][owners][token
        // tile][128]; the owner count grows with the SM count, bounded here for
        // up to 1024 SMs
        const int ntiles = (N + kBM - 1) / kBM;
        pb = (size_t)ntiles * decode_max_owners(N, cols, 1024) * decode_token_tile(M, cols) * kBM * sizeof(float);
    }
    w.counters = w.partial + align256(pb);
    const size_t nb = small_m ? (size_t)((N + kBM - 1) / kBM) * sizeof(int) : 0;
    w.total = w.counters + align256(nb);
    return w;
}

}  // namespace

extern "C" {

const char* w4a4_status_string(int status) {
    switch (status) {
        case W4A4_OK: return "ok";
        case W4A4_ERR_INVALID_ARG: return "invalid argument";
        case W4A4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
        case W4A4_ERR_WORKSPACE: return "workspace missing or too small";
        case W4A4_ERR_ARCH: return "device is not sm_100";
        case W4A4_ERR_CUDA: return "CUDA error";
        case W4A4_ERR_DEVICE_TIMEOUT: return "in-kernel wait timed out";
        default: return "unknown status";
    }
}

int w4a4_qtensor_bytes(int format, int rows, int cols, int scale_mode, size_t* codes_bytes, size_t* scales_bytes,
                       size_t* s2_bytes) {
    const int g = group_of(format);
    if (g < 0 || rows < 0 || cols < 0 || cols % 128) return W4A4_ERR_INVALID_ARG;
    size_t c = (size_t)rows * (cols / 2);
    size_t s = format == W4A4_INT4 ? (size_t)(cols / 128) * pad128(rows) * sizeof(float)
                                   : (size_t)pad128(rows) * (cols / g);
    size_t t = 0;
    if (format == W4A4_NVFP4) t = scale_mode == W4A4_SCALE_TOKEN ? (size_t)(rows > 0 ? rows : 1) * 4 : 16;
    if (codes_bytes) *codes_bytes = c;
    if (scales_bytes) *scales_bytes = s;
    if (s2_bytes) *s2_bytes = t;
    return W4A4_OK;
}

int w4a4_quantize_act(const uint16_t* X, int M, int K, int ldx, int format, int group, int scale_mode,
                      const float* static_s2, w4a4_qtensor* out, void* stream) {
    if (M < 0 || K < 128 || K % 128 || K > kMaxK || ldx < K) return W4A4_ERR_INVALID_ARG;
    if (!group_ok(format, group) || K % group) return W4A4_ERR_INVALID_ARG;
    int rc = check_qtensor(out);
    if (rc != W4A4_OK) return rc;
    if (out->format != format || out->group != group || out->rows != M || out->cols < K ||
        (format == W4A4_NVFP4 && out->scale_mode != scale_mode))
        return W4A4_ERR_INVALID_ARG;
    if (format != W4A4_NVFP4 && static_s2) return W4A4_ERR_INVALID_ARG;
    if (M == 0) return W4A4_OK;
    if (!X) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(X) || ldx % 8) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    return quantize_rows(X, M, K, ldx, nullptr, K, static_s2, out, sms, as_stream(stream));
}

int w4a4_quantize_weight(const uint16_t* W, int N, int K, int ldw, int format, int group, const int32_t* S, int nS,
                         w4a4_qtensor* out, void* stream) {
    if (N < 0 || K < 128 || K % 128 || K > kMaxK || ldw < K) return W4A4_ERR_INVALID_ARG;
    if (!group_ok(format, group) || K % group) return W4A4_ERR_INVALID_ARG;
    int rc = check_S_args(S, nS, K);
    if (rc != W4A4_OK) return rc;
    rc = check_qtensor(out);
    if (rc != W4A4_OK) return rc;
    if (out->format != format || out->group != group || out->rows != N || out->cols != K + nS)
        return W4A4_ERR_INVALID_ARG;
    if (format == W4A4_NVFP4 && out->scale_mode != W4A4_SCALE_TENSOR) return W4A4_ERR_INVALID_ARG;
    if (nS && out->flags) return W4A4_ERR_INVALID_ARG;
    if (N == 0) return W4A4_OK;
    if (!W) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(W) || ldw % 8) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    return quantize_rows(W, N, K + nS, ldw, nS ? S : nullptr, K, nullptr, out, sms, as_stream(stream), nullptr, 0, 1,
                         true);
}

int w4a4_quantize_weight_segments(const uint16_t* W, int N, int K, int ldw, const int32_t* seg, int nseg,
                                  const int32_t* S, int nS, w4a4_qtensor* out, void* stream) {
    if (N < 0 || K < 128 || K % 128 || K > kMaxK || ldw < K) return W4A4_ERR_INVALID_ARG;
    if (!seg || nseg < 1 || seg[0] != 0 || seg[nseg] != N) return W4A4_ERR_INVALID_ARG;
    for (int i = 0; i < nseg; ++i)
        if (seg[i + 1] <= seg[i] || seg[i + 1] % 128) return W4A4_ERR_INVALID_ARG;
    int rc = check_S_args(S, nS, K);
    if (rc != W4A4_OK) return rc;
    rc = check_qtensor(out);
    if (rc != W4A4_OK) return rc;
    if (out->format != W4A4_NVFP4 || out->scale_mode != W4A4_SCALE_TOKEN || out->rows != N || out->cols != K + nS)
        return W4A4_ERR_INVALID_ARG;
    if (nS && out->flags) return W4A4_ERR_INVALID_ARG;
    rc = check_weight_s2(out);
    if (rc != W4A4_OK) return rc;
    if (!W) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(W) || ldw % 8) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    cudaStream_t st = as_stream(stream);
    const int cols = K + nS;
    for (int i = 0; i < nseg; ++i) {
        // the segment as a tensor of its own: rows r0..r1 of codes, its 128-row
        // scale atoms, and s2[r0] as its tensor scale (s2[r0 + 1], s2[r0 + 2]
        // are its scratch, inside the segment's rows and overwritten by the
        // spread below)
        const int r0 = seg[i], rows = seg[i + 1] - seg[i];
        w4a4_qtensor q = *out;
        q.rows = rows;
        q.scale_mode = W4A4_SCALE_TENSOR;
        q.codes = static_cast<uint8_t*>(out->codes) + (size_t)r0 * (cols / 2);
        q.scales = static_cast<uint8_t*>(out->scales) + (size_t)(r0 / 128) * (cols / 16 / 4) * 512;
        q.s2 = out->s2 + r0;
        rc = quantize_rows(W + (size_t)r0 * ldw, rows, cols, ldw, nS ? S : nullptr, K, nullptr, &q, sms, st, nullptr, 0,
                           1, true);
        if (rc != W4A4_OK) return rc;
        if (launch_spread_first(q.s2, rows, st) != cudaSuccess) return W4A4_ERR_CUDA;
    }
    return W4A4_OK;
}

int w4a4_quantize_act_msd(const uint16_t* X, int M, int K, int ldx, int passes, w4a4_qtensor* out, void* stream) {
    if (M < 0 || K < 128 || K % 128 || K > kMaxK || ldx < K || passes < 1 || passes > kMaxPasses)
        return W4A4_ERR_INVALID_ARG;
    int rc = check_qtensor(out);
    if (rc != W4A4_OK) return rc;
    if (out->format != W4A4_MXFP4 || out->rows != M || out->cols != passes * K || out->flags)
        return W4A4_ERR_INVALID_ARG;
    if (M == 0) return W4A4_OK;
    if (!X) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(X) || ldx % 8) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    return quantize_rows(X, M, K, ldx, nullptr, K, nullptr, out, sms, as_stream(stream), nullptr, 0, passes);
}

// The weight side of the multi-pass product: W quantized once into the first
// K columns, then copied into the other passes' columns (codes row by row,
// scale atoms row tile by row tile).
int w4a4_quantize_weight_msd(const uint16_t* W, int N, int K, int ldw, int passes, w4a4_qtensor* out, void* stream) {
    if (N < 0 || K < 128 || K % 128 || K > kMaxK || ldw < K || passes < 1 || passes > kMaxPasses)
        return W4A4_ERR_INVALID_ARG;
    int rc = check_qtensor(out);
    if (rc != W4A4_OK) return rc;
    if (out->format != W4A4_MXFP4 || out->rows != N || out->cols != passes * K || out->flags)
        return W4A4_ERR_INVALID_ARG;
    if (N == 0) return W4A4_OK;
    if (!W) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(W) || ldw % 8) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    cudaStream_t st = as_stream(stream);
    rc = quantize_rows(W, N, K, ldw, nullptr, K, nullptr, out, sms, st);
    if (rc != W4A4_OK) return rc;
    uint8_t* codes = static_cast<uint8_t*>(out->codes);
    uint8_t* scales = static_cast<uint8_t*>(out->scales);
    const size_t row_b = (size_t)passes * K / 2, part_b = (size_t)K / 2;
    const size_t atoms = (size_t)K / 32 / 4, tile_b = (size_t)passes * atoms * 512;
    for (int p = 1; p < passes; ++p) {
        cudaError_t e = cudaMemcpy2DAsync(codes + p * part_b, row_b, codes, row_b, part_b, N, cudaMemcpyDeviceToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(scales + p * atoms * 512, tile_b, scales, tile_b, atoms * 512, pad128(N) / 128,
                                  cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return W4A4_ERR_CUDA;
    }
    return W4A4_OK;
}

int w4a4_gemm(const w4a4_qtensor* A, const w4a4_qtensor* B, uint16_t* Y, int ldy, void* stream) {
    int rc = check_qtensor(A);
    if (rc == W4A4_OK) rc = check_qtensor(B);
    if (rc != W4A4_OK) return rc;
    if (A->format != B->format || A->cols != B->cols || B->rows < 128 || B->rows % 128 || ldy < B->rows ||
        A->flags != B->flags || A->group != B->group)
        return W4A4_ERR_INVALID_ARG;
    rc = check_weight_s2(B);
    if (rc != W4A4_OK) return rc;
    if (A->rows == 0) return W4A4_OK;
    if (!Y) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(Y) || ldy % 8) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    return run_gemm(A, B, Y, ldy, nullptr, sms, false, as_stream(stream));
}

int w4a4_int4_group_for_rho(double rho) {
    // rescales per tensor-core step scale as 1/G: keep them in step with the
    // MMAs as rho grows past the value (16) where g128 still pays
    if (!(rho > 0.0)) return 128;
    int g = 128;
    while (g < 512 && rho > 16.0 * (g / 128)) g *= 2;
    return g;
}

size_t w4a4_linear_workspace(int M, int N, int K, int format, int nS) {
    if (M < 0 || N < 128 || N % 128 || K < 128 || K % 128 || group_of(format) < 0 || nS < 0 || nS % 128)
        return 0;
    return ws_layout(M, N, K, format, nS).total;
}

int w4a4_linear(const uint16_t* X, int M, int K, int ldx, const w4a4_qtensor* Wq, int scale_mode, const int32_t* S,
                int nS, uint16_t* Y, int ldy, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_qtensor(Wq);
    if (rc != W4A4_OK) return rc;
    const int fmt = Wq->format;
    if (M < 0 || K < 128 || K % 128 || K > kMaxK || ldx < K) return W4A4_ERR_INVALID_ARG;
    rc = check_S_args(S, nS, K);
    if (rc != W4A4_OK) return rc;
    if (nS && (fmt != W4A4_NVFP4 || Wq->flags)) return W4A4_ERR_INVALID_ARG;
    if (Wq->cols != K + nS || Wq->rows < 128 || Wq->rows % 128 || ldy < Wq->rows) return W4A4_ERR_INVALID_ARG;
    if (fmt == W4A4_NVFP4 && scale_mode != W4A4_SCALE_TENSOR && scale_mode != W4A4_SCALE_TOKEN)
        return W4A4_ERR_INVALID_ARG;
    rc = check_weight_s2(Wq);
    if (rc != W4A4_OK) return rc;
    if (M == 0) return W4A4_OK;
    if (!X || !Y) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(X) || ldx % 8 || !aligned16(Y) || ldy % 8) return W4A4_ERR_MISALIGNED;
    const int N = Wq->rows;
    const WsLayout L = ws_layout(M, N, K, fmt, nS);
    if (!ws || ws_bytes < L.total) return W4A4_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    cudaStream_t st = as_stream(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    w4a4_qtensor xq{};
    xq.format = fmt;
    xq.rows = M;
    xq.cols = K + nS;
    xq.group = fmt == W4A4_INT4 ? Wq->group : group_of(fmt);  // INT4: the weights' scale groups
    xq.scale_mode = fmt == W4A4_NVFP4 ? scale_mode : 0;
    xq.flags = Wq->flags;  // rotated weights: rotate the activations the same way
    if (fmt == W4A4_INT4) xq.flags |= kFlagInt8Codes;
    xq.codes = base + L.codes;
    xq.scales = base + L.scales;
    xq.s2 = reinterpret_cast<float*>(base + L.s2);
    const bool small_m = use_small_m(fmt, M, N, xq.cols, sms);
    int* counters = small_m ? reinterpret_cast<int*>(base + L.counters) : nullptr;
    // the quantizer clears the decode GEMM's per-tile counters on its way
    bool res_done = false;
    rc = quantize_rows(X, M, K, ldx, nullptr, K, nullptr, &xq, sms, st, counters, small_m ? (N + kBM - 1) / kBM : 0,
                       1, false, false, nS ? S : nullptr, nS, &res_done, true);
    if (rc != W4A4_OK) return rc;
    if (nS && !res_done) {
        ResidualArgs r{X, M, K, ldx, pad128(M), S, nS, static_cast<uint8_t*>(xq.codes), xq.cols / 2,
                       static_cast<uint8_t*>(xq.scales), xq.cols / 16 / 4, xq.s2, xq.scale_mode};
        if (launch_residual(r, st) != cudaSuccess) return W4A4_ERR_CUDA;
    }
    float* partial = small_m ? reinterpret_cast<float*>(base + L.partial) : nullptr;
    return run_gemm(&xq, Wq, Y, ldy, partial, sms, true, st, counters);
}

int w4a4_linear_msd(const uint16_t* X, int M, int K, int ldx, const w4a4_qtensor* Wq, int passes, uint16_t* Y,
                    int ldy, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_qtensor(Wq);
    if (rc != W4A4_OK) return rc;
    if (M < 0 || K < 128 || K % 128 || K > kMaxK || ldx < K || passes < 1 || passes > kMaxPasses)
        return W4A4_ERR_INVALID_ARG;
    if (Wq->format != W4A4_MXFP4 || Wq->cols != passes * K || Wq->rows < 128 || Wq->rows % 128 || ldy < Wq->rows ||
        Wq->flags)
        return W4A4_ERR_INVALID_ARG;
    if (M == 0) return W4A4_OK;
    if (!X || !Y) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(X) || ldx % 8 || !aligned16(Y) || ldy % 8) return W4A4_ERR_MISALIGNED;
    const int N = Wq->rows;
    const WsLayout L = ws_layout(M, N, K, W4A4_MXFP4, (passes - 1) * K);
    if (!ws || ws_bytes < L.total) return W4A4_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return W4A4_ERR_MISALIGNED;
    int sms = 0;
    rc = device_check(&sms);
    if (rc != W4A4_OK) return rc;
    cudaStream_t st = as_stream(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    w4a4_qtensor xq{};
    xq.format = W4A4_MXFP4;
    xq.rows = M;
    xq.cols = passes * K;
    xq.group = 32;
    xq.codes = base + L.codes;
    xq.scales = base + L.scales;
    xq.s2 = nullptr;
    const bool small_m = use_small_m(W4A4_MXFP4, M, N, xq.cols, sms);
    int* counters = small_m ? reinterpret_cast<int*>(base + L.counters) : nullptr;
    rc = quantize_rows(X, M, K, ldx, nullptr, K, nullptr, &xq, sms, st, counters, small_m ? (N + kBM - 1) / kBM : 0,
                       passes, false, false);
    if (rc != W4A4_OK) return rc;
    float* partial = small_m ? reinterpret_cast<float*>(base + L.partial) : nullptr;
    return run_gemm(&xq, Wq, Y, ldy, partial, sms, true, st, counters);
}

int w4a4_augment_residual(const uint16_t* X, int M, int K, int ldx, const int32_t* S, int nS, w4a4_qtensor* Xaug,
                          void* stream) {
    if (M < 0 || K < 128 || K % 128 || K > kMaxK || ldx < K || nS <= 0) return W4A4_ERR_INVALID_ARG;
    int rc = check_S_args(S, nS, K);
    if (rc == W4A4_OK) rc = check_qtensor(Xaug);
    if (rc != W4A4_OK) return rc;
    if (Xaug->format != W4A4_NVFP4 || Xaug->rows != M || Xaug->cols != K + nS || Xaug->flags)
        return W4A4_ERR_INVALID_ARG;
    if (M == 0) return W4A4_OK;
    if (!X) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(X) || ldx % 8) return W4A4_ERR_MISALIGNED;
    rc = device_check(nullptr);
    if (rc != W4A4_OK) return rc;
    ResidualArgs r{X, M, K, ldx, pad128(M), S, nS, static_cast<uint8_t*>(Xaug->codes), Xaug->cols / 2,
                   static_cast<uint8_t*>(Xaug->scales), Xaug->cols / 16 / 4, Xaug->s2, Xaug->scale_mode};
    return cuda_status(launch_residual(r, as_stream(stream)));
}

int w4a4_select_channels(const uint16_t* Xcal, int Mc, int K, int ldx, int nS, int32_t* S_out, void* ws,
                         size_t ws_bytes, void* stream) {
    if (Mc < 1 || K < 1 || ldx < K || nS < 0 || nS > K || !Xcal || (nS > 0 && !S_out)) return W4A4_ERR_INVALID_ARG;
    if (!ws || ws_bytes < (size_t)K * 8) return W4A4_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 15) return W4A4_ERR_MISALIGNED;
    int rc = device_check(nullptr);
    if (rc != W4A4_OK) return rc;
    if (nS == 0) return W4A4_OK;
    float* amax = static_cast<float*>(ws);
    int* sel = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + (size_t)K * 4);
    return cuda_status(launch_select(Xcal, Mc, K, ldx, nS, S_out, amax, sel, as_stream(stream)));
}

int w4a4_device_status(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return W4A4_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return W4A4_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return W4A4_ERR_CUDA;
        return v == kErrTimeout ? W4A4_ERR_DEVICE_TIMEOUT : v == kErrBadIndex ? W4A4_ERR_INVALID_ARG : W4A4_ERR_CUDA;
    }
    return W4A4_OK;
}

void w4a4_debug_set(int skip_k_tile, unsigned long long wait_limit_ns) {
    g_skip_k_tile = skip_k_tile < 0 ? -1 : skip_k_tile;
    g_wait_limit_ns = wait_limit_ns ? wait_limit_ns : 2000000000ull;
}

}  // extern "C"
