/*
 * w4a4.h -- C-ABI of the B200 (sm_100a) W4A4 quantized linear layer.
 *
 * The operation: a linear layer Y[M,N] = X[M,K] * W[N,K]^T whose activations
 * X (bf16) are quantized to 4 bits on the fly, per token, and whose weights W
 * are quantized to 4 bits once, offline; the 4-bit x 4-bit product applies
 * the block scales, accumulates in FP32 and writes bf16.  Passages defining
 * it (page title, paragraph):
 *   - "Depth Registers Unlock W4A4 on SwiGLU: A Reader/Generator
 *     Decomposition" (mlsanity page), abstract: post-training W4A4,
 *     round-to-nearest quantization of every linear's input activations.
 *   - "Depth Registers..." (thelatestinai page), para 2 (APEX4): W4A4-g128
 *     INT4 GEMM whose per-group dequantization runs on the CUDA cores;
 *     para 1: open-standard MXFP4.
 *   - "Daily Papers", para 4 (Minima): NVFP4 W4A4 with 16-element block
 *     scaling, a global scale, per-token activation quantization.
 *   - "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute
 *     Rebalancing" page, para 2 (ARCQuant): residual channels quantized to
 *     NVFP4 and appended to the activation along the reduction dimension,
 *     the matching weight columns duplicated, one standard NVFP4 GEMM.
 *
 * Formats (the bit-level rules are those of the public OCP Microscaling /
 * NVFP4 definitions the paragraphs above name):
 *   W4A4_NVFP4  E2M1 elements, one E4M3 scale per 16 elements along K, one
 *               FP32 second-level scale per tensor or per row (token).
 *   W4A4_MXFP4  E2M1 elements, one E8M0 (power of two) scale per 32.
 *   W4A4_INT4   4-bit two's-complement integers, one FP32 scale amax/7 per
 *               128 elements along K (symmetric, round to nearest even).
 *
 * Conventions for every entry point:
 *   - bf16 tensors are uint16_t bit patterns, row-major, leading dimension in
 *     elements; pointers to them are DEVICE pointers.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).  All
 *     device work is asynchronous on it; nothing synchronizes except
 *     w4a4_device_status().
 *   - The library allocates no device memory.  The caller owns every buffer,
 *     including the workspace of w4a4_linear.  w4a4_qtensor descriptors are
 *     host structs whose pointer members point to device memory.
 *   - Entry points return a W4A4_* status and never abort or print.  On an
 *     argument error nothing is launched.
 *   - Shapes: M >= 0 (M == 0 is a no-op), N and K multiples of 128,
 *     K <= 65536.  Device pointers 16-byte aligned; leading dimensions
 *     multiples of 8 elements.
 */
#ifndef W4A4_H
#define W4A4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define W4A4_OK                 0
#define W4A4_ERR_INVALID_ARG    1  /* null pointer, bad shape, format/group mismatch, S invalid */
#define W4A4_ERR_MISALIGNED     2  /* pointer not 16-byte aligned or leading dim not a multiple of 8 */
#define W4A4_ERR_WORKSPACE      3  /* workspace missing or smaller than w4a4_linear_workspace() */
#define W4A4_ERR_ARCH           4  /* current device is not sm_100 */
#define W4A4_ERR_CUDA           5  /* a CUDA runtime/driver call or a launch failed */
#define W4A4_ERR_DEVICE_TIMEOUT 6  /* a bounded in-kernel wait expired (read by w4a4_device_status) */

/* ---- formats ------------------------------------------------------------ */
#define W4A4_NVFP4 0   /* group 16 */
#define W4A4_MXFP4 1   /* group 32 */
#define W4A4_INT4  2   /* group 128 */

/* w4a4_qtensor.flags */
#define W4A4_FLAG_HADAMARD 1  /* each quantization block (16 / 32 / 128 elements along K) was
                                 rotated by a Walsh-Hadamard matrix before quantization */

/* NVFP4 second-level scale granularity */
#define W4A4_SCALE_TENSOR 0  /* one FP32 scale for the whole tensor */
#define W4A4_SCALE_TOKEN  1  /* one FP32 scale per row (per token) */

/*
 * A quantized tensor of `rows` x `cols` elements (cols along K).
 *
 * codes   [rows][cols/2] bytes: element 2j in the low nibble of byte j.
 * scales  NVFP4: E4M3 bytes, MXFP4: E8M0 bytes, both in the layout the
 *         block-scaled tensor-core MMA reads: 512-byte atoms of 128 rows x 4
 *         consecutive scales, the scale of (row r, block c) at byte
 *           ((r/128) * (cols/g/4) + c/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + c%4
 *         (g = 16 or 32); rows are padded to a multiple of 128 with zero
 *         scales.  INT4: FP32, group-major [cols/group][pad128(rows)], the
 *         scale of (row r, group c) at index c * pad128(rows) + r.
 * s2      NVFP4 only: FP32 second-level scales; TENSOR: s2[0] is the scale and
 *         s2[1..3] are scratch (the tensor amax, the one-pass quantizer's CTA
 *         count); TOKEN: s2[r] per row.
 *
 * An "augmented" activation tensor has cols = K + nS: its first K columns
 * come from w4a4_quantize_act, the last nS from w4a4_augment_residual.
 *
 * W4A4_FLAG_HADAMARD (block-local rotation: the "Depth Registers Unlock W4A4
 * on SwiGLU" (mlsanity) abstract names QuaRot's Hadamard rotations; the
 * "APEX4..." page, para 2 (ARCQuant) notes that full rotations compromise
 * block isolation, so here each quantization block is rotated on its own).
 * When set on the output of a quantizer, each n-element block along K (n = 16
 * NVFP4, 32 MXFP4, 128 INT4) is first transformed by the fast Walsh-Hadamard
 * butterflies in FP32 (stages h = 1, 2, ..., n/2, (a, b) -> (a + b, a - b),
 * Sylvester order), then quantized by the format's rule (NVFP4 amaxes, per
 * token or per tensor, are those of the rotated values).  Activations
 * (w4a4_quantize_act, w4a4_linear) are also multiplied by 1/n; weights
 * (w4a4_quantize_weight, w4a4_quantize_weight_segments) are not, so that the
 * product of a rotated activation and a rotated weight is X W^T unchanged
 * (H H^T = n I): the GEMM needs no change.  w4a4_gemm requires both operands
 * to carry the same flag; w4a4_linear rotates the activations when Wq
 * carries it.  Not combined with residual channels (nS > 0) nor with the
 * multi-pass decomposition (those calls return W4A4_ERR_INVALID_ARG).
 */
typedef struct w4a4_qtensor {
    int32_t format;      /* W4A4_NVFP4 / W4A4_MXFP4 / W4A4_INT4 */
    int32_t rows;
    int32_t cols;
    int32_t group;       /* 16 (NVFP4) / 32 (MXFP4) / 128, 256 or 512 (INT4; cols % group == 0) */
    int32_t scale_mode;  /* NVFP4: W4A4_SCALE_TENSOR or W4A4_SCALE_TOKEN; else ignored */
    int32_t flags;       /* 0, or W4A4_FLAG_HADAMARD (see below); other bits must be 0 */
    void*   codes;       /* device */
    void*   scales;      /* device */
    float*  s2;          /* device, NVFP4 only (else may be NULL) */
} w4a4_qtensor;

/* Bytes each buffer of a quantized tensor needs.  Host only, no device work.
 * Any of the out-pointers may be NULL.  Returns W4A4_OK or
 * W4A4_ERR_INVALID_ARG.  INT4 scales are sized for group 128, which bounds
 * the coarser groups too. */
int w4a4_qtensor_bytes(int format, int rows, int cols, int scale_mode,
                       size_t* codes_bytes, size_t* scales_bytes, size_t* s2_bytes);

/*
 * Quantize activations X[M,K] (bf16, row stride ldx) into `out`, per token
 * ("Daily Papers" para 4: per-token quantization; "Depth Registers..."
 * abstract: round to nearest).
 *   format/group: (NVFP4,16), (MXFP4,32) or (INT4, 128 / 256 / 512; K a
 *     multiple of the group).  INT4 groups coarser than 128 are the
 *     granularity knob of the "Depth Registers..." thelatestinai page, para 2
 *     (APEX4: rho-aware granularity adaptation): the GEMM rescales once per
 *     group, so a group of 512 takes a quarter of g128's CUDA-core work; the
 *     weights must use the same group (w4a4_int4_group_for_rho picks one).
 *   scale_mode (NVFP4): TOKEN -> s2[r] = amax(row r)/2688; TENSOR ->
 *     s2[0] = amax(X)/2688 from an extra reduction pass (two reads of X).
 *     A zero amax, or a quotient below the smallest normal float, gives 1.
 *   static_s2 (nullable, device, NVFP4): caller-fixed second-level scale(s),
 *     [1] for TENSOR, [M] for TOKEN; no amax pass is made.
 *   out: out->format/group/scale_mode must equal the arguments, out->rows ==
 *     M, out->cols >= K (== K + nS for an augmented tensor, whose first K
 *     columns this call writes).
 * Block rule, NVFP4: scale = E4M3((amax_block/6)/s2), element code =
 *   E2M1(x/(scale*s2)) (FP32 divides, nearest even, saturating at 6; a
 *   negative element that rounds to zero keeps its sign bit; a zero scale
 *   gives zero codes).  MXFP4: scale exponent floor(log2(amax_block)) - 2,
 *   clamped to E8M0's range, code = E2M1(x * 2^-exp); zero block -> exponent
 *   code 0, zero codes.  INT4: s = amax_group/7, q = clamp(rint(x/s),-8,7);
 *   zero group -> s = 0, zero codes.
 */
int w4a4_quantize_act(const uint16_t* X, int M, int K, int ldx,
                      int format, int group, int scale_mode,
                      const float* static_s2, w4a4_qtensor* out, void* stream);

/*
 * Quantize weights W[N,K] (bf16, row stride ldw) once, offline.  Same block
 * rules as w4a4_quantize_act; NVFP4 weights here use one tensor scale
 * (out->scale_mode must be TENSOR; w4a4_quantize_weight_segments gives one
 * scale per row segment).  With S (device int32[nS], channel indices in
 * [0,K) in any order, nS a multiple of 128) the quantized
 * tensor is [W | W[:,S]] with cols = K + nS: the weight side of the
 * dual-stage residual augmentation ("APEX4..." page, para 2, ARCQuant).
 */
int w4a4_quantize_weight(const uint16_t* W, int N, int K, int ldw,
                         int format, int group, const int32_t* S, int nS,
                         w4a4_qtensor* out, void* stream);

/*
 * NVFP4 weights of a fused module (q/k/v, gate/up stacked along N) with one
 * global scale per constituent module ("Daily Papers" page, para 4, Minima:
 * one NVFP4 global scale per module, calibrated separately).  Row segment i
 * is rows [seg[i], seg[i+1]) of W[N,K]; it is quantized exactly as
 * w4a4_quantize_weight quantizes that slice alone (tensor scale
 * s2_i = amax(segment)/2688), and every row of it stores s2_i.
 *   seg: HOST int32[nseg+1], seg[0] = 0 < seg[1] < ... < seg[nseg] = N, every
 *     boundary a multiple of 128 (so each segment owns whole scale atoms);
 *     nseg >= 1.  nseg = 1 gives the tensor rule with the scale repeated.
 *   S, nS: as w4a4_quantize_weight (cols = K + nS; the appended channels use
 *     their segment's scale).
 *   out: format NVFP4, scale_mode W4A4_SCALE_TOKEN (s2 holds one scale per
 *     row, N floats, 16-byte aligned), rows = N, cols = K + nS.
 * The GEMM and the linear layer read s2[n] for output column n; with the
 * same rows in one segment the result equals a tensor-scale weight's.
 * Returns W4A4_ERR_INVALID_ARG on a bad segment list, W4A4_ERR_MISALIGNED on
 * an unaligned s2; nothing is launched then.
 */
int w4a4_quantize_weight_segments(const uint16_t* W, int N, int K, int ldw,
                                  const int32_t* seg, int nseg,
                                  const int32_t* S, int nS,
                                  w4a4_qtensor* out, void* stream);

/*
 * Multi-pass MXFP4 decomposition of activations ("APEX4: Efficient Pure W4A4
 * LLM Inference via Intra-SM Compute Rebalancing" page, para 1, MSD: the
 * activation is split into several low-precision components, each multiplied
 * directly with the quantized weights).  Pass 0 is w4a4_quantize_act's MXFP4
 * rule on X; pass p applies the same rule, with its own shared exponents, to
 * the residual X - (values of passes 0..p-1), formed exactly in FP32 (it is
 * always a bf16 value).  Pass p fills columns [p*K, (p+1)*K) of `out`.
 *   passes: 1 .. 4 (1 is plain MXFP4).
 *   out: format MXFP4, rows = M, cols = passes * K.
 * Multiplied with w4a4_quantize_weight_msd's [W | W | ...] (one GEMM over
 * passes * K), the product is sum_p X_p W^T.
 */
int w4a4_quantize_act_msd(const uint16_t* X, int M, int K, int ldx, int passes,
                          w4a4_qtensor* out, void* stream);

/*
 * The weight side of the multi-pass product: W[N,K] quantized to MXFP4 once
 * and repeated `passes` times along K (cols = passes * K), so that one GEMM
 * multiplies every activation pass with the same weights.
 *   out: format MXFP4, rows = N, cols = passes * K.
 */
int w4a4_quantize_weight_msd(const uint16_t* W, int N, int K, int ldw, int passes,
                             w4a4_qtensor* out, void* stream);

/*
 * Y[M,N] = A * B^T for quantized A (activations, rows = M) and B (weights,
 * rows = N) of the same format and the same cols (= K, or K + nS).
 *   NVFP4/MXFP4: block-scaled tensor-core MMA, FP32 accumulation;
 *     NVFP4 result of (m, n) multiplied by alpha = s2_A (row m, or the
 *     tensor's) * s2_B (the tensor's, or row n's when B->scale_mode is
 *     TOKEN, e.g. per-segment weights; B->s2 must then be 16-byte aligned).
 *   INT4: exact int32 partial sum per 128-group, rescaled by
 *     scale_A[m,g]*scale_B[n,g] and accumulated in FP32 ("Depth
 *     Registers..." thelatestinai page, para 2: group dequantization).
 * Y: device bf16, row stride ldy >= N.  Result rounded to nearest bf16.
 */
int w4a4_gemm(const w4a4_qtensor* A, const w4a4_qtensor* B,
              uint16_t* Y, int ldy, void* stream);

/* INT4 group size for a device whose tensor-core / CUDA-core throughput
 * ratio is rho ("Depth Registers..." thelatestinai page, para 2: APEX4's
 * rho; g128 pays at rho = 16, not at 64): 128 up to rho = 16, then doubled
 * per doubling of rho, at most 512.  B200's int8-tensor to FP32-FMA ratio is
 * about 60, which gives 512.  Host only. */
int w4a4_int4_group_for_rho(double rho);

/* Workspace bytes w4a4_linear needs for these sizes (0 on bad arguments). */
size_t w4a4_linear_workspace(int M, int N, int K, int format, int nS);

/*
 * The whole linear layer: quantize X[M,K] per token in the format of Wq,
 * optionally append the nS residual channels of S (NVFP4 only; Wq must then
 * have cols = K + nS and have been made with the same S), and multiply with
 * Wq, writing Y[M,N] bf16.  scale_mode selects the NVFP4 activation scale
 * (TOKEN: dynamic per token; TENSOR: dynamic per tensor).  Small M (<= 16)
 * takes a bandwidth-bound split-K variant.  ws: device workspace of at least
 * w4a4_linear_workspace(M, N, K, Wq->format, nS) bytes, 256-byte aligned.
 */
int w4a4_linear(const uint16_t* X, int M, int K, int ldx,
                const w4a4_qtensor* Wq, int scale_mode,
                const int32_t* S, int nS,
                uint16_t* Y, int ldy, void* ws, size_t ws_bytes, void* stream);

/*
 * w4a4_linear without a caller workspace (the pages have no counterpart: it
 * only changes where the scratch lives).  Same operation, arguments, layout
 * and results as w4a4_linear; the scratch is a static device array inside
 * this library, W4A4_NOALLOC_SCRATCH_BYTES per device, and the call
 * allocates nothing.  It serves callers that hold no device allocator and so
 * cannot provide a workspace.
 *  - Sizes whose w4a4_linear_workspace() exceeds W4A4_NOALLOC_SCRATCH_BYTES
 *    return W4A4_ERR_WORKSPACE and launch nothing (16 MiB covers, e.g., every
 *    Llama-2-70B-sized linear at M <= 16, the small-M decode case).
 *  - The first call in a CUDA context (with its device current) looks up
 *    the array's address in that context and caches it per context handle;
 *    make that first call before any stream capture.  Calls made in another
 *    context (a driver-API context of the caller's, or the primary context
 *    re-created after cudaDeviceReset) look the address up again there.
 *  - No scratch byte needs to start at zero: the call writes all it reads.
 *  - One scratch per device: calls on one device whose kernels could overlap
 *    (unordered streams, several host threads) race on it and must be
 *    ordered by the caller.
 */
#define W4A4_NOALLOC_SCRATCH_BYTES (16u << 20)
int w4a4_linear_noalloc(const uint16_t* X, int M, int K, int ldx,
                        const w4a4_qtensor* Wq, int scale_mode,
                        const int32_t* S, int nS,
                        uint16_t* Y, int ldy, void* stream);

/*
 * The multi-pass MXFP4 linear layer: w4a4_quantize_act_msd of X[M,K] into the
 * workspace, then one MXFP4 GEMM over passes * K columns with Wq (made by
 * w4a4_quantize_weight_msd with the same passes), Y[M,N] bf16.  ws: at least
 * w4a4_linear_workspace(M, N, K, W4A4_MXFP4, (passes - 1) * K) bytes,
 * 256-byte aligned.  M <= 16 takes the split-K decode variant.
 */
int w4a4_linear_msd(const uint16_t* X, int M, int K, int ldx,
                    const w4a4_qtensor* Wq, int passes,
                    uint16_t* Y, int ldy, void* ws, size_t ws_bytes, void* stream);

/*
 * Second stage of the dual-stage NVFP4 quantization ("APEX4..." page,
 * para 2, ARCQuant): for every row, R_j = x[S_j] - x^[S_j] in FP32, where
 * x^ is the first-stage dequantized value (code * block scale * s2, rounded
 * to FP32) read from Xaug's first K columns, and R is quantized to NVFP4
 * with the row's own s2 into columns K .. K+nS-1 of Xaug.
 * S: device int32[nS], in [0,K), in any order (w4a4_select_channels writes
 * them ascending; the order is the order of the residual columns, and the
 * weights must be quantized with the same S); nS a multiple of 128.  An
 * index outside [0,K) is replaced by channel 0 and makes
 * w4a4_device_status return W4A4_ERR_INVALID_ARG.
 * Xaug: NVFP4, rows = M, cols = K + nS, first K columns already quantized.
 */
int w4a4_augment_residual(const uint16_t* X, int M, int K, int ldx,
                          const int32_t* S, int nS, w4a4_qtensor* Xaug, void* stream);

/*
 * Offline channel selection for the augmentation: the nS channels with the
 * largest max|x| over the Mc calibration rows Xcal[Mc,K] (device bf16, row
 * stride ldx), ties to the lower index, written ascending to S_out (device
 * int32[nS]).  ws: device workspace of at least 8*K bytes (per-channel
 * maxima and ranks).
 */
int w4a4_select_channels(const uint16_t* Xcal, int Mc, int K, int ldx, int nS,
                         int32_t* S_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronize `stream`, then read and clear the library's device error word.
 * Returns W4A4_OK, W4A4_ERR_DEVICE_TIMEOUT (a kernel's bounded wait expired
 * and the kernel returned early; its outputs are undefined),
 * W4A4_ERR_INVALID_ARG (a channel index in a device-side S was outside
 * [0,K); it was replaced by channel 0) or W4A4_ERR_CUDA.
 */
int w4a4_device_status(void* stream);

/*
 * Test hook for the bounded waits (process-wide, not thread-safe): every
 * later GEMM launch uses `wait_limit_ns` as the limit of each in-kernel wait
 * (0 restores the default of 2 s), and when skip_k_tile >= 0 the GEMM's
 * loader skips loading k-tile `skip_k_tile` of every output tile, so the
 * consumer's wait runs out and the kernel reports W4A4_ERR_DEVICE_TIMEOUT.
 */
void w4a4_debug_set(int skip_k_tile, unsigned long long wait_limit_ns);

/* Static description of a status code. */
const char* w4a4_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* W4A4_H */
