/*
 * W4A4 oracle: plain, slow, obviously-correct CPU reference of the W4A4
 * quantized linear layer.  TEST INFRASTRUCTURE ONLY: the library under
 * w4a4_quantized_gemm_token_b200/ never includes, links or calls it; only the
 * tests, the smoke check and the benchmark's CPU-baseline leg do.
 *
 * What it follows (page title, paragraph):
 *  - "Daily Papers", para 4 (Minima): NVFP4 = 16-element block scaling plus a
 *    global (FP32) scale; per-token activation quantization.
 *  - "Depth Registers Unlock W4A4 on SwiGLU" (thelatestinai page), para 1:
 *    open-standard MXFP4; "APEX4: Efficient Pure W4A4 LLM Inference via
 *    Intra-SM Compute Rebalancing" page, para 1 (MSD): two-pass MXFP4.
 *  - "Depth Registers..." (thelatestinai page), para 2 (APEX4): W4A4-g128
 *    INT4 with per-group dequantization; "Depth Registers..." (mlsanity
 *    page), abstract: naive round-to-nearest W4A4.
 *  - "APEX4..." page, para 2 (ARCQuant): augmented residual channels, the
 *    dual-stage NVFP4 residual appended along the reduction dimension.
 * The bit-level encodings (E2M1, E4M3, E8M0) are not printed on the pages;
 * the rules below are the plain reading of the public OCP Microscaling and
 * NVFP4 format definitions that those paragraphs name.
 *
 * Conventions: bf16 tensors are passed as uint16_t bit patterns, row-major
 * with a leading dimension in elements.  4-bit codes are packed two per byte,
 * element 2j in the low nibble of byte j.  Scales here are plain row-major
 * ([rows][blocks]); the GPU library stores them in the MMA layout and the
 * tests undo that with their own index function.
 *
 * All float arithmetic of the quantizers is IEEE binary32 with round to
 * nearest even, no contraction (built with -ffp-contract=off); the GEMM
 * reference sums are exact (int128 or fp64) and rounded once to bf16.
 */
#ifndef W4A4_ORACLE_H
#define W4A4_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- scalar encodings -------------------------------------------------- */
uint8_t orc_e2m1_encode(float v);     /* nearest of {0,.5,1,1.5,2,3,4,6}, ties to even code, |v|>6 -> 6, sign = signbit(v) */
float   orc_e2m1_decode(uint8_t code);
uint8_t orc_e4m3_encode(float v);     /* v >= 0: E4M3 (bias 7, max 448), nearest even, saturating */
float   orc_e4m3_decode(uint8_t code);
float   orc_e8m0_decode(uint8_t code); /* 2^(code-127) */
int     orc_floor_log2(float a);      /* a > 0 finite, subnormals included */
float   orc_bf16_to_f32(uint16_t b);
uint16_t orc_f64_to_bf16(double v);   /* one rounding, nearest even */

/* ---- NVFP4 second-level scale ------------------------------------------ */
float orc_nvfp4_s2_from_amax(float amax);

/* ---- quantizers -------------------------------------------------------- */
/* mode: 0 = one FP32 scale for the whole tensor, 1 = one per row (token).
 * static_s2 (nullable): caller-fixed second-level scale(s), [1] or [M].
 * codes [M][K/2], scales [M][K/16] E4M3 bytes, s2 [1] or [M].            */
int orc_quant_nvfp4(const uint16_t* X, int M, int K, int ldx, int mode,
                    const float* static_s2, uint8_t* codes, uint8_t* scales,
                    float* s2);
/* Fused modules ("Daily Papers", para 4 (Minima): a global-scale mismatch
 * when modules quantized with their own global scales are fused into one
 * GEMM): rows [seg[i], seg[i+1]) form module i, quantized as its own tensor
 * (one FP32 scale from the module's amax); s2_rows[M] receives every row's
 * module scale.  seg: nseg+1 ascending boundaries, seg[0] = 0, seg[nseg] = M. */
int orc_quant_nvfp4_segments(const uint16_t* X, int M, int K, int ldx,
                             const int32_t* seg, int nseg, uint8_t* codes,
                             uint8_t* scales, float* s2_rows);
/* codes [M][K/2], scales [M][K/32] E8M0 bytes                             */
int orc_quant_mxfp4(const uint16_t* X, int M, int K, int ldx,
                    uint8_t* codes, uint8_t* scales);
/* Multi-pass MXFP4 ("APEX4: Efficient Pure W4A4..." page, para 1, MSD): pass
 * p quantizes the residual left by passes 0..p-1 (exact, a bf16 value) with
 * its own shared exponents into columns [p*K, (p+1)*K).  codes
 * [M][passes*K/2], scales [M][passes*K/32].  Returns -2 if a residual were
 * not exact (never, under the MXFP4 rule above).                           */
int orc_quant_mxfp4_msd(const uint16_t* X, int M, int K, int ldx, int passes,
                        uint8_t* codes, uint8_t* scales);
/* Block-local Walsh-Hadamard rotation of X (bf16 [M][ldx]) into FP32
 * out[M][K]: each n-element block along K (n = 16, 32 or 128: the block of
 * the format) is transformed by the fast Walsh-Hadamard butterflies in FP32
 * (stages h = 1, 2, ..., n/2; (a, b) -> (a + b, a - b)), then multiplied by
 * 1/n when act_side (activations), left unscaled otherwise (weights), so
 * that (X H/n)(W H)^T = X W^T.                                             */
int orc_rotate_blocks(const uint16_t* X, int M, int K, int ldx, int n, int act_side, float* out);
/* The quantizers on FP32 input X[M][K] (rotated values), same rules.        */
int orc_quant_nvfp4_f32(const float* X, int M, int K, int mode,
                        uint8_t* codes, uint8_t* scales, float* s2);
int orc_quant_mxfp4_f32(const float* X, int M, int K, uint8_t* codes, uint8_t* scales);
int orc_quant_int4_f32(const float* X, int M, int K, uint8_t* codes, float* scales);
/* INT4 with groups of G elements (G a multiple of 128, K a multiple of G;
 * "Depth Registers..." thelatestinai page, para 2: rho-aware granularity):
 * the same rule per group; scales [M][K/G].                                */
int orc_quant_int4_g(const uint16_t* X, int M, int K, int ldx, int G,
                     uint8_t* codes, float* scales);
int orc_quant_int4_f32_g(const float* X, int M, int K, int G, uint8_t* codes, float* scales);
int orc_gemm_int4_g(const uint8_t* ca, const float* sa, const uint8_t* cw, const float* sw,
                    int M, int N, int K, int G, uint16_t* Y, double* yref, double* absdot);
/* codes [M][K/2] two's-complement nibbles, scales [M][K/128] FP32          */
int orc_quant_int4(const uint16_t* X, int M, int K, int ldx,
                   uint8_t* codes, float* scales);

/* ---- dequantization to fp64 [M][K] ------------------------------------- */
void orc_dequant_nvfp4(const uint8_t* codes, const uint8_t* scales,
                       const float* s2, int mode, int M, int K, double* out);
void orc_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales,
                       int M, int K, double* out);
void orc_dequant_int4(const uint8_t* codes, const float* scales,
                      int M, int K, double* out);

/* ---- GEMM reference: Y[m,n] = alpha * sum_k a^[m,k] w^[n,k] ------------
 * Y: bf16 bits [M][N]; yref (nullable): exact value in fp64; absdot
 * (nullable): |alpha| * sum_k |a^ w^| in fp64 (the tolerance term).        */
int orc_gemm_nvfp4(const uint8_t* ca, const uint8_t* sa, const float* s2a, int a_mode,
                   const uint8_t* cw, const uint8_t* sw, const float* s2w,
                   int M, int N, int K, uint16_t* Y, double* yref, double* absdot);
/* The same with the weights' second-level scale per output row (w_mode 1:
 * s2w[N], alpha = s2a * s2w[n]) or per tensor (w_mode 0).                  */
int orc_gemm_nvfp4_wrows(const uint8_t* ca, const uint8_t* sa, const float* s2a, int a_mode,
                         const uint8_t* cw, const uint8_t* sw, const float* s2w, int w_mode,
                         int M, int N, int K, uint16_t* Y, double* yref, double* absdot);
int orc_gemm_mxfp4(const uint8_t* ca, const uint8_t* sa,
                   const uint8_t* cw, const uint8_t* sw,
                   int M, int N, int K, uint16_t* Y, double* yref, double* absdot);
int orc_gemm_int4(const uint8_t* ca, const float* sa,
                  const uint8_t* cw, const float* sw,
                  int M, int N, int K, uint16_t* Y, double* yref, double* absdot);

/* ---- dual-stage residual augmentation (NVFP4) --------------------------
 * Given the first-stage NVFP4 quantization (codes [M][K/2], scales
 * [M][K/16], s2 with `mode`), the channel list S (nS ascending, nS % 16 == 0)
 * computes R[m,j] = x[m,S_j] - x^[m,S_j] in FP32 and quantizes R by the
 * NVFP4 block rule with the row's own second-level scale:
 * rcodes [M][nS/2], rscales [M][nS/16].                                   */
int orc_augment_nvfp4(const uint16_t* X, int M, int K, int ldx,
                      const int32_t* S, int nS,
                      const uint8_t* codes, const uint8_t* scales,
                      const float* s2, int mode,
                      uint8_t* rcodes, uint8_t* rscales);
/* Offline channel selection: per-channel max|x| over Mc calibration rows,
 * the nS largest (ties to the lower index), returned ascending.           */
int orc_select_channels(const uint16_t* Xcal, int Mc, int K, int nS, int32_t* S);

#ifdef __cplusplus
}
#endif
#endif
