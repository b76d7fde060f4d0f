/*
 * convrot_nvfp4.h -- C ABI of the NVFP4 variant of the rotated linear layer
 * (library libconvrot_nvfp4.so): activations and weights rotated by the
 * same block Hadamard as in the W4A4 layer, quantised to NVFP4 and
 * multiplied on the sm_100a block-scaled FP4 tensor cores
 * (tcgen05.mma kind::mxf4nvf4, E2M1 x E2M1 with E4M3 scales per 16 values).
 *
 * The pages name NVFP4 as the target of the official ConvRot implementation
 * ("convrot-mlx" README, "Why this repository exists") without defining the
 * format or the scaling.  Reading taken here, the plainest one the rest of
 * the pages supports (the rotation of Comfy-Org/comfy-quants issue, section
 * 1, and the rowwise absmax scale of "convrot-mlx" README, "What is
 * included"), decided in fp32 for every row y of x R (or of W R):
 *
 *   a    = max_k |y_k|,  s = a / 2688  (6 x 448),  r = 448 / a
 *          (a == 0: s = r = 0);
 *   per block b of 16 consecutive k:
 *          sf_b = e4m3(max_{k in b} |y_k| * r)      (round to nearest even,
 *                                                     saturating at 448),
 *          d_b  = value(sf_b) * s,  inv_b = 1 / d_b  (0 when d_b == 0),
 *          q_k  = e2m1(y_k * inv_b)                  (nearest even, +-6 max);
 *   y[m][n] = bf16_rne((sum_b value(sfx_b) value(sfw_b)
 *                       sum_{k in b} e2m1(qx_k) e2m1(qw_k)) * sx[m] * sw[n] + b[n]).
 *
 * The tensor cores accumulate in fp32 and the epilogue is fp32
 * ((acc * sx) * sw + b), so results match the exact definition within the
 * rounding of that arithmetic, not bit for bit.
 *
 * Layouts:
 *   - codes: [rows][K/2] bytes, two E2M1 codes per byte, low nibble = even
 *     k (bit 3 of a code is its sign);
 *   - block scales: convrot_nvfp4_scale_bytes(rows, K) bytes of E4M3 codes
 *     in 512-byte atoms of 128 rows x 4 blocks: the scale of row r, block j
 *     is at ((r / 128) * (K / 64) + j / 4) * 512 + 16 (r mod 32)
 *     + 4 ((r / 32) mod 4) + j mod 4, rows padded to a multiple of 128 (the
 *     layout the tensor cores read, so atoms go to them unchanged); the
 *     quantisation writes every byte, code 0 for the padding rows;
 *   - row scales: fp32 [rows].
 * Conventions are those of convrot.h: device pointers on the current device
 * (CONVROT_ERR_NOT_DEVICE otherwise), 16-byte aligned (CONVROT_ERR_ALIGN),
 * caller-owned, work enqueued on `stream`, arguments validated before any
 * launch, M = 0 or N = 0 a no-op, K a multiple of 64 and of `group`
 * (64 <= K <= CONVROT_MAX_K), group 64 or 256.  Device waits are bounded; a
 * wait that runs out is reported by convrot_nvfp4_check_device_error.
 */
#ifndef CONVROT_NVFP4_H_
#define CONVROT_NVFP4_H_

#include "convrot.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of the block-scale buffer of `rows` rows: ceil(rows / 128) * 128 *
 * K / 16.  Host-only; 0 for rows <= 0 or K <= 0. */
size_t convrot_nvfp4_scale_bytes(int64_t rows, int64_t K);

/*
 * Rotation and NVFP4 quantisation of bf16 rows x [rows][K] (activations, or
 * weights offline): writes q [rows][K/2], sf (convrot_nvfp4_scale_bytes) and
 * s fp32 [rows].  One kernel.  The rotation is Comfy-Org/comfy-quants issue,
 * section 1; the quantisation the reading above.
 */
convrot_status convrot_nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t K, int group,
                                      uint8_t *q, uint8_t *sf, float *s,
                                      convrot_stream_t stream);

/* Bytes of workspace convrot_nvfp4_linear needs: the activations' codes,
 * block scales and row scales, each rounded up to 256 bytes. */
size_t convrot_nvfp4_workspace_size(int64_t M, int64_t K);

/*
 * The product on prepared operands: qx [M][K/2], sfx, sx [M] (from
 * convrot_nvfp4_quantize of the activations) and qw [N][K/2], sfw, sw [N]
 * (of the weights), bias bf16 [N] or NULL, y bf16 [M][N].  One block-scaled
 * tensor-core kernel.  "convrot-mlx" README, "Install and test": the
 * product, then scaling and bias.
 */
convrot_status convrot_nvfp4_linear_prepared(const uint8_t *qx, const uint8_t *sfx,
                                             const float *sx, const uint8_t *qw,
                                             const uint8_t *sfw, const float *sw,
                                             const void *bias_bf16, int64_t M, int64_t N,
                                             int64_t K, void *y_bf16, convrot_stream_t stream);

/*
 * Test hook: convrot_nvfp4_linear_prepared with the GEMM's tile width
 * forced.  form:
 *          0  automatic: 128-wide weight tiles where twice the number of
 *             256-wide tiles fits in one wave of CTAs (one per SM), else
 *             256-wide;
 *          1  tiles of 128 tokens x 256 weight rows;
 *          2  tiles of 128 tokens x 128 weight rows.
 * Returns CONVROT_ERR_SHAPE for any other form.  Exposes the product of
 * "convrot-mlx" README, "Install and test" per tile width.
 */
convrot_status convrot_nvfp4_debug_gemm_form(const uint8_t *qx, const uint8_t *sfx,
                                             const float *sx, const uint8_t *qw,
                                             const uint8_t *sfw, const float *sw,
                                             const void *bias_bf16, int64_t M, int64_t N,
                                             int64_t K, int form, void *y_bf16,
                                             convrot_stream_t stream);

/*
 * The whole NVFP4 layer: quantisation of x into `workspace`
 * (ws_bytes >= convrot_nvfp4_workspace_size(M, K), 256-byte aligned,
 * CONVROT_ERR_WORKSPACE otherwise), then the product.  Two kernels.
 */
convrot_status convrot_nvfp4_linear(const void *x_bf16, const uint8_t *qw, const uint8_t *sfw,
                                    const float *sw, const void *bias_bf16, int64_t M,
                                    int64_t N, int64_t K, int group, void *workspace,
                                    size_t ws_bytes, void *y_bf16, convrot_stream_t stream);

/* Failure detection (no counterpart on the pages).  Synchronise `stream`,
 * then return and clear this library's device error word. */
convrot_status convrot_nvfp4_check_device_error(convrot_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_NVFP4_H_ */
