/*
 * convrot_w4a16.h -- C ABI of the W4A16 variant of the rotated linear layer
 * (library libconvrot_w4a16.so): bf16 activations times the same packed,
 * rotated INT4 weights, on the sm_100a tensor cores.
 *
 * The pages name this sibling of the W4A4 path ("convrot-mlx" README, "What
 * is included": Metal 4 MPP W4A4/W4A16 TensorOps paths; "Requirements": the
 * MPP paths perform signed INT8 x INT4 or BF16 x INT4 TensorOps) without
 * spelling out its arithmetic.  Reading taken here, the plainest one the
 * rest of the pages support:
 *
 *   1. the weights are prepared exactly as for W4A4 (convrot_quantize_weight:
 *      rotated by R = I_G (x) H_n, one absmax scale sw[n] per row, codes
 *      q[n][k] in [-7, 7], packed two per byte, low nibble = even k);
 *   2. since the weights were rotated, the activations are rotated by the
 *      same R (Comfy-Org/comfy-quants issue, section 1: X W^T = (X R)(W R)^T
 *      for orthogonal R) but NOT quantised: each rotated value is rounded
 *      once to bf16, the operand type of a BF16 x INT4 product,
 *          xr[m][k] = bf16_rne((x_m R)[k]);
 *   3. y[m][n] = bf16_rne( (sum_k xr[m][k] q[n][k]) * sw[n] + b[n] ).
 *
 * The GPU evaluates step 2 with fp32 butterflies and step 3 with fp32
 * tensor-core accumulation and an fp32 epilogue ((acc * sw) + b, two
 * roundings), so results match the exact definition within the rounding of
 * that arithmetic, not bit for bit.
 *
 * Conventions are those of convrot.h: device pointers on the current device
 * (CONVROT_ERR_NOT_DEVICE otherwise, checked before any launch),
 * row-major, contiguous, 16-byte aligned (CONVROT_ERR_ALIGN otherwise); the
 * caller owns every buffer and the library allocates nothing; work is
 * enqueued on `stream`; arguments are validated before any launch, so a
 * status other than CONVROT_OK or CONVROT_ERR_CUDA means nothing ran; M = 0
 * or N = 0 is a no-op; 64 <= K <= CONVROT_MAX_K with K % 64 == 0 (and
 * K % group == 0 where a group is given); group is 64 or 256.  Device waits
 * are bounded; a wait that runs out is reported by
 * convrot_w4a16_check_device_error.
 */
#ifndef CONVROT_W4A16_H_
#define CONVROT_W4A16_H_

#include "convrot.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Step 2 alone: xr [M][K] bf16 = bf16_rne(x R), R = I_G (x) H_group.
 * x: bf16 [M][K] (read).  xr: bf16 [M][K] (written).  One kernel.
 * Source: the block rotation of Comfy-Org/comfy-quants issue, section 1,
 * applied to the activations of the BF16 x INT4 path ("convrot-mlx" README,
 * "Requirements").
 */
convrot_status convrot_w4a16_prepare_act(const void *x_bf16, int64_t M, int64_t K, int group,
                                         void *xr_bf16, convrot_stream_t stream);

/* Bytes of workspace convrot_w4a16_linear needs: the rotated activations,
 * M * K * 2 rounded up to 256 (0 for M <= 0 or K <= 0).  Host-only.  It holds
 * step 2's output, the bf16 operand of the BF16 x INT4 product ("convrot-mlx"
 * README, "Requirements"). */
size_t convrot_w4a16_workspace_size(int64_t M, int64_t K);

/*
 * Step 3 on rotated activations: y [M][N] bf16 from xr bf16 [M][K], the
 * packed weights qw uint8 [N][K/2] and their scales sw fp32 [N], bias bf16
 * [N] or NULL (zeros).  One tensor-core kernel.  Requires K % 64 == 0.
 * Source: "convrot-mlx" README, "What is included" (the W4A16 TensorOps path)
 * and "Install and test" (the product, then scaling and bias).
 */
convrot_status convrot_w4a16_linear_prepared(const void *xr_bf16, const uint8_t *qw,
                                             const float *sw, const void *bias_bf16, int64_t M,
                                             int64_t N, int64_t K, void *y_bf16,
                                             convrot_stream_t stream);

/*
 * The whole W4A16 layer ("convrot-mlx" README, "What is included": the
 * W4A16 path beside W4A4): steps 2 and 3, two kernels on `stream` (the GEMM's
 * set-up overlaps the end of the rotation through programmatic dependent
 * launch).  workspace: device memory of at least
 * convrot_w4a16_workspace_size(M, K) bytes, 256-byte aligned
 * (CONVROT_ERR_WORKSPACE otherwise); it receives xr.
 */
convrot_status convrot_w4a16_linear(const void *x_bf16, const uint8_t *qw, const float *sw,
                                    const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                    int group, void *workspace, size_t ws_bytes, void *y_bf16,
                                    convrot_stream_t stream);

/*
 * convrot_w4a16_linear and convrot_w4a16_linear_prepared with the weights
 * given in the repacked layout of convrot_repack_weight (include/convrot.h;
 * "convrot-mlx" README, "What is included": lossless repacking), same
 * arguments otherwise, bit-identical results.
 */
convrot_status convrot_w4a16_linear_repacked(const void *x_bf16, const uint8_t *qw_rep,
                                             const float *sw, const void *bias_bf16, int64_t M,
                                             int64_t N, int64_t K, int group, void *workspace,
                                             size_t ws_bytes, void *y_bf16,
                                             convrot_stream_t stream);
convrot_status convrot_w4a16_linear_prepared_repacked(const void *xr_bf16, const uint8_t *qw_rep,
                                                      const float *sw, const void *bias_bf16,
                                                      int64_t M, int64_t N, int64_t K,
                                                      void *y_bf16, convrot_stream_t stream);

/*
 * Test hook: the product on prepared operands (as
 * convrot_w4a16_linear_prepared) with the GEMM forced to one form, so that
 * every form is checked whatever the automatic choice for (M, N, K):
 *   form = 0  automatic (as the entry points above: form 3 up to 64 tokens,
 *             form 1 beyond);
 *          1  128 x 256 token-by-weight tiles;
 *          2  few tokens (M <= 64), weights widened to bf16 in shared memory
 *             on the MMA's 128-row side;
 *          3  few tokens (M <= 64), weights widened to bf16 straight into
 *             TMEM (the MMA's A operand), one CTA per slice of weight rows.
 * form | CONVROT_TILES_REPACKED takes qw in the repacked layout.  Returns
 * CONVROT_ERR_SHAPE for any other form or for 2 / 3 with M > 64.  Exposes
 * the product of "convrot-mlx" README, "What is included" (the W4A16 path)
 * per GEMM form.
 */
convrot_status convrot_w4a16_debug_gemm_form(const void *xr_bf16, const uint8_t *qw,
                                             const float *sw, const void *bias_bf16, int64_t M,
                                             int64_t N, int64_t K, int form, void *y_bf16,
                                             convrot_stream_t stream);

/* Failure detection (no counterpart on the pages).  Synchronise `stream`,
 * then return and clear this library's device error word (CONVROT_OK, or
 * CONVROT_ERR_DEVICE_TIMEOUT after a wait ran out). */
convrot_status convrot_w4a16_check_device_error(convrot_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_W4A16_H_ */
