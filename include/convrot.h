/*
 * convrot.h -- C ABI of the B200 (sm_100a) rotated W4A4 linear layer.
 *
 * The layer (pages: "convrot-mlx" README, "What is included" and "Install and
 * test"; Comfy-Org/comfy-quants issue "convrot is exactly same as or a wrapper
 * around QuaRot Stage 1c", sections 1 and 2):
 *
 *   1. every K-group of n in {64, 256} channels of a bf16 row is multiplied by
 *      the normalised regular Hadamard matrix H_n = (J - 2I)^{(x)log4 n}/sqrt(n),
 *      i.e. the row is multiplied by the block-diagonal R = I_G (x) H_n;
 *   2. the rotated row is quantised with ONE symmetric absmax scale per row to
 *      signed INT4 codes in [-7, 7]:
 *          a = max|y|,  s = a / 7,  q = round_half_away(y * (7 / a))   (fp32)
 *      (a == 0 gives s = 0 and all codes 0), and packed two codes per byte,
 *      low nibble = even channel, 4-bit two's complement;
 *   3. activations and offline-prepared weights are multiplied with exact
 *      integer accumulation, acc[m][n] = sum_k qx[m][k] qw[n][k], and
 *   4. the epilogue writes y[m][n] = bf16_rne((float(acc) * sx[m]) * sw[n] + b[n])
 *      evaluated in fp32 in that order.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers on the current CUDA device unless stated
 *     otherwise, row-major and contiguous, 16-byte aligned (CONVROT_ERR_ALIGN
 *     otherwise).  bf16 tensors are passed as const void* to raw bf16 data.
 *     Each pointer is looked up with cudaPointerGetAttributes before anything
 *     is launched: host memory (pinned or not), another GPU's memory or an
 *     address the CUDA runtime does not know gives CONVROT_ERR_NOT_DEVICE.
 *     Sizes cannot be checked through a raw pointer: buffers must hold the
 *     bytes each entry point states.
 *   - Ownership stays with the caller: the library allocates nothing, frees
 *     nothing, never synchronises and never changes the current device.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Arguments are validated before anything is launched: a non-OK status
 *     means nothing was enqueued, except CONVROT_ERR_CUDA (a launch failed).
 *   - Shapes: M, N >= 1 (M = 0 or N = 0 is a no-op returning OK), K a
 *     multiple of `group`, 64 <= K <= CONVROT_MAX_K; group is 64 or 256.
 *   - Results are deterministic: identical inputs give identical bytes.
 *   - Device-side waits are bounded; a wait that runs out records
 *     CONVROT_ERR_DEVICE_TIMEOUT, which convrot_check_device_error reports.
 */
#ifndef CONVROT_H_
#define CONVROT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                        /* the CUDA runtime's stream type */
typedef struct CUstream_st *convrot_stream_t;  /* same object as cudaStream_t */

#define CONVROT_MAX_K 32768

typedef enum {
    CONVROT_OK = 0,
    CONVROT_ERR_NULL = 1,            /* a required pointer is NULL */
    CONVROT_ERR_GROUP = 2,           /* group is not 64 or 256 */
    CONVROT_ERR_SHAPE = 3,           /* negative dim, K % group, K out of range */
    CONVROT_ERR_ALIGN = 4,           /* a pointer is not 16-byte aligned */
    CONVROT_ERR_WORKSPACE = 5,       /* workspace smaller than required */
    CONVROT_ERR_CUDA = 6,            /* a CUDA runtime call or launch failed */
    CONVROT_ERR_DEVICE_TIMEOUT = 7,  /* a bounded device wait ran out */
    CONVROT_ERR_UNSUPPORTED = 8,     /* device is not sm_100 */
    CONVROT_ERR_SCRATCH_LIMIT = 9,   /* needs more than the built-in scratch array */
    CONVROT_ERR_NOT_DEVICE = 10,     /* a pointer is not memory of the current device */
    CONVROT_ERR_OVERLAP = 11         /* input and output buffers overlap */
} convrot_status;

/* Human-readable name of a status (static storage, never NULL).  The pages
 * have no counterpart: their Python API raises instead ("mlx-nf4" README,
 * "Quantize and multiply": an explicit reference path, no silent fallback). */
const char *convrot_status_string(convrot_status s);

/*
 * Steps 1-2 on weights (offline).  w_bf16: [N][K] bf16.  Writes qw: [N][K/2]
 * bytes (packed codes) and sw: [N] fp32 scales.  Source: "convrot-mlx"
 * README, "Install and test" (quantize_convrot_weight -> qweight, scales).
 */
convrot_status convrot_quantize_weight(const void *w_bf16, int64_t N, int64_t K, int group,
                                       uint8_t *qw, float *sw, convrot_stream_t stream);

/*
 * Steps 1-2 on activations: the fused prep kernel (one CTA per row).
 * x_bf16: [M][K] bf16.  Writes qx: [M][K/2] bytes and sx: [M] fp32.
 * Source: "convrot-mlx" README, "What is included" (fused activation prep).
 */
convrot_status convrot_prepare_act(const void *x_bf16, int64_t M, int64_t K, int group,
                                   uint8_t *qx, float *sx, convrot_stream_t stream);

/*
 * Split K (the pages have no counterpart: it is how the integer product is
 * scheduled on 148 SMs, not what it computes).  Where the output tiles leave
 * the last wave of the persistent GEMM part-filled, the tiles of that wave
 * are split into 2-4 ranges of K; each part writes its int32 partial sums to
 * a split area, and the part that finishes last adds them and runs the
 * epilogue.  Integer addition is exact, so the result is bit-identical to
 * the unsplit product.  A split area is CONVROT_SPLIT_AREA_BYTES bytes,
 * 256-byte aligned: CONVROT_SPLIT_COUNTER_BYTES of counters that must be
 * zero before a launch (each launch that completes leaves them zero), then
 * the partial slots (one wave of 256 x 256 int32 tiles).
 */
#define CONVROT_SPLIT_COUNTER_BYTES ((size_t)8192)
#define CONVROT_SPLIT_AREA_BYTES (CONVROT_SPLIT_COUNTER_BYTES + (size_t)160 * 128 * 256 * 4)

/* Bytes of workspace convrot_linear needs: the packed codes [M][K/2] and the
 * fp32 scales [M] of the prepared activations, each region rounded up to 256
 * bytes, then (M > 128, where the token-major GEMM runs) a split area of
 * CONVROT_SPLIT_AREA_BYTES.  Host-only; 0 for M <= 0 or K <= 0.  Source:
 * "convrot-mlx" README, "What is included" (fused activation preparation
 * into the N x packed-K layout and one absmax scale per row). */
size_t convrot_linear_workspace_size(int64_t M, int64_t K);

/*
 * Steps 1-4, the whole layer: prep kernel into `workspace`, then the
 * tcgen05 INT GEMM with the fused scale/bias/bf16 epilogue.
 * x_bf16 [M][K] bf16; qw [N][K/2] and sw [N] from convrot_quantize_weight
 * with the same group; bias_bf16 [N] bf16 or NULL (zeros); y_bf16 [M][N].
 * workspace: ws_bytes >= convrot_linear_workspace_size(M, K), 256-byte
 * aligned.  A workspace that holds the codes and scales but not the split
 * area (ws_bytes >= the size less CONVROT_SPLIT_AREA_BYTES) is accepted and
 * runs without split K, with the same results.  The prep kernel zeroes the
 * split counters, so the workspace needs no initialisation.  Source:
 * "convrot-mlx" README, "Install and test" (the complete path is rotation,
 * activation quantisation, the integer product, scaling and bias).
 */
convrot_status convrot_linear(const void *x_bf16, const uint8_t *qw, const float *sw,
                              const void *bias_bf16, int64_t M, int64_t N, int64_t K, int group,
                              void *workspace, size_t ws_bytes, void *y_bf16,
                              convrot_stream_t stream);

/*
 * Steps 3-4 only, on prepared operands: qx [M][K/2], sx [M], qw [N][K/2],
 * sw [N], bias [N] bf16 or NULL, y [M][N] bf16.  K is the unpacked length
 * (a multiple of 64).  Source: "convrot-mlx" README, "What is included"
 * (the packed INT4 product) and "Install and test" (the integer product,
 * then scaling and bias).
 */
convrot_status convrot_linear_prepared(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                       const float *sw, const void *bias_bf16, int64_t M,
                                       int64_t N, int64_t K, void *y_bf16,
                                       convrot_stream_t stream);

/*
 * convrot_linear_prepared with a split area (split_ws, split_bytes >=
 * CONVROT_SPLIT_AREA_BYTES, 256-byte aligned, else CONVROT_ERR_WORKSPACE),
 * so that the GEMM may split K as convrot_linear does.  Its counters must be
 * zero before the first call (e.g. one memset when the area is allocated);
 * every call that completes leaves them zero, so later calls need nothing.
 * After CONVROT_ERR_DEVICE_TIMEOUT zero them again.  Calls that use one area
 * must be ordered on the GPU.  split_ws = NULL runs without split K.
 */
convrot_status convrot_linear_prepared_split(const uint8_t *qx, const float *sx,
                                             const uint8_t *qw, const float *sw,
                                             const void *bias_bf16, int64_t M, int64_t N,
                                             int64_t K, void *split_ws, size_t split_bytes,
                                             void *y_bf16, convrot_stream_t stream);

/*
 * The reversible weight repack.  "convrot-mlx" README, "What is included"
 * (lossless repacking of the packed weights for the kernels that read them)
 * and "Install and test" (repack_nk_weight_for_mpp).  The pages repack for
 * Apple's MPP layout; here the same bytes are reordered, without loss, into
 * the order the B200 kernels stream them: every row of the canonical
 * N x packed-K layout qw [N][K/2] is cut into 128-byte column blocks (256
 * codes), and block b of all N rows is stored before block b + 1:
 *     qw_rep[(b * N + n) * 128 + j] = qw[n * (K/2) + b * 128 + j],
 * b < ceil(K / 256), j < 128, zero where b * 128 + j >= K/2.  A kernel's
 * slice of rows then reads each block as one contiguous run instead of N
 * strided 128-byte pieces.
 *
 * convrot_repacked_weight_size: bytes of qw_rep, N * ceil(K/256) * 128
 * (host-only; 0 for N <= 0 or K <= 0).
 * convrot_repack_weight: qw [N][K/2] -> qw_rep.  convrot_unpack_weight: the
 * exact inverse, qw_rep -> qw.  Device pointers, 16-byte aligned, the two
 * buffers must not overlap (CONVROT_ERR_OVERLAP); K a multiple of 64 up to
 * CONVROT_MAX_K.  One kernel on `stream`.
 *
 * convrot_linear_repacked / convrot_linear_prepared_repacked: convrot_linear
 * and convrot_linear_prepared with the weights given as qw_rep (same
 * arguments otherwise); the results are bit-identical to the canonical
 * calls on the unpacked weights.
 */
size_t convrot_repacked_weight_size(int64_t N, int64_t K);
convrot_status convrot_repack_weight(const uint8_t *qw, int64_t N, int64_t K, uint8_t *qw_rep,
                                     convrot_stream_t stream);
convrot_status convrot_unpack_weight(const uint8_t *qw_rep, int64_t N, int64_t K, uint8_t *qw,
                                     convrot_stream_t stream);
convrot_status convrot_linear_repacked(const void *x_bf16, const uint8_t *qw_rep, const float *sw,
                                       const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                       int group, void *workspace, size_t ws_bytes, void *y_bf16,
                                       convrot_stream_t stream);
convrot_status convrot_linear_prepared_repacked(const uint8_t *qx, const float *sx,
                                                const uint8_t *qw_rep, const float *sw,
                                                const void *bias_bf16, int64_t M, int64_t N,
                                                int64_t K, void *y_bf16, convrot_stream_t stream);

/*
 * Test hook: step 1 alone, through the same prep kernel.  Writes the
 * normalised rotated rows y_rot [M][K] as fp32.  Exposes the block rotation
 * X R = [X_1 H, ..., X_G H] (Comfy-Org/comfy-quants issue, section 1).
 */
convrot_status convrot_debug_rotate_f32(const void *x_bf16, int64_t M, int64_t K, int group,
                                        float *y_rot, convrot_stream_t stream);

/*
 * Test hook: step 3 alone, through the same GEMM kernel.  Writes the exact
 * integer accumulators acc [M][N] as int32 (|acc| <= 49 K always fits).
 * Exposes the integer product of "convrot-mlx" README, "Install and test".
 */
convrot_status convrot_debug_gemm_s32(const uint8_t *qx, const uint8_t *qw, int64_t M, int64_t N,
                                      int64_t K, int32_t *acc, convrot_stream_t stream);

/*
 * Whether convrot_linear runs a layer of this shape as one kernel: 1 when
 * 1 <= M <= 4, K is a multiple of 2048 up to 16384 and the few token rows'
 * buffers fit in shared memory beside the weight ring, so the rows are
 * prepared inside the GEMM kernel (activation preparation fused into a
 * CUDA-core GEMV; the workspace is then not touched); 0 when it runs the
 * prep kernel and the GEMM.  Depends on (M, K, group) only.  Host-only, no
 * device work; invalid arguments give 0.  Both forms give bit-identical
 * results.  The pages' analogue is the skinny verification kernel that reads
 * each weight once for a few rows ("mlx-kquant" METADATA, "Performance").
 */
int convrot_linear_single_kernel(int64_t M, int64_t K, int group);

/*
 * Test hook: steps 3-4 (out_s32 = 0: y [M][N] bf16, as convrot_linear_prepared)
 * or step 3 alone (out_s32 = 1: acc [M][N] int32, sx / sw / bias unused) with
 * the token-major GEMM forced to one tile shape, so that each shape can be
 * checked whatever the automatic choice for (M, N, K) would be:
 *   tiles = 0  automatic (as the entry points above);
 *           1  128 x 256 tiles, both operands widened in shared memory;
 *           2  128 x 192 tiles, A widened into TMEM;
 *           3  256 x 192 tiles on CTA pairs (cta_group::2);
 *           4  few-token form (M <= 128): weights widened into TMEM, one
 *              CTA per slice of weight rows (the automatic choice there);
 *           5  few-token form with both operands widened in shared memory;
 *           6  256 x 128 tiles on CTA pairs (four TMEM A stages);
 *           7  few-token form on CTA pairs (M <= 128): each CTA widens its
 *              slice of weight rows into its TMEM and holds half of the
 *              token columns; one cta_group::2 MMA covers both slices.
 * tiles | CONVROT_TILES_REPACKED takes qw in the repacked layout
 * (convrot_repack_weight); form 5 with M <= 16 reads 256-byte boxes and
 * does not take it (CONVROT_ERR_UNSUPPORTED).
 * Returns CONVROT_ERR_SHAPE for any other value or for 4 / 5 / 7 with
 * M > 128, and CONVROT_ERR_UNSUPPORTED when the device cannot co-schedule
 * CTA pairs (tiles = 3, 6, 7).  Exposes steps 3-4 ("convrot-mlx" README,
 * "Install and test": the integer product, scaling and bias) per GEMM form.
 */
#define CONVROT_TILES_REPACKED 0x100
convrot_status convrot_debug_gemm_tiles(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                        const float *sw, const void *bias_bf16, int64_t M,
                                        int64_t N, int64_t K, int tiles, int out_s32, void *out,
                                        convrot_stream_t stream);

/*
 * Test hook, host-only (no device work): the GEMM form and split-K plan
 * convrot_linear chooses for (M, N, K) on a device with `pairs` co-resident
 * CTA pairs (0: none) and `sms` SMs, given a split area of split_bytes
 * (0: none).  *tiles is the form as numbered for convrot_debug_gemm_tiles
 * (4 for the few-token form, M <= 128); the first *split_tiles output tiles
 * are cut into *splits ranges of K (0 and 1: no split).  CONVROT_ERR_NULL
 * for a NULL output, CONVROT_ERR_SHAPE for K outside 64 .. CONVROT_MAX_K or
 * not a multiple of 64, negative sizes, pairs < 0 or sms <= 0.  Exposes the
 * scheduling of step 3 ("convrot-mlx" README, "Install and test": the
 * integer product), which changes no result.
 */
convrot_status convrot_debug_gemm_plan(int64_t M, int64_t N, int64_t K, int pairs, int sms,
                                       size_t split_bytes, int *tiles, int *split_tiles,
                                       int *splits);

/*
 * Test hook: convrot_debug_gemm_tiles for a token-major form (tiles 0-3 or
 * 6, optionally | CONVROT_TILES_REPACKED) with a given split-K plan: the
 * first split_tiles output tiles (tile t covers rows (t mod TA) x TM and
 * columns (t / TA) x BN, TA = ceil(M / TM)) are each cut into `splits`
 * contiguous ranges of K-stages; split_tiles = 0 runs every tile whole,
 * split_tiles = -1 takes the planner's choice for this area.  The split area
 * is that of convrot_linear_prepared_split (counters zero on entry, zero
 * again when the call completes).  CONVROT_ERR_SHAPE when the plan does not
 * fit: split_tiles above the tile count, splits outside 2 .. the K-stages of
 * a tile, or slots or counters beyond the area.  Exposes the scheduling of
 * step 3 ("convrot-mlx" README, "Install and test": the integer product) and
 * shows it does not change a bit of the result.
 */
convrot_status convrot_debug_gemm_split(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                        const float *sw, const void *bias_bf16, int64_t M,
                                        int64_t N, int64_t K, int tiles, int split_tiles,
                                        int splits, void *split_ws, size_t split_bytes,
                                        int out_s32, void *out, convrot_stream_t stream);

/*
 * The whole layer, like convrot_linear, for callers that cannot give the
 * library any device memory of their own: a plugin called by a host runtime
 * that owns every allocation and passes no workspace, or a caller on a
 * latency-critical path that must not call cudaMalloc (it can synchronise the
 * device and take milliseconds).  The pages have no counterpart to this
 * entry point; it exists only for such callers.
 *
 * Instead of a caller-provided workspace it uses one fixed array of
 * CONVROT_NOALLOC_SCRATCH_BYTES in the library's own device memory.  Every
 * GPU that loads the library holds that array until the process exits.
 * Requests needing more (round256(M*K/2) + round256(4*M) bytes, the codes
 * and scales of convrot_linear_workspace_size without its split area; this
 * entry point does not split K) fail with
 * CONVROT_ERR_SCRATCH_LIMIT before anything is launched; e.g. M = 4096 with
 * K = 4096 fits (8 MiB), M = 8192 with K = 4096 (16 MiB + 32 KiB) does not.
 *
 * The array is shared by every call on a device and keeps the last call's
 * contents; the prep kernel overwrites every byte the GEMM then reads, so
 * nothing needs clearing between calls.  Calls whose work overlaps on the
 * GPU (for example on two streams without ordering between them) race on the
 * array and give undefined results: order them.  The first call on each
 * device looks up the array's device address once (cudaGetSymbolAddress with
 * that device current); make that first call before any stream capture.
 * Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * Shapes that convrot_linear runs as one kernel (convrot_linear_single_kernel)
 * run as that kernel here too and do not touch the array.
 * Arguments, layouts and errors are otherwise those of convrot_linear.
 */
#define CONVROT_NOALLOC_SCRATCH_BYTES (16u << 20)
convrot_status convrot_linear_noalloc(const void *x_bf16, const uint8_t *qw, const float *sw,
                                      const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                      int group, void *y_bf16, convrot_stream_t stream);

/*
 * Failure detection (the pages have no counterpart: their kernels do not
 * report device-side errors).  Synchronises `stream`, then returns and
 * clears the device error word of the current device: CONVROT_ERR_DEVICE_TIMEOUT if a bounded wait in any kernel
 * of this library ran out since the last check, CONVROT_ERR_CUDA if the
 * synchronisation itself failed, CONVROT_OK otherwise.
 */
convrot_status convrot_check_device_error(convrot_stream_t stream);

/*
 * Test hook for the timeout path (no counterpart on the pages; it exercises
 * the failure detection above): launches one CTA that waits on a
 * shared-memory barrier nothing ever signals, giving up after timeout_ns
 * nanoseconds (clamped to [1e3, 5e9]); it then records
 * CONVROT_ERR_DEVICE_TIMEOUT in the device error word and returns normally.
 */
convrot_status convrot_debug_timeout_probe(int64_t timeout_ns, convrot_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H_ */
