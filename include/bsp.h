/*
 * bsp.h -- C ABI of libbsp: block-scaled (NVFP4 W4A4 / MXFP8 W8A8) linear
 * layers on NVIDIA B200 (sm_100a).
 *
 * The library is the hot path of a quantized linear layer:
 *
 *   codes, scales = quantize(x)                     (bf16 -> block-scaled)
 *   D = alpha * (A (x) sfA) (B (x) sfB)^T + bias     (tensor cores, fp32 accumulate)
 *
 * Sources (page title, then the symbol or section on it):
 *   hao-ai-lab-FastVideo  fastvideo/layers/quantization/nvfp4_qat_config.py
 *       NVFP4QATQuantizeMethod.apply, convert_model_to_fp4
 *   hao-ai-lab-FastVideo  fastvideo/layers/quantization/nvfp4_config.py
 *       module docstring, _nvfp4_quantize, _mm_fp4, the fastvideo_fp4 custom
 *       ops and their register_fake shape functions, NVFP4QuantizeMethod.apply
 *   sgl-project sglang    python/sglang/srt/layers/quantization/nvfp4_online.py
 *       ModelOptNvFp4OnlineFusedMoEMethod._quantize_weight_nvfp4,
 *       NvFp4OnlineConfig (per-token activation scales)
 *   vllm-omni             vllm_omni/quantization/mxfp8_config.py
 *       DiffusionMXFP8Config, NPUMxfp8LinearMethod._quant_matmul
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless stated; the caller
 *     allocates and owns every buffer.  The library never allocates, frees,
 *     synchronises, or reads device memory from the host (except
 *     bsp_device_status, which exists to do exactly that).  Calls are
 *     asynchronous on `stream` (NULL = the legacy default stream).
 *   - bf16 tensors are passed as `const uint16_t*` (their bit patterns).
 *   - Matrices are row-major; `ld_*` is the row stride in ELEMENTS.
 *   - Return value: a bsp_status.  Arguments are checked on the host first;
 *     a non-zero status means nothing was launched.
 *   - The current CUDA device must be an sm_100 GPU (B200/GB200), else
 *     BSP_ERR_UNSUPPORTED_DEVICE.  (The pages gate NVFP4 on compute
 *     capability 100: NVFP4QATConfig.get_min_capability.)
 *   - Kernels bound every wait on the GPU.  A wait that runs out sets a
 *     device error word instead of hanging; bsp_device_status reports it.
 */
#ifndef BSP_H
#define BSP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (pointer to the runtime's opaque stream). */
typedef struct CUstream_st *bsp_stream_t;

typedef enum {
    BSP_OK = 0,
    BSP_ERR_INVALID_ARG = 1,        /* a size, mode or pointer argument is not allowed */
    BSP_ERR_ALIGNMENT = 2,          /* a pointer or leading dimension is misaligned */
    BSP_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100 */
    BSP_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    BSP_ERR_TIMEOUT = 5             /* a bounded wait on the GPU ran out (bsp_device_status) */
} bsp_status;

/* Scale modes of nvfp4_quantize. */
enum {
    BSP_SF_PER_TENSOR = 0, /* one fp32 encode scale for the whole tensor */
    BSP_SF_PER_ROW = 1     /* one fp32 encode scale per row, computed in-kernel */
};

/* Output element types of the GEMMs. */
enum {
    BSP_OUT_BF16 = 0,
    BSP_OUT_F32 = 1
};

/* Input element types of nvfp4_quantize_ex. */
enum {
    BSP_IN_BF16 = 0,
    BSP_IN_F16 = 1
};

/* Scale-factor tile layouts (FastVideo nvfp4_config.py: SfLayout.layout_128x4
 * and layout_8x4, the latter with rows padded to 8, `row_tile = 8`). */
enum {
    BSP_SF_LAYOUT_128X4 = 0,
    BSP_SF_LAYOUT_8X4 = 1
};

/* Norms of the fused norm + quantize producers (bsp_debug_norm_stats). */
enum {
    BSP_NORM_RMS = 0,
    BSP_NORM_LAYER = 1
};

/* Human-readable name of a status code (static string, never NULL). */
const char *bsp_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int bsp_version(void);

/* ------------------------------------------------------------------------
 * Scale-factor buffer sizes.
 * Scales are stored in the 128x4 tile layout the pages name ("layout_128x4
 * scale layout", nvfp4_config.py module docstring; _nvfp4_quantize pads rows
 * to 128 for it).  Logical scale (r, c) of a [rows, cols] scale matrix lives at
 *   ((r/128) * (cols4/4) + c/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + c%4
 * with cols4 = cols rounded up to a multiple of 4; padding bytes are 0.
 * The buffer holds round_up(rows,128) * round_up(cols,4) bytes.
 * ---------------------------------------------------------------------- */

/* NVFP4: cols = K/16 (one e4m3 scale per 16 elements).  0 if K % 16 != 0. */
size_t bsp_nvfp4_sf_bytes(int64_t rows, int64_t K);
/* The same for a scale layout: BSP_SF_LAYOUT_128X4 as above; BSP_SF_LAYOUT_8X4
 * stores 32-byte tiles of 8 rows x 4 columns, row-major inside a tile, tiles
 * ordered by row tile then column tile:
 *   ((r/8) * (cols4/4) + c/4) * 32 + (r%8)*4 + c%4
 * in round_up(rows,8) * round_up(cols,4) bytes.  (The pages name layout_8x4
 * and its 8-row padding but not its byte order; this row-major tile is the
 * reading taken.)  0 for an unknown layout or K % 16 != 0. */
size_t bsp_nvfp4_sf_bytes_layout(int64_t rows, int64_t K, int sf_layout);
/* MXFP8: cols = K/32 (one e8m0 scale per 32 elements).  0 if K % 32 != 0. */
size_t bsp_mxfp8_sf_bytes(int64_t rows, int64_t K);

/* ------------------------------------------------------------------------
 * Global (per-tensor) scales.
 * ---------------------------------------------------------------------- */

/* amax = max |x_i| over n bf16 values, as the weight conversion computes it
 * (x.abs().nan_to_num().amax(): NaN counts as 0, +-inf as the largest finite
 * bf16).  nvfp4_qat_config.py, convert_model_to_fp4.
 *   x     : bf16 [n], 16-byte aligned
 *   amax  : fp32 [1], overwritten (the call zeroes it, then reduces into it)
 * Errors: n < 0 -> INVALID_ARG; misaligned x -> ALIGNMENT. */
int bsp_amax_bf16(const uint16_t *x, int64_t n, float *amax, bsp_stream_t stream);

/* As bsp_amax_bf16, but folds max |x_i| into the caller's *amax (which must
 * hold a previous amax, e.g. from bsp_amax_bf16) instead of overwriting it:
 * the amax over several tensors that must share one global scale, such as the
 * gated w1/w3 pair that nvfp4_online.py quantizes together
 * (process_loaded_weight: torch.cat of the pair, one amax-derived scale).
 *   x     : bf16 [n], 16-byte aligned
 *   amax  : fp32 [1], read and updated on the device
 * Errors as bsp_amax_bf16. */
int bsp_amax_bf16_into(const uint16_t *x, int64_t n, float *amax, bsp_stream_t stream);

/* bsp_amax_bf16 / bsp_amax_bf16_into for fp16 data (the weight of an fp16
 * model, convert_model_to_fp4): NaN counts as 0, +-inf as 65504.
 *   x : fp16 [n] bit patterns, 16-byte aligned; the rest as bsp_amax_bf16. */
int bsp_amax_f16(const uint16_t *x, int64_t n, float *amax, bsp_stream_t stream);
int bsp_amax_f16_into(const uint16_t *x, int64_t n, float *amax, bsp_stream_t stream);

/* NVFP4 encode scale from an amax, on the device (no host sync):
 *   gs = amax > 0 ? fl32(448*6 / amax) : 1.0     (convert_model_to_fp4; the
 *        all-zero guard is nvfp4_online.py _quantize_weight_nvfp4)
 *   inv_gs = fl32(1 / gs)                         (the decode scale)
 * amax, gs, inv_gs: fp32 [1].  gs or inv_gs may be NULL. */
int bsp_nvfp4_global_scale(const float *amax, float *gs, float *inv_gs, bsp_stream_t stream);

/* The same with the numerator as a parameter: gs = amax > 0 ?
 * fl32(fp8_fp4_max / amax) : 1.0, inv_gs = fl32(1 / gs).  fp8_fp4_max is
 * e4m3_max * 6: 448 * 6 = 2688 (bsp_nvfp4_global_scale) or, with the 4over6
 * setting of nvfp4_online.py _quantize_weight_nvfp4 (e4m3_max = 256 so that
 * every group scale stays <= 256), 256 * 6 = 1536.
 *   fp8_fp4_max: host value, finite and > 0 (else INVALID_ARG, nothing
 *                launched)
 * Other arguments and errors as bsp_nvfp4_global_scale. */
int bsp_nvfp4_global_scale_max(const float *amax, float fp8_fp4_max, float *gs, float *inv_gs,
                               bsp_stream_t stream);

/* alpha = fl32(1 / fl32(gs_x * gs_w)), the GEMM output scale of
 * NVFP4QATQuantizeMethod.apply.  All fp32 [1]. */
int bsp_nvfp4_alpha(const float *gs_x, const float *gs_w, float *alpha, bsp_stream_t stream);

/* Load-time weight conversion in one launch: the sequence
 *   bsp_amax_{bf16,f16}(w) -> bsp_nvfp4_global_scale_max(amax, fp8_fp4_max)
 *   -> nvfp4_quantize(w, gs) (per-tensor, layout_128x4)
 * of the weight path of nvfp4_online.py (_quantize_weight_nvfp4: amax, the
 * e4m3_max * 6 / amax global scale, quantize) and nvfp4_config.py
 * (process_weights_after_loading), with bit-identical results.  One grid of
 * co-resident blocks reduces max|w| through the workspace, meets at a grid
 * barrier, derives gs on every block and quantizes the rows last row first,
 * so that a weight smaller than L2 is read from DRAM once.
 *   w            : bf16 / fp16 [N, K] (w_dtype BSP_IN_BF16 / BSP_IN_F16), row
 *                  stride ld_w elements, 16-byte aligned
 *   N, K, ld_w   : N >= 0, K > 0 and K % 64 == 0, ld_w >= K and ld_w % 8 == 0
 *   fp8_fp4_max  : host value, finite and > 0 (2688, or 1536 for 4over6)
 *   amax         : fp32 [1] max|w| (NaN 0, +-inf the largest finite), or NULL
 *   gs, inv_gs   : fp32 [1], as bsp_nvfp4_global_scale_max
 *   codes, sf    : outputs as nvfp4_quantize (N rows; round_up(N, 128) rows of
 *                  scales, the padding rows zero); non-NULL even when N = 0
 *                  (a zero-row weight still gets its amax 0, gs 1, inv_gs 1)
 *   workspace    : device memory of workspace_bytes >= the size that
 *                  bsp_nvfp4_quantize_weight_workspace_bytes reports for this
 *                  device and w_dtype, 16-byte aligned, any content: the call
 *                  sets its two barrier words to 0 on `stream` before the
 *                  launch, so a workspace left behind by a call that timed out
 *                  is fit for the next call.  Owned by the caller; calls that
 *                  overlap in time on one workspace race.
 * Launched cooperatively (every block resident at once).  Errors:
 * INVALID_ARG (sizes, modes, NULL pointers, workspace too small), ALIGNMENT,
 * UNSUPPORTED_DEVICE, CUDA (the launch failed, e.g. a cooperative launch the
 * context does not allow); a barrier wait that runs out (2 s) raises the
 * device error word (bsp_device_status: TIMEOUT) and leaves the outputs
 * unspecified. */
int nvfp4_quantize_weight(const uint16_t *w, int w_dtype, int64_t N, int64_t K, int64_t ld_w, float fp8_fp4_max,
                          float *amax, float *gs, float *inv_gs, uint8_t *codes, uint8_t *sf, void *workspace,
                          int64_t workspace_bytes, bsp_stream_t stream);

/* Workspace bytes nvfp4_quantize_weight and nvfp4_quantize_weights need on
 * the current device for w_dtype (a 256-byte header and two words per block of
 * their grid).  Host-only. */
int bsp_nvfp4_quantize_weight_workspace_bytes(int w_dtype, int64_t *bytes);

/* One weight of an nvfp4_quantize_weights call: the arguments of
 * nvfp4_quantize_weight that differ from weight to weight (all device
 * pointers; amax may be NULL). */
#define BSP_WEIGHT_BATCH_MAX 256
typedef struct bsp_weight_desc {
    const uint16_t *w;       /* [N, K], row stride ld_w elements, 16-byte aligned */
    int64_t N, K, ld_w;      /* N >= 0, K % 64 == 0, ld_w >= K, ld_w % 8 == 0 */
    float *amax, *gs, *inv_gs;
    uint8_t *codes, *sf;
} bsp_weight_desc;

/* nvfp4_quantize_weight for up to BSP_WEIGHT_BATCH_MAX weights of one input
 * format and one fp8_fp4_max in a single cooperative launch: per weight the
 * amax, a grid barrier, gs and the quantization, with one weight's last rows
 * overlapping the next weight's amax reads (the load-time conversion of a
 * model's linears, nvfp4_qat_config.py convert_model_to_fp4, as one call).
 * Results are bit-identical to nvfp4_quantize_weight on each weight.
 *   descs    : HOST array of count descriptors (copied into the launch; the
 *              caller may reuse it as soon as the call returns)
 *   count    : 0 .. BSP_WEIGHT_BATCH_MAX (0: nothing launched)
 *   workspace: as nvfp4_quantize_weight (its size from
 *              bsp_nvfp4_quantize_weight_workspace_bytes; the two entries may
 *              share one workspace if their calls do not overlap in time)
 * Errors: INVALID_ARG or ALIGNMENT for any descriptor as nvfp4_quantize_weight
 * (nothing launched), CUDA if the launch fails; a barrier wait that runs out
 * raises the device error word. */
int nvfp4_quantize_weights(const bsp_weight_desc *descs, int count, int w_dtype, float fp8_fp4_max, void *workspace,
                           int64_t workspace_bytes, bsp_stream_t stream);

/* nvfp4_quantize_weight with no workspace argument and no allocation: its
 * scratch is a static device array inside the library (16,640 bytes: room
 * for the size bsp_nvfp4_quantize_weight_workspace_bytes reports up to grids
 * of 2048 blocks; a B200 grid is 444).  The
 * pages have no counterpart; it serves callers that can provide neither
 * scratch memory nor an allocator.  Results are those of
 * nvfp4_quantize_weight.
 *   Arguments and errors as nvfp4_quantize_weight, less the workspace; also
 *   INVALID_ARG if this device's grid needs more scratch than the array holds.
 * The first call on each device looks up the array's address
 * (cudaGetSymbolAddress, under a lock) and keeps it for the life of the
 * process; make that first call before any stream capture.  Every call clears
 * the barrier words on `stream` before its launch.  The address belongs to
 * the device's primary context: after cudaDeviceReset this entry must not be
 * called again in the same process.  There is one array per device: calls
 * that overlap in time (other streams, other host threads) race. */
int nvfp4_quantize_weight_static(const uint16_t *w, int w_dtype, int64_t N, int64_t K, int64_t ld_w,
                                 float fp8_fp4_max, float *amax, float *gs, float *inv_gs, uint8_t *codes,
                                 uint8_t *sf, bsp_stream_t stream);

/* ------------------------------------------------------------------------
 * NVFP4 quantization (nvfp4_config.py: fastvideo_fp4::nvfp4_quantize and
 * _nvfp4_quantize; module docstring: e2m1 elements, group size 16, e4m3
 * scales, fp32 global scale, layout_128x4).
 *
 * Per row m and group g of 16 consecutive elements along K:
 *   amax = max |x|;  s = fl32(fl32(amax / 6) * gs);  sfb = e4m3_rne_sat(s)
 *   inv  = sfb == 0 ? 0 : fl32(gs / value(sfb))
 *   code_i = e2m1_rne_sat(fl32(x_i * inv))  (sign kept)
 *
 *   x        : bf16 [M, K], row stride ld_x >= K elements; 16-byte aligned,
 *              ld_x % 8 == 0
 *   global_sf: PER_TENSOR -- fp32 [1], the encode scale gs (the caller passes
 *              it, so there is no hidden reduction or host sync; activations
 *              use a static 1.0 as NVFP4QATQuantizeMethod.__init__ does).
 *              PER_ROW -- ignored (may be NULL).
 *   sf_mode  : BSP_SF_PER_TENSOR or BSP_SF_PER_ROW.  PER_ROW computes
 *              gs[m] = amax(row m) > 0 ? fl32(448*6/amax) : 1 in-kernel (the
 *              dynamic per-token activation scales of nvfp4_online.py,
 *              NvFp4OnlineConfig.use_per_token_activation).
 *   row_gs   : PER_ROW: fp32 [M] receives gs[m] (may be NULL); else unused.
 *   row_inv_gs: PER_ROW: fp32 [M] receives fl32(1/gs[m]), the per-row factor
 *              nvfp4_gemm takes as row_scale (may be NULL); else unused.
 *   codes    : uint8 [M, K/2] (dense), element 2j in the low nibble of byte j
 *              (torch.float4_e2m1fn_x2 packing, _mm_fp4); 16-byte aligned.
 *   sf       : uint8 [bsp_nvfp4_sf_bytes(M, K)] e4m3 bytes, 128x4 layout;
 *              padding rows/columns are written as 0.  16-byte aligned.
 * Rows are not padded in `codes` (the pages pad with F.pad and narrow back;
 * here padding rows exist only in `sf`).
 * Errors: K % 16 != 0, K <= 0, M < 0, ld_x < K, bad sf_mode, NULL required
 * pointer -> INVALID_ARG; alignment -> ALIGNMENT.  M == 0 is a no-op. */
int nvfp4_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                   const float *global_sf, int sf_mode, float *row_gs, float *row_inv_gs,
                   uint8_t *codes, uint8_t *sf, bsp_stream_t stream);

/* The same for fp16 input.  nvfp4_config.py (_coerce_fp4_input_dtype and
 * NVFP4QuantizeMethod.apply) feeds bf16 and fp16 activations to the quantizer
 * as they are; x_i are the exact fp16 values, and the per-row amax treats NaN
 * as 0 and +-inf as the largest finite fp16 (65504).
 *   x : fp16 [M, K] bit patterns, row stride ld_x; other arguments, layouts
 *       and errors as nvfp4_quantize. */
int nvfp4_quantize_f16(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                       const float *global_sf, int sf_mode, float *row_gs, float *row_inv_gs,
                       uint8_t *codes, uint8_t *sf, bsp_stream_t stream);

/* nvfp4_quantize with the input type and the scale layout as arguments:
 *   x_dtype  : BSP_IN_BF16 (as nvfp4_quantize) or BSP_IN_F16 (as
 *              nvfp4_quantize_f16)
 *   sf_layout: BSP_SF_LAYOUT_128X4 (as nvfp4_quantize) or BSP_SF_LAYOUT_8X4
 *              (sf holds bsp_nvfp4_sf_bytes_layout(M, K, BSP_SF_LAYOUT_8X4)
 *              bytes; padding rows up to a multiple of 8 are 0).  An 8x4
 *              activation is consumed by nvfp4_gemm_ex for M <= 64.
 * Other arguments and errors as nvfp4_quantize; an unknown x_dtype or
 * sf_layout -> INVALID_ARG. */
int nvfp4_quantize_ex(const uint16_t *x, int x_dtype, int64_t M, int64_t K, int64_t ld_x,
                      const float *global_sf, int sf_mode, int sf_layout, float *row_gs,
                      float *row_inv_gs, uint8_t *codes, uint8_t *sf, bsp_stream_t stream);

/* RMSNorm fused into the NVFP4 quantizer: the producer of the pre-quantized
 * activation that NVFP4QuantizeMethod.apply (nvfp4_config.py) accepts from a
 * fused norm+quant call.  The pages name the fused call but not its norm; this
 * is RMSNorm with a weight, whose normalised output is quantized as if it had
 * been written as bf16 and passed to nvfp4_quantize.  Per row m:
 *   ms   = mean_k x_k^2, the exact mean rounded once to fp32 (an fp64 sum with
 *          a proven error bound decides it, or, where that bound does not
 *          decide the rounding, exact integer sums)
 *   rstd = fl32(1 / sqrt(fl32(ms + eps)))   (correctly rounded)
 *   y_k  = bf16(fl32(fl32(x_k * rstd) * gamma_k))
 *   then y is quantized as nvfp4_quantize does (per-tensor global_sf, or per
 *   row gs[m] from the row amax of y), without y being stored.
 *   x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf:
 *              as nvfp4_quantize (bf16 x); K <= 2^20
 *   gamma    : bf16 [K], 16-byte aligned
 *   eps      : host fp32, finite and >= 0
 *   row_rstd : fp32 [M] receives rstd of each row (may be NULL)
 * Errors as nvfp4_quantize; eps negative or not finite, K > 2^20 ->
 * INVALID_ARG. */
int nvfp4_rmsnorm_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                           const uint16_t *gamma, float eps, const float *global_sf, int sf_mode,
                           float *row_gs, float *row_inv_gs, float *row_rstd, uint8_t *codes,
                           uint8_t *sf, bsp_stream_t stream);

/* LayerNorm fused into the NVFP4 quantizer: the same producer as
 * nvfp4_rmsnorm_quantize with the norm of the Wan-2.1 blocks whose attention
 * and FFN projections the pages quantize (nvfp4_qat_config.py
 * DEFAULT_FP4_LAYERS; nvfp4_config.py names the fused norm+quant call, not its
 * norm).  Per row m:
 *   mean = (1/K) sum_k x_k          the exact mean rounded once to fp32
 *   var  = (1/K) sum_k (x_k - mu)^2 with mu the exact mean: the exact
 *                                   population variance rounded once to fp32
 *   rstd = fl32(1 / sqrt(fl32(var + eps)))   (correctly rounded)
 *   y_k  = bf16(fl32(fl32(fl32(fl32(x_k - mean) * rstd) * gamma_k) + beta_k))
 *          (gamma and beta optional: absent, their steps are left out)
 *   then y is quantized as nvfp4_quantize does, without y being stored.
 *   x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf:
 *              as nvfp4_quantize (bf16 x); K <= 32768
 *   gamma    : bf16 [K], 16-byte aligned, or NULL (no scale)
 *   beta     : bf16 [K], 16-byte aligned, or NULL (no shift)
 *   eps      : host fp32, finite and >= 0
 *   row_mean, row_rstd : fp32 [M] receive mean and rstd of each row (each
 *              may be NULL)
 * Errors as nvfp4_quantize; eps negative or not finite, K > 32768 ->
 * INVALID_ARG. */
int nvfp4_layernorm_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                             const uint16_t *gamma, const uint16_t *beta, float eps,
                             const float *global_sf, int sf_mode, float *row_gs, float *row_inv_gs,
                             float *row_mean, float *row_rstd, uint8_t *codes, uint8_t *sf,
                             bsp_stream_t stream);

/* ------------------------------------------------------------------------
 * NVFP4 GEMM (nvfp4_qat_config.py, NVFP4QATQuantizeMethod.apply:
 * mm_fp4(x_fp4, w_fp4.T, x_scale, w_scale.T, 1/(gs_x*gs_w), bf16) then
 * out + bias).  TN: both operands are K-major.
 *
 *   D[m, n] = alpha * row_scale[m] * sum_k A(m,k) sfA(m,k/16) B(n,k) sfB(n,k/16)
 *             + bias[n]
 * computed on tcgen05 block-scaled tensor cores with fp32 accumulation, then
 * rounded once to the output type.
 *
 *   A, sfA    : nvfp4_quantize output for the activations, [M, K/2] + sf(M, K)
 *   B, sfB    : nvfp4_quantize output for the weight, [N, K/2] + sf(N, K)
 *   alpha     : fp32 [1] (device), or NULL for 1.0
 *   row_scale : fp32 [M] per-row factor (1/gs[m] of PER_ROW quantization), or NULL
 *   bias      : bf16 [N], 16-byte aligned, or NULL
 *   D         : [M, ld_d] of d_dtype (BSP_OUT_BF16 or BSP_OUT_F32), 16-byte
 *               aligned, ld_d >= N, ld_d * sizeof(elem) % 16 == 0
 * Errors: M < 0, N < 0, K <= 0, K % 32 != 0 (the packed rows must be a
 * multiple of 16 bytes for the tensor-memory-access engine), N % 8 != 0,
 * ld_d < N, bad d_dtype, NULL A/B/sfA/sfB/D -> INVALID_ARG; alignment ->
 * ALIGNMENT.  M == 0 or N == 0 is a no-op. */
int nvfp4_gemm(const uint8_t *A, const uint8_t *sfA, const uint8_t *B, const uint8_t *sfB,
               int64_t M, int64_t N, int64_t K, const float *alpha, const float *row_scale,
               const uint16_t *bias, void *D, int d_dtype, int64_t ld_d, bsp_stream_t stream);

/* nvfp4_gemm with the activation scales in a given layout (mm_fp4's
 * use_8x4_sf_layout, nvfp4_config.py _mm_fp4):
 *   a_sf_layout: BSP_SF_LAYOUT_128X4 (as nvfp4_gemm) or BSP_SF_LAYOUT_8X4, for
 *                M <= 64: sfA holds bsp_nvfp4_sf_bytes_layout(M, K,
 *                BSP_SF_LAYOUT_8X4) bytes (nvfp4_quantize_ex with that
 *                layout).  The weight scales sfB are always 128x4.
 * Other arguments and errors as nvfp4_gemm; an unknown layout, or 8X4 with
 * M > 64 -> INVALID_ARG. */
int nvfp4_gemm_ex(const uint8_t *A, const uint8_t *sfA, int a_sf_layout, const uint8_t *B,
                  const uint8_t *sfB, int64_t M, int64_t N, int64_t K, const float *alpha,
                  const float *row_scale, const uint16_t *bias, void *D, int d_dtype, int64_t ld_d,
                  bsp_stream_t stream);

/* ------------------------------------------------------------------------
 * MXFP8 quantization (mxfp8_config.py, DiffusionMXFP8Config: groups of 32
 * K-elements share one float8_e8m0fnu scale, e4m3 elements, OCP MX).
 * Per group: E = floor(log2 amax) (-inf for amax 0), e = clamp(E - 8, -127, 127),
 * scale byte = e + 127, q_i = e4m3_rne_sat(x_i * 2^-e).
 *   x  : bf16 [M, K], ld_x as for nvfp4_quantize
 *   q  : uint8 e4m3 [M, K] (dense), 16-byte aligned
 *   sf : uint8 [bsp_mxfp8_sf_bytes(M, K)] e8m0 bytes, 128x4 layout, padding 0
 * Errors: K % 32 != 0 and the rest as nvfp4_quantize. */
int mxfp8_quantize(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x,
                   uint8_t *q, uint8_t *sf, bsp_stream_t stream);

/* ------------------------------------------------------------------------
 * MXFP8 GEMM (mxfp8_config.py, NPUMxfp8LinearMethod._quant_matmul: per-group
 * e8m0 scales on both operands, bias, output in the activation dtype).
 *   D[m, n] = alpha * sum_k A(m,k) 2^eA(m,k/32) B(n,k) 2^eB(n,k/32) + bias[n]
 * Arguments as nvfp4_gemm, with A [M, K] / B [N, K] e4m3 bytes and e8m0
 * scales from mxfp8_quantize.  K % 32 != 0 -> INVALID_ARG. */
int mxfp8_gemm(const uint8_t *A, const uint8_t *sfA, const uint8_t *B, const uint8_t *sfB,
               int64_t M, int64_t N, int64_t K, const float *alpha,
               const uint16_t *bias, void *D, int d_dtype, int64_t ld_d, bsp_stream_t stream);

/* ------------------------------------------------------------------------
 * Device error word.
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns BSP_OK, BSP_ERR_TIMEOUT if a kernel's bounded wait ran out
 * since the last call, or BSP_ERR_CUDA if the synchronisation failed.
 * ---------------------------------------------------------------------- */
int bsp_device_status(bsp_stream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostics (used by the tests to pin the hardware conversions that the
 * quantize kernels use).  All buffers are device buffers of n elements.
 * ---------------------------------------------------------------------- */

/* codes[i] = e2m1 code (0..15) of v[i] by the kernels' conversion path. */
int bsp_debug_encode_e2m1(const float *v, int64_t n, uint8_t *codes, bsp_stream_t stream);
/* bytes[i] = e4m3 byte of v[i] by the kernels' conversion path. */
int bsp_debug_encode_e4m3(const float *v, int64_t n, uint8_t *bytes, bsp_stream_t stream);
/* Launches one block that waits on a shared-memory barrier nobody arrives at,
 * with a limit of `limit_ns` nanoseconds (1e3 .. 1e10).  The wait runs out and
 * sets the error word, so bsp_device_status then returns BSP_ERR_TIMEOUT. */
int bsp_debug_wait_timeout(int64_t limit_ns, bsp_stream_t stream);
/* The row statistics of the fused norms alone, as those kernels decide them:
 * per row r of bf16 x [M, K] (row stride ld_x), norm BSP_NORM_RMS writes
 * stat0[r] = ms (the exact mean of squares rounded to fp32), BSP_NORM_LAYER
 * writes stat0[r] = mean and stat1[r] = var (each exact, rounded to fp32).
 * exact_only != 0 skips the fp64 decision and always takes the exact integer
 * sums; path (int [M], or NULL) receives 0 where the fp64 error bounds settled
 * the row, 2 where the LayerNorm mean was decided from a provably exact fp64
 * sum, and 1 where the exact integer sums did.  K % 16 == 0 and the K limits
 * of the fused calls; errors as nvfp4_rmsnorm_quantize. */
int bsp_debug_norm_stats(const uint16_t *x, int64_t M, int64_t K, int64_t ld_x, int norm,
                         int exact_only, float *stat0, float *stat1, int *path, bsp_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSP_H */
