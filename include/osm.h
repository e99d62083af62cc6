/*
 * osm.h -- C ABI of libosm, a B200 (sm_100a) implementation of the
 * smoothed, outlier-split W4A4 linear layer described in
 * "W4A4 Quantization for Inference on Wan2.2-I2V-A14B" (ICME 2026
 * Low-Bit-width Large-Model Quantization Challenge, Sub-Challenge 1).
 *
 * The layer computes Y = X W (Eq. (1)) as
 *     Y = (X/s)_{:,J} W'^(q)_{J,:} + (X/s)_{:,O} W'^(hp)_{O,:}      (Eq. (5))
 * where s is the SmoothQuant vector of Eq. (2), W' = s (.) W are the
 * folded weights, O is the static top-k outlier channel set of Eq. (4),
 * J its complement, (q) is MXFP4 (OCP MX v1.0: E2M1 elements, one E8M0
 * scale per 32 consecutive bulk channels, round-to-nearest-even) and
 * (hp) is BF16. The 4-bit format stands in for the paper's HiF4, whose
 * bit layout the paper does not give.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless the parameter name ends in
 *     _host. BF16 tensors are passed as uint16_t bit patterns. All device
 *     pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Device work is enqueued on it and the call returns without
 *     synchronising, except where stated.
 *   - The caller allocates every tensor; sizes come from osm_plan_sizes().
 *     The library allocates device memory only in osm_plan_create() and
 *     frees it in osm_plan_destroy(). Hot-path calls allocate nothing.
 *   - Return value: OSM_OK or an OSM_ERR_* code. Nothing is enqueued when
 *     an argument check fails. osm_last_error() gives a message for the
 *     calling thread's last failure. No call aborts the process; no device
 *     code traps.
 *
 * Index sets and packed layouts (shared by activations and weights)
 *   K = input channels, k = |O|, Kb = K - k, Kbp = Kb rounded up to 128,
 *   kp = k rounded up to 64. O ascending; J = ascending complement of O,
 *   compacted to bulk positions p = 0..Kb-1. For a matrix with R rows:
 *   codes  [R][Kbp/2] u8   E2M1 of bulk position p of row r in byte
 *                          r*Kbp/2 + p/2, low nibble for even p; padding
 *                          positions p >= Kb hold code 0.
 *   scales E8M0 of 32-block b = p/32 of row r (exponent + 127), in the
 *          tcgen05 block-scale layout: 128-row x 4-block atoms of 512
 *          bytes; atom (r/128, b/4) at byte offset
 *          ((r/128) * (Kbp/128) + b/4) * 512, and inside the atom
 *          (r%32)*16 + ((r%128)/32)*4 + b%4. Rows are padded to a multiple
 *          of 128; a block with no real element (and every padding row)
 *          holds 0.
 *          NVFP4 plans (osm_plan_set_format) store one UE4M3 scale per
 *          16-block b = p/16 in the same atom layout with four 16-blocks
 *          per atom row: Kbp/64 atoms per 128 rows, Kbp/16 bytes per row.
 *   hp     [R][kp] BF16    the outlier channels O_0..O_{k-1}, zero padded
 *          (binary16 for an FP16 outlier branch; NVFP4 plans store them
 *          times 2^-g, see osm_plan_set_format).
 */
#ifndef OSM_H
#define OSM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define OSM_API __attribute__((visibility("default")))
#else
#define OSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes --------------------------------------------------- */
#define OSM_OK                 0
#define OSM_ERR_INVALID_ARG    1  /* null / misaligned pointer, bad size or mode          */
#define OSM_ERR_UNSUPPORTED    2  /* device is not sm_100, or a shape the kernels refuse  */
#define OSM_ERR_CUDA           3  /* a CUDA runtime call or a launch failed               */
#define OSM_ERR_TIMEOUT        4  /* a device-side wait gave up (reported via status)     */
#define OSM_ERR_NONFINITE      5  /* calibration statistics contain inf or NaN           */
#define OSM_ERR_NOMEM          6  /* plan allocation failed                               */

/* device status bits, returned by osm_plan_status() */
#define OSM_STATUS_TIMEOUT     1u  /* a pipeline wait of a plan's kernel ran out of time */
#define OSM_STATUS_NONFINITE   2u  /* osm_plan_refresh saw a non-finite statistic          */

typedef struct osm_plan osm_plan;

/* Weight block-scale layouts evaluated in the paper's packing paragraph
 * (Fig. 8): the exponent of a 32-block is taken from the amax of
 *   OSM_WSCALE_1x32       the block itself (plain MXFP4);
 *   OSM_WSCALE_TILE32x32  its 32 (bulk channel) x 32 (output channel) tile;
 *   OSM_WSCALE_STRIP128x1 its 128-channel K-major stripe of one output row;
 * and replicated to every 32-block inside the tile or stripe. */
typedef enum {
    OSM_WSCALE_1x32 = 0,
    OSM_WSCALE_TILE32x32 = 1,
    OSM_WSCALE_STRIP128x1 = 2
} osm_wscale_mode;

/* Epilogues of osm_dual_gemm. GELU below is the FFN's tanh form,
 * 0.5 x (1 + tanh(u)), u = sqrt(2/pi)(x + 0.044715 x^3), evaluated in FP32
 * as x / (1 + 2^z), z = -2 u log2(e), with the power of two and the
 * reciprocal on the special-function unit (osm_gelu_f32 exposes the
 * routine). It stays within 5e-7 |GELU(x)| + 2e-8 |x| of the exact
 * function; a BF16 result adds one rounding. */
typedef enum {
    OSM_EPI_F32 = 0,          /* Y [M][N] float32                                     */
    OSM_EPI_BF16 = 1,         /* Y [M][N] BF16 (RNE of the FP32 accumulator)          */
    OSM_EPI_GELU_REQUANT = 2, /* FFN hidden layer handed to `next` already quantised  */
    OSM_EPI_GELU_BF16 = 3     /* Y [M][N] BF16 = bf16(GELU(acc (+ bias)))             */
} osm_epi;

/* ---- calibration (offline) ------------------------------------------
 * "For each targeted FFN linear map we record per-input-channel activation
 * maxima, weight column ranges" (implementation/calibration paragraph).
 */

/* amax[j] = max(amax[j], max_t |X[t][j]|) for X [T][K] BF16 row-major.
 * amax is device float[K], max-merged in place (zero it before the first
 * batch), so several calibration batches accumulate. T >= 0, K > 0. */
OSM_API int osm_act_amax_accumulate(const uint16_t* X, int64_t T, int64_t K, float* amax, void* stream);

/* wmax[j] = max_n |W[j][n]| for W [K][N] BF16 row-major (input channel j,
 * output channel n); the "weight column range" of Eq. (2). Overwrites wmax
 * (device float[K]). */
OSM_API int osm_weight_amax(const uint16_t* W, int64_t K, int64_t N, float* wmax, void* stream);

/* Host-side finalisation of Eq. (2) and Eq. (4):
 *   s_j     = fp32( max(amax_j,1e-5)^alpha / max(wmax_j,1e-5)^(1-alpha) )
 *             evaluated in double;
 *   inv_s_j = 1.0f / s_j (IEEE fp32 division);
 *   O       = the k channels with the largest amax_j (score of Eq. (4);
 *             ties: lower index first), written ascending.
 * All arrays are host memory of length K (O_host: k). 0 < alpha < 1,
 * 0 <= k <= K. Returns OSM_ERR_NONFINITE if a statistic is inf/NaN. */
OSM_API int osm_calibrate_finalize(const float* amax_host, const float* wmax_host, int64_t K, float alpha,
                           int64_t k, float* s_host, float* inv_s_host, int32_t* O_host);

/* Tail-aware channel score (the activation-tail-aware percentile
 * calibration of the Tail-Aware HiFloat4 page, which builds the channel
 * mask from the tail of the activation distribution so that rare
 * calibration spikes do not decide the outlier set). score[j] = the
 * nearest-rank q-percentile of |x_tj| over the T tokens of X [T][K] BF16:
 * the value of rank ceil(q T) (clamped to [1, T], computed in FP64) in
 * ascending order. q in (0, 1]; q = 1 gives the maximum. score: device
 * float[K]. All T tokens in one call (percentiles do not merge across
 * batches). K % 32 == 0. */
OSM_API int osm_act_percentile(const uint16_t* X, int64_t T, int64_t K, float q, float* score, void* stream);

/* As osm_calibrate_finalize, with Eq. (4)'s top-k taken by score_host
 * (e.g. osm_act_percentile) while Eq. (2) keeps amax_host. Host arrays. */
OSM_API int osm_calibrate_finalize_scored(const float* amax_host, const float* score_host, const float* wmax_host,
                                          int64_t K, float alpha, int64_t k, float* s_host, float* inv_s_host,
                                          int32_t* O_host);

/* ---- plans ------------------------------------------------------------ */

/* Build a plan for one linear map with K input and N output channels,
 * smoothing vector s (host float[K], > 0, finite) and ascending outlier set
 * O (host int32[k], distinct, in [0, K)). The plan owns device copies of
 * inv_s = 1.0f/s, the channel routing table and a status word.
 * Requirements: K % 32 == 0, N % 32 == 0, 0 <= k <= K, K <= 65536.
 * The plan is bound to the current CUDA device. */
OSM_API int osm_plan_create(int64_t K, int64_t N, int64_t k, const float* s_host, const int32_t* O_host,
                    int wscale_mode, osm_plan** out);
OSM_API int osm_plan_destroy(osm_plan* plan);

/* Bytes of the packed buffers for `rows` rows (activations: rows = M;
 * weights: rows = N). scales_bytes includes the padding to 128 rows
 * (Kbp/32 bytes per row for MXFP4, Kbp/16 for NVFP4). */
OSM_API int osm_plan_sizes(const osm_plan* plan, int64_t rows, size_t* codes_bytes, size_t* scales_bytes,
                   size_t* hp_bytes);

/* K, N, k, Kb, Kbp, kp of the plan (any pointer may be NULL). */
OSM_API int osm_plan_dims(const osm_plan* plan, int64_t* K, int64_t* N, int64_t* k, int64_t* Kb,
                  int64_t* Kbp, int64_t* kp);

/* Reads (and, if clear != 0, resets) the plan's device status word. Waits
 * for `stream` to finish. status_host receives OSM_STATUS_* bits. */
OSM_API int osm_plan_status(const osm_plan* plan, void* stream, uint32_t* status_host, int clear);

/* Debug knob for failure-detection tests: the wait limit, in nanoseconds,
 * of every pipeline wait inside osm_dual_gemm and osm_quantize_act for this
 * plan (default 2e9). A wait that runs out sets OSM_STATUS_TIMEOUT and the
 * kernel returns early (its outputs are then incomplete); the context stays
 * usable. */
OSM_API int osm_plan_set_wait_limit(osm_plan* plan, uint64_t ns);

/* Number format of the outlier (high-precision) branch. The paper's
 * implementation paragraph names an FP16 outlier path; OSM_HP_BF16 is the
 * default. With OSM_HP_FP16 the outlier slots of activations and weights
 * hold the same FP32 products x * inv_s and w * s rounded once to binary16
 * (ties to even; magnitudes of 65520 and above become infinite), and the
 * branch runs as FP16 x FP16 -> FP32 MMAs; the bulk path is unchanged. Set
 * it before packing: data packed under the other type must not be used. */
#define OSM_HP_BF16 0
#define OSM_HP_FP16 1
OSM_API int osm_plan_set_outlier_dtype(osm_plan* plan, int dtype);

/* ---- second 4-bit block format: NVFP4 --------------------------------------
 * The implementation paragraph of "W4A4 Quantization for Inference on
 * Wan2.2-I2V-A14B" leaves the block format of the W4A4 bulk path open to
 * exploration. OSM_FMT_MXFP4 (default) is the OCP MXFP4 path described
 * above. OSM_FMT_NVFP4 runs the same dual product with:
 *   - E2M1 elements in blocks of 16 consecutive compacted bulk positions;
 *   - one unsigned E4M3 scale per block (bias 7, 3 mantissa bits, largest
 *     448), laid out like the E8M0 scales (128 x 4 atoms: four 16-blocks
 *     per atom row), so a scales buffer holds Kbp/16 bytes per padded row;
 *   - one power-of-two factor per tensor, 2^g_act for activations and 2^g_w
 *     for weights (see osm_nvfp4_tensor_exponent);
 *   - block scale S = E4M3_RNE_satfinite(fp32(amax_b * k)), k = fp32(1/6) *
 *     2^-g; element code = E2M1_RNE_sat(fp32(x * R)), R = fp32(1 / (S * 2^g))
 *     (R = 0 for S = 0, the block then encodes as signed zeros); the decoded
 *     element is e2m1 * S * 2^g;
 *   - the BF16 outlier branch shares the accumulator, so its stored operands
 *     carry the inverse factors: a_hp = bf16(fp32(x' * 2^-g_act)), w_hp =
 *     bf16(fp32(w' * 2^-g_w)); the epilogue multiplies the accumulator by
 *     2^(g_act + g_w) (exact) before the bias.
 * Requirements: the plan's weight scale mode is OSM_WSCALE_1x32 (read as one
 * scale per 16-block of each output channel), its outlier branch BF16, and
 * -100 <= g <= 100 with |g_act + g_w| <= 126. OSM_EPI_GELU_REQUANT needs
 * both plans in MXFP4. Set the
 * format before packing or quantising; data packed under the other format
 * must not be used. */
#define OSM_FMT_MXFP4 0
#define OSM_FMT_NVFP4 1
OSM_API int osm_plan_set_format(osm_plan* plan, int format, int g_act, int g_w);

/* Host-only: the per-tensor exponent for a tensor maximum amax (finite,
 * >= 0): the smallest g in [-100, 100] with amax <= 6 * 448 * 2^g, so that
 * the largest block scale fits E4M3; 0 for amax == 0. */
OSM_API int osm_nvfp4_tensor_exponent(float amax, int* g);

/* Host-only: g_act and g_w of a plan from its calibration statistics (the
 * inputs of osm_calibrate_finalize and its outputs s, inv_s, O): the
 * activations' tensor maximum is max over bulk channels of
 * bf16(fp32(amax_j * inv_s_j)) -- the largest smoothed calibration value --
 * and the weights' max over bulk channels of bf16(fp32(wmax_j * s_j)).
 * Activations beyond the calibration range saturate (scale 448, element 6). */
OSM_API int osm_nvfp4_plan_exponents(const float* amax_host, const float* wmax_host, const float* s_host,
                                     const float* inv_s_host, const int32_t* O_host, int64_t K, int64_t k,
                                     int* g_act, int* g_w);

/* Debug flags for failure-detection tests (no counterpart in the paper).
 * OSM_DEBUG_STARVE_QUANTIZE: osm_quantize_act expects 16 bytes more per row
 * group than its copies deliver, so every wait on a row group runs out after
 * the wait limit: the kernel sets OSM_STATUS_TIMEOUT, waits (bounded) for
 * its copies and returns; its outputs are incomplete. Nothing faults: the
 * copies themselves complete. 0 restores normal operation. */
#define OSM_DEBUG_STARVE_QUANTIZE 1u
OSM_API int osm_plan_set_debug(osm_plan* plan, uint32_t flags);

/* Channel order in which a previous layer must produce this plan's input
 * for OSM_EPI_GELU_REQUANT: order_host[c] = J[c] for c < Kb (bulk channels
 * ascending), O[c - Kb] for Kb <= c < K (outlier channels ascending).
 * order_host: host int32[K]. */
OSM_API int osm_plan_channel_order(const osm_plan* plan, int32_t* order_host);

/* ---- offline weight packing --------------------------------------------
 * "SmoothQuant scales are folded into master weights before HiF4 packing"
 * and "remaining weights are packed with block-wise scales" (packing and
 * implementation paragraphs, Fig. 8).
 * W [K][N] BF16 row-major. w' = bf16(fp32(w_jn) * s_j). Writes
 *   w_codes  [N][Kbp/2], w_scales (layout above, rows = N), w_hp [N][kp]
 * with the plan's block-scale mode. */
OSM_API int osm_pack_weights(const osm_plan* plan, const uint16_t* W, uint8_t* w_codes, uint8_t* w_scales,
                     uint16_t* w_hp, void* stream);

/* As osm_pack_weights, for the first projection of an FFN whose output
 * feeds `next` through OSM_EPI_GELU_REQUANT: packed row c (output channel)
 * is column osm_plan_channel_order(next)[c] of W, so the layer's output
 * columns come out in next's [J | O] order and every 32 consecutive bulk
 * columns form one MXFP4 block of next's input (paper: GELU and smoothing
 * act per channel, so the permutation changes no value). Requires
 * plan->N == next->K. With OSM_WSCALE_TILE32x32 the 32-row tiles are taken
 * in the permuted order. */
OSM_API int osm_pack_weights_for_next(const osm_plan* plan, const osm_plan* next, const uint16_t* W,
                                      uint8_t* w_codes, uint8_t* w_scales, uint16_t* w_hp, void* stream);

/* ---- dynamic outlier set (on-device re-calibration) -----------------------
 * Eq. (2) and Eq. (4) recomputed on the device from device statistics, so
 * that the outlier set can follow the activations per batch or per
 * denoising step (the paper leaves a dynamic set to future work; MixQ keeps
 * it online). amax, wmax: device float[K], the same statistics
 * osm_calibrate_finalize takes (osm_act_amax_accumulate, osm_weight_amax).
 * The plan keeps K, N, k and its weight-scale mode; s, inv_s, O, J and
 * every routing table are rebuilt in place with osm_calibrate_finalize's
 * arithmetic (FP64 pow may differ from the host's in the last double bit,
 * so s can differ by one FP32 ulp in rare cases; O is exact). Stream-
 * ordered, no host synchronisation. Afterwards the weights must be packed
 * again (osm_pack_weights): s is folded into them and J has changed; data
 * packed for the old plan must not be used with the new one. A non-finite
 * statistic sets OSM_STATUS_NONFINITE and leaves the plan unchanged.
 * alpha in (0, 1). The format and an NVFP4 plan's exponents g_act, g_w are
 * kept as set (they are host-side settings); a caller that wants them to
 * follow the new s sets them again with osm_plan_set_format before
 * packing. */
OSM_API int osm_plan_refresh(osm_plan* plan, const float* amax, const float* wmax, float alpha, void* stream);

/* As osm_plan_refresh, with the top-k taken by a separate device score
 * (e.g. osm_act_percentile) while s follows amax. */
OSM_API int osm_plan_refresh_scored(osm_plan* plan, const float* amax, const float* score, const float* wmax,
                                    float alpha, void* stream);

/* Copies of the plan's s, inv_s (float[K]) and O (int32[k], ascending) to
 * host memory; any pointer may be NULL. Synchronous. */
OSM_API int osm_plan_tables(const osm_plan* plan, float* s_host, float* inv_s_host, int32_t* O_host);

/* ---- per-layer alpha / k search support -----------------------------------
 * The paper suggests tuning alpha and k per layer; a search scores each
 * candidate by the relative error of the layer's output against its
 * unquantised product. out (device double[2], 8-byte aligned) receives
 * sum (Y - Yref)^2 and sum Yref^2 over `count` FP32 values, accumulated in
 * FP64 (the summation order varies between runs in the last bits). */
OSM_API int osm_error_norms(const float* Y, const float* Yref, int64_t count, double* out, void* stream);

/* The FP32 GELU routine of the FFN epilogues (OSM_EPI_GELU_BF16 and
 * OSM_EPI_GELU_REQUANT) applied element-wise: y[i] = GELU(x[i]) with exactly
 * the epilogues' arithmetic, so that tests can hold the routine to the exact
 * function. x, y: device float[n], n >= 1. */
OSM_API int osm_gelu_f32(const float* x, float* y, int64_t n, void* stream);

/* ---- runtime activation path ----------------------------------------------
 * "activations are divided in-place by s, quantized ..., and routed through
 * either the W4A4 bulk path or a narrow FP16 outlier path" (implementation
 * paragraph). X [M][K] BF16 row-major, 1 <= M < 2^31. For each row:
 *   x' = bf16(fp32(x_j) * inv_s_j);
 *   a_hp[t][i] = x'[O_i];
 *   bulk x'[J_p] -> MXFP4 with the exponent floor(log2 amax_b) - 2 of each
 *   32-block (clamped to [-127,127]; amax 0 -> -127), elements E2M1 RNE,
 *   saturating at 6; the sign bit is the sign of x'.
 * (NVFP4 plans: 16-blocks with UE4M3 scales and 2^-g_act outlier slots, as
 * osm_plan_set_format defines.)
 * Writes a_codes [M][Kbp/2], a_scales (rows padded to 128), a_hp [M][kp].
 * Rows stream through shared memory by asynchronous bulk copies; a copy
 * that does not arrive within the plan's wait limit sets OSM_STATUS_TIMEOUT
 * in the plan status (osm_plan_status). */
OSM_API int osm_quantize_act(const osm_plan* plan, const uint16_t* X, int64_t M, uint8_t* a_codes,
                     uint8_t* a_scales, uint16_t* a_hp, void* stream);

/* ---- the dual-branch GEMM ------------------------------------------------
 * Eq. (5) with Eq. (3)'s per-group scales taken per 32-block:
 *   acc[t][n] = sum_b 2^(Xa(t,b)+Xw(n,b)) sum_{p in b} e2m1(a_tp) e2m1(w_np)
 *             + sum_{i<kp} a_hp[t][i] w_hp[n][i]             (FP32 accumulate)
 *   y = acc (+ bias[n] if bias != NULL).
 * NVFP4 plans: kind::mxf4nvf4 MMAs with the 16-block UE4M3 scales, and
 *   y = 2^(g_act + g_w) acc (+ bias[n]).
 * Both branches accumulate into one tensor-memory accumulator on tcgen05
 * (block-scaled MXFP4 MMA, then BF16 MMA) before a single epilogue.
 * Operands come from osm_quantize_act / osm_pack_weights with the same
 * plan. 1 <= M < 2^31.
 *   epi = OSM_EPI_F32:       Y is float [M][N].
 *   epi = OSM_EPI_BF16:      Y is BF16  [M][N].
 *   epi = OSM_EPI_GELU_BF16: Y is BF16  [M][N] = bf16(GELU(acc + bias)).
 *   epi = OSM_EPI_GELU_REQUANT (the FFN up-projection fused with the next
 *         layer's activation path; implementation paragraph: activations
 *         are divided by s, quantised and routed): Y and bias must be NULL;
 *         the weights must come from osm_pack_weights_for_next(plan, next);
 *         for each row, h = bf16(GELU(acc)) is written straight into the
 *         next layer's packed activations, exactly as osm_quantize_act(next)
 *         would write them for the BF16 matrix H = h in next's natural
 *         channel order: next_codes [M][Kbp'/2], next_scales (rows padded to
 *         128, padding rows 0), next_hp [M][kp'] (primes: next's sizes).
 *   `next` and next_* must be NULL for the other epilogues.
 * A pipeline wait that exceeds the plan's wait limit sets the plan's
 * OSM_STATUS_TIMEOUT bit (see osm_plan_status). */
OSM_API int osm_dual_gemm(const osm_plan* plan, const uint8_t* a_codes, const uint8_t* a_scales,
                  const uint16_t* a_hp, int64_t M, const uint8_t* w_codes, const uint8_t* w_scales,
                  const uint16_t* w_hp, const float* bias, int epi, void* Y, const osm_plan* next,
                  uint8_t* next_codes, uint8_t* next_scales, uint16_t* next_hp, void* stream);

/* ---- end-to-end layer from host memory ------------------------------------
 * One forward of the layer for a host (preferably pinned) X_host [M][K]
 * BF16: copies X to the device, runs osm_quantize_act and osm_dual_gemm
 * against resident packed weights, and copies Y (F32 or BF16, per epi)
 * back to Y_host. workspace is caller-owned device memory of at least
 * osm_linear_workspace_size(plan, M, epi) bytes. Enqueued on `stream`; the
 * caller synchronises before reading Y_host. */
OSM_API size_t osm_linear_workspace_size(const osm_plan* plan, int64_t M, int epi);
OSM_API int osm_linear_host(const osm_plan* plan, const uint16_t* X_host, int64_t M, const uint8_t* w_codes,
                    const uint8_t* w_scales, const uint16_t* w_hp, const float* bias, int epi,
                    void* Y_host, void* workspace, size_t workspace_bytes, void* stream);

/* ---- one FFN block (up-projection, GELU, down-projection) -----------------
 * The FFN of a transformer block as the implementation paragraph deploys it:
 * every FFN linear map runs the smoothed, outlier-split W4A4 path, and the
 * hidden activations are "divided in-place by s, quantized ..., and routed"
 * before the down-projection. One call enqueues
 *   osm_quantize_act(up, X)                      -> up's packed activations,
 *   osm_dual_gemm(up, OSM_EPI_GELU_REQUANT, down) -> down's packed activations
 *                                                   (GELU, smoothing by down's
 *                                                   s, MXFP4 encoding fused),
 *   osm_dual_gemm(down, OSM_EPI_BF16)            -> Y [M][down->N] BF16
 *                                                   (+ bias_down[n] if given).
 * up->N must equal down->K; both plans MXFP4. Weights: wu_* packed by
 * osm_pack_weights_for_next(up, down, W_up), wd_* by osm_pack_weights(down,
 * W_down). X [M][up->K] BF16 and Y are device pointers; workspace is
 * caller-owned device memory of at least osm_ffn_workspace_size(up, down, M)
 * bytes (both layers' packed activations; contents need no clearing). The
 * result is bit-identical to issuing the three calls on separate buffers.
 * 1 <= M < 2^31. Returns the first failing call's error; a failure of the
 * second or third call leaves the earlier work enqueued. */
OSM_API size_t osm_ffn_workspace_size(const osm_plan* up, const osm_plan* down, int64_t M);
OSM_API int osm_ffn_block(const osm_plan* up, const osm_plan* down, const uint16_t* X, int64_t M,
                          const uint8_t* wu_codes, const uint8_t* wu_scales, const uint16_t* wu_hp,
                          const uint8_t* wd_codes, const uint8_t* wd_scales, const uint16_t* wd_hp,
                          const float* bias_down, uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream);

/* As osm_ffn_block for a host (preferably pinned) X_host [M][up->K] BF16 and
 * a host Y_host [M][down->N] BF16: copies X in, runs the block and copies Y
 * out, all enqueued on `stream` (the caller synchronises before reading
 * Y_host). workspace: device memory of at least
 * osm_ffn_host_workspace_size(up, down, M) bytes (the device X and Y plus
 * osm_ffn_workspace_size). */
OSM_API size_t osm_ffn_host_workspace_size(const osm_plan* up, const osm_plan* down, int64_t M);
OSM_API int osm_ffn_block_host(const osm_plan* up, const osm_plan* down, const uint16_t* X_host, int64_t M,
                               const uint8_t* wu_codes, const uint8_t* wu_scales, const uint16_t* wu_hp,
                               const uint8_t* wd_codes, const uint8_t* wd_scales, const uint16_t* wd_hp,
                               const float* bias_down, uint16_t* Y_host, void* workspace, size_t workspace_bytes,
                               void* stream);

/* ---- allocation-free device forward --------------------------------------
 * The paper has no counterpart to this entry point; it serves callers that
 * build their plans and pack their weights at load time but cannot
 * allocate device memory while the layer runs: a serving runtime that
 * reserves the GPU's memory up front for its own pool (a cudaMalloc would
 * find none, and cudaMalloc / cudaFree synchronise the device), or a
 * plug-in that its host framework hands only tensors and a stream.
 *
 * Same result as osm_quantize_act followed by osm_dual_gemm, on device
 * X [M][K] BF16 and device Y [M][N] (F32 or BF16, per epi), with no
 * activation buffers from the caller: the packed activations live in a
 * static device array of OSM_NOALLOC_SCRATCH_BYTES inside the library
 * (every GPU that loads the library holds one until the process exits).
 * It calls no allocator. A call whose packed activations (codes + scales +
 * outlier slots, each rounded up to 256 bytes; see osm_plan_sizes) exceed
 * the array -- at K = 5120, k = 128 about 5 700 tokens -- returns
 * OSM_ERR_UNSUPPORTED before launching anything (so does any M above
 * OSM_NOALLOC_SCRATCH_BYTES, checked before the sizes are computed).
 * The first call on a device looks up the array's device address; make
 * that first call before any stream capture. All calls share the array:
 * calls whose work overlaps on the GPU (different streams, or different
 * host threads, without ordering between them) race on it. A timeout sets
 * the plan's status word as osm_dual_gemm does. */
#define OSM_NOALLOC_SCRATCH_BYTES (16u << 20)
OSM_API int osm_linear_noalloc(const osm_plan* plan, const uint16_t* X, int64_t M, const uint8_t* w_codes,
                               const uint8_t* w_scales, const uint16_t* w_hp, const float* bias, int epi, void* Y,
                               void* stream);

/* ---- helpers ------------------------------------------------------------ */

/* Host-only: un-swizzle a scales buffer (layout above) of `rows` rows and
 * `nblocks` blocks (Kbp/32 for MXFP4, Kbp/16 for NVFP4) into a row-major
 * [rows][nblocks] host array. */
OSM_API int osm_scales_to_logical(const uint8_t* swizzled_host, int64_t rows, int64_t nblocks,
                          uint8_t* logical_host);

/* Message for the calling thread's most recent failed call ("" if none). */
OSM_API const char* osm_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* OSM_H */
