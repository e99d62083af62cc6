// Internal declarations shared by the libosm translation units.
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>

#include "osm.h"

struct osm_plan {
    int device;
    int64_t K, N, k, Kb, Kbp, kp;
    int wmode;
    int hp_fp16;         // outlier branch in binary16 (OSM_HP_FP16) instead of BF16
    int fmt;             // OSM_FMT_MXFP4 or OSM_FMT_NVFP4
    int g_act, g_w;      // NVFP4 per-tensor exponents (activations, weights)
    // device tables, owned by the plan
    float* d_s;          // [K]  smoothing vector s (Eq. (2))
    float* d_inv_s;      // [K]  1.0f / s
    int32_t* d_route;    // [K]  byte offset of channel j inside a row staged by quantize_act:
                         //      bulk position p -> (p/32)*QA_BLOCK_BYTES + (p%32)*2,
                         //      outlier slot i  -> (Kbp/32)*QA_BLOCK_BYTES + 2*i
    int32_t* d_J;        // [Kb] bulk position -> channel (ascending)
    int32_t* d_O;        // [k]  outlier slot -> channel (ascending)
    int32_t* d_order;    // [K]  channel order [J ascending | O ascending] (bulk positions, then slots)
    float* d_inv_s_ord;  // [K]  inv_s in that order: inv_s[d_order[c]]
    uint32_t* d_status;  // OSM_STATUS_* bits written by kernels
    float* d_s_new;      // [3K] scratch of osm_plan_refresh: s, inv_s, then the channels' ranks (int32)
    uint32_t* d_bad;     // scratch of osm_plan_refresh: a statistic was not finite
    uint64_t wait_limit_ns;
    uint32_t debug_flags;  // OSM_DEBUG_* (failure-detection tests)
};

namespace osm {

// Bytes of one 32-value bulk block in a row staged by quantize_act
// (64 bytes of BF16 plus 16 bytes of padding against bank conflicts).
constexpr int QA_BLOCK_BYTES = 80;

// thread-local error message
void set_error(const char* fmt, ...);
int fail(int code, const char* fmt, ...);
int check_cuda(cudaError_t e, const char* what);

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Elements per scale block: 32 (MXFP4) or 16 (NVFP4).
inline int64_t block_elems(int fmt) { return fmt == OSM_FMT_NVFP4 ? 16 : 32; }

// Bytes of one scales buffer for `rows` rows of a plan.
inline int64_t scales_bytes(int64_t rows, int64_t Kbp, int fmt) {
    return round_up(rows, 128) * (Kbp / block_elems(fmt));
}

// fp32(1/6) * 2^-g and 2^g as floats (exact for |g| <= 100).
float nvfp4_k(int g);
float pow2f(int g);

// launchers (return OSM_OK or an error code; arguments already validated)
int launch_act_amax(const uint16_t* X, int64_t T, int64_t K, float* amax, cudaStream_t st);
int launch_act_percentile(const uint16_t* X, int64_t T, int64_t K, int64_t rank, float* score, cudaStream_t st);
int launch_weight_amax(const uint16_t* W, int64_t K, int64_t N, float* wmax, cudaStream_t st);
int launch_pack_weights(const osm_plan* p, const uint16_t* W, const int32_t* col_order, uint8_t* codes,
                        uint8_t* scales, uint16_t* hp, cudaStream_t st);
int launch_plan_refresh(osm_plan* p, const float* amax, const float* score, const float* wmax, float alpha,
                        cudaStream_t st);
int launch_error_norms(const float* y, const float* r, int64_t count, double* out, cudaStream_t st);
int launch_gelu_f32(const float* x, float* y, int64_t n, cudaStream_t st);
int launch_quantize_act(const osm_plan* p, const uint16_t* X, int64_t M, uint8_t* codes,
                        uint8_t* scales, uint16_t* hp, cudaStream_t st);
int launch_dual_gemm(const osm_plan* p, const uint8_t* a_codes, const uint8_t* a_scales,
                     const uint16_t* a_hp, int64_t M, const uint8_t* w_codes,
                     const uint8_t* w_scales, const uint16_t* w_hp, const float* bias, int epi,
                     void* Y, const osm_plan* next, uint8_t* next_codes, uint8_t* next_scales,
                     uint16_t* next_hp, cudaStream_t st);

}  // namespace osm
