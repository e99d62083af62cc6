// C ABI of libosm: argument checking, plans, host-side calibration
// finalisation and the host-buffer end-to-end entry point. The device work
// itself lives in osm_quant.cu and osm_gemm.cu.

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <numeric>
#include <vector>

#include "osm_internal.h"

namespace osm {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
}

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int check_cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return OSM_OK;
    return fail(OSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

float pow2f(int g) { return std::ldexp(1.0f, g); }
float nvfp4_k(int g) { return std::ldexp(1.0f / 6.0f, -g); }

// The kernels are built for sm_100a only.
static int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(OSM_ERR_CUDA, "no CUDA device");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(OSM_ERR_UNSUPPORTED, "device %d is sm_%d%d; libosm kernels are built for sm_100a", dev,
                    major, minor);
    return OSM_OK;
}

static int check_plan(const osm_plan* p) {
    if (!p) return fail(OSM_ERR_INVALID_ARG, "plan is NULL");
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != p->device) return fail(OSM_ERR_INVALID_ARG, "plan belongs to device %d, current is %d", p->device, dev);
    return OSM_OK;
}

#define OSM_REQUIRE(cond, ...)                                        \
    do {                                                              \
        if (!(cond)) return fail(OSM_ERR_INVALID_ARG, __VA_ARGS__);   \
    } while (0)

#define OSM_TRY(expr)             \
    do {                          \
        int rc_ = (expr);         \
        if (rc_) return rc_;      \
    } while (0)

}  // namespace osm

using namespace osm;

extern "C" {

const char* osm_last_error(void) { return g_err; }

int osm_act_amax_accumulate(const uint16_t* X, int64_t T, int64_t K, float* amax, void* stream) {
    g_err[0] = 0;
    OSM_REQUIRE(T >= 0 && K > 0 && K % 32 == 0, "act_amax: need T >= 0, K > 0, K %% 32 == 0 (T=%lld K=%lld)",
                (long long)T, (long long)K);
    OSM_REQUIRE(amax && aligned16(amax), "act_amax: amax must be a 16-byte aligned device pointer");
    OSM_REQUIRE(T == 0 || (X && aligned16(X)), "act_amax: X must be a 16-byte aligned device pointer");
    OSM_TRY(check_device());
    return launch_act_amax(X, T, K, amax, static_cast<cudaStream_t>(stream));
}

int osm_weight_amax(const uint16_t* W, int64_t K, int64_t N, float* wmax, void* stream) {
    g_err[0] = 0;
    OSM_REQUIRE(K > 0 && N > 0 && N % 32 == 0 && K <= 0x7FFFFFFF, "weight_amax: need K > 0, N %% 32 == 0");
    OSM_REQUIRE(W && aligned16(W) && wmax, "weight_amax: null or misaligned pointer");
    OSM_TRY(check_device());
    return launch_weight_amax(W, K, N, wmax, static_cast<cudaStream_t>(stream));
}

int osm_calibrate_finalize_scored(const float* amax_host, const float* score_host, const float* wmax_host, int64_t K,
                                  float alpha, int64_t k, float* s_host, float* inv_s_host, int32_t* O_host) {
    g_err[0] = 0;
    OSM_REQUIRE(amax_host && score_host && wmax_host && s_host && inv_s_host, "calibrate_finalize: null pointer");
    OSM_REQUIRE(K > 0 && k >= 0 && k <= K, "calibrate_finalize: need 0 <= k <= K");
    OSM_REQUIRE(k == 0 || O_host, "calibrate_finalize: O_host is NULL");
    OSM_REQUIRE(alpha > 0.0f && alpha < 1.0f, "calibrate_finalize: alpha must lie in (0, 1)");
    for (int64_t j = 0; j < K; ++j)
        if (!std::isfinite(amax_host[j]) || !std::isfinite(wmax_host[j]) || !std::isfinite(score_host[j]))
            return fail(OSM_ERR_NONFINITE, "calibrate_finalize: statistic of channel %lld is not finite",
                        (long long)j);
    // Eq. (2) in double, statistics floored at 1e-5, rounded once to float
    const double a = static_cast<double>(alpha);
    for (int64_t j = 0; j < K; ++j) {
        const double am = std::max(static_cast<double>(amax_host[j]), 1e-5);
        const double wm = std::max(static_cast<double>(wmax_host[j]), 1e-5);
        s_host[j] = static_cast<float>(std::pow(am, a) / std::pow(wm, 1.0 - a));
        inv_s_host[j] = 1.0f / s_host[j];
    }
    // Eq. (4): top-k by score, ties to the lower channel index
    if (k > 0) {
        std::vector<int32_t> idx(static_cast<size_t>(K));
        std::iota(idx.begin(), idx.end(), 0);
        std::partial_sort(idx.begin(), idx.begin() + k, idx.end(), [&](int32_t x, int32_t y) {
            if (score_host[x] != score_host[y]) return score_host[x] > score_host[y];
            return x < y;
        });
        std::sort(idx.begin(), idx.begin() + k);
        std::copy(idx.begin(), idx.begin() + k, O_host);
    }
    return OSM_OK;
}

int osm_calibrate_finalize(const float* amax_host, const float* wmax_host, int64_t K, float alpha, int64_t k,
                           float* s_host, float* inv_s_host, int32_t* O_host) {
    return osm_calibrate_finalize_scored(amax_host, amax_host, wmax_host, K, alpha, k, s_host, inv_s_host, O_host);
}

int osm_act_percentile(const uint16_t* X, int64_t T, int64_t K, float q, float* score, void* stream) {
    g_err[0] = 0;
    OSM_REQUIRE(T >= 1 && K > 0 && K % 32 == 0 && K <= 0x7FFFFFFF, "act_percentile: need T >= 1, K %% 32 == 0");
    OSM_REQUIRE(q > 0.0f && q <= 1.0f, "act_percentile: q must lie in (0, 1]");
    OSM_REQUIRE(X && aligned16(X) && score, "act_percentile: null or misaligned pointer");
    OSM_TRY(check_device());
    double r = std::ceil(static_cast<double>(q) * static_cast<double>(T));
    if (r < 1.0) r = 1.0;
    if (r > static_cast<double>(T)) r = static_cast<double>(T);
    return launch_act_percentile(X, T, K, static_cast<int64_t>(r), score, static_cast<cudaStream_t>(stream));
}

int osm_plan_create(int64_t K, int64_t N, int64_t k, const float* s_host, const int32_t* O_host, int wscale_mode,
                    osm_plan** out) {
    g_err[0] = 0;
    OSM_REQUIRE(out, "plan_create: out is NULL");
    *out = nullptr;
    OSM_REQUIRE(K > 0 && K % 32 == 0 && K <= 65536, "plan_create: need 0 < K <= 65536, K %% 32 == 0 (K=%lld)",
                (long long)K);
    OSM_REQUIRE(N > 0 && N % 32 == 0 && N <= (int64_t(1) << 30), "plan_create: need N > 0, N %% 32 == 0 (N=%lld)",
                (long long)N);
    OSM_REQUIRE(k >= 0 && k <= K, "plan_create: need 0 <= k <= K (k=%lld)", (long long)k);
    OSM_REQUIRE(s_host, "plan_create: s_host is NULL");
    OSM_REQUIRE(k == 0 || O_host, "plan_create: O_host is NULL");
    OSM_REQUIRE(wscale_mode >= OSM_WSCALE_1x32 && wscale_mode <= OSM_WSCALE_STRIP128x1,
                "plan_create: unknown weight scale mode %d", wscale_mode);
    for (int64_t j = 0; j < K; ++j)
        OSM_REQUIRE(std::isfinite(s_host[j]) && s_host[j] > 0.0f, "plan_create: s[%lld] is not finite and positive",
                    (long long)j);
    for (int64_t i = 0; i < k; ++i) {
        OSM_REQUIRE(O_host[i] >= 0 && O_host[i] < K, "plan_create: O[%lld] out of range", (long long)i);
        OSM_REQUIRE(i == 0 || O_host[i] > O_host[i - 1], "plan_create: O must be strictly ascending");
    }
    OSM_TRY(check_device());

    osm_plan* p = new (std::nothrow) osm_plan();
    if (!p) return fail(OSM_ERR_NOMEM, "plan_create: host allocation failed");
    cudaGetDevice(&p->device);
    p->K = K;
    p->N = N;
    p->k = k;
    p->Kb = K - k;
    p->Kbp = round_up(K - k, 128);
    p->kp = round_up(k, 64);
    p->wmode = wscale_mode;
    p->hp_fp16 = 0;
    p->fmt = OSM_FMT_MXFP4;
    p->g_act = 0;
    p->g_w = 0;
    p->wait_limit_ns = 2000000000ull;
    p->debug_flags = 0;

    std::vector<float> inv_s(static_cast<size_t>(K));
    for (int64_t j = 0; j < K; ++j) inv_s[j] = 1.0f / s_host[j];
    std::vector<int32_t> route(static_cast<size_t>(K)), J, order;
    J.reserve(static_cast<size_t>(K - k));
    {
        std::vector<int32_t> slot(static_cast<size_t>(K), -1);
        for (int64_t i = 0; i < k; ++i) slot[O_host[i]] = static_cast<int32_t>(i);
        for (int64_t j = 0; j < K; ++j) {
            if (slot[j] >= 0) {
                route[j] = static_cast<int32_t>((p->Kbp / 32) * QA_BLOCK_BYTES + 2 * slot[j]);
            } else {
                const int64_t pos = static_cast<int64_t>(J.size());
                route[j] = static_cast<int32_t>((pos / 32) * QA_BLOCK_BYTES + (pos % 32) * 2);
                J.push_back(static_cast<int32_t>(j));
            }
        }
    }
    order = J;
    order.insert(order.end(), O_host, O_host + k);
    std::vector<float> inv_s_ord(static_cast<size_t>(K));
    for (int64_t c = 0; c < K; ++c) inv_s_ord[c] = inv_s[order[c]];
    auto cleanup = [&](int code) {
        osm_plan_destroy(p);
        return code;
    };
    cudaError_t e = cudaSuccess;
    e = cudaMalloc(&p->d_s, sizeof(float) * K);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_inv_s, sizeof(float) * K);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_route, sizeof(int32_t) * K);
    if (e == cudaSuccess && K - k > 0) e = cudaMalloc(&p->d_J, sizeof(int32_t) * (K - k));
    if (e == cudaSuccess && k > 0) e = cudaMalloc(&p->d_O, sizeof(int32_t) * k);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_status, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMalloc(&p->d_order, sizeof(int32_t) * K);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_inv_s_ord, sizeof(float) * K);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_s_new, sizeof(float) * 3 * K);  // s, inv_s, ranks
    if (e == cudaSuccess) e = cudaMalloc(&p->d_bad, sizeof(uint32_t));
    if (e != cudaSuccess) return cleanup(fail(OSM_ERR_NOMEM, "plan_create: %s", cudaGetErrorString(e)));
    e = cudaMemcpy(p->d_s, s_host, sizeof(float) * K, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(p->d_inv_s, inv_s.data(), sizeof(float) * K, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(p->d_route, route.data(), sizeof(int32_t) * K, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && K - k > 0)
        e = cudaMemcpy(p->d_J, J.data(), sizeof(int32_t) * (K - k), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && k > 0) e = cudaMemcpy(p->d_O, O_host, sizeof(int32_t) * k, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(p->d_status, 0, sizeof(uint32_t));
    // osm_plan_refresh expects its flag and rank scratch zeroed on entry
    if (e == cudaSuccess) e = cudaMemset(p->d_bad, 0, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(p->d_s_new + 2 * K, 0, sizeof(float) * K);
    if (e == cudaSuccess) e = cudaMemcpy(p->d_order, order.data(), sizeof(int32_t) * K, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(p->d_inv_s_ord, inv_s_ord.data(), sizeof(float) * K, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cleanup(fail(OSM_ERR_CUDA, "plan_create: %s", cudaGetErrorString(e)));
    *out = p;
    return OSM_OK;
}

int osm_plan_destroy(osm_plan* p) {
    if (!p) return OSM_OK;
    cudaFree(p->d_s);
    cudaFree(p->d_inv_s);
    cudaFree(p->d_route);
    cudaFree(p->d_J);
    cudaFree(p->d_O);
    cudaFree(p->d_status);
    cudaFree(p->d_order);
    cudaFree(p->d_inv_s_ord);
    cudaFree(p->d_s_new);
    cudaFree(p->d_bad);
    delete p;
    return OSM_OK;
}

int osm_plan_sizes(const osm_plan* p, int64_t rows, size_t* codes_bytes, size_t* scales_bytes, size_t* hp_bytes) {
    g_err[0] = 0;
    OSM_REQUIRE(p, "plan_sizes: plan is NULL");
    OSM_REQUIRE(rows >= 0, "plan_sizes: rows < 0");
    if (codes_bytes) *codes_bytes = static_cast<size_t>(rows * (p->Kbp / 2));
    if (scales_bytes) *scales_bytes = static_cast<size_t>(osm::scales_bytes(rows, p->Kbp, p->fmt));
    if (hp_bytes) *hp_bytes = static_cast<size_t>(rows * p->kp * 2);
    return OSM_OK;
}

int osm_plan_dims(const osm_plan* p, int64_t* K, int64_t* N, int64_t* k, int64_t* Kb, int64_t* Kbp, int64_t* kp) {
    g_err[0] = 0;
    OSM_REQUIRE(p, "plan_dims: plan is NULL");
    if (K) *K = p->K;
    if (N) *N = p->N;
    if (k) *k = p->k;
    if (Kb) *Kb = p->Kb;
    if (Kbp) *Kbp = p->Kbp;
    if (kp) *kp = p->kp;
    return OSM_OK;
}

int osm_plan_status(const osm_plan* p, void* stream, uint32_t* status_host, int clear) {
    g_err[0] = 0;
    OSM_REQUIRE(status_host, "plan_status: status_host is NULL");
    OSM_TRY(check_plan(p));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    OSM_TRY(check_cuda(cudaStreamSynchronize(st), "plan_status: stream synchronize"));
    OSM_TRY(check_cuda(cudaMemcpy(status_host, p->d_status, sizeof(uint32_t), cudaMemcpyDeviceToHost),
                       "plan_status: read"));
    if (clear) OSM_TRY(check_cuda(cudaMemset(p->d_status, 0, sizeof(uint32_t)), "plan_status: clear"));
    return OSM_OK;
}

int osm_plan_set_wait_limit(osm_plan* p, uint64_t ns) {
    g_err[0] = 0;
    OSM_REQUIRE(p, "plan_set_wait_limit: plan is NULL");
    OSM_REQUIRE(ns >= 1000ull, "plan_set_wait_limit: limit below 1 us");
    p->wait_limit_ns = ns;
    return OSM_OK;
}

int osm_plan_set_outlier_dtype(osm_plan* p, int dtype) {
    g_err[0] = 0;
    OSM_REQUIRE(p, "plan_set_outlier_dtype: plan is NULL");
    OSM_REQUIRE(dtype == OSM_HP_BF16 || dtype == OSM_HP_FP16, "plan_set_outlier_dtype: unknown type %d", dtype);
    OSM_REQUIRE(dtype == OSM_HP_BF16 || p->fmt == OSM_FMT_MXFP4,
                "plan_set_outlier_dtype: an NVFP4 plan keeps a BF16 outlier branch");
    p->hp_fp16 = dtype == OSM_HP_FP16;
    return OSM_OK;
}

int osm_plan_set_format(osm_plan* p, int format, int g_act, int g_w) {
    g_err[0] = 0;
    OSM_REQUIRE(p, "plan_set_format: plan is NULL");
    OSM_REQUIRE(format == OSM_FMT_MXFP4 || format == OSM_FMT_NVFP4, "plan_set_format: unknown format %d", format);
    if (format == OSM_FMT_NVFP4) {
        OSM_REQUIRE(g_act >= -100 && g_act <= 100 && g_w >= -100 && g_w <= 100 && std::abs(g_act + g_w) <= 126,
                    "plan_set_format: exponents must lie in [-100, 100], |g_act + g_w| <= 126 (%d, %d)", g_act, g_w);
        OSM_REQUIRE(p->wmode == OSM_WSCALE_1x32, "plan_set_format: NVFP4 needs the OSM_WSCALE_1x32 weight mode");
        OSM_REQUIRE(!p->hp_fp16, "plan_set_format: NVFP4 needs the BF16 outlier branch");
    }
    p->fmt = format;
    p->g_act = format == OSM_FMT_NVFP4 ? g_act : 0;
    p->g_w = format == OSM_FMT_NVFP4 ? g_w : 0;
    return OSM_OK;
}

int osm_nvfp4_tensor_exponent(float amax, int* g) {
    g_err[0] = 0;
    OSM_REQUIRE(g, "nvfp4_tensor_exponent: g is NULL");
    OSM_REQUIRE(std::isfinite(amax) && amax >= 0.0f, "nvfp4_tensor_exponent: amax must be finite and >= 0");
    int e = 0;
    if (amax > 0.0f) {
        e = -100;
        while (e < 100 && static_cast<double>(amax) > std::ldexp(2688.0, e)) ++e;
    }
    *g = e;
    return OSM_OK;
}

// bf16(fp32 v), round to nearest even (v finite)
static float bf16_round_host(float v) {
    uint32_t u;
    std::memcpy(&u, &v, 4);
    const uint32_t lsb = (u >> 16) & 1u;
    u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
    float r;
    std::memcpy(&r, &u, 4);
    return r;
}

int osm_nvfp4_plan_exponents(const float* amax, const float* wmax, const float* s, const float* inv_s,
                             const int32_t* O, int64_t K, int64_t k, int* g_act, int* g_w) {
    g_err[0] = 0;
    OSM_REQUIRE(amax && wmax && s && inv_s && g_act && g_w, "nvfp4_plan_exponents: null pointer");
    OSM_REQUIRE(K > 0 && k >= 0 && k <= K && (k == 0 || O), "nvfp4_plan_exponents: bad K / k / O");
    std::vector<char> out(static_cast<size_t>(K), 0);
    for (int64_t i = 0; i < k; ++i) {
        OSM_REQUIRE(O[i] >= 0 && O[i] < K, "nvfp4_plan_exponents: O[%lld] out of range", (long long)i);
        out[O[i]] = 1;
    }
    float am = 0.0f, wm = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        if (out[j]) continue;
        const float a = std::fabs(bf16_round_host(amax[j] * inv_s[j]));
        const float w = std::fabs(bf16_round_host(wmax[j] * s[j]));
        OSM_REQUIRE(std::isfinite(a) && std::isfinite(w), "nvfp4_plan_exponents: statistic %lld not finite",
                    (long long)j);
        am = std::max(am, a);
        wm = std::max(wm, w);
    }
    OSM_TRY(osm_nvfp4_tensor_exponent(am, g_act));
    return osm_nvfp4_tensor_exponent(wm, g_w);
}

int osm_plan_set_debug(osm_plan* p, uint32_t flags) {
    g_err[0] = 0;
    OSM_REQUIRE(p, "plan_set_debug: plan is NULL");
    OSM_REQUIRE((flags & ~static_cast<uint32_t>(OSM_DEBUG_STARVE_QUANTIZE)) == 0, "plan_set_debug: unknown flag");
    p->debug_flags = flags;
    return OSM_OK;
}

int osm_pack_weights(const osm_plan* p, const uint16_t* W, uint8_t* w_codes, uint8_t* w_scales, uint16_t* w_hp,
                     void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    OSM_REQUIRE(W && aligned16(W), "pack_weights: W must be a 16-byte aligned device pointer");
    OSM_REQUIRE(p->Kbp == 0 || (w_codes && aligned16(w_codes) && w_scales && aligned16(w_scales)),
                "pack_weights: w_codes / w_scales null or misaligned");
    OSM_REQUIRE(p->kp == 0 || (w_hp && aligned16(w_hp)), "pack_weights: w_hp null or misaligned");
    OSM_TRY(check_device());
    return launch_pack_weights(p, W, nullptr, w_codes, w_scales, w_hp, static_cast<cudaStream_t>(stream));
}

int osm_pack_weights_for_next(const osm_plan* p, const osm_plan* next, const uint16_t* W, uint8_t* w_codes,
                              uint8_t* w_scales, uint16_t* w_hp, void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    OSM_TRY(check_plan(next));
    OSM_REQUIRE(next->K == p->N, "pack_weights_for_next: next->K (%lld) must equal plan->N (%lld)",
                (long long)next->K, (long long)p->N);
    OSM_REQUIRE(W && aligned16(W), "pack_weights_for_next: W must be a 16-byte aligned device pointer");
    OSM_REQUIRE(p->Kbp == 0 || (w_codes && aligned16(w_codes) && w_scales && aligned16(w_scales)),
                "pack_weights_for_next: w_codes / w_scales null or misaligned");
    OSM_REQUIRE(p->kp == 0 || (w_hp && aligned16(w_hp)), "pack_weights_for_next: w_hp null or misaligned");
    OSM_TRY(check_device());
    return launch_pack_weights(p, W, next->d_order, w_codes, w_scales, w_hp, static_cast<cudaStream_t>(stream));
}

int osm_plan_channel_order(const osm_plan* p, int32_t* order_host) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    OSM_REQUIRE(order_host, "plan_channel_order: order_host is NULL");
    return check_cuda(cudaMemcpy(order_host, p->d_order, sizeof(int32_t) * p->K, cudaMemcpyDeviceToHost),
                      "plan_channel_order: read");
}

int osm_plan_refresh_scored(osm_plan* p, const float* amax, const float* score, const float* wmax, float alpha,
                            void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    auto ok = [](const float* x) { return x && (reinterpret_cast<uintptr_t>(x) & 3) == 0; };
    OSM_REQUIRE(ok(amax) && ok(score) && ok(wmax), "plan_refresh: amax / score / wmax null or misaligned");
    OSM_REQUIRE(alpha > 0.0f && alpha < 1.0f, "plan_refresh: alpha must lie in (0, 1)");
    return launch_plan_refresh(p, amax, score, wmax, alpha, static_cast<cudaStream_t>(stream));
}

int osm_plan_refresh(osm_plan* p, const float* amax, const float* wmax, float alpha, void* stream) {
    return osm_plan_refresh_scored(p, amax, amax, wmax, alpha, stream);
}

int osm_plan_tables(const osm_plan* p, float* s_host, float* inv_s_host, int32_t* O_host) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    cudaError_t e = cudaSuccess;
    if (s_host) e = cudaMemcpy(s_host, p->d_s, sizeof(float) * p->K, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && inv_s_host)
        e = cudaMemcpy(inv_s_host, p->d_inv_s, sizeof(float) * p->K, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && O_host && p->k > 0)
        e = cudaMemcpy(O_host, p->d_O, sizeof(int32_t) * p->k, cudaMemcpyDeviceToHost);
    return check_cuda(e, "plan_tables: read");
}

int osm_error_norms(const float* Y, const float* Yref, int64_t count, double* out, void* stream) {
    g_err[0] = 0;
    OSM_REQUIRE(count >= 1, "error_norms: count must be >= 1");
    OSM_REQUIRE(Y && Yref && out && (reinterpret_cast<uintptr_t>(out) & 7) == 0,
                "error_norms: null or misaligned pointer");
    OSM_TRY(check_device());
    return launch_error_norms(Y, Yref, count, out, static_cast<cudaStream_t>(stream));
}

int osm_gelu_f32(const float* x, float* y, int64_t n, void* stream) {
    g_err[0] = 0;
    OSM_REQUIRE(n >= 1, "gelu_f32: n must be >= 1");
    OSM_REQUIRE(x && y && (reinterpret_cast<uintptr_t>(x) & 3) == 0 && (reinterpret_cast<uintptr_t>(y) & 3) == 0,
                "gelu_f32: null or misaligned pointer");
    OSM_TRY(check_device());
    return launch_gelu_f32(x, y, n, static_cast<cudaStream_t>(stream));
}

int osm_quantize_act(const osm_plan* p, const uint16_t* X, int64_t M, uint8_t* a_codes, uint8_t* a_scales,
                     uint16_t* a_hp, void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    OSM_REQUIRE(M >= 1 && M <= (int64_t(1) << 31) - 1, "quantize_act: need 1 <= M < 2^31");
    OSM_REQUIRE(X && aligned16(X), "quantize_act: X must be a 16-byte aligned device pointer");
    OSM_REQUIRE(p->Kbp == 0 || (a_codes && aligned16(a_codes) && a_scales && aligned16(a_scales)),
                "quantize_act: a_codes / a_scales null or misaligned");
    OSM_REQUIRE(p->kp == 0 || (a_hp && aligned16(a_hp)), "quantize_act: a_hp null or misaligned");
    return launch_quantize_act(p, X, M, a_codes, a_scales, a_hp, static_cast<cudaStream_t>(stream));
}

int osm_dual_gemm(const osm_plan* p, const uint8_t* a_codes, const uint8_t* a_scales, const uint16_t* a_hp,
                  int64_t M, const uint8_t* w_codes, const uint8_t* w_scales, const uint16_t* w_hp,
                  const float* bias, int epi, void* Y, const osm_plan* next, uint8_t* next_codes,
                  uint8_t* next_scales, uint16_t* next_hp, void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    OSM_REQUIRE(M >= 1 && M <= (int64_t(1) << 31) - 1, "dual_gemm: need 1 <= M < 2^31");
    OSM_REQUIRE(epi == OSM_EPI_F32 || epi == OSM_EPI_BF16 || epi == OSM_EPI_GELU_BF16 || epi == OSM_EPI_GELU_REQUANT,
                "dual_gemm: unknown epilogue %d", epi);
    if (epi == OSM_EPI_GELU_REQUANT) {
        OSM_TRY(check_plan(next));
        OSM_REQUIRE(next->K == p->N, "dual_gemm: next->K (%lld) must equal plan->N (%lld)", (long long)next->K,
                    (long long)p->N);
        OSM_REQUIRE(!Y && !bias, "dual_gemm: GELU_REQUANT writes next_* only; Y and bias must be NULL");
        OSM_REQUIRE(p->fmt == OSM_FMT_MXFP4 && next->fmt == OSM_FMT_MXFP4,
                    "dual_gemm: GELU_REQUANT needs MXFP4 plans");
        OSM_REQUIRE(next->Kbp == 0 || (next_codes && aligned16(next_codes) && next_scales && aligned16(next_scales)),
                    "dual_gemm: next_codes / next_scales null or misaligned");
        OSM_REQUIRE(next->kp == 0 || (next_hp && aligned16(next_hp)), "dual_gemm: next_hp null or misaligned");
    } else {
        OSM_REQUIRE(!next && !next_codes && !next_scales && !next_hp,
                    "dual_gemm: next-layer buffers need OSM_EPI_GELU_REQUANT");
        OSM_REQUIRE(Y && aligned16(Y), "dual_gemm: Y must be a 16-byte aligned device pointer");
        OSM_REQUIRE(!bias || aligned16(bias), "dual_gemm: bias must be 16-byte aligned");
    }
    OSM_REQUIRE(p->Kbp == 0 || (a_codes && aligned16(a_codes) && a_scales && aligned16(a_scales) && w_codes &&
                                aligned16(w_codes) && w_scales && aligned16(w_scales)),
                "dual_gemm: bulk operands null or misaligned");
    OSM_REQUIRE(p->kp == 0 || (a_hp && aligned16(a_hp) && w_hp && aligned16(w_hp)),
                "dual_gemm: outlier operands null or misaligned");
    OSM_TRY(check_device());
    return launch_dual_gemm(p, a_codes, a_scales, a_hp, M, w_codes, w_scales, w_hp, bias, epi, Y, next, next_codes,
                            next_scales, next_hp, static_cast<cudaStream_t>(stream));
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t osm_linear_workspace_size(const osm_plan* p, int64_t M, int epi) {
    if (!p || M < 1 || M > (int64_t(1) << 31) - 1) return 0;
    size_t cb, sb, hb;
    osm_plan_sizes(p, M, &cb, &sb, &hb);
    const size_t yb = static_cast<size_t>(M * p->N) * (epi == OSM_EPI_BF16 ? 2 : 4);
    return align256(static_cast<size_t>(M * p->K * 2)) + align256(cb) + align256(sb) + align256(hb) + align256(yb);
}

int osm_linear_host(const osm_plan* p, const uint16_t* X_host, int64_t M, const uint8_t* w_codes,
                    const uint8_t* w_scales, const uint16_t* w_hp, const float* bias, int epi, void* Y_host,
                    void* workspace, size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(p));
    OSM_REQUIRE(X_host && Y_host, "linear_host: X_host / Y_host is NULL");
    OSM_REQUIRE(M >= 1 && M <= (int64_t(1) << 31) - 1, "linear_host: need 1 <= M < 2^31");
    OSM_REQUIRE(epi == OSM_EPI_F32 || epi == OSM_EPI_BF16, "linear_host: epilogue must be F32 or BF16");
    const size_t need = osm_linear_workspace_size(p, M, epi);
    OSM_REQUIRE(workspace && aligned16(workspace) && workspace_bytes >= need,
                "linear_host: workspace needs %zu bytes", need);
    size_t cb, sb, hb;
    osm_plan_sizes(p, M, &cb, &sb, &hb);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t* dX = reinterpret_cast<uint16_t*>(ws);
    ws += align256(static_cast<size_t>(M * p->K * 2));
    uint8_t* codes = ws;
    ws += align256(cb);
    uint8_t* scales = ws;
    ws += align256(sb);
    uint16_t* hp = reinterpret_cast<uint16_t*>(ws);
    ws += align256(hb);
    void* dY = ws;
    const size_t yb = static_cast<size_t>(M * p->N) * (epi == OSM_EPI_BF16 ? 2 : 4);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    OSM_TRY(check_cuda(cudaMemcpyAsync(dX, X_host, static_cast<size_t>(M * p->K * 2), cudaMemcpyHostToDevice, st),
                       "linear_host: copy X"));
    OSM_TRY(osm_quantize_act(p, dX, M, codes, scales, hp, stream));
    OSM_TRY(osm_dual_gemm(p, codes, scales, hp, M, w_codes, w_scales, w_hp, bias, epi, dY, nullptr, nullptr,
                          nullptr, nullptr, stream));
    return check_cuda(cudaMemcpyAsync(Y_host, dY, yb, cudaMemcpyDeviceToHost, st), "linear_host: copy Y");
}

// ---- one FFN block: quantize_act(up) -> dual_gemm(up, GELU_REQUANT) -> dual_gemm(down, BF16)

size_t osm_ffn_workspace_size(const osm_plan* up, const osm_plan* down, int64_t M) {
    if (!up || !down || M < 1 || M > (int64_t(1) << 31) - 1 || up->N != down->K) return 0;
    size_t cu, su, hu, cd, sd, hd;
    osm_plan_sizes(up, M, &cu, &su, &hu);
    osm_plan_sizes(down, M, &cd, &sd, &hd);
    return align256(cu) + align256(su) + align256(hu) + align256(cd) + align256(sd) + align256(hd);
}

size_t osm_ffn_host_workspace_size(const osm_plan* up, const osm_plan* down, int64_t M) {
    const size_t inner = osm_ffn_workspace_size(up, down, M);
    if (!inner) return 0;
    return inner + align256(static_cast<size_t>(M * up->K * 2)) + align256(static_cast<size_t>(M * down->N * 2));
}

int osm_ffn_block(const osm_plan* up, const osm_plan* down, const uint16_t* X, int64_t M, const uint8_t* wu_codes,
                  const uint8_t* wu_scales, const uint16_t* wu_hp, const uint8_t* wd_codes, const uint8_t* wd_scales,
                  const uint16_t* wd_hp, const float* bias_down, uint16_t* Y, void* workspace,
                  size_t workspace_bytes, void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(up));
    OSM_TRY(check_plan(down));
    OSM_REQUIRE(up->N == down->K, "ffn_block: up->N (%lld) must equal down->K (%lld)", (long long)up->N,
                (long long)down->K);
    OSM_REQUIRE(M >= 1 && M <= (int64_t(1) << 31) - 1, "ffn_block: need 1 <= M < 2^31");
    const size_t need = osm_ffn_workspace_size(up, down, M);
    OSM_REQUIRE(workspace && aligned16(workspace) && workspace_bytes >= need, "ffn_block: workspace needs %zu bytes",
                need);
    size_t cu, su, hu, cd, sd, hd;
    osm_plan_sizes(up, M, &cu, &su, &hu);
    osm_plan_sizes(down, M, &cd, &sd, &hd);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* a_codes = ws;
    ws += align256(cu);
    uint8_t* a_scales = ws;
    ws += align256(su);
    uint16_t* a_hp = reinterpret_cast<uint16_t*>(ws);
    ws += align256(hu);
    uint8_t* h_codes = ws;
    ws += align256(cd);
    uint8_t* h_scales = ws;
    ws += align256(sd);
    uint16_t* h_hp = reinterpret_cast<uint16_t*>(ws);
    // every argument of the three calls is checked by them before anything is
    // enqueued; a failure of the second or third leaves the earlier work queued
    OSM_TRY(osm_quantize_act(up, X, M, a_codes, a_scales, a_hp, stream));
    OSM_TRY(osm_dual_gemm(up, a_codes, a_scales, a_hp, M, wu_codes, wu_scales, wu_hp, nullptr, OSM_EPI_GELU_REQUANT,
                          nullptr, down, h_codes, h_scales, h_hp, stream));
    return osm_dual_gemm(down, h_codes, h_scales, h_hp, M, wd_codes, wd_scales, wd_hp, bias_down, OSM_EPI_BF16, Y,
                         nullptr, nullptr, nullptr, nullptr, stream);
}

int osm_ffn_block_host(const osm_plan* up, const osm_plan* down, const uint16_t* X_host, int64_t M,
                       const uint8_t* wu_codes, const uint8_t* wu_scales, const uint16_t* wu_hp,
                       const uint8_t* wd_codes, const uint8_t* wd_scales, const uint16_t* wd_hp,
                       const float* bias_down, uint16_t* Y_host, void* workspace, size_t workspace_bytes,
                       void* stream) {
    g_err[0] = 0;
    OSM_TRY(check_plan(up));
    OSM_TRY(check_plan(down));
    OSM_REQUIRE(X_host && Y_host, "ffn_block_host: X_host / Y_host is NULL");
    OSM_REQUIRE(up->N == down->K, "ffn_block_host: up->N (%lld) must equal down->K (%lld)", (long long)up->N,
                (long long)down->K);
    OSM_REQUIRE(M >= 1 && M <= (int64_t(1) << 31) - 1, "ffn_block_host: need 1 <= M < 2^31");
    const size_t need = osm_ffn_host_workspace_size(up, down, M);
    OSM_REQUIRE(workspace && aligned16(workspace) && workspace_bytes >= need,
                "ffn_block_host: workspace needs %zu bytes", need);
    const size_t xb = static_cast<size_t>(M * up->K * 2), yb = static_cast<size_t>(M * down->N * 2);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t* dX = reinterpret_cast<uint16_t*>(ws);
    ws += align256(xb);
    uint16_t* dY = reinterpret_cast<uint16_t*>(ws);
    ws += align256(yb);
    const size_t inner = osm_ffn_workspace_size(up, down, M);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    OSM_TRY(check_cuda(cudaMemcpyAsync(dX, X_host, xb, cudaMemcpyHostToDevice, st), "ffn_block_host: copy X"));
    OSM_TRY(osm_ffn_block(up, down, dX, M, wu_codes, wu_scales, wu_hp, wd_codes, wd_scales, wd_hp, bias_down, dY, ws,
                          inner, stream));
    return check_cuda(cudaMemcpyAsync(Y_host, dY, yb, cudaMemcpyDeviceToHost, st), "ffn_block_host: copy Y");
}

int osm_scales_to_logical(const uint8_t* sw, int64_t rows, int64_t nblocks, uint8_t* logical) {
    g_err[0] = 0;
    OSM_REQUIRE(rows >= 0 && nblocks >= 0 && nblocks % 4 == 0, "scales_to_logical: nblocks must be a multiple of 4");
    OSM_REQUIRE((rows == 0 || nblocks == 0) || (sw && logical), "scales_to_logical: null pointer");
    const int64_t katoms = nblocks / 4;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nblocks; ++b)
            logical[r * nblocks + b] =
                sw[((r / 128) * katoms + b / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (b % 4)];
    return OSM_OK;
}

}  // extern "C"
