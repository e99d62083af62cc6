// Allocation-free device forward of the layer: quantize_act -> dual_gemm
// with the packed activations (codes, scales, outlier slots) held in a
// file-scope static device array instead of caller-provided buffers.
//
// Who needs this: callers that create their plans and pack their weights
// at load time but cannot allocate device memory when the layer runs. A
// serving runtime that reserves the GPU's memory up front for its own pool
// leaves nothing for a cudaMalloc, and a plug-in that a host framework
// hands only tensors and a stream has no access to that framework's
// allocator; cudaMalloc and cudaFree would also synchronise the whole
// device in the middle of other streams' work. Such callers pass only X,
// the packed weights and Y; the scratch is in this file.
//
// The array is module data: every GPU that loads the library holds its own
// copy of it until the process exits. In host code `g_act_scratch` is only
// a host-side stand-in for the symbol, never a device address, so the
// device address is looked up with cudaGetSymbolAddress, once per device,
// with that device current.

#include <cuda_runtime.h>

#include <mutex>

#include "osm_internal.h"

namespace {

static __device__ __align__(256) uint8_t g_act_scratch[OSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t* g_scratch_dev[kMaxDevices] = {};  // device address of g_act_scratch, per device

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of the scratch array on the current device (set up on the
// first call on each device).
int scratch_for_current_device(uint8_t** out) {
    int dev = 0;
    if (int rc = osm::check_cuda(cudaGetDevice(&dev), "linear_noalloc: cudaGetDevice")) return rc;
    if (dev < 0 || dev >= kMaxDevices) return osm::fail(OSM_ERR_UNSUPPORTED, "linear_noalloc: device index %d", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_dev[dev]) {
        void* ptr = nullptr;
        if (int rc = osm::check_cuda(cudaGetSymbolAddress(&ptr, g_act_scratch),
                                     "linear_noalloc: cudaGetSymbolAddress of the static scratch"))
            return rc;
        g_scratch_dev[dev] = static_cast<uint8_t*>(ptr);
    }
    *out = g_scratch_dev[dev];
    return OSM_OK;
}

}  // namespace

extern "C" OSM_API int osm_linear_noalloc(const osm_plan* p, const uint16_t* X, int64_t M, const uint8_t* w_codes,
                                          const uint8_t* w_scales, const uint16_t* w_hp, const float* bias, int epi,
                                          void* Y, void* stream) {
    using namespace osm;
    if (!p) return fail(OSM_ERR_INVALID_ARG, "linear_noalloc: plan is NULL");
    if (M < 1) return fail(OSM_ERR_INVALID_ARG, "linear_noalloc: M must be >= 1");
    // Every row takes at least one byte of packed activations, so a batch
    // above this many rows cannot fit; checked before the size arithmetic
    // below, whose 64-bit products would wrap for absurd M.
    if (M > static_cast<int64_t>(OSM_NOALLOC_SCRATCH_BYTES))
        return fail(OSM_ERR_UNSUPPORTED,
                    "linear_noalloc: M=%lld rows cannot fit the static scratch of %u bytes; split the batch or use "
                    "osm_quantize_act + osm_dual_gemm",
                    (long long)M, (unsigned)OSM_NOALLOC_SCRATCH_BYTES);
    if (epi != OSM_EPI_F32 && epi != OSM_EPI_BF16)
        return fail(OSM_ERR_INVALID_ARG, "linear_noalloc: epilogue must be OSM_EPI_F32 or OSM_EPI_BF16");
    size_t cb = 0, sb = 0, hb = 0;
    if (int rc = osm_plan_sizes(p, M, &cb, &sb, &hb)) return rc;
    const size_t need = align256(cb) + align256(sb) + align256(hb);
    if (need > OSM_NOALLOC_SCRATCH_BYTES) {
        const size_t per_row = (cb + sb + hb) / static_cast<size_t>(M) + 1;
        return fail(OSM_ERR_UNSUPPORTED,
                    "linear_noalloc: M=%lld needs %zu bytes of packed activations but the static scratch holds %u "
                    "(about %zu rows for this plan); split the batch or use osm_quantize_act + osm_dual_gemm",
                    (long long)M, need, (unsigned)OSM_NOALLOC_SCRATCH_BYTES,
                    static_cast<size_t>(OSM_NOALLOC_SCRATCH_BYTES) / per_row);
    }
    uint8_t* base = nullptr;
    if (int rc = scratch_for_current_device(&base)) return rc;
    // quantize_act rewrites every byte that dual_gemm reads (all codes, all
    // scale bytes including the padding rows, all outlier slots), so nothing
    // left by an earlier call needs clearing.
    uint8_t* codes = base;
    uint8_t* scales = codes + align256(cb);
    uint16_t* hp = reinterpret_cast<uint16_t*>(scales + align256(sb));
    if (int rc = osm_quantize_act(p, X, M, codes, scales, hp, stream)) return rc;
    return osm_dual_gemm(p, codes, scales, hp, M, w_codes, w_scales, w_hp, bias, epi, Y, nullptr, nullptr, nullptr,
                         nullptr, stream);
}
