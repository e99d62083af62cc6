// On-device plan refresh: the calibration of "W4A4 Quantization for
// Inference on Wan2.2-I2V-A14B" (Eq. (2) smoothing vector, Eq. (4) top-k
// outlier set) recomputed from device-resident statistics, and every plan
// table derived from it rebuilt in place, so that a new outlier set can be
// adopted per batch or per denoising step without a host round trip. The
// arithmetic is that of osm_calibrate_finalize followed by osm_plan_create.
//
// Kernel 1, one thread per channel: s_j = fp32(max(amax_j,1e-5)^alpha /
// max(wmax_j,1e-5)^(1-alpha)) in FP64 and inv_s_j = 1.0f / s_j into plan
// scratch, and a flag if any statistic is not finite. For K <=
// RF_RANK_MAX_K and 0 < k < K the same launch spreads over the whole GPU
// and also counts, for every channel, the keys larger than its own (its
// rank), each CTA for 256 channels against a slice of the keys staged in
// shared memory, adding its counts atomically; channel j is selected iff
// its rank is below k (keys are unique). Two launches per refresh in all.
// Kernel 2, one CTA of 1024 threads (K <= 65536):
//  1. flag set -> OSM_STATUS_NONFINITE, every table untouched;
//  2. s, inv_s adopted from scratch;
//  3. O = the k channels with the largest key (the score -- amax for Eq. (4),
//     from the ranks of kernel 1b when it ran, otherwise as follows
//     or a tail-aware percentile -- mapped to an unsigned integer of the
//     same order, << 16 | 0xFFFF - j): keys are unique, and their order is
//     score descending, then channel index ascending.
//     The k-th largest key is found by a radix select over the 48 key bits,
//     8 bits per pass: a shared 256-bin histogram (one increment per
//     distinct digit of a warp) and a warp-parallel search from the top;
//  4. J (unselected, ascending) and O (selected, ascending) by block-wide
//     ballot scans over chunks of 1024 channels; route, order and
//     inv_s in that order follow from each channel's rank.

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "osm_internal.h"

namespace osm {
namespace {

constexpr int RF_THREADS = 1024;

struct RefreshParams {
    const float* amax;     // Eq. (2)
    const float* score;    // Eq. (4)
    const float* wmax;
    double alpha;
    int K, k, Kb, Kbp;
    const float* s_new;    // [2K]: s, then inv_s
    const uint32_t* bad;
    float* s;
    float* inv_s;
    int32_t* route;
    int32_t* J;
    int32_t* O;
    int32_t* order;
    float* inv_s_ord;
    uint32_t* status;
    const int32_t* rank;   // ranks from kernel 1b, or NULL (radix select)
};

constexpr int RF_RANK_MAX_K = 16384;  // above this the K^2 counting costs more than the radix select
constexpr int RF_RANK_SLICE = 4096;   // keys per CTA slice (16 KB of shared memory)

constexpr int RF_SMEM_KEYS = 32768;  // statistics staged in shared memory (128 KB)

// The statistic mapped to an unsigned integer of the same order (-0 taken
// as +0, so that equal values tie).
__device__ __forceinline__ uint32_t rf_ord(float a) {
    uint32_t u = __float_as_uint(a);
    if (u == 0x80000000u) u = 0u;
    return u ^ ((u >> 31) ? 0xFFFFFFFFu : 0x80000000u);
}

// 48-bit key of channel j: its ordered statistic, then 0xFFFF - j. `sk`
// holds the ordered statistics of channels below RF_SMEM_KEYS.
__device__ __forceinline__ uint64_t rf_key(const uint32_t* sk, const float* amax, int j) {
    const uint32_t u = j < RF_SMEM_KEYS ? sk[j] : rf_ord(amax[j]);
    return (static_cast<uint64_t>(u) << 16) | static_cast<uint64_t>(0xFFFF - j);
}

// Exclusive prefix of `flag` over the CTA (thread order), and the total.
__device__ __forceinline__ int block_exclusive_scan(int flag, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned b = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(b & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(b);
    __syncthreads();
    if (warp == 0) {
        const int v = warp_tot[lane];
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        warp_tot[lane] = incl - v;  // exclusive
        if (lane == 31) *total = incl;
    }
    __syncthreads();
    const int r = warp_tot[warp] + in_warp;
    __syncthreads();  // warp_tot is reused by the next call
    return r;
}

// Kernel 1: CTA (x, y) covers channels 256x .. 256x+255. The CTAs of row
// y = 0 compute s and inv_s of their channels; with `rank` set, the CTAs of
// row y >= 1 count, for their channels, the larger keys among keys
// slice*(y-1) .. slice*y-1 and add the counts to rank (zero on entry: the
// plan is created with it zeroed and plan_refresh_kernel zeroes it again).
__global__ void __launch_bounds__(256) refresh_stats_kernel(const float* __restrict__ amax,
                                                            const float* __restrict__ score,
                                                            const float* __restrict__ wmax, double alpha, int K,
                                                            int slice, float* __restrict__ s_new,
                                                            uint32_t* __restrict__ bad, int32_t* __restrict__ rank) {
    __shared__ uint32_t so[RF_RANK_SLICE];
    const int j = static_cast<int>(blockIdx.x) * 256 + threadIdx.x;
    if (blockIdx.y == 0) {
        if (j >= K) return;
        const float a = amax[j], w = wmax[j];
        if (!isfinite(a) || !isfinite(w) || !isfinite(score[j])) {
            atomicOr(bad, 1u);
        } else {
            const double am = fmax(static_cast<double>(a), 1e-5);
            const double wm = fmax(static_cast<double>(w), 1e-5);
            const float sj = static_cast<float>(pow(am, alpha) / pow(wm, 1.0 - alpha));
            s_new[j] = sj;
            s_new[K + j] = __fdiv_rn(1.0f, sj);
        }
        return;
    }
    // rows y >= 1 count (with a non-finite statistic the counts are
    // meaningless, and unused)
    const int i0 = static_cast<int>(blockIdx.y - 1) * slice;
    const int n = min(slice, K - i0);
    if (n <= 0) return;
    for (int t = threadIdx.x; t < n; t += 256) so[t] = rf_ord(score[i0 + t]);
    __syncthreads();
    if (j >= K) return;
    // key i > key j  <=>  ord_i > ord_j, or ord_i == ord_j and i < j: the
    // keys of channels below j count when >=, the others when >
    const uint32_t oj = rf_ord(score[j]);
    const int split = min(max(j - i0, 0), n);
    int cnt = 0;
#pragma unroll 4
    for (int t = 0; t < split; ++t) cnt += so[t] >= oj ? 1 : 0;
#pragma unroll 4
    for (int t = split; t < n; ++t) cnt += so[t] > oj ? 1 : 0;
    atomicAdd(rank + j, cnt);
}

__global__ void __launch_bounds__(RF_THREADS) plan_refresh_kernel(RefreshParams p) {
    extern __shared__ uint32_t sk[];  // ordered statistics of the first min(K, RF_SMEM_KEYS) channels
    __shared__ unsigned hist[256];
    __shared__ int warp_tot[32];
    __shared__ int total;
    __shared__ uint64_t prefix_sh;
    __shared__ int need_sh;
    const int tid = threadIdx.x;

    // 1. statistics must be finite (the scratch flag and ranks are left
    // zeroed for the next refresh in every case)
    if (*p.bad) {
        __syncthreads();  // every thread has read the flag
        if (tid == 0) {
            atomicOr(p.status, OSM_STATUS_NONFINITE);
            *const_cast<uint32_t*>(p.bad) = 0;
        }
        if (p.rank != nullptr)
            for (int j = tid; j < p.K; j += RF_THREADS) const_cast<int32_t*>(p.rank)[j] = 0;
        return;
    }

    // inputs of the table rebuild (step 4), loaded one chunk ahead; with
    // ranks the first chunk's are loaded before anything else
    const bool use_rank = p.rank != nullptr && p.k > 0 && p.k < p.K;
    auto fetch = [&](int c0, int32_t& rk, uint64_t& key, float& iv) {
        const int j = c0 + tid;
        if (j < p.K) {
            if (use_rank) rk = p.rank[j];
            else key = rf_key(sk, p.score, j);
            iv = p.s_new[p.K + j];
        }
    };
    int32_t rk_n = 0;
    uint64_t key_n = 0;
    float iv_n = 0.0f;
    if (use_rank) fetch(0, rk_n, key_n, iv_n);

    // 2. Eq. (2), computed by refresh_stats_kernel; stage the keys
    for (int j = tid; j < p.K; j += RF_THREADS) {
        p.s[j] = p.s_new[j];
        p.inv_s[j] = p.s_new[p.K + j];
        if (j < RF_SMEM_KEYS) sk[j] = rf_ord(p.score[j]);
    }
    __syncthreads();

    // 3. the k-th largest key (k = 0: none selected; k = K: all)
    uint64_t thresh = 0;  // selected <=> key >= thresh
    if (p.k == 0) {
        thresh = ~0ull;
    } else if (p.k < p.K && p.rank == nullptr) {
        if (tid == 0) {
            prefix_sh = 0;
            need_sh = p.k;
        }
        __syncthreads();
        for (int shift = 40; shift >= 0; shift -= 8) {
            for (int b = tid; b < 256; b += RF_THREADS) hist[b] = 0;
            __syncthreads();
            const uint64_t prefix = prefix_sh;
            const uint64_t hi_mask = shift == 40 ? 0ull : (~0ull << (shift + 8)) & 0xFFFFFFFFFFFFull;
            for (int j0 = 0; j0 < p.K; j0 += RF_THREADS) {  // uniform trip count: whole warps stay converged
                const int j = j0 + tid;
                const uint64_t key = j < p.K ? rf_key(sk, p.score, j) : 0;
                const bool in = j < p.K && (key & hi_mask) == prefix;
                const unsigned digit = in ? static_cast<unsigned>((key >> shift) & 0xFF) : 256u;
                // one shared-memory increment per distinct digit of the warp
                const unsigned peers = __match_any_sync(0xffffffffu, digit);
                if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns digits 255 - 8l .. 248 - 8l; a prefix sum over lanes
                // runs from the top digit down
                const int lane = tid;
                int own = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) own += static_cast<int>(hist[255 - 8 * lane - i]);
                int incl = own;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int o = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += o;
                }
                const int need = need_sh;
                const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
                const int l = __ffs(hit) - 1;  // first lane whose digits reach the k-th key
                if (lane == l) {
                    int rem = need - (incl - own);
                    int d = 255 - 8 * lane;
                    for (int i = 0; i < 7; ++i, --d) {
                        if (static_cast<int>(hist[d]) >= rem) break;
                        rem -= static_cast<int>(hist[d]);
                    }
                    prefix_sh = prefix | (static_cast<uint64_t>(d) << shift);
                    need_sh = rem;
                }
            }
            __syncthreads();
        }
        thresh = prefix_sh;  // exact: keys are unique, so the k-th largest is one key
    }

    // 4. ranks, J, O, route, order, inv_s in order. Each chunk's inputs (the
    // channel's rank or key and its inv_s) are loaded one chunk ahead, so
    // that their latency overlaps the previous chunk's scan and stores.
    __syncthreads();
    const int nbp = p.Kbp / 32;
    if (!use_rank) fetch(0, rk_n, key_n, iv_n);  // the keys are staged by now
    int base_o = 0, base_j = 0;
    for (int c0 = 0; c0 < p.K; c0 += RF_THREADS) {
        const int j = c0 + tid;
        const bool valid = j < p.K;
        const int32_t rk = rk_n;
        const uint64_t key = key_n;
        const float iv = iv_n;
        if (c0 + RF_THREADS < p.K) fetch(c0 + RF_THREADS, rk_n, key_n, iv_n);
        const int sel = !valid ? 0 : use_rank ? (rk < p.k ? 1 : 0) : (key >= thresh ? 1 : 0);
        const int r_o = block_exclusive_scan(sel, warp_tot, &total) + base_o;
        const int n_sel = total;
        const int r_j = base_j + tid - (r_o - base_o);  // unselected channels before j
        if (valid) {
            if (sel) {
                p.O[r_o] = j;
                p.route[j] = nbp * QA_BLOCK_BYTES + 2 * r_o;
                p.order[p.Kb + r_o] = j;
                p.inv_s_ord[p.Kb + r_o] = iv;
            } else {
                p.J[r_j] = j;
                p.route[j] = (r_j / 32) * QA_BLOCK_BYTES + (r_j % 32) * 2;
                p.order[r_j] = j;
                p.inv_s_ord[r_j] = iv;
            }
        }
        base_o += n_sel;
        base_j += min(RF_THREADS, p.K - c0) - n_sel;
        __syncthreads();
    }
    if (p.rank != nullptr)
        for (int j = tid; j < p.K; j += RF_THREADS) const_cast<int32_t*>(p.rank)[j] = 0;
    if (tid == 0) *const_cast<uint32_t*>(p.bad) = 0;
}

}  // namespace

int launch_plan_refresh(osm_plan* pl, const float* amax, const float* score, const float* wmax, float alpha,
                        cudaStream_t st) {
    const int K = static_cast<int>(pl->K);
    const int k = static_cast<int>(pl->k);
    int rc;
    // the flag and the ranks are zero here: zeroed at plan creation and by
    // every plan_refresh_kernel before it exits
    int32_t* rank = nullptr;
    const int cx = (K + 255) / 256;
    int gy = 1, slice = K;
    if (k > 0 && k < K && K <= RF_RANK_MAX_K) {
        rank = reinterpret_cast<int32_t*>(pl->d_s_new + 2 * static_cast<size_t>(K));
        const int g = std::max((K + RF_RANK_SLICE - 1) / RF_RANK_SLICE, std::min(64, 296 / cx));  // ~2 CTAs per SM
        slice = (K + g - 1) / g;  // <= RF_RANK_SLICE
        gy = (K + slice - 1) / slice;
    }
    // row y = 0 of the grid: Eq. (2) per channel; rows 1 .. gy: the rank counts
    refresh_stats_kernel<<<dim3(cx, rank ? gy + 1 : 1), 256, 0, st>>>(amax, score, wmax, static_cast<double>(alpha), K, slice,
                                                      pl->d_s_new, pl->d_bad, rank);
    if ((rc = check_cuda(cudaGetLastError(), "plan_refresh statistics launch"))) return rc;
    RefreshParams p{amax, score, wmax, static_cast<double>(alpha), K, k, static_cast<int>(pl->Kb),
                    static_cast<int>(pl->Kbp), pl->d_s_new, pl->d_bad, pl->d_s, pl->d_inv_s, pl->d_route,
                    pl->d_J, pl->d_O, pl->d_order, pl->d_inv_s_ord, pl->d_status, rank};
    const size_t smem = sizeof(uint32_t) * static_cast<size_t>(K < RF_SMEM_KEYS ? K : RF_SMEM_KEYS);
    static bool attr_set[64] = {};
    int dev = 0;
    if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((rc = check_cuda(cudaFuncSetAttribute(plan_refresh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(sizeof(uint32_t) * RF_SMEM_KEYS)),
                             "plan_refresh smem attribute")))
            return rc;
        attr_set[dev] = true;
    }
    plan_refresh_kernel<<<1, RF_THREADS, smem, st>>>(p);
    return check_cuda(cudaGetLastError(), "plan_refresh launch");
}

}  // namespace osm

// ---------------------------------------------------------------------------
// Error norms for the per-layer alpha / k search: out[0] += sum (y - r)^2,
// out[1] += sum r^2 over `count` FP32 values, accumulated in FP64.

namespace osm {
namespace {

__global__ void __launch_bounds__(256) error_norms_kernel(const float* __restrict__ y, const float* __restrict__ r,
                                                          int64_t count, double* __restrict__ out) {
    double e = 0.0, n = 0.0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
        const double d = static_cast<double>(y[i]) - static_cast<double>(r[i]);
        e = fma(d, d, e);
        n = fma(static_cast<double>(r[i]), static_cast<double>(r[i]), n);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        e += __shfl_xor_sync(0xffffffffu, e, o);
        n += __shfl_xor_sync(0xffffffffu, n, o);
    }
    __shared__ double part[2][8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        part[0][warp] = e;
        part[1][warp] = n;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double se = 0.0, sn = 0.0;
        for (int w = 0; w < 8; ++w) {
            se += part[0][w];
            sn += part[1][w];
        }
        atomicAdd(out, se);
        atomicAdd(out + 1, sn);
    }
}

}  // namespace

int launch_error_norms(const float* y, const float* r, int64_t count, double* out, cudaStream_t st) {
    int rc = check_cuda(cudaMemsetAsync(out, 0, 2 * sizeof(double), st), "error_norms clear");
    if (rc) return rc;
    int64_t blocks = (count + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    error_norms_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(y, r, count, out);
    return check_cuda(cudaGetLastError(), "error_norms launch");
}

}  // namespace osm
