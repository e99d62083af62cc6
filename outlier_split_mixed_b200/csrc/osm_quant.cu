// Calibration statistics, weight packing and the runtime activation
// quantiser of the smoothed, outlier-split W4A4 layer
// ("W4A4 Quantization for Inference on Wan2.2-I2V-A14B", Eq. (1), (2),
// (4), (5), and the block-packing paragraph with Fig. 8).
//
// All kernels here are HBM-bound streaming passes: 128-bit vector loads,
// per-channel tables served from L1/L2, and coalesced 32/128-bit stores.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>
#include <type_traits>
#include <utility>

#include "osm_internal.h"
#include "osm_mx.cuh"
#include "osm_ptx.cuh"

namespace osm {
namespace {

// ------------------------------------------------------------ helpers

using mx::sf_offset;

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t encode8_words(uint4 q, float inv) { return mx::encode8_words(q.x, q.y, q.z, q.w, inv); }

// Two BF16 inputs (one packed word) times their inv_s -> two BF16 x' values
// (packed): x' = bf16(fp32(x) * inv_s), one IEEE multiply per lane.
__device__ __forceinline__ uint32_t smooth2(uint32_t w, float2 s) {
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)), s);
    return mx::bf16x2_bits(v.x, v.y);
}

// As smooth2 with the halves selected by `f16mask` (0xFFFF per half) rounded
// to binary16 instead of BF16: the outlier slots of an FP16 outlier branch.
__device__ __forceinline__ uint32_t smooth2_mixed(uint32_t w, float2 s, uint32_t f16mask) {
    const float2 v = __fmul2_rn(make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)), s);
    const uint32_t b = mx::bf16x2_bits(v.x, v.y);
    const uint32_t h = mx::f16x2_bits(v.x, v.y);
    return (h & f16mask) | (b & ~f16mask);
}

// Mask for smooth2_mixed: the halves whose routed offset is an outlier slot
// (offsets from `slot0` on) when the outlier branch is FP16.
__device__ __forceinline__ uint32_t slot_mask(int2 dv, int slot0) {
    return (dv.x >= slot0 ? 0x0000FFFFu : 0u) | (dv.y >= slot0 ? 0xFFFF0000u : 0u);
}

// ------------------------------------------------------------ calibration

constexpr int AMAX_THREADS = 256;
constexpr int AMAX_ROWS = 256;  // rows per CTA (at most; fewer for small batches)

// amax[j] = max(amax[j], max_t |X[t][j]|). A CTA covers 256 channels (a
// lane takes 8 channels, 16 bytes of a row) and `rows` rows (warp w takes
// rows w, w + 8, ...), with eight 16-byte row loads per lane in
// flight; the maxima are kept as packed u16 pairs of |x| bit patterns
// (integer order, so a NaN pattern propagates and the finiteness check of
// the calibration sees it), combined over the warps in shared memory and
// merged with one atomicMax per channel and CTA on the IEEE bit pattern of
// the FP32 value (monotone for non-negative floats).
__global__ void __launch_bounds__(AMAX_THREADS) act_amax_kernel(const uint16_t* __restrict__ X, int64_t T,
                                                                int64_t K, float* __restrict__ amax, int rows) {
    constexpr int NW = AMAX_THREADS / 32;
    __shared__ uint32_t red[NW][32][4];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t v = static_cast<int64_t>(blockIdx.x) * 32 + lane;  // 8-channel group
    const bool active = v * 8 < K;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * rows;
    const int64_t t1 = min(T, t0 + rows);
    uint32_t m[4] = {0, 0, 0, 0};
    const uint16_t* src = X + v * 8;
    if (active) {
        for (int64_t t = t0 + warp; t < t1; t += 8 * NW) {
            uint4 q[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t tu = t + u * NW;
                q[u] = tu < t1 ? ldg_nc_v4(src + tu * K) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                m[0] = vmax_u16x2(m[0], q[u].x & 0x7FFF7FFFu);
                m[1] = vmax_u16x2(m[1], q[u].y & 0x7FFF7FFFu);
                m[2] = vmax_u16x2(m[2], q[u].z & 0x7FFF7FFFu);
                m[3] = vmax_u16x2(m[3], q[u].w & 0x7FFF7FFFu);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane][i] = m[i];
    __syncthreads();
    if (warp == 0 && active) {
#pragma unroll
        for (int w = 1; w < NW; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i) m[i] = vmax_u16x2(m[i], red[w][lane][i]);
        unsigned int* dst = reinterpret_cast<unsigned int*>(amax) + v * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            atomicMax(dst + 2 * i, (m[i] & 0xFFFFu) << 16);
            atomicMax(dst + 2 * i + 1, m[i] & 0xFFFF0000u);
        }
    }
}

// Tail-aware channel score (the activation-tail-aware percentile
// calibration of the Tail-Aware HiFloat4 page): score[j] = the rank-th
// smallest |x_tj| over the T tokens (rank 1-based; the host derives it from
// the percentile q as ceil(q T)). Per-channel shared histograms are padded
// so that equal buckets of different channels fall in different banks.
constexpr int PCT_THREADS = 256;
constexpr int PCT_SPLIT = 4;   // CTAs of a cluster, each taking a quarter of the rows
constexpr int PCT_UNROLL = 8;  // rows per warp loaded before their histogram updates

// score[j] = the rank-th smallest |x_tj| (1-based) for 32 channels per
// cluster of PCT_SPLIT CTAs: BF16 magnitudes are 15-bit keys, so two
// histogram passes (the high 8 bits, then the low 7 bits inside the chosen
// bucket) find the rank exactly. Each CTA histograms its share of the rows
// (eight independent row loads per warp in flight), the shares are added
// into the first CTA's histogram through distributed shared memory, the
// first CTA picks the bucket and hands it back to the others.
__global__ void __cluster_dims__(PCT_SPLIT, 1, 1) __launch_bounds__(PCT_THREADS)
    act_percentile_kernel(const uint16_t* __restrict__ X, int64_t T, int64_t K, int64_t rank,
                          float* __restrict__ score) {
    __shared__ unsigned hist[32][257];
    __shared__ unsigned pick[32], rem[32];
    constexpr int NW = PCT_THREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t crank = ptx::cluster_ctarank();
    const int64_t j = static_cast<int64_t>(blockIdx.y) * 32 + lane;  // K % 32 == 0
    const int64_t chunk = (T + PCT_SPLIT - 1) / PCT_SPLIT;
    const int64_t t0 = static_cast<int64_t>(crank) * chunk;
    const int64_t t1 = min(T, t0 + chunk);
    const uint32_t hist0 = ptx::mapa(ptx::smem_u32(&hist[0][0]), 0);
    for (int pass = 0; pass < 2; ++pass) {
        for (int i = threadIdx.x; i < 32 * 257; i += PCT_THREADS) (&hist[0][0])[i] = 0;
        __syncthreads();
        const unsigned hi = pass ? pick[lane] : 0u;
        for (int64_t t = t0 + warp; t < t1; t += PCT_UNROLL * NW) {
            unsigned key[PCT_UNROLL];
#pragma unroll
            for (int u = 0; u < PCT_UNROLL; ++u) {
                const int64_t tu = t + u * NW;
                key[u] = tu < t1 ? (__ldg(X + tu * K + j) & 0x7FFFu) : 0xFFFFFFFFu;
            }
#pragma unroll
            for (int u = 0; u < PCT_UNROLL; ++u) {
                if (key[u] == 0xFFFFFFFFu) continue;
                if (pass == 0) atomicAdd(&hist[lane][key[u] >> 7], 1u);
                else if ((key[u] >> 7) == hi) atomicAdd(&hist[lane][key[u] & 127u], 1u);
            }
        }
        ptx::cluster_sync();  // every share complete
        if (crank != 0)
            for (int i = threadIdx.x; i < 32 * 257; i += PCT_THREADS) {
                const unsigned v = (&hist[0][0])[i];
                if (v) ptx::red_add_cluster_u32(hist0 + 4u * i, v);
            }
        ptx::cluster_sync();  // the first CTA holds the whole histogram
        if (crank == 0 && threadIdx.x < 32) {
            const int c = threadIdx.x;
            unsigned need = pass ? rem[c] : static_cast<unsigned>(rank);
            const int nb = pass ? 128 : 256;
            int b = 0;
            for (; b < nb - 1; ++b) {
                if (hist[c][b] >= need) break;
                need -= hist[c][b];
            }
            if (pass == 0) {
                pick[c] = static_cast<unsigned>(b);
                rem[c] = need;
                for (uint32_t r = 1; r < PCT_SPLIT; ++r)
                    ptx::st_cluster_u32(ptx::mapa(ptx::smem_u32(&pick[c]), r), static_cast<unsigned>(b));
            } else {
                score[static_cast<int64_t>(blockIdx.y) * 32 + c] = __uint_as_float(((pick[c] << 7) | b) << 16);
            }
        }
        ptx::cluster_sync();  // the bucket of pass 0 is known everywhere; no CTA touches another's memory after
    }
}

// wmax[j] = max_n |W[j][n]|: one block per input channel row.
__global__ void __launch_bounds__(256) weight_amax_kernel(const uint16_t* __restrict__ W, int64_t N,
                                                          float* __restrict__ wmax) {
    const int64_t j = blockIdx.x;
    const uint16_t* row = W + j * N;
    uint32_t m = 0;
    for (int64_t v = threadIdx.x; v * 8 < N; v += blockDim.x) {
        const uint4 q = ldg_nc_v4(row + v * 8);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, w[i] >> 16 & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ uint32_t part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r = max(r, part[i]);
        wmax[j] = __uint_as_float(r << 16);
    }
}

// ------------------------------------------------------------ weight packing

struct PackParams {
    const uint16_t* W;  // [K][N]
    const int32_t* col_order;  // packed row n takes W column col_order[n] (NULL: n)
    const float* s;     // [K]
    const int32_t* J;   // [Kb]
    const int32_t* O;   // [k]
    int64_t K, N, k, Kb, Kbp, kp;
    int mode;
    uint8_t* codes;     // [N][Kbp/2]
    uint8_t* scales;    // layout, rows padded to 128
    uint16_t* hp;       // [N][kp]
    int katoms;         // scale atoms per 128-row tile: Kbp/128 (MXFP4) or Kbp/64 (NVFP4)
    int nv;             // NVFP4 encoding
    float nv_k;         // NVFP4: fp32(1/6) * 2^-g_w
    float nv_p2g;       // NVFP4: 2^g_w
    float hp_scale;     // NVFP4: 2^-g_w on the outlier rows
};

// Tiled forms of the two packing kernels: a CTA gathers whole W rows (input
// channels) with coalesced 16-byte loads, folds s and rounds to BF16 on the
// way into shared memory, and reads the tile back transposed, so that every
// global access is wide and contiguous whatever the packing order.

constexpr int PK_THREADS = 256;

// Load rows src_row(r) of W (r < nrows <= 128; a negative row is zero),
// columns n0 .. n0+127 (packed order: W column col_order[n] when col_order
// is set), as w' = bf16(fp32(w) * s[row]) into tile[r][0..63] (BF16
// pairs). Each thread issues all its 16-byte row loads (up to eight) before
// it folds and stores any of them, so that they are in flight together.
template <bool F16, typename RowOf>
__device__ __forceinline__ void load_folded_rows(const PackParams& p, int64_t n0, int nrows, RowOf src_row,
                                                 uint32_t (*tile)[64]) {
    constexpr int PER = 128 * 16 / PK_THREADS;
    uint4 w[PER];
    float sj[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int t = threadIdx.x + i * PK_THREADS;
        w[i] = make_uint4(0, 0, 0, 0);
        sj[i] = 0.0f;
        if (t >= nrows * 16) continue;
        const int r = t >> 4, c = t & 15;
        const int64_t j = src_row(r);
        const int64_t n = n0 + 8 * c;
        if (j < 0 || n >= p.N) continue;
        sj[i] = __ldg(p.s + j);
        if (p.col_order == nullptr) {
            w[i] = ldg_nc_v4(p.W + j * p.N + n);
        } else {
            uint32_t e[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) e[u] = p.W[j * p.N + __ldg(p.col_order + n + u)];
            w[i] = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
        }
    }
    const uint32_t m = F16 ? 0xFFFFFFFFu : 0u;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int t = threadIdx.x + i * PK_THREADS;
        if (t >= nrows * 16) continue;
        const int r = t >> 4, c = t & 15;
        const float2 s2 = make_float2(sj[i], sj[i]);
        // a zero row (j < 0 or n >= N) folds to +0 either way
        const uint4 v = make_uint4(smooth2_mixed(w[i].x, s2, m), smooth2_mixed(w[i].y, s2, m),
                                   smooth2_mixed(w[i].z, s2, m), smooth2_mixed(w[i].w, s2, m));
        *reinterpret_cast<uint4*>(&tile[r][4 * c]) = v;
    }
}

// Bulk channels: CTA = 128 bulk positions (one strip, four MX blocks) x 128
// packed output channels. Warp w encodes block q = w / 2 for the 64 channel
// pairs 32 (w % 2) + lane: its 32 words are (channel n, channel n + 1) pairs
// down the block, so one packed abs-max chain gives both channels' block
// maxima. 1x32: the block maximum; 32x32: the maximum over 32 channels (16
// lanes); 128x1: the maximum over the strip's four blocks (four warps, via
// shared memory). NV: the 32 positions are two NVFP4 16-blocks, each with
// its own E4M3 scale and element multiplier.
// Five CTAs per SM (48 registers): the tile loads of more CTAs are in
// flight at once (the kernel waits on memory latency: 83.4-85.8 -> 72.9-74.5
// us for the 5120 x 13824 weights against four CTAs; six CTAs spill).
template <bool NV>
__global__ void __launch_bounds__(PK_THREADS, 5) pack_bulk_tiled_kernel(PackParams p) {
    __shared__ __align__(16) uint32_t tile[128][64];
    __shared__ uint32_t red[4][64];
    __shared__ uint32_t sxs[4][64];  // scale codes per quarter and pair: MX (n | n+1 << 8), NV (n: 2 bytes | n+1: 2 bytes)
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128;
    const int64_t p0 = static_cast<int64_t>(blockIdx.y) * 128;
    const int64_t katoms = p.katoms;
    load_folded_rows<false>(p, n0, 128, [&](int r) -> int64_t { return p0 + r < p.Kb ? __ldg(p.J + p0 + r) : -1; },
                            tile);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp >> 1;
    const int c = 32 * (warp & 1) + lane;  // channel pair: columns n0 + 2c, n0 + 2c + 1
    uint32_t wv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) wv[i] = tile[32 * q + i][c];
    using mx::bf16x2_absmax;
    const int64_t n = n0 + 2 * c;
    if constexpr (NV) {
        uint32_t ma = wv[0], mb = wv[16];
#pragma unroll
        for (int i = 1; i < 16; ++i) {
            ma = bf16x2_absmax(ma, wv[i]);
            mb = bf16x2_absmax(mb, wv[16 + i]);
        }
        float r0a, r0b, r1a, r1b;  // multipliers of channel n (blocks 2q, 2q+1) and n + 1
        const uint32_t s0 = mx::nv_block_scales(ma & 0x7FFFu, mb & 0x7FFFu, p.nv_k, p.nv_p2g, &r0a, &r0b);
        const uint32_t s1 =
            mx::nv_block_scales((ma >> 16) & 0x7FFFu, (mb >> 16) & 0x7FFFu, p.nv_k, p.nv_p2g, &r1a, &r1b);
        if (n < p.N) {
            uint32_t lo[16], hi[16];
#pragma unroll
            for (int k2 = 0; k2 < 16; ++k2) {
                lo[k2] = __byte_perm(wv[2 * k2], wv[2 * k2 + 1], 0x5410);
                hi[k2] = __byte_perm(wv[2 * k2], wv[2 * k2 + 1], 0x7632);
            }
            const uint4 clo = make_uint4(mx::encode8_words(lo[0], lo[1], lo[2], lo[3], r0a),
                                         mx::encode8_words(lo[4], lo[5], lo[6], lo[7], r0a),
                                         mx::encode8_words(lo[8], lo[9], lo[10], lo[11], r0b),
                                         mx::encode8_words(lo[12], lo[13], lo[14], lo[15], r0b));
            const uint4 chi = make_uint4(mx::encode8_words(hi[0], hi[1], hi[2], hi[3], r1a),
                                         mx::encode8_words(hi[4], hi[5], hi[6], hi[7], r1a),
                                         mx::encode8_words(hi[8], hi[9], hi[10], hi[11], r1b),
                                         mx::encode8_words(hi[12], hi[13], hi[14], hi[15], r1b));
            *reinterpret_cast<uint4*>(p.codes + n * (p.Kbp / 2) + p0 / 2 + 16 * q) = clo;
            *reinterpret_cast<uint4*>(p.codes + (n + 1) * (p.Kbp / 2) + p0 / 2 + 16 * q) = chi;
        }
        sxs[q][c] = (s0 & 0xFFFFu) | (s1 << 16);
        __syncthreads();
        if (warp < 2) {  // a channel's eight scale bytes of the strip: one word in each of two atoms
            uint32_t w0lo = (sxs[0][c] & 0xFFFFu) | (sxs[1][c] << 16), w1lo = (sxs[2][c] & 0xFFFFu) | (sxs[3][c] << 16);
            uint32_t w0hi = (sxs[0][c] >> 16) | (sxs[1][c] & 0xFFFF0000u), w1hi = (sxs[2][c] >> 16) | (sxs[3][c] & 0xFFFF0000u);
            if (n >= p.N) w0lo = w1lo = 0;
            if (n + 1 >= p.N) w0hi = w1hi = 0;
            const int64_t b0 = static_cast<int64_t>(blockIdx.y) * 8;
            *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n, b0, katoms)) = w0lo;
            *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n, b0 + 4, katoms)) = w1lo;
            *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n + 1, b0, katoms)) = w0hi;
            *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n + 1, b0 + 4, katoms)) = w1hi;
        }
        return;
    }
    uint32_t m = wv[0];
#pragma unroll
    for (int i = 1; i < 32; ++i) m = bf16x2_absmax(m, wv[i]);
    if (p.mode == OSM_WSCALE_TILE32x32) {
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) m = bf16x2_absmax(m, __shfl_xor_sync(0xffffffffu, m, o));
        const uint32_t mm = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
        m = mm | (mm << 16);
    } else if (p.mode == OSM_WSCALE_STRIP128x1) {
        red[q][c] = m;
        __syncthreads();
        m = bf16x2_absmax(bf16x2_absmax(red[0][c], red[1][c]), bf16x2_absmax(red[2][c], red[3][c]));
    }
    const bool real = p0 + 32 * q < p.Kb;  // the block holds at least one real position
    float inv_lo, inv_hi;
    const int X_lo = mx::bf16_block_exponent(m & 0x7FFFu, &inv_lo);
    const int X_hi = mx::bf16_block_exponent((m >> 16) & 0x7FFFu, &inv_hi);
    if (n < p.N) {
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) {
            lo[k2] = __byte_perm(wv[2 * k2], wv[2 * k2 + 1], 0x5410);
            hi[k2] = __byte_perm(wv[2 * k2], wv[2 * k2 + 1], 0x7632);
        }
        const uint4 clo = make_uint4(mx::encode8_words(lo[0], lo[1], lo[2], lo[3], inv_lo),
                                     mx::encode8_words(lo[4], lo[5], lo[6], lo[7], inv_lo),
                                     mx::encode8_words(lo[8], lo[9], lo[10], lo[11], inv_lo),
                                     mx::encode8_words(lo[12], lo[13], lo[14], lo[15], inv_lo));
        const uint4 chi = make_uint4(mx::encode8_words(hi[0], hi[1], hi[2], hi[3], inv_hi),
                                     mx::encode8_words(hi[4], hi[5], hi[6], hi[7], inv_hi),
                                     mx::encode8_words(hi[8], hi[9], hi[10], hi[11], inv_hi),
                                     mx::encode8_words(hi[12], hi[13], hi[14], hi[15], inv_hi));
        *reinterpret_cast<uint4*>(p.codes + n * (p.Kbp / 2) + p0 / 2 + 16 * q) = clo;
        *reinterpret_cast<uint4*>(p.codes + (n + 1) * (p.Kbp / 2) + p0 / 2 + 16 * q) = chi;
    }
    sxs[q][c] = real ? static_cast<uint32_t>(X_lo + 127) | (static_cast<uint32_t>(X_hi + 127) << 8) : 0u;
    __syncthreads();
    if (warp < 2) {  // the four scale bytes of a channel are one word of its atom row; padding rows get 0
        uint32_t wlo = 0, whi = 0;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            wlo |= (sxs[qq][c] & 0xFFu) << (8 * qq);
            whi |= ((sxs[qq][c] >> 8) & 0xFFu) << (8 * qq);
        }
        if (n >= p.N) wlo = 0;
        if (n + 1 >= p.N) whi = 0;
        const int64_t strip = blockIdx.y;
        *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n, strip * 4, katoms)) = wlo;
        *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n + 1, strip * 4, katoms)) = whi;
    }
}

// Outlier channels: CTA = 64 outlier slots x 128 packed output channels;
// w_hp[n][i] = bf16(fp32(w[O_i][n]) * s[O_i]) (binary16 for an FP16 outlier
// branch) for i < k, 0 for k <= i < kp.
// Thread (n, 8-slot group) gathers its eight values down the tile and writes
// them as one 16-byte store.
template <bool F16>
__global__ void __launch_bounds__(PK_THREADS) pack_hp_tiled_kernel(PackParams p) {
    __shared__ __align__(16) uint32_t tile[64][64];
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 128;
    const int64_t i0 = static_cast<int64_t>(blockIdx.y) * 64;
    load_folded_rows<F16>(p, n0, 64, [&](int r) -> int64_t { return i0 + r < p.k ? __ldg(p.O + i0 + r) : -1; },
                          tile);
    __syncthreads();
    const uint16_t* t16 = reinterpret_cast<const uint16_t*>(&tile[0][0]);
    for (int t = threadIdx.x; t < 128 * 8; t += PK_THREADS) {
        const int nl = t & 127, g = t >> 7;  // channel, group of 8 slots
        const int64_t n = n0 + nl;
        if (n >= p.N) continue;
        uint32_t e[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = t16[(8 * g + i) * 128 + nl];
        uint4 v = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
        if (p.nv) v = mx::scale_bf16x8(v, p.hp_scale);  // NVFP4: w_hp = bf16(fp32(w') * 2^-g_w)
        *reinterpret_cast<uint4*>(p.hp + n * p.kp + i0 + 8 * g) = v;
    }
}

// ------------------------------------------------------------ quantize_act

struct QuantParams {
    const uint16_t* X;       // [M][K]
    const float* inv_s;      // [K]
    const int32_t* route;    // [K] byte offset of channel j inside a staged row
    int M, K, k, Kb, Kbp, kp;
    uint8_t* codes;          // [M][Kbp/2]
    uint8_t* scales;         // layout, rows padded to 128
    uint16_t* hp;            // [M][kp]
    uint32_t* status;        // OSM_STATUS_* bits
    uint64_t wait_limit_ns;  // bound of every wait on an incoming row group
    uint32_t extra_tx;       // bytes expected beyond each group's copy (0; 16 when starved for a test)
    int hp_fp16;             // outlier slots in binary16 instead of BF16
    int katoms;              // scale atoms per 128-row tile: Kbp/128 (MXFP4) or Kbp/64 (NVFP4)
    float nv_k;              // NVFP4: fp32(1/6) * 2^-g_act
    float nv_p2g;            // NVFP4: 2^g_act
    float hp_scale;          // NVFP4: 2^-g_act on the outlier slots
};

// Encodings of quantize_act: MXFP4 with BF16 or FP16 outlier slots, NVFP4.
enum QaMode { QA_MX = 0, QA_MX_F16 = 1, QA_NV = 2 };

constexpr int QA_THREADS = 256;
constexpr int STREAM_NT = 512;  // threads of the streaming form

__host__ __device__ constexpr int qa_row_stride(int nb, int kp) { return (nb * QA_BLOCK_BYTES + kp * 2 + 15) & ~15; }

// Each CTA handles R consecutive rows, staged in shared memory in
// [bulk blocks | outlier slots] order; a bulk block of 32 BF16 values takes
// 80 bytes (64 + 16 padding) so that phase 2's 128-bit reads by consecutive
// threads hit distinct banks.
//  phase 1: each lane loads 2 channels (32-bit) of each of the R rows -- a
//           warp reads 128 contiguous bytes per row -- computes
//           x' = bf16(x * inv_s) (a packed pair of IEEE multiplies) and
//           stores both values at their routed offsets (bulk position or
//           outlier slot); consecutive lanes write into one 128-byte window,
//           so the stores are conflict-free (eight channels per lane would
//           put a warp's stores 16 bytes apart: a 4-way bank conflict);
//  phases 2 and 3 (encode_staged): one thread per (row, 32-block) encodes
//           the block (MXFP4, or two NVFP4 16-blocks) from four 128-bit
//           shared loads; the outlier slots go out as 128-bit stores.
// This staged, phase-serial form serves rows too wide for the streaming
// form's ring (quantize_act_stream_kernel below).
template <int MODE>
__device__ __forceinline__ void encode_staged(const QuantParams& p, uint32_t sbuf, int stride, int row0, int nrows);
__device__ __forceinline__ void zero_padding_scale_rows(const QuantParams& p);

template <int R, int MODE>
__global__ void __launch_bounds__(QA_THREADS) quantize_act_kernel(QuantParams p) {
    constexpr bool HPF = MODE == QA_MX_F16;
    ptx::grid_dep_launch();  // the dual_gemm that follows may start its prologue
    extern __shared__ __align__(16) uint8_t sbuf[];
    const int nb = p.Kbp >> 5;
    const int stride = qa_row_stride(nb, p.kp);
    const int row0 = blockIdx.x * R;
    const int tid = threadIdx.x;

    // zero the padding slots: bulk positions [Kb, Kbp) and outlier slots [k, kp)
    {
        const int npb = p.Kbp - p.Kb, npad = npb + (p.kp - p.k);
        for (int i = tid; i < R * npad; i += QA_THREADS) {
            const int r = i / npad, c = i - r * npad;
            const int pos = p.Kb + c;
            const int off = c < npb ? (pos >> 5) * QA_BLOCK_BYTES + (pos & 31) * 2
                                    : nb * QA_BLOCK_BYTES + (p.k + c - npb) * 2;
            *reinterpret_cast<uint16_t*>(sbuf + r * stride + off) = 0;
        }
    }

    // phase 1: each lane takes channel pairs c = tid, tid + 256, ... (a warp
    // reads 128 contiguous bytes of each row); the pair's inv_s and routes
    // are loaded once and serve all R rows. Consecutive lanes store into one
    // 128-byte window of the staged row, so the routed stores do not conflict.
    const int npairs = p.K >> 1;
    const uint32_t* xrow[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
        xrow[r] = reinterpret_cast<const uint32_t*>(p.X) + static_cast<size_t>(row0 + r < p.M ? row0 + r : row0) * npairs;
    constexpr int U = 4;
    for (int c0 = tid; c0 < npairs; c0 += U * QA_THREADS) {
        uint32_t w[U][R];
        float2 sv[U];
        int2 dv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * QA_THREADS;
            if (c < npairs) {
                sv[u] = __ldg(reinterpret_cast<const float2*>(p.inv_s) + c);
                dv[u] = __ldg(reinterpret_cast<const int2*>(p.route) + c);
#pragma unroll
                for (int r = 0; r < R; ++r) w[u][r] = ldg_nc_u32(xrow[r] + c);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * QA_THREADS;
            if (c < npairs) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint32_t h = HPF ? smooth2_mixed(w[u][r], sv[u], slot_mask(dv[u], nb * QA_BLOCK_BYTES))
                                           : smooth2(w[u][r], sv[u]);
                    *reinterpret_cast<uint16_t*>(sbuf + r * stride + dv[u].x) = static_cast<uint16_t>(h);
                    *reinterpret_cast<uint16_t*>(sbuf + r * stride + dv[u].y) = static_cast<uint16_t>(h >> 16);
                }
            }
        }
    }
    __syncthreads();

    // phases 2 and 3
    encode_staged<MODE>(p, ptx::smem_u32(sbuf), stride, row0, min(R, p.M - row0));
    if (row0 <= p.M - 1 && p.M - 1 < row0 + R) zero_padding_scale_rows(p);
}


// Encode the staged rows [0, nrows) of a routed buffer: one thread per
// (row, 32-block) -- four 128-bit shared loads, amax by packed u16 max, the
// block scale(s), sixteen E2M1x2 conversions, one 16-byte code store and the
// scale byte(s) -- then the outlier slots as 16-byte copies. MXFP4: one E8M0
// exponent per 32-block. NVFP4: the 32-block is two 16-blocks, each with its
// E4M3 scale and element multiplier; the outlier slots are scaled by
// 2^-g_act. Rows are row0 + r of the output.
template <int MODE>
__device__ __forceinline__ void encode_staged(const QuantParams& p, uint32_t sbuf, int stride, int row0,
                                              int nrows) {
    const int nb = p.Kbp >> 5;
    const int katoms = p.katoms;
    const int tid = threadIdx.x;
    const float inv_nb = 1.0f / static_cast<float>(nb);
    for (int wi = tid; wi < nrows * nb; wi += blockDim.x) {
        // r = wi / nb (exact: wi < 2^20 and the quotient is below 8)
        int r = static_cast<int>((static_cast<float>(wi) + 0.5f) * inv_nb);
        r -= (r * nb > wi);
        r += ((r + 1) * nb <= wi);
        const int b = wi - r * nb;
        const int t = row0 + r;
        const uint32_t src = sbuf + r * stride + b * QA_BLOCK_BYTES;
        const uint4 q0 = ptx::ld_shared_v4(src), q1 = ptx::ld_shared_v4(src + 16), q2 = ptx::ld_shared_v4(src + 32),
                    q3 = ptx::ld_shared_v4(src + 48);
        using mx::bf16x2_absmax;
        const uint32_t m01 = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(q0.x, q0.y), bf16x2_absmax(q0.z, q0.w)),
                                           bf16x2_absmax(bf16x2_absmax(q1.x, q1.y), bf16x2_absmax(q1.z, q1.w)));
        const uint32_t m23 = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(q2.x, q2.y), bf16x2_absmax(q2.z, q2.w)),
                                           bf16x2_absmax(bf16x2_absmax(q3.x, q3.y), bf16x2_absmax(q3.z, q3.w)));
        uint8_t* codes = p.codes + static_cast<size_t>(t) * (p.Kbp >> 1) + b * 16;
        if constexpr (MODE == QA_NV) {
            float r_lo, r_hi;
            const uint32_t s2 = mx::nv_block_scales(max(m01 & 0x7FFFu, (m01 >> 16) & 0x7FFFu),
                                                    max(m23 & 0x7FFFu, (m23 >> 16) & 0x7FFFu), p.nv_k, p.nv_p2g,
                                                    &r_lo, &r_hi);
            *reinterpret_cast<uint4*>(codes) = make_uint4(encode8_words(q0, r_lo), encode8_words(q1, r_lo),
                                                          encode8_words(q2, r_hi), encode8_words(q3, r_hi));
            // 16-blocks 2b and 2b + 1: adjacent bytes of one atom row
            *reinterpret_cast<uint16_t*>(p.scales + sf_offset(t, 2 * b, katoms)) = static_cast<uint16_t>(s2);
        } else {
            const uint32_t m = bf16x2_absmax(m01, m23);
            const uint32_t amax = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
            float inv;
            const int X = mx::bf16_block_exponent(amax, &inv);
            *reinterpret_cast<uint4*>(codes) = make_uint4(encode8_words(q0, inv), encode8_words(q1, inv),
                                                          encode8_words(q2, inv), encode8_words(q3, inv));
            p.scales[sf_offset(t, b, katoms)] = static_cast<uint8_t>(b * 32 < p.Kb ? X + 127 : 0);
        }
    }
    const int hv = p.kp >> 3;
    for (int i = tid; i < nrows * hv; i += blockDim.x) {
        const int r = i / hv, c = i - r * hv;
        uint4 v = ptx::ld_shared_v4(sbuf + r * stride + nb * QA_BLOCK_BYTES + c * 16);
        if constexpr (MODE == QA_NV) v = mx::scale_bf16x8(v, p.hp_scale);
        *reinterpret_cast<uint4*>(p.hp + static_cast<size_t>(row0 + r) * p.kp + c * 8) = v;
    }
}

// Scale bytes of the padding rows [M, round_up(M, 128)) are zero; done by
// the CTA that handles row M - 1.
__device__ __forceinline__ void zero_padding_scale_rows(const QuantParams& p) {
    const int katoms = p.katoms;
    const int tile = (p.M - 1) >> 7;
    const int rem = p.M & 127;
    if (rem == 0) return;
    const int nwords = (128 - rem) * katoms;
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) {
        const int a = i / (128 - rem), rr = rem + (i - a * (128 - rem));
        *reinterpret_cast<uint32_t*>(p.scales + sf_offset(tile * 128 + rr, a * 4, katoms)) = 0u;
    }
}

// The streaming form. Persistent CTAs take groups of R consecutive rows
// g = blockIdx.x, blockIdx.x + gridDim.x, ...; the R rows of a group are
// contiguous in X, so one bulk asynchronous copy (issued by thread 0, S
// groups ahead, into a ring of S raw slots, completion on an mbarrier) brings
// them into shared memory while the CTA works on earlier groups. Per group:
//  route: each thread takes channel pairs c = tid, tid + 256, ... of each row
//         from the raw slot (conflict-free 32-bit shared loads), computes
//         x' = bf16(x * inv_s) and stores the two values at their routed
//         offsets in the staged buffer ([bulk blocks | outlier slots], a
//         32-block in 80 bytes); consecutive lanes write one 128-byte window;
//  then the raw slot is refilled with the group S ahead, and the staged rows
//  are encoded (encode_staged).
// Every wait on a slot is bounded; a wait that runs out sets
// OSM_STATUS_TIMEOUT, and the CTA lets its copies land before it returns.
// Two CTAs per SM, except with more than six register-held pairs per
// thread (one CTA per SM then has the registers and the shared memory for
// a deeper ring).
// FP: 2 when the threads' register-held pairs cover exactly the K / 2
// channel pairs (K / 2 == TR * NT: no pair needs a bound check), 1 when only
// the last of each thread's TR pairs may lie past K / 2 (K / 2 >= (TR - 1) *
// NT), 0 otherwise (every pair checked).
template <int R, int S, int NT, int TR, int MODE, int FP>
__global__ void __launch_bounds__(NT, (NT <= 256 ? 3 : (TR > 6 ? 1 : 2))) quantize_act_stream_kernel(QuantParams p) {
    constexpr bool HPF = MODE == QA_MX_F16;
    ptx::grid_dep_launch();  // the dual_gemm that follows may start its prologue
    extern __shared__ __align__(128) uint8_t smem[];
    const int nb = p.Kbp >> 5;
    const int stride = qa_row_stride(nb, p.kp);
    const int raw_bytes = R * p.K * 2;
    uint8_t* raw = smem;
    uint8_t* sbuf = smem + S * raw_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sbuf + R * stride);
    __shared__ int never;  // a flag nothing sets
    const int tid = threadIdx.x;
    const int ngroups = (p.M + R - 1) / R;
    const int mine = blockIdx.x < ngroups ? (ngroups - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;

    auto issue = [&](int i) {
        const int g = blockIdx.x + i * gridDim.x;
        const int rows = min(R, p.M - g * R);
        const uint32_t bar = ptx::smem_u32(&full[i % S]);
        const uint32_t bytes = static_cast<uint32_t>(rows) * p.K * 2u;
        ptx::mbar_arrive_expect_tx(bar, bytes + p.extra_tx);
        ptx::bulk_load(ptx::smem_u32(raw + (i % S) * raw_bytes), p.X + static_cast<size_t>(g) * R * p.K, bytes, bar);
    };

    if (tid == 0) {
        for (int s = 0; s < S; ++s) ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
        never = 0;
        ptx::fence_mbar_init();
    }
    // the padding positions of the staged rows (bulk [Kb, Kbp), slots [k, kp))
    // are never written by the routing step: zero them once
    {
        const int npb = p.Kbp - p.Kb, npad = npb + (p.kp - p.k);
        for (int i = tid; i < R * npad; i += NT) {
            const int r = i / npad, c = i - r * npad;
            const int pos = p.Kb + c;
            const int off = c < npb ? (pos >> 5) * QA_BLOCK_BYTES + (pos & 31) * 2
                                    : nb * QA_BLOCK_BYTES + (p.k + c - npb) * 2;
            *reinterpret_cast<uint16_t*>(sbuf + r * stride + off) = 0;
        }
    }
    __syncthreads();
    if (tid == 0)
        for (int i = 0; i < S && i < mine; ++i) issue(i);

    const int npairs = p.K >> 1;
    const float2* is2 = reinterpret_cast<const float2*>(p.inv_s);
    const int2* rt2 = reinterpret_cast<const int2*>(p.route);
    // with TR > 0 (npairs <= TR * NT) each thread keeps its pairs' inv_s and
    // routes in registers for all its groups
    const uint32_t raw_u32 = ptx::smem_u32(raw), sbuf_u32 = ptx::smem_u32(sbuf);
    const uint32_t row_bytes = static_cast<uint32_t>(p.K) * 2u;
    // with TR > 0 (npairs <= TR * NT) each thread keeps its pairs' inv_s and
    // the shared addresses of their routed slots (row 0) in registers
    float2 tsv[TR > 0 ? TR : 1];
    uint2 tad[TR > 0 ? TR : 1];
    uint32_t tmask[TR > 0 ? TR : 1];  // FP16 outlier branch: halves that are outlier slots
    if constexpr (TR > 0) {
#pragma unroll
        for (int j = 0; j < TR; ++j) {
            const int c = tid + j * NT;
            tsv[j] = c < npairs ? __ldg(is2 + c) : make_float2(0.f, 0.f);
            const int2 dv = c < npairs ? __ldg(rt2 + c) : make_int2(0, 0);
            tad[j] = make_uint2(sbuf_u32 + dv.x, sbuf_u32 + dv.y);
            tmask[j] = HPF ? slot_mask(dv, nb * QA_BLOCK_BYTES) : 0u;
        }
    }
    int issued = min(S, mine);
    for (int i = 0; i < mine; ++i) {
        const int g = blockIdx.x + i * gridDim.x;
        const int rows = min(R, p.M - g * R);
        const uint32_t bar = ptx::smem_u32(&full[i % S]);
        const bool ok = ptx::mbar_wait_bounded(bar, static_cast<uint32_t>((i / S) & 1), p.wait_limit_ns, &never);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(p.status, OSM_STATUS_TIMEOUT);
                // let every copy already issued land in this CTA's shared memory
                for (int j = i; j < issued; ++j)
                    if (!ptx::mbar_wait_bounded(ptx::smem_u32(&full[j % S]), static_cast<uint32_t>((j / S) & 1),
                                                20000000ull, &never))
                        ptx::spin_ns(1000000);
            }
            __syncthreads();
            return;
        }
        const uint32_t src = raw_u32 + (i % S) * raw_bytes + tid * 4;  // this thread's first pair, row 0
        if constexpr (TR > 0) {
            // A whole group (rows == R) routes without per-row checks, and
            // pairs known to lie inside K/2 (FP) without bound checks; only
            // the batch's last group can be partial. The loads of a chunk of
            // CH pairs are issued before any of its routed stores (the
            // shared accesses keep their program order), so their latencies
            // overlap (100.4 against 102.4 us at 32760 x 5120).
            auto route_rows = [&](auto rr) {
                constexpr int RR = decltype(rr)::value;
                constexpr int CH = FP == 0 ? 1 : (TR <= 6 ? TR : (TR + 1) / 2);  // every pair checked: one at a time
#pragma unroll
                for (int j0 = 0; j0 < TR; j0 += CH) {
                    uint32_t x[CH][RR];
#pragma unroll
                    for (int jj = 0; jj < CH; ++jj) {
                        const int j = j0 + jj;
                        if (j < TR && (FP == 2 || (FP == 1 && j < TR - 1) || tid + j * NT < npairs)) {
#pragma unroll
                            for (int r = 0; r < RR; ++r) x[jj][r] = ptx::ld_shared_u32(src + r * row_bytes + j * NT * 4);
                        }
                    }
#pragma unroll
                    for (int jj = 0; jj < CH; ++jj) {
                        const int j = j0 + jj;
                        if (j < TR && (FP == 2 || (FP == 1 && j < TR - 1) || tid + j * NT < npairs)) {
#pragma unroll
                            for (int r = 0; r < RR; ++r) {
                                const uint32_t h = HPF ? smooth2_mixed(x[jj][r], tsv[j], tmask[j]) : smooth2(x[jj][r], tsv[j]);
                                ptx::st_shared_u16(tad[j].x + r * stride, h);
                                ptx::st_shared_u16(tad[j].y + r * stride, h >> 16);
                            }
                        }
                    }
                }
            };
            if (rows == R) {
                route_rows(std::integral_constant<int, R>{});
            } else {
                static_assert(R <= 2, "a partial group of the register-held form has one row");
                route_rows(std::integral_constant<int, 1>{});
            }
        } else {
            for (int c = tid; c < npairs; c += NT) {
                const float2 sv = __ldg(is2 + c);
                const int2 dv = __ldg(rt2 + c);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (r < rows) {
                        const uint32_t x = ptx::ld_shared_u32(src + r * row_bytes + (c - tid) * 4);
                        const uint32_t h = HPF ? smooth2_mixed(x, sv, slot_mask(dv, nb * QA_BLOCK_BYTES))
                                               : smooth2(x, sv);
                        ptx::st_shared_u16(sbuf_u32 + r * stride + dv.x, h);
                        ptx::st_shared_u16(sbuf_u32 + r * stride + dv.y, h >> 16);
                    }
                }
            }
        }
        __syncthreads();  // raw slot consumed, staged rows complete
        if (tid == 0 && issued < mine) issue(issued++);
        encode_staged<MODE>(p, sbuf_u32, stride, g * R, rows);
        if (g * R <= p.M - 1 && p.M - 1 < g * R + rows) zero_padding_scale_rows(p);
        __syncthreads();  // staged rows free for the next group
    }
}

// ------------------------------------------------- two-row groups, paired staging
//
// The streaming form for two-row groups with register-held pairs stages the
// two rows interleaved: routed position p of the bulk (or outlier slot i)
// is one 32-bit word, row 0's BF16 value in the low half and row 1's in the
// high half. A routing thread then stores each channel of both rows with
// one 32-bit store (two per channel pair instead of four 16-bit stores and
// two row offsets), and an encoding thread takes one 32-block of both rows
// from eight 128-bit loads: one packed abs-max chain gives both rows' block
// maxima, and the E2M1 conversion unpacks the low or high halves exactly as
// it would unpack a row's packed pairs. A staged block of the pair is 32
// words plus 16 bytes of padding (144 bytes: an odd number of 16-byte units,
// so the 16-byte reads of consecutive blocks hit distinct banks); the
// outlier slots follow the nb blocks.
constexpr int IP_BLOCK = 144;
__host__ __device__ constexpr int qa_ip_bytes(int nb, int kp) { return nb * IP_BLOCK + kp * 4; }

// Eight BF16 values, the low (HI = false) or high (HI = true) halves of
// eight consecutive staged words, scaled by `inv` (a power of two, or the
// NVFP4 element multiplier) -> eight E2M1 codes, element i in nibble i.
template <bool HI>
__device__ __forceinline__ uint32_t encode8_halves(const uint32_t* w, float inv) {
    auto f = [](uint32_t x) { return __uint_as_float(HI ? (x & 0xFFFF0000u) : (x << 16)); };
    const float2 iv = make_float2(inv, inv);
    const float2 v0 = __fmul2_rn(make_float2(f(w[0]), f(w[1])), iv);
    const float2 v1 = __fmul2_rn(make_float2(f(w[2]), f(w[3])), iv);
    const float2 v2 = __fmul2_rn(make_float2(f(w[4]), f(w[5])), iv);
    const float2 v3 = __fmul2_rn(make_float2(f(w[6]), f(w[7])), iv);
    uint32_t out;
    asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
        "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
        : "=r"(out)
        : "f"(v0.x), "f"(v0.y), "f"(v1.x), "f"(v1.y), "f"(v2.x), "f"(v2.y), "f"(v3.x), "f"(v3.y));
    return out;
}

// Encode staged block b of both rows of the pair (output rows t0, t0 + 1;
// the second only when rows == 2). The block is read twice -- once for the
// maxima, once, eight words at a time, for the codes -- so that the 32
// words never need registers of their own next to the routing thread's
// register-held pairs.
template <int MODE>
__device__ __forceinline__ void encode_pair_block(const QuantParams& p, uint32_t sbuf, int t0, int rows, int b) {
    const uint32_t src = sbuf + b * IP_BLOCK;
    using mx::bf16x2_absmax;
    uint32_t mq[2];  // packed maxima of positions 0-15 and 16-31 (row 0 low, row 1 high)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 v0 = ptx::ld_shared_v4(src + 64 * h), v1 = ptx::ld_shared_v4(src + 64 * h + 16),
                    v2 = ptx::ld_shared_v4(src + 64 * h + 32), v3 = ptx::ld_shared_v4(src + 64 * h + 48);
        mq[h] = bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(v0.x, v0.y), bf16x2_absmax(v0.z, v0.w)),
                              bf16x2_absmax(bf16x2_absmax(v1.x, v1.y), bf16x2_absmax(v1.z, v1.w)));
        mq[h] = bf16x2_absmax(mq[h], bf16x2_absmax(bf16x2_absmax(bf16x2_absmax(v2.x, v2.y), bf16x2_absmax(v2.z, v2.w)),
                                                   bf16x2_absmax(bf16x2_absmax(v3.x, v3.y), bf16x2_absmax(v3.z, v3.w))));
    }
    // element multipliers of each row for positions 0-15 and 16-31
    float f0[2], f1[2];
    const size_t cstride = static_cast<size_t>(p.Kbp >> 1);
    uint8_t* codes0 = p.codes + static_cast<size_t>(t0) * cstride + b * 16;
    if constexpr (MODE == QA_NV) {
        const uint32_t s0 = mx::nv_block_scales(mq[0] & 0x7FFFu, mq[1] & 0x7FFFu, p.nv_k, p.nv_p2g, &f0[0], &f0[1]);
        const uint32_t s1 = mx::nv_block_scales((mq[0] >> 16) & 0x7FFFu, (mq[1] >> 16) & 0x7FFFu, p.nv_k, p.nv_p2g,
                                                &f1[0], &f1[1]);
        *reinterpret_cast<uint16_t*>(p.scales + sf_offset(t0, 2 * b, p.katoms)) = static_cast<uint16_t>(s0);
        if (rows == 2)
            *reinterpret_cast<uint16_t*>(p.scales + sf_offset(t0 + 1, 2 * b, p.katoms)) = static_cast<uint16_t>(s1);
    } else {
        const uint32_t m = bf16x2_absmax(mq[0], mq[1]);
        const bool real = b * 32 < p.Kb;
        const int X0 = mx::bf16_block_exponent(m & 0x7FFFu, &f0[0]);
        const int X1 = mx::bf16_block_exponent((m >> 16) & 0x7FFFu, &f1[0]);
        f0[1] = f0[0];
        f1[1] = f1[0];
        p.scales[sf_offset(t0, b, p.katoms)] = static_cast<uint8_t>(real ? X0 + 127 : 0);
        if (rows == 2) p.scales[sf_offset(t0 + 1, b, p.katoms)] = static_cast<uint8_t>(real ? X1 + 127 : 0);
    }
    uint32_t c0[4], c1[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 a = ptx::ld_shared_v4(src + 32 * q), d = ptx::ld_shared_v4(src + 32 * q + 16);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, d.x, d.y, d.z, d.w};
        c0[q] = encode8_halves<false>(w, f0[q >> 1]);
        c1[q] = encode8_halves<true>(w, f1[q >> 1]);
    }
    *reinterpret_cast<uint4*>(codes0) = make_uint4(c0[0], c0[1], c0[2], c0[3]);
    if (rows == 2) *reinterpret_cast<uint4*>(codes0 + cstride) = make_uint4(c1[0], c1[1], c1[2], c1[3]);
}

// Outlier slots 8c .. 8c + 7 of both rows (32 staged bytes) -> two 16-byte
// stores (NVFP4: scaled by 2^-g_act).
template <int MODE>
__device__ __forceinline__ void copy_pair_slots(const QuantParams& p, uint32_t sbuf, int nb, int t0, int rows, int c) {
    const uint32_t src = sbuf + nb * IP_BLOCK + c * 32;
    const uint4 a = ptx::ld_shared_v4(src), d = ptx::ld_shared_v4(src + 16);
    uint4 r0 = make_uint4(__byte_perm(a.x, a.y, 0x5410), __byte_perm(a.z, a.w, 0x5410), __byte_perm(d.x, d.y, 0x5410),
                          __byte_perm(d.z, d.w, 0x5410));
    if constexpr (MODE == QA_NV) r0 = mx::scale_bf16x8(r0, p.hp_scale);
    *reinterpret_cast<uint4*>(p.hp + static_cast<size_t>(t0) * p.kp + c * 8) = r0;
    if (rows == 2) {
        uint4 r1 = make_uint4(__byte_perm(a.x, a.y, 0x7632), __byte_perm(a.z, a.w, 0x7632),
                              __byte_perm(d.x, d.y, 0x7632), __byte_perm(d.z, d.w, 0x7632));
        if constexpr (MODE == QA_NV) r1 = mx::scale_bf16x8(r1, p.hp_scale);
        *reinterpret_cast<uint4*>(p.hp + static_cast<size_t>(t0 + 1) * p.kp + c * 8) = r1;
    }
}

// The streaming kernel for two-row groups with register-held pairs (the
// structure of quantize_act_stream_kernel: persistent CTAs, a ring of S raw
// slots filled by one bulk copy per group, bounded waits) on the paired
// staging. FP as for quantize_act_stream_kernel.
template <int S, int NT, int TR, int MODE, int FP>
__global__ void __launch_bounds__(NT, (NT <= 256 ? 3 : 2)) quantize_act_pair_kernel(QuantParams p) {
    constexpr int R = 2;
    constexpr bool HPF = MODE == QA_MX_F16;
    static_assert(TR > 0, "the paired form keeps its pairs in registers");
    ptx::grid_dep_launch();  // the dual_gemm that follows may start its prologue
    extern __shared__ __align__(128) uint8_t smem[];
    const int nb = p.Kbp >> 5;
    const int raw_bytes = R * p.K * 2;
    uint8_t* raw = smem;
    uint8_t* sbuf = smem + S * raw_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sbuf + ((qa_ip_bytes(nb, p.kp) + 7) & ~7));
    __shared__ int never;  // a flag nothing sets
    const int tid = threadIdx.x;
    const int ngroups = (p.M + R - 1) / R;
    const int mine = blockIdx.x < ngroups ? (ngroups - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;

    auto issue = [&](int i) {
        const int g = blockIdx.x + i * gridDim.x;
        const int rows = min(R, p.M - g * R);
        const uint32_t bar = ptx::smem_u32(&full[i % S]);
        const uint32_t bytes = static_cast<uint32_t>(rows) * p.K * 2u;
        ptx::mbar_arrive_expect_tx(bar, bytes + p.extra_tx);
        ptx::bulk_load(ptx::smem_u32(raw + (i % S) * raw_bytes), p.X + static_cast<size_t>(g) * R * p.K, bytes, bar);
    };
    // staged word of a position given by its offset in one unpaired staged row
    // ([blocks of 80 bytes | outlier slots], as the plan's route table)
    auto ip_off = [&](int off) -> int {
        if (off < nb * QA_BLOCK_BYTES) {
            const int b = off / QA_BLOCK_BYTES;
            return b * IP_BLOCK + ((off - b * QA_BLOCK_BYTES) >> 1) * 4;
        }
        return nb * IP_BLOCK + ((off - nb * QA_BLOCK_BYTES) >> 1) * 4;
    };

    if (tid == 0) {
        for (int s = 0; s < S; ++s) ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
        never = 0;
        ptx::fence_mbar_init();
    }
    // the padding positions (bulk [Kb, Kbp), slots [k, kp)) of both rows are
    // never written by the routing step: zero them once
    {
        const int npb = p.Kbp - p.Kb, npad = npb + (p.kp - p.k);
        for (int c = tid; c < npad; c += NT) {
            const int pos = p.Kb + c;
            const int off = c < npb ? (pos >> 5) * IP_BLOCK + (pos & 31) * 4 : nb * IP_BLOCK + (p.k + c - npb) * 4;
            *reinterpret_cast<uint32_t*>(sbuf + off) = 0u;
        }
    }
    __syncthreads();
    if (tid == 0)
        for (int i = 0; i < S && i < mine; ++i) issue(i);

    const int npairs = p.K >> 1;
    const float2* is2 = reinterpret_cast<const float2*>(p.inv_s);
    const int2* rt2 = reinterpret_cast<const int2*>(p.route);
    const uint32_t raw_u32 = ptx::smem_u32(raw), sbuf_u32 = ptx::smem_u32(sbuf);
    const uint32_t row_bytes = static_cast<uint32_t>(p.K) * 2u;
    // each thread keeps its pairs' inv_s and the staged addresses of their
    // two channels in registers for all its groups
    float2 tsv[TR];
    uint2 tad[TR];
    uint32_t tmask[TR];  // FP16 outlier branch: halves that are outlier slots
#pragma unroll
    for (int j = 0; j < TR; ++j) {
        const int c = tid + j * NT;
        tsv[j] = c < npairs ? __ldg(is2 + c) : make_float2(0.f, 0.f);
        const int2 dv = c < npairs ? __ldg(rt2 + c) : make_int2(0, 0);
        tad[j] = make_uint2(sbuf_u32 + ip_off(dv.x), sbuf_u32 + ip_off(dv.y));
        tmask[j] = HPF ? slot_mask(dv, nb * QA_BLOCK_BYTES) : 0u;
    }
    const int hv = p.kp >> 3;
    int issued = min(S, mine);
    for (int i = 0; i < mine; ++i) {
        const int g = blockIdx.x + i * gridDim.x;
        const int rows = min(R, p.M - g * R);
        const uint32_t bar = ptx::smem_u32(&full[i % S]);
        const bool ok = ptx::mbar_wait_bounded(bar, static_cast<uint32_t>((i / S) & 1), p.wait_limit_ns, &never);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(p.status, OSM_STATUS_TIMEOUT);
                // let every copy already issued land in this CTA's shared memory
                for (int j = i; j < issued; ++j)
                    if (!ptx::mbar_wait_bounded(ptx::smem_u32(&full[j % S]), static_cast<uint32_t>((j / S) & 1),
                                                20000000ull, &never))
                        ptx::spin_ns(1000000);
            }
            __syncthreads();
            return;
        }
        const uint32_t src = raw_u32 + (i % S) * raw_bytes + tid * 4;  // this thread's first pair, row 0
        // Routing: the loads of a chunk of CH pairs (both rows) are issued
        // before any of its stores; a one-row group stages zeros as row 1.
        auto route = [&](auto two) {
            constexpr bool TWO = decltype(two)::value;
            constexpr int CH = FP == 0 ? 1 : (TR <= 6 ? TR : (TR + 1) / 2);
#pragma unroll
            for (int j0 = 0; j0 < TR; j0 += CH) {
                uint32_t x0[CH], x1[CH];
#pragma unroll
                for (int jj = 0; jj < CH; ++jj) {
                    const int j = j0 + jj;
                    if (j < TR && (FP == 2 || (FP == 1 && j < TR - 1) || tid + j * NT < npairs)) {
                        x0[jj] = ptx::ld_shared_u32(src + j * NT * 4);
                        x1[jj] = TWO ? ptx::ld_shared_u32(src + row_bytes + j * NT * 4) : 0u;
                    }
                }
#pragma unroll
                for (int jj = 0; jj < CH; ++jj) {
                    const int j = j0 + jj;
                    if (j < TR && (FP == 2 || (FP == 1 && j < TR - 1) || tid + j * NT < npairs)) {
                        const uint32_t h0 = HPF ? smooth2_mixed(x0[jj], tsv[j], tmask[j]) : smooth2(x0[jj], tsv[j]);
                        const uint32_t h1 = HPF ? smooth2_mixed(x1[jj], tsv[j], tmask[j]) : smooth2(x1[jj], tsv[j]);
                        ptx::st_shared_u32(tad[j].x, __byte_perm(h0, h1, 0x5410));
                        ptx::st_shared_u32(tad[j].y, __byte_perm(h0, h1, 0x7632));
                    }
                }
            }
        };
        if (rows == R) route(std::true_type{});
        else route(std::false_type{});
        __syncthreads();  // raw slot consumed, staged rows complete
        if (tid == 0 && issued < mine) issue(issued++);
        for (int b = tid; b < nb; b += NT) encode_pair_block<MODE>(p, sbuf_u32, g * R, rows, b);
        for (int c = NT - 1 - tid; c < hv; c += NT) copy_pair_slots<MODE>(p, sbuf_u32, nb, g * R, rows, c);
        if (g * R <= p.M - 1 && p.M - 1 < g * R + rows) zero_padding_scale_rows(p);
        __syncthreads();  // staged rows free for the next group
    }
}

template <int S>
size_t pair_smem_bytes(int K, int nb, int kp) {
    return static_cast<size_t>(S) * 2 * K * 2 + ((qa_ip_bytes(nb, kp) + 7) & ~7) + 8 * S;
}

template <int R, int S>
size_t stream_smem_bytes(int K, int stride) {
    return static_cast<size_t>(S) * R * K * 2 + static_cast<size_t>(R) * stride + 8 * S;
}

}  // namespace

// ------------------------------------------------------------ launchers

int launch_act_amax(const uint16_t* X, int64_t T, int64_t K, float* amax, cudaStream_t st) {
    if (T == 0) return OSM_OK;
    // rows per CTA: AMAX_ROWS, or fewer (a multiple of 64) when that would
    // leave the GPU with less than about one wave of resident CTAs (small
    // batches: 4096 x 5120 took 15.1 us with 256 rows per CTA; one wave of
    // 128-row CTAs beat two of 64 rows by 1.3 us)
    const int64_t groups = ceil_div(K / 8, 32);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t target = static_cast<int64_t>(sms) * 6;
    int64_t rows = ceil_div(ceil_div(T * groups, target), 64) * 64;
    rows = rows < 64 ? 64 : (rows > AMAX_ROWS ? AMAX_ROWS : rows);
    dim3 grid(static_cast<unsigned>(groups), static_cast<unsigned>(ceil_div(T, rows)));
    if (ceil_div(T, rows) > 65535) return fail(OSM_ERR_UNSUPPORTED, "act_amax: T too large for one launch");
    act_amax_kernel<<<grid, AMAX_THREADS, 0, st>>>(X, T, K, amax, static_cast<int>(rows));
    return check_cuda(cudaGetLastError(), "act_amax launch");
}

int launch_act_percentile(const uint16_t* X, int64_t T, int64_t K, int64_t rank, float* score, cudaStream_t st) {
    act_percentile_kernel<<<dim3(PCT_SPLIT, static_cast<unsigned>(K / 32)), PCT_THREADS, 0, st>>>(X, T, K, rank,
                                                                                              score);
    return check_cuda(cudaGetLastError(), "act_percentile launch");
}

int launch_weight_amax(const uint16_t* W, int64_t K, int64_t N, float* wmax, cudaStream_t st) {
    weight_amax_kernel<<<static_cast<unsigned>(K), 256, 0, st>>>(W, N, wmax);
    return check_cuda(cudaGetLastError(), "weight_amax launch");
}

int launch_pack_weights(const osm_plan* pl, const uint16_t* W, const int32_t* col_order, uint8_t* codes,
                        uint8_t* scales, uint16_t* hp, cudaStream_t st) {
    const bool nv = pl->fmt == OSM_FMT_NVFP4;
    PackParams p{W, col_order, pl->d_s, pl->d_J, pl->d_O, pl->K, pl->N, pl->k, pl->Kb, pl->Kbp, pl->kp,
                 pl->wmode, codes, scales, hp, static_cast<int>(pl->Kbp / (4 * block_elems(pl->fmt))), nv ? 1 : 0,
                 nvfp4_k(pl->g_w), pow2f(pl->g_w), pow2f(-pl->g_w)};
    if (pl->Kbp > 0) {
        dim3 grid(static_cast<unsigned>(round_up(pl->N, 128) / 128), static_cast<unsigned>(pl->Kbp / 128));
        if (nv) pack_bulk_tiled_kernel<true><<<grid, PK_THREADS, 0, st>>>(p);
        else pack_bulk_tiled_kernel<false><<<grid, PK_THREADS, 0, st>>>(p);
        int rc = check_cuda(cudaGetLastError(), "pack_bulk launch");
        if (rc) return rc;
    }
    if (pl->kp > 0) {
        dim3 grid(static_cast<unsigned>(round_up(pl->N, 128) / 128), static_cast<unsigned>(pl->kp / 64));
        if (pl->hp_fp16) pack_hp_tiled_kernel<true><<<grid, PK_THREADS, 0, st>>>(p);
        else pack_hp_tiled_kernel<false><<<grid, PK_THREADS, 0, st>>>(p);
        return check_cuda(cudaGetLastError(), "pack_hp launch");
    }
    return OSM_OK;
}

// Per device and kernel, once: raise the dynamic shared-memory limit to
// what a launch needs and look up CTAs per SM for that size and the SM
// count, so that a launch costs no driver queries after the first.
static int prepare_kernel(const void* kern, int threads, size_t smem, int* per_sm_out, int* sms_out) {
    struct Setup {
        size_t smem_set = 0;
        std::map<size_t, int> per_sm;
    };
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, Setup> cache;
    static int sms_cache[64] = {};
    int dev = 0;
    int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
    if (rc) return rc;
    if (dev < 0 || dev >= 64) return fail(OSM_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(mu);
    Setup& su = cache[{kern, dev}];
    if (smem > 48 * 1024 && su.smem_set < smem) {
        if ((rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(smem)),
                             "quantize_act smem attribute")))
            return rc;
        su.smem_set = smem;
    }
    if (per_sm_out) {
        auto it = su.per_sm.find(smem);
        if (it == su.per_sm.end()) {
            int n = 0;
            if ((rc = check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem),
                                 "quantize_act occupancy")))
                return rc;
            it = su.per_sm.emplace(smem, n).first;
        }
        *per_sm_out = it->second;
    }
    if (sms_out) {
        if (!sms_cache[dev] &&
            (rc = check_cuda(cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev), "SM count")))
            return rc;
        *sms_out = sms_cache[dev];
    }
    return OSM_OK;
}

template <int R>
static int launch_qa(const QuantParams& p, int mode, size_t smem, cudaStream_t st) {
    auto kern = mode == QA_NV ? quantize_act_kernel<R, QA_NV>
                              : (mode == QA_MX_F16 ? quantize_act_kernel<R, QA_MX_F16> : quantize_act_kernel<R, QA_MX>);
    int rc = prepare_kernel(reinterpret_cast<const void*>(kern), QA_THREADS, smem, nullptr, nullptr);
    if (rc) return rc;
    const int64_t grid = ceil_div(p.M, R);
    kern<<<static_cast<unsigned>(grid), QA_THREADS, smem, st>>>(p);
    return check_cuda(cudaGetLastError(), "quantize_act launch");
}

template <int R, int S, int NT, int TR>
static int launch_stream(const QuantParams& p, int mode, int stride, cudaStream_t st) {
    const size_t smem = stream_smem_bytes<R, S>(p.K, stride);
    const int np = p.K / 2;
    const int fp = TR == 0 ? 0 : (np == TR * NT ? 2 : (np >= (TR - 1) * NT ? 1 : 0));
    auto pick = [&](auto f) {
        constexpr int F = decltype(f)::value;
        return mode == QA_NV ? quantize_act_stream_kernel<R, S, NT, TR, QA_NV, F>
                             : (mode == QA_MX_F16 ? quantize_act_stream_kernel<R, S, NT, TR, QA_MX_F16, F>
                                                  : quantize_act_stream_kernel<R, S, NT, TR, QA_MX, F>);
    };
    auto kern = fp == 2 ? pick(std::integral_constant<int, 2>{})
                        : (fp == 1 ? pick(std::integral_constant<int, 1>{}) : pick(std::integral_constant<int, 0>{}));
    int per_sm = 0, sms = 0;
    int rc = prepare_kernel(reinterpret_cast<const void*>(kern), NT, smem, &per_sm, &sms);
    if (rc) return rc;
    if (per_sm < 1) return fail(OSM_ERR_UNSUPPORTED, "quantize_act: no CTA fits");
    const int64_t groups = ceil_div(p.M, R);
    const int64_t grid = groups < static_cast<int64_t>(sms) * per_sm ? groups : static_cast<int64_t>(sms) * per_sm;
    kern<<<static_cast<unsigned>(grid), NT, smem, st>>>(p);
    return check_cuda(cudaGetLastError(), "quantize_act launch");
}

template <int S, int NT, int TR>
static int launch_pair(const QuantParams& p, int mode, cudaStream_t st) {
    const size_t smem = pair_smem_bytes<S>(p.K, p.Kbp >> 5, p.kp);
    const int np = p.K / 2;
    const int fp = np == TR * NT ? 2 : (np >= (TR - 1) * NT ? 1 : 0);
    auto pick = [&](auto f) {
        constexpr int F = decltype(f)::value;
        return mode == QA_NV ? quantize_act_pair_kernel<S, NT, TR, QA_NV, F>
                             : (mode == QA_MX_F16 ? quantize_act_pair_kernel<S, NT, TR, QA_MX_F16, F>
                                                  : quantize_act_pair_kernel<S, NT, TR, QA_MX, F>);
    };
    auto kern = fp == 2 ? pick(std::integral_constant<int, 2>{})
                        : (fp == 1 ? pick(std::integral_constant<int, 1>{}) : pick(std::integral_constant<int, 0>{}));
    int per_sm = 0, sms = 0;
    int rc = prepare_kernel(reinterpret_cast<const void*>(kern), NT, smem, &per_sm, &sms);
    if (rc) return rc;
    if (per_sm < 1) return fail(OSM_ERR_UNSUPPORTED, "quantize_act: no CTA fits");
    const int64_t groups = ceil_div(p.M, 2);
    const int64_t grid = groups < static_cast<int64_t>(sms) * per_sm ? groups : static_cast<int64_t>(sms) * per_sm;
    kern<<<static_cast<unsigned>(grid), NT, smem, st>>>(p);
    return check_cuda(cudaGetLastError(), "quantize_act launch");
}

int launch_quantize_act(const osm_plan* pl, const uint16_t* X, int64_t M, uint8_t* codes,
                        uint8_t* scales, uint16_t* hp, cudaStream_t st) {
    if (M > 0x7FFFFFFF) return fail(OSM_ERR_UNSUPPORTED, "quantize_act: M too large");
    QuantParams p{X, pl->d_inv_s, pl->d_route, static_cast<int>(M), static_cast<int>(pl->K),
                  static_cast<int>(pl->k), static_cast<int>(pl->Kb), static_cast<int>(pl->Kbp),
                  static_cast<int>(pl->kp), codes, scales, hp, pl->d_status, pl->wait_limit_ns,
                  (pl->debug_flags & OSM_DEBUG_STARVE_QUANTIZE) ? 16u : 0u, pl->hp_fp16,
                  static_cast<int>(pl->Kbp / (4 * block_elems(pl->fmt))), nvfp4_k(pl->g_act), pow2f(pl->g_act),
                  pow2f(-pl->g_act)};
    const int mode = pl->fmt == OSM_FMT_NVFP4 ? QA_NV : (pl->hp_fp16 ? QA_MX_F16 : QA_MX);
    const int stride = qa_row_stride(static_cast<int>(pl->Kbp / 32), static_cast<int>(pl->kp));
    // streaming form: two CTAs of at most 110 KB per SM
    const size_t two_per_sm = 110 * 1024;
    const int npairs = p.K / 2;
    if (stream_smem_bytes<2, 3>(p.K, stride) <= two_per_sm) {
        // Large batches: three CTAs of 256 threads per SM with a two-slot ring
        // (a block barrier spans fewer warps; measured 111.6 against 118.8 us
        // for 32760 x 5120). Small batches keep two 512-thread CTAs with three
        // slots (23.6 against 24.6 us for 4096 x 5120), whose deeper ring
        // matters when each CTA sees only a few row groups.
        if (p.M >= 8192 && npairs <= 10 * 256 && stream_smem_bytes<2, 2>(p.K, stride) * 3 <= 220 * 1024)
            return launch_pair<2, 256, 10>(p, mode, st);
        if (npairs == 5 * STREAM_NT) return launch_pair<3, STREAM_NT, 5>(p, mode, st);
        if (npairs <= 6 * STREAM_NT) return launch_pair<3, STREAM_NT, 6>(p, mode, st);
        return launch_stream<2, 3, STREAM_NT, 0>(p, mode, stride, st);
    }
    if (stream_smem_bytes<1, 3>(p.K, stride) <= two_per_sm) return launch_stream<1, 3, STREAM_NT, 0>(p, mode, stride, st);
    // rows whose ring would get only two slots at two CTAs per SM (e.g. K =
    // 13824): one CTA per SM with five slots, each thread's (up to 14)
    // channel pairs and routes held in registers
    const size_t one_per_sm = 220 * 1024;
    if (npairs <= 14 * STREAM_NT && stream_smem_bytes<1, 5>(p.K, stride) <= one_per_sm)
        return launch_stream<1, 5, STREAM_NT, 14>(p, mode, stride, st);
    if (stream_smem_bytes<1, 2>(p.K, stride) <= two_per_sm) return launch_stream<1, 2, STREAM_NT, 0>(p, mode, stride, st);
    // very wide rows: the staged, phase-serial form
    const size_t row_bytes = static_cast<size_t>(stride);
    const size_t budget = 72 * 1024;
    if (row_bytes * 8 <= budget) return launch_qa<8>(p, mode, row_bytes * 8, st);
    if (row_bytes * 4 <= budget) return launch_qa<4>(p, mode, row_bytes * 4, st);
    if (row_bytes * 2 <= budget) return launch_qa<2>(p, mode, row_bytes * 2, st);
    if (row_bytes <= 200 * 1024) return launch_qa<1>(p, mode, row_bytes, st);
    return fail(OSM_ERR_UNSUPPORTED, "quantize_act: K too large for one staged row");
}

}  // namespace osm
