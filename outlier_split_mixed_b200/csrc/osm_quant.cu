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

#include "osm_internal.h"

namespace osm {
namespace {

// ------------------------------------------------------------ helpers

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// FP32 -> BF16 bits, round to nearest even (cvt.rn.bf16.f32).
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// MX shared exponent X = floor(log2 amax) - 2, clamped to [-127, 127],
// amax == 0 -> -127. amax is a finite, non-negative float; floor(log2) is
// read from the exponent field (subnormals from the leading mantissa bit).
__device__ __forceinline__ int mx_exponent(float amax) {
    const uint32_t u = __float_as_uint(amax);
    if (u == 0u) return -127;
    const int e = static_cast<int>((u >> 23) & 0xFFu);
    const int fl = e ? e - 127 : (31 - __clz(u & 0x7FFFFFu)) - 149;
    int X = fl - 2;
    X = X < -127 ? -127 : X;
    X = X > 127 ? 127 : X;
    return X;
}

// 2^-X as an exact float for X in [-127, 127].
__device__ __forceinline__ float exp2_neg(int X) {
    return X <= 126 ? __uint_as_float(static_cast<uint32_t>(127 - X) << 23)
                    : __uint_as_float(0x00400000u >> (X - 127));
}

// Eight non-negative magnitudes -> eight E2M1 codes (round to nearest even,
// saturating at 6), element i in nibble i.
__device__ __forceinline__ uint32_t e2m1x8(const float (&a)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
    return out;
}

// Encode 8 BF16 values (bits in h[0..7]) with shared exponent X. The sign
// bit of each code is the sign bit of the BF16 input.
__device__ __forceinline__ uint32_t encode8(const uint32_t (&h)[8], int X) {
    const float inv = exp2_neg(X);
    float a[8];
    uint32_t signs = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        a[i] = bf16_bits_to_f32(h[i] & 0x7FFFu) * inv;  // exact: power-of-two scaling
        signs |= ((h[i] >> 15) & 1u) << (4 * i + 3);
    }
    return e2m1x8(a) | signs;
}

// Byte offset of E8M0 scale (row r, 32-block b) in the tcgen05 block-scale
// layout: 512-byte atoms of 128 rows x 4 blocks.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int64_t katoms) {
    return ((r >> 7) * katoms + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ------------------------------------------------------------ calibration

constexpr int AMAX_ROWS = 64;

// amax[j] = max(amax[j], max_t |X[t][j]|). One thread per 8 channels and
// AMAX_ROWS rows; the per-thread maxima are merged with atomicMax on the
// IEEE bit pattern (monotone for non-negative floats).
__global__ void __launch_bounds__(128) act_amax_kernel(const uint16_t* __restrict__ X, int64_t T,
                                                       int64_t K, float* __restrict__ amax) {
    const int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (v * 8 >= K) return;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * AMAX_ROWS;
    const int64_t t1 = min(T, t0 + AMAX_ROWS);
    uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // |x| bit patterns (bf16 << 16)
    for (int64_t t = t0; t < t1; ++t) {
        const uint4 q = ldg_nc_v4(X + t * K + v * 8);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m[2 * i] = max(m[2 * i], (w[i] & 0x7FFFu) << 16);
            m[2 * i + 1] = max(m[2 * i + 1], (w[i] >> 16 & 0x7FFFu) << 16);
        }
    }
    unsigned int* dst = reinterpret_cast<unsigned int*>(amax) + v * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) atomicMax(dst + i, m[i]);
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
    const float* s;     // [K]
    const int32_t* J;   // [Kb]
    const int32_t* O;   // [k]
    int64_t K, N, k, Kb, Kbp, kp;
    int mode;
    uint8_t* codes;     // [N][Kbp/2]
    uint8_t* scales;    // layout, rows padded to 128
    uint16_t* hp;       // [N][kp]
};

// One thread per (output channel n, 128-wide bulk strip). Threads of a warp
// take 32 consecutive n, so every W row read is a coalesced 64-byte segment
// and a 32x32 tile is exactly one warp.
__global__ void __launch_bounds__(256) pack_bulk_kernel(PackParams p) {
    const int64_t n = static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x;
    const int64_t strip = static_cast<int64_t>(blockIdx.y) * 8 + threadIdx.y;
    const int64_t katoms = p.Kbp / 128;
    if (strip >= katoms) return;  // uniform per warp
    const bool nvalid = n < p.N;
    uint32_t h[128];
    float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 128; ++i) {
        const int64_t pos = strip * 128 + i;
        uint32_t bits = 0;
        if (nvalid && pos < p.Kb) {
            const int32_t j = __ldg(p.J + pos);
            const float w = bf16_bits_to_f32(p.W[static_cast<int64_t>(j) * p.N + n]);
            bits = f32_to_bf16_bits(w * __ldg(p.s + j));
        }
        h[i] = bits;
        am[i >> 5] = fmaxf(am[i >> 5], bf16_bits_to_f32(bits & 0x7FFFu));
    }
    if (p.mode == OSM_WSCALE_STRIP128x1) {
        const float m = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
        am[0] = am[1] = am[2] = am[3] = m;
    } else if (p.mode == OSM_WSCALE_TILE32x32) {
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int o = 16; o; o >>= 1) am[b] = fmaxf(am[b], __shfl_xor_sync(0xffffffffu, am[b], o));
    }
    uint32_t sc = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const int X = mx_exponent(am[b]);
        const int64_t pos0 = strip * 128 + b * 32;
        const uint32_t code = (nvalid && pos0 < p.Kb) ? static_cast<uint32_t>(X + 127) : 0u;
        sc |= code << (8 * b);
        if (nvalid) {
            uint4 out;
            uint32_t* o4 = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t hh[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) hh[e] = h[b * 32 + g * 8 + e];
                o4[g] = encode8(hh, X);
            }
            *reinterpret_cast<uint4*>(p.codes + n * (p.Kbp / 2) + strip * 64 + b * 16) = out;
        }
    }
    // four scales of this strip are contiguous bytes of one atom row
    if (n < (p.N + 127) / 128 * 128) {
        *reinterpret_cast<uint32_t*>(p.scales + sf_offset(n, strip * 4, katoms)) = sc;
    }
}

// w_hp[n][i] = bf16(w[O_i][n] * s[O_i]) for i < k, zero for k <= i < kp.
__global__ void __launch_bounds__(256) pack_hp_kernel(PackParams p) {
    const int64_t n = static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x;
    const int64_t i = static_cast<int64_t>(blockIdx.y) * 8 + threadIdx.y;
    if (n >= p.N || i >= p.kp) return;
    uint32_t bits = 0;
    if (i < p.k) {
        const int32_t j = p.O[i];
        bits = f32_to_bf16_bits(bf16_bits_to_f32(p.W[static_cast<int64_t>(j) * p.N + n]) * p.s[j]);
    }
    p.hp[n * p.kp + i] = static_cast<uint16_t>(bits);
}

// ------------------------------------------------------------ quantize_act

struct QuantParams {
    const uint16_t* X;       // [M][K]
    const float* inv_s;      // [K]
    const int32_t* route;    // [K]
    int64_t M, K, k, Kb, Kbp, kp;
    uint8_t* codes;          // [M][Kbp/2]
    uint8_t* scales;         // layout, rows padded to 128
    uint16_t* hp;            // [M][kp]
};

constexpr int QA_THREADS = 256;

// Each CTA handles R consecutive rows.
//  phase 1: coalesced 16-byte loads of the rows; x' = bf16(x * inv_s) is
//           scattered into a shared-memory row in [bulk J | outliers O]
//           order (the routing table is the channel -> slot map);
//  phase 2: four threads per 32-block of the compacted bulk row: 16-byte
//           shared loads, amax by two xor-shuffles, E8M0 scale, E2M1 codes
//           (one coalesced 32-bit store per thread);
//  phase 3: the outlier slots go out as 16-byte stores.
template <int R>
__global__ void __launch_bounds__(QA_THREADS) quantize_act_kernel(QuantParams p) {
    extern __shared__ __align__(16) uint16_t srow[];
    const int64_t W = p.Kbp + p.kp;             // staged row length (elements)
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * R;
    const int tid = threadIdx.x;

    // zero the padding slots [Kb, Kbp) and [Kbp + k, Kbp + kp)
    const int64_t npad_b = p.Kbp - p.Kb, npad_h = p.kp - p.k;
    for (int64_t i = tid; i < R * (npad_b + npad_h); i += QA_THREADS) {
        const int64_t r = i / (npad_b + npad_h), c = i % (npad_b + npad_h);
        const int64_t col = c < npad_b ? p.Kb + c : p.Kbp + p.k + (c - npad_b);
        srow[r * W + col] = 0;
    }

    // phase 1
    const int64_t nvec = p.K / 8;
    for (int64_t v = tid; v < nvec; v += QA_THREADS) {
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(p.inv_s + v * 8));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(p.inv_s + v * 8 + 4));
        const int4 d0 = __ldg(reinterpret_cast<const int4*>(p.route + v * 8));
        const int4 d1 = __ldg(reinterpret_cast<const int4*>(p.route + v * 8 + 4));
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        const int dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        uint4 xv[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t t = row0 + r;
            xv[r] = (t < p.M) ? ldg_nc_v4(p.X + t * p.K + v * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t w[4] = {xv[r].x, xv[r].y, xv[r].z, xv[r].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t hb = (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu);
                const float xs = bf16_bits_to_f32(hb) * sv[i];
                srow[r * W + dv[i]] = static_cast<uint16_t>(f32_to_bf16_bits(xs));
            }
        }
    }
    __syncthreads();

    // phase 2
    const int64_t G = p.Kbp / 8;   // 8-element groups per row
    const int64_t katoms = p.Kbp / 128;
    const int lane = tid & 31;
    for (int64_t gb = (tid & ~31); gb < R * G; gb += QA_THREADS) {
        const int64_t g = gb + lane;
        const bool valid = g < R * G;
        const int64_t r = valid ? g / G : 0, q = valid ? g % G : 0;
        uint32_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (valid) {
            const uint4 u = *reinterpret_cast<const uint4*>(srow + r * W + q * 8);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                h[2 * i] = w[i] & 0xFFFFu;
                h[2 * i + 1] = w[i] >> 16;
            }
        }
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = max(m, h[i] & 0x7FFFu);
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const int X = mx_exponent(bf16_bits_to_f32(m));
        const uint32_t word = encode8(h, X);
        const int64_t t = row0 + r;
        if (valid && t < p.M) {
            *reinterpret_cast<uint32_t*>(p.codes + t * (p.Kbp / 2) + q * 4) = word;
            if ((q & 3) == 0) {
                const int64_t b = q >> 2;
                p.scales[sf_offset(t, b, katoms)] =
                    static_cast<uint8_t>(b * 32 < p.Kb ? X + 127 : 0);
            }
        }
    }

    // phase 3: outlier slots
    const int64_t hv = p.kp / 8;
    for (int64_t i = tid; i < R * hv; i += QA_THREADS) {
        const int64_t r = i / hv, c = i % hv;
        const int64_t t = row0 + r;
        if (t < p.M)
            *reinterpret_cast<uint4*>(p.hp + t * p.kp + c * 8) =
                *reinterpret_cast<const uint4*>(srow + r * W + p.Kbp + c * 8);
    }

    // scale bytes of the padding rows [M, round_up(M,128)) are zero
    if (row0 <= p.M - 1 && p.M - 1 < row0 + R && (p.M & 127) != 0) {
        const int64_t tile = (p.M - 1) >> 7;
        const int64_t rem = p.M & 127;
        const int64_t nwords = (128 - rem) * katoms;
        for (int64_t i = tid; i < nwords; i += QA_THREADS) {
            const int64_t rr = rem + i % (128 - rem), a = i / (128 - rem);
            *reinterpret_cast<uint32_t*>(p.scales + sf_offset(tile * 128 + rr, a * 4, katoms)) = 0u;
        }
    }
}

}  // namespace

// ------------------------------------------------------------ launchers

int launch_act_amax(const uint16_t* X, int64_t T, int64_t K, float* amax, cudaStream_t st) {
    if (T == 0) return OSM_OK;
    dim3 grid(static_cast<unsigned>(ceil_div(K / 8, 128)), static_cast<unsigned>(ceil_div(T, AMAX_ROWS)));
    if (grid.y > 65535u) return fail(OSM_ERR_UNSUPPORTED, "act_amax: T too large for one launch");
    act_amax_kernel<<<grid, 128, 0, st>>>(X, T, K, amax);
    return check_cuda(cudaGetLastError(), "act_amax launch");
}

int launch_weight_amax(const uint16_t* W, int64_t K, int64_t N, float* wmax, cudaStream_t st) {
    weight_amax_kernel<<<static_cast<unsigned>(K), 256, 0, st>>>(W, N, wmax);
    return check_cuda(cudaGetLastError(), "weight_amax launch");
}

int launch_pack_weights(const osm_plan* pl, const uint16_t* W, uint8_t* codes, uint8_t* scales,
                        uint16_t* hp, cudaStream_t st) {
    PackParams p{W, pl->d_s, pl->d_J, pl->d_O, pl->K, pl->N, pl->k, pl->Kb, pl->Kbp, pl->kp,
                 pl->wmode, codes, scales, hp};
    if (pl->Kbp > 0) {
        dim3 grid(static_cast<unsigned>(round_up(pl->N, 128) / 32),
                  static_cast<unsigned>(ceil_div(pl->Kbp / 128, 8)));
        pack_bulk_kernel<<<grid, dim3(32, 8), 0, st>>>(p);
        int rc = check_cuda(cudaGetLastError(), "pack_bulk launch");
        if (rc) return rc;
    }
    if (pl->kp > 0) {
        dim3 grid(static_cast<unsigned>(ceil_div(pl->N, 32)), static_cast<unsigned>(ceil_div(pl->kp, 8)));
        pack_hp_kernel<<<grid, dim3(32, 8), 0, st>>>(p);
        return check_cuda(cudaGetLastError(), "pack_hp launch");
    }
    return OSM_OK;
}

template <int R>
static int launch_qa(const QuantParams& p, size_t smem, cudaStream_t st) {
    auto kern = quantize_act_kernel<R>;
    if (smem > 48 * 1024) {
        int rc = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem)),
                            "quantize_act smem attribute");
        if (rc) return rc;
    }
    const int64_t grid = ceil_div(p.M, R);
    if (grid > 0x7FFFFFFF) return fail(OSM_ERR_UNSUPPORTED, "quantize_act: M too large");
    kern<<<static_cast<unsigned>(grid), QA_THREADS, smem, st>>>(p);
    return check_cuda(cudaGetLastError(), "quantize_act launch");
}

int launch_quantize_act(const osm_plan* pl, const uint16_t* X, int64_t M, uint8_t* codes,
                        uint8_t* scales, uint16_t* hp, cudaStream_t st) {
    QuantParams p{X, pl->d_inv_s, pl->d_route, M, pl->K, pl->k, pl->Kb, pl->Kbp, pl->kp, codes, scales, hp};
    const size_t row_bytes = static_cast<size_t>(pl->Kbp + pl->kp) * 2;
    const size_t budget = 64 * 1024;
    if (row_bytes * 8 <= budget) return launch_qa<8>(p, row_bytes * 8, st);
    if (row_bytes * 4 <= budget) return launch_qa<4>(p, row_bytes * 4, st);
    if (row_bytes * 2 <= budget) return launch_qa<2>(p, row_bytes * 2, st);
    if (row_bytes <= 200 * 1024) return launch_qa<1>(p, row_bytes, st);
    return fail(OSM_ERR_UNSUPPORTED, "quantize_act: K too large for one staged row");
}

}  // namespace osm
