// Dual-branch W4A4 GEMM for sm_100a: Eq. (5) of "W4A4 Quantization for
// Inference on Wan2.2-I2V-A14B" with Eq. (3)'s group scales taken per
// 32-element block (OCP MXFP4).
//
//   acc = sum over bulk K-steps of tcgen05.mma kind::mxf4 (block-scaled,
//         E8M0 scales in tensor memory)
//       + sum over outlier K-steps of tcgen05.mma kind::f16 (BF16 x BF16)
//
// Both branches accumulate into the same FP32 tensor-memory accumulator
// before one epilogue. Persistent CTAs (one per SM, 128x256 output tiles),
// warp-specialised:
//   warp 0     TMA producer (tiled 128B-swizzled loads of codes / BF16
//              chunks, 1-D bulk copies of the scale atoms) into a 4-deep
//              shared-memory ring guarded by mbarriers;
//   warp 1     tensor-memory allocation and the single MMA-issuing thread
//              (tcgen05.cp of the scale atoms into tensor memory, then the
//              MMAs, then tcgen05.commit to release the ring slot);
//   warps 2-5  epilogue: tcgen05.ld of the accumulator, optional bias,
//              FP32 or BF16 stores.
// Every wait is bounded by %globaltimer; a wait that runs out sets the
// plan's status word, raises a CTA-wide abort flag, and the CTA drains its
// in-flight copies and MMAs, frees tensor memory and returns.
// No TMA multicast is used anywhere.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "osm_internal.h"
#include "osm_ptx.cuh"

namespace osm {
namespace {

constexpr int BM = 128;                 // output rows per tile (TMEM lanes)
constexpr int BN = 256;                 // output columns per tile (TMEM columns)
constexpr int STAGES = 4;
constexpr int A_TILE = BM * 128;        // one K-step of A: 128 rows x 128 bytes
constexpr int B_TILE = BN * 128;        // one K-step of B: 256 rows x 128 bytes
constexpr int SFA_TILE = 2 * 512;       // two 128x4 scale atoms
constexpr int SFB_TILE = 2 * 2 * 512;   // two row tiles x two atoms
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;       // scale factors live after the accumulator
constexpr uint32_t SF_STAGE_COLS = 24;  // 8 columns for A, 16 for B per ring slot
constexpr int GROUP_M = 16;             // raster: 16 M-blocks sweep the N-blocks together

// Instruction descriptors (tcgen05 instruction-descriptor format).
// kind::mxf4 block-scaled: A/B E2M1 (1), K-major, N>>3 @17, UE8M0 scales
// (bit 23), M>>4 @24; scale-factor byte ids at bits 29-30 (A) and 4-5 (B).
constexpr uint32_t IDESC_MXF4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) |
                                ((uint32_t)(BM >> 4) << 24);
// kind::f16: FP32 accumulate (bit 4), A/B BF16 (1 @7, 1 @10), K-major.
constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(BM >> 4) << 24);

struct __align__(1024) Smem {
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint8_t sfa[STAGES][SFA_TILE];
    uint8_t sfb[STAGES][SFB_TILE];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct GemmParams {
    CUtensorMap tm_a;    // a_codes  [M][Kbp/2] u8, box 128 x 128
    CUtensorMap tm_b;    // w_codes  [N][Kbp/2] u8, box 128 x 256
    CUtensorMap tm_ah;   // a_hp     [M][kp] bf16, box 64 x 128
    CUtensorMap tm_bh;   // w_hp     [N][kp] bf16, box 64 x 256
    const uint8_t* a_scales;
    const uint8_t* w_scales;
    const float* bias;
    void* Y;
    uint32_t* status;
    uint64_t wait_limit_ns;
    int64_t M, N;
    int katoms;      // Kbp / 128
    int n_fp4;       // K-steps of the bulk branch: ceil(katoms / 2)
    int n_hp;        // K-steps of the outlier branch: kp / 64
    int num_m, num_n;
    int n_row_tiles; // ceil(N / 128): scale-atom rows of W
    int epi;
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& m_blk, int& n_blk) {
    const int group = GROUP_M * num_n;
    const int g = tile / group;
    const int first_m = g * GROUP_M;
    const int gm = min(num_m - first_m, GROUP_M);
    const int local = tile % group;
    m_blk = first_m + local % gm;
    n_blk = local / gm;
}

__device__ __forceinline__ void raise_abort(Smem& S, uint32_t* status) {
    S.abort_flag = 1;
    atomicOr(status, OSM_STATUS_TIMEOUT);
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    return ptx::smem_desc(saddr, 16, 1024, ptx::LAYOUT_SW128);
}

__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
    // 32 rows x 16 bytes, core matrices of 8 rows stacked every 128 bytes
    return ptx::smem_desc(saddr, 0, 128, ptx::LAYOUT_NONE);
}

__device__ __forceinline__ void store_chunk(const GemmParams& p, int64_t row, int64_t col0,
                                            const uint32_t (&r)[32]) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    if (p.bias) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            const float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + col0 + i));
            v[i] += b.x;
            v[i + 1] += b.y;
            v[i + 2] += b.z;
            v[i + 3] += b.w;
        }
    }
    if (p.epi == OSM_EPI_F32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.Y) + row * p.N + col0);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.Y) + row * p.N + col0);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) dual_gemm_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles = p.num_m * p.num_n;
    const int ksteps = p.n_fp4 + p.n_hp;
    const volatile int* abort = &S.abort_flag;
    __shared__ int never;  // a flag nothing sets: drain waits use it instead of the abort flag
    // Drains wait for work that always completes (copies, MMAs); they get a
    // generous limit even when the pipeline limit is set very short.
    const uint64_t drain_ns = p.wait_limit_ns > 200000000ull ? p.wait_limit_ns : 200000000ull;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(ptx::smem_u32(&S.full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(&S.acc_full), 1);
        ptx::mbar_init(ptx::smem_u32(&S.acc_empty), 4);
        ptx::mbar_init(ptx::smem_u32(&S.drain), 1);
        S.abort_flag = 0;
        never = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        if (p.n_fp4) { ptx::prefetch_tmap(&p.tm_a); ptx::prefetch_tmap(&p.tm_b); }
        if (p.n_hp) { ptx::prefetch_tmap(&p.tm_ah); ptx::prefetch_tmap(&p.tm_bh); }
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&S.tmem_base), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (ptx::elect_one()) {
            int stage = 0;
            uint32_t phase = 0;
            int issued[STAGES];
            uint32_t issued_phase[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = 0, issued_phase[s] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(tile, p.num_m, p.num_n, m_blk, n_blk);
                const int m0 = m_blk * BM, n0 = n_blk * BN;
                const int nbt = min(2, p.n_row_tiles - 2 * n_blk);  // valid 128-row scale tiles of W
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint32_t eb = ptx::smem_u32(&S.empty[stage]);
                    if (!ptx::mbar_wait_bounded(eb, phase ^ 1u, p.wait_limit_ns, abort)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = ptx::smem_u32(&S.full[stage]);
                    if (ks < p.n_fp4) {
                        const int natoms = min(2, p.katoms - 2 * ks);
                        const uint32_t sf_bytes = natoms * 512u;
                        ptx::mbar_arrive_expect_tx(fb, A_TILE + B_TILE + sf_bytes * (1 + nbt));
                        ptx::tma_load_2d(ptx::smem_u32(S.a[stage]), &p.tm_a, ks * 128, m0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(S.b[stage]), &p.tm_b, ks * 128, n0, fb);
                        ptx::bulk_load(ptx::smem_u32(S.sfa[stage]),
                                       p.a_scales + ((int64_t)m_blk * p.katoms + 2 * ks) * 512, sf_bytes, fb);
                        for (int h = 0; h < nbt; ++h)
                            ptx::bulk_load(ptx::smem_u32(S.sfb[stage]) + h * 1024,
                                           p.w_scales + ((int64_t)(2 * n_blk + h) * p.katoms + 2 * ks) * 512,
                                           sf_bytes, fb);
                    } else {
                        const int kh = ks - p.n_fp4;
                        ptx::mbar_arrive_expect_tx(fb, A_TILE + B_TILE);
                        ptx::tma_load_2d(ptx::smem_u32(S.a[stage]), &p.tm_ah, kh * 64, m0, fb);
                        ptx::tma_load_2d(ptx::smem_u32(S.b[stage]), &p.tm_bh, kh * 64, n0, fb);
                    }
                    issued[stage] = 1;
                    issued_phase[stage] = phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) raise_abort(S, p.status);
            // every copy this thread issued has landed before the CTA can exit
            for (int s = 0; s < STAGES; ++s)
                if (issued[s])
                    ptx::mbar_wait_bounded(ptx::smem_u32(&S.full[s]), issued_phase[s], drain_ns, &never);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (ptx::elect_one()) {
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            const uint32_t acc = tmem;  // lane 0, column 0
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                if (!ptx::mbar_wait_bounded(ptx::smem_u32(&S.acc_empty), acc_phase ^ 1u, p.wait_limit_ns, abort)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                uint32_t accumulate = 0;
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (!ptx::mbar_wait_bounded(ptx::smem_u32(&S.full[stage]), phase, p.wait_limit_ns, abort)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_base = ptx::smem_u32(S.a[stage]);
                    const uint32_t b_base = ptx::smem_u32(S.b[stage]);
                    if (ks < p.n_fp4) {
                        const int natoms = min(2, p.katoms - 2 * ks);
                        const uint32_t sfa_col = tmem + SF_COL0 + stage * SF_STAGE_COLS;
                        const uint32_t sfb_col = sfa_col + 8;
                        const uint32_t sfa_s = ptx::smem_u32(S.sfa[stage]);
                        const uint32_t sfb_s = ptx::smem_u32(S.sfb[stage]);
                        for (int a = 0; a < natoms; ++a) {
                            ptx::tc_cp_32x128_x4(sfa_col + 4 * a, desc_sf(sfa_s + 512 * a));
                            ptx::tc_cp_32x128_x4(sfb_col + 8 * a, desc_sf(sfb_s + 512 * a));
                            ptx::tc_cp_32x128_x4(sfb_col + 8 * a + 4, desc_sf(sfb_s + 1024 + 512 * a));
                        }
                        for (int kk = 0; kk < 2 * natoms; ++kk) {
                            const uint32_t sf_id = (uint32_t)(kk & 1) * 2u;  // bytes 0-1 or 2-3 of the atom
                            const uint32_t idesc = IDESC_MXF4 | (sf_id << 29) | (sf_id << 4);
                            ptx::mma_mxf4(acc, desc_sw128(a_base + kk * 32), desc_sw128(b_base + kk * 32), idesc,
                                          sfa_col + 4 * (kk >> 1), sfb_col + 8 * (kk >> 1), accumulate);
                            accumulate = 1;
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            ptx::mma_bf16(acc, desc_sw128(a_base + kk * 32), desc_sw128(b_base + kk * 32),
                                          IDESC_BF16, accumulate);
                            accumulate = 1;
                        }
                    }
                    ptx::tc_commit(ptx::smem_u32(&S.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::tc_commit(ptx::smem_u32(&S.acc_full));
                acc_phase ^= 1u;
            }
            if (!ok) raise_abort(S, p.status);
            // all issued tensor-core work has finished before tensor memory is freed
            ptx::tc_commit(ptx::smem_u32(&S.drain));
            ptx::mbar_wait_bounded(ptx::smem_u32(&S.drain), 0, drain_ns, &never);
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lanes 32q..32q+31 are reachable from this warp
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            int m_blk, n_blk;
            tile_coords(tile, p.num_m, p.num_n, m_blk, n_blk);
            int ok = 1;
            if (lane == 0)
                ok = ptx::mbar_wait_bounded(ptx::smem_u32(&S.acc_full), acc_phase, p.wait_limit_ns, abort) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) raise_abort(S, p.status);
                break;
            }
            ptx::tc_fence_after();
            const int64_t row = (int64_t)m_blk * BM + q * 32 + lane;
            const int64_t n0 = (int64_t)n_blk * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                ptx::tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + c * 32, r);
                ptx::tmem_ld_wait();
                const int64_t col0 = n0 + c * 32;
                if (row < p.M && col0 < p.N) store_chunk(p, row, col0, r);
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&S.acc_empty));
            acc_phase ^= 1u;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

int make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, const char* what) {
    auto enc = get_encode_fn();
    if (!enc) return fail(OSM_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OSM_ERR_CUDA, "tensor map for %s: CUresult %d", what, (int)r);
    return OSM_OK;
}

}  // namespace

size_t dual_gemm_smem_bytes() { return sizeof(Smem) + 1024; }

int launch_dual_gemm(const osm_plan* pl, const uint8_t* a_codes, const uint8_t* a_scales, const uint16_t* a_hp,
                     int64_t M, const uint8_t* w_codes, const uint8_t* w_scales, const uint16_t* w_hp,
                     const float* bias, int epi, void* Y, cudaStream_t st) {
    static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory budget");
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    int rc;
    if (pl->Kbp > 0) {
        if ((rc = make_map(&p.tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, pl->Kbp / 2, M, pl->Kbp / 2, 128, BM,
                           "a_codes")))
            return rc;
        if ((rc = make_map(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, pl->Kbp / 2, pl->N, pl->Kbp / 2, 128,
                           BN, "w_codes")))
            return rc;
    }
    if (pl->kp > 0) {
        if ((rc = make_map(&p.tm_ah, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_hp, pl->kp, M, pl->kp * 2, 64, BM,
                           "a_hp")))
            return rc;
        if ((rc = make_map(&p.tm_bh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_hp, pl->kp, pl->N, pl->kp * 2, 64, BN,
                           "w_hp")))
            return rc;
    }
    p.a_scales = a_scales;
    p.w_scales = w_scales;
    p.bias = bias;
    p.Y = Y;
    p.status = pl->d_status;
    p.wait_limit_ns = pl->wait_limit_ns;
    p.M = M;
    p.N = pl->N;
    p.katoms = static_cast<int>(pl->Kbp / 128);
    p.n_fp4 = (p.katoms + 1) / 2;
    p.n_hp = static_cast<int>(pl->kp / 64);
    p.num_m = static_cast<int>(ceil_div(M, BM));
    p.num_n = static_cast<int>(ceil_div(pl->N, BN));
    p.n_row_tiles = static_cast<int>(ceil_div(pl->N, 128));
    p.epi = epi;

    int dev = 0, sms = 0;
    if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
    if ((rc = check_cuda(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "SM count")))
        return rc;
    const size_t smem = sizeof(Smem) + 1024;
    if ((rc = check_cuda(cudaFuncSetAttribute(dual_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem)),
                         "dual_gemm smem attribute")))
        return rc;
    const int64_t tiles = (int64_t)p.num_m * p.num_n;
    if (tiles > 0x7FFFFFFF) return fail(OSM_ERR_UNSUPPORTED, "dual_gemm: too many tiles");
    const int grid = static_cast<int>(tiles < sms ? tiles : sms);
    dual_gemm_kernel<<<grid, NUM_THREADS, smem, st>>>(p);
    return check_cuda(cudaGetLastError(), "dual_gemm launch");
}

}  // namespace osm
