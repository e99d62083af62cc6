// Dual-branch W4A4 GEMM for sm_100a: Eq. (5) of "W4A4 Quantization for
// Inference on Wan2.2-I2V-A14B" with Eq. (3)'s group scales taken per
// 32-element block (OCP MXFP4), or per 16-element block (NVFP4).
//
//   acc = sum over bulk K-steps of tcgen05.mma kind::mxf4 (block-scaled,
//         E8M0 scales in tensor memory) or kind::mxf4nvf4 (UE4M3 scales)
//       + sum over outlier K-steps of tcgen05.mma kind::f16 (BF16 or FP16)
//
// Both branches accumulate into the same FP32 tensor-memory accumulator
// before one epilogue.
//
// Work decomposition: persistent CTA pairs (clusters of 2, one CTA per SM);
// each pair owns a 256 x 256 output tile at a time and issues cta_group::2
// MMAs (M = 256 split across the two SMs, N = 256 with B split likewise),
// so each SM streams 128 rows of A and 128 rows of B per K-step for a
// 128 x 256 share of the output.
//
// Roles in each CTA (warp-specialised):
//   warps 0-7  epilogue: each warp drains 32 lanes x 128 columns of its
//              CTA's accumulator into registers (two per TMEM lane
//              quadrant), hands tensor memory back (arrivals counted in the
//              leader), then converts and stores straight from registers
//              in full 32-byte sectors while the next tile's MMAs run.
//   warp 8     TMA producer: 128B-swizzled tiles of its A rows and B rows,
//              and the scale atoms (its 128 A rows; all 256 B rows), into
//              a shared-memory ring (6 slots for MXFP4, 5 for NVFP4). All
//              copies of both CTAs complete on the LEADER CTA's ring
//              barrier.
//   warp 9     in the leader CTA the single MMA-issuing thread: tcgen05.cp
//              of the scale atoms into tensor memory (both CTAs), the MMAs,
//              and multicast tcgen05.commits that free the ring slot and
//              publish the finished accumulator in both CTAs.
//   warp 1     allocates and frees the pair's tensor memory; warps 10-11
//              only complete the control warpgroup.
// Every wait is bounded by %globaltimer; a wait that runs out sets the
// plan's status word and raises a CTA-wide abort flag; the CTA then lets
// its in-flight copies and MMAs finish, frees tensor memory and returns.
// No TMA multicast is used anywhere.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "osm_internal.h"
#include "osm_mx.cuh"
#include "osm_ptx.cuh"

namespace osm {
namespace {

constexpr int BM = 128;                 // accumulator rows per CTA (TMEM lanes); pair tile M = 256
constexpr int BN = 256;                 // output columns per tile; each CTA loads BN/2 rows of B
constexpr int A_TILE = BM * 128;        // one K-step of A: 128 rows x 128 bytes
constexpr int B_TILE = (BN / 2) * 128;  // one K-step of this CTA's half of B
constexpr int NUM_EPI_WARPS = 8;        // two per TMEM lane quadrant, 128 columns each
constexpr int CTRL_WG = 2;              // warpgroup of the producer (warp 8) and MMA issuer (warp 9)
constexpr int PRODUCER_WARP = 4 * CTRL_WG;
constexpr int MMA_WARP = PRODUCER_WARP + 1;
constexpr int NUM_THREADS = 32 * NUM_EPI_WARPS + 128;  // epilogue = warpgroups 0 and 1
// Register split. The kernel is launched with LAUNCH_REGS per thread (the
// most 384 threads may hold: a warp's registers come from one SM
// sub-partition of 16384, and each sub-partition holds three warps).
// Warpgroup 2 (producer, MMA issuer, two idle warps) then gives registers
// back and the epilogue warpgroups take them: a lane's 128 accumulators,
// 64 packed x' words and the loop state must fit in EPI_REGS.
constexpr int LAUNCH_REGS = 168;
constexpr int CTRL_REGS = 56;
constexpr int EPI_REGS = 224;
static_assert(NUM_THREADS == 384, "three warpgroups");
static_assert((LAUNCH_REGS - CTRL_REGS) * 128 >= (EPI_REGS - LAUNCH_REGS) * 256, "register split exceeds the launch");
static_assert(CTRL_REGS + 2 * EPI_REGS <= 512, "register split exceeds a sub-partition");
static_assert(LAUNCH_REGS * 3 <= 512 && CTRL_REGS % 8 == 0 && EPI_REGS % 8 == 0, "register counts");
// Each epilogue kind is its own kernel instantiation with its own register
// allocation; only the FFN requantisation needs more than LAUNCH_REGS.
__host__ __device__ constexpr bool uses_register_split(int epi) { return epi == OSM_EPI_GELU_REQUANT; }
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;       // scale factors live after the accumulator
// Tile raster. When the packed weights fit comfortably in L2 (the FFN
// projections: about 40 MB), every M-tile sweeps all N-tiles before the next
// (group of 1): all of W stays resident and each activation tile is read
// from HBM once. Larger weights use groups of GROUP_M M-tiles, which bound
// the weight bytes streamed per group.
constexpr int GROUP_M = 8;
constexpr int64_t W_RESIDENT_BYTES = 48ll << 20;
constexpr uint16_t PAIR_MASK = 0x3;

// Ring shape per 4-bit format. A slot carries one K-step of 256 FP4 values;
// its scales are 128 x 4 atoms of 512 bytes: two atoms per 128-row tile for
// MXFP4 (8 E8M0 scales per row), four for NVFP4 (16 E4M3 scales). Each atom
// is copied to four tensor-memory columns (A) or eight (B: two 128-row
// tiles). NVFP4's larger slots leave room for five in shared and tensor
// memory, MXFP4's for six.
template <bool NV>
struct Fmt {
    static constexpr int STAGES = NV ? 5 : 6;
    static constexpr int APS = NV ? 4 : 2;                // scale atoms per K-step and 128-row tile
    static constexpr int SFA_TILE = APS * 512;
    static constexpr int SFB_HALF = APS * 512;            // one 128-row tile of B
    static constexpr int SFB_TILE = 2 * SFB_HALF;
    static constexpr uint32_t SF_STAGE_COLS = 12 * APS;   // 4 columns per atom for A, 8 for B
};
static_assert(SF_COL0 + Fmt<false>::STAGES * Fmt<false>::SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");
static_assert(SF_COL0 + Fmt<true>::STAGES * Fmt<true>::SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");

// Instruction descriptors (tcgen05 instruction-descriptor format), M = 256
// over the CTA pair, N = 256.
// kind::mxf4 block-scaled: A/B E2M1 (1), K-major, N>>3 @17, UE8M0 scales
// (bit 23), M>>4 @24; scale-factor byte ids at bits 29-30 (A) and 4-5 (B).
constexpr uint32_t IDESC_MXF4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) |
                                ((uint32_t)((2 * BM) >> 4) << 24);
// kind::mxf4nvf4 with UE4M3 scales (bit 23 clear), four scales per row and
// MMA: scale-factor byte ids 0.
constexpr uint32_t IDESC_NVF4 = IDESC_MXF4 & ~(1u << 23);
// kind::f16: FP32 accumulate (bit 4), A/B BF16 (1 @7, 1 @10), K-major;
// IDESC_F16: the same with A and B binary16 (type 0 in both fields).
constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)((2 * BM) >> 4) << 24);
constexpr uint32_t IDESC_F16 = IDESC_BF16 & ~((1u << 7) | (1u << 10));

template <bool NV>
struct __align__(1024) Smem {
    static constexpr int STAGES = Fmt<NV>::STAGES;
    uint8_t a[STAGES][A_TILE];
    uint8_t b[STAGES][B_TILE];
    uint8_t sfa[STAGES][Fmt<NV>::SFA_TILE];
    uint8_t sfb[STAGES][Fmt<NV>::SFB_TILE];
    uint64_t full[STAGES];   // leader: all copies of both CTAs for the slot have landed
    uint64_t empty[STAGES];  // both: the MMAs reading the slot have completed
    uint64_t acc_full;       // both: the tile's accumulator is complete
    uint64_t acc_empty;      // leader: both CTAs' epilogues have drained the accumulator
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct GemmParams {
    CUtensorMap tm_a;    // a_codes  [M][Kbp/2] u8, box 128 x 128
    CUtensorMap tm_b;    // w_codes  [N][Kbp/2] u8, box 128 x 128
    CUtensorMap tm_ah;   // a_hp     [M][kp] bf16, box 64 x 128
    CUtensorMap tm_bh;   // w_hp     [N][kp] bf16, box 64 x 128
    CUtensorMap tm_sa;   // a_scales as [bytes/128][128] u8, box 128 x 4 (one 512-byte atom)
    CUtensorMap tm_sb;   // w_scales likewise
    const float* bias;
    void* Y;
    uint32_t* status;
    uint64_t wait_limit_ns;
    int64_t M, N;
    int katoms;      // scale atoms per 128-row tile: Kbp / 128 (MXFP4), Kbp / 64 (NVFP4)
    int n_fp4;       // K-steps of the bulk branch: ceil(Kbp / 256)
    int n_hp;        // K-steps of the outlier branch: kp / 64
    int num_m, num_n;
    int group_m;     // tile raster: groups of group_m M-tiles sweep the N-tiles (M fastest inside a group)
    int n_row_tiles; // ceil(N / 128): scale-atom rows of W
    int epi;
    uint32_t idesc_hp;        // instruction descriptor of the outlier K-steps (BF16 or FP16 operands)
    float out_scale;          // NVFP4: 2^(g_act + g_w), applied to the accumulator before the bias
    // OSM_EPI_GELU_REQUANT: the next layer's packed activations
    uint8_t* next_codes;      // [M][nKbp/2]
    uint8_t* next_scales;     // layout, rows padded to 128
    uint16_t* next_hp;        // [M][nkp]
    const float* inv_s_ord;   // next's inv_s in its [J | O] channel order (= this layer's column order)
    int nKb, nKbp, nk, nkp;   // next's bulk / outlier widths
    int next_hp_fp16;         // next's outlier slots in binary16
    int64_t m_pad;            // M rounded up to 128 (rows of next_scales)
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m, int& m_blk, int& n_blk) {
    const int group = group_m * num_n;
    const int g = tile / group;
    const int first_m = g * group_m;
    const int gm = min(num_m - first_m, group_m);
    const int local = tile % group;
    m_blk = first_m + local % gm;
    n_blk = local / gm;
}

template <class SM>
__device__ __forceinline__ void raise_abort(SM& S, uint32_t* status) {
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

// Load one 16-lane slab of the accumulator: 16 TMEM lanes x 128 columns.
// Thread t receives lanes t/4 and t/4 + 8 and, for each 8-column block j,
// columns 8j + 2(t%4) and 8j + 2(t%4) + 1 (registers 4j .. 4j+3), so the
// four lanes of a quad hold one row's 32 contiguous bytes.
__device__ __forceinline__ void tmem_ld_16x256b_x16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}
// Add the bias and store one 16-row x 128-column slab from registers: each
// store instruction of the warp writes eight full 32-byte sectors (one per
// row), FP32 as 8-byte pairs or BF16 as 4-byte pairs. Rows >= M and
// columns >= N (N % 32 == 0, so whole 8-column blocks) are skipped.
template <int EPI, bool NV>
__device__ __forceinline__ void store_slab(const GemmParams& p, int64_t row0, int64_t col0, int lane, const uint32_t* r) {
    const int64_t ra = row0 + (lane >> 2), rb = ra + 8;
    const int cq = 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int64_t col = col0 + 8 * j + cq;
        if (col >= p.N) break;
        float2 a = make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]));
        float2 b = make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        if constexpr (NV) {
            a = __fmul2_rn(a, make_float2(p.out_scale, p.out_scale));
            b = __fmul2_rn(b, make_float2(p.out_scale, p.out_scale));
        }
        if (p.bias) {
            const float2 bb = __ldg(reinterpret_cast<const float2*>(p.bias + col));
            a = __fadd2_rn(a, bb);
            b = __fadd2_rn(b, bb);
        }
        if constexpr (EPI == OSM_EPI_GELU_BF16) {
            a = mx::gelu2(a);
            b = mx::gelu2(b);
        }
        if constexpr (EPI == OSM_EPI_F32) {
            if (ra < p.M) *reinterpret_cast<float2*>(static_cast<float*>(p.Y) + ra * p.N + col) = a;
            if (rb < p.M) *reinterpret_cast<float2*>(static_cast<float*>(p.Y) + rb * p.N + col) = b;
        } else {
            if (ra < p.M) *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.Y) + ra * p.N + col) = mx::bf16x2_bits(a.x, a.y);
            if (rb < p.M) *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.Y) + rb * p.N + col) = mx::bf16x2_bits(b.x, b.y);
        }
    }
}
// Wait for this warp's tensor-memory loads, then tell the leader CTA's
// MMA warp that the accumulator may be overwritten (16 arrivals: 8 warps in
// each CTA of the pair). The only ordering this hand-off needs is that of
// the tensor-memory reads before the next tile's MMAs: tcgen05.wait::ld
// returns once the loads have completed and tcgen05.fence::before_thread_sync
// orders them before the arrival, so the arrival itself is relaxed; the
// epilogue publishes no memory that the MMA warp reads. (A release arrival
// at cluster scope waited for this lane's earlier global stores and cost
// about 0.9 us of idle tensor pipe at every tile boundary.)
__device__ __forceinline__ void release_accumulator(uint32_t acc_empty_leader, int lane) {
    ptx::tmem_ld_wait();
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive_remote_relaxed(acc_empty_leader);
}
// OSM_EPI_GELU_REQUANT for one 32-column group of one row (the lane's row),
// columns c0 .. c0+31 (c0 < N; N % 32 == 0, so all 32 are real). Column c
// of this layer is channel order[c] of the next layer, with reciprocal
// smoothing factor inv_s_ord[c]; column c < nKb is bulk position c, column
// c >= nKb is outlier slot c - nKb. h = bf16(GELU(acc)), x' = bf16(h * inv_s),
// then the bulk part is MXFP4-encoded as one block (codes 16 bytes, one scale
// byte; in a partial last block the positions >= nKb are padding, code 0)
// and the outlier part goes to next_hp. The group holding the last bulk
// position also writes the next layer's padding blocks (code 0, scale 0),
// the group holding the last column the outlier padding slots, and lanes of
// padding rows (M <= row < M rounded up to 128) write scale 0 only.
__device__ __forceinline__ void requant_group(const GemmParams& p, int64_t row, int64_t c0, const uint32_t* r) {
    const int katoms = p.nKbp >> 7;
    const bool holds_last_bulk = p.nKb > 0 && c0 <= p.nKb - 1 && p.nKb - 1 < c0 + 32;
    if (row >= p.M) {
        if (row < p.m_pad) {
            if (c0 < p.nKb) p.next_scales[mx::sf_offset(row, c0 >> 5, katoms)] = 0;
            if (holds_last_bulk)
                for (int b = (p.nKb + 31) >> 5; b < (p.nKbp >> 5); ++b) p.next_scales[mx::sf_offset(row, b, katoms)] = 0;
        }
        return;
    }
    // x' = round(bf16(GELU(acc)) * inv_s) as pairs, element 2i in the low
    // half of word i: BF16 for the bulk columns; for an FP16 outlier branch
    // of the next layer, binary16 in the columns from nKb on (the same
    // product, rounded to the other format)
    const bool f16_tail = p.next_hp_fp16 && c0 + 32 > p.nKb;  // uniform across the warp
    const int d = static_cast<int>(c0 - p.nKb);
    uint32_t hw[16];
    const float4* iv = reinterpret_cast<const float4*>(p.inv_s_ord + c0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 sv = __ldg(iv + i);
        const float2 g0 = mx::gelu2(make_float2(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1])));
        const float2 g1 = mx::gelu2(make_float2(__uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
        const uint32_t h0 = mx::bf16x2_bits(g0.x, g0.y), h1 = mx::bf16x2_bits(g1.x, g1.y);
        const float2 x0 = __fmul2_rn(make_float2(__uint_as_float(h0 << 16), __uint_as_float(h0 & 0xFFFF0000u)),
                                     make_float2(sv.x, sv.y));
        const float2 x1 = __fmul2_rn(make_float2(__uint_as_float(h1 << 16), __uint_as_float(h1 & 0xFFFF0000u)),
                                     make_float2(sv.z, sv.w));
        hw[2 * i] = mx::bf16x2_bits(x0.x, x0.y);
        hw[2 * i + 1] = mx::bf16x2_bits(x1.x, x1.y);
        if (f16_tail) {
            const int o = d + 4 * i;  // column of element 4i, relative to nKb
            const uint32_t m0 = (o >= 0 ? 0x0000FFFFu : 0u) | (o + 1 >= 0 ? 0xFFFF0000u : 0u);
            const uint32_t m1 = (o + 2 >= 0 ? 0x0000FFFFu : 0u) | (o + 3 >= 0 ? 0xFFFF0000u : 0u);
            hw[2 * i] = (hw[2 * i] & ~m0) | (mx::f16x2_bits(x0.x, x0.y) & m0);
            hw[2 * i + 1] = (hw[2 * i + 1] & ~m1) | (mx::f16x2_bits(x1.x, x1.y) & m1);
        }
    }
    if (c0 < p.nKb) {
        uint32_t bw[16];
        if (p.nKb - c0 >= 32) {  // a whole bulk block (the same for every lane of the warp)
#pragma unroll
            for (int i = 0; i < 16; ++i) bw[i] = hw[i];
        } else {                 // the last, partial block: positions >= nKb are padding (0)
            const int nreal = static_cast<int>(p.nKb - c0);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t lo = (2 * i < nreal) ? (hw[i] & 0xFFFFu) : 0u;
                const uint32_t hi = (2 * i + 1 < nreal) ? (hw[i] & 0xFFFF0000u) : 0u;
                bw[i] = lo | hi;
            }
        }
        // block maximum of |x'| by a tree of packed BF16 abs-max (sign bits cleared after)
        uint32_t t8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) t8[i] = mx::bf16x2_absmax(bw[2 * i], bw[2 * i + 1]);
#pragma unroll
        for (int i = 0; i < 4; ++i) t8[i] = mx::bf16x2_absmax(t8[2 * i], t8[2 * i + 1]);
        t8[0] = mx::bf16x2_absmax(mx::bf16x2_absmax(t8[0], t8[1]), mx::bf16x2_absmax(t8[2], t8[3]));
        const uint32_t amax = max(t8[0] & 0x7FFFu, (t8[0] >> 16) & 0x7FFFu);
        float inv;
        const int X = mx::bf16_block_exponent(amax, &inv);
        const uint4 out = make_uint4(mx::encode8_words(bw[0], bw[1], bw[2], bw[3], inv),
                                     mx::encode8_words(bw[4], bw[5], bw[6], bw[7], inv),
                                     mx::encode8_words(bw[8], bw[9], bw[10], bw[11], inv),
                                     mx::encode8_words(bw[12], bw[13], bw[14], bw[15], inv));
        *reinterpret_cast<uint4*>(p.next_codes + row * (p.nKbp >> 1) + (c0 >> 1)) = out;
        p.next_scales[mx::sf_offset(row, c0 >> 5, katoms)] = static_cast<uint8_t>(X + 127);
        if (holds_last_bulk) {
            for (int b = (p.nKb + 31) >> 5; b < (p.nKbp >> 5); ++b) {
                *reinterpret_cast<uint4*>(p.next_codes + row * (p.nKbp >> 1) + b * 16) = make_uint4(0, 0, 0, 0);
                p.next_scales[mx::sf_offset(row, b, katoms)] = 0;
            }
        }
    }
    if (c0 + 32 > p.nKb) {
        // outlier part: columns max(c0, nKb) .. c0+31 -> slots c - nKb
        uint16_t* hp = p.next_hp + row * p.nkp;
        if (c0 >= p.nKb && ((c0 - p.nKb) & 7) == 0) {
            uint4* dst = reinterpret_cast<uint4*>(hp + (c0 - p.nKb));
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(hw[4 * i], hw[4 * i + 1], hw[4 * i + 2], hw[4 * i + 3]);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (c0 + e >= p.nKb)
                    hp[c0 + e - p.nKb] = static_cast<uint16_t>((e & 1) ? (hw[e >> 1] >> 16) : (hw[e >> 1] & 0xFFFFu));
        }
        if (p.nkp > p.nk && c0 <= p.N - 1 && p.N - 1 < c0 + 32)
            for (int i = p.nk; i < p.nkp; ++i) hp[i] = 0;
    }
}

// The epilogue code for a whole 128-column strip, unrolled, does not fit
// the instruction cache; the strips are processed in a rolled loop over
// column groups instead. Registers cannot be indexed at run time, so after
// each step the accumulator array shifts down by the step's width (register
// moves) and the loop body always reads r[0 ..].
template <int STEP, int N>
__device__ __forceinline__ void shift_down(uint32_t (&r)[N]) {
#pragma unroll
    for (int j = 0; j + STEP < N; ++j) r[j] = r[j + STEP];
}

// TMA producer, one elected thread in each CTA of the pair.
template <bool NV>
__device__ __forceinline__ void producer_role(const GemmParams& p, Smem<NV>& S, uint32_t rank, bool leader, int pair,
                                              int npairs, int tiles, int ksteps, const volatile int* abort,
                                              const volatile int* never, uint64_t drain_ns) {
    if (ptx::elect_one()) {
        int stage = 0;
        uint32_t phase = 0;
        int last_stage = -1;
        uint32_t last_phase = 0;
        bool ok = true;
        for (int tile = pair; tile < tiles && ok; tile += npairs) {
            int m_blk, n_blk;
            tile_coords(tile, p.num_m, p.num_n, p.group_m, m_blk, n_blk);
            const int arow = m_blk * 2 * BM + static_cast<int>(rank) * BM;        // this CTA's A rows
            const int brow = n_blk * BN + static_cast<int>(rank) * (BN / 2);      // this CTA's B rows
            const int nbt = min(2, p.n_row_tiles - 2 * n_blk);                   // valid B scale row tiles
            const int sfa_tile = 2 * m_blk + static_cast<int>(rank);              // A scale row tile
            for (int ks = 0; ks < ksteps; ++ks) {
                if (!ptx::mbar_wait_bounded(ptx::smem_u32(&S.empty[stage]), phase ^ 1u, p.wait_limit_ns,
                                            abort)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = ptx::mapa(ptx::smem_u32(&S.full[stage]), 0);  // leader's barrier
                if (ks < p.n_fp4) {
                    constexpr int APS = Fmt<NV>::APS;
                    const int natoms = min(APS, p.katoms - APS * ks);
                    if (leader)
                        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&S.full[stage]),
                                                   2u * (A_TILE + B_TILE + natoms * 512u * (1u + nbt)));
                    ptx::tma_load_2d_pair(ptx::smem_u32(S.a[stage]), &p.tm_a, ks * 128, arow, fb);
                    ptx::tma_load_2d_pair(ptx::smem_u32(S.b[stage]), &p.tm_b, ks * 128, brow, fb);
                    for (int a = 0; a < natoms; ++a) {
                        ptx::tma_load_2d_pair(ptx::smem_u32(S.sfa[stage]) + 512 * a, &p.tm_sa, 0,
                                              (sfa_tile * p.katoms + APS * ks + a) * 4, fb);
                        for (int h = 0; h < nbt; ++h)
                            ptx::tma_load_2d_pair(ptx::smem_u32(S.sfb[stage]) + Fmt<NV>::SFB_HALF * h + 512 * a,
                                                  &p.tm_sb, 0, ((2 * n_blk + h) * p.katoms + APS * ks + a) * 4, fb);
                    }
                } else {
                    const int kh = ks - p.n_fp4;
                    if (leader)
                        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&S.full[stage]), 2u * (A_TILE + B_TILE));
                    ptx::tma_load_2d_pair(ptx::smem_u32(S.a[stage]), &p.tm_ah, kh * 64, arow, fb);
                    ptx::tma_load_2d_pair(ptx::smem_u32(S.b[stage]), &p.tm_bh, kh * 64, brow, fb);
                }
                last_stage = stage;
                last_phase = phase;
                if (++stage == Fmt<NV>::STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        if (!ok) raise_abort(S, p.status);
        // Let every copy this thread issued land before the pair exits: the
        // last slot it filled is released (empty) only after the MMAs that
        // read it completed, which implies all earlier copies completed too.
        if (last_stage >= 0) {
            if (!ptx::mbar_wait_bounded_cluster(ptx::smem_u32(&S.empty[last_stage]), last_phase, drain_ns,
                                                never))
                ptx::spin_ns(1000000);  // an aborted pipeline: give any in-flight copy ample time to land
        }
    }
}

// MMA issuer, one elected thread of the leader CTA.
template <bool NV>
__device__ __forceinline__ void mma_role(const GemmParams& p, Smem<NV>& S, bool leader, int pair, int npairs, int tiles,
                                         int ksteps, const volatile int* abort, const volatile int* never,
                                         uint64_t drain_ns, uint32_t tmem) {
    if (leader && ptx::elect_one()) {
        int stage = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        const uint32_t acc = tmem;  // lane 0, column 0
        // K-step ks of the slot `stage`: wait for its operands, then copy its
        // scale atoms into the slot's tensor-memory columns. Neither touches
        // the accumulator, so a tile's first K-step is prepared before the
        // epilogue hands the accumulator back (the copies queue behind the
        // previous tile's MMAs on the tensor pipe).
        auto prepare = [&](int ks) -> bool {
            if (!ptx::mbar_wait_bounded(ptx::smem_u32(&S.full[stage]), phase, p.wait_limit_ns, abort)) return false;
            ptx::tc_fence_after();
            if (ks < p.n_fp4) {
                constexpr int APS = Fmt<NV>::APS;
                const int natoms = min(APS, p.katoms - APS * ks);
                const uint32_t sfa_col = tmem + SF_COL0 + stage * Fmt<NV>::SF_STAGE_COLS;
                const uint32_t sfb_col = sfa_col + 4 * APS;
                const uint32_t sfa_s = ptx::smem_u32(S.sfa[stage]);
                const uint32_t sfb_s = ptx::smem_u32(S.sfb[stage]);
                for (int a = 0; a < natoms; ++a) {
                    ptx::tc_cp_32x128_x4_pair(sfa_col + 4 * a, desc_sf(sfa_s + 512 * a));
                    ptx::tc_cp_32x128_x4_pair(sfb_col + 8 * a, desc_sf(sfb_s + 512 * a));
                    ptx::tc_cp_32x128_x4_pair(sfb_col + 8 * a + 4, desc_sf(sfb_s + Fmt<NV>::SFB_HALF + 512 * a));
                }
            }
            return true;
        };
        for (int tile = pair; tile < tiles && ok; tile += npairs) {
            if (!prepare(0)) {
                ok = false;
                break;
            }
            if (!ptx::mbar_wait_bounded_cluster(ptx::smem_u32(&S.acc_empty), acc_phase ^ 1u, p.wait_limit_ns,
                                                abort)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            uint32_t accumulate = 0;
            for (int ks = 0; ks < ksteps; ++ks) {
                if (ks > 0 && !prepare(ks)) {
                    ok = false;
                    break;
                }
                const uint32_t a_base = ptx::smem_u32(S.a[stage]);
                const uint32_t b_base = ptx::smem_u32(S.b[stage]);
                if (ks < p.n_fp4) {
                    constexpr int APS = Fmt<NV>::APS;
                    const int natoms = min(APS, p.katoms - APS * ks);
                    const uint32_t sfa_col = tmem + SF_COL0 + stage * Fmt<NV>::SF_STAGE_COLS;
                    const uint32_t sfb_col = sfa_col + 4 * APS;
                    if constexpr (NV) {
                        // one atom (four 16-blocks per row) per MMA of K = 64
                        for (int kk = 0; kk < natoms; ++kk) {
                            ptx::mma_nvf4_pair(acc, desc_sw128(a_base + kk * 32), desc_sw128(b_base + kk * 32),
                                               IDESC_NVF4, sfa_col + 4 * kk, sfb_col + 8 * kk, accumulate);
                            accumulate = 1;
                        }
                    } else {
                        for (int kk = 0; kk < 2 * natoms; ++kk) {
                            const uint32_t sf_id = (uint32_t)(kk & 1) * 2u;  // bytes 0-1 or 2-3 of the atom
                            const uint32_t idesc = IDESC_MXF4 | (sf_id << 29) | (sf_id << 4);
                            ptx::mma_mxf4_pair(acc, desc_sw128(a_base + kk * 32), desc_sw128(b_base + kk * 32),
                                               idesc, sfa_col + 4 * (kk >> 1), sfb_col + 8 * (kk >> 1), accumulate);
                            accumulate = 1;
                        }
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        ptx::mma_bf16_pair(acc, desc_sw128(a_base + kk * 32), desc_sw128(b_base + kk * 32),
                                           p.idesc_hp, accumulate);
                        accumulate = 1;
                    }
                }
                ptx::tc_commit_pair_mc(ptx::smem_u32(&S.empty[stage]), PAIR_MASK);
                if (++stage == Fmt<NV>::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            ptx::tc_commit_pair_mc(ptx::smem_u32(&S.acc_full), PAIR_MASK);
            acc_phase ^= 1u;
        }
        if (!ok) raise_abort(S, p.status);
        // all issued tensor-core work has finished before tensor memory is freed
        ptx::tc_commit_pair_mc(ptx::smem_u32(&S.drain), 0x1);
        ptx::mbar_wait_bounded(ptx::smem_u32(&S.drain), 0, drain_ns, never);
    }
}

// Epilogue, warps 0..7 of both CTAs: drain the accumulator, release
// it to the MMA issuer, then convert and store.
template <int EPI, bool NV>
__device__ __forceinline__ void epilogue_role(const GemmParams& p, Smem<NV>& S, int warp, int lane, uint32_t rank,
                                              int pair, int npairs, int tiles, const volatile int* abort,
                                              uint32_t tmem) {
    const int q = warp & 3;                   // TMEM lanes 32q..32q+31 are reachable from this warp
    const int half = warp >> 2;  // columns [128*half, 128*half + 128) of the tile
    const uint32_t acc_empty_leader = ptx::mapa(ptx::smem_u32(&S.acc_empty), 0);
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < tiles; tile += npairs) {
        int m_blk, n_blk;
        tile_coords(tile, p.num_m, p.num_n, p.group_m, m_blk, n_blk);
        int ok = 1;
        if (lane == 0)
            // the accumulator completes once per tile (about 10 us of MMAs):
            // a suspending wait polls less (1-2 % on the power-capped FFN step)
            ok = ptx::mbar_wait_bounded_long(ptx::smem_u32(&S.acc_full), acc_phase, p.wait_limit_ns, abort, 20000u)
                     ? 1
                     : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) raise_abort(S, p.status);
            break;
        }
        ptx::tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + half * 128;
        const int64_t y0 = (int64_t)m_blk * 2 * BM + (int64_t)rank * BM + q * 32;
        const int64_t x0 = (int64_t)n_blk * BN + half * 128;
        if constexpr (EPI == OSM_EPI_GELU_REQUANT) {
            static_assert(!NV, "the fused requantisation takes MXFP4 operands");
            // lane = row, 32 consecutive columns per load: whole MX blocks per lane
            uint32_t r[128];
            ptx::tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            ptx::tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            ptx::tmem_ld_32x32b_x32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
            ptx::tmem_ld_32x32b_x32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
            release_accumulator(acc_empty_leader, lane);
#pragma unroll 1
            for (int g = 0; g < 4; g += 2) {
                if (x0 + 32 * g < p.N) requant_group(p, y0 + lane, x0 + 32 * g, r);
                if (x0 + 32 * g + 32 < p.N) requant_group(p, y0 + lane, x0 + 32 * g + 32, r + 32);
                shift_down<64>(r);
            }
        } else {
            // four lanes per row: full 32-byte sectors per store
            uint32_t r[128];
            tmem_ld_16x256b_x16(taddr, r);
            tmem_ld_16x256b_x16(taddr + (16u << 16), r + 64);
            release_accumulator(acc_empty_leader, lane);
            if (x0 < p.N) {
#pragma unroll 1
                for (int sl = 0; sl < 2; ++sl) {
                    store_slab<EPI, NV>(p, y0 + 16 * sl, x0, lane, r);
                    shift_down<64>(r);
                }
            }
        }
        acc_phase ^= 1u;
    }
}

// Both CTAs done (no MMA, copy or tensor-memory read in flight), then warp 1
// frees the pair's tensor memory. Lanes that skipped a single-thread role
// wait for their elected lane first.
__device__ __forceinline__ void teardown(int warp, uint32_t tmem) {
    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

template <int EPI, bool NV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    dual_gemm_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    Smem<NV>& S = *reinterpret_cast<Smem<NV>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();  // 0 = leader (issues the MMAs), 1 = peer
    const bool leader = rank == 0;
    const int pair = static_cast<int>(ptx::cluster_id_x());
    const int npairs = static_cast<int>(ptx::num_clusters_x());
    const int tiles = p.num_m * p.num_n;
    const int ksteps = p.n_fp4 + p.n_hp;
    const volatile int* abort = &S.abort_flag;
    __shared__ int never;  // a flag nothing sets: drain waits use it instead of the abort flag
    // Drains wait for work that always completes (copies, MMAs); they get a
    // generous limit even when the pipeline limit is set very short.
    const uint64_t drain_ns = p.wait_limit_ns > 200000000ull ? p.wait_limit_ns : 200000000ull;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Fmt<NV>::STAGES; ++s) {
            ptx::mbar_init(ptx::smem_u32(&S.full[s]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(&S.acc_full), 1);
        ptx::mbar_init(ptx::smem_u32(&S.acc_empty), 2 * NUM_EPI_WARPS);
        ptx::mbar_init(ptx::smem_u32(&S.drain), 1);
        S.abort_flag = 0;
        never = 0;
        ptx::fence_mbar_init();
    }
    if (warp == PRODUCER_WARP && lane == 0) {
        if (p.n_fp4) {
            ptx::prefetch_tmap(&p.tm_a);
            ptx::prefetch_tmap(&p.tm_b);
            ptx::prefetch_tmap(&p.tm_sa);
            ptx::prefetch_tmap(&p.tm_sb);
        }
        if (p.n_hp) { ptx::prefetch_tmap(&p.tm_ah); ptx::prefetch_tmap(&p.tm_bh); }
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_u32(&S.tmem_base), TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
    ptx::tc_fence_after();
    // Everything above overlaps the tail of the previous kernel on the stream
    // (a dependent launch); operands and outputs are touched only after it.
    ptx::grid_dep_wait();
    ptx::grid_dep_launch();
    const uint32_t tmem = S.tmem_base;
    // Warpgroup-uniform register split (for the epilogues that need it). Each
    // side ends with its own copy of the teardown, so that no code is shared
    // between the two budgets.
    if (warp >= PRODUCER_WARP) {
        if constexpr (uses_register_split(EPI)) ptx::setmaxnreg_dec<CTRL_REGS>();
        if (warp == PRODUCER_WARP) producer_role(p, S, rank, leader, pair, npairs, tiles, ksteps, abort, &never, drain_ns);
        else if (warp == MMA_WARP) mma_role(p, S, leader, pair, npairs, tiles, ksteps, abort, &never, drain_ns, tmem);
        teardown(warp, tmem);
    } else {
        if constexpr (uses_register_split(EPI)) ptx::setmaxnreg_inc<EPI_REGS>();
        epilogue_role<EPI, NV>(p, S, warp, lane, rank, pair, npairs, tiles, abort, tmem);
        teardown(warp, tmem);
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
             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz,
             const char* what) {
    auto enc = get_encode_fn();
    if (!enc) return fail(OSM_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(OSM_ERR_CUDA, "tensor map for %s: CUresult %d", what, (int)r);
    return OSM_OK;
}

struct LaunchInfo {
    int max_pairs = 0;
    bool ready = false;
};

// The epilogues' GELU routine applied element-wise (a test hook for its
// accuracy): y[i] = GELU(x[i]) exactly as the FFN epilogues compute it.
__global__ void gelu_f32_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x * 2) {
        const float2 v = mx::gelu2(make_float2(x[i], i + 1 < n ? x[i + 1] : 0.0f));
        y[i] = v.x;
        if (i + 1 < n) y[i + 1] = v.y;
    }
}

}  // namespace


int launch_gelu_f32(const float* x, float* y, int64_t n, cudaStream_t st) {
    const int64_t blocks = std::min<int64_t>((n + 511) / 512, 148 * 8);
    gelu_f32_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(x, y, n);
    return check_cuda(cudaGetLastError(), "gelu_f32 launch");
}

int launch_dual_gemm(const osm_plan* pl, const uint8_t* a_codes, const uint8_t* a_scales, const uint16_t* a_hp,
                     int64_t M, const uint8_t* w_codes, const uint8_t* w_scales, const uint16_t* w_hp,
                     const float* bias, int epi, void* Y, const osm_plan* next, uint8_t* next_codes,
                     uint8_t* next_scales, uint16_t* next_hp, cudaStream_t st) {
    static_assert(sizeof(Smem<false>) + 1024 <= 232448 && sizeof(Smem<true>) + 1024 <= 232448,
                  "shared memory budget");
    const bool nv = pl->fmt == OSM_FMT_NVFP4;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    int rc;
    const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B, NOSW = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (pl->Kbp > 0) {
        if ((rc = make_map(&p.tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, pl->Kbp / 2, M, pl->Kbp / 2, 128, BM, SW,
                           "a_codes")))
            return rc;
        if ((rc = make_map(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, pl->Kbp / 2, pl->N, pl->Kbp / 2, 128,
                           BN / 2, SW, "w_codes")))
            return rc;
        // scale atoms are contiguous 512-byte runs: view them as 128-byte rows so
        // that one atom is four wide TMA requests rather than 32 narrow ones
        const uint64_t sa_rows = static_cast<uint64_t>(scales_bytes(M, pl->Kbp, pl->fmt)) / 128;
        const uint64_t sb_rows = static_cast<uint64_t>(scales_bytes(pl->N, pl->Kbp, pl->fmt)) / 128;
        if ((rc = make_map(&p.tm_sa, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_scales, 128, sa_rows, 128, 128, 4, NOSW,
                           "a_scales")))
            return rc;
        if ((rc = make_map(&p.tm_sb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_scales, 128, sb_rows, 128, 128, 4, NOSW,
                           "w_scales")))
            return rc;
    }
    if (pl->kp > 0) {
        const CUtensorMapDataType hpt = pl->hp_fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        if ((rc = make_map(&p.tm_ah, hpt, a_hp, pl->kp, M, pl->kp * 2, 64, BM, SW,
                           "a_hp")))
            return rc;
        if ((rc = make_map(&p.tm_bh, hpt, w_hp, pl->kp, pl->N, pl->kp * 2, 64, BN / 2,
                           SW, "w_hp")))
            return rc;
    }
    p.bias = bias;
    p.Y = Y;
    p.status = pl->d_status;
    p.wait_limit_ns = pl->wait_limit_ns;
    p.M = M;
    p.N = pl->N;
    p.katoms = static_cast<int>(pl->Kbp / (4 * block_elems(pl->fmt)));
    p.n_fp4 = static_cast<int>(ceil_div(pl->Kbp, 256));
    p.n_hp = static_cast<int>(pl->kp / 64);
    p.num_m = static_cast<int>(ceil_div(M, 2 * BM));
    p.num_n = static_cast<int>(ceil_div(pl->N, BN));
    {
        size_t wc = 0, ws = 0, wh = 0;
        osm_plan_sizes(pl, pl->N, &wc, &ws, &wh);
        p.group_m = static_cast<int64_t>(wc + ws + wh) <= W_RESIDENT_BYTES ? 1 : GROUP_M;
    }
    p.n_row_tiles = static_cast<int>(ceil_div(pl->N, 128));
    p.epi = epi;
    p.idesc_hp = pl->hp_fp16 ? IDESC_F16 : IDESC_BF16;
    p.out_scale = nv ? pow2f(pl->g_act + pl->g_w) : 1.0f;
    if (epi == OSM_EPI_GELU_REQUANT) {
        p.next_codes = next_codes;
        p.next_scales = next_scales;
        p.next_hp = next_hp;
        p.inv_s_ord = next->d_inv_s_ord;
        p.nKb = static_cast<int>(next->Kb);
        p.nKbp = static_cast<int>(next->Kbp);
        p.nk = static_cast<int>(next->k);
        p.nkp = static_cast<int>(next->kp);
        p.m_pad = round_up(M, 128);
        p.next_hp_fp16 = next->hp_fp16;
    }

    void (*kernel)(GemmParams) = nullptr;
    switch (epi) {
        case OSM_EPI_F32:
            kernel = nv ? dual_gemm_kernel<OSM_EPI_F32, true> : dual_gemm_kernel<OSM_EPI_F32, false>;
            break;
        case OSM_EPI_BF16:
            kernel = nv ? dual_gemm_kernel<OSM_EPI_BF16, true> : dual_gemm_kernel<OSM_EPI_BF16, false>;
            break;
        case OSM_EPI_GELU_REQUANT:
            if (nv) return fail(OSM_ERR_UNSUPPORTED, "dual_gemm: GELU_REQUANT takes MXFP4 operands");
            kernel = dual_gemm_kernel<OSM_EPI_GELU_REQUANT, false>;
            break;
        case OSM_EPI_GELU_BF16:
            kernel = nv ? dual_gemm_kernel<OSM_EPI_GELU_BF16, true> : dual_gemm_kernel<OSM_EPI_GELU_BF16, false>;
            break;
        default: return fail(OSM_ERR_INVALID_ARG, "dual_gemm: epilogue %d", epi);
    }

    // co-resident clusters of two CTAs, queried once per device and epilogue
    static LaunchInfo info[64][8];
    static std::mutex mu;
    int dev = 0;
    if ((rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice"))) return rc;
    if (dev < 0 || dev >= 64) return fail(OSM_ERR_UNSUPPORTED, "device index %d", dev);
    const size_t smem = (nv ? sizeof(Smem<true>) : sizeof(Smem<false>)) + 1024;
    LaunchInfo& li = info[dev][2 * epi + (nv ? 1 : 0)];
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!li.ready) {
            // The register split assumes the launch gives every thread exactly
            // LAUNCH_REGS: with fewer, the epilogue's increase could never be met.
            cudaFuncAttributes fa;
            if ((rc = check_cuda(cudaFuncGetAttributes(&fa, kernel), "dual_gemm attributes"))) return rc;
            if (uses_register_split(epi) && fa.numRegs != LAUNCH_REGS)
                return fail(OSM_ERR_UNSUPPORTED, "dual_gemm: built with %d registers per thread, the split needs %d",
                            fa.numRegs, LAUNCH_REGS);
            if ((rc = check_cuda(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(smem)),
                                 "dual_gemm smem attribute")))
                return rc;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2, 1, 1);
            cfg.blockDim = dim3(NUM_THREADS, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if ((rc = check_cuda(cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg),
                                 "dual_gemm cluster occupancy")))
                return rc;
            if (clusters < 1) return fail(OSM_ERR_UNSUPPORTED, "dual_gemm: no CTA pair fits on this device");
            li.max_pairs = clusters;
            li.ready = true;
        }
    }
    const int64_t tiles = (int64_t)p.num_m * p.num_n;
    if (tiles > 0x7FFFFFFF) return fail(OSM_ERR_UNSUPPORTED, "dual_gemm: too many tiles");
    const int pairs = static_cast<int>(tiles < li.max_pairs ? tiles : li.max_pairs);
    // a dependent launch: the prologue may run while the previous kernel on
    // the stream (normally quantize_act) finishes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return check_cuda(cudaLaunchKernelEx(&cfg, kernel, p), "dual_gemm launch");
}

}  // namespace osm
