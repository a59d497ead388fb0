// gemm_mx.cu -- persistent grouped GEMM on MXFP8 operands with the
// block-scaled 5th-generation tensor-core MMA (tcgen05.mma kind::mxf8f6f4
// .block_scale): C[rows of one expert, :] = A[rows, K] * B_e[:, K]^T where A
// and B hold E4M3 codes (K-major) and every 32 consecutive K elements of a
// row share one E8M0 scale. The tensor core applies the scales; C is fp32 in
// tensor memory (TMEM).
//
// The pages' low-precision expert pipeline ("Current Bug: CuTeDSLMoERunner
// produces wrong output") broke on the layout of the per-expert activation
// scales: padded 128-row scale blocks per expert did not match the
// contiguous expert offsets the GEMM indexes by. Here the scales of each
// 128-row x 128-element tile are stored as one 512-byte atom in the order the
// tensor core wants (mxfp8.cuh), keyed for activations by the m-tile's index
// in the device-built tile list (the kernels that produce x's and h's scales
// place them there) and for weights by row / 128. Expert segments stay
// contiguous and unpadded, tiles start at any row, and a stage's scales
// arrive with one 512-byte bulk copy per operand.
//
// Structure (one CTA per SM, 192 threads), as in gemm_tc.cu:
//   warp 0     producer (one thread): TMA of the 128 x 128-byte A and B code
//              tiles (128-byte swizzle) and bulk copies of their two scale
//              atoms, all completing on the stage's barrier; STAGES-deep ring
//   warp 1     allocates TMEM (two 128-column accumulators + the scale
//              columns); one thread copies the stage's scales into TMEM
//              (tcgen05.cp 32x128b.warpx4) and issues four M=128 N=128 K=32
//              block-scaled MMAs, selecting the scale byte of each K step in
//              the instruction descriptor
//   warps 2-5  epilogue: SwiGLU followed by MXFP8 quantization of h (each
//              thread holds one 32-column block of its row, so the block
//              maximum needs no exchange), or the routing-weighted scatter-add,
//              or a plain fp32 store
// Tensor-core copies and MMAs issued by one thread execute in order. Each
// ring stage has its own 8 TMEM scale columns (after the 256 accumulator
// columns), so a stage's copy never waits for the previous stage's MMAs to
// finish reading; a stage's columns are rewritten only after its MMAs have
// committed (the producer refills its buffers only then).
//
// NVFP4 operands (FMT_NV4, nvfp4.cuh) run on the same engine with
// tcgen05.mma kind::mxf4nvf4 .block_scale.scale_vec::4X: packed E2M1 codes
// (a 128-byte K stage holds 256 elements), one E4M3 scale per 16 elements, so
// a stage brings four 512-byte scale atoms per operand (one 2 KB bulk copy),
// owns 32 TMEM scale columns, and issues four M=128 N=128 K=64 MMAs, each
// reading a whole 32-bit scale word per row. The epilogue multiplies the
// accumulators by 1 / (gs_A * gs_B[expert]) (the two global encode scales).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "mxfp8.cuh"
#include "nvfp4.cuh"
#include "tiles.cuh"

namespace moe {

#ifndef MOE_GM_MX_W13
#define MOE_GM_MX_W13 32
#endif
#ifndef MOE_GM_MX_W2
#define MOE_GM_MX_W2 16
#endif

struct MxArgs {
    int kblocks;            // K stages (K / 128 E4M3 or K / 256 E2M1 elements)
    int n_tiles;
    int group_m;
    // band order over the routed list (band_coords); NULL: plain bands
    const int32_t *mt_first;
    int n_groups;
    int band_g;
    int b_rows_per_group;
    const int32_t *mt_row0;
    const int32_t *mt_group;
    const int32_t *num_mt_dev;
    int num_mt_host;
    const int32_t *seg_offsets;
    long long rows_valid;
    const uint8_t *A_sf;
    const uint8_t *B_sf;
    void *out;
    long long ldo;
    uint8_t *out_sf;
    const int32_t *perm_token;
    const int32_t *slot_pos;
    const float *topk_w;
    int k;
    const float *perm_w;
    uint32_t *status;
    const float *b_gs;        // NVFP4: B's global encode scale per group
    float a_gs, out_gs;       // NVFP4: A's global encode scale; h's (EPI_SWIGLU_MX)
};

template <int FMT>
struct MxCfg {
    static constexpr int BM = 128, BN = 128;
    static constexpr int BK_BYTES = 128;                  // one K stage: 128 bytes per row
    static constexpr int BK = FMT == FMT_NV4 ? 256 : 128; // ... = 256 E2M1 or 128 E4M3 elements
    static constexpr int A_BYTES = BM * BK_BYTES;
    static constexpr int B_BYTES = BN * BK_BYTES;
    static constexpr int SF_ATOMS = FMT == FMT_NV4 ? 4 : 1;   // K groups (512-byte atoms) per stage
    // per stage: B's scale atoms; A's scales in the activation layout for
    // NVFP4 (two 4 KB tcgen05.cp 128x256b sources, nvfp4.cuh), else atoms
    static constexpr int SFB_BYTES = 512 * SF_ATOMS;
    static constexpr int SFA_BYTES = FMT == FMT_NV4 ? 8192 : 512;
    static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
    static constexpr int STAGES = FMT == FMT_NV4 ? 5 : 6;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_COL = 2 * BN;                 // scale columns after the accumulators
    static constexpr int SF_COLS_PER_STAGE = 8 * SF_ATOMS; // 4 per K group, A's then B's
    static constexpr int SMEM_BYTES =
        1024 + STAGES * (A_BYTES + B_BYTES) + STAGES * SF_STAGE_BYTES + 256;
    static_assert(SF_COL + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS,
                  "accumulators and per-stage scale columns must fit the TMEM allocation");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ void mx_tile_coords(long long tile, int num_mt, int n_tiles,
                                               int group_m, int &m_idx, int &n_idx)
{
    const long long band_size = (long long)group_m * n_tiles;
    const int band = (int)(tile / band_size);
    const int first_m = band * group_m;
    const int rows = min(group_m, num_mt - first_m);
    const int r = (int)(tile - (long long)band * band_size);
    m_idx = first_m + r % rows;
    n_idx = r / rows;
}

__device__ __forceinline__ void mx_coords(const MxArgs &p, long long tile, int num_mt, int &m_idx,
                                          int &n_idx)
{
    if (p.mt_first)
        band_coords(tile, num_mt, p.n_tiles, p.band_g, kBlockM, p.mt_first, p.n_groups, p.mt_group,
                    p.seg_offsets, m_idx, n_idx);
    else
        mx_tile_coords(tile, num_mt, p.n_tiles, p.group_m, m_idx, n_idx);
}

// Shared-memory descriptor of one 32-row x 16-byte scale atom (no swizzle:
// 8-row core matrices of 16-byte rows, 128 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(16u >> 4) << 16;    // leading byte offset (a single 16-byte column)
    d |= (uint64_t)(128u >> 4) << 32;   // stride byte offset: next 8 rows
    d |= (uint64_t)1 << 46;             // descriptor version
    return d;                           // layout type 0: no swizzle
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: E4M3 A and B
// (format 0), K-major, E8M0 scales, fp32 D, M = 128, N = 128; `sf_id` picks
// the scale byte (K block) of each 32-bit TMEM scale word for A and B.
__device__ __forceinline__ uint32_t idesc_mx(uint32_t sf_id)
{
    return (sf_id << 4)                      // B scale factor id
           | (1u << 23)                      // scale format: E8M0
           | ((uint32_t)(128 >> 3) << 17)    // N = 128
           | ((uint32_t)(128 >> 4) << 24)    // M = 128
           | (sf_id << 29);                  // A scale factor id
}

// Instruction descriptor, kind::mxf4nvf4 block-scaled with 16-element
// blocks: E2M1 A and B (format 1), K-major, E4M3 scales (scale format 0),
// fp32 D, M = 128, N = 128, dense K = 64; each MMA reads a whole 32-bit
// scale word (four blocks) per row, so the scale ids stay 0.
__device__ __forceinline__ uint32_t idesc_nv4()
{
    return (1u << 7) | (1u << 10)            // A and B: E2M1
           | ((uint32_t)(128 >> 3) << 17)    // N = 128
           | ((uint32_t)(128 >> 4) << 24);   // M = 128
}

// Shared-memory descriptor of one 4 KB activation-scale copy source
// (nvfp4.cuh nv_sfa_offset): 128 lane rows of two 16-byte chunks, the first
// chunks of all rows (2 KB) before the second ones; no swizzle, 8-row core
// matrices 128 bytes apart, the two chunk columns 2 KB apart.
__device__ __forceinline__ uint64_t smem_desc_sfa(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(2048u >> 4) << 16;   // leading byte offset: the second 16-byte chunk
    d |= (uint64_t)(128u >> 4) << 32;    // stride byte offset: next 8 rows
    d |= (uint64_t)1 << 46;              // descriptor version
    return d;                            // layout type 0: no swizzle
}

// 128 lanes x 256 bits (eight TMEM columns) from a shared-memory source, no
// replication over the lane quarters.
__device__ __forceinline__ void tc_cp_sf_128x256(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
                 : "memory");
}

__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ void tc_mma_nv4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

template <int MODE, int FMT>
__device__ __forceinline__ void mx_epilogue(const MxArgs &p, uint32_t tb, long long row,
                                            bool valid, int n_idx, int m_idx, int m, float alpha)
{
    constexpr int BN = 128;
    if (MODE == EPI_SWIGLU_MX && FMT == FMT_NV4) {
        // h columns n_idx*64 .. +63: 32 bytes of packed codes per row, two
        // 16-element blocks (and scales) per 32-column chunk
        uint8_t *hq = static_cast<uint8_t *>(p.out) + row * (p.ldo / 2) + n_idx * 32;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            float g[32], u[32];
            tmem_ld32(tb + c * 32, g);
            tmem_ld32(tb + 64 + c * 32, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
                g[i] = silu_mul(g[i] * alpha, u[i] * alpha);
            uint2 q0, q1;
            const uint32_t s0 = nv_quantize16(g, p.out_gs, q0);
            const uint32_t s1 = nv_quantize16(g + 16, p.out_gs, q1);
            if (valid) {
                *reinterpret_cast<uint4 *>(hq + c * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
                // blocks 4 n_idx + 2c and + 1: adjacent bytes of one atom word
                *reinterpret_cast<uint16_t *>(p.out_sf +
                                              nv_sfa_offset(m_idx, m, 4 * n_idx + 2 * c, (int)p.ldo)) =
                    (uint16_t)(s0 | (s1 << 8));
            }
        }
    } else if (MODE == EPI_SWIGLU_MX) {
        // columns [0,64) = gate, [64,128) = up of h columns n_idx*64 ..
        uint8_t *hq = static_cast<uint8_t *>(p.out) + row * p.ldo + n_idx * 64;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            float g[32], u[32];
            tmem_ld32(tb + c * 32, g);
            tmem_ld32(tb + 64 + c * 32, u);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
                g[i] = silu_mul(g[i], u[i]);
            uint32_t q[8];
            const uint8_t sc = mx_quantize32(g, q);
            if (valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(hq + c * 32);
                dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
                dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
                // h's scales in the atom layout of this m-tile (K of h = ldo)
                p.out_sf[sf_atom_offset(m_idx, m, 2 * n_idx + c, (int)p.ldo)] = sc;
            }
        }
    } else if (MODE == EPI_COMBINE) {
        int t = 0;
        float wgt = 0.f;
        if (valid) {
            t = p.perm_token[row];
            if (p.perm_w) {
                wgt = p.perm_w[row];
            } else {
                for (int j = 0; j < p.k; ++j)
                    if (p.slot_pos[(long long)t * p.k + j] == row)
                        wgt = p.topk_w[(long long)t * p.k + j];
            }
            wgt *= alpha;
        }
        float *o = static_cast<float *>(p.out) + (long long)t * p.ldo + n_idx * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (valid) {
                float4 *dst = reinterpret_cast<float4 *>(o + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    atomicAdd(dst + i, make_float4(wgt * v[4 * i], wgt * v[4 * i + 1],
                                                   wgt * v[4 * i + 2], wgt * v[4 * i + 3]));
            }
        }
    } else {   // EPI_STORE_F32
        float *o = static_cast<float *>(p.out) + row * p.ldo + n_idx * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (valid) {
                float4 *dst = reinterpret_cast<float4 *>(o + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(alpha * v[4 * i], alpha * v[4 * i + 1],
                                         alpha * v[4 * i + 2], alpha * v[4 * i + 3]);
            }
        }
    }
}

template <int MODE, int FMT>
__global__ void __launch_bounds__(192, 1)
    k_gemm_mx(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const MxArgs p)
{
    using C = MxCfg<FMT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + C::STAGES * C::A_BYTES;
    uint8_t *sSF = sB + C::STAGES * C::B_BYTES;   // per stage: A's scale atoms, then B's
    uint64_t *full = reinterpret_cast<uint64_t *>(sSF + C::STAGES * C::SF_STAGE_BYTES);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_mt = p.num_mt_dev ? *p.num_mt_dev : p.num_mt_host;
    const long long total = (long long)num_mt * p.n_tiles;

    if (warp == 0) {
        if (lane == 0) {   // ---------------- producer
            uint32_t it = 0;
            bool ok = true;
            for (long long tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                int m_idx, n_idx;
                mx_coords(p, tile, num_mt, m_idx, n_idx);
                const long long row0 = p.mt_row0 ? p.mt_row0[m_idx] : (long long)m_idx * C::BM;
                const int grp = p.mt_group ? (p.mt_group[m_idx] & ~kHalfTileBit) : 0;
                const long long brow = (long long)grp * p.b_rows_per_group + (long long)n_idx * C::BN;
                // a 128-row band's scales: kblocks stages of SFA / SFB bytes each
                const uint8_t *sfa = p.A_sf + (long long)m_idx * p.kblocks * C::SFA_BYTES;
                const uint8_t *sfb = p.B_sf + (brow >> 7) * p.kblocks * C::SFB_BYTES;
                for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sf = sSF + s * C::SF_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES + C::SF_STAGE_BYTES);
                    tma_load_2d(sA + s * C::A_BYTES, &tmA, kb * C::BK_BYTES, (int)row0, &full[s]);
                    tma_load_2d(sB + s * C::B_BYTES, &tmB, kb * C::BK_BYTES, (int)brow, &full[s]);
                    bulk_load(sf, sfa + (long long)kb * C::SFA_BYTES, C::SFA_BYTES, &full[s]);
                    bulk_load(sf + C::SFA_BYTES, sfb + (long long)kb * C::SFB_BYTES, C::SFB_BYTES,
                              &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {   // ---------------- MMA issuer
            uint32_t it = 0, local = 0;
            for (long long tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
                const uint32_t b = local & 1u, aph = (local >> 1) & 1u;
                if (!mbar_wait(&tempty[b], aph ^ 1u, abort_flag, p.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * C::BN;
                bool ok = true;
                for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf0 = smem_u32(sSF + s * C::SF_STAGE_BYTES);
                    // each stage has its own scale columns: the copy for this
                    // stage never overwrites columns that earlier MMAs still read
                    const uint32_t sf_a = tmem_base + C::SF_COL + s * C::SF_COLS_PER_STAGE;
                    const uint32_t sf_b = sf_a + 4 * C::SF_ATOMS;
                    if constexpr (FMT == FMT_NV4) {
                        // A: two 128x256b copies, K groups 2h and 2h + 1 in the
                        // 4-column slots sf_a + 8h and sf_a + 8h + 4 (each lane
                        // quarter reads its own column of a slot)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tc_cp_sf_128x256(sf_a + 8 * h, smem_desc_sfa(sf0 + 4096 * h));
                    } else {
                        tc_cp_sf(sf_a, smem_desc_sf(sf0));
                    }
#pragma unroll
                    for (int i = 0; i < C::SF_ATOMS; ++i)
                        tc_cp_sf(sf_b + 4 * i, smem_desc_sf(sf0 + C::SFA_BYTES + 512 * i));
                    const uint32_t a0 = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + s * C::B_BYTES);
                    // four MMAs of 32 bytes of K each (K = 32 E4M3 or 64 E2M1)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        if constexpr (FMT == FMT_NV4)
                            tc_mma_nv4(d_tmem, smem_desc_k128(a0 + kk * 32),
                                       smem_desc_k128(b0 + kk * 32), idesc_nv4(), sf_a + 4 * kk,
                                       sf_b + 4 * kk, (kb | kk) != 0);
                        else
                            tc_mma_mx(d_tmem, smem_desc_k128(a0 + kk * 32),
                                      smem_desc_k128(b0 + kk * 32), idesc_mx(kk), sf_a, sf_b,
                                      (kb | kk) != 0);
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok)
                    break;
                tc_commit(&tfull[b]);
            }
        }
    } else {   // ---------------- epilogue warps 2..5
        const int q = warp & 3;
        uint32_t local = 0;
        for (long long tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
            int m_idx, n_idx;
            mx_coords(p, tile, num_mt, m_idx, n_idx);
            const long long row0 = p.mt_row0 ? p.mt_row0[m_idx] : (long long)m_idx * C::BM;
            const int grp = p.mt_group ? (p.mt_group[m_idx] & ~kHalfTileBit) : 0;
            const long long row_end = p.seg_offsets ? p.seg_offsets[grp + 1] : p.rows_valid;
            const uint32_t b = local & 1u, aph = (local >> 1) & 1u;
            if (!mbar_wait(&tfull[b], aph, abort_flag, p.status))
                break;
            tc_fence_after();
            const long long row = row0 + q * 32 + lane;
            const bool valid = row < row_end;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * C::BN;
            const float alpha = FMT == FMT_NV4 ? 1.0f / (p.a_gs * p.b_gs[grp]) : 1.0f;
            mx_epilogue<MODE, FMT>(p, tb, row, valid, n_idx, m_idx, q * 32 + lane, alpha);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&tempty[b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_mx()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Row-major byte matrix [rows, cols] as a 2-D TMA tensor; box 128 x 128 bytes,
// 128-byte swizzle, zero fill out of bounds.
static int make_tmap_u8(CUtensorMap *m, const void *base, long long cols, long long rows)
{
    auto fn = encode_fn_mx();
    if (!fn)
        return MOE_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {128u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Byte matrix [rows, cols] as a 2-D TMA tensor with a 128-byte-swizzled box
// of 128 bytes x box_rows (the operand layout of the block-scaled MMAs).
int make_tmap_u8_sw128(CUtensorMap *m, const void *base, long long cols, long long rows,
                       int box_rows)
{
    auto fn = encode_fn_mx();
    if (!fn)
        return MOE_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Byte matrix [rows, cols] as a 2-D TMA tensor with an unswizzled box of
// 128 bytes x box_rows (rows land 128 bytes apart in shared memory), for
// kernels that read the tile with CUDA cores.
int make_tmap_u8_rows(CUtensorMap *m, const void *base, long long cols, long long rows,
                      int box_rows)
{
    auto fn = encode_fn_mx();
    if (!fn)
        return MOE_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

template <int MODE, int FMT>
static int launch_mx_impl(const GemmArgs &g, cudaStream_t st)
{
    using C = MxCfg<FMT>;
    if (g.K % C::BK != 0 || g.N % C::BN != 0)
        return MOE_ERR_INVALID_ARG;
    if (FMT == FMT_NV4 && !g.b_gs)
        return MOE_ERR_INVALID_ARG;
    // code rows are K bytes (E4M3) or K / 2 bytes (packed E2M1)
    const long long row_bytes = FMT == FMT_NV4 ? g.K / 2 : g.K;
    CUtensorMap tA, tB;
    int rc = make_tmap_u8(&tA, g.Aq, row_bytes, g.a_rows);
    if (rc)
        return rc;
    rc = make_tmap_u8(&tB, g.Bq, row_bytes, g.b_rows_total);
    if (rc)
        return rc;
    MxArgs p;
    std::memset(&p, 0, sizeof p);
    p.kblocks = g.K / C::BK;
    p.n_tiles = g.N / C::BN;
    p.group_m = (MODE == EPI_SWIGLU_MX) ? MOE_GM_MX_W13 : MOE_GM_MX_W2;
    // bands hold at most 48 MiB of activation codes
    p.mt_first = g.mt_row0 ? g.mt_first : nullptr;
    p.n_groups = g.n_groups;
    p.band_g = (int)std::min<long long>(
        std::max<long long>((48LL << 20) / std::max(128 * row_bytes, 1LL), 1), 1 << 20);
    p.b_rows_per_group = g.b_rows_per_group;
    p.mt_row0 = g.mt_row0;
    p.mt_group = g.mt_group;
    p.num_mt_dev = g.num_mt_dev;
    p.num_mt_host = g.num_mt_host;
    p.seg_offsets = g.seg_offsets;
    p.rows_valid = g.rows_valid;
    p.A_sf = g.A_sf;
    p.B_sf = g.B_sf;
    p.out = g.out;
    p.ldo = g.ldo;
    p.out_sf = g.out_sf;
    p.perm_token = g.perm_token;
    p.slot_pos = g.slot_pos;
    p.topk_w = g.topk_w;
    p.k = g.k;
    p.perm_w = g.perm_w;
    p.status = g.status;
    p.b_gs = g.b_gs;
    p.a_gs = g.a_gs;
    p.out_gs = g.out_gs;

    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(k_gemm_mx<MODE, FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = 1;
    }
    const int max_mt = g.num_mt_dev ? g.max_mt : g.num_mt_host;
    const long long tiles = (long long)max_mt * p.n_tiles;
    if (tiles <= 0)
        return MOE_OK;
    const int grid = (int)std::min<long long>(tiles, num_sms());
    k_gemm_mx<MODE, FMT><<<grid, 192, C::SMEM_BYTES, st>>>(tA, tB, p);
    return launched();
}

int launch_gemm_mx(const GemmArgs &g, cudaStream_t st)
{
    if (g.fmt == FMT_NV4) {
        switch (g.mode) {
        case EPI_SWIGLU_MX: return launch_mx_impl<EPI_SWIGLU_MX, FMT_NV4>(g, st);
        case EPI_COMBINE: return launch_mx_impl<EPI_COMBINE, FMT_NV4>(g, st);
        case EPI_STORE_F32: return launch_mx_impl<EPI_STORE_F32, FMT_NV4>(g, st);
        default: return MOE_ERR_INVALID_ARG;
        }
    }
    switch (g.mode) {
    case EPI_SWIGLU_MX: return launch_mx_impl<EPI_SWIGLU_MX, FMT_MX8>(g, st);
    case EPI_COMBINE: return launch_mx_impl<EPI_COMBINE, FMT_MX8>(g, st);
    case EPI_STORE_F32: return launch_mx_impl<EPI_STORE_F32, FMT_MX8>(g, st);
    default: return MOE_ERR_INVALID_ARG;
    }
}

} // namespace moe
