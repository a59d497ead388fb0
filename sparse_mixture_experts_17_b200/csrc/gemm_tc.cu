// gemm_tc.cu -- persistent grouped GEMM on the 5th-generation tensor cores.
//
// C[rows of one expert, :] = A[rows, K] * B_e[:, K]^T with A, B bf16 K-major,
// fp32 accumulation in tensor memory (TMEM), and one of four fused
// epilogues (EpiMode): the SwiGLU of the w1/w3 GEMM ("Expert FFN" on
// "MoE Model Architectures"), the routing-weighted scatter-add of the w2 GEMM
// ("Sparse MoE Block": scale by the routing weight and index_add into token
// order), a plain fp32 store, and the router logits with bias.
//
// Structure (one CTA per SM, 192 threads):
//   warp 0     TMA producer: 128 x 64 A tile + BN x 64 B tile per stage,
//              128-byte swizzle, STAGES-deep ring of shared-memory buffers
//   warp 1     allocates 2*BN TMEM columns; one thread issues
//              tcgen05.mma (M=128, N=BN, K=16) x4 per stage, commits the
//              stage back to the producer and the finished accumulator to
//              the epilogue
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (each warp owns the
//              32 TMEM lanes = tile rows of its lane quarter), fused math,
//              global stores / fp32 vector atomics
// Two TMEM accumulators alternate so the epilogue of tile i overlaps the
// main loop of tile i+1. Tiles never mix experts: the m-tile list (built on
// the device from the expert offsets) gives each 128-row tile one expert; rows
// past the expert's end are computed and discarded by the epilogue.
// Every CTA fetches its own tiles; no copy is shared across CTAs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tiles.cuh"

namespace moe {

// Rasterisation bands (m-tiles per band) of the grouped GEMMs.
#ifndef MOE_GM_1SM_W13
#define MOE_GM_1SM_W13 32
#endif
#ifndef MOE_GM_1SM_W2
#define MOE_GM_1SM_W2 16
#endif
#ifndef MOE_GM_2SM_W13
#define MOE_GM_2SM_W13 16
#endif
#ifndef MOE_GM_2SM_W2
#define MOE_GM_2SM_W2 8
#endif

struct TcArgs {
    int kblocks;
    int n_tiles;
    int group_m;
    // band order over a routed list (band_coords); mt_first NULL: plain bands
    // of group_m m-tiles
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
    void *out;
    long long ldo;
    const int32_t *perm_token;
    const int32_t *slot_pos;
    const float *topk_w;
    int k;
    const float *perm_w;
    const float *bias;
    int n_valid;
    uint32_t *status;
    int32_t *route_idx;
    float *route_w;
    int32_t *counter_zero;
    void *out2;
    const uint16_t *gu;
    float *row_dot;
    const int32_t *grp_kb0;
    const int32_t *grp_nkb;
    long long out_group_stride;
    int32_t *hist_chunk, *hist_rank, *hist_counter, *hist_counts, *hist_offsets, *hist_n_kept;
    int32_t *hist_mt_row0, *hist_mt_group, *hist_num_mt, *hist_mt2_row0, *hist_mt2_group,
        *hist_num_mt2, *hist_mt_first, *hist_mt2_first;
    int capacity;
    // bound of every pipeline wait; `starve` (test only): the producer issues
    // no loads, so the first wait on a full stage runs out and every role unwinds
    unsigned long long wait_ns;
    int starve;
};

// Shared memory of the histogram folded into the router (E <= 64): per-warp
// lane masks and prefixes of one 128-token tile, then the last CTA's scan.
struct RouterHistSmem {
    uint32_t mask[4][64];
    int wpre[4][64];
    int kept[MOE_MAX_E];
    int off[MOE_MAX_E + 1];
    int warp[17];
    int last;
};

__device__ __forceinline__ void epi_barrier()   // the 4 epilogue warps (128 threads)
{
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Histogram of one 128-token m-tile (the router's rows), as the histogram
// kernel computes it for its chunks: lane masks per slot with match_any
// (leaders are unique per round; rounds ordered by __syncwarp), per-expert
// prefixes over the 4 warps in tile-row order, the tile's counts, and each
// kept slot's rank among the earlier tokens of the tile that chose the same
// expert. All 128 epilogue threads call it once per tile.
__device__ __forceinline__ void router_hist_tile(const TcArgs &p, RouterHistSmem &H, long long row,
                                                 bool valid, int q, int lane, int m_idx)
{
    const int E = p.n_valid, k = p.k;
    H.mask[q][lane] = 0u;
    H.mask[q][lane + 32] = 0u;
    __syncwarp();
    for (int j = 0; j < k; ++j) {
        const int e = valid ? p.route_idx[row * k + j] : -1;
        const uint32_t g = __match_any_sync(kFullMask, e);
        if (e >= 0 && lane == __ffs(g) - 1)
            H.mask[q][e] |= g;
        __syncwarp();
    }
    epi_barrier();
    const int tix = q * 32 + lane;
    if (tix < E) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            H.wpre[w][tix] = run;
            run += __popc(H.mask[w][tix]);
        }
        p.hist_chunk[(long long)m_idx * E + tix] = run;
    }
    epi_barrier();
    if (valid)
        for (int j = 0; j < k; ++j) {
            const int e = p.route_idx[row * k + j];
            p.hist_rank[row * k + j] = H.wpre[q][e] + __popc(H.mask[q][e] & lanemask_lt());
        }
    epi_barrier();
}

template <int BN>
struct TcCfg {
    static constexpr int BM = 128, BK = 64;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN == 256) ? 4 : (BN == 128 ? 6 : 8);
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
};

__device__ __forceinline__ void tile_coords(long long tile, int num_mt, int n_tiles, int group_m,
                                            int &m_idx, int &n_idx)
{
    const long long band_size = (long long)group_m * n_tiles;
    const int band = (int)(tile / band_size);
    const int first_m = band * group_m;
    const int rows = min(group_m, num_mt - first_m);
    const int r = (int)(tile - (long long)band * band_size);
    m_idx = first_m + r % rows;
    n_idx = r / rows;
}

// Tile -> (m-tile, n-tile): band order over a routed list, else plain bands.
__device__ __forceinline__ void tc_coords(const TcArgs &p, long long tile, int num_mt, int tile_m,
                                          int &m_idx, int &n_idx)
{
    if (p.mt_first)
        band_coords(tile, num_mt, p.n_tiles, p.band_g, tile_m, p.mt_first, p.n_groups,
                    p.mt_group, p.seg_offsets, m_idx, n_idx);
    else
        tile_coords(tile, num_mt, p.n_tiles, p.group_m, m_idx, n_idx);
}

// Epilogue of one accumulator tile for this thread's row (TMEM lane): `tb`
// addresses the row's BN fp32 columns. tcgen05.ld is warp-collective, so all
// lanes run it; only rows inside the expert's segment (`valid`) are written.
// Per-warp staging of the combine epilogue: 32 rows x 32 floats, rows padded
// to 36 floats (144 bytes: 16-byte aligned rows).
constexpr int kXposeStride = 36;
constexpr int kXposeBytes = 4 * 32 * kXposeStride * 4;   // the four epilogue warps

template <int BN, int MODE>
__device__ __forceinline__ void epilogue_tile(const TcArgs &p, uint32_t tb, long long row,
                                              bool valid, int n_idx, int grp, bool empty_k,
                                              float *xpose = nullptr)
{
    if (MODE == EPI_SWIGLU_SAVE) {
        // as EPI_SWIGLU, and the raw accumulators (gate | up of this 128-column
        // block, the packed W13 order) as bf16 for the backward pass
        uint16_t *H = static_cast<uint16_t *>(p.out) + row * p.ldo + n_idx * 128;
        uint16_t *GU = static_cast<uint16_t *>(p.out2) + row * 2 * p.ldo + n_idx * 256;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float g[32], u[32];
            tmem_ld32(tb + c * 32, g);
            tmem_ld32(tb + 128 + c * 32, u);
            tmem_ld_wait();
            uint32_t ph[16], pg[16], pu[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                ph[i] = pack_bf16x2(silu_mul(g[2 * i], u[2 * i]), silu_mul(g[2 * i + 1], u[2 * i + 1]));
                pg[i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
                pu[i] = pack_bf16x2(u[2 * i], u[2 * i + 1]);
            }
            if (valid) {
                uint4 *dh = reinterpret_cast<uint4 *>(H + c * 32);
                uint4 *dg = reinterpret_cast<uint4 *>(GU + c * 32);
                uint4 *du = reinterpret_cast<uint4 *>(GU + 128 + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dh[i] = make_uint4(ph[4 * i], ph[4 * i + 1], ph[4 * i + 2], ph[4 * i + 3]);
                    dg[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
                    du[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
                }
            }
        }
    } else if (MODE == EPI_SWIGLU_BWD) {
        // acc columns = dh for h columns n_idx*BN ..; with s = sigmoid(g):
        //   du = dh * g s,  dg = dh * u * s (1 + g (1 - s)),  row_dot += dh * g s u
        // written as [dg | du] in the packed W13 order (block of 128 columns)
        float dot = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (valid) {
                const int col = n_idx * BN + c * 32;               // h column
                const long long pk = row * 2 * p.ldo + (long long)(col / 128) * 256 + (col % 128);
                const uint4 *gsrc = reinterpret_cast<const uint4 *>(p.gu + pk);
                const uint4 *usrc = reinterpret_cast<const uint4 *>(p.gu + pk + 128);
                uint32_t og[16], ou[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 gw = gsrc[i], uw = usrc[i];
                    const uint32_t gg[4] = {gw.x, gw.y, gw.z, gw.w};
                    const uint32_t uu[4] = {uw.x, uw.y, uw.z, uw.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float dg2[2], du2[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const float g = h ? bf16hi(gg[q]) : bf16lo(gg[q]);
                            const float u = h ? bf16hi(uu[q]) : bf16lo(uu[q]);
                            const float dh = v[8 * i + 2 * q + h];
                            const float sg = __fdividef(1.f, 1.f + __expf(-g));
                            const float silu = g * sg;
                            du2[h] = dh * silu;
                            dg2[h] = dh * u * sg * (1.f + g * (1.f - sg));
                            dot = fmaf(dh, silu * u, dot);
                        }
                        og[4 * i + q] = pack_bf16x2(dg2[0], dg2[1]);
                        ou[4 * i + q] = pack_bf16x2(du2[0], du2[1]);
                    }
                }
                uint16_t *dst = static_cast<uint16_t *>(p.out) + pk;
                uint4 *dg = reinterpret_cast<uint4 *>(dst);
                uint4 *du = reinterpret_cast<uint4 *>(dst + 128);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    dg[i] = make_uint4(og[4 * i], og[4 * i + 1], og[4 * i + 2], og[4 * i + 3]);
                    du[i] = make_uint4(ou[4 * i], ou[4 * i + 1], ou[4 * i + 2], ou[4 * i + 3]);
                }
            }
        }
        if (valid)
            atomicAdd(p.row_dot + row, dot);
    } else if (MODE == EPI_SWIGLU) {
        // accumulator columns [0,128) = gate, [128,256) = up of H columns n_idx*128..
        uint16_t *H = static_cast<uint16_t *>(p.out) + row * p.ldo + n_idx * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float g[32], u[32];
            tmem_ld32(tb + c * 32, g);
            tmem_ld32(tb + 128 + c * 32, u);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(silu_mul(g[2 * i], u[2 * i]),
                                    silu_mul(g[2 * i + 1], u[2 * i + 1]));
            if (valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(H + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    } else if (MODE == EPI_COMBINE) {
        int t = 0;
        float wgt = 0.f;
        if (valid) {
            t = p.perm_token ? p.perm_token[row] : (int)row;   // NULL: rows are tokens
            if (p.perm_w) {
                wgt = p.perm_w[row];
            } else if (!p.slot_pos) {
                wgt = 1.f;   // unweighted scatter-add (the backward pass's dx)
            } else {
                for (int j = 0; j < p.k; ++j)
                    if (p.slot_pos[(long long)t * p.k + j] == row)
                        wgt = p.topk_w[(long long)t * p.k + j];
            }
        }
        if (xpose) {
            // lanes hold rows, so each thread's 16-byte atomics would go to 32
            // different rows at once; staging 32 x 32 floats per warp in shared
            // memory lets eight lanes cover one row's 128 contiguous bytes, a
            // quarter of the L2 atomic requests per warp instruction
            const int lane = threadIdx.x & 31;
            float4 *mine = reinterpret_cast<float4 *>(xpose + lane * kXposeStride);
            float *obase = static_cast<float *>(p.out) + n_idx * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld32(tb + c * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mine[i] = make_float4(wgt * v[4 * i], wgt * v[4 * i + 1], wgt * v[4 * i + 2],
                                          wgt * v[4 * i + 3]);
                __syncwarp();
#pragma unroll
                for (int pass = 0; pass < 8; ++pass) {
                    const int r = 4 * pass + (lane >> 3), seg = lane & 7;
                    const int tr = __shfl_sync(kFullMask, t, r);
                    const int vr = __shfl_sync(kFullMask, valid ? 1 : 0, r);
                    const float4 val = reinterpret_cast<const float4 *>(xpose + r * kXposeStride)[seg];
                    if (vr)
                        atomicAdd(reinterpret_cast<float4 *>(obase + (long long)tr * p.ldo + c * 32) + seg,
                                  val);
                }
                __syncwarp();
            }
        } else {
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
        }
    } else if (MODE == EPI_STORE_F32 && xpose && (p.ldo & 3) == 0) {
        // rows through shared memory: eight lanes store one row's 128 bytes
        const int lane = threadIdx.x & 31;
        float4 *mine = reinterpret_cast<float4 *>(xpose + lane * kXposeStride);
        float *obase = static_cast<float *>(p.out) + (long long)grp * p.out_group_stride + n_idx * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (empty_k) {   // a group with no k-blocks: its output block is zero
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mine[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            __syncwarp();
#pragma unroll
            for (int pass = 0; pass < 8; ++pass) {
                const int r = 4 * pass + (lane >> 3), seg = lane & 7;
                const long long rr = __shfl_sync(kFullMask, row, r);
                const int vr = __shfl_sync(kFullMask, valid ? 1 : 0, r);
                if (vr)
                    reinterpret_cast<float4 *>(obase + rr * p.ldo + c * 32)[seg] =
                        reinterpret_cast<const float4 *>(xpose + r * kXposeStride)[seg];
            }
            __syncwarp();
        }
    } else if (MODE == EPI_STORE_F32) {
        float *o = static_cast<float *>(p.out) + (long long)grp * p.out_group_stride +
                   row * p.ldo + n_idx * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (empty_k) {   // a group with no k-blocks: its output block is zero
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] = 0.f;
            }
            if (valid) {
                float4 *dst = reinterpret_cast<float4 *>(o + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    } else if (MODE == EPI_ROUTER_TOPK) {
        // the whole row (E <= 64 logits) is this thread's: logits + bias, then
        // "Sparse MoE Block" routing in registers: k rounds of arg-max (larger
        // logit, then lower index; -0.0 == +0.0) and the weights
        // exp(l_j - l_max) / sum over the chosen k
        float v[64];
        tmem_ld32(tb, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(tb + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_ld_wait();
        if (valid) {
            const int E = p.n_valid;
            float *o = static_cast<float *>(p.out) + row * p.ldo;
            bool bad = false;
#pragma unroll
            for (int n = 0; n < 64; ++n) {
                if (n < E) {
                    v[n] += p.bias ? p.bias[n] : 0.f;
                    o[n] = v[n];
                    bad |= isnan(v[n]);
                }
            }
            uint64_t taken = 0;
            int sel[MOE_MAX_K];
            float ex[MOE_MAX_K];
            float M = 0.f, sum = 0.f;
            for (int j = 0; j < p.k; ++j) {
                float bv = -INFINITY;
                int bi = -1;
#pragma unroll
                for (int n = 0; n < 64; ++n)
                    if (n < E && !((taken >> n) & 1ull) && (bi < 0 || v[n] > bv)) {
                        bv = v[n];
                        bi = n;
                    }
                taken |= 1ull << bi;
                if (j == 0)
                    M = bv;
                sel[j] = bi;
                ex[j] = expf(bv - M);
                sum += ex[j];
            }
            if (bad || !isfinite(M))
                flag_status(p.status, MOE_ERR_NONFINITE);
            for (int j = 0; j < p.k; ++j) {
                p.route_idx[row * p.k + j] = sel[j];
                p.route_w[row * p.k + j] = ex[j] / sum;
            }
        }
    } else if (xpose && (p.n_valid & 3) == 0 && (p.ldo & 3) == 0) {   // EPI_ROUTER, staged
        // as the combine epilogue: rows through shared memory so that eight
        // lanes write one row's 128 contiguous bytes
        const int lane = threadIdx.x & 31;
        float4 *mine = reinterpret_cast<float4 *>(xpose + lane * kXposeStride);
        const long long row_base = row - lane;   // this warp's first row (M = 128 tiles)
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            const int n0 = n_idx * BN + c * 32;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mine[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            __syncwarp();
#pragma unroll
            for (int pass = 0; pass < 8; ++pass) {
                const int r = 4 * pass + (lane >> 3), seg = lane & 7;
                const int vr = __shfl_sync(kFullMask, valid ? 1 : 0, r);
                const int n = n0 + seg * 4;
                if (vr && n < p.n_valid) {
                    float4 val = reinterpret_cast<const float4 *>(xpose + r * kXposeStride)[seg];
                    if (p.bias) {
                        val.x += p.bias[n];
                        val.y += p.bias[n + 1];
                        val.z += p.bias[n + 2];
                        val.w += p.bias[n + 3];
                    }
                    *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (row_base + r) * p.ldo + n) = val;
                }
            }
            __syncwarp();
        }
    } else {   // EPI_ROUTER
        float *o = static_cast<float *>(p.out) + row * p.ldo;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld32(tb + c * 32, v);
            tmem_ld_wait();
            if (valid) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int n = n_idx * BN + c * 32 + i;
                    if (n < p.n_valid)
                        o[n] = v[i] + (p.bias ? p.bias[n] : 0.f);
                }
            }
        }
    }
}

template <int BN, int MODE>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmA64, const TcArgs p)
{
    using C = TcCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + C::STAGES * C::A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + C::STAGES * C::B_BYTES);
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
        tma_prefetch_desc(&tmA64);

    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // launched with programmatic stream serialization: the setup above overlaps
    // the predecessor's tail; nothing the predecessor writes is read before this
    pdl_wait();
    pdl_trigger();

    // the fused router also re-arms the histogram kernel's ticket (which runs
    // after this kernel in stream order)
    if (MODE == EPI_ROUTER_TOPK && blockIdx.x == 0 && threadIdx.x == 0 && p.counter_zero)
        *p.counter_zero = 0;

    const int num_mt = p.num_mt_dev ? *p.num_mt_dev : p.num_mt_host;
    const long long total = (long long)num_mt * p.n_tiles;

    if (warp == 0) {
        if (lane == 0 && !p.starve) {   // ---------------- TMA producer
            uint32_t it = 0;
            for (long long tile = blockIdx.x; tile < total; tile += gridDim.x) {
                int m_idx, n_idx;
                tc_coords(p, tile, num_mt, C::BM, m_idx, n_idx);
                const int row0 = p.mt_row0 ? p.mt_row0[m_idx] : m_idx * C::BM;
                const int grp = p.mt_group ? (p.mt_group[m_idx] & ~kHalfTileBit) : 0;
                const int brow = grp * p.b_rows_per_group + n_idx * BN;
                // a tile of <= 64 rows runs M = 64 MMAs, which read A's first 64
                // rows only: it loads those (a 64-row box), not 128
                const bool half = p.mt_group && (p.mt_group[m_idx] & kHalfTileBit);
                const void *ta = half ? static_cast<const void *>(&tmA64)
                                      : static_cast<const void *>(&tmA);
                const uint32_t stage_bytes = half ? C::STAGE_BYTES - C::A_BYTES / 2 : C::STAGE_BYTES;
                // K-grouped GEMMs contract over their group's own k-block range
                const int kb0 = p.grp_kb0 ? p.grp_kb0[grp] : 0;
                const int nkb = p.grp_kb0 ? p.grp_nkb[grp] : p.kblocks;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], stage_bytes);
                    tma_load_2d(sA + s * C::A_BYTES, ta, (kb0 + kb) * C::BK, row0, &full[s]);
                    tma_load_2d(sB + s * C::B_BYTES, &tmB, (kb0 + kb) * C::BK, brow, &full[s]);
                }
                if (!ok)
                    break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {   // ---------------- MMA issuer
            constexpr uint32_t IDESC128 = idesc_bf16_f32(128, BN);
            constexpr uint32_t IDESC64 = idesc_bf16_f32(64, BN);
            uint32_t it = 0, local = 0;
            for (long long tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
                const uint32_t b = local & 1u, aph = (local >> 1) & 1u;
                int m_idx, n_idx;
                tc_coords(p, tile, num_mt, C::BM, m_idx, n_idx);
                const bool half = p.mt_group && (p.mt_group[m_idx] & kHalfTileBit);
                const uint32_t IDESC = half ? IDESC64 : IDESC128;
                const int grp = p.mt_group ? (p.mt_group[m_idx] & ~kHalfTileBit) : 0;
                const int nkb = p.grp_kb0 ? p.grp_nkb[grp] : p.kblocks;
                if (!mbar_wait(&tempty[b], aph ^ 1u, abort_flag, p.status, p.wait_ns))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * BN;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag, p.status, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)
                        tc_mma_bf16(d_tmem, smem_desc_k128(a0 + kk * 32),
                                    smem_desc_k128(b0 + kk * 32), IDESC, (kb | kk) != 0);
                    tc_commit(&empty[s]);
                }
                if (!ok)
                    break;
                tc_commit(&tfull[b]);
            }
        }
    } else {   // ---------------- epilogue warps 2..5
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        uint32_t local = 0;
        for (long long tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
            int m_idx, n_idx;
            tc_coords(p, tile, num_mt, C::BM, m_idx, n_idx);
            const long long row0 = p.mt_row0 ? p.mt_row0[m_idx] : (long long)m_idx * C::BM;
            const int gword = p.mt_group ? p.mt_group[m_idx] : 0;
            const int grp = gword & ~kHalfTileBit;
            const bool half = (gword & kHalfTileBit) != 0;
            const long long row_end = p.seg_offsets ? p.seg_offsets[grp + 1] : p.rows_valid;
            const uint32_t b = local & 1u, aph = (local >> 1) & 1u;
            const bool got = mbar_wait(&tfull[b], aph, abort_flag, p.status, p.wait_ns);
            // the folded histogram's named barriers need every epilogue warp on
            // every tile, so a warp whose wait gave up keeps going without work
            if (!got && !(MODE == EPI_ROUTER_TOPK && p.hist_chunk))
                break;
            tc_fence_after();
            // M = 128: tile row q*32 + lane sits in lane q*32 + lane. M = 64: tile
            // row 16 q + l sits in lane 32 q + l (l < 16); lanes 16..31 hold nothing.
            const long long row = row0 + (half ? q * 16 + lane : q * 32 + lane);
            const bool valid = got && (!half || lane < 16) && row < row_end;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
            const bool empty_k = p.grp_kb0 && p.grp_nkb[grp] == 0;

            if (got)
                epilogue_tile<BN, MODE>(
                    p, tb, row, valid, n_idx, grp, empty_k,
                    (MODE == EPI_COMBINE || MODE == EPI_STORE_F32 || (MODE == EPI_ROUTER && !half))
                        ? reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(full) + C::BAR_BYTES) +
                              q * 32 * kXposeStride
                        : nullptr);
            if constexpr (MODE == EPI_ROUTER_TOPK) {
                if (p.hist_chunk)
                    router_hist_tile(p, *reinterpret_cast<RouterHistSmem *>(
                                            reinterpret_cast<uint8_t *>(full) + C::BAR_BYTES),
                                     row, valid, q, lane, m_idx);
            }
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
    if constexpr (MODE == EPI_ROUTER_TOPK) {
        // the folded histogram: the last CTA to finish scans every tile's counts
        if (p.hist_chunk) {
            RouterHistSmem &H = *reinterpret_cast<RouterHistSmem *>(
                reinterpret_cast<uint8_t *>(full) + C::BAR_BYTES);
            __threadfence();
            if (threadIdx.x == 0)
                H.last = (atomicAdd(p.hist_counter, 1) == (int)gridDim.x - 1);
            __syncthreads();
            if (H.last) {
                __threadfence();
                hist_finish(p.hist_chunk, num_mt, 1, p.n_valid, p.capacity, p.hist_counts,
                            p.hist_offsets, p.hist_n_kept, p.hist_mt_row0, p.hist_mt_group,
                            p.hist_num_mt, p.hist_mt2_row0, p.hist_mt2_group, p.hist_num_mt2,
                            nullptr, p.hist_counter, H.kept, H.off, H.warp, p.hist_mt_first,
                            p.hist_mt2_first);
            }
        }
    }
}

// ---------------------------------------------------------------- 2-SM pair variant
// A cluster of two CTAs computes one 256 x 256 tile with tcgen05.mma
// cta_group::2 issued by the leader (rank 0): each CTA loads its own 128 rows
// of A and its own half of B (128 rows: the gate half on rank 0, the up half
// on rank 1 for the SwiGLU layout), so each SM moves a third less operand
// data per FLOP than the single-CTA kernel. Both CTAs' TMA copies complete on
// the leader's `full` barrier; the leader's commits arrive on both CTAs'
// `empty` / `tfull` barriers; both epilogues release an accumulator buffer by
// arriving on the leader's `tempty` barrier (8 arrivals: 4 warps x 2 CTAs).
// m-tiles are 256 rows (one expert each); each CTA's epilogue owns its 128.
struct TcPairCfg {
    static constexpr int BK = 64;
    static constexpr int A_BYTES = 128 * BK * 2;
    static constexpr int B_BYTES = 128 * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = 6;
    static constexpr int TMEM_COLS = 512;   // two 256-column accumulators
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + kXposeBytes;
};

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const TcArgs p)
{
    using C = TcPairCfg;
    constexpr int BN = 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + C::STAGES * C::A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + C::STAGES * C::B_BYTES);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = (rank == 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers exist and TMEM is allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_mt = p.num_mt_dev ? *p.num_mt_dev : p.num_mt_host;
    const long long total = (long long)num_mt * p.n_tiles;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {   // ---------------- TMA producer (both CTAs)
            uint32_t it = 0;
            for (long long tile = pair; tile < total; tile += npairs) {
                int m_idx, n_idx;
                tc_coords(p, tile, num_mt, 256, m_idx, n_idx);
                const int row0 = (p.mt_row0 ? p.mt_row0[m_idx] : m_idx * 256) + 128 * (int)rank;
                const int grp = p.mt_group ? (p.mt_group[m_idx] & ~kHalfTileBit) : 0;
                const int brow = grp * p.b_rows_per_group + n_idx * BN + 128 * (int)rank;
                bool ok = true;
                for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (leader)
                        mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
                    const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
                    tma_load_2d_pair(sA + s * C::A_BYTES, &tmA, kb * C::BK, row0, fbar);
                    tma_load_2d_pair(sB + s * C::B_BYTES, &tmB, kb * C::BK, brow, fbar);
                }
                if (!ok)
                    break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {   // ---------------- MMA issuer (leader only)
            constexpr uint32_t IDESC = idesc_bf16_f32(256, BN);
            uint32_t it = 0, local = 0;
            for (long long tile = pair; tile < total; tile += npairs, ++local) {
                const uint32_t b = local & 1u, aph = (local >> 1) & 1u;
                if (!mbar_wait_cluster(&tempty[b], aph ^ 1u, abort_flag, p.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * BN;
                bool ok = true;
                for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (it / C::STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)
                        tc_mma_bf16_pair(d_tmem, smem_desc_k128(a0 + kk * 32),
                                         smem_desc_k128(b0 + kk * 32), IDESC, (kb | kk) != 0);
                    tc_commit_pair(&empty[s], 0x3);
                }
                if (!ok)
                    break;
                tc_commit_pair(&tfull[b], 0x3);
            }
        }
    } else {   // ---------------- epilogue warps 2..5 (both CTAs)
        const int q = warp & 3;
        uint32_t local = 0;
        for (long long tile = pair; tile < total; tile += npairs, ++local) {
            int m_idx, n_idx;
            tc_coords(p, tile, num_mt, 256, m_idx, n_idx);
            const long long row0 = (p.mt_row0 ? p.mt_row0[m_idx] : (long long)m_idx * 256) + 128 * rank;
            const int grp = p.mt_group ? (p.mt_group[m_idx] & ~kHalfTileBit) : 0;
            const long long row_end = p.seg_offsets ? p.seg_offsets[grp + 1] : p.rows_valid;
            const uint32_t b = local & 1u, aph = (local >> 1) & 1u;
            if (!mbar_wait(&tfull[b], aph, abort_flag, p.status))
                break;
            tc_fence_after();
            const long long row = row0 + q * 32 + lane;
            const bool valid = row < row_end;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
            epilogue_tile<BN, MODE>(p, tb, row, valid, n_idx, grp, false,
                                    reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(full) +
                                                              C::BAR_BYTES) +
                                        q * 32 * kXposeStride);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[b]), 0));
        }
    }

    tc_fence_before();
    cluster_sync_all();   // neither CTA leaves while the pair's MMAs may read its memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

// Wait bound of the test-only starved launch (GemmArgs::test_starve).
constexpr unsigned long long kTestWaitLimitNs = 50000000ull;

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
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

// Row-major bf16 matrix [rows, cols] as a 2-D TMA tensor; box = 64 x box_rows
// elements (128 B inner extent), 128-byte swizzle, zero fill out of bounds.
static int make_tmap(CUtensorMap *m, const void *base, long long cols, long long rows,
                     int box_rows)
{
    auto fn = encode_fn();
    if (!fn)
        return MOE_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Band height of a routed GEMM (band_coords): a band's activation rows stay
// in L2 while it sweeps the n-tiles, so its m-tiles are bounded by
// MOE_BAND_MB MiB of bf16 rows of length K.
#ifndef MOE_BAND_MB
#define MOE_BAND_MB 48
#endif
static int band_tiles(long long tile_rows, int K)
{
    const long long per = std::max(tile_rows * K * 2, 1LL);
    return (int)std::min<long long>(std::max<long long>(((long long)MOE_BAND_MB << 20) / per, 1),
                                    1 << 20);
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

template <int BN, int MODE>
static int launch_tc_impl(const GemmArgs &g, cudaStream_t st)
{
    using C = TcCfg<BN>;
    CUtensorMap tA, tB;
    CUtensorMap tA64;
    int rc = make_tmap(&tA, g.A, g.K, g.a_rows, 128);
    if (rc)
        return rc;
    if ((rc = make_tmap(&tA64, g.A, g.K, g.a_rows, 64)))
        return rc;
    rc = make_tmap(&tB, g.B, g.K, g.b_rows_total, BN);
    if (rc)
        return rc;
    TcArgs p;
    std::memset(&p, 0, sizeof p);
    p.kblocks = g.K / 64;
    p.n_tiles = (MODE == EPI_SWIGLU || MODE == EPI_SWIGLU_SAVE) ? g.N / 256 : (g.N + BN - 1) / BN;
    // Rasterisation: consecutive tiles sweep a band of group_m m-tiles across
    // all n-tiles, so a band's B tiles are fetched from HBM about once while
    // its A rows stay in L2. Measured on the Mixtral-shape prefill: bands of 32
    // cut w1/w3 DRAM reads by ~15% and time by ~5% against 8; w2 is flat.
    p.group_m = (MODE == EPI_SWIGLU) ? MOE_GM_1SM_W13 : MOE_GM_1SM_W2;
    p.mt_first = g.mt_row0 ? g.mt_first : nullptr;
    p.n_groups = g.n_groups;
    p.band_g = band_tiles(C::BM, g.K);
    p.b_rows_per_group = g.b_rows_per_group;
    p.mt_row0 = g.mt_row0;
    p.mt_group = g.mt_group;
    p.num_mt_dev = g.num_mt_dev;
    p.num_mt_host = g.num_mt_host;
    p.seg_offsets = g.seg_offsets;
    p.rows_valid = g.rows_valid;
    p.out = g.out;
    p.ldo = g.ldo;
    p.perm_token = g.perm_token;
    p.slot_pos = g.slot_pos;
    p.topk_w = g.topk_w;
    p.k = g.k;
    p.perm_w = g.perm_w;
    p.bias = g.bias;
    p.n_valid = g.n_valid;
    p.status = g.status;
    p.route_idx = g.route_idx;
    p.route_w = g.route_w;
    p.counter_zero = g.counter_zero;
    p.out2 = g.out2;
    p.gu = g.gu;
    p.row_dot = g.row_dot;
    p.grp_kb0 = g.grp_kb0;
    p.grp_nkb = g.grp_nkb;
    p.out_group_stride = g.out_group_stride;
    p.hist_chunk = g.hist_chunk;
    p.hist_rank = g.hist_rank;
    p.hist_counter = g.hist_counter;
    p.hist_counts = g.hist_counts;
    p.hist_offsets = g.hist_offsets;
    p.hist_n_kept = g.hist_n_kept;
    p.hist_mt_row0 = g.hist_mt_row0;
    p.hist_mt_group = g.hist_mt_group;
    p.hist_num_mt = g.hist_num_mt;
    p.hist_mt2_row0 = g.hist_mt2_row0;
    p.hist_mt2_group = g.hist_mt2_group;
    p.hist_num_mt2 = g.hist_num_mt2;
    p.hist_mt_first = g.hist_mt_first;
    p.hist_mt2_first = g.hist_mt2_first;
    p.capacity = g.capacity;
    p.starve = g.test_starve;
    p.wait_ns = g.test_starve ? kTestWaitLimitNs : kWaitLimitNs;

    // the router with the folded histogram also needs its tile-histogram area
    constexpr int SMEM = C::SMEM_BYTES + (MODE == EPI_ROUTER_TOPK ? (int)sizeof(RouterHistSmem) : 0) +
                         ((MODE == EPI_COMBINE || MODE == EPI_ROUTER || MODE == EPI_STORE_F32)
                              ? kXposeBytes
                              : 0);
    static_assert(SMEM <= 232448, "shared memory per CTA");
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(k_gemm_tc<BN, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = 1;
    }
    const int max_mt = g.num_mt_dev ? g.max_mt : g.num_mt_host;
    const long long tiles = (long long)max_mt * p.n_tiles;
    if (tiles <= 0)
        return MOE_OK;
    const int grid = (int)std::min<long long>(tiles, num_sms());
    launch_pdl_ex(k_gemm_tc<BN, MODE>, dim3(grid), dim3(192), SMEM, st, tA, tB, tA64, p);
    return launched();
}

template <int MODE>
static int launch_tc2_impl(const GemmArgs &g, cudaStream_t st)
{
    using C = TcPairCfg;
    CUtensorMap tA, tB;
    int rc = make_tmap(&tA, g.A, g.K, g.a_rows, 128);
    if (rc)
        return rc;
    rc = make_tmap(&tB, g.B, g.K, g.b_rows_total, 128);
    if (rc)
        return rc;
    TcArgs p;
    std::memset(&p, 0, sizeof p);
    p.kblocks = g.K / 64;
    p.n_tiles = g.N / 256;
    p.group_m = (MODE == EPI_SWIGLU) ? MOE_GM_2SM_W13 : MOE_GM_2SM_W2;
    p.mt_first = g.mt_row0 ? g.mt_first : nullptr;
    p.n_groups = g.n_groups;
    p.band_g = band_tiles(256, g.K);
    p.b_rows_per_group = g.b_rows_per_group;
    p.mt_row0 = g.mt_row0;
    p.mt_group = g.mt_group;
    p.num_mt_dev = g.num_mt_dev;
    p.num_mt_host = g.num_mt_host;
    p.seg_offsets = g.seg_offsets;
    p.rows_valid = g.rows_valid;
    p.out = g.out;
    p.ldo = g.ldo;
    p.perm_token = g.perm_token;
    p.slot_pos = g.slot_pos;
    p.topk_w = g.topk_w;
    p.k = g.k;
    p.perm_w = g.perm_w;
    p.bias = g.bias;
    p.n_valid = g.n_valid;
    p.status = g.status;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(k_gemm_tc2<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_done[dev] = 1;
    }
    const int max_mt = g.num_mt_dev ? g.max_mt : g.num_mt_host;
    const long long tiles = (long long)max_mt * p.n_tiles;
    if (tiles <= 0)
        return MOE_OK;
    const int pairs = (int)std::min<long long>(tiles, num_sms() / 2);
    k_gemm_tc2<MODE><<<2 * pairs, 192, C::SMEM_BYTES, st>>>(tA, tB, p);
    return launched();
}

int launch_gemm_tc(const GemmArgs &g, cudaStream_t st)
{
    if (g.pair) {
        switch (g.mode) {
        case EPI_SWIGLU: return launch_tc2_impl<EPI_SWIGLU>(g, st);
        case EPI_COMBINE: return launch_tc2_impl<EPI_COMBINE>(g, st);
        case EPI_STORE_F32: return launch_tc2_impl<EPI_STORE_F32>(g, st);
        default: return MOE_ERR_INVALID_ARG;
        }
    }
    switch (g.mode) {
    case EPI_SWIGLU:
        return launch_tc_impl<256, EPI_SWIGLU>(g, st);
    case EPI_COMBINE:
        return (g.N % 256 == 0) ? launch_tc_impl<256, EPI_COMBINE>(g, st)
                                : launch_tc_impl<128, EPI_COMBINE>(g, st);
    case EPI_STORE_F32:
        return (g.N % 256 == 0) ? launch_tc_impl<256, EPI_STORE_F32>(g, st)
                                : launch_tc_impl<128, EPI_STORE_F32>(g, st);
    case EPI_ROUTER:
        // 64-column tiles: more CTAs for few 128-token tiles; x re-reads hit L2
        return launch_tc_impl<64, EPI_ROUTER>(g, st);
    case EPI_SWIGLU_SAVE:
        return launch_tc_impl<256, EPI_SWIGLU_SAVE>(g, st);
    case EPI_SWIGLU_BWD:
        return (g.N % 256 == 0) ? launch_tc_impl<256, EPI_SWIGLU_BWD>(g, st)
                                : launch_tc_impl<128, EPI_SWIGLU_BWD>(g, st);
    case EPI_ROUTER_TOPK:
        if (g.N > 64 || g.k < 1 || g.k > MOE_MAX_K)
            return MOE_ERR_INVALID_ARG;
        return launch_tc_impl<64, EPI_ROUTER_TOPK>(g, st);
    default:
        return MOE_ERR_INVALID_ARG;
    }
}

} // namespace moe
