// tiles.cuh -- the histogram's last step, shared by the histogram kernel and
// the router kernel that folds the histogram into its epilogue: per-chunk
// expert counts become exclusive chunk bases, the capacity is applied, and
// the offsets and the grouped GEMMs' m-tile lists are written.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

// Exclusive scan of one int per thread over the block (blockDim.x a multiple
// of 32, at most 256). s_warp holds 17 ints.
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(kFullMask, inc, off);
        if (lane >= off)
            inc += o;
    }
    if (lane == 31)
        s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int wv = (lane < nw) ? s_warp[lane] : 0;
        int winc = wv;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
            const int o = __shfl_up_sync(kFullMask, winc, off);
            if (lane >= off)
                winc += o;
        }
        if (lane < 8)
            s_warp[8 + lane] = winc - wv;
        if (lane == 7)
            s_warp[16] = winc;
    }
    __syncthreads();
    const int r = s_warp[8 + warp] + inc - v;
    *total = s_warp[16];
    __syncthreads();
    return r;
}

// Writes the grouped-GEMM m-tile list for kept counts in s_kept[E]: expert e
// contributes ceil(kept/tile_m) tiles starting at rows offsets[e] + tile_m i.
// Thread e handles expert e (blockDim.x >= E).
//
// Order. With tile_start == NULL the list holds first the experts of several
// tiles, then the experts of one tile, each part in expert order and each
// expert's tiles together and in order. The grouped GEMMs interleave the two
// parts tile by tile (band_coords): one-tile experts stream a whole weight
// block for few rows and are bound by DRAM, multi-tile experts share each
// weight block between their tiles through L2 and are bound by the tensor
// cores, so the mix keeps both busy. With tile_start set (block-scaled
// operands, whose activation scales are keyed by tile index) the list is in
// plain expert order and tile_start receives each expert's first tile index.
// `first` (E + 1 ints, may be NULL) receives each expert's first position in
// the list and, at [E], the length of the first part (the whole list in
// plain order).
__device__ inline void build_tiles(const int *s_kept, const int32_t *offsets_smem_or_global, int E,
                                   int tile_m, int32_t *mt_row0, int32_t *mt_group,
                                   int32_t *num_mt, int *s_warp, int32_t *tile_start = nullptr,
                                   int32_t *first = nullptr)
{
    const int e = threadIdx.x;
    const int nt = (e < E) ? (s_kept[e] + tile_m - 1) / tile_m : 0;
    const bool multi = tile_start != nullptr || nt >= 2;
    int n_multi, n_single;
    const int start_m = block_excl_scan(multi ? nt : 0, s_warp, &n_multi);
    const int start_s = block_excl_scan(multi ? 0 : nt, s_warp, &n_single);
    const int start = multi ? start_m : n_multi + start_s;
    if (e < E) {
        if (tile_start)
            tile_start[e] = start;
        if (first)
            first[e] = start;
        const int base = offsets_smem_or_global[e];
        // a last tile of <= 64 rows is marked for the M = 64 MMA (128-row lists only)
        const int rem = s_kept[e] - (nt - 1) * tile_m;
        for (int i = 0; i < nt; ++i) {
            mt_row0[start + i] = base + i * tile_m;
            const bool half = (tile_m == kBlockM) && (i == nt - 1) && rem <= 64;
            mt_group[start + i] = e | (half ? kHalfTileBit : 0);
        }
    }
    if (e == 0) {
        *num_mt = n_multi + n_single;
        if (first)
            first[E] = n_multi;
    }
}

// Maps tile t (0 <= t < num_mt * n_tiles) of a grouped GEMM to its m-tile and
// n-tile, over a list in build_tiles' order (first[e]: expert e's first
// position; first[E] = nh, the multi-tile part). The tiles of the two parts
// are interleaved evenly: position t belongs to the multi-tile part when
// floor((t + 1) Th / Tt) > floor(t Th / Tt), Th and Tt being that part's and
// the whole list's tile counts.
//  - Multi-tile part: each expert's m-tiles form bands of at most gmax
//    (split into near-equal bands when it has more), and a band's tiles run
//    m-tile fastest, then n-tile, so every weight block of the expert is
//    fetched from DRAM once per band and its other m-tiles read it from L2;
//    bands never hold two experts. gmax bounds the activation rows a band
//    keeps in L2 while it sweeps the n-tiles.
//  - One-tile part: each expert's n-tiles in order (its activation tile stays
//    in L2 across them).
// tile_m is the list's tile height (counts come from the kept offsets seg).
__host__ __device__ __forceinline__ void band_coords(long long t, int num_mt, int n_tiles, int gmax,
                                            int tile_m, const int32_t *first, int E,
                                            const int32_t *mt_group, const int32_t *seg,
                                            int &m_idx, int &n_idx)
{
    const int nh = first[E];
    const long long Tt = (long long)num_mt * n_tiles, Th = (long long)nh * n_tiles;
    const long long a = (t + 1) * Th / Tt;   // multi-part tiles among positions 0..t
    if (a > t * Th / Tt) {
        const long long u = a - 1;
        const int pm = (int)(u / n_tiles);
        const int e = mt_group[pm] & ~kHalfTileBit;
        const int f = first[e];
        const int cnt = (seg[e + 1] - seg[e] + tile_m - 1) / tile_m;
        const int nb = (cnt + gmax - 1) / gmax;
        const int q = cnt / nb, r = cnt - q * nb;   // r bands of q + 1, then bands of q
        const int j = pm - f, big = r * (q + 1);
        const int bi = j < big ? j / (q + 1) : r + (j - big) / q;
        const int b0 = f + (bi < r ? bi * (q + 1) : big + (bi - r) * q);
        const int rows = q + (bi < r ? 1 : 0);
        const long long rr = u - (long long)b0 * n_tiles;
        m_idx = b0 + (int)(rr % rows);
        n_idx = (int)(rr / rows);
    } else {
        const long long v = t - a;
        m_idx = nh + (int)(v / n_tiles);
        n_idx = (int)(v - (long long)(v / n_tiles) * n_tiles);
    }
}

// Run by every thread of the last CTA (after a fence that makes the other
// CTAs' chunk counts visible). chunk_counts[(c * nj + j) * E + e] holds the
// count of expert e in chunk c (for slot j when nj = k, slot-major order);
// it is replaced by the exclusive prefix in rank order (slots, then chunks).
// Then counts, capacity, offsets (E + 1), n_kept, the 128-row m-tile list
// (and the 256-row one when mt2_row0 is set), and the ticket is re-armed.
// s_kept, s_off: MOE_MAX_E (+1) ints of shared memory; s_warp: 17 ints.
__device__ inline void hist_finish(int32_t *chunk_counts, int nchunks, int nj, int E, int C,
                                   int32_t *counts, int32_t *offsets, int32_t *n_kept,
                                   int32_t *mt_row0, int32_t *mt_group, int32_t *num_mt,
                                   int32_t *mt2_row0, int32_t *mt2_group, int32_t *num_mt2,
                                   int32_t *tile_start, int32_t *counter, int *s_kept, int *s_off,
                                   int *s_warp, int32_t *mt_first, int32_t *mt2_first)
{
    const int tid = threadIdx.x;
    const int R = nj * nchunks;   // count rows of one expert, in rank order r = j * nchunks + c
    auto row_at = [&](int r, int e) -> size_t {
        const int j = r / nchunks, c = r - j * nchunks;
        return ((size_t)c * nj + j) * E + e;
    };
    const int nwarps = blockDim.x >> 5;
    if (E * 4 <= nwarps * 32 && R >= 64) {
        // few experts, many rows: a warp per expert, each lane a contiguous
        // range of rows (loads in flight together), then a warp scan of the
        // lane totals
        // A lane holds up to 8 consecutive rows in registers (all loads in
        // flight together); longer lists take rounds of 256 rows.
        const int lane = tid & 31, warp = tid >> 5;
        constexpr int V = 8;
        for (int e = warp; e < MOE_MAX_E; e += nwarps) {
            int kept = 0;
            if (e < E) {
                int carry = 0;
                for (int base = 0; base < R; base += 32 * V) {
                    const int r0 = base + lane * V;
                    int v[V];
#pragma unroll
                    for (int u = 0; u < V; ++u)
                        v[u] = (r0 + u < R) ? __ldcg(&chunk_counts[row_at(r0 + u, e)]) : 0;
                    int sum = 0;
#pragma unroll
                    for (int u = 0; u < V; ++u)
                        sum += v[u];
                    int inc = sum;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const int o = __shfl_up_sync(kFullMask, inc, off);
                        if (lane >= off)
                            inc += o;
                    }
                    int run = carry + inc - sum;
#pragma unroll
                    for (int u = 0; u < V; ++u) {
                        if (r0 + u < R)
                            __stcg(&chunk_counts[row_at(r0 + u, e)], run);
                        run += v[u];
                    }
                    carry += __shfl_sync(kFullMask, inc, 31);
                }
                if (lane == 0)
                    counts[e] = carry;
                kept = (C > 0 && carry > C) ? C : carry;
            }
            if (lane == 0)
                s_kept[e] = kept;
        }
    } else {
        // many experts: a thread per expert, 16 loads in flight
        constexpr int U = 16;
        for (int e = tid; e < MOE_MAX_E; e += blockDim.x) {
            int kept = 0;
            if (e < E) {
                int run = 0;
                for (int r0 = 0; r0 < R; r0 += U) {
                    int v[U];
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        v[u] = (r0 + u) < R ? __ldcg(&chunk_counts[row_at(r0 + u, e)]) : 0;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        if (r0 + u < R)
                            __stcg(&chunk_counts[row_at(r0 + u, e)], run);
                        run += v[u];
                    }
                }
                counts[e] = run;
                kept = (C > 0 && run > C) ? C : run;
            }
            s_kept[e] = kept;
        }
    }
    __syncthreads();
    int total;
    const int ex = block_excl_scan(tid < E ? s_kept[tid] : 0, s_warp, &total);
    if (tid < E) {
        offsets[tid] = ex;
        s_off[tid] = ex;
    }
    if (tid == 0) {
        offsets[E] = total;
        *n_kept = total;
    }
    __syncthreads();
    build_tiles(s_kept, s_off, E, kBlockM, mt_row0, mt_group, num_mt, s_warp, tile_start, mt_first);
    if (mt2_row0)
        build_tiles(s_kept, s_off, E, 2 * kBlockM, mt2_row0, mt2_group, num_mt2, s_warp, nullptr,
                    mt2_first);
    if (tid == 0)
        *counter = 0;
}

} // namespace moe
