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

// Position of element j of one sorted list (length n) in the merge of two
// lists of lengths n and m spread evenly over each other: element j carries
// the key (j + 1/2) / n, the other list's element i the key (i + 1/2) / m,
// and ties go to `first` (the list whose elements precede on equal keys).
__device__ __forceinline__ int spread_merge_pos(int j, int n, int m, bool first)
{
    if (m == 0)
        return j;
    const long long a = (long long)(2 * j + 1) * m;   // key of j, scaled by 2 n m
    long long before;                                 // elements of the other list before j
    if (first) {   // other elements i with (2i + 1) n < a
        const long long num = a - n;
        before = num <= 0 ? 0 : (num + 2LL * n - 1) / (2LL * n);
    } else {       // other elements i with (2i + 1) n <= a
        const long long num = a - n;
        before = num < 0 ? 0 : num / (2LL * n) + 1;
    }
    return j + (int)(before < m ? before : m);
}

// Writes the grouped-GEMM m-tile list for kept counts in s_kept[E]: expert e
// contributes ceil(kept/tile_m) tiles starting at rows offsets[e] + tile_m i.
// Thread e handles expert e (blockDim.x >= E).
//
// Order. With tile_start == NULL the list interleaves two kinds of expert:
// experts of one tile (few rows: their GEMM tiles stream a whole weight
// block for few rows, so they are bound by DRAM) and experts of several
// tiles (their tiles share each weight block through L2, so they are bound
// by the tensor cores). Each list keeps expert order, and the two are spread
// evenly over each other, so every stretch of the list that the GEMM runs at
// once holds both kinds and the weight stream of the first overlaps the
// arithmetic of the second. An expert's tiles stay in order. With tile_start
// set (block-scaled operands, whose activation scales are keyed by tile
// index) the list is in plain expert order and tile_start receives each
// expert's first tile index.
__device__ inline void build_tiles(const int *s_kept, const int32_t *offsets_smem_or_global, int E,
                                   int tile_m, int32_t *mt_row0, int32_t *mt_group,
                                   int32_t *num_mt, int *s_warp, int32_t *tile_start = nullptr)
{
    const int tid = threadIdx.x;
    const int e = tid;
    const int nt = (e < E) ? (s_kept[e] + tile_m - 1) / tile_m : 0;
    const bool spread = tile_start == nullptr;
    const bool multi = nt >= 2;
    int total, n_multi, n_single;
    const int start = block_excl_scan(nt, s_warp, &total);
    const int start_m = block_excl_scan(spread && multi ? nt : 0, s_warp, &n_multi);
    const int start_s = block_excl_scan(spread && !multi ? nt : 0, s_warp, &n_single);
    if (e < E && tile_start)
        tile_start[e] = start;
    if (e < E) {
        const int base = offsets_smem_or_global[e];
        // a last tile of <= 64 rows is marked for the M = 64 MMA (128-row lists only)
        const int rem = s_kept[e] - (nt - 1) * tile_m;
        for (int i = 0; i < nt; ++i) {
            int pos = start + i;
            if (spread)
                pos = multi ? spread_merge_pos(start_m + i, n_multi, n_single, true)
                            : spread_merge_pos(start_s + i, n_single, n_multi, false);
            mt_row0[pos] = base + i * tile_m;
            const bool half = (tile_m == kBlockM) && (i == nt - 1) && rem <= 64;
            mt_group[pos] = e | (half ? kHalfTileBit : 0);
        }
    }
    if (tid == 0)
        *num_mt = total;
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
                                   int *s_warp)
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
    build_tiles(s_kept, s_off, E, kBlockM, mt_row0, mt_group, num_mt, s_warp, tile_start);
    if (mt2_row0)
        build_tiles(s_kept, s_off, E, 2 * kBlockM, mt2_row0, mt2_group, num_mt2, s_warp);
    if (tid == 0)
        *counter = 0;
}

} // namespace moe
