// dispatch.cu -- router (CUDA-core path), softmax/top-k, expert histogram and
// offsets, token permutation, fixed-order combine and W1/W3 packing.
//
// Layer definition: "MoE Model Architectures" (architectures.md), section
// "Mixtral 8x7B", "Sparse MoE Block"; offsets as in "Current Bug:
// CuTeDSLMoERunner produces wrong output", "How the pipeline works".
#include <climits>
#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "tiles.cuh"
#include "topk.cuh"

namespace moe {

// ---------------------------------------------------------------- router (CUDA cores)
// logits[t, e] = sum_i x[t, i] * Wg[e, i] + bias[e]. A CTA computes a tile of
// 64 tokens x EC experts; each thread owns TPT tokens x 4 experts; K is staged
// through shared memory 32 at a time. Used for decode-sized T, for the
// CUDA-core debugging path, and as the router when tensor cores are not used.
template <int EC>
__global__ void __launch_bounds__(256) k_router_simt(const uint16_t *__restrict__ x,
                                                     const uint16_t *__restrict__ Wg,
                                                     const float *__restrict__ bias, int T, int d,
                                                     int E, float *__restrict__ logits)
{
    constexpr int EG = EC / 4;      // expert groups of 4
    constexpr int TG = 256 / EG;    // token groups
    constexpr int TPT = 64 / TG;    // tokens per thread
    __shared__ float xs[32][64 + 1];
    __shared__ float ws[32][EC + 1];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * 64, e0 = blockIdx.y * EC;
    const int eg = tid % EG, tg = tid / EG;
    float acc[TPT][4];
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += 32) {
        {   // x tile: 64 tokens x 32 k, one 16-B load per thread
            const int tt = tid / 4, kk = (tid % 4) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t0 + tt < T)
                v = *reinterpret_cast<const uint4 *>(x + (size_t)(t0 + tt) * d + k0 + kk);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                xs[kk + 2 * q][tt] = bf16lo(u[q]);
                xs[kk + 2 * q + 1][tt] = bf16hi(u[q]);
            }
        }
        if (tid < EC * 4) {   // Wg tile: EC experts x 32 k
            const int ee = tid / 4, kk = (tid % 4) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (e0 + ee < E)
                v = *reinterpret_cast<const uint4 *>(Wg + (size_t)(e0 + ee) * d + k0 + kk);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                ws[kk + 2 * q][ee] = bf16lo(u[q]);
                ws[kk + 2 * q + 1][ee] = bf16hi(u[q]);
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            float a[TPT], b[4];
#pragma unroll
            for (int i = 0; i < TPT; ++i)
                a[i] = xs[kk][tg + i * TG];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                b[j] = ws[kk][eg + j * EG];
#pragma unroll
            for (int i = 0; i < TPT; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int t = t0 + tg + i * TG;
        if (t >= T)
            continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + eg + j * EG;
            if (e < E)
                logits[(size_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.f);
        }
    }
}

int launch_router_simt(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                       const float *bias, float *logits, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const dim3 block(256);
    if (s.E <= 16) {
        k_router_simt<16><<<dim3((s.T + 63) / 64, 1), block, 0, st>>>(x, Wg, bias, s.T, s.d, s.E,
                                                                        logits);
    } else {
        k_router_simt<64><<<dim3((s.T + 63) / 64, (s.E + 63) / 64), block, 0, st>>>(
            x, Wg, bias, s.T, s.d, s.E, logits);
    }
    return launched();
}

// ---------------------------------------------------------------- softmax + top-k
template <int VPL>
__global__ void __launch_bounds__(256) k_topk(const float *__restrict__ logits, int T, int E,
                                              int k, int32_t *__restrict__ idx,
                                              float *__restrict__ w, int32_t *counter_to_zero,
                                              uint32_t *status)
{
    pdl_wait();      // the logits come from the router kernel
    pdl_trigger();
    if (counter_to_zero && blockIdx.x == 0 && threadIdx.x == 0)
        *counter_to_zero = 0;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T)
        return;
    warp_topk_row<VPL>(logits + (size_t)t * E, E, k, idx + (size_t)t * k, w + (size_t)t * k,
                       status);
}

int launch_topk(const moe_shape_t &s, const float *logits, int32_t *idx, float *w,
                int32_t *counter_to_zero, uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int blocks = (s.T + 7) / 8;
    const int vpl = (s.E + 31) / 32;
    auto kern = vpl <= 1 ? k_topk<1> : vpl <= 2 ? k_topk<2> : vpl <= 4 ? k_topk<4> : k_topk<8>;
    launch_pdl_ex(kern, dim3(blocks), dim3(256), 0, st, logits, s.T, s.E, s.k, idx, w,
                  counter_to_zero, status);
    return launched();
}

// ---------------------------------------------------------------- histogram + scan
// One CTA per chunk of 256 tokens (thread = token). For each slot j the warp
// groups equal expert ids with __match_any_sync; the group leader ORs the
// group's lane mask into mask[warp][e] (no atomics: leaders are unique per
// round, rounds are ordered by __syncwarp). A token's rank within the chunk
// is the popcount of earlier warps' masks plus the lower lanes of its own.
// The last CTA to finish (ticket counter) scans the per-chunk counts in chunk
// order, applies the capacity, writes offsets and the GEMM tile list, and
// re-arms the counter. The result depends only on idx: bit-exact.
// Slot-major priority: the same per slot, with counts per (chunk, slot), and
// the scan runs over slots, then chunks, so that every first choice ranks
// before any second choice.
__global__ void __launch_bounds__(256) k_hist_scan(
    const int32_t *__restrict__ idx, int T, int E, int k, int C, int slot_major,
    int32_t *chunk_counts, int32_t *__restrict__ rank_local, int32_t *counter,
    int32_t *__restrict__ counts, int32_t *__restrict__ offsets, int32_t *__restrict__ n_kept,
    int32_t *mt_row0, int32_t *mt_group, int32_t *num_mt, int32_t *mt2_row0, int32_t *mt2_group,
    int32_t *num_mt2, int32_t *tile_start, int32_t *mt_first, int32_t *mt2_first, uint32_t *status)
{
    pdl_wait();      // the expert ids come from the routing kernels
    pdl_trigger();
    __shared__ uint32_t mask[8][MOE_MAX_E];
    __shared__ int32_t wpre[8][MOE_MAX_E];
    __shared__ int s_last;
    __shared__ int s_warp[17];
    __shared__ int s_kept[MOE_MAX_E];
    __shared__ int s_off[MOE_MAX_E + 1];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = blockIdx.x * kChunkTokens + tid;
    const bool live = t < T;

    // the token's expert ids, read once; an id out of range or repeating an
    // earlier slot becomes -1 (and is flagged)
    int ids[MOE_MAX_K];
    bool flagged = false;
#pragma unroll
    for (int j = 0; j < MOE_MAX_K; ++j) {
        int e = (live && j < k) ? idx[(size_t)t * k + j] : -1;
        if (live && j < k && (e < 0 || e >= E)) {
            flagged = true;
            e = -1;
        }
#pragma unroll
        for (int jj = 0; jj < j; ++jj)
            if (e >= 0 && ids[jj] == e) {
                flagged = true;
                e = -1;
            }
        ids[j] = e;
    }
    auto slot_expert = [&](int j) {
        int e = -1;
#pragma unroll
        for (int jj = 0; jj < MOE_MAX_K; ++jj)
            if (jj == j)
                e = ids[jj];
        return e;
    };
    // one group of slots [j0, j1): per-warp lane masks, then per-expert warp
    // prefixes and the chunk's count (written at chunk_counts[row])
    auto count_slots = [&](int j0, int j1, size_t row) {
        for (int i = tid; i < 8 * MOE_MAX_E; i += 256)
            (&mask[0][0])[i] = 0u;
        __syncthreads();
        for (int j = j0; j < j1; ++j) {
            const int e = slot_expert(j);
            const uint32_t g = __match_any_sync(kFullMask, e);
            if (e >= 0 && lane == __ffs(g) - 1)
                mask[warp][e] |= g;
            __syncwarp();
        }
        __syncthreads();
        for (int e = tid; e < E; e += 256) {
            int run = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                wpre[w][e] = run;
                run += __popc(mask[w][e]);
            }
            chunk_counts[row * E + e] = run;
        }
        __syncthreads();
        if (live) {
            for (int j = j0; j < j1; ++j) {
                const int e = slot_expert(j);
                rank_local[(size_t)t * k + j] =
                    e >= 0 ? wpre[warp][e] + __popc(mask[warp][e] & lanemask_lt()) : -1;
            }
        }
        __syncthreads();
    };
    if (slot_major) {
        // chunk_counts[(chunk k + j) E + e]: slot j's assignments only
        for (int j = 0; j < k; ++j)
            count_slots(j, j + 1, (size_t)blockIdx.x * k + j);
    } else {
        count_slots(0, k, blockIdx.x);
    }
    if (flagged)
        flag_status(status, MOE_ERR_BAD_EXPERT);

    // ---- the last CTA scans all chunks
    __threadfence();
    __syncthreads();
    if (tid == 0)
        s_last = (atomicAdd(counter, 1) == (int)gridDim.x - 1);
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    hist_finish(chunk_counts, gridDim.x, slot_major ? k : 1, E, C, counts, offsets, n_kept,
                mt_row0, mt_group, num_mt, mt2_row0, mt2_group, num_mt2, tile_start, counter,
                s_kept, s_off, s_warp, mt_first, mt2_first);
}

int launch_hist_scan(const moe_shape_t &s, const int32_t *idx, int32_t *chunk_counts,
                     int32_t *rank_local, int32_t *counter, int32_t *counts, int32_t *offsets,
                     int32_t *n_kept, int32_t *mt_row0, int32_t *mt_group, int32_t *num_mt,
                     int32_t *mt2_row0, int32_t *mt2_group, int32_t *num_mt2, uint32_t *status,
                     cudaStream_t st, int32_t *tile_start, int32_t *mt_first, int32_t *mt2_first)
{
    const int nchunks = (s.T + kChunkTokens - 1) / kChunkTokens;
    if (nchunks == 0)
        return MOE_OK;
    launch_pdl_ex(k_hist_scan, dim3(nchunks), dim3(256), 0, st, idx, s.T, s.E, s.k, s.capacity,
                  slot_major(s), chunk_counts, rank_local, counter, counts, offsets, n_kept,
                  mt_row0, mt_group, num_mt, mt2_row0, mt2_group, num_mt2, tile_start, mt_first,
                  mt2_first, status);
    return launched();
}

// ---------------------------------------------------------------- permutation
// One warp per token: lane j < k resolves slot j's permuted row
// (offsets[e] + chunk base + rank within the chunk of chunk_tokens tokens,
// -1 past the capacity;
// with slot-major priority the base is per (chunk, slot));
// then the warp copies x[t] once into every kept row with 16-B loads/stores
// and, when asked, zeroes out[t] (the fused combine accumulates into it).
__global__ void __launch_bounds__(256) k_permute(
    const int32_t *__restrict__ idx, int T, int E, int k, int C, int slot_major, int d,
    int chunk_tokens, const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ rank_local,
    const int32_t *__restrict__ offsets, const uint4 *__restrict__ x, int32_t *__restrict__ slot_pos,
    int32_t *__restrict__ perm_token, uint4 *__restrict__ x_perm, float4 *__restrict__ out_zero)
{
    pdl_wait();      // offsets, chunk bases and ranks come from the histogram
    pdl_trigger();
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;
    int pos = -1;
    if (lane < k) {
        const int e = idx[(size_t)t * k + lane];
        const int rl = rank_local[(size_t)t * k + lane];
        if (e >= 0 && e < E && rl >= 0) {
            const size_t row = slot_major ? (size_t)(t / chunk_tokens) * k + lane
                                          : (size_t)(t / chunk_tokens);
            const int r = chunk_base[row * E + e] + rl;
            if (C <= 0 || r < C)
                pos = offsets[e] + r;
        }
        slot_pos[(size_t)t * k + lane] = pos;
        if (pos >= 0)
            perm_token[pos] = t;
    }
    if (x_perm) {
        int pj[MOE_MAX_K];
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j)
            pj[j] = __shfl_sync(kFullMask, pos, j);
        const int nv = d / 8;   // a multiple of 16 (d % 128 == 0)
        const uint4 *src = x + (size_t)t * nv;
        // four 16-byte loads in flight per lane, each copied to every kept row
        for (int c0 = 0; c0 < nv; c0 += 128) {
            uint4 v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = c0 + lane + 32 * i;
                if (c < nv)
                    v[i] = src[c];
            }
#pragma unroll
            for (int j = 0; j < MOE_MAX_K; ++j) {
                if (j < k && pj[j] >= 0) {
                    uint4 *dst = x_perm + (size_t)pj[j] * nv;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = c0 + lane + 32 * i;
                        if (c < nv)
                            dst[c] = v[i];
                    }
                }
            }
        }
    }
    if (out_zero) {
        const int nv = d / 4;
        for (int c = lane; c < nv; c += 32)
            out_zero[(size_t)t * nv + c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

int launch_permute(const moe_shape_t &s, const int32_t *idx, const int32_t *chunk_base,
                   const int32_t *rank_local, const int32_t *offsets, const uint16_t *x,
                   int32_t *slot_pos, int32_t *perm_token, uint16_t *x_perm, float *out_zero,
                   cudaStream_t st, int chunk_tokens)
{
    if (s.T == 0)
        return MOE_OK;
    launch_pdl_ex(k_permute, dim3((s.T + 7) / 8), dim3(256), 0, st, idx, s.T, s.E, s.k, s.capacity,
                  slot_major(s), s.d, chunk_tokens, chunk_base, rank_local, offsets,
                  reinterpret_cast<const uint4 *>(x), slot_pos, perm_token,
                  reinterpret_cast<uint4 *>(x_perm), reinterpret_cast<float4 *>(out_zero));
    return launched();
}

// ---------------------------------------------------------------- tile list from offsets
__global__ void __launch_bounds__(256) k_tiles_from_offsets(const int32_t *__restrict__ offsets,
                                                            int E, int32_t *mt_row0,
                                                            int32_t *mt_group, int32_t *num_mt,
                                                            int32_t *mt2_row0, int32_t *mt2_group,
                                                            int32_t *num_mt2, int32_t *mt_first,
                                                            int32_t *mt2_first)
{
    __shared__ int s_kept[MOE_MAX_E];
    __shared__ int s_off[MOE_MAX_E];
    __shared__ int s_warp[17];
    const int e = threadIdx.x;
    s_kept[e] = (e < E) ? max(0, offsets[e + 1] - offsets[e]) : 0;
    s_off[e] = (e < E) ? offsets[e] : 0;
    __syncthreads();
    build_tiles(s_kept, s_off, E, kBlockM, mt_row0, mt_group, num_mt, s_warp, nullptr, mt_first);
    if (mt2_row0)
        build_tiles(s_kept, s_off, E, 2 * kBlockM, mt2_row0, mt2_group, num_mt2, s_warp, nullptr,
                    mt2_first);
}

int launch_tiles_from_offsets(const moe_shape_t &s, const int32_t *offsets, int32_t *mt_row0,
                              int32_t *mt_group, int32_t *num_mt, int32_t *mt2_row0,
                              int32_t *mt2_group, int32_t *num_mt2, cudaStream_t st,
                              int32_t *mt_first, int32_t *mt2_first)
{
    k_tiles_from_offsets<<<1, 256, 0, st>>>(offsets, s.E, mt_row0, mt_group, num_mt, mt2_row0,
                                            mt2_group, num_mt2, mt_first, mt2_first);
    return launched();
}

// ---------------------------------------------------------------- combine (fixed order)
__global__ void __launch_bounds__(256) k_combine(const float4 *__restrict__ y,
                                                 const int32_t *__restrict__ slot_pos,
                                                 const float *__restrict__ w, int T, int k, int d,
                                                 const float4 *shared_out, float4 *out)
{
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;
    int pj = -1;
    float wj = 0.f;
    if (lane < k) {
        pj = slot_pos[(size_t)t * k + lane];
        wj = w[(size_t)t * k + lane];
    }
    int ps[MOE_MAX_K];
    float ws[MOE_MAX_K];
#pragma unroll
    for (int j = 0; j < MOE_MAX_K; ++j) {
        ps[j] = __shfl_sync(kFullMask, pj, j);
        ws[j] = __shfl_sync(kFullMask, wj, j);
    }
    const int nv = d / 4;
    for (int c = lane; c < nv; c += 32) {
        float4 acc = shared_out ? shared_out[(size_t)t * nv + c] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) {
            const int p = ps[j];
            const float ww = ws[j];
            if (j >= k || p < 0)
                continue;
            const float4 v = y[(size_t)p * nv + c];
            acc.x = fmaf(ww, v.x, acc.x);
            acc.y = fmaf(ww, v.y, acc.y);
            acc.z = fmaf(ww, v.z, acc.z);
            acc.w = fmaf(ww, v.w, acc.w);
        }
        out[(size_t)t * nv + c] = acc;
    }
}

int launch_combine(const moe_shape_t &s, const float *y_perm, const int32_t *slot_pos,
                   const float *topk_w, const float *shared_out, float *out, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_combine<<<(s.T + 7) / 8, 256, 0, st>>>(reinterpret_cast<const float4 *>(y_perm), slot_pos,
                                             topk_w, s.T, s.k, s.d,
                                             reinterpret_cast<const float4 *>(shared_out),
                                             reinterpret_cast<float4 *>(out));
    return launched();
}

// ---------------------------------------------------------------- W1/W3 packing
// W13[e, 256 b + r] = r < 128 ? W1[e, 128 b + r] : W3[e, 128 b + r - 128].
__global__ void k_pack_w13(const uint4 *__restrict__ W1, const uint4 *__restrict__ W3,
                           uint4 *__restrict__ W13, int E, int d_ff, int d)
{
    const int nv = d / 8;
    const long long rows = (long long)E * 2 * d_ff;
    const long long total = rows * nv;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long row = i / nv;
        const int c = (int)(i - row * nv);
        const int e = (int)(row / (2 * d_ff));
        const int r = (int)(row - (long long)e * 2 * d_ff);
        const int b = r / 256, within = r % 256;
        const long long src_row = (long long)e * d_ff + b * 128 + (within & 127);
        W13[i] = (within < 128 ? W1 : W3)[src_row * nv + c];
    }
}

int launch_pack_w13(int E, int d_ff, int d, const uint16_t *W1, const uint16_t *W3,
                    uint16_t *W13, cudaStream_t st)
{
    const long long total = (long long)E * 2 * d_ff * (d / 8);
    if (total == 0)
        return MOE_OK;
    const int blocks = (int)std::min<long long>((total + 255) / 256, 148LL * 16);
    k_pack_w13<<<blocks, 256, 0, st>>>(reinterpret_cast<const uint4 *>(W1),
                                       reinterpret_cast<const uint4 *>(W3),
                                       reinterpret_cast<uint4 *>(W13), E, d_ff, d);
    return launched();
}


// ---------------------------------------------------------------- dispatch consistency checks
// Debug bounds checks of a dispatch (moe_check_dispatch): three passes, each
// of which bounds-checks every index before it reads with it.
//   pass 1: zero the per-row counters; one thread checks the offsets
//   pass 2: one thread per assignment: id range, the row inside its expert's
//           segment, perm_token of the row, and one count on the row
//   pass 3: every row below n_kept was counted exactly once
__global__ void k_dbg_offsets(const int32_t *__restrict__ offsets, const int32_t *__restrict__ n_kept,
                              int E, long long N, int capacity, int32_t *__restrict__ seen,
                              uint32_t *status)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < N;
         i += (long long)gridDim.x * blockDim.x)
        seen[i] = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        bool ok = offsets[0] == 0;
        for (int e = 0; e < E; ++e) {
            const int32_t a = offsets[e], b = offsets[e + 1];
            ok = ok && a <= b && (capacity <= 0 || b - a <= capacity);
        }
        const int32_t nk = *n_kept;
        ok = ok && offsets[E] == nk && nk >= 0 && (long long)nk <= N;
        if (!ok)
            flag_status(status, MOE_ERR_CHECK);
    }
}

__global__ void k_dbg_assign(const int32_t *__restrict__ idx, const int32_t *__restrict__ slot_pos,
                             const int32_t *__restrict__ perm_token,
                             const int32_t *__restrict__ offsets, int T, int k, int E, int capacity,
                             int32_t *__restrict__ seen, uint32_t *status)
{
    const long long N = (long long)T * k;
    for (long long a = blockIdx.x * (long long)blockDim.x + threadIdx.x; a < N;
         a += (long long)gridDim.x * blockDim.x) {
        const int e = idx[a];
        const int32_t pos = slot_pos[a];
        const int t = (int)(a / k);
        if (e < 0 || e >= E) {
            flag_status(status, MOE_ERR_BAD_EXPERT);
            continue;
        }
        if (pos == -1) {
            if (capacity <= 0)
                flag_status(status, MOE_ERR_CHECK);   // nothing is dropped without a capacity
            continue;
        }
        if (pos < 0 || (long long)pos >= N) {
            flag_status(status, MOE_ERR_CHECK);
            continue;
        }
        if (pos < offsets[e] || pos >= offsets[e + 1] || perm_token[pos] != t)
            flag_status(status, MOE_ERR_CHECK);
        atomicAdd(seen + pos, 1);
    }
}

__global__ void k_dbg_rows(const int32_t *__restrict__ seen, const int32_t *__restrict__ n_kept,
                           long long N, uint32_t *status)
{
    const long long nk = min((long long)max(*n_kept, 0), N);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nk;
         i += (long long)gridDim.x * blockDim.x)
        if (seen[i] != 1)
            flag_status(status, MOE_ERR_CHECK);
}

int launch_check_dispatch(const moe_shape_t &s, const int32_t *idx, const int32_t *offsets,
                          const int32_t *slot_pos, const int32_t *perm_token,
                          const int32_t *n_kept, int32_t *seen, uint32_t *status, cudaStream_t st)
{
    const long long N = (long long)s.T * s.k;
    if (N == 0)
        return MOE_OK;
    const int grid = (int)std::min<long long>((N + 255) / 256, 4LL * num_sms());
    k_dbg_offsets<<<grid, 256, 0, st>>>(offsets, n_kept, s.E, N, s.capacity, seen, status);
    int rc = launched();
    if (rc)
        return rc;
    k_dbg_assign<<<grid, 256, 0, st>>>(idx, slot_pos, perm_token, offsets, s.T, s.k, s.E,
                                       s.capacity, seen, status);
    if ((rc = launched()))
        return rc;
    k_dbg_rows<<<grid, 256, 0, st>>>(seen, n_kept, N, status);
    return launched();
}

} // namespace moe
