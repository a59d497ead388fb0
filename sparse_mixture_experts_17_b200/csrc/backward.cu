// backward.cu -- helper kernels of the MoE backward pass (the GEMMs run on the
// tensor-core kernel of gemm_tc.cu).
//
// Gradients of the layer with the routing decisions held fixed ("Sparse MoE
// Block" / "Expert FFN" on "MoE Model Architectures"): for a kept assignment
// (t, j) to expert e with weight w and dout row delta,
//   dW2_e += w delta h^T, dh = w W2_e^T delta, du = dh silu(g),
//   dg = dh u silu'(g), dW1_e += dg x^T, dW3_e += du x^T,
//   dx += W1_e^T dg + W3_e^T du,
// and through the router (softmax renormalised over the chosen experts)
//   dl_j = w_j G_j - w_j sum_i w_i G_i with G_j = <delta, y_j>,
//   dWg += dl^T x, dbias += sum_t dl, dx += dl Wg.
// The per-row sum w <delta, y> = <dh, h> comes out of the dh GEMM's epilogue,
// so the unweighted expert outputs y are never formed.
//
// The weight gradients contract over the rows routed to each expert. Their
// operands are transposed here into [columns, padded rows] with every
// expert's segment starting at a multiple of 64 rows (TMA coordinates stay
// 16-byte aligned) and zero-filled up to the next segment.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kTr = 64;   // transpose tile

// dst[b][c][r] = src[b][r][c] for R x C matrices (R, C multiples of 64).
__global__ void __launch_bounds__(256) k_transpose_batched(const uint16_t *__restrict__ src,
                                                           int R, int C,
                                                           uint16_t *__restrict__ dst)
{
    __shared__ uint16_t tile[kTr][kTr + 2];
    const size_t b = blockIdx.z;
    const int r0 = blockIdx.y * kTr, c0 = blockIdx.x * kTr;
    const uint16_t *s = src + b * (size_t)R * C;
    uint16_t *d = dst + b * (size_t)R * C;
    for (int i = threadIdx.x; i < kTr * kTr; i += blockDim.x) {
        const int rr = i / kTr, cc = i % kTr;
        tile[rr][cc] = s[(size_t)(r0 + rr) * C + c0 + cc];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kTr * kTr; i += blockDim.x) {
        const int cc = i / kTr, rr = i % kTr;
        d[(size_t)(c0 + cc) * R + r0 + rr] = tile[rr][cc];
    }
}

// Expert of a permuted row: the e with offsets[e] <= r < offsets[e + 1].
__device__ __forceinline__ int row_expert(const int32_t *offsets, int E, int r)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= r)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// dst[c][pstart[e] + (r - offsets[e])] = src[r][c] for the n kept rows
// (C a multiple of 64, ld of src = C, ld of dst = ldd).
__global__ void __launch_bounds__(256) k_transpose_grouped(const uint16_t *__restrict__ src,
                                                           int n, int C,
                                                           const int32_t *__restrict__ offsets,
                                                           const int32_t *__restrict__ pstart,
                                                           int E, uint16_t *__restrict__ dst,
                                                           long long ldd)
{
    __shared__ uint16_t tile[kTr][kTr + 2];
    __shared__ int dcol[kTr];
    const int r0 = blockIdx.y * kTr, c0 = blockIdx.x * kTr;
    const int n_kept = min(n, offsets[E]);   // rows past the kept ones (drops) are absent
    if (threadIdx.x < kTr) {
        const int r = r0 + threadIdx.x;
        int dc = -1;
        if (r < n_kept) {
            const int e = row_expert(offsets, E, r);
            dc = pstart[e] + (r - offsets[e]);
        }
        dcol[threadIdx.x] = dc;
    }
    for (int i = threadIdx.x; i < kTr * kTr; i += blockDim.x) {
        const int rr = i / kTr, cc = i % kTr;
        tile[rr][cc] = (r0 + rr < n_kept) ? src[(size_t)(r0 + rr) * C + c0 + cc] : 0;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kTr * kTr; i += blockDim.x) {
        const int cc = i / kTr, rr = i % kTr;
        const int dc = dcol[rr];
        if (dc >= 0)
            dst[(size_t)(c0 + cc) * ldd + dc] = tile[rr][cc];
    }
}

// Zero the padding columns [pstart[e] + n_e, pstart[e + 1]) of every dst row.
__global__ void __launch_bounds__(256) k_zero_pads(const int32_t *__restrict__ offsets,
                                                   const int32_t *__restrict__ pstart, int E,
                                                   int rows, uint16_t *__restrict__ dst,
                                                   long long ldd)
{
    const int row = blockIdx.x;
    if (row >= rows)
        return;
    for (int e = 0; e < E; ++e) {
        const int a = pstart[e] + (offsets[e + 1] - offsets[e]), b = pstart[e + 1];
        for (int c = a + (int)threadIdx.x; c < b; c += blockDim.x)
            dst[(size_t)row * ldd + c] = 0;
    }
}

// Per expert: padded row start (multiple of 64), its first k-block and count
// (blocks of 64 rows); plus the K-grouped m-tile lists for outputs of M1 and
// M2 rows (identity tiles per expert).
__global__ void k_group_ranges(const int32_t *__restrict__ offsets, int E, int32_t *pstart,
                               int32_t *kb0, int32_t *nkb, int M1, int32_t *mt1_row0,
                               int32_t *mt1_group, int M2, int32_t *mt2_row0, int32_t *mt2_group)
{
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int ne = offsets[e + 1] - offsets[e];
            const int pad = (ne + 63) / 64;
            pstart[e] = run;
            kb0[e] = run / 64;
            nkb[e] = pad;
            run += pad * 64;
        }
        pstart[E] = run;
    }
    const int n1 = M1 / kBlockM, n2 = M2 / kBlockM;
    for (int i = threadIdx.x; i < E * n1; i += blockDim.x) {
        mt1_row0[i] = (i % n1) * kBlockM;
        mt1_group[i] = i / n1;
    }
    for (int i = threadIdx.x; i < E * n2; i += blockDim.x) {
        mt2_row0[i] = (i % n2) * kBlockM;
        mt2_group[i] = i / n2;
    }
}

// dYw[slot row] = w[t, j] * dout[t] in bf16, for every kept slot of token t
// (one warp per token).
__global__ void __launch_bounds__(256) k_bwd_dyw(const float *__restrict__ dout,
                                                 const int32_t *__restrict__ slot_pos,
                                                 const float *__restrict__ topk_w, int T, int k,
                                                 int d, uint16_t *__restrict__ dyw)
{
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;
    const int mp = (lane < k) ? slot_pos[(size_t)t * k + lane] : -1;
    const float mw = (lane < k) ? topk_w[(size_t)t * k + lane] : 0.f;
    const float4 *src = reinterpret_cast<const float4 *>(dout + (size_t)t * d);
    for (int j = 0; j < k; ++j) {
        const int pos = __shfl_sync(kFullMask, mp, j);
        const float wj = __shfl_sync(kFullMask, mw, j);
        if (pos < 0)
            continue;
        uint2 *dst = reinterpret_cast<uint2 *>(dyw + (size_t)pos * d);
        for (int c = lane; c < d / 4; c += 32) {
            const float4 v = src[c];
            dst[c] = make_uint2(pack_bf16x2(wj * v.x, wj * v.y), pack_bf16x2(wj * v.z, wj * v.w));
        }
    }
}

// Router: dl[t, e_j] = Gw_j - w_j sum_i Gw_i over the chosen slots, where
// Gw_j = w_j <dout_t, y_j> is the dh GEMM's row sum (0 for a dropped slot);
// 0 for the other experts. One warp per token.
__global__ void __launch_bounds__(256) k_router_bwd_dl(const int32_t *__restrict__ idx,
                                                       const float *__restrict__ topk_w,
                                                       const int32_t *__restrict__ slot_pos,
                                                       const float *__restrict__ row_dot, int T,
                                                       int E, int k, float *__restrict__ dl)
{
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;
    float gw = 0.f, wj = 0.f;
    int e = -1;
    if (lane < k) {
        const int pos = slot_pos[(size_t)t * k + lane];
        gw = pos >= 0 ? row_dot[pos] : 0.f;
        wj = topk_w[(size_t)t * k + lane];
        e = idx[(size_t)t * k + lane];
    }
    float sum = gw;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        sum += __shfl_xor_sync(kFullMask, sum, off);
    for (int c = lane; c < E; c += 32)
        dl[(size_t)t * E + c] = 0.f;
    __syncwarp();
    if (lane < k && e >= 0 && e < E)
        dl[(size_t)t * E + e] = gw - wj * sum;
}

// dWg[e, i] = sum_t dl[t, e] x[t, i] in two fixed-order passes (deterministic):
// chunk c of kDwgChunk tokens -> part[c][e][i], then the chunks summed in order.
// Thread (e, i) with consecutive i across a warp.
constexpr int kDwgChunk = 1024;

__global__ void __launch_bounds__(256) k_router_bwd_dwg_part(const float *__restrict__ dl,
                                                             const uint16_t *__restrict__ x,
                                                             int T, int E, int d,
                                                             float *__restrict__ part)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int e = blockIdx.y, c = blockIdx.z;
    if (i >= d)
        return;
    const int t1 = min(T, (c + 1) * kDwgChunk);
    float acc = 0.f;
    for (int t = c * kDwgChunk; t < t1; ++t) {
        const uint16_t xb = x[(size_t)t * d + i];
        acc = fmaf(dl[(size_t)t * E + e], __uint_as_float((uint32_t)xb << 16), acc);
    }
    part[((size_t)c * E + e) * d + i] = acc;
}

__global__ void __launch_bounds__(256) k_router_bwd_dwg_sum(const float *__restrict__ part,
                                                            int nchunks, int E, int d,
                                                            float *__restrict__ dWg)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int e = blockIdx.y;
    if (i >= d)
        return;
    float acc = 0.f;
    for (int c = 0; c < nchunks; ++c)
        acc += part[((size_t)c * E + e) * d + i];
    dWg[(size_t)e * d + i] = acc;
}

// dbias[e] = sum_t dl[t, e] (block reduction in a fixed order).
__global__ void __launch_bounds__(256) k_router_bwd_dbias(const float *__restrict__ dl, int T,
                                                          int E, float *__restrict__ dbias)
{
    __shared__ float red[256];
    const int e = blockIdx.x;
    float acc = 0.f;
    for (int t = threadIdx.x; t < T; t += blockDim.x)
        acc += dl[(size_t)t * E + e];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if ((int)threadIdx.x < s)
            red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        dbias[e] = red[0];
}

// dx[t, i] += sum_e dl[t, e] Wg[e, i]; thread (t, i).
__global__ void __launch_bounds__(256) k_router_bwd_dx(const float *__restrict__ dl,
                                                       const uint16_t *__restrict__ Wg, int T,
                                                       int E, int d, float *__restrict__ dx)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int t = blockIdx.y;
    if (i >= d || t >= T)
        return;
    float acc = 0.f;
    for (int e = 0; e < E; ++e) {
        const float g = dl[(size_t)t * E + e];
        if (g != 0.f)
            acc = fmaf(g, __uint_as_float((uint32_t)Wg[(size_t)e * d + i] << 16), acc);
    }
    dx[(size_t)t * d + i] += acc;
}

// bf16 copy of dout (the shared expert's w * dout with w = 1), and the
// single-group offsets {0, T} its weight gradients contract over.
__global__ void __launch_bounds__(256) k_bwd_shared_prep(const float *__restrict__ dout,
                                                         long long n4, int T,
                                                         uint16_t *__restrict__ dout_bf,
                                                         int32_t *__restrict__ offs)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) {
        offs[0] = 0;
        offs[1] = T;
    }
    if (i >= n4)
        return;
    const float4 v = reinterpret_cast<const float4 *>(dout)[i];
    reinterpret_cast<uint2 *>(dout_bf)[i] =
        make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

// ---------------------------------------------------------------- host side
int launch_bwd_shared_prep(const float *dout, int T, int d, uint16_t *dout_bf, int32_t *offs,
                           cudaStream_t st)
{
    const long long n4 = (long long)T * d / 4;
    k_bwd_shared_prep<<<(unsigned)((std::max(n4, 1LL) + 255) / 256), 256, 0, st>>>(dout, n4, T,
                                                                                dout_bf, offs);
    return launched();
}

int launch_transpose_batched(const uint16_t *src, int batch, int R, int C, uint16_t *dst,
                             cudaStream_t st)
{
    if (batch == 0 || R == 0 || C == 0)
        return MOE_OK;
    k_transpose_batched<<<dim3(C / kTr, R / kTr, batch), 256, 0, st>>>(src, R, C, dst);
    return launched();
}

int launch_transpose_grouped(const uint16_t *src, int n, int C, const int32_t *offsets,
                             const int32_t *pstart, int E, uint16_t *dst, long long ldd,
                             cudaStream_t st)
{
    if (n > 0) {
        k_transpose_grouped<<<dim3(C / kTr, (n + kTr - 1) / kTr), 256, 0, st>>>(
            src, n, C, offsets, pstart, E, dst, ldd);
        int rc = launched();
        if (rc)
            return rc;
    }
    k_zero_pads<<<C, 256, 0, st>>>(offsets, pstart, E, C, dst, ldd);
    return launched();
}

int launch_group_ranges(const int32_t *offsets, int E, int32_t *pstart, int32_t *kb0,
                        int32_t *nkb, int M1, int32_t *mt1_row0, int32_t *mt1_group, int M2,
                        int32_t *mt2_row0, int32_t *mt2_group, cudaStream_t st)
{
    k_group_ranges<<<1, 256, 0, st>>>(offsets, E, pstart, kb0, nkb, M1, mt1_row0, mt1_group, M2,
                                      mt2_row0, mt2_group);
    return launched();
}

int launch_bwd_dyw(const moe_shape_t &s, const float *dout, const int32_t *slot_pos,
                   const float *topk_w, uint16_t *dyw, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_bwd_dyw<<<(s.T + 7) / 8, 256, 0, st>>>(dout, slot_pos, topk_w, s.T, s.k, s.d, dyw);
    return launched();
}

size_t router_bwd_part_bytes(const moe_shape_t &s)
{
    return (size_t)((s.T + kDwgChunk - 1) / kDwgChunk) * s.E * s.d * 4;
}

int launch_router_bwd(const moe_shape_t &s, const int32_t *idx, const float *topk_w,
                      const int32_t *slot_pos, const float *row_dot, const uint16_t *x,
                      const uint16_t *Wg, float *dl, float *part, float *dWg, float *dbias,
                      float *dx, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_router_bwd_dl<<<(s.T + 7) / 8, 256, 0, st>>>(idx, topk_w, slot_pos, row_dot, s.T, s.E, s.k,
                                                   dl);
    int rc = launched();
    if (rc)
        return rc;
    const int nchunks = (s.T + kDwgChunk - 1) / kDwgChunk;
    k_router_bwd_dwg_part<<<dim3((s.d + 255) / 256, s.E, nchunks), 256, 0, st>>>(dl, x, s.T, s.E,
                                                                                  s.d, part);
    if ((rc = launched()))
        return rc;
    k_router_bwd_dwg_sum<<<dim3((s.d + 255) / 256, s.E), 256, 0, st>>>(part, nchunks, s.E, s.d,
                                                                      dWg);
    if ((rc = launched()))
        return rc;
    k_router_bwd_dbias<<<s.E, 256, 0, st>>>(dl, s.T, s.E, dbias);
    if ((rc = launched()))
        return rc;
    k_router_bwd_dx<<<dim3((s.d + 255) / 256, s.T), 256, 0, st>>>(dl, Wg, s.T, s.E, s.d, dx);
    return launched();
}

} // namespace moe
