// mx_quant.cu -- MXFP8 quantization of expert weights and activations (the
// encoding is defined in mxfp8.cuh).
//
//   k_mx_quantize_rows  a bf16 matrix [rows, K] -> codes [rows, K] + scales in
//                       the atom layout of mxfp8.cuh (tile = row / 128); one
//                       thread per 32-element block
//   k_mx_pack_w13       W1, W3 [E, d_ff, d] -> the packed gate/up operand of
//                       the MXFP8 w1/w3 GEMM: for each block b of 64 h
//                       columns, packed rows 128b..128b+63 are W1 rows
//                       64b.., rows 128b+64..128b+127 are W3 rows 64b.. (one
//                       128-column accumulator tile holds matching gate and
//                       up columns); quantized along d
//   k_mx_gather         x [T, d] -> every kept permuted row of token t:
//                       each token is quantized once and its codes and scales
//                       copied to the rows slot_pos[t, :] names (scales in the
//                       atom layout keyed by the row's m-tile)
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "mxfp8.cuh"

namespace moe {

__device__ __forceinline__ void load_bf16x32(const uint16_t *src, float (&v)[32])
{
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(s + i);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = bf16lo(ww[j]);
            v[8 * i + 2 * j + 1] = bf16hi(ww[j]);
        }
    }
}

__device__ __forceinline__ void store_codes32(uint8_t *dst, const uint32_t (&q)[8])
{
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    d[0] = make_uint4(q[0], q[1], q[2], q[3]);
    d[1] = make_uint4(q[4], q[5], q[6], q[7]);
}

__global__ void __launch_bounds__(256) k_mx_quantize_rows(const uint16_t *__restrict__ src,
                                                          long long nblocks, int K,
                                                          uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nblocks)
        return;
    const int bpr = K / kMxBlock;
    const long long row = i / bpr;
    const int b = (int)(i - row * bpr);
    float v[32];
    load_bf16x32(src + i * kMxBlock, v);
    uint32_t q[8];
    scales[sf_atom_offset(row >> 7, (int)(row & 127), b, K)] = mx_quantize32(v, q);
    store_codes32(codes + i * kMxBlock, q);
}

__global__ void __launch_bounds__(256) k_mx_pack_w13(const uint16_t *__restrict__ W1,
                                                     const uint16_t *__restrict__ W3, int E,
                                                     int d_ff, int d,
                                                     uint8_t *__restrict__ codes,
                                                     uint8_t *__restrict__ scales)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int bpr = d / kMxBlock;
    const long long nblocks = (long long)E * 2 * d_ff * bpr;
    if (i >= nblocks)
        return;
    const long long prow = i / bpr;          // packed row over all experts
    const int b = (int)(i - prow * bpr);
    const int e = (int)(prow / (2 * d_ff));
    const int p = (int)(prow - (long long)e * 2 * d_ff);
    const int blk = p / 128, r = p % 128;
    const uint16_t *src = (r < 64 ? W1 : W3) + ((long long)e * d_ff + 64 * blk + (r & 63)) * d;
    float v[32];
    load_bf16x32(src + b * kMxBlock, v);
    uint32_t q[8];
    scales[sf_atom_offset(prow >> 7, (int)(prow & 127), b, d)] = mx_quantize32(v, q);
    store_codes32(codes + i * kMxBlock, q);
}

// One warp per token; lane j < k holds slot j's permuted row, and the row's
// m-tile (the expert's first tile + its position in the segment / 128) and
// row within the tile, which place its scales in the atom layout.
__global__ void __launch_bounds__(256) k_mx_gather(const uint16_t *__restrict__ x,
                                                   const int32_t *__restrict__ idx,
                                                   const int32_t *__restrict__ slot_pos,
                                                   const int32_t *__restrict__ offsets,
                                                   const int32_t *__restrict__ tile_start, int T,
                                                   int k, int d, uint8_t *__restrict__ xq,
                                                   uint8_t *__restrict__ xsf)
{
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;
    int mine = -1, mtile = 0, mrow = 0;
    if (lane < k) {
        mine = slot_pos[(size_t)t * k + lane];
        if (mine >= 0) {
            const int e = idx[(size_t)t * k + lane];
            const int p = mine - offsets[e];
            mtile = tile_start[e] + (p >> 7);
            mrow = p & 127;
        }
    }
    int pos[MOE_MAX_K], tl[MOE_MAX_K], rw[MOE_MAX_K];
#pragma unroll
    for (int j = 0; j < MOE_MAX_K; ++j) {
        pos[j] = __shfl_sync(kFullMask, mine, j);
        tl[j] = __shfl_sync(kFullMask, mtile, j);
        rw[j] = __shfl_sync(kFullMask, mrow, j);
    }
    const int bpr = d / kMxBlock;
    for (int b = lane; b < bpr; b += 32) {
        float v[32];
        load_bf16x32(x + (size_t)t * d + b * kMxBlock, v);
        uint32_t q[8];
        const uint8_t sc = mx_quantize32(v, q);
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) {
            if (j < k && pos[j] >= 0) {
                store_codes32(xq + (size_t)pos[j] * d + b * kMxBlock, q);
                xsf[sf_atom_offset(tl[j], rw[j], b, d)] = sc;
            }
        }
    }
}

// Blocks of 32 values (bf16 or fp32) through MXFP8 and back, written as bf16:
// an E4M3 value times a power of two has at most 4 significant bits, so the
// bf16 result is exact (outside the far subnormal range). Programmatic
// dependent launch: waits for its predecessor before reading.
template <typename InT>
__global__ void __launch_bounds__(256) k_mx_qdq(const InT *__restrict__ src, long long nblocks,
                                                uint16_t *__restrict__ dst)
{
    pdl_wait();
    pdl_trigger();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nblocks)
        return;
    float v[32];
    if constexpr (sizeof(InT) == 2) {
        load_bf16x32(reinterpret_cast<const uint16_t *>(src) + i * kMxBlock, v);
    } else {
        const float4 *s4 = reinterpret_cast<const float4 *>(src) + i * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 f = s4[j];
            v[4 * j] = f.x;
            v[4 * j + 1] = f.y;
            v[4 * j + 2] = f.z;
            v[4 * j + 3] = f.w;
        }
    }
    uint32_t q[8];
    const float sc = mx_scale_value(mx_quantize32(v, q));
    uint32_t o[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 lo = mx_decode2((uint16_t)(q[j] & 0xffffu));
        const float2 hi = mx_decode2((uint16_t)(q[j] >> 16));
        o[2 * j] = pack_bf16x2(lo.x * sc, lo.y * sc);
        o[2 * j + 1] = pack_bf16x2(hi.x * sc, hi.y * sc);
    }
    uint4 *d4 = reinterpret_cast<uint4 *>(dst + i * kMxBlock);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        d4[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

// ---------------------------------------------------------------- host side
int launch_mx_quantize_rows(const uint16_t *src, long long rows, int K, uint8_t *codes,
                            uint8_t *scales, cudaStream_t st)
{
    const long long nblocks = rows * (K / kMxBlock);
    if (nblocks <= 0)
        return MOE_OK;
    k_mx_quantize_rows<<<(unsigned)((nblocks + 255) / 256), 256, 0, st>>>(src, nblocks, K, codes,
                                                                          scales);
    return launched();
}

int launch_mx_pack_w13(const moe_shape_t &s, const uint16_t *W1, const uint16_t *W3,
                       uint8_t *codes, uint8_t *scales, cudaStream_t st)
{
    const long long nblocks = (long long)s.E * 2 * s.d_ff * (s.d / kMxBlock);
    if (nblocks <= 0)
        return MOE_OK;
    k_mx_pack_w13<<<(unsigned)((nblocks + 255) / 256), 256, 0, st>>>(W1, W3, s.E, s.d_ff, s.d,
                                                                     codes, scales);
    return launched();
}

int launch_mx_gather(const moe_shape_t &s, const uint16_t *x, const int32_t *idx,
                     const int32_t *slot_pos, const int32_t *offsets, const int32_t *tile_start,
                     uint8_t *xq, uint8_t *xsf, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_mx_gather<<<(s.T + 7) / 8, 256, 0, st>>>(x, idx, slot_pos, offsets, tile_start, s.T, s.k,
                                               s.d, xq, xsf);
    return launched();
}

template <typename InT>
static int launch_qdq(const InT *src, long long n, uint16_t *dst, cudaStream_t st)
{
    const long long nblocks = n / kMxBlock;
    if (nblocks <= 0)
        return MOE_OK;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)((nblocks + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, k_mx_qdq<InT>, src, nblocks, dst);
    return launched();
}

int launch_mx_qdq_bf16(const uint16_t *src, long long n, uint16_t *dst, cudaStream_t st)
{
    return launch_qdq(src, n, dst, st);
}

int launch_mx_qdq_f32(const float *src, long long n, uint16_t *dst, cudaStream_t st)
{
    return launch_qdq(src, n, dst, st);
}

} // namespace moe
