// nv_quant.cu -- NVFP4 quantization of expert weights and activations (the
// encoding is defined in nvfp4.cuh). Codes are packed two per byte, element
// 2i in the low nibble of byte i, rows of K / 2 bytes.
//
//   k_nv_amax           per-expert max |W| of bf16 weights, as fp32 bits
//                       (non-negative floats order like their bits), by
//                       atomicMax; several tensors may share one maximum
//   k_nv_gs_finalize    max -> global encode scale 448 * 6 / max (1 for 0)
//   k_nv_quantize_rows  bf16 [rows, K] -> codes + scales in the atom layout
//                       (weights) or the activation layout (nv_sfa_offset)
//                       (tile = row / 128); the global scale per group of
//                       rows, or one constant
//   k_nv_pack_w13       W1, W3 [E, d_ff, d] -> the packed gate/up operand of
//                       the w1/w3 GEMM (64-row gate/up interleave, as for
//                       MXFP8), with expert e's global scale
//   k_nv_gather         x [T, d] -> every kept permuted row of token t,
//                       quantized once with the activations' global scale;
//                       scales keyed by the row's m-tile
//   k_nv_qrows_f16      rows of x or h for the decode kernels: the codes'
//                       values in f16 and the scales' values in fp32
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "nvfp4.cuh"

namespace moe {

__device__ __forceinline__ void load_bf16x16(const uint16_t *src, float (&v)[16])
{
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 w = __ldg(s + i);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = bf16lo(ww[j]);
            v[8 * i + 2 * j + 1] = bf16hi(ww[j]);
        }
    }
}

// grid (x: slices, y: group); each group is n8 runs of 8 bf16
__global__ void __launch_bounds__(256) k_nv_amax(const uint16_t *__restrict__ src, long long n8,
                                                 uint32_t *__restrict__ amax_bits)
{
    const uint4 *s = reinterpret_cast<const uint4 *>(src) + (long long)blockIdx.y * n8;
    float m = 0.f;
    for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n8;
         i += (long long)gridDim.x * 256) {
        const uint4 w = __ldg(s + i);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            m = fmaxf(m, fmaxf(fabsf(bf16lo(ww[j])), fabsf(bf16hi(ww[j]))));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1)
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    __shared__ float s_m[8];
    if ((threadIdx.x & 31) == 0)
        s_m[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = s_m[0];
        for (int i = 1; i < 8; ++i)
            b = fmaxf(b, s_m[i]);
        atomicMax(&amax_bits[blockIdx.y], __float_as_uint(b));
    }
}

__global__ void k_nv_gs_finalize(float *__restrict__ gs, int n)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        const float a = gs[i];   // holds the maximum on entry
        gs[i] = a > 0.f ? __fdiv_rn(kNvGsNum, a) : 1.0f;
    }
}

__global__ void __launch_bounds__(256) k_nv_quantize_rows(const uint16_t *__restrict__ src,
                                                          long long nblocks, int K,
                                                          const float *__restrict__ gs_arr,
                                                          long long rows_per_gs, float gs_const,
                                                          uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales,
                                                          int a_layout)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nblocks)
        return;
    const int bpr = K / kNvBlock;
    const long long row = i / bpr;
    const int b = (int)(i - row * bpr);
    float v[16];
    load_bf16x16(src + i * kNvBlock, v);
    const float gs = gs_arr ? gs_arr[row / rows_per_gs] : gs_const;
    uint2 q;
    const long long off = a_layout ? nv_sfa_offset(row >> 7, (int)(row & 127), b, K)
                                   : nv_sf_offset(row >> 7, (int)(row & 127), b, K);
    scales[off] = nv_quantize16(v, gs, q);
    reinterpret_cast<uint2 *>(codes)[i] = q;
}

__global__ void __launch_bounds__(256) k_nv_pack_w13(const uint16_t *__restrict__ W1,
                                                     const uint16_t *__restrict__ W3, int E,
                                                     int d_ff, int d, const float *__restrict__ gs13,
                                                     uint8_t *__restrict__ codes,
                                                     uint8_t *__restrict__ scales)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const int bpr = d / kNvBlock;
    const long long nblocks = (long long)E * 2 * d_ff * bpr;
    if (i >= nblocks)
        return;
    const long long prow = i / bpr;   // packed row over all experts
    const int b = (int)(i - prow * bpr);
    const int e = (int)(prow / (2 * d_ff));
    const int p = (int)(prow - (long long)e * 2 * d_ff);
    const int blk = p / 128, r = p % 128;
    const uint16_t *src = (r < 64 ? W1 : W3) + ((long long)e * d_ff + 64 * blk + (r & 63)) * d;
    float v[16];
    load_bf16x16(src + b * kNvBlock, v);
    uint2 q;
    scales[nv_sf_offset(prow >> 7, (int)(prow & 127), b, d)] = nv_quantize16(v, gs13[e], q);
    reinterpret_cast<uint2 *>(codes)[i] = q;
}

// Rows for the NVFP4 decode kernels: each 16-element block of `src` (bf16 or
// fp32) quantized with global scale gs by the same rule as every other
// NVFP4 producer here (nv_quantize16), written as the 16 E2M1 values in f16
// (exact) and the block's E4M3 scale value in fp32. One thread per block;
// launched with programmatic stream serialization.
__device__ __forceinline__ void load16(const uint16_t *src, float (&v)[16]) { load_bf16x16(src, v); }
__device__ __forceinline__ void load16(const float *src, float (&v)[16])
{
    const float4 *s = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 f = s[i];
        v[4 * i] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
    }
}

template <typename InT>
__global__ void __launch_bounds__(256) k_nv_qrows_f16(const InT *__restrict__ src, long long nblocks,
                                                      float gs, uint16_t *__restrict__ dst_h,
                                                      float *__restrict__ dst_s)
{
    pdl_wait();
    pdl_trigger();
    const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (i >= nblocks)
        return;
    float v[16];
    load16(src + i * kNvBlock, v);
    uint2 q;
    const uint8_t sc = nv_quantize16(v, gs, q);
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const __half2 h = nv_pair_h2((j < 4 ? q.x : q.y) >> (8 * (j & 3)));
        o[j] = *reinterpret_cast<const uint32_t *>(&h);
    }
    uint4 *d4 = reinterpret_cast<uint4 *>(dst_h + i * kNvBlock);
    d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
    dst_s[i] = nv_scale_value(sc);
}

// One warp per token (as k_mx_gather): lane j < k holds slot j's permuted
// row, its m-tile and its row within the tile.
__global__ void __launch_bounds__(256) k_nv_gather(const uint16_t *__restrict__ x,
                                                   const int32_t *__restrict__ idx,
                                                   const int32_t *__restrict__ slot_pos,
                                                   const int32_t *__restrict__ offsets,
                                                   const int32_t *__restrict__ tile_start, int T,
                                                   int k, int d, float gs,
                                                   uint8_t *__restrict__ xq,
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
    const int bpr = d / kNvBlock;
    for (int b = lane; b < bpr; b += 32) {
        float v[16];
        load_bf16x16(x + (size_t)t * d + b * kNvBlock, v);
        uint2 q;
        const uint8_t sc = nv_quantize16(v, gs, q);
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) {
            if (j < k && pos[j] >= 0) {
                reinterpret_cast<uint2 *>(xq + (size_t)pos[j] * (d / 2))[b] = q;
                xsf[nv_sfa_offset(tl[j], rw[j], b, d)] = sc;
            }
        }
    }
}

// ---------------------------------------------------------------- host side
static int nv_amax(const uint16_t *src, long long per_group, int groups, float *amax,
                   cudaStream_t st)
{
    const long long n8 = per_group / 8;
    if (n8 <= 0 || groups <= 0)
        return MOE_OK;
    const unsigned gx = (unsigned)std::min<long long>((n8 + 255) / 256, 256);
    k_nv_amax<<<dim3(gx, (unsigned)groups), 256, 0, st>>>(src, n8,
                                                          reinterpret_cast<uint32_t *>(amax));
    return launched();
}

int launch_nv_weight_scales(const moe_shape_t &s, const uint16_t *W1, const uint16_t *W3,
                            const uint16_t *W2, float *gs13, float *gs2, cudaStream_t st)
{
    const int E = s.E;
    if (cudaMemsetAsync(gs13, 0, sizeof(float) * E, st) != cudaSuccess ||
        cudaMemsetAsync(gs2, 0, sizeof(float) * E, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    const long long n13 = (long long)s.d_ff * s.d;
    int rc;
    if ((rc = nv_amax(W1, n13, E, gs13, st)) || (rc = nv_amax(W3, n13, E, gs13, st)) ||
        (rc = nv_amax(W2, n13, E, gs2, st)))
        return rc;
    k_nv_gs_finalize<<<(E + 127) / 128, 128, 0, st>>>(gs13, E);
    if ((rc = launched()))
        return rc;
    k_nv_gs_finalize<<<(E + 127) / 128, 128, 0, st>>>(gs2, E);
    return launched();
}

int launch_nv_quantize_rows(const uint16_t *src, long long rows, int K, const float *gs_arr,
                            long long rows_per_gs, float gs_const, uint8_t *codes,
                            uint8_t *scales, cudaStream_t st, bool a_layout)
{
    const long long nblocks = rows * (K / kNvBlock);
    if (nblocks <= 0)
        return MOE_OK;
    k_nv_quantize_rows<<<(unsigned)((nblocks + 255) / 256), 256, 0, st>>>(
        src, nblocks, K, gs_arr, rows_per_gs > 0 ? rows_per_gs : 1, gs_const, codes, scales,
        a_layout ? 1 : 0);
    return launched();
}

int launch_nv_pack_w13(const moe_shape_t &s, const uint16_t *W1, const uint16_t *W3,
                       const float *gs13, uint8_t *codes, uint8_t *scales, cudaStream_t st)
{
    const long long nblocks = (long long)s.E * 2 * s.d_ff * (s.d / kNvBlock);
    if (nblocks <= 0)
        return MOE_OK;
    k_nv_pack_w13<<<(unsigned)((nblocks + 255) / 256), 256, 0, st>>>(W1, W3, s.E, s.d_ff, s.d,
                                                                     gs13, codes, scales);
    return launched();
}

int launch_nv_gather(const moe_shape_t &s, const uint16_t *x, const int32_t *idx,
                     const int32_t *slot_pos, const int32_t *offsets, const int32_t *tile_start,
                     float gs, uint8_t *xq, uint8_t *xsf, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_nv_gather<<<(s.T + 7) / 8, 256, 0, st>>>(x, idx, slot_pos, offsets, tile_start, s.T, s.k,
                                               s.d, gs, xq, xsf);
    return launched();
}

template <typename InT>
static int launch_nv_qrows(const InT *src, long long n, float gs, uint16_t *dst_h, float *dst_s,
                           cudaStream_t st)
{
    const long long nblocks = n / kNvBlock;
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
    cudaLaunchKernelEx(&cfg, k_nv_qrows_f16<InT>, src, nblocks, gs, dst_h, dst_s);
    return launched();
}

int launch_nv_qrows_f16_bf16(const uint16_t *src, long long n, float gs, uint16_t *dst_h,
                             float *dst_s, cudaStream_t st)
{
    return launch_nv_qrows(src, n, gs, dst_h, dst_s, st);
}

int launch_nv_qrows_f16_f32(const float *src, long long n, float gs, uint16_t *dst_h,
                            float *dst_s, cudaStream_t st)
{
    return launch_nv_qrows(src, n, gs, dst_h, dst_s, st);
}

} // namespace moe
