// nvfp4.cuh -- NVFP4 blocks on the device: E2M1 elements (magnitudes 0, 0.5,
// 1, 1.5, 2, 3, 4, 6), one E4M3 scale per 16 consecutive elements along the
// contraction dimension, and one fp32 global encode scale gs per tensor.
//
// Encoding of a block (every step one IEEE fp32 operation, in this order):
//   sd = (amax / 6) * gs; s = E4M3(sd), nearest, ties to even, saturating at
//   448; r = gs / s (0 when s = 0); code_i = E2M1(v_i * r), nearest, ties to
//   even, saturating at 6. The value of a code is E2M1 * s / gs.
// For a weight tensor gs = 448 * 6 / amax(tensor) (1 for an all-zero tensor);
// for activations it is a constant the caller supplies.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {

constexpr int kNvBlock = 16;
constexpr float kNvGsNum = 2688.0f;   // 448 * 6: E4M3 max times E2M1 max

// E4M3 code of a non-negative value (nearest, ties to even, saturating) and
// the value it stands for.
__device__ __forceinline__ uint8_t nv_e4m3(float v, float &val)
{
    const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
    const __half_raw h = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);
    val = __half2float(*reinterpret_cast<const __half *>(&h));
    return (uint8_t)c;
}

// Two values -> two E2M1 codes in one byte, the first in the low nibble.
__device__ __forceinline__ uint32_t nv_e2m1x2(float a, float b)
{
    return (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest);
}

// Quantize 16 fp32 values with global scale gs: 8 bytes of codes (element 2i
// in the low nibble of byte i) and the E4M3 scale code.
__device__ __forceinline__ uint8_t nv_quantize16(const float *v, float gs, uint2 &codes)
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
        amax = fmaxf(amax, fabsf(v[i]));
    float s;
    const uint8_t sc = nv_e4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs), s);
    const float r = s > 0.f ? __fdiv_rn(gs, s) : 0.f;
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t acc = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc |= nv_e2m1x2(__fmul_rn(v[8 * h + 2 * j], r), __fmul_rn(v[8 * h + 2 * j + 1], r))
                   << (8 * j);
        w[h] = acc;
    }
    codes = make_uint2(w[0], w[1]);
    return sc;
}

// Two E2M1 codes (one byte, the first element in the low nibble) -> the two
// values as f16x2 (exact: every E2M1 value is an f16).
__device__ __forceinline__ __half2 nv_pair_h2(uint32_t byte)
{
    const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xffu), __NV_E2M1);
    return *reinterpret_cast<const __half2 *>(&r);
}

// The value of an E4M3 scale code (exact in fp32).
__device__ __forceinline__ float nv_scale_value(uint32_t code)
{
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xffu), __NV_E4M3);
    return __half2float(*reinterpret_cast<const __half *>(&h));
}

// Scale layout for the block-scaled MMA with 16-element blocks: the scales
// of a 128-row x 64-element tile form one 512-byte atom in which the scale of
// tile row m and block b (0..3) sits at byte (m % 32) * 16 + (m / 32) * 4 + b
// (the order tcgen05.cp 32x128b.warpx4 expects; one atom feeds one K = 64
// MMA). Atoms are stored tile by tile, K groups innermost: atom (tile, g) at
// byte (tile * (K / 64) + g) * 512, so the four atoms of one 256-element
// K stage are contiguous.
__host__ __device__ __forceinline__ long long nv_sf_offset(long long tile, int m, int b, int K)
{
    return (tile * (K / 64) + (b >> 2)) * 512 + (m & 31) * 16 + (m >> 5) * 4 + (b & 3);
}

// Scale bytes of a [rows, K] operand in this layout (rows padded to 128).
__host__ __device__ __forceinline__ long long nv_sf_bytes(long long rows, int K)
{
    return (rows + 127) / 128 * (K / 64) * 512;
}

// Activation (A operand) scales of the block-scaled GEMM in the layout one
// tcgen05.cp 128x256b copy per two K groups serves: the MMA's lane quarter q
// (rows 32 q .. 32 q + 31) reads column slot + q of a K group's 4-column
// slot, so row m needs its four block scales only at bytes 4 q .. 4 q + 3 of
// that slot's 16-byte lane chunk, and no replication over the quarters.
// Per 128-row tile and 256-element K stage an 8 KB region: two 4 KB copy
// sources (K groups 0-1 and 2-3 of the stage), each two 2 KB chunks (the
// first and the second K group), each 128 lane rows of 16 bytes. The other
// 12 bytes of a lane row are never read.
__host__ __device__ __forceinline__ long long nv_sfa_offset(long long tile, int m, int b, int K)
{
    const int stage = b >> 4, g = (b >> 2) & 3;   // K stage (16 blocks), K group within it
    return (tile * ((K + 255) / 256) + stage) * 8192 + (g >> 1) * 4096 + (g & 1) * 2048 + m * 16 +
           (m >> 5) * 4 + (b & 3);
}

// Bytes of an activation scale buffer in that layout (rows padded to 128).
__host__ __device__ __forceinline__ long long nv_sfa_bytes(long long rows, int K)
{
    return (rows + 127) / 128 * ((K + 255) / 256) * 8192;
}

} // namespace moe
