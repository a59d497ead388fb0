// mxfp8.cuh -- MXFP8 blocks on the device: E4M3 elements with one E8M0
// (power-of-two) scale per 32 consecutive elements along the contraction
// dimension (OCP "Microscaling (MX) Formats" v1.0).
//
// The shared scale of a block is 2^X with X = floor(log2(max|v|)) - 8 (8 is
// the exponent of E4M3's largest normal binade), clamped to [-127, 127]; an
// all-zero block takes -127. Its E8M0 code is X + 127. Elements are v * 2^-X
// rounded to the nearest E4M3 value, ties to even, saturating at 448
// (cvt.rn.satfinite): the block maximum scales into [256, 512), so scaled
// magnitudes of 464 and above clamp to 448, as the standard's conversion
// does. Multiplying by a power of two is exact here, so the encoding is a
// function of the fp32 inputs alone.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {

constexpr int kMxBlock = 32;

// X for a block maximum amax = 1.m * 2^E (normal): E - 8, the unbiased
// exponent field minus 8. Zero and fp32 subnormals (< 2^-126, where E - 8 is
// below -127 anyway) take -127.
__device__ __forceinline__ int mx_scale_exp(float amax)
{
    const uint32_t b = __float_as_uint(amax) & 0x7fffffffu;
    if (b < 0x00800000u)
        return -127;
    const int X = (int)(b >> 23) - 127 - 8;
    return max(-127, min(127, X));
}

// 2^X as a float for X in [-127, 127] (2^-127 is an fp32 subnormal).
__device__ __forceinline__ float mx_exp2(int X)
{
    return X >= -126 ? __uint_as_float((uint32_t)(X + 127) << 23) : __uint_as_float(0x00400000u);
}

// Four E4M3 codes of v[0..3] * s, packed little-endian (v[0] in the low byte).
__device__ __forceinline__ uint32_t mx_pack4(float a, float b, float c, float d, float s)
{
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a * s, b * s), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c * s, d * s), __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
}

// Quantize one block of 32 fp32 values: 8 words of codes and the E8M0 byte.
__device__ __forceinline__ uint8_t mx_quantize32(const float (&v)[32], uint32_t (&codes)[8])
{
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
        amax = fmaxf(amax, fabsf(v[i]));
    const int X = mx_scale_exp(amax);
    // 2^-X: X = -127 needs 2^127 (normal), X = 127 needs 2^-127 (subnormal)
    const float s = mx_exp2(-X);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        codes[i] = mx_pack4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], s);
    return (uint8_t)(X + 127);
}

// Scale layout for the block-scaled MMA ("scale atoms"): the scales of a
// 128-row x 128-element tile form one 512-byte atom in which the scale of
// tile row m and 32-element block kb (0..3) sits at byte
// (m % 32) * 16 + (m / 32) * 4 + kb, the order tcgen05.cp 32x128b.warpx4
// expects. Atoms are stored tile by tile, K groups innermost: atom
// (tile, g) at byte (tile * (K / 128) + g) * 512. For weights the tile is
// row / 128; for routed activations it is the row's m-tile in the GEMM's tile
// list, so expert segments need no padding.
constexpr int kSfAtomBytes = 512;

__host__ __device__ __forceinline__ long long sf_atom_offset(long long tile, int m, int b, int K)
{
    return (tile * (K / 128) + (b >> 2)) * kSfAtomBytes + (m & 31) * 16 + (m >> 5) * 4 + (b & 3);
}

// Scale bytes of a [rows, K] operand in the atom layout (rows padded to 128).
__host__ __device__ __forceinline__ long long sf_atom_bytes(long long rows, int K)
{
    return (rows + 127) / 128 * (K / 128) * kSfAtomBytes;
}

// Two E4M3 codes (low byte first) -> two floats, exact.
__device__ __forceinline__ float2 mx_decode2(uint16_t c2)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c2, __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// The scale 2^(code - 127) of an E8M0 byte.
__device__ __forceinline__ float mx_scale_value(uint8_t code)
{
    return mx_exp2((int)code - 127);
}

} // namespace moe
