// gemm_simt.cu -- grouped GEMM on CUDA cores (fp32 FMA), the slow debugging
// path that cross-checks the tensor-core kernels. Same m-tile list, same
// epilogue semantics (EpiMode) as gemm_tc.cu, no tensor cores.
#include "common.cuh"
#include "internal.h"

namespace moe {

// One CTA: one 128-row m-tile x 64 output columns; 256 threads, each owning
// 8 rows x 4 columns (two accumulators for the SwiGLU gate/up pair).
template <int MODE>
__global__ void __launch_bounds__(256) k_gemm_simt(const GemmArgs g)
{
    constexpr int BM = 128, BN = 64, BK = 32;
    constexpr bool SWIGLU = (MODE == EPI_SWIGLU);
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[SWIGLU ? 2 : 1][BK][BN + 4];
    const int num_mt = g.num_mt_dev ? *g.num_mt_dev : g.num_mt_host;
    const int m_idx = blockIdx.x;
    if (m_idx >= num_mt)
        return;
    const long long row0 = g.mt_row0 ? g.mt_row0[m_idx] : (long long)m_idx * BM;
    const int grp = g.mt_group ? (g.mt_group[m_idx] & ~kHalfTileBit) : 0;
    const long long row_end = g.seg_offsets ? g.seg_offsets[grp + 1] : g.rows_valid;
    const int n0 = blockIdx.y * BN;   // output column (H column for SWIGLU)
    const long long bgrp = (long long)grp * g.b_rows_per_group;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    float acc[2][8][4] = {};

    for (int k0 = 0; k0 < g.K; k0 += BK) {
        for (int i = tid; i < BM * BK / 8; i += 256) {
            const int r = i / (BK / 8), kk = (i % (BK / 8)) * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row0 + r < g.a_rows)
                v = *reinterpret_cast<const uint4 *>(g.A + (size_t)(row0 + r) * g.K + k0 + kk);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                As[kk + 2 * q][r] = bf16lo(u[q]);
                As[kk + 2 * q + 1][r] = bf16hi(u[q]);
            }
        }
        for (int i = tid; i < (SWIGLU ? 2 : 1) * BN * BK / 8; i += 256) {
            const int h = i / (BN * BK / 8);
            const int ii = i % (BN * BK / 8);
            const int c = ii / (BK / 8), kk = (ii % (BK / 8)) * 8;
            long long brow;
            if (SWIGLU) {
                const int col = n0 + c;   // H column; gate row / up row in the packed W13
                brow = bgrp + (long long)(col / 128) * 256 + (col % 128) + (h ? 128 : 0);
            } else {
                brow = bgrp + n0 + c;
            }
            uint4 v = make_uint4(0, 0, 0, 0);
            if (brow < g.b_rows_total && (SWIGLU || n0 + c < g.N))
                v = *reinterpret_cast<const uint4 *>(g.B + (size_t)brow * g.K + k0 + kk);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                Bs[h][kk + 2 * q][c] = bf16lo(u[q]);
                Bs[h][kk + 2 * q + 1][c] = bf16hi(u[q]);
            }
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < BK; ++kk) {
            float a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                a[i] = As[kk][ty + 16 * i];
#pragma unroll
            for (int h = 0; h < (SWIGLU ? 2 : 1); ++h) {
                float b[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    b[j] = Bs[h][kk][tx + 16 * j];
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        acc[h][i][j] = fmaf(a[i], b[j], acc[h][i][j]);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const long long row = row0 + ty + 16 * i;
        if (row >= row_end)
            continue;
        if (MODE == EPI_SWIGLU) {
            uint16_t *H = static_cast<uint16_t *>(g.out) + row * g.ldo;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = n0 + tx + 16 * j;
                const float h = silu_mul(acc[0][i][j], acc[1][i][j]);
                const __nv_bfloat16 hb = __float2bfloat16_rn(h);
                H[col] = *reinterpret_cast<const uint16_t *>(&hb);
            }
        } else if (MODE == EPI_COMBINE) {
            const int t = g.perm_token[row];
            float wgt = 0.f;
            if (g.perm_w) {
                wgt = g.perm_w[row];
            } else {
                for (int j = 0; j < g.k; ++j)
                    if (g.slot_pos[(size_t)t * g.k + j] == row)
                        wgt = g.topk_w[(size_t)t * g.k + j];
            }
            float *o = static_cast<float *>(g.out) + (long long)t * g.ldo;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                atomicAdd(o + n0 + tx + 16 * j, wgt * acc[0][i][j]);
        } else if (MODE == EPI_STORE_F32) {
            float *o = static_cast<float *>(g.out) + row * g.ldo;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o[n0 + tx + 16 * j] = acc[0][i][j];
        } else {   // EPI_ROUTER
            float *o = static_cast<float *>(g.out) + row * g.ldo;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx + 16 * j;
                if (n < g.n_valid)
                    o[n] = acc[0][i][j] + (g.bias ? g.bias[n] : 0.f);
            }
        }
    }
}

int launch_gemm_simt(const GemmArgs &g, cudaStream_t st)
{
    const int max_mt = g.num_mt_dev ? g.max_mt : g.num_mt_host;
    if (max_mt <= 0)
        return MOE_OK;
    const int ncols = (g.mode == EPI_SWIGLU) ? g.N / 2 : g.N;
    const dim3 grid(max_mt, (ncols + 63) / 64);
    switch (g.mode) {
    case EPI_SWIGLU: k_gemm_simt<EPI_SWIGLU><<<grid, 256, 0, st>>>(g); break;
    case EPI_COMBINE: k_gemm_simt<EPI_COMBINE><<<grid, 256, 0, st>>>(g); break;
    case EPI_STORE_F32: k_gemm_simt<EPI_STORE_F32><<<grid, 256, 0, st>>>(g); break;
    default: k_gemm_simt<EPI_ROUTER><<<grid, 256, 0, st>>>(g); break;
    }
    return launched();
}

} // namespace moe
