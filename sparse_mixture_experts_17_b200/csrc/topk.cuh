// topk.cuh -- one warp selects the top-k experts of one token.
//
// "MoE Model Architectures", "Mixtral 8x7B" / "Sparse MoE Block": softmax over
// all experts, top-k, divide by the top-k sum. Lane l holds logits l, l+32, ...
// (VPL per lane). k rounds of a butterfly arg-max on the key (larger value,
// then smaller index) pick the experts in selection order (equal logits: the
// lower index first; -0.0 == +0.0). The weights are exp(l_j - l_max) divided
// by their sum over the chosen k, which equals the softmax over all E
// renormalised over the top-k (the full-E denominator cancels).
#pragma once

#include <climits>

#include "common.cuh"

namespace moe {

template <int VPL>
__device__ __forceinline__ void warp_topk_row(const float *l, int E, int k, int32_t *idx_out,
                                              float *w_out, uint32_t *status)
{
    const int lane = threadIdx.x & 31;
    float v[VPL];
    uint32_t avail = 0;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = -INFINITY;
        if (e < E) {
            v[i] = l[e];
            avail |= 1u << i;
            bad |= isnan(v[i]);
        }
    }
    float my_v = 0.f;
    int my_i = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = INT_MAX;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            if (((avail >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
                bv = v[i];
                bi = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(kFullMask, bv, off);
            const int oi = __shfl_xor_sync(kFullMask, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (bi != INT_MAX && (bi & 31) == lane)
            avail &= ~(1u << (bi >> 5));
        if (lane == j) {
            my_v = bv;
            my_i = bi;
        }
    }
    const float M = __shfl_sync(kFullMask, my_v, 0);
    bad |= !isfinite(M);
    if (__any_sync(kFullMask, bad)) {
        if (lane == 0)
            flag_status(status, MOE_ERR_NONFINITE);
    }
    const float ex = (lane < k) ? expf(my_v - M) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        sum += __shfl_xor_sync(kFullMask, sum, off);
    if (lane < k) {
        idx_out[lane] = my_i;
        w_out[lane] = ex / sum;
    }
}

} // namespace moe
