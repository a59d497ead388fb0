// expert_choice.cu -- expert-choice routing ("MoE Model Architectures",
// "Design Patterns", "Pattern 3: Expert Choice Routing": each expert selects
// its top tokens from all tokens, instead of tokens choosing experts).
//
// Score of (t, e): the softmax over experts of token t's logits ("Sparse MoE
// Block"). Expert e takes the K = min(C, T) tokens with the largest scores in
// column e (equal scores: the lower token first), listed in ascending token
// order with weight S[t, e]. The selected rows are laid out expert-major
// (expert e owns rows [e K, (e+1) K)), so the same grouped tensor-core GEMMs
// run on them; the w2 epilogue adds w * y into out[token] as in top-k routing.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace moe {

// ---------------------------------------------------------------- softmax over experts
template <int VPL>
__global__ void __launch_bounds__(256) k_softmax_rows(const float *__restrict__ logits, int T,
                                                      int E, float *__restrict__ scores,
                                                      uint32_t *status)
{
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= T)
        return;
    const float *l = logits + (size_t)t * E;
    float v[VPL];
    float m = -INFINITY;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? l[e] : -INFINITY;
        bad |= isnan(v[i]);
        m = fmaxf(m, v[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    bad |= !isfinite(m);
    if (__any_sync(kFullMask, bad)) {
        if (lane == 0)
            flag_status(status, MOE_ERR_NONFINITE);
    }
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        v[i] = (lane + 32 * i < E) ? expf(v[i] - m) : 0.f;
        z += v[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        z += __shfl_xor_sync(kFullMask, z, off);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E)
            scores[(size_t)t * E + e] = v[i] / z;
    }
}

// ---------------------------------------------------------------- per-expert selection
// One CTA of 1024 threads per expert. Scores are >= 0, so their bit patterns
// order like the values. Four 8-bit radix passes find the exact key of the
// K-th largest score and how many of its ties to take; a token-order pass
// then writes every token above it plus the first ties, in ascending order.
// Counts use shared-memory atomics (order-independent): the result is a
// function of the scores alone. Block e also writes offsets[e] = e K and its
// own grouped-GEMM m-tiles.
constexpr int kEcThreads = 1024;

__global__ void __launch_bounds__(kEcThreads) k_ec_select(
    const float *__restrict__ scores, int T, int E, int K, int32_t *__restrict__ tokens,
    float *__restrict__ weights, int32_t *__restrict__ offsets, int32_t *__restrict__ mt_row0,
    int32_t *__restrict__ mt_group, int32_t *__restrict__ num_mt, int32_t *__restrict__ mt_first,
    uint32_t *status)
{
    __shared__ int hist[256];
    __shared__ uint32_t s_prefix;
    __shared__ int s_remaining;
    __shared__ int s_tie[kEcThreads / 32];
    __shared__ int s_take[kEcThreads / 32];
    __shared__ int s_run[2];
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto key = [&](int t) { return __float_as_uint(scores[(size_t)t * E + e]); };

    if (tid == 0) {
        s_prefix = 0;
        s_remaining = K;
    }
    __syncthreads();
    bool bad = false;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kEcThreads)
            hist[i] = 0;
        __syncthreads();
        const uint32_t prefix = s_prefix;
        const uint32_t hi_mask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
        for (int t = tid; t < T; t += kEcThreads) {
            const uint32_t u = key(t);
            if (shift == 24)
                bad |= (u > 0x7F800000u);   // NaN (or a negative score)
            if ((u & hi_mask) == (prefix & hi_mask))
                atomicAdd(&hist[(u >> shift) & 255], 1);
        }
        __syncthreads();
        if (tid == 0) {
            int cum = 0, rem = s_remaining;
            for (int b = 255; b >= 0; --b) {
                if (cum + hist[b] >= rem) {
                    s_prefix = prefix | ((uint32_t)b << shift);
                    s_remaining = rem - cum;
                    break;
                }
                cum += hist[b];
            }
        }
        __syncthreads();
    }
    if (__syncthreads_or(bad) && tid == 0)
        flag_status(status, MOE_ERR_NONFINITE);
    const uint32_t kth = s_prefix;     // key of the K-th largest score
    const int ties = s_remaining;      // how many tokens equal to it are taken
    if (tid == 0) {
        s_run[0] = 0;   // tokens written so far
        s_run[1] = 0;   // ties seen so far
    }
    __syncthreads();
    for (int base = 0; base < T; base += kEcThreads) {
        const int t = base + tid;
        const uint32_t u = (t < T) ? key(t) : 0u;
        const bool tie = (t < T) && (u == kth);
        const bool above = (t < T) && (u > kth);
        const uint32_t tb = __ballot_sync(kFullMask, tie);
        if (lane == 0)
            s_tie[warp] = __popc(tb);
        __syncthreads();
        int tie_before = s_run[1] + __popc(tb & lanemask_lt());
        for (int w = 0; w < warp; ++w)
            tie_before += s_tie[w];
        const bool take = above || (tie && tie_before < ties);
        const uint32_t sb = __ballot_sync(kFullMask, take);
        if (lane == 0)
            s_take[warp] = __popc(sb);
        __syncthreads();
        int pos = s_run[0] + __popc(sb & lanemask_lt());
        for (int w = 0; w < warp; ++w)
            pos += s_take[w];
        if (take) {
            tokens[(size_t)e * K + pos] = t;
            weights[(size_t)e * K + pos] = __uint_as_float(u);
        }
        __syncthreads();
        if (tid == 0) {
            int nt = 0, nk = 0;
            for (int w = 0; w < kEcThreads / 32; ++w) {
                nt += s_tie[w];
                nk += s_take[w];
            }
            s_run[0] += nk;
            s_run[1] += nt;
        }
        __syncthreads();
    }
    // layout for the grouped GEMMs: expert e owns rows [e K, (e + 1) K)
    const int nt = (K + kBlockM - 1) / kBlockM;
    if (tid == 0) {
        offsets[e] = e * K;
        mt_first[e] = e * nt;   // plain expert order: one part, bands per expert
        if (e == E - 1) {
            offsets[E] = E * K;
            *num_mt = E * nt;
            mt_first[E] = E * nt;
        }
    }
    const int rem = K - (nt - 1) * kBlockM;
    for (int i = tid; i < nt; i += kEcThreads) {
        mt_row0[e * nt + i] = e * K + i * kBlockM;
        mt_group[e * nt + i] = e | ((i == nt - 1 && rem <= 64) ? kHalfTileBit : 0);
    }
}

// ---------------------------------------------------------------- gather + zero
// Row r < E K: x_perm[r] = x[tokens[r]]; row t < T (when zero_out): out[t] = 0.
__global__ void __launch_bounds__(256) k_ec_gather(const uint4 *__restrict__ x,
                                                   const int32_t *__restrict__ tokens, int rows,
                                                   int T, int d, uint4 *__restrict__ x_perm,
                                                   float4 *__restrict__ out_zero)
{
    const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r < rows) {
        const int t = tokens[r];
        const int nv = d / 8;
        for (int c = lane; c < nv; c += 32)
            x_perm[(size_t)r * nv + c] = x[(size_t)t * nv + c];
    }
    if (out_zero && r < T) {
        const int nv = d / 4;
        for (int c = lane; c < nv; c += 32)
            out_zero[(size_t)r * nv + c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------- host side
int launch_softmax_rows(const moe_shape_t &s, const float *logits, float *scores,
                        uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int blocks = (s.T + 7) / 8, vpl = (s.E + 31) / 32;
    if (vpl <= 1)
        k_softmax_rows<1><<<blocks, 256, 0, st>>>(logits, s.T, s.E, scores, status);
    else if (vpl <= 2)
        k_softmax_rows<2><<<blocks, 256, 0, st>>>(logits, s.T, s.E, scores, status);
    else if (vpl <= 4)
        k_softmax_rows<4><<<blocks, 256, 0, st>>>(logits, s.T, s.E, scores, status);
    else
        k_softmax_rows<8><<<blocks, 256, 0, st>>>(logits, s.T, s.E, scores, status);
    return launched();
}

int launch_ec_select(const moe_shape_t &s, int K, const float *scores, int32_t *tokens,
                     float *weights, int32_t *offsets, int32_t *mt_row0, int32_t *mt_group,
                     int32_t *num_mt, int32_t *mt_first, uint32_t *status, cudaStream_t st)
{
    if (s.T == 0 || K == 0)
        return MOE_OK;
    k_ec_select<<<s.E, kEcThreads, 0, st>>>(scores, s.T, s.E, K, tokens, weights, offsets, mt_row0,
                                            mt_group, num_mt, mt_first, status);
    return launched();
}

int launch_ec_gather(const moe_shape_t &s, int rows, const uint16_t *x, const int32_t *tokens,
                     uint16_t *x_perm, float *out_zero, cudaStream_t st)
{
    const int n = std::max(rows, out_zero ? s.T : 0);
    if (n == 0)
        return MOE_OK;
    k_ec_gather<<<(n + 7) / 8, 256, 0, st>>>(reinterpret_cast<const uint4 *>(x), tokens, rows, s.T,
                                             s.d, reinterpret_cast<uint4 *>(x_perm),
                                             reinterpret_cast<float4 *>(out_zero));
    return launched();
}

} // namespace moe
