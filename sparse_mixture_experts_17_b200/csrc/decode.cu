// decode.cu -- the small-T forward: stream only the chosen experts' weights.
//
// "Faster writing: run only the chosen experts; uncap the large profile"
// (mini-AGI) describes the failure this path avoids: a single-token forward
// that multiplied against every expert on the card read all their weights to
// use top_k of them. "perf(moe): route granite-4.0-h single-token MoE through
// the fused kernel" (mlxcel) routes one-token decode to a fused kernel fed by
// the router's top-k indices and renormalised scores. Here the chosen experts
// are known only on the device, so every CTA rebuilds the (tiny) plan in
// shared memory from topk_idx, and the weight stream is spread over all SMs.
//
// Routing (k_dec_route): one CTA computes the T x E logits (warps over
// experts, lanes over d) and then the top-k (one warp per token), when W_g is
// small; otherwise k_dec_router (one warp per expert) feeds k_topk.
// The plan applies the capacity (in the same rank order as the histogram
// kernel), so a dropped assignment reads no weights and adds nothing.
// Phase 1 (k_dec_w13): work unit = one SwiGLU column c of one chosen expert:
//   h[a, c] = bf16(silu(W1_e[c] . x_t) * (W3_e[c] . x_t)) for every
//   assignment a = (t, j) routed to e. Each unit streams the gate row and the
//   up row once (2 * d * 2 bytes), dotted against the routed tokens' x (L1).
// Phase 2 (k_dec_w2): work unit = one output row r:
//   out[t, r] = sum over the chosen experts e (ascending), then the shared
//   expert, of w[a] * (W2_e[r] . h[a]). Each unit streams W2_e[r] once per
//   chosen expert; h is L1/L2 resident. Fixed order: deterministic.
// The kernels are instantiated for MAXT in {1, 2, 4, 8, 16} >= T, the most
// assignments one expert can have (a token picks an expert at most once), so
// the per-token accumulators stay in registers and the code stays small.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "mxfp8.cuh"
#include "nvfp4.cuh"
#include "decode_split.cuh"
#include "topk.cuh"

namespace moe {

constexpr int kDecMaxA = MOE_DECODE_MAX_T * MOE_MAX_K;   // 256 assignments

struct DecPlanSmem {
    int U;                        // chosen experts (distinct)
    int uniq[MOE_MAX_E];          // ascending expert ids
    int ustart[MOE_MAX_E + 1];    // their assignment ranges in `list`
    int list[kDecMaxA];           // assignment ids a = t*k + j, by expert then token
    int cnt[MOE_MAX_E];
    int start[MOE_MAX_E];
};

// Rank of assignment a among the assignments to the same expert that come
// before it in the capacity order: row-major (t, j), or slot-major (j, t).
__device__ __forceinline__ int plan_rank(const int32_t *__restrict__ idx, int A, int k, int a,
                                         int slot_major)
{
    const int e = idx[a];
    int r = 0;
    if (!slot_major) {
        for (int b = 0; b < a; ++b)
            r += (idx[b] == e);
    } else {
        const int ja = a % k;
        for (int b = 0; b < A; ++b) {
            const int jb = b % k;
            r += (idx[b] == e) && (jb < ja || (jb == ja && b < a));
        }
    }
    return r;
}

// Every thread of the CTA participates; ends with __syncthreads(). An
// assignment whose rank reaches the capacity C (> 0) is dropped: it is in no
// expert's list, so it gets no h row and adds nothing to out.
__device__ void build_plan(DecPlanSmem &P, const int32_t *__restrict__ idx, int T, int E, int k,
                           int C, int slot_major, uint32_t *status)
{
    const int A = T * k;
    for (int e = threadIdx.x; e < MOE_MAX_E; e += blockDim.x)
        P.cnt[e] = 0;
    __syncthreads();
    for (int a = threadIdx.x; a < A; a += blockDim.x) {
        const int e = idx[a];
        if (e < 0 || e >= E) {
            if (blockIdx.x == 0)
                flag_status(status, MOE_ERR_BAD_EXPERT);
            continue;
        }
        if (C > 0 && plan_rank(idx, A, k, a, slot_major) >= C)
            continue;
        atomicAdd(&P.cnt[e], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0, u = 0;
        for (int e = 0; e < E; ++e) {
            P.start[e] = run;
            if (P.cnt[e] > 0) {
                P.uniq[u] = e;
                P.ustart[u] = run;
                ++u;
            }
            run += P.cnt[e];
        }
        P.ustart[u] = run;
        P.U = u;
    }
    __syncthreads();
    // each kept assignment at its rank within its expert's list
    for (int a = threadIdx.x; a < A; a += blockDim.x) {
        const int e = idx[a];
        if (e < 0 || e >= E)
            continue;
        const int r = plan_rank(idx, A, k, a, slot_major);
        if (C > 0 && r >= C)
            continue;
        P.list[P.start[e] + r] = a;
    }
    __syncthreads();
}

__device__ __forceinline__ float dot8(uint4 w, uint4 x, float acc)
{
    acc = fmaf(bf16lo(w.x), bf16lo(x.x), acc);
    acc = fmaf(bf16hi(w.x), bf16hi(x.x), acc);
    acc = fmaf(bf16lo(w.y), bf16lo(x.y), acc);
    acc = fmaf(bf16hi(w.y), bf16hi(x.y), acc);
    acc = fmaf(bf16lo(w.z), bf16lo(x.z), acc);
    acc = fmaf(bf16hi(w.z), bf16hi(x.z), acc);
    acc = fmaf(bf16lo(w.w), bf16lo(x.w), acc);
    acc = fmaf(bf16hi(w.w), bf16hi(x.w), acc);
    return acc;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(kFullMask, v, off);
    return v;
}

// ---------------------------------------------------------------- routing for small T

// One warp per expert: logits[t, e] = Wg[e] . x[t] + bias[e] for all t < T.
template <int MAXT>
__global__ void __launch_bounds__(256) k_dec_router(const uint16_t *__restrict__ x,
                                                    const uint16_t *__restrict__ Wg,
                                                    const float *__restrict__ bias, int T, int d,
                                                    int E, float *__restrict__ logits)
{
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const int nv = d / 8;
    for (int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; e < E; e += nwarps) {
        float acc[MAXT];
#pragma unroll
        for (int t = 0; t < MAXT; ++t)
            acc[t] = 0.f;
        const uint4 *wr = reinterpret_cast<const uint4 *>(Wg + (size_t)e * d);
        for (int c = lane; c < nv; c += 32) {
            const uint4 wv = ld_stream_v4(wr + c);
#pragma unroll
            for (int t = 0; t < MAXT; ++t)
                if (t < T)
                    acc[t] = dot8(wv, __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * d) + c), acc[t]);
        }
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            if (t < T) {
                const float s = warp_sum(acc[t]);
                if (lane == 0)
                    logits[(size_t)t * E + e] = s + (bias ? bias[e] : 0.f);
            }
        }
    }
}

// Router and top-k in one CTA of 512 threads, for W_g up to kFusedRouteBytes.
// Work item = (expert e, slice of d): with E < 16 each expert's row is split
// into 16/E slices so all 16 warps stream W_g; each lane keeps eight 16-byte
// loads in flight. Partial dot products meet in shared memory, then warp t
// selects token t's experts.
constexpr size_t kFusedRouteBytes = 256 * 1024;

template <int MAXT, int VPL>
__global__ void __launch_bounds__(512) k_dec_route(const uint16_t *__restrict__ x,
                                                   const uint16_t *__restrict__ Wg,
                                                   const float *__restrict__ bias, int T, int d,
                                                   int E, int k, float *__restrict__ logits,
                                                   int32_t *__restrict__ idx,
                                                   float *__restrict__ w, int32_t *counter_to_zero,
                                                   uint32_t *status)
{
    __shared__ float part[MAXT * 256];   // [t][e * S + slice], E * S <= 256
    pdl_trigger();   // the weight-streaming kernel may be scheduled on the other SMs
    if (counter_to_zero && threadIdx.x == 0)
        *counter_to_zero = 0;   // re-arms the histogram's ticket for a following permute
    __shared__ float sl[MAXT * MOE_MAX_E];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = d / 8;
    const int S = E < 16 ? 16 / E : 1;
    const int slice = (nv + S - 1) / S;
    for (int item = warp; item < E * S; item += 16) {
        const int e = item / S, sidx = item - e * S;
        const int c0 = sidx * slice, c1 = min(nv, c0 + slice);
        float acc[MAXT];
#pragma unroll
        for (int t = 0; t < MAXT; ++t)
            acc[t] = 0.f;
        const uint4 *wr = reinterpret_cast<const uint4 *>(Wg + (size_t)e * d);
        // eight 16-byte loads of W_g per lane in flight (a 2048-element slice
        // in one round trip), and for T <= 2 the matching x loads with them
        for (int cb = c0; cb < c1; cb += 256) {
            uint4 wv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = cb + lane + 32 * i;
                if (c < c1)
                    wv[i] = ld_stream_v4(wr + c);
            }
            if (MAXT <= 2) {
                uint4 xv[MAXT][8];
#pragma unroll
                for (int t = 0; t < MAXT; ++t)
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int c = cb + lane + 32 * i;
                        if (t < T && c < c1)
                            xv[t][i] = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * d) + c);
                    }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int c = cb + lane + 32 * i;
                    if (c >= c1)
                        continue;
#pragma unroll
                    for (int t = 0; t < MAXT; ++t)
                        if (t < T)
                            acc[t] = dot8(wv[i], xv[t][i], acc[t]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int c = cb + lane + 32 * i;
                    if (c >= c1)
                        continue;
#pragma unroll
                    for (int t = 0; t < MAXT; ++t)
                        if (t < T)
                            acc[t] = dot8(wv[i], __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * d) + c), acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            if (t < T) {
                const float v = warp_sum(acc[t]);
                if (lane == 0)
                    part[t * 256 + item] = v;
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * E; i += blockDim.x) {
        const int t = i / E, e = i - t * E;
        float v = bias ? bias[e] : 0.f;
        for (int q = 0; q < S; ++q)
            v += part[t * 256 + e * S + q];
        sl[t * E + e] = v;
        logits[(size_t)t * E + e] = v;
    }
    __syncthreads();
    if (warp < T)
        warp_topk_row<VPL>(sl + warp * E, E, k, idx + (size_t)warp * k, w + (size_t)warp * k,
                           status);
}

// ---------------------------------------------------------------- phase 1: W1/W3 + SwiGLU
constexpr int kDecUnroll = 4;

template <int MAXT>
__global__ void __launch_bounds__(256, (MAXT <= 2) ? 4 : 2)
    k_dec_w13(const uint16_t *__restrict__ x, const int32_t *__restrict__ idx, int T, int d,
              int d_ff, int E, int k, int C, int slot_major, const uint16_t *__restrict__ W13,
              int d_ff_s,
              const uint16_t *__restrict__ W13s, uint16_t *__restrict__ Hdec,
              uint16_t *__restrict__ Hs, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    pdl_wait();      // topk_idx comes from the routing kernel
    pdl_trigger();
    build_plan(P, idx, T, E, k, C, slot_major, status);
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const long long routed_units = (long long)P.U * d_ff;
    const long long units = routed_units + (W13s ? d_ff_s : 0);
    const int nv = d / 8;
    for (long long unit = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; unit < units;
         unit += nwarps) {
        const uint4 *gate, *up;
        int a0, na, c, ldh;
        uint16_t *hout;
        const bool shared = unit >= routed_units;
        if (!shared) {
            const int u = (int)(unit / d_ff);
            c = (int)(unit - (long long)u * d_ff);
            const int e = P.uniq[u];
            const size_t rbase = (size_t)e * 2 * d_ff + (size_t)(c / 128) * 256 + (c % 128);
            gate = reinterpret_cast<const uint4 *>(W13 + rbase * d);
            up = reinterpret_cast<const uint4 *>(W13 + (rbase + 128) * d);
            a0 = P.ustart[u];
            na = P.ustart[u + 1] - a0;
            hout = Hdec;
            ldh = d_ff;
        } else {
            c = (int)(unit - routed_units);
            const size_t rbase = (size_t)(c / 128) * 256 + (c % 128);
            gate = reinterpret_cast<const uint4 *>(W13s + rbase * d);
            up = reinterpret_cast<const uint4 *>(W13s + (rbase + 128) * d);
            a0 = 0;
            na = T;
            hout = Hs;
            ldh = d_ff_s;
        }
        const uint4 *xr[MAXT];
#pragma unroll
        for (int s = 0; s < MAXT; ++s)
            xr[s] = reinterpret_cast<const uint4 *>(
                x + (size_t)((s < na) ? (shared ? s : P.list[a0 + s] / k) : 0) * d);
        float ag[MAXT], au[MAXT];
#pragma unroll
        for (int s = 0; s < MAXT; ++s)
            ag[s] = au[s] = 0.f;
        for (int cb = 0; cb < nv; cb += 32 * kDecUnroll) {
            uint4 wg[kDecUnroll], wu[kDecUnroll];
#pragma unroll
            for (int i = 0; i < kDecUnroll; ++i) {
                const int ci = cb + lane + 32 * i;
                if (ci < nv) {
                    wg[i] = ld_stream_v4(gate + ci);
                    wu[i] = ld_stream_v4(up + ci);
                }
            }
#pragma unroll
            for (int i = 0; i < kDecUnroll; ++i) {
                const int ci = cb + lane + 32 * i;
                if (ci >= nv)
                    continue;
#pragma unroll
                for (int s = 0; s < MAXT; ++s) {
                    if (s < na) {
                        const uint4 xv = __ldg(xr[s] + ci);
                        ag[s] = dot8(wg[i], xv, ag[s]);
                        au[s] = dot8(wu[i], xv, au[s]);
                    }
                }
            }
        }
#pragma unroll
        for (int s = 0; s < MAXT; ++s) {
            if (s < na) {
                const float g = warp_sum(ag[s]);
                const float uu = warp_sum(au[s]);
                if (lane == 0) {
                    const int row = shared ? s : P.list[a0 + s];
                    const __nv_bfloat16 hb = __float2bfloat16_rn(silu_mul(g, uu));
                    hout[(size_t)row * ldh + c] = *reinterpret_cast<const uint16_t *>(&hb);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- phase 2: W2 + combine
// Work item = (output row r, source): one chosen expert's W2_e[r], or the
// shared expert's row, streamed once by one warp. A CTA takes RG consecutive
// rows at a time (RG * n_src items, n_src = chosen experts + shared; RG = 8 /
// n_src, at least 1), its eight warps take the items, and each item leaves its
// per-token contribution w * (W2_e[r] . h) in shared memory; the CTA then adds
// the sources of each row in a fixed order (ascending expert, then the shared
// expert): deterministic. Splitting a row's sources over warps doubles (at
// top-2) the streams in flight against one warp per row.
// At MAXT = 1 the weight stream is software-pipelined (two 16-byte loads per
// lane in flight while two are consumed); at MAXT >= 2 a batch of eight (four
// above MAXT = 2) loads is issued and then consumed.
constexpr int kDecW2MaxItems = MOE_MAX_E + 8;

template <int MAXT>
__global__ void __launch_bounds__(256, (MAXT <= 2) ? 4 : 2)
    k_dec_w2(const int32_t *__restrict__ idx, const float *__restrict__ topk_w, int T, int d,
             int d_ff, int E, int k, int C, int slot_major, const uint16_t *__restrict__ W2,
             int d_ff_s,
             const uint16_t *__restrict__ W2s, const uint16_t *__restrict__ Hdec,
             const uint16_t *__restrict__ Hs, float *__restrict__ out, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    __shared__ float contrib[kDecW2MaxItems][MAXT];
    pdl_wait();      // h comes from the w1/w3 kernel
    build_plan(P, idx, T, E, k, C, slot_major, status);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_src = P.U + (W2s ? 1 : 0);
    if (n_src == 0) {   // every assignment dropped and no shared expert: out = 0
        for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)T * d;
             i += (long long)gridDim.x * blockDim.x)
            out[i] = 0.f;
        return;
    }
    const int RG = max(1, 8 / n_src);
    const int items = RG * n_src;   // <= max(8, n_src) <= kDecW2MaxItems
    for (int r0 = blockIdx.x * RG; r0 < d; r0 += gridDim.x * RG) {
        for (int it = warp; it < items; it += 8) {
            const int r = r0 + it / n_src, u = it % n_src;
            float tok[MAXT];
#pragma unroll
            for (int t = 0; t < MAXT; ++t)
                tok[t] = 0.f;
            if (r < d) {
                const bool shared = (u == P.U);
                const int ff = shared ? d_ff_s : d_ff;
                const uint4 *wrow = reinterpret_cast<const uint4 *>(
                    shared ? W2s + (size_t)r * d_ff_s : W2 + ((size_t)P.uniq[u] * d + r) * d_ff);
                const int a0 = shared ? 0 : P.ustart[u];
                const int na = shared ? T : P.ustart[u + 1] - a0;
                const uint16_t *hb = shared ? Hs : Hdec;
                const uint4 *hr[MAXT];
                int tk[MAXT];
                float wt[MAXT];
#pragma unroll
                for (int s = 0; s < MAXT; ++s) {
                    const int a = (s < na) ? (shared ? s : P.list[a0 + s]) : 0;
                    hr[s] = reinterpret_cast<const uint4 *>(hb + (size_t)a * ff);
                    tk[s] = shared ? s : a / k;
                    wt[s] = (s < na) ? (shared ? 1.f : topk_w[a]) : 0.f;
                }
                const int nv = ff / 8;
                float pa[MAXT];
#pragma unroll
                for (int s = 0; s < MAXT; ++s)
                    pa[s] = 0.f;
                if constexpr (MAXT == 1) {
                    constexpr int UNR = 2;
                    uint4 cur[UNR], nxt[UNR];
#pragma unroll
                    for (int i = 0; i < UNR; ++i) {
                        const int ci = lane + 32 * i;
                        if (ci < nv)
                            cur[i] = ld_stream_v4(wrow + ci);
                    }
                    for (int cb = 0; cb < nv; cb += 32 * UNR) {
                        const int nb = cb + 32 * UNR;
#pragma unroll
                        for (int i = 0; i < UNR; ++i) {
                            const int ci = nb + lane + 32 * i;
                            if (ci < nv)
                                nxt[i] = ld_stream_v4(wrow + ci);
                        }
#pragma unroll
                        for (int i = 0; i < UNR; ++i) {
                            const int ci = cb + lane + 32 * i;
                            if (ci < nv && na > 0)
                                pa[0] = dot8(cur[i], __ldg(hr[0] + ci), pa[0]);
                        }
#pragma unroll
                        for (int i = 0; i < UNR; ++i)
                            cur[i] = nxt[i];
                    }
                } else {
                    constexpr int UNR = (MAXT <= 2) ? 8 : kDecUnroll;
                    for (int cb = 0; cb < nv; cb += 32 * UNR) {
                        uint4 wv[UNR];
#pragma unroll
                        for (int i = 0; i < UNR; ++i) {
                            const int ci = cb + lane + 32 * i;
                            if (ci < nv)
                                wv[i] = ld_stream_v4(wrow + ci);
                        }
#pragma unroll
                        for (int i = 0; i < UNR; ++i) {
                            const int ci = cb + lane + 32 * i;
                            if (ci >= nv)
                                continue;
#pragma unroll
                            for (int s = 0; s < MAXT; ++s)
                                if (s < na)
                                    pa[s] = dot8(wv[i], __ldg(hr[s] + ci), pa[s]);
                        }
                    }
                }
                // this source's weighted contribution to each token of row r
#pragma unroll
                for (int s = 0; s < MAXT; ++s) {
                    if (s < na) {
                        const float v = wt[s] * warp_sum(pa[s]);
#pragma unroll
                        for (int tt = 0; tt < MAXT; ++tt)
                            if (tt == tk[s])
                                tok[tt] += v;
                    }
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < MAXT; ++t)
                    contrib[it][t] = tok[t];
            }
        }
        __syncthreads();
        // fixed-order sum of each row's sources
        for (int q = threadIdx.x; q < RG * T; q += blockDim.x) {
            const int j = q / T, t = q - j * T;
            const int r = r0 + j;
            if (r < d) {
                float v = 0.f;
                for (int u = 0; u < n_src; ++u)
                    v += contrib[j * n_src + u][t];
                out[(size_t)t * d + r] = v;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- MXFP8 experts
// The same two phases on MXFP8 weights: a lane's 16-byte load carries 16 E4M3
// codes (twice the elements of a bf16 load) and each 32-element block adds one
// E8M0 byte, so a chosen expert streams 8.25 bits per weight instead of 16.
// The activations arrive already through MXFP8 and back (exact in bf16): x
// before phase 1, h between the phases. Phase 1 writes h in fp32.

// sum over 16 elements of E4M3 code value * bf16 value (fp32)
__device__ __forceinline__ float dot16_mx(uint4 w, uint4 xa, uint4 xb, float acc)
{
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    const uint32_t xx[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 lo = mx_decode2((uint16_t)(ww[i] & 0xffffu));
        const float2 hi = mx_decode2((uint16_t)(ww[i] >> 16));
        acc = fmaf(lo.x, bf16lo(xx[2 * i]), acc);
        acc = fmaf(lo.y, bf16hi(xx[2 * i]), acc);
        acc = fmaf(hi.x, bf16lo(xx[2 * i + 1]), acc);
        acc = fmaf(hi.y, bf16hi(xx[2 * i + 1]), acc);
    }
    return acc;
}

template <int MAXT>
__global__ void __launch_bounds__(256, (MAXT <= 2) ? 4 : 2)
    k_dec_w13_mx(const uint16_t *__restrict__ xdq, const int32_t *__restrict__ idx, int T, int d,
                 int d_ff, int E, int k, int C, int slot_major, const uint8_t *__restrict__ W13q,
                 const uint8_t *__restrict__ W13sf, int d_ff_s, const uint8_t *__restrict__ W13s_q,
                 const uint8_t *__restrict__ W13s_sf, float *__restrict__ H32,
                 float *__restrict__ Hs32, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    pdl_wait();
    pdl_trigger();
    build_plan(P, idx, T, E, k, C, slot_major, status);
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const long long routed_units = (long long)P.U * d_ff;
    const long long units = routed_units + (W13s_q ? d_ff_s : 0);
    const int nv = d / 16;
    for (long long unit = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; unit < units;
         unit += nwarps) {
        const uint8_t *qb, *sb;
        int a0, na, c, ldh;
        float *hout;
        const bool shared = unit >= routed_units;
        size_t prow;
        if (!shared) {
            const int u = (int)(unit / d_ff);
            c = (int)(unit - (long long)u * d_ff);
            // packed gate row of h column c; the up row is 64 rows further
            prow = (size_t)P.uniq[u] * 2 * d_ff + (size_t)(c / 64) * 128 + (c % 64);
            qb = W13q;
            sb = W13sf;
            a0 = P.ustart[u];
            na = P.ustart[u + 1] - a0;
            hout = H32;
            ldh = d_ff;
        } else {
            c = (int)(unit - routed_units);
            prow = (size_t)(c / 64) * 128 + (c % 64);
            qb = W13s_q;
            sb = W13s_sf;
            a0 = 0;
            na = T;
            hout = Hs32;
            ldh = d_ff_s;
        }
        const uint4 *gate = reinterpret_cast<const uint4 *>(qb + prow * d);
        const uint4 *up = reinterpret_cast<const uint4 *>(qb + (prow + 64) * d);
        // scale atoms of the gate and up rows (tile = row / 128)
        const long long gt = (long long)(prow >> 7), ut = (long long)((prow + 64) >> 7);
        const int gm = (int)(prow & 127), um = (int)((prow + 64) & 127);
        const uint4 *xr[MAXT];
#pragma unroll
        for (int s = 0; s < MAXT; ++s)
            xr[s] = reinterpret_cast<const uint4 *>(
                xdq + (size_t)((s < na) ? (shared ? s : P.list[a0 + s] / k) : 0) * d);
        float ag[MAXT], au[MAXT];
#pragma unroll
        for (int s = 0; s < MAXT; ++s)
            ag[s] = au[s] = 0.f;
        for (int cb = 0; cb < nv; cb += 32 * kDecUnroll) {
            uint4 wg[kDecUnroll], wu[kDecUnroll];
            uint8_t sg[kDecUnroll], su[kDecUnroll];
#pragma unroll
            for (int i = 0; i < kDecUnroll; ++i) {
                const int ci = cb + lane + 32 * i;
                if (ci < nv) {
                    wg[i] = ld_stream_v4(gate + ci);
                    wu[i] = ld_stream_v4(up + ci);
                    sg[i] = __ldg(sb + sf_atom_offset(gt, gm, ci >> 1, d));
                    su[i] = __ldg(sb + sf_atom_offset(ut, um, ci >> 1, d));
                }
            }
#pragma unroll
            for (int i = 0; i < kDecUnroll; ++i) {
                const int ci = cb + lane + 32 * i;
                if (ci >= nv)
                    continue;
                const float fg = mx_scale_value(sg[i]), fu = mx_scale_value(su[i]);
#pragma unroll
                for (int s = 0; s < MAXT; ++s) {
                    if (s < na) {
                        const uint4 xa = __ldg(xr[s] + 2 * ci), xb = __ldg(xr[s] + 2 * ci + 1);
                        ag[s] = fmaf(fg, dot16_mx(wg[i], xa, xb, 0.f), ag[s]);
                        au[s] = fmaf(fu, dot16_mx(wu[i], xa, xb, 0.f), au[s]);
                    }
                }
            }
        }
#pragma unroll
        for (int s = 0; s < MAXT; ++s) {
            if (s < na) {
                const float g = warp_sum(ag[s]);
                const float uu = warp_sum(au[s]);
                if (lane == 0) {
                    const int row = shared ? s : P.list[a0 + s];
                    hout[(size_t)row * ldh + c] = silu_mul(g, uu);
                }
            }
        }
    }
}

template <int MAXT>
__global__ void __launch_bounds__(256, (MAXT <= 2) ? 4 : 2)
    k_dec_w2_mx(const int32_t *__restrict__ idx, const float *__restrict__ topk_w, int T, int d,
                int d_ff, int E, int k, int C, int slot_major, const uint8_t *__restrict__ W2q,
                const uint8_t *__restrict__ W2sf, int d_ff_s, const uint8_t *__restrict__ W2s_q,
                const uint8_t *__restrict__ W2s_sf, const uint16_t *__restrict__ Hdq,
                const uint16_t *__restrict__ Hsdq, float *__restrict__ out, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    pdl_wait();      // h comes from the quantization between the phases
    build_plan(P, idx, T, E, k, C, slot_major, status);
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const int n_src = P.U + (W2s_q ? 1 : 0);
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < d; r += nwarps) {
        float acc[MAXT];
#pragma unroll
        for (int t = 0; t < MAXT; ++t)
            acc[t] = 0.f;
        for (int u = 0; u < n_src; ++u) {
            const bool shared = (u == P.U);
            const int ff = shared ? d_ff_s : d_ff;
            const size_t wr = shared ? (size_t)r : (size_t)P.uniq[u] * d + r;
            const uint4 *wrow = reinterpret_cast<const uint4 *>((shared ? W2s_q : W2q) + wr * ff);
            const uint8_t *wsf = shared ? W2s_sf : W2sf;
            const long long wt_tile = (long long)(wr >> 7);
            const int wt_m = (int)(wr & 127);
            const int a0 = shared ? 0 : P.ustart[u];
            const int na = shared ? T : P.ustart[u + 1] - a0;
            const uint16_t *hb = shared ? Hsdq : Hdq;
            const uint4 *hr[MAXT];
            int tk[MAXT];
            float wt[MAXT];
#pragma unroll
            for (int s = 0; s < MAXT; ++s) {
                const int a = (s < na) ? (shared ? s : P.list[a0 + s]) : 0;
                hr[s] = reinterpret_cast<const uint4 *>(hb + (size_t)a * ff);
                tk[s] = shared ? s : a / k;
                wt[s] = (s < na) ? (shared ? 1.f : topk_w[a]) : 0.f;
            }
            const int nv = ff / 16;
            float pa[MAXT];
#pragma unroll
            for (int s = 0; s < MAXT; ++s)
                pa[s] = 0.f;
            for (int cb = 0; cb < nv; cb += 32 * kDecUnroll) {
                uint4 wv[kDecUnroll];
                uint8_t sc[kDecUnroll];
#pragma unroll
                for (int i = 0; i < kDecUnroll; ++i) {
                    const int ci = cb + lane + 32 * i;
                    if (ci < nv) {
                        wv[i] = ld_stream_v4(wrow + ci);
                        sc[i] = __ldg(wsf + sf_atom_offset(wt_tile, wt_m, ci >> 1, ff));
                    }
                }
#pragma unroll
                for (int i = 0; i < kDecUnroll; ++i) {
                    const int ci = cb + lane + 32 * i;
                    if (ci >= nv)
                        continue;
                    const float f = mx_scale_value(sc[i]);
#pragma unroll
                    for (int s = 0; s < MAXT; ++s)
                        if (s < na)
                            pa[s] = fmaf(f, dot16_mx(wv[i], __ldg(hr[s] + 2 * ci),
                                                     __ldg(hr[s] + 2 * ci + 1), 0.f),
                                         pa[s]);
                }
            }
#pragma unroll
            for (int s = 0; s < MAXT; ++s) {
                if (s < na) {
#pragma unroll
                    for (int tt = 0; tt < MAXT; ++tt)
                        if (tt == tk[s])
                            acc[tt] = fmaf(wt[s], pa[s], acc[tt]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            if (t < T) {
                const float s = warp_sum(acc[t]);
                if (lane == 0)
                    out[(size_t)t * d + r] = s;
            }
        }
    }
}

// ---------------------------------------------------------------- NVFP4 experts (T <= 2)
// The same two phases on NVFP4 weights (packed E2M1 codes, an E4M3 scale per
// 16 elements in the atom layout, a global scale per expert), with x and h
// quantized to NVFP4 as the tensor-core chain quantizes them and handed over
// as their codes' values in f16 plus each block's scale value in fp32.
//
// One 16-element block is a dot product of E2M1 values: every product is a
// multiple of 1/4 of magnitude <= 36, so each f16 lane of the half2
// accumulator (8 products) stays a multiple of 1/4 below 288 and is exact in
// f16; the block sum is then scaled by s_w * s_x (two E4M3 values: exact in
// fp32) and accumulated in fp32. The global scales divide the row's sum once.

// Exact dot product of one 16-element block: the 8 code bytes (w0, w1; the
// first element in the low nibble) against 8 f16x2 values.
__device__ __forceinline__ float nv_block_dot(uint32_t w0, uint32_t w1, const uint4 &xa,
                                              const uint4 &xb)
{
    const uint32_t xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
    __half2 acc = __float2half2_rn(0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t wb = (j < 4 ? w0 : w1) >> (8 * (j & 3));
        acc = __hfma2(nv_pair_h2(wb), *reinterpret_cast<const __half2 *>(&xv[j]), acc);
    }
    const float2 f = __half22float2(acc);
    return f.x + f.y;
}

// One 16-byte chunk of a code row (32 elements = two blocks) against the
// same 32 values of x or h (f16, x[0..3]) and their two block scales: the sum
// over both blocks of the exact block dot times s_w(block) * s_x(block).
__device__ __forceinline__ float nv_chunk_dot(const uint4 &w, float sw0, float sw1, const uint4 (&x)[4],
                                              const float2 &xs)
{
    const float b0 = nv_block_dot(w.x, w.y, x[0], x[1]);
    const float b1 = nv_block_dot(w.z, w.w, x[2], x[3]);
    return fmaf(b1, sw1 * xs.y, b0 * (sw0 * xs.x));
}

// Phase 1, fed by the TMA. Work item = one 128-row tile of a source's packed
// W13: 64 gate and 64 up rows, i.e. h columns 64 t .. 64 t + 63 of source u
// (a chosen expert, or the shared expert after them). A producer thread
// streams the tile through a ring of K stages: 128 rows x 128 bytes of codes
// (256 elements, one TMA box) and the stage's four 512-byte scale atoms (one
// bulk copy); the copy engine keeps kNdStages stages in flight whatever the
// consumers' registers. Eight consumer warps own 16 rows each: lane l takes
// the 32-element chunk l % 8 of rows l / 8 + 4 j (j < 4), so one load of x's
// chunk serves eight rows and each 16-byte code read is conflict-free. At
// the end of a tile the eight lanes of a row reduce their sums, and the h
// columns are formed from the gate and up row sums in shared memory.
constexpr int kNdStages = 4;
constexpr int kNdStageBytes = 128 * 128;   // codes of one K stage (256 elements x 128 rows)
constexpr int kNdSfBytes = 4 * 512;        // its four scale atoms
constexpr int kNdConsumers = 8;            // consumer warps (16 rows each)
constexpr int kNdRowsPerLane = 128 / kNdConsumers / 4;
constexpr int kNdThreads = 32 * kNdConsumers + 32;   // the consumers, then the producer warp

template <int MAXT>
struct NdSmem {
    uint8_t code[kNdStages][kNdStageBytes];
    uint8_t sf[kNdStages][kNdSfBytes];
    uint64_t full[kNdStages], empty[kNdStages];
    float rowsum[128][MAXT];
    int abort;
};

// Bytes of NdSmem<MAXT> rounded up to 16 (x is staged after it).
template <int MAXT>
__host__ __device__ constexpr size_t nd_smem_bytes()
{
    return (sizeof(NdSmem<MAXT>) + 15) / 16 * 16;
}

__device__ __forceinline__ void nd_bulk_load(void *smem_dst, const void *src, uint32_t bytes,
                                             uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// named barrier of the consumer warps
__device__ __forceinline__ void nd_consumer_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kNdConsumers) : "memory");
}

template <int MAXT>
__global__ void __launch_bounds__(kNdThreads, 2)
    k_dec_w13_nv(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmS,
                 const uint16_t *__restrict__ xh, const float *__restrict__ xs, float x_gs,
                 const int32_t *__restrict__ idx, int T, int d, int d_ff, int E, int k, int C,
                 int slot_major, const uint8_t *__restrict__ W13sf,
                 const float *__restrict__ gs13, int d_ff_s, int has_shared,
                 const uint8_t *__restrict__ W13s_sf, const float *__restrict__ gs13s,
                 float *__restrict__ H32, float *__restrict__ Hs32, uint32_t *status)
{
    extern __shared__ uint8_t nd_raw[];
    NdSmem<MAXT> &S = *reinterpret_cast<NdSmem<MAXT> *>(
        (reinterpret_cast<uintptr_t>(nd_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ DecPlanSmem P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kNdStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kNdConsumers);
        }
        S.abort = 0;
        fence_mbar_init();
    }
    pdl_wait();
    pdl_trigger();
    build_plan(P, idx, T, E, k, C, slot_major, status);   // ends with __syncthreads
    // x (T rows of f16 values) and its block scales, staged in shared memory
    // once: every tile reads them again, and global loads there left the
    // consumers waiting on L2 latency at each stage
    uint4 *x_sm = reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(&S) + nd_smem_bytes<MAXT>());
    float *xs_sm = reinterpret_cast<float *>(x_sm + (size_t)T * (d / 8));
    for (int i = threadIdx.x; i < T * (d / 8); i += blockDim.x)
        x_sm[i] = __ldg(reinterpret_cast<const uint4 *>(xh) + i);
    for (int i = threadIdx.x; i < T * (d / 16); i += blockDim.x)
        xs_sm[i] = __ldg(xs + i);
    __syncthreads();
    volatile int *abort_flag = &S.abort;
    const int tpr = 2 * d_ff / 128;                        // tiles of a routed expert
    const int routed_items = P.U * tpr;
    const int items = routed_items + (has_shared ? 2 * d_ff_s / 128 : 0);
    const int nks = (d + 255) / 256;   // K stages of a tile; the last holds 128 or 256 elements

    if (warp == kNdConsumers) {
        if (lane == 0) {   // ---------------- producer
            uint32_t it = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
                const bool shared = item >= routed_items;
                const int t = shared ? item - routed_items : item % tpr;
                const long long row0 =
                    shared ? (long long)t * 128 : (long long)P.uniq[item / tpr] * 2 * d_ff + t * 128;
                const uint8_t *sfb = (shared ? W13s_sf : W13sf) + (size_t)(row0 / 128) * (d / 64) * 512;
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % kNdStages;
                    const uint32_t ph = (it / kNdStages) & 1u;
                    if (!mbar_wait(&S.empty[s], ph ^ 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    // a 128-element last stage: the TMA box still spans 128 bytes per
                    // row (the half past the row reads as zeros), the scales two atoms
                    const uint32_t sf_bytes = (uint32_t)min(256, d - ks * 256) / 64 * 512;
                    mbar_arrive_expect_tx(&S.full[s], kNdStageBytes + sf_bytes);
                    tma_load_2d(S.code[s], shared ? &tmS : &tmR, ks * 128, (int)row0, &S.full[s]);
                    nd_bulk_load(S.sf[s], sfb + (size_t)ks * kNdSfBytes, sf_bytes, &S.full[s]);
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                int never = 0;
                const uint32_t first = it >= kNdStages ? it - kNdStages : 0;
                for (uint32_t i = first; i < it; ++i)
                    mbar_wait(&S.full[i % kNdStages], (i / kNdStages) & 1u, &never, status);
            }
        }
        return;
    }
    // ---------------- consumers (warps 0 .. kNdConsumers - 1)
    const int c = lane & 7, rsub = lane >> 3;
    uint32_t it = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const bool shared = item >= routed_items;
        const int u = shared ? 0 : item / tpr;
        const int t = shared ? item - routed_items : item % tpr;
        const int a0 = shared ? 0 : P.ustart[u];
        const int na = shared ? T : P.ustart[u + 1] - a0;
        const float gsw = shared ? gs13s[0] : gs13[P.uniq[u]];
        const uint4 *xr[MAXT];
        const float2 *sr[MAXT];
#pragma unroll
        for (int q = 0; q < MAXT; ++q) {
            const int tok = (q < na) ? (shared ? q : P.list[a0 + q] / k) : 0;
            xr[q] = x_sm + (size_t)tok * (d / 8);
            sr[q] = reinterpret_cast<const float2 *>(xs_sm + (size_t)tok * (d / 16));
        }
        float acc[kNdRowsPerLane][MAXT];
#pragma unroll
        for (int j = 0; j < kNdRowsPerLane; ++j)
#pragma unroll
            for (int q = 0; q < MAXT; ++q)
                acc[j][q] = 0.f;
        for (int ks = 0; ks < nks; ++ks, ++it) {
            const int s = it % kNdStages;
            const uint32_t ph = (it / kNdStages) & 1u;
            const bool got = mbar_wait(&S.full[s], ph, abort_flag, status);
            // chunk c (elements ks * 256 + 32 c ..) lies inside the row
            if (got && ks * 256 + c * 32 < d) {
                // x's chunk c of this stage (32 values) and its two block scales
                uint4 xv[MAXT][4];
                float2 xsc[MAXT];
#pragma unroll
                for (int q = 0; q < MAXT; ++q) {
                    if (q < na) {
                        const int x4 = ks * 32 + c * 4;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            xv[q][i] = xr[q][x4 + i];
                        xsc[q] = sr[q][ks * 8 + c];
                    }
                }
#pragma unroll
                for (int j = 0; j < kNdRowsPerLane; ++j) {
                    const int r = warp * (4 * kNdRowsPerLane) + rsub + 4 * j;
                    const uint4 w = *reinterpret_cast<const uint4 *>(S.code[s] + r * 128 + c * 16);
                    // blocks 2c and 2c + 1 of this stage: K group c / 2, row r
                    const uint32_t sw = *reinterpret_cast<const uint16_t *>(
                        S.sf[s] + (c >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4 + 2 * (c & 1));
                    const float s0 = nv_scale_value(sw), s1 = nv_scale_value(sw >> 8);
#pragma unroll
                    for (int q = 0; q < MAXT; ++q)
                        if (q < na)
                            acc[j][q] += nv_chunk_dot(w, s0, s1, xv[q], xsc[q]);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&S.empty[s]);
        }
        // row sums: the eight lanes of a row differ in bits 0..2 of the lane id
        const float inv = 1.0f / (x_gs * gsw);
#pragma unroll
        for (int j = 0; j < kNdRowsPerLane; ++j)
#pragma unroll
            for (int q = 0; q < MAXT; ++q) {
                float v = acc[j][q];
                v += __shfl_xor_sync(kFullMask, v, 1);
                v += __shfl_xor_sync(kFullMask, v, 2);
                v += __shfl_xor_sync(kFullMask, v, 4);
                if (c == 0)
                    S.rowsum[warp * (4 * kNdRowsPerLane) + rsub + 4 * j][q] = v * inv;
            }
        nd_consumer_sync();
        // h columns 64 t + i: gate row i, up row 64 + i of the tile
        if (threadIdx.x < 64) {
            const int i = threadIdx.x;
#pragma unroll
            for (int q = 0; q < MAXT; ++q) {
                if (q < na) {
                    const float h = silu_mul(S.rowsum[i][q], S.rowsum[64 + i][q]);
                    if (shared)
                        Hs32[(size_t)q * d_ff_s + 64 * t + i] = h;
                    else
                        H32[(size_t)P.list[a0 + q] * d_ff + 64 * t + i] = h;
                }
            }
        }
        nd_consumer_sync();
    }
}

// Phase 2: one work unit = output row r: for each chosen expert (ascending),
// then the shared expert, stream W2_e[r] once and dot it with each of the
// expert's assignments' h rows; fixed order (deterministic).
template <int MAXT>
__global__ void __launch_bounds__(256, 2)
    k_dec_w2_nv(const int32_t *__restrict__ idx, const float *__restrict__ topk_w, int T, int d,
                int d_ff, int E, int k, int C, int slot_major, const uint8_t *__restrict__ W2q,
                const uint8_t *__restrict__ W2sf, const float *__restrict__ gs2, int d_ff_s,
                const uint8_t *__restrict__ W2s_q, const uint8_t *__restrict__ W2s_sf,
                const float *__restrict__ gs2s, const uint16_t *__restrict__ hh,
                const float *__restrict__ hsc, float h_gs, float *__restrict__ out,
                uint32_t *status)
{
    __shared__ DecPlanSmem P;
    pdl_wait();      // h comes from the quantization between the phases
    build_plan(P, idx, T, E, k, C, slot_major, status);
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const int n_src = P.U + (W2s_q ? 1 : 0);
    // shared-expert rows follow the T * k routed rows
    const uint16_t *hh_s = hh + (size_t)T * k * d_ff;
    const float *hsc_s = hsc + (size_t)T * k * (d_ff / 16);
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < d; r += nwarps) {
        float acc[MAXT];
#pragma unroll
        for (int t = 0; t < MAXT; ++t)
            acc[t] = 0.f;
        for (int u = 0; u < n_src; ++u) {
            const bool shared = (u == P.U);
            const int ff = shared ? d_ff_s : d_ff;
            const size_t wr = shared ? (size_t)r : (size_t)P.uniq[u] * d + r;
            const uint4 *wrow = reinterpret_cast<const uint4 *>((shared ? W2s_q : W2q) + wr * (ff / 2));
            const uint8_t *wsf = shared ? W2s_sf : W2sf;
            const long long wt_tile = (long long)(wr >> 7);
            const int wt_m = (int)(wr & 127);
            const int a0 = shared ? 0 : P.ustart[u];
            const int na = shared ? T : P.ustart[u + 1] - a0;
            const float inv = 1.0f / (h_gs * (shared ? gs2s[0] : gs2[P.uniq[u]]));
            const uint4 *hr[MAXT];
            const float2 *sr[MAXT];
            int tk[MAXT];
            float wt[MAXT];
#pragma unroll
            for (int s = 0; s < MAXT; ++s) {
                const int a = (s < na) ? (shared ? s : P.list[a0 + s]) : 0;
                hr[s] = reinterpret_cast<const uint4 *>((shared ? hh_s : hh) + (size_t)a * ff);
                sr[s] = reinterpret_cast<const float2 *>((shared ? hsc_s : hsc) + (size_t)a * (ff / 16));
                tk[s] = shared ? s : a / k;
                wt[s] = (s < na) ? (shared ? 1.f : topk_w[a]) * inv : 0.f;
            }
            const int nv = ff / 32;
            float pa[MAXT];
#pragma unroll
            for (int s = 0; s < MAXT; ++s)
                pa[s] = 0.f;
            constexpr int UNR = 8;
            for (int cb = 0; cb < nv; cb += 32 * UNR) {
                uint4 wv[UNR];
                uint32_t sc[UNR];
#pragma unroll
                for (int i = 0; i < UNR; ++i) {
                    const int ci = cb + lane + 32 * i;
                    if (ci < nv) {
                        wv[i] = ld_stream_v4(wrow + ci);
                        sc[i] = __ldg(reinterpret_cast<const uint16_t *>(
                            wsf + nv_sf_offset(wt_tile, wt_m, 2 * ci, ff)));
                    }
                }
#pragma unroll
                for (int i = 0; i < UNR; ++i) {
                    const int ci = cb + lane + 32 * i;
                    if (ci >= nv)
                        continue;
                    const float f0 = nv_scale_value(sc[i]), f1 = nv_scale_value(sc[i] >> 8);
#pragma unroll
                    for (int s = 0; s < MAXT; ++s)
                        if (s < na) {
                            const uint4 hv[4] = {__ldg(hr[s] + 4 * ci), __ldg(hr[s] + 4 * ci + 1),
                                                 __ldg(hr[s] + 4 * ci + 2), __ldg(hr[s] + 4 * ci + 3)};
                            pa[s] += nv_chunk_dot(wv[i], f0, f1, hv, __ldg(sr[s] + ci));
                        }
                }
            }
#pragma unroll
            for (int s = 0; s < MAXT; ++s) {
                if (s < na) {
#pragma unroll
                    for (int tt = 0; tt < MAXT; ++tt)
                        if (tt == tk[s])
                            acc[tt] = fmaf(wt[s], pa[s], acc[tt]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            if (t < T) {
                const float v = warp_sum(acc[t]);
                if (lane == 0)
                    out[(size_t)t * d + r] = v;
            }
        }
    }
}

// ---------------------------------------------------------------- NVFP4 decode w1/w3, tensor cores
// NVFP4 decode w1/w3 on the tensor cores: the chosen experts' weights are
// the M side of block-scaled MMAs (128 packed W13 rows per tile) and the
// tokens the N side (16 columns; rows past T are zeros), so the 4-bit codes
// are multiplied where they land in shared memory and no CUDA core converts
// them. Work item = one 128-row tile of a chosen expert's packed W13 (64 gate
// and 64 up rows: h columns 64 t .. 64 t + 63), or of the shared expert after
// them.
//
// Structure (one CTA per SM, 192 threads), as the block-scaled GEMM:
//   all        x quantized to NVFP4 (the prefill quantizer's arithmetic,
//              global scale gs_x) straight into the MMA's operand layout:
//              every K stage's 16 x 128-byte token tile (128-byte swizzle)
//              and its four scale atoms stay resident for the whole launch
//   warp 0     producer: per 256-element K stage, TMA of the 128 x 128-byte
//              weight tile (128-byte swizzle) and a bulk copy of its four
//              scale atoms, through a ring of nst stages
//   warp 1     TMEM (256 columns: two 16-column accumulators, then the
//              stages' scale columns); one thread copies both operands' scale atoms into
//              TMEM (32x128b.warpx4) and issues four M=128 N=16 K=64
//              kind::mxf4nvf4 MMAs per stage
//   warps 2-5  epilogue: the tile's 128 x 16 sums to shared memory, then
//              h[a, c] = silu(gate) * up for each assignment a of the tile's
//              expert, scaled by 1 / (gs_x gs_w), in fp32 (as the CUDA-core
//              decode kernel writes it for the w2 phase)
// Load balance: with G CTAs, the first items / G rounds are whole tiles; the
// R = items mod G tiles left over are cut along K into pieces (dt_split) so
// that the last round spreads over all CTAs. A piece writes its fp32 sums
// to `part`, and k_dec_w13_nvtc_fix adds a tile's pieces in piece order
// (deterministic) and forms its h columns.
// Every pipeline wait is bounded (mbar_wait); on expiry the roles unwind.
namespace {

constexpr int kDtMaxStages = 6;
constexpr int kDtN = 16;                  // token columns of an MMA
constexpr int kDtABytes = 128 * 128;      // weight codes of one K stage (256 elements x 128 rows)
constexpr int kDtBBytes = kDtN * 128;     // token codes of one K stage
constexpr int kDtSfBytes = 2048;          // four scale atoms per operand and stage
constexpr int kDtSfCols = 32;             // TMEM scale columns per stage (A's 16, then B's)
constexpr int kDtMaxRing = 6;             // ring stages: 2 x 16 accumulator + 6 x 32 scale columns <= 256

// Dynamic shared memory of k_dec_w13_nvtc (byte offsets from a 1024-aligned
// base; every operand region starts on a 1024-byte boundary):
//   a    [nst][128 x 128 B]  weight codes of a K stage
//   sfa  [nst][2 KB]         their scale atoms
//   xb   [nks][16 x 128 B]   the tokens' codes, every K stage (resident)
//   xsf  [nks][2 KB]         their scale atoms (resident)
//   d    [128][17] fp32      one tile's sums
//   hb   [16][64] fp32       one tile's h columns, per assignment (quantized
//                            to NVFP4 from here)
struct DtCarve {
    uint32_t a, sfa, xb, xsf, d, hb, total;
};

__host__ __device__ __forceinline__ DtCarve dt_carve(int nst, int nks)
{
    DtCarve c;
    c.a = 0;
    c.sfa = c.a + (uint32_t)nst * kDtABytes;
    c.xb = c.sfa + (uint32_t)nst * kDtSfBytes;
    c.xsf = c.xb + (uint32_t)nks * kDtBBytes;
    c.d = c.xsf + (uint32_t)nks * kDtSfBytes;
    c.hb = c.d + 128u * (kDtN + 1) * 4u;
    c.total = c.hb + kDtN * 64u * 4u;
    return c;
}

__device__ __forceinline__ uint64_t dt_desc_atom(uint32_t smem_addr)
{
    uint64_t d = 0;   // one 32-row x 16-byte scale atom: no swizzle, 8-row core matrices
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(16u >> 4) << 16;
    d |= (uint64_t)(128u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

__device__ __forceinline__ void dt_cp_atom(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
                 : "memory");
}

// kind::mxf4nvf4 with 16-element E4M3 scales, E2M1 A and B, M = 128, N = 16
constexpr uint32_t kDtIdesc =
    (1u << 7) | (1u << 10) | ((uint32_t)(kDtN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ void dt_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kDtIdesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ void dt_bulk_load(void *smem_dst, const void *src, uint32_t bytes,
                                             uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane (32x32b shape).
__device__ __forceinline__ void dt_tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void dt_epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads (tcgen05.cp, tcgen05.mma).
__device__ __forceinline__ void dt_fence_proxy_async()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Tile `item` of a launch: whether it is the shared expert's, its index t
// within its source (h columns 64 t ..), and its source's unique-expert slot.
struct DtTile {
    bool shared;
    int u, t;
};

__device__ __forceinline__ DtTile dt_tile(int item, int routed_items, int tpr)
{
    DtTile r;
    r.shared = item >= routed_items;
    r.u = r.shared ? 0 : item / tpr;
    r.t = r.shared ? item - routed_items : item % tpr;
    return r;
}

// h block bi (columns 64 t + 16 bi ..) of row `row` of an NVFP4 operand with
// K columns: 8 bytes of codes and the E4M3 scale in the atom layout, the
// arithmetic of every other NVFP4 quantizer here (nv_quantize16).
__device__ __forceinline__ void dt_quantize_h(const float *hrow16, float h_gs, int row, int t, int bi,
                                              int K, uint8_t *codes, uint8_t *sf)
{
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = hrow16[i];
    uint2 q;
    const uint8_t sc = nv_quantize16(v, h_gs, q);
    const int col = 64 * t + 16 * bi;
    *reinterpret_cast<uint2 *>(codes + (size_t)row * (K / 2) + col / 2) = q;
    sf[nv_sf_offset(row >> 7, row & 127, col / kNvBlock, K)] = sc;
}

} // namespace

__global__ void __launch_bounds__(192, 1)
    k_dec_w13_nvtc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                   const uint16_t *__restrict__ x, float x_gs, const int32_t *__restrict__ idx,
                   int T, int d, int d_ff, int E, int k, int C, int slot_major, int nst,
                   const uint8_t *__restrict__ W13sf, const float *__restrict__ gs13, int d_ff_s,
                   int has_shared, const uint8_t *__restrict__ W13s_sf,
                   const float *__restrict__ gs13s, float *__restrict__ H32,
                   float *__restrict__ Hs32, float *__restrict__ part, float h_gs,
                   uint8_t *__restrict__ hq, uint8_t *__restrict__ hsf, uint8_t *__restrict__ hqs,
                   uint8_t *__restrict__ hsfs, uint32_t *status)
{
    extern __shared__ uint8_t dt_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dt_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int nks = d / 256;   // K stages of a tile
    const DtCarve cv = dt_carve(nst, nks);
    uint8_t *const sa = base + cv.a, *const ssfa = base + cv.sfa;
    uint8_t *const sxb = base + cv.xb, *const sxsf = base + cv.xsf;
    float(*const sd)[kDtN + 1] = reinterpret_cast<float(*)[kDtN + 1]>(base + cv.d);
    float(*const shb)[64] = reinterpret_cast<float(*)[64]>(base + cv.hb);
    __shared__ uint64_t full[kDtMaxStages], empty[kDtMaxStages], tfull[2], tempty[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_s;
    __shared__ DecPlanSmem P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        if (has_shared)
            tma_prefetch_desc(&tmAs);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 256);
        tmem_relinquish();
    }
    // x (an input of the layer, final before the routing kernel started):
    // rows past T and their scales are zeros
    {
        uint4 *z = reinterpret_cast<uint4 *>(sxb);
        const int n16 = nks * (kDtBBytes + kDtSfBytes) / 16;
        for (int i = threadIdx.x; i < n16; i += blockDim.x)
            z[i] = make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        const int bpr = d / kNvBlock;   // 16-element blocks of a row
        for (int i = threadIdx.x; i < T * bpr; i += blockDim.x) {
            const int r = i / bpr, b = i - r * bpr;
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)r * d + b * kNvBlock);
            float v[16];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 w = __ldg(src + h);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[8 * h + 2 * j] = bf16lo(ww[j]);
                    v[8 * h + 2 * j + 1] = bf16hi(ww[j]);
                }
            }
            uint2 q;
            const uint8_t sc = nv_quantize16(v, x_gs, q);
            // block ib of K stage kb: bytes 8 ib .. 8 ib + 7 of the stage's
            // 128-byte row r, whose 16-byte chunk c sits at chunk c ^ (r & 7)
            const int kb = b >> 4, ib = b & 15;
            *reinterpret_cast<uint2 *>(sxb + kb * kDtBBytes + r * 128 +
                                       (((ib >> 1) ^ (r & 7)) << 4) + (ib & 1) * 8) = q;
            sxsf[nv_sf_offset(0, r, b, d)] = sc;
        }
        dt_fence_proxy_async();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    pdl_wait();
    pdl_trigger();
    build_plan(P, idx, T, E, k, C, slot_major, status);   // ends with __syncthreads
    volatile int *abort_flag = &abort_s;
    const int tpr = 2 * d_ff / 128;                        // tiles of a routed expert
    const int routed_items = P.U * tpr;
    const int items = routed_items + (has_shared ? 2 * d_ff_s / 128 : 0);
    const int G = gridDim.x, c = blockIdx.x;
    const DtSplit sp = dt_split(items, G, nks);
    const int nw = dt_num_works(sp, G, c);

    if (warp == 0) {
        if (lane == 0) {   // ---------------- producer
            uint32_t it = 0;
            bool ok = true;
            for (int w = 0; ok && w < nw; ++w) {
                int item, kb0, kb1, unit;
                dt_work(sp, G, c, w, nks, item, kb0, kb1, unit);
                const DtTile tl = dt_tile(item, routed_items, tpr);
                const long long row0 = tl.shared ? (long long)tl.t * 128
                                                 : (long long)P.uniq[tl.u] * 2 * d_ff + tl.t * 128;
                const uint8_t *sfa = (tl.shared ? W13s_sf : W13sf) + (size_t)(row0 / 128) * (d / 64) * 512;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % nst;
                    const uint32_t ph = (it / nst) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], kDtABytes + kDtSfBytes);
                    tma_load_2d(sa + s * kDtABytes, tl.shared ? &tmAs : &tmA, kb * 128, (int)row0, &full[s]);
                    dt_bulk_load(ssfa + s * kDtSfBytes, sfa + (size_t)kb * kDtSfBytes, kDtSfBytes, &full[s]);
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                int never = 0;
                const uint32_t first = it >= (uint32_t)nst ? it - nst : 0;
                for (uint32_t i = first; i < it; ++i)
                    mbar_wait(&full[i % nst], (i / nst) & 1u, &never, status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {   // ---------------- MMA issuer
            uint32_t it = 0;
            for (int w = 0; w < nw; ++w) {
                int item, kb0, kb1, unit;
                dt_work(sp, G, c, w, nks, item, kb0, kb1, unit);
                const uint32_t b = w & 1, aph = (w >> 1) & 1u;
                if (!mbar_wait(&tempty[b], aph ^ 1u, abort_flag, status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * kDtN;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % nst;
                    const uint32_t ph = (it / nst) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // each stage has its own scale columns after the accumulators
                    const uint32_t sf_a = tmem_base + 2 * kDtN + s * kDtSfCols;
                    const uint32_t sf_b = sf_a + 16;
                    const uint32_t a_sf = smem_u32(ssfa + s * kDtSfBytes);
                    const uint32_t b_sf = smem_u32(sxsf + kb * kDtSfBytes);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        dt_cp_atom(sf_a + 4 * g, dt_desc_atom(a_sf + 512 * g));
                        dt_cp_atom(sf_b + 4 * g, dt_desc_atom(b_sf + 512 * g));
                    }
                    const uint32_t a0 = smem_u32(sa + s * kDtABytes), b0 = smem_u32(sxb + kb * kDtBBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        dt_mma(d_tmem, smem_desc_k128(a0 + kk * 32), smem_desc_k128(b0 + kk * 32),
                               sf_a + 4 * kk, sf_b + 4 * kk, (kb != kb0 || kk != 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                if (!ok)
                    break;
                tc_commit(&tfull[b]);
            }
        }
    } else {   // ---------------- epilogue warps 2..5
        const int q = warp & 3;            // TMEM lane quarter this warp may access
        const int et = threadIdx.x - 64;   // 0..127
        for (int w = 0; w < nw; ++w) {
            int item, kb0, kb1, unit;
            dt_work(sp, G, c, w, nks, item, kb0, kb1, unit);
            const uint32_t b = w & 1, aph = (w >> 1) & 1u;
            const bool got = mbar_wait(&tfull[b], aph, abort_flag, status);
            tc_fence_after();
            if (got) {
                float v[16];
                dt_tmem_ld16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * kDtN, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < kDtN; ++i)
                    sd[q * 32 + lane][i] = v[i];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&tempty[b]);
            dt_epi_sync();
            if (got && unit >= 0) {
                // a piece: its sums, row et of token column tok
                for (int tok = 0; tok < T; ++tok)
                    part[((size_t)unit * T + tok) * 128 + et] = sd[et][tok];
            } else if (got && et < 64) {
                const DtTile tl = dt_tile(item, routed_items, tpr);
                const int a0 = tl.shared ? 0 : P.ustart[tl.u];
                const int na = tl.shared ? T : P.ustart[tl.u + 1] - a0;
                const float inv = 1.0f / (x_gs * (tl.shared ? gs13s[0] : gs13[P.uniq[tl.u]]));
                for (int qa = 0; qa < na; ++qa) {
                    const int a = tl.shared ? qa : P.list[a0 + qa];
                    const int tok = tl.shared ? qa : a / k;
                    const float h = silu_mul(sd[et][tok] * inv, sd[64 + et][tok] * inv);
                    shb[qa][et] = h;
                    if (tl.shared)
                        Hs32[(size_t)qa * d_ff_s + 64 * tl.t + et] = h;
                    else
                        H32[(size_t)a * d_ff + 64 * tl.t + et] = h;
                }
            }
            dt_epi_sync();
            if (got && unit < 0 && hq) {
                // h as the w2 kernel's NVFP4 operand: block et & 3 of assignment et >> 2
                const DtTile tl = dt_tile(item, routed_items, tpr);
                const int a0 = tl.shared ? 0 : P.ustart[tl.u];
                const int na = tl.shared ? T : P.ustart[tl.u + 1] - a0;
                if (et < 4 * na) {
                    const int qa = et >> 2, bi = et & 3;
                    const int row = tl.shared ? qa : P.list[a0 + qa];
                    dt_quantize_h(&shb[qa][16 * bi], h_gs, row, tl.t, bi, tl.shared ? d_ff_s : d_ff,
                                  tl.shared ? hqs : hq, tl.shared ? hsfs : hsf);
                }
            }
            dt_epi_sync();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 256);
    }
}

// The leftover tiles of k_dec_w13_nvtc (same G): block j adds the np pieces
// of leftover tile j in piece order and forms its 64 h columns.
__global__ void __launch_bounds__(64)
    k_dec_w13_nvtc_fix(const int32_t *__restrict__ idx, int T, int d, int d_ff, int E, int k, int C,
                       int slot_major, int G, int d_ff_s, int has_shared, float x_gs,
                       const float *__restrict__ gs13, const float *__restrict__ gs13s,
                       const float *__restrict__ part, float *__restrict__ H32,
                       float *__restrict__ Hs32, float h_gs, uint8_t *__restrict__ hq,
                       uint8_t *__restrict__ hsf, uint8_t *__restrict__ hqs,
                       uint8_t *__restrict__ hsfs, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    __shared__ float shb[kDtN][64];
    build_plan(P, idx, T, E, k, C, slot_major, status);   // idx is final: the w1/w3 kernel read it
    pdl_wait();      // the pieces come from the w1/w3 kernel
    pdl_trigger();
    const int tpr = 2 * d_ff / 128;
    const int routed_items = P.U * tpr;
    const int items = routed_items + (has_shared ? 2 * d_ff_s / 128 : 0);
    const DtSplit sp = dt_split(items, G, d / 256);
    const int j = blockIdx.x;
    if (j >= sp.R)
        return;
    const DtTile tl = dt_tile(sp.full * G + j, routed_items, tpr);
    const int a0 = tl.shared ? 0 : P.ustart[tl.u];
    const int na = tl.shared ? T : P.ustart[tl.u + 1] - a0;
    const float inv = 1.0f / (x_gs * (tl.shared ? gs13s[0] : gs13[P.uniq[tl.u]]));
    const int et = threadIdx.x;
    for (int qa = 0; qa < na; ++qa) {
        const int a = tl.shared ? qa : P.list[a0 + qa];
        const int tok = tl.shared ? qa : a / k;
        const float *pp = part + ((size_t)j * sp.np * T + tok) * 128 + et;
        const size_t stride = (size_t)T * 128;   // from one piece to the next
        float g = 0.f, u = 0.f;
        // eight pieces' loads in flight at a time, added in piece order
        for (int p0 = 0; p0 < sp.np; p0 += 8) {
            float vg[8], vu[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const bool in = p0 + i < sp.np;
                vg[i] = in ? __ldcg(pp + (p0 + i) * stride) : 0.f;
                vu[i] = in ? __ldcg(pp + (p0 + i) * stride + 64) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (p0 + i < sp.np) {
                    g += vg[i];
                    u += vu[i];
                }
        }
        const float h = silu_mul(g * inv, u * inv);
        shb[qa][et] = h;
        if (tl.shared)
            Hs32[(size_t)qa * d_ff_s + 64 * tl.t + et] = h;
        else
            H32[(size_t)a * d_ff + 64 * tl.t + et] = h;
    }
    if (!hq)
        return;
    __syncthreads();
    if (et < 4 * na) {
        const int qa = et >> 2, bi = et & 3;
        const int row = tl.shared ? qa : P.list[a0 + qa];
        dt_quantize_h(&shb[qa][16 * bi], h_gs, row, tl.t, bi, tl.shared ? d_ff_s : d_ff,
                      tl.shared ? hqs : hq, tl.shared ? hsfs : hsf);
    }
}

// ---------------------------------------------------------------- NVFP4 decode w2, tensor cores
// NVFP4 decode w2 on the tensor cores: a chosen expert's W2 rows are the M
// side (128 output rows per tile, K = d_ff) and the assignments' h rows the N
// side (16 columns: routed h rows a = t k + j, quantized by the w1/w3 kernel;
// the shared expert's tiles take the T shared h rows). Tiles: source u (the
// chosen experts ascending, then the shared expert) x row tile rt. There are
// few of them (64 at one token), so the launch is split evenly over its G
// CTAs along the flattened (tile, K stage) sequence ("stream-K"): CTA c runs
// stages [c F / G, (c + 1) F / G), one piece per tile it touches. A piece's
// epilogue weights column a by w_a / (gs_h gs_w2[e]) and writes, for every
// token, its rows' sums to `part` (zero where the token did not choose the
// expert); k_dec_w2_nvtc_reduce adds, per output, the pieces of every source
// in (source, CTA) order: deterministic.
// Roles as k_dec_w13_nvtc; the ring carries the weight tile (16 KB), the h
// tile (2 KB) and both operands' scale atoms (2 KB each) per K stage.
namespace {

constexpr uint32_t kD2StageBytes = kDtABytes + kDtBBytes + 2 * kDtSfBytes;
constexpr int kD2MaxCtas = 1024;   // CTAs of one k_dec_w2_nvtc launch

} // namespace

__global__ void __launch_bounds__(192, 1)
    k_dec_w2_nvtc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                  const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBs,
                  const int32_t *__restrict__ idx, const float *__restrict__ topk_w, int T, int d,
                  int d_ff, int E, int k, int C, int slot_major, int nst,
                  const uint8_t *__restrict__ W2sf, const float *__restrict__ gs2, int d_ff_s,
                  int has_shared, const uint8_t *__restrict__ W2s_sf, const float *__restrict__ gs2s,
                  const uint8_t *__restrict__ hsf, const uint8_t *__restrict__ hsfs, float h_gs,
                  float *__restrict__ part, int pmax, uint32_t *status)
{
    extern __shared__ uint8_t dt_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(dt_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // ring: a [nst][16 KB], b [nst][2 KB], sfa [nst][2 KB], sfb [nst][2 KB]
    uint8_t *const sa = base, *const sb = base + nst * kDtABytes;
    uint8_t *const ssfa = sb + nst * kDtBBytes, *const ssfb = ssfa + nst * kDtSfBytes;
    __shared__ uint64_t full[kDtMaxStages], empty[kDtMaxStages], tfull[2], tempty[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_s;
    __shared__ DecPlanSmem P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (has_shared) {
            tma_prefetch_desc(&tmAs);
            tma_prefetch_desc(&tmBs);
        }
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    build_plan(P, idx, T, E, k, C, slot_major, status);   // idx: final before the w1/w3 kernel ran
    pdl_wait();      // h comes from the w1/w3 kernels
    pdl_trigger();
    volatile int *abort_flag = &abort_s;
    const D2Space z = d2_space(P.U, has_shared, d, d_ff, d_ff_s);
    const int G = gridDim.x, c = blockIdx.x;

    if (warp == 0) {
        if (lane == 0) {   // ---------------- producer
            uint32_t it = 0;
            bool ok = true;
            int item, kb0, kb1;
            for (int lp = 0; ok && lp < pmax && d2_piece(z, G, c, lp, item, kb0, kb1); ++lp) {
                const bool shared = item >= z.routed_items;
                const int rt = item % z.RT;
                const long long row0 = shared ? (long long)rt * 128
                                              : ((long long)P.uniq[item / z.RT] * d + rt * 128);
                const int K = shared ? d_ff_s : d_ff;
                const uint8_t *sfa = (shared ? W2s_sf : W2sf) + (size_t)(row0 / 128) * (K / 64) * 512;
                const uint8_t *sfb = shared ? hsfs : hsf;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % nst;
                    const uint32_t ph = (it / nst) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], kD2StageBytes);
                    tma_load_2d(sa + s * kDtABytes, shared ? &tmAs : &tmA, kb * 128, (int)row0, &full[s]);
                    tma_load_2d(sb + s * kDtBBytes, shared ? &tmBs : &tmB, kb * 128, 0, &full[s]);
                    dt_bulk_load(ssfa + s * kDtSfBytes, sfa + (size_t)kb * kDtSfBytes, kDtSfBytes, &full[s]);
                    dt_bulk_load(ssfb + s * kDtSfBytes, sfb + (size_t)kb * kDtSfBytes, kDtSfBytes, &full[s]);
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                int never = 0;
                const uint32_t first = it >= (uint32_t)nst ? it - nst : 0;
                for (uint32_t i = first; i < it; ++i)
                    mbar_wait(&full[i % nst], (i / nst) & 1u, &never, status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {   // ---------------- MMA issuer
            uint32_t it = 0;
            int item, kb0, kb1;
            for (int lp = 0; lp < pmax && d2_piece(z, G, c, lp, item, kb0, kb1); ++lp) {
                const uint32_t b = lp & 1, aph = (lp >> 1) & 1u;
                if (!mbar_wait(&tempty[b], aph ^ 1u, abort_flag, status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * kDtN;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % nst;
                    const uint32_t ph = (it / nst) & 1u;
                    if (!mbar_wait(&full[s], ph, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_a = tmem_base + 2 * kDtN + s * kDtSfCols;
                    const uint32_t sf_b = sf_a + 16;
                    const uint32_t a_sf = smem_u32(ssfa + s * kDtSfBytes);
                    const uint32_t b_sf = smem_u32(ssfb + s * kDtSfBytes);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        dt_cp_atom(sf_a + 4 * g, dt_desc_atom(a_sf + 512 * g));
                        dt_cp_atom(sf_b + 4 * g, dt_desc_atom(b_sf + 512 * g));
                    }
                    const uint32_t a0 = smem_u32(sa + s * kDtABytes), b0 = smem_u32(sb + s * kDtBBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        dt_mma(d_tmem, smem_desc_k128(a0 + kk * 32), smem_desc_k128(b0 + kk * 32),
                               sf_a + 4 * kk, sf_b + 4 * kk, (kb != kb0 || kk != 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                if (!ok)
                    break;
                tc_commit(&tfull[b]);
            }
        }
    } else {   // ---------------- epilogue warps 2..5: one output row per thread
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int item, kb0, kb1;
        for (int lp = 0; lp < pmax && d2_piece(z, G, c, lp, item, kb0, kb1); ++lp) {
            const uint32_t b = lp & 1, aph = (lp >> 1) & 1u;
            const bool got = mbar_wait(&tfull[b], aph, abort_flag, status);
            tc_fence_after();
            float v[16];
            if (got) {
                dt_tmem_ld16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * kDtN, v);
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&tempty[b]);
            if (!got)
                continue;
            const bool shared = item >= z.routed_items;
            const int u = shared ? 0 : item / z.RT;
            const float inv = 1.0f / (h_gs * (shared ? gs2s[0] : gs2[P.uniq[u]]));
            float *dst = part + (size_t)(c * pmax + lp) * T * 128 + row;
            for (int tok = 0; tok < T; ++tok) {
                float val = 0.f;
                if (shared) {
#pragma unroll
                    for (int j = 0; j < kDtN; ++j)
                        val = (j == tok) ? v[j] * inv : val;
                } else {
                    for (int qa = P.ustart[u]; qa < P.ustart[u + 1]; ++qa) {
                        const int a = P.list[qa];
                        if (a / k != tok)
                            continue;
                        float pick = 0.f;
#pragma unroll
                        for (int j = 0; j < kDtN; ++j)
                            pick = (j == a) ? v[j] : pick;
                        val = topk_w[a] * inv * pick;
                    }
                }
                dst[(size_t)tok * 128] = val;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 256);
    }
}

// out[t, r] = the sum, over the sources in order (chosen experts ascending,
// then the shared expert) and over the CTAs that ran pieces of the source's
// row tile (ascending), of the pieces' sums. One block per (row tile, token),
// 128 threads (one output row each); G and pmax as for k_dec_w2_nvtc. One
// thread lists the pieces' slots, up to 512 at a time, and every thread adds
// its row of them in list order, eight loads in flight.
__global__ void __launch_bounds__(128)
    k_dec_w2_nvtc_reduce(const int32_t *__restrict__ idx, int T, int d, int d_ff, int E, int k, int C,
                         int slot_major, int G, int pmax, int d_ff_s, int has_shared,
                         const float *__restrict__ part, float *__restrict__ out, uint32_t *status)
{
    constexpr int kList = 512;
    __shared__ DecPlanSmem P;
    __shared__ int terms[kList];   // piece slots (units of T x 128 floats), in summation order
    __shared__ long long f0s[kD2MaxCtas + 1];   // the CTAs' first stages
    __shared__ int nterms, g_src, g_cc, g_done;
    build_plan(P, idx, T, E, k, C, slot_major, status);
    const D2Space z = d2_space(P.U, has_shared, d, d_ff, d_ff_s);
    for (int cc = threadIdx.x; cc <= G; cc += blockDim.x)
        f0s[cc] = d2_f0(z, G, cc);
    pdl_wait();      // the pieces come from the w2 kernel
    pdl_trigger();
    const int rt = blockIdx.x, tok = blockIdx.y, r = threadIdx.x;
    if (r == 0) {
        g_src = 0;
        g_cc = -1;
    }
    const float *pp = part + (size_t)tok * 128 + r;
    const size_t stride = (size_t)T * 128;
    float acc = 0.f;
    for (;;) {
        __syncthreads();   // the previous list is consumed
        if (r == 0) {
            int n = 0, src = g_src, cc = g_cc;
            while (n < kList && src < z.src) {
                const int item = src * z.RT + rt;
                const long long s0 = d2_item_start(z, item), s1 = d2_item_start(z, item + 1);
                if (cc < 0)
                    cc = d2_first_cta(z, G, s0);
                const long long a = cc < G ? f0s[cc] : s1;
                if (a >= s1) {
                    ++src;
                    cc = -1;
                    continue;
                }
                const long long b = f0s[cc + 1];
                if (b > s0 && b > a)   // a non-empty range that meets the tile
                    terms[n++] = cc * pmax + (item - d2_item_of(z, a));
                ++cc;
            }
            nterms = n;
            g_src = src;
            g_cc = cc;
            g_done = src >= z.src;
        }
        __syncthreads();
        const int n = nterms;
        for (int i0 = 0; i0 < n; i0 += 8) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = i0 + i < n ? __ldcg(pp + (size_t)terms[i0 + i] * stride) : 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i0 + i < n)
                    acc += v[i];
        }
        if (g_done)
            break;
    }
    out[(size_t)tok * d + rt * 128 + r] = acc;
}

// ---------------------------------------------------------------- host side

// Launch with programmatic stream serialization (the kernel calls pdl_wait()
// before reading its predecessor's output), hiding the launch gap.
template <typename... KArgs, typename... Args>
static void launch_pdl(void (*kernel)(KArgs...), int grid, int block, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raises a kernel's dynamic shared memory limit to the device's opt-in
// maximum once per (kernel, device); fails if `smem` exceeds it.
static int smem_attr_once(const void *kernel, size_t smem)
{
    constexpr int kMax = 64;
    static std::mutex mu;
    static const void *done_k[kMax];
    static int done_d[kMax];
    static int n_done = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_done; ++i)
        if (done_k[i] == kernel && done_d[i] == dev)
            return MOE_OK;
    // the device's opt-in maximum less the kernel's static shared memory, so
    // that every later size fits as well
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int dyn_max = optin - (int)fa.sharedSizeBytes;
    if (dyn_max < (int)smem ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (n_done < kMax) {
        done_k[n_done] = kernel;
        done_d[n_done] = dev;
        ++n_done;
    }
    return MOE_OK;
}

// The same, with dynamic shared memory.
// The dynamic shared memory a launch of `kernel` may take on this device:
// the opt-in maximum less the kernel's static shared memory.
static int smem_limit(const void *kernel, int &dyn_max)
{
    constexpr int kMax = 64;
    static std::mutex mu;
    static const void *seen_k[kMax];
    static int seen_d[kMax], seen_v[kMax];
    static int n_seen = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_seen; ++i)
        if (seen_k[i] == kernel && seen_d[i] == dev) {
            dyn_max = seen_v[i];
            return MOE_OK;
        }
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
        return MOE_ERR_CUDA;
    dyn_max = optin - (int)fa.sharedSizeBytes;
    if (n_seen < kMax) {
        seen_k[n_seen] = kernel;
        seen_d[n_seen] = dev;
        seen_v[n_seen] = dyn_max;
        ++n_seen;
    }
    return MOE_OK;
}

template <typename... KArgs, typename... Args>
static int launch_pdl_smem(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                           cudaStream_t st, Args... args)
{
    if (const int rc = smem_attr_once(reinterpret_cast<const void *>(kernel), smem))
        return rc;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, args...);
    return MOE_OK;
}

static int maxt_for(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16; }

int launch_dec_router(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                      const float *bias, float *logits, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int blocks = (s.E + 7) / 8;
    switch (maxt_for(s.T)) {
    case 1: k_dec_router<1><<<blocks, 256, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, logits); break;
    case 2: k_dec_router<2><<<blocks, 256, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, logits); break;
    case 4: k_dec_router<4><<<blocks, 256, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, logits); break;
    case 8: k_dec_router<8><<<blocks, 256, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, logits); break;
    default: k_dec_router<16><<<blocks, 256, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, logits); break;
    }
    return launched();
}

bool dec_route_fusable(const moe_shape_t &s)
{
    return s.T <= MOE_DECODE_MAX_T && (size_t)s.E * s.d * 2 <= kFusedRouteBytes;
}

template <int MAXT>
static void launch_dec_route_t(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                               const float *bias, float *logits, int32_t *idx, float *w,
                               int32_t *ctr, uint32_t *status, cudaStream_t st)
{
    const int vpl = (s.E + 31) / 32;
    if (vpl <= 1)
        k_dec_route<MAXT, 1><<<1, 512, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, s.k, logits, idx, w, ctr, status);
    else if (vpl <= 2)
        k_dec_route<MAXT, 2><<<1, 512, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, s.k, logits, idx, w, ctr, status);
    else if (vpl <= 4)
        k_dec_route<MAXT, 4><<<1, 512, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, s.k, logits, idx, w, ctr, status);
    else
        k_dec_route<MAXT, 8><<<1, 512, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, s.k, logits, idx, w, ctr, status);
}

int launch_dec_route(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                     const float *bias, float *logits, int32_t *idx, float *w,
                     int32_t *counter_to_zero, uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    int32_t *c = counter_to_zero;
    switch (maxt_for(s.T)) {
    case 1: launch_dec_route_t<1>(s, x, Wg, bias, logits, idx, w, c, status, st); break;
    case 2: launch_dec_route_t<2>(s, x, Wg, bias, logits, idx, w, c, status, st); break;
    case 4: launch_dec_route_t<4>(s, x, Wg, bias, logits, idx, w, c, status, st); break;
    case 8: launch_dec_route_t<8>(s, x, Wg, bias, logits, idx, w, c, status, st); break;
    default: launch_dec_route_t<16>(s, x, Wg, bias, logits, idx, w, c, status, st); break;
    }
    return launched();
}

int launch_dec_w13(const moe_shape_t &s, const uint16_t *x, const int32_t *topk_idx,
                   const uint16_t *W13, const uint16_t *W13s, uint16_t *Hdec, uint32_t *status,
                   cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int mt = maxt_for(s.T);
    const int blocks = num_sms() * ((mt <= 2) ? 4 : 2);
    uint16_t *Hs = Hdec + (size_t)s.T * s.k * s.d_ff;
    const uint16_t *ws = s.d_ff_shared ? W13s : nullptr;
#define MOE_DEC13(M)                                                                            \
    launch_pdl(k_dec_w13<M>, blocks, 256, st, x, topk_idx, s.T, s.d, s.d_ff, s.E, s.k,        \
               s.capacity, slot_major(s), W13, s.d_ff_shared, ws, Hdec, Hs, status)
    switch (mt) {
    case 1: MOE_DEC13(1); break;
    case 2: MOE_DEC13(2); break;
    case 4: MOE_DEC13(4); break;
    case 8: MOE_DEC13(8); break;
    default: MOE_DEC13(16); break;
    }
#undef MOE_DEC13
    return launched();
}

int launch_dec_w2(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                  const uint16_t *W2, const uint16_t *W2s, const uint16_t *Hdec, float *out,
                  uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int mt = maxt_for(s.T);
    const int blocks = num_sms() * ((mt <= 2) ? 4 : 2);
    const uint16_t *Hs = Hdec + (size_t)s.T * s.k * s.d_ff;
    const uint16_t *ws = s.d_ff_shared ? W2s : nullptr;
#define MOE_DEC2(M)                                                                             \
    launch_pdl(k_dec_w2<M>, blocks, 256, st, topk_idx, topk_w, s.T, s.d, s.d_ff, s.E, s.k,     \
               s.capacity, slot_major(s), W2, s.d_ff_shared, ws, Hdec, Hs, out, status)
    switch (mt) {
    case 1: MOE_DEC2(1); break;
    case 2: MOE_DEC2(2); break;
    case 4: MOE_DEC2(4); break;
    case 8: MOE_DEC2(8); break;
    default: MOE_DEC2(16); break;
    }
#undef MOE_DEC2
    return launched();
}

int launch_dec_w13_mx(const moe_shape_t &s, const uint16_t *xdq, const int32_t *topk_idx,
                      const uint8_t *W13q, const uint8_t *W13sf, const uint8_t *W13s_q,
                      const uint8_t *W13s_sf, float *H32, uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int mt = maxt_for(s.T);
    const int blocks = num_sms() * ((mt <= 2) ? 4 : 2);
    float *Hs = H32 + (size_t)s.T * s.k * s.d_ff;
    const uint8_t *wq = s.d_ff_shared ? W13s_q : nullptr;
#define MOE_DEC13MX(M)                                                                          \
    launch_pdl(k_dec_w13_mx<M>, blocks, 256, st, xdq, topk_idx, s.T, s.d, s.d_ff, s.E, s.k,    \
               s.capacity, slot_major(s), W13q, W13sf, s.d_ff_shared, wq, W13s_sf, H32, Hs,     \
               status)
    switch (mt) {
    case 1: MOE_DEC13MX(1); break;
    case 2: MOE_DEC13MX(2); break;
    case 4: MOE_DEC13MX(4); break;
    case 8: MOE_DEC13MX(8); break;
    default: MOE_DEC13MX(16); break;
    }
#undef MOE_DEC13MX
    return launched();
}

int launch_dec_w2_mx(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                     const uint8_t *W2q, const uint8_t *W2sf, const uint8_t *W2s_q,
                     const uint8_t *W2s_sf, const uint16_t *Hdq, float *out, uint32_t *status,
                     cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int mt = maxt_for(s.T);
    const int blocks = num_sms() * ((mt <= 2) ? 4 : 2);
    const uint16_t *Hs = Hdq + (size_t)s.T * s.k * s.d_ff;
    const uint8_t *wq = s.d_ff_shared ? W2s_q : nullptr;
#define MOE_DEC2MX(M)                                                                           \
    launch_pdl(k_dec_w2_mx<M>, blocks, 256, st, topk_idx, topk_w, s.T, s.d, s.d_ff, s.E, s.k,  \
               s.capacity, slot_major(s), W2q, W2sf, s.d_ff_shared, wq, W2s_sf, Hdq, Hs, out,   \
               status)
    switch (mt) {
    case 1: MOE_DEC2MX(1); break;
    case 2: MOE_DEC2MX(2); break;
    case 4: MOE_DEC2MX(4); break;
    case 8: MOE_DEC2MX(8); break;
    default: MOE_DEC2MX(16); break;
    }
#undef MOE_DEC2MX
    return launched();
}

int launch_dec_w13_nv(const moe_shape_t &s, const uint16_t *xh, const float *xs, float x_gs,
                      const int32_t *topk_idx, const uint8_t *W13q, const uint8_t *W13sf,
                      const float *gs13, const uint8_t *W13s_q, const uint8_t *W13s_sf,
                      const float *gs13s, float *H32, uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    if (s.T > 2)
        return MOE_ERR_UNSUPPORTED;
    // packed code rows of d / 2 bytes, read 128 rows x 128 bytes per K stage
    CUtensorMap tmR, tmS;
    int rc = make_tmap_u8_rows(&tmR, W13q, s.d / 2, (long long)s.E * 2 * s.d_ff, 128);
    if (rc)
        return rc;
    const bool shared = s.d_ff_shared > 0 && W13s_q;
    if (shared) {
        if ((rc = make_tmap_u8_rows(&tmS, W13s_q, s.d / 2, 2LL * s.d_ff_shared, 128)))
            return rc;
    } else {
        tmS = tmR;
    }
    // at most min(E, T k) chosen experts of 2 d_ff / 128 tiles, then the shared expert's
    const long long items = (long long)std::min(s.E, s.T * s.k) * (2 * s.d_ff / 128) +
                            (shared ? 2 * s.d_ff_shared / 128 : 0);
    const int blocks = (int)std::max<long long>(1, std::min<long long>(items, 2LL * num_sms()));
    float *Hs = H32 + (size_t)s.T * s.k * s.d_ff;
    // x staged in shared memory: T rows of d f16 values and d / 16 fp32 scales
    const size_t xbytes = (size_t)s.T * s.d * 2 + (size_t)s.T * (s.d / 16) * 4;
    rc = s.T == 1
             ? launch_pdl_smem(k_dec_w13_nv<1>, blocks, kNdThreads, nd_smem_bytes<1>() + 1024 + xbytes, st,
                               tmR, tmS, xh, xs, x_gs, topk_idx, s.T, s.d, s.d_ff, s.E, s.k,
                               s.capacity, slot_major(s), W13sf, gs13, s.d_ff_shared,
                               shared ? 1 : 0, W13s_sf, gs13s, H32, Hs, status)
             : launch_pdl_smem(k_dec_w13_nv<2>, blocks, kNdThreads, nd_smem_bytes<2>() + 1024 + xbytes, st,
                               tmR, tmS, xh, xs, x_gs, topk_idx, s.T, s.d, s.d_ff, s.E, s.k,
                               s.capacity, slot_major(s), W13sf, gs13, s.d_ff_shared,
                               shared ? 1 : 0, W13s_sf, gs13s, H32, Hs, status);
    if (rc)
        return rc;
    return launched();
}

int launch_dec_w13_nvtc(const moe_shape_t &s, const uint16_t *x, float x_gs,
                        const int32_t *topk_idx, const uint8_t *W13q, const uint8_t *W13sf,
                        const float *gs13, const uint8_t *W13s_q, const uint8_t *W13s_sf,
                        const float *gs13s, float *H32, float *part, size_t part_floats,
                        float h_gs, uint8_t *hq, uint8_t *hsf, uint8_t *hqs, uint8_t *hsfs,
                        uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const bool shared = s.d_ff_shared > 0 && W13s_q;
    if (s.T > kDtN || s.d % 256 != 0 || (2 * s.d_ff) % 128 != 0 ||
        (shared && (2 * s.d_ff_shared) % 128 != 0))
        return MOE_ERR_UNSUPPORTED;
    const int nks = s.d / 256;
    const long long items = (long long)std::min(s.E, s.T * s.k) * (2 * s.d_ff / 128) +
                            (shared ? 2 * s.d_ff_shared / 128 : 0);
    const int blocks = (int)std::max<long long>(1, std::min<long long>(items, num_sms()));
    // pieces: fewer than 2 G units of T x 128 sums
    if ((size_t)2 * blocks * s.T * 128 > part_floats)
        return MOE_ERR_UNSUPPORTED;
    // the deepest ring (2..kDtMaxStages stages) that fits beside the resident x
    int dyn_max = 0;
    if (const int rc = smem_limit(reinterpret_cast<const void *>(k_dec_w13_nvtc), dyn_max))
        return rc;
    int nst = kDtMaxRing;
    while (nst >= 2 && (int)dt_carve(nst, nks).total + 1024 > dyn_max)
        --nst;
    if (nst < 2)
        return MOE_ERR_UNSUPPORTED;
    CUtensorMap tmA, tmAs;
    int rc = make_tmap_u8_sw128(&tmA, W13q, s.d / 2, (long long)s.E * 2 * s.d_ff, 128);
    if (rc)
        return rc;
    if (shared) {
        if ((rc = make_tmap_u8_sw128(&tmAs, W13s_q, s.d / 2, 2LL * s.d_ff_shared, 128)))
            return rc;
    } else {
        tmAs = tmA;
    }
    float *Hs = H32 + (size_t)s.T * s.k * s.d_ff;
    rc = launch_pdl_smem(k_dec_w13_nvtc, blocks, 192, dt_carve(nst, nks).total + 1024, st, tmA, tmAs,
                         x, x_gs, topk_idx, s.T, s.d, s.d_ff, s.E, s.k, s.capacity, slot_major(s), nst,
                         W13sf, gs13, s.d_ff_shared, shared ? 1 : 0, W13s_sf, gs13s, H32, Hs, part,
                         h_gs, hq, hsf, hqs, hsfs, status);
    if (rc)
        return rc;
    if ((rc = launched()))
        return rc;
    launch_pdl(k_dec_w13_nvtc_fix, blocks, 64, st, topk_idx, s.T, s.d, s.d_ff, s.E, s.k, s.capacity,
               slot_major(s), blocks, s.d_ff_shared, shared ? 1 : 0, x_gs, gs13, gs13s,
               (const float *)part, H32, Hs, h_gs, hq, hsf, hqs, hsfs, status);
    return launched();
}

int launch_dec_w2_nvtc(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                       const uint8_t *W2q, const uint8_t *W2sf, const float *gs2,
                       const uint8_t *W2s_q, const uint8_t *W2s_sf, const float *gs2s,
                       const uint8_t *hq, const uint8_t *hsf, const uint8_t *hqs, const uint8_t *hsfs,
                       float h_gs, float *part, size_t part_floats, float *out, uint32_t *status,
                       cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const bool shared = s.d_ff_shared > 0 && W2s_q;
    // h rows are the N side: every routed row (and the T shared rows) in 16 columns
    if (s.T * s.k > kDtN || s.d % 128 != 0 || s.d_ff % 256 != 0 ||
        (shared && s.d_ff_shared % 256 != 0))
        return MOE_ERR_UNSUPPORTED;
    const int RT = s.d / 128, nks = s.d_ff / 256, nks_s = shared ? s.d_ff_shared / 256 : nks;
    const long long Fmax = (long long)std::min(s.E, s.T * s.k) * RT * nks +
                           (shared ? (long long)RT * nks_s : 0);
    const int G = (int)std::max<long long>(1, std::min<long long>(Fmax, num_sms()));
    if (G > kD2MaxCtas)
        return MOE_ERR_UNSUPPORTED;
    // pieces per CTA: a range of at most ceil(F / G) stages meets at most
    // ceil(that / the shortest tile) + 1 tiles
    const int pmax = d2_pmax(Fmax, G, std::min(nks, nks_s));
    if ((size_t)G * pmax * s.T * 128 > part_floats)
        return MOE_ERR_UNSUPPORTED;
    int dyn_max = 0;
    if (const int rc = smem_limit(reinterpret_cast<const void *>(k_dec_w2_nvtc), dyn_max))
        return rc;
    int nst = kDtMaxRing;
    while (nst >= 2 && (int)(nst * kD2StageBytes) + 1024 > dyn_max)
        --nst;
    if (nst < 2)
        return MOE_ERR_UNSUPPORTED;
    CUtensorMap tmA, tmAs, tmB, tmBs;
    int rc = make_tmap_u8_sw128(&tmA, W2q, s.d_ff / 2, (long long)s.E * s.d, 128);
    if (!rc)
        rc = make_tmap_u8_sw128(&tmB, hq, s.d_ff / 2, (long long)s.T * s.k, kDtN);
    if (!rc && shared) {
        rc = make_tmap_u8_sw128(&tmAs, W2s_q, s.d_ff_shared / 2, s.d, 128);
        if (!rc)
            rc = make_tmap_u8_sw128(&tmBs, hqs, s.d_ff_shared / 2, s.T, kDtN);
    } else {
        tmAs = tmA;
        tmBs = tmB;
    }
    if (rc)
        return rc;
    rc = launch_pdl_smem(k_dec_w2_nvtc, G, 192, (size_t)nst * kD2StageBytes + 1024, st, tmA, tmAs, tmB,
                         tmBs, topk_idx, topk_w, s.T, s.d, s.d_ff, s.E, s.k, s.capacity, slot_major(s),
                         nst, W2sf, gs2, s.d_ff_shared, shared ? 1 : 0, W2s_sf, gs2s, hsf, hsfs, h_gs,
                         part, pmax, status);
    if (rc)
        return rc;
    if ((rc = launched()))
        return rc;
    launch_pdl_ex(k_dec_w2_nvtc_reduce, dim3(RT, s.T), dim3(128), 0, st, topk_idx, s.T, s.d, s.d_ff,
                  s.E, s.k, s.capacity, slot_major(s), G, pmax, s.d_ff_shared, shared ? 1 : 0,
                  (const float *)part, out, status);
    return launched();
}

int launch_dec_w2_nv(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                     const uint8_t *W2q, const uint8_t *W2sf, const float *gs2,
                     const uint8_t *W2s_q, const uint8_t *W2s_sf, const float *gs2s,
                     const uint16_t *hh, const float *hs, float h_gs, float *out,
                     uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    if (s.T > 2)
        return MOE_ERR_UNSUPPORTED;
    const int blocks = num_sms() * 2;
    const uint8_t *wq = s.d_ff_shared ? W2s_q : nullptr;
    if (s.T == 1)
        launch_pdl(k_dec_w2_nv<1>, blocks, 256, st, topk_idx, topk_w, s.T, s.d, s.d_ff, s.E, s.k,
                   s.capacity, slot_major(s), W2q, W2sf, gs2, s.d_ff_shared, wq, W2s_sf, gs2s,
                   hh, hs, h_gs, out, status);
    else
        launch_pdl(k_dec_w2_nv<2>, blocks, 256, st, topk_idx, topk_w, s.T, s.d, s.d_ff, s.E, s.k,
                   s.capacity, slot_major(s), W2q, W2sf, gs2, s.d_ff_shared, wq, W2s_sf, gs2s,
                   hh, hs, h_gs, out, status);
    return launched();
}

} // namespace moe
