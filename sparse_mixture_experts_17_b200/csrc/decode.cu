// decode.cu -- the small-T forward: stream only the chosen experts' weights.
//
// "Faster writing: run only the chosen experts; uncap the large profile"
// (mini-AGI) describes the failure this path avoids: a single-token forward
// that multiplied against every expert on the card read all their weights to
// use top_k of them. "perf(moe): route granite-4.0-h single-token MoE through
// the fused kernel" (mlxcel) routes one-token decode to a fused kernel fed by
// the router's top-k indices and renormalised scores. Here the chosen experts
// are known only on the device, so every CTA rebuilds the (tiny) plan in
// shared memory from topk_idx and the weight stream is spread over all SMs.
//
// Phase 1 (k_dec_w13): work unit = one SwiGLU column c of one chosen expert:
//   h[a, c] = bf16(silu(W1_e[c] . x_t) * (W3_e[c] . x_t)) for every
//   assignment a = (t, j) routed to e. Each unit streams the gate row and the
//   up row once (2 * d * 2 bytes), dotted against the routed tokens' x (L1).
// Phase 2 (k_dec_w2): work unit = one output row r:
//   out[t, r] = sum over the chosen experts e (ascending), then the shared
//   expert, of w[a] * (W2_e[r] . h[a]). Each unit streams W2_e[r] once per
//   chosen expert; h is L1/L2 resident. Fixed order: deterministic.
#include "common.cuh"
#include "internal.h"

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

// Every thread of the CTA participates; ends with __syncthreads().
__device__ void build_plan(DecPlanSmem &P, const int32_t *__restrict__ idx, int T, int E, int k,
                           uint32_t *status)
{
    const int A = T * k;
    for (int e = threadIdx.x; e < MOE_MAX_E; e += blockDim.x)
        P.cnt[e] = 0;
    __syncthreads();
    // rank of each assignment among earlier ones of the same expert
    for (int a = threadIdx.x; a < A; a += blockDim.x) {
        const int e = idx[a];
        if (e < 0 || e >= E) {
            if (blockIdx.x == 0)
                flag_status(status, MOE_ERR_BAD_EXPERT);
            continue;
        }
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
    for (int a = threadIdx.x; a < A; a += blockDim.x) {
        const int e = idx[a];
        if (e < 0 || e >= E)
            continue;
        int r = 0;
        for (int b = 0; b < a; ++b)
            r += (idx[b] == e);
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

// ---------------------------------------------------------------- router for small T
// One warp per expert: logits[t, e] = Wg[e] . x[t] + bias[e] for all t < T.
__global__ void __launch_bounds__(256) k_dec_router(const uint16_t *__restrict__ x,
                                                    const uint16_t *__restrict__ Wg,
                                                    const float *__restrict__ bias, int T, int d,
                                                    int E, float *__restrict__ logits)
{
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const int nv = d / 8;
    for (int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; e < E; e += nwarps) {
        float acc[MOE_DECODE_MAX_T];
#pragma unroll
        for (int t = 0; t < MOE_DECODE_MAX_T; ++t)
            acc[t] = 0.f;
        const uint4 *wr = reinterpret_cast<const uint4 *>(Wg + (size_t)e * d);
        for (int c = lane; c < nv; c += 32) {
            const uint4 wv = ld_stream_v4(wr + c);
#pragma unroll
            for (int t = 0; t < MOE_DECODE_MAX_T; ++t)
                if (t < T)
                    acc[t] = dot8(wv, reinterpret_cast<const uint4 *>(x + (size_t)t * d)[c], acc[t]);
        }
#pragma unroll
        for (int t = 0; t < MOE_DECODE_MAX_T; ++t) {
            if (t < T) {
                const float s = warp_sum(acc[t]);
                if (lane == 0)
                    logits[(size_t)t * E + e] = s + (bias ? bias[e] : 0.f);
            }
        }
    }
}

// ---------------------------------------------------------------- phase 1: W1/W3 + SwiGLU
constexpr int kDecUnroll = 4;

__global__ void __launch_bounds__(256) k_dec_w13(const uint16_t *__restrict__ x,
                                                 const int32_t *__restrict__ idx, int T, int d,
                                                 int d_ff, int E, int k,
                                                 const uint16_t *__restrict__ W13, int d_ff_s,
                                                 const uint16_t *__restrict__ W13s,
                                                 uint16_t *__restrict__ Hdec,
                                                 uint16_t *__restrict__ Hs, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    build_plan(P, idx, T, E, k, status);
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
        int tok[MOE_DECODE_MAX_T];
#pragma unroll
        for (int s = 0; s < MOE_DECODE_MAX_T; ++s)
            tok[s] = (s < na) ? (shared ? s : P.list[a0 + s] / k) : 0;
        float ag[MOE_DECODE_MAX_T], au[MOE_DECODE_MAX_T];
#pragma unroll
        for (int s = 0; s < MOE_DECODE_MAX_T; ++s)
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
                for (int s = 0; s < MOE_DECODE_MAX_T; ++s) {
                    if (s < na) {
                        const uint4 xv = reinterpret_cast<const uint4 *>(x + (size_t)tok[s] * d)[ci];
                        ag[s] = dot8(wg[i], xv, ag[s]);
                        au[s] = dot8(wu[i], xv, au[s]);
                    }
                }
            }
        }
#pragma unroll
        for (int s = 0; s < MOE_DECODE_MAX_T; ++s) {
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
__global__ void __launch_bounds__(256) k_dec_w2(const int32_t *__restrict__ idx,
                                                const float *__restrict__ topk_w, int T, int d,
                                                int d_ff, int E, int k,
                                                const uint16_t *__restrict__ W2, int d_ff_s,
                                                const uint16_t *__restrict__ W2s,
                                                const uint16_t *__restrict__ Hdec,
                                                const uint16_t *__restrict__ Hs,
                                                float *__restrict__ out, uint32_t *status)
{
    __shared__ DecPlanSmem P;
    build_plan(P, idx, T, E, k, status);
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const int n_src = P.U + (W2s ? 1 : 0);
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < d; r += nwarps) {
        float acc[MOE_DECODE_MAX_T];
#pragma unroll
        for (int t = 0; t < MOE_DECODE_MAX_T; ++t)
            acc[t] = 0.f;
        for (int u = 0; u < n_src; ++u) {
            const bool shared = (u == P.U);
            const int ff = shared ? d_ff_s : d_ff;
            const uint4 *wrow = reinterpret_cast<const uint4 *>(
                shared ? W2s + (size_t)r * d_ff_s : W2 + ((size_t)P.uniq[u] * d + r) * d_ff);
            const int a0 = shared ? 0 : P.ustart[u];
            const int na = shared ? T : P.ustart[u + 1] - a0;
            int arow[MOE_DECODE_MAX_T];
#pragma unroll
            for (int s = 0; s < MOE_DECODE_MAX_T; ++s)
                arow[s] = (s < na) ? (shared ? s : P.list[a0 + s]) : 0;
            const uint16_t *hb = shared ? Hs : Hdec;
            const int nv = ff / 8;
            float pa[MOE_DECODE_MAX_T];
#pragma unroll
            for (int s = 0; s < MOE_DECODE_MAX_T; ++s)
                pa[s] = 0.f;
            for (int cb = 0; cb < nv; cb += 32 * kDecUnroll) {
                uint4 wv[kDecUnroll];
#pragma unroll
                for (int i = 0; i < kDecUnroll; ++i) {
                    const int ci = cb + lane + 32 * i;
                    if (ci < nv)
                        wv[i] = ld_stream_v4(wrow + ci);
                }
#pragma unroll
                for (int i = 0; i < kDecUnroll; ++i) {
                    const int ci = cb + lane + 32 * i;
                    if (ci >= nv)
                        continue;
#pragma unroll
                    for (int s = 0; s < MOE_DECODE_MAX_T; ++s)
                        if (s < na)
                            pa[s] = dot8(wv[i],
                                         reinterpret_cast<const uint4 *>(hb + (size_t)arow[s] * ff)[ci],
                                         pa[s]);
                }
            }
            // fold the lane partials into the tokens' accumulators, weighted
#pragma unroll
            for (int s = 0; s < MOE_DECODE_MAX_T; ++s) {
                if (s < na) {
                    const int t = shared ? s : arow[s] / k;
                    const float wgt = shared ? 1.f : topk_w[arow[s]];
#pragma unroll
                    for (int tt = 0; tt < MOE_DECODE_MAX_T; ++tt)
                        if (tt == t)
                            acc[tt] = fmaf(wgt, pa[s], acc[tt]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MOE_DECODE_MAX_T; ++t) {
            if (t < T) {
                const float s = warp_sum(acc[t]);
                if (lane == 0)
                    out[(size_t)t * d + r] = s;
            }
        }
    }
}

int launch_dec_w13(const moe_shape_t &s, const uint16_t *x, const int32_t *topk_idx,
                   const uint16_t *W13, const uint16_t *W13s, uint16_t *Hdec, uint32_t *status,
                   cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_dec_w13<<<num_sms() * 4, 256, 0, st>>>(x, topk_idx, s.T, s.d, s.d_ff, s.E, s.k, W13,
                                            s.d_ff_shared, s.d_ff_shared ? W13s : nullptr, Hdec,
                                            Hdec + (size_t)s.T * s.k * s.d_ff, status);
    return launched();
}

int launch_dec_w2(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                  const uint16_t *W2, const uint16_t *W2s, const uint16_t *Hdec, float *out,
                  uint32_t *status, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    k_dec_w2<<<num_sms() * 4, 256, 0, st>>>(topk_idx, topk_w, s.T, s.d, s.d_ff, s.E, s.k, W2,
                                           s.d_ff_shared, s.d_ff_shared ? W2s : nullptr, Hdec,
                                           Hdec + (size_t)s.T * s.k * s.d_ff, out, status);
    return launched();
}

int launch_dec_router(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                      const float *bias, float *logits, cudaStream_t st)
{
    if (s.T == 0)
        return MOE_OK;
    const int blocks = (s.E + 7) / 8;
    k_dec_router<<<blocks, 256, 0, st>>>(x, Wg, bias, s.T, s.d, s.E, logits);
    return launched();
}

} // namespace moe
