/*
 * moe.h -- C ABI of libmoe.so: the forward pass of a top-k routed
 * Mixture-of-Experts SwiGLU FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer (defined on "MoE Model Architectures", architectures.md, section
 * "Mixtral 8x7B", subsections "Sparse MoE Block" and "Expert FFN"; the bias
 * and the shared expert from section "DeepSeek-V3"):
 *   logits = x W_g^T + b                          router GEMM, fp32
 *   idx, w = top-k of softmax(logits), w / sum(w)  lowest index wins ties
 *   counts, offsets, permutation                   grouped by expert
 *   h      = silu(x W1_e^T) * (x W3_e^T)           per chosen expert, bf16
 *   out[t] = sum_j w[t,j] * (h W2_e^T) [+ shared]  fp32
 *
 * Conventions for every call
 *  - Tensor arguments are DEVICE pointers owned by the caller, contiguous and
 *    row-major, at least 16-byte aligned (256-byte alignment recommended).
 *    The library never allocates device memory, never frees the caller's
 *    memory and never synchronises the stream.
 *  - Scratch space comes from a caller-provided workspace `ws` of `ws_bytes`
 *    bytes (at least moe_workspace_size()), 256-byte aligned. Calls that
 *    share one workspace must be ordered on the GPU (same stream).
 *  - Every call is asynchronous on `stream` and performs no host<->device
 *    synchronisation, so a sequence of calls can be captured in a CUDA graph.
 *  - The return value is a host-detected status (MOE_OK or an MOE_ERR_* code).
 *    On any non-zero return nothing was launched. A launch failure reported
 *    by the CUDA runtime returns MOE_ERR_CUDA.
 *  - Errors found on the device are OR-ed into `*status` (a device uint32,
 *    which may be NULL to ignore them) as the bit (1u << MOE_ERR_*). The
 *    caller clears it and reads it whenever it chooses. When a device error
 *    is flagged, the outputs of that call are unspecified.
 *  - T = 0 is a valid no-op for every call (pointers may then be NULL);
 *    moe_permute then only zeroes the counts, offsets and n_kept it is given.
 *
 * Types: bf16 is the 16-bit bfloat16 bit pattern (uint16_t here); fp32 is
 * float; ids and positions are int32_t.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t;
typedef struct CUstream_st *moe_stream_t; /* same object as cudaStream_t; NULL = legacy default stream */

/* Status codes (host return values, and bit positions of the device word). */
enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, bad shape (see moe_shape_t), misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2, /* valid request that the library does not implement */
    MOE_ERR_WORKSPACE = 3,   /* ws too small or misaligned */
    MOE_ERR_CUDA = 4,        /* the CUDA runtime refused a launch or query */
    MOE_ERR_NONFINITE = 5,   /* device: a logit row holds NaN, or its maximum is +-inf */
    MOE_ERR_BAD_EXPERT = 6,  /* device: an expert id outside [0,E) or repeated within a token */
    MOE_ERR_TIMEOUT = 7,     /* device: a pipeline wait gave up (the kernel returned, no hang) */
    MOE_ERR_CHECK = 8        /* device: a dispatch consistency check failed (MOE_FLAG_DEBUG_CHECKS,
                                moe_check_dispatch) */
};

/* Flags (moe_shape_t.flags). */
enum {
    MOE_FLAG_DETERMINISTIC = 1 << 0, /* combine in a fixed order (y_perm + moe_combine) instead
                                        of fused fp32 atomics in the w2 epilogue */
    MOE_FLAG_FORCE_PREFILL = 1 << 1, /* moe_forward: never take the small-T decode kernels */
    MOE_FLAG_FORCE_DECODE = 1 << 2,  /* moe_forward: take the decode kernels whenever
                                        T <= MOE_DECODE_MAX_T (else MOE_ERR_UNSUPPORTED) */
    MOE_FLAG_SIMT_FFN = 1 << 3,      /* expert GEMMs on CUDA cores (slow debugging path that
                                        cross-checks the tensor-core kernels) */
    MOE_FLAG_HOST_IO = 1 << 4,       /* workspace also holds device staging for x and out,
                                        as moe_forward_host needs */
    MOE_FLAG_GEMM_1SM = 1 << 5,      /* tensor-core GEMMs: always the single-SM kernel */
    MOE_FLAG_GEMM_2SM = 1 << 6,      /* tensor-core GEMMs: the 2-SM pair kernel (256 x 256
                                        tiles, cta_group::2) wherever the output width is a
                                        multiple of 256 (default: the pair kernel for w2 when
                                        experts average >= 1024 rows, else single-SM) */
    MOE_FLAG_EXPERT_CHOICE = 1 << 7, /* workspace sized for the expert-choice calls
                                        (moe_route_expert_choice, moe_forward_expert_choice) */
    MOE_FLAG_SLOT_PRIORITY = 1 << 8, /* capacity ranks in slot-major order (see moe_shape_t) */
    MOE_FLAG_MXFP8 = 1 << 9,         /* workspace for moe_forward_mxfp8 (MXFP8 experts); the
                                        bf16 layer calls reject it */
    MOE_FLAG_BACKWARD = 1 << 10,     /* workspace also sized for moe_backward */
    MOE_FLAG_NVFP4 = 1 << 11,        /* workspace for moe_forward_nvfp4 (NVFP4 experts); the
                                        bf16 layer calls reject it */
    MOE_FLAG_DEBUG_CHECKS = 1 << 12  /* moe_permute and the prefill moe_forward also check the
                                        dispatch they built (moe_check_dispatch) and flag
                                        MOE_ERR_CHECK; the workspace holds one int32 per
                                        assignment more. A build with -DMOE_DEBUG sets it on
                                        every call */,
    MOE_FLAG_TEST_TIMEOUT = 1 << 13  /* test only, honoured by moe_expert_ffn alone: its w1/w3
                                        GEMM runs on the single-SM tensor-core kernel with a
                                        producer that issues no loads and pipeline waits
                                        bounded at 50 ms, so every CTA gives up its first wait,
                                        flags MOE_ERR_TIMEOUT, frees its tensor memory and
                                        returns with nothing in flight. Exercises the bounded
                                        waits; the call's results are meaningless */
};

#define MOE_MAX_E 256
#define MOE_MAX_K 16
#define MOE_DECODE_MAX_T 16     /* largest T the decode kernels accept */
#define MOE_DECODE_DEFAULT_T 2  /* moe_forward takes them for T <= this (measured crossover
                                   with the tensor-core chain on the Mixtral shape) */

/* Layer shape. Requirements (else MOE_ERR_INVALID_ARG):
 *   0 <= T <= 2^24; 1 <= E <= MOE_MAX_E; 1 <= k <= min(E, MOE_MAX_K);
 *   d and d_ff multiples of 128 in [128, 32768]; d_ff_shared 0 or a multiple
 *   of 128 in [128, 32768]; capacity <= 0 means uncapped.
 * capacity (reading of "Switch Transformers" / "Top-1 Routing" on the
 * architectures page, whose mask is garbled, and of "Faster writing: run only
 * the chosen experts", where a capacity factor of 0 means uncapped): an
 * assignment (t, j) is kept iff fewer than `capacity` assignments to the same
 * expert precede it in row-major (token, slot) order. Dropped assignments
 * contribute nothing and the kept weights are not renormalised.
 * With MOE_FLAG_SLOT_PRIORITY the order is slot-major (slot, token) instead:
 * every token's first choice ranks before any token's second choice (the
 * first-expert priority of top-2 dispatch with a capacity factor, the
 * "Capacity factor tuning" of the page's GLaM row), and an expert's kept
 * rows are laid out in that order (by slot, then ascending token). */
typedef struct moe_shape {
    int32_t T, d, d_ff, E, k;
    int32_t capacity;
    int32_t d_ff_shared;
    int32_t flags;
} moe_shape_t;

/* Short text for a status code (static storage). */
MOE_API const char *moe_status_string(int code);

/* Bytes of workspace that every call below needs for this shape and flags. */
MOE_API int moe_workspace_size(const moe_shape_t *shape, size_t *bytes);

/* Pack the expert gate and up projections for the tensor-core GEMM.
 *   W1, W3  [E, d_ff, d] bf16 (nn.Linear [out, in], "Expert FFN": w1, w3)
 *   W13     [E, 2*d_ff, d] bf16 output: for each block b of 128 columns,
 *           rows 256b..256b+127 are W1 rows 128b.., rows 256b+128..256b+255
 *           are W3 rows 128b.. (gate and up of a column side by side).
 * With E = 1 it packs a shared expert (d_ff = d_ff_shared). */
MOE_API int moe_pack_w13(const moe_shape_t *shape, const moe_bf16_t *W1, const moe_bf16_t *W3,
                 moe_bf16_t *W13, moe_stream_t stream);

/* Router and top-k ("Sparse MoE Block": gate -> softmax -> topk -> divide by
 * the sum; bias from "Auxiliary-Loss-Free Load Balancing").
 *   x       [T, d] bf16, or NULL: then `logits` is an INPUT [T, E] fp32
 *   Wg      [E, d] bf16 (ignored when x is NULL)
 *   bias    [E] fp32 or NULL (ignored when x is NULL)
 *   logits  [T, E] fp32, output (x != NULL) or input (x == NULL)
 *   topk_idx [T, k] int32 out: experts in selection order (largest logit
 *            first; equal logits -> lower index first; -0.0 == +0.0)
 *   topk_w  [T, k] fp32 out: exp(l_j - max) / sum over the chosen k, which
 *           equals the softmax over all E renormalised over the top-k
 * Device errors: MOE_ERR_NONFINITE. */
MOE_API int moe_route(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
              const float *bias, float *logits, int32_t *topk_idx, float *topk_w,
              uint32_t *status, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Expert histogram, offsets, capacity and token permutation ("Current Bug:
 * CuTeDSLMoERunner produces wrong output", "How the pipeline works": counts
 * [4,4,0] -> offsets [0,4,8,8]; "Sparse MoE Block": torch.where order).
 *   topk_idx       [T, k] int32 in: distinct ids in [0, E) per token
 *   x              [T, d] bf16 in (may be NULL: then x_perm is not written)
 *   expert_counts  [E] int32 out: routed assignments per expert (before capacity)
 *   expert_offsets [E+1] int32 out: exclusive scan of min(count, capacity)
 *   slot_pos       [T, k] int32 out: permuted row of (t, j), -1 if dropped
 *   perm_token     [T*k] int32 out: token of each permuted row; rows within an
 *                  expert are in ascending token order (MOE_FLAG_SLOT_PRIORITY:
 *                  by slot, then token); rows >= n_kept untouched
 *   x_perm         [T*k, d] bf16 out: x_perm[slot_pos[t,j]] = x[t]
 *   n_kept         [1] int32 out: expert_offsets[E]
 * Bit-exact: the result is a function of topk_idx alone.
 * Device errors: MOE_ERR_BAD_EXPERT. */
MOE_API int moe_permute(const moe_shape_t *shape, const int32_t *topk_idx, const moe_bf16_t *x,
                int32_t *expert_counts, int32_t *expert_offsets, int32_t *slot_pos,
                int32_t *perm_token, moe_bf16_t *x_perm, int32_t *n_kept, uint32_t *status,
                void *ws, size_t ws_bytes, moe_stream_t stream);

/* Grouped expert FFN over the chosen experts only ("Expert FFN", run on the
 * rows [offsets[e], offsets[e+1]) of each expert as "Sparse MoE Block" does).
 *   x_perm   [T*k, d] bf16 in; expert_offsets [E+1] int32 in
 *   W13      [E, 2*d_ff, d] bf16 (moe_pack_w13); W2 [E, d, d_ff] bf16
 *   perm_token [T*k], slot_pos [T, k] int32, topk_w [T, k] fp32 (used only
 *            by the fused combine)
 *   y_perm   [T*k, d] fp32 or NULL. Non-NULL: writes the UNWEIGHTED expert
 *            output of each kept row (for moe_combine); `out` is ignored.
 *            NULL: fused combine, out[perm_token[r]] += w * y[r] with fp32
 *            atomics; `out` [T, d] fp32 must hold zeros or a partial sum
 *            (e.g. the shared expert's output).
 * H, the bf16 SwiGLU product [T*k, d_ff], lives in the workspace. */
MOE_API int moe_expert_ffn(const moe_shape_t *shape, const moe_bf16_t *x_perm,
                   const int32_t *expert_offsets, const moe_bf16_t *W13, const moe_bf16_t *W2,
                   const int32_t *perm_token, const int32_t *slot_pos, const float *topk_w,
                   float *y_perm, float *out, uint32_t *status, void *ws, size_t ws_bytes,
                   moe_stream_t stream);

/* Routing-weighted combine in a fixed order ("Sparse MoE Block": scale by
 * the routing weight, index_add into token order; "DeepSeekMoE Architecture":
 * shared_output + routed_output):
 *   out[t] = shared_out[t] + sum_{j = 0..k-1, slot_pos[t,j] >= 0} w[t,j] * y_perm[slot_pos[t,j]]
 *   y_perm [T*k, d] fp32; slot_pos [T, k]; topk_w [T, k]; shared_out [T, d]
 *   fp32 or NULL; out [T, d] fp32 (may alias shared_out). Deterministic. */
MOE_API int moe_combine(const moe_shape_t *shape, const float *y_perm, const int32_t *slot_pos,
                const float *topk_w, const float *shared_out, float *out, moe_stream_t stream);

/* The whole layer forward, one stream, no host synchronisation.
 *   x [T, d] bf16; Wg [E, d] bf16; bias [E] fp32 or NULL;
 *   W13 [E, 2*d_ff, d] bf16 packed; W2 [E, d, d_ff] bf16;
 *   W13_shared [2*d_ff_shared, d] bf16 packed and W2_shared [d, d_ff_shared]
 *   bf16 when d_ff_shared > 0 (else NULL);
 *   out [T, d] fp32 (fully written);
 *   logits_out [T, E] fp32, topk_idx_out [T, k] int32: optional copies.
 * T <= MOE_DECODE_DEFAULT_T takes the decode kernels, which stream only the
 * chosen experts' weights once ("Faster writing: run only the chosen
 * experts"; "perf(moe): route granite-4.0-h single-token MoE through the fused
 * kernel"); larger T takes router -> top-k -> histogram -> permute -> grouped
 * tensor-core GEMMs with the SwiGLU and the weighted combine in their
 * epilogues, which also read only the chosen experts (tiles exist only for
 * experts with rows). Device errors: NONFINITE, BAD_EXPERT, TIMEOUT. */
MOE_API int moe_forward(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W2,
                const moe_bf16_t *W13_shared, const moe_bf16_t *W2_shared, float *out,
                float *logits_out, int32_t *topk_idx_out, uint32_t *status, void *ws,
                size_t ws_bytes, moe_stream_t stream);

/* moe_forward from and to HOST memory: copies x_host [T, d] bf16 into the
 * workspace, runs the layer, copies out [T, d] fp32 back into out_host, all
 * asynchronously on `stream` (cudaMemcpyAsync; use pinned host buffers for
 * true asynchrony). The caller synchronises the stream before reading
 * out_host. Weights and bias are device pointers as in moe_forward. The
 * workspace must be sized with MOE_FLAG_HOST_IO set in shape->flags.
 * An uncapped batch of at least 4096 tokens (each token's output depends on
 * its own row only) is processed in up to 4 chunks: the library forks two
 * copy streams of its own (created once per device) from `stream`, so each
 * chunk's upload and download overlap the other chunks' compute, and joins
 * them back into `stream` before returning. Results equal the unchunked ones
 * (bit for bit with MOE_FLAG_DETERMINISTIC or k <= 2; otherwise up to the order
 * of the fp32 atomic additions of the combine).
 * Not for concurrent calls from several host threads on one device. */
MOE_API int moe_forward_host(const moe_shape_t *shape, const moe_bf16_t *x_host, const moe_bf16_t *Wg,
                     const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W2,
                     const moe_bf16_t *W13_shared, const moe_bf16_t *W2_shared, float *out_host,
                     uint32_t *status, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Expert-choice routing ("MoE Model Architectures", "Design Patterns",
 * "Pattern 3: Expert Choice Routing": experts choose tokens instead of tokens
 * choosing experts). Requires MOE_FLAG_EXPERT_CHOICE in shape->flags (also
 * for moe_workspace_size) and shape->capacity = C >= 1; shape->k is not used
 * (any valid value, e.g. 1). MOE_FLAG_DETERMINISTIC and MOE_FLAG_HOST_IO are
 * rejected with MOE_ERR_INVALID_ARG: the combine adds each expert's weighted
 * rows into out with atomics, so the last bits of out may differ between runs.
 *   score S[t, e] = softmax over experts of token t's logits (fp32);
 *   expert e takes the K = min(C, T) tokens with the largest S[:, e], equal
 *   scores going to the lower token index;
 *   out[t] = sum over the experts that took t of S[t, e] * FFN_e(x_t)
 *            (+ the shared expert), not renormalised; a token no expert takes
 *            gets only the shared expert (or zero).
 * moe_route_expert_choice:
 *   x [T, d] bf16 or NULL: with x, logits [T, E] (out, or NULL to keep them in
 *   the workspace) and scores [T, E] (out) are computed; with x == NULL,
 *   scores [T, E] fp32 is the INPUT (identical scores give bit-identical
 *   selections).
 *   expert_tokens [E, K] int32 out: each expert's tokens, ascending;
 *   expert_w [E, K] fp32 out: their scores S[t, e].
 *   Device errors: MOE_ERR_NONFINITE (NaN logit or score). */
MOE_API int moe_route_expert_choice(const moe_shape_t *shape, const moe_bf16_t *x,
                                    const moe_bf16_t *Wg, const float *bias, float *logits,
                                    float *scores, int32_t *expert_tokens, float *expert_w,
                                    uint32_t *status, void *ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* The whole layer under expert-choice routing: router, softmax, per-expert
 * top-K, gather, grouped w1/w3 GEMM + SwiGLU, grouped w2 GEMM with the
 * score-weighted combine into out [T, d] fp32 (fully written). Arguments as
 * in moe_forward. */
MOE_API int moe_forward_expert_choice(const moe_shape_t *shape, const moe_bf16_t *x,
                                      const moe_bf16_t *Wg, const float *bias,
                                      const moe_bf16_t *W13, const moe_bf16_t *W2,
                                      const moe_bf16_t *W13_shared, const moe_bf16_t *W2_shared,
                                      float *out, uint32_t *status, void *ws, size_t ws_bytes,
                                      moe_stream_t stream);

/* ---- MXFP8 experts: block-scaled 8-bit weights and activations
 * (the low-precision expert pipeline of "Current Bug: CuTeDSLMoERunner
 * produces wrong output": per-expert weight and activation scale factors
 * feeding a block-scaled grouped GEMM; the encoding is OCP "Microscaling (MX)
 * Formats" v1.0 MXFP8, which the page does not fix):
 *   - a block is 32 consecutive elements along the contraction dimension
 *     (d for x and w1/w3, d_ff for h and w2);
 *   - its scale is 2^X, X the smallest integer in [-127, 127] with
 *     max|v| <= 448 * 2^X (no element saturates), stored as the E8M0 byte
 *     X + 127;
 *   - its elements are E4M3 codes of v * 2^-X, rounded to nearest even.
 * The router, top-k and dispatch are those of moe_forward (bf16 W_g, fp32
 * logits); x and h are quantized on the fly; the GEMMs accumulate in fp32;
 * out is fp32.
 *
 * moe_quantize_experts_mxfp8: one-time conversion of bf16 experts.
 *   W1, W3  [E, d_ff, d] bf16 in; W2 [E, d, d_ff] bf16 in
 *   W13q    [E, 2*d_ff, d] E4M3 out, packed: for each block b of 64 h
 *           columns, rows 128b..128b+63 are W1 rows 64b.., rows 128b+64..
 *           128b+127 are W3 rows 64b.. (gate and up side by side in one
 *           128-column tile)
 *   W13sf   E*2*d_ff*d/32 E8M0 bytes out, in the scale-atom order the
 *           block-scaled tensor-core MMA reads: the scales of rows
 *           128t..128t+127 and K elements 128g..128g+127 form the 512-byte
 *           atom (t * (K/128) + g), inside which row 128t + m, 32-element
 *           block 4g + j sits at byte (m % 32) * 16 + (m / 32) * 4 + j
 *           (K = d; rows in W13q's packed order)
 *   W2q     [E, d, d_ff] E4M3 out; W2sf E*d*d_ff/32 E8M0 bytes out, atoms as
 *           above with K = d_ff
 * With E = 1 and d_ff = d_ff_shared it converts a shared expert. All four
 * arrays 16-byte aligned. */
MOE_API int moe_quantize_experts_mxfp8(const moe_shape_t *shape, const moe_bf16_t *W1,
                                       const moe_bf16_t *W3, const moe_bf16_t *W2,
                                       uint8_t *W13q, uint8_t *W13sf, uint8_t *W2q,
                                       uint8_t *W2sf, moe_stream_t stream);

/* The layer with MXFP8 experts. Requires MOE_FLAG_MXFP8 in shape->flags
 * (also when sizing the workspace); MOE_FLAG_HOST_IO is rejected
 * (MOE_ERR_INVALID_ARG). Arguments as in moe_forward, with the experts (and
 * the shared expert, when d_ff_shared > 0) as moe_quantize_experts_mxfp8
 * writes them. MOE_FLAG_DETERMINISTIC, capacity, MOE_FLAG_SLOT_PRIORITY and
 * the decode / prefill choice (MOE_FLAG_FORCE_*) act as in moe_forward: small
 * T streams only the chosen experts' codes and scales (8.25 bits a weight);
 * larger T runs the block-scaled tensor-core GEMMs.
 * Device errors: MOE_ERR_NONFINITE, MOE_ERR_BAD_EXPERT, MOE_ERR_TIMEOUT. */
MOE_API int moe_forward_mxfp8(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                              const float *bias, const uint8_t *W13q, const uint8_t *W13sf,
                              const uint8_t *W2q, const uint8_t *W2sf, const uint8_t *W13s_q,
                              const uint8_t *W13s_sf, const uint8_t *W2s_q,
                              const uint8_t *W2s_sf, float *out, float *logits_out,
                              int32_t *topk_idx_out, uint32_t *status, void *ws, size_t ws_bytes,
                              moe_stream_t stream);

/* ---- NVFP4 experts: block-scaled 4-bit weights and activations
 * (the NVFP4 grouped GEMM of "Current Bug: CuTeDSLMoERunner produces wrong
 * output", "How the pipeline works": per-expert weight scales and activation
 * scales feeding a block-scaled grouped GEMM; the page does not spell the
 * format out, this is NVIDIA's NVFP4):
 *   - an element is E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), packed two
 *     to a byte, element 2i in the low nibble of byte i;
 *   - a block is 16 consecutive elements along the contraction dimension,
 *     with one E4M3 scale s;
 *   - a tensor has one fp32 global encode scale gs: 448 * 6 / max|W| per
 *     expert for the weights (W1 and W3 of an expert share one, W2 has its
 *     own; 1 for an all-zero tensor), and the caller's constants x_gs and
 *     h_gs for x and for the SwiGLU product h;
 *   - encoding, each step an IEEE fp32 operation: s = E4M3((amax / 6) * gs),
 *     nearest even, saturating; r = gs / s (0 when s = 0); code = E2M1(v * r),
 *     nearest even, saturating at 6. A code stands for E2M1 * s / gs.
 * The router, top-k and dispatch are those of moe_forward; x and h are
 * quantized on the fly; the GEMMs (tcgen05 kind::mxf4nvf4, 16-element
 * blocks) accumulate in fp32 and multiply by 1 / (gs_activation * gs_weight);
 * out is fp32. d, d_ff and d_ff_shared must be multiples of 256
 * (MOE_ERR_UNSUPPORTED otherwise).
 *
 * moe_quantize_experts_nvfp4: one-time conversion of bf16 experts.
 *   W1, W3  [E, d_ff, d] bf16 in; W2 [E, d, d_ff] bf16 in
 *   W13q    [E, 2*d_ff, d/2] bytes out: packed E2M1 codes, rows in the
 *           64-row gate/up interleave of moe_quantize_experts_mxfp8
 *   W13sf   E*2*d_ff*d/16 E4M3 bytes out, in 512-byte atoms: the scales of
 *           rows 128t..128t+127 and K elements 64g..64g+63 form atom
 *           (t * (K/64) + g), inside which row 128t + m, block 4g + j sits at
 *           byte (m % 32) * 16 + (m / 32) * 4 + j (K = d, packed rows)
 *   W13_gs  [E] fp32 out: the global encode scale of expert e's W1 and W3
 *   W2q     [E, d, d_ff/2] bytes out; W2sf E*d*d_ff/16 bytes out, atoms as
 *           above with K = d_ff; W2_gs [E] fp32 out
 * With E = 1 and d_ff = d_ff_shared it converts a shared expert. Code and
 * scale arrays 16-byte aligned, scale vectors 4-byte aligned. */
MOE_API int moe_quantize_experts_nvfp4(const moe_shape_t *shape, const moe_bf16_t *W1,
                                       const moe_bf16_t *W3, const moe_bf16_t *W2,
                                       uint8_t *W13q, uint8_t *W13sf, float *W13_gs,
                                       uint8_t *W2q, uint8_t *W2sf, float *W2_gs,
                                       moe_stream_t stream);

/* The layer with NVFP4 experts. Requires MOE_FLAG_NVFP4 in shape->flags (also
 * when sizing the workspace); MOE_FLAG_HOST_IO and MOE_FLAG_MXFP8 are
 * rejected (MOE_ERR_INVALID_ARG), as are x_gs or h_gs that are not positive
 * and finite. Arguments as in moe_forward_mxfp8, with each weight set's
 * global scales (device pointers, as moe_quantize_experts_nvfp4 writes them).
 * T <= MOE_DECODE_DEFAULT_T takes the NVFP4 decode kernels ("perf(moe): route
 * granite-4.0-h single-token MoE through the fused kernel": a 4-bit
 * single-token path fed by the top-k indices and weights): x and h are
 * quantized as the tensor-core chain quantizes them, and each chosen expert's
 * codes and scales are streamed once into block-scaled tensor-core MMAs whose
 * N side is the tokens (d a multiple of 256, T k <= 16 for w2; other shapes
 * stream them through CUDA cores, every 16-element block dot product exact
 * in f16). The output is the same bit for bit on every call with the same
 * inputs and launch shape (fixed-order sums). Larger T runs the block-scaled tensor-core
 * GEMMs, which also read each chosen expert's codes and scales once (4.5
 * bits a weight). MOE_FLAG_FORCE_DECODE takes the decode kernels for T <= 2
 * and is MOE_ERR_UNSUPPORTED above; MOE_FLAG_FORCE_PREFILL takes the chain.
 * MOE_FLAG_DETERMINISTIC, capacity and MOE_FLAG_SLOT_PRIORITY act as in
 * moe_forward.
 * Device errors: MOE_ERR_NONFINITE, MOE_ERR_BAD_EXPERT, MOE_ERR_TIMEOUT. */
MOE_API int moe_forward_nvfp4(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                              const float *bias, const uint8_t *W13q, const uint8_t *W13sf,
                              const float *W13_gs, const uint8_t *W2q, const uint8_t *W2sf,
                              const float *W2_gs, const uint8_t *W13s_q, const uint8_t *W13s_sf,
                              const float *W13s_gs, const uint8_t *W2s_q, const uint8_t *W2s_sf,
                              const float *W2s_gs, float x_gs, float h_gs, float *out,
                              float *logits_out, int32_t *topk_idx_out, uint32_t *status,
                              void *ws, size_t ws_bytes, moe_stream_t stream);

/* ---- Backward pass ("Sparse MoE Block" / "Expert FFN" differentiated with the
 * routing decisions held fixed: top-k set, capacity drops, slot order).
 *
 * moe_pack_backward: the transposed expert weights the backward GEMMs read,
 * from the forward's packed W13 and W2 (once per weight update):
 *   W13T [E, d, 2*d_ff] bf16 out: W13T[e][i][p] = W13[e][p][i]
 *   W2T  [E, d_ff, d]   bf16 out: W2T[e][c][i]  = W2[e][i][c] */
MOE_API int moe_pack_backward(const moe_shape_t *shape, const moe_bf16_t *W13,
                              const moe_bf16_t *W2, moe_bf16_t *W13T, moe_bf16_t *W2T,
                              moe_stream_t stream);

/* Gradients of sum(out * dout) for the layer moe_forward computes (routing
 * recomputed with the same kernels, so it is identical). Requires
 * MOE_FLAG_BACKWARD in shape->flags (also for moe_workspace_size); rejects
 * MOE_FLAG_MXFP8, MOE_FLAG_NVFP4 and MOE_FLAG_SIMT_FFN (MOE_ERR_INVALID_ARG).
 *   x, Wg, bias, W13  as moe_forward; W13T, W2T as moe_pack_backward writes
 *   W13_shared, W13T_shared, W2T_shared: with d_ff_shared > 0, the shared
 *         expert's packed W13 [2*d_ff_shared, d] and its transposes (from
 *         moe_pack_backward with E = 1, d_ff = d_ff_shared); else NULL
 *   dout  [T, d] fp32 in
 *   dx    [T, d] fp32 out: through the experts and through the router
 *   dW13  [E, 2*d_ff, d] fp32 out, in the packed W13 order (rows of dW1 and
 *         dW3 interleaved by 128 as in moe_pack_w13)
 *   dW2   [E, d, d_ff] fp32 out
 *   dW13_shared [2*d_ff_shared, d], dW2_shared [d, d_ff_shared] fp32 out
 *         (with d_ff_shared > 0; else NULL)
 *   dWg   [E, d] fp32 out; dbias [E] fp32 out (written even if bias is NULL)
 *   dlogits [T, E] fp32 out, or NULL
 * For a kept assignment (t, j) to expert e with weight w: dW2_e += w dout_t
 * h^T, dh = w W2_e^T dout_t, du = dh silu(g), dg = dh u silu'(g),
 * dW1_e += dg x^T, dW3_e += du x^T, dx_t += W1_e^T dg + W3_e^T du; the
 * router: dl_j = w_j G_j - w_j sum_i w_i G_i with G_j = <dout_t, y_j> over the
 * chosen experts, dWg += dl^T x, dbias += sum_t dl, dx += dl Wg. bf16
 * operands (x, h, w*dout, [dg | du], gate/up), fp32 accumulation. The weight
 * gradients are plain per-expert GEMMs (bitwise repeatable); dx and dlogits
 * use fp32 atomic adds. */
MOE_API int moe_backward(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                         const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W13T,
                         const moe_bf16_t *W2T, const moe_bf16_t *W13_shared,
                         const moe_bf16_t *W13T_shared, const moe_bf16_t *W2T_shared,
                         const float *dout, float *dx, float *dW13, float *dW2,
                         float *dW13_shared, float *dW2_shared, float *dWg, float *dbias,
                         float *dlogits, uint32_t *status, void *ws, size_t ws_bytes,
                         moe_stream_t stream);

/* Consistency check of a dispatch (the debug bounds checks of the permutation,
 * which the pages do not describe; they guard the offsets bug class of
 * "Current Bug: CuTeDSLMoERunner produces wrong output", "Root Cause:
 * scale_a layout doesn't match expert_offsets"). Reads, never writes, the
 * dispatch; sets the bit (1u << MOE_ERR_CHECK) of *status when any of these
 * fails, and (1u << MOE_ERR_BAD_EXPERT) for an id outside [0, E):
 *   expert_offsets[0] = 0, nondecreasing, expert_offsets[E] = *n_kept <= T*k,
 *   and with a capacity C > 0 no expert holds more than C rows;
 *   every kept slot_pos[t, j] lies in [expert_offsets[e], expert_offsets[e+1])
 *   of its expert e = topk_idx[t, j], and perm_token of that row is t;
 *   without a capacity no assignment is dropped (slot_pos = -1 only with C > 0;
 *   any other negative value fails);
 *   every row in [0, n_kept) is the slot of exactly one assignment.
 *   Every read is bounds-checked first, so a corrupt dispatch raises the
 *   status bit and nothing else. The workspace must be sized with
 *   MOE_FLAG_DEBUG_CHECKS in shape->flags (one int32 per assignment). */
MOE_API int moe_check_dispatch(const moe_shape_t *shape, const int32_t *topk_idx,
                               const int32_t *expert_offsets, const int32_t *slot_pos,
                               const int32_t *perm_token, const int32_t *n_kept, uint32_t *status,
                               void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory: engines that reserve all device memory for their own pool, and
 * paths that cannot pay for cudaMalloc/cudaFree (cudaFree synchronises the
 * device). The pages have no counterpart of this call.
 *   Arguments, outputs and results are those of moe_permute (bit-identical),
 *   minus ws/ws_bytes: the scratch is one fixed 4 MiB array inside the
 *   library's device image, held on every GPU that loads the library until
 *   the process exits. Shapes whose scratch does not fit return
 *   MOE_ERR_UNSUPPORTED and launch nothing; every shape with T*k <= 262144
 *   and T <= 262144 fits.
 *   The call allocates nothing. Its first call on a device looks up the
 *   array's device address (cudaGetSymbolAddress, with that device current)
 *   and caches it with the device's context; make that first call before any
 *   stream capture. After a device reset the next call looks the address up
 *   again.
 *   All calls share the one array and each call clears what must start at
 *   zero, so calls that overlap on the GPU (other streams, other host threads)
 *   race and corrupt each other's results: order them on one stream. */
MOE_API int moe_permute_static(const moe_shape_t *shape, const int32_t *topk_idx,
                               const moe_bf16_t *x, int32_t *expert_counts, int32_t *expert_offsets,
                               int32_t *slot_pos, int32_t *perm_token, moe_bf16_t *x_perm,
                               int32_t *n_kept, uint32_t *status, moe_stream_t stream);

/* ---- Instrumentation (computes nothing; for measurement and tests). ---- */

/* Stages of moe_forward (and moe_backward) timed by the profiler below; in
 * moe_backward, W13 is the w1/w3 recompute and W2 the dh GEMM. */
enum {
    MOE_STAGE_ROUTER = 0,   /* router logits */
    MOE_STAGE_TOPK = 1,     /* softmax / top-k / weights */
    MOE_STAGE_HIST = 2,     /* histogram, offsets, tile list */
    MOE_STAGE_PERMUTE = 3,  /* permutation and gather of x */
    MOE_STAGE_SHARED = 4,   /* shared expert (both GEMMs) */
    MOE_STAGE_W13 = 5,      /* grouped w1/w3 GEMM + SwiGLU */
    MOE_STAGE_W2 = 6,       /* grouped w2 GEMM + weighted combine */
    MOE_STAGE_COMBINE = 7,  /* fixed-order combine (deterministic mode) */
    MOE_STAGE_DEC_W13 = 8,  /* decode: chosen experts' w1/w3 + SwiGLU */
    MOE_STAGE_DEC_W2 = 9,   /* decode: chosen experts' w2 + combine */
    MOE_STAGE_BWD_DX = 10,  /* backward: dx through the experts */
    MOE_STAGE_BWD_DW = 11,  /* backward: transposes + per-expert weight-gradient GEMMs */
    MOE_STAGE_BWD_ROUTER = 12, /* backward: router gradient (dlogits, dWg, dbias, dx) */
    MOE_NUM_STAGES = 13
};

/* Number of kernels this library has launched in this process. */
MOE_API uint64_t moe_kernel_launches(void);

/* on != 0: from now on moe_forward records a CUDA event before and after each
 * stage, on the caller's stream (events are created here, once); on == 0:
 * stop recording. Not for concurrent use from several host threads. */
MOE_API int moe_profile_enable(int on);

/* Wait for the recorded events, then write per-stage total milliseconds and
 * call counts since the last read (arrays of n <= MOE_NUM_STAGES entries;
 * either may be NULL) and forget the records. */
MOE_API int moe_profile_read(double *ms, int64_t *calls, int n);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
