// internal.h -- host-side interface between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Counts every kernel launch of this library (moe_kernel_launches).
void note_launch();

// Call right after one kernel launch: counts it and maps the launch result.
inline int launched()
{
    note_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may start while
// its predecessor in the stream is still running, so it must execute
// griddepcontrol.wait (pdl_wait) before it reads anything a predecessor
// writes. Returns the launch's error code.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr int kBlockM = 128;      // rows of one grouped-GEMM m-tile
// Bit of an m-tile's group entry marking a tail tile of at most 64 rows: the
// single-SM tensor-core GEMM runs it with M = 64 MMAs and loads 64 A rows
// (an M = 64 MMA takes as many tensor-pipe cycles as an M = 128 one).
constexpr int32_t kHalfTileBit = 1 << 30;
constexpr int kChunkTokens = 256; // tokens per histogram chunk (one CTA)

// Capacity ranks in slot-major order (MOE_FLAG_SLOT_PRIORITY with a capacity).
inline int slot_major(const moe_shape_t &s)
{
    return (s.flags & MOE_FLAG_SLOT_PRIORITY) ? 1 : 0;
}
// Per-chunk count rows of the histogram: one per chunk, or one per (chunk, slot).
inline size_t chunk_count_rows(const moe_shape_t &s, size_t nchunks)
{
    return nchunks * (slot_major(s) ? (size_t)s.k : 1);
}

// Scratch layout inside the caller's workspace (byte offsets, 256-B aligned).
struct WsLayout {
    size_t logits, topk_idx, topk_w;
    size_t counts, offsets, n_kept, counter, num_mt;
    size_t chunk_counts, rank_local;
    size_t slot_pos, perm_token;
    size_t mt_row0, mt_group;
    size_t mt2_row0, mt2_group, num_mt2;   // 256-row tiles of the 2-SM GEMM
    size_t mt_first, mt2_first;            // E + 1 ints each (build_tiles)
    size_t x_perm, H, H_shared, Y;
    size_t dec_H;
    size_t x_stage, out_stage;
    size_t scores, ec_w;   // expert-choice routing
    size_t xq, xsf, Hq, Hsf, xq_s, xsf_s, Hsq, Hssf;   // MXFP8 operands
    size_t dec_xdq, dec_H32;                             // MXFP8 / NVFP4 decode
    size_t dec_xs, dec_hs;                               // NVFP4 decode: scale values
    size_t dec_part;                                     // NVFP4 decode: split-K sums
    size_t dec_hq, dec_hsf, dec_hqs, dec_hsfs;           // NVFP4 decode: h as the w2 operand
    size_t tile_start;                                   // first m-tile of each expert
    size_t dbg_seen;                                     // dispatch checks: count per row
    // backward pass
    size_t GU, dYw, dGU, row_dot, pstart, kb0, nkb, mtk1_row0, mtk1_group, mtk2_row0,
        mtk2_group, dYwT, HT, dGUT, XpT, dl, dwg_part;
    // backward of the shared expert
    size_t s_GU, s_dout, s_dGU, s_rowdot, s_offs, s_pstart, s_kb0, s_nkb, s_mt1_row0,
        s_mt1_group, s_mt2_row0, s_mt2_group, s_doutT, s_HT, s_dGUT, s_xT;
    long long Tp;
    long long Np;                                        // padded rows of the transposes
    size_t total;
    int nchunks, max_mt, max_mt2;
};

WsLayout ws_layout(const moe_shape_t &s);

// The shape rules every entry point applies (MOE_OK or MOE_ERR_INVALID_ARG).
int check_shape(const moe_shape_t *s);

// ---- routing / dispatch (dispatch.cu)
int launch_router_simt(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                       const float *bias, float *logits, cudaStream_t st);
int launch_topk(const moe_shape_t &s, const float *logits, int32_t *idx, float *w,
                int32_t *counter_to_zero, uint32_t *status, cudaStream_t st);
// Also writes the 256-row m-tile list of the 2-SM GEMM when mt2_row0 is non-NULL.
// mt_first / mt2_first (E + 1 ints each, may be NULL): the lists' expert
// positions for the GEMMs' band order (build_tiles in tiles.cuh).
int launch_hist_scan(const moe_shape_t &s, const int32_t *idx, int32_t *chunk_counts,
                     int32_t *rank_local, int32_t *counter, int32_t *counts, int32_t *offsets,
                     int32_t *n_kept, int32_t *mt_row0, int32_t *mt_group, int32_t *num_mt,
                     int32_t *mt2_row0, int32_t *mt2_group, int32_t *num_mt2, uint32_t *status,
                     cudaStream_t st, int32_t *tile_start = nullptr, int32_t *mt_first = nullptr,
                     int32_t *mt2_first = nullptr);
int launch_permute(const moe_shape_t &s, const int32_t *idx, const int32_t *chunk_base,
                   const int32_t *rank_local, const int32_t *offsets, const uint16_t *x,
                   int32_t *slot_pos, int32_t *perm_token, uint16_t *x_perm, float *out_zero,
                   cudaStream_t st, int chunk_tokens = kChunkTokens);
int launch_tiles_from_offsets(const moe_shape_t &s, const int32_t *offsets, int32_t *mt_row0,
                              int32_t *mt_group, int32_t *num_mt, int32_t *mt2_row0,
                              int32_t *mt2_group, int32_t *num_mt2, cudaStream_t st,
                              int32_t *mt_first = nullptr, int32_t *mt2_first = nullptr);
int launch_combine(const moe_shape_t &s, const float *y_perm, const int32_t *slot_pos,
                   const float *topk_w, const float *shared_out, float *out, cudaStream_t st);
int launch_pack_w13(int E, int d_ff, int d, const uint16_t *W1, const uint16_t *W3,
                    uint16_t *W13, cudaStream_t st);
// Debug consistency checks of a dispatch (seen: T*k int32 of scratch).
int launch_check_dispatch(const moe_shape_t &s, const int32_t *idx, const int32_t *offsets,
                          const int32_t *slot_pos, const int32_t *perm_token,
                          const int32_t *n_kept, int32_t *seen, uint32_t *status, cudaStream_t st);
// Whether the dispatch checks run: MOE_FLAG_DEBUG_CHECKS, or every call in a
// build compiled with -DMOE_DEBUG.
inline bool debug_checks(const moe_shape_t &s)
{
#ifdef MOE_DEBUG
    (void)s;
    return true;
#else
    return (s.flags & MOE_FLAG_DEBUG_CHECKS) != 0;
#endif
}

// ---- grouped GEMMs (gemm_tc.cu: tcgen05 + TMA; gemm_simt.cu: CUDA cores)
enum EpiMode {
    EPI_SWIGLU = 0,     // H[row, n*128 + c] = bf16(silu(acc[c]) * acc[128 + c])
    EPI_COMBINE = 1,    // out[perm_token[row], :] += w(row) * acc  (fp32 atomics)
    EPI_STORE_F32 = 2,  // out[row, :] = acc  (fp32)
    EPI_ROUTER = 3,     // out[row, n] = acc[n] + bias[n] for n < n_valid
    EPI_SWIGLU_MX = 4,  // MXFP8 GEMM: h = silu(gate) * up, quantized to MXFP8 codes (out)
                        // and block scales (out_sf)
    EPI_ROUTER_TOPK = 5,// EPI_ROUTER, then (E <= 64, one 64-column tile) the top-k of each
                        // row and its renormalised weights into route_idx / route_w
    EPI_SWIGLU_SAVE = 6,// EPI_SWIGLU, and the raw gate / up accumulators as bf16 in the packed
                        // W13 order into out2 [rows, 2 N/2] (for the backward pass)
    EPI_SWIGLU_BWD = 7  // backward through SwiGLU: acc = dh; reads the saved gate / up (gu),
                        // writes [dg | du] bf16 in the packed order into out and adds
                        // sum_c dh * h per row into row_dot (fp32)
};

// Block-scaled operand formats of launch_gemm_mx (GemmArgs::fmt).
enum BlockFormat { FMT_MX8 = 0, FMT_NV4 = 1 };

struct GemmArgs {
    int mode;
    // A [a_rows, K] bf16 row-major; B [groups * b_rows_per_group, K] bf16 row-major
    const uint16_t *A;
    long long a_rows;
    const uint16_t *B;
    long long b_rows_total;
    int K;
    int N;                    // output columns of one group (2*d_ff for SWIGLU)
    int b_rows_per_group;
    // m-tiles: routed (list on device) or identity (row0 = 128 * i)
    const int32_t *mt_row0;   // NULL: identity tiles
    const int32_t *mt_group;
    const int32_t *num_mt_dev; // NULL: use num_mt_host
    int num_mt_host;
    int max_mt;               // upper bound of the m-tile count (grid sizing)
    // routed lists in build_tiles' order: each group's first position, and at
    // [n_groups] the multi-tile part's length; NULL: plain bands of m-tiles
    const int32_t *mt_first;
    int n_groups;
    const int32_t *seg_offsets; // group g rows end at seg_offsets[g+1]; NULL: rows_valid
    long long rows_valid;
    // epilogue
    void *out;
    long long ldo;
    const int32_t *perm_token;
    const int32_t *slot_pos;
    const float *topk_w;
    int k;
    const float *perm_w;      // EPI_COMBINE: weight of each row (else found via slot_pos)
    const float *bias;
    int n_valid;
    uint32_t *status;
    // 1: 2-SM pair kernel (256 x 256 tiles; the m-tile list must hold 256-row tiles)
    int pair;
    // MXFP8 GEMM (launch_gemm_mx): E4M3 codes of A and B and their E8M0 scales
    // in the atom layout (mxfp8.cuh): A's keyed by m-tile index, B's by row/128
    const uint8_t *Aq, *A_sf, *Bq, *B_sf;
    uint8_t *out_sf;          // EPI_SWIGLU_MX: scales of h, atom layout keyed by m-tile
    // NVFP4 operands instead (fmt = FMT_NV4, nvfp4.cuh): packed E2M1 codes, E4M3
    // scales per 16 in the 64-element atom layout; A's global encode scale
    // a_gs, B's per group b_gs[g]; the accumulators are multiplied by
    // 1 / (a_gs * b_gs[g]); EPI_SWIGLU_MX quantizes h with out_gs
    int fmt;                  // FMT_MX8 or FMT_NV4
    const float *b_gs;
    float a_gs, out_gs;
    // EPI_ROUTER_TOPK: top-k outputs [rows, k]; counter_zero (one word) is zeroed
    int32_t *route_idx;
    float *route_w;
    int32_t *counter_zero;
    // backward pass
    void *out2;                  // EPI_SWIGLU_SAVE: gate / up [rows, 2 * ldo]
    const uint16_t *gu;          // EPI_SWIGLU_BWD: the saved gate / up [rows, 2 * ldo/2]
    float *row_dot;              // EPI_SWIGLU_BWD: per-row sum of dh * h (atomic adds)
    // K-grouped GEMM (weight gradients): group g of the m-tile list contracts
    // over k-blocks [grp_kb0[g], grp_kb0[g] + grp_nkb[g]); its output starts at
    // out + g * out_group_stride; B rows are shared (b_rows_per_group = 0)
    const int32_t *grp_kb0;
    const int32_t *grp_nkb;
    long long out_group_stride;
    // EPI_ROUTER_TOPK with the histogram folded in (hist_chunk set): per
    // 128-token m-tile expert counts and ranks, then the last CTA's scan
    int32_t *hist_chunk, *hist_rank, *hist_counter, *hist_counts, *hist_offsets, *hist_n_kept;
    int32_t *hist_mt_row0, *hist_mt_group, *hist_num_mt, *hist_mt2_row0, *hist_mt2_group,
        *hist_num_mt2, *hist_mt_first, *hist_mt2_first;
    int capacity;
    // test only (single-SM tensor-core kernel): the producer issues no loads and
    // the pipeline waits give up after 50 ms, so the launch returns with
    // MOE_ERR_TIMEOUT flagged and nothing in flight
    int test_starve;
};

int launch_gemm_tc(const GemmArgs &g, cudaStream_t st);
int launch_gemm_mx(const GemmArgs &g, cudaStream_t st);
// 2-D TMA map of a byte matrix [rows, cols], unswizzled box of 128 bytes x
// box_rows (gemm_mx.cu). Returns MOE_OK or MOE_ERR_CUDA.
int make_tmap_u8_rows(CUtensorMap *m, const void *base, long long cols, long long rows,
                      int box_rows);
// The same with a 128-byte-swizzled box (the block-scaled MMAs' operand layout).
int make_tmap_u8_sw128(CUtensorMap *m, const void *base, long long cols, long long rows,
                       int box_rows);
// NVFP4 decode w1/w3 on the tensor cores (T <= 16): quantizes x (bf16
// [T, d]) with x_gs inside the kernel and writes H32 like launch_dec_w13_nv;
// tiles left over after the whole rounds are split along K, their pieces'
// sums go to `part` (part_floats floats, at least 2 x CTAs x T x 128) and a
// second kernel adds them. With hq != NULL it also writes h as the NVFP4
// operand of launch_dec_w2_nvtc (h_gs; routed rows a = t k + j into hq/hsf,
// the shared expert's rows into hqs/hsfs). Returns MOE_ERR_UNSUPPORTED
// (nothing launched) for shapes it does not take.
int launch_dec_w13_nvtc(const moe_shape_t &s, const uint16_t *x, float x_gs,
                        const int32_t *topk_idx, const uint8_t *W13q, const uint8_t *W13sf,
                        const float *gs13, const uint8_t *W13s_q, const uint8_t *W13s_sf,
                        const float *gs13s, float *H32, float *part, size_t part_floats,
                        float h_gs, uint8_t *hq, uint8_t *hsf, uint8_t *hqs, uint8_t *hsfs,
                        uint32_t *status, cudaStream_t st);
// NVFP4 decode w2 on the tensor cores (T k <= 16): h as the NVFP4 operand the
// w1/w3 kernel wrote (hq [T k, d_ff / 2] with atom-layout scales hsf; the
// shared expert's hqs [T, d_ff_shared / 2], hsfs), split evenly over the
// CTAs along (tile, K stage); its pieces' sums go to `part` and a second
// kernel adds them into out [T, d] in a fixed order. MOE_ERR_UNSUPPORTED
// (nothing launched) for shapes it does not take.
int launch_dec_w2_nvtc(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                       const uint8_t *W2q, const uint8_t *W2sf, const float *gs2,
                       const uint8_t *W2s_q, const uint8_t *W2s_sf, const float *gs2s,
                       const uint8_t *hq, const uint8_t *hsf, const uint8_t *hqs, const uint8_t *hsfs,
                       float h_gs, float *part, size_t part_floats, float *out, uint32_t *status,
                       cudaStream_t st);
int launch_gemm_simt(const GemmArgs &g, cudaStream_t st);
int num_sms();

// ---- decode (decode.cu): small T, only the chosen experts' weights are read
int launch_dec_router(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                      const float *bias, float *logits, cudaStream_t st);
// Router + top-k in one single-CTA launch (small T and small W_g only).
bool dec_route_fusable(const moe_shape_t &s);
int launch_dec_route(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                     const float *bias, float *logits, int32_t *idx, float *w,
                     int32_t *counter_to_zero, uint32_t *status, cudaStream_t st);
int launch_dec_w13(const moe_shape_t &s, const uint16_t *x, const int32_t *topk_idx,
                   const uint16_t *W13, const uint16_t *W13s, uint16_t *Hdec, uint32_t *status,
                   cudaStream_t st);
int launch_dec_w2(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                  const uint16_t *W2, const uint16_t *W2s, const uint16_t *Hdec, float *out,
                  uint32_t *status, cudaStream_t st);

// ---- MXFP8 quantization (mx_quant.cu)
int launch_mx_quantize_rows(const uint16_t *src, long long rows, int K, uint8_t *codes,
                            uint8_t *scales, cudaStream_t st);
int launch_mx_pack_w13(const moe_shape_t &s, const uint16_t *W1, const uint16_t *W3,
                       uint8_t *codes, uint8_t *scales, cudaStream_t st);
int launch_mx_gather(const moe_shape_t &s, const uint16_t *x, const int32_t *idx,
                     const int32_t *slot_pos, const int32_t *offsets, const int32_t *tile_start,
                     uint8_t *xq, uint8_t *xsf, cudaStream_t st);
// ---- NVFP4 quantization (nv_quant.cu)
// per-expert global encode scales of W1 and W3 together (gs13 [E]) and of W2
int launch_nv_weight_scales(const moe_shape_t &s, const uint16_t *W1, const uint16_t *W3,
                            const uint16_t *W2, float *gs13, float *gs2, cudaStream_t st);
// rows of a bf16 matrix; global scale gs_arr[row / rows_per_gs], or gs_const
// a_layout: scales in the activation layout (nv_sfa_offset, an A operand)
// instead of the weights' atom layout.
int launch_nv_quantize_rows(const uint16_t *src, long long rows, int K, const float *gs_arr,
                            long long rows_per_gs, float gs_const, uint8_t *codes,
                            uint8_t *scales, cudaStream_t st, bool a_layout = false);
int launch_nv_pack_w13(const moe_shape_t &s, const uint16_t *W1, const uint16_t *W3,
                       const float *gs13, uint8_t *codes, uint8_t *scales, cudaStream_t st);
int launch_nv_gather(const moe_shape_t &s, const uint16_t *x, const int32_t *idx,
                     const int32_t *slot_pos, const int32_t *offsets, const int32_t *tile_start,
                     float gs, uint8_t *xq, uint8_t *xsf, cudaStream_t st);
// n values (a multiple of 16) through NVFP4 with global scale gs, as the codes'
// values in f16 (dst_h, n) and the block scales' values in fp32 (dst_s, n / 16)
int launch_nv_qrows_f16_bf16(const uint16_t *src, long long n, float gs, uint16_t *dst_h,
                             float *dst_s, cudaStream_t st);
int launch_nv_qrows_f16_f32(const float *src, long long n, float gs, uint16_t *dst_h,
                            float *dst_s, cudaStream_t st);
// decode phases on NVFP4 experts (decode.cu), T <= 2: x and h as given by
// launch_nv_qrows_f16_*; H32 receives h in fp32 (routed rows, then shared)
int launch_dec_w13_nv(const moe_shape_t &s, const uint16_t *xh, const float *xs, float x_gs,
                      const int32_t *topk_idx, const uint8_t *W13q, const uint8_t *W13sf,
                      const float *gs13, const uint8_t *W13s_q, const uint8_t *W13s_sf,
                      const float *gs13s, float *H32, uint32_t *status, cudaStream_t st);
int launch_dec_w2_nv(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                     const uint8_t *W2q, const uint8_t *W2sf, const float *gs2,
                     const uint8_t *W2s_q, const uint8_t *W2s_sf, const float *gs2s,
                     const uint16_t *hh, const float *hs, float h_gs, float *out,
                     uint32_t *status, cudaStream_t st);
// n values (a multiple of 32) through MXFP8 and back, as bf16 (PDL launch)
int launch_mx_qdq_bf16(const uint16_t *src, long long n, uint16_t *dst, cudaStream_t st);
int launch_mx_qdq_f32(const float *src, long long n, uint16_t *dst, cudaStream_t st);
// decode phases on MXFP8 experts (decode.cu); xdq and Hdq are bf16 values
// already through MXFP8; H32 receives h in fp32 (routed rows, then shared)
int launch_dec_w13_mx(const moe_shape_t &s, const uint16_t *xdq, const int32_t *topk_idx,
                      const uint8_t *W13q, const uint8_t *W13sf, const uint8_t *W13s_q,
                      const uint8_t *W13s_sf, float *H32, uint32_t *status, cudaStream_t st);
int launch_dec_w2_mx(const moe_shape_t &s, const int32_t *topk_idx, const float *topk_w,
                     const uint8_t *W2q, const uint8_t *W2sf, const uint8_t *W2s_q,
                     const uint8_t *W2s_sf, const uint16_t *Hdq, float *out, uint32_t *status,
                     cudaStream_t st);

// ---- backward pass helpers (backward.cu)
int launch_transpose_batched(const uint16_t *src, int batch, int R, int C, uint16_t *dst,
                             cudaStream_t st);
int launch_transpose_grouped(const uint16_t *src, int n, int C, const int32_t *offsets,
                             const int32_t *pstart, int E, uint16_t *dst, long long ldd,
                             cudaStream_t st);
int launch_group_ranges(const int32_t *offsets, int E, int32_t *pstart, int32_t *kb0,
                        int32_t *nkb, int M1, int32_t *mt1_row0, int32_t *mt1_group, int M2,
                        int32_t *mt2_row0, int32_t *mt2_group, cudaStream_t st);
int launch_bwd_dyw(const moe_shape_t &s, const float *dout, const int32_t *slot_pos,
                   const float *topk_w, uint16_t *dyw, cudaStream_t st);
size_t router_bwd_part_bytes(const moe_shape_t &s);
int launch_bwd_shared_prep(const float *dout, int T, int d, uint16_t *dout_bf, int32_t *offs,
                           cudaStream_t st);
int launch_router_bwd(const moe_shape_t &s, const int32_t *idx, const float *topk_w,
                      const int32_t *slot_pos, const float *row_dot, const uint16_t *x,
                      const uint16_t *Wg, float *dl, float *part, float *dWg, float *dbias,
                      float *dx, cudaStream_t st);

// ---- expert-choice routing (expert_choice.cu)
int launch_softmax_rows(const moe_shape_t &s, const float *logits, float *scores,
                        uint32_t *status, cudaStream_t st);
int launch_ec_select(const moe_shape_t &s, int K, const float *scores, int32_t *tokens,
                     float *weights, int32_t *offsets, int32_t *mt_row0, int32_t *mt_group,
                     int32_t *num_mt, int32_t *mt_first, uint32_t *status, cudaStream_t st);
int launch_ec_gather(const moe_shape_t &s, int rows, const uint16_t *x, const int32_t *tokens,
                     uint16_t *x_perm, float *out_zero, cudaStream_t st);

} // namespace moe
