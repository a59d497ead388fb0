// moe_api.cu -- the extern "C" entry points of libmoe.so (declared in moe.h):
// argument validation, workspace carving, and the launch sequences.
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"
#include "mxfp8.cuh"
#include "nvfp4.cuh"

namespace moe {

// ---------------------------------------------------------------- instrumentation
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {
struct StageRecord {
    int stage;
    cudaEvent_t a, b;
};
struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<cudaEvent_t> pool;   // created once, reused
    size_t next = 0;
    std::vector<StageRecord> recs;
};
Profiler &prof()
{
    static Profiler p;
    return p;
}
cudaEvent_t take_event(Profiler &P)
{
    if (P.next == P.pool.size()) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess)
            return nullptr;
        P.pool.push_back(e);
    }
    return P.pool[P.next++];
}
} // namespace

// Brackets one stage of moe_forward with two events when profiling is on.
struct StageMark {
    int stage;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    StageMark(int stage_, cudaStream_t st_) : stage(stage_), st(st_)
    {
        Profiler &P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        if (P.on && (a = take_event(P)))
            cudaEventRecord(a, st);
    }
    // Close the stage here (the destructor then does nothing).
    void end()
    {
        if (!a)
            return;
        Profiler &P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        cudaEvent_t b = take_event(P);
        if (b && cudaEventRecord(b, st) == cudaSuccess)
            P.recs.push_back({stage, a, b});
        a = nullptr;
    }
    ~StageMark() { end(); }
};
int launch_dec_router(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                      const float *bias, float *logits, cudaStream_t st);

static bool dim_ok(int v) { return v >= 128 && v <= 32768 && v % 128 == 0; }

int check_shape(const moe_shape_t *s)
{
    if (!s)
        return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->T > (1 << 24))
        return MOE_ERR_INVALID_ARG;
    if (s->E < 1 || s->E > MOE_MAX_E)
        return MOE_ERR_INVALID_ARG;
    if (s->k < 1 || s->k > s->E || s->k > MOE_MAX_K)
        return MOE_ERR_INVALID_ARG;
    if (!dim_ok(s->d) || !dim_ok(s->d_ff))
        return MOE_ERR_INVALID_ARG;
    if (s->d_ff_shared != 0 && !dim_ok(s->d_ff_shared))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

static bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// fp32 split-K sums of the NVFP4 decode w1/w3 kernel: 2 x 1024 CTAs x
// (T <= 2) x 128 (non-decreasing in T)
static size_t dec_part_floats(const moe_shape_t &s)
{
    return (size_t)2 * 1024 * (size_t)std::min(s.T, 2) * 128;
}

WsLayout ws_layout(const moe_shape_t &s)
{
    WsLayout L;
    std::memset(&L, 0, sizeof L);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~static_cast<size_t>(255);
        return o;
    };
    const bool ec = (s.flags & MOE_FLAG_EXPERT_CHOICE) != 0;
    const size_t Kec = ec ? (size_t)std::min(std::max(s.capacity, 0), s.T) : 0;
    const size_t T = s.T, k = s.k, E = s.E, N = std::max(T * k, E * Kec);
    L.nchunks = (int)((T + kChunkTokens - 1) / kChunkTokens);
    L.max_mt = (int)((N + kBlockM - 1) / kBlockM + E);
    L.max_mt2 = (int)((N + 2 * kBlockM - 1) / (2 * kBlockM) + E);
    L.logits = take(T * E * 4);
    L.topk_idx = take(N * 4);
    L.topk_w = take(N * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.n_kept = take(4);
    L.counter = take(4);
    L.num_mt = take(4);
    // 256-token chunks of the histogram kernel, or the router's 128-token
    // m-tiles when it folds the histogram in
    L.chunk_counts = take(std::max(chunk_count_rows(s, L.nchunks), (size_t)((T + kBlockM - 1) / kBlockM)) *
                          E * 4);
    L.rank_local = take(N * 4);
    L.slot_pos = take(N * 4);
    L.perm_token = take(N * 4);
    L.mt_row0 = take((size_t)L.max_mt * 4);
    L.mt_group = take((size_t)L.max_mt * 4);
    L.mt2_row0 = take((size_t)L.max_mt2 * 4);
    L.mt2_group = take((size_t)L.max_mt2 * 4);
    L.num_mt2 = take(4);
    L.mt_first = take((E + 1) * 4);
    L.mt2_first = take((E + 1) * 4);
    const bool mx = (s.flags & MOE_FLAG_MXFP8) != 0;
    const bool nv = (s.flags & MOE_FLAG_NVFP4) != 0;
    const bool lowp = mx || nv;   // block-scaled experts: codes instead of bf16 copies
    const size_t dfs = s.d_ff_shared;
    L.x_perm = take(lowp ? 0 : N * s.d * 2);
    L.H = take(lowp ? 0 : N * s.d_ff * 2);
    L.H_shared = take(!lowp && dfs ? T * dfs * 2 : 0);
    L.Y = take((s.flags & MOE_FLAG_DETERMINISTIC) ? N * s.d * 4 : 0);
    const size_t Td = T < (size_t)MOE_DECODE_MAX_T ? T : (size_t)MOE_DECODE_MAX_T;
    L.dec_H = take((Td * k * s.d_ff + Td * dfs) * 2);
    L.dec_xdq = take(lowp ? Td * s.d * 2 : 0);
    L.dec_H32 = take(lowp ? (Td * k * s.d_ff + Td * dfs) * 4 : 0);
    L.dec_xs = take(nv ? Td * (s.d / 16) * 4 : 0);
    L.dec_hs = take(nv ? (Td * k * s.d_ff + Td * dfs) / 16 * 4 : 0);
    L.dec_part = take(nv ? dec_part_floats(s) * 4 : 0);
    {
        // h of at most two tokens as the NVFP4 w2 operand (codes, atom-layout scales)
        const size_t Th = std::min<size_t>(T, 2);
        L.dec_hq = take(nv ? Th * k * s.d_ff / 2 : 0);
        L.dec_hsf = take(nv ? (size_t)nv_sf_bytes((long long)(Th * k), (int)s.d_ff) : 0);
        L.dec_hqs = take(nv && dfs ? Th * dfs / 2 : 0);
        L.dec_hsfs = take(nv && dfs ? (size_t)nv_sf_bytes((long long)Th, (int)dfs) : 0);
    }
    // activation scales: routed operands keyed by m-tile (at most max_mt
    // tiles of 128 rows), shared-expert operands by row / 128; MXFP8 in the
    // atom layout, NVFP4 (16-element blocks) in the activation layout of
    // nvfp4.cuh (8 KB per tile and 256-element K stage)
    const size_t mt_rows = (size_t)L.max_mt * 128;
    auto sf_bytes = [&](size_t rows, size_t K) {
        return (size_t)(nv ? nv_sfa_bytes((long long)rows, (int)K) : sf_atom_bytes((long long)rows, (int)K));
    };
    L.xq = take(lowp ? N * s.d : 0);
    L.xsf = take(lowp ? sf_bytes(mt_rows, s.d) : 0);
    L.Hq = take(lowp ? N * s.d_ff : 0);
    L.Hsf = take(lowp ? sf_bytes(mt_rows, s.d_ff) : 0);
    L.xq_s = take(lowp && dfs ? T * s.d : 0);
    L.xsf_s = take(lowp && dfs ? sf_bytes(T, s.d) : 0);
    L.Hsq = take(lowp && dfs ? T * dfs : 0);
    L.Hssf = take(lowp && dfs ? sf_bytes(T, dfs) : 0);
    L.tile_start = take(lowp ? E * 4 : 0);
    // backward pass: saved gate/up, w * dout, [dg | du], per-row <dh, h>, the
    // K-grouped GEMMs' ranges and tile lists, and the padded transposes
    const bool bw = (s.flags & MOE_FLAG_BACKWARD) != 0;
    const size_t Np = bw ? ((N + 64 * E + 63) / 64) * 64 : 0;
    L.Np = (long long)Np;
    L.GU = take(bw ? N * 2 * s.d_ff * 2 : 0);
    L.dYw = take(bw ? N * s.d * 2 : 0);
    L.dGU = take(bw ? N * 2 * s.d_ff * 2 : 0);
    L.row_dot = take(bw ? N * 4 : 0);
    L.pstart = take(bw ? (E + 1) * 4 : 0);
    L.kb0 = take(bw ? E * 4 : 0);
    L.nkb = take(bw ? E * 4 : 0);
    L.mtk1_row0 = take(bw ? E * (s.d / kBlockM) * 4 : 0);
    L.mtk1_group = take(bw ? E * (s.d / kBlockM) * 4 : 0);
    L.mtk2_row0 = take(bw ? E * (2 * s.d_ff / kBlockM) * 4 : 0);
    L.mtk2_group = take(bw ? E * (2 * s.d_ff / kBlockM) * 4 : 0);
    L.dYwT = take(bw ? s.d * Np * 2 : 0);
    L.HT = take(bw ? s.d_ff * Np * 2 : 0);
    L.dGUT = take(bw ? 2 * s.d_ff * Np * 2 : 0);
    L.XpT = take(bw ? s.d * Np * 2 : 0);
    L.dl = take(bw ? T * E * 4 : 0);
    L.dwg_part = take(bw ? router_bwd_part_bytes(s) : 0);
    // shared expert: one group of all T rows
    const bool bws = bw && dfs > 0;
    const size_t Tp = bws ? ((T + 63) / 64) * 64 : 0;
    L.Tp = (long long)Tp;
    L.s_GU = take(bws ? T * 2 * dfs * 2 : 0);
    L.s_dout = take(bws ? T * s.d * 2 : 0);
    L.s_dGU = take(bws ? T * 2 * dfs * 2 : 0);
    L.s_rowdot = take(bws ? T * 4 : 0);
    L.s_offs = take(bws ? 2 * 4 : 0);
    L.s_pstart = take(bws ? 2 * 4 : 0);
    L.s_kb0 = take(bws ? 4 : 0);
    L.s_nkb = take(bws ? 4 : 0);
    L.s_mt1_row0 = take(bws ? (s.d / kBlockM) * 4 : 0);
    L.s_mt1_group = take(bws ? (s.d / kBlockM) * 4 : 0);
    L.s_mt2_row0 = take(bws ? (2 * dfs / kBlockM) * 4 : 0);
    L.s_mt2_group = take(bws ? (2 * dfs / kBlockM) * 4 : 0);
    L.s_doutT = take(bws ? s.d * Tp * 2 : 0);
    L.s_HT = take(bws ? dfs * Tp * 2 : 0);
    L.s_dGUT = take(bws ? 2 * dfs * Tp * 2 : 0);
    L.s_xT = take(bws ? s.d * Tp * 2 : 0);
    L.scores = take(ec ? T * E * 4 : 0);
    L.ec_w = take(ec ? N * 4 : 0);
    L.dbg_seen = take(debug_checks(s) ? N * 4 : 0);
    L.x_stage = take((s.flags & MOE_FLAG_HOST_IO) ? T * s.d * 2 : 0);
    L.out_stage = take((s.flags & MOE_FLAG_HOST_IO) ? T * s.d * 4 : 0);
    L.total = off;
    return L;
}

template <class P>
static P *at(void *ws, size_t off)
{
    return reinterpret_cast<P *>(static_cast<char *>(ws) + off);
}

static int check_ws(const moe_shape_t &s, void *ws, size_t ws_bytes, WsLayout &L)
{
    L = ws_layout(s);
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

static int run_gemm(const moe_shape_t &s, const GemmArgs &g, cudaStream_t st)
{
    if (s.flags & MOE_FLAG_SIMT_FFN) {
        GemmArgs g1 = g;
        g1.pair = 0;
        return launch_gemm_simt(g1, st);
    }
    return launch_gemm_tc(g, st);
}

// Engine choice. The 2-SM pair kernel (256-row tiles) moves a third less
// operand data per FLOP from L2 into shared memory, the other limit of a
// stage beside the tensor pipe. With experts of >= 1024 rows it is the faster
// engine for both GEMMs in interleaved measurements on the power-capped B200
// (the prefill layer about 6% faster with w1/w3 on it as well). Short groups
// would pad up to 255 rows per tile, so they stay on the single-SM kernel.
// Output widths must be multiples of 256.
static bool use_pair(const moe_shape_t &s, long long avg_rows, int n_out, bool is_w2)
{
    (void)is_w2;
    if ((s.flags & (MOE_FLAG_SIMT_FFN | MOE_FLAG_GEMM_1SM)) || n_out % 256 != 0)
        return false;
    if (s.flags & MOE_FLAG_GEMM_2SM)
        return true;
    return avg_rows >= 1024;
}

// Point a routed GEMM at the m-tile list of its engine.
static void set_tiles(GemmArgs &g, const moe_shape_t &s, const WsLayout &L, void *ws, bool pair)
{
    g.pair = pair ? 1 : 0;
    g.mt_first = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + (pair ? L.mt2_first : L.mt_first));
    g.n_groups = s.E;
    g.mt_row0 = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + (pair ? L.mt2_row0 : L.mt_row0));
    g.mt_group = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + (pair ? L.mt2_group : L.mt_group));
    g.num_mt_dev = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + (pair ? L.num_mt2 : L.num_mt));
    g.max_mt = pair ? L.max_mt2 : L.max_mt;
}

static GemmArgs gemm_base()
{
    GemmArgs g;
    std::memset(&g, 0, sizeof g);
    return g;
}

// Routed grouped GEMMs: SwiGLU into H, then w2 with the chosen epilogue.
static int expert_ffn_core(const moe_shape_t &s, const WsLayout &L, void *ws,
                           const uint16_t *x_perm, const int32_t *offsets, const uint16_t *W13,
                           const uint16_t *W2, const int32_t *perm_token, const int32_t *slot_pos,
                           const float *topk_w, float *y_perm, float *out, uint32_t *status,
                           cudaStream_t st, long long n_rows = -1, const float *perm_w = nullptr,
                           bool allow_pair = true, bool test_starve = false)
{
    const long long N = n_rows >= 0 ? n_rows : (long long)s.T * s.k;
    uint16_t *H = at<uint16_t>(ws, L.H);
    GemmArgs g = gemm_base();
    g.mode = EPI_SWIGLU;
    g.A = x_perm;
    g.a_rows = N;
    g.B = W13;
    g.b_rows_total = (long long)s.E * 2 * s.d_ff;
    g.K = s.d;
    g.N = 2 * s.d_ff;
    g.b_rows_per_group = 2 * s.d_ff;
    const long long avg_rows = N / s.E;
    set_tiles(g, s, L, ws, allow_pair && use_pair(s, avg_rows, g.N, false));
    g.seg_offsets = offsets;
    g.out = H;
    g.ldo = s.d_ff;
    g.status = status;
    g.test_starve = test_starve ? 1 : 0;
    int rc;
    {
        StageMark m(MOE_STAGE_W13, st);
        rc = run_gemm(s, g, st);
    }
    if (rc)
        return rc;
    g.test_starve = 0;
    g.A = H;
    g.B = W2;
    g.b_rows_total = (long long)s.E * s.d;
    g.K = s.d_ff;
    g.N = s.d;
    g.b_rows_per_group = s.d;
    g.ldo = s.d;
    set_tiles(g, s, L, ws, allow_pair && use_pair(s, avg_rows, g.N, true));
    if (y_perm) {
        g.mode = EPI_STORE_F32;
        g.out = y_perm;
    } else {
        g.mode = EPI_COMBINE;
        g.out = out;
        g.perm_token = perm_token;
        g.slot_pos = slot_pos;
        g.topk_w = topk_w;
        g.k = s.k;
        g.perm_w = perm_w;
    }
    StageMark m(MOE_STAGE_W2, st);
    return run_gemm(s, g, st);
}

// Shared expert on all T tokens: out = W2s (silu(W1s x) * W3s x), plain store.
static int shared_expert(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                         const uint16_t *W13s, const uint16_t *W2s, float *out, uint32_t *status,
                         cudaStream_t st)
{
    uint16_t *Hs = at<uint16_t>(ws, L.H_shared);
    const bool pair1 = use_pair(s, s.T, 2 * s.d_ff_shared, false);
    const int mt = (s.T + (pair1 ? 256 : kBlockM) - 1) / (pair1 ? 256 : kBlockM);
    GemmArgs g = gemm_base();
    g.pair = pair1 ? 1 : 0;
    g.mode = EPI_SWIGLU;
    g.A = x;
    g.a_rows = s.T;
    g.B = W13s;
    g.b_rows_total = 2LL * s.d_ff_shared;
    g.K = s.d;
    g.N = 2 * s.d_ff_shared;
    g.b_rows_per_group = 2 * s.d_ff_shared;
    g.num_mt_host = mt;
    g.max_mt = mt;
    g.rows_valid = s.T;
    g.out = Hs;
    g.ldo = s.d_ff_shared;
    g.status = status;
    int rc = run_gemm(s, g, st);
    if (rc)
        return rc;
    g.mode = EPI_STORE_F32;
    g.A = Hs;
    g.B = W2s;
    g.b_rows_total = s.d;
    g.K = s.d_ff_shared;
    g.N = s.d;
    g.b_rows_per_group = s.d;
    g.out = out;
    g.ldo = s.d;
    const bool pair2 = use_pair(s, s.T, s.d, true);
    g.pair = pair2 ? 1 : 0;
    g.num_mt_host = g.max_mt = (s.T + (pair2 ? 256 : kBlockM) - 1) / (pair2 ? 256 : kBlockM);
    return run_gemm(s, g, st);
}

static int router(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg, const float *bias,
                  float *logits, uint32_t *status, cudaStream_t st)
{
    if (s.T <= MOE_DECODE_MAX_T)
        return launch_dec_router(s, x, Wg, bias, logits, st);
    if (s.flags & MOE_FLAG_SIMT_FFN)
        return launch_router_simt(s, x, Wg, bias, logits, st);
    GemmArgs g = gemm_base();
    g.mode = EPI_ROUTER;
    g.A = x;
    g.a_rows = s.T;
    g.B = Wg;
    g.b_rows_total = s.E;
    g.K = s.d;
    g.N = s.E;
    g.b_rows_per_group = 0;
    g.num_mt_host = (s.T + kBlockM - 1) / kBlockM;
    g.max_mt = g.num_mt_host;
    g.rows_valid = s.T;
    g.out = logits;
    g.ldo = s.E;
    g.bias = bias;
    g.n_valid = s.E;
    g.status = status;
    return launch_gemm_tc(g, st);
}

// Router GEMM with the top-k in its epilogue (one launch): the tensor-core
// router with all E <= 64 logits of a token in one 64-column tile.
static bool router_topk_fusable(const moe_shape_t &s)
{
    return s.T > MOE_DECODE_MAX_T && s.E <= 64 && !(s.flags & MOE_FLAG_SIMT_FFN);
}

static int router_topk(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                       const float *bias, float *logits, int32_t *idx, float *w,
                       int32_t *counter, uint32_t *status, cudaStream_t st)
{
    GemmArgs g = gemm_base();
    g.mode = EPI_ROUTER_TOPK;
    g.A = x;
    g.a_rows = s.T;
    g.B = Wg;
    g.b_rows_total = s.E;
    g.K = s.d;
    g.N = s.E;
    g.num_mt_host = (s.T + kBlockM - 1) / kBlockM;
    g.max_mt = g.num_mt_host;
    g.rows_valid = s.T;
    g.out = logits;
    g.ldo = s.E;
    g.bias = bias;
    g.n_valid = s.E;
    g.k = s.k;
    g.route_idx = idx;
    g.route_w = w;
    g.counter_zero = counter;
    g.status = status;
    return launch_gemm_tc(g, st);
}

// The prefill router with the top-k and the expert histogram in its
// epilogue: per 128-token m-tile counts and ranks, then the last CTA's scan
// into counts, offsets and the grouped GEMMs' tile lists (token-major
// priority only; slot-major priority needs every slot's counts first).
static bool router_hist_fusable(const moe_shape_t &s)
{
    return router_topk_fusable(s) && !slot_major(s);
}

struct HistOut {
    int32_t *chunk, *rank, *counts, *offsets, *n_kept, *mt_row0, *mt_group, *num_mt, *mt2_row0,
        *mt2_group, *num_mt2, *mt_first, *mt2_first;
};

static int router_topk_hist(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                            const float *bias, float *logits, int32_t *idx, float *w,
                            int32_t *counter, const HistOut &h, uint32_t *status, cudaStream_t st)
{
    GemmArgs g = gemm_base();
    g.mode = EPI_ROUTER_TOPK;
    g.A = x;
    g.a_rows = s.T;
    g.B = Wg;
    g.b_rows_total = s.E;
    g.K = s.d;
    g.N = s.E;
    g.num_mt_host = (s.T + kBlockM - 1) / kBlockM;
    g.max_mt = g.num_mt_host;
    g.rows_valid = s.T;
    g.out = logits;
    g.ldo = s.E;
    g.bias = bias;
    g.n_valid = s.E;
    g.k = s.k;
    g.route_idx = idx;
    g.route_w = w;
    g.status = status;
    g.hist_chunk = h.chunk;
    g.hist_rank = h.rank;
    g.hist_counter = counter;
    g.hist_counts = h.counts;
    g.hist_offsets = h.offsets;
    g.hist_n_kept = h.n_kept;
    g.hist_mt_row0 = h.mt_row0;
    g.hist_mt_group = h.mt_group;
    g.hist_num_mt = h.num_mt;
    g.hist_mt2_row0 = h.mt2_row0;
    g.hist_mt2_group = h.mt2_group;
    g.hist_num_mt2 = h.num_mt2;
    g.hist_mt_first = h.mt_first;
    g.hist_mt2_first = h.mt2_first;
    g.capacity = s.capacity;
    // the ticket starts at zero whatever an earlier, aborted call left in it
    if (cudaMemsetAsync(counter, 0, sizeof(int32_t), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_gemm_tc(g, st);
}

// Router, softmax / top-k / renormalisation: one launch when a fused form
// applies (single-CTA for small T and W_g; the GEMM epilogue for E <= 64).
static int route_tokens(const moe_shape_t &s, const uint16_t *x, const uint16_t *Wg,
                        const float *bias, float *logits, int32_t *idx, float *w,
                        int32_t *counter, uint32_t *status, cudaStream_t st)
{
    if (dec_route_fusable(s)) {
        StageMark m(MOE_STAGE_ROUTER, st);
        return launch_dec_route(s, x, Wg, bias, logits, idx, w, counter, status, st);
    }
    if (router_topk_fusable(s)) {
        StageMark m(MOE_STAGE_ROUTER, st);
        return router_topk(s, x, Wg, bias, logits, idx, w, counter, status, st);
    }
    int rc;
    {
        StageMark m(MOE_STAGE_ROUTER, st);
        rc = router(s, x, Wg, bias, logits, status, st);
    }
    if (rc)
        return rc;
    StageMark m(MOE_STAGE_TOPK, st);
    return launch_topk(s, logits, idx, w, counter, status, st);
}

static int forward_impl(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                        const uint16_t *Wg, const float *bias, const uint16_t *W13,
                        const uint16_t *W2, const uint16_t *W13s, const uint16_t *W2s,
                        float *out, float *logits_out, int32_t *idx_out, uint32_t *status,
                        cudaStream_t st)
{
    float *logits = logits_out ? logits_out : at<float>(ws, L.logits);
    int32_t *idx = idx_out ? idx_out : at<int32_t>(ws, L.topk_idx);
    float *w = at<float>(ws, L.topk_w);
    const bool force_dec = (s.flags & MOE_FLAG_FORCE_DECODE) != 0;
    const bool force_pre = (s.flags & MOE_FLAG_FORCE_PREFILL) != 0;
    if (force_dec && s.T > MOE_DECODE_MAX_T)
        return MOE_ERR_UNSUPPORTED;
    const bool decode = force_dec || (!force_pre && s.T <= MOE_DECODE_DEFAULT_T);
    int32_t *counter = at<int32_t>(ws, L.counter);
    const HistOut hist = {at<int32_t>(ws, L.chunk_counts), at<int32_t>(ws, L.rank_local),
                          at<int32_t>(ws, L.counts),       at<int32_t>(ws, L.offsets),
                          at<int32_t>(ws, L.n_kept),       at<int32_t>(ws, L.mt_row0),
                          at<int32_t>(ws, L.mt_group),     at<int32_t>(ws, L.num_mt),
                          at<int32_t>(ws, L.mt2_row0),     at<int32_t>(ws, L.mt2_group),
                          at<int32_t>(ws, L.num_mt2),      at<int32_t>(ws, L.mt_first),
                          at<int32_t>(ws, L.mt2_first)};
    const bool hist_fused = !decode && router_hist_fusable(s);
    int rc;
    if (hist_fused) {
        StageMark m(MOE_STAGE_ROUTER, st);
        rc = router_topk_hist(s, x, Wg, bias, logits, idx, w, counter, hist, status, st);
    } else {
        rc = route_tokens(s, x, Wg, bias, logits, idx, w, counter, status, st);
    }
    if (rc)
        return rc;
    if (decode) {
        uint16_t *Hdec = at<uint16_t>(ws, L.dec_H);
        {
            StageMark m(MOE_STAGE_DEC_W13, st);
            rc = launch_dec_w13(s, x, idx, W13, W13s, Hdec, status, st);
        }
        if (rc)
            return rc;
        StageMark m(MOE_STAGE_DEC_W2, st);
        return launch_dec_w2(s, idx, w, W2, W2s, Hdec, out, status, st);
    }

    const bool det = (s.flags & MOE_FLAG_DETERMINISTIC) != 0;
    const bool shared = s.d_ff_shared > 0;
    int32_t *counts = at<int32_t>(ws, L.counts);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *chunk = at<int32_t>(ws, L.chunk_counts);
    int32_t *rank = at<int32_t>(ws, L.rank_local);
    int32_t *slot_pos = at<int32_t>(ws, L.slot_pos);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token);
    uint16_t *x_perm = at<uint16_t>(ws, L.x_perm);
    if (!hist_fused) {
        StageMark m(MOE_STAGE_HIST, st);
        rc = launch_hist_scan(s, idx, chunk, rank, counter, counts, offsets,
                              at<int32_t>(ws, L.n_kept), at<int32_t>(ws, L.mt_row0),
                              at<int32_t>(ws, L.mt_group), at<int32_t>(ws, L.num_mt),
                              at<int32_t>(ws, L.mt2_row0), at<int32_t>(ws, L.mt2_group),
                              at<int32_t>(ws, L.num_mt2), status, st, nullptr,
                              at<int32_t>(ws, L.mt_first), at<int32_t>(ws, L.mt2_first));
    }
    if (rc)
        return rc;
    {
        StageMark m(MOE_STAGE_PERMUTE, st);
        rc = launch_permute(s, idx, chunk, rank, offsets, x, slot_pos, perm_token, x_perm,
                            (!shared && !det) ? out : nullptr, st,
                            hist_fused ? kBlockM : kChunkTokens);
    }
    if (rc)
        return rc;
    if (debug_checks(s) &&
        (rc = launch_check_dispatch(s, idx, offsets, slot_pos, perm_token,
                                    at<int32_t>(ws, L.n_kept), at<int32_t>(ws, L.dbg_seen),
                                    status, st)))
        return rc;
    if (shared) {
        StageMark m(MOE_STAGE_SHARED, st);
        rc = shared_expert(s, L, ws, x, W13s, W2s, out, status, st);
        if (rc)
            return rc;
    }
    float *Y = det ? at<float>(ws, L.Y) : nullptr;
    rc = expert_ffn_core(s, L, ws, x_perm, offsets, W13, W2, perm_token, slot_pos, w, Y, out,
                         status, st);
    if (rc)
        return rc;
    if (det) {
        StageMark m(MOE_STAGE_COMBINE, st);
        rc = launch_combine(s, Y, slot_pos, w, shared ? out : nullptr, out, st);
    }
    return rc;
}

// ---------------------------------------------------------------- MXFP8 experts
// Grouped MXFP8 GEMMs over the routed rows: w1/w3 with the SwiGLU + MXFP8
// epilogue into Hq/Hsf, then w2 with the chosen epilogue.
// Block-scaled expert weights: MXFP8 (FMT_MX8) or NVFP4 (FMT_NV4, with global
// encode scales per expert and the activations' constants x_gs, h_gs).
struct LowpWeights {
    int fmt;
    const uint8_t *W13q, *W13sf, *W2q, *W2sf;
    const float *W13gs, *W2gs;
    const uint8_t *W13s_q, *W13s_sf, *W2s_q, *W2s_sf;
    const float *W13s_gs, *W2s_gs;
    float x_gs, h_gs;
};

static int expert_ffn_mx(const moe_shape_t &s, const WsLayout &L, void *ws, const LowpWeights &lw,
                         const int32_t *offsets, const int32_t *perm_token,
                         const int32_t *slot_pos, const float *topk_w, float *y_perm, float *out,
                         uint32_t *status, cudaStream_t st)
{
    const long long N = (long long)s.T * s.k;
    GemmArgs g = gemm_base();
    g.mode = EPI_SWIGLU_MX;
    g.fmt = lw.fmt;
    g.Aq = at<uint8_t>(ws, L.xq);
    g.A_sf = at<uint8_t>(ws, L.xsf);
    g.a_rows = N;
    g.Bq = lw.W13q;
    g.B_sf = lw.W13sf;
    g.b_gs = lw.W13gs;
    g.a_gs = lw.x_gs;
    g.out_gs = lw.h_gs;
    g.b_rows_total = (long long)s.E * 2 * s.d_ff;
    g.K = s.d;
    g.N = 2 * s.d_ff;
    g.b_rows_per_group = 2 * s.d_ff;
    set_tiles(g, s, L, ws, false);
    g.seg_offsets = offsets;
    g.out = at<uint8_t>(ws, L.Hq);
    g.ldo = s.d_ff;
    g.out_sf = at<uint8_t>(ws, L.Hsf);
    g.status = status;
    int rc;
    {
        StageMark m(MOE_STAGE_W13, st);
        rc = launch_gemm_mx(g, st);
    }
    if (rc)
        return rc;
    g.Aq = at<uint8_t>(ws, L.Hq);
    g.A_sf = at<uint8_t>(ws, L.Hsf);
    g.Bq = lw.W2q;
    g.B_sf = lw.W2sf;
    g.b_gs = lw.W2gs;
    g.a_gs = lw.h_gs;
    g.b_rows_total = (long long)s.E * s.d;
    g.K = s.d_ff;
    g.N = s.d;
    g.b_rows_per_group = s.d;
    g.ldo = s.d;
    g.out_sf = nullptr;
    if (y_perm) {
        g.mode = EPI_STORE_F32;
        g.out = y_perm;
    } else {
        g.mode = EPI_COMBINE;
        g.out = out;
        g.perm_token = perm_token;
        g.slot_pos = slot_pos;
        g.topk_w = topk_w;
        g.k = s.k;
    }
    StageMark m(MOE_STAGE_W2, st);
    return launch_gemm_mx(g, st);
}

// Shared expert on all T tokens in MXFP8: quantize x, w1/w3 + SwiGLU + MXFP8,
// w2 with a plain store into out.
static int shared_expert_mx(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                            const LowpWeights &lw, float *out, uint32_t *status, cudaStream_t st)
{
    const int dfs = s.d_ff_shared;
    int rc = lw.fmt == FMT_NV4 ? launch_nv_quantize_rows(x, s.T, s.d, nullptr, 0, lw.x_gs,
                                                   at<uint8_t>(ws, L.xq_s), at<uint8_t>(ws, L.xsf_s), st,
                                                   true)
                         : launch_mx_quantize_rows(x, s.T, s.d, at<uint8_t>(ws, L.xq_s),
                                                   at<uint8_t>(ws, L.xsf_s), st);
    if (rc)
        return rc;
    const int mt = (s.T + kBlockM - 1) / kBlockM;
    GemmArgs g = gemm_base();
    g.mode = EPI_SWIGLU_MX;
    g.fmt = lw.fmt;
    g.Aq = at<uint8_t>(ws, L.xq_s);
    g.A_sf = at<uint8_t>(ws, L.xsf_s);
    g.a_rows = s.T;
    g.Bq = lw.W13s_q;
    g.B_sf = lw.W13s_sf;
    g.b_gs = lw.W13s_gs;
    g.a_gs = lw.x_gs;
    g.out_gs = lw.h_gs;
    g.b_rows_total = 2LL * dfs;
    g.K = s.d;
    g.N = 2 * dfs;
    g.b_rows_per_group = 2 * dfs;
    g.num_mt_host = mt;
    g.max_mt = mt;
    g.rows_valid = s.T;
    g.out = at<uint8_t>(ws, L.Hsq);
    g.ldo = dfs;
    g.out_sf = at<uint8_t>(ws, L.Hssf);
    g.status = status;
    if ((rc = launch_gemm_mx(g, st)))
        return rc;
    g.mode = EPI_STORE_F32;
    g.Aq = at<uint8_t>(ws, L.Hsq);
    g.A_sf = at<uint8_t>(ws, L.Hssf);
    g.Bq = lw.W2s_q;
    g.B_sf = lw.W2s_sf;
    g.b_gs = lw.W2s_gs;
    g.a_gs = lw.h_gs;
    g.b_rows_total = s.d;
    g.K = dfs;
    g.N = s.d;
    g.b_rows_per_group = s.d;
    g.out = out;
    g.ldo = s.d;
    g.out_sf = nullptr;
    return launch_gemm_mx(g, st);
}

static int forward_mx_impl(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                           const uint16_t *Wg, const float *bias, const LowpWeights &lw,
                           float *out, float *logits_out, int32_t *idx_out, uint32_t *status,
                           cudaStream_t st)
{
    const uint8_t *W13q = lw.W13q, *W13sf = lw.W13sf, *W2q = lw.W2q, *W2sf = lw.W2sf;
    const uint8_t *W13s_q = lw.W13s_q, *W13s_sf = lw.W13s_sf, *W2s_q = lw.W2s_q,
                  *W2s_sf = lw.W2s_sf;
    float *logits = logits_out ? logits_out : at<float>(ws, L.logits);
    int32_t *idx = idx_out ? idx_out : at<int32_t>(ws, L.topk_idx);
    float *w = at<float>(ws, L.topk_w);
    int32_t *counter = at<int32_t>(ws, L.counter);
    const bool force_dec = (s.flags & MOE_FLAG_FORCE_DECODE) != 0;
    const bool force_pre = (s.flags & MOE_FLAG_FORCE_PREFILL) != 0;
    if (force_dec && s.T > MOE_DECODE_MAX_T)
        return MOE_ERR_UNSUPPORTED;
    // the NVFP4 decode kernels take T <= 2 (x and h staged as f16 code values)
    const bool nv = lw.fmt == FMT_NV4;
    const bool decode = force_dec || (!force_pre && s.T <= MOE_DECODE_DEFAULT_T);
    if (nv && decode && s.T > 2)
        return MOE_ERR_UNSUPPORTED;
    int rc = route_tokens(s, x, Wg, bias, logits, idx, w, counter, status, st);
    if (rc)
        return rc;
    if (decode && nv) {
        // only the chosen experts' codes and scales are read, each once
        uint16_t *xh = at<uint16_t>(ws, L.dec_xdq);
        float *xs = at<float>(ws, L.dec_xs);
        float *H32 = at<float>(ws, L.dec_H32);
        uint16_t *hh = at<uint16_t>(ws, L.dec_H);
        float *hs = at<float>(ws, L.dec_hs);
        const long long nh = (long long)s.T * s.k * s.d_ff + (long long)s.T * s.d_ff_shared;
        // h as the tensor-core w2 kernel's NVFP4 operand, written by the w1/w3 kernel
        float *part = at<float>(ws, L.dec_part);
        uint8_t *hq = at<uint8_t>(ws, L.dec_hq), *hsf = at<uint8_t>(ws, L.dec_hsf);
        uint8_t *hqs = s.d_ff_shared ? at<uint8_t>(ws, L.dec_hqs) : nullptr;
        uint8_t *hsfs = s.d_ff_shared ? at<uint8_t>(ws, L.dec_hsfs) : nullptr;
        bool hq_written = false;
        {
            StageMark m(MOE_STAGE_DEC_W13, st);
            // w1/w3 on the tensor cores; shapes that kernel does not take go
            // through the CUDA-core kernel on f16 code values
            rc = launch_dec_w13_nvtc(s, x, lw.x_gs, idx, W13q, W13sf, lw.W13gs, W13s_q, W13s_sf,
                                     lw.W13s_gs, H32, part, dec_part_floats(s), lw.h_gs, hq, hsf,
                                     hqs, hsfs, status, st);
            hq_written = rc == MOE_OK;
            if (rc == MOE_ERR_UNSUPPORTED) {
                rc = launch_nv_qrows_f16_bf16(x, (long long)s.T * s.d, lw.x_gs, xh, xs, st);
                if (!rc)
                    rc = launch_dec_w13_nv(s, xh, xs, lw.x_gs, idx, W13q, W13sf, lw.W13gs, W13s_q,
                                           W13s_sf, lw.W13s_gs, H32, status, st);
            }
        }
        if (rc)
            return rc;
        StageMark m(MOE_STAGE_DEC_W2, st);
        // w2 on the tensor cores; otherwise on the CUDA cores from f16 code values
        rc = hq_written ? launch_dec_w2_nvtc(s, idx, w, W2q, W2sf, lw.W2gs, W2s_q, W2s_sf, lw.W2s_gs,
                                             hq, hsf, hqs, hsfs, lw.h_gs, part, dec_part_floats(s),
                                             out, status, st)
                        : MOE_ERR_UNSUPPORTED;
        if (rc == MOE_ERR_UNSUPPORTED) {
            rc = launch_nv_qrows_f16_f32(H32, nh, lw.h_gs, hh, hs, st);
            if (!rc)
                rc = launch_dec_w2_nv(s, idx, w, W2q, W2sf, lw.W2gs, W2s_q, W2s_sf, lw.W2s_gs, hh,
                                      hs, lw.h_gs, out, status, st);
        }
        return rc;
    }
    if (decode) {
        // only the chosen experts' codes and scales are read, each once
        uint16_t *xdq = at<uint16_t>(ws, L.dec_xdq);
        float *H32 = at<float>(ws, L.dec_H32);
        uint16_t *Hdq = at<uint16_t>(ws, L.dec_H);
        const long long nh = (long long)s.T * s.k * s.d_ff + (long long)s.T * s.d_ff_shared;
        {
            StageMark m(MOE_STAGE_DEC_W13, st);
            rc = launch_mx_qdq_bf16(x, (long long)s.T * s.d, xdq, st);
            if (!rc)
                rc = launch_dec_w13_mx(s, xdq, idx, W13q, W13sf, W13s_q, W13s_sf, H32, status, st);
        }
        if (rc)
            return rc;
        StageMark m(MOE_STAGE_DEC_W2, st);
        rc = launch_mx_qdq_f32(H32, nh, Hdq, st);
        if (!rc)
            rc = launch_dec_w2_mx(s, idx, w, W2q, W2sf, W2s_q, W2s_sf, Hdq, out, status, st);
        return rc;
    }
    const bool det = (s.flags & MOE_FLAG_DETERMINISTIC) != 0;
    const bool shared = s.d_ff_shared > 0;
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *chunk = at<int32_t>(ws, L.chunk_counts);
    int32_t *rank = at<int32_t>(ws, L.rank_local);
    int32_t *slot_pos = at<int32_t>(ws, L.slot_pos);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token);
    {
        StageMark m(MOE_STAGE_HIST, st);
        rc = launch_hist_scan(s, idx, chunk, rank, counter, at<int32_t>(ws, L.counts), offsets,
                              at<int32_t>(ws, L.n_kept), at<int32_t>(ws, L.mt_row0),
                              at<int32_t>(ws, L.mt_group), at<int32_t>(ws, L.num_mt), nullptr,
                              nullptr, nullptr, status, st, at<int32_t>(ws, L.tile_start),
                              at<int32_t>(ws, L.mt_first));
    }
    if (rc)
        return rc;
    {
        StageMark m(MOE_STAGE_PERMUTE, st);
        rc = launch_permute(s, idx, chunk, rank, offsets, nullptr, slot_pos, perm_token, nullptr,
                            (!shared && !det) ? out : nullptr, st);
        if (!rc)
            rc = lw.fmt == FMT_NV4
                     ? launch_nv_gather(s, x, idx, slot_pos, offsets, at<int32_t>(ws, L.tile_start),
                                        lw.x_gs, at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.xsf), st)
                     : launch_mx_gather(s, x, idx, slot_pos, offsets, at<int32_t>(ws, L.tile_start),
                                        at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.xsf), st);
    }
    if (rc)
        return rc;
    if (shared) {
        StageMark m(MOE_STAGE_SHARED, st);
        rc = shared_expert_mx(s, L, ws, x, lw, out, status, st);
        if (rc)
            return rc;
    }
    float *Y = det ? at<float>(ws, L.Y) : nullptr;
    rc = expert_ffn_mx(s, L, ws, lw, offsets, perm_token, slot_pos, w, Y, out,
                       status, st);
    if (rc || !det)
        return rc;
    StageMark m(MOE_STAGE_COMBINE, st);
    return launch_combine(s, Y, slot_pos, w, shared ? out : nullptr, out, st);
}

// ---------------------------------------------------------------- backward pass
// Backward of the shared expert ([DSK]: added with weight 1 on every token):
// the routed path's kernels with identity tiles and one K-group of all T rows.
static int backward_shared(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                           const uint16_t *W13s, const uint16_t *W13sT, const uint16_t *W2sT,
                           const float *dout, float *dx, float *dW13s, float *dW2s,
                           uint32_t *status, cudaStream_t st)
{
    const int dfs = s.d_ff_shared;
    const int mt = (s.T + kBlockM - 1) / kBlockM;
    uint16_t *Hs = at<uint16_t>(ws, L.H_shared), *GUs = at<uint16_t>(ws, L.s_GU);
    uint16_t *dout_bf = at<uint16_t>(ws, L.s_dout), *dGUs = at<uint16_t>(ws, L.s_dGU);
    float *srow = at<float>(ws, L.s_rowdot);
    int32_t *soffs = at<int32_t>(ws, L.s_offs);
    int rc;
    StageMark mark(MOE_STAGE_SHARED, st);
    // recompute w1s/w3s keeping gate / up
    GemmArgs g = gemm_base();
    g.mode = EPI_SWIGLU_SAVE;
    g.A = x;
    g.a_rows = s.T;
    g.B = W13s;
    g.b_rows_total = 2LL * dfs;
    g.K = s.d;
    g.N = 2 * dfs;
    g.b_rows_per_group = 2 * dfs;
    g.num_mt_host = g.max_mt = mt;
    g.rows_valid = s.T;
    g.out = Hs;
    g.ldo = dfs;
    g.out2 = GUs;
    g.status = status;
    if ((rc = launch_gemm_tc(g, st)) || (rc = launch_bwd_shared_prep(dout, s.T, s.d, dout_bf, soffs, st)))
        return rc;
    if (cudaMemsetAsync(srow, 0, sizeof(float) * (size_t)s.T, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    // dh = dout W2s, through SwiGLU
    g = gemm_base();
    g.mode = EPI_SWIGLU_BWD;
    g.A = dout_bf;
    g.a_rows = s.T;
    g.B = W2sT;
    g.b_rows_total = dfs;
    g.K = s.d;
    g.N = dfs;
    g.b_rows_per_group = dfs;
    g.num_mt_host = g.max_mt = mt;
    g.rows_valid = s.T;
    g.out = dGUs;
    g.ldo = dfs;
    g.gu = GUs;
    g.row_dot = srow;
    g.status = status;
    if ((rc = launch_gemm_tc(g, st)))
        return rc;
    // dx += [dg | du] W13s (rows are tokens)
    g = gemm_base();
    g.mode = EPI_COMBINE;
    g.A = dGUs;
    g.a_rows = s.T;
    g.B = W13sT;
    g.b_rows_total = s.d;
    g.K = 2 * dfs;
    g.N = s.d;
    g.b_rows_per_group = s.d;
    g.num_mt_host = g.max_mt = mt;
    g.rows_valid = s.T;
    g.out = dx;
    g.ldo = s.d;
    g.status = status;
    if ((rc = launch_gemm_tc(g, st)))
        return rc;
    // dW2s = dout^T h_s, dW13s = [dg | du]^T x: one group of all T rows
    int32_t *pst = at<int32_t>(ws, L.s_pstart), *kb0 = at<int32_t>(ws, L.s_kb0);
    int32_t *nkb = at<int32_t>(ws, L.s_nkb);
    if ((rc = launch_group_ranges(soffs, 1, pst, kb0, nkb, s.d, at<int32_t>(ws, L.s_mt1_row0),
                                  at<int32_t>(ws, L.s_mt1_group), 2 * dfs,
                                  at<int32_t>(ws, L.s_mt2_row0), at<int32_t>(ws, L.s_mt2_group),
                                  st)))
        return rc;
    const long long Tp = L.Tp;
    uint16_t *doutT = at<uint16_t>(ws, L.s_doutT), *HT = at<uint16_t>(ws, L.s_HT);
    uint16_t *dGUT = at<uint16_t>(ws, L.s_dGUT), *xT = at<uint16_t>(ws, L.s_xT);
    if ((rc = launch_transpose_grouped(dout_bf, s.T, s.d, soffs, pst, 1, doutT, Tp, st)) ||
        (rc = launch_transpose_grouped(Hs, s.T, dfs, soffs, pst, 1, HT, Tp, st)) ||
        (rc = launch_transpose_grouped(dGUs, s.T, 2 * dfs, soffs, pst, 1, dGUT, Tp, st)) ||
        (rc = launch_transpose_grouped(x, s.T, s.d, soffs, pst, 1, xT, Tp, st)))
        return rc;
    g = gemm_base();
    g.mode = EPI_STORE_F32;
    g.A = doutT;
    g.a_rows = s.d;
    g.B = HT;
    g.b_rows_total = dfs;
    g.K = (int)Tp;
    g.N = dfs;
    g.b_rows_per_group = 0;
    g.mt_row0 = at<int32_t>(ws, L.s_mt1_row0);
    g.mt_group = at<int32_t>(ws, L.s_mt1_group);
    g.num_mt_host = g.max_mt = s.d / kBlockM;
    g.rows_valid = s.d;
    g.grp_kb0 = kb0;
    g.grp_nkb = nkb;
    g.out = dW2s;
    g.ldo = dfs;
    g.status = status;
    if ((rc = launch_gemm_tc(g, st)))
        return rc;
    g.A = dGUT;
    g.a_rows = 2LL * dfs;
    g.B = xT;
    g.b_rows_total = s.d;
    g.N = s.d;
    g.mt_row0 = at<int32_t>(ws, L.s_mt2_row0);
    g.mt_group = at<int32_t>(ws, L.s_mt2_group);
    g.num_mt_host = g.max_mt = 2 * dfs / kBlockM;
    g.rows_valid = 2LL * dfs;
    g.out = dW13s;
    g.ldo = s.d;
    return launch_gemm_tc(g, st);
}

static int backward_impl(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                         const uint16_t *Wg, const float *bias, const uint16_t *W13,
                         const uint16_t *W13T, const uint16_t *W2T, const uint16_t *W13s,
                         const uint16_t *W13sT, const uint16_t *W2sT, const float *dout, float *dx,
                         float *dW13, float *dW2, float *dW13s, float *dW2s, float *dWg,
                         float *dbias, float *dlogits, uint32_t *status, cudaStream_t st)
{
    const long long N = (long long)s.T * s.k;
    float *logits = at<float>(ws, L.logits);
    int32_t *idx = at<int32_t>(ws, L.topk_idx);
    float *w = at<float>(ws, L.topk_w);
    int32_t *counter = at<int32_t>(ws, L.counter);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *chunk = at<int32_t>(ws, L.chunk_counts);
    int32_t *rank = at<int32_t>(ws, L.rank_local);
    int32_t *slot_pos = at<int32_t>(ws, L.slot_pos);
    int32_t *perm_token = at<int32_t>(ws, L.perm_token);
    uint16_t *x_perm = at<uint16_t>(ws, L.x_perm);
    uint16_t *H = at<uint16_t>(ws, L.H);
    uint16_t *GU = at<uint16_t>(ws, L.GU);
    uint16_t *dYw = at<uint16_t>(ws, L.dYw);
    uint16_t *dGU = at<uint16_t>(ws, L.dGU);
    float *row_dot = at<float>(ws, L.row_dot);
    float *dl = dlogits ? dlogits : at<float>(ws, L.dl);
    int rc;
    // routing and dispatch: the forward's kernels, so the decisions are identical
    if ((rc = route_tokens(s, x, Wg, bias, logits, idx, w, counter, status, st)))
        return rc;
    {
        StageMark m(MOE_STAGE_HIST, st);
        rc = launch_hist_scan(s, idx, chunk, rank, counter, at<int32_t>(ws, L.counts), offsets,
                              at<int32_t>(ws, L.n_kept), at<int32_t>(ws, L.mt_row0),
                              at<int32_t>(ws, L.mt_group), at<int32_t>(ws, L.num_mt), nullptr,
                              nullptr, nullptr, status, st, nullptr, at<int32_t>(ws, L.mt_first));
    }
    if (rc)
        return rc;
    {
        StageMark m(MOE_STAGE_PERMUTE, st);
        if ((rc = launch_permute(s, idx, chunk, rank, offsets, x, slot_pos, perm_token, x_perm,
                                 nullptr, st)))
            return rc;
        if ((rc = launch_bwd_dyw(s, dout, slot_pos, w, dYw, st)))
            return rc;
    }
    // w1/w3 again, keeping the gate / up accumulators
    GemmArgs g = gemm_base();
    g.mode = EPI_SWIGLU_SAVE;
    g.A = x_perm;
    g.a_rows = N;
    g.B = W13;
    g.b_rows_total = (long long)s.E * 2 * s.d_ff;
    g.K = s.d;
    g.N = 2 * s.d_ff;
    g.b_rows_per_group = 2 * s.d_ff;
    set_tiles(g, s, L, ws, false);
    g.seg_offsets = offsets;
    g.out = H;
    g.ldo = s.d_ff;
    g.out2 = GU;
    g.status = status;
    {
        StageMark m(MOE_STAGE_W13, st);
        if ((rc = launch_gemm_tc(g, st)))
            return rc;
    }
    // dh = (w dout) W2_e, then through SwiGLU: [dg | du] and row sums <dh, h>
    if (cudaMemsetAsync(row_dot, 0, sizeof(float) * (size_t)std::max(N, 1LL), st) != cudaSuccess ||
        cudaMemsetAsync(dx, 0, sizeof(float) * (size_t)s.T * s.d, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    g = gemm_base();
    g.mode = EPI_SWIGLU_BWD;
    g.A = dYw;
    g.a_rows = N;
    g.B = W2T;
    g.b_rows_total = (long long)s.E * s.d_ff;
    g.K = s.d;
    g.N = s.d_ff;
    g.b_rows_per_group = s.d_ff;
    set_tiles(g, s, L, ws, false);
    g.seg_offsets = offsets;
    g.out = dGU;
    g.ldo = s.d_ff;
    g.gu = GU;
    g.row_dot = row_dot;
    g.status = status;
    {
        StageMark m(MOE_STAGE_W2, st);
        if ((rc = launch_gemm_tc(g, st)))
            return rc;
    }
    // dx += [dg | du] [W1; W3]_e, scattered back to the tokens (weight 1)
    g = gemm_base();
    g.mode = EPI_COMBINE;
    g.A = dGU;
    g.a_rows = N;
    g.B = W13T;
    g.b_rows_total = (long long)s.E * s.d;
    g.K = 2 * s.d_ff;
    g.N = s.d;
    g.b_rows_per_group = s.d;
    set_tiles(g, s, L, ws, false);
    g.seg_offsets = offsets;
    g.out = dx;
    g.ldo = s.d;
    g.perm_token = perm_token;
    g.status = status;
    {
        StageMark m(MOE_STAGE_BWD_DX, st);
        if ((rc = launch_gemm_tc(g, st)))
            return rc;
    }
    // weight gradients: contractions over each expert's rows
    StageMark mdw(MOE_STAGE_BWD_DW, st);
    int32_t *pstart = at<int32_t>(ws, L.pstart);
    int32_t *kb0 = at<int32_t>(ws, L.kb0);
    int32_t *nkb = at<int32_t>(ws, L.nkb);
    if ((rc = launch_group_ranges(offsets, s.E, pstart, kb0, nkb, s.d, at<int32_t>(ws, L.mtk1_row0),
                                  at<int32_t>(ws, L.mtk1_group), 2 * s.d_ff,
                                  at<int32_t>(ws, L.mtk2_row0), at<int32_t>(ws, L.mtk2_group), st)))
        return rc;
    const long long Np = L.Np;
    uint16_t *dYwT = at<uint16_t>(ws, L.dYwT), *HT = at<uint16_t>(ws, L.HT);
    uint16_t *dGUT = at<uint16_t>(ws, L.dGUT), *XpT = at<uint16_t>(ws, L.XpT);
    if ((rc = launch_transpose_grouped(dYw, (int)N, s.d, offsets, pstart, s.E, dYwT, Np, st)) ||
        (rc = launch_transpose_grouped(H, (int)N, s.d_ff, offsets, pstart, s.E, HT, Np, st)) ||
        (rc = launch_transpose_grouped(dGU, (int)N, 2 * s.d_ff, offsets, pstart, s.E, dGUT, Np, st)) ||
        (rc = launch_transpose_grouped(x_perm, (int)N, s.d, offsets, pstart, s.E, XpT, Np, st)))
        return rc;
    // dW2_e = (w dout)_e^T h_e  [d, d_ff]
    g = gemm_base();
    g.mode = EPI_STORE_F32;
    g.A = dYwT;
    g.a_rows = s.d;
    g.B = HT;
    g.b_rows_total = s.d_ff;
    g.K = (int)Np;
    g.N = s.d_ff;
    g.b_rows_per_group = 0;
    g.mt_row0 = at<int32_t>(ws, L.mtk1_row0);
    g.mt_group = at<int32_t>(ws, L.mtk1_group);
    g.num_mt_host = s.E * (s.d / kBlockM);
    g.max_mt = g.num_mt_host;
    g.rows_valid = s.d;
    g.grp_kb0 = kb0;
    g.grp_nkb = nkb;
    g.out = dW2;
    g.ldo = s.d_ff;
    g.out_group_stride = (long long)s.d * s.d_ff;
    g.status = status;
    if ((rc = launch_gemm_tc(g, st)))
        return rc;
    // dW13_e = [dg | du]_e^T x_e  [2 d_ff, d] (the packed W13 order)
    g.A = dGUT;
    g.a_rows = 2LL * s.d_ff;
    g.B = XpT;
    g.b_rows_total = s.d;
    g.N = s.d;
    g.mt_row0 = at<int32_t>(ws, L.mtk2_row0);
    g.mt_group = at<int32_t>(ws, L.mtk2_group);
    g.num_mt_host = s.E * (2 * s.d_ff / kBlockM);
    g.max_mt = g.num_mt_host;
    g.rows_valid = 2LL * s.d_ff;
    g.out = dW13;
    g.ldo = s.d;
    g.out_group_stride = 2LL * s.d_ff * s.d;
    if ((rc = launch_gemm_tc(g, st)))
        return rc;
    mdw.end();
    if (s.d_ff_shared > 0 &&
        (rc = backward_shared(s, L, ws, x, W13s, W13sT, W2sT, dout, dx, dW13s, dW2s, status, st)))
        return rc;
    // router: dl, dWg, dbias, and dx += dl Wg (after every scatter-add into dx)
    StageMark m(MOE_STAGE_BWD_ROUTER, st);
    return launch_router_bwd(s, idx, w, slot_pos, row_dot, x, Wg, dl, at<float>(ws, L.dwg_part),
                             dWg, dbias, dx, st);
}

// ---------------------------------------------------------------- expert-choice routing
// Expert choice needs its flag (workspace sizing) and a capacity. Its combine
// is the w2 epilogue's atomic add (a token may be taken by any number of
// experts), so the bitwise-repeatable mode is not offered for it.
static int ec_check(const moe_shape_t &s)
{
    if (!(s.flags & MOE_FLAG_EXPERT_CHOICE) || s.capacity <= 0 ||
        (s.flags & (MOE_FLAG_DETERMINISTIC | MOE_FLAG_HOST_IO)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Router + softmax (when x is given) and the per-expert selection; writes the
// selected tokens / weights, the expert offsets and the GEMM m-tile list.
static int ec_route(const moe_shape_t &s, const WsLayout &L, void *ws, const uint16_t *x,
                    const uint16_t *Wg, const float *bias, float *logits, float *scores,
                    int32_t *tokens, float *weights, uint32_t *status, cudaStream_t st)
{
    const int K = std::min(s.capacity, s.T);
    int rc;
    if (x) {
        {
            StageMark m(MOE_STAGE_ROUTER, st);
            rc = router(s, x, Wg, bias, logits, status, st);
        }
        if (rc)
            return rc;
        StageMark m(MOE_STAGE_TOPK, st);
        if ((rc = launch_softmax_rows(s, logits, scores, status, st)))
            return rc;
    }
    StageMark m(MOE_STAGE_HIST, st);
    return launch_ec_select(s, K, scores, tokens, weights, at<int32_t>(ws, L.offsets),
                            at<int32_t>(ws, L.mt_row0), at<int32_t>(ws, L.mt_group),
                            at<int32_t>(ws, L.num_mt), at<int32_t>(ws, L.mt_first), status, st);
}

// ---------------------------------------------------------------- host I/O pipeline
// moe_forward_host splits a token-separable batch (uncapped: every token's
// output depends only on its own row) into chunks, so chunk c+1's upload and
// chunk c-1's download run on the copy engines while chunk c computes. The two
// copy streams and the events are created once per device and kept.
namespace {
constexpr int kHostIoMaxChunks = 4;
constexpr int kHostIoMinChunkRows = 2048;

struct HostIo {
    std::mutex mu;
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t in_done[kHostIoMaxChunks] = {};
    cudaEvent_t compute_done[kHostIoMaxChunks] = {};
};

HostIo *host_io_for_current_device()
{
    static HostIo per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    HostIo &h = per_dev[dev];
    std::lock_guard<std::mutex> g(h.mu);
    if (!h.ready) {
        bool ok = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&h.fork, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&h.join, cudaEventDisableTiming) == cudaSuccess;
        for (int c = 0; ok && c < kHostIoMaxChunks; ++c)
            ok = cudaEventCreateWithFlags(&h.in_done[c], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h.compute_done[c], cudaEventDisableTiming) == cudaSuccess;
        if (!ok)
            return nullptr;
        h.ready = true;
    }
    return &h;
}
} // namespace

static int forward_host_pipelined(const moe_shape_t &s, const WsLayout &L, void *ws,
                                  const uint16_t *x_host, const uint16_t *Wg, const float *bias,
                                  const uint16_t *W13, const uint16_t *W2, const uint16_t *W13s,
                                  const uint16_t *W2s, float *out_host, uint32_t *status,
                                  cudaStream_t st, int nchunks)
{
    HostIo *h = host_io_for_current_device();
    if (!h)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> g(h->mu);
    uint16_t *xd = at<uint16_t>(ws, L.x_stage);
    float *od = at<float>(ws, L.out_stage);
    // fork: the copy streams start after everything already queued on `st`
    if (cudaEventRecord(h->fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(h->in, h->fork, 0) != cudaSuccess ||
        cudaStreamWaitEvent(h->out, h->fork, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int rows = (s.T + nchunks - 1) / nchunks;
    for (int c = 0; c < nchunks; ++c) {
        const int r0 = c * rows, n = std::min(rows, s.T - r0);
        if (cudaMemcpyAsync(xd + (size_t)r0 * s.d, x_host + (size_t)r0 * s.d, (size_t)n * s.d * 2,
                            cudaMemcpyHostToDevice, h->in) != cudaSuccess ||
            cudaEventRecord(h->in_done[c], h->in) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    for (int c = 0; c < nchunks; ++c) {
        const int r0 = c * rows, n = std::min(rows, s.T - r0);
        moe_shape_t sc = s;
        sc.T = n;
        if (cudaStreamWaitEvent(st, h->in_done[c], 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        int rc = forward_impl(sc, L, ws, xd + (size_t)r0 * s.d, Wg, bias, W13, W2, W13s, W2s,
                              od + (size_t)r0 * s.d, nullptr, nullptr, status, st);
        if (rc)
            return rc;
        if (cudaEventRecord(h->compute_done[c], st) != cudaSuccess ||
            cudaStreamWaitEvent(h->out, h->compute_done[c], 0) != cudaSuccess ||
            cudaMemcpyAsync(out_host + (size_t)r0 * s.d, od + (size_t)r0 * s.d,
                            (size_t)n * s.d * 4, cudaMemcpyDeviceToHost, h->out) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // join: `st` completes only after the last download
    if (cudaEventRecord(h->join, h->out) != cudaSuccess ||
        cudaStreamWaitEvent(st, h->join, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

} // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(int code)
{
    switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_NONFINITE: return "non-finite router logit";
    case MOE_ERR_BAD_EXPERT: return "expert id out of range or repeated";
    case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MOE_ERR_CHECK: return "dispatch consistency check failed";
    default: return "unknown status";
    }
}

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_profile_enable(int on)
{
    Profiler &P = prof();
    std::lock_guard<std::mutex> g(P.mu);
    P.on = on != 0;
    return MOE_OK;
}

int moe_profile_read(double *ms, int64_t *calls, int n)
{
    if (n < 0 || n > MOE_NUM_STAGES)
        return MOE_ERR_INVALID_ARG;
    Profiler &P = prof();
    std::lock_guard<std::mutex> g(P.mu);
    for (int i = 0; i < n; ++i) {
        if (ms)
            ms[i] = 0.0;
        if (calls)
            calls[i] = 0;
    }
    int rc = MOE_OK;
    for (const StageRecord &r : P.recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
            rc = MOE_ERR_CUDA;
            continue;
        }
        if (r.stage < n) {
            if (ms)
                ms[r.stage] += t;
            if (calls)
                calls[r.stage] += 1;
        }
    }
    P.recs.clear();
    P.next = 0;
    return rc;
}

int moe_workspace_size(const moe_shape_t *shape, size_t *bytes)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (!bytes)
        return MOE_ERR_INVALID_ARG;
    *bytes = ws_layout(*shape).total;
    return MOE_OK;
}

int moe_pack_w13(const moe_shape_t *shape, const moe_bf16_t *W1, const moe_bf16_t *W3,
                 moe_bf16_t *W13, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;   // empty batch: nothing to read or write
    if (!W1 || !W3 || !W13 || !al16(W1) || !al16(W3) || !al16(W13))
        return MOE_ERR_INVALID_ARG;
    return launch_pack_w13(shape->E, shape->d_ff, shape->d, W1, W3, W13,
                           reinterpret_cast<cudaStream_t>(stream));
}

int moe_route(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
              const float *bias, float *logits, int32_t *topk_idx, float *topk_w,
              uint32_t *status, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;   // empty batch: nothing to read or write
    const moe_shape_t &s = *shape;
    if (!logits || !topk_idx || !topk_w || (x && !Wg) || (x && (!al16(x) || !al16(Wg))))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    if (s.T == 0)
        return MOE_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (x && dec_route_fusable(s))
        return launch_dec_route(s, x, Wg, bias, logits, topk_idx, topk_w, nullptr, status, st);
    if (x && router_topk_fusable(s))
        return router_topk(s, x, Wg, bias, logits, topk_idx, topk_w, nullptr, status, st);
    if (x && (rc = router(s, x, Wg, bias, logits, status, st)))
        return rc;
    return launch_topk(s, logits, topk_idx, topk_w, nullptr, status, st);
}

int moe_permute(const moe_shape_t *shape, const int32_t *topk_idx, const moe_bf16_t *x,
                int32_t *expert_counts, int32_t *expert_offsets, int32_t *slot_pos,
                int32_t *perm_token, moe_bf16_t *x_perm, int32_t *n_kept, uint32_t *status,
                void *ws, size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    const moe_shape_t &s = *shape;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (s.T == 0) {
        // empty batch: every expert has 0 rows (async memsets, no kernel)
        if ((expert_counts && cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * s.E, st) != cudaSuccess) ||
            (expert_offsets && cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (s.E + 1), st) != cudaSuccess) ||
            (n_kept && cudaMemsetAsync(n_kept, 0, sizeof(int32_t), st) != cudaSuccess))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!topk_idx || !expert_counts || !expert_offsets || !slot_pos || !perm_token ||
        (x && !x_perm) || (x && (!al16(x) || !al16(x_perm))))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    int32_t *counter = at<int32_t>(ws, L.counter);
    if (cudaMemsetAsync(counter, 0, sizeof(int32_t), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    int32_t *chunk = at<int32_t>(ws, L.chunk_counts);
    int32_t *rank = at<int32_t>(ws, L.rank_local);
    int32_t *nk = n_kept ? n_kept : at<int32_t>(ws, L.n_kept);
    rc = launch_hist_scan(s, topk_idx, chunk, rank, counter, expert_counts, expert_offsets, nk,
                          at<int32_t>(ws, L.mt_row0), at<int32_t>(ws, L.mt_group),
                          at<int32_t>(ws, L.num_mt), at<int32_t>(ws, L.mt2_row0),
                          at<int32_t>(ws, L.mt2_group), at<int32_t>(ws, L.num_mt2), status, st,
                          nullptr, at<int32_t>(ws, L.mt_first), at<int32_t>(ws, L.mt2_first));
    if (rc)
        return rc;
    rc = launch_permute(s, topk_idx, chunk, rank, expert_offsets, x, slot_pos, perm_token,
                        x ? x_perm : nullptr, nullptr, st);
    if (rc || !debug_checks(s))
        return rc;
    return launch_check_dispatch(s, topk_idx, expert_offsets, slot_pos, perm_token, nk,
                                 at<int32_t>(ws, L.dbg_seen), status, st);
}

int moe_check_dispatch(const moe_shape_t *shape, const int32_t *topk_idx,
                       const int32_t *expert_offsets, const int32_t *slot_pos,
                       const int32_t *perm_token, const int32_t *n_kept, uint32_t *status,
                       void *ws, size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    const moe_shape_t &s = *shape;
    if (s.T == 0)
        return MOE_OK;
    if (!debug_checks(s) || !topk_idx || !expert_offsets || !slot_pos || !perm_token || !n_kept ||
        !status)
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    return launch_check_dispatch(s, topk_idx, expert_offsets, slot_pos, perm_token, n_kept,
                                 at<int32_t>(ws, L.dbg_seen), status,
                                 reinterpret_cast<cudaStream_t>(stream));
}

int moe_expert_ffn(const moe_shape_t *shape, const moe_bf16_t *x_perm,
                   const int32_t *expert_offsets, const moe_bf16_t *W13, const moe_bf16_t *W2,
                   const int32_t *perm_token, const int32_t *slot_pos, const float *topk_w,
                   float *y_perm, float *out, uint32_t *status, void *ws, size_t ws_bytes,
                   moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->flags & (MOE_FLAG_MXFP8 | MOE_FLAG_NVFP4))
        return MOE_ERR_INVALID_ARG;   // bf16 experts: block-scaled workspaces have no bf16 buffers
    if (shape->T == 0)
        return MOE_OK;   // empty batch: nothing to read or write
    const moe_shape_t &s = *shape;
    if (!x_perm || !expert_offsets || !W13 || !W2 || !al16(x_perm) || !al16(W13) || !al16(W2))
        return MOE_ERR_INVALID_ARG;
    if (y_perm ? !al16(y_perm) : (!out || !perm_token || !slot_pos || !topk_w || !al16(out)))
        return MOE_ERR_INVALID_ARG;
    // the test-only starved w1/w3 launch: single-SM tensor-core kernel only
    const bool starve = (s.flags & MOE_FLAG_TEST_TIMEOUT) != 0;
    if (starve && (s.flags & MOE_FLAG_SIMT_FFN))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    if (s.T == 0)
        return MOE_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    rc = launch_tiles_from_offsets(s, expert_offsets, at<int32_t>(ws, L.mt_row0),
                                   at<int32_t>(ws, L.mt_group), at<int32_t>(ws, L.num_mt),
                                   at<int32_t>(ws, L.mt2_row0), at<int32_t>(ws, L.mt2_group),
                                   at<int32_t>(ws, L.num_mt2), st, at<int32_t>(ws, L.mt_first),
                                   at<int32_t>(ws, L.mt2_first));
    if (rc)
        return rc;
    return expert_ffn_core(s, L, ws, x_perm, expert_offsets, W13, W2, perm_token, slot_pos, topk_w,
                           y_perm, out, status, st, -1, nullptr, !starve, starve);
}

int moe_combine(const moe_shape_t *shape, const float *y_perm, const int32_t *slot_pos,
                const float *topk_w, const float *shared_out, float *out, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;   // empty batch: nothing to read or write
    if (!y_perm || !slot_pos || !topk_w || !out || !al16(y_perm) || !al16(out) ||
        (shared_out && !al16(shared_out)))
        return MOE_ERR_INVALID_ARG;
    return launch_combine(*shape, y_perm, slot_pos, topk_w, shared_out, out,
                          reinterpret_cast<cudaStream_t>(stream));
}

int moe_forward(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W2,
                const moe_bf16_t *W13_shared, const moe_bf16_t *W2_shared, float *out,
                float *logits_out, int32_t *topk_idx_out, uint32_t *status, void *ws,
                size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->flags & (MOE_FLAG_MXFP8 | MOE_FLAG_NVFP4))
        return MOE_ERR_INVALID_ARG;   // bf16 experts: block-scaled workspaces have no bf16 buffers
    if (shape->T == 0)
        return MOE_OK;   // empty batch: nothing to read or write
    const moe_shape_t &s = *shape;
    if (!x || !Wg || !W13 || !W2 || !out || !al16(x) || !al16(Wg) || !al16(W13) || !al16(W2) ||
        !al16(out))
        return MOE_ERR_INVALID_ARG;
    if (s.d_ff_shared > 0 &&
        (!W13_shared || !W2_shared || !al16(W13_shared) || !al16(W2_shared)))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    if (s.T == 0)
        return MOE_OK;
    return forward_impl(s, L, ws, x, Wg, bias, W13, W2, W13_shared, W2_shared, out, logits_out,
                        topk_idx_out, status, reinterpret_cast<cudaStream_t>(stream));
}

int moe_forward_host(const moe_shape_t *shape, const moe_bf16_t *x_host, const moe_bf16_t *Wg,
                     const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W2,
                     const moe_bf16_t *W13_shared, const moe_bf16_t *W2_shared, float *out_host,
                     uint32_t *status, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->flags & (MOE_FLAG_MXFP8 | MOE_FLAG_NVFP4))
        return MOE_ERR_INVALID_ARG;   // bf16 experts: block-scaled workspaces have no bf16 buffers
    if (shape->T == 0)
        return MOE_OK;   // empty batch: nothing to read or write
    const moe_shape_t &s = *shape;
    if (!(s.flags & MOE_FLAG_HOST_IO))
        return MOE_ERR_INVALID_ARG;
    if (!x_host || !out_host || !Wg || !W13 || !W2 || !al16(Wg) || !al16(W13) || !al16(W2))
        return MOE_ERR_INVALID_ARG;
    if (s.d_ff_shared > 0 &&
        (!W13_shared || !W2_shared || !al16(W13_shared) || !al16(W2_shared)))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    if (s.T == 0)
        return MOE_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // token-separable batches large enough to split: overlap copies with compute
    const int nchunks = std::min(kHostIoMaxChunks, s.T / kHostIoMinChunkRows);
    if (s.capacity <= 0 && nchunks >= 2)
        return forward_host_pipelined(s, L, ws, x_host, Wg, bias, W13, W2, W13_shared, W2_shared,
                                      out_host, status, st, nchunks);
    uint16_t *xd = at<uint16_t>(ws, L.x_stage);
    float *od = at<float>(ws, L.out_stage);
    const size_t xb = (size_t)s.T * s.d * 2, ob = (size_t)s.T * s.d * 4;
    if (cudaMemcpyAsync(xd, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    rc = forward_impl(s, L, ws, xd, Wg, bias, W13, W2, W13_shared, W2_shared, od, nullptr, nullptr,
                      status, st);
    if (rc)
        return rc;
    if (cudaMemcpyAsync(out_host, od, ob, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_route_expert_choice(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                            const float *bias, float *logits, float *scores,
                            int32_t *expert_tokens, float *expert_w, uint32_t *status, void *ws,
                            size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if ((rc = ec_check(*shape)))
        return rc;
    if (shape->T == 0)
        return MOE_OK;
    const moe_shape_t &s = *shape;
    if (!scores || !expert_tokens || !expert_w || (x && (!Wg || !al16(x) || !al16(Wg))))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    return ec_route(s, L, ws, x, Wg, bias, logits ? logits : at<float>(ws, L.logits), scores,
                    expert_tokens, expert_w, status, reinterpret_cast<cudaStream_t>(stream));
}

int moe_forward_expert_choice(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                              const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W2,
                              const moe_bf16_t *W13_shared, const moe_bf16_t *W2_shared,
                              float *out, uint32_t *status, void *ws, size_t ws_bytes,
                              moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->flags & (MOE_FLAG_MXFP8 | MOE_FLAG_NVFP4))
        return MOE_ERR_INVALID_ARG;   // bf16 experts: block-scaled workspaces have no bf16 buffers
    if ((rc = ec_check(*shape)))
        return rc;
    if (shape->T == 0)
        return MOE_OK;
    const moe_shape_t &s = *shape;
    if (!x || !Wg || !W13 || !W2 || !out || !al16(x) || !al16(Wg) || !al16(W13) || !al16(W2) ||
        !al16(out))
        return MOE_ERR_INVALID_ARG;
    if (s.d_ff_shared > 0 &&
        (!W13_shared || !W2_shared || !al16(W13_shared) || !al16(W2_shared)))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int K = std::min(s.capacity, s.T);
    const long long rows = (long long)s.E * K;
    int32_t *tokens = at<int32_t>(ws, L.perm_token);
    float *wts = at<float>(ws, L.ec_w);
    if ((rc = ec_route(s, L, ws, x, Wg, bias, at<float>(ws, L.logits), at<float>(ws, L.scores),
                       tokens, wts, status, st)))
        return rc;
    const bool shared = s.d_ff_shared > 0;
    uint16_t *x_perm = at<uint16_t>(ws, L.x_perm);
    {
        StageMark m(MOE_STAGE_PERMUTE, st);
        if ((rc = launch_ec_gather(s, (int)rows, x, tokens, x_perm, shared ? nullptr : out, st)))
            return rc;
    }
    if (shared) {
        StageMark m(MOE_STAGE_SHARED, st);
        if ((rc = shared_expert(s, L, ws, x, W13_shared, W2_shared, out, status, st)))
            return rc;
    }
    return expert_ffn_core(s, L, ws, x_perm, at<int32_t>(ws, L.offsets), W13, W2, tokens, nullptr,
                           nullptr, nullptr, out, status, st, rows, wts, false);
}

int moe_quantize_experts_mxfp8(const moe_shape_t *shape, const moe_bf16_t *W1,
                               const moe_bf16_t *W3, const moe_bf16_t *W2, uint8_t *W13q,
                               uint8_t *W13sf, uint8_t *W2q, uint8_t *W2sf, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;
    const moe_shape_t &s = *shape;
    if (!W1 || !W3 || !W2 || !W13q || !W13sf || !W2q || !W2sf || !al16(W1) || !al16(W3) ||
        !al16(W2) || !al16(W13q) || !al16(W2q) || !al16(W13sf) || !al16(W2sf))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = launch_mx_pack_w13(s, W1, W3, W13q, W13sf, st)))
        return rc;
    return launch_mx_quantize_rows(W2, (long long)s.E * s.d, s.d_ff, W2q, W2sf, st);
}

int moe_forward_mxfp8(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                      const float *bias, const uint8_t *W13q, const uint8_t *W13sf,
                      const uint8_t *W2q, const uint8_t *W2sf, const uint8_t *W13s_q,
                      const uint8_t *W13s_sf, const uint8_t *W2s_q, const uint8_t *W2s_sf,
                      float *out, float *logits_out, int32_t *topk_idx_out, uint32_t *status,
                      void *ws, size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;
    const moe_shape_t &s = *shape;
    if (!(s.flags & MOE_FLAG_MXFP8) || (s.flags & MOE_FLAG_HOST_IO))
        return MOE_ERR_INVALID_ARG;
    if (!x || !Wg || !W13q || !W13sf || !W2q || !W2sf || !out || !al16(x) || !al16(Wg) ||
        !al16(W13q) || !al16(W2q) || !al16(W13sf) || !al16(W2sf) || !al16(out))
        return MOE_ERR_INVALID_ARG;
    if (s.d_ff_shared > 0 && (!W13s_q || !W13s_sf || !W2s_q || !W2s_sf || !al16(W13s_q) ||
                              !al16(W2s_q) || !al16(W13s_sf) || !al16(W2s_sf)))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    LowpWeights lw;
    std::memset(&lw, 0, sizeof lw);
    lw.fmt = FMT_MX8;
    lw.W13q = W13q;
    lw.W13sf = W13sf;
    lw.W2q = W2q;
    lw.W2sf = W2sf;
    lw.W13s_q = W13s_q;
    lw.W13s_sf = W13s_sf;
    lw.W2s_q = W2s_q;
    lw.W2s_sf = W2s_sf;
    return forward_mx_impl(s, L, ws, x, Wg, bias, lw, out, logits_out, topk_idx_out, status,
                           reinterpret_cast<cudaStream_t>(stream));
}

// NVFP4 GEMMs take 256-element K stages: every contraction length (d, d_ff,
// d_ff_shared) must be a multiple of 256.
static int nv_dims_ok(const moe_shape_t &s)
{
    return s.d % 256 == 0 && s.d_ff % 256 == 0 && s.d_ff_shared % 256 == 0;
}

int moe_quantize_experts_nvfp4(const moe_shape_t *shape, const moe_bf16_t *W1,
                               const moe_bf16_t *W3, const moe_bf16_t *W2, uint8_t *W13q,
                               uint8_t *W13sf, float *W13_gs, uint8_t *W2q, uint8_t *W2sf,
                               float *W2_gs, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    const moe_shape_t &s = *shape;
    if (!nv_dims_ok(s))
        return MOE_ERR_UNSUPPORTED;
    if (!W1 || !W3 || !W2 || !W13q || !W13sf || !W13_gs || !W2q || !W2sf || !W2_gs || !al16(W1) ||
        !al16(W3) || !al16(W2) || !al16(W13q) || !al16(W2q) || !al16(W13sf) || !al16(W2sf) ||
        (reinterpret_cast<uintptr_t>(W13_gs) & 3u) || (reinterpret_cast<uintptr_t>(W2_gs) & 3u))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = launch_nv_weight_scales(s, W1, W3, W2, W13_gs, W2_gs, st)))
        return rc;
    if ((rc = launch_nv_pack_w13(s, W1, W3, W13_gs, W13q, W13sf, st)))
        return rc;
    return launch_nv_quantize_rows(W2, (long long)s.E * s.d, s.d_ff, W2_gs, s.d, 0.f, W2q, W2sf,
                                   st);
}

int moe_forward_nvfp4(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                      const float *bias, const uint8_t *W13q, const uint8_t *W13sf,
                      const float *W13_gs, const uint8_t *W2q, const uint8_t *W2sf,
                      const float *W2_gs, const uint8_t *W13s_q, const uint8_t *W13s_sf,
                      const float *W13s_gs, const uint8_t *W2s_q, const uint8_t *W2s_sf,
                      const float *W2s_gs, float x_gs, float h_gs, float *out,
                      float *logits_out, int32_t *topk_idx_out, uint32_t *status, void *ws,
                      size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    const moe_shape_t &s = *shape;
    if (!(s.flags & MOE_FLAG_NVFP4) || (s.flags & (MOE_FLAG_HOST_IO | MOE_FLAG_MXFP8)))
        return MOE_ERR_INVALID_ARG;
    if (!nv_dims_ok(s))
        return MOE_ERR_UNSUPPORTED;
    if (!(x_gs > 0.f) || !(h_gs > 0.f) || !std::isfinite(x_gs) || !std::isfinite(h_gs))
        return MOE_ERR_INVALID_ARG;
    if (s.T == 0)
        return MOE_OK;
    if (!x || !Wg || !W13q || !W13sf || !W13_gs || !W2q || !W2sf || !W2_gs || !out || !al16(x) ||
        !al16(Wg) || !al16(W13q) || !al16(W2q) || !al16(W13sf) || !al16(W2sf) || !al16(out))
        return MOE_ERR_INVALID_ARG;
    if (s.d_ff_shared > 0 &&
        (!W13s_q || !W13s_sf || !W13s_gs || !W2s_q || !W2s_sf || !W2s_gs || !al16(W13s_q) ||
         !al16(W2s_q) || !al16(W13s_sf) || !al16(W2s_sf)))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    LowpWeights lw;
    std::memset(&lw, 0, sizeof lw);
    lw.fmt = FMT_NV4;
    lw.W13q = W13q;
    lw.W13sf = W13sf;
    lw.W13gs = W13_gs;
    lw.W2q = W2q;
    lw.W2sf = W2sf;
    lw.W2gs = W2_gs;
    lw.W13s_q = W13s_q;
    lw.W13s_sf = W13s_sf;
    lw.W13s_gs = W13s_gs;
    lw.W2s_q = W2s_q;
    lw.W2s_sf = W2s_sf;
    lw.W2s_gs = W2s_gs;
    lw.x_gs = x_gs;
    lw.h_gs = h_gs;
    return forward_mx_impl(s, L, ws, x, Wg, bias, lw, out, logits_out, topk_idx_out, status,
                           reinterpret_cast<cudaStream_t>(stream));
}

int moe_pack_backward(const moe_shape_t *shape, const moe_bf16_t *W13, const moe_bf16_t *W2,
                      moe_bf16_t *W13T, moe_bf16_t *W2T, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;
    const moe_shape_t &s = *shape;
    if (!W13 || !W2 || !W13T || !W2T || !al16(W13) || !al16(W2) || !al16(W13T) || !al16(W2T))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = launch_transpose_batched(W13, s.E, 2 * s.d_ff, s.d, W13T, st)))
        return rc;
    return launch_transpose_batched(W2, s.E, s.d, s.d_ff, W2T, st);
}

int moe_backward(const moe_shape_t *shape, const moe_bf16_t *x, const moe_bf16_t *Wg,
                 const float *bias, const moe_bf16_t *W13, const moe_bf16_t *W13T,
                 const moe_bf16_t *W2T, const moe_bf16_t *W13_shared,
                 const moe_bf16_t *W13T_shared, const moe_bf16_t *W2T_shared, const float *dout,
                 float *dx, float *dW13, float *dW2, float *dW13_shared, float *dW2_shared,
                 float *dWg, float *dbias, float *dlogits, uint32_t *status, void *ws,
                 size_t ws_bytes, moe_stream_t stream)
{
    int rc = check_shape(shape);
    if (rc)
        return rc;
    if (shape->T == 0)
        return MOE_OK;
    const moe_shape_t &s = *shape;
    if (!(s.flags & MOE_FLAG_BACKWARD) || (s.flags & (MOE_FLAG_MXFP8 | MOE_FLAG_NVFP4 | MOE_FLAG_SIMT_FFN)))
        return MOE_ERR_INVALID_ARG;
    if (!x || !Wg || !W13 || !W13T || !W2T || !dout || !dx || !dW13 || !dW2 || !dWg || !dbias ||
        !al16(x) || !al16(Wg) || !al16(W13) || !al16(W13T) || !al16(W2T) || !al16(dout) ||
        !al16(dx) || !al16(dW13) || !al16(dW2))
        return MOE_ERR_INVALID_ARG;
    if (s.d_ff_shared > 0 &&
        (!W13_shared || !W13T_shared || !W2T_shared || !dW13_shared || !dW2_shared ||
         !al16(W13_shared) || !al16(W13T_shared) || !al16(W2T_shared) || !al16(dW13_shared) ||
         !al16(dW2_shared)))
        return MOE_ERR_INVALID_ARG;
    WsLayout L;
    if ((rc = check_ws(s, ws, ws_bytes, L)))
        return rc;
    return backward_impl(s, L, ws, x, Wg, bias, W13, W13T, W2T, W13_shared, W13T_shared,
                         W2T_shared, dout, dx, dW13, dW2, dW13_shared, dW2_shared, dWg, dbias,
                         dlogits, status, reinterpret_cast<cudaStream_t>(stream));
}

} // extern "C"
