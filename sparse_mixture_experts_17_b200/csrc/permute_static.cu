// permute_static.cu -- moe_permute for callers that cannot allocate.
//
// Some callers have no way to hand the library a workspace: engines that
// reserve every byte of device memory for their own pool up front, and
// latency-critical paths that cannot afford cudaMalloc/cudaFree (cudaFree
// synchronises the whole device). For them,
// moe_permute_static runs the same histogram/offsets/permutation kernels as
// moe_permute, with their scratch in one fixed array that the library carries
// in device memory, so the call itself allocates nothing.
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "internal.h"

namespace moe {

// Fixed scratch of the no-allocation permute: per-chunk expert counts, ranks
// within a chunk, the last-CTA ticket, n_kept and the grouped-GEMM tile list.
// Every GPU that loads the library holds these 4 MiB until the process exits.
constexpr size_t kPermuteStaticBytes = 4u << 20;
static __device__ __align__(256) unsigned char g_permute_scratch[kPermuteStaticBytes];

namespace {

struct StaticLayout {
    size_t chunk_counts, rank_local, counter, n_kept, mt_row0, mt_group, num_mt, total;
};

StaticLayout static_layout(const moe_shape_t &s)
{
    StaticLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~static_cast<size_t>(255);
        return o;
    };
    const size_t T = s.T, k = s.k, E = s.E, N = T * k;
    const size_t nchunks = (T + kChunkTokens - 1) / kChunkTokens;
    const size_t max_mt = (N + kBlockM - 1) / kBlockM + E;
    L.counter = take(4);
    L.n_kept = take(4);
    L.num_mt = take(4);
    L.chunk_counts = take(chunk_count_rows(s, nchunks) * E * 4);
    L.rank_local = take(N * 4);
    L.mt_row0 = take(max_mt * 4);
    L.mt_group = take(max_mt * 4);
    L.total = off;
    return L;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

// cuCtxGetCurrent through the runtime's driver entry-point table (the library
// does not link the driver API directly).
CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

// Device address of the scratch array in the current device's context. It is
// looked up with cudaGetSymbolAddress, with that device current, the first
// time a device (or a new context of it, after a reset) is seen, and cached
// per device together with the context it belongs to. Host code must never
// pass g_permute_scratch itself to a kernel: on the host it names a shadow,
// not device memory.
int scratch_for_current_device(unsigned char **out)
{
    struct Entry {
        CUcontext ctx;
        unsigned char *ptr;
    };
    static std::mutex mu;
    static Entry cache[256] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256)
        return MOE_ERR_CUDA;
    CtxGetCurrentFn get_ctx = ctx_get_current();
    if (!get_ctx)
        return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> g(mu);
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS)
        return MOE_ERR_CUDA;
    if (!cache[dev].ptr || !ctx || cache[dev].ctx != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p)
            return MOE_ERR_CUDA;
        // the lookup made the device's context current on this thread
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
            return MOE_ERR_CUDA;
        cache[dev] = Entry{ctx, static_cast<unsigned char *>(p)};
    }
    *out = cache[dev].ptr;
    return MOE_OK;
}

} // namespace
} // namespace moe

using namespace moe;

extern "C" int moe_permute_static(const moe_shape_t *shape, const int32_t *topk_idx,
                                  const moe_bf16_t *x, int32_t *expert_counts,
                                  int32_t *expert_offsets, int32_t *slot_pos, int32_t *perm_token,
                                  moe_bf16_t *x_perm, int32_t *n_kept, uint32_t *status,
                                  moe_stream_t stream)
{
    if (check_shape(shape) != MOE_OK)
        return MOE_ERR_INVALID_ARG;
    const moe_shape_t &s = *shape;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (s.T == 0) {
        if ((expert_counts && cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * s.E, st) != cudaSuccess) ||
            (expert_offsets && cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (s.E + 1), st) != cudaSuccess) ||
            (n_kept && cudaMemsetAsync(n_kept, 0, sizeof(int32_t), st) != cudaSuccess))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!topk_idx || !expert_counts || !expert_offsets || !slot_pos || !perm_token ||
        (x && !x_perm) || (x && (!al16(x) || !al16(x_perm))))
        return MOE_ERR_INVALID_ARG;
    const StaticLayout L = static_layout(s);
    if (L.total > kPermuteStaticBytes)
        return MOE_ERR_UNSUPPORTED;
    unsigned char *base = nullptr;
    int rc = scratch_for_current_device(&base);
    if (rc)
        return rc;
    int32_t *counter = reinterpret_cast<int32_t *>(base + L.counter);
    // the array keeps the previous call's contents: the ticket must start at 0
    if (cudaMemsetAsync(counter, 0, sizeof(int32_t), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    int32_t *chunk = reinterpret_cast<int32_t *>(base + L.chunk_counts);
    int32_t *rank = reinterpret_cast<int32_t *>(base + L.rank_local);
    rc = launch_hist_scan(s, topk_idx, chunk, rank, counter, expert_counts, expert_offsets,
                          n_kept ? n_kept : reinterpret_cast<int32_t *>(base + L.n_kept),
                          reinterpret_cast<int32_t *>(base + L.mt_row0),
                          reinterpret_cast<int32_t *>(base + L.mt_group),
                          reinterpret_cast<int32_t *>(base + L.num_mt), nullptr, nullptr,
                          nullptr, status, st);
    if (rc)
        return rc;
    return launch_permute(s, topk_idx, chunk, rank, expert_offsets, x, slot_pos, perm_token,
                          x ? x_perm : nullptr, nullptr, st);
}
