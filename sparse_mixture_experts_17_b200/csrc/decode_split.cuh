// decode_split.cuh -- how the tensor-core decode kernels divide their work
// over a launch's CTAs (host and device: the kernels, their launchers and a
// host-compiled test use the same functions).
#pragma once

#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- w1/w3
// The work of one launch over G CTAs: `full` rounds of whole tiles (CTA c
// takes tiles c + r G), then the R = items - full G tiles left over, each cut
// into np pieces of ps K stages (the last piece may be shorter). Unit u =
// piece u % np of leftover tile u / np goes to CTA u mod G.
struct DtSplit {
    int full, R, ps, np, units;
};

__host__ __device__ __forceinline__ DtSplit dt_split(int items, int G, int nks)
{
    DtSplit s;
    s.full = items / G;
    s.R = items - s.full * G;
    s.ps = s.R ? (s.R * nks + G - 1) / G : nks;
    s.np = (nks + s.ps - 1) / s.ps;
    s.units = s.R * s.np;
    return s;
}

// Work w of CTA c: the tile, its K-stage range, and the unit (-1: whole tile).
__host__ __device__ __forceinline__ void dt_work(const DtSplit &sp, int G, int c, int w, int nks, int &item,
                                        int &kb0, int &kb1, int &unit)
{
    if (w < sp.full) {
        item = c + w * G;
        kb0 = 0;
        kb1 = nks;
        unit = -1;
    } else {
        unit = c + (w - sp.full) * G;
        item = sp.full * G + unit / sp.np;
        kb0 = (unit % sp.np) * sp.ps;
        kb1 = kb0 + sp.ps < nks ? kb0 + sp.ps : nks;
    }
}

__host__ __device__ __forceinline__ int dt_num_works(const DtSplit &sp, int G, int c)
{
    return sp.full + (c < sp.units ? (sp.units - 1 - c) / G + 1 : 0);
}

// ---------------------------------------------------------------- w2
// The w2 kernel's tiles: source u (the chosen experts ascending, then the
// shared expert) x row tile rt (128 output rows), item = u RT + rt, with nks
// K stages (nks_s for the shared expert's). F stages in all, in item order;
// CTA c of G runs stages [c F / G, (c + 1) F / G), one piece per tile it
// meets.
struct D2Space {
    int U, src, RT, nks, nks_s, routed_items, items;
    long long Fr, F;   // routed stages, all stages
};

__host__ __device__ __forceinline__ D2Space d2_space(int U, int has_shared, int d, int d_ff, int d_ff_s)
{
    D2Space z;
    z.U = U;
    z.src = U + (has_shared ? 1 : 0);
    z.RT = d / 128;
    z.nks = d_ff / 256;
    z.nks_s = has_shared ? d_ff_s / 256 : 0;
    z.routed_items = U * z.RT;
    z.items = z.src * z.RT;
    z.Fr = (long long)z.routed_items * z.nks;
    z.F = z.Fr + (long long)(has_shared ? z.RT : 0) * z.nks_s;
    return z;
}

__host__ __device__ __forceinline__ long long d2_f0(const D2Space &z, int G, int c)
{
    return (long long)c * z.F / G;
}

__host__ __device__ __forceinline__ int d2_item_of(const D2Space &z, long long f)
{
    return f < z.Fr ? (int)(f / z.nks) : z.routed_items + (int)((f - z.Fr) / z.nks_s);
}

__host__ __device__ __forceinline__ long long d2_item_start(const D2Space &z, int i)
{
    return i <= z.routed_items ? (long long)i * z.nks : z.Fr + (long long)(i - z.routed_items) * z.nks_s;
}

// Piece lp of CTA c: its tile and K-stage range; false past the CTA's range.
__host__ __device__ __forceinline__ bool d2_piece(const D2Space &z, int G, int c, int lp, int &item, int &kb0,
                                         int &kb1)
{
    const long long a = d2_f0(z, G, c), b = d2_f0(z, G, c + 1);
    if (a >= b)
        return false;
    item = d2_item_of(z, a) + lp;
    const long long s0 = d2_item_start(z, item), s1 = d2_item_start(z, item + 1);
    const long long lo = a > s0 ? a : s0, hi = b < s1 ? b : s1;
    if (lo >= hi)
        return false;
    kb0 = (int)(lo - s0);
    kb1 = (int)(hi - s0);
    return true;
}

// The last CTA whose stage range starts at or before stage s0 (F > 0).
__host__ __device__ __forceinline__ int d2_first_cta(const D2Space &z, int G, long long s0)
{
    const int c = (int)(((s0 + 1) * G + z.F - 1) / z.F) - 1;
    return c < 0 ? 0 : c;
}

// Pieces one CTA may run, for any launch of at most Fmax stages over G CTAs
// whose tiles have at least nks_min stages: a range of at most ceil(Fmax / G)
// stages meets at most ceil(that / nks_min) + 1 tiles.
__host__ __device__ __forceinline__ int d2_pmax(long long Fmax, int G, int nks_min)
{
    const long long per = (Fmax + G - 1) / G;
    return (int)((per + nks_min - 1) / nks_min) + 1;
}

} // namespace moe
