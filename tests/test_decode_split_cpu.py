"""How the tensor-core decode kernels divide their work over a launch's CTAs:
the functions of csrc/decode_split.cuh compiled for the host and run over
decode shapes. No GPU.

w1/w3 (dt_split, dt_work, dt_num_works): with G CTAs, whole tiles for
items / G rounds, then the R leftover tiles cut along K into np pieces of ps
stages, unit u = piece u mod np of leftover tile u / np on CTA u mod G.
Every (tile, K stage) must be run exactly once, the pieces of leftover tile
j must be units j np .. j np + np - 1 (where the second kernel reads them),
there are at most 2 G units (the size of the sums buffer), and the CTAs'
work differs by at most the tail's pieces.

w2 (d2_space, d2_piece, d2_first_cta, d2_pmax): CTA c runs stages
[c F / G, (c + 1) F / G) of the (tile, K stage) sequence. Every stage must be
run exactly once, no CTA may have more pieces than d2_pmax allows for the
launch's largest F, and the reduce's list for a tile (the CTAs from
d2_first_cta on whose ranges meet it, each with piece index
tile - first tile of its range) must name exactly the pieces that ran it, in
ascending CTA order.
"""
import os
import subprocess
import tempfile

import pytest

from sparse_mixture_experts_17_b200 import build as B

HARNESS = r"""
#include <cstdio>
#include <map>
#include <set>
#include <utility>
#include <vector>
#include "decode_split.cuh"
using namespace moe;

static int fail(const char *what, int a, int b, int c)
{
    std::printf("FAIL %s %d %d %d\n", what, a, b, c);
    return 1;
}

// w1/w3: items tiles of nks stages over G CTAs
static int check_w13(int items, int G, int nks)
{
    const DtSplit sp = dt_split(items, G, nks);
    std::map<std::pair<int, int>, int> runs;
    std::map<int, std::pair<int, int>> unit_item;   // unit -> (tile, first stage)
    int max_stages = 0, min_stages = 1 << 30;
    for (int c = 0; c < G; ++c) {
        const int nw = dt_num_works(sp, G, c);
        int stages = 0;
        for (int w = 0; w < nw; ++w) {
            int item, kb0, kb1, unit;
            dt_work(sp, G, c, w, nks, item, kb0, kb1, unit);
            if (item < 0 || item >= items || kb0 < 0 || kb1 > nks || kb0 >= kb1)
                return fail("w13 range", items, G, c);
            if ((unit >= 0) != (w >= sp.full) || (unit >= 0 && unit % G != c))
                return fail("w13 unit owner", items, G, c);
            if (unit >= 0)
                unit_item[unit] = std::make_pair(item, kb0);
            for (int kb = kb0; kb < kb1; ++kb)
                ++runs[std::make_pair(item, kb)];
            stages += kb1 - kb0;
        }
        max_stages = stages > max_stages ? stages : max_stages;
        min_stages = stages < min_stages ? stages : min_stages;
    }
    if ((long long)runs.size() != (long long)items * nks)
        return fail("w13 coverage", items, G, nks);
    for (auto &kv : runs)
        if (kv.second != 1)
            return fail("w13 twice", kv.first.first, kv.first.second, kv.second);
    if (sp.units > 2 * G)
        return fail("w13 units", items, G, sp.units);
    // leftover tile j: pieces p = 0 .. np-1 are units j np + p, from stage p ps
    for (int j = 0; j < sp.R; ++j)
        for (int p = 0; p < sp.np; ++p) {
            auto it = unit_item.find(j * sp.np + p);
            if (it == unit_item.end() || it->second.first != sp.full * G + j ||
                it->second.second != p * sp.ps)
                return fail("w13 piece index", items, G, j);
        }
    // the whole rounds are equal; the tail adds at most ceil(units / G) pieces
    if (max_stages - min_stages > sp.ps * ((sp.units + G - 1) / G))
        return fail("w13 balance", items, G, max_stages - min_stages);
    return 0;
}

// w2: U chosen experts (+ shared) over G CTAs, G and pmax from the largest U
static int check_w2(int U, int Umax, int has_shared, int d, int d_ff, int d_ff_s, int nsm)
{
    const D2Space zmax = d2_space(Umax, has_shared, d, d_ff, d_ff_s);
    const int G = (int)(zmax.F < nsm ? (zmax.F > 0 ? zmax.F : 1) : nsm);
    const int nks_min = has_shared && zmax.nks_s < zmax.nks ? zmax.nks_s : zmax.nks;
    const int pmax = d2_pmax(zmax.F, G, nks_min);
    const D2Space z = d2_space(U, has_shared, d, d_ff, d_ff_s);
    std::map<std::pair<int, int>, int> runs;
    std::map<int, std::vector<std::pair<int, int>>> ran;   // tile -> (CTA, piece)
    long long lo = z.F, hi = 0;
    for (int c = 0; c < G; ++c) {
        int lp = 0, item, kb0, kb1;
        for (; d2_piece(z, G, c, lp, item, kb0, kb1); ++lp) {
            const int nk = item < z.routed_items ? z.nks : z.nks_s;
            if (item < 0 || item >= z.items || kb0 < 0 || kb1 > nk || kb0 >= kb1)
                return fail("w2 range", U, G, c);
            for (int kb = kb0; kb < kb1; ++kb)
                ++runs[std::make_pair(item, kb)];
            ran[item].push_back(std::make_pair(c, lp));
        }
        if (lp > pmax)
            return fail("w2 pmax", U, c, lp);
        const long long len = d2_f0(z, G, c + 1) - d2_f0(z, G, c);
        lo = len < lo ? len : lo;
        hi = len > hi ? len : hi;
    }
    long long want = 0;
    for (int i = 0; i < z.items; ++i)
        want += i < z.routed_items ? z.nks : z.nks_s;
    if ((long long)runs.size() != want)
        return fail("w2 coverage", U, G, (int)runs.size());
    for (auto &kv : runs)
        if (kv.second != 1)
            return fail("w2 twice", kv.first.first, kv.first.second, kv.second);
    if (z.F > 0 && hi - lo > 1)
        return fail("w2 balance", U, G, (int)(hi - lo));
    // the reduce's list, generated as the reduce kernel does
    for (int item = 0; item < z.items; ++item) {
        const long long s0 = d2_item_start(z, item), s1 = d2_item_start(z, item + 1);
        std::vector<std::pair<int, int>> got;
        for (int cc = d2_first_cta(z, G, s0);; ++cc) {
            const long long a = cc < G ? d2_f0(z, G, cc) : s1;
            if (a >= s1)
                break;
            const long long b = d2_f0(z, G, cc + 1);
            if (b > s0 && b > a)
                got.push_back(std::make_pair(cc, item - d2_item_of(z, a)));
        }
        if (got != ran[item])
            return fail("w2 reduce list", U, G, item);
    }
    return 0;
}

int main()
{
    char kind[8];
    int bad = 0;
    while (std::scanf("%7s", kind) == 1) {
        if (kind[0] == 'a') {
            int items, G, nks;
            std::scanf("%d %d %d", &items, &G, &nks);
            bad |= check_w13(items, G, nks);
        } else {
            int U, Umax, sh, d, d_ff, d_ff_s, nsm;
            std::scanf("%d %d %d %d %d %d %d", &U, &Umax, &sh, &d, &d_ff, &d_ff_s, &nsm);
            bad |= check_w2(U, Umax, sh, d, d_ff, d_ff_s, nsm);
        }
    }
    std::printf(bad ? "bad\n" : "ok\n");
    return bad;
}
"""


@pytest.fixture(scope="module")
def harness():
    d = tempfile.mkdtemp(prefix="decode_split_")
    src = os.path.join(d, "h.cu")
    exe = os.path.join(d, "h")
    with open(src, "w") as f:
        f.write(HARNESS)
    r = subprocess.run([B.nvcc(), *B.ARCH, "-std=c++17", "-O1", "-I", B.CSRC, "-I", B.INCLUDE, src, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def run(exe, lines):
    r = subprocess.run([exe], input="\n".join(lines) + "\n", capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]


def test_w13_split_mixtral_and_edges(harness):
    lines = []
    # one and two tokens at the Mixtral shape on 148 SMs (448 / 896 tiles of 16 stages)
    lines += ["a 448 148 16", "a 896 148 16", "a 672 148 16", "a 452 148 16"]
    # fewer tiles than CTAs (everything split), exact multiples, one CTA, no tiles
    for items in (0, 1, 7, 47, 48, 96, 147, 148, 149, 295, 296, 297, 1000):
        for G in (1, 3, 37, 148):
            if G <= max(items, 1):
                for nks in (1, 2, 4, 16, 28, 56):
                    lines.append(f"a {items} {G} {nks}")
    run(harness, lines)


def test_w2_stream_k_mixtral_and_edges(harness):
    lines = []
    for U in range(0, 5):   # the launch is sized for U = min(E, T k)
        lines.append(f"b {U} 2 0 4096 14336 0 148")
        lines.append(f"b {U} 4 0 4096 14336 0 148")
        lines.append(f"b {U} 4 1 4096 14336 2048 148")
    for U in range(0, 17):
        lines.append(f"b {U} 16 1 1024 512 256 148")    # many small experts, shared expert
        lines.append(f"b {U} 16 0 512 256 0 148")       # fewer stages than CTAs
    lines += ["b 2 2 1 1024 9728 256 148", "b 1 1 1 256 256 512 148", "b 3 3 0 4096 1536 0 7"]
    run(harness, lines)
