"""The grouped GEMMs' tile order: band_coords (csrc/tiles.cuh) compiled for the
host and run over m-tile lists laid out as build_tiles lays them out.

build_tiles writes the experts of two or more tiles first and the experts of
one tile after them, each part in expert order with an expert's tiles
together; first[e] is expert e's first position and first[E] the length of the
first part (the whole list in the block-scaled, plain-order case). Every CTA of
a grouped GEMM walks tiles t = blockIdx.x, blockIdx.x + gridDim.x, ... and
maps each through band_coords. What has to hold:

- the map is a bijection onto every (m-tile, n-tile) pair, so no output tile
  is skipped or computed twice;
- a multi-tile expert's m-tiles for one n-tile sit together in t (one band),
  or, past gmax m-tiles, in ceil(cnt / gmax) near-equal bands, and a band
  never holds two experts: its weight block then leaves DRAM once per band;
- the two parts are interleaved evenly (any window holds its share of
  multi-part tiles to within one);
- a one-tile expert's n-tiles follow each other.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

from sparse_mixture_experts_17_b200 import build as B

HALF = 1 << 30

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "tiles.cuh"
int main()
{
    int E, tile_m, n_tiles, gmax, num_mt;
    while (std::scanf("%d %d %d %d %d", &E, &tile_m, &n_tiles, &gmax, &num_mt) == 5) {
        std::vector<int32_t> first(E + 1), seg(E + 1), grp(num_mt > 0 ? num_mt : 1);
        for (int i = 0; i <= E; ++i) std::scanf("%d", &first[i]);
        for (int i = 0; i <= E; ++i) std::scanf("%d", &seg[i]);
        for (int i = 0; i < num_mt; ++i) std::scanf("%d", &grp[i]);
        const long long total = (long long)num_mt * n_tiles;
        for (long long t = 0; t < total; ++t) {
            int m, n;
            moe::band_coords(t, num_mt, n_tiles, gmax, tile_m, first.data(), E, grp.data(),
                             seg.data(), m, n);
            std::printf("%d %d\n", m, n);
        }
        std::printf("end\n");
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def harness():
    d = tempfile.mkdtemp(prefix="tile_order_")
    src = os.path.join(d, "h.cu")
    exe = os.path.join(d, "h")
    with open(src, "w") as f:
        f.write(HARNESS)
    r = subprocess.run([B.nvcc(), *B.ARCH, "-std=c++17", "-O1", "-I", B.CSRC, "-I", B.INCLUDE, src, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def make_list(kept, tile_m, plain=False):
    """An m-tile list in build_tiles' documented order."""
    E = len(kept)
    nt = [(int(c) + tile_m - 1) // tile_m for c in kept]
    multi = [plain or n >= 2 for n in nt]
    order = [e for e in range(E) if multi[e]] + [e for e in range(E) if not multi[e]]
    first = [0] * (E + 1)
    grp = []
    pos = 0
    for e in order:
        first[e] = pos
        rem = int(kept[e]) - (nt[e] - 1) * tile_m
        for i in range(nt[e]):
            half = tile_m == 128 and i == nt[e] - 1 and rem <= 64
            grp.append(e | (HALF if half else 0))
        pos += nt[e]
    first[E] = sum(nt[e] for e in range(E) if multi[e])
    for e in range(E):   # experts without tiles: a position in their part (unused)
        if nt[e] == 0:
            first[e] = 0
    seg = np.concatenate([[0], np.cumsum(kept)]).astype(int).tolist()
    return first, seg, grp, nt


def run(exe, E, tile_m, n_tiles, gmax, first, seg, grp):
    inp = f"{E} {tile_m} {n_tiles} {gmax} {len(grp)}\n" + " ".join(map(str, first)) + "\n" + \
        " ".join(map(str, seg)) + "\n" + " ".join(map(str, grp)) + "\n"
    out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout.split("\n")
    assert out[-2] == "end"
    return np.array([list(map(int, l.split())) for l in out[:-2]], dtype=np.int64).reshape(-1, 2)


def check(exe, kept, tile_m, n_tiles, gmax, plain=False):
    E = len(kept)
    first, seg, grp, nt = make_list(kept, tile_m, plain)
    num_mt = len(grp)
    mn = run(exe, E, tile_m, n_tiles, gmax, first, seg, grp)
    total = num_mt * n_tiles
    assert mn.shape == (total, 2)
    if total == 0:
        return
    # a bijection onto all (m-tile, n-tile) pairs
    assert (mn[:, 0] >= 0).all() and (mn[:, 0] < num_mt).all()
    assert (mn[:, 1] >= 0).all() and (mn[:, 1] < n_tiles).all()
    flat = mn[:, 0] * n_tiles + mn[:, 1]
    assert np.array_equal(np.sort(flat), np.arange(total))
    nh = first[E]
    heavy = mn[:, 0] < nh
    # even interleave: every prefix holds its share of multi-part tiles, to within one
    share = np.cumsum(heavy)
    ideal = np.arange(1, total + 1) * (nh * n_tiles) / total
    assert np.all(np.abs(share - ideal) < 1.0 + 1e-9)
    # the multi-tile part: positions among its own tiles (u), band structure
    u_of_t = np.cumsum(heavy) - 1
    expert = np.array([g & ~HALF for g in grp])
    for e in range(E):
        if nt[e] == 0 or first[e] >= nh and not plain:
            continue
        sel = heavy & (expert[mn[:, 0]] == e)
        us = np.sort(u_of_t[sel])
        # the expert's tiles are one contiguous run of the multi part
        assert us[-1] - us[0] + 1 == len(us) == nt[e] * n_tiles
        nb = -(-nt[e] // gmax)
        sizes = sorted(((nt[e] // nb) + (1 if b < nt[e] % nb else 0)) for b in range(nb))
        assert max(sizes) <= gmax
        # each band: a fixed set of m-tiles that sweeps every n-tile, m fastest
        t_e = np.where(sel)[0]
        m_e, n_e = mn[t_e, 0], mn[t_e, 1]
        got_sizes = []
        i = 0
        while i < len(t_e):
            rows = set()
            j = i
            while j < len(t_e) and n_e[j] == n_e[i]:
                rows.add(int(m_e[j]))
                j += 1
            band = sorted(rows)
            assert band == list(range(band[0], band[0] + len(band)))   # consecutive m-tiles
            for n in range(n_tiles):   # the same m-tiles for every n-tile, in order
                blk = slice(i + n * len(band), i + (n + 1) * len(band))
                assert (n_e[blk] == n).all() and sorted(m_e[blk].tolist()) == band
            got_sizes.append(len(band))
            i += n_tiles * len(band)
        assert sorted(got_sizes) == sizes
    # the one-tile part: each expert's n-tiles back to back, in order
    light_t = np.where(~heavy)[0]
    lm, ln = mn[light_t, 0], mn[light_t, 1]
    for i in range(0, len(light_t), n_tiles):
        assert (lm[i:i + n_tiles] == lm[i]).all()
        assert np.array_equal(ln[i:i + n_tiles], np.arange(n_tiles))


def test_prefill_shape_one_band_per_expert(harness):
    # 16384 tokens x k = 2 over 8 experts (31..34 m-tiles each); bands of up to 48
    kept = [4139, 3944, 4239, 4050, 4140, 4021, 4041, 4194]
    check(harness, kept, 128, 112, 48)


def test_skewed_experts_split_into_bands(harness):
    rng = np.random.default_rng(0)
    kept = (rng.zipf(1.6, 64) * 9) % 3000
    kept[5] = 0
    kept[7] = 1
    kept[9] = 64
    kept[11] = 65
    kept[13] = 129
    check(harness, kept.tolist(), 128, 7, 5)


def test_gmax_boundaries(harness):
    # counts of tiles around gmax and its multiples: 1 band, 2 bands, 3 bands
    kept = [128 * 6, 128 * 7, 128 * 12, 128 * 13, 128 * 2 + 1, 64, 0, 128 * 18]
    check(harness, kept, 128, 3, 6)


def test_only_one_tile_experts(harness):
    check(harness, [100, 5, 0, 128, 64], 128, 4, 8)


def test_only_multi_tile_experts(harness):
    check(harness, [300, 1000, 257], 128, 5, 3)


def test_plain_order_block_scaled(harness):
    # block-scaled lists: plain expert order, one part (first[E] = list length)
    check(harness, [500, 20, 0, 129, 7000], 128, 6, 16, plain=True)


def test_pair_list_256_rows(harness):
    kept = [4139, 3944, 4239, 4050, 300, 100, 0, 256]
    check(harness, kept, 256, 16, 6)


def test_empty_list(harness):
    check(harness, [0, 0, 0], 128, 4, 8)
