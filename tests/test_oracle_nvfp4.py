"""Pins of the oracle's NVFP4 experts (CPU only).

The E2M1 table is checked against the bit-field definition of the format;
the encoder against midpoints (ties to the even code), saturation and the
sign rule; the E4M3 scale encoder against the C oracle's (itself pinned) and
torch's float8_e4m3fn cast; the block rule against special cases that reduce
to plain E2M1 rounding, exact round trips and its error bound; the layer
against the C oracle's fp64 layer when quantization is the identity, and the
quantization placement (which tensor, which global scale, which axis).
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as N
from sparse_mixture_experts_17_b200 import inputs as I


def _f32(a):
    return np.asarray(a, np.float32)


def test_e2m1_table_from_bit_fields():
    for c in range(16):
        s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
        mag = (m / 2.0) * 2.0 ** 0 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
        assert N.e2m1_decode(np.array([c]))[0] == (-mag if s else mag)


def test_e2m1_encode_grid_midpoints_saturation():
    grid = N.e2m1_decode(np.arange(8))
    # every representable magnitude encodes to itself, both signs
    assert (N.e2m1_encode(_f32(grid)) == np.arange(8)).all()
    assert (N.e2m1_encode(_f32(-grid[1:])) == np.arange(1, 8) | 8).all()
    # midpoints go to the neighbour with the even code
    mids = (grid[:-1] + grid[1:]) / 2
    lo, hi = np.arange(7), np.arange(1, 8)
    want = np.where(lo % 2 == 0, lo, hi)
    assert (N.e2m1_encode(_f32(mids)) == want).all()
    # just off a midpoint goes to the nearer neighbour
    eps = np.float32(1e-3)
    assert (N.e2m1_encode(_f32(mids) - eps) == lo).all()
    assert (N.e2m1_encode(_f32(mids) + eps) == hi).all()
    # saturation, and the sign of a zero result is the sign of the input
    assert (N.e2m1_encode(_f32([6.5, 7.0, 1e30, -1e30])) == [7, 7, 7, 15]).all()
    assert (N.e2m1_encode(_f32([0.0, -0.0, 0.2, -0.2])) == [0, 8, 0, 8]).all()


def test_e2m1_encode_is_nearest():
    rng = np.random.default_rng(0)
    v = _f32(rng.uniform(-7, 7, 20000))
    dec = N.e2m1_decode(N.e2m1_encode(v))
    grid = N.e2m1_decode(np.arange(8))
    best = np.abs(np.abs(v)[:, None] - grid).min(1)
    # |v| <= 6: the decoded value is a nearest grid point; beyond, 6
    inside = np.abs(v) <= 6
    assert np.allclose(np.abs(np.abs(dec[inside]) - np.abs(v[inside])), best[inside], atol=0)
    assert (np.abs(dec[~inside]) == 6.0).all()
    assert (np.sign(dec[dec != 0]) == np.sign(v[dec != 0])).all()


def test_e4m3_encoder_matches_c_oracle_and_torch(orc):
    rng = np.random.default_rng(1)
    v = np.concatenate([_f32(np.exp2(rng.uniform(-12, 9.2, 4000))),
                        _f32([0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -6, 448.0, 464.0,
                              479.0, 1e6, 240.0, 0.0625 * 1.0625])])
    mine = N.e4m3_encode_pos(v)
    c = np.array([orc.e4m3_encode(float(x)) for x in v])
    assert (mine == c).all()
    ok = v <= 448
    t = torch.from_numpy(v[ok]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (mine[ok] == t).all()
    assert (N.e4m3_decode(mine) == N.e4m3_decode(c)).all()


def test_block_rule_reduces_to_plain_rounding():
    """gs = 1 and a block maximum of 6: scale 1, r = 1, codes = E2M1(v)."""
    rng = np.random.default_rng(2)
    v = _f32(rng.uniform(-6, 6, (5, 16)))
    v[:, 0] = 6.0
    codes, sc = N.quantize(v, 1.0)
    assert (N.e4m3_decode(sc) == 1.0).all()
    assert (codes == N.e2m1_encode(v)).all()
    # an all-zero block: scale code 0, codes 0
    z = np.zeros((1, 32), np.float32)
    c0, s0 = N.quantize(z, 3.0)
    assert (s0 == 0).all() and (c0 == 0).all()


def test_round_trip_exact_on_representable_values():
    """Blocks of E2M1 grid values times 2^j, with a tensor maximum of 6 * 2^J:
    gs = 448 * 2^-J, the scales are powers of two times 448, r = 2^-j, so
    quantizing and dequantizing returns the input exactly."""
    rng = np.random.default_rng(3)
    grid = N.e2m1_decode(np.arange(16))
    J = 3
    rows = []
    for j in range(-4, J + 1):
        b = grid[rng.integers(0, 16, 16)]
        b[rng.integers(0, 16)] = 6.0          # block maximum 6 * 2^j
        rows.append(b * 2.0 ** j)
    v = _f32(np.stack(rows))
    gs = N.global_scale(np.abs(v).max())
    assert gs == np.float32(448 * 2.0 ** -J)
    assert (N.qdq(v, gs) == v).all()


def test_error_bound_and_global_scale():
    """|qdq(v) - v| <= s / gs per element (E2M1 half-spacing <= 1 up to 6, and
    the scale rounding keeps |v r| <= 6.4 < 7), and the block holding the
    tensor's maximum gets the scale 448."""
    rng = np.random.default_rng(4)
    v = _f32(rng.standard_normal((64, 256)) * 0.02)
    gs = N.global_scale(np.abs(v).max())
    codes, sc = N.quantize(v, gs)
    s = N.e4m3_decode(sc)
    dq = N.dequantize(codes, sc, gs)
    err = np.abs(dq - v).reshape(64, 16, 16)
    assert (err <= (s / gs)[..., None] * (1 + 1e-6)).all()
    r, c = np.unravel_index(np.abs(v).argmax(), v.shape)
    assert sc[r, c // 16] == N.e4m3_encode_pos(_f32([448.0]))[0]
    # relative Frobenius error of 4-bit values with 16-element blocks is a few percent
    rel = np.linalg.norm(dq - v) / np.linalg.norm(v)
    assert 0.02 < rel < 0.15, rel


def _layer_inputs(seed, shared):
    w = I.Workload("nv", T=12, d=32, d_ff=48, E=4, k=2, capacity=0,
                   d_ff_shared=32 if shared else 0, zipf_s=0.3)
    inp = I.oracle_arrays(I.make_inputs(w, "cpu", seed=seed))
    return w, inp


@pytest.mark.parametrize("shared", [False, True])
def test_layer_matches_fp64_layer_without_quantization(orc, monkeypatch, shared):
    """With quantization replaced by the identity the NVFP4 layer is the fp64
    layer of the C oracle (h rounded once to fp32: relative 1e-6)."""
    w, inp = _layer_inputs(5, shared)
    _, L32 = orc.router_logits(inp["x"], inp["wg"], inp["bias"])
    idx, wts = orc.route(L32, w.k)
    disp = orc.dispatch(idx, w.E, 3)                 # with drops
    assert (disp["slot_pos"] < 0).any()
    tokens = np.arange(w.T, dtype=np.int32)
    kw = {k: inp[k] for k in ("W1s", "W3s", "W2s")} if shared else {}
    ref = orc.moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, wts, disp["slot_pos"],
                         tokens, h_bf16=False, **kw)
    monkeypatch.setattr(N, "qdq", lambda v, gs: np.asarray(v, np.float64))
    got = N.moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, wts, disp["slot_pos"],
                       tokens, **kw)
    np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-9)


def test_layer_quantizes_each_operand_once_along_k(orc, monkeypatch):
    """x along d with gs_x, W1/W3 of expert e along d with gs13[e], h along
    d_ff with gs_h, W2 of expert e along d_ff with gs2[e]."""
    w, inp = _layer_inputs(6, False)
    _, L32 = orc.router_logits(inp["x"], inp["wg"], inp["bias"])
    idx, wts = orc.route(L32, w.k)
    disp = orc.dispatch(idx, w.E, 0)
    gs13, gs2 = N.weight_global_scales(inp["W1"], inp["W3"], inp["W2"])
    assert len(set(gs13.tolist())) == w.E            # distinct per expert
    calls = []
    real = N.qdq
    monkeypatch.setattr(N, "qdq", lambda v, gs: (calls.append((np.shape(v), float(gs))), real(v, gs))[1])
    N.moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, wts, disp["slot_pos"],
                 np.arange(w.T), gs_x=0.75, gs_h=1.25)
    assert calls[0] == ((w.T, w.d), 0.75)
    used = sorted(set(idx[disp["slot_pos"] >= 0].tolist()))
    per_expert = calls[1:]
    assert len(per_expert) == 4 * len(used)
    for n, e in enumerate(used):
        c = per_expert[4 * n: 4 * n + 4]
        assert c[0] == ((w.d_ff, w.d), float(gs13[e])) and c[1] == ((w.d_ff, w.d), float(gs13[e]))
        assert c[2] == ((w.d, w.d_ff), float(gs2[e]))
        rows = int(((idx == e) & (disp["slot_pos"] >= 0)).sum())
        assert c[3] == ((rows, w.d_ff), 1.25)
