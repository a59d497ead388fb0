"""Pins of the oracle's MXFP8 arithmetic (OCP "Microscaling (MX) Formats"
v1.0: E4M3 elements, one E8M0 power-of-two scale per 32 elements) to things
other than itself: the format's closed-form values, torch's float8_e4m3fn
conversions, a brute-force nearest-even search over all codes, the shared
exponent rule's defining inequalities and hand-worked blocks (saturation
included), and a numpy composition of the quantized
expert FFN (CPU only)."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_mixture_experts_17_b200 import inputs as I


def test_e4m3_decode_closed_forms(orc):
    fixed = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x3C: 1.5, 0x40: 2.0, 0x7E: 448.0, 0x77: 240.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0}
    v = orc.e4m3_decode(list(fixed))
    assert (v == np.array(list(fixed.values()))).all()
    assert np.isnan(orc.e4m3_decode([0x7F, 0xFF])).all()


def test_e4m3_decode_matches_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = orc.e4m3_decode(codes)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert ((ref == got) | both_nan).all()


def _finite_values():
    c = np.arange(0x7F, dtype=np.uint8)          # non-negative finite codes 0x00..0x7E
    return torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()


def _brute_encode(v):
    """Nearest non-negative finite E4M3 value by exhaustive search, ties to the
    even code, saturating at 448; sign copied."""
    vals = _finite_values()
    a = abs(v)
    d = np.abs(vals - a)
    best = np.nonzero(d == d.min())[0]
    c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    return c | (0x80 if math.copysign(1.0, v) < 0 else 0)


def test_e4m3_encode_brute_force_and_ties(orc):
    vals = _finite_values()
    mids = (vals[:-1] + vals[1:]) / 2            # exact midpoints: ties
    rng = np.random.default_rng(0)
    rnd = np.concatenate([rng.uniform(0, 448, 300), np.exp2(rng.uniform(-12, 8.8, 300)),
                          rng.uniform(0, 2.0 ** -6, 100)])
    for v in np.concatenate([vals, mids, rnd, [450.0, 1e9]]):
        for sv in (v, -v):
            assert orc.e4m3_encode(sv) == _brute_encode(min(abs(sv), 448.0) * np.sign(sv)
                                                        if sv != 0 else sv), sv


def test_e4m3_encode_matches_torch(orc):
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 30, 2000), np.exp2(rng.uniform(-11, 8.7, 2000)),
                        -np.exp2(rng.uniform(-11, 8.7, 500))]).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(x)) for x in v], np.uint8)
    assert (got == ref).all()


def test_mx_scale_exponent_rule(orc):
    """OCP MX v1.0's conversion of a block: the shared exponent is
    floor(log2(max|v|)) - emax_elem, emax_elem = 8 for E4M3 (its largest
    normal binade is [256, 512)), clamped to E8M0's [-127, 127]. Pinned by its
    defining inequality 2^(8+X) <= amax < 2^(9+X) and by hand-worked values."""
    rng = np.random.default_rng(2)
    for amax in np.concatenate([np.exp2(rng.uniform(-60, 60, 500)), [448.0, 448.0 * 2 ** -3,
                                                                        448.0 * 2 ** 5 + 1e-9]]):
        X = orc.mx_scale_exp(amax)
        assert 2.0 ** (8 + X) <= amax < 2.0 ** (9 + X), (amax, X)
    # hand-worked: the binade [256, 512) is X = 0, whatever saturates in it
    for amax, X in ((256.0, 0), (448.0, 0), (480.0, 0), (np.nextafter(512.0, 0), 0), (512.0, 1),
                    (255.0, -1), (1.0, -8), (0.75, -9), (2.0 ** -119, -127), (3e38, 119)):
        assert orc.mx_scale_exp(amax) == X, (amax, X)
    # clamped to the E8M0 range; an all-zero block takes the smallest scale
    assert orc.mx_scale_exp(2.0 ** -120) == -127
    assert orc.mx_scale_exp(0.0) == -127
    assert orc.mx_scale_exp(1e-45) == -127


def test_mx_quantize_error_bound_and_identity(orc):
    rng = np.random.default_rng(3)
    a = rng.normal(0, 1, (16, 256)) * np.exp2(rng.integers(-20, 20, (16, 1)))
    a[3, 32:64] = 0.0                                   # an all-zero block
    a[5, 64:96] = np.linspace(-505.0, 505.0, 32) * 2.0 ** -7   # saturating block
    codes, scales = orc.mx_quantize(a)
    back = orc.mx_dequantize(codes, scales)
    X = scales.astype(np.int64) - 127
    n_sat = 0
    for r in range(16):
        for b in range(8):
            blk, q = a[r, 32 * b:32 * b + 32], back[r, 32 * b:32 * b + 32]
            if not blk.any():
                assert (q == 0).all()
                continue
            assert X[r, b] == orc.mx_scale_exp(np.abs(blk).max())
            top = 448.0 * 2.0 ** X[r, b]
            sat = np.abs(blk) >= 464.0 * 2.0 ** X[r, b]   # round to nearest past 448: clamp
            n_sat += int(sat.sum())
            assert (q[sat] == np.sign(blk[sat]) * top).all()
            # elsewhere |error| <= half a spacing: 2^-4 relative in a binade (3
            # mantissa bits), or half the subnormal step 2^(X-10) near zero
            bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** (X[r, b] - 10))
            assert (np.abs(q - blk)[~sat] <= bound[~sat]).all()
    assert n_sat >= 2                                   # the saturating block did saturate
    # values already on the grid come back unchanged: their block maximum
    # stays in the same binade, so the scale and the codes repeat
    assert (orc.mx_dequantize(*orc.mx_quantize(back)) == back).all()
    # a block that reaches 448 * 2^X keeps its scale and codes exactly
    c1, s1 = orc.mx_quantize(back * 0 + np.where(np.arange(256) % 32 == 0, 448.0, 1.0))
    assert (s1 == 127).all() and (c1[:, ::32] == 0x7E).all() and (c1[:, 1::32] == 0x38).all()
    # hand-worked saturation: a block of maximum 500 takes X = 0, and 500,
    # 470 and 464 clamp to 448 (code 0x7E) while 463 rounds to 448 and 440 to 448
    # (spacing 32 in [256, 512)), 430 to 416 (0x7D)
    blk = np.zeros((1, 32))
    blk[0, :7] = [500.0, 470.0, 464.0, 463.0, 440.0, 430.0, -500.0]
    c2, s2 = orc.mx_quantize(blk)
    assert s2[0, 0] == 127
    assert c2[0, :7].tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7D, 0xFE]


def test_layer_mx_mode_vs_numpy_composition(orc):
    """Precision mode 2 against an fp64 numpy composition that quantizes x, the
    weight rows and h with mx_quantize and runs the FFN with numpy matmuls."""
    w = I.Workload("mx", T=12, d=64, d_ff=96, E=4, k=2, d_ff_shared=64, zipf_s=0.5)
    inp = I.oracle_arrays(I.make_inputs(w, "cpu", seed=7))
    _, L32 = orc.router_logits(inp["x"], inp["wg"], inp["bias"])
    idx, wts = orc.route(L32, w.k)
    disp = orc.dispatch(idx, w.E, 0)
    toks = np.arange(w.T, dtype=np.int32)
    got = orc.moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, wts, disp["slot_pos"],
                         toks, W1s=inp["W1s"], W3s=inp["W3s"], W2s=inp["W2s"], mx=True)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).double().numpy()

    def qdq(a):
        a2 = a.reshape(-1, a.shape[-1])
        return orc.mx_dequantize(*orc.mx_quantize(a2)).reshape(a.shape)

    def ffn(xq, W1, W3, W2):
        g = xq @ qdq(bf(W1)).T
        u = xq @ qdq(bf(W3)).T
        h = qdq((F.silu(torch.from_numpy(g)).numpy() * u))
        return h @ qdq(bf(W2)).T

    xq = qdq(bf(inp["x"]))
    ref = ffn(xq, inp["W1s"], inp["W3s"], inp["W2s"])
    for t in range(w.T):
        for j in range(w.k):
            e = idx[t, j]
            ref[t] += wts[t, j] * ffn(xq[t:t + 1], inp["W1"][e], inp["W3"][e], inp["W2"][e])[0]
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12)
    # and the quantization matters: mode 2 differs from the bf16-h mode
    plain = orc.moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, wts, disp["slot_pos"],
                           toks, W1s=inp["W1s"], W3s=inp["W3s"], W2s=inp["W2s"])
    assert np.abs(plain - got).max() > 5e-3 * np.abs(plain).max()


def test_mx_mode_rejects_unaligned_width(orc):
    x = np.zeros((1, 48), np.uint16)
    W = np.zeros((1, 32, 48), np.uint16)
    with pytest.raises(orc.OracleError):
        orc.moe_tokens(x, W, W, np.zeros((1, 48, 32), np.uint16), np.zeros((1, 1), np.int32),
                       np.ones((1, 1)), np.zeros((1, 1), np.int32), np.zeros(1, np.int32),
                       mx=True)
