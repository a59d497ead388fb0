"""NVFP4 experts for the oracle: plain numpy, fp64 products and sums.

TEST INFRASTRUCTURE. Only ``tests/``, the package smoke check and the
benchmark's CPU-baseline leg may import this module. The product (the CUDA
library and its binding) never calls it and shares no code with it.

What it follows. The page "Current Bug: CuTeDSLMoERunner produces wrong
output" runs the routed experts of the layer ("MoE Model Architectures",
"Mixtral 8x7B", "Sparse MoE Block" and "Expert FFN") as an NVFP4 grouped GEMM
with per-expert activation scales ("How the pipeline works"). The pages do not
spell the format out; this module takes NVFP4 as NVIDIA publishes it:

  * element: E2M1, 1 sign, 2 exponent (bias 1) and 1 mantissa bit; the
    magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7, sign in bit 3);
  * block: 16 consecutive elements along the contraction dimension share one
    E4M3 scale (the 8-bit format of oracle_e4m3_decode in moe_oracle.c);
  * tensor: one fp32 global encode scale gs. For a weight tensor it is
    448 * 6 / amax over the tensor (one tensor per expert for W1 and W3
    together, one for W2; gs = 1 when amax = 0). For the activations (x and
    the SwiGLU product h) it is a constant the caller supplies (calibration).

Encoding of a block v[0..15] (float32 values) with global scale gs, every
step an IEEE float32 operation so that a kernel takes the same decisions:
  sd = fl32(fl32(amax / 6) * gs); s = E4M3(sd) (nearest, ties to even,
  saturating at 448); r = fl32(gs / s) (0 when s = 0);
  code_i = E2M1(fl32(v_i * r)) (nearest, ties to the even code, saturating
  at 6, the sign of a zero result is the sign of v_i).
Decoding: value = E2M1 value * s / gs.
"""
from __future__ import annotations

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0
NV_BLOCK = 16
GS_NUM = np.float32(E4M3_MAX * E2M1_MAX)    # 2688, exact in fp32

# E2M1 magnitude of codes 0..7: 0 and 0.5 (exponent 0: m * 0.5), then
# (1 + m / 2) * 2^(e - 1) for e = 1..3
_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes):
    """E2M1 codes (uint8, low 4 bits) -> float64 values."""
    c = np.asarray(codes, np.int64) & 0xF
    mag = _E2M1_MAG[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(v):
    """float32 values -> E2M1 codes: the nearest representable magnitude, ties
    to the even code, |v| > 6 saturating to 6; the sign bit is v's sign."""
    v = np.asarray(v, np.float32)
    if v.size > (1 << 20):   # in slices, to bound the distance table's memory
        flat = v.reshape(-1)
        return np.concatenate([_e2m1_encode(flat[i:i + (1 << 20)])
                               for i in range(0, flat.size, 1 << 20)]).reshape(v.shape)
    return _e2m1_encode(v)


def _e2m1_encode(v):
    a = np.abs(v.astype(np.float64))
    dist = np.abs(a[..., None] - _E2M1_MAG)               # [..., 8]
    best = dist.min(-1, keepdims=True)
    cand = dist == best                                    # one or two nearest codes
    even = cand & ((np.arange(8) & 1) == 0)
    code = np.where(even.any(-1), np.argmax(even, -1), np.argmax(cand, -1))
    code = np.where(a > E2M1_MAX, 7, code)
    return (code | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def e4m3_decode(codes):
    """E4M3 codes -> float64 (bias 7, subnormals m/8 * 2^-6, 448 max, S.1111.111 NaN)."""
    c = np.asarray(codes, np.int64)
    s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
    v = np.where(e == 0, np.ldexp(m.astype(np.float64), -9), np.ldexp(8.0 + m, e - 10))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return np.where(s == 1, -v, v)


def e4m3_encode_pos(v):
    """Non-negative float32 values -> E4M3 codes: nearest value, ties to even,
    saturating at 448 (the same rule as oracle_e4m3_encode)."""
    a = np.asarray(v, np.float64)
    _, e = np.frexp(a)                                   # a = f * 2^e, 0.5 <= f < 1
    q = np.where(a < 2.0 ** -6, -9, e - 4)               # weight of the last kept bit
    r = np.minimum(np.ldexp(np.rint(np.ldexp(a, -q)), q), E4M3_MAX)
    _, er = np.frexp(r)
    sub = r < 2.0 ** -6
    m_norm = np.rint((np.ldexp(r, -(er - 1)) - 1.0) * 8.0).astype(np.int64)
    code = np.where(sub, np.rint(np.ldexp(r, 9)).astype(np.int64), ((er - 1 + 7) << 3) | m_norm)
    return code.astype(np.uint8)


def global_scale(amax) -> np.float32:
    """fl32(448 * 6 / amax), or 1 for an all-zero tensor."""
    a = np.float32(amax)
    return np.float32(1.0) if a == 0 else np.float32(GS_NUM / a)


def quantize(v, gs):
    """Rows of float32 values [.., K] (K a multiple of 16) -> (E2M1 codes
    [.., K] one per byte, E4M3 scale codes [.., K/16]). `gs` is a scalar or
    broadcasts against the leading dimensions."""
    v = np.asarray(v, np.float32)
    K = v.shape[-1]
    assert K % NV_BLOCK == 0
    b = v.reshape(v.shape[:-1] + (K // NV_BLOCK, NV_BLOCK))
    gs = np.asarray(gs, np.float32)
    gsb = gs.reshape(gs.shape + (1,)) if gs.ndim else gs   # broadcast over blocks
    amax = np.abs(b).max(-1)
    sd = (amax / np.float32(6.0)).astype(np.float32) * gsb
    sd = sd.astype(np.float32)
    sc = e4m3_encode_pos(sd)
    s = e4m3_decode(sc).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s > 0, (gsb / np.where(s > 0, s, np.float32(1))).astype(np.float32),
                     np.float32(0))
    y = (b * r[..., None]).astype(np.float32)
    codes = e2m1_encode(y).reshape(v.shape)
    return codes, sc


def dequantize(codes, scales, gs):
    """E2M1 codes [.., K] and E4M3 scales [.., K/16] -> float64 values / gs."""
    codes = np.asarray(codes)
    K = codes.shape[-1]
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (K // NV_BLOCK, NV_BLOCK))
    s = e4m3_decode(scales)[..., None]
    gs = np.asarray(gs, np.float64)
    gsb = gs.reshape(gs.shape + (1, 1)) if gs.ndim else gs
    return (vals * s / gsb).reshape(codes.shape)


def qdq(v, gs):
    """float32 rows through NVFP4 and back (float64)."""
    c, s = quantize(v, gs)
    return dequantize(c, s, gs)


def _bf16_to_f32(u16):
    u = np.asarray(u16, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32)


def weight_global_scales(W1, W3, W2):
    """Per-expert global scales (gs13 [E], gs2 [E]) of bf16 weights (uint16
    bit patterns, [E, ...])."""
    E = W1.shape[0]
    a13 = np.maximum(np.abs(_bf16_to_f32(W1)).reshape(E, -1).max(1),
                     np.abs(_bf16_to_f32(W3)).reshape(E, -1).max(1))
    a2 = np.abs(_bf16_to_f32(W2)).reshape(E, -1).max(1)
    return (np.array([global_scale(a) for a in a13], np.float32),
            np.array([global_scale(a) for a in a2], np.float32))


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _expert(xq, W1, W3, W2, gs13, gs2, gs_h):
    """[MIX] "Expert FFN" on NVFP4 operands: rows xq (already dequantized),
    W1/W3/W2 dequantized with their global scales, h rounded once to fp32 and
    quantized along d_ff with gs_h."""
    w1 = qdq(_bf16_to_f32(W1), gs13)
    w3 = qdq(_bf16_to_f32(W3), gs13)
    w2 = qdq(_bf16_to_f32(W2), gs2)
    g = xq @ w1.T
    u = xq @ w3.T
    h = (_silu(g) * u).astype(np.float32)
    return qdq(h, gs_h) @ w2.T


def moe_tokens(x, W1, W3, W2, idx, w, slot_pos, tokens, gs_x=1.0, gs_h=1.0, W1s=None, W3s=None,
               W2s=None, gs13=None, gs2=None):
    """The layer output of `tokens` with NVFP4 x, weights and h, given the
    routing ([MIX] "Sparse MoE Block": routed experts in ascending expert
    order, weighted by w; [DSK] shared expert added with weight 1). Inputs
    are bf16 bit patterns; gs13/gs2 default to the weights' own scales."""
    tokens = np.asarray(tokens, np.int64)
    E, d = W1.shape[0], x.shape[1]
    if gs13 is None:
        gs13, gs2 = weight_global_scales(W1, W3, W2)
    xq = qdq(_bf16_to_f32(x[tokens]), np.float32(gs_x))
    out = np.zeros((len(tokens), d))
    idx_t, w_t, sp_t = idx[tokens], np.asarray(w, np.float64)[tokens], slot_pos[tokens]
    for e in range(E):
        rows, slots = np.nonzero((idx_t == e) & (sp_t >= 0))
        if len(rows) == 0:
            continue
        y = _expert(xq[rows], W1[e], W3[e], W2[e], gs13[e], gs2[e], np.float32(gs_h))
        np.add.at(out, rows, w_t[rows, slots][:, None] * y)
    if W1s is not None:
        s13, s2 = weight_global_scales(W1s[None], W3s[None], W2s[None])
        out = _expert(xq, W1s, W3s, W2s, s13[0], s2[0], np.float32(gs_h)) + out
    return out
