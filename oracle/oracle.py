"""Python face of the fp64 CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE. Only ``tests/``, the package smoke check and the
benchmark's CPU-baseline leg may import this module. It marshals numpy arrays
into the C oracle and back; it holds no arithmetic of the layer itself.

bf16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, EINVAL, ENONFINITE, EBADEXPERT = 0, 1, 5, 6


class OracleError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"oracle {fn} returned {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (plain gcc, OpenMP, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_round_bf16.argtypes = [ctypes.c_double]
        L.oracle_round_bf16.restype = ctypes.c_double
        L.oracle_router_logits.argtypes = [i, i, i, P, P, P, P, P]
        L.oracle_route.argtypes = [i, i, i, P, P, P]
        L.oracle_dispatch.argtypes = [i, i, i, i, i, P, P, P, P, P, P]
        L.oracle_moe_tokens.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P,
                                        i, i, P, P]
        L.oracle_expert_rows.argtypes = [i, i, i, i, P, P, P, P, i, i, P, P, P]
        L.oracle_num_threads.argtypes = []
        L.oracle_softmax_rows.argtypes = [i, i, P, P]
        L.oracle_expert_choice.argtypes = [i, i, i, P, P, P, P]
        L.oracle_e4m3_decode.argtypes = [i]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_int
        L.oracle_mx_scale_exp.argtypes = [ctypes.c_double]
        L.oracle_mx_scale_exp.restype = ctypes.c_int
        L.oracle_mx_quantize.argtypes = [ctypes.c_int64, i, P, P, P]
        L.oracle_mx_quantize.restype = ctypes.c_int
        L.oracle_moe_backward.argtypes = [i] * 6 + [P] * 23
        L.oracle_moe_backward.restype = ctypes.c_int
        L.oracle_softmax_rows.restype = ctypes.c_int
        L.oracle_expert_choice.restype = ctypes.c_int
        for f in (L.oracle_router_logits, L.oracle_route, L.oracle_dispatch,
                  L.oracle_moe_tokens, L.oracle_expert_rows, L.oracle_num_threads):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _check(fn, rc):
    if rc != OK:
        raise OracleError(fn, rc)


def num_threads() -> int:
    return lib().oracle_num_threads()


def round_bf16(v: float) -> float:
    return lib().oracle_round_bf16(float(v))


def router_logits(x, wg, bias=None):
    """x [T,d] u16, wg [E,d] u16, bias [E] f32|None -> (L64 [T,E] f64, L32 [T,E] f32)."""
    x, wg = _u16(x), _u16(wg)
    T, d = x.shape
    E = wg.shape[0]
    L64 = np.empty((T, E), np.float64)
    L32 = np.empty((T, E), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float32)
    _check("router_logits", lib().oracle_router_logits(T, d, E, _p(x), _p(wg), _p(b), _p(L64), _p(L32)))
    return L64, L32


def route(L32, k):
    """L32 [T,E] f32 -> (idx [T,k] i32, w [T,k] f64)."""
    L = np.ascontiguousarray(L32, np.float32)
    T, E = L.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    _check("route", lib().oracle_route(T, E, k, _p(L), _p(idx), _p(w)))
    return idx, w


def dispatch(idx, E, C=0, slot_priority=False):
    """idx [T,k] -> dict(counts [E], offsets [E+1], slot_pos [T,k], perm_token [T*k], n_kept).
    slot_priority: capacity ranks (and segment order) in slot-major order."""
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    slot_pos = np.empty((T, k), np.int32)
    perm_token = np.empty(max(T * k, 1), np.int32)
    n_kept = np.zeros(1, np.int32)
    _check("dispatch", lib().oracle_dispatch(T, E, k, int(C), int(bool(slot_priority)), _p(idx),
                                             _p(counts), _p(offsets),
                                             _p(slot_pos), _p(perm_token), _p(n_kept)))
    return dict(counts=counts, offsets=offsets, slot_pos=slot_pos,
                perm_token=perm_token[: T * k], n_kept=int(n_kept[0]))


def _mode(h_bf16, mx):
    """Precision mode of the oracle's expert FFN: 0 fp64, 1 bf16 h, 2 MXFP8."""
    return 2 if mx else int(bool(h_bf16))


def moe_tokens(x, W1, W3, W2, idx, w, slot_pos, tokens, h_bf16=True, W1s=None, W3s=None, W2s=None,
               mx=False):
    """Layer output rows (fp64) for the listed tokens, given the routing.
    mx: MXFP8 experts (x, weights and h through MXFP8)."""
    x, W1, W3, W2 = _u16(x), _u16(W1), _u16(W3), _u16(W2)
    T, d = x.shape
    E, d_ff, _ = W1.shape
    k = idx.shape[1]
    d_ff_s = 0
    if W1s is not None:
        W1s, W3s, W2s = _u16(W1s), _u16(W3s), _u16(W2s)
        d_ff_s = W1s.shape[0]
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    slot_pos = np.ascontiguousarray(slot_pos, np.int32)
    tokens = np.ascontiguousarray(tokens, np.int32)
    out = np.empty((len(tokens), d), np.float64)
    _check("moe_tokens", lib().oracle_moe_tokens(
        T, d, d_ff, E, k, d_ff_s, _p(x), _p(W1), _p(W3), _p(W2), _p(W1s), _p(W3s), _p(W2s),
        _p(idx), _p(w), _p(slot_pos), _mode(h_bf16, mx), len(tokens), _p(tokens), _p(out)))
    return out


def expert_rows(x, W1, W3, W2, tokens, experts, h_bf16=True, mx=False):
    """Unweighted expert outputs y[s] = FFN_{experts[s]}(x[tokens[s]]) in fp64."""
    x, W1, W3, W2 = _u16(x), _u16(W1), _u16(W3), _u16(W2)
    T, d = x.shape
    E, d_ff, _ = W1.shape
    tokens = np.ascontiguousarray(tokens, np.int32)
    experts = np.ascontiguousarray(experts, np.int32)
    y = np.empty((len(tokens), d), np.float64)
    _check("expert_rows", lib().oracle_expert_rows(T, d, d_ff, E, _p(x), _p(W1), _p(W3), _p(W2),
                                                   _mode(h_bf16, mx), len(tokens), _p(tokens),
                                                   _p(experts), _p(y)))
    return y


def forward(inp: dict, tokens=None, logits=None, h_bf16=True, mx=False):
    """Whole layer: logits (or the given fp32 logits), routing over all T tokens,
    dispatch with the capacity, then outputs for ``tokens`` (default: all).

    ``inp`` holds numpy arrays: x, wg, bias (or None), W1, W3, W2, optional
    W1s/W3s/W2s, ints k, capacity, and an optional bool slot_priority.
    """
    T = inp["x"].shape[0]
    E = inp["wg"].shape[0]
    L64 = None
    if logits is None:
        L64, L32 = router_logits(inp["x"], inp["wg"], inp.get("bias"))
    else:
        L32 = np.ascontiguousarray(logits, np.float32)
    idx, w = route(L32, inp["k"])
    disp = dispatch(idx, E, inp.get("capacity", 0), inp.get("slot_priority", False))
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    out = moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, w, disp["slot_pos"], tokens,
                     h_bf16=h_bf16, W1s=inp.get("W1s"), W3s=inp.get("W3s"), W2s=inp.get("W2s"),
                     mx=mx)
    return dict(L64=L64, L32=L32, idx=idx, w=w, out=out, tokens=np.asarray(tokens, np.int32), **disp)


def softmax_rows(L32):
    """fp64 softmax over experts of fp32 logits [T,E]."""
    L = np.ascontiguousarray(L32, np.float32)
    T, E = L.shape
    S = np.empty((T, E), np.float64)
    _check("softmax_rows", lib().oracle_softmax_rows(T, E, _p(L), _p(S)))
    return S


def expert_choice(S32, C):
    """Expert-choice selection on fp32 scores [T,E] -> (tokens [E,Ceff], w [E,Ceff])."""
    S = np.ascontiguousarray(S32, np.float32)
    T, E = S.shape
    K = min(C, T)
    tokens = np.empty((E, K), np.int32)
    w = np.empty((E, K), np.float64)
    ceff = np.zeros(1, np.int32)
    _check("expert_choice", lib().oracle_expert_choice(T, E, int(C), _p(S), _p(tokens), _p(w),
                                                       _p(ceff)))
    return tokens, w


def expert_choice_layer(inp, S32, C, tokens=None, h_bf16=True):
    """Layer output under expert-choice routing, for `tokens` (default all):
    out[t] = sum over the experts that selected t of S[t,e] * FFN_e(x_t)
    (+ the shared expert), via the per-token evaluation with E slots where
    slot e is kept iff expert e selected the token."""
    T, E = S32.shape
    sel_tok, sel_w = expert_choice(S32, C)
    idx = np.tile(np.arange(E, dtype=np.int32), (T, 1))
    w = np.zeros((T, E), np.float64)
    slot = np.full((T, E), -1, np.int32)
    for e in range(E):
        w[sel_tok[e], e] = sel_w[e]
        slot[sel_tok[e], e] = 0
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    out = moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, w, slot, tokens,
                     h_bf16=h_bf16, W1s=inp.get("W1s"), W3s=inp.get("W3s"), W2s=inp.get("W2s"))
    return dict(out=out, tokens=sel_tok, w=sel_w, tokens_eval=np.asarray(tokens, np.int32))


# ---------------------------------------------------------------- MXFP8

def e4m3_decode(codes):
    """E4M3 codes (uint8 array) -> float64 values."""
    table = np.array([lib().oracle_e4m3_decode(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(v))


def mx_scale_exp(amax: float) -> int:
    return lib().oracle_mx_scale_exp(float(amax))


def mx_quantize(a):
    """Rows of a [rows, K] (K % 32 == 0) -> (codes u8 [rows, K], scales u8 [rows, K/32])."""
    a = np.ascontiguousarray(a, np.float64)
    rows, K = a.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    _check("mx_quantize", lib().oracle_mx_quantize(rows, K, _p(a), _p(codes), _p(scales)))
    return codes, scales


def mx_dequantize(codes, scales):
    """Inverse map of mx_quantize's output back to float64 values."""
    v = e4m3_decode(codes)
    X = scales.astype(np.int64) - 127
    return v * np.repeat(np.exp2(X.astype(np.float64)), 32, axis=1)


# ---------------------------------------------------------------- backward

def moe_backward(inp, idx, w, slot_pos, dout):
    """Gradients of the fp64 layer with the routing held fixed (see
    oracle_moe_backward). inp: x, wg, W1, W3, W2 (+ W1s, W3s, W2s) as uint16;
    idx/w/slot_pos from route/dispatch; dout [T, d] float32. Returns a dict of
    float64 arrays: dx, dW1, dW3, dW2, (dW1s, dW3s, dW2s), dlogits, dWg, dbias, G."""
    x, W1, W3, W2, wg = (_u16(inp[kk]) for kk in ("x", "W1", "W3", "W2", "wg"))
    T, d = x.shape
    E, d_ff, _ = W1.shape
    k = idx.shape[1]
    has_s = inp.get("W1s") is not None
    W1s = W3s = W2s = None
    d_ff_s = 0
    if has_s:
        W1s, W3s, W2s = _u16(inp["W1s"]), _u16(inp["W3s"]), _u16(inp["W2s"])
        d_ff_s = W1s.shape[0]
    out = dict(dx=np.empty((T, d)), dW1=np.empty((E, d_ff, d)), dW3=np.empty((E, d_ff, d)),
               dW2=np.empty((E, d, d_ff)), dlogits=np.empty((T, E)), dWg=np.empty((E, d)),
               dbias=np.empty(E), G=np.empty((T, k)))
    if has_s:
        out.update(dW1s=np.empty((d_ff_s, d)), dW3s=np.empty((d_ff_s, d)), dW2s=np.empty((d, d_ff_s)))
    dout = np.ascontiguousarray(dout, np.float32)
    _check("moe_backward", lib().oracle_moe_backward(
        T, d, d_ff, E, k, d_ff_s, _p(x), _p(W1), _p(W3), _p(W2), _p(W1s), _p(W3s), _p(W2s),
        _p(wg), _p(np.ascontiguousarray(idx, np.int32)), _p(np.ascontiguousarray(w, np.float64)),
        _p(np.ascontiguousarray(slot_pos, np.int32)), _p(dout), _p(out["dx"]), _p(out["dW1"]),
        _p(out["dW3"]), _p(out["dW2"]), _p(out.get("dW1s")), _p(out.get("dW3s")),
        _p(out.get("dW2s")), _p(out["dlogits"]), _p(out["dWg"]), _p(out["dbias"]), _p(out["G"])))
    return out
