"""Thin Python binding of libmoe.so (the C ABI declared in include/moe.h).

Argument marshalling only: every function here checks tensor dtypes and
devices, turns torch tensors into raw device pointers and the current torch
stream into a cudaStream_t, and calls the entry point of the same name. All
arithmetic runs in the library's CUDA kernels. There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_NONFINITE = 5
MOE_ERR_BAD_EXPERT = 6
MOE_ERR_TIMEOUT = 7
MOE_ERR_CHECK = 8

MOE_FLAG_DETERMINISTIC = 1 << 0
MOE_FLAG_FORCE_PREFILL = 1 << 1
MOE_FLAG_FORCE_DECODE = 1 << 2
MOE_FLAG_SIMT_FFN = 1 << 3
MOE_FLAG_HOST_IO = 1 << 4
MOE_FLAG_GEMM_1SM = 1 << 5
MOE_FLAG_GEMM_2SM = 1 << 6
MOE_FLAG_EXPERT_CHOICE = 1 << 7
MOE_FLAG_SLOT_PRIORITY = 1 << 8
MOE_FLAG_MXFP8 = 1 << 9
MOE_FLAG_BACKWARD = 1 << 10
MOE_FLAG_NVFP4 = 1 << 11
MOE_FLAG_DEBUG_CHECKS = 1 << 12
MOE_FLAG_TEST_TIMEOUT = 1 << 13

MOE_MAX_E = 256
MOE_MAX_K = 16
MOE_DECODE_MAX_T = 16


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {code} ({msg})")
        self.code = code


class moe_shape_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("d_ff_shared", ctypes.c_int32), ("flags", ctypes.c_int32)]

    def __repr__(self):
        return "moe_shape_t(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_shape(T, d, d_ff, E, k, capacity=0, d_ff_shared=0, flags=0) -> moe_shape_t:
    return moe_shape_t(T, d, d_ff, E, k, capacity, d_ff_shared, flags)


def shape_of(workload, flags=0, T=None) -> moe_shape_t:
    w = workload
    return make_shape(w.T if T is None else T, w.d, w.d_ff, w.E, w.k, w.capacity, w.d_ff_shared,
                      flags)


_lib = None
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_SHP = ctypes.POINTER(moe_shape_t)

_SIGS = {
    "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "moe_workspace_size": ([_SHP, ctypes.POINTER(_SZ)], ctypes.c_int),
    "moe_pack_w13": ([_SHP, _P, _P, _P, _P], ctypes.c_int),
    "moe_route": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_permute": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_expert_ffn": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_combine": ([_SHP, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_forward": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_forward_host": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_permute_static": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_check_dispatch": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_quantize_experts_mxfp8": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_forward_mxfp8": ([_SHP] + [_P] * 16 + [_SZ, _P], ctypes.c_int),
    "moe_quantize_experts_nvfp4": ([_SHP] + [_P] * 10, ctypes.c_int),
    "moe_forward_nvfp4": ([_SHP] + [_P] * 15 + [ctypes.c_float, ctypes.c_float] + [_P] * 5 +
                          [_SZ, _P], ctypes.c_int),
    "moe_pack_backward": ([_SHP, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_backward": ([_SHP] + [_P] * 20 + [_SZ, _P], ctypes.c_int),
    "moe_route_expert_choice": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_forward_expert_choice": ([_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
                                  ctypes.c_int),
    "moe_kernel_launches": ([], ctypes.c_uint64),
    "moe_profile_enable": ([ctypes.c_int], ctypes.c_int),
    "moe_profile_read": ([_P, _P, ctypes.c_int], ctypes.c_int),
}

STAGES = ["router", "topk", "hist", "permute", "shared", "w13", "w2", "combine", "dec_w13",
          "dec_w2", "bwd_dx", "bwd_dw", "bwd_router"]


def header_entry_points() -> list[str]:
    """Names of the entry points that include/moe.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not found at {LIB_PATH}: build it with "
                               "`python -m sparse_mixture_experts_17_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def _check(fn, rc):
    if rc != MOE_OK:
        raise MoeError(fn, rc, status_string(rc))


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _host_ptr(t, dtype, name):
    if t.is_cuda or not t.is_contiguous() or t.dtype != dtype:
        raise ValueError(f"{name}: must be a contiguous host tensor of {dtype}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


BF16, F32, I32, U32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.int32, torch.uint8


# ---------------------------------------------------------------- entry points

def moe_workspace_size(shape: moe_shape_t) -> int:
    n = _SZ(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def alloc_workspace(shape: moe_shape_t, device="cuda") -> torch.Tensor:
    """A workspace of the right size (torch allocates; the library never does)."""
    return torch.empty(max(moe_workspace_size(shape), 256), dtype=torch.uint8, device=device)


def moe_pack_w13(shape, W1, W3, W13=None, stream=None):
    if W13 is None:
        W13 = torch.empty(shape.E, 2 * shape.d_ff, shape.d, dtype=BF16, device=W1.device)
    _check("moe_pack_w13", lib().moe_pack_w13(ctypes.byref(shape), _ptr(W1, BF16, "W1"),
                                              _ptr(W3, BF16, "W3"), _ptr(W13, BF16, "W13"),
                                              _stream(stream)))
    return W13


def moe_route(shape, x, Wg, bias, logits, topk_idx, topk_w, status, ws, stream=None):
    _check("moe_route", lib().moe_route(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(logits, F32, "logits"), _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel() if ws is not None else 0,
        _stream(stream)))


def moe_permute(shape, topk_idx, x, expert_counts, expert_offsets, slot_pos, perm_token, x_perm,
                n_kept, status, ws, stream=None):
    _check("moe_permute", lib().moe_permute(
        ctypes.byref(shape), _ptr(topk_idx, I32, "topk_idx"), _ptr(x, BF16, "x"),
        _ptr(expert_counts, I32, "expert_counts"), _ptr(expert_offsets, I32, "expert_offsets"),
        _ptr(slot_pos, I32, "slot_pos"), _ptr(perm_token, I32, "perm_token"),
        _ptr(x_perm, BF16, "x_perm"), _ptr(n_kept, I32, "n_kept"), _ptr(status, U32, "status"),
        _ptr(ws, name="ws"), ws.numel(), _stream(stream)))


def moe_check_dispatch(shape, topk_idx, expert_offsets, slot_pos, perm_token, n_kept, status, ws,
                       stream=None):
    """Debug consistency checks of a dispatch; failures set bits of `status`."""
    _check("moe_check_dispatch", lib().moe_check_dispatch(
        ctypes.byref(shape), _ptr(topk_idx, I32, "topk_idx"),
        _ptr(expert_offsets, I32, "expert_offsets"), _ptr(slot_pos, I32, "slot_pos"),
        _ptr(perm_token, I32, "perm_token"), _ptr(n_kept, I32, "n_kept"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel(), _stream(stream)))


def moe_permute_static(shape, topk_idx, x, expert_counts, expert_offsets, slot_pos, perm_token,
                       x_perm, n_kept, status, stream=None):
    """moe_permute with the library's own fixed scratch: allocates nothing."""
    _check("moe_permute_static", lib().moe_permute_static(
        ctypes.byref(shape), _ptr(topk_idx, I32, "topk_idx"), _ptr(x, BF16, "x"),
        _ptr(expert_counts, I32, "expert_counts"), _ptr(expert_offsets, I32, "expert_offsets"),
        _ptr(slot_pos, I32, "slot_pos"), _ptr(perm_token, I32, "perm_token"),
        _ptr(x_perm, BF16, "x_perm"), _ptr(n_kept, I32, "n_kept"), _ptr(status, U32, "status"),
        _stream(stream)))


def moe_route_expert_choice(shape, x, Wg, bias, logits, scores, expert_tokens, expert_w, status,
                            ws, stream=None):
    _check("moe_route_expert_choice", lib().moe_route_expert_choice(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(logits, F32, "logits"), _ptr(scores, F32, "scores"),
        _ptr(expert_tokens, I32, "expert_tokens"), _ptr(expert_w, F32, "expert_w"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel(), _stream(stream)))


def moe_forward_expert_choice(shape, x, Wg, bias, W13, W2, W13_shared, W2_shared, out, status, ws,
                              stream=None):
    _check("moe_forward_expert_choice", lib().moe_forward_expert_choice(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(W13, BF16, "W13"), _ptr(W2, BF16, "W2"), _ptr(W13_shared, BF16, "W13_shared"),
        _ptr(W2_shared, BF16, "W2_shared"), _ptr(out, F32, "out"), _ptr(status, U32, "status"),
        _ptr(ws, name="ws"), ws.numel(), _stream(stream)))


def moe_quantize_experts_mxfp8(shape, W1, W3, W2, stream=None) -> dict:
    """MXFP8 experts from bf16 ones: dict(W13q, W13sf, W2q, W2sf) (uint8 tensors; the
    scale arrays are flat, in the scale-atom order moe.h describes)."""
    E, d_ff, d = shape.E, shape.d_ff, shape.d
    dev = W1.device
    q = dict(W13q=torch.empty(E, 2 * d_ff, d, dtype=U8, device=dev),
             W13sf=torch.empty(E * 2 * d_ff * d // 32, dtype=U8, device=dev),
             W2q=torch.empty(E, d, d_ff, dtype=U8, device=dev),
             W2sf=torch.empty(E * d * d_ff // 32, dtype=U8, device=dev))
    _check("moe_quantize_experts_mxfp8", lib().moe_quantize_experts_mxfp8(
        ctypes.byref(shape), _ptr(W1, BF16, "W1"), _ptr(W3, BF16, "W3"), _ptr(W2, BF16, "W2"),
        _ptr(q["W13q"], U8, "W13q"), _ptr(q["W13sf"], U8, "W13sf"), _ptr(q["W2q"], U8, "W2q"),
        _ptr(q["W2sf"], U8, "W2sf"), _stream(stream)))
    return q


def moe_forward_mxfp8(shape, x, Wg, bias, q, qs, out, logits_out, topk_idx_out, status, ws,
                      stream=None):
    """q: routed experts, qs: shared expert (or None), both as moe_quantize_experts_mxfp8 gives."""
    qs = qs or {}
    _check("moe_forward_mxfp8", lib().moe_forward_mxfp8(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(q["W13q"], U8, "W13q"), _ptr(q["W13sf"], U8, "W13sf"), _ptr(q["W2q"], U8, "W2q"),
        _ptr(q["W2sf"], U8, "W2sf"), _ptr(qs.get("W13q"), U8, "W13s_q"),
        _ptr(qs.get("W13sf"), U8, "W13s_sf"), _ptr(qs.get("W2q"), U8, "W2s_q"),
        _ptr(qs.get("W2sf"), U8, "W2s_sf"), _ptr(out, F32, "out"),
        _ptr(logits_out, F32, "logits_out"), _ptr(topk_idx_out, I32, "topk_idx_out"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel(), _stream(stream)))
    return out


def moe_quantize_experts_nvfp4(shape, W1, W3, W2, stream=None) -> dict:
    """NVFP4 experts from bf16 ones: dict(W13q, W13sf, W13gs, W2q, W2sf, W2gs): packed
    E2M1 codes (uint8, two per byte), flat E4M3 scale atoms and fp32 global scales [E]."""
    E, d_ff, d = shape.E, shape.d_ff, shape.d
    dev = W1.device
    q = dict(W13q=torch.empty(E, 2 * d_ff, d // 2, dtype=U8, device=dev),
             W13sf=torch.empty(E * 2 * d_ff * d // 16, dtype=U8, device=dev),
             W13gs=torch.empty(E, dtype=F32, device=dev),
             W2q=torch.empty(E, d, d_ff // 2, dtype=U8, device=dev),
             W2sf=torch.empty(E * d * d_ff // 16, dtype=U8, device=dev),
             W2gs=torch.empty(E, dtype=F32, device=dev))
    _check("moe_quantize_experts_nvfp4", lib().moe_quantize_experts_nvfp4(
        ctypes.byref(shape), _ptr(W1, BF16, "W1"), _ptr(W3, BF16, "W3"), _ptr(W2, BF16, "W2"),
        _ptr(q["W13q"], U8, "W13q"), _ptr(q["W13sf"], U8, "W13sf"), _ptr(q["W13gs"], F32, "W13gs"),
        _ptr(q["W2q"], U8, "W2q"), _ptr(q["W2sf"], U8, "W2sf"), _ptr(q["W2gs"], F32, "W2gs"),
        _stream(stream)))
    return q


def moe_forward_nvfp4(shape, x, Wg, bias, q, qs, x_gs, h_gs, out, logits_out, topk_idx_out,
                      status, ws, stream=None):
    """q: routed experts, qs: shared expert (or None), both as moe_quantize_experts_nvfp4
    gives; x_gs, h_gs: the activations' global encode scales."""
    qs = qs or {}
    _check("moe_forward_nvfp4", lib().moe_forward_nvfp4(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(q["W13q"], U8, "W13q"), _ptr(q["W13sf"], U8, "W13sf"), _ptr(q["W13gs"], F32, "W13gs"),
        _ptr(q["W2q"], U8, "W2q"), _ptr(q["W2sf"], U8, "W2sf"), _ptr(q["W2gs"], F32, "W2gs"),
        _ptr(qs.get("W13q"), U8, "W13s_q"), _ptr(qs.get("W13sf"), U8, "W13s_sf"),
        _ptr(qs.get("W13gs"), F32, "W13s_gs"), _ptr(qs.get("W2q"), U8, "W2s_q"),
        _ptr(qs.get("W2sf"), U8, "W2s_sf"), _ptr(qs.get("W2gs"), F32, "W2s_gs"),
        float(x_gs), float(h_gs), _ptr(out, F32, "out"), _ptr(logits_out, F32, "logits_out"),
        _ptr(topk_idx_out, I32, "topk_idx_out"), _ptr(status, U32, "status"),
        _ptr(ws, name="ws"), ws.numel(), _stream(stream)))
    return out


def moe_expert_ffn(shape, x_perm, expert_offsets, W13, W2, perm_token, slot_pos, topk_w, y_perm,
                   out, status, ws, stream=None):
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        ctypes.byref(shape), _ptr(x_perm, BF16, "x_perm"),
        _ptr(expert_offsets, I32, "expert_offsets"), _ptr(W13, BF16, "W13"), _ptr(W2, BF16, "W2"),
        _ptr(perm_token, I32, "perm_token"), _ptr(slot_pos, I32, "slot_pos"),
        _ptr(topk_w, F32, "topk_w"), _ptr(y_perm, F32, "y_perm"), _ptr(out, F32, "out"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel(), _stream(stream)))


def moe_combine(shape, y_perm, slot_pos, topk_w, shared_out, out, stream=None):
    _check("moe_combine", lib().moe_combine(
        ctypes.byref(shape), _ptr(y_perm, F32, "y_perm"), _ptr(slot_pos, I32, "slot_pos"),
        _ptr(topk_w, F32, "topk_w"), _ptr(shared_out, F32, "shared_out"), _ptr(out, F32, "out"),
        _stream(stream)))


def moe_forward(shape, x, Wg, bias, W13, W2, W13_shared, W2_shared, out, logits_out=None,
                topk_idx_out=None, status=None, ws=None, stream=None):
    _check("moe_forward", lib().moe_forward(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(W13, BF16, "W13"), _ptr(W2, BF16, "W2"), _ptr(W13_shared, BF16, "W13_shared"),
        _ptr(W2_shared, BF16, "W2_shared"), _ptr(out, F32, "out"),
        _ptr(logits_out, F32, "logits_out"), _ptr(topk_idx_out, I32, "topk_idx_out"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel() if ws is not None else 0,
        _stream(stream)))


def moe_forward_host(shape, x_host, Wg, bias, W13, W2, W13_shared, W2_shared, out_host, status,
                     ws, stream=None):
    _check("moe_forward_host", lib().moe_forward_host(
        ctypes.byref(shape), _host_ptr(x_host, BF16, "x_host"), _ptr(Wg, BF16, "Wg"),
        _ptr(bias, F32, "bias"), _ptr(W13, BF16, "W13"), _ptr(W2, BF16, "W2"),
        _ptr(W13_shared, BF16, "W13_shared"), _ptr(W2_shared, BF16, "W2_shared"),
        _host_ptr(out_host, F32, "out_host"), _ptr(status, U32, "status"), _ptr(ws, name="ws"),
        ws.numel(), _stream(stream)))


# ---------------------------------------------------------------- convenience

class MoeLayer:
    """Device-resident weights (packed once) plus a workspace; forward() runs
    the whole layer through moe_forward on the current stream."""

    def __init__(self, inp: dict, flags: int = 0, T_max: int | None = None):
        w = inp["workload"]
        self.workload = w
        self.flags = flags
        dev = inp["x"].device
        self.Wg = inp["wg"].contiguous()
        self.bias = None if inp.get("bias") is None else inp["bias"].to(dev, torch.float32).contiguous()
        s = shape_of(w, flags)
        self.W13 = moe_pack_w13(s, inp["W1"].contiguous(), inp["W3"].contiguous())
        self.W2 = inp["W2"].contiguous()
        self.W13s = self.W2s = None
        if w.d_ff_shared:
            ss = make_shape(w.T, w.d, w.d_ff_shared, 1, 1)
            self.W13s = moe_pack_w13(ss, inp["W1s"].contiguous()[None], inp["W3s"].contiguous()[None])[0]
            self.W2s = inp["W2s"].contiguous()
        self.T_max = T_max or w.T
        self.ws = alloc_workspace(shape_of(w, flags, T=self.T_max), dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def shape(self, T, flags=None):
        return shape_of(self.workload, self.flags if flags is None else flags, T=T)

    def forward(self, x, out=None, logits_out=None, topk_idx_out=None, flags=None, stream=None):
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError("T exceeds the workspace's T_max")
        if out is None:
            out = torch.empty(T, self.workload.d, dtype=torch.float32, device=x.device)
        moe_forward(self.shape(T, flags), x, self.Wg, self.bias, self.W13, self.W2, self.W13s,
                    self.W2s, out, logits_out, topk_idx_out, self.status, self.ws, stream)
        return out


def sf_atoms_to_rows(sf, rows: int, K: int):
    """Scale bytes in the atom order -> [rows, K/32] row-major (numpy or torch)."""
    a = sf.reshape(rows // 128, K // 128, 32, 4, 4)     # [tile, group, m%32, m/32, block]
    a = a.permute(0, 3, 2, 1, 4) if isinstance(a, torch.Tensor) else a.transpose(0, 3, 2, 1, 4)
    return a.reshape(rows, K // 32)


def moe_pack_backward(shape, W13, W2, stream=None):
    """Transposed expert weights for moe_backward: (W13T [E, d, 2 d_ff], W2T [E, d_ff, d])."""
    E, d_ff, d = shape.E, shape.d_ff, shape.d
    W13T = torch.empty(E, d, 2 * d_ff, dtype=BF16, device=W13.device)
    W2T = torch.empty(E, d_ff, d, dtype=BF16, device=W13.device)
    _check("moe_pack_backward", lib().moe_pack_backward(
        ctypes.byref(shape), _ptr(W13, BF16, "W13"), _ptr(W2, BF16, "W2"), _ptr(W13T, BF16, "W13T"),
        _ptr(W2T, BF16, "W2T"), _stream(stream)))
    return W13T, W2T


def moe_backward(shape, x, Wg, bias, W13, W13T, W2T, dout, status, ws, want_dlogits=False,
                 shared=None, stream=None) -> dict:
    """Gradients of sum(out * dout): dict(dx, dW13 (packed order), dW2, dWg, dbias[, dlogits]
    [, dW13s, dW2s]). shared = (W13s [2 dfs, d], W13sT, W2sT) when d_ff_shared > 0."""
    T, d, d_ff, E, dfs = shape.T, shape.d, shape.d_ff, shape.E, shape.d_ff_shared
    dev = x.device
    g = dict(dx=torch.empty(T, d, dtype=F32, device=dev),
             dW13=torch.empty(E, 2 * d_ff, d, dtype=F32, device=dev),
             dW2=torch.empty(E, d, d_ff, dtype=F32, device=dev),
             dWg=torch.empty(E, d, dtype=F32, device=dev),
             dbias=torch.empty(E, dtype=F32, device=dev))
    if want_dlogits:
        g["dlogits"] = torch.empty(T, E, dtype=F32, device=dev)
    W13s = W13sT = W2sT = None
    if dfs:
        W13s, W13sT, W2sT = shared
        g["dW13s"] = torch.empty(2 * dfs, d, dtype=F32, device=dev)
        g["dW2s"] = torch.empty(d, dfs, dtype=F32, device=dev)
    _check("moe_backward", lib().moe_backward(
        ctypes.byref(shape), _ptr(x, BF16, "x"), _ptr(Wg, BF16, "Wg"), _ptr(bias, F32, "bias"),
        _ptr(W13, BF16, "W13"), _ptr(W13T, BF16, "W13T"), _ptr(W2T, BF16, "W2T"),
        _ptr(W13s, BF16, "W13s"), _ptr(W13sT, BF16, "W13sT"), _ptr(W2sT, BF16, "W2sT"),
        _ptr(dout, F32, "dout"), _ptr(g["dx"], F32, "dx"), _ptr(g["dW13"], F32, "dW13"),
        _ptr(g["dW2"], F32, "dW2"), _ptr(g.get("dW13s"), F32, "dW13s"),
        _ptr(g.get("dW2s"), F32, "dW2s"), _ptr(g["dWg"], F32, "dWg"),
        _ptr(g["dbias"], F32, "dbias"), _ptr(g.get("dlogits"), F32, "dlogits"),
        _ptr(status, U32, "status"), _ptr(ws, name="ws"), ws.numel(), _stream(stream)))
    return g


class MoeLayerMx:
    """The layer with MXFP8 experts: quantizes the bf16 experts of `inp` once
    (moe_quantize_experts_mxfp8) and runs moe_forward_mxfp8."""

    def __init__(self, inp: dict, flags: int = 0, T_max: int | None = None):
        w = inp["workload"]
        self.workload = w
        self.flags = flags | MOE_FLAG_MXFP8
        dev = inp["x"].device
        self.Wg = inp["wg"].contiguous()
        self.bias = None if inp.get("bias") is None else inp["bias"].to(dev, torch.float32).contiguous()
        s = shape_of(w, self.flags)
        self.q = moe_quantize_experts_mxfp8(s, inp["W1"].contiguous(), inp["W3"].contiguous(),
                                            inp["W2"].contiguous())
        self.qs = None
        if w.d_ff_shared:
            ss = make_shape(w.T, w.d, w.d_ff_shared, 1, 1)
            self.qs = moe_quantize_experts_mxfp8(ss, inp["W1s"].contiguous()[None],
                                                 inp["W3s"].contiguous()[None],
                                                 inp["W2s"].contiguous()[None])
        self.T_max = T_max or w.T
        self.ws = alloc_workspace(shape_of(w, self.flags, T=self.T_max), dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def shape(self, T, flags=None):
        return shape_of(self.workload, self.flags if flags is None else flags | MOE_FLAG_MXFP8, T=T)

    def forward(self, x, out=None, logits_out=None, topk_idx_out=None, flags=None, stream=None):
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError("T exceeds the workspace's T_max")
        if out is None:
            out = torch.empty(T, self.workload.d, dtype=torch.float32, device=x.device)
        return moe_forward_mxfp8(self.shape(T, flags), x, self.Wg, self.bias, self.q, self.qs, out,
                                 logits_out, topk_idx_out, self.status, self.ws, stream)


class MoeLayerNv4:
    """The layer with NVFP4 experts: quantizes the bf16 experts of `inp` once
    (moe_quantize_experts_nvfp4) and runs moe_forward_nvfp4 with the
    activations' global encode scales x_gs and h_gs (calibration constants;
    1.0 leaves the E4M3 block scales to cover the values alone)."""

    def __init__(self, inp: dict, flags: int = 0, T_max: int | None = None, x_gs: float = 1.0,
                 h_gs: float = 1.0):
        w = inp["workload"]
        self.workload = w
        self.flags = flags | MOE_FLAG_NVFP4
        dev = inp["x"].device
        self.Wg = inp["wg"].contiguous()
        self.bias = None if inp.get("bias") is None else inp["bias"].to(dev, torch.float32).contiguous()
        self.x_gs, self.h_gs = float(x_gs), float(h_gs)
        s = shape_of(w, self.flags)
        self.q = moe_quantize_experts_nvfp4(s, inp["W1"].contiguous(), inp["W3"].contiguous(),
                                            inp["W2"].contiguous())
        self.qs = None
        if w.d_ff_shared:
            ss = make_shape(w.T, w.d, w.d_ff_shared, 1, 1)
            self.qs = moe_quantize_experts_nvfp4(ss, inp["W1s"].contiguous()[None],
                                                 inp["W3s"].contiguous()[None],
                                                 inp["W2s"].contiguous()[None])
        self.T_max = T_max or w.T
        self.ws = alloc_workspace(shape_of(w, self.flags, T=self.T_max), dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def shape(self, T, flags=None):
        return shape_of(self.workload, self.flags if flags is None else flags | MOE_FLAG_NVFP4, T=T)

    def forward(self, x, out=None, logits_out=None, topk_idx_out=None, flags=None, stream=None):
        T = x.shape[0]
        if T > self.T_max:
            raise ValueError("T exceeds the workspace's T_max")
        if out is None:
            out = torch.empty(T, self.workload.d, dtype=torch.float32, device=x.device)
        return moe_forward_nvfp4(self.shape(T, flags), x, self.Wg, self.bias, self.q, self.qs,
                                 self.x_gs, self.h_gs, out, logits_out, topk_idx_out, self.status,
                                 self.ws, stream)


# ---------------------------------------------------------------- instrumentation

def moe_kernel_launches() -> int:
    return int(lib().moe_kernel_launches())


def moe_profile_enable(on: bool = True):
    _check("moe_profile_enable", lib().moe_profile_enable(int(bool(on))))


def moe_profile_read() -> dict:
    """{stage: (total ms, calls)} since the last read (waits for the events)."""
    import numpy as np
    n = len(STAGES)
    ms = np.zeros(n, np.float64)
    calls = np.zeros(n, np.int64)
    _check("moe_profile_read", lib().moe_profile_read(ms.ctypes.data, calls.ctypes.data, n))
    return {STAGES[i]: (float(ms[i]), int(calls[i])) for i in range(n) if calls[i]}
