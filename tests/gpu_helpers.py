"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

# Layer tolerance (bf16 weights, fp32 accumulation, bf16 SwiGLU product).
MAX_ABS = 2e-2
REL_FRO = 1e-2
# Router logits vs fp64: fp32 accumulation of d bf16 products.
LOGIT_ABS = 1e-3
# Routing weights vs fp64 (fp32 exp and division on identical fp32 logits).
W_ABS = 1e-6


def layer_errors(got, ref):
    g = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    d = g - r
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(r), 1e-30)) if d.size else 0.0
    return max_abs, rel


def assert_layer_close(got, ref, what=""):
    max_abs, rel = layer_errors(got, ref)
    assert max_abs <= MAX_ABS and rel <= REL_FRO, f"{what}: max_abs={max_abs:.3e} rel_fro={rel:.3e}"
    return max_abs, rel


def small_workload(name, T, d, d_ff, E, k, capacity=0, d_ff_shared=0, zipf_s=0.0):
    return I.Workload(name, T=T, d=d, d_ff=d_ff, E=E, k=k, capacity=capacity,
                      d_ff_shared=d_ff_shared, zipf_s=zipf_s)


def u16(t):
    return I.to_numpy_u16(t)


class Buffers:
    """Device outputs of the step-by-step pipeline for one shape."""

    def __init__(self, w, dev="cuda", flags=0):
        T, E, k, d = w.T, w.E, w.k, w.d
        self.shape = M.shape_of(w, flags)
        self.ws = M.alloc_workspace(self.shape, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        z = lambda *s, dt=torch.int32: torch.full(s, -7, dtype=dt, device=dev)
        self.logits = torch.empty(T, E, dtype=torch.float32, device=dev)
        self.idx = z(T, k)
        self.w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = z(E)
        self.offsets = z(E + 1)
        self.slot_pos = z(T, k)
        self.perm_token = z(max(T * k, 1))
        self.n_kept = z(1)
        self.x_perm = torch.zeros(max(T * k, 1), d, dtype=torch.bfloat16, device=dev)
        self.y_perm = torch.zeros(max(T * k, 1), d, dtype=torch.float32, device=dev)
        self.out = torch.zeros(T, d, dtype=torch.float32, device=dev)


def pipeline_from_logits(inp, logits, flags=0, fused=True):
    """moe_route (logits given) -> moe_permute -> moe_expert_ffn [-> moe_combine]."""
    w = inp["workload"]
    b = Buffers(w, flags=flags)
    b.logits.copy_(logits)
    s = b.shape
    M.moe_route(s, None, None, None, b.logits, b.idx, b.w, b.status, b.ws)
    M.moe_permute(s, b.idx, inp["x"], b.counts, b.offsets, b.slot_pos, b.perm_token, b.x_perm,
                  b.n_kept, b.status, b.ws)
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    shared = None
    if w.d_ff_shared:
        # the shared expert through the same calls: one group of all T rows, unweighted
        ss = M.make_shape(w.T, w.d, w.d_ff_shared, 1, 1)
        W13s = M.moe_pack_w13(ss, inp["W1s"][None].contiguous(), inp["W3s"][None].contiguous())
        offs = torch.tensor([0, w.T], dtype=torch.int32, device=inp["x"].device)
        shared = torch.empty(w.T, w.d, dtype=torch.float32, device=inp["x"].device)
        M.moe_expert_ffn(ss, inp["x"], offs, W13s, inp["W2s"][None].contiguous(), None, None, None,
                         shared, None, b.status, M.alloc_workspace(ss, inp["x"].device))
    if fused:
        if shared is not None:
            b.out.copy_(shared)
        else:
            b.out.zero_()
        M.moe_expert_ffn(s, b.x_perm, b.offsets, W13, inp["W2"], b.perm_token, b.slot_pos, b.w,
                         None, b.out, b.status, b.ws)
    else:
        M.moe_expert_ffn(s, b.x_perm, b.offsets, W13, inp["W2"], None, None, None, b.y_perm, None,
                         b.status, b.ws)
        M.moe_combine(s, b.y_perm, b.slot_pos, b.w, shared, b.out)
    torch.cuda.synchronize()
    return b


def oracle_tokens_subset(inp, idx, w, slot_pos, tokens, h_bf16=True, mx=False):
    """Oracle layer rows for `tokens`, copying to the host only the experts
    those tokens keep (the large configurations do not fit on the host whole)."""
    tokens = np.asarray(tokens, np.int32)
    idx_t, w_t, sp_t = idx[tokens], w[tokens], slot_pos[tokens]
    need = np.unique(idx_t[sp_t >= 0])
    remap = np.zeros(inp["workload"].E, np.int32)
    remap[need] = np.arange(len(need), dtype=np.int32)
    sel = torch.from_numpy(need.astype(np.int64)).to(inp["W1"].device)
    W1 = u16(inp["W1"].index_select(0, sel))
    W3 = u16(inp["W3"].index_select(0, sel))
    W2 = u16(inp["W2"].index_select(0, sel))
    x = u16(inp["x"][torch.from_numpy(tokens.astype(np.int64)).to(inp["x"].device)])
    kw = {}
    if inp.get("W1s") is not None:
        kw = dict(W1s=u16(inp["W1s"]), W3s=u16(inp["W3s"]), W2s=u16(inp["W2s"]))
    idx_r = np.where(sp_t >= 0, remap[np.clip(idx_t, 0, None)], 0).astype(np.int32)
    # dropped slots keep distinct placeholder ids only if the expert count allows; the
    # oracle skips them (slot_pos < 0) after checking the id range
    return O.moe_tokens(x, W1, W3, W2, idx_r, w_t, sp_t, np.arange(len(tokens)), h_bf16=h_bf16,
                        mx=mx, **kw)


def sample_tokens(T, disp, n_random=24, seed=0, extra=()):
    """A token sample: random tokens, the first and last token, the first and
    last rows of the largest and smallest non-empty experts' segments, and
    (with capacity) some tokens that lost an assignment."""
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    s.update([0, T - 1])
    off = disp["offsets"]
    pt = disp["perm_token"]
    kept = np.diff(off)
    nz = np.nonzero(kept)[0]
    if len(nz):
        for e in (nz[np.argmax(kept[nz])], nz[np.argmin(kept[nz])]):
            s.add(int(pt[off[e]]))
            s.add(int(pt[off[e + 1] - 1]))
    dropped = np.nonzero((disp["slot_pos"] < 0).any(1))[0]
    s.update(dropped[:4].tolist())
    s.update(extra)
    return np.array(sorted(s), np.int32)
