"""MoE backward pass on the GPU vs the oracle's fp64 backward, through the C ABI.

The oracle is given the routing the GPU takes: the oracle's own top-k and
dispatch on the GPU's fp32 logits (identical decisions). Every gradient is
checked three ways, so that one wrong expert block or a few wrong token rows
cannot hide inside a small whole-tensor error:

- whole tensor: relative Frobenius error within 2e-2 for the expert gradients
  (dx, dW1, dW3, dW2 and the shared expert's), 5e-2 for the router gradients
  (dWg, dbias, dlogits), which difference terms of similar size;
- element by element: |got - ref| <= 2e-2 * max|ref| (expert gradients) or
  5e-2 * max|ref| (router gradients);
- block by block: each expert's dW1 / dW3 / dW2 block and each token's dx row
  within 3e-2 relative Frobenius error, plus a floor of 1e-3 times the
  tensor's root-mean-square block norm for blocks that are (near) zero.

The bounds come from the arithmetic: every GEMM operand is rounded once to
bf16 (relative error <= 2^-9 per operand) and accumulated in fp32, and the
SwiGLU backward reads gate and up saved in bf16, so an element carries a
relative error of a few 2^-9 of its own dot product's scale.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import Buffers, small_workload

pytestmark = pytest.mark.gpu
EXPERT_REL = 2e-2
ROUTER_REL = 5e-2
EXPERT_ELEM = 2e-2     # of max|ref|
ROUTER_ELEM = 5e-2     # of max|ref|
BLOCK_REL = 3e-2       # per expert block / per token row
BLOCK_FLOOR = 1e-3     # of the RMS block norm


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _np(a):
    return a.double().cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a, np.float64)


def check_grad(name, got, ref, rel_fro, elem, blocks=False, stats=None):
    """Whole-tensor, element-wise and (blocks=True: along axis 0) per-block
    bounds; returns the measured figures."""
    g, r = _np(got), np.asarray(ref, np.float64)
    assert g.shape == r.shape, (name, g.shape, r.shape)
    d = g - r
    fro = float(np.linalg.norm(d) / max(np.linalg.norm(r), 1e-30))
    rmax = float(np.abs(r).max()) if r.size else 0.0
    el = float(np.abs(d).max() / max(rmax, 1e-30)) if r.size else 0.0
    out = {"fro": fro, "elem": el}
    assert fro <= rel_fro, (name, out)
    assert el <= elem, (name, out)
    if blocks and r.shape[0] > 0:
        dn = np.linalg.norm(d.reshape(r.shape[0], -1), axis=1)
        rn = np.linalg.norm(r.reshape(r.shape[0], -1), axis=1)
        floor = BLOCK_FLOOR * float(np.sqrt(np.mean(rn ** 2)))
        worst = float(np.max(dn / (BLOCK_REL * rn + floor)))
        out["block_worst_vs_bound"] = worst
        out["block_rel_max"] = float(np.max(dn[rn > 0] / rn[rn > 0])) if (rn > 0).any() else 0.0
        bad = np.nonzero(dn > BLOCK_REL * rn + floor)[0]
        assert len(bad) == 0, (name, "blocks beyond bound", bad[:8].tolist(), out)
    if stats is not None:
        stats[name] = out
    return out


def _unpack13(dW13, d_ff):
    E, _, d = dW13.shape
    b = dW13.reshape(E, d_ff // 128, 2, 128, d)
    return b[:, :, 0].reshape(E, d_ff, d), b[:, :, 1].reshape(E, d_ff, d)


BWD_CASES = [
    # name, T, d, d_ff, E, k, capacity, zipf
    ("basic", 300, 256, 256, 8, 2, 0, 0.0),
    ("ragged_skewed", 700, 256, 384, 8, 2, 0, 1.0),
    ("capacity_drops", 500, 256, 256, 16, 4, 60, 1.2),
    ("many_experts", 400, 512, 128, 64, 6, 0, 1.1),
    ("small_T", 10, 256, 256, 4, 2, 0, 0.0),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: c[0])
def test_backward_parity(case):
    name, T, d, d_ff, E, k, C, zipf = case
    w = small_workload(name, T, d, d_ff, E, k, capacity=C, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + d + E)
    s = M.shape_of(w, M.MOE_FLAG_BACKWARD)
    ws = M.alloc_workspace(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    W13T, W2T = M.moe_pack_backward(s, W13, inp["W2"])
    g = torch.Generator("cuda").manual_seed(T)
    dout = torch.randn(T, d, generator=g, device="cuda")
    grads = M.moe_backward(s, inp["x"], inp["wg"], inp["bias"], W13, W13T, W2T, dout, status, ws,
                           want_dlogits=True)
    # the logits the GPU routes on (same kernels as the forward and the backward)
    b = Buffers(w)
    M.moe_route(b.shape, inp["x"], inp["wg"], inp["bias"], b.logits, b.idx, b.w, b.status, b.ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and int(b.status.item()) == 0
    idx_o, w_o = O.route(b.logits.cpu().numpy(), k)
    disp = O.dispatch(idx_o, E, C)
    if C:
        assert (disp["slot_pos"] < 0).any()
    ref = O.moe_backward(I.oracle_arrays(inp), idx_o, w_o, disp["slot_pos"], dout.cpu().numpy())
    dW1, dW3 = _unpack13(grads["dW13"].cpu().numpy(), d_ff)
    st = {}
    for key, got, blk in (("dx", grads["dx"], True), ("dW1", dW1, True), ("dW3", dW3, True),
                          ("dW2", grads["dW2"], True)):
        check_grad(key, got, ref[key], EXPERT_REL, EXPERT_ELEM, blocks=blk, stats=st)
    for key in ("dWg", "dbias", "dlogits"):
        check_grad(key, grads[key], ref[key], ROUTER_REL, ROUTER_ELEM, stats=st)
    print(f"backward {name}: " + ", ".join(f"{k} {v}" for k, v in st.items()))
    # experts that received no rows have exactly zero weight gradients
    counts = np.bincount(idx_o[disp["slot_pos"] >= 0], minlength=E)
    for e in np.nonzero(counts == 0)[0]:
        assert (grads["dW2"][e] == 0).all() and (grads["dW13"][e] == 0).all()


def test_backward_weight_grads_repeatable():
    """The weight gradients are plain per-expert GEMMs: bitwise repeatable."""
    w = small_workload("rep", 600, 256, 256, 8, 2, zipf_s=1.0)
    inp = I.make_inputs(w, "cuda", seed=11)
    s = M.shape_of(w, M.MOE_FLAG_BACKWARD)
    ws = M.alloc_workspace(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    W13T, W2T = M.moe_pack_backward(s, W13, inp["W2"])
    dout = torch.randn(600, 256, device="cuda")
    a = M.moe_backward(s, inp["x"], inp["wg"], inp["bias"], W13, W13T, W2T, dout, status, ws)
    b = M.moe_backward(s, inp["x"], inp["wg"], inp["bias"], W13, W13T, W2T, dout, status, ws)
    torch.cuda.synchronize()
    for key in ("dW13", "dW2", "dWg", "dbias"):
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("T,d,d_ff,E,k,dfs,C", [(300, 256, 256, 8, 2, 256, 0),
                                                (90, 512, 128, 16, 4, 384, 0),
                                                (400, 256, 256, 16, 4, 256, 80)])
def test_backward_shared_expert(T, d, d_ff, E, k, dfs, C):
    """With a shared expert ([DSK]: weight 1 on every token): its gradients and
    its share of dx against the oracle, uncapped and with capacity drops."""
    w = small_workload("bsh", T, d, d_ff, E, k, capacity=C, d_ff_shared=dfs, zipf_s=1.0)
    inp = I.make_inputs(w, "cuda", seed=T + dfs)
    s = M.shape_of(w, M.MOE_FLAG_BACKWARD)
    ws = M.alloc_workspace(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    W13T, W2T = M.moe_pack_backward(s, W13, inp["W2"])
    ss = M.make_shape(T, d, dfs, 1, 1)
    W13s = M.moe_pack_w13(ss, inp["W1s"][None].contiguous(), inp["W3s"][None].contiguous())
    W13sT, W2sT = M.moe_pack_backward(ss, W13s, inp["W2s"][None].contiguous())
    dout = torch.randn(T, d, generator=torch.Generator("cuda").manual_seed(3), device="cuda")
    grads = M.moe_backward(s, inp["x"], inp["wg"], inp["bias"], W13, W13T, W2T, dout, status, ws,
                           shared=(W13s[0], W13sT[0], W2sT[0]))
    b = Buffers(w)
    M.moe_route(b.shape, inp["x"], inp["wg"], inp["bias"], b.logits, b.idx, b.w, b.status, b.ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx_o, w_o = O.route(b.logits.cpu().numpy(), k)
    disp = O.dispatch(idx_o, E, C)
    if C:
        assert (disp["slot_pos"] < 0).any()
    ref = O.moe_backward(I.oracle_arrays(inp), idx_o, w_o, disp["slot_pos"], dout.cpu().numpy())
    dW1s, dW3s = _unpack13(grads["dW13s"].cpu().numpy()[None], dfs)
    dW1, dW3 = _unpack13(grads["dW13"].cpu().numpy(), d_ff)
    st = {}
    for key, got, blk in (("dx", grads["dx"], True), ("dW1s", dW1s[0], False),
                          ("dW3s", dW3s[0], False), ("dW2s", grads["dW2s"], False),
                          ("dW1", dW1, True), ("dW3", dW3, True), ("dW2", grads["dW2"], True)):
        check_grad(key, got, ref[key], EXPERT_REL, EXPERT_ELEM, blocks=blk, stats=st)
    for key in ("dWg", "dbias"):
        check_grad(key, grads[key], ref[key], ROUTER_REL, ROUTER_ELEM, stats=st)
    print(f"backward shared T={T} dfs={dfs}: " + ", ".join(f"{k} {v}" for k, v in st.items()))
