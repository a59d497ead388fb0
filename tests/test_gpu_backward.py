"""MoE backward pass on the GPU vs the oracle's fp64 backward, through the C ABI.

The oracle is given the routing the GPU takes: the oracle's own top-k and
dispatch on the GPU's fp32 logits (identical decisions). Every gradient is
compared in relative Frobenius norm: the expert gradients (dx, dW1, dW3, dW2)
within 2e-2 (bf16 operands, fp32 accumulation), the router gradients (dWg,
dbias, dlogits) within 5e-2 (they difference terms of similar size).
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _rel(got, ref):
    g = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))


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
    errs = {
        "dx": _rel(grads["dx"], ref["dx"]),
        "dW1": _rel(dW1, ref["dW1"]),
        "dW3": _rel(dW3, ref["dW3"]),
        "dW2": _rel(grads["dW2"], ref["dW2"]),
        "dWg": _rel(grads["dWg"], ref["dWg"]),
        "dbias": _rel(grads["dbias"], ref["dbias"]),
        "dlogits": _rel(grads["dlogits"], ref["dlogits"]),
    }
    for key in ("dx", "dW1", "dW3", "dW2"):
        assert errs[key] <= EXPERT_REL, (name, errs)
    for key in ("dWg", "dbias", "dlogits"):
        assert errs[key] <= ROUTER_REL, (name, errs)
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


@pytest.mark.parametrize("T,d,d_ff,E,k,dfs", [(300, 256, 256, 8, 2, 256), (90, 512, 128, 16, 4, 384)])
def test_backward_shared_expert(T, d, d_ff, E, k, dfs):
    """With a shared expert ([DSK]: weight 1 on every token): its gradients and
    its share of dx against the oracle."""
    w = small_workload("bsh", T, d, d_ff, E, k, d_ff_shared=dfs, zipf_s=1.0)
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
    disp = O.dispatch(idx_o, E, 0)
    ref = O.moe_backward(I.oracle_arrays(inp), idx_o, w_o, disp["slot_pos"], dout.cpu().numpy())
    dW1s, dW3s = _unpack13(grads["dW13s"].cpu().numpy()[None], dfs)
    errs = {"dx": _rel(grads["dx"], ref["dx"]), "dW1s": _rel(dW1s[0], ref["dW1s"]),
            "dW3s": _rel(dW3s[0], ref["dW3s"]), "dW2s": _rel(grads["dW2s"], ref["dW2s"]),
            "dW2": _rel(grads["dW2"], ref["dW2"]), "dWg": _rel(grads["dWg"], ref["dWg"])}
    for key in ("dx", "dW1s", "dW3s", "dW2s", "dW2"):
        assert errs[key] <= EXPERT_REL, errs
    assert errs["dWg"] <= ROUTER_REL, errs
