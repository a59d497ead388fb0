"""Pins of the oracle's backward pass (CPU only).

A plain numpy fp64 forward with the routing held fixed is first checked
against the oracle's own fp64 forward on the same bf16 inputs; central finite
differences of that forward then pin every gradient the oracle returns (x,
W_g, bias, W1, W3, W2 and the shared expert), including a capacity drop."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_17_b200 import inputs as I


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).double().numpy()


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _forward(P, idx, slot_pos):
    """fp64 layer with fixed top-k sets and drops; weights from the fp64 logits."""
    x, Wg, b = P["x"], P["wg"], P["bias"]
    T = x.shape[0]
    L = x @ Wg.T + b
    out = np.zeros_like(x)
    for t in range(T):
        sel = idx[t]
        p = np.exp(L[t, sel] - L[t, sel].max())
        w = p / p.sum()
        for j, e in enumerate(sel):
            if slot_pos[t, j] < 0:
                continue
            h = _silu(P["W1"][e] @ x[t]) * (P["W3"][e] @ x[t])
            out[t] += w[j] * (P["W2"][e] @ h)
        if "W1s" in P:
            out[t] += P["W2s"] @ (_silu(P["W1s"] @ x[t]) * (P["W3s"] @ x[t]))
    return out, L


def _setup(orc, shared, C, seed):
    w = I.Workload("bwd", T=6, d=16, d_ff=24, E=4, k=2, capacity=C,
                   d_ff_shared=16 if shared else 0, zipf_s=0.5)
    inp = I.oracle_arrays(I.make_inputs(w, "cpu", seed=seed))
    P = {key: _bf(inp[key]) for key in ("x", "wg", "W1", "W3", "W2") + (("W1s", "W3s", "W2s") if shared else ())}
    P["bias"] = np.asarray(inp["bias"], np.float64) if inp["bias"] is not None else np.zeros(w.E)
    inp["bias"] = P["bias"].astype(np.float32)
    _, L32 = orc.router_logits(inp["x"], inp["wg"], inp["bias"])
    idx, _ = orc.route(L32, w.k)
    disp = orc.dispatch(idx, w.E, C)
    return w, inp, P, idx, disp


@pytest.mark.parametrize("shared,C", [(True, 0), (False, 0), (True, 2)])
def test_numpy_forward_matches_oracle(orc, shared, C):
    w, inp, P, idx, disp = _setup(orc, shared, C, seed=3)
    out, L = _forward(P, idx, disp["slot_pos"])
    wts = np.stack([np.exp(L[t, idx[t]] - L[t, idx[t]].max()) for t in range(w.T)])
    wts /= wts.sum(1, keepdims=True)
    ref = orc.moe_tokens(inp["x"], inp["W1"], inp["W3"], inp["W2"], idx, wts, disp["slot_pos"],
                         np.arange(w.T, dtype=np.int32), h_bf16=False,
                         **({k: inp[k] for k in ("W1s", "W3s", "W2s")} if shared else {}))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("shared,C", [(True, 0), (False, 0), (True, 2)])
def test_backward_finite_differences(orc, shared, C):
    w, inp, P, idx, disp = _setup(orc, shared, C, seed=5)
    rng = np.random.default_rng(1)
    dout = rng.standard_normal((w.T, w.d)).astype(np.float32)
    out, L = _forward(P, idx, disp["slot_pos"])
    wts = np.stack([np.exp(L[t, idx[t]] - L[t, idx[t]].max()) for t in range(w.T)])
    wts /= wts.sum(1, keepdims=True)
    if C:
        assert (disp["slot_pos"] < 0).any()
    g = orc.moe_backward(inp, idx, wts, disp["slot_pos"], dout)

    def loss(PP):
        return float((_forward(PP, idx, disp["slot_pos"])[0] * dout.astype(np.float64)).sum())

    names = [("x", "dx"), ("wg", "dWg"), ("bias", "dbias"), ("W1", "dW1"), ("W3", "dW3"),
             ("W2", "dW2")] + ([("W1s", "dW1s"), ("W3s", "dW3s"), ("W2s", "dW2s")] if shared else [])
    eps = 1e-6
    for pname, gname in names:
        flat = P[pname].reshape(-1)
        for i in rng.choice(flat.size, size=min(12, flat.size), replace=False):
            Pp = {kk: v.copy() for kk, v in P.items()}
            Pm = {kk: v.copy() for kk, v in P.items()}
            Pp[pname].reshape(-1)[i] += eps
            Pm[pname].reshape(-1)[i] -= eps
            fd = (loss(Pp) - loss(Pm)) / (2 * eps)
            an = g[gname].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (pname, i, fd, an)
    # G is the gradient of the loss w.r.t. each kept assignment's weight: <dout, y>
    for t in range(w.T):
        for j in range(w.k):
            if disp["slot_pos"][t, j] < 0:
                assert g["G"][t, j] == 0.0
    # the router gradient of each token sums to zero (softmax over the chosen set)
    np.testing.assert_allclose(g["dlogits"].sum(1), 0.0, atol=1e-12)
