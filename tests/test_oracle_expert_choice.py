"""Pins of the oracle's expert-choice routing ("MoE Model Architectures",
"Design Patterns", "Pattern 3: Expert Choice Routing") to things other than
itself: brute-force sorting, ties, closed special cases, torch's softmax, and a
dense every-expert evaluation with the selection mask (CPU only)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_mixture_experts_17_b200 import inputs as I


def _brute(S, C):
    T, E = S.shape
    K = min(C, T)
    toks = []
    for e in range(E):
        order = sorted(range(T), key=lambda t: (-float(S[t, e]), t))[:K]
        toks.append(sorted(order))
    return np.array(toks, np.int32).reshape(E, K)


@pytest.mark.parametrize("T,E,C,kind", [(50, 4, 10, "cont"), (64, 8, 16, "ties"), (7, 3, 20, "cont"),
                                        (200, 16, 25, "ties"), (33, 1, 5, "cont")])
def test_expert_choice_brute_force(orc, T, E, C, kind):
    rng = np.random.default_rng(T + E + C)
    if kind == "cont":
        S = rng.random((T, E)).astype(np.float32)
    else:
        S = rng.choice(np.array([0.1, 0.25, 0.5, 0.0], np.float32), size=(T, E))
    tok, w = orc.expert_choice(S, C)
    assert (tok == _brute(S, C)).all()
    for e in range(E):
        assert (w[e] == S[tok[e], e].astype(np.float64)).all()
        assert (np.diff(tok[e]) > 0).all()          # ascending token order


def test_expert_choice_takes_all_when_capacity_exceeds_tokens(orc):
    S = np.random.default_rng(0).random((6, 3)).astype(np.float32)
    tok, _ = orc.expert_choice(S, 100)
    assert (tok == np.arange(6)).all()


def test_softmax_rows_matches_torch(orc):
    L = (np.random.default_rng(1).standard_normal((40, 17)) * 3).astype(np.float32)
    S = orc.softmax_rows(L)
    ref = F.softmax(torch.from_numpy(L).double(), dim=1).numpy()
    np.testing.assert_allclose(S, ref, rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(S.sum(1), 1.0, rtol=0, atol=1e-14)


def test_expert_choice_layer_vs_dense_masked(orc):
    """out[t] = sum_e m[t,e] S[t,e] FFN_e(x_t), every expert on every token (fp64)."""
    w = I.Workload("ec", T=40, d=32, d_ff=48, E=6, k=2, d_ff_shared=32, zipf_s=1.0)
    inp = I.oracle_arrays(I.make_inputs(w, "cpu", seed=4))
    _, L32 = orc.router_logits(inp["x"], inp["wg"], inp["bias"])
    S32 = orc.softmax_rows(L32).astype(np.float32)
    C = 9
    res = orc.expert_choice_layer(inp, S32, C, h_bf16=False)
    cv = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double()
    x, W1, W3, W2 = cv(inp["x"]), cv(inp["W1"]), cv(inp["W3"]), cv(inp["W2"])
    m = torch.zeros(w.T, w.E, dtype=torch.float64)
    for e in range(w.E):
        m[_brute(S32, C)[e], e] = 1.0
    out = torch.zeros(w.T, w.d, dtype=torch.float64)
    for e in range(w.E):
        y = (F.silu(x @ W1[e].T) * (x @ W3[e].T)) @ W2[e].T
        out += (m[:, e] * torch.from_numpy(S32[:, e]).double())[:, None] * y
    W1s, W3s, W2s = cv(inp["W1s"]), cv(inp["W3s"]), cv(inp["W2s"])
    out = (F.silu(x @ W1s.T) * (x @ W3s.T)) @ W2s.T + out
    np.testing.assert_allclose(res["out"], out.numpy(), rtol=1e-10, atol=1e-12)
    # every expert took exactly C tokens; a token may be taken by 0..E experts
    assert res["tokens"].shape == (w.E, C)
