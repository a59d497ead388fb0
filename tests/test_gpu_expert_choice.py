"""Expert-choice routing ("MoE Model Architectures", "Design Patterns",
"Pattern 3: Expert Choice Routing") on the GPU vs the fp64 oracle, through the
C ABI.

The selection (which K = min(C, T) tokens each expert takes, in ascending
token order, and their weights) is compared bit for bit on identical fp32
scores; the softmax against the oracle's fp64 softmax of the same fp32 logits;
the layer output within max-abs 2e-2 and relative Frobenius 1e-2 against the
oracle evaluated on the GPU's own scores (so both sides select the same
tokens).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import LOGIT_ABS, assert_layer_close, small_workload, u16

pytestmark = pytest.mark.gpu
EC = M.MOE_FLAG_EXPERT_CHOICE
# fp32 exp and division vs the fp64 softmax of the same fp32 logits
S_ABS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _scores(T, E, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "continuous":
        S = rng.random((T, E)).astype(np.float32)
    elif kind == "ties":
        S = rng.choice(np.array([0.0, 0.125, 0.25, 0.5, 1.0], np.float32), size=(T, E))
    else:  # "flat": every score equal, so every choice is decided by token order
        S = np.full((T, E), 0.25, np.float32)
    return S


def _route(T, E, C, S=None, x=None, inp=None, flags=0):
    K = min(C, T)
    s = M.make_shape(T, 128 if inp is None else inp["workload"].d, 128, E, 1, C, 0, EC | flags)
    ws = M.alloc_workspace(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    logits = torch.full((T, E), -7.0, dtype=torch.float32, device="cuda")
    scores = torch.full((T, E), -7.0, dtype=torch.float32, device="cuda")
    if S is not None:
        scores.copy_(torch.from_numpy(S))
    tok = torch.full((E, K), -7, dtype=torch.int32, device="cuda")
    wt = torch.full((E, K), -7.0, dtype=torch.float32, device="cuda")
    if inp is None:
        M.moe_route_expert_choice(s, None, None, None, None, scores, tok, wt, status, ws)
    else:
        M.moe_route_expert_choice(s, inp["x"], inp["wg"], inp["bias"], logits, scores, tok, wt,
                                  status, ws)
    torch.cuda.synchronize()
    return dict(status=int(status.item()), logits=logits.cpu().numpy(),
                scores=scores.cpu().numpy(), tok=tok.cpu().numpy(), w=wt.cpu().numpy())


# ---------------------------------------------------------------- selection on identical scores

@pytest.mark.parametrize("T,E,C", [(1000, 8, 250), (1000, 8, 1), (1000, 1, 999), (300, 64, 37),
                                   (5000, 16, 625), (4099, 256, 129), (17, 4, 100),
                                   (2048, 32, 2048), (70000, 8, 17500)])
@pytest.mark.parametrize("kind", ["continuous", "ties", "flat"])
def test_selection_bitexact(T, E, C, kind):
    S = _scores(T, E, kind, seed=T + E + C)
    tok_o, w_o = O.expert_choice(S, C)
    r = _route(T, E, C, S=S)
    assert r["status"] == 0
    assert (r["tok"] == tok_o).all()
    # weights are the selected scores themselves, bit for bit
    assert (r["w"].astype(np.float64) == w_o).all()


def test_selection_nan_flagged():
    S = _scores(500, 8, "continuous", seed=3)
    S[123, 5] = np.nan
    r = _route(500, 8, 100, S=S)
    assert r["status"] == 1 << 5          # MOE_ERR_NONFINITE


# ---------------------------------------------------------------- router + softmax

@pytest.mark.parametrize("T,d,E,C,zipf", [(700, 256, 8, 175, 0.0), (300, 512, 64, 12, 1.0),
                                          (200, 7168, 256, 3, 1.1), (5, 4096, 8, 2, 0.0)])
def test_router_softmax_selection(T, d, E, C, zipf):
    w = small_workload("ecr", T, d, 128, E, 1, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + E)
    bias = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    L64, _ = O.router_logits(u16(inp["x"]), u16(inp["wg"]), bias)
    r = _route(T, E, C, inp=inp)
    assert r["status"] == 0
    assert np.abs(r["logits"].astype(np.float64) - L64).max() <= LOGIT_ABS
    S_o = O.softmax_rows(r["logits"])
    assert np.abs(r["scores"].astype(np.float64) - S_o).max() <= S_ABS
    tok_o, w_o = O.expert_choice(r["scores"], C)
    assert (r["tok"] == tok_o).all()
    assert (r["w"].astype(np.float64) == w_o).all()


# ---------------------------------------------------------------- the layer

EC_CASES = [
    # name, T, d, d_ff, E, C, d_ff_shared, zipf
    ("tiles_ragged", 700, 256, 384, 8, 150, 0, 0.0),        # K=150: 128 + a 22-row half tile
    ("full_tail", 700, 256, 256, 8, 200, 0, 1.0),           # K=200: 128 + a 72-row tile
    ("shared", 520, 256, 256, 6, 100, 256, 0.5),
    ("one_expert", 300, 128, 256, 1, 300, 0, 0.0),          # every token, once
    ("cap_above_T", 90, 256, 128, 4, 500, 128, 0.0),        # K = T: every expert takes all
    ("many_experts", 1024, 512, 256, 64, 40, 0, 1.1),
    ("one_token_each", 400, 128, 128, 16, 1, 0, 0.0),
]


@pytest.mark.parametrize("case", EC_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("flags", [0, M.MOE_FLAG_SIMT_FFN], ids=["tc", "simt"])
def test_forward_expert_choice(case, flags):
    name, T, d, d_ff, E, C, dfs, zipf = case
    w = small_workload(name, T, d, d_ff, E, 1, capacity=C, d_ff_shared=dfs, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + d + E)
    s = M.shape_of(w, EC | flags)
    ws = M.alloc_workspace(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    W13s = W2s = None
    if dfs:
        ss = M.make_shape(T, d, dfs, 1, 1)
        W13s = M.moe_pack_w13(ss, inp["W1s"][None].contiguous(), inp["W3s"][None].contiguous())
        W2s = inp["W2s"]
    out = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    M.moe_forward_expert_choice(s, inp["x"], inp["wg"], inp["bias"], W13, inp["W2"], W13s, W2s,
                                out, status, ws)
    # the scores this forward selected on (same kernels, same inputs)
    r = _route(T, E, C, inp=inp)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and r["status"] == 0
    ref = O.expert_choice_layer(I.oracle_arrays(inp), r["scores"], C)
    assert_layer_close(out, ref["out"], name)
    if C >= T and not dfs:
        return
    # tokens no expert took are exactly the shared expert's output (or zero)
    taken = np.zeros(T, bool)
    taken[ref["tokens"].ravel()] = True
    if (~taken).any() and not dfs:
        assert (out.cpu().numpy()[~taken] == 0).all()


def test_forward_expert_choice_rejects_bad_flags():
    w = small_workload("bad", 64, 128, 128, 4, 1, capacity=16)
    inp = I.make_inputs(w, "cuda", seed=1)
    for flags in (0, EC | M.MOE_FLAG_DETERMINISTIC):
        s = M.shape_of(w, flags)
        ws = M.alloc_workspace(M.shape_of(w, EC))
        out = torch.empty(64, 128, dtype=torch.float32, device="cuda")
        with pytest.raises(M.MoeError):
            M.moe_forward_expert_choice(s, inp["x"], inp["wg"], None, inp["W1"], inp["W2"], None,
                                        None, out, None, ws)
    w0 = small_workload("nocap", 64, 128, 128, 4, 1, capacity=0)
    s = M.shape_of(w0, EC)
    with pytest.raises(M.MoeError):
        M.moe_forward_expert_choice(s, inp["x"], inp["wg"], None, inp["W1"], inp["W2"], None,
                                    None, torch.empty(64, 128, device="cuda"), None,
                                    M.alloc_workspace(M.shape_of(w, EC)))


def test_expert_choice_empty_batch():
    s = M.make_shape(0, 128, 128, 4, 1, 8, 0, EC)
    M.moe_forward_expert_choice(s, None, None, None, None, None, None, None, None, None,
                                torch.empty(256, dtype=torch.uint8, device="cuda"))


# ---------------------------------------------------------------- the Mixtral shape

@pytest.mark.slow
def test_forward_expert_choice_mixtral_t4096():
    """d 4096, d_ff 14336, E 8, C = T k / E with k = 2 (the same number of
    expert rows as top-2 routing): sampled tokens against the oracle."""
    T, C = 4096, 1024
    w = I.PREFILL.with_T(T)
    inp = I.make_inputs(w, "cuda", seed=11)
    s = M.make_shape(T, w.d, w.d_ff, w.E, 1, C, 0, EC)
    ws = M.alloc_workspace(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    out = torch.empty(T, w.d, dtype=torch.float32, device="cuda")
    M.moe_forward_expert_choice(s, inp["x"], inp["wg"], inp["bias"], W13, inp["W2"], None, None,
                                out, status, ws)
    r = _route(T, w.E, C, inp=inp)
    assert int(status.item()) == 0 and r["status"] == 0
    tok, wt = O.expert_choice(r["scores"], C)
    rng = np.random.default_rng(0)
    sample = sorted(set(rng.choice(T, 12, replace=False).tolist()) | {0, T - 1,
                                                                     int(tok[0, 0]),
                                                                     int(tok[-1, -1])})
    pairs = [(t, e) for t in sample for e in range(w.E) if t in set(tok[e].tolist())]
    ref = np.zeros((len(sample), w.d))
    if pairs:
        toks = np.array([p[0] for p in pairs], np.int32)
        exps = np.array([p[1] for p in pairs], np.int32)
        y = O.expert_rows(u16(inp["x"]), u16(inp["W1"]), u16(inp["W3"]), u16(inp["W2"]), toks,
                          exps)
        pos = {t: i for i, t in enumerate(sample)}
        for (t, e), row in zip(pairs, y):
            j = int(np.nonzero(tok[e] == t)[0][0])
            ref[pos[t]] += wt[e, j] * row
    got = out[torch.tensor(sample, device="cuda")]
    assert_layer_close(got, ref, "mixtral expert choice")
