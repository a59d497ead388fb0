"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test checks the oracle against one of: a value printed on the pages
(tests/golden), a hand-worked case, brute force on tiny inputs, a closed form,
an invariant, or a special case that reduces to a library routine (torch fp64
softmax / topk / matmul / index_add_, torch's bf16 conversion).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_mixture_experts_17_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = line.split(":", 1)
        out[key.strip()] = [int(v) for v in val.split()]
    return out


# ---------------------------------------------------------------- page values

def test_p3_worked_offsets(orc):
    """counts [4,4,0] -> offsets [4,8,8] / [0,4,8,8] (the page's example)."""
    g = _read_kv(os.path.join(GOLDEN, "p3_offsets.txt"))
    E = g["E"][0]
    counts = g["counts"]
    # build an idx array that realises these counts with k = 1
    idx = np.array([[e] for e in range(E) for _ in range(counts[e])], np.int32)
    d = orc.dispatch(idx, E, 0)
    assert d["counts"].tolist() == counts
    assert d["offsets"].tolist() == g["offsets_exclusive"]
    assert d["offsets"][1:].tolist() == g["offsets_inclusive"]


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "hand_cases.json")))["cases"],
                         ids=lambda c: c["name"])
def test_hand_cases(orc, case):
    L = np.array(case["logits"], np.float32)
    idx, w = orc.route(L, case["k"])
    assert idx.tolist() == case["idx"]
    np.testing.assert_allclose(w, np.array(case["w"]), rtol=0, atol=case["w_tol"])
    d = orc.dispatch(idx, case["E"], case["capacity"])
    assert d["counts"].tolist() == case["counts"]
    assert d["offsets"].tolist() == case["offsets"]
    assert d["slot_pos"].tolist() == case["slot_pos"]
    assert d["perm_token"].tolist() == case["perm_token"]
    assert d["n_kept"] == case["n_kept"]


def test_hand_case_dropped_token_output_is_zero(orc):
    """Capacity 3 in the [4,4,0] case drops token 3 from both experts: out[3] = 0."""
    rng = np.random.default_rng(5)
    T, d, d_ff, E, k = 4, 8, 16, 3, 2
    bf = lambda a: I.to_numpy_u16(torch.tensor(a, dtype=torch.float32).to(torch.bfloat16))
    x = bf(rng.standard_normal((T, d)))
    W1, W3 = bf(rng.standard_normal((E, d_ff, d)) * 0.3), bf(rng.standard_normal((E, d_ff, d)) * 0.3)
    W2 = bf(rng.standard_normal((E, d, d_ff)) * 0.3)
    L = np.tile(np.array([1, 1, 0], np.float32), (T, 1))
    idx, w = orc.route(L, k)
    disp = orc.dispatch(idx, E, 3)
    out = orc.moe_tokens(x, W1, W3, W2, idx, w, disp["slot_pos"], np.arange(T))
    assert np.all(out[3] == 0.0)
    assert np.all(np.abs(out[:3]).sum(1) > 0)


# ---------------------------------------------------------------- top-k by brute force

def _brute_topk(l, k):
    """All k-subsets; the chosen set is the one whose every member beats every
    non-member under (larger logit, then smaller index); order likewise."""
    E = len(l)
    beats = lambda a, b: (l[a] > l[b]) or (l[a] == l[b] and a < b)
    winners = []
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if all(beats(a, b) for a in S for b in rest):
            winners.append(S)
    assert len(winners) == 1
    return sorted(winners[0], key=lambda e: (-l[e], e))


@pytest.mark.parametrize("E,k", [(3, 1), (3, 2), (5, 3), (8, 2), (8, 4), (8, 8)])
def test_topk_brute_force_with_ties(orc, E, k):
    rng = np.random.default_rng(E * 100 + k)
    # a small discrete set of values makes ties frequent; include -0.0 / +0.0
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 2.0, -np.inf], np.float32)
    T = 300
    L = vals[rng.integers(0, len(vals), size=(T, E))]
    L[:, 0] = np.where(np.isinf(L[:, 0]), 1.0, L[:, 0])   # a finite max per row
    idx, w = orc.route(L, k)
    for t in range(T):
        assert idx[t].tolist() == _brute_topk(L[t].tolist(), k), (t, L[t])


def test_topk_equals_softmax_topk(orc):
    """On continuous logits the selection equals torch.topk of the fp64 softmax
    (the page's order), and the weights equal the renormalised probabilities."""
    rng = np.random.default_rng(1)
    for E, k in [(8, 2), (64, 6), (256, 8), (128, 8)]:
        L = (rng.standard_normal((200, E)) * 2).astype(np.float32)
        idx, w = orc.route(L, k)
        p = F.softmax(torch.from_numpy(L).double(), dim=1)
        pv, pi = torch.topk(p, k, dim=-1)
        assert (pi.numpy() == idx).all()
        pv = pv / pv.sum(-1, keepdim=True)
        np.testing.assert_allclose(w, pv.numpy(), rtol=1e-13, atol=0)


def test_special_cases_k1_kE_equal(orc):
    rng = np.random.default_rng(2)
    L = (rng.standard_normal((50, 8)) * 3).astype(np.float32)
    # k = 1 (Switch top-1): weight exactly 1, expert = argmax
    idx, w = orc.route(L, 1)
    assert (w == 1.0).all()
    assert (idx[:, 0] == np.argmax(L, axis=1)).all()
    # k = E: weights are the full softmax (numpy exp), every expert once
    idx, w = orc.route(L, 8)
    ex = np.exp(L.astype(np.float64) - L.max(1, keepdims=True))
    sm = ex / ex.sum(1, keepdims=True)
    full = np.take_along_axis(sm, idx, 1)
    np.testing.assert_allclose(w, full, rtol=1e-14)
    assert (np.sort(idx, 1) == np.arange(8)).all()
    # all-equal logits: idx = 0..k-1 and w = 1/k
    Z = np.full((7, 8), 0.25, np.float32)
    for k in (1, 3, 8):
        idx, w = orc.route(Z, k)
        assert (idx == np.arange(k)).all()
        np.testing.assert_allclose(w, 1.0 / k, rtol=1e-15)


def test_route_rejects_nan(orc):
    L = np.zeros((3, 4), np.float32)
    L[1, 2] = np.nan
    with pytest.raises(orc.OracleError) as ei:
        orc.route(L, 2)
    assert ei.value.code == orc.ENONFINITE


def test_weights_sum_to_one(orc):
    rng = np.random.default_rng(3)
    L = (rng.standard_normal((500, 128)) * 1.5).astype(np.float32)
    _, w = orc.route(L, 8)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- dispatch invariants

def _random_idx(rng, T, E, k, skew=0.0):
    p = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k,C", [(37, 5, 2, 0), (64, 8, 2, 0), (200, 16, 4, 30),
                                     (300, 12, 3, 40), (128, 8, 8, 0), (64, 8, 2, 1)])
def test_dispatch_invariants_and_brute_rank(orc, T, E, k, C):
    rng = np.random.default_rng(T + E + k + C)
    idx = _random_idx(rng, T, E, k, skew=1.0)
    d = orc.dispatch(idx, E, C)
    flat = idx.reshape(-1)
    # counts are the histogram
    assert (d["counts"] == np.bincount(flat, minlength=E)).all()
    # brute-force rank: earlier assignments (row-major) to the same expert
    rank = np.array([(flat[:a] == flat[a]).sum() for a in range(len(flat))])
    kept = (rank < C) if C > 0 else np.ones_like(rank, bool)
    kc = np.array([kept[flat == e].sum() for e in range(E)])
    assert (d["offsets"] == np.concatenate([[0], np.cumsum(kc)])).all()
    assert d["n_kept"] == kept.sum() == d["offsets"][-1]
    sp = d["slot_pos"].reshape(-1)
    assert ((sp >= 0) == kept).all()
    assert (sp[kept] == d["offsets"][flat[kept]] + rank[kept]).all()
    # inverse bijection between kept assignments and rows [0, n_kept)
    assert sorted(sp[kept].tolist()) == list(range(d["n_kept"]))
    pt = d["perm_token"]
    assert (pt[sp[kept]] == (np.arange(T * k) // k)[kept]).all()
    assert (pt[d["n_kept"]:] == -1).all()
    # uncapped: each token appears exactly k times
    if C <= 0:
        assert (np.bincount(pt, minlength=T) == k).all()
    # rows within each expert segment are in ascending token order
    for e in range(E):
        seg = pt[d["offsets"][e]:d["offsets"][e + 1]]
        assert (np.diff(seg) > 0).all()
        # drops are a token-order suffix: every kept token precedes every dropped one
        toks = (np.arange(T * k) // k)[flat == e]
        dropped = toks[~kept[flat == e]]
        if len(dropped) and len(seg):
            assert seg.max() < dropped.min()


@pytest.mark.parametrize("T,E,k,C", [(37, 5, 2, 5), (200, 16, 4, 30), (300, 12, 3, 40),
                                     (64, 8, 2, 1), (50, 4, 1, 7), (80, 6, 3, 0)])
def test_dispatch_slot_priority_brute_force(orc, T, E, k, C):
    """Slot-priority capacity: per expert, its assignments sorted by (slot, token)
    with a plain Python sort; the first C are kept, in that order."""
    rng = np.random.default_rng(T * 3 + E + k + C)
    idx = _random_idx(rng, T, E, k, skew=1.2)
    d = orc.dispatch(idx, E, C, slot_priority=True)
    off = [0]
    order = {}
    for e in range(E):
        a_e = sorted(((j, t) for t in range(T) for j in range(k) if idx[t, j] == e))
        keep = a_e if C <= 0 else a_e[:C]
        order[e] = keep
        off.append(off[-1] + len(keep))
    assert d["offsets"].tolist() == off
    assert (d["counts"] == np.bincount(idx.reshape(-1), minlength=E)).all()
    sp = np.full((T, k), -1)
    for e in range(E):
        for r, (j, t) in enumerate(order[e]):
            sp[t, j] = off[e] + r
            assert d["perm_token"][off[e] + r] == t
    assert (d["slot_pos"] == sp).all()


def test_dispatch_slot_priority_special_cases(orc):
    rng = np.random.default_rng(9)
    # k = 1: slot-major and row-major orders coincide
    idx1 = _random_idx(rng, 120, 6, 1, skew=1.0)
    a, b = orc.dispatch(idx1, 6, 9), orc.dispatch(idx1, 6, 9, slot_priority=True)
    for key in ("counts", "offsets", "slot_pos", "perm_token"):
        assert (a[key] == b[key]).all()
    # uncapped: the same rows per expert (only their order differs)
    idx = _random_idx(rng, 90, 8, 3, skew=0.5)
    a, b = orc.dispatch(idx, 8, 0), orc.dispatch(idx, 8, 0, slot_priority=True)
    assert (a["offsets"] == b["offsets"]).all()
    for e in range(8):
        sa = a["perm_token"][a["offsets"][e]:a["offsets"][e + 1]]
        sb = b["perm_token"][b["offsets"][e]:b["offsets"][e + 1]]
        assert sorted(sa.tolist()) == sorted(sb.tolist())
    # every first choice survives whenever C covers the first choices
    idx = _random_idx(rng, 100, 5, 2, skew=0.0)
    C = int(np.bincount(idx[:, 0], minlength=5).max())
    b = orc.dispatch(idx, 5, C, slot_priority=True)
    assert (b["slot_pos"][:, 0] >= 0).all()
    a = orc.dispatch(idx, 5, C)
    assert a["n_kept"] == b["n_kept"]          # same kept count per expert: min(count, C)


def test_dispatch_rejects_bad_ids(orc):
    with pytest.raises(orc.OracleError) as ei:
        orc.dispatch(np.array([[0, 3]], np.int32), 3, 0)
    assert ei.value.code == orc.EBADEXPERT
    with pytest.raises(orc.OracleError) as ei:
        orc.dispatch(np.array([[1, 1]], np.int32), 3, 0)
    assert ei.value.code == orc.EBADEXPERT


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch(orc):
    """fp32 values round to bf16 exactly as torch's fp32 -> bf16 conversion."""
    rng = np.random.default_rng(4)
    mags = (10.0 ** rng.integers(-30, 30, 3000)).astype(np.float32)
    v = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * mags,
        # exact ties between two bf16 neighbours (lower 16 bits 0x8000)
        (rng.integers(0, 2 ** 16, 500).astype(np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([1e-40, -3e-39, 3.3e38, -3.39e38, 0.0, -0.0], np.float32),
    ]).astype(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.round_bf16(float(a)) for a in v])
    np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------- layer: closed form

def test_ffn_closed_form_permutation_weights(orc):
    """W1 = P, W3 = Q, W2 = R (permutation matrices, all different and not
    symmetric): y = R (silu(P x) * (Q x)), element by element with math.exp."""
    d = d_ff = 16
    rng = np.random.default_rng(6)
    perms = [rng.permutation(d) for _ in range(3)]
    mats = []
    for p in perms:
        m = np.zeros((d, d), np.float32)
        m[np.arange(d), p] = 1.0
        mats.append(m)
    P, Q, R = mats
    x32 = rng.standard_normal((3, d)).astype(np.float32) * 2
    bf = lambda a: I.to_numpy_u16(torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16))
    x = bf(x32)
    xv = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    y = orc.expert_rows(x, bf(P[None]), bf(Q[None]), bf(R[None]), np.arange(3), np.zeros(3), h_bf16=False)
    for t in range(3):
        g = xv[t][perms[0]]
        u = xv[t][perms[1]]
        h = np.array([gi / (1 + math.exp(-gi)) * ui for gi, ui in zip(g, u)])
        np.testing.assert_allclose(y[t], h[perms[2]], rtol=1e-15, atol=0)


# ---------------------------------------------------------------- layer: dense brute force

def _dense_brute(inp, L32, C, h_bf16):
    """Every expert on every token, times a masked weight (fp64 torch)."""
    x = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).double()
    cv = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double()
    W1, W3, W2 = cv(inp["W1"]), cv(inp["W3"]), cv(inp["W2"])
    T, E, k = x.shape[0], W1.shape[0], inp["k"]
    Ld = torch.from_numpy(L32).double()
    p = torch.softmax(Ld, dim=1)
    # the top-k mask from the (logit desc, index asc) order
    m = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(L32[t, e]), e))[:k]
        m[t, order] = 1.0
    wfull = p * m
    wfull = wfull / wfull.sum(1, keepdim=True)
    # capacity: keep an assignment iff fewer than C earlier tokens chose that expert
    if C > 0:
        before = torch.cumsum(m, 0) - m
        wfull = torch.where(before < C, wfull, torch.zeros_like(wfull))
    def rnd(h):
        if not h_bf16:
            return h
        return torch.tensor([orc_round(v) for v in h.reshape(-1).tolist()],
                            dtype=torch.float64).reshape(h.shape)

    out = torch.zeros(T, x.shape[1], dtype=torch.float64)
    for e in range(E):
        h = rnd(F.silu(x @ W1[e].T) * (x @ W3[e].T))
        out += wfull[:, e:e + 1] * (h @ W2[e].T)
    if "W1s" in inp:
        W1s, W3s, W2s = cv(inp["W1s"]), cv(inp["W3s"]), cv(inp["W2s"])
        out = rnd(F.silu(x @ W1s.T) * (x @ W3s.T)) @ W2s.T + out
    return out.numpy()


orc_round = None


def _small_inputs(T, d, d_ff, E, k, C=0, shared=0, zipf=0.0, seed=0):
    w = I.Workload("pin", T=T, d=d, d_ff=d_ff, E=E, k=k, capacity=C, d_ff_shared=shared, zipf_s=zipf)
    return I.oracle_arrays(I.make_inputs(w, "cpu", seed=seed))


@pytest.mark.parametrize("T,d,d_ff,E,k,C,shared,zipf", [
    (24, 32, 48, 4, 2, 0, 0, 0.0),
    (40, 32, 32, 8, 3, 12, 0, 1.0),
    (16, 64, 32, 6, 2, 0, 48, 1.1),
    (32, 16, 16, 5, 5, 0, 0, 0.0),
])
@pytest.mark.parametrize("h_bf16", [False, True])
def test_layer_vs_dense_brute_force(orc, T, d, d_ff, E, k, C, shared, zipf, h_bf16):
    global orc_round
    orc_round = orc.round_bf16
    inp = _small_inputs(T, d, d_ff, E, k, C, shared, zipf, seed=T + E)
    res = orc.forward(inp, h_bf16=h_bf16)
    ref = _dense_brute(inp, res["L32"], C, h_bf16)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)


def test_router_logits_vs_torch(orc):
    inp = _small_inputs(50, 96, 32, 7, 2, zipf=1.0, seed=9)
    L64, L32 = orc.router_logits(inp["x"], inp["wg"], inp["bias"])
    x = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).double()
    wg = torch.from_numpy(inp["wg"].view(np.int16)).view(torch.bfloat16).double()
    ref = x @ wg.T + torch.from_numpy(inp["bias"]).double()
    np.testing.assert_allclose(L64, ref.numpy(), rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(L32, torch.from_numpy(L64).float().numpy())


# ---------------------------------------------------------------- layer: the page's loop

def _mixtral_loop(inp, L32):
    """The page's Sparse MoE Block, restated with torch fp64 library calls:
    softmax, topk, divide by the sum, then for each expert torch.where,
    gather, expert FFN, scale by the routing weight and index_add_."""
    cv = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double()
    hidden = cv(inp["x"])
    W1, W3, W2 = cv(inp["W1"]), cv(inp["W3"]), cv(inp["W2"])
    routing_weights = F.softmax(torch.from_numpy(L32).double(), dim=1)
    routing_weights, selected = torch.topk(routing_weights, inp["k"], dim=-1)
    routing_weights /= routing_weights.sum(dim=-1, keepdim=True)
    final = torch.zeros_like(hidden)
    for e in range(W1.shape[0]):
        idx, top_x = torch.where(selected == e)
        if idx.shape[0] == 0:
            continue
        cur = hidden[idx]
        cur = (F.silu(cur @ W1[e].T) * (cur @ W3[e].T)) @ W2[e].T
        cur = cur * routing_weights[idx, top_x, None]
        final.index_add_(0, idx, cur)
    return final.numpy(), selected.numpy()


@pytest.mark.parametrize("wl", ["tiny", "tiny_E16_k4"])
def test_layer_vs_mixtral_loop(orc, wl):
    if wl == "tiny":
        inp = I.oracle_arrays(I.make_inputs(I.TINY, "cpu", seed=0))
    else:
        inp = _small_inputs(48, 64, 128, 16, 4, zipf=1.0, seed=3)
    res = orc.forward(inp, h_bf16=False)
    ref, sel = _mixtral_loop(inp, res["L32"])
    assert (sel == res["idx"]).all()
    np.testing.assert_allclose(res["out"], ref, rtol=1e-11, atol=1e-13)


def test_sampled_tokens_equal_full(orc):
    """A token's output depends on its own row and the global drop set only,
    so evaluating a sample gives exactly the full run's rows."""
    inp = _small_inputs(96, 32, 32, 8, 2, C=20, zipf=1.0, seed=11)
    full = orc.forward(inp)
    sample = np.array([0, 5, 17, 50, 95], np.int32)
    part = orc.forward(inp, tokens=sample)
    np.testing.assert_array_equal(part["out"], full["out"][sample])
