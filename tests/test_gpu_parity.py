"""CUDA path vs the fp64 oracle, through the C ABI, on seeded inputs.

Routing, offsets, permutation and drops are compared bit for bit on
identical fp32 logits; the router logits against fp64 within LOGIT_ABS; the
layer output within max-abs 2e-2 and relative Frobenius 1e-2. Sizes span
several tiles and a ragged tail; the edge cases of the method are covered.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import (LOGIT_ABS, W_ABS, Buffers, assert_layer_close, layer_errors,
                         pipeline_from_logits, small_workload, u16)

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _logits(T, E, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "continuous":
        return (rng.standard_normal((T, E)) * 2).astype(np.float32)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 2.0, -np.inf], np.float32)
    L = vals[rng.integers(0, len(vals), size=(T, E))]
    L[:, 0] = np.where(np.isinf(L[:, 0]), 1.0, L[:, 0])
    return L


# ---------------------------------------------------------------- S2: top-k on identical logits

@pytest.mark.parametrize("E,k", [(3, 2), (8, 2), (16, 4), (32, 1), (40, 3), (64, 6), (96, 5),
                                 (128, 8), (256, 8), (256, 16)])
@pytest.mark.parametrize("kind", ["continuous", "ties"])
def test_route_bitexact(E, k, kind):
    T = 1000
    L = _logits(T, E, kind, seed=E * 7 + k)
    idx_o, w_o = O.route(L, k)
    w = small_workload("r", T, 128, 128, E, k)
    b = Buffers(w)
    b.logits.copy_(torch.from_numpy(L))
    M.moe_route(b.shape, None, None, None, b.logits, b.idx, b.w, b.status, b.ws)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    assert (b.idx.cpu().numpy() == idx_o).all()
    assert np.abs(b.w.double().cpu().numpy() - w_o).max() <= W_ABS


# ---------------------------------------------------------------- S1: router logits

@pytest.mark.parametrize("T,d,E,zipf,flags", [
    (300, 256, 8, 0.0, 0),            # tensor-core router, BN = 64
    (300, 512, 128, 1.0, 0),          # BN = 128
    (200, 7168, 256, 1.1, 0),         # BN = 256, the fine-grained router shape
    (5, 4096, 8, 0.0, 0),             # small-T router (one warp per expert)
    (16, 2048, 256, 1.0, 0),
    (300, 512, 64, 1.0, M.MOE_FLAG_SIMT_FFN),   # CUDA-core router
])
def test_router_logits(T, d, E, zipf, flags):
    w = small_workload("lg", T, d, 128, E, 2, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + E)
    L64, _ = O.router_logits(u16(inp["x"]), u16(inp["wg"]),
                             None if inp["bias"] is None else inp["bias"].cpu().numpy())
    b = Buffers(w, flags=flags)
    M.moe_route(b.shape, inp["x"], inp["wg"], inp["bias"], b.logits, b.idx, b.w, b.status, b.ws)
    torch.cuda.synchronize()
    err = np.abs(b.logits.double().cpu().numpy() - L64).max()
    assert err <= LOGIT_ABS, err


# ---------------------------------------------------------------- S1+S2 fused (router GEMM epilogue)

@pytest.mark.parametrize("T,E,k,ties", [(300, 8, 2, False), (1000, 64, 8, False), (257, 40, 3, False),
                                        (500, 16, 1, False), (300, 8, 2, True), (200, 64, 6, True)])
def test_router_topk_fused_matches_separate(T, E, k, ties):
    """moe_route on x (E <= 64: top-k in the router GEMM's epilogue) against the
    separate top-k kernel on the very logits it produced: indices bit for bit,
    weights within W_ABS, and the logits against the fp64 oracle."""
    w = small_workload("rtk", T, 512, 128, E, k)
    inp = I.make_inputs(w, "cuda", seed=T + E + k)
    wg, bias = inp["wg"], inp["bias"]
    if ties:   # logits = bias only, with repeated values: ties decided by expert index
        wg = torch.zeros_like(wg)
        bias = torch.tensor([0.5, -1.0, 0.5, 2.0, 2.0, 0.0, -0.0, 0.5] * (E // 8),
                            dtype=torch.float32, device="cuda")
    b1 = Buffers(w)
    M.moe_route(b1.shape, inp["x"], wg, bias, b1.logits, b1.idx, b1.w, b1.status, b1.ws)
    b2 = Buffers(w)
    b2.logits.copy_(b1.logits)
    M.moe_route(b2.shape, None, None, None, b2.logits, b2.idx, b2.w, b2.status, b2.ws)
    torch.cuda.synchronize()
    assert int(b1.status.item()) == 0 and int(b2.status.item()) == 0
    assert torch.equal(b1.idx, b2.idx)
    assert (b1.w - b2.w).abs().max().item() <= W_ABS
    idx_o, w_o = O.route(b1.logits.cpu().numpy(), k)
    assert (b1.idx.cpu().numpy() == idx_o).all()
    assert np.abs(b1.w.double().cpu().numpy() - w_o).max() <= W_ABS
    L64, _ = O.router_logits(u16(inp["x"]), u16(wg), None if bias is None else bias.cpu().numpy())
    assert np.abs(b1.logits.double().cpu().numpy() - L64).max() <= LOGIT_ABS


# ---------------------------------------------------------------- S3/S4: histogram, offsets, permutation

def _random_idx(rng, T, E, k, skew):
    p = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k,C,skew", [
    (1, 8, 2, 0, 0.0), (37, 5, 2, 0, 0.0), (256, 8, 2, 0, 0.5), (257, 8, 2, 0, 0.5),
    (1000, 16, 4, 200, 1.0), (4096, 128, 8, 320, 1.0), (3000, 256, 8, 0, 1.1),
    (2000, 64, 16, 100, 0.8), (700, 8, 8, 0, 0.0), (513, 3, 1, 50, 2.0),
])
@pytest.mark.parametrize("prio", [False, True], ids=["rowmajor", "slotmajor"])
def test_permute_bitexact(T, E, k, C, skew, prio):
    rng = np.random.default_rng(T * 3 + E)
    idx = _random_idx(rng, T, E, k, skew)
    ref = O.dispatch(idx, E, C, slot_priority=prio)
    w = small_workload("p", T, 128, 128, E, k, capacity=C)
    b = Buffers(w, flags=M.MOE_FLAG_SLOT_PRIORITY if prio else 0)
    x = torch.randn(T, 128, device="cuda").to(torch.bfloat16)
    b.idx.copy_(torch.from_numpy(idx))
    M.moe_permute(b.shape, b.idx, x, b.counts, b.offsets, b.slot_pos, b.perm_token, b.x_perm,
                  b.n_kept, b.status, b.ws)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    assert (b.counts.cpu().numpy() == ref["counts"]).all()
    assert (b.offsets.cpu().numpy() == ref["offsets"]).all()
    assert int(b.n_kept.item()) == ref["n_kept"]
    assert (b.slot_pos.cpu().numpy() == ref["slot_pos"]).all()
    n = ref["n_kept"]
    pt = b.perm_token.cpu().numpy()[:n]
    assert (pt == ref["perm_token"][:n]).all()
    assert torch.equal(b.x_perm[:n], x[torch.from_numpy(pt.astype(np.int64)).cuda()])
    # a second call on the same workspace gives the same answer (the ticket re-arms)
    M.moe_permute(b.shape, b.idx, x, b.counts, b.offsets, b.slot_pos, b.perm_token, b.x_perm,
                  b.n_kept, b.status, b.ws)
    torch.cuda.synchronize()
    assert (b.offsets.cpu().numpy() == ref["offsets"]).all()


def test_p3_worked_example_on_gpu():
    """counts [4,4,0] -> offsets [0,4,8,8]; with capacity 3 -> [0,3,6,6]."""
    cases = json.load(open(os.path.join(GOLDEN, "hand_cases.json")))["cases"]
    for case in cases:
        L = np.array(case["logits"], np.float32)
        T, E, k = L.shape[0], case["E"], case["k"]
        w = small_workload("p3", T, 128, 128, E, k, capacity=case["capacity"])
        b = Buffers(w)
        b.logits.copy_(torch.from_numpy(L))
        M.moe_route(b.shape, None, None, None, b.logits, b.idx, b.w, b.status, b.ws)
        M.moe_permute(b.shape, b.idx, None, b.counts, b.offsets, b.slot_pos, b.perm_token, None,
                      b.n_kept, b.status, b.ws)
        torch.cuda.synchronize()
        assert b.idx.cpu().tolist() == case["idx"], case["name"]
        np.testing.assert_allclose(b.w.cpu().numpy(), np.array(case["w"]), atol=max(case["w_tol"], 1e-7))
        assert b.counts.cpu().tolist() == case["counts"]
        assert b.offsets.cpu().tolist() == case["offsets"]
        assert b.slot_pos.cpu().tolist() == case["slot_pos"]
        assert b.perm_token.cpu().tolist()[:case["n_kept"]] == case["perm_token"][:case["n_kept"]]


# ---------------------------------------------------------------- S5/S6: expert FFN and combine

FFN_CASES = [
    # name, T, d, d_ff, E, k, capacity, zipf
    ("ragged8", 700, 256, 384, 8, 2, 0, 0.0),
    ("long_groups", 2600, 512, 512, 4, 2, 0, 0.0),      # > 1024 rows per expert, ragged tails
    ("peer_tail", 1100, 256, 256, 8, 1, 0, 0.0),         # segments just past 128 rows
    ("cap16", 1500, 1024, 512, 16, 4, 400, 1.0),
    ("d128", 300, 128, 256, 8, 2, 0, 0.0),
    ("many_tiles", 3000, 512, 640, 32, 4, 0, 0.8),
]


@pytest.mark.parametrize("case", FFN_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("flags", [M.MOE_FLAG_GEMM_1SM, M.MOE_FLAG_GEMM_2SM, M.MOE_FLAG_SIMT_FFN],
                         ids=["tc1", "tc2", "simt"])
@pytest.mark.parametrize("fused", [True, False], ids=["fused", "yperm"])
def test_expert_ffn_parity(case, flags, fused):
    name, T, d, d_ff, E, k, C, zipf = case
    w = small_workload(name, T, d, d_ff, E, k, capacity=C, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=11)
    oi = I.oracle_arrays(inp)
    _, L32 = O.router_logits(oi["x"], oi["wg"], oi["bias"])
    ref = O.forward(oi, logits=L32)
    b = pipeline_from_logits(inp, torch.from_numpy(L32).cuda(), flags=flags, fused=fused)
    assert int(b.status.item()) == 0
    assert (b.idx.cpu().numpy() == ref["idx"]).all()
    assert (b.offsets.cpu().numpy() == ref["offsets"]).all()
    assert (b.slot_pos.cpu().numpy() == ref["slot_pos"]).all()
    assert_layer_close(b.out, ref["out"], f"{name} flags={flags} fused={fused}")
    if not fused:   # unweighted per-row expert outputs in permuted order
        n = ref["n_kept"]
        rows = np.linspace(0, n - 1, num=min(n, 64)).astype(np.int64)
        toks = ref["perm_token"][rows]
        exps = np.searchsorted(ref["offsets"], rows, side="right") - 1
        y_ref = O.expert_rows(oi["x"], oi["W1"], oi["W3"], oi["W2"], toks, exps)
        assert_layer_close(b.y_perm[torch.from_numpy(rows).cuda()], y_ref, "y_perm rows")


# ---------------------------------------------------------------- whole layer

FWD_CASES = [
    ("tiny", I.TINY),
    ("shared", small_workload("shared", 600, 256, 256, 16, 4, d_ff_shared=384, zipf_s=1.1)),
    ("capacity", small_workload("capacity", 1024, 256, 256, 32, 8,
                                capacity=I.capacity_for(1024, 8, 32), zipf_s=1.0)),
    ("T17", small_workload("T17", 17, 512, 256, 8, 2)),
    ("T1_prefill", small_workload("T1", 1, 256, 256, 8, 2)),
]


def _gap_ok(L64, k, margin):
    """Tokens whose k-th and (k+1)-th fp64 logits differ by more than `margin`:
    their routing is decided by more than fp32 accumulation noise."""
    s = -np.sort(-L64, axis=1)
    if s.shape[1] <= k:
        return np.ones(s.shape[0], bool)
    return (s[:, k - 1] - s[:, k]) > margin


@pytest.mark.parametrize("case", FWD_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("flags", [0, M.MOE_FLAG_DETERMINISTIC, M.MOE_FLAG_SIMT_FFN,
                                   M.MOE_FLAG_FORCE_PREFILL, M.MOE_FLAG_GEMM_2SM,
                                   M.MOE_FLAG_GEMM_2SM | M.MOE_FLAG_DETERMINISTIC],
                         ids=["default", "det", "simt", "prefill", "tc2", "tc2det"])
def test_forward_parity(case, flags):
    name, w = case
    inp = I.make_inputs(w, "cuda", seed=0)
    oi = I.oracle_arrays(inp)
    layer = M.MoeLayer(inp, flags=flags)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi)
    assert np.abs(logits.double().cpu().numpy() - ref["L64"]).max() <= LOGIT_ABS
    same = (idx.cpu().numpy() == ref["idx"]).all(1)
    sure = _gap_ok(ref["L64"], w.k, 2 * LOGIT_ABS)
    assert same[sure].all(), "routing differs on a token with a clear top-k margin"
    if w.capacity:
        # a flip anywhere can move later ranks; require none for an exact comparison
        assert same.all()
    assert_layer_close(out[torch.from_numpy(np.nonzero(same)[0]).cuda()], ref["out"][same], name)


@pytest.mark.parametrize("T,E,k,C,zipf", [(300, 8, 2, 0, 0.0), (129, 16, 4, 30, 1.0),
                                          (1000, 64, 8, 150, 1.0), (20000, 64, 8, 3000, 1.2),
                                          (19000, 8, 2, 0, 0.5)])
def test_forward_router_histogram_fused(T, E, k, C, zipf):
    """Prefill with E <= 64 folds the expert histogram into the router GEMM
    (per 128-token tile counts and ranks, last-CTA scan). moe_forward against
    the step-by-step pipeline (separate histogram kernel) on the logits the
    forward produced: identical top-k, and outputs that agree to fp32
    rounding of the weights, so every capacity drop and permuted row agrees.
    20000 tokens are 157 tiles: some CTAs take two."""
    w = small_workload("rhist", T, 256, 256, E, k, capacity=C, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + E)
    layer = M.MoeLayer(inp, flags=M.MOE_FLAG_DETERMINISTIC)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    b = pipeline_from_logits(inp, logits, flags=M.MOE_FLAG_DETERMINISTIC, fused=False)
    assert int(b.status.item()) == 0
    assert torch.equal(b.idx, idx)
    if C:
        assert (b.slot_pos < 0).any()
    scale = max(b.out.abs().max().item(), 1e-30)
    assert (out - b.out).abs().max().item() <= 1e-5 * scale
    # the second call re-uses the ticket the first call's last CTA re-armed
    out2 = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    assert torch.equal(out, out2)


@pytest.mark.parametrize("flags", [0, M.MOE_FLAG_DETERMINISTIC, M.MOE_FLAG_SIMT_FFN],
                         ids=["default", "det", "simt"])
def test_forward_slot_priority(flags):
    """Capacity with slot-major priority, through moe_forward, on a skewed load
    where most experts overflow."""
    w = small_workload("slotprio", 1200, 256, 256, 16, 4, capacity=150, zipf_s=1.2)
    inp = I.make_inputs(w, "cuda", seed=5)
    oi = dict(I.oracle_arrays(inp), slot_priority=True)
    layer = M.MoeLayer(inp, flags=flags | M.MOE_FLAG_SLOT_PRIORITY)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy())   # identical fp32 logits
    assert (idx.cpu().numpy() == ref["idx"]).all()
    drops = (ref["slot_pos"] < 0)
    assert drops.any() and not drops[:, 0].all()
    # the row-major order would keep a different set of assignments here
    kept_rm = O.dispatch(ref["idx"], w.E, w.capacity)["slot_pos"] >= 0
    assert (kept_rm != (ref["slot_pos"] >= 0)).any()
    assert_layer_close(out, ref["out"], "slot priority")


@pytest.mark.parametrize("T,C", [(2, 1), (8, 2), (16, 3)])
@pytest.mark.parametrize("prio", [False, True], ids=["rowmajor", "slotmajor"])
def test_decode_kernels_apply_capacity(T, C, prio):
    """The decode kernels drop the same assignments as the histogram path."""
    # a steep load skew (Zipf 3) makes every token pick the same two experts
    w = small_workload("deccap", T, 512, 256, 4, 2, capacity=C, d_ff_shared=128, zipf_s=3.0)
    inp = I.make_inputs(w, "cuda", seed=T + C)
    fl = M.MOE_FLAG_SLOT_PRIORITY if prio else 0
    oi = dict(I.oracle_arrays(inp), slot_priority=prio)
    layer = M.MoeLayer(inp, flags=fl)
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    out_d = layer.forward(inp["x"], logits_out=logits, flags=fl | M.MOE_FLAG_FORCE_DECODE)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy())
    assert (ref["slot_pos"] < 0).any()
    assert_layer_close(out_d, ref["out"], f"decode kernels with capacity T={T}")
    out_p = layer.forward(inp["x"], flags=fl | M.MOE_FLAG_FORCE_PREFILL)
    torch.cuda.synchronize()
    assert_layer_close(out_p, ref["out"], f"tensor-core chain with capacity T={T}")


def test_deterministic_flag_is_bitwise_repeatable():
    w = small_workload("detrep", 900, 256, 256, 16, 8, d_ff_shared=256, zipf_s=1.0)
    inp = I.make_inputs(w, "cuda", seed=3)
    layer = M.MoeLayer(inp, flags=M.MOE_FLAG_DETERMINISTIC)
    a = layer.forward(inp["x"]).clone()
    b = layer.forward(inp["x"]).clone()
    assert torch.equal(a, b)


# ---------------------------------------------------------------- decode path

@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_decode_mixtral_shape(T):
    w = I.DECODE.with_T(T)
    inp = I.make_inputs(w, "cuda", seed=0)
    oi = I.oracle_arrays(inp)
    layer = M.MoeLayer(inp)
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    # the decode kernels (streaming only the chosen experts' rows)
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx,
                        flags=M.MOE_FLAG_FORCE_DECODE)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy())   # routing: identical fp32 logits
    L64, _ = O.router_logits(oi["x"], oi["wg"], None)
    assert np.abs(logits.double().cpu().numpy() - L64).max() <= LOGIT_ABS
    assert (idx.cpu().numpy() == ref["idx"]).all()
    assert_layer_close(out, ref["out"], f"decode kernels T={T}")
    # the tensor-core chain (taken by default from T = 3 on) on the same input
    out_p = layer.forward(inp["x"], flags=M.MOE_FLAG_FORCE_PREFILL)
    torch.cuda.synchronize()
    assert_layer_close(out_p, ref["out"], f"tensor-core chain T={T}")
    # the default choice is one of them, bit for bit (k = 2: the fp32 atomic
    # combine adds two terms onto zero, which is order-independent)
    out_def = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(out_def, out if T <= 2 else out_p)


def test_decode_shared_many_experts():
    w = small_workload("dec_shared", 3, 1024, 512, 64, 8, d_ff_shared=256, zipf_s=1.1)
    inp = I.make_inputs(w, "cuda", seed=2)
    oi = I.oracle_arrays(inp)
    layer = M.MoeLayer(inp, flags=M.MOE_FLAG_FORCE_DECODE)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    ref = O.forward(oi, logits=logits.cpu().numpy())
    assert_layer_close(out, ref["out"], "decode with shared expert")


# ---------------------------------------------------------------- device-side errors

def test_nonfinite_logit_flagged():
    w = small_workload("nan", 64, 128, 128, 8, 2)
    b = Buffers(w)
    L = torch.randn(64, 8)
    L[5, 3] = float("nan")
    b.logits.copy_(L)
    M.moe_route(b.shape, None, None, None, b.logits, b.idx, b.w, b.status, b.ws)
    torch.cuda.synchronize()
    assert int(b.status.item()) & (1 << M.MOE_ERR_NONFINITE)


def test_bad_expert_flagged():
    w = small_workload("bad", 40, 128, 128, 8, 2)
    b = Buffers(w)
    idx = torch.zeros(40, 2, dtype=torch.int32)
    idx[:, 1] = 1
    idx[7, 1] = 9      # out of range
    idx[9, 1] = 0      # repeated within a token
    b.idx.copy_(idx)
    M.moe_permute(b.shape, b.idx, None, b.counts, b.offsets, b.slot_pos, b.perm_token, None,
                  b.n_kept, b.status, b.ws)
    torch.cuda.synchronize()
    assert int(b.status.item()) & (1 << M.MOE_ERR_BAD_EXPERT)
    sp = b.slot_pos.cpu().numpy()
    assert sp[7, 1] == -1 and sp[9, 1] == -1


def test_empty_batch_is_noop():
    w = small_workload("empty", 0, 128, 128, 8, 2)
    inp = I.make_inputs(small_workload("e1", 4, 128, 128, 8, 2), "cuda")
    layer = M.MoeLayer(inp)
    out = torch.full((0, 128), 5.0, device="cuda")
    M.moe_forward(M.shape_of(w), inp["x"][:0].contiguous(), layer.Wg, None, layer.W13, layer.W2,
                  None, None, out, None, None, layer.status, layer.ws)
    torch.cuda.synchronize()


# ---------------------------------------------------------------- graphs and host I/O

@pytest.mark.parametrize("T", [2, 4, 500])
def test_cuda_graph_capture_replay(T):
    w = small_workload("graph", T, 256, 256, 16, 4, d_ff_shared=128, zipf_s=1.0)
    inp = I.make_inputs(w, "cuda", seed=5)
    layer = M.MoeLayer(inp, flags=M.MOE_FLAG_DETERMINISTIC)
    x = inp["x"].clone()
    out = torch.zeros(T, w.d, dtype=torch.float32, device="cuda")
    ref = layer.forward(x).clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(x, out=out)      # warm up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    x.copy_(torch.randn_like(x.float()).to(torch.bfloat16))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, layer.forward(x).clone())


@pytest.mark.parametrize("T,k,flags", [(300, 2, 0), (5000, 2, 0), (9000, 4, M.MOE_FLAG_DETERMINISTIC)],
                         ids=["single", "chunked2", "chunked4_det"])
def test_forward_host_matches_device(T, k, flags):
    """Host-buffer forward; from 4096 tokens on it runs in overlapped chunks."""
    w = small_workload("hostio", T, 256, 256, 8, k)
    inp = I.make_inputs(w, "cuda", seed=8)
    layer = M.MoeLayer(inp, flags=M.MOE_FLAG_HOST_IO | flags)
    ref = layer.forward(inp["x"]).clone()
    x_h = inp["x"].cpu().pin_memory()
    out_h = torch.empty(w.T, w.d, dtype=torch.float32).pin_memory()
    M.moe_forward_host(layer.shape(w.T), x_h, layer.Wg, layer.bias, layer.W13, layer.W2, None,
                       None, out_h, layer.status, layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref.cpu())
