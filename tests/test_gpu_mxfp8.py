"""MXFP8 experts on the GPU vs the oracle's MXFP8 mode, through the C ABI.

The expert quantizer is compared bit for bit (codes and scales) with the
oracle's quantizer; the layer (moe_forward_mxfp8: bf16 router, MXFP8 x, w1/w3,
h and w2, tcgen05 block-scaled GEMMs) against the oracle on identical fp32
logits, within the layer tolerance (max-abs 2e-2, relative Frobenius 1e-2).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import (assert_layer_close, oracle_tokens_subset, sample_tokens, small_workload,
                         u16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _unpack_w13(W13, d_ff):
    """Packed [E, 2 d_ff, K] (64-row gate/up interleave) -> (W1 rows, W3 rows)."""
    E, _, K = W13.shape
    blk = W13.reshape(E, d_ff // 64, 2, 64, K)
    return blk[:, :, 0].reshape(E, d_ff, K), blk[:, :, 1].reshape(E, d_ff, K)


def _f64(t):
    return t.double().cpu().numpy()


def _weights(E, d_ff, d, kind, seed):
    g = torch.Generator("cuda").manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, device="cuda") * 0.02
    W1, W3, W2 = mk(E, d_ff, d), mk(E, d_ff, d), mk(E, d, d_ff)
    if kind == "wide":
        # row scales from 2^-40 to 2^40: E8M0 exponents far from zero
        for W in (W1, W3, W2):
            W *= torch.exp2(torch.randint(-40, 40, W.shape[:-1] + (1,), generator=g,
                                          device="cuda").float())
    elif kind == "special":
        W1[0, :, :64] = 0.0                              # all-zero blocks
        W3[0, 3, :] = 1e-39                              # bf16 subnormals
        W2[0, 1, :32] = 3e38                             # near the bf16 maximum
        W1[-1, 5, :] = torch.linspace(-448, 448, d, device="cuda")  # exact E4M3 grid points
        # blocks whose maximum scales past 448: elements of 464 and above clamp
        W1[-1, 6, 0::2] = 500.0
        W1[-1, 6, 1::2] = 470.0
        W3[-1, 7, :] = torch.linspace(-511, 511, d, device="cuda")
    return [W.to(torch.bfloat16).contiguous() for W in (W1, W3, W2)]


@pytest.mark.parametrize("E,d_ff,d", [(3, 256, 256), (2, 384, 512), (1, 128, 7168)])
@pytest.mark.parametrize("kind", ["normal", "wide", "special"])
def test_quantize_experts_bitexact(E, d_ff, d, kind):
    W1, W3, W2 = _weights(E, d_ff, d, kind, seed=E + d)
    s = M.make_shape(1, d, d_ff, E, 1)
    q = M.moe_quantize_experts_mxfp8(s, W1, W3, W2)
    torch.cuda.synchronize()
    c1, c3 = _unpack_w13(q["W13q"].cpu().numpy(), d_ff)
    sf13 = M.sf_atoms_to_rows(q["W13sf"].cpu().numpy(), E * 2 * d_ff, d).reshape(E, 2 * d_ff, -1)
    s1, s3 = _unpack_w13(sf13, d_ff)
    for W, c, sc in ((W1, c1, s1), (W3, c3, s3)):
        oc, os_ = O.mx_quantize(_f64(W).reshape(-1, d))
        assert (c.reshape(-1, d) == oc).all()
        assert (sc.reshape(-1, d // 32) == os_).all()
    oc, os_ = O.mx_quantize(_f64(W2).reshape(-1, d_ff))
    assert (q["W2q"].cpu().numpy().reshape(-1, d_ff) == oc).all()
    assert (M.sf_atoms_to_rows(q["W2sf"].cpu().numpy(), E * d, d_ff) == os_).all()


MX_CASES = [
    # name, T, d, d_ff, E, k, capacity, d_ff_shared, zipf
    ("tiles_ragged", 700, 256, 384, 8, 2, 0, 0, 0.0),
    ("shared", 520, 256, 256, 6, 2, 0, 256, 0.5),
    ("capacity", 1000, 256, 256, 16, 4, 100, 0, 1.0),
    ("many_experts", 800, 512, 256, 64, 6, 0, 0, 1.1),
    ("one_token", 1, 512, 256, 8, 2, 0, 128, 0.0),
    ("five_tokens", 5, 256, 128, 4, 2, 0, 0, 0.0),
]


@pytest.mark.parametrize("case", MX_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("flags", [0, M.MOE_FLAG_DETERMINISTIC], ids=["default", "det"])
def test_forward_mxfp8_parity(case, flags):
    name, T, d, d_ff, E, k, C, dfs, zipf = case
    w = small_workload(name, T, d, d_ff, E, k, capacity=C, d_ff_shared=dfs, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + d + E)
    oi = I.oracle_arrays(inp)
    layer = M.MoeLayerMx(inp, flags=flags)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy(), mx=True)   # identical fp32 logits
    assert (idx.cpu().numpy() == ref["idx"]).all()
    assert_layer_close(out, ref["out"], f"mxfp8 {name}")


def test_forward_mxfp8_slot_priority():
    w = small_workload("mxprio", 900, 256, 256, 16, 4, capacity=120, zipf_s=1.2)
    inp = I.make_inputs(w, "cuda", seed=9)
    oi = dict(I.oracle_arrays(inp), slot_priority=True)
    layer = M.MoeLayerMx(inp, flags=M.MOE_FLAG_SLOT_PRIORITY)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy(), mx=True)
    assert (ref["slot_pos"] < 0).any()
    assert_layer_close(out, ref["out"], "mxfp8 slot priority")


def test_mxfp8_flag_checks():
    w = small_workload("mxbad", 64, 128, 128, 4, 2)
    inp = I.make_inputs(w, "cuda", seed=1)
    layer = M.MoeLayerMx(inp)
    x = inp["x"]
    out = torch.empty(64, 128, dtype=torch.float32, device="cuda")
    # the MXFP8 call without its flag, and the bf16 call with it, are refused
    with pytest.raises(M.MoeError):
        M.moe_forward_mxfp8(M.shape_of(w, 0), x, layer.Wg, None, layer.q, None, out, None, None,
                            layer.status, layer.ws)
    bf = M.MoeLayer(inp)
    with pytest.raises(M.MoeError):
        M.moe_forward(M.shape_of(w, M.MOE_FLAG_MXFP8), x, bf.Wg, None, bf.W13, bf.W2, None, None,
                      out, None, None, bf.status, bf.ws)


@pytest.mark.slow
def test_forward_mxfp8_mixtral_t4096():
    """The Mixtral layer shape at T = 4096: all routing bit-exact on identical
    logits, sampled tokens against the oracle's MXFP8 mode."""
    w = I.PREFILL.with_T(4096)
    inp = I.make_inputs(w, "cuda", seed=2)
    layer = M.MoeLayerMx(inp)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    idx_o, w_o = O.route(logits.cpu().numpy(), w.k)
    disp = O.dispatch(idx_o, w.E, w.capacity)
    tokens = sample_tokens(w.T, disp, n_random=10)
    ref = oracle_tokens_subset(inp, idx_o, w_o, disp["slot_pos"], tokens, mx=True)
    assert_layer_close(out[torch.from_numpy(tokens.astype(np.int64)).cuda()], ref,
                       "mxfp8 mixtral T=4096")


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_mxfp8_decode_mixtral_shape(T):
    """The decode kernels on MXFP8 experts (only the chosen experts' codes and
    scales streamed) and the block-scaled tensor-core chain, both against the
    oracle's MXFP8 mode."""
    w = I.DECODE.with_T(T)
    inp = I.make_inputs(w, "cuda", seed=0)
    oi = I.oracle_arrays(inp)
    layer = M.MoeLayerMx(inp)
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, flags=M.MOE_FLAG_FORCE_DECODE).clone()
    out_p = layer.forward(inp["x"], flags=M.MOE_FLAG_FORCE_PREFILL).clone()
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy(), mx=True)
    assert_layer_close(out, ref["out"], f"mxfp8 decode kernels T={T}")
    assert_layer_close(out_p, ref["out"], f"mxfp8 tensor-core chain T={T}")


@pytest.mark.parametrize("C", [0, 2])
def test_mxfp8_decode_shared_many_experts(C):
    w = small_workload("mxdec", 3, 1024, 512, 64, 8, capacity=C, d_ff_shared=256, zipf_s=3.0)
    inp = I.make_inputs(w, "cuda", seed=2)
    oi = I.oracle_arrays(inp)
    layer = M.MoeLayerMx(inp, flags=M.MOE_FLAG_FORCE_DECODE)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(oi, logits=logits.cpu().numpy(), mx=True)
    if C:
        assert (ref["slot_pos"] < 0).any()
    assert_layer_close(out, ref["out"], "mxfp8 decode with shared expert")
