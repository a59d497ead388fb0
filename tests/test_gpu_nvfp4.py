"""NVFP4 experts on the GPU vs the oracle's NVFP4 module, through the C ABI.

The expert quantizer is compared bit for bit (packed codes, E4M3 scales in
the atom layout, per-expert global scales) with the oracle's quantizer; the
layer (moe_forward_nvfp4: bf16 router, NVFP4 x, w1/w3, h and w2 on tcgen05
kind::mxf4nvf4 GEMMs) against the oracle on the routing of identical fp32
logits. x and the weights take identical codes on both sides; h can take a
different code where its fp32 value (accumulated in another order than the
oracle's fp64) sits at an E2M1 rounding boundary. Such a flip moves h by one
E2M1 step, at most 2 s / gs_h with s / gs_h <= 1.0625 max|h| / 6 (about 1
here), and an output by that times a W2 weight (|w| < 0.1 for N(0, 0.02)
weights): at most 0.1. So: relative Frobenius error <= 1e-2, at most 1e-4 of
the outputs beyond the layer's 2e-2, none beyond 0.1.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as NV
from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import MAX_ABS, REL_FRO, layer_errors, small_workload, u16

pytestmark = pytest.mark.gpu
FLIP_ABS = 0.1
FLIP_FRAC = 1e-4


def assert_layer_close(got, ref, what=""):
    max_abs, rel = layer_errors(got, ref)
    g = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    frac = float((np.abs(g - np.asarray(ref)) > MAX_ABS).mean())
    assert rel <= REL_FRO and frac <= FLIP_FRAC and max_abs <= FLIP_ABS, \
        f"{what}: max_abs={max_abs:.3e} rel_fro={rel:.3e} beyond {MAX_ABS}: {frac:.2e}"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _unpack_codes(packed):
    """[.., K/2] bytes -> [.., K] E2M1 codes (element 2i in the low nibble)."""
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def _atoms_to_rows(sf, rows, K):
    """Scale atoms (128 rows x 64 elements, 512 bytes) -> [rows, K/16]."""
    a = np.asarray(sf).reshape(rows // 128, K // 64, 32, 4, 4)   # [tile, group, m%32, m/32, b]
    return a.transpose(0, 3, 2, 1, 4).reshape(rows, K // 16)


def _unpack_w13(W13, d_ff):
    E, _, K = W13.shape
    blk = W13.reshape(E, d_ff // 64, 2, 64, K)
    return blk[:, :, 0].reshape(E, d_ff, K), blk[:, :, 1].reshape(E, d_ff, K)


def _weights(E, d_ff, d, kind, seed):
    g = torch.Generator("cuda").manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, device="cuda") * 0.02
    W1, W3, W2 = mk(E, d_ff, d), mk(E, d_ff, d), mk(E, d, d_ff)
    if kind == "wide":
        # row scales from 2^-12 to 2^12 inside one expert: small rows' block
        # scales fall into the E4M3 subnormals or to zero
        for W in (W1, W3, W2):
            W *= torch.exp2(torch.randint(-12, 12, W.shape[:-1] + (1,), generator=g,
                                          device="cuda").float())
    elif kind == "special":
        W1[0, :, :64] = 0.0                              # all-zero blocks
        W3[0, 3, :] = 1e-39                              # bf16 subnormals
        W2[0, 1, :32] = 3e38                             # near the bf16 maximum
        W1[-1, 5, :] = torch.linspace(-6, 6, d, device="cuda")   # midpoints of the E2M1 grid
        if E > 1:
            for W in (W1, W3, W2):
                W[1] = 0.0                               # an all-zero expert: global scale 1
    return [W.to(torch.bfloat16).contiguous() for W in (W1, W3, W2)]


@pytest.mark.parametrize("E,d_ff,d", [(3, 256, 256), (2, 512, 768), (1, 256, 1024)])
@pytest.mark.parametrize("kind", ["normal", "wide", "special"])
def test_quantize_experts_bitexact(E, d_ff, d, kind):
    W1, W3, W2 = _weights(E, d_ff, d, kind, seed=E + d)
    s = M.make_shape(1, d, d_ff, E, 1)
    q = M.moe_quantize_experts_nvfp4(s, W1, W3, W2)
    torch.cuda.synchronize()
    gs13, gs2 = NV.weight_global_scales(u16(W1), u16(W3), u16(W2))
    assert (q["W13gs"].cpu().numpy() == gs13).all()
    assert (q["W2gs"].cpu().numpy() == gs2).all()
    c1, c3 = _unpack_w13(_unpack_codes(q["W13q"].cpu().numpy()), d_ff)
    sf13 = _atoms_to_rows(q["W13sf"].cpu().numpy(), E * 2 * d_ff, d).reshape(E, 2 * d_ff, -1)
    s1, s3 = _unpack_w13(sf13, d_ff)
    for W, c, sc in ((W1, c1, s1), (W3, c3, s3)):
        f = u16(W).astype(np.uint32) << 16
        for e in range(E):
            oc, os_ = NV.quantize(f[e].view(np.float32), gs13[e])
            assert (sc[e] == os_).all(), e
            assert (c[e] == oc).all(), e
    f2 = u16(W2).astype(np.uint32) << 16
    c2 = _unpack_codes(q["W2q"].cpu().numpy())
    s2 = _atoms_to_rows(q["W2sf"].cpu().numpy(), E * d, d_ff).reshape(E, d, -1)
    for e in range(E):
        oc, os_ = NV.quantize(f2[e].view(np.float32), gs2[e])
        assert (s2[e] == os_).all() and (c2[e] == oc).all(), e


NV_CASES = [
    # name, T, d, d_ff, E, k, capacity, d_ff_shared, zipf
    ("tiles_ragged", 700, 256, 512, 8, 2, 0, 0, 0.0),
    ("shared", 520, 256, 256, 6, 2, 0, 256, 0.5),
    ("capacity", 1000, 256, 256, 16, 4, 100, 0, 1.0),
    ("many_experts", 800, 512, 256, 64, 6, 0, 0, 1.1),
    ("one_token", 1, 512, 256, 8, 2, 0, 256, 0.0),
    ("five_tokens", 5, 256, 256, 4, 2, 0, 0, 0.0),
    ("wider", 2048, 1024, 2048, 8, 2, 0, 0, 0.3),
]


def _oracle_out(inp, logits, k, C, x_gs, h_gs, slot_priority=False):
    idx, w = O.route(logits, k)
    disp = O.dispatch(idx, inp["workload"].E, C, slot_priority=slot_priority)
    oi = I.oracle_arrays(inp)
    kw = {}
    if inp.get("W1s") is not None:
        kw = dict(W1s=oi["W1s"], W3s=oi["W3s"], W2s=oi["W2s"])
    T = logits.shape[0]
    out = NV.moe_tokens(oi["x"], oi["W1"], oi["W3"], oi["W2"], idx, w, disp["slot_pos"],
                        np.arange(T), gs_x=x_gs, gs_h=h_gs, **kw)
    return idx, disp, out


@pytest.mark.parametrize("case", NV_CASES, ids=lambda c: c[0])
@pytest.mark.parametrize("flags", [0, M.MOE_FLAG_DETERMINISTIC], ids=["default", "det"])
def test_forward_nvfp4_parity(case, flags):
    name, T, d, d_ff, E, k, C, dfs, zipf = case
    w = small_workload(name, T, d, d_ff, E, k, capacity=C, d_ff_shared=dfs, zipf_s=zipf)
    inp = I.make_inputs(w, "cuda", seed=T + d + E)
    # calibration constants: x's from its maximum, h's a fixed value
    x_gs = float(2688.0 / inp["x"].float().abs().max().item())
    h_gs = 3.0
    layer = M.MoeLayerNv4(inp, flags=flags, x_gs=x_gs, h_gs=h_gs)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    idx_o, disp, ref = _oracle_out(inp, logits.cpu().numpy(), k, C, np.float32(x_gs),
                                   np.float32(h_gs))
    assert (idx.cpu().numpy() == idx_o).all()
    if C:
        assert (disp["slot_pos"] < 0).any()
    assert_layer_close(out, ref, f"nvfp4 {name}")


def test_forward_nvfp4_slot_priority_and_repeat():
    w = small_workload("nvprio", 900, 256, 256, 16, 4, capacity=120, zipf_s=1.2)
    inp = I.make_inputs(w, "cuda", seed=9)
    layer = M.MoeLayerNv4(inp, flags=M.MOE_FLAG_SLOT_PRIORITY)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits).clone()
    out2 = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    _, disp, ref = _oracle_out(inp, logits.cpu().numpy(), w.k, w.capacity, np.float32(1.0),
                               np.float32(1.0), slot_priority=True)
    assert (disp["slot_pos"] < 0).any()
    assert_layer_close(out, ref, "nvfp4 slot priority")
    # only the combine's fp32 atomics may reorder: the same codes either way
    assert (out - out2).abs().max().item() <= 1e-5 * max(out.abs().max().item(), 1e-30)


@pytest.mark.parametrize("T", [1, 2, 8])
def test_nvfp4_small_batches(T):
    """Decode-sized batches: T <= 2 takes the NVFP4 decode kernels, T = 8 the
    block-scaled tensor-core chain; both read each chosen expert's codes once."""
    w = small_workload("nvdec", T, 1024, 2048, 16, 2, d_ff_shared=256)
    inp = I.make_inputs(w, "cuda", seed=T)
    layer = M.MoeLayerNv4(inp, h_gs=2.0)
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    _, _, ref = _oracle_out(inp, logits.cpu().numpy(), w.k, 0, np.float32(1.0), np.float32(2.0))
    assert_layer_close(out, ref, f"nvfp4 T={T}")


@pytest.mark.parametrize("T", [1, 2])
def test_nvfp4_decode_kernels_and_chain(T):
    """The NVFP4 decode kernels (w1/w3 as M = 128, N = 16 block-scaled MMAs;
    w2 as exact 16-element block dot products on the CUDA cores) and the
    tensor-core chain on the same inputs, both against the oracle, at
    d = 4096."""
    w = small_workload("nvdk", T, 4096, 1536, 8, 2, zipf_s=0.5)
    inp = I.make_inputs(w, "cuda", seed=10 + T)
    x_gs = float(2688.0 / inp["x"].float().abs().max().item())
    layer = M.MoeLayerNv4(inp, x_gs=x_gs, h_gs=2.0)
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    out_d = layer.forward(inp["x"], logits_out=logits, flags=M.MOE_FLAG_FORCE_DECODE).clone()
    out_p = layer.forward(inp["x"], flags=M.MOE_FLAG_FORCE_PREFILL).clone()
    out_0 = layer.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    _, _, ref = _oracle_out(inp, logits.cpu().numpy(), w.k, 0, np.float32(x_gs), np.float32(2.0))
    assert_layer_close(out_d, ref, f"nvfp4 decode kernels T={T}")
    assert_layer_close(out_p, ref, f"nvfp4 tensor-core chain T={T}")
    # the default path at T <= 2 is the decode kernels (deterministic: fixed order)
    assert torch.equal(out_0, out_d)


@pytest.mark.parametrize("T", [1, 2])
def test_nvfp4_decode_split_tail(T):
    """More w1/w3 tiles than SMs with some left over (2 x 152 routed + 4
    shared tiles): the decode kernel cuts the leftover tiles along K and a
    second kernel adds their pieces in a fixed order."""
    w = small_workload("nvsplit", T, 1024, 9728, 2, 2, d_ff_shared=256)
    inp = I.make_inputs(w, "cuda", seed=20 + T)
    layer = M.MoeLayerNv4(inp, h_gs=2.0)
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits).clone()
    out2 = layer.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    _, _, ref = _oracle_out(inp, logits.cpu().numpy(), w.k, 0, np.float32(1.0), np.float32(2.0))
    assert_layer_close(out, ref, f"nvfp4 decode split T={T}")
    assert torch.equal(out, out2)


@pytest.mark.parametrize("C", [0, 1])
def test_nvfp4_decode_shared_many_experts(C):
    """Decode kernels with 64 experts, top-8, a shared expert and (C = 1) a
    capacity that drops the second token's repeated experts."""
    w = small_workload("nvdec2", 2, 1024, 512, 64, 8, capacity=C, d_ff_shared=256, zipf_s=3.0)
    inp = I.make_inputs(w, "cuda", seed=2)
    layer = M.MoeLayerNv4(inp, h_gs=1.5)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    _, disp, ref = _oracle_out(inp, logits.cpu().numpy(), w.k, C, np.float32(1.0), np.float32(1.5))
    if C:
        assert (disp["slot_pos"] < 0).any()
    assert_layer_close(out, ref, f"nvfp4 decode shared C={C}")


def test_nvfp4_is_closer_to_bf16_than_its_error_bound():
    """The NVFP4 layer against the bf16 layer on the same inputs: a few
    percent apart (4-bit values, 16-element blocks), far from unrelated."""
    w = small_workload("nvbf", 512, 512, 512, 8, 2)
    inp = I.make_inputs(w, "cuda", seed=4)
    out4 = M.MoeLayerNv4(inp).forward(inp["x"])
    out16 = M.MoeLayer(inp).forward(inp["x"])
    torch.cuda.synchronize()
    rel = ((out4 - out16).norm() / out16.norm()).item()
    assert 0.01 < rel < 0.3, rel


def test_nvfp4_flag_checks():
    w = small_workload("nvbad", 64, 256, 256, 4, 2)
    inp = I.make_inputs(w, "cuda", seed=1)
    layer = M.MoeLayerNv4(inp)
    x = inp["x"]
    out = torch.empty(64, 256, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError):
        M.moe_forward_nvfp4(M.shape_of(w, 0), x, layer.Wg, None, layer.q, None, 1.0, 1.0, out,
                            None, None, layer.status, layer.ws)
    with pytest.raises(M.MoeError):
        layer.forward(x, flags=M.MOE_FLAG_FORCE_DECODE)
    bf = M.MoeLayer(inp)
    with pytest.raises(M.MoeError):
        M.moe_forward(M.shape_of(w, M.MOE_FLAG_NVFP4), x, bf.Wg, None, bf.W13, bf.W2, None, None,
                      out, None, None, bf.status, bf.ws)
