"""The three large workloads at full size, in the configuration the benchmark
times (moe_forward, default flags), against the oracle.

Routing (logits -> top-k -> histogram -> offsets -> permutation -> drops) is
compared on ALL tokens, bit for bit, on identical fp32 logits (the oracle's
own fp32-rounded logits, fed to moe_route with x = NULL). Layer outputs are
compared on a token sample the oracle evaluates one by one: a token's output
depends only on its own row and the global drop set, so the sample is exact.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import (LOGIT_ABS, assert_layer_close, oracle_tokens_subset,
                         pipeline_from_logits, sample_tokens, u16)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("wl", [I.PREFILL, I.FINE_GRAINED, I.CAPACITY], ids=lambda w: w.name)
def test_full_size(wl):
    torch.cuda.empty_cache()
    inp = I.make_inputs(wl, "cuda", seed=0)
    bias = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    L64, L32 = O.router_logits(u16(inp["x"]), u16(inp["wg"]), bias)
    idx_o, w_o = O.route(L32, wl.k)
    disp = O.dispatch(idx_o, wl.E, wl.capacity)

    # (1) the step-by-step pipeline on the oracle's fp32 logits
    b = pipeline_from_logits(inp, torch.from_numpy(L32).cuda())
    assert int(b.status.item()) == 0
    assert (b.idx.cpu().numpy() == idx_o).all()
    assert (b.counts.cpu().numpy() == disp["counts"]).all()
    assert (b.offsets.cpu().numpy() == disp["offsets"]).all()
    assert (b.slot_pos.cpu().numpy() == disp["slot_pos"]).all()
    n = disp["n_kept"]
    assert (b.perm_token.cpu().numpy()[:n] == disp["perm_token"][:n]).all()
    tokens = sample_tokens(wl.T, disp, n_random=16)
    ref = oracle_tokens_subset(inp, idx_o, w_o, disp["slot_pos"], tokens)
    assert_layer_close(b.out[torch.from_numpy(tokens.astype(np.int64)).cuda()], ref,
                       f"{wl.name} pipeline")
    out_pipe = b.out
    del b

    # (2) moe_forward end to end, as the benchmark runs it
    layer = M.MoeLayer(inp)
    logits = torch.empty(wl.T, wl.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    out = layer.forward(inp["x"], logits_out=logits, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    assert np.abs(logits.double().cpu().numpy() - L64).max() <= LOGIT_ABS
    same = (idx.cpu().numpy() == idx_o).all(1)
    # a routing difference can only come from a near-tie of fp32 accumulations
    assert same.mean() > 0.999, same.mean()
    if same.all():
        assert_layer_close(out[torch.from_numpy(tokens.astype(np.int64)).cuda()], ref,
                           f"{wl.name} forward")
    else:
        keep = tokens[same[tokens]] if not wl.capacity else np.array([], np.int32)
        if len(keep):
            sel = np.searchsorted(tokens, keep)
            assert_layer_close(out[torch.from_numpy(keep.astype(np.int64)).cuda()], ref[sel],
                               f"{wl.name} forward (tokens with identical routing)")
    # the fused path and the step-by-step path agree everywhere routing agrees
    rows = torch.from_numpy(np.nonzero(same)[0]).cuda()
    if not wl.capacity and len(rows):
        d = (out[rows] - out_pipe[rows]).abs().max().item()
        assert d <= 2e-2, d
