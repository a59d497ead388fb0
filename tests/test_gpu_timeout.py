"""The bounded pipeline waits of the tensor-core GEMM, exercised on the GPU
without a fault or a hang.

MOE_FLAG_TEST_TIMEOUT makes moe_expert_ffn's w1/w3 GEMM run with a producer
that issues no loads and with waits bounded at 50 ms. No stage ever fills, so
every CTA's MMA thread gives up its first wait on a full stage (before it has
issued any MMA), raises the CTA's abort flag and flags MOE_ERR_TIMEOUT; the
epilogue warps see the abort and stop waiting; every role reaches the final
barrier and the tensor memory is freed. Nothing asynchronous is in flight at
that point: no copy was issued and no MMA. The call therefore returns within
a fraction of a second, the status word carries the timeout bit, and the next
normal forward in the same process matches the oracle."""
import time

import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import Buffers, assert_layer_close

pytestmark = pytest.mark.gpu
TIMEOUT_BIT = 1 << M.MOE_ERR_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def test_starved_pipeline_times_out_and_the_context_stays_usable():
    w = I.TINY
    inp = I.make_inputs(w, "cuda", seed=0)
    b = Buffers(w)
    s = b.shape
    M.moe_route(s, inp["x"], inp["wg"], inp["bias"], b.logits, b.idx, b.w, b.status, b.ws)
    M.moe_permute(s, b.idx, inp["x"], b.counts, b.offsets, b.slot_pos, b.perm_token, b.x_perm,
                  b.n_kept, b.status, b.ws)
    W13 = M.moe_pack_w13(s, inp["W1"], inp["W3"])
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0

    starved = M.make_shape(w.T, w.d, w.d_ff, w.E, w.k, flags=M.MOE_FLAG_TEST_TIMEOUT)
    out = torch.zeros(w.T, w.d, dtype=torch.float32, device="cuda")
    t0 = time.perf_counter()
    M.moe_expert_ffn(starved, b.x_perm, b.offsets, W13, inp["W2"], b.perm_token, b.slot_pos, b.w,
                     None, out, b.status, b.ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    st = int(b.status.item())
    assert st & TIMEOUT_BIT, st
    assert st == TIMEOUT_BIT, st            # no other error on the way
    assert elapsed < 1.5, elapsed           # 50 ms waits, not the 2 s production bound

    # the context is intact: a normal forward in the same process matches the oracle
    layer = M.MoeLayer(inp)
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    got = layer.forward(inp["x"], logits_out=logits)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = O.forward(I.oracle_arrays(inp), logits=logits.cpu().numpy())
    assert_layer_close(got, ref["out"], "forward after the timeout")


def test_timeout_flag_is_rejected_on_the_cuda_core_path():
    w = I.TINY
    s = M.make_shape(w.T, w.d, w.d_ff, w.E, w.k,
                     flags=M.MOE_FLAG_TEST_TIMEOUT | M.MOE_FLAG_SIMT_FFN)
    z = torch.zeros(w.T * w.k, w.d, dtype=torch.bfloat16, device="cuda")
    offs = torch.zeros(w.E + 1, dtype=torch.int32, device="cuda")
    W = torch.zeros(w.E, 2 * w.d_ff, w.d, dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros(w.E, w.d, w.d_ff, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(w.T * w.k, w.d, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_expert_ffn(s, z, offs, W, W2, None, None, None, y, None, None,
                         M.alloc_workspace(s))
    assert ei.value.code == M.MOE_ERR_INVALID_ARG
