"""moe_permute_static: the permute for callers that cannot allocate device
memory (stream capture in global mode, engines owning all device memory,
paths that cannot pay for cudaMalloc/cudaFree). It must give exactly what
moe_permute gives with a caller workspace, call after call, although every
call reuses the same fixed scratch array inside the library."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_17_b200 import moe as M

pytestmark = pytest.mark.gpu


def _idx(T, E, k, seed):
    rng = np.random.default_rng(seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.0
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _outputs(T, E, k, d):
    z = lambda *s: torch.full(s, -9, dtype=torch.int32, device="cuda")
    return dict(counts=z(E), offsets=z(E + 1), slot_pos=z(T, k), perm_token=z(T * k), n_kept=z(1),
                x_perm=torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("T,E,k,C", [(3000, 64, 8, 300), (777, 8, 2, 0)])
def test_static_permute_matches_workspace_permute_twice(T, E, k, C):
    from sparse_mixture_experts_17_b200 import build
    build.build()
    d = 256
    s = M.make_shape(T, d, 256, E, k, capacity=C)
    idx = torch.from_numpy(_idx(T, E, k, seed=T + E)).cuda()
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = _outputs(T, E, k, d)
    M.moe_permute(s, idx, x, ref["counts"], ref["offsets"], ref["slot_pos"], ref["perm_token"],
                  ref["x_perm"], ref["n_kept"], status, M.alloc_workspace(s))
    torch.cuda.synchronize()
    n = int(ref["n_kept"].item())
    for call in range(2):
        got = _outputs(T, E, k, d)
        M.moe_permute_static(s, idx, x, got["counts"], got["offsets"], got["slot_pos"],
                             got["perm_token"], got["x_perm"], got["n_kept"], status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for key in ("counts", "offsets", "slot_pos", "n_kept"):
            assert torch.equal(got[key], ref[key]), (call, key)
        assert torch.equal(got["perm_token"][:n], ref["perm_token"][:n]), call
        assert torch.equal(got["x_perm"][:n], ref["x_perm"][:n]), call


def test_static_permute_rejects_oversize():
    s = M.make_shape(1 << 19, 128, 128, 8, 2)   # T*k = 2^20: its scratch exceeds the 4 MiB array
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_permute_static(s, dummy, None, dummy, dummy, dummy, dummy, None, None, None)
    assert ei.value.code == M.MOE_ERR_UNSUPPORTED
