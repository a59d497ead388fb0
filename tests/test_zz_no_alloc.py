"""moe_permute_static: the permute for callers that cannot allocate device
memory (engines owning all device memory, paths that cannot pay for
cudaMalloc/cudaFree). It must give exactly what moe_permute gives with a
caller workspace, and what the oracle's dispatch computes, call after call,
although every call reuses the same fixed scratch array inside the library."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
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


@pytest.mark.parametrize("T,E,k,C,slot", [(3000, 64, 8, 300, False), (777, 8, 2, 0, False),
                                          (16384, 256, 16, 1280, True)],
                         ids=["capped", "uncapped", "slot_priority_at_bound"])
def test_static_permute_matches_workspace_permute_twice(T, E, k, C, slot):
    """The last case sits at the documented bound T * k = 262144 with the
    slot-major count rows (k per chunk), the largest scratch layout."""
    from sparse_mixture_experts_17_b200 import build
    build.build()
    O.build()
    d = 256
    s = M.make_shape(T, d, 256, E, k, capacity=C, flags=M.MOE_FLAG_SLOT_PRIORITY if slot else 0)
    idx_np = _idx(T, E, k, seed=T + E)
    idx = torch.from_numpy(idx_np).cuda()
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = _outputs(T, E, k, d)
    M.moe_permute(s, idx, x, ref["counts"], ref["offsets"], ref["slot_pos"], ref["perm_token"],
                  ref["x_perm"], ref["n_kept"], status, M.alloc_workspace(s))
    torch.cuda.synchronize()
    n = int(ref["n_kept"].item())
    orc = O.dispatch(idx_np, E, C, slot_priority=slot)
    if C:
        assert (orc["slot_pos"] < 0).any()
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
        # and the oracle's dispatch of the same indices, bit for bit
        assert n == orc["n_kept"]
        assert (got["counts"].cpu().numpy() == orc["counts"]).all(), call
        assert (got["offsets"].cpu().numpy() == orc["offsets"]).all(), call
        assert (got["slot_pos"].cpu().numpy() == orc["slot_pos"]).all(), call
        assert (got["perm_token"][:n].cpu().numpy() == orc["perm_token"][:n]).all(), call
        kept_counts = np.minimum(orc["counts"], C) if C else orc["counts"]
        assert (np.diff(got["offsets"].cpu().numpy()) == kept_counts).all(), call
        rows = torch.from_numpy(orc["perm_token"][:n].astype(np.int64)).cuda()
        assert torch.equal(got["x_perm"][:n], x[rows]), call


def test_static_permute_rejects_oversize():
    s = M.make_shape(1 << 19, 128, 128, 8, 2)   # T*k = 2^20: its scratch exceeds the 4 MiB array
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_permute_static(s, dummy, None, dummy, dummy, dummy, dummy, None, None, None)
    assert ei.value.code == M.MOE_ERR_UNSUPPORTED
