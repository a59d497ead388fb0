"""Debug consistency checks of the dispatch (MOE_FLAG_DEBUG_CHECKS and
moe_check_dispatch): expert ids in [0, E), offsets monotone and ending at
n_kept, every kept row inside its expert's segment with the right token, and
every permuted row written exactly once.

A correct dispatch, as moe_permute and moe_forward build it, passes the checks
with the results unchanged; dispatches corrupted on the host in each of the
ways the checks name raise the status bit. The check kernels bound-check every
index before they read with it, so a corrupt dispatch only sets a bit."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_mixture_experts_17_b200 import inputs as I
from sparse_mixture_experts_17_b200 import moe as M

from gpu_helpers import Buffers, small_workload

pytestmark = pytest.mark.gpu
CHECK = 1 << M.MOE_ERR_CHECK
BAD = 1 << M.MOE_ERR_BAD_EXPERT


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_17_b200 import build
    build.build()
    M.lib()


def _idx(T, E, k, seed, zipf=1.0):
    rng = np.random.default_rng(seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** -zipf
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _permute(s, idx, x, ws):
    T, k, E, d = s.T, s.k, s.E, s.d
    z = lambda *sh: torch.full(sh, -9, dtype=torch.int32, device="cuda")
    o = dict(counts=z(E), offsets=z(E + 1), slot_pos=z(T, k), perm_token=z(T * k), n_kept=z(1),
             x_perm=torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda"),
             status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    M.moe_permute(s, idx, x, o["counts"], o["offsets"], o["slot_pos"], o["perm_token"],
                  o["x_perm"], o["n_kept"], o["status"], ws)
    torch.cuda.synchronize()
    return o


@pytest.mark.parametrize("T,E,k,C,flags", [(1000, 16, 2, 0, 0), (3000, 64, 8, 300, 0),
                                           (777, 8, 2, 150, M.MOE_FLAG_SLOT_PRIORITY)],
                         ids=["uncapped", "capped", "slot_priority"])
def test_permute_with_checks_passes_and_matches(T, E, k, C, flags):
    d = 128
    idx = torch.from_numpy(_idx(T, E, k, seed=T)).cuda()
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    s0 = M.make_shape(T, d, 128, E, k, capacity=C, flags=flags)
    s1 = M.make_shape(T, d, 128, E, k, capacity=C, flags=flags | M.MOE_FLAG_DEBUG_CHECKS)
    assert M.moe_workspace_size(s1) >= M.moe_workspace_size(s0) + T * k * 4
    ref = _permute(s0, idx, x, M.alloc_workspace(s0))
    got = _permute(s1, idx, x, M.alloc_workspace(s1))
    assert int(got["status"].item()) == 0
    n = int(ref["n_kept"].item())
    for key in ("counts", "offsets", "slot_pos", "n_kept"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["perm_token"][:n], ref["perm_token"][:n])
    assert torch.equal(got["x_perm"][:n], ref["x_perm"][:n])


@pytest.mark.parametrize("name,T,E,k,C", [("fused_hist", 600, 8, 2, 0), ("hist_kernel", 900, 128, 2, 0)])
def test_forward_with_checks_passes_and_matches(name, T, E, k, C):
    """The prefill forward with the checks on: no status bit, and the same
    output bit for bit (k = 2 adds two products onto zero in either order)."""
    w = small_workload(name, T, 256, 256, E, k, capacity=C, zipf_s=1.0)
    inp = I.make_inputs(w, "cuda", seed=T)
    a = M.MoeLayer(inp)
    b = M.MoeLayer(inp, flags=M.MOE_FLAG_DEBUG_CHECKS)
    oa = a.forward(inp["x"])
    ob = b.forward(inp["x"])
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0 and int(a.status.item()) == 0
    assert torch.equal(oa, ob)


def _valid_dispatch(T=400, E=16, k=4, C=0, seed=5):
    d = 128
    flags = M.MOE_FLAG_DEBUG_CHECKS
    s = M.make_shape(T, d, 128, E, k, capacity=C, flags=flags)
    idx_np = _idx(T, E, k, seed=seed)
    idx = torch.from_numpy(idx_np).cuda()
    ws = M.alloc_workspace(s)
    o = _permute(s, idx, None, ws)
    o["idx"] = idx
    # the dispatch is the oracle's, bit for bit
    orc = O.dispatch(idx_np, E, C)
    assert (o["slot_pos"].cpu().numpy() == orc["slot_pos"]).all()
    return s, ws, o


def _check(s, ws, o, **override):
    d = {key: o[key].clone() for key in ("idx", "offsets", "slot_pos", "perm_token", "n_kept")}
    for key, fn in override.items():
        fn(d[key])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_check_dispatch(s, d["idx"], d["offsets"], d["slot_pos"], d["perm_token"], d["n_kept"],
                         status, ws)
    torch.cuda.synchronize()
    return int(status.item())


def test_check_dispatch_accepts_a_valid_dispatch():
    s, ws, o = _valid_dispatch()
    assert _check(s, ws, o) == 0
    s, ws, o = _valid_dispatch(C=60)
    assert (o["slot_pos"] < 0).any()
    assert _check(s, ws, o) == 0


def _set(i, v):
    def f(t):
        t.view(-1)[i] = v
    return f


def test_check_dispatch_flags_each_corruption():
    s, ws, o = _valid_dispatch()
    sp = o["slot_pos"].cpu().numpy()
    pt = o["perm_token"].cpu().numpy()
    off = o["offsets"].cpu().numpy()
    nk = int(o["n_kept"].item())
    N = s.T * s.k
    # two rows of different tokens swapped in perm_token
    r0 = int(sp[0, 0])
    r1 = int(sp[1, 0]) if pt[int(sp[1, 0])] != pt[r0] else int(sp[2, 0])
    swap = lambda t: t.copy_(t[torch.tensor(
        [r1 if i == r0 else r0 if i == r1 else i for i in range(N)], device="cuda")])
    assert _check(s, ws, o, perm_token=swap) & CHECK
    # one row claimed twice (and another row by no one)
    assert _check(s, ws, o, slot_pos=_set(1, int(sp.flat[0]))) & CHECK
    # offsets not monotone
    e = int(np.nonzero(np.diff(off) > 0)[0][0])
    assert _check(s, ws, o, offsets=_set(e + 1, int(off[e + 1]) + 10 ** 6)) & CHECK
    # offsets[0] != 0
    assert _check(s, ws, o, offsets=_set(0, 1)) & CHECK
    # n_kept disagrees with offsets[E], and n_kept beyond T * k
    assert _check(s, ws, o, n_kept=_set(0, nk - 1)) & CHECK
    assert _check(s, ws, o, n_kept=_set(0, N + 7)) & CHECK
    # an expert id outside [0, E)
    assert _check(s, ws, o, idx=_set(3, s.E)) & BAD
    assert _check(s, ws, o, idx=_set(3, -2)) & BAD
    # a slot outside [0, T k), a negative slot other than -1, and a drop without capacity
    assert _check(s, ws, o, slot_pos=_set(2, N + 5)) & CHECK
    assert _check(s, ws, o, slot_pos=_set(2, -3)) & CHECK
    assert _check(s, ws, o, slot_pos=_set(2, -1)) & CHECK
    # a slot outside its own expert's segment (the first row of another expert)
    e0 = int(o["idx"].view(-1)[0].item())
    other = int(off[(e0 + 1) % s.E]) if off[(e0 + 1) % s.E] != off[e0] else 0
    if not (off[e0] <= other < off[e0 + 1]):
        assert _check(s, ws, o, slot_pos=_set(0, other)) & CHECK


def test_check_dispatch_flags_capacity_overflow():
    s, ws, o = _valid_dispatch(C=60)
    off = o["offsets"].cpu().numpy()
    # a segment made longer than C by moving the boundary after it
    e = int(np.argmax(np.diff(off)))
    assert _check(s, ws, o, offsets=_set(e + 1, int(off[e]) + s.capacity + 1)) & CHECK


def test_check_dispatch_needs_the_flag_in_the_shape():
    s, ws, o = _valid_dispatch()
    s2 = M.make_shape(s.T, s.d, s.d_ff, s.E, s.k, capacity=s.capacity)
    with pytest.raises(M.MoeError) as ei:
        M.moe_check_dispatch(s2, o["idx"], o["offsets"], o["slot_pos"], o["perm_token"],
                             o["n_kept"], o["status"], ws)
    assert ei.value.code == M.MOE_ERR_INVALID_ARG
