"""The C ABI on a machine without a GPU: the library loads, exports every entry
point the header declares, and rejects bad arguments on the host (no compute
call is made here)."""
import ctypes
import os
import subprocess
import sys

import pytest

from sparse_mixture_experts_17_b200 import build as B
from sparse_mixture_experts_17_b200 import moe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.lib()


def test_exports_every_header_entry_point(lib):
    names = M.header_entry_points()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    # and nothing else is exported (the static CUDA runtime stays private)
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(line.split()[-1] for line in out.splitlines() if line.strip())
    assert exported == names


def test_status_strings(lib):
    assert M.status_string(M.MOE_OK) == "ok"
    assert "workspace" in M.status_string(M.MOE_ERR_WORKSPACE)
    assert M.status_string(99) == "unknown status"


def test_workspace_size_scales(lib):
    a = M.moe_workspace_size(M.make_shape(64, 128, 256, 8, 2))
    b = M.moe_workspace_size(M.make_shape(6400, 128, 256, 8, 2))
    assert b > a > 0
    c = M.moe_workspace_size(M.make_shape(6400, 128, 256, 8, 2, flags=M.MOE_FLAG_DETERMINISTIC))
    assert c >= b + 6400 * 2 * 128 * 4
    h = M.moe_workspace_size(M.make_shape(6400, 128, 256, 8, 2, flags=M.MOE_FLAG_HOST_IO))
    assert h >= b + 6400 * 128 * 6


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(d=100), dict(d=0), dict(d_ff=200), dict(E=0), dict(E=257),
    dict(k=0), dict(k=9, E=8), dict(k=17, E=64), dict(d_ff_shared=64), dict(T=(1 << 24) + 1),
    dict(d=32896),
])
def test_invalid_shapes(lib, bad):
    kw = dict(T=64, d=128, d_ff=256, E=8, k=2)
    kw.update(bad)
    s = M.make_shape(**kw)
    n = ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(s), ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG


FAKE = 0x100000  # an aligned non-null address that is never dereferenced


def _forward(lib, s, ws=FAKE, ws_bytes=1 << 40, x=FAKE, wg=FAKE, w13=FAKE, w2=FAKE, out=FAKE,
             w13s=None, w2s=None):
    return lib.moe_forward(ctypes.byref(s), x, wg, None, w13, w2, w13s, w2s, out, None, None,
                           None, ws, ws_bytes, None)


def test_forward_host_validation(lib):
    s = M.make_shape(64, 128, 256, 8, 2)
    assert _forward(lib, s, x=None) == M.MOE_ERR_INVALID_ARG
    assert _forward(lib, s, out=None) == M.MOE_ERR_INVALID_ARG
    assert _forward(lib, s, x=FAKE + 8) == M.MOE_ERR_INVALID_ARG      # misaligned
    assert _forward(lib, s, ws=None) == M.MOE_ERR_WORKSPACE
    assert _forward(lib, s, ws=FAKE + 16) == M.MOE_ERR_WORKSPACE      # not 256-B aligned
    assert _forward(lib, s, ws_bytes=1024) == M.MOE_ERR_WORKSPACE
    sh = M.make_shape(64, 128, 256, 8, 2, d_ff_shared=256)
    assert _forward(lib, sh) == M.MOE_ERR_INVALID_ARG                 # shared weights missing
    # T = 0 is a valid no-op that touches no device
    assert _forward(lib, M.make_shape(0, 128, 256, 8, 2)) == M.MOE_OK


def test_other_entry_points_validation(lib):
    s = M.make_shape(64, 128, 256, 8, 2)
    # moe_route: logits is required; x without Wg is rejected
    assert lib.moe_route(ctypes.byref(s), None, None, None, None, FAKE, FAKE, None, FAKE, 1 << 40,
                         None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_route(ctypes.byref(s), FAKE, None, None, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                         None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_route(ctypes.byref(s), None, None, None, FAKE, FAKE, FAKE, None, FAKE, 16,
                         None) == M.MOE_ERR_WORKSPACE
    # moe_permute: outputs required; x without x_perm rejected
    assert lib.moe_permute(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None,
                           FAKE, 1 << 40, None) == M.MOE_ERR_INVALID_ARG
    # moe_expert_ffn: the fused combine needs out, perm_token, slot_pos, topk_w
    assert lib.moe_expert_ffn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, None, None, None,
                              FAKE, None, FAKE, 1 << 40, None) == M.MOE_ERR_INVALID_ARG
    # moe_combine
    assert lib.moe_combine(ctypes.byref(s), None, FAKE, FAKE, None, FAKE, None) == \
        M.MOE_ERR_INVALID_ARG
    # moe_pack_w13
    assert lib.moe_pack_w13(ctypes.byref(s), FAKE, None, FAKE, None) == M.MOE_ERR_INVALID_ARG
    # moe_forward_host needs the HOST_IO workspace flag
    assert lib.moe_forward_host(ctypes.byref(s), FAKE, FAKE, None, FAKE, FAKE, None, None, FAKE,
                                None, FAKE, 1 << 40, None) == M.MOE_ERR_INVALID_ARG
    # NVFP4: dimensions must be multiples of 256; the flag is required; the
    # activations' global scales must be positive and finite
    f, P = ctypes.c_float, [FAKE] * 6
    def nv(shape, xgs=1.0, hgs=1.0):
        return lib.moe_forward_nvfp4(ctypes.byref(shape), FAKE, FAKE, None, *P, *P, f(xgs), f(hgs),
                                     FAKE, None, None, FAKE, FAKE, 1 << 40, None)
    assert nv(M.make_shape(64, 128, 256, 8, 2, flags=M.MOE_FLAG_NVFP4)) == M.MOE_ERR_UNSUPPORTED
    assert nv(M.make_shape(64, 256, 384, 8, 2, flags=M.MOE_FLAG_NVFP4)) == M.MOE_ERR_UNSUPPORTED
    s4 = M.make_shape(64, 256, 512, 8, 2, flags=M.MOE_FLAG_NVFP4)
    assert nv(M.make_shape(64, 256, 512, 8, 2)) == M.MOE_ERR_INVALID_ARG
    assert nv(s4, xgs=0.0) == M.MOE_ERR_INVALID_ARG
    assert nv(s4, hgs=float("inf")) == M.MOE_ERR_INVALID_ARG
    assert nv(M.make_shape(64, 256, 512, 8, 2, flags=M.MOE_FLAG_NVFP4 | M.MOE_FLAG_MXFP8)) == \
        M.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_experts_nvfp4(ctypes.byref(s4), FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                          FAKE, FAKE, FAKE, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_quantize_experts_nvfp4(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                          FAKE, FAKE, FAKE, None) == M.MOE_ERR_UNSUPPORTED
    # the NVFP4 workspace is smaller than the bf16 one (no bf16 copies of x and h)
    sb = M.make_shape(4096, 4096, 14336, 8, 2)
    assert M.moe_workspace_size(s4) > 0
    assert M.moe_workspace_size(M.make_shape(4096, 4096, 14336, 8, 2, flags=M.MOE_FLAG_NVFP4)) < \
        M.moe_workspace_size(sb)
    # FORCE_DECODE above the decode limit is unsupported (checked before launching)
    sd = M.make_shape(64, 128, 256, 8, 2, flags=M.MOE_FLAG_FORCE_DECODE)
    ws = M.moe_workspace_size(sd)
    # a workspace size check passes with a fake aligned pointer, then the path is refused
    assert _forward(lib, sd, ws_bytes=ws) == M.MOE_ERR_UNSUPPORTED


def test_product_does_not_import_oracle():
    """The product path (binding + inputs) never imports or loads the oracle."""
    code = ("import sys; import sparse_mixture_experts_17_b200.moe as m; "
            "import sparse_mixture_experts_17_b200.inputs; m.lib(); "
            "assert not any(k == 'oracle' or k.startswith('oracle.') for k in sys.modules), "
            "sorted(k for k in sys.modules if 'oracle' in k)")
    subprocess.run([sys.executable, "-c", code], cwd=ROOT, check=True)
    for dirpath, _, files in os.walk(os.path.join(ROOT, "sparse_mixture_experts_17_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                for needle in ("import oracle", "from oracle", "liboracle", "moe_oracle"):
                    assert needle not in text, (f, needle)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="libmoe.so not found"):
        M.lib()


def _header_signatures():
    """{name: [parameter declarations]} of every MOE_API function in moe.h."""
    import re
    text = open(M.HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)   # drop comments
    sigs = {}
    for m in re.finditer(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(([^)]*)\)", text):
        params = [p.strip() for p in m.group(2).split(",")]
        sigs[m.group(1)] = [] if params == ["void"] else params
    return sigs


def test_binding_signatures_match_header():
    """Every ctypes signature in the binding has the header's parameter count,
    and each parameter's kind matches: pointers (and the stream handle) as
    pointers, size_t / int / float as themselves. A miscounted argument list
    would pass garbage on the GPU instead of failing here."""
    sigs = _header_signatures()
    assert set(sigs) == set(M._SIGS), set(sigs) ^ set(M._SIGS)
    for name, params in sigs.items():
        args = M._SIGS[name][0]
        assert len(args) == len(params), (name, len(args), len(params))
        for decl, a in zip(params, args):
            if "*" in decl or decl.startswith("moe_stream_t"):
                assert a in (ctypes.c_void_p, ctypes.c_char_p) or \
                    issubclass(a, ctypes._Pointer), (name, decl, a)
            elif decl.startswith("size_t"):
                assert a is ctypes.c_size_t, (name, decl, a)
            elif decl.startswith("float"):
                assert a is ctypes.c_float, (name, decl, a)
            elif decl.startswith("int"):
                assert a is ctypes.c_int, (name, decl, a)
            else:
                raise AssertionError(f"unexpected parameter {decl!r} of {name}")


@pytest.mark.parametrize("flags", [0, M.MOE_FLAG_DETERMINISTIC, M.MOE_FLAG_MXFP8, M.MOE_FLAG_NVFP4,
                                   M.MOE_FLAG_BACKWARD, M.MOE_FLAG_EXPERT_CHOICE,
                                   M.MOE_FLAG_HOST_IO, M.MOE_FLAG_SLOT_PRIORITY])
@pytest.mark.parametrize("dims", [(256, 512, 8, 2, 0, 0), (512, 256, 64, 6, 0, 256),
                                  (256, 256, 16, 4, 100, 0)])
def test_workspace_never_shrinks_with_T(lib, flags, dims):
    """A layer sizes its workspace once for T_max and runs smaller batches in
    it, so the size must be non-decreasing in T for every flag."""
    d, d_ff, E, k, C, dfs = dims
    prev = 0
    for T in [1, 2, 3, 16, 17, 100, 127, 128, 129, 255, 256, 257, 1000, 4096, 4097, 16384]:
        if flags & M.MOE_FLAG_EXPERT_CHOICE and C <= 0:
            C = 64
        n = M.moe_workspace_size(M.make_shape(T, d, d_ff, E, k, C, dfs, flags))
        assert n >= prev, (T, n, prev)
        prev = n
