"""Seeded synthetic inputs for the MoE layer, and the workload shapes.

This module is shared by the tests, the benchmark, the oracle checks and the
CUDA path. It draws random numbers and holds shapes only: none of the layer's
arithmetic lives here.

Recipe (one generator, seeded, draws in this fixed order):
  x   [T, d]        ~ N(0, 1)            -> bf16
  W_g [E, d]        ~ N(0, 0.02)         -> bf16   (nn.Linear layout [out, in])
  W1  [E, d_ff, d]  ~ N(0, 0.02) per expert, expert 0 first -> bf16
  W3  [E, d_ff, d]  same
  W2  [E, d, d_ff]  same
  shared expert W1s [d_ff_s, d], W3s [d_ff_s, d], W2s [d, d_ff_s], same law
  bias b[E] (fp32): zero, or for a Zipf(s) load skew b[e] = -s * ln(r_e) with
  r a permutation of 1..E drawn from a CPU generator seeded with seed + 1;
  softmax(b) alone is then exactly Zipf(s) over the experts.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    d_ff: int
    E: int
    k: int
    capacity: int = 0        # <= 0: uncapped
    d_ff_shared: int = 0     # 0: no shared expert
    zipf_s: float = 0.0      # 0: no router bias

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")


def capacity_for(T: int, k: int, E: int, factor: float = 1.25) -> int:
    """Per-expert capacity ceil(factor * T * k / E)."""
    return int(math.ceil(factor * T * k / E))


# The five workloads the layer is measured and checked on.
TINY = Workload("tiny", T=64, d=128, d_ff=256, E=8, k=2)
DECODE = Workload("decode", T=1, d=4096, d_ff=14336, E=8, k=2)
PREFILL = Workload("prefill", T=16384, d=4096, d_ff=14336, E=8, k=2)
FINE_GRAINED = Workload("fine_grained", T=8192, d=7168, d_ff=2048, E=256, k=8,
                        d_ff_shared=2048, zipf_s=1.1)
CAPACITY = Workload("capacity", T=4096, d=2048, d_ff=768, E=128, k=8,
                    capacity=capacity_for(4096, 8, 128), zipf_s=1.0)
DECODE_TS = (1, 2, 4, 8)

WORKLOADS = {w.name: w for w in (TINY, DECODE, PREFILL, FINE_GRAINED, CAPACITY)}


def zipf_bias(E: int, s: float, seed: int) -> torch.Tensor:
    if s == 0.0:
        return torch.zeros(E, dtype=torch.float32)
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    r = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    return (-s * torch.log(r)).to(torch.float32)


def make_inputs(w: Workload, device="cpu", seed: int = 0, with_bias: bool | None = None,
                router_only: bool = False) -> dict:
    """Draw the workload's tensors on ``device`` (bf16 weights, fp32 bias).
    router_only: stop after x and W_g (the same values as the full draw) and
    the bias; no expert weights."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(seed)
    bf = torch.bfloat16

    def normal(shape, std):
        t = torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t.to(bf)

    def stacked(E, rows, cols):
        out = torch.empty(E, rows, cols, dtype=bf, device=dev)
        for e in range(E):
            out[e] = normal((rows, cols), 0.02)
        return out

    inp = dict(workload=w)
    inp["x"] = normal((w.T, w.d), 1.0)
    inp["wg"] = normal((w.E, w.d), 0.02)
    if router_only:
        use_bias = (w.zipf_s != 0.0) if with_bias is None else with_bias
        inp["bias"] = zipf_bias(w.E, w.zipf_s, seed).to(dev) if use_bias else None
        inp["k"] = w.k
        inp["capacity"] = w.capacity
        return inp
    inp["W1"] = stacked(w.E, w.d_ff, w.d)
    inp["W3"] = stacked(w.E, w.d_ff, w.d)
    inp["W2"] = stacked(w.E, w.d, w.d_ff)
    if w.d_ff_shared:
        inp["W1s"] = normal((w.d_ff_shared, w.d), 0.02)
        inp["W3s"] = normal((w.d_ff_shared, w.d), 0.02)
        inp["W2s"] = normal((w.d, w.d_ff_shared), 0.02)
    use_bias = (w.zipf_s != 0.0) if with_bias is None else with_bias
    inp["bias"] = zipf_bias(w.E, w.zipf_s, seed).to(dev) if use_bias else None
    inp["k"] = w.k
    inp["capacity"] = w.capacity
    return inp


def to_numpy_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def oracle_arrays(inp: dict) -> dict:
    """The same tensors as host numpy arrays in the oracle's conventions."""
    out = {}
    for key in ("x", "wg", "W1", "W3", "W2", "W1s", "W3s", "W2s"):
        if key in inp and inp[key] is not None:
            out[key] = to_numpy_u16(inp[key])
    out["bias"] = None if inp.get("bias") is None else inp["bias"].detach().cpu().numpy()
    out["k"] = inp["k"]
    out["capacity"] = inp["capacity"]
    return out
