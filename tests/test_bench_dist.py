"""The multi-rank host logic of bench.py (replicas: max-over-ranks time, summed
tokens, rank 0 prints) on CPU with the gloo backend, world size 2."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(use_cuda=False)
    assert (w, r) == (world, rank)
    t = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
    n = bench.sum_over_ranks(1000.0, world, torch.device("cpu"))
    bench.barrier(world)
    q.put((rank, t, n))
    dist.destroy_process_group()


def test_max_and_sum_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 11.0, 2000.0), (1, 11.0, 2000.0)]


def test_reference_arm_rank0_prints_other_ranks_exit():
    """`--impl reference` under two ranks: rank 0 prints one JSON line, rank 1 exits 0."""
    port = _free_port()
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "1",
           "--ref-step-s", "0.2"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    # the line describes what ran: K steps of one sample each, K * ms_per_step
    # is the timed region, and the config has the keys our arm prints
    assert d["steps"] == 3 and d["warmup"] == 1
    assert abs(d["steps"] * d["ms_per_step"] / 1e3 - d["timed_region_s"]) <= 0.5 * d["timed_region_s"]
    assert abs(d["sample_tokens_per_step"] / (d["ms_per_step"] / 1e3) - d["value"]) <= 1e-3 * d["value"] + 1e-3
    sys.path.insert(0, ROOT)
    import bench
    from sparse_mixture_experts_17_b200 import inputs as I
    assert d["config"] == bench.config_of(I.TINY, 2)


def test_summary_lists_the_five_workloads():
    """The compact summary printed last in the bench line names every workload."""
    sys.path.insert(0, ROOT)
    import bench
    res = {"ms_per_step": 9.0, "value": 1.8e6, "active_tflops": 1200.0,
           "roofline": {"frac": 0.8},
           "configs": {n: {"ms_per_step": 1.0, "tokens_per_s": 2.0, "frac_of_roof": 0.5,
                           "roof_bound": "hbm"} for n in ("tiny", "fine_grained", "capacity")},
           "decode": {f"T{t}": {"ms_per_step": 0.1, "frac_hbm_measured": 0.7} for t in (1, 2, 4, 8)}}
    sm = bench.summarize(res)
    assert set(sm) == {"C1_tiny", "C2_decode", "C3_prefill", "C4_fine_grained", "C5_capacity"}
    assert len(json.dumps(sm)) < 1200
