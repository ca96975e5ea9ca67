"""The N > 1 paths, on CPU ranks over gloo.

With N GPUs bench.py runs an independent replica of the layer per rank, so
its only cross-rank work is the max over ranks of the device times and the
whole-job rate computed from it.  These tests run that logic with
world_size 2 on the gloo backend, run the reference arm under torchrun
(rank 0 alone times the oracle), and run the exchange step of the layer's
all_reduce form (ep_allreduce.all_reduce_partial) on partials the oracle
computes for each rank.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r is slower on the first timer and faster on the second
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], torch.device("cpu"))
        rate = bench.whole_job_rate(1000, world, got[0])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, rate in res:
        assert got == [2.0, 10.0, 5.0]            # every rank sees the slowest rank's times
        assert rate == pytest.approx(2 * 1000 / 2e-3)   # all ranks' tokens / max time


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5], torch.device("cpu")) == [3.0, 4.5]
    assert bench.whole_job_rate(8192, 1, 8.0) == pytest.approx(8192 / 8e-3)


def test_reference_arm_under_torchrun_world2():
    """Two ranks under torchrun: rank 0 times the oracle on a bounded sample
    and prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "1",
           "--warmup", "1", "--ref-seconds", "0.2"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "tiny"


def _allreduce_rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from expert_parallelism_b200 import ep_allreduce
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the same batch on both ranks; dyadic values keep every sum exact
        T, k, E, H = 50, 4, 8, 16
        g = torch.Generator().manual_seed(31)
        idx, _ = oracle.route_topk(torch.randn(T, E, generator=g), k)
        lay = oracle.dispatch_layout(idx, E, world)
        y = torch.randint(-64, 65, (T * k, H), generator=g).float() / 8
        w = torch.randint(1, 16, (T, k), generator=g).float() / 16
        part = oracle.combine_rank(y, lay["slot_of_pair"], w, lay["rank_offsets"], rank, "f32")
        ep_allreduce.all_reduce_partial(part)
        whole = oracle.combine(y, lay["slot_of_pair"], w, "f32")
        q.put((rank, bool(torch.equal(part, whole)), int((part != 0).any(dim=1).sum())))
    finally:
        dist.destroy_process_group()


def test_all_reduce_form_exchange_gloo_world2():
    """Each rank's partial covers its own experts' picks only; after the
    all-reduce both ranks hold the full combine, bit for bit."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_allreduce_rank_main, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [True, True]
