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


def _ep_rank_main(rank, world, port, payload, q):
    """One expert-parallel rank on CPU: its own tokens, the count exchange
    over gloo (expert_parallelism_b200.ep.exchange_counts), the oracle's
    plan, the rows sent to their owners as point-to-point messages (one per
    peer: the sender's rank slab), the owner's experts on what it received,
    the outputs sent back the same way, and the combine."""
    sys.path.insert(0, ROOT)
    import oracle
    from expert_parallelism_b200 import ep, workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        base = workloads.Workload("ep", 24, 256, 8, 2, 64, world, "bf16", payload, "bf16")
        full = workloads.layer_inputs(base)                    # every expert's weights
        mine = base.replace(seed=100 + rank)
        inp = {"logits": workloads.router_logits(mine), "x": workloads.hidden_states(mine)}
        E, k, H, Er = base.E, base.k, base.H, base.E // world
        idx, w = oracle.route_topk(inp["logits"], k)
        lay = oracle.dispatch_layout(idx, E, world)
        counts_all = torch.empty(world, E, dtype=torch.int32)
        ep.exchange_counts(lay["expert_counts"], counts_all)
        plans = [oracle.ep_plan(counts_all, s) for s in range(world)]
        recv_off = plans[rank][1]
        xp, sc = oracle.permute(inp["x"], k, lay["pair_of_slot"], payload)
        rows = xp.view(torch.uint8) if payload == "e4m3" else xp.view(torch.int16)
        if sc is not None:      # scales travel in the same message, as raw bits
            rows = torch.cat([rows, sc.view(torch.uint8 if payload == "e4m3" else torch.int16)
                              .reshape(rows.shape[0], -1)], dim=1)
        ro = lay["rank_offsets"].tolist()

        def exchange(send_for, recv_len, width, dtype):
            """Point-to-point: send_for(d) to every peer d, receive recv_len(s)
            rows from every peer s (the own share is copied locally)."""
            got = {rank: send_for(rank)}
            ops = []
            for d in range(world):
                if d == rank:
                    continue
                got[d] = torch.empty(recv_len(d), width, dtype=dtype)
                ops.append(dist.P2POp(dist.isend, send_for(d).contiguous(), d))
                ops.append(dist.P2POp(dist.irecv, got[d], d))
            for wk in dist.batch_isend_irecv(ops) if ops else []:
                wk.wait()
            return got

        rows_from = lambda s: int(counts_all[s, rank * Er:(rank + 1) * Er].sum())
        got = exchange(lambda d: rows[ro[d]:ro[d + 1]], rows_from, rows.shape[1], rows.dtype)
        # place every source's chunk of every local expert by the plan
        n_recv = int(recv_off[-1])
        recv = torch.empty(n_recv, rows.shape[1], dtype=rows.dtype)
        for s in range(world):
            pos = 0
            for j in range(Er):
                e, c = rank * Er + j, int(counts_all[s, rank * Er + j])
                b = int(plans[s][0][e])
                recv[b:b + c] = got[s][pos:pos + c]
                pos += c
        if payload == "e4m3":
            codes = recv[:, :H].contiguous().view(torch.float8_e4m3fn)
            rsc = recv[:, H:].contiguous().view(torch.float32)
        else:
            codes, rsc = recv.contiguous().view(torch.bfloat16), None
        _, y, _ = oracle.grouped_gemm(codes, rsc, recv_off, 0, Er,
                                      full["w13"][rank * Er:(rank + 1) * Er].contiguous(),
                                      full["w2"][rank * Er:(rank + 1) * Er].contiguous())

        def y_for(s):       # owner -> source s: its chunks, local expert by expert
            parts = []
            for j in range(Er):
                e, c = rank * Er + j, int(counts_all[s, rank * Er + j])
                b = int(plans[s][0][e])
                parts.append(y[b:b + c])
            return torch.cat(parts)

        back = exchange(y_for, lambda d: int(ro[d + 1] - ro[d]), H, torch.float64)
        y_home = torch.zeros(xp.shape[0], H, dtype=torch.float64)
        for d in range(world):
            y_home[ro[d]:ro[d + 1]] = back[d]
        out = oracle.combine(y_home, lay["slot_of_pair"], w)
        ref = oracle.layer(base, dict(inp, w13=full["w13"], w2=full["w2"]))
        q.put((rank, bool(torch.equal(out, ref["out"])), n_recv,
               int(counts_all.sum()), int(lay["expert_counts"].sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("payload", ["bf16", "e4m3"])
def test_expert_parallel_layer_gloo_world2(payload):
    """Real expert parallelism on two CPU ranks: each rank's output equals the
    single-rank layer on its own tokens, bit for bit, and the count exchange
    accounts for every routed row."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_rank_main, args=(r, world, port, payload, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [True, True]
    assert sum(r[2] for r in res) == res[0][3] == sum(r[4] for r in res)
