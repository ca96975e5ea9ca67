"""Expert parallelism as separate processes: two ranks, each its own
process with its own tokens and its own E/2 experts, share one GPU.  Each
maps the other's receive and output buffers through CUDA IPC records
(moe_ipc_export / moe_ipc_import), the count exchange and the barriers run
over a gloo group, and the dispatch stores and combine loads go through the
mapped addresses -- the multi-GPU code path (ep.DistributedEP), with the
peer buffers on the same device.  No kernel of one rank waits for the
other's: the barriers are host-side, after each rank's device work.

Each rank's out equals this library's single-rank layer on its tokens, bit
for bit, and the oracle's layer within the bf16 bar.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, payload, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    import oracle
    from expert_parallelism_b200 import ep, moe, workloads
    from parity_helpers import BF16_TOL, bits, rowwise_ok
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    # a short group timeout: a rank that fails ends the other's next collective
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cuda:0")
        torch.cuda.set_device(dev)
        base = workloads.Workload("ep_ipc", 96, 256, 8, 2, 192, world, "bf16", payload, "bf16")
        full = workloads.layer_inputs(base)
        Er = base.E // world
        mine = base.replace(seed=100 + rank)
        logits = workloads.router_logits(mine)
        x = workloads.hidden_states(mine)
        w13, w2 = full["w13"].to(dev), full["w2"].to(dev)
        run = ep.DistributedEP(base, device=dev)
        outs = []
        for _ in range(2):                 # two layers in a row on the same buffers
            out = run.forward(logits.to(dev), x.to(dev), w13[rank * Er:(rank + 1) * Er],
                              w2[rank * Er:(rank + 1) * Er])
            torch.cuda.synchronize()
            outs.append(out.clone())
        st = moe.moe_check_status(run.state.dev_status)
        run.close()
        one = base.replace(W=world)
        buf = moe.LayerBuffers(one, dev)
        moe.layer_forward(one, logits.to(dev), x.to(dev), w13, w2, buf)
        torch.cuda.synchronize()
        same = all(bool(torch.equal(bits(o), bits(buf.out))) for o in outs)
        ref = oracle.layer(base, {"logits": logits, "x": x, "w13": full["w13"], "w2": full["w2"]})
        ok, worst = rowwise_ok(outs[0].cpu(), ref["out"], BF16_TOL)
        q.put((rank, st, same, ok, worst))
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
@pytest.mark.parametrize("payload", ["bf16", "e4m3"])
def test_expert_parallel_processes_over_ipc(payload, cuda_device):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, payload, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    for p in procs:
        if p.exitcode is None:
            p.terminate()
            p.join(10)
    assert [p.exitcode for p in procs] == [0] * world
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, st, same, ok, worst in res:
        assert st == 0, (rank, st)
        assert same, rank
        assert ok, (rank, worst)
