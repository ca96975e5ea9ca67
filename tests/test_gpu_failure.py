"""Failure detection without a GPU fault: a bounded wait that runs out.

Every spin-wait in the library is bounded; when its limit passes, the kernel
records MOE_DEV_TIMEOUT in the caller's status word and returns, and the
context stays usable.  moe_diag_layout_wait_timeout runs the dispatch
layout's own scan kernel on a look-back flag that nothing sets, with a
caller-chosen limit, so the wait can only run out.  The test checks that the
status word reports it, that the kernel gave up after about the limit (not
the library's 2 s), and that the next ordinary layout, a multi-chunk scan on
the same context, is bit-exact with the oracle again.
"""
import time

import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads


@pytest.mark.gpu
@pytest.mark.parametrize("limit_ns", [0, 20_000_000])
def test_layout_wait_runs_out_then_next_layout_is_exact(limit_ns, cuda_device):
    ws = torch.empty(moe.load_library().moe_diag_layout_wait_timeout_workspace_bytes(),
                     dtype=torch.uint8, device=cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.moe_diag_layout_wait_timeout(ws, limit_ns, st)
    rc = moe.moe_check_status(st)                  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert moe.STATUS[rc] == "MOE_ERR_TIMEOUT"
    assert elapsed >= 0.9 * limit_ns * 1e-9        # it waited for its limit ...
    assert elapsed < 1.0                           # ... not for the library's 2 s
    assert moe.moe_check_status(st) == 0           # the status word was cleared
    # the context still works: a five-chunk scan with the default limit
    T, k, E, W = 20000, 8, 256, 8
    wl = workloads.Workload("after_timeout", T, 64, E, k, 32, W, "bf16", "bf16", "bf16")
    logits = workloads.router_logits(wl)
    idx_o, _ = oracle.route_topk(logits, k)
    lay = oracle.dispatch_layout(idx_o, E, W)
    i32 = dict(dtype=torch.int32, device=cuda_device)
    got = dict(expert_counts=torch.empty(E, **i32), expert_offsets=torch.empty(E + 1, **i32),
               rank_offsets=torch.empty(W + 1, **i32), slot_of_pair=torch.empty(T * k, **i32),
               pair_of_slot=torch.empty(T * k, **i32))
    lws = torch.empty(moe.moe_dispatch_layout_workspace_bytes(T, k, E), dtype=torch.uint8,
                      device=cuda_device)
    moe.moe_dispatch_layout(idx_o.to(cuda_device), E, W, got["expert_counts"],
                            got["expert_offsets"], got["rank_offsets"], got["slot_of_pair"],
                            got["pair_of_slot"], lws, st)
    assert moe.moe_check_status(st) == 0
    for key, v in got.items():
        assert torch.equal(v.cpu(), lay[key]), key
