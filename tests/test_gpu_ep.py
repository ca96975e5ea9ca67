"""Expert parallelism on one GPU: W ranks, each with its own tokens and its
E/W experts, run through the real entry points (moe_ep_plan,
moe_ep_dispatch, moe_grouped_gemm on the receive buffer, moe_ep_combine);
the per-rank buffer table holds W buffers of this GPU instead of
peer-mapped ones, and no rank's kernels wait for another's.

Checks: the plan equals the oracle's bit for bit; every received row holds
exactly the payload the oracle's exchange puts there; each rank's out is
within the bf16 bar of the oracle's layer on its tokens, and bit-exact with
this library's own single-rank layer (moving rows changes no arithmetic);
rows that would miss a too-small receive buffer are skipped and reported.
"""
import pytest
import torch

import oracle
from expert_parallelism_b200 import ep, moe, workloads

from parity_helpers import BF16_TOL, bits, rowwise_ok


def _inputs(base, W, dev):
    full = workloads.layer_inputs(base)
    per = []
    for r in range(W):
        wl_r = base.replace(seed=100 + r)
        per.append({"logits": workloads.router_logits(wl_r), "x": workloads.hidden_states(wl_r)})
    return full, per


CASES = {
    "bf16_w2": (workloads.Workload("ep_bf16", 96, 256, 8, 2, 192, 2, "bf16", "bf16", "bf16"), 2),
    "fp8_w4": (workloads.Workload("ep_fp8", 80, 384, 16, 4, 320, 4, "bf16", "e4m3", "bf16"), 4),
    "fp8y_w4": (workloads.Workload("ep_fp8y", 64, 256, 8, 2, 128, 4, "bf16", "e4m3", "bf16",
                                   ydt="e4m3"), 4),
    "bf16_w8_pairs": (workloads.Workload("ep_pairs", 700, 256, 16, 4, 192, 8, "bf16", "bf16",
                                         "bf16"), 8),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_expert_parallel_layer_on_one_gpu(name, cuda_device):
    base, W = CASES[name]
    full, per = _inputs(base, W, cuda_device)
    w13, w2 = full["w13"].to(cuda_device), full["w2"].to(cuda_device)
    run = ep.EmulatedEP(base, W, cuda_device)
    outs = run.forward([p["logits"].to(cuda_device) for p in per],
                       [p["x"].to(cuda_device) for p in per], w13, w2)
    torch.cuda.synchronize()
    assert run.status() == [0] * W
    ref = oracle.ep_layer(base, per, full["w13"], full["w2"])
    Er = base.E // W
    for r in range(W):
        R = run.ranks[r]
        assert torch.equal(R.counts_all.cpu(), ref[r]["counts_all"])
        assert torch.equal(R.send_base.cpu(), ref[r]["send_base"])
        assert torch.equal(R.recv_offsets.cpu(), ref[r]["recv_offsets"])
    # every received row: the oracle's payload for the pair the plan sends there
    for s in range(W):
        lay = oracle.dispatch_layout(run.ranks[s].topk_idx.cpu(), base.E, W)
        xp_o, sc_o = oracle.permute(per[s]["x"], base.k, lay["pair_of_slot"], base.payload)
        owner, row = ref[s]["owner"], ref[s]["row"]
        sop = lay["slot_of_pair"].long()
        for r in range(W):
            sel = torch.nonzero(owner == r).flatten()
            got = run.ranks[r].recv.cpu()[row[sel]]
            assert torch.equal(bits(got), bits(xp_o[sop[sel]])), (s, r)
            if sc_o is not None:
                assert torch.equal(bits(run.ranks[r].recv_scales.cpu()[row[sel]]),
                                   bits(sc_o[sop[sel]]))
    for r in range(W):
        if base.ydt != "e4m3":
            ok, worst = rowwise_ok(outs[r].cpu(), ref[r]["out"], BF16_TOL)
            assert ok, (r, worst)
        # the single-rank layer on the same tokens, with all E experts
        wl1 = base.replace(W=1)
        buf = moe.LayerBuffers(wl1, cuda_device)
        moe.layer_forward(wl1, per[r]["logits"].to(cuda_device), per[r]["x"].to(cuda_device),
                          w13, w2, buf)
        torch.cuda.synchronize()
        assert torch.equal(bits(outs[r]), bits(buf.out)), r


@pytest.mark.gpu
def test_expert_parallel_dsv3_shape_equals_single_rank(cuda_device):
    """The DeepSeek-V3 shape split over 8 ranks of 1024 tokens each (the
    same 65,536 routed rows as the one-GPU dsv3 batch): every rank's out is
    the single-rank layer's, bit for bit, and the plans are the oracle's."""
    W = 8
    base = workloads.WORKLOADS["dsv3"].replace(T=1024, W=W, name="dsv3_ep8")
    dev = cuda_device
    w13 = torch.empty(base.E, 2 * base.I, base.H, dtype=torch.bfloat16, device=dev)
    w2 = torch.empty(base.E, base.H, base.I, dtype=torch.bfloat16, device=dev)
    workloads.fill_expert_weights(base, w13, w2)
    per = [{"logits": workloads.router_logits(base.replace(seed=100 + r)).to(dev),
            "x": workloads.hidden_states(base.replace(seed=100 + r)).to(dev)} for r in range(W)]
    run = ep.EmulatedEP(base, W, dev)
    outs = run.forward([p["logits"] for p in per], [p["x"] for p in per], w13, w2)
    torch.cuda.synchronize()
    assert run.status() == [0] * W
    counts = run.ranks[0].counts_all.cpu()
    assert int(counts.sum()) == W * base.T * base.k
    for r in range(W):
        sb, ro = oracle.ep_plan(counts, r)
        assert torch.equal(run.ranks[r].send_base.cpu(), sb)
        assert torch.equal(run.ranks[r].recv_offsets.cpu(), ro)
    one = base.replace(W=8)
    buf = moe.LayerBuffers(one, dev)
    for r in range(W):
        moe.layer_forward(one, per[r]["logits"], per[r]["x"], w13, w2, buf)
        torch.cuda.synchronize()
        assert torch.equal(bits(outs[r]), bits(buf.out)), r


@pytest.mark.gpu
def test_rows_past_the_receive_buffer_are_skipped_and_reported(cuda_device):
    """A receive buffer smaller than what arrives: the rows that do not fit
    are not written (the guard rows past the stated capacity keep their
    sentinel), and the status word reports MOE_ERR_OVERFLOW."""
    base, W = workloads.Workload("ep_small", 64, 256, 8, 2, 128, 2, "bf16", "bf16", "bf16"), 2
    full, per = _inputs(base, W, cuda_device)
    run = ep.EmulatedEP(base, W, cuda_device)
    R = run.ranks
    for r in range(W):
        R[r].route_and_layout(per[r]["logits"].to(cuda_device))
    counts = torch.stack([R[r].expert_counts for r in range(W)])
    for r in range(W):
        R[r].counts_all.copy_(counts)
        R[r].plan(r)
    cap = 40                                  # far fewer than the ~64 rows each owner gets
    for r in range(W):
        R[r].recv.fill_(7.0)
    tables = [R[r].recv for r in range(W)]
    for s in range(W):
        moe.moe_ep_dispatch(per[s]["x"].to(cuda_device), base.k, R[s].topk_idx,
                            R[s].slot_of_pair, R[s].expert_offsets, R[s].send_base, tables, None,
                            torch.bfloat16, cap, R[s].dev_status)
    torch.cuda.synchronize()
    assert any(moe.STATUS[moe.moe_check_status(R[s].dev_status)] == "MOE_ERR_OVERFLOW"
               for s in range(W))
    for r in range(W):
        assert bool((R[r].recv[cap:] == 7.0).all())
