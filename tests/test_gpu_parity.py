"""GPU parity: every step of the hot path, called through the C ABI, against
the CPU oracle on the same seeded inputs.

Small workloads (tiny and the extra ragged ones) are compared in full.
The full-size workloads (mid, dsv3, skew, decode) are compared in full for
routing and layout, and on a seeded sample of rows for the permute, the
GEMM and the combine, with the same launches and sizes the benchmark
times: all k rows of sampled tokens; the first, the last and 8 more seeded
rows of every expert; and every row of 8 experts, among them the largest
one, one whose rows take a pass with a second chunk (257..320 rows) and one
that takes several passes (parity_helpers.full_experts).  Full-size combine is also checked
against a property that holds at any size: with identity experts it
returns x bit for bit.
"""
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

from parity_helpers import (BF16_TOL, F32_TOL, GpuLayer, bits, h_ok, oracle_gemm_rows,
                            rowwise_ok, sample_rows, tol_for, workload)

SMALL = ["tiny", "small_f32", "small_bf16", "small_fp8", "small_fp8v", "ragged_bf16", "pair_bf16",
         "pair_fp8"]
FULL = {"decode": 64, "mid": 192, "skew": 128, "dsv3": 96,    # name -> sampled tokens
        "dsv3_cap": 96, "skew_cap": 128, "dsv3_grouped": 96}


def _check_route_layout(wl, g: GpuLayer):
    b = g.buf
    if wl.route_groups:
        idx_o, w_o = oracle.route_topk_grouped(g.inputs["logits"], wl.k, wl.route_groups,
                                               wl.route_max_groups)
    else:
        idx_o, w_o = oracle.route_topk(g.inputs["logits"], wl.k)
    assert torch.equal(b.topk_idx.cpu(), idx_o), "topk_idx differs"
    wg = b.topk_w.cpu().double()
    assert bool(((wg - w_o.double()).abs() <= 1e-5 * w_o.double().abs()).all()), "topk_w"
    if wl.capacity_factor is None:
        lay = oracle.dispatch_layout(idx_o, wl.E, wl.W)
    else:
        C = oracle.capacity_rows(wl.T, wl.k, wl.E, wl.capacity_factor)
        lay = oracle.dispatch_layout_capacity(idx_o, wl.E, wl.W, C)
        assert int(b.n_dropped.cpu()[0]) == lay["dropped"]
    for key in ["expert_counts", "expert_offsets", "rank_offsets", "slot_of_pair",
                "pair_of_slot"]:
        got = getattr(b, key).cpu()[:lay[key].numel()]
        assert torch.equal(got, lay[key]), f"{key} differs"
    return idx_o, w_o, lay


@pytest.mark.gpu
@pytest.mark.parametrize("name", SMALL)
def test_small_layer_full_parity(name, cuda_device):
    wl = workload(name)
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    idx_o, w_o, lay = _check_route_layout(wl, g)
    b = g.buf
    xp_o, sc_o = oracle.permute(g.inputs["x"], wl.k, lay["pair_of_slot"], wl.payload)
    assert torch.equal(bits(b.xp), bits(xp_o)), "xp differs"
    if sc_o is not None:
        assert torch.equal(bits(b.xp_scales), bits(sc_o)), "xp_scales differ"
    h_o, y_o, done = oracle.grouped_gemm(xp_o, sc_o, lay["expert_offsets"], 0, wl.E,
                                         g.inputs["w13"], g.inputs["w2"])
    assert done == wl.N
    wdt = workloads.TORCH_DTYPE[wl.wdt]
    ok, worst = h_ok(b.h.cpu(), h_o, wdt)
    assert ok, f"h: worst excess {worst:.3g}"
    ok, worst = rowwise_ok(b.y.cpu(), y_o, tol_for(wdt))
    assert ok, f"y: worst err/rms {worst:.3g} > {tol_for(wdt)}"
    out_o = oracle.combine(y_o, lay["slot_of_pair"], w_o)
    ok, worst = rowwise_ok(b.out.cpu(), out_o, tol_for(wdt))
    assert ok, f"out: worst err/rms {worst:.3g}"


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(FULL))
def test_full_size_layer_sampled_parity(name, cuda_device):
    wl = workload(name)
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    idx_o, w_o, lay = _check_route_layout(wl, g)
    b = g.buf
    toks, mask, experts = sample_rows(lay, wl.T, wl.k, FULL[name])
    cnt = lay["expert_counts"]
    assert all(int(mask[lay["expert_offsets"][e]:][:int(cnt[e])].sum()) == int(cnt[e])
               for e in experts)
    # permute: the oracle writes only the sampled slots
    pos = lay["pair_of_slot"].clone()
    pos[~mask] = -1
    xp_o, sc_o = oracle.permute(g.inputs["x"], wl.k, pos, wl.payload)
    xp_g = b.xp.cpu()
    assert torch.equal(bits(xp_g[mask]), bits(xp_o[mask])), "xp differs on sampled slots"
    if sc_o is not None:
        assert torch.equal(bits(b.xp_scales.cpu()[mask]), bits(sc_o[mask])), "scales differ"
    slots, h_o, y_o = oracle_gemm_rows(wl, xp_o, sc_o, lay["expert_offsets"], mask)
    ok, worst = h_ok(b.h.cpu()[slots], h_o, torch.bfloat16)
    assert ok, f"h: worst excess {worst:.3g}"
    ok, worst = rowwise_ok(b.y.cpu()[slots], y_o, BF16_TOL)
    assert ok, f"y: worst err/rms {worst:.3g}"
    # combine for the sampled tokens, from the oracle's own (exact) y rows
    # (a dropped pair, slot -1, stays -1 and adds nothing)
    sop = lay["slot_of_pair"].view(wl.T, wl.k)[toks].reshape(-1)
    kept = sop >= 0
    compact = torch.full_like(sop, -1)
    compact[kept] = torch.searchsorted(slots, sop[kept].long()).to(torch.int32)
    assert torch.equal(slots[compact[kept].long()], sop[kept].long())
    out_o = oracle.combine(y_o, compact, w_o[toks].contiguous())
    ok, worst = rowwise_ok(b.out.cpu()[toks], out_o, BF16_TOL)
    assert ok, f"out: worst err/rms {worst:.3g}"
    # full size, identity experts: combine(xp) returns x exactly (bf16 payloads)
    if wl.payload == "bf16" and wl.capacity_factor is None:
        moe.moe_combine(b.xp, b.slot_of_pair, b.topk_w, b.out)
        torch.cuda.synchronize()
        assert torch.equal(bits(b.out), bits(g.inputs["x"])), "identity combine != x"
