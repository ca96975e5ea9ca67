"""GPU parity of the fixed-capacity dispatch layout (token dropping) with
the oracle: every output bit-exact, including the dropped-pair count.

Source: "Expert Parallelism" (aiwiki), "Implementation", closing note on
fixed capacity.  Reading: expert e owns rows [e*C, (e+1)*C); its earliest
pairs fill them; later pairs are dropped.
"""
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads


def _capacity_layout(idx, E, W, C, dev):
    T, k = idx.shape
    i32 = dict(dtype=torch.int32, device=dev)
    b = dict(expert_counts=torch.full((E,), -5, **i32),
             expert_offsets=torch.full((E + 1,), -5, **i32),
             rank_offsets=torch.full((W + 1,), -5, **i32),
             slot_of_pair=torch.full((max(T * k, 1),), -5, **i32),
             pair_of_slot=torch.full((max(E * C, 1),), -5, **i32),
             n_dropped=torch.full((1,), -5, **i32),
             dev_status=torch.zeros(1, **i32))
    ws = torch.empty(max(moe.moe_dispatch_layout_workspace_bytes(T, k, E), 16),
                     dtype=torch.uint8, device=dev)
    moe.moe_dispatch_layout_capacity(idx.to(dev), E, W, C, b["expert_counts"],
                                     b["expert_offsets"], b["rank_offsets"], b["slot_of_pair"],
                                     b["pair_of_slot"], ws, b["dev_status"],
                                     n_dropped=b["n_dropped"])
    assert moe.moe_check_status(b["dev_status"]) == 0
    return {key: v.cpu() for key, v in b.items()}


def _assert_equal(got, ref, T, k, E, C):
    assert torch.equal(got["expert_counts"], ref["expert_counts"])
    assert torch.equal(got["expert_offsets"], ref["expert_offsets"])
    assert torch.equal(got["rank_offsets"], ref["rank_offsets"])
    assert torch.equal(got["slot_of_pair"][:T * k], ref["slot_of_pair"])
    assert torch.equal(got["pair_of_slot"][:E * C], ref["pair_of_slot"])
    assert int(got["n_dropped"][0]) == ref["dropped"]


@pytest.mark.gpu
@pytest.mark.parametrize("T,k,E,W,factor", [
    (8192, 8, 256, 8, 1.0),      # DeepSeek-V3 shape, C = 256: a few pairs drop
    (8192, 8, 256, 8, 1.25),     # C = 320: nothing drops on balanced routing
    (4096, 6, 64, 4, 0.5),       # heavy dropping
    (3000, 4, 16, 2, 0.1),       # several 2048-pair tiles per expert all past C
    (1, 2, 8, 2, 1.0),           # one token
])
def test_capacity_layout_matches_oracle(T, k, E, W, factor, cuda_device):
    g = torch.Generator().manual_seed(T + E)
    logits = torch.randn(T, E, generator=g)
    idx, _ = oracle.route_topk(logits, k)
    C = oracle.capacity_rows(T, k, E, factor)
    ref = oracle.dispatch_layout_capacity(idx, E, W, C)
    got = _capacity_layout(idx, E, W, C, cuda_device)
    _assert_equal(got, ref, T, k, E, C)


@pytest.mark.gpu
def test_capacity_layout_skewed_routing_and_degenerate_capacities(cuda_device):
    wl = workloads.WORKLOADS["skew"].replace(T=4096)
    idx, _ = oracle.route_topk(workloads.router_logits(wl), wl.k)
    for C in (0, 1, 7, 128, 4096 * 4):
        ref = oracle.dispatch_layout_capacity(idx, wl.E, wl.W, C)
        got = _capacity_layout(idx, wl.E, wl.W, C, cuda_device)
        _assert_equal(got, ref, wl.T, wl.k, wl.E, C)
    assert ref["dropped"] == 0                              # C above every count


@pytest.mark.gpu
def test_capacity_layout_empty_batch_and_bad_ids(cuda_device):
    E, W, C = 8, 2, 3
    got = _capacity_layout(torch.empty(0, 2, dtype=torch.int32), E, W, C, cuda_device)
    assert got["expert_counts"].tolist() == [0] * E
    assert got["expert_offsets"].tolist() == [e * C for e in range(E + 1)]
    assert bool((got["pair_of_slot"][:E * C] == -1).all()) and int(got["n_dropped"][0]) == 0
    idx = torch.tensor([[0, 9], [1, -1], [0, 1], [0, 2]], dtype=torch.int32)
    ref = oracle.dispatch_layout_capacity(idx, E, W, 2)
    dev = cuda_device
    i32 = dict(dtype=torch.int32, device=dev)
    st = torch.zeros(1, **i32)
    outs = [torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(W + 1, **i32),
            torch.empty(8, **i32), torch.empty(E * 2, **i32)]
    nd = torch.empty(1, **i32)
    ws = torch.empty(moe.moe_dispatch_layout_workspace_bytes(4, 2, E), dtype=torch.uint8,
                     device=dev)
    moe.moe_dispatch_layout_capacity(idx.to(dev), E, W, 2, *outs, ws, st, n_dropped=nd)
    assert moe.moe_check_status(st) == 3                 # MOE_ERR_BAD_INDEX: ids 9 and -1
    assert torch.equal(outs[3].cpu(), ref["slot_of_pair"])
    assert torch.equal(outs[4].cpu(), ref["pair_of_slot"])
    assert int(nd.cpu()[0]) == ref["dropped"] == 1 and ref["skipped"] == 2


CAP_LAYERS = {
    # (workload, capacity factor): heavy dropping, mild dropping, none
    "cap_bf16_drop": (workloads.Workload("cap_bf16", 600, 256, 8, 2, 192, 2, "bf16", "bf16",
                                         "bf16"), 0.6),
    "cap_fp8_drop": (workloads.Workload("cap_fp8", 400, 384, 16, 4, 320, 4, "bf16", "e4m3",
                                        "bf16"), 0.9),
    "cap_bf16_none": (workloads.Workload("cap_bf16n", 300, 256, 8, 2, 192, 2, "bf16", "bf16",
                                         "bf16"), 2.0),
    "cap_f32": (workloads.Workload("cap_f32", 130, 72, 5, 3, 40, 5, "f32", "f32", "f32"), 0.7),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CAP_LAYERS))
def test_capacity_layer_parity(name, cuda_device):
    """moe_layer_forward with fixed slabs against the oracle layer: layout,
    kept payload rows and dropped count bit-exact; the kept rows' h and y
    and the combined out within the GEMM dtype's tolerance."""
    from parity_helpers import GpuLayer, bits, h_ok, rowwise_ok, tol_for
    base, factor = CAP_LAYERS[name]
    wl = base.replace(capacity_factor=factor)
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    b = g.buf
    ref = oracle.layer(wl, g.inputs)
    C = oracle.capacity_rows(wl.T, wl.k, wl.E, factor)
    assert b.capacity == C
    for key in ("expert_counts", "expert_offsets", "rank_offsets", "slot_of_pair",
                "pair_of_slot"):
        assert torch.equal(getattr(b, key).cpu()[:ref[key].numel()], ref[key]), key
    assert int(b.n_dropped.cpu()[0]) == ref["dropped"]
    kept = ref["pair_of_slot"] >= 0
    assert torch.equal(bits(b.xp)[kept], bits(ref["xp"])[kept])
    if ref["xp_scales"] is not None:
        assert torch.equal(bits(b.xp_scales)[kept], bits(ref["xp_scales"])[kept])
    wdt = workloads.TORCH_DTYPE[wl.wdt]
    ok, worst = h_ok(b.h.cpu()[kept], ref["h"][kept], wdt)
    assert ok, f"h: {worst:.3g}"
    ok, worst = rowwise_ok(b.y.cpu()[kept], ref["y"][kept], tol_for(wdt))
    assert ok, f"y: {worst:.3g}"
    ok, worst = rowwise_ok(b.out.cpu(), ref["out"], tol_for(wdt))
    assert ok, f"out: {worst:.3g}"
    if factor < 1.0:
        assert ref["dropped"] > 0
