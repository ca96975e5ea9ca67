"""GPU parity of group-limited routing with the oracle: picks bit-exact,
weights within 1e-5 relative.

Source: "Expert Parallelism" (aiwiki), "Hiding the latency", topology-aware
routing (each token reaches at most M nodes).  Reading: G equal groups of
consecutive experts, scored by their largest logit; the M best are kept.
"""
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,k,G,M,ties", [
    (4096, 256, 8, 8, 4, False),    # DeepSeek-V3 shape: 8 rank groups, at most 4
    (1000, 64, 6, 8, 2, False),
    (500, 12, 5, 3, 2, False),      # one logit per lane (E < 32), 4 experts per group
    (300, 160, 4, 32, 3, False),    # 32 groups of 5 experts, groups straddle lanes
    (200, 256, 8, 8, 8, False),     # every group kept: plain top-k
    (700, 64, 4, 8, 2, True),       # logits on a coarse grid: ties between groups
])
def test_grouped_route_matches_oracle(T, E, k, G, M, ties, cuda_device):
    g = torch.Generator().manual_seed(T + E + G)
    lg = torch.randn(T, E, generator=g)
    if ties:
        lg = (lg * 2).round() / 2
    idx_o, w_o = oracle.route_topk_grouped(lg, k, G, M)
    dev = cuda_device
    idx = torch.full((T, k), -9, dtype=torch.int32, device=dev)
    w = torch.full((T, k), -9.0, dtype=torch.float32, device=dev)
    moe.moe_route_topk_grouped(lg.to(dev), G, M, idx, w)
    torch.cuda.synchronize()
    assert torch.equal(idx.cpu(), idx_o)
    wg, wo = w.cpu().double(), w_o.double()
    assert bool(((wg - wo).abs() <= 1e-5 * wo.abs()).all())
    if M == G:
        i0, _ = oracle.route_topk(lg, k)
        assert torch.equal(idx.cpu(), i0)


@pytest.mark.gpu
def test_grouped_route_layer_parity(cuda_device):
    """The whole layer with group-limited routing: routing and layout
    bit-exact, out within the bf16 bar."""
    from parity_helpers import GpuLayer, rowwise_ok, BF16_TOL
    wl = workloads.Workload("grp", 400, 256, 16, 4, 192, 4, "bf16", "bf16", "bf16",
                            route_groups=4, route_max_groups=2)
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    ref = oracle.layer(wl, g.inputs)
    b = g.buf
    assert torch.equal(b.topk_idx.cpu(), ref["topk_idx"])
    for key in ("expert_counts", "expert_offsets", "slot_of_pair", "pair_of_slot"):
        assert torch.equal(getattr(b, key).cpu()[:ref[key].numel()], ref[key]), key
    per = wl.E // wl.route_groups
    groups = (b.topk_idx.cpu().long() // per)
    assert all(len(set(r)) <= wl.route_max_groups for r in groups.tolist())
    ok, worst = rowwise_ok(b.out.cpu(), ref["out"], BF16_TOL)
    assert ok, worst
