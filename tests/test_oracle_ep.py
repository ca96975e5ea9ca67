"""Pins of the oracle's expert-parallel dispatch plan and of the simulated
expert-parallel layer, against things other than the plan's own formula.

Sources: "Expert Parallelism" (aiwiki), "The two all-to-alls" and
"Implementation" (rows travel to their expert's owner and back; a count
exchange tells each owner how much arrives; the sketch counts rows per
destination with bincount(idx // per_rank)); "Expert parallelism"
(Transformers), "How the sizes combine" (rank r owns experts
[r*E/W, (r+1)*E/W)).
"""
import itertools

import pytest
import torch

import oracle
from expert_parallelism_b200 import workloads


def _counts(W, E, seed, hi=6):
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(0, hi, (W, E), generator=g, dtype=torch.int32)
    c[0, 0] = 0                                    # empty (source, expert) pairs too
    return c


@pytest.mark.parametrize("W,E,seed", [(1, 5, 0), (2, 4, 1), (3, 6, 2), (4, 8, 3), (4, 4, 4),
                                       (8, 16, 5), (8, 64, 6)])
def test_plan_tiles_every_owner_buffer_in_expert_then_source_order(W, E, seed):
    """Brute force over every (source, expert) chunk: for each owner the
    chunks [send_base, send_base + count) are disjoint, cover [0, total)
    exactly, and sort by (expert, source); recv_offsets marks each local
    expert's first row."""
    c = _counts(W, E, seed)
    Er = E // W
    plans = [oracle.ep_plan(c, s) for s in range(W)]
    for r in range(W):
        chunks = []
        for s, j in itertools.product(range(W), range(Er)):
            e = r * Er + j
            chunks.append((int(plans[s][0][e]), int(c[s, e]), j, s))
        covered = torch.zeros(int(c[:, r * Er:(r + 1) * Er].sum()), dtype=torch.int32)
        for start, n, _, _ in chunks:
            covered[start:start + n] += 1
        assert bool((covered == 1).all())
        # non-empty chunks in buffer order are sorted by (expert, source)
        order = [(j, s) for start, n, j, s in sorted(chunks) if n > 0]
        assert order == sorted(order)
        ro = plans[r][1]
        assert int(ro[-1]) == covered.numel()
        for j in range(Er):
            firsts = [start for start, n, jj, s in chunks if jj == j and n > 0]
            if firsts:
                assert int(ro[j]) == min(firsts)
            assert int(ro[j + 1] - ro[j]) == int(c[:, r * Er + j].sum())


def test_plan_on_one_rank_is_the_local_layout():
    """W = 1: nothing moves, so the plan's rows are the single-rank layout's
    expert offsets."""
    idx, _ = oracle.route_topk(torch.randn(50, 8, generator=torch.Generator().manual_seed(5)), 3)
    lay = oracle.dispatch_layout(idx, 8, 1)
    sb, ro = oracle.ep_plan(lay["expert_counts"][None], 0)
    assert torch.equal(sb, lay["expert_offsets"][:-1])
    assert torch.equal(ro, lay["expert_offsets"])


def test_rows_per_owner_equal_the_sketch_bincount():
    """What an owner receives is the sum over senders of the aiwiki sketch's
    per-destination bincount(idx // per_rank)."""
    W, E, k, T = 4, 16, 3, 40
    g = torch.Generator().manual_seed(9)
    per = []
    for s in range(W):
        idx, _ = oracle.route_topk(torch.randn(T, E, generator=g), k)
        per.append((idx, oracle.dispatch_layout(idx, E, W)))
    c = torch.stack([lay["expert_counts"] for _, lay in per])
    sketch = sum(torch.bincount(idx.reshape(-1).long() // (E // W), minlength=W)
                 for idx, _ in per)
    for r in range(W):
        assert int(oracle.ep_plan(c, r)[1][-1]) == int(sketch[r])


def test_dest_rows_are_a_bijection_onto_each_owner_buffer():
    W, E, k, T = 3, 9, 2, 30
    g = torch.Generator().manual_seed(11)
    per = []
    for s in range(W):
        idx, _ = oracle.route_topk(torch.randn(T, E, generator=g), k)
        per.append((idx, oracle.dispatch_layout(idx, E, W)))
    c = torch.stack([lay["expert_counts"] for _, lay in per])
    hits = [torch.zeros(int(oracle.ep_plan(c, r)[1][-1]), dtype=torch.int32) for r in range(W)]
    for s, (idx, lay) in enumerate(per):
        sb, _ = oracle.ep_plan(c, s)
        owner, row = oracle.ep_dest_rows(lay, idx, sb, E, W)
        assert bool((owner == idx.reshape(-1).long() // (E // W)).all())
        for o, r_ in zip(owner.tolist(), row.tolist()):
            hits[o][r_] += 1
    assert all(bool((h == 1).all()) for h in hits)


@pytest.mark.parametrize("W,payload", [(2, "bf16"), (4, "bf16"), (2, "e4m3"), (8, "e4m3")])
def test_expert_parallel_layer_equals_the_single_rank_layer(W, payload):
    """Moving rows to their owners and back changes nothing: every rank's out
    equals the single-GPU layer on its own tokens, bit for bit (fp64, each
    output row depends only on its own input row and its expert)."""
    base = workloads.Workload("ep", 24, 256, 8, 2, 64, W, "bf16", payload, "bf16")
    full = workloads.layer_inputs(base)
    inputs = []
    for s in range(W):
        wl_s = base.replace(seed=100 + s)
        inputs.append({"logits": workloads.router_logits(wl_s),
                       "x": workloads.hidden_states(wl_s)})
    res = oracle.ep_layer(base, inputs, full["w13"], full["w2"])
    for s in range(W):
        ref = oracle.layer(base, dict(inputs[s], w13=full["w13"], w2=full["w2"]))
        assert torch.equal(res[s]["out"], ref["out"]), s
