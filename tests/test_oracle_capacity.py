"""Pins of the oracle's fixed-capacity dispatch layout (token dropping).

Source: "Expert Parallelism" (aiwiki), "Implementation", closing note: fixed
buffers make every destination's size known in advance, at the price of
the tokens that do not fit.  Reading: expert e owns rows [e*C, (e+1)*C);
its earliest pairs (pair order) fill them; later pairs are dropped and
contribute nothing to the combine.
"""
import numpy as np
import pytest
import torch

import oracle


def _brute(idx: np.ndarray, E: int, C: int):
    """Per expert, the ordered list of its pairs; the first C are kept."""
    flat = idx.reshape(-1)
    kept, dropped = {}, 0
    for e in range(E):
        pairs = [p for p in range(flat.size) if flat[p] == e]
        kept[e] = pairs[:C]
        dropped += max(0, len(pairs) - C)
    return kept, dropped


@pytest.mark.parametrize("seed", range(40))
def test_capacity_layout_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    T, k, E = int(rng.integers(1, 12)), int(rng.integers(1, 4)), int(rng.integers(2, 6))
    k = min(k, E)
    W = 1 if E % 2 else 2
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    C = int(rng.integers(0, 5))
    lay = oracle.dispatch_layout_capacity(torch.from_numpy(idx), E, W, C)
    kept, dropped = _brute(idx, E, C)
    assert lay["dropped"] == dropped and lay["skipped"] == 0
    assert lay["expert_offsets"].tolist() == [e * C for e in range(E + 1)]
    assert lay["rank_offsets"].tolist() == [r * (E // W) * C for r in range(W + 1)]
    assert lay["expert_counts"].tolist() == [len(kept[e]) for e in range(E)]
    sop = lay["slot_of_pair"].tolist()
    pos = lay["pair_of_slot"].tolist()
    assert len(pos) == E * C
    want_sop = [-1] * (T * k)
    want_pos = [-1] * (E * C)
    for e in range(E):
        for i, p in enumerate(kept[e]):
            want_sop[p] = e * C + i
            want_pos[e * C + i] = p
    assert sop == want_sop and pos == want_pos


def test_capacity_above_every_count_is_the_dropless_layout_in_fixed_slabs():
    """With C >= the largest count nothing drops, and every pair keeps its
    rank inside its expert's segment from the (separately pinned) dropless
    layout."""
    g = torch.Generator().manual_seed(3)
    T, k, E, W = 300, 4, 16, 4
    logits = torch.randn(T, E, generator=g)
    idx, _ = oracle.route_topk(logits, k)
    free = oracle.dispatch_layout(idx, E, W)
    C = int(free["expert_counts"].max())
    cap = oracle.dispatch_layout_capacity(idx, E, W, C)
    assert cap["dropped"] == 0
    assert torch.equal(cap["expert_counts"], free["expert_counts"])
    off = free["expert_offsets"]
    e_of = idx.reshape(-1).long()
    want = e_of * C + (free["slot_of_pair"].long() - off[e_of].long())
    assert torch.equal(cap["slot_of_pair"].long(), want)


def test_capacity_zero_drops_everything_and_counts_add_up():
    g = torch.Generator().manual_seed(5)
    T, k, E = 64, 2, 8
    idx, _ = oracle.route_topk(torch.randn(T, E, generator=g), k)
    lay = oracle.dispatch_layout_capacity(idx, E, 2, 0)
    assert lay["dropped"] == T * k
    assert bool((lay["slot_of_pair"] == -1).all()) and lay["expert_counts"].sum() == 0
    free = oracle.dispatch_layout(idx, E, 2)
    for C in (1, 5, 16, 40):
        lay = oracle.dispatch_layout_capacity(idx, E, 2, C)
        kept = torch.clamp(free["expert_counts"], max=C)
        assert torch.equal(lay["expert_counts"], kept)
        assert int(kept.sum()) + lay["dropped"] == T * k


def test_out_of_range_ids_are_skipped_not_dropped():
    idx = torch.tensor([[0, 9], [1, -1], [0, 1]], dtype=torch.int32)
    lay = oracle.dispatch_layout_capacity(idx, 2, 1, 1)
    assert lay["skipped"] == 2 and lay["dropped"] == 2       # pairs 4 and 5 exceed C = 1
    assert lay["slot_of_pair"].tolist() == [0, -1, 1, -1, -1, -1]


def test_dropped_pairs_contribute_nothing_to_the_combine():
    """Identity experts (y = xp): each token's output is x times the sum of
    the router weights of its kept pairs, exactly (dyadic weights)."""
    T, k, E, C = 6, 2, 3, 2
    idx = torch.tensor([[0, 1], [0, 2], [0, 1], [1, 2], [2, 0], [1, 0]], dtype=torch.int32)
    w = torch.tensor([[0.5, 0.5]] * T, dtype=torch.float32)
    x = torch.randn(T, 8, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    lay = oracle.dispatch_layout_capacity(idx, E, 1, C)
    y = torch.zeros(E * C, 8, dtype=torch.float64)
    for s, p in enumerate(lay["pair_of_slot"].tolist()):
        if p >= 0:
            y[s] = x[p // k]
    out = oracle.combine(y, lay["slot_of_pair"], w)
    kept = (lay["slot_of_pair"].reshape(T, k) >= 0).double()
    want = x * (kept * w.double()).sum(dim=1, keepdim=True)
    assert torch.equal(out, want)
    # in pair order, expert 0 is picked by tokens 0, 1, 2, 4, 5 (keeps 0, 1),
    # expert 1 by 0, 2, 3, 5 (keeps 0, 2) and expert 2 by 1, 3, 4 (keeps 1, 3)
    assert kept[:, 0].tolist() == [1, 1, 0, 0, 0, 0] and kept[:, 1].tolist() == [1, 1, 1, 1, 0, 0]


def test_capacity_rows_formula():
    assert oracle.capacity_rows(8192, 8, 256, 1.0) == 256
    assert oracle.capacity_rows(8192, 8, 256, 1.25) == 320
    assert oracle.capacity_rows(10, 3, 7, 1.0) == 5          # ceil(30 / 7)


def test_capacity_layer_is_the_dropless_layer_minus_the_dropped_pairs():
    """The whole oracle layer with fixed slabs: every kept pair's expert
    output equals the dropless layer's for that pair, and each token's
    output is the weighted sum over its kept pairs only (same fp64 values,
    same j order: bit-exact)."""
    from expert_parallelism_b200 import workloads
    wl = workloads.Workload("cap", 96, 64, 8, 3, 48, 2, "bf16", "bf16", "bf16", seed=4)
    inputs = workloads.layer_inputs(wl)
    free = oracle.layer(wl, inputs)
    for factor in (0.5, 1.0, 5.0):
        cap = oracle.layer(wl.replace(capacity_factor=factor), inputs)
        sop_c, sop_f = cap["slot_of_pair"].long(), free["slot_of_pair"].long()
        kept = sop_c >= 0
        assert torch.equal(cap["y"][sop_c[kept]], free["y"][sop_f[kept]])
        w = cap["topk_w"].double()
        want = torch.zeros(wl.T, wl.H, dtype=torch.float64)
        for t in range(wl.T):
            for j in range(wl.k):
                p = t * wl.k + j
                if kept[p]:
                    want[t] += w[t, j] * free["y"][sop_f[p]]
        assert torch.equal(cap["out"], want)
        if factor == 5.0:
            assert bool(kept.all()) and torch.equal(cap["out"], free["out"])
        else:
            assert not bool(kept.all())
