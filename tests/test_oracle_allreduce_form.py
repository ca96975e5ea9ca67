"""Pins of the oracle's all_reduce form of the layer: each rank's partial
(its own picks only) and the sum of the partials over ranks.

Source: "Expert parallelism" (Transformers docs), "Choosing an
implementation", the all_reduce row: no token moves, every rank runs its
experts over the whole batch, and the ranks' outputs are summed by an
all-reduce.
"""
import torch

import oracle


def _layout(T, k, E, W, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    idx, w = oracle.route_topk(logits, k)
    return idx, w, oracle.dispatch_layout(idx, E, W)


def test_partials_by_brute_force():
    """Pure-Python loops over a tiny case: each rank's partial takes exactly
    the picks whose expert it owns (E/W consecutive experts per rank)."""
    T, k, E, W, H = 7, 3, 6, 3, 4
    idx, w, lay = _layout(T, k, E, W, 11)
    g = torch.Generator().manual_seed(12)
    y = torch.randn(T * k, H, generator=g, dtype=torch.float64)
    sop = lay["slot_of_pair"]
    for r in range(W):
        got = oracle.combine_rank(y, sop, w, lay["rank_offsets"], r)
        for t in range(T):
            for c in range(H):
                ref = 0.0
                for j in range(k):
                    if int(idx[t, j]) // (E // W) == r:     # the expert's owner
                        ref += float(w[t, j]) * float(y[int(sop[t * k + j]), c])
                assert abs(float(got[t, c]) - ref) <= 1e-12 * (1 + abs(ref))


def test_sum_of_partials_is_the_combine_exactly():
    """With dyadic values (small integers times powers of two) every sum is
    exact in fp64, so the ranks' partials add up to the combine bit for
    bit, whatever the order."""
    T, k, E, W, H = 64, 4, 16, 4, 8
    idx, _, lay = _layout(T, k, E, W, 13)
    g = torch.Generator().manual_seed(14)
    y = torch.randint(-64, 65, (T * k, H), generator=g).double() / 8
    w = torch.randint(1, 16, (T, k), generator=g).float() / 16
    sop = lay["slot_of_pair"]
    parts = torch.stack([oracle.combine_rank(y, sop, w, lay["rank_offsets"], r)
                         for r in range(W)])
    assert torch.equal(oracle.reduce_partials(parts), oracle.combine(y, sop, w))


def test_a_token_served_by_one_rank_only():
    """All of token 0's picks on rank 0's experts: rank 0's partial is its
    whole combine and every other rank contributes an exact zero row."""
    T, k, E, W, H = 3, 2, 8, 4, 5
    logits = torch.full((T, E), -5.0)
    logits[0, 0], logits[0, 1] = 2.0, 1.0                       # experts 0, 1: rank 0
    logits[1, 6], logits[1, 2] = 3.0, 2.5                       # ranks 3 and 1
    logits[2, 4], logits[2, 5] = 1.0, 0.5                       # rank 2
    idx, w = oracle.route_topk(logits, k)
    lay = oracle.dispatch_layout(idx, E, W)
    y = torch.randn(T * k, H, generator=torch.Generator().manual_seed(15), dtype=torch.float64)
    sop = lay["slot_of_pair"]
    full = oracle.combine(y, sop, w)
    p0 = oracle.combine_rank(y, sop, w, lay["rank_offsets"], 0)
    assert torch.equal(p0[0], full[0])
    for r in (1, 2, 3):
        assert bool((oracle.combine_rank(y, sop, w, lay["rank_offsets"], r)[0] == 0).all())
    assert bool((p0[1:] == 0).all())                           # tokens 1, 2 have no rank-0 pick


def test_dropped_pairs_belong_to_no_rank():
    """Under a capacity, a dropped pair (slot -1) lies in no rank's slab."""
    T, k, E, W, H = 40, 2, 4, 2, 3
    g = torch.Generator().manual_seed(16)
    logits = torch.randn(T, E, generator=g)
    logits[:, 0] += 4.0                                         # expert 0 overflows
    idx, w = oracle.route_topk(logits, k)
    lay = oracle.dispatch_layout_capacity(idx, E, W, 6)
    assert lay["dropped"] > 0
    y = torch.randn(E * 6, H, generator=g, dtype=torch.float64)
    sop = lay["slot_of_pair"]
    parts = torch.stack([oracle.combine_rank(y, sop, w, lay["rank_offsets"], r)
                         for r in range(W)])
    ref = oracle.combine(y, sop, w)
    assert bool(((oracle.reduce_partials(parts) - ref).abs() <= 1e-12 * (1 + ref.abs())).all())


def test_reduce_rounds_once():
    """Rounding happens after the sum (bf16 spacing at 1 is 2^-7): (1 + 2^-9)
    + (2^-9 + 2^-10) = 1 + 0.625 * 2^-7 rounds up to 1 + 2^-7, while rounding
    the first partial to bf16 on its own (to 1) would lead to 1."""
    parts = torch.tensor([[[1.0 + 2.0 ** -9]], [[2.0 ** -9 + 2.0 ** -10]]], dtype=torch.float64)
    assert float(oracle.reduce_partials(parts, "bf16").float()) == 1.0 + 2.0 ** -7
    assert float(oracle.round_to(parts[0], "bf16").float()) == 1.0
