"""Pins for the oracle's router top-k and dispatch layout.

Router: "Expert parallelism and all-to-all", "Walking through one MoE
layer" (each token gets a list of (expert, weight) picks) and the
Transformers docs' (top_k_index, top_k_weights) call signature.  Layout:
"Expert Parallelism" (aiwiki), "Implementation" (sort by destination so
each peer's tokens are one slab; per-rank bincount) and the Transformers
docs, "How the sizes combine" (rank r owns E/ep_size consecutive experts).
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _key(vals, e):
    return (-float(vals[e]), e)


# ----------------------------------------------------------------- top-k
@pytest.mark.parametrize("E", [3, 5, 8, 10])
def test_topk_brute_force_subsets(E):
    rng = np.random.default_rng(E)
    T = 40
    # coarse values make ties common
    logits = torch.tensor(rng.integers(-3, 4, size=(T, E)).astype(np.float32) * 0.5)
    for k in range(1, E + 1):
        idx, w = oracle.route_topk(logits, k)
        for t in range(T):
            row = logits[t].tolist()
            picked = idx[t].tolist()
            # the unique k-subset whose every member beats every non-member
            dominating = [S for S in itertools.combinations(range(E), k)
                          if all(_key(row, a) < _key(row, b)
                                 for a in S for b in range(E) if b not in S)]
            assert len(dominating) == 1
            assert sorted(picked) == list(dominating[0])
            # within the picks: logit descending, id ascending
            assert picked == sorted(picked, key=lambda e: _key(row, e))


def test_topk_ties_lower_id_first_and_signed_zero():
    logits = torch.tensor([[1.0, 1.0, 1.0, 1.0],
                           [0.0, -0.0, 0.0, -1.0],
                           [-0.0, 0.0, 2.0, 2.0]], dtype=torch.float32)
    idx, w = oracle.route_topk(logits, 2)
    assert idx.tolist() == [[0, 1], [0, 1], [2, 3]]
    # two equal top logits with k=2: both weights exactly 1/2
    assert w.tolist() == [[0.5, 0.5], [0.5, 0.5], [0.5, 0.5]]


def test_topk_weights_equal_renormalised_full_softmax():
    rng = np.random.default_rng(7)
    T, E, k = 64, 32, 6
    logits = torch.tensor(rng.normal(0, 2, (T, E)).astype(np.float32))
    idx, w = oracle.route_topk(logits, k)
    L = logits.double().numpy()
    full = np.exp(L - L.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)           # softmax over all E
    picked = np.take_along_axis(full, idx.long().numpy(), axis=1)
    ref = picked / picked.sum(axis=1, keepdims=True)  # restrict, renormalise
    np.testing.assert_allclose(w.double().numpy(), ref, rtol=1e-6, atol=0)
    np.testing.assert_allclose(w.double().sum(1).numpy(), 1.0, atol=1e-6)
    # k = E: the weights are the full softmax, in picked order
    idx, w = oracle.route_topk(logits, E)
    np.testing.assert_allclose(w.double().numpy(),
                               np.take_along_axis(full, idx.long().numpy(), axis=1),
                               rtol=1e-6)


# ----------------------------------------------------------------- layout
def _check_layout(idx, E, W, lay):
    T, k = idx.shape
    N = T * k
    flat = idx.reshape(-1).tolist()
    valid = [p for p in range(N) if 0 <= flat[p] < E]
    counts = lay["expert_counts"].tolist()
    off = lay["expert_offsets"].tolist()
    sop = lay["slot_of_pair"].tolist()
    pos = lay["pair_of_slot"].tolist()
    assert sum(counts) == len(valid)
    assert off[0] == 0 and all(off[e + 1] - off[e] == counts[e] for e in range(E))
    # bijection between valid pairs and slots [0, off[E])
    assert sorted(sop[p] for p in valid) == list(range(off[E]))
    for p in valid:
        assert pos[sop[p]] == p
    assert all(sop[p] == -1 for p in range(N) if p not in set(valid))
    assert all(pos[s] == -1 for s in range(off[E], N))
    # every slot of segment e holds a pair routed to e; pair index strictly
    # increases inside a segment (stability)
    for e in range(E):
        seg = pos[off[e]:off[e + 1]]
        assert all(flat[p] == e for p in seg)
        assert all(a < b for a, b in zip(seg, seg[1:]))
    ro = lay["rank_offsets"].tolist()
    assert ro == [off[r * E // W] for r in range(W + 1)]


@pytest.mark.parametrize("T,k,E,W", [(0, 2, 8, 2), (1, 1, 4, 4), (1, 4, 8, 2), (37, 3, 16, 4),
                                     (256, 2, 8, 2), (129, 8, 64, 8)])
def test_layout_invariants(T, k, E, W):
    rng = np.random.default_rng(T * 131 + k)
    # distinct experts per token, skewed so some experts get nothing
    p = np.arange(E, 0, -1, dtype=np.float64) ** 2
    p /= p.sum()
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]) \
        if T else np.zeros((0, k), np.int64)
    idx = torch.tensor(idx, dtype=torch.int32).reshape(T, k)
    lay = oracle.dispatch_layout(idx, E, W)
    assert lay["skipped"] == 0
    _check_layout(idx, E, W, lay)


def test_layout_k1_is_stable_argsort_and_bincount():
    """k=1 reduces to the aiwiki sketch: order = argsort(idx) (read as
    stable), counts = bincount(idx // per_rank, minlength=world)."""
    rng = np.random.default_rng(11)
    T, E, W = 500, 16, 4
    idx = rng.integers(0, E, size=T)
    lay = oracle.dispatch_layout(torch.tensor(idx[:, None], dtype=torch.int32), E, W)
    order = np.argsort(idx, kind="stable")
    assert lay["pair_of_slot"].tolist() == order.tolist()
    per_rank = E // W
    counts = np.bincount(idx // per_rank, minlength=W)
    assert np.diff(lay["rank_offsets"].numpy()).tolist() == counts.tolist()


def test_layout_rank_slabs_match_ownership_picture():
    g = json.load(open(os.path.join(GOLDEN, "rank_ownership_e8.json")))
    E = g["num_experts"]
    rng = np.random.default_rng(5)
    T, k = 300, 2
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    flat = idx.reshape(-1)
    for ep, owned in g["ep_size"].items():
        W = int(ep)
        lay = oracle.dispatch_layout(torch.tensor(idx, dtype=torch.int32), E, W)
        ro = lay["rank_offsets"].tolist()
        pos = lay["pair_of_slot"].tolist()
        for r in range(W):
            slab = pos[ro[r]:ro[r + 1]]
            assert sorted(set(int(flat[p]) for p in slab)) == \
                sorted(e for e in owned[r] if (flat == e).any())
            assert len(slab) == int(np.isin(flat, owned[r]).sum())


def test_layout_skips_out_of_range_ids():
    idx = torch.tensor([[0, 9], [-1, 3], [3, 0]], dtype=torch.int32)
    lay = oracle.dispatch_layout(idx, 8, 2)
    assert lay["skipped"] == 2
    assert lay["slot_of_pair"].tolist() == [0, -1, -1, 2, 3, 1]
    assert lay["pair_of_slot"].tolist() == [0, 5, 3, 4, -1, -1]
    assert lay["expert_counts"].tolist() == [2, 0, 0, 2, 0, 0, 0, 0]
