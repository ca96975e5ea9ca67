"""Pins of the oracle's group-limited routing.

Source: "Expert Parallelism" (aiwiki), "Hiding the latency", topology-aware
routing: each token goes to experts on at most M nodes.  Reading: G equal
groups of consecutive experts; a group's score is its largest logit; the M
best groups are kept (ties: lower id); the top k of their experts are the
picks; softmax over the picks.
"""
import numpy as np
import pytest
import torch

import oracle


def _groups_of(idx, per):
    return [set(int(e) // per for e in row) for row in idx]


def test_all_groups_kept_is_plain_topk():
    g = torch.Generator().manual_seed(11)
    for (T, E, k, G) in [(200, 64, 6, 8), (50, 256, 8, 8), (30, 12, 5, 3)]:
        lg = torch.randn(T, E, generator=g)
        i0, w0 = oracle.route_topk(lg, k)
        i1, w1 = oracle.route_topk_grouped(lg, k, G, G)
        assert torch.equal(i0, i1) and torch.equal(w0, w1)


def test_unconstrained_picks_on_few_groups_are_unchanged():
    """A group holding one of the plain top-k picks scores at least the k-th
    largest logit, and a group holding none scores less; so when the plain
    picks span at most M groups those groups are among the M kept and the
    result is the plain top-k."""
    g = torch.Generator().manual_seed(12)
    T, E, k, G, M = 2000, 64, 4, 8, 3
    lg = torch.randn(T, E, generator=g)
    i0, w0 = oracle.route_topk(lg, k)
    i1, w1 = oracle.route_topk_grouped(lg, k, G, M)
    per = E // G
    few = torch.tensor([len(s) <= M for s in _groups_of(i0.tolist(), per)])
    assert few.sum() > 100 and (~few).sum() > 100          # both kinds occur
    assert torch.equal(i1[few], i0[few]) and torch.equal(w1[few], w0[few])
    assert not torch.equal(i1[~few], i0[~few])


def test_picks_span_at_most_m_groups_and_are_the_top_of_the_kept_ones():
    g = torch.Generator().manual_seed(13)
    T, E, k, G, M = 500, 256, 8, 8, 4
    lg = torch.randn(T, E, generator=g)
    idx, w = oracle.route_topk_grouped(lg, k, G, M)
    per = E // G
    L = lg.numpy()
    for t in range(T):
        picks = idx[t].tolist()
        groups = {e // per for e in picks}
        assert len(groups) <= M
        scores = L[t].reshape(G, per).max(axis=1)
        kept = sorted(range(G), key=lambda q: (-scores[q], q))[:M]
        # the group of the token's best expert is always kept
        assert int(np.argmax(L[t])) // per in kept
        # every pick is in a kept group and beats every unpicked expert of the kept groups
        allowed = [e for e in range(E) if e // per in kept]
        assert set(picks) <= set(allowed)
        worst = min(L[t][e] for e in picks)
        assert all(L[t][e] <= worst for e in allowed if e not in picks)
        # picks in (logit desc, id asc) order; weights are the softmax of the picks
        vals = [L[t][e] for e in picks]
        assert all(vals[i] >= vals[i + 1] for i in range(k - 1))
        z = np.exp(np.array(vals, dtype=np.float64) - vals[0])
        assert np.allclose(w[t].numpy(), z / z.sum(), rtol=1e-6, atol=0)


def test_worked_examples():
    lg = torch.tensor([[0.1, 5.0, 0.2, 0.3, 4.0, 4.5, 0.0, -1.0],
                       [3.0, 0.0, 2.9, 2.8, 2.7, 0.0, 0.0, 0.0],
                       [1.0, 1.0, 2.0, 2.0, 2.0, 0.5, 2.0, 2.0]])
    # 4 groups of 2: token 0 keeps groups {0, 2} -> experts 1, 5, 4
    # token 1 keeps {0, 1} -> 0, 2, 3; token 2: groups 1, 2, 3 tie at 2.0,
    # the lower ids 1 and 2 are kept -> experts 2, 3, 4
    idx, w = oracle.route_topk_grouped(lg, 3, 4, 2)
    assert idx.tolist() == [[1, 5, 4], [0, 2, 3], [2, 3, 4]]
    assert abs(float(w[2].sum()) - 1.0) < 1e-6 and float(w[2][0]) == float(w[2][1])
    # one group: token 0 keeps group 0 only -> experts 1, 0
    idx, _ = oracle.route_topk_grouped(lg[:1], 2, 4, 1)
    assert idx.tolist() == [[1, 0]]


def test_invalid_sizes_are_rejected():
    lg = torch.zeros(2, 8)
    for (k, G, M) in [(3, 4, 1), (2, 3, 1), (2, 4, 5), (2, 4, 0)]:
        with pytest.raises(ValueError):
            oracle.route_topk_grouped(lg, k, G, M)
