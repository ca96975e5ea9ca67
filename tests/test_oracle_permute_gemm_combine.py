"""Pins for the oracle's permute, grouped SwiGLU GEMM and combine.

Permute = "sent = x[order]" of "Expert Parallelism" (aiwiki),
"Implementation", with the FP8 payload of "Expert parallelism and
all-to-all", "Traffic math".  GEMM = "each GPU runs its local experts ... as
one grouped matrix multiply" ("Walking through one MoE layer").  Combine =
"y[order] = back" (aiwiki) plus "takes a weighted sum into the residual
stream" (step 4 of "Walking through one MoE layer").
"""
import numpy as np
import pytest
import torch

import oracle
from expert_parallelism_b200 import workloads


def _layout_for(T, k, E, W, seed=0):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    idx = torch.tensor(idx, dtype=torch.int32)
    return idx, oracle.dispatch_layout(idx, E, W)


# ----------------------------------------------------------------- permute
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_permute_is_row_copy(dt):
    T, H, k, E = 33, 64, 3, 8
    idx, lay = _layout_for(T, k, E, 2)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(1)).to(workloads.TORCH_DTYPE[dt])
    xp, sc = oracle.permute(x, k, lay["pair_of_slot"], dt)
    assert sc is None
    pos = lay["pair_of_slot"].long()
    ref = x[pos // k]
    assert torch.equal(xp.view(torch.int16 if dt == "bf16" else torch.int32),
                       ref.view(torch.int16 if dt == "bf16" else torch.int32))


def test_permute_fp8_blocks():
    T, H, k, E = 9, 384, 2, 4
    idx, lay = _layout_for(T, k, E, 2, seed=3)
    g = torch.Generator().manual_seed(2)
    x = torch.randn(T, H, generator=g)
    x[0, 0:128] = 0.0                                   # zero block -> scale 1
    x[1, 128:256] = torch.linspace(-1, 1, 128)
    x[1, 200] = 448.0 * 2.0 ** -3                       # amax = 448 * 2^-3
    x[2, 256:384] *= 0.0
    x[2, 300] = -448.0 * 4.0                            # amax = 448 * 2^2, negative
    x = x.to(torch.bfloat16)
    xp, sc = oracle.permute(x, k, lay["pair_of_slot"], "e4m3")
    q = xp.view(torch.uint8)
    pos = lay["pair_of_slot"].tolist()
    for s, p in enumerate(pos):
        t = p // k
        if t == 0:
            assert sc[s, 0].item() == 1.0 and int(q[s, :128].abs().sum()) == 0
        if t == 1:
            assert sc[s, 1].item() == 2.0 ** -3 and q[s, 200].item() == 0x7E
        if t == 2:
            assert sc[s, 2].item() == 4.0 and q[s, 300].item() == 0xFE
    # every slot of one token carries identical bytes and scales
    for t in range(T):
        slots = [s for s, p in enumerate(pos) if p // k == t]
        for s in slots[1:]:
            assert torch.equal(q[s], q[slots[0]]) and torch.equal(sc[s], sc[slots[0]])
    # reconstruction error within e4m3's spacing: relative 2^-4 for normals,
    # absolute 2^-10 * scale in the subnormal range
    deq = oracle.e4m3_decode(q).reshape(len(pos), H // 128, 128) * sc.double()[:, :, None]
    ref = x.double()[torch.tensor(pos) // k].reshape(len(pos), H // 128, 128)
    bound = torch.maximum(ref.abs() * 2.0 ** -4, sc.double()[:, :, None] * 2.0 ** -10)
    assert bool(((deq - ref).abs() <= bound * (1 + 1e-12)).all())


# ----------------------------------------------------------------- gemm
def _np_swiglu_expert(a, w13, w2, I, round_h):
    """h unrounded; y from h rounded to its storage type (as the path stores
    it before the down projection)."""
    g = a @ w13[:I].T
    u = a @ w13[I:].T
    h = g / (1 + np.exp(-g)) * u
    return h, round_h(h) @ w2.T


@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_gemm_matches_numpy_fp64(wdt):
    wl = workloads.Workload("t", 48, 64, 4, 2, 96, 2, wdt, wdt, wdt)
    inp = workloads.layer_inputs(wl)
    idx, w = oracle.route_topk(inp["logits"], wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    xp, _ = oracle.permute(inp["x"], wl.k, lay["pair_of_slot"], wl.payload)
    h, y, done = oracle.grouped_gemm(xp, None, lay["expert_offsets"], 0, wl.E,
                                     inp["w13"], inp["w2"])
    assert done == wl.N
    tdt = workloads.TORCH_DTYPE[wdt]
    rnd = lambda v: torch.tensor(v).to(tdt).double().numpy()
    off = lay["expert_offsets"].tolist()
    for e in range(wl.E):
        a = xp[off[e]:off[e + 1]].double().numpy()
        hr, yr = _np_swiglu_expert(a, inp["w13"][e].double().numpy(),
                                   inp["w2"][e].double().numpy(), wl.I, rnd)
        # both sides fp64; only the summation order differs
        np.testing.assert_allclose(h[off[e]:off[e + 1]].numpy(), hr, rtol=1e-12,
                                   atol=1e-12 * np.abs(hr).max())
        np.testing.assert_allclose(y[off[e]:off[e + 1]].numpy(), yr, rtol=1e-12,
                                   atol=1e-12 * np.abs(yr).max())


def test_gemm_one_hot_weights_pin_indices():
    """One-hot W13 / W2: gate row i picks x[pi(i)], up row i picks
    x[sigma(i)], W2 row o picks h[tau(o)].  Then h_i = silu(x_pi(i)) *
    x_sigma(i) and y_o = h_tau(o): a swapped gate/up or a transposed weight
    fails."""
    H = I = 16
    rng = np.random.default_rng(4)
    pi, sigma, tau = rng.permutation(H), rng.permutation(H), rng.permutation(I)
    w13 = np.zeros((1, 2 * I, H), np.float32)
    w13[0, np.arange(I), pi] = 1.0
    w13[0, I + np.arange(I), sigma] = 1.0
    w2 = np.zeros((1, H, I), np.float32)
    w2[0, np.arange(H), tau] = 1.0
    xp = torch.tensor(rng.normal(0, 1, (5, H)).astype(np.float32))
    off = torch.tensor([0, 5], dtype=torch.int32)
    h, y, _ = oracle.grouped_gemm(xp, None, off, 0, 1, torch.tensor(w13), torch.tensor(w2))
    x = xp.double().numpy()
    hr = x[:, pi] / (1 + np.exp(-x[:, pi])) * x[:, sigma]
    np.testing.assert_allclose(h.numpy(), hr, rtol=1e-15, atol=0)
    # the down projection reads h as stored (fp32 here)
    assert np.array_equal(y.numpy(), h.numpy().astype(np.float32).astype(np.float64)[:, tau])


def test_gemm_fp8_payload_dequant_then_bf16():
    wl = workloads.Workload("t8", 24, 256, 4, 2, 64, 2, "bf16", "e4m3", "bf16")
    inp = workloads.layer_inputs(wl)
    idx, w = oracle.route_topk(inp["logits"], wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    xp, sc = oracle.permute(inp["x"], wl.k, lay["pair_of_slot"], "e4m3")
    h, y, _ = oracle.grouped_gemm(xp, sc, lay["expert_offsets"], 0, wl.E, inp["w13"], inp["w2"])
    # library route: torch's e4m3 -> fp32, fp32 multiply by the block scale,
    # torch's fp32 -> bf16, then numpy fp64 matmuls
    deq = (xp.to(torch.float32).reshape(-1, 2, 128) * sc[:, :, None]).reshape(-1, 256)
    a_all = deq.to(torch.bfloat16).double().numpy()
    rnd = lambda v: torch.tensor(v).to(torch.bfloat16).double().numpy()
    off = lay["expert_offsets"].tolist()
    for e in range(wl.E):
        hr, yr = _np_swiglu_expert(a_all[off[e]:off[e + 1]], inp["w13"][e].double().numpy(),
                                   inp["w2"][e].double().numpy(), wl.I, rnd)
        np.testing.assert_allclose(h[off[e]:off[e + 1]].numpy(), hr, rtol=1e-12,
                                   atol=1e-12 * np.abs(hr).max())
        np.testing.assert_allclose(y[off[e]:off[e + 1]].numpy(), yr, rtol=1e-12,
                                   atol=1e-12 * np.abs(yr).max())


def test_gemm_expert_subset_and_row_mask():
    wl = workloads.Workload("ts", 40, 64, 8, 2, 32, 4, "bf16", "bf16", "bf16")
    inp = workloads.layer_inputs(wl)
    idx, w = oracle.route_topk(inp["logits"], wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    xp, _ = oracle.permute(inp["x"], wl.k, lay["pair_of_slot"], "bf16")
    off = lay["expert_offsets"]
    h, y, _ = oracle.grouped_gemm(xp, None, off, 0, wl.E, inp["w13"], inp["w2"])
    # rank 1 of 4 holds experts 2, 3 and only their weights
    h1, y1, d1 = oracle.grouped_gemm(xp, None, off, 2, 2, inp["w13"][2:4].contiguous(),
                                     inp["w2"][2:4].contiguous())
    lo, hi = off[2].item(), off[4].item()
    assert d1 == hi - lo
    assert torch.equal(y1[lo:hi], y[lo:hi])
    assert torch.isnan(y1[:lo]).all() and torch.isnan(y1[hi:]).all()
    mask = torch.zeros(wl.N, dtype=torch.bool)
    mask[::3] = True
    hm, ym, dm = oracle.grouped_gemm(xp, None, off, 0, wl.E, inp["w13"], inp["w2"], mask)
    assert dm == int(mask.sum())
    assert torch.equal(ym[mask], y[mask])
    # storage rounding on request
    hb, yb, _ = oracle.grouped_gemm(xp, None, off, 0, wl.E, inp["w13"], inp["w2"], out="bf16")
    assert torch.equal(yb.view(torch.int16), oracle.bf16_round(y).view(torch.int16))


# ----------------------------------------------------------------- combine
def test_combine_identity_experts_return_x_bf16():
    """Identity experts (y := xp) and renormalised router weights give
    back x bit-exactly in bf16: the weights sum to 1 within a few fp32
    ulps, far below half a bf16 ulp."""
    wl = workloads.Workload("ci", 200, 64, 16, 4, 8, 4, "bf16", "bf16", "bf16")
    inp = workloads.layer_inputs(wl, with_weights=False)
    idx, w = oracle.route_topk(inp["logits"], wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    xp, _ = oracle.permute(inp["x"], wl.k, lay["pair_of_slot"], "bf16")
    out = oracle.combine(xp, lay["slot_of_pair"], w)
    assert torch.equal(oracle.bf16_round(out).view(torch.int16), inp["x"].view(torch.int16))
    assert torch.equal(oracle.combine(xp, lay["slot_of_pair"], w, "bf16").view(torch.int16),
                       inp["x"].view(torch.int16))


def test_combine_identity_experts_fp32_and_dyadic():
    wl = workloads.Workload("cf", 100, 32, 8, 3, 8, 2, "f32", "f32", "f32")
    inp = workloads.layer_inputs(wl, with_weights=False)
    idx, w = oracle.route_topk(inp["logits"], wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    xp, _ = oracle.permute(inp["x"], wl.k, lay["pair_of_slot"], "f32")
    out = oracle.combine(xp, lay["slot_of_pair"], w, "f32")
    x = inp["x"]
    ulp = torch.abs(x) * 2.0 ** -23
    assert bool(((out - x).abs() <= (wl.k + 1) * ulp).all())
    wd = torch.tensor([[0.25, 0.5, 0.25]] * wl.T, dtype=torch.float32)  # dyadic
    out = oracle.combine(xp, lay["slot_of_pair"], wd)
    assert torch.equal(out, x.double())


def test_combine_fp8_identity_returns_dequantised_x():
    wl = workloads.Workload("c8", 30, 256, 8, 2, 8, 2, "bf16", "e4m3", "bf16")
    inp = workloads.layer_inputs(wl, with_weights=False)
    idx, w = oracle.route_topk(inp["logits"], wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    xp, sc = oracle.permute(inp["x"], wl.k, lay["pair_of_slot"], "e4m3")
    deq = (xp.to(torch.float32).reshape(wl.N, 2, 128) * sc[:, :, None]).reshape(wl.N, 256)
    y = deq.to(torch.bfloat16)                         # identity expert on the FP8 payload
    out = oracle.combine(y, lay["slot_of_pair"], w, "bf16")
    first = lay["slot_of_pair"].view(wl.T, wl.k)[:, 0].long()
    assert torch.equal(out.view(torch.int16), y[first].view(torch.int16))


def test_combine_k1_unit_weight_is_unsort():
    """k=1, w=1: combine is the sketch's y[order] = back."""
    rng = np.random.default_rng(9)
    T, E, H = 50, 8, 16
    idx = rng.integers(0, E, size=T)
    lay = oracle.dispatch_layout(torch.tensor(idx[:, None], dtype=torch.int32), E, 2)
    back = torch.tensor(rng.normal(0, 1, (T, H)).astype(np.float32))
    out = oracle.combine(back, lay["slot_of_pair"], torch.ones(T, 1))
    order = np.argsort(idx, kind="stable")
    yref = torch.empty_like(back)
    yref[torch.tensor(order)] = back
    assert torch.equal(out, yref.double())


def test_combine_skips_dropped_pairs():
    y = torch.arange(12, dtype=torch.float32).reshape(3, 4)
    sop = torch.tensor([0, -1, 2, 1], dtype=torch.int32)
    w = torch.tensor([[0.5, 0.5], [0.25, 0.75]])
    out = oracle.combine(y, sop, w)
    assert out.tolist() == [[0.0, 0.5, 1.0, 1.5], [5.0, 6.0, 7.0, 8.0]]


# ----------------------------------------------------------------- whole layer
def test_layer_matches_plain_torch_fp64_tiny():
    """The whole tiny layer against a composition of plain torch fp64 ops:
    a stable descending sort for top-k, softmax, a stable argsort for the
    layout, torch matmuls, index_add for combine."""
    wl = workloads.WORKLOADS["tiny"]
    inp = workloads.layer_inputs(wl)
    r = oracle.layer(wl, inp)
    L = inp["logits"]
    order = torch.sort(L, dim=1, descending=True, stable=True).indices[:, :wl.k]
    assert torch.equal(r["topk_idx"].long(), order)
    pick = torch.gather(L.double(), 1, order)
    wref = torch.softmax(pick, dim=1)
    assert torch.allclose(r["topk_w"].double(), wref, rtol=1e-6, atol=0)
    flat = order.reshape(-1)
    perm = torch.sort(flat, stable=True).indices
    assert torch.equal(r["pair_of_slot"].long(), perm)
    x = inp["x"].double()
    xp = x[perm // wl.k]
    y = torch.empty(wl.N, wl.H, dtype=torch.float64)
    for e in range(wl.E):
        m = flat[perm] == e
        a = xp[m]
        w13, w2 = inp["w13"][e].double(), inp["w2"][e].double()
        g, u = a @ w13[:wl.I].T, a @ w13[wl.I:].T
        h = (torch.nn.functional.silu(g) * u).float().double()      # h as stored (fp32)
        y[m] = h @ w2.T
    rel = lambda a, b: float(((a - b).abs() / b.pow(2).mean(1, keepdim=True).sqrt()).max())
    assert rel(r["y"], y) < 1e-12
    out = torch.zeros(wl.T, wl.H, dtype=torch.float64)
    out.index_add_(0, perm // wl.k, y * r["topk_w"].double().reshape(-1)[perm][:, None])
    assert rel(r["out"], out) < 1e-12


def test_traffic_worked_example():
    import json
    import os
    from expert_parallelism_b200 import traffic
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "traffic_example.json")))
    b = traffic.dispatch_combine_bytes_per_token(g["k"], g["H"], g["bytes_per_element"])
    assert b == g["per_token_per_layer_bytes"] == 114688
    assert b // 1024 == g["per_token_per_layer_kib"]
    assert g["layers"] * b // 1024 == g["per_token_all_layers_kib"]
    total = g["prefill_tokens"] * b * g["layers"]
    assert total == 45_875_200_000 and round(total / 1e9) == 46
    assert abs(total / 1e9 - g["prefill_all_layers_gb_approx"]) < 1.0
    # dispatch bytes from a layout: every routed row once
    wl = workloads.Workload("tr", 64, 7168, 256, 8, 8, 8, "bf16", "e4m3", "bf16")
    idx, w = oracle.route_topk(workloads.router_logits(wl), wl.k)
    lay = oracle.dispatch_layout(idx, wl.E, wl.W)
    assert traffic.dispatch_bytes_from_layout(int(lay["rank_offsets"][-1]), wl.H, 1) == \
        wl.T * wl.k * wl.H == 64 * b // 2
