"""GPU edge cases: empty and one-token batches, skipped expert ids, the
kernels' maximum sizes, multi-chunk scans, one logical rank's slab run on
its own, invalid calls that must not touch outputs, and CUDA-graph capture
of the whole layer."""
import numpy as np
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

from parity_helpers import BF16_TOL, GpuLayer, bits, h_ok, rowwise_ok

SENT = -7


def _layout_bufs(T, k, E, W, dev):
    i32 = dict(dtype=torch.int32, device=dev)
    N = max(T * k, 1)
    return dict(expert_counts=torch.full((E,), SENT, **i32),
                expert_offsets=torch.full((E + 1,), SENT, **i32),
                rank_offsets=torch.full((W + 1,), SENT, **i32),
                slot_of_pair=torch.full((N,), SENT, **i32),
                pair_of_slot=torch.full((N,), SENT, **i32),
                ws=torch.empty(moe.moe_dispatch_layout_workspace_bytes(T, k, E), dtype=torch.uint8,
                               device=dev),
                st=torch.zeros(1, **i32))


def _run_layout(idx, E, W, dev):
    T, k = idx.shape
    b = _layout_bufs(T, k, E, W, dev)
    moe.moe_dispatch_layout(idx.to(dev), E, W, b["expert_counts"], b["expert_offsets"],
                            b["rank_offsets"], b["slot_of_pair"], b["pair_of_slot"], b["ws"],
                            b["st"])
    status = moe.moe_check_status(b["st"])
    return b, status


def _assert_layout_equal(b, lay, N):
    for key in ["expert_counts", "expert_offsets", "rank_offsets"]:
        assert torch.equal(b[key].cpu(), lay[key]), key
    for key in ["slot_of_pair", "pair_of_slot"]:
        assert torch.equal(b[key].cpu()[:N], lay[key]), key


@pytest.mark.gpu
def test_empty_batch(cuda_device):
    E, W, k = 8, 2, 2
    b, st = _run_layout(torch.zeros(0, k, dtype=torch.int32), E, W, cuda_device)
    assert st == 0
    assert b["expert_counts"].cpu().tolist() == [0] * E
    assert b["expert_offsets"].cpu().tolist() == [0] * (E + 1)
    assert b["rank_offsets"].cpu().tolist() == [0] * (W + 1)
    logits = torch.zeros(0, E, device=cuda_device)
    idx = torch.zeros(0, k, dtype=torch.int32, device=cuda_device)
    w = torch.zeros(0, k, device=cuda_device)
    moe.moe_route_topk(logits, idx, w)
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device=cuda_device)
    xp = torch.zeros(0, 64, dtype=torch.bfloat16, device=cuda_device)
    moe.moe_permute(x, k, b["slot_of_pair"], xp)
    out = torch.zeros(0, 64, dtype=torch.bfloat16, device=cuda_device)
    moe.moe_combine(xp, b["slot_of_pair"], w, out)
    torch.cuda.synchronize()


@pytest.mark.gpu
@pytest.mark.parametrize("T,k,E,W", [(1, 1, 1, 1), (1, 4, 8, 2), (3, 2, 64, 8)])
def test_one_token_and_empty_experts(T, k, E, W, cuda_device):
    wl = workloads.Workload("e", T, 64, E, k, 32, W, "bf16", "bf16", "bf16")
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    r = oracle.layer(wl, g.inputs)
    assert torch.equal(g.buf.topk_idx.cpu(), r["topk_idx"])
    assert torch.equal(g.buf.expert_offsets.cpu(), r["expert_offsets"])
    ok, worst = rowwise_ok(g.buf.out.cpu(), r["out"], BF16_TOL)
    assert ok, worst


@pytest.mark.gpu
def test_bad_expert_ids_are_skipped_and_reported(cuda_device):
    E, W = 8, 2
    idx = torch.tensor([[0, 9], [-1, 3], [3, 0], [7, 100]], dtype=torch.int32)
    b, st = _run_layout(idx, E, W, cuda_device)
    assert moe.STATUS[st] == "MOE_ERR_BAD_INDEX"
    lay = oracle.dispatch_layout(idx, E, W)
    _assert_layout_equal(b, lay, idx.numel())
    # permute and combine skip the dropped pairs
    T, k, H = 4, 2, 64
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    xp = torch.zeros(T * k, H, dtype=torch.bfloat16, device=cuda_device)
    moe.moe_permute(x.to(cuda_device), k, b["slot_of_pair"], xp)
    w = torch.full((T, k), 0.5, device=cuda_device)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=cuda_device)
    moe.moe_combine(xp, b["slot_of_pair"], w, out)
    torch.cuda.synchronize()
    xp_o, _ = oracle.permute(x, k, lay["pair_of_slot"], "bf16")
    out_o = oracle.combine(xp_o, lay["slot_of_pair"], w.cpu(), "bf16")   # dyadic weights: exact
    assert torch.equal(bits(out), bits(out_o))
    assert moe.moe_check_status(b["st"]) == 0       # the status word was cleared


@pytest.mark.gpu
@pytest.mark.parametrize("T,k,E,W", [(300, 16, 1024, 8), (20000, 8, 256, 8), (4097, 6, 64, 4)])
def test_route_layout_max_sizes_and_multichunk_scan(T, k, E, W, cuda_device):
    wl = workloads.Workload("m", T, 64, E, k, 32, W, "bf16", "bf16", "bf16")
    logits = workloads.router_logits(wl)
    idx = torch.empty(T, k, dtype=torch.int32, device=cuda_device)
    w = torch.empty(T, k, device=cuda_device)
    moe.moe_route_topk(logits.to(cuda_device), idx, w)
    idx_o, w_o = oracle.route_topk(logits, k)
    assert torch.equal(idx.cpu(), idx_o)
    assert bool(((w.cpu().double() - w_o.double()).abs() <= 1e-5 * w_o.double().abs()).all())
    b, st = _run_layout(idx_o, E, W, cuda_device)
    assert st == 0
    _assert_layout_equal(b, oracle.dispatch_layout(idx_o, E, W), T * k)


@pytest.mark.gpu
def test_one_rank_slab_gemm(cuda_device):
    """Logical rank r runs only its experts [r*E/W, (r+1)*E/W) with its own
    weight shard; rows outside its slab stay untouched."""
    wl = workloads.Workload("r", 512, 256, 16, 4, 192, 4, "bf16", "bf16", "bf16")
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    b = g.buf
    r, Er = 2, wl.E // wl.W
    h = torch.full_like(b.h, 3.0)
    y = torch.full_like(b.y, 3.0)
    moe.moe_grouped_gemm(b.xp, None, b.expert_offsets, r * Er, Er,
                         g.w13[r * Er:(r + 1) * Er].contiguous(),
                         g.w2[r * Er:(r + 1) * Er].contiguous(), h, y, None, b.dev_status)
    torch.cuda.synchronize()
    ro = b.rank_offsets.cpu().tolist()
    lo, hi = ro[r], ro[r + 1]
    assert torch.equal(bits(y[lo:hi]), bits(b.y[lo:hi]))
    assert bool((y[:lo] == 3.0).all()) and bool((y[hi:] == 3.0).all())


@pytest.mark.gpu
def test_invalid_calls_touch_nothing(cuda_device):
    E, W, T, k = 8, 3, 16, 2           # E % W != 0
    idx = torch.zeros(T, k, dtype=torch.int32, device=cuda_device)
    b = _layout_bufs(T, k, E, 2, cuda_device)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_dispatch_layout(idx, E, W, b["expert_counts"], b["expert_offsets"],
                                b["rank_offsets"], b["slot_of_pair"], b["pair_of_slot"], b["ws"],
                                b["st"])
    assert ei.value.status == "MOE_ERR_INVALID_ARG"
    logits = torch.zeros(T, E, device=cuda_device)
    ti = torch.full((T, 9), SENT, dtype=torch.int32, device=cuda_device)
    tw = torch.full((T, 9), float(SENT), device=cuda_device)
    with pytest.raises(moe.MoEError):
        moe.moe_route_topk(logits, ti, tw)                     # k > E
    x = torch.zeros(T, 136, dtype=torch.bfloat16, device=cuda_device)
    xp = torch.full((T * k, 136), 5, dtype=torch.uint8, device=cuda_device).view(torch.float8_e4m3fn)
    sc = torch.full((T * k, 2), float(SENT), device=cuda_device)
    with pytest.raises(moe.MoEError):
        moe.moe_permute(x, k, b["slot_of_pair"], xp, sc)       # H % 128 != 0 for FP8
    torch.cuda.synchronize()
    for key in ["expert_counts", "expert_offsets", "rank_offsets", "slot_of_pair",
                "pair_of_slot"]:
        assert bool((b[key] == SENT).all()), key
    assert bool((ti == SENT).all()) and bool((tw == SENT).all())
    assert bool((xp.view(torch.uint8) == 5).all()) and bool((sc == SENT).all())


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["decode"])
def test_layer_captures_in_a_cuda_graph(name, cuda_device):
    """No host synchronisation inside the chain: the five calls capture in
    one CUDA graph, and a replay reproduces the eager result bit for bit."""
    wl = workloads.WORKLOADS[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    eager = g.buf.out.clone()
    g.buf.out.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        moe.layer_forward(wl, g.logits, g.x, g.w13, g.w2, g.buf, stream=s)   # warm-up
        s.synchronize()
        with torch.cuda.graph(graph, stream=s):
            moe.layer_forward(wl, g.logits, g.x, g.w13, g.w2, g.buf, stream=s)
    g.buf.out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(bits(g.buf.out), bits(eager))
    assert moe.moe_check_status(g.buf.dev_status) == 0
    del graph


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["small_fp8", "ragged_bf16"])
def test_layer_call_equals_the_five_calls(name, cuda_device):
    """moe_layer_forward (one call, events between steps) and
    moe_layer_forward_host (host inputs/output) give the five-call chain's
    results bit for bit."""
    from parity_helpers import workload
    wl = workload(name)
    g = GpuLayer(wl, cuda_device)
    b = g.buf
    moe.moe_route_topk(g.logits, b.topk_idx, b.topk_w)
    moe.moe_dispatch_layout(b.topk_idx, wl.E, wl.W, b.expert_counts, b.expert_offsets,
                            b.rank_offsets, b.slot_of_pair, b.pair_of_slot, b.layout_ws,
                            b.dev_status)
    moe.moe_permute(g.x, wl.k, b.slot_of_pair, b.xp, b.xp_scales)
    moe.moe_grouped_gemm(b.xp, b.xp_scales, b.expert_offsets, 0, wl.E, g.w13, g.w2, b.h, b.y,
                         b.gemm_ws, b.dev_status)
    moe.moe_combine(b.y, b.slot_of_pair, b.topk_w, b.out)
    torch.cuda.synchronize()
    five = b.out.clone()
    b.out.zero_()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    moe.moe_layer_forward(wl, g.logits, g.x, g.w13, g.w2, b, step_events=evs)
    torch.cuda.synchronize()
    assert torch.equal(bits(b.out), bits(five))
    assert all(evs[i].elapsed_time(evs[i + 1]) >= 0 for i in range(7))
    h_out = torch.zeros(b.out.shape, dtype=b.out.dtype).pin_memory()
    moe.moe_layer_forward_host(wl, g.inputs["logits"].pin_memory(), g.inputs["x"].pin_memory(),
                               h_out, torch.empty_like(g.logits), torch.empty_like(g.x), g.w13,
                               g.w2, b)
    torch.cuda.synchronize()
    assert torch.equal(bits(h_out), bits(five))
    assert moe.moe_check_status(b.dev_status) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("ydt", ["f32", "bf16"])
def test_gemm_rows_on_chunk_boundaries(ydt, cuda_device):
    """Expert row counts on and around every padding boundary of the grouped
    GEMM (multiples of 16 and of 256, empty experts), H and I not multiples
    of the weight tile: every row of h and y against the oracle."""
    counts = [0, 1, 15, 16, 17, 31, 32, 33, 0, 255, 256, 257, 511, 512, 513]
    E, H, I = len(counts), 320, 200
    wl = workloads.Workload("chunks", 1, H, E, 1, I, 1, "bf16", "bf16", "bf16", ydt=ydt)
    off = torch.tensor([0] + list(np.cumsum(counts)), dtype=torch.int32)
    n = int(off[-1])
    g = torch.Generator().manual_seed(7)
    xp = torch.randn(n, H, generator=g).to(torch.bfloat16)
    w13 = torch.stack([workloads.expert_w13(wl, e) for e in range(E)])
    w2 = torch.stack([workloads.expert_w2(wl, e) for e in range(E)])
    h_ref, y_ref, done = oracle.grouped_gemm(xp, None, off, 0, E, w13, w2)
    assert done == n
    dev = cuda_device
    h = torch.full((n, I), float("nan"), dtype=torch.bfloat16, device=dev)
    y = torch.full((n, H), float("nan"), dtype=workloads.TORCH_DTYPE[ydt], device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    moe.moe_grouped_gemm(xp.to(dev), None, off.to(dev), 0, E, w13.to(dev), w2.to(dev), h, y,
                         None, st)
    assert moe.moe_check_status(st) == 0
    ok, worst = h_ok(h.cpu(), h_ref, torch.bfloat16)
    assert ok, worst
    ok, worst = rowwise_ok(y.cpu(), y_ref, BF16_TOL)
    assert ok, worst
