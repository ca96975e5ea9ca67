"""GPU parity of the fused gather: the gate/up GEMM reads each routed row
from the token-major activations through pair_of_slot instead of from a
permuted copy.

Source: "Expert parallelism" (Transformers docs), "Choosing an
implementation": the Mega MoE implementation fuses the dispatch, the
experts and the combine into one kernel; on one GPU the dispatch's data
movement is this gather of the routed rows.

The gathered rows hold the very values the permute would have written (x's
rows for a bf16 payload; each token's bf16(decode(q) * scale) for an FP8
payload), and the MMA shapes, their order and the epilogue are unchanged,
so h, y (and its FP8 scales) and out must equal the unfused path's bit for
bit.  Small cases are also compared with the oracle directly.
"""
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

from parity_helpers import BF16_TOL, GpuLayer, bits, rowwise_ok, workload

W = workloads.Workload
CASES = {
    "small_bf16": workload("small_bf16"),
    "small_fp8": workload("small_fp8"),
    "small_fp8v": workload("small_fp8v"),
    # H = 200: the last k-step holds one 8-element piece, the rest read zeros
    "ragged_bf16": workload("ragged_bf16"),
    # > 320 rows per expert: balanced multi-pass experts
    "pair_bf16": workload("pair_bf16"),
    "pair_fp8": workload("pair_fp8"),
    # ~280 rows per expert: one pass with a second (tail) chunk
    "tail_bf16": W("tail_bf16", 560, 256, 4, 2, 192, 2, "bf16", "bf16", "bf16"),
    "tail_fp8": W("tail_fp8", 600, 384, 4, 2, 128, 2, "bf16", "e4m3", "bf16"),
    # fixed capacity: slots past each expert's count hold no pair
    "cap_fp8": W("cap_fp8", 600, 256, 8, 2, 192, 2, "bf16", "e4m3", "bf16",
                 capacity_factor=0.7),
    # fewer slots (E * C = 304) than tokens (600): the token rows need their own room
    "cap_fp8_few_slots": W("cap_fp8_few", 600, 256, 8, 2, 192, 2, "bf16", "e4m3", "bf16",
                           capacity_factor=0.25),
    # FP8 combine payload out of the same GEMM
    "fp8y": W("fp8y_f", 300, 256, 8, 2, 192, 2, "bf16", "e4m3", "bf16", ydt="e4m3"),
    # k = 8 picks per token
    "k8": W("k8_f", 256, 256, 16, 8, 128, 4, "bf16", "bf16", "bf16"),
}

SENTINEL = 0x5A


def _fused_buffers(wl, device):
    fb = moe.LayerBuffers(wl.replace(fused_gather=True), device)
    fb.xp.view(torch.uint8).fill_(SENTINEL)       # the fused path never writes xp
    return fb


def _run(wl, g, buf):
    moe.layer_forward(wl.replace(fused_gather=True), g.logits, g.x, g.w13, g.w2, buf)
    torch.cuda.synchronize()
    return moe.moe_check_status(buf.dev_status)


def _kept(buf, wl):
    n = moe.slot_rows(wl)
    return (buf.pair_of_slot[:n] >= 0).cpu()


def _assert_same(ref, fused, wl, skip_xp_check=False):
    """Bit-for-bit equality of the layer's results, over the computed slots."""
    kept = _kept(ref, wl)
    assert torch.equal(bits(fused.slot_of_pair), bits(ref.slot_of_pair))
    assert torch.equal(bits(fused.h.cpu()[kept]), bits(ref.h.cpu()[kept])), "h differs"
    assert torch.equal(bits(fused.y.cpu()[kept]), bits(ref.y.cpu()[kept])), "y differs"
    if ref.y_scales is not None:
        assert torch.equal(bits(fused.y_scales.cpu()[kept]), bits(ref.y_scales.cpu()[kept]))
    assert torch.equal(bits(fused.out), bits(ref.out)), "out differs"
    if not skip_xp_check:
        assert bool((fused.xp.view(torch.uint8) == SENTINEL).all()), "the permute ran"


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_fused_gather_small(name, cuda_device):
    wl = CASES[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    fb = _fused_buffers(wl, cuda_device)
    assert _run(wl, g, fb) == 0
    _assert_same(g.buf, fb, wl)
    # and against the oracle: out of the exact layer
    ref = oracle.layer(wl, g.inputs)
    y_o = torch.nan_to_num(ref["y"], nan=0.0)
    out_o = oracle.combine(y_o, ref["slot_of_pair"], ref["topk_w"])
    if wl.ydt == "e4m3":
        return     # FP8 y: test_gpu_fp8_combine holds the bounds; equality above covers it
    ok, worst = rowwise_ok(fb.out.cpu(), out_o, BF16_TOL)
    assert ok, f"out: worst err/rms {worst:.3g}"


@pytest.mark.gpu
def test_fused_gather_flag_is_ignored_where_the_kernel_does_not_apply(cuda_device):
    """decode-sized batches (< 16 rows per expert) run the token-major GEMM,
    which has no gather: the layer permutes as usual and gives the same
    results."""
    wl = workloads.WORKLOADS["decode"].replace(T=16)
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    fb = _fused_buffers(wl, cuda_device)
    assert _run(wl, g, fb) == 0
    _assert_same(g.buf, fb, wl, skip_xp_check=True)
    assert torch.equal(bits(fb.xp), bits(g.buf.xp))


def _device_inputs(wl, device):
    """Seeded inputs of the workload's shapes and distributions drawn on the
    device (equality of two paths holds for any inputs; this skips the
    host-side draw of the full-size weights)."""
    gen = torch.Generator(device=device).manual_seed(20251)
    bf = torch.bfloat16
    logits = torch.randn(wl.T, wl.E, generator=gen, device=device)
    if wl.router == "zipf":
        logits += workloads.zipf_bias(wl).to(device)
    x = torch.randn(wl.T, wl.H, generator=gen, device=device).to(bf)
    w13 = torch.randn(wl.E, 2 * wl.I, wl.H, generator=gen, device=device, dtype=bf)
    w13.mul_(wl.H ** -0.5)
    w2 = torch.randn(wl.E, wl.H, wl.I, generator=gen, device=device, dtype=bf)
    w2.mul_(wl.I ** -0.5)
    return {"logits": logits, "x": x, "w13": w13, "w2": w2}


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["dsv3", "mid", "skew", "dsv3_cap"])
def test_fused_gather_full_size_equals_unfused(name, cuda_device):
    """Full-size workloads: the fused layer equals the unfused one bit for
    bit (the unfused layer is compared with the oracle at these sizes in
    test_gpu_parity)."""
    wl = workloads.WORKLOADS[name]
    g = GpuLayer(wl, cuda_device, inputs=_device_inputs(wl, cuda_device))
    assert g.run() == 0
    fb = _fused_buffers(wl, cuda_device)
    assert _run(wl, g, fb) == 0
    _assert_same(g.buf, fb, wl)
