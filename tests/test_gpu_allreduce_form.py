"""GPU parity of the all_reduce form of the layer: each logical rank's
partial over its own slab of slots (moe_combine_rank), and the sum of the
partials in rank order, rounded once (moe_reduce_partials).

Source: "Expert parallelism" (Transformers docs), "Choosing an
implementation", the all_reduce row.

moe_combine_rank is checked against the oracle's partial of the GPU's own y
(fp32 accumulation of at most k terms: |err| <= k * 2^-24 * sum |w y|);
moe_reduce_partials bit for bit against the same fp32 additions in rank
order on the CPU, followed by one rounding; and the whole layer in this
form against the oracle's exact layer (the bf16 bar) and against the
default combine (the same sum, associated differently: apart by the two
sums' fp32 errors plus one rounding step of out).
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
    "pair_fp8": workload("pair_fp8"),
    "ragged_bf16": workload("ragged_bf16"),
    "cap_bf16": W("cap_ar", 600, 256, 8, 2, 192, 4, "bf16", "bf16", "bf16", capacity_factor=0.5),
    "fp8y": W("fp8y_ar", 300, 256, 8, 2, 192, 2, "bf16", "e4m3", "bf16", ydt="e4m3"),
    "f32": workload("small_f32"),
}


def _y_f32(buf):
    """y as fp32 values: fp32 / bf16 y as stored, or decode(q) * scale (fp32
    product) for an FP8 y."""
    y = buf.y.cpu()
    if y.dtype == torch.float8_e4m3fn:
        return y.float() * buf.y_scales.cpu().repeat_interleave(128, dim=1)
    return y.float()


def _assert_close_to_default(a, d, buf, k, act):
    """Two fp32 sums of the same <= k products, associated differently, each
    rounded once to act: apart by at most both sums' fp32 errors (k * 2^-24
    * sum |w y| each) plus one rounding step of act (2^-7 relative for bf16)."""
    y = _y_f32(buf)
    mag = oracle.combine(y.abs(), buf.slot_of_pair.cpu(), buf.topk_w.cpu().abs())
    step = 2.0 ** -7 if act == "bf16" else 0.0
    a, d = a.double(), d.double()
    bound = step * torch.maximum(a.abs(), d.abs()) + 2 * k * 2.0 ** -24 * mag
    assert bool(((a - d).abs() <= bound).all()), f"worst excess {float(((a - d).abs() - bound).max()):.3g}"


def _fp32_rank_sum(parts):
    acc = parts[0].clone()
    for r in range(1, parts.shape[0]):
        acc = acc + parts[r]                  # fp32, round to nearest even
    return acc


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_rank_partials_and_their_sum(name, cuda_device):
    wl = CASES[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    b = g.buf
    T, H = wl.T, wl.H
    parts = torch.empty(wl.W, T, H, dtype=torch.float32, device=cuda_device)
    for r in range(wl.W):
        moe.moe_combine_rank(b.y, b.slot_of_pair, b.topk_w, b.rank_offsets, r, parts[r],
                             y_scales=b.y_scales)
    torch.cuda.synchronize()
    y = _y_f32(b)
    sop, w, ro = b.slot_of_pair.cpu(), b.topk_w.cpu(), b.rank_offsets.cpu()
    absw = w.abs()
    # fp32 roundings per pick: one (the fused add) for fp32 / bf16 y; for an
    # FP8 y the GPU weights each code by (w * scale), rounded once per piece,
    # while y here holds decode * scale rounded: up to three
    per_pick = 3 if wl.ydt == "e4m3" else 1
    for r in range(wl.W):
        ref = oracle.combine_rank(y, sop, w, ro, r)
        mag = oracle.combine_rank(y.abs(), sop, absw, ro, r)
        err = (parts[r].cpu().double() - ref).abs()
        assert bool((err <= per_pick * wl.k * 2.0 ** -24 * mag).all()), f"rank {r}"
    # the ranks' partials cover every kept pick exactly once
    whole = oracle.combine(y, sop, w)
    mag = oracle.combine(y.abs(), sop, absw)
    got = _fp32_rank_sum(parts.cpu()).double()
    assert bool(((got - whole).abs() <= (per_pick * wl.k + wl.W) * 2.0 ** -24 * mag).all())
    # the reduction: fp32 additions in rank order, one rounding, bit for bit
    out = torch.empty(T, H, dtype=workloads.TORCH_DTYPE[wl.act], device=cuda_device)
    moe.moe_reduce_partials(parts, out)
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(_fp32_rank_sum(parts.cpu()).to(out.dtype)))


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["small_bf16", "small_fp8", "cap_bf16", "f32"])
def test_layer_in_all_reduce_form(name, cuda_device):
    """moe_layer_forward with all_reduce_form: out against the oracle's
    exact layer, and within one rounding step of the default combine."""
    wl = CASES[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    wla = wl.replace(all_reduce_form=True)
    ab = moe.LayerBuffers(wla, cuda_device)
    moe.layer_forward(wla, g.logits, g.x, g.w13, g.w2, ab)
    torch.cuda.synchronize()
    assert moe.moe_check_status(ab.dev_status) == 0
    ref = oracle.layer(wl, g.inputs)
    y_o = torch.nan_to_num(ref["y"], nan=0.0)
    out_o = oracle.combine(y_o, ref["slot_of_pair"], ref["topk_w"])
    tol = BF16_TOL if wl.wdt == "bf16" else 1e-5
    ok, worst = rowwise_ok(ab.out.cpu(), out_o, tol)
    assert ok, f"out: worst err/rms {worst:.3g}"
    _assert_close_to_default(ab.out.cpu(), g.buf.out.cpu(), g.buf, wl.k, wl.act)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["dsv3", "decode"])
def test_full_size_all_reduce_form_matches_the_default_combine(name, cuda_device):
    """Full size: the layer in the all_reduce form gives the default
    layer's out up to one rounding step (the default layer is compared with
    the oracle at these sizes in test_gpu_parity); route, layout and y are
    the same kernels, bit for bit."""
    wl = workloads.WORKLOADS[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    wla = wl.replace(all_reduce_form=True)
    ab = moe.LayerBuffers(wla, cuda_device)
    moe.layer_forward(wla, g.logits, g.x, g.w13, g.w2, ab)
    torch.cuda.synchronize()
    assert moe.moe_check_status(ab.dev_status) == 0
    assert torch.equal(ab.slot_of_pair.cpu(), g.buf.slot_of_pair.cpu())
    _assert_close_to_default(ab.out.cpu(), g.buf.out.cpu(), g.buf, wl.k, wl.act)
    # each logical rank's partial holds exactly the tokens it serves
    ro = ab.rank_offsets.cpu()
    sop = ab.slot_of_pair.cpu().view(wl.T, wl.k)
    for r in range(wl.W):
        served = ((sop >= ro[r]) & (sop < ro[r + 1])).any(dim=1)
        zero_rows = (ab.partials[r].cpu() == 0).all(dim=1)
        assert bool(zero_rows[~served].all())
