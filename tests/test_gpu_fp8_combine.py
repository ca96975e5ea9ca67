"""GPU parity of the FP8 combine payload (y as e4m3 codes with per-128 block
scales, written by the down GEMM's epilogue and read by the combine).

Source: "Expert parallelism and all-to-all", "Traffic math": 1-byte
activations both ways.

The GPU quantises its fp32 y, which meets the bf16 GEMM's bar against the
exact y (|Δy| <= TAU * RMS(row), TAU = 2e-2: h is a bf16 operand, and the
GPU's and the exact gate/up values can round to neighbouring bf16 values),
and quantisation adds at most half a code step times the block scale.  The
checks, against the oracle's exact y:
  - block scales: |Δscale| <= TAU * RMS(row) / 448 (a block's amax moves
    by at most the largest |Δy|);
  - every dequantised element: |decode(q) * scale - y| <= step/2 * scale +
    TAU * RMS(row), step = the e4m3 spacing at that code (doubled, to cover
    a binade edge);
  - out: |Δ| <= Σ_j w_j (step_j * scale_j + TAU * RMS_j) + 1e-5 Σ_j w_j |y_j|
    + 2^-8 |out| (the picks' bounds, the fp32 sums, out's bf16 rounding),
    against the combine of the exact y.
"""
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

from parity_helpers import BF16_TOL as TAU
from parity_helpers import GpuLayer, oracle_gemm_rows, sample_rows


def _spacing(m):
    """e4m3 spacing at magnitude m (in code units)."""
    e = torch.floor(torch.log2(m.clamp(min=2.0 ** -6)))
    return torch.where(m >= 2.0 ** -6, 2.0 ** (e - 3), torch.full_like(m, 2.0 ** -9))


def _check_rows(q_gpu, sc_gpu, y_exact):
    """Codes and scales of GPU rows against the exact rows they encode."""
    y = y_exact.double()
    rms = y.pow(2).mean(dim=1, keepdim=True).sqrt()
    amax = y.abs().view(y.shape[0], -1, 128).amax(dim=2)
    ds = (sc_gpu.double() - amax / 448.0).abs()
    assert bool((ds <= TAU * rms / 448.0 + 1e-7 * amax).all()), "block scales"
    s = sc_gpu.double().repeat_interleave(128, dim=1)
    dq = q_gpu.float().double()
    err = (dq * s - y).abs()
    bound = _spacing(dq.abs()) * s + TAU * rms          # half a step, doubled
    assert bool((err <= bound).all()), f"worst excess {float((err - bound).max()):.3g}"


def _out_bound(y_exact, sc, sop, w, out_exact):
    """Per-element bound on |out_gpu - out_exact| (rows indexed by sop;
    -1 = dropped)."""
    T, k = w.shape
    y = y_exact.double()
    rms = y.pow(2).mean(dim=1, keepdim=True).sqrt()
    s = sc.double().repeat_interleave(128, dim=1)
    bound = torch.zeros(T, y.shape[1], dtype=torch.float64)
    mag = torch.zeros_like(bound)
    for j in range(k):
        rows = sop[:, j].long()
        ok = (rows >= 0).double().unsqueeze(1)
        r = rows.clamp(min=0)
        wj = w[:, j].double().unsqueeze(1) * ok
        bound += wj * (2 * _spacing((y[r] / s[r]).abs()) * s[r] + TAU * rms[r])
        mag += wj * y[r].abs()
    return bound + 1e-5 * mag + 2.0 ** -8 * out_exact.abs()


SMALL = {
    "fp8y_bf16": workloads.Workload("fp8y_bf16", 300, 256, 8, 2, 192, 2, "bf16", "bf16", "bf16",
                                    ydt="e4m3"),
    "fp8y_fp8": workloads.Workload("fp8y_fp8", 200, 384, 16, 4, 320, 4, "bf16", "e4m3", "bf16",
                                   ydt="e4m3"),
    "fp8y_pairs": workloads.Workload("fp8y_pairs", 1500, 384, 4, 3, 320, 4, "bf16", "e4m3",
                                     "bf16", ydt="e4m3"),
    "fp8y_capacity": workloads.Workload("fp8y_cap", 600, 256, 8, 2, 192, 2, "bf16", "bf16",
                                        "bf16", ydt="e4m3", capacity_factor=0.7),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_combine_layer_parity(name, cuda_device):
    wl = SMALL[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    b = g.buf
    ref = oracle.layer(wl, g.inputs)
    kept = ref["pair_of_slot"] >= 0
    _check_rows(b.y.cpu()[kept], b.y_scales.cpu()[kept], ref["y"][kept])
    sop = ref["slot_of_pair"].view(wl.T, wl.k)
    y_exact = torch.nan_to_num(ref["y"], nan=0.0)
    out_exact = oracle.combine(y_exact, ref["slot_of_pair"], ref["topk_w"])
    bound = _out_bound(y_exact, b.y_scales.cpu(), sop, ref["topk_w"], out_exact)
    err = (b.out.cpu().double() - out_exact).abs()
    assert bool((err <= bound).all()), f"worst excess {float((err - bound).max()):.3g}"


@pytest.mark.gpu
def test_fp8_combine_full_size_sampled(cuda_device):
    """dsv3_fp8y at full size: codes and scales of the sampled rows (every
    row of 8 experts, 8 seeded rows and both ends of every other expert, and
    all rows of the sampled tokens), and the sampled tokens' out, against the
    oracle's exact rows."""
    wl = workloads.WORKLOADS["dsv3_fp8y"]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    b = g.buf
    idx_o, w_o = oracle.route_topk(g.inputs["logits"], wl.k)
    lay = oracle.dispatch_layout(idx_o, wl.E, wl.W)
    assert torch.equal(b.slot_of_pair.cpu(), lay["slot_of_pair"])
    toks, mask, _ = sample_rows(lay, wl.T, wl.k, 96)
    pos = lay["pair_of_slot"].clone()
    pos[~mask] = -1
    xp_o, sc_o = oracle.permute(g.inputs["x"], wl.k, pos, wl.payload)
    slots, _, y_o = oracle_gemm_rows(wl, xp_o, sc_o, lay["expert_offsets"], mask)
    _check_rows(b.y.cpu()[slots], b.y_scales.cpu()[slots], y_o)
    sop = lay["slot_of_pair"].view(wl.T, wl.k)[toks]
    compact = torch.searchsorted(slots, sop.reshape(-1).long()).to(torch.int32).view(-1, wl.k)
    out_exact = oracle.combine(y_o, compact.reshape(-1), w_o[toks].contiguous())
    bound = _out_bound(y_o, b.y_scales.cpu()[slots], compact, w_o[toks], out_exact)
    err = (b.out.cpu()[toks].double() - out_exact).abs()
    assert bool((err <= bound).all()), f"worst excess {float((err - bound).max()):.3g}"
