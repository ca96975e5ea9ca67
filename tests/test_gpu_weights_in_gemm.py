"""The router weights applied in the down GEMM's epilogue (layer option
weights_in_gemm), the second half of the fused layer ("Expert parallelism"
(Transformers docs), "Choosing an implementation": deepgemm_megamoe fuses
dispatch, experts and combine): y row s becomes w * (the expert's output)
with w = topk_w of the row's pair, and the combine sums the k rows with unit
weights.

Checks: every y row equals the default layer's fp32 y row times its weight,
bit for bit (the same accumulator, one fp32 product); out is within the
bf16 bar of the oracle; the fused gather and the capacity layout compose
with it."""
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

from parity_helpers import BF16_TOL, GpuLayer, bits, rowwise_ok, workload

CASES = ["small_bf16", "small_fp8", "ragged_bf16", "pair_bf16", "pair_fp8"]


def _weights_of_slots(buf, n_slots):
    pos = buf.pair_of_slot.cpu()[:n_slots].long()
    w = buf.topk_w.cpu().reshape(-1)
    return torch.where(pos >= 0, w[pos.clamp(min=0)], torch.zeros_like(pos, dtype=torch.float32))


def _run(wl, g, **kw):
    wlw = wl.replace(**kw)
    buf = moe.LayerBuffers(wlw, g.x.device)
    moe.layer_forward(wlw, g.logits, g.x, g.w13, g.w2, buf)
    torch.cuda.synchronize()
    assert moe.moe_check_status(buf.dev_status) == 0
    return buf


@pytest.mark.gpu
@pytest.mark.parametrize("name", CASES + ["cap"])
def test_weights_in_gemm_small(name, cuda_device):
    wl = (workloads.Workload("cap_w", 600, 256, 8, 2, 192, 2, "bf16", "bf16", "bf16",
                             capacity_factor=0.7) if name == "cap" else workload(name))
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    base = g.buf
    wb = _run(wl, g, weights_in_gemm=True)
    n = int(base.expert_offsets[-1]) if wl.capacity_factor is None else wb.pair_of_slot.numel()
    w = _weights_of_slots(wb, n)
    keep = wb.pair_of_slot.cpu()[:n] >= 0
    want = (base.y.cpu()[:n] * w[:, None])[keep]
    assert torch.equal(bits(wb.y.cpu()[:n][keep]), bits(want))
    ref = oracle.layer(wl, g.inputs)
    ok, worst = rowwise_ok(wb.out.cpu(), ref["out"], BF16_TOL)
    assert ok, worst


@pytest.mark.gpu
def test_weights_in_gemm_with_fused_gather(cuda_device):
    wl = workload("small_fp8")
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    a = _run(wl, g, weights_in_gemm=True)
    b = _run(wl, g, weights_in_gemm=True, fused_gather=True)
    assert torch.equal(bits(a.y), bits(b.y))
    assert torch.equal(bits(a.out), bits(b.out))


@pytest.mark.gpu
def test_weights_in_gemm_full_size_dsv3(cuda_device):
    """dsv3 at full size: every y row is the default fp32 y row times its
    router weight, bit for bit; out differs from the default layer's out by
    at most one bf16 rounding plus the fp32 roundings of the k terms."""
    wl = workloads.WORKLOADS["dsv3"]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    base = g.buf
    y0, out0 = base.y.clone(), base.out.clone()
    wb = _run(wl, g, weights_in_gemm=True)
    n = wl.N
    w = _weights_of_slots(wb, n).to(cuda_device)
    assert torch.equal(bits(wb.y), bits(y0 * w[:, None]))
    # the two fp32 sums (of fl(w*y) terms, and of fused w*y + acc steps)
    # differ by a few fp32 roundings of the terms; each is then rounded to
    # bf16 once: |d| <= one bf16 ulp of out (2^-7 |out|) + 2^-20 sum_j |w_j y_j|
    sop = wb.slot_of_pair.view(wl.T, wl.k).long()
    tw = wb.topk_w.view(wl.T, wl.k)
    mag = torch.zeros(wl.T, wl.H, device=cuda_device)
    for j in range(wl.k):
        mag += (tw[:, j:j + 1] * y0[sop[:, j]]).abs()
    d = (wb.out.float() - out0.float()).abs()
    assert bool((d <= 2.0 ** -7 * out0.float().abs() + 2.0 ** -20 * mag).all())
