"""The packed weight layout (moe_pack_expert_weights): the blocks hold
exactly the stacked weights' values in the documented order, and the
grouped GEMM on packed weights gives the stacked GEMM's h and y bit for bit
(same operands, same MMA order), standalone and inside the layer call."""
import numpy as np
import pytest
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

from parity_helpers import BF16_TOL, GpuLayer, bits, h_ok, rowwise_ok


def _reference_pack(w13, w2):
    """The layout written out with tensor ops on the host: W13 blocks
    (e, f, c) = [gate rows 64f.., up rows I+64f..] x columns 64c..; W2 blocks
    (e, r, c) = rows 128r.. x columns 64c..; zero padding to whole tiles."""
    E, H, I = w2.shape
    FB, KB13 = 2 * ((I + 127) // 128), (H + 63) // 64
    RB, KB2 = 2 * ((H + 255) // 256), (I + 63) // 64
    g = torch.zeros(E, FB * 64, KB13 * 64, dtype=w13.dtype)
    u = torch.zeros_like(g)
    g[:, :I, :H] = w13[:, :I]
    u[:, :I, :H] = w13[:, I:]
    gb = g.view(E, FB, 64, KB13, 64).permute(0, 1, 3, 2, 4)
    ub = u.view(E, FB, 64, KB13, 64).permute(0, 1, 3, 2, 4)
    p13 = torch.cat([gb, ub], dim=3).contiguous()              # [E, FB, KB, 128, 64]
    d = torch.zeros(E, RB * 128, KB2 * 64, dtype=w2.dtype)
    d[:, :H, :I] = w2
    p2 = d.view(E, RB, 128, KB2, 64).permute(0, 1, 3, 2, 4).contiguous()
    return p13.view(-1), p2.view(-1)


@pytest.mark.gpu
@pytest.mark.parametrize("E,H,I", [(3, 320, 200), (2, 2880, 2880), (4, 256, 64)])
def test_pack_layout_matches_the_documented_blocks(E, H, I, cuda_device):
    wl = workloads.Workload("pk", 1, H, E, 1, I, 1, "bf16", "bf16", "bf16")
    w13 = torch.stack([workloads.expert_w13(wl, e) for e in range(E)])
    w2 = torch.stack([workloads.expert_w2(wl, e) for e in range(E)])
    p13, p2 = moe.packed_weight_tensors(E, H, I, cuda_device)
    moe.moe_pack_expert_weights(w13.to(cuda_device), w2.to(cuda_device), p13, p2)
    torch.cuda.synchronize()
    r13, r2 = _reference_pack(w13, w2)
    assert torch.equal(p13.cpu().view(torch.int16), r13.view(torch.int16))
    assert torch.equal(p2.cpu().view(torch.int16), r2.view(torch.int16))


@pytest.mark.gpu
@pytest.mark.parametrize("ydt", ["f32", "bf16"])
def test_packed_gemm_equals_stacked_gemm_on_chunk_boundaries(ydt, cuda_device):
    counts = [0, 1, 15, 16, 17, 31, 32, 33, 0, 255, 256, 257, 511, 512, 513]
    E, H, I = len(counts), 320, 200
    wl = workloads.Workload("pkc", 1, H, E, 1, I, 1, "bf16", "bf16", "bf16", ydt=ydt)
    off = torch.tensor([0] + list(np.cumsum(counts)), dtype=torch.int32)
    n = int(off[-1])
    xp = torch.randn(n, H, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16)
    w13 = torch.stack([workloads.expert_w13(wl, e) for e in range(E)]).to(cuda_device)
    w2 = torch.stack([workloads.expert_w2(wl, e) for e in range(E)]).to(cuda_device)
    dev = cuda_device
    ydtype = workloads.TORCH_DTYPE[ydt]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    outs = []
    for packed in (False, True):
        h = torch.full((n, I), float("nan"), dtype=torch.bfloat16, device=dev)
        y = torch.full((n, H), float("nan"), dtype=ydtype, device=dev)
        if packed:
            p13, p2 = moe.packed_weight_tensors(E, H, I, dev)
            moe.moe_pack_expert_weights(w13, w2, p13, p2)
            moe.moe_grouped_gemm_packed(xp.to(dev), None, off.to(dev), 0, E, p13, p2, H, I, h, y,
                                        None, st)
        else:
            moe.moe_grouped_gemm(xp.to(dev), None, off.to(dev), 0, E, w13, w2, h, y, None, st)
        assert moe.moe_check_status(st) == 0
        outs.append((h.cpu(), y.cpu()))
    assert torch.equal(bits(outs[0][0]), bits(outs[1][0]))
    assert torch.equal(bits(outs[0][1]), bits(outs[1][1]))
    h_ref, y_ref, _ = oracle.grouped_gemm(xp, None, off, 0, E, w13.cpu(), w2.cpu())
    assert h_ok(outs[1][0], h_ref, torch.bfloat16)[0]
    assert rowwise_ok(outs[1][1], y_ref, BF16_TOL)[0]


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["dsv3", "skew", "decode"])
def test_packed_layer_equals_stacked_layer(name, cuda_device):
    """The layer call on packed weights gives the stacked layer's out, h and
    y bit for bit at full size (decode included: packed weights always take
    the operand-swapped kernel)."""
    wl = workloads.WORKLOADS[name]
    g = GpuLayer(wl, cuda_device)
    assert g.run() == 0
    h0, y0, out0 = g.buf.h.clone(), g.buf.y.clone(), g.buf.out.clone()
    wlp = wl.replace(packed_weights=True)
    p13, p2 = moe.packed_weight_tensors(wl.E, wl.H, wl.I, cuda_device)
    moe.moe_pack_expert_weights(g.w13, g.w2, p13, p2)
    for t in (g.buf.h, g.buf.y, g.buf.out):
        t.zero_()
    moe.layer_forward(wlp, g.logits, g.x, p13, p2, g.buf)
    torch.cuda.synchronize()
    assert moe.moe_check_status(g.buf.dev_status) == 0
    rows = int(g.buf.expert_offsets[-1])
    if name == "decode":       # the stacked decode layer ran the token-major kernel
        ok, worst = rowwise_ok(g.buf.y[:rows].cpu(), y0[:rows].cpu(), BF16_TOL)
        assert ok, worst
        ok, worst = rowwise_ok(g.buf.out.cpu(), out0.cpu(), BF16_TOL)
        assert ok, worst
    else:
        assert torch.equal(bits(g.buf.h[:rows]), bits(h0[:rows]))
        assert torch.equal(bits(g.buf.y[:rows]), bits(y0[:rows]))
        assert torch.equal(bits(g.buf.out), bits(out0))
