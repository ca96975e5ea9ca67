"""Poison-fill checks of what each kernel writes: every output buffer of
the layer is filled with a sentinel before the call; afterwards every row
that holds a routed pair has been written (no sentinel left in it) and
every row that holds none still holds the sentinel (nothing wrote past the
rows it owns).  Fixed-capacity layouts leave unused slab rows, so they show
both sides; the dropless layout must write every row."""
import pytest
import torch

from expert_parallelism_b200 import moe, workloads

from parity_helpers import GpuLayer

CASES = {
    "cap_bf16": workloads.Workload("cap_p", 600, 256, 8, 2, 192, 2, "bf16", "bf16", "bf16",
                                   capacity_factor=0.7),
    "cap_fp8": workloads.Workload("cap_p8", 500, 384, 16, 4, 320, 4, "bf16", "e4m3", "bf16",
                                  capacity_factor=1.2),
    "dropless_fp8": workloads.Workload("free_p8", 300, 256, 8, 2, 192, 2, "bf16", "e4m3", "bf16"),
}


def _poison(t):
    v = t.view(torch.uint8) if t.element_size() == 1 else t
    if t.is_floating_point() and t.element_size() > 1:
        t.fill_(float("nan"))
    else:
        v.fill_(0xA5)


def _is_poison(t):
    if t.is_floating_point() and t.element_size() > 1:
        return torch.isnan(t.float())
    return t.view(torch.uint8) == 0xA5


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_every_owned_row_written_and_no_other(name, cuda_device):
    wl = CASES[name]
    g = GpuLayer(wl, cuda_device)
    b = g.buf
    outs = [t for t in (b.xp, b.xp_scales, b.h, b.y, b.out) if t is not None]
    for t in outs:
        _poison(t)
    moe.layer_forward(wl, g.logits, g.x, g.w13, g.w2, b)
    torch.cuda.synchronize()
    assert moe.moe_check_status(b.dev_status) == 0
    held = (b.pair_of_slot >= 0).cpu()
    for t in (b.xp, b.xp_scales, b.h, b.y):
        if t is None:
            continue
        p = _is_poison(t).cpu()
        rows_touched = ~p.all(dim=1)
        # bf16 / fp32 rows: no finite result is NaN, so a written row holds
        # no sentinel at all; FP8 codes can equal the sentinel byte, so a
        # written code row only has to differ from it somewhere
        rows_written = rows_touched if t.element_size() == 1 else ~p.any(dim=1)
        assert bool(rows_written[held].all()), "a held row was not (fully) written"
        assert not bool(rows_touched[~held].any()), "a row holding no pair was written"
    assert not bool(_is_poison(b.out).any().cpu()), "out not fully written"
