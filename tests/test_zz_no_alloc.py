"""The allocation-free layout entry point, for callers that cannot allocate
device memory (no cudaMalloc during stream capture, or a host framework that
owns all device memory).  It must give exactly what moe_dispatch_layout
gives with a caller workspace, on consecutive calls that reuse its
library-internal scratch.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

from expert_parallelism_b200 import moe, workloads

KEYS = ["expert_counts", "expert_offsets", "rank_offsets", "slot_of_pair", "pair_of_slot"]


def _outputs(T, k, E, W, dev):
    i32 = dict(dtype=torch.int32, device=dev)
    N = max(T * k, 1)
    return {"expert_counts": torch.full((E,), -5, **i32),
            "expert_offsets": torch.full((E + 1,), -5, **i32),
            "rank_offsets": torch.full((W + 1,), -5, **i32),
            "slot_of_pair": torch.full((N,), -5, **i32),
            "pair_of_slot": torch.full((N,), -5, **i32),
            "st": torch.zeros(1, **i32)}


def test_noalloc_rejects_oversize_on_the_host():
    lib = moe.load_library()
    assert lib.moe_dispatch_layout_noalloc_max_scratch_bytes() == 2 << 20
    fake = ctypes.c_void_p(4096)   # never dereferenced: the size check fails first
    T = 3_000_000                  # 256 experts x ceil(24M pairs / 2048) > the scratch
    rc = lib.moe_dispatch_layout_noalloc(fake, T, 8, 256, 8, fake, fake, fake, fake, fake,
                                         fake, None)
    assert moe.STATUS[rc] == "MOE_ERR_UNSUPPORTED"


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["dsv3", "skew"])
def test_noalloc_matches_workspace_entry_point_twice(name, cuda_device):
    wl = workloads.WORKLOADS[name]
    logits = workloads.router_logits(wl).to(cuda_device)
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=cuda_device)
    w = torch.empty(wl.T, wl.k, device=cuda_device)
    moe.moe_route_topk(logits, idx, w)
    ref = _outputs(wl.T, wl.k, wl.E, wl.W, cuda_device)
    ws = torch.empty(moe.moe_dispatch_layout_workspace_bytes(wl.T, wl.k, wl.E),
                     dtype=torch.uint8, device=cuda_device)
    moe.moe_dispatch_layout(idx, wl.E, wl.W, *[ref[k] for k in KEYS], ws, ref["st"])
    assert moe.moe_check_status(ref["st"]) == 0
    # two calls in a row; the second one also runs on a different batch
    # first, so it cannot pass on stale scratch contents from the first
    other = torch.flip(idx, dims=[0]).contiguous()
    for call in range(2):
        got = _outputs(wl.T, wl.k, wl.E, wl.W, cuda_device)
        if call == 1:
            scratch_dirty = _outputs(wl.T, wl.k, wl.E, wl.W, cuda_device)
            moe.moe_dispatch_layout_noalloc(other, wl.E, wl.W, *[scratch_dirty[k] for k in KEYS],
                                            scratch_dirty["st"])
        moe.moe_dispatch_layout_noalloc(idx, wl.E, wl.W, *[got[k] for k in KEYS], got["st"])
        assert moe.moe_check_status(got["st"]) == 0
        for key in KEYS:
            assert torch.equal(got[key], ref[key]), (call, key)
