"""The grouped GEMM's in-kernel clock record (moe_diag_gemm_clock): after a
layer call whose experts run on the tensor-core GEMM, both phases have
recorded SM cycles and nanoseconds, their ratio is a plausible SM clock,
the record sums over launches, and a reset clears it."""
import pytest
import torch

from expert_parallelism_b200 import moe, workloads

from parity_helpers import GpuLayer

# ~128 routed rows per expert: the operand-swapped tensor-core GEMM
WL = workloads.Workload("clock_rec", 512, 256, 8, 2, 256, 2, "bf16", "bf16", "bf16")


@pytest.mark.gpu
def test_clock_record_counts_both_phases_and_resets(cuda_device):
    g = GpuLayer(WL, cuda_device)
    moe.moe_diag_gemm_clock(reset=True)
    assert moe.moe_diag_gemm_clock() == {"gate_up": (0, 0), "down": (0, 0)}
    moe.layer_forward(WL, g.logits, g.x, g.w13, g.w2, g.buf)
    one = moe.moe_diag_gemm_clock()
    assert moe.moe_check_status(g.buf.dev_status) == 0
    for phase in ("gate_up", "down"):
        cycles, ns = one[phase]
        assert cycles > 0 and ns > 0, phase
        mhz = cycles / ns * 1e3
        assert 100.0 < mhz < 3000.0, (phase, mhz)
    moe.layer_forward(WL, g.logits, g.x, g.w13, g.w2, g.buf)
    two = moe.moe_diag_gemm_clock(reset=True)
    for phase in ("gate_up", "down"):
        assert two[phase][0] > one[phase][0] and two[phase][1] > one[phase][1], phase
    assert moe.moe_diag_gemm_clock() == {"gate_up": (0, 0), "down": (0, 0)}
