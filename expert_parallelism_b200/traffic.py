"""Byte and flop accounting for the MoE-layer hot path (host-side only).

``dispatch_combine_bytes_per_token`` is the traffic rule of "Expert
parallelism and all-to-all", section "Traffic math": each token's hidden
vector travels to its k experts and back, 2 * k * H * bytes per token per
MoE layer.  The rest gives the algorithmic HBM bytes and flops of each
kernel on one GPU, the figures the roofline fractions divide by.
"""
from __future__ import annotations

from .workloads import ELEM_BYTES, Workload


def dispatch_combine_bytes_per_token(k: int, H: int, bytes_per_elem: int) -> int:
    """2 * k * H * bytes: dispatch plus combine, one token, one MoE layer."""
    return 2 * k * H * bytes_per_elem


def dispatch_bytes_from_layout(rank_offsets_last: int, H: int, bytes_per_elem: int) -> int:
    """Bytes the dispatch all-to-all would move for one GPU: every routed
    row (rank_offsets[W] of them) of H elements."""
    return rank_offsets_last * H * bytes_per_elem


def kernel_bytes(wl: Workload, rows: int | None = None) -> dict:
    """Algorithmic HBM bytes per launch of each step (each input read once,
    each output written once) for ``rows`` routed rows kept (all T*k by
    default; fewer when a fixed capacity drops pairs)."""
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    N = wl.N if rows is None else rows
    xb, pb, yb = ELEM_BYTES[wl.act], ELEM_BYTES[wl.payload], ELEM_BYTES[wl.ydt]
    scales = N * (H // 128) * 4 if wl.payload == "e4m3" else 0
    return {
        "route_topk": T * E * 4 + T * k * 8,
        "dispatch_layout": N * 4 + N * 8 + (2 * E + 1) * 4 + (wl.W + 1) * 4,
        "permute": T * H * xb + N * H * pb + scales,
        # inside moe_layer_forward an FP8 permute also writes the GEMM's bf16
        # rows; with the fused gather the permuted copy is never made: an FP8
        # payload's tokens make one bf16 round trip each (T rows), a bf16
        # payload has no step here at all
        "permute_layer": ((T * H * xb + T * H * 2 if wl.payload == "e4m3" else 0)
                          if wl.fused_gather else
                          T * H * xb + N * H * pb + scales
                          + (N * H * 2 if wl.payload == "e4m3" else 0)),
        # the all_reduce form reads slot_of_pair and topk_w once per rank,
        # writes W fp32 partials and reads them back for the sum
        "combine": N * H * yb + (N * (H // 128) * 4 if wl.ydt == "e4m3" else 0)
                   + T * k * 8 * (wl.W if wl.all_reduce_form else 1) + T * H * xb
                   + (2 * wl.W * T * H * 4 if wl.all_reduce_form else 0),
    }


def gemm_flops(wl: Workload, rows: int | None = None) -> dict:
    """Dense flops of the two GEMM phases for ``rows`` routed rows."""
    n = wl.N if rows is None else rows
    return {"gate_up": 2 * n * wl.H * 2 * wl.I, "down": 2 * n * wl.I * wl.H,
            "total": 6 * n * wl.H * wl.I}


def touched_weight_bytes(wl: Workload, experts_touched: int) -> int:
    """Expert-weight bytes a pass must read at least once."""
    return experts_touched * 3 * wl.I * wl.H * ELEM_BYTES[wl.wdt]


def section8_bytes(wl: Workload, rows: int | None = None) -> dict:
    """The permute's and the combine's algorithmic bytes as the step table
    counts them: the send buffer (x read once, the payload and its block
    scales written once per routed row), and the combine reading each routed
    row of y once in a 2-byte type (1 byte plus block scales for the FP8
    combine payload) and writing out once.  Whatever y's storage dtype, the
    combine's fraction of peak on these bytes is what the step's target
    refers to."""
    T, H, k = wl.T, wl.H, wl.k
    N = wl.N if rows is None else rows
    xb, pb = ELEM_BYTES[wl.act], ELEM_BYTES[wl.payload]
    scales = N * (H // 128) * 4 if wl.payload == "e4m3" else 0
    y_row = H + (H // 128) * 4 if wl.ydt == "e4m3" else 2 * H
    return {"permute": T * H * xb + N * H * pb + scales,
            "combine": N * y_row + T * H * xb}


def gemm_phase_bytes(wl: Workload, rows: int, experts_touched: int) -> dict:
    """DRAM bytes each GEMM phase must move at least: its weights once per
    touched expert, its row operand once, its output once (h in the weight
    dtype; y in its storage dtype, plus block scales for an FP8 y)."""
    wb = ELEM_BYTES[wl.wdt]
    H, I = wl.H, wl.I
    y_row = H + (H // 128) * 4 if wl.ydt == "e4m3" else H * ELEM_BYTES[wl.ydt]
    return {"gate_up": experts_touched * 2 * I * H * wb + rows * H * wb + rows * I * wb,
            "down": experts_touched * H * I * wb + rows * I * wb + rows * y_row}
