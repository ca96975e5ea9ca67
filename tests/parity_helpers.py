"""Shared helpers for the GPU parity tests: run the hot path through the
C ABI and compare with the CPU oracle on the same seeded inputs.

The oracle's floating-point results are exact (fp64, unrounded); the only
narrow type inside its chain is h, the bf16 (or fp32) operand of the down
projection.  Tolerances:
  y, out of a bf16 GEMM: per row, max |gpu - oracle| <= 2e-2 * RMS(oracle row)
  y, out, h of the fp32 GEMM: per row, max |gpu - oracle| <= 1e-5 * RMS(oracle row)
  h (bf16, the GEMM's internal activation): per element,
                  |gpu - oracle| <= 2^-8 * |oracle| + 1e-3 * RMS(oracle row),
                  i.e. the bf16 rounding of that element (at most half an
                  ulp, 2^-8 relative) plus a floor for fp32 accumulation
                  order; h is heavy-tailed (silu(g) * u), so a row-RMS bound
                  would be smaller than the rounding of its largest entries
  router weights: elementwise |dw| <= 1e-5 * |w|.
Everything integer (indices, counts, offsets, permutation order, FP8 codes
and their fp32 scales, same-dtype payload copies) must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from expert_parallelism_b200 import moe, workloads

BF16_TOL = 2e-2
F32_TOL = 1e-5

EXTRA = {
    # sizes the oracle finishes in seconds that still span several tiles
    # and ragged tails of the GEMM (partial M, N and K tiles)
    "small_bf16": workloads.Workload("small_bf16", 300, 256, 8, 2, 192, 2, "bf16", "bf16", "bf16"),
    "small_fp8": workloads.Workload("small_fp8", 200, 384, 16, 4, 320, 4, "bf16", "e4m3", "bf16"),
    # H/128 a multiple of 4: block scales leave the permute as 16-byte vectors
    "small_fp8v": workloads.Workload("small_fp8v", 120, 512, 8, 4, 64, 2, "bf16", "e4m3", "bf16"),
    "ragged_bf16": workloads.Workload("ragged_bf16", 777, 200, 6, 3, 136, 3, "bf16", "bf16",
                                      "bf16"),
    "small_f32": workloads.Workload("small_f32", 130, 72, 5, 3, 40, 5, "f32", "f32", "f32"),
    # >= 512 rows per expert: the GEMM runs 256-row tiles on CTA pairs
    "pair_bf16": workloads.Workload("pair_bf16", 2100, 256, 4, 2, 192, 2, "bf16", "bf16", "bf16"),
    "pair_fp8": workloads.Workload("pair_fp8", 1500, 384, 4, 3, 320, 4, "bf16", "e4m3", "bf16"),
}


def workload(name):
    return workloads.WORKLOADS.get(name) or EXTRA[name]


def tol_for(gemm_dtype: torch.dtype) -> float:
    """Row tolerance for y and out: by the dtype the GEMM computes in (a bf16
    GEMM's fp32-stored y is still a bf16-GEMM result)."""
    return F32_TOL if gemm_dtype == torch.float32 else BF16_TOL


def rowwise_ok(got: torch.Tensor, ref: torch.Tensor, tol: float):
    """Per-row max abs error <= tol * RMS(ref row); returns (ok, worst ratio)."""
    g, r = got.double(), ref.double()
    rms = r.pow(2).mean(dim=1).sqrt()
    err = (g - r).abs().amax(dim=1)
    ratio = torch.where(rms > 0, err / rms, err)
    worst = float(ratio.max()) if ratio.numel() else 0.0
    return bool((ratio <= tol).all()), worst


def h_ok(got: torch.Tensor, ref: torch.Tensor, dtype: torch.dtype):
    """The h check above; returns (ok, worst excess over the bound / RMS)."""
    if dtype == torch.float32:
        return rowwise_ok(got, ref, F32_TOL)
    g, r = got.double(), ref.double()
    rms = r.pow(2).mean(dim=1, keepdim=True).sqrt()
    bound = 2.0 ** -8 * r.abs() + 1e-3 * rms
    excess = ((g - r).abs() - bound) / rms
    worst = float(excess.max()) if excess.numel() else 0.0
    return bool((excess <= 0).all()), worst


def bits(t: torch.Tensor) -> torch.Tensor:
    t = t.detach().cpu().contiguous()
    return t.view({4: torch.int32, 2: torch.int16, 1: torch.uint8}[t.element_size()])


class GpuLayer:
    """Device copies of a workload's inputs plus the layer's buffers."""

    def __init__(self, wl, device, inputs=None):
        self.wl = wl
        self.inputs = inputs if inputs is not None else workloads.layer_inputs(wl)
        self.logits = self.inputs["logits"].to(device)
        self.x = self.inputs["x"].to(device)
        self.w13 = self.inputs["w13"].to(device)
        self.w2 = self.inputs["w2"].to(device)
        self.buf = moe.LayerBuffers(wl, device)

    def run(self):
        b, wl = self.buf, self.wl
        moe.layer_forward(wl, self.logits, self.x, self.w13, self.w2, b)
        torch.cuda.synchronize()
        return moe.moe_check_status(b.dev_status)


def full_experts(lay: dict, n: int = 8, seed: int = 0):
    """Experts whose every row a full-size check compares: the largest
    expert; the largest one whose rows make one pass with a second chunk
    (257..320 rows); the largest one that needs several passes (> 320 rows);
    then seeded picks among the other non-empty experts, up to ``n``."""
    cnt = lay["expert_counts"].numpy()
    order = [int(e) for e in np.argsort(-cnt, kind="stable") if cnt[e] > 0]
    chosen = []

    def add(e):
        if e is not None and e not in chosen and len(chosen) < n:
            chosen.append(e)

    if order:
        add(order[0])
    add(next((e for e in order if 256 < cnt[e] <= 320), None))
    add(next((e for e in order if cnt[e] > 320), None))
    rest = [e for e in order if e not in chosen]
    rng = np.random.default_rng(seed + 1)
    for e in rng.permutation(rest)[:max(0, n - len(chosen))]:
        add(int(e))
    return chosen


def sample_rows(lay: dict, T: int, k: int, n_tokens: int, seed: int = 0, per_expert: int = 8,
                n_full: int = 8):
    """Slots a full-size check compares: every kept pair of a seeded token
    sample; the first and last computed row of every non-empty expert (the
    ragged tails) and ``per_expert`` more seeded rows of each; and every row
    of ``n_full`` experts (``full_experts``).  Returns (tokens, slot mask,
    those experts).  Works for the dropless and the fixed-capacity
    layouts."""
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(T, size=min(n_tokens, T), replace=False))
    sop = lay["slot_of_pair"].numpy().reshape(T, k)
    mask = np.zeros(lay["pair_of_slot"].numel(), dtype=bool)
    picked = sop[toks].reshape(-1)
    mask[picked[picked >= 0]] = True
    off = lay["expert_offsets"].numpy()
    cnt = lay["expert_counts"].numpy()
    for e in range(len(off) - 1):
        if cnt[e] > 0:
            mask[off[e]] = True
            mask[off[e] + cnt[e] - 1] = True
            mask[off[e] + rng.choice(cnt[e], size=min(per_expert, cnt[e]), replace=False)] = True
    experts = full_experts(lay, n_full, seed)
    for e in experts:
        mask[off[e]:off[e] + cnt[e]] = True
    return torch.from_numpy(toks), torch.from_numpy(mask), experts


def oracle_gemm_rows(wl, xp, sc, offsets, mask, w13=None, w2=None, batch=16):
    """Oracle h and y for the masked slots.  Every output row depends only
    on its own input row and its expert's weights, so the oracle runs on a
    compact sub-problem: the sampled rows of up to ``batch`` experts at a
    time, with those experts' weights (re-drawn per expert on the host
    unless given).  Returns (slots, h, y), rows in ascending slot order."""
    off = offsets.tolist()
    todo = []
    for e in range(wl.E):
        lo, hi = off[e], off[e + 1]
        sel = torch.nonzero(mask[lo:hi]).flatten() + lo
        if sel.numel():
            todo.append((e, sel))
    slots, hs, ys = [], [], []
    for i in range(0, len(todo), batch):
        chunk = todo[i:i + batch]
        sel = torch.cat([s for _, s in chunk])
        a13 = torch.stack([w13[e] if w13 is not None else workloads.expert_w13(wl, e)
                           for e, _ in chunk]).contiguous()
        a2 = torch.stack([w2[e] if w2 is not None else workloads.expert_w2(wl, e)
                          for e, _ in chunk]).contiguous()
        xe = xp[sel].contiguous()
        se = sc[sel].contiguous() if sc is not None else None
        oe = torch.tensor([0] + list(np.cumsum([s.numel() for _, s in chunk])), dtype=torch.int32)
        he, ye, done = oracle.grouped_gemm(xe, se, oe, 0, len(chunk), a13, a2)
        assert done == sel.numel()
        slots.append(sel)
        hs.append(he)
        ys.append(ye)
    return torch.cat(slots), torch.cat(hs), torch.cat(ys)
