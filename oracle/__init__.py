"""CPU oracle for the MoE-layer hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it
and shares no code with it.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, OpenMP over the
GEMM's rows); this module compiles it on first use and marshals CPU torch
tensors in and out.  Every function takes and returns CPU tensors; bf16
data travels as its bit pattern.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

F32, BF16, E4M3, F64 = 0, 1, 2, 3
_CODE = {"f32": F32, "bf16": BF16, "e4m3": E4M3, "f64": F64}
_TDT = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn,
        "f64": torch.float64}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmoe_oracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I32, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        lib.oracle_route_topk.argtypes = [P, I64, I32, I32, P, P]
        lib.oracle_route_topk.restype = I
        lib.oracle_dispatch_layout.argtypes = [P, I64, I32, I32, I32, P, P, P, P, P]
        lib.oracle_dispatch_layout.restype = I64
        lib.oracle_quantize_rows_e4m3.argtypes = [P, I64, I32, P, P]
        lib.oracle_quantize_rows_e4m3.restype = I
        lib.oracle_combine_e4m3.argtypes = [P, P, P, P, I64, I32, I32, P, I]
        lib.oracle_combine_e4m3.restype = I
        lib.oracle_route_topk_grouped.argtypes = [P, I64, I32, I32, I32, I32, P, P]
        lib.oracle_route_topk_grouped.restype = I
        lib.oracle_dispatch_layout_capacity.argtypes = [P, I64, I32, I32, I32, I32, P, P, P, P,
                                                         P, P]
        lib.oracle_dispatch_layout_capacity.restype = I64
        lib.oracle_permute.argtypes = [P, I, I64, I32, I32, P, I64, P, I, P]
        lib.oracle_permute.restype = I
        lib.oracle_grouped_gemm.argtypes = [P, I, P, P, I32, I32, I32, I32, P, P, I, P, P, P, I]
        lib.oracle_grouped_gemm.restype = I64
        lib.oracle_combine.argtypes = [P, I, P, P, I64, I32, I32, P, I]
        lib.oracle_combine.restype = I
        lib.oracle_combine_rank.argtypes = [P, I, P, P, I64, I32, I32, P, I32, I32, P, I]
        lib.oracle_combine_rank.restype = I
        lib.oracle_reduce_partials.argtypes = [P, I, I32, I64, P, I]
        lib.oracle_reduce_partials.restype = I
        lib.oracle_ep_plan.argtypes = [P, I32, I32, I32, P, P]
        lib.oracle_ep_plan.restype = I64
        lib.oracle_e4m3_encode.argtypes = [P, I64, P]
        lib.oracle_e4m3_decode.argtypes = [P, I64, P]
        lib.oracle_bf16_round.argtypes = [P, I64, P]
        _lib = lib
    return _lib


def _p(t: torch.Tensor | None):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


def _dt_name(t: torch.Tensor) -> str:
    for k, v in _TDT.items():
        if t.dtype == v:
            return k
    raise TypeError(f"oracle: unsupported dtype {t.dtype}")


# ---------------------------------------------------------------- codecs
def e4m3_encode(v: torch.Tensor) -> torch.Tensor:
    """fp32 -> e4m3 code bytes (uint8), RNE with saturation to +-448."""
    v = v.to(torch.float32).contiguous()
    out = torch.empty(v.shape, dtype=torch.uint8)
    _load().oracle_e4m3_encode(_p(v), v.numel(), _p(out))
    return out


def e4m3_decode(c: torch.Tensor) -> torch.Tensor:
    """e4m3 code bytes -> fp64 values."""
    c = c.contiguous().view(torch.uint8)
    out = torch.empty(c.shape, dtype=torch.float64)
    _load().oracle_e4m3_decode(_p(c), c.numel(), _p(out))
    return out


def bf16_round(v: torch.Tensor) -> torch.Tensor:
    """fp64 -> bf16 (RNE), returned as a bfloat16 tensor."""
    v = v.to(torch.float64).contiguous()
    out = torch.empty(v.shape, dtype=torch.int16)
    _load().oracle_bf16_round(_p(v), v.numel(), _p(out))
    return out.view(torch.bfloat16)


# ---------------------------------------------------------------- the five steps
def route_topk(logits: torch.Tensor, k: int):
    logits = logits.to(torch.float32).contiguous()
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32)
    w = torch.empty(T, k, dtype=torch.float32)
    _load().oracle_route_topk(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def route_topk_grouped(logits: torch.Tensor, k: int, groups: int, max_groups: int):
    """Top-k restricted to the ``max_groups`` best of ``groups`` equal expert
    groups (a group's score: its largest logit); softmax over the picks."""
    logits = logits.to(torch.float32).contiguous()
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32)
    w = torch.empty(T, k, dtype=torch.float32)
    rc = _load().oracle_route_topk_grouped(_p(logits), T, E, k, groups, max_groups, _p(idx),
                                           _p(w))
    if rc != 0:
        raise ValueError("route_topk_grouped: need groups | E and k <= max_groups * E / groups")
    return idx, w


def dispatch_layout(topk_idx: torch.Tensor, E: int, W: int):
    topk_idx = topk_idx.to(torch.int32).contiguous()
    T, k = topk_idx.shape
    N = T * k
    counts = torch.empty(E, dtype=torch.int32)
    offsets = torch.empty(E + 1, dtype=torch.int32)
    rank_offsets = torch.empty(W + 1, dtype=torch.int32)
    slot_of_pair = torch.empty(N, dtype=torch.int32)
    pair_of_slot = torch.empty(N, dtype=torch.int32)
    bad = _load().oracle_dispatch_layout(_p(topk_idx), T, k, E, W, _p(counts), _p(offsets),
                                         _p(rank_offsets), _p(slot_of_pair), _p(pair_of_slot))
    return dict(expert_counts=counts, expert_offsets=offsets, rank_offsets=rank_offsets,
                slot_of_pair=slot_of_pair, pair_of_slot=pair_of_slot, skipped=int(bad))


def dispatch_layout_capacity(topk_idx: torch.Tensor, E: int, W: int, C: int):
    """Fixed-capacity layout: expert e's slab is rows [e*C, (e+1)*C), filled
    by its earliest pairs; later pairs are dropped (slot -1).  Returns the
    dropless layout's keys plus ``dropped``; ``expert_counts`` holds the
    kept rows per expert and ``pair_of_slot`` has E*C entries."""
    topk_idx = topk_idx.to(torch.int32).contiguous()
    T, k = topk_idx.shape
    counts = torch.empty(E, dtype=torch.int32)
    offsets = torch.empty(E + 1, dtype=torch.int32)
    rank_offsets = torch.empty(W + 1, dtype=torch.int32)
    slot_of_pair = torch.empty(T * k, dtype=torch.int32)
    pair_of_slot = torch.empty(max(E * C, 1), dtype=torch.int32)
    skipped = ctypes.c_int64(0)
    dropped = _load().oracle_dispatch_layout_capacity(
        _p(topk_idx), T, k, E, W, C, _p(counts), _p(offsets), _p(rank_offsets),
        _p(slot_of_pair), _p(pair_of_slot), ctypes.byref(skipped))
    return dict(expert_counts=counts, expert_offsets=offsets, rank_offsets=rank_offsets,
                slot_of_pair=slot_of_pair, pair_of_slot=pair_of_slot[:E * C],
                dropped=int(dropped), skipped=int(skipped.value))


def capacity_rows(T: int, k: int, E: int, capacity_factor: float) -> int:
    """Rows per expert slab: ceil(capacity_factor * T * k / E) (the plainest
    reading; the pages give no formula)."""
    import math
    return int(math.ceil(capacity_factor * T * k / E))


def permute(x: torch.Tensor, k: int, pair_of_slot: torch.Tensor, payload: str,
            fill: float = 0.0):
    """Returns (xp, xp_scales or None).  Slots holding -1 keep ``fill``."""
    x = x.contiguous()
    T, H = x.shape
    n_slots = pair_of_slot.numel()
    xdt = _dt_name(x)
    if payload == "e4m3":
        xp = torch.full((n_slots, H), 0, dtype=torch.uint8)
        sc = torch.full((n_slots, H // 128), fill, dtype=torch.float32)
    else:
        xp = torch.full((n_slots, H), fill, dtype=_TDT[payload])
        sc = None
    rc = _load().oracle_permute(_p(x), _CODE[xdt], T, H, k, _p(pair_of_slot.contiguous()),
                                n_slots, _p(xp), _CODE[payload], _p(sc))
    if rc != 0:
        raise ValueError("oracle.permute: unsupported dtype pair")
    if payload == "e4m3":
        xp = xp.view(torch.float8_e4m3fn)
    return xp, sc


def grouped_gemm(xp: torch.Tensor, xp_scales, expert_offsets: torch.Tensor,
                 expert_begin: int, n_experts: int, w13: torch.Tensor, w2: torch.Tensor,
                 row_mask: torch.Tensor | None = None, out: str = "f64"):
    """Returns (h, y, rows_done).  h and y come back in ``out``: "f64" =
    unrounded (the default: what parity compares against), or the weight
    dtype's storage rounding.  The down projection always consumes h
    rounded to the weight dtype.  Rows outside the mask (or outside the
    experts' segments) are left as NaN."""
    xp = xp.contiguous()
    n_rows, H = xp.shape
    I = w2.shape[2]
    wdt = _dt_name(w13)
    h = torch.full((n_rows, I), float("nan"), dtype=_TDT[out])
    y = torch.full((n_rows, H), float("nan"), dtype=_TDT[out])
    mask = None if row_mask is None else row_mask.to(torch.uint8).contiguous()
    xdt = _dt_name(xp)
    done = _load().oracle_grouped_gemm(
        _p(xp.view(torch.uint8) if xdt == "e4m3" else xp), _CODE[xdt],
        _p(xp_scales.contiguous() if xp_scales is not None else None),
        _p(expert_offsets.to(torch.int32).contiguous()), expert_begin, n_experts, H, I,
        _p(w13.contiguous()), _p(w2.contiguous()), _CODE[wdt], _p(mask), _p(h), _p(y),
        _CODE[out])
    return h, y, int(done)


def combine(y: torch.Tensor, slot_of_pair: torch.Tensor, topk_w: torch.Tensor,
            out_dtype: str = "f64"):
    """Weighted sum of each token's k rows of y (read in y's own dtype), in
    fp64; "f64" returns it unrounded."""
    y = y.contiguous()
    T, k = topk_w.shape
    H = y.shape[1]
    out = torch.empty(T, H, dtype=_TDT[out_dtype])
    _load().oracle_combine(_p(y), _CODE[_dt_name(y)], _p(slot_of_pair.to(torch.int32).contiguous()),
                           _p(topk_w.to(torch.float32).contiguous()), T, k, H, _p(out),
                           _CODE[out_dtype])
    return out


def combine_rank(y: torch.Tensor, slot_of_pair: torch.Tensor, topk_w: torch.Tensor,
                 rank_offsets: torch.Tensor, rank: int, out_dtype: str = "f64"):
    """Rank ``rank``'s partial of the all_reduce form: each token's weighted
    sum over only the picks whose slot lies in the rank's slab
    [rank_offsets[rank], rank_offsets[rank+1]) (zero rows for tokens it does
    not serve); fp64, "f64" unrounded."""
    y = y.contiguous()
    T, k = topk_w.shape
    H = y.shape[1]
    ro = rank_offsets.to(torch.int32).contiguous()
    out = torch.empty(T, H, dtype=_TDT[out_dtype])
    rc = _load().oracle_combine_rank(_p(y), _CODE[_dt_name(y)],
                                     _p(slot_of_pair.to(torch.int32).contiguous()),
                                     _p(topk_w.to(torch.float32).contiguous()), T, k, H, _p(ro),
                                     ro.numel() - 1, rank, _p(out), _CODE[out_dtype])
    if rc != 0:
        raise ValueError("combine_rank: rank outside [0, world)")
    return out


def reduce_partials(partials: torch.Tensor, out_dtype: str = "f64"):
    """Sum of the ranks' partials [n, T, H] (the all-reduce), in fp64,
    rounded once to ``out_dtype``."""
    p = partials.contiguous()
    n = p.shape[0]
    out = torch.empty(p.shape[1:], dtype=_TDT[out_dtype])
    _load().oracle_reduce_partials(_p(p), _CODE[_dt_name(p)], n, p[0].numel(), _p(out),
                                   _CODE[out_dtype])
    return out


def quantize_rows_e4m3(v: torch.Tensor):
    """Per-128 block FP8 e4m3 quantisation of rows of fp32 values (the
    combine payload's rule: scale = amax / 448, codes e4m3(v * (1 / scale)));
    returns (codes as float8_e4m3fn, fp32 scales)."""
    v = v.to(torch.float32).contiguous()
    rows, H = v.shape
    q = torch.empty(rows, H, dtype=torch.uint8)
    sc = torch.empty(rows, H // 128, dtype=torch.float32)
    if _load().oracle_quantize_rows_e4m3(_p(v), rows, H, _p(q), _p(sc)) != 0:
        raise ValueError("quantize_rows_e4m3: H must be a multiple of 128")
    return q.view(torch.float8_e4m3fn), sc


def combine_e4m3(q: torch.Tensor, scales: torch.Tensor, slot_of_pair: torch.Tensor,
                 topk_w: torch.Tensor, out_dtype: str = "f64"):
    """Weighted sum of each token's k FP8 rows, each dequantised as the fp32
    product decode(q) * scale; summed in fp64 ("f64": unrounded)."""
    q = q.contiguous().view(torch.uint8)
    T, k = topk_w.shape
    H = q.shape[1]
    out = torch.empty(T, H, dtype=_TDT[out_dtype])
    rc = _load().oracle_combine_e4m3(_p(q), _p(scales.to(torch.float32).contiguous()),
                                     _p(slot_of_pair.to(torch.int32).contiguous()),
                                     _p(topk_w.to(torch.float32).contiguous()), T, k, H,
                                     _p(out), _CODE[out_dtype])
    if rc != 0:
        raise ValueError("combine_e4m3: H must be a multiple of 128")
    return out


def round_to(v: torch.Tensor, dtype: str) -> torch.Tensor:
    """fp64 values rounded to a storage type with the oracle's own rounding."""
    if dtype == "bf16":
        return bf16_round(v)
    if dtype == "f32":
        return v.to(torch.float32)      # IEEE round-to-nearest-even
    return v


def layer(wl, inputs, row_mask=None):
    """The whole hot path on one workload's inputs; returns every
    intermediate (dict).  h, y and out are unrounded (fp64): out is the
    weighted sum of the exact y.  ``row_mask`` (per slot) samples the GEMM
    rows; combine is then only meaningful for tokens whose pairs were all
    computed.  A workload with a capacity_factor uses the fixed-capacity
    layout (dropped pairs add nothing to out)."""
    if getattr(wl, "route_groups", 0):
        idx, w = route_topk_grouped(inputs["logits"], wl.k, wl.route_groups, wl.route_max_groups)
    else:
        idx, w = route_topk(inputs["logits"], wl.k)
    if getattr(wl, "capacity_factor", None) is None:
        lay = dispatch_layout(idx, wl.E, wl.W)
    else:   # fixed slabs: only the slab rows holding a pair are computed
        C = capacity_rows(wl.T, wl.k, wl.E, wl.capacity_factor)
        lay = dispatch_layout_capacity(idx, wl.E, wl.W, C)
        kept = lay["pair_of_slot"] >= 0
        row_mask = kept if row_mask is None else (row_mask & kept)
    xp, sc = permute(inputs["x"], wl.k, lay["pair_of_slot"], wl.payload)
    h, y, _ = grouped_gemm(xp, sc, lay["expert_offsets"], 0, wl.E, inputs["w13"], inputs["w2"],
                           row_mask)
    if getattr(wl, "ydt", None) == "e4m3":
        # FP8 combine payload: the exact y, held in fp32, quantised per 128 block
        yq, ysc = quantize_rows_e4m3(torch.nan_to_num(y, nan=0.0).float())
        out = combine_e4m3(yq, ysc, lay["slot_of_pair"], w)
        return dict(topk_idx=idx, topk_w=w, xp=xp, xp_scales=sc, h=h, y=y, y_q=yq, y_scales=ysc,
                    out=out, **lay)
    out = combine(y, lay["slot_of_pair"], w)
    return dict(topk_idx=idx, topk_w=w, xp=xp, xp_scales=sc, h=h, y=y, out=out, **lay)


# ---------------------------------------------------------------- expert parallelism
def ep_plan(counts_all: torch.Tensor, rank: int):
    """The dispatch plan of rank ``rank`` from every rank's expert counts
    ``counts_all`` [W, E] (the count exchange).  Returns (send_base [E]: the
    row of each expert's owner's receive buffer where this rank's rows for
    it begin; recv_offsets [E/W + 1]: where each local expert begins in this
    rank's own receive buffer).  Receive order: expert by expert, inside an
    expert by source rank, each source's rows in its slot order."""
    c = counts_all.to(torch.int32).contiguous()
    W, E = c.shape
    send_base = torch.empty(E, dtype=torch.int32)
    recv_offsets = torch.empty(E // W + 1, dtype=torch.int32)
    if _load().oracle_ep_plan(_p(c), W, E, rank, _p(send_base), _p(recv_offsets)) < 0:
        raise ValueError("ep_plan: W must divide E and rank lie in [0, W)")
    return send_base, recv_offsets


def ep_dest_rows(lay: dict, topk_idx: torch.Tensor, send_base: torch.Tensor, E: int, W: int):
    """Where each of a rank's routed pairs lands: (owner rank [N], row of the
    owner's receive buffer [N]); -1 for a skipped pair.  A pair in slot s of
    the sender's own expert-major layout, routed to expert e, is the
    (s - expert_offsets[e])-th row the sender sends to e."""
    idx = topk_idx.reshape(-1).long()
    sop = lay["slot_of_pair"].long()
    ok = sop >= 0
    e = idx.clamp(0, E - 1)
    owner = torch.where(ok, e // (E // W), torch.full_like(e, -1))
    row = torch.where(ok, send_base.long()[e] + sop - lay["expert_offsets"].long()[e],
                      torch.full_like(e, -1))
    return owner, row


def ep_layer(wl, inputs_per_rank, w13, w2):
    """The expert-parallel layer over W = len(inputs_per_rank) ranks, simulated
    in one process: every rank routes its own tokens and lays them out
    (route_topk, dispatch_layout), the counts are exchanged, each row is moved
    to its owner's receive buffer by the plan, each owner runs its own
    experts on what it received (grouped_gemm with w13/w2 rows
    [r*E/W, (r+1)*E/W)), the rows travel back, and each rank combines its
    tokens' k rows.  Returns per rank a dict with out (fp64, unrounded), the
    plan and the receive buffer's offsets."""
    W, E, k = len(inputs_per_rank), wl.E, wl.k
    Er = E // W
    per = []
    for inp in inputs_per_rank:
        idx, w = route_topk(inp["logits"], k)
        per.append(dict(idx=idx, w=w, lay=dispatch_layout(idx, E, W), x=inp["x"]))
    counts_all = torch.stack([p["lay"]["expert_counts"] for p in per])
    for r, p in enumerate(per):
        p["send_base"], p["recv_offsets"] = ep_plan(counts_all, r)
        p["owner"], p["row"] = ep_dest_rows(p["lay"], p["idx"], p["send_base"], E, W)
    # dispatch: each pair's payload row goes to (owner, row)
    recv = []
    for r in range(W):
        n = int(per[r]["recv_offsets"][-1])
        H = wl.H
        if wl.payload == "e4m3":
            buf = (torch.zeros(n, H, dtype=torch.uint8), torch.zeros(n, H // 128))
        else:
            buf = (torch.zeros(n, H, dtype=_TDT[wl.payload]), None)
        recv.append(buf)
    for s, p in enumerate(per):
        xp, sc = permute(p["x"], k, p["lay"]["pair_of_slot"], wl.payload)
        sop = p["lay"]["slot_of_pair"].long()
        for q in torch.nonzero(p["owner"] >= 0).flatten().tolist():
            r, row = int(p["owner"][q]), int(p["row"][q])
            src = int(sop[q])
            if wl.payload == "e4m3":
                recv[r][0][row] = xp.view(torch.uint8)[src]
                recv[r][1][row] = sc[src]
            else:
                recv[r][0][row] = xp[src]
    # every owner runs its own experts on its receive buffer
    ys = []
    for r in range(W):
        q, sc = recv[r]
        if wl.payload == "e4m3":
            q = q.view(torch.float8_e4m3fn)
        _, y, _ = grouped_gemm(q, sc, per[r]["recv_offsets"], 0, Er,
                               w13[r * Er:(r + 1) * Er].contiguous(),
                               w2[r * Er:(r + 1) * Er].contiguous())
        ys.append(y)
    # combine: the rows come back to their sender's slots, then the k-way sum
    outs = []
    for s, p in enumerate(per):
        N = p["lay"]["slot_of_pair"].numel()
        y_home = torch.zeros(N, wl.H, dtype=torch.float64)
        sop = p["lay"]["slot_of_pair"].long()
        for q in torch.nonzero(p["owner"] >= 0).flatten().tolist():
            y_home[sop[q]] = ys[int(p["owner"][q])][int(p["row"][q])]
        outs.append(dict(out=combine(y_home, p["lay"]["slot_of_pair"], p["w"]),
                         send_base=p["send_base"], recv_offsets=p["recv_offsets"],
                         counts_all=counts_all, owner=p["owner"], row=p["row"]))
    return outs
