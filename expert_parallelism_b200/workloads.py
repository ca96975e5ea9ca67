"""Seeded synthetic inputs for the MoE-layer hot path.

This module only draws random numbers and lays them out; it holds none of
the layer's arithmetic (no top-k, no layout, no quantisation, no GEMM).  Both
the CUDA path and the CPU oracle take their inputs from here, so that the two
sides see bit-identical bytes.

Workloads (shapes from the pages' problem statement: x[T, H] tokens,
idx/weights[T, k], E experts, E/world experts per logical rank; see
"Expert Parallelism" (aiwiki), section "Implementation", and "Expert
parallelism" (Transformers docs), section "How the sizes combine"):

  name    T      H     E    k  I     W  activations / payload / GEMM
  tiny    256    128   8    2  256   2  fp32 / fp32 / fp32
  mid     4096   2048  64   6  1408  4  bf16 / bf16 / bf16
  dsv3    8192   7168  256  8  2048  8  bf16 / e4m3 + per-128 scales / bf16
  skew    16384  2880  128  4  2880  8  bf16 / bf16 / bf16, Zipf(1.2) router bias
  decode  64     7168  256  8  2048  8  bf16 / bf16 / bf16

Expert outputs y are stored in fp32 for every workload (the combine then
rounds only once, into out); h, the down projection's operand, has the
GEMM's dtype.

Distributions: router logits ~ N(0, 1) in fp32 (plus, for ``skew``, a
per-expert bias log p_{pi(e)} with p_r proportional to r^-1.2 over a seeded
permutation pi); x ~ N(0, 1) cast to the activation dtype; W13[e] ~
N(0, 1/H) and W2[e] ~ N(0, 1/I) (fan-in scaling), drawn in fp32 and cast
to the weight dtype.

Every tensor is drawn from its own CPU ``torch.Generator`` whose seed is
derived from (seed, tensor tag, expert index).  Each expert's weights can
therefore be re-drawn on their own, which lets a check on a sample of
experts regenerate just those experts on the host.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import hashlib
import math
import os

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    H: int          # hidden size
    E: int          # experts
    k: int          # experts per token
    I: int          # expert FFN intermediate size
    W: int          # logical EP ranks (E/W experts each)
    act: str        # activation dtype of x / out: "f32" | "bf16"
    payload: str    # dispatch payload dtype: "f32" | "bf16" | "e4m3"
    wdt: str        # expert weight / GEMM dtype: "f32" | "bf16"
    router: str = "normal"   # "normal" | "zipf"
    zipf_s: float = 1.2
    seed: int = 0
    ydt: str = "f32"         # storage of the experts' outputs y (combine's input)
    capacity_factor: float | None = None   # None: dropless; else fixed slabs per expert
    route_groups: int = 0                  # 0: plain top-k; G: group-limited routing
    route_max_groups: int = 0              # M: groups a token may reach (with route_groups)
    fused_gather: bool = False             # the gate/up GEMM gathers rows from x (no xp copy)
    all_reduce_form: bool = False          # combine as W per-rank partials summed over ranks
    packed_weights: bool = False           # expert weights re-laid out in 16 KB blocks
    weights_in_gemm: bool = False          # router weights applied in the down GEMM's epilogue

    @property
    def N(self) -> int:
        """Routed (token, expert) pairs."""
        return self.T * self.k

    @property
    def experts_per_rank(self) -> int:
        return self.E // self.W

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 256, 128, 8, 2, 256, 2, "f32", "f32", "f32"),
    "mid": Workload("mid", 4096, 2048, 64, 6, 1408, 4, "bf16", "bf16", "bf16"),
    "dsv3": Workload("dsv3", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3", "bf16"),
    "skew": Workload("skew", 16384, 2880, 128, 4, 2880, 8, "bf16", "bf16", "bf16",
                     router="zipf"),
    "decode": Workload("decode", 64, 7168, 256, 8, 2048, 8, "bf16", "bf16", "bf16"),
    # fixed-capacity variants: slabs of ceil(factor * T*k / E) rows per expert
    "dsv3_cap": Workload("dsv3_cap", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3", "bf16",
                         capacity_factor=1.0),
    "skew_cap": Workload("skew_cap", 16384, 2880, 128, 4, 2880, 8, "bf16", "bf16", "bf16",
                         router="zipf", capacity_factor=1.25),
    # FP8 combine payload: the experts' outputs travel back as e4m3 + block scales
    "dsv3_fp8y": Workload("dsv3_fp8y", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3", "bf16",
                          ydt="e4m3"),
    # group-limited routing: each token reaches at most 4 of the 8 rank groups
    "dsv3_grouped": Workload("dsv3_grouped", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3",
                             "bf16", route_groups=8, route_max_groups=4),
    # fused gather: the gate/up GEMM reads each routed row from the token-major
    # activations through pair_of_slot, with no permuted copy in between
    "dsv3_fused": Workload("dsv3_fused", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3", "bf16",
                           fused_gather=True),
    "mid_fused": Workload("mid_fused", 4096, 2048, 64, 6, 1408, 4, "bf16", "bf16", "bf16",
                          fused_gather=True),
    "skew_fused": Workload("skew_fused", 16384, 2880, 128, 4, 2880, 8, "bf16", "bf16", "bf16",
                           router="zipf", fused_gather=True),
    # the all_reduce form: each logical rank's partial sum over its own
    # experts' picks, then the sum over ranks (the all-reduce) rounded once
    "dsv3_allreduce": Workload("dsv3_allreduce", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3",
                               "bf16", all_reduce_form=True),
    "decode_allreduce": Workload("decode_allreduce", 64, 7168, 256, 8, 2048, 8, "bf16", "bf16",
                                 "bf16", all_reduce_form=True),
    # expert weights re-laid out once (moe_pack_expert_weights) into 16 KB blocks
    "dsv3_packed": Workload("dsv3_packed", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3", "bf16",
                            packed_weights=True),
    "mid_packed": Workload("mid_packed", 4096, 2048, 64, 6, 1408, 4, "bf16", "bf16", "bf16",
                           packed_weights=True),
    "skew_packed": Workload("skew_packed", 16384, 2880, 128, 4, 2880, 8, "bf16", "bf16", "bf16",
                            router="zipf", packed_weights=True),
    "decode_packed": Workload("decode_packed", 64, 7168, 256, 8, 2048, 8, "bf16", "bf16", "bf16",
                              packed_weights=True),
    # the router weights applied in the down GEMM's epilogue; the combine sums
    "dsv3_wgemm": Workload("dsv3_wgemm", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3", "bf16",
                           weights_in_gemm=True),
    # both halves of the fused row: the gather and the weights in the GEMM
    "dsv3_fused_wgemm": Workload("dsv3_fused_wgemm", 8192, 7168, 256, 8, 2048, 8, "bf16", "e4m3",
                                 "bf16", fused_gather=True, weights_in_gemm=True),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16,
               "e4m3": torch.float8_e4m3fn}
ELEM_BYTES = {"f32": 4, "bf16": 2, "e4m3": 1}


def derived_seed(seed: int, tag: str, index: int = 0) -> int:
    """A 63-bit generator seed for one tensor (or one expert's slice of it)."""
    h = hashlib.sha256(f"{seed}:{tag}:{index}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, tag: str, index: int = 0) -> torch.Generator:
    return torch.Generator().manual_seed(derived_seed(seed, tag, index))


def zipf_bias(wl: Workload) -> torch.Tensor:
    """Per-expert additive router bias log p_{pi(e)}, p_r = r^-s / sum r'^-s."""
    perm = torch.randperm(wl.E, generator=_gen(wl.seed, "perm"))  # pi, 0-based ranks
    r = torch.arange(1, wl.E + 1, dtype=torch.float64)
    p = r.pow(-wl.zipf_s)
    p = p / p.sum()
    return torch.log(p)[perm].to(torch.float32)


def router_logits(wl: Workload) -> torch.Tensor:
    """fp32 [T, E] router logits."""
    logits = torch.randn(wl.T, wl.E, generator=_gen(wl.seed, "logits"),
                         dtype=torch.float32)
    if wl.router == "zipf":
        logits = logits + zipf_bias(wl)[None, :]
    return logits.contiguous()


def hidden_states(wl: Workload) -> torch.Tensor:
    """[T, H] token activations in the activation dtype."""
    x = torch.randn(wl.T, wl.H, generator=_gen(wl.seed, "x"), dtype=torch.float32)
    return x.to(TORCH_DTYPE[wl.act]).contiguous()


def expert_w13(wl: Workload, e: int) -> torch.Tensor:
    """[2I, H] gate rows 0..I-1 then up rows I..2I-1 of expert e."""
    w = torch.randn(2 * wl.I, wl.H, generator=_gen(wl.seed, "w13", e),
                    dtype=torch.float32)
    w.mul_(1.0 / math.sqrt(wl.H))
    return w.to(TORCH_DTYPE[wl.wdt])


def expert_w2(wl: Workload, e: int) -> torch.Tensor:
    """[H, I] down projection of expert e."""
    w = torch.randn(wl.H, wl.I, generator=_gen(wl.seed, "w2", e), dtype=torch.float32)
    w.mul_(1.0 / math.sqrt(wl.I))
    return w.to(TORCH_DTYPE[wl.wdt])


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def fill_expert_weights(wl: Workload, w13: torch.Tensor, w2: torch.Tensor,
                        experts: range | list | None = None) -> None:
    """Draw experts' weights into preallocated [E', 2I, H] / [E', H, I] tensors.

    ``w13[j]`` receives expert ``experts[j]``.  The target tensors may live
    on any device; experts are drawn on the host in a thread pool (each
    expert has its own generator, so the result does not depend on the
    thread count) and copied over one by one.
    """
    experts = list(range(wl.E)) if experts is None else list(experts)

    def one(j_e):
        j, e = j_e
        return j, expert_w13(wl, e), expert_w2(wl, e)

    with _cf.ThreadPoolExecutor(_threads()) as pool:
        for j, a, b in pool.map(one, enumerate(experts)):
            w13[j].copy_(a)
            w2[j].copy_(b)


def layer_inputs(wl: Workload, with_weights: bool = True, device="cpu"):
    """All inputs of one layer: dict(logits, x, w13, w2) on ``device``."""
    out = {"logits": router_logits(wl).to(device), "x": hidden_states(wl).to(device)}
    if with_weights:
        dt = TORCH_DTYPE[wl.wdt]
        w13 = torch.empty(wl.E, 2 * wl.I, wl.H, dtype=dt, device=device)
        w2 = torch.empty(wl.E, wl.H, wl.I, dtype=dt, device=device)
        fill_expert_weights(wl, w13, w2)
        out["w13"], out["w2"] = w13, w2
    return out
