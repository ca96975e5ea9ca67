#!/usr/bin/env python3
"""Benchmark of the single-GPU MoE-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dsv3]
                    [--impl ours|reference] [--no-cpu-baseline]

One step = one pass of the whole hot path (router top-k -> dispatch layout
-> permute -> grouped SwiGLU GEMM -> combine) over one batch of the
workload, inputs resident in HBM.  When a step streams more than 4x the L2
(126 MB) in expert weights, that alone evicts L2 between steps ("inputs
larger than L2"); smaller workloads get an explicit 512 MiB write-flush
before every step, outside the step's CUDA events.  With N > 1 (torchrun), every
rank runs an independent replica of the layer on its own GPU (no
collective on the data path: weak scaling); the per-step time is the max
over ranks.  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle instead (the only other place
that runs it), on a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_parallelism_b200 import moe, traffic, workloads  # noqa: E402

METRIC = "MoE-layer tokens/s (dispatch+grouped GEMM+combine); permute/combine HBM GB/s"
L2_FLUSH_BYTES = 512 << 20
L2_BYTES = 126 << 20


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the timed
    region runs, kept sample by sample.  Two read-only sources run side by
    side: NVML polled every 5 ms from a thread (for the device whose UUID the
    CUDA runtime gives), and ``nvidia-smi -lms 50`` (the tool the recipe's
    clocks line uses).  Changes no setting."""

    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    SMI_NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device: torch.device, period_s: float = 0.005):
        self.device = device
        self.period = period_s
        self.nvml, self.smi = [], []      # (ms since start, MHz, reason names)
        self.max_mhz = None
        self.stop = threading.Event()
        self.threads = []
        self.proc = None
        self.t0 = None

    def _uuid(self):
        u = str(torch.cuda.get_device_properties(self.device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u

    def _now_ms(self):
        return (time.perf_counter() - self.t0) * 1e3

    def _poll_nvml(self, nv, h):
        self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop.is_set():
            mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            names = [n for n, b in self.REASONS.items() if bits & b]
            self.nvml.append((self._now_ms(), mhz, names))
            self.stop.wait(self.period)

    def _read_smi(self):
        for ln in self.proc.stdout:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 6:
                continue
            try:
                mhz, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            self.max_mhz = self.max_mhz or mx
            names = [n for n, v in zip(self.SMI_NAMES, parts[2:6]) if v.lower() == "active"]
            self.smi.append((self._now_ms(), mhz, names))

    def __enter__(self):
        self.t0 = time.perf_counter()
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self._uuid())
            self.threads.append(threading.Thread(target=self._poll_nvml, args=(nv, h),
                                                 daemon=True))
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._uuid(), f"--query-gpu={self.SMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.threads.append(threading.Thread(target=self._read_smi, daemon=True))
        except Exception:
            self.proc = None
        for t in self.threads:
            t.start()
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        for t in self.threads:
            t.join(timeout=5)

    @staticmethod
    def _stats(samples):
        if not samples:
            return None
        mhz = sorted(s[1] for s in samples)
        cap = sum(1 for s in samples if "sw_power_cap" in s[2])
        return {"samples": len(samples), "sm_mhz_median": statistics.median(mhz),
                "sm_mhz_p10": mhz[min(len(mhz) - 1, int(0.1 * len(mhz)))], "sm_mhz_min": mhz[0],
                "sw_power_cap_frac": cap / len(samples),
                "reasons": sorted({n for s in samples for n in s[2]}),
                # (ms from the start of the timed region, MHz, active reasons)
                "trace": [[round(s[0], 1), s[1], s[2]] for s in samples[:64]]}

    def summary(self, ms_per_step=None):
        """Median and spread per source; the headline figures take
        nvidia-smi's when it gave at least 3 samples, else NVML's.
        ``ms_x_mhz`` (step time x median SM MHz) lets step times taken at
        different clocks be compared."""
        nv, smi = self._stats(self.nvml), self._stats(self.smi)
        head = smi if smi and smi["samples"] >= 3 else (nv or smi)
        out = {"sm_mhz": head["sm_mhz_median"] if head else None, "sm_max_mhz": self.max_mhz,
               "reasons": sorted(set((nv or {}).get("reasons", [])) |
                                 set((smi or {}).get("reasons", []))),
               "source": ("nvidia-smi, 50 ms" if head is smi else "nvml, 5 ms") if head else None,
               "nvml": nv, "nvidia_smi": smi}
        if head and ms_per_step:
            out["ms_x_mhz"] = ms_per_step * head["sm_mhz_median"]
        return out


def max_over_ranks(values, device):
    """Element-wise max of per-rank times over the process group (identity
    without one).  Every rank must call it, in the same order."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(units_per_rank: int, world_size: int, ms_max: float) -> float:
    """Units all ranks processed divided by the slowest rank's time (weak
    scaling: every rank runs the same per-GPU work)."""
    return world_size * units_per_rank / (ms_max * 1e-3)


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------- CPU oracle leg
class OracleSample:
    """The CPU oracle run on the first S tokens of a workload: all five
    steps (route, layout, permute, GEMM, combine) in fp64.  The touched
    experts' weights are drawn on the host once, outside the timed calls,
    and kept for later runs of the same or a smaller sample."""

    def __init__(self, wl):
        self.wl = wl
        self.logits = workloads.router_logits(wl)
        self.x = workloads.hidden_states(wl)
        self.cache = {}

    def _route_layout(self, S):
        import oracle
        wl = self.wl
        lg, x = self.logits[:S].contiguous(), self.x[:S].contiguous()
        if wl.route_groups:
            idx, w = oracle.route_topk_grouped(lg, wl.k, wl.route_groups, wl.route_max_groups)
        else:
            idx, w = oracle.route_topk(lg, wl.k)
        if wl.capacity_factor is None:
            lay = oracle.dispatch_layout(idx, wl.E, wl.W)
        else:
            lay = oracle.dispatch_layout_capacity(
                idx, wl.E, wl.W, oracle.capacity_rows(S, wl.k, wl.E, wl.capacity_factor))
        return x, w, lay

    def prepare(self, S):
        """Draws (untimed) the weights of every expert the first S tokens
        reach."""
        import concurrent.futures as cf
        _, _, lay = self._route_layout(S)
        cnt = lay["expert_counts"].tolist()
        need = [e for e in range(self.wl.E) if cnt[e] > 0 and e not in self.cache]
        draw = lambda e: (e, workloads.expert_w13(self.wl, e), workloads.expert_w2(self.wl, e))
        with cf.ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as pool:
            for e, a, b in pool.map(draw, need):
                self.cache[e] = (a, b)

    def run(self, S):
        """Seconds of oracle work for the first S tokens (weight drawing
        excluded)."""
        import oracle
        wl = self.wl
        self.prepare(S)
        t0 = time.perf_counter()
        x, w, lay = self._route_layout(S)
        xp, sc = oracle.permute(x, wl.k, lay["pair_of_slot"], wl.payload)
        el = time.perf_counter() - t0
        off = lay["expert_offsets"].tolist()
        cnt = lay["expert_counts"].tolist()         # rows each expert computes
        touched = [e for e in range(wl.E) if cnt[e] > 0]
        y = torch.zeros(xp.shape[0], wl.H, dtype=torch.float64)
        for i in range(0, len(touched), 32):
            grp = touched[i:i + 32]
            rows = torch.cat([torch.arange(off[e], off[e] + cnt[e]) for e in grp])
            oe = torch.tensor([0] + list(torch.tensor([cnt[e] for e in grp])
                                         .cumsum(0).tolist()), dtype=torch.int32)
            a13 = torch.stack([self.cache[e][0] for e in grp])
            a2 = torch.stack([self.cache[e][1] for e in grp])
            t0 = time.perf_counter()
            _, ye, _ = oracle.grouped_gemm(xp[rows].contiguous(),
                                           sc[rows].contiguous() if sc is not None else None,
                                           oe, 0, len(grp), a13, a2)
            el += time.perf_counter() - t0
            y[rows] = ye
        t0 = time.perf_counter()
        oracle.combine(y, lay["slot_of_pair"], w, wl.act)
        el += time.perf_counter() - t0
        return el

    def tokens_for(self, seconds, probe=8):
        """Sample size whose oracle time is about ``seconds`` (the oracle's
        time is linear in the tokens: one probe run, then scaled)."""
        S = min(self.wl.T, probe)
        el = self.run(S)
        return max(1, min(self.wl.T, int(S * seconds / max(el, 1e-6))))


def _cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def oracle_sample(wl, target_s: float = 12.0, max_tokens: int | None = None):
    """cpu_baseline of the GPU line: the oracle on about ``target_s`` seconds
    of work (a token sample of the workload)."""
    o = OracleSample(wl)
    S = o.tokens_for(target_s)
    if max_tokens is not None:
        S = min(S, max_tokens)
    el = o.run(S)
    return {"value": S / el, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
            "sample": f"first {S} of {wl.T} tokens of workload {wl.name}, all five steps "
                      f"(fp64 C oracle, OpenMP over GEMM rows); {el:.2f} s of oracle time"}


def run_reference(args, wl):
    """The reference arm: the oracle as it stands, on rank 0 only.  Each of
    the W + K steps is the same bounded token sample S, sized once so that
    the whole run takes about ``--ref-budget`` seconds; ``ms_per_step`` is the
    measured time of those S-token steps, and ``value`` = S / that time."""
    ws, rank, local = _dist()
    if rank != 0:
        return
    o = OracleSample(wl)
    per_step = min(args.ref_seconds, args.ref_budget / max(1, args.steps + args.warmup))
    S = o.tokens_for(per_step)
    o.prepare(S)
    for _ in range(args.warmup):
        o.run(S)
    times = [o.run(S) for _ in range(args.steps)]
    sec = statistics.mean(times)
    v = S / sec
    sample = (f"first {S} of {wl.T} tokens of workload {wl.name} per step, all five steps "
              f"(fp64 C oracle, OpenMP over GEMM rows); {args.steps} timed steps of "
              f"{sec:.2f} s mean after {args.warmup} warm-up steps")
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * sec,
            "tokens_per_step": S, "ms_per_full_batch_extrapolated": 1000.0 * wl.T / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": _config(wl),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _weight_bytes(wl):
    return wl.E * 3 * wl.I * wl.H * workloads.ELEM_BYTES[wl.wdt]


def _needs_flush(wl):
    return _weight_bytes(wl) < 4 * L2_BYTES


def _capacity_info(buf, dropped):
    if buf.capacity < 0:
        return {}
    return {"capacity_rows_per_expert": buf.capacity, "pairs_dropped": dropped}


def _config(wl):
    l2 = (f"flushed ({L2_FLUSH_BYTES >> 20} MiB write) before every step" if _needs_flush(wl)
          else f"inputs larger than L2: {_weight_bytes(wl) / 1e9:.1f} GB of expert weights "
               f"streamed per step")
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
            "logical_ranks": wl.W, "activations": wl.act, "payload": wl.payload,
            "gemm": wl.wdt, "y": wl.ydt, "router": wl.router, "seed": wl.seed, "l2": l2,
            **({"capacity_factor": wl.capacity_factor} if wl.capacity_factor is not None else {}),
            **({"route_groups": wl.route_groups, "route_max_groups": wl.route_max_groups}
               if wl.route_groups else {}),
            "fused_gather": wl.fused_gather,
            **({"packed_weights": True} if wl.packed_weights else {}),
            **({"weights_in_gemm": True} if wl.weights_in_gemm else {}),
            **({"all_reduce_form": True} if wl.all_reduce_form else {}),
            "parallelism": "replicas (one independent layer per GPU)"}


# ---------------------------------------------------------------- GPU leg
def run_ours(args, wl):
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    lib = moe.load_library()
    inp = workloads.layer_inputs(wl, with_weights=False, device="cpu")
    logits, x = inp["logits"].to(dev), inp["x"].to(dev)
    wdt = workloads.TORCH_DTYPE[wl.wdt]
    w13 = torch.empty(wl.E, 2 * wl.I, wl.H, dtype=wdt, device=dev)
    w2 = torch.empty(wl.E, wl.H, wl.I, dtype=wdt, device=dev)
    workloads.fill_expert_weights(wl, w13, w2)
    if wl.packed_weights:
        # one-time re-layout of the weights (at load, outside every timed region)
        p13, p2 = moe.packed_weight_tensors(wl.E, wl.H, wl.I, dev)
        moe.moe_pack_expert_weights(w13, w2, p13, p2)
        torch.cuda.synchronize()
        del w13, w2
        w13, w2 = p13, p2
    buf = moe.LayerBuffers(wl, dev)
    flush = torch.empty(L2_FLUSH_BYTES if _needs_flush(wl) else 16, dtype=torch.uint8,
                        device=dev)
    stream = torch.cuda.current_stream()

    # spans between the 8 events moe_layer_forward records
    names = ["route_topk", "dispatch_layout", "permute", "dequant_e4m3", "gemm_gate_up",
             "gemm_down", "combine"]

    def step(evs):
        # one C call: the five steps, with an event before, between and after them
        moe.moe_layer_forward(wl, logits, x, w13, w2, buf, step_events=evs)

    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    for _ in range(args.warmup):
        flush.fill_(1)
        step(mk())
    torch.cuda.synchronize()
    st = moe.moe_check_status(buf.dev_status)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {moe.STATUS.get(st, st)}")

    moe.moe_diag_gemm_clock(reset=True)      # the GEMM's in-kernel clock record
    launches0 = lib.moe_launch_count()
    all_evs = [mk() for _ in range(args.steps)]
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        for i in range(args.steps):
            flush.fill_(1)
            step(all_evs[i])
        torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    launches = lib.moe_launch_count() - launches0      # over the whole timed region
    gemm_clock = moe.moe_diag_gemm_clock()
    per = {n: [] for n in names}
    step_ms = []
    for evs in all_evs:
        for j, n in enumerate(names):
            per[n].append(evs[j].elapsed_time(evs[j + 1]))
        step_ms.append(evs[0].elapsed_time(evs[7]))
    ms = statistics.mean(step_ms)
    layer_ms = ms - statistics.mean(per["route_topk"])      # dispatch + GEMM + combine
    ms, layer_ms = max_over_ranks([ms, layer_ms], dev)

    # end to end through the C ABI with HOST buffers: each call copies that
    # step's logits and x from pinned host memory, runs the layer and copies
    # out back.  Two steps are in flight on two streams with their own
    # device buffers, so one step's host copies overlap the other's kernels
    # (the copy engines and the SMs work at the same time); the time is the
    # whole run of K steps, every copy included.
    h_logits = inp["logits"].pin_memory()
    h_x = inp["x"].pin_memory()
    sets = [(buf, logits, x), (moe.LayerBuffers(wl, dev), torch.empty_like(logits),
                               torch.empty_like(x))]
    h_outs = [torch.empty(buf.out.shape, dtype=buf.out.dtype).pin_memory() for _ in sets]
    e2e_streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]

    def e2e_run(n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for st in e2e_streams:
            st.wait_stream(stream)
        for i in range(n):
            bset, lg, xx = sets[i % 2]
            st = e2e_streams[i % 2]
            if _needs_flush(wl):
                with torch.cuda.stream(st):
                    flush.fill_(1)
            moe.moe_layer_forward_host(wl, h_logits, h_x, h_outs[i % 2], lg, xx, w13, w2, bset,
                                       stream=st)
        for st in e2e_streams:
            stream.wait_stream(st)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    e2e_run(args.warmup)
    e2e = e2e_run(args.steps) / args.steps
    (e2e,) = max_over_ranks([e2e], dev)
    for bset, _, _ in sets:
        st = moe.moe_check_status(bset.dev_status)
        if st != 0:
            raise RuntimeError(f"device status after the host-buffer steps: {moe.STATUS.get(st, st)}")
    del sets[1]
    # the permute alone (moe_permute: the send buffer only, as a standalone
    # call), L2 flushed before each launch
    perm_alone_us = _permute_alone_us(wl, x, buf, 10)
    # the whole layer captured once in a CUDA graph and replayed: median
    # device time per replay (launch overhead of the separate calls removed)
    graph_us, replays = _graph_replay_us(wl, logits, x, w13, w2, buf, 100 if wl.T <= 1024 else 20)
    (graph_us,) = max_over_ranks([graph_us], dev)
    st = moe.moe_check_status(buf.dev_status)
    if st != 0:
        raise RuntimeError(f"device status after timing: {moe.STATUS.get(st, st)}")

    if rank == 0:
        peaks = _peaks()
        # rows the experts computed: all T*k, or the kept ones under a capacity
        dropped = int(buf.n_dropped.cpu()[0]) if buf.capacity >= 0 else 0
        rows = wl.N - dropped
        kb = traffic.kernel_bytes(wl, rows)
        fl = traffic.gemm_flops(wl, rows)
        avg = {n: statistics.mean(v) for n, v in per.items()}
        gemm_ms = avg["dequant_e4m3"] + avg["gemm_gate_up"] + avg["gemm_down"]
        counts = buf.expert_counts.cpu()
        touched = int((counts > 0).sum())
        tf = lambda flops, ms: flops / (ms * 1e-3) / 1e12
        gbs = lambda b, ms: b / (ms * 1e-3) / 1e9 if b and ms > 0 else None
        kernels = {
            "route_topk": {"us": avg["route_topk"] * 1e3,
                           "gbs": gbs(kb["route_topk"], avg["route_topk"])},
            "dispatch_layout": {"us": avg["dispatch_layout"] * 1e3},
            "permute": {"us": avg["permute"] * 1e3, "bytes": kb["permute_layer"],
                        "gbs": gbs(kb["permute_layer"], avg["permute"]),
                        "note": ("fused gather: one bf16 round trip per token (FP8 payload), "
                                 "no permuted copy" if wl.fused_gather else
                                 "inside the layer call an FP8 permute also writes the GEMM's "
                                 "bf16 rows" if wl.payload == "e4m3" else "send buffer only")},
            "permute_standalone": {"us": perm_alone_us, "bytes": kb["permute"],
                                   "gbs": gbs(kb["permute"], perm_alone_us * 1e-3),
                                   "l2": "flushed before each launch"},
            "grouped_gemm": {"us": gemm_ms * 1e3, "flops": fl["total"],
                             "tflops": tf(fl["total"], gemm_ms),
                             "dequant_e4m3_us": avg["dequant_e4m3"] * 1e3,
                             "gate_up_us": avg["gemm_gate_up"] * 1e3,
                             "gate_up_tflops": tf(fl["gate_up"], avg["gemm_gate_up"]),
                             "down_us": avg["gemm_down"] * 1e3,
                             "down_tflops": tf(fl["down"], avg["gemm_down"]),
                             "weight_gbs": gbs(traffic.touched_weight_bytes(wl, touched), gemm_ms),
                             "experts_touched": touched},
            "combine": {"us": avg["combine"] * 1e3, "bytes": kb["combine"],
                        "gbs": gbs(kb["combine"], avg["combine"])},
        }
        for n in ["permute", "permute_standalone", "combine", "route_topk"]:
            g = kernels[n]["gbs"]
            kernels[n]["hbm_frac"] = g / peaks["hbm_gbs"] if g is not None else None
        # The dominant kernel is the gate/up grouped GEMM (SwiGLU fused).  A
        # step is a few ms and the timed region well under a second, so the
        # burst bf16 peak is the denominator; the sustained figure (for
        # kernels timed inside seconds-long runs) is kept beside it.
        achieved = tf(fl["gate_up"], avg["gemm_gate_up"])
        roof = {"kernel": "grouped GEMM, gate/up + SwiGLU phase", "bound": "tensor",
                "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "traffic": _profile_traffic(wl), "algorithmic_flops_per_launch": fl["gate_up"],
                "launch_us": avg["gemm_gate_up"] * 1e3,
                "peak_source": peaks["source"] + " bf16 burst"}
        # The SM clock the GEMM phases ran at, read inside the kernel (CTA 0's
        # clock64 cycles over its globaltimer nanoseconds, over the timed
        # launches), and the tensor rate at that clock: 8192 dense bf16
        # flop per cycle per SM (148 SMs at 1.855 GHz give the nominal
        # 2.25 PFLOP/s).  A nominal per-clock figure, reported beside the
        # measured-peak fractions, not instead of them.
        n_sms = torch.cuda.get_device_properties(dev).multi_processor_count

        def at_kernel_clock(entry, phase):
            cycles, ns = gemm_clock[phase]
            if not ns:
                return entry
            mhz = cycles / ns * 1e3
            peak_clk = n_sms * 8192 * mhz * 1e6 / 1e12
            entry.update({"sm_mhz_in_kernel": mhz, "peak_at_kernel_clock": peak_clk,
                          "frac_at_kernel_clock": entry["achieved"] / peak_clk,
                          "peak_at_kernel_clock_is": "nominal 8192 bf16 flop/cycle/SM x the "
                                                     "clock measured inside the kernel"})
            return entry

        at_kernel_clock(roof, "gate_up")
        # every other kernel against its own bound (same CUDA-event spans)
        gb_w = traffic.gemm_phase_bytes(wl, rows, touched)
        s8 = traffic.section8_bytes(wl, rows)
        hbm = peaks["hbm_gbs"]

        def hbm_entry(name, nbytes, us, what):
            g = gbs(nbytes, us * 1e-3)
            return {"kernel": name, "bound": "hbm", "achieved": g, "peak": hbm, "unit": "GB/s",
                    "frac": g / hbm if g else None, "bytes": nbytes, "launch_us": us,
                    "bytes_are": what}

        others = [
            at_kernel_clock({
                "kernel": "grouped GEMM, down phase", "bound": "tensor",
                "achieved": tf(fl["down"], avg["gemm_down"]), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": tf(fl["down"], avg["gemm_down"]) / peaks["bf16_tflops"],
                "launch_us": avg["gemm_down"] * 1e3, "algorithmic_flops_per_launch": fl["down"],
                "dram_bytes": gb_w["down"], "dram_gbs": gbs(gb_w["down"], avg["gemm_down"]),
                "dram_frac": (gbs(gb_w["down"], avg["gemm_down"]) or 0) / hbm}, "down"),
            {"kernel": "grouped GEMM, gate/up + SwiGLU phase (DRAM view)", "bound": "hbm",
             "achieved": gbs(gb_w["gate_up"], avg["gemm_gate_up"]), "peak": hbm, "unit": "GB/s",
             "frac": (gbs(gb_w["gate_up"], avg["gemm_gate_up"]) or 0) / hbm,
             "bytes": gb_w["gate_up"], "launch_us": avg["gemm_gate_up"] * 1e3},
            {"kernel": "grouped GEMM, both phases", "bound": "tensor",
             "achieved": tf(fl["total"], gemm_ms), "peak": peaks["bf16_tflops"],
             "unit": "TFLOP/s", "frac": tf(fl["total"], gemm_ms) / peaks["bf16_tflops"],
             "launch_us": gemm_ms * 1e3},
            hbm_entry("permute (in the layer call)", kb["permute_layer"], avg["permute"] * 1e3,
                      "bytes it moves"),
            hbm_entry("permute (in the layer call)", s8["permute"], avg["permute"] * 1e3,
                      "the send buffer's algorithmic bytes"),
            hbm_entry("permute (standalone moe_permute)", kb["permute"], perm_alone_us,
                      "the send buffer's algorithmic bytes"),
            hbm_entry("combine", kb["combine"], avg["combine"] * 1e3, "bytes it moves"),
            hbm_entry("combine", s8["combine"], avg["combine"] * 1e3,
                      "algorithmic bytes with a bf16 (or the FP8) y"),
        ]
        line = {
            "metric": METRIC, "value": whole_job_rate(wl.T, ws, ms), "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": dict(_config(wl), **_capacity_info(buf, dropped)),
            "layer_tokens_per_s": whole_job_rate(wl.T, ws, layer_ms),
            "layer_ms_excl_route": layer_ms,
            "kernels": kernels, "roofline": roof, "roofline_other": others,
            "e2e": {"value": whole_job_rate(wl.T, ws, e2e), "unit": "tokens/s",
                    "h2d_bytes_per_step": h_logits.numel() * 4 + h_x.numel() * h_x.element_size(),
                    "d2h_bytes_per_step": h_outs[0].numel() * h_outs[0].element_size(),
                    "ms_per_step": e2e, "steps_in_flight": 2},
            "graph": {"us_median_per_layer": graph_us, "replays": replays,
                      "tokens_per_s": whole_job_rate(wl.T, ws, graph_us * 1e-3)},
            "gpu_launches": int(launches),
            "gpu_launches_per_step": int(launches) // max(args.steps, 1),
            "clocks": clk.summary(ms),
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample(wl)
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_ep(args, wl):
    """Expert parallelism (``--ep``).  Under torchrun with N GPUs: N ranks,
    each with its own T tokens and E/N experts, rows moved to their owners
    through peer buffers mapped with CUDA IPC (DistributedEP); weak
    scaling.  On one GPU: ``--ep-ranks`` W ranks emulated on the device, each
    with T/W tokens (EmulatedEP), the same total batch as the plain step.
    A step is one layer on every rank; the time is the max over ranks."""
    from expert_parallelism_b200 import ep
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    moe.load_library()
    stream = torch.cuda.current_stream()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        W, Er = ws, wl.E // ws
        wl_r = wl.replace(W=W, seed=wl.seed + 100 + rank)
        w13 = torch.empty(Er, 2 * wl.I, wl.H, dtype=torch.bfloat16, device=dev)
        w2 = torch.empty(Er, wl.H, wl.I, dtype=torch.bfloat16, device=dev)
        workloads.fill_expert_weights(wl, w13, w2, experts=range(rank * Er, (rank + 1) * Er))
        logits = workloads.router_logits(wl_r).to(dev)
        x = workloads.hidden_states(wl_r).to(dev)
        runner = ep.DistributedEP(wl.replace(W=W), device=dev)
        step = lambda: runner.forward(logits, x, w13, w2)
        tokens = wl.T
        status = lambda: [moe.moe_check_status(runner.state.dev_status)]
    else:
        W = args.ep_ranks
        wl_r = wl.replace(T=wl.T // W, W=W)
        w13 = torch.empty(wl.E, 2 * wl.I, wl.H, dtype=torch.bfloat16, device=dev)
        w2 = torch.empty(wl.E, wl.H, wl.I, dtype=torch.bfloat16, device=dev)
        workloads.fill_expert_weights(wl, w13, w2)
        lg = [workloads.router_logits(wl_r.replace(seed=wl.seed + 100 + r)).to(dev)
              for r in range(W)]
        xs = [workloads.hidden_states(wl_r.replace(seed=wl.seed + 100 + r)).to(dev)
              for r in range(W)]
        runner = ep.EmulatedEP(wl_r, W, dev)
        step = lambda: runner.forward(lg, xs, w13, w2)
        tokens = wl_r.T * W
        status = runner.status
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if any(st != 0 for st in status()):
        raise RuntimeError(f"device status after warm-up: {status()}")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = moe.load_library().moe_launch_count()
    with ClockSampler(dev) as clk:
        for a, b in evs:
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
    launches = moe.load_library().moe_launch_count() - launches0
    if ws > 1:
        torch.distributed.barrier()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    (ms,) = max_over_ranks([ms], dev)
    if rank == 0:
        line = {"metric": METRIC, "value": whole_job_rate(tokens, ws, ms), "unit": "tokens/s",
                "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": dict(_config(wl_r), parallelism=(
                    f"expert parallel over {W} GPUs (peer-mapped buffers)" if ws > 1 else
                    f"expert parallel, {W} ranks emulated on one GPU"),
                    tokens_per_rank=wl_r.T),
                "gpu_launches": int(launches), "clocks": clk.summary(ms)}
        print(json.dumps(line), flush=True)
    if ws > 1:
        runner.close()
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def _permute_alone_us(wl, x, buf, iters):
    """Mean device time of moe_permute on the step's routing (its send
    buffer, payload dtype of the workload), with a 512 MiB write before each
    launch so x starts outside L2."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=x.device)
    ts = []
    for i in range(iters + 2):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        moe.moe_permute(x, wl.k, buf.slot_of_pair, buf.xp, buf.xp_scales)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            ts.append(e0.elapsed_time(e1) * 1e3)
    del flush
    return statistics.mean(ts)


def _graph_replay_us(wl, logits, x, w13, w2, buf, replays):
    """Capture moe_layer_forward in one CUDA graph on a side stream, replay
    it ``replays`` times with events around each replay; median in us."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        moe.moe_layer_forward(wl, logits, x, w13, w2, buf, stream=s)
        s.synchronize()
        with torch.cuda.graph(graph, stream=s):
            moe.moe_layer_forward(wl, logits, x, w13, w2, buf, stream=s)
        for _ in range(3):
            graph.replay()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(replays)]
        for a, b in evs:
            a.record(s)
            graph.replay()
            b.record(s)
        s.synchronize()
    times = [a.elapsed_time(b) * 1e3 for a, b in evs]
    del graph
    return statistics.median(times), replays


def _profile_traffic(wl):
    """DRAM bytes per launch of the gate/up GEMM kernel on this workload, from
    the committed ncu summary -- None unless that summary was taken on the
    same kernel source file (named in it, checked by hash) and for this
    workload."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "expert_parallelism_b200", "csrc", rec.get("source", "?"))
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if rec.get("source_sha256") != digest:
            return None
        return rec.get("gate_up_dram_bytes_per_launch", {}).get(wl.name)
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsv3", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=12.0,
                    help="reference arm: at most this many seconds of oracle work per step")
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="reference arm: about this many seconds for all warm-up and timed steps")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (smaller cases of the same kernels, for profiling)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (must stay a multiple of the logical ranks)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism: one rank per GPU under torchrun, or --ep-ranks "
                         "ranks emulated on one GPU")
    ap.add_argument("--ep-ranks", type=int, default=8)
    args = ap.parse_args()
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens is not None or args.experts is not None:
        wl = wl.replace(T=args.tokens or wl.T, E=args.experts or wl.E,
                        name=f"{wl.name}[T={args.tokens or wl.T},E={args.experts or wl.E}]")
    if args.impl == "reference":
        run_reference(args, wl)
    elif args.ep:
        run_ep(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
