"""Expert parallelism over W ranks: each rank holds its own tokens and the
weights of E/W experts, and the routed rows travel to their experts' owners
and back.

Source: "Expert Parallelism" (aiwiki), "The two all-to-alls" (dispatch
sends each token's row to the ranks owning its experts, combine returns
the outputs), "Implementation" (a count exchange first tells each owner how
many rows arrive) and "Hiding the latency"; "Expert parallelism and
all-to-all", "Walking through one MoE layer", steps 1-4; ownership from
"Expert parallelism" (Transformers docs), "How the sizes combine".

Per rank and layer: moe_route_topk and moe_dispatch_layout on its own
tokens; the count exchange (every rank's expert_counts into counts_all
[W, E]); moe_ep_plan; moe_ep_dispatch (each routed row stored into its
owner's receive buffer); a barrier; moe_grouped_gemm on the local receive
buffer; a barrier; moe_ep_combine (each pick's output row loaded from its
owner and weighted into the token's home row).  Every step is a libmoe
kernel; this module only allocates buffers and orders the calls.

Two ways to run the W ranks:
  - ``EmulatedEP``: all W ranks on one GPU, each with its own buffers.
    The kernels of different ranks never wait for one another (stream
    order is the only synchronisation), so this is an exact stand-in for
    the data flow, not for its timing.
  - ``DistributedEP``: one process per GPU of an NVLink domain.  Each
    rank maps the other ranks' receive and output buffers through CUDA IPC
    records; the dispatch stores to them and the combine loads from them
    (peer memory over NVLink); the count exchange is an all-gather; the
    barriers are stream-ordered collectives.  No TMA or cluster multicast
    reads another GPU's memory.
"""
from __future__ import annotations

import torch

from . import moe
from .workloads import TORCH_DTYPE


def recv_capacity_rows(wl, world: int) -> int:
    """Rows a receive buffer may need: every token of every rank can send at
    most min(k, E/W) of its picks to one owner."""
    return world * wl.T * min(wl.k, wl.E // world)


class RankState:
    """One rank's buffers for the expert-parallel layer (its own layout, its
    plan, its receive buffer and its experts' outputs)."""

    def __init__(self, wl, world: int, device, rows_capacity: int, alloc=None):
        T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        alloc = alloc or (lambda shape, dtype: torch.empty(shape, dtype=dtype, device=dev))
        self.wl, self.world, self.cap = wl, world, rows_capacity
        self.topk_idx = torch.empty(T, k, **i32)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.rank_offsets = torch.empty(world + 1, **i32)
        self.slot_of_pair = torch.empty(max(T * k, 1), **i32)
        self.pair_of_slot = torch.empty(max(T * k, 1), **i32)
        self.layout_ws = torch.empty(max(moe.moe_dispatch_layout_workspace_bytes(T, k, E), 16),
                                     dtype=torch.uint8, device=dev)
        self.counts_all = torch.empty(world, E, **i32)
        self.send_base = torch.empty(E, **i32)
        self.recv_offsets = torch.empty(E // world + 1, **i32)
        self.dev_status = torch.zeros(1, **i32)
        pdt = TORCH_DTYPE[wl.payload]
        cap = max(rows_capacity, 1)
        # the buffers other ranks store to (payload) and load from (y)
        self.recv = alloc((cap, H), pdt)
        self.recv_scales = alloc((cap, H // 128), torch.float32) if wl.payload == "e4m3" else None
        self.y = alloc((cap, H), TORCH_DTYPE[wl.ydt])
        self.y_scales = alloc((cap, H // 128), torch.float32) if wl.ydt == "e4m3" else None
        self.h = torch.empty(cap, I, dtype=TORCH_DTYPE[wl.wdt], device=dev)
        gb = moe.moe_grouped_gemm_workspace_bytes(cap, H, I, pdt, TORCH_DTYPE[wl.wdt])
        self.gemm_ws = torch.empty(gb, dtype=torch.uint8, device=dev) if gb else None
        self.out = torch.empty(T, H, dtype=TORCH_DTYPE[wl.act], device=dev)

    # ------------------------------------------------------------ the steps
    def route_and_layout(self, logits, stream=None):
        wl = self.wl
        moe.moe_route_topk(logits, self.topk_idx, self.topk_w, stream=stream)
        moe.moe_dispatch_layout(self.topk_idx, wl.E, self.world, self.expert_counts,
                                self.expert_offsets, self.rank_offsets, self.slot_of_pair,
                                self.pair_of_slot, self.layout_ws, self.dev_status, stream=stream)

    def plan(self, rank, stream=None):
        moe.moe_ep_plan(self.counts_all, rank, self.send_base, self.recv_offsets, self.dev_status,
                        stream=stream)

    def dispatch(self, x, recv_rows, recv_scales, stream=None):
        moe.moe_ep_dispatch(x, self.wl.k, self.topk_idx, self.slot_of_pair, self.expert_offsets,
                            self.send_base, recv_rows, recv_scales, TORCH_DTYPE[self.wl.payload],
                            self.cap, self.dev_status, stream=stream)

    def experts(self, w13_local, w2_local, stream=None):
        moe.moe_grouped_gemm(self.recv, self.recv_scales, self.recv_offsets, 0,
                             self.wl.E // self.world, w13_local, w2_local, self.h, self.y,
                             self.gemm_ws, self.dev_status, stream=stream,
                             y_scales=self.y_scales)

    def combine(self, y_rows, y_scales, stream=None):
        moe.moe_ep_combine(y_rows, y_scales, TORCH_DTYPE[self.wl.ydt], self.topk_idx,
                           self.slot_of_pair, self.expert_offsets, self.send_base, self.topk_w,
                           self.cap, self.out, self.dev_status, stream=stream)


class EmulatedEP:
    """W expert-parallel ranks run on one GPU: rank r's tokens are its own
    inputs, rank r's experts the weight rows [r*E/W, (r+1)*E/W).  The count
    exchange is a copy of the W count vectors; the barriers are stream
    order."""

    def __init__(self, wl, world: int, device="cuda"):
        self.wl, self.world = wl, world
        self.cap = recv_capacity_rows(wl, world)
        self.ranks = [RankState(wl, world, device, self.cap) for _ in range(world)]

    def forward(self, logits_per_rank, x_per_rank, w13, w2, stream=None):
        W, Er = self.world, self.wl.E // self.world
        R = self.ranks
        for r in range(W):
            R[r].route_and_layout(logits_per_rank[r], stream=stream)
        # the count exchange (every rank gets every rank's counts)
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            counts = torch.stack([R[r].expert_counts for r in range(W)])
            for r in range(W):
                R[r].counts_all.copy_(counts)
        for r in range(W):
            R[r].plan(r, stream=stream)
        recv = [R[r].recv for r in range(W)]
        recv_sc = [R[r].recv_scales for r in range(W)] if self.wl.payload == "e4m3" else None
        for r in range(W):
            R[r].dispatch(x_per_rank[r], recv, recv_sc, stream=stream)
        for r in range(W):
            R[r].experts(w13[r * Er:(r + 1) * Er], w2[r * Er:(r + 1) * Er], stream=stream)
        ys = [R[r].y for r in range(W)]
        ysc = [R[r].y_scales for r in range(W)] if self.wl.ydt == "e4m3" else None
        for r in range(W):
            R[r].combine(ys, ysc, stream=stream)
        return [R[r].out for r in range(W)]

    def status(self):
        """Device status of every rank (synchronises)."""
        return [moe.moe_check_status(R.dev_status) for R in self.ranks]


def exchange_counts(expert_counts: torch.Tensor, counts_all: torch.Tensor, group=None):
    """The count exchange: counts_all[s] = rank s's expert_counts on every
    rank (an all-gather: NCCL on GPU tensors; a gloo group takes the counts
    through host memory)."""
    import torch.distributed as dist
    if expert_counts.is_cuda and dist.get_backend(group) != "nccl":
        host = torch.empty(counts_all.shape, dtype=counts_all.dtype)
        dist.all_gather(list(host.unbind(0)), expert_counts.cpu(), group=group)
        counts_all.copy_(host)
        return counts_all
    dist.all_gather(list(counts_all.unbind(0)), expert_counts.contiguous(), group=group)
    return counts_all


class DistributedEP:
    """One expert-parallel rank per process.  Every rank exports its receive
    and output buffers as CUDA IPC records (moe_ipc_export), gathers the
    others' records, and maps them (moe_ipc_import): the tables that the
    dispatch stores through and the combine loads through then hold the
    peers' buffers (peer memory over NVLink between GPUs).  No multicast
    object is created and no TMA load reads a peer's memory.

    Barriers: with NCCL, a one-element all-reduce on the compute stream
    (ordered after this rank's kernels and before its next ones); with gloo
    (several processes sharing one GPU, as in the tests), the device is
    synchronised and the host group meets."""

    def __init__(self, wl, group=None, device=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group or dist.group.WORLD
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        self.nccl = dist.get_backend(self.group) == "nccl"
        self.wl = wl
        dev = device or torch.device("cuda", torch.cuda.current_device())
        self.cap = recv_capacity_rows(wl, self.world)
        self.state = RankState(wl, self.world, dev, self.cap)
        self._tick = torch.zeros(1, dtype=torch.int32, device=dev)
        self.imported = []
        S = self.state
        self.recv_rows = self._share(S.recv)
        self.recv_scales = self._share(S.recv_scales)
        self.y_rows = self._share(S.y)
        self.y_scales = self._share(S.y_scales)

    def _share(self, t):
        """Every rank's address of the buffer ``t`` of each rank (its own
        pointer at its own index)."""
        if t is None:
            return None
        rec = moe.moe_ipc_export(t)
        recs = [None] * self.world
        self.dist.all_gather_object(recs, rec, group=self.group)
        ptrs = []
        for r, other in enumerate(recs):
            if r == self.rank:
                ptrs.append(t.data_ptr())
            else:
                p = moe.moe_ipc_import(other)
                self.imported.append((other, p))
                ptrs.append(p)
        return ptrs

    def barrier(self):
        if self.nccl:
            self.dist.all_reduce(self._tick, group=self.group)
        else:
            torch.cuda.synchronize()
            self.dist.barrier(group=self.group)

    def forward(self, logits, x, w13_local, w2_local, stream=None):
        """One layer on this rank.  With ``stream`` given, the kernels and the
        collectives (count exchange, barriers) are all ordered on it."""
        if stream is not None:
            with torch.cuda.stream(stream):
                return self.forward(logits, x, w13_local, w2_local)
        S = self.state
        S.route_and_layout(logits)
        exchange_counts(S.expert_counts, S.counts_all, self.group)
        S.plan(self.rank)
        S.dispatch(x, self.recv_rows, self.recv_scales)
        self.barrier()                       # every rank's rows have landed
        S.experts(w13_local, w2_local)
        self.barrier()                       # every owner's y is written
        S.combine(self.y_rows, self.y_scales)
        self.barrier()                       # nobody reads this rank's y any more
        return S.out

    def close(self):
        """Unmaps the peers' buffers (every rank, after its last forward)."""
        torch.cuda.synchronize()
        for rec, p in self.imported:
            moe.moe_ipc_close(rec, p)
        self.imported = []
