"""Python binding of libmoe's C ABI (include/moe.h): argument marshalling only.

Each ``moe_*`` function mirrors the C entry point of the same name: it
takes CUDA torch tensors (PyTorch supplies device memory and the current
stream), passes their raw pointers and sizes through ctypes, and raises
``MoEError`` for any status other than MOE_OK.  All computation happens in
the library's CUDA kernels; there is no Python or CPU fallback, and
loading fails loudly when ``libmoe.so`` has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
MOE_DEV_BAD_INDEX, MOE_DEV_TIMEOUT, MOE_DEV_OVERFLOW = 0x1, 0x2, 0x4
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_BAD_INDEX",
          4: "MOE_ERR_TIMEOUT", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_OVERFLOW"}
_DT = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16, torch.float8_e4m3fn: MOE_E4M3}

# exported symbols and their ctypes signatures (P = pointer, I64/I32 = ints)
_P, _I64, _I32, _SZ, _I = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t,
                           ctypes.c_int)
SIGNATURES = {
    "moe_route_topk": ([_P, _I64, _I32, _I32, _P, _P, _P], _I),
    "moe_route_topk_grouped": ([_P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P], _I),
    "moe_dispatch_layout_workspace_bytes": ([_I64, _I32, _I32], _SZ),
    "moe_dispatch_layout": ([_P, _I64, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P, _P], _I),
    "moe_dispatch_layout_capacity": ([_P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P,
                                      _P, _SZ, _P, _P], _I),
    "moe_dispatch_layout_noalloc_max_scratch_bytes": ([], _SZ),
    "moe_dispatch_layout_noalloc": ([_P, _I64, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _P], _I),
    "moe_permute": ([_P, _I, _I64, _I32, _I32, _P, _P, _I, _P, _P], _I),
    "moe_grouped_gemm_workspace_bytes": ([_I64, _I32, _I32, _I, _I], _SZ),
    "moe_grouped_gemm": ([_P, _I, _P, _P, _P, _I32, _I32, _I64, _I32, _I32, _P, _P, _I, _P, _P,
                          _I, _P, _P, _SZ, _P, _P], _I),
    "moe_packed_weights_bytes": ([_I32, _I32, _I32, _I32], _SZ),
    "moe_pack_expert_weights": ([_P, _P, _I32, _I32, _I32, _I, _P, _P, _P], _I),
    "moe_grouped_gemm_packed": ([_P, _I, _P, _P, _P, _I32, _I32, _I64, _I32, _I32, _P, _P, _I, _P,
                                 _P, _I, _P, _P, _SZ, _P, _P], _I),
    "moe_combine": ([_P, _I, _P, _P, _P, _I64, _I32, _I32, _P, _I, _P], _I),
    "moe_combine_rank": ([_P, _I, _P, _P, _P, _I64, _I32, _I32, _P, _I32, _I32, _P, _P], _I),
    "moe_reduce_partials": ([_P, _I32, _I64, _I32, _P, _I, _P], _I),
    "moe_layer_forward": ([_P, _P, _I, _I64, _I32, _I32, _I32, _I32, _I32, _P, _P, _I, _I, _I,
                           _P, _P, _P, _P, _P], _I),
    "moe_layer_forward_host": ([_P, _P, _P, _P, _P, _P, _I, _I64, _I32, _I32, _I32, _I32, _I32,
                                _P, _P, _I, _I, _I, _P, _P, _P, _P], _I),
    "moe_check_status": ([_P, _P], _I),
    "moe_status_str": ([_I], ctypes.c_char_p),
    "moe_launch_count": ([], ctypes.c_uint64),
    "moe_ep_plan": ([_P, _I32, _I32, _I32, _P, _P, _P, _P], _I),
    "moe_ep_dispatch": ([_P, _I, _I64, _I32, _I32, _P, _P, _P, _P, _I32, _I32, _P, _P, _I, _I64,
                         _P, _P], _I),
    "moe_ep_combine": ([_P, _P, _I, _P, _P, _P, _P, _P, _I64, _I32, _I32, _I32, _I32, _I64, _P,
                        _I, _P, _P], _I),
    "moe_ipc_handle_bytes": ([], _SZ),
    "moe_ipc_export": ([_P, _P], _I),
    "moe_ipc_import": ([_P, ctypes.POINTER(ctypes.c_void_p)], _I),
    "moe_ipc_close": ([_P, _P], _I),
    "moe_diag_layout_wait_timeout_workspace_bytes": ([], _SZ),
    "moe_diag_layout_wait_timeout": ([_P, _SZ, ctypes.c_uint64, _P, _P], _I),
    "moe_diag_gemm_clock": ([_P, ctypes.c_int32], _I),
}


class LayerOptionsC(ctypes.Structure):
    """moe_layer_options (include/moe.h)."""
    _fields_ = [("capacity", _I32), ("route_groups", _I32), ("route_max_groups", _I32),
                ("fused_gather", _I32), ("all_reduce_form", _I32), ("packed_weights", _I32),
                ("weights_in_gemm", _I32)]


class LayerBuffersC(ctypes.Structure):
    """moe_layer_buffers (include/moe.h)."""
    _fields_ = [("topk_idx", _P), ("topk_w", _P), ("expert_counts", _P),
                ("expert_offsets", _P), ("rank_offsets", _P), ("slot_of_pair", _P),
                ("pair_of_slot", _P), ("layout_workspace", _P),
                ("layout_workspace_bytes", _SZ), ("xp", _P), ("xp_scales", _P), ("h", _P),
                ("y", _P), ("y_scales", _P), ("gemm_workspace", _P), ("gemm_workspace_bytes", _SZ),
                ("dev_status", _P), ("n_dropped", _P), ("partials", _P)]


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, code)}")
        self.code = code
        self.status = STATUS.get(code, str(code))


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe.so once; raises if it is missing (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"libmoe.so not built at {path}: run "
                              "`python -m expert_parallelism_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes, fn.restype = args, res
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(name, rc):
    if rc != 0:
        raise MoEError(name, rc)


def dtype_code(t: torch.Tensor) -> int:
    return _DT[t.dtype]


# ----------------------------------------------------------------- the C ABI
def moe_route_topk(logits, topk_idx, topk_w, stream=None):
    T, E = logits.shape
    k = topk_idx.shape[1]
    _check("moe_route_topk", load_library().moe_route_topk(
        _ptr(logits), T, E, k, _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_route_topk_grouped(logits, groups, max_groups, topk_idx, topk_w, stream=None):
    T, E = logits.shape
    k = topk_idx.shape[1]
    _check("moe_route_topk_grouped", load_library().moe_route_topk_grouped(
        _ptr(logits), T, E, k, groups, max_groups, _ptr(topk_idx), _ptr(topk_w),
        _stream(stream)))


def moe_dispatch_layout_workspace_bytes(T, k, E) -> int:
    return int(load_library().moe_dispatch_layout_workspace_bytes(T, k, E))


def moe_dispatch_layout(topk_idx, E, W, expert_counts, expert_offsets, rank_offsets,
                        slot_of_pair, pair_of_slot, workspace, dev_status, stream=None):
    T, k = topk_idx.shape
    _check("moe_dispatch_layout", load_library().moe_dispatch_layout(
        _ptr(topk_idx), T, k, E, W, _ptr(expert_counts), _ptr(expert_offsets),
        _ptr(rank_offsets), _ptr(slot_of_pair), _ptr(pair_of_slot), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))


def moe_dispatch_layout_capacity(topk_idx, E, W, capacity, expert_counts, expert_offsets,
                                 rank_offsets, slot_of_pair, pair_of_slot, workspace, dev_status,
                                 n_dropped=None, stream=None):
    T, k = topk_idx.shape
    _check("moe_dispatch_layout_capacity", load_library().moe_dispatch_layout_capacity(
        _ptr(topk_idx), T, k, E, W, capacity, _ptr(expert_counts), _ptr(expert_offsets),
        _ptr(rank_offsets), _ptr(slot_of_pair), _ptr(pair_of_slot), _ptr(n_dropped),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
        _stream(stream)))


def moe_dispatch_layout_noalloc(topk_idx, E, W, expert_counts, expert_offsets, rank_offsets,
                                slot_of_pair, pair_of_slot, dev_status, stream=None):
    """moe_dispatch_layout without a workspace (scratch inside the library)."""
    T, k = topk_idx.shape
    _check("moe_dispatch_layout_noalloc", load_library().moe_dispatch_layout_noalloc(
        _ptr(topk_idx), T, k, E, W, _ptr(expert_counts), _ptr(expert_offsets),
        _ptr(rank_offsets), _ptr(slot_of_pair), _ptr(pair_of_slot), _ptr(dev_status),
        _stream(stream)))


def moe_permute(x, k, slot_of_pair, xp, xp_scales=None, stream=None):
    T, H = x.shape
    _check("moe_permute", load_library().moe_permute(
        _ptr(x), dtype_code(x), T, H, k, _ptr(slot_of_pair), _ptr(xp), dtype_code(xp),
        _ptr(xp_scales), _stream(stream)))


def moe_grouped_gemm_workspace_bytes(n_rows, H, I, xp_dtype, w_dtype) -> int:
    return int(load_library().moe_grouped_gemm_workspace_bytes(n_rows, H, I, _DT[xp_dtype],
                                                                _DT[w_dtype]))


def moe_grouped_gemm(xp, xp_scales, expert_offsets, expert_begin, n_experts, w13, w2, h, y,
                     workspace, dev_status, stream=None, expert_counts=None, y_scales=None):
    n_rows, H = xp.shape
    I = w2.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_grouped_gemm", load_library().moe_grouped_gemm(
        _ptr(xp), dtype_code(xp), _ptr(xp_scales), _ptr(expert_offsets), _ptr(expert_counts),
        expert_begin,
        n_experts, n_rows, H, I, _ptr(w13), _ptr(w2), dtype_code(w13), _ptr(h), _ptr(y),
        dtype_code(y), _ptr(y_scales), _ptr(workspace), ws_bytes, _ptr(dev_status),
        _stream(stream)))


def packed_weight_tensors(E, H, I, device):
    """Empty uint8 buffers for the packed W13 and W2 of E experts."""
    lib = load_library()
    return (torch.empty(lib.moe_packed_weights_bytes(E, H, I, 0), dtype=torch.uint8,
                        device=device),
            torch.empty(lib.moe_packed_weights_bytes(E, H, I, 1), dtype=torch.uint8,
                        device=device))


def moe_pack_expert_weights(w13, w2, packed13, packed2, stream=None):
    """Re-lay stacked bf16 weights [E, 2I, H] / [E, H, I] into 16 KB blocks."""
    E, H, I = w2.shape
    _check("moe_pack_expert_weights", load_library().moe_pack_expert_weights(
        _ptr(w13), _ptr(w2), E, H, I, dtype_code(w2), _ptr(packed13), _ptr(packed2),
        _stream(stream)))


def moe_grouped_gemm_packed(xp, xp_scales, expert_offsets, expert_begin, n_experts, packed13,
                            packed2, H, I, h, y, workspace, dev_status, stream=None,
                            expert_counts=None, y_scales=None):
    n_rows = xp.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_grouped_gemm_packed", load_library().moe_grouped_gemm_packed(
        _ptr(xp), dtype_code(xp), _ptr(xp_scales), _ptr(expert_offsets), _ptr(expert_counts),
        expert_begin, n_experts, n_rows, H, I, _ptr(packed13), _ptr(packed2), MOE_BF16,
        _ptr(h), _ptr(y), dtype_code(y), _ptr(y_scales), _ptr(workspace), ws_bytes,
        _ptr(dev_status), _stream(stream)))


def moe_combine(y, slot_of_pair, topk_w, out, stream=None, y_scales=None):
    T, k = topk_w.shape
    H = y.shape[1]
    _check("moe_combine", load_library().moe_combine(
        _ptr(y), dtype_code(y), _ptr(y_scales), _ptr(slot_of_pair), _ptr(topk_w), T, k, H,
        _ptr(out), dtype_code(out), _stream(stream)))


def moe_combine_rank(y, slot_of_pair, topk_w, rank_offsets, rank, partial, stream=None,
                     y_scales=None):
    """Rank ``rank``'s fp32 partial of the all_reduce form (its own slab of
    slots only); ``rank_offsets`` has world + 1 entries."""
    T, k = topk_w.shape
    H = y.shape[1]
    _check("moe_combine_rank", load_library().moe_combine_rank(
        _ptr(y), dtype_code(y), _ptr(y_scales), _ptr(slot_of_pair), _ptr(topk_w), T, k, H,
        _ptr(rank_offsets), rank_offsets.numel() - 1, rank, _ptr(partial), _stream(stream)))


def moe_reduce_partials(partials, out, stream=None):
    """out = the sum of partials [n, T, H] (fp32, rank order), rounded once."""
    n, T, H = partials.shape
    _check("moe_reduce_partials", load_library().moe_reduce_partials(
        _ptr(partials), n, T, H, _ptr(out), dtype_code(out), _stream(stream)))


def moe_check_status(dev_status, stream=None) -> int:
    """Synchronises the stream; returns the raw status code (0 = OK)."""
    return int(load_library().moe_check_status(_ptr(dev_status), _stream(stream)))


def _ptr_array(ptrs):
    """A host array of device pointers (ints or tensors; None -> NULL)."""
    vals = [None if p is None else (p.data_ptr() if isinstance(p, torch.Tensor) else int(p))
            for p in ptrs]
    return (ctypes.c_void_p * len(vals))(*vals)


def moe_ipc_export(t: torch.Tensor) -> bytes:
    """IPC record (handle of the allocation + the tensor's offset) of a
    device tensor, as bytes to send to another process."""
    lib = load_library()
    rec = ctypes.create_string_buffer(lib.moe_ipc_handle_bytes())
    _check("moe_ipc_export", lib.moe_ipc_export(_ptr(t), rec))
    return rec.raw


def moe_ipc_import(record: bytes) -> int:
    """Device address, in this process, of the buffer another process
    exported."""
    lib = load_library()
    out = ctypes.c_void_p()
    _check("moe_ipc_import", lib.moe_ipc_import(ctypes.c_char_p(record), ctypes.byref(out)))
    return int(out.value)


def moe_ipc_close(record: bytes, ptr: int):
    _check("moe_ipc_close", load_library().moe_ipc_close(ctypes.c_char_p(record),
                                                          ctypes.c_void_p(ptr)))


def moe_ep_plan(counts_all, rank, send_base, recv_offsets, dev_status, stream=None):
    """This rank's dispatch plan from every rank's expert counts [W, E]."""
    W, E = counts_all.shape
    _check("moe_ep_plan", load_library().moe_ep_plan(
        _ptr(counts_all), W, E, rank, _ptr(send_base), _ptr(recv_offsets), _ptr(dev_status),
        _stream(stream)))


def moe_ep_dispatch(x, k, topk_idx, slot_of_pair, expert_offsets, send_base, recv_rows,
                    recv_scales, payload_dtype, rows_capacity, dev_status, stream=None):
    """Every routed row of this rank into its owner's receive buffer.
    ``recv_rows``/``recv_scales``: one entry per rank (tensors on this GPU,
    or raw peer-mapped device pointers)."""
    T, H = x.shape
    W = len(recv_rows)
    E = expert_offsets.numel() - 1
    sc = _ptr_array(recv_scales) if recv_scales is not None else None
    _check("moe_ep_dispatch", load_library().moe_ep_dispatch(
        _ptr(x), dtype_code(x), T, H, k, _ptr(topk_idx), _ptr(slot_of_pair),
        _ptr(expert_offsets), _ptr(send_base), E, W, _ptr_array(recv_rows), sc,
        _DT[payload_dtype], rows_capacity, _ptr(dev_status), _stream(stream)))


def moe_ep_combine(y_rows, y_scales, y_dtype, topk_idx, slot_of_pair, expert_offsets, send_base,
                   topk_w, rows_capacity, out, dev_status, stream=None):
    """out[t] = sum_j w[t,j] * (pick j's output row in its owner's y)."""
    T, k = topk_w.shape
    H = out.shape[1]
    W = len(y_rows)
    E = expert_offsets.numel() - 1
    sc = _ptr_array(y_scales) if y_scales is not None else None
    _check("moe_ep_combine", load_library().moe_ep_combine(
        _ptr_array(y_rows), sc, _DT[y_dtype], _ptr(topk_idx), _ptr(slot_of_pair),
        _ptr(expert_offsets), _ptr(send_base), _ptr(topk_w), T, k, H, E, W, rows_capacity,
        _ptr(out), dtype_code(out), _ptr(dev_status), _stream(stream)))


def moe_diag_gemm_clock(reset=False):
    """The grouped GEMM's clock record: {"gate_up": (cycles, ns), "down":
    (cycles, ns)} summed over launches since the last reset (synchronises the
    device); with reset, clears it afterwards."""
    out = (ctypes.c_uint64 * 4)()
    _check("moe_diag_gemm_clock", load_library().moe_diag_gemm_clock(out, 1 if reset else 0))
    return {"gate_up": (int(out[0]), int(out[1])), "down": (int(out[2]), int(out[3]))}


def moe_diag_layout_wait_timeout(workspace, wait_limit_ns, dev_status, stream=None):
    """Runs the layout scan on a flag that nothing sets; its bounded wait
    gives up after ``wait_limit_ns`` and records MOE_DEV_TIMEOUT."""
    _check("moe_diag_layout_wait_timeout", load_library().moe_diag_layout_wait_timeout(
        _ptr(workspace), workspace.numel() * workspace.element_size(), wait_limit_ns,
        _ptr(dev_status), _stream(stream)))


def moe_status_str(code: int) -> str:
    return load_library().moe_status_str(code).decode()


# ----------------------------------------------------------------- buffers
def capacity_rows(wl) -> int:
    """Rows per expert slab for a fixed-capacity workload, ceil(factor * T*k
    / E); -1 for a dropless one."""
    if wl.capacity_factor is None:
        return -1
    return int(math.ceil(wl.capacity_factor * wl.T * wl.k / wl.E))


def slot_rows(wl) -> int:
    """Rows of the permuted buffers: T*k, or E * capacity."""
    c = capacity_rows(wl)
    return wl.T * wl.k if c < 0 else wl.E * c


class LayerBuffers:
    """Device buffers for one layer of a workload (outputs and workspaces).

    Plain torch allocations made once; every step reuses them.
    """

    def __init__(self, wl, device="cuda"):
        from .workloads import TORCH_DTYPE
        T, H, E, k, I, W = wl.T, wl.H, wl.E, wl.k, wl.I, wl.W
        self.capacity = capacity_rows(wl)
        N = slot_rows(wl)                      # rows of the permuted buffers
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.wl = wl
        self.topk_idx = torch.empty(T, k, **i32)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.rank_offsets = torch.empty(W + 1, **i32)
        self.slot_of_pair = torch.empty(max(T * k, 1), **i32)
        self.pair_of_slot = torch.empty(max(N, 1), **i32)
        self.n_dropped = torch.zeros(1, **i32)
        self.layout_ws = torch.empty(max(moe_dispatch_layout_workspace_bytes(T, k, E), 16),
                                     dtype=torch.uint8, device=dev)
        self.dev_status = torch.zeros(1, **i32)
        pdt = TORCH_DTYPE[wl.payload]
        self.xp = torch.empty(N, H, dtype=pdt, device=dev)
        self.xp_scales = (torch.empty(N, H // 128, dtype=torch.float32, device=dev)
                          if wl.payload == "e4m3" else None)
        wdt = TORCH_DTYPE[wl.wdt]
        self.h = torch.empty(N, I, dtype=wdt, device=dev)
        self.y = torch.empty(N, H, dtype=TORCH_DTYPE[wl.ydt], device=dev)
        self.y_scales = (torch.empty(N, H // 128, dtype=torch.float32, device=dev)
                         if wl.ydt == "e4m3" else None)
        gb = moe_grouped_gemm_workspace_bytes(N, H, I, pdt, wdt)
        if wl.fused_gather and wl.payload == "e4m3":
            gb = max(gb, T * H * 2)            # the fused gather's one bf16 row per token
        self.gemm_ws = torch.empty(gb, dtype=torch.uint8, device=dev) if gb else None
        self.out = torch.empty(T, H, dtype=TORCH_DTYPE[wl.act], device=dev)
        self.partials = (torch.empty(W, T, H, dtype=torch.float32, device=dev)
                         if wl.all_reduce_form else None)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def layer_buffers_c(buf: "LayerBuffers") -> LayerBuffersC:
    return LayerBuffersC(
        _ptr(buf.topk_idx), _ptr(buf.topk_w), _ptr(buf.expert_counts), _ptr(buf.expert_offsets),
        _ptr(buf.rank_offsets), _ptr(buf.slot_of_pair), _ptr(buf.pair_of_slot),
        _ptr(buf.layout_ws), _nbytes(buf.layout_ws), _ptr(buf.xp), _ptr(buf.xp_scales),
        _ptr(buf.h), _ptr(buf.y), _ptr(buf.y_scales), _ptr(buf.gemm_ws), _nbytes(buf.gemm_ws),
        _ptr(buf.dev_status),
        _ptr(buf.n_dropped), _ptr(buf.partials))


def _events(step_events, stream=None):
    if step_events is None:
        return None
    s = torch.cuda.current_stream() if stream is None else stream
    for e in step_events:
        if not e.cuda_event:      # torch creates the CUDA event on its first record
            e.record(s)
    assert len(step_events) == 8, "8 events: see moe_layer_forward in include/moe.h"
    arr = (ctypes.c_void_p * 8)(*[ctypes.c_void_p(e.cuda_event) for e in step_events])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def _weight_code(wl) -> int:
    """The weights' dtype code from the workload (packed weights live in byte
    buffers, so their tensors do not carry it)."""
    from .workloads import TORCH_DTYPE
    return _DT[TORCH_DTYPE[wl.wdt]]


def layer_options(wl, buf: "LayerBuffers") -> LayerOptionsC:
    return LayerOptionsC(buf.capacity, wl.route_groups, wl.route_max_groups,
                         1 if wl.fused_gather else 0, 1 if wl.all_reduce_form else 0,
                         1 if getattr(wl, "packed_weights", False) else 0,
                         1 if getattr(wl, "weights_in_gemm", False) else 0)


def moe_layer_forward(wl, logits, x, w13, w2, buf: "LayerBuffers", step_events=None,
                      stream=None):
    """The whole hot path in one C call (route, layout, permute, grouped
    GEMM, combine); optionally records 8 torch.cuda.Events between the
    kernels (see include/moe.h for their positions)."""
    cb = layer_buffers_c(buf)
    ev = _events(step_events, stream)
    _check("moe_layer_forward", load_library().moe_layer_forward(
        _ptr(logits), _ptr(x), dtype_code(x), wl.T, wl.H, wl.E, wl.k, wl.W, wl.I, _ptr(w13),
        _ptr(w2), _weight_code(wl), dtype_code(buf.xp), dtype_code(buf.y),
        ctypes.byref(layer_options(wl, buf)), ctypes.byref(cb), _ptr(buf.out),
        ev[0] if ev else None, _stream(stream)))
    return buf.out


def moe_layer_forward_host(wl, logits_host, x_host, out_host, logits_dev, x_dev, w13, w2,
                           buf: "LayerBuffers", step_events=None, stream=None):
    """moe_layer_forward with host inputs/output (copies inside the call)."""
    cb = layer_buffers_c(buf)
    ev = _events(step_events, stream)
    _check("moe_layer_forward_host", load_library().moe_layer_forward_host(
        _ptr(logits_host), _ptr(x_host), _ptr(out_host), _ptr(logits_dev), _ptr(x_dev),
        _ptr(buf.out), dtype_code(x_dev), wl.T, wl.H, wl.E, wl.k, wl.W, wl.I, _ptr(w13), _ptr(w2),
        _weight_code(wl), dtype_code(buf.xp), dtype_code(buf.y),
        ctypes.byref(layer_options(wl, buf)), ctypes.byref(cb), ev[0] if ev else None,
        _stream(stream)))


def layer_forward(wl, logits, x, w13, w2, buf: "LayerBuffers", stream=None):
    """The whole hot path: route -> layout -> permute -> grouped GEMM -> combine."""
    return moe_layer_forward(wl, logits, x, w13, w2, buf, stream=stream)
