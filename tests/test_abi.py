"""The C-ABI library loads, exports every symbol include/moe.h declares,
and rejects invalid arguments on the host before launching anything.

These run without a GPU: invalid calls return before any CUDA call, and
the workspace-size queries are pure host arithmetic.
"""
import ctypes
import os
import re

import pytest

from expert_parallelism_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

FAKE = ctypes.c_void_p(4096)   # never dereferenced: validation fails first


@pytest.fixture(scope="module")
def lib():
    from expert_parallelism_b200 import build
    build.build()
    return moe.load_library()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_five_steps():
    names = _declared()
    for n in ["moe_route_topk", "moe_dispatch_layout", "moe_permute", "moe_grouped_gemm",
              "moe_combine", "moe_check_status", "moe_status_str"]:
        assert n in names


def test_every_declared_symbol_is_exported_and_bound(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in moe.SIGNATURES, f"binding lacks {name}"


def _struct_fields(name):
    """Field names of `typedef struct <name> {...} <name>;` in the header,
    in order."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct " + name + r"\s*\{(.*?)\}\s*" + name + ";", src, re.S)
    assert body, name
    return re.findall(r"(\w+)\s*;", body.group(1))      # each declaration ends "name;"


def test_layer_structs_match_the_header():
    """The ctypes mirrors of moe_layer_options and moe_layer_buffers list the
    header's fields in the header's order (a drift would shift every later
    field)."""
    assert [f[0] for f in moe.LayerOptionsC._fields_] == _struct_fields("moe_layer_options")
    assert [f[0] for f in moe.LayerBuffersC._fields_] == _struct_fields("moe_layer_buffers")


def test_status_strings(lib):
    assert moe.moe_status_str(0) == "MOE_OK"
    assert moe.moe_status_str(1) == "MOE_ERR_INVALID_ARG"
    assert moe.moe_status_str(4) == "MOE_ERR_TIMEOUT"


def test_workspace_queries(lib):
    n = lib.moe_dispatch_layout_workspace_bytes(8192, 8, 256)
    assert n > 0 and n % 16 == 0
    assert lib.moe_dispatch_layout_workspace_bytes(0, 8, 256) > 0     # T=0 still writes offsets
    assert lib.moe_dispatch_layout_workspace_bytes(-1, 8, 256) == 0
    assert lib.moe_grouped_gemm_workspace_bytes(100, 256, 64, moe.MOE_BF16, moe.MOE_BF16) == 0


def test_route_rejects_before_launch(lib):
    f = lib.moe_route_topk
    assert f(FAKE, 10, 8, 9, FAKE, FAKE, None) == 1          # k > E
    assert f(FAKE, 10, 8, 0, FAKE, FAKE, None) == 1          # k < 1
    assert f(FAKE, -1, 8, 2, FAKE, FAKE, None) == 1          # T < 0
    assert f(None, 10, 8, 2, FAKE, FAKE, None) == 1          # null input
    assert f(FAKE, 10, 2048, 2, FAKE, FAKE, None) == 2       # E > 1024
    assert f(FAKE, 10, 64, 17, FAKE, FAKE, None) == 2        # k > 16
    assert f(None, 0, 8, 2, None, None, None) == 0           # empty batch: no-op


def test_layout_rejects_before_launch(lib):
    f = lib.moe_dispatch_layout
    ws = lib.moe_dispatch_layout_workspace_bytes(10, 2, 8)
    args = lambda **kw: [kw.get("idx", FAKE), 10, kw.get("k", 2), kw.get("E", 8), kw.get("W", 2),
                         FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("ws", FAKE),
                         kw.get("wsb", ws), kw.get("st", FAKE), None]
    assert f(*args(W=3)) == 1                 # ep_size must divide the number of experts
    assert f(*args(W=16)) == 1                # more ranks than experts
    assert f(*args(W=0)) == 1
    assert f(*args(wsb=ws - 1)) == 1          # workspace too small
    assert f(*args(ws=ctypes.c_void_p(4100))) == 1   # misaligned workspace
    assert f(*args(st=None)) == 1             # no status word
    assert f(*args(idx=None)) == 1
    assert f(*args(E=2048, W=2)) == 2


def test_capacity_layout_rejects_before_launch(lib):
    f = lib.moe_dispatch_layout_capacity
    ws = lib.moe_dispatch_layout_workspace_bytes(10, 2, 8)
    args = lambda **kw: [FAKE, 10, 2, kw.get("E", 8), kw.get("W", 2), kw.get("C", 4), FAKE, FAKE,
                         FAKE, FAKE, kw.get("pos", FAKE), None, FAKE, ws, FAKE, None]
    assert f(*args(C=-1)) == 1                # negative capacity
    assert f(*args(W=3)) == 1                 # same checks as the dropless layout
    assert f(*args(pos=None)) == 1            # slab map missing
    assert f(*args(E=1024, W=1, C=1 << 21)) == 2   # E * C rows do not fit int32


def test_permute_combine_gemm_reject_before_launch(lib):
    p = lib.moe_permute
    assert p(FAKE, moe.MOE_BF16, 10, 100, 2, FAKE, FAKE, moe.MOE_BF16, None, None) == 1   # H % 8
    assert p(FAKE, moe.MOE_BF16, 10, 136, 2, FAKE, FAKE, moe.MOE_E4M3, FAKE, None) == 1   # H % 128
    assert p(FAKE, moe.MOE_BF16, 10, 128, 2, FAKE, FAKE, moe.MOE_E4M3, None, None) == 1   # scales
    assert p(FAKE, moe.MOE_E4M3, 10, 128, 2, FAKE, FAKE, moe.MOE_E4M3, FAKE, None) == 1   # x dtype
    assert p(FAKE, moe.MOE_BF16, 10, 128, 2, FAKE, FAKE, moe.MOE_F32, None, None) == 1    # cast
    assert p(ctypes.c_void_p(4098), moe.MOE_BF16, 10, 128, 2, FAKE, FAKE, moe.MOE_BF16, None,
             None) == 1                                                                 # align
    # FP8 block scales go out as 16-byte vectors: a scale buffer at an odd
    # float offset (a sliced tensor, say) is refused instead of faulting
    assert p(FAKE, moe.MOE_BF16, 10, 512, 2, FAKE, FAKE, moe.MOE_E4M3, ctypes.c_void_p(4100),
             None) == 1
    c = lib.moe_combine
    assert c(FAKE, moe.MOE_E4M3, None, FAKE, FAKE, 10, 2, 128, FAKE, moe.MOE_BF16, None) == 1  # scales
    assert c(FAKE, moe.MOE_E4M3, FAKE, FAKE, FAKE, 10, 2, 136, FAKE, moe.MOE_BF16, None) == 1  # H%128
    assert c(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 10, 0, 128, FAKE, moe.MOE_BF16, None) == 1
    assert c(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 10, 17, 128, FAKE, moe.MOE_BF16, None) == 2
    g = lib.moe_grouped_gemm
    base = [FAKE, moe.MOE_BF16, None, FAKE, None, 0, 8, 100, 256, 64, FAKE, FAKE, moe.MOE_BF16,
            FAKE, FAKE, moe.MOE_F32, None, None, 0, FAKE, None]
    bad = list(base); bad[9] = 60                      # I % 8
    assert g(*bad) == 1
    bad = list(base); bad[1] = moe.MOE_F32             # f32 payload with bf16 weights
    assert g(*bad) == 1
    bad = list(base); bad[1] = moe.MOE_E4M3            # FP8 payload needs scales
    assert g(*bad) == 1
    bad = list(base); bad[19] = None                   # status word
    assert g(*bad) == 1
    bad = list(base); bad[15] = moe.MOE_E4M3           # FP8 y needs its block scales
    assert g(*bad) == 1
    bad = list(base); bad[15] = moe.MOE_E4M3; bad[16] = FAKE; bad[8] = 200   # and H % 128
    assert g(*bad) == 1
    bad = list(base); bad[1] = moe.MOE_F32; bad[12] = moe.MOE_F32; bad[15] = moe.MOE_BF16
    assert g(*bad) == 1                                # fp32 GEMM stores y in fp32
    bad = list(base); bad[6] = 0                       # no experts
    assert g(*bad) == 1


def test_missing_library_fails_loudly(tmp_path):
    saved = moe._lib
    moe._lib = None
    try:
        with pytest.raises(ImportError):
            moe.load_library(str(tmp_path / "nope.so"))
    finally:
        moe._lib = saved


def test_layer_call_rejects_before_launch(lib):
    f = lib.moe_layer_forward
    # no buffer struct
    assert f(FAKE, FAKE, moe.MOE_BF16, 10, 128, 8, 2, 2, 64, FAKE, FAKE, moe.MOE_BF16,
             moe.MOE_BF16, moe.MOE_F32, None, None, FAKE, None, None) == 1
    cb = moe.LayerBuffersC(*([FAKE] * 8 + [0] + [FAKE] * 6 + [0] + [FAKE, None]))
    # E % W != 0 is caught before anything runs (workspace size 0 too)
    assert f(FAKE, FAKE, moe.MOE_BF16, 10, 128, 8, 2, 3, 64, FAKE, FAKE, moe.MOE_BF16,
             moe.MOE_BF16, moe.MOE_F32, None, ctypes.byref(cb), FAKE, None, None) == 1
    # a capacity whose E * C rows do not fit int32
    big = moe.LayerOptionsC(1 << 28, 0, 0)
    assert f(FAKE, FAKE, moe.MOE_BF16, 10, 128, 8, 2, 2, 64, FAKE, FAKE, moe.MOE_BF16,
             moe.MOE_BF16, moe.MOE_F32, ctypes.byref(big), ctypes.byref(cb), FAKE, None,
             None) == 2
    # group-limited routing that cannot give k picks (2 groups of 4, 1 kept, k = 5)
    grp = moe.LayerOptionsC(-1, 2, 1)
    assert f(FAKE, FAKE, moe.MOE_BF16, 10, 128, 8, 5, 2, 64, FAKE, FAKE, moe.MOE_BF16,
             moe.MOE_BF16, moe.MOE_F32, ctypes.byref(grp), ctypes.byref(cb), FAKE, None,
             None) == 1


def test_all_reduce_form_calls_reject_before_launch(lib):
    cr = lib.moe_combine_rank
    assert cr(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 10, 2, 128, FAKE, 4, 4, FAKE, None) == 1  # rank
    assert cr(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 10, 2, 128, FAKE, 4, -1, FAKE, None) == 1
    assert cr(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 10, 2, 128, None, 4, 0, FAKE, None) == 1  # offsets
    assert cr(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 10, 2, 100, FAKE, 4, 0, FAKE, None) == 1  # H % 8
    assert cr(FAKE, moe.MOE_BF16, None, FAKE, FAKE, 0, 2, 128, None, 4, 0, None, None) == 0   # empty
    rp = lib.moe_reduce_partials
    assert rp(FAKE, 0, 10, 128, FAKE, moe.MOE_BF16, None) == 1             # no partials
    assert rp(FAKE, 2, 10, 100, FAKE, moe.MOE_BF16, None) == 1             # H % 8
    assert rp(FAKE, 2, 10, 128, FAKE, moe.MOE_E4M3, None) == 1             # out dtype
    assert rp(ctypes.c_void_p(4100), 2, 10, 128, FAKE, moe.MOE_BF16, None) == 1   # alignment
    assert rp(None, 2, 0, 128, None, moe.MOE_BF16, None) == 0              # empty
    # the layer's all_reduce form needs the partials buffer
    lw = moe.moe_dispatch_layout_workspace_bytes(10, 2, 8)
    cb = moe.LayerBuffersC(*([FAKE] * 8 + [lw] + [FAKE] * 6 + [0] + [FAKE, None, None]))
    o = moe.LayerOptionsC(-1, 0, 0, 0, 1)
    assert lib.moe_layer_forward(FAKE, FAKE, moe.MOE_BF16, 10, 128, 8, 2, 2, 64, FAKE, FAKE,
                                 moe.MOE_BF16, moe.MOE_BF16, moe.MOE_F32, ctypes.byref(o),
                                 ctypes.byref(cb), FAKE, None, None) == 1


def test_layer_call_rejects_misaligned_fp8_scales(lib):
    """The layer call checks the permute's scale buffer as moe_permute does."""
    T, H, E, k, W, I = 10, 512, 8, 2, 2, 64
    lw = moe.moe_dispatch_layout_workspace_bytes(T, k, E)
    gw = T * k * H * 2                                 # the FP8 payload's bf16 rows
    fields = [FAKE] * 8 + [lw] + [FAKE] * 6 + [gw] + [FAKE, None, None]
    fields[10] = ctypes.c_void_p(4100)                 # xp_scales, 4-byte aligned only
    cb = moe.LayerBuffersC(*fields)
    assert lib.moe_layer_forward(FAKE, FAKE, moe.MOE_BF16, T, H, E, k, W, I, FAKE, FAKE,
                                 moe.MOE_BF16, moe.MOE_E4M3, moe.MOE_F32, None, ctypes.byref(cb),
                                 FAKE, None, None) == 1


def test_fused_gather_needs_one_workspace_row_per_token(lib):
    """With an FP8 payload the fused gather keeps one bf16 row per token in
    the GEMM workspace: a workspace sized only for the GEMM's slots (here 8
    slots from capacity 1, fewer than the 10 tokens) is rejected up front."""
    T, H, E, k, W, I = 10, 128, 8, 2, 2, 64
    lw = moe.moe_dispatch_layout_workspace_bytes(T, k, E)
    cb = moe.LayerBuffersC(*([FAKE] * 8 + [lw] + [FAKE] * 6 + [E * 1 * H * 2] + [FAKE, None]))
    fused = moe.LayerOptionsC(1, 0, 0, 1, 0)
    assert lib.moe_layer_forward(FAKE, FAKE, moe.MOE_BF16, T, H, E, k, W, I, FAKE, FAKE,
                                 moe.MOE_BF16, moe.MOE_E4M3, moe.MOE_F32, ctypes.byref(fused),
                                 ctypes.byref(cb), FAKE, None, None) == 1


def test_wait_timeout_diagnostic_rejects_before_launch(lib):
    f = lib.moe_diag_layout_wait_timeout
    n = lib.moe_diag_layout_wait_timeout_workspace_bytes()
    assert n > 0 and n % 16 == 0
    assert f(None, n, 1000, FAKE, None) == 1                    # no workspace
    assert f(FAKE, n - 1, 1000, FAKE, None) == 1                # too small
    assert f(ctypes.c_void_p(4100), n, 1000, FAKE, None) == 1   # misaligned
    assert f(FAKE, n, 1000, None, None) == 1                    # no status word
    assert f(FAKE, n, 3 * 10 ** 9, FAKE, None) == 1             # above the library's 2 s


def test_ep_calls_reject_before_launch(lib):
    W = 2
    table = (ctypes.c_void_p * W)(4096, 8192)
    bad_table = (ctypes.c_void_p * W)(4096, 4100)            # misaligned peer buffer
    null_table = (ctypes.c_void_p * W)(4096, None)
    pl = lib.moe_ep_plan
    assert pl(FAKE, 3, 8, 0, FAKE, FAKE, FAKE, None) == 1       # W must divide E
    assert pl(FAKE, 2, 8, 2, FAKE, FAKE, FAKE, None) == 1       # rank outside [0, W)
    assert pl(FAKE, 128, 128, 0, FAKE, FAKE, FAKE, None) == 2   # more than 64 ranks
    assert pl(None, 2, 8, 0, FAKE, FAKE, FAKE, None) == 1
    d = lib.moe_ep_dispatch
    args = lambda **kw: [FAKE, moe.MOE_BF16, 10, kw.get("H", 128), 2, FAKE, FAKE, FAKE, FAKE,
                         kw.get("E", 8), W, kw.get("rows", table), kw.get("sc", None),
                         kw.get("pd", moe.MOE_BF16), kw.get("cap", 100), FAKE, None]
    assert d(*args(E=7)) == 1                                  # W does not divide E
    assert d(*args(rows=bad_table)) == 1
    assert d(*args(rows=null_table)) == 1
    assert d(*args(pd=moe.MOE_E4M3)) == 1                      # FP8 needs the scale table
    assert d(*args(pd=moe.MOE_E4M3, sc=table, H=136)) == 1     # and H % 128
    assert d(*args(pd=moe.MOE_F32)) == 1                       # no dtype cast
    assert d(*args(cap=-1)) == 1
    assert d(*args(cap=1 << 31)) == 2
    c = lib.moe_ep_combine
    cargs = lambda **kw: [kw.get("rows", table), kw.get("sc", None), kw.get("yd", moe.MOE_F32),
                          FAKE, FAKE, FAKE, FAKE, FAKE, 10, 2, 128, 8, W, 100,
                          kw.get("out", FAKE), moe.MOE_BF16, FAKE, None]
    assert c(*cargs(rows=null_table)) == 1
    assert c(*cargs(yd=moe.MOE_E4M3)) == 1                     # FP8 y needs the scale table
    assert c(*cargs(out=ctypes.c_void_p(4100))) == 1            # misaligned out
    assert moe.moe_status_str(6) == "MOE_ERR_OVERFLOW"
    rec = ctypes.create_string_buffer(lib.moe_ipc_handle_bytes())
    assert lib.moe_ipc_handle_bytes() >= 64
    assert lib.moe_ipc_export(None, rec) == 1
    assert lib.moe_ipc_import(None, ctypes.byref(ctypes.c_void_p())) == 1
    assert lib.moe_ipc_close(rec, None) == 1


def test_pack_calls_reject_before_launch(lib):
    assert lib.moe_packed_weights_bytes(256, 7168, 2048, 0) == 256 * 32 * 112 * 16384
    assert lib.moe_packed_weights_bytes(256, 7168, 2048, 1) == 256 * 56 * 32 * 16384
    assert lib.moe_packed_weights_bytes(128, 2880, 2880, 1) == 128 * 24 * 45 * 16384
    assert lib.moe_packed_weights_bytes(4, 256, 64, 2) == 0
    f = lib.moe_pack_expert_weights
    assert f(FAKE, FAKE, 4, 256, 64, moe.MOE_F32, FAKE, FAKE, None) == 1     # bf16 only
    assert f(FAKE, FAKE, 4, 250, 64, moe.MOE_BF16, FAKE, FAKE, None) == 1    # H % 8
    assert f(FAKE, FAKE, 4, 256, 64, moe.MOE_BF16, None, FAKE, None) == 1    # no output
    assert f(None, None, 4, 256, 64, moe.MOE_BF16, FAKE, FAKE, None) == 1    # nothing to pack
    assert f(ctypes.c_void_p(4100), None, 4, 256, 64, moe.MOE_BF16, FAKE, None, None) == 1
    g = lib.moe_grouped_gemm_packed
    base = [FAKE, moe.MOE_BF16, None, FAKE, None, 0, 8, 100, 256, 64, FAKE, FAKE, moe.MOE_BF16,
            FAKE, FAKE, moe.MOE_F32, None, None, 0, FAKE, None]
    bad = list(base); bad[12] = moe.MOE_F32            # packed weights are bf16
    assert g(*bad) == 1
    bad = list(base); bad[9] = 60                      # I % 8
    assert g(*bad) == 1


def test_grouped_route_rejects_before_launch(lib):
    f = lib.moe_route_topk_grouped
    assert f(FAKE, 10, 8, 2, 3, 1, FAKE, FAKE, None) == 1      # groups must divide E
    assert f(FAKE, 10, 8, 5, 4, 2, FAKE, FAKE, None) == 1      # 2 groups of 2: < 5 experts
    assert f(FAKE, 10, 8, 2, 4, 5, FAKE, FAKE, None) == 1      # more kept groups than groups
    assert f(FAKE, 10, 8, 2, 4, 0, FAKE, FAKE, None) == 1
    assert f(FAKE, 10, 128, 2, 64, 4, FAKE, FAKE, None) == 2   # more than 32 groups
    assert f(None, 0, 8, 2, 4, 2, None, None, None) == 0       # empty batch: no-op
