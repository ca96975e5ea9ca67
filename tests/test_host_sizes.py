"""Host-side sizing of the layer's variants, on CPU: the algorithmic byte
counts the roofline fractions divide by, and the buffers the binding
allocates for each option.  (The kernels themselves are covered by the -m
gpu tests.)"""
import torch

from expert_parallelism_b200 import moe, traffic, workloads


def test_kernel_bytes_of_the_layer_variants():
    wl = workloads.WORKLOADS["dsv3"]
    T, H, E, k, W = wl.T, wl.H, wl.E, wl.k, wl.W
    N = T * k
    base = traffic.kernel_bytes(wl)
    # the permute inside the layer: x once, FP8 codes + scales + the GEMM's bf16 rows
    assert base["permute_layer"] == T * H * 2 + N * H + N * (H // 128) * 4 + N * H * 2
    # fused gather, FP8 payload: one bf16 round trip per token, nothing per slot
    fused = traffic.kernel_bytes(wl.replace(fused_gather=True))
    assert fused["permute_layer"] == T * H * 2 + T * H * 2
    assert fused["permute"] == base["permute"]          # the standalone send buffer is unchanged
    # fused gather, bf16 payload: no step at all
    mid = workloads.WORKLOADS["mid"]
    assert traffic.kernel_bytes(mid.replace(fused_gather=True))["permute_layer"] == 0
    # all_reduce form: slot_of_pair and topk_w per rank, W fp32 partials written and read
    ar = traffic.kernel_bytes(wl.replace(all_reduce_form=True))
    assert ar["combine"] - base["combine"] == (W - 1) * T * k * 8 + 2 * W * T * H * 4


def test_buffers_for_the_options():
    # FP8 payload with fewer slots than tokens: the fused gather's token rows need room
    wl = workloads.Workload("few", 600, 256, 8, 2, 64, 2, "bf16", "e4m3", "bf16",
                            capacity_factor=0.25)
    slots = moe.slot_rows(wl)
    assert slots < wl.T
    plain = moe.LayerBuffers(wl, "cpu")
    assert plain.gemm_ws.numel() == slots * wl.H * 2 and plain.partials is None
    fused = moe.LayerBuffers(wl.replace(fused_gather=True), "cpu")
    assert fused.gemm_ws.numel() == wl.T * wl.H * 2
    # the all_reduce form: one fp32 [T, H] partial per logical rank
    ar = moe.LayerBuffers(wl.replace(all_reduce_form=True), "cpu")
    assert tuple(ar.partials.shape) == (wl.W, wl.T, wl.H) and ar.partials.dtype == torch.float32
    opts = moe.layer_options(wl.replace(fused_gather=True, all_reduce_form=True), ar)
    assert (opts.capacity, opts.fused_gather, opts.all_reduce_form) == (ar.capacity, 1, 1)
    assert moe.layer_buffers_c(ar).partials == ar.partials.data_ptr()


def test_permute_bytes_and_gemm_flops_of_the_five_workloads():
    """Hand-computed: the permute reads x once and writes T*k payload rows
    (plus fp32 scales per 128 for FP8); the expert FFN is 6 N H I flops."""
    want_permute_mb = {"tiny": 0.393, "mid": 117.4, "dsv3": 601.9, "skew": 471.9, "decode": 8.26}
    want_gflops = {"tiny": 0.1007, "mid": 425.2, "dsv3": 5772.0, "skew": 3261.4, "decode": 45.10}
    for name in want_permute_mb:
        wl = workloads.WORKLOADS[name]
        mb = traffic.kernel_bytes(wl)["permute"] / 1e6
        gf = traffic.gemm_flops(wl)["total"] / 1e9
        assert abs(mb - want_permute_mb[name]) <= 0.002 * want_permute_mb[name], (name, mb)
        assert abs(gf - want_gflops[name]) <= 0.002 * want_gflops[name], (name, gf)
