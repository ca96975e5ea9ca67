// api.cu -- the extern "C" boundary of libmoe (declared in include/moe.h).
//
// Every entry point validates its arguments on the host first and returns
// MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED before anything is enqueued,
// then launches its kernels on the caller's stream and returns without
// waiting.  Nothing here allocates or frees device memory.
#include <stdio.h>

#include <atomic>

#include "common.cuh"

namespace moe {
cudaError_t launch_route_topk(const float*, int64_t, int, int, int, int, int32_t*, float*,
                              cudaStream_t);
size_t layout_workspace_bytes(int64_t T, int k, int E);
cudaError_t launch_dispatch_layout(const int32_t*, int64_t, int, int, int, int, int32_t*,
                                   int32_t*, int32_t*, int32_t*, int32_t*, int32_t*, void*,
                                   int32_t*, cudaStream_t);
cudaError_t launch_permute(const void*, moe_dtype, int64_t, int, int, const int32_t*, void*,
                           moe_dtype, float*, __nv_bfloat16*, cudaStream_t);
cudaError_t launch_combine(const void*, moe_dtype, const float*, const int32_t*, const float*,
                           int64_t, int, int, void*, moe_dtype, cudaStream_t,
                           const int32_t* rank_offsets = nullptr, int rank = 0);
cudaError_t launch_reduce_partials(const float*, int, int64_t, void*, moe_dtype, cudaStream_t);
cudaError_t launch_dequant_e4m3(const uint8_t*, const float*, const int32_t*, int, int, int64_t,
                                int, __nv_bfloat16*, cudaStream_t);
cudaError_t launch_grouped_gemm_simt_f32(const float*, const int32_t*, const int32_t*, int, int,
                                         int64_t, int, int, const float*, const float*, float*,
                                         float*, cudaEvent_t, cudaStream_t);
cudaError_t launch_grouped_gemm_tc(const __nv_bfloat16*, const int32_t*, const int32_t*, int, int,
                                   int64_t, int, int, const __nv_bfloat16*, const __nv_bfloat16*,
                                   __nv_bfloat16*, void*, moe_dtype, float*, int32_t*,
                                   const gemm_gather*, cudaEvent_t, cudaStream_t, bool,
                                   const float*, const int32_t*);
size_t packed_weights_bytes(int64_t E, int H, int I, int which);
cudaError_t launch_pack_weights(const __nv_bfloat16*, const __nv_bfloat16*, int64_t, int, int,
                                __nv_bfloat16*, __nv_bfloat16*, cudaStream_t);
bool grouped_gemm_tc_uses_swap(int64_t n_rows, int n_experts, moe_dtype y_dtype);
cudaError_t launch_quantize_tokens_e4m3(const void*, moe_dtype, int64_t, int, __nv_bfloat16*,
                                       cudaStream_t);
size_t layout_wait_selftest_bytes();
cudaError_t launch_layout_wait_selftest(void*, uint64_t, int32_t*, cudaStream_t);
}  // namespace moe

namespace moe {
static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace moe

namespace moe {

moe_status report_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    fprintf(stderr, "libmoe: CUDA error: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

// The layout's argument rules, except for the caller workspace (shared by
// every layout entry point).
moe_status check_layout_args(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E, int32_t W,
                             const int32_t* expert_counts, const int32_t* expert_offsets,
                             const int32_t* rank_offsets, const int32_t* slot_of_pair,
                             const int32_t* pair_of_slot, const int32_t* dev_status) {
    if (T < 0 || k < 1 || E < 1 || W < 1 || W > E || (E % W) != 0) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (T * (int64_t)k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    if (!expert_counts || !expert_offsets || !rank_offsets || !dev_status)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !slot_of_pair || !pair_of_slot)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

namespace {

bool is_act_dtype(moe_dtype d) { return d == MOE_F32 || d == MOE_BF16; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

moe_status cuda_status(cudaError_t e) { return moe::report_cuda(e); }


// Host-side validation of each step (no launch).  *noop is set when the
// arguments are valid and there is nothing to launch (an empty batch).
moe_status check_route(const float* logits, int64_t T, int32_t E, int32_t k,
                       const int32_t* topk_idx, const float* topk_w, bool* noop) {
    *noop = false;
    if (T < 0 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return *noop = true, MOE_OK;
    if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Group-limited routing: G equal groups (G | E, 1 <= G <= 32), at most M
// of them per token (1 <= M <= G) with enough experts for k picks.
moe_status check_route_groups(int32_t E, int32_t k, int32_t G, int32_t M) {
    if (G < 1 || M < 1 || M > G || (E % G) != 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)k > (int64_t)M * (E / G)) return MOE_ERR_INVALID_ARG;
    if (G > 32) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_layout(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E, int32_t W,
                        const int32_t* expert_counts, const int32_t* expert_offsets,
                        const int32_t* rank_offsets, const int32_t* slot_of_pair,
                        const int32_t* pair_of_slot, const void* workspace,
                        size_t workspace_bytes, const int32_t* dev_status) {
    const moe_status st = moe::check_layout_args(topk_idx, T, k, E, W, expert_counts,
                                                 expert_offsets, rank_offsets, slot_of_pair,
                                                 pair_of_slot, dev_status);
    if (st != MOE_OK) return st;
    if (!workspace || workspace_bytes < layout_workspace_bytes(T, k, E) || !aligned16(workspace))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status check_permute(const void* x, moe_dtype x_dtype, int64_t T, int32_t H, int32_t k,
                         const int32_t* slot_of_pair, const void* xp, moe_dtype xp_dtype,
                         const float* xp_scales, bool* noop) {
    *noop = false;
    if (T < 0 || H < 1 || k < 1 || (H % 8) != 0) return MOE_ERR_INVALID_ARG;
    if (!is_act_dtype(x_dtype)) return MOE_ERR_INVALID_ARG;
    if (xp_dtype != x_dtype && xp_dtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
    // the block scales leave the kernel as 16-byte vectors: 16-byte aligned
    if (xp_dtype == MOE_E4M3 && ((H % 128) != 0 || !xp_scales || !aligned16(xp_scales)))
        return MOE_ERR_INVALID_ARG;
    if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return *noop = true, MOE_OK;
    if (!x || !slot_of_pair || !xp || !aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

size_t gemm_workspace_bytes(int64_t n_rows, int32_t H, moe_dtype xp_dtype) {
    if (n_rows < 0 || H < 1) return 0;
    // FP8 payload: a bf16 copy of the dequantised rows for the GEMM's A.
    return xp_dtype == MOE_E4M3 ? (size_t)n_rows * H * 2 : 0;
}

moe_status check_gemm(const void* xp, moe_dtype xp_dtype, const float* xp_scales,
                      const int32_t* expert_offsets, int32_t expert_begin, int32_t n_experts,
                      int64_t n_rows, int32_t H, int32_t I, const void* w13, const void* w2,
                      moe_dtype w_dtype, const void* h, const void* y, moe_dtype y_dtype,
                      const float* y_scales, const void* workspace, size_t workspace_bytes,
                      const int32_t* dev_status, bool* noop) {
    *noop = false;
    if (n_rows < 0 || H < 1 || I < 1 || (H % 8) != 0 || (I % 8) != 0) return MOE_ERR_INVALID_ARG;
    if (expert_begin < 0 || n_experts < 1) return MOE_ERR_INVALID_ARG;
    if (n_experts > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    const bool f32 = (w_dtype == MOE_F32 && xp_dtype == MOE_F32);
    const bool bf16 = (w_dtype == MOE_BF16 && (xp_dtype == MOE_BF16 || xp_dtype == MOE_E4M3));
    if (!f32 && !bf16) return MOE_ERR_INVALID_ARG;
    // y: fp32 (either path), bf16 or the FP8 combine payload (bf16 path only)
    if (y_dtype != MOE_F32 && !(bf16 && (y_dtype == MOE_BF16 || y_dtype == MOE_E4M3)))
        return MOE_ERR_INVALID_ARG;
    if (y_dtype == MOE_E4M3 && ((H % 128) != 0 || !y_scales)) return MOE_ERR_INVALID_ARG;
    if (xp_dtype == MOE_E4M3 && ((H % 128) != 0 || !xp_scales)) return MOE_ERR_INVALID_ARG;
    if (!expert_offsets || !w13 || !w2 || !dev_status) return MOE_ERR_INVALID_ARG;
    if (n_rows == 0) return *noop = true, MOE_OK;
    if (!xp || !h || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(w13) || !aligned16(w2) || !aligned16(h) || !aligned16(y))
        return MOE_ERR_INVALID_ARG;
    const size_t need = gemm_workspace_bytes(n_rows, H, xp_dtype);
    if (need > 0 && (workspace_bytes < need || !workspace || ((uintptr_t)workspace & 127u)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status check_combine(const void* y, moe_dtype y_dtype, const float* y_scales,
                         const int32_t* slot_of_pair, const float* topk_w, int64_t T, int32_t k,
                         int32_t H, const void* out, moe_dtype out_dtype, bool* noop) {
    *noop = false;
    if (T < 0 || H < 1 || k < 1 || (H % 8) != 0) return MOE_ERR_INVALID_ARG;
    if (!(is_act_dtype(y_dtype) || y_dtype == MOE_E4M3) || !is_act_dtype(out_dtype))
        return MOE_ERR_INVALID_ARG;
    if (y_dtype == MOE_E4M3 && ((H % 128) != 0 || !y_scales)) return MOE_ERR_INVALID_ARG;
    if (k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return *noop = true, MOE_OK;
    // topk_w may be null: unit weights (outputs that already carry them)
    if (!y || !slot_of_pair || !out || !aligned16(y) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// ev_a (after the FP8 dequantisation, or at the start) and ev_b (between
// the two GEMM phases) may be null.  g (bf16 weights, operand-swapped
// kernel only): the gate/up rows are gathered from g->src; xp is not read.
cudaError_t run_gemm(const void* xp, moe_dtype xp_dtype, const float* xp_scales,
                     const int32_t* expert_offsets, const int32_t* expert_counts,
                     int32_t expert_begin, int32_t n_experts,
                     int64_t n_rows, int32_t H, int32_t I, const void* w13, const void* w2,
                     moe_dtype w_dtype, void* h, void* y, moe_dtype y_dtype, float* y_scales,
                     void* workspace, int32_t* dev_status, cudaStream_t s,
                     cudaEvent_t ev_a = nullptr, cudaEvent_t ev_b = nullptr,
                     bool a_ready = false, const gemm_gather* g = nullptr, bool packed = false,
                     const float* row_weights = nullptr, const int32_t* weight_pairs = nullptr) {
    cudaError_t e = cudaSuccess;
    if (w_dtype == MOE_F32) {
        if (ev_a) e = cudaEventRecord(ev_a, s);
        if (e != cudaSuccess) return e;
        return launch_grouped_gemm_simt_f32((const float*)xp, expert_offsets, expert_counts,
                                            expert_begin, n_experts, n_rows, H, I,
                                            (const float*)w13, (const float*)w2, (float*)h,
                                            (float*)y, ev_b, s);
    }
    const __nv_bfloat16* a = (const __nv_bfloat16*)xp;
    if (xp_dtype == MOE_E4M3 && !g) {
        // the FP8 rows' bf16 operand, unless the permute already wrote it
        if (!a_ready)
            e = launch_dequant_e4m3((const uint8_t*)xp, xp_scales, expert_offsets, expert_begin,
                                    n_experts, n_rows, H, (__nv_bfloat16*)workspace, s);
        if (e != cudaSuccess) return e;
        a = (const __nv_bfloat16*)workspace;
    }
    if (ev_a) e = cudaEventRecord(ev_a, s);
    if (e != cudaSuccess) return e;
    return launch_grouped_gemm_tc(a, expert_offsets, expert_counts, expert_begin, n_experts,
                                  n_rows, H, I,
                                  (const __nv_bfloat16*)w13, (const __nv_bfloat16*)w2,
                                  (__nv_bfloat16*)h, y, y_dtype, y_scales, dev_status, g, ev_b,
                                  s, packed, row_weights, weight_pairs);
}

}  // namespace

extern "C" {

moe_status moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k,
                          int32_t* topk_idx, float* topk_w, void* stream) {
    bool noop;
    const moe_status st = check_route(logits, T, E, k, topk_idx, topk_w, &noop);
    if (st != MOE_OK || noop) return st;
    return cuda_status(
        launch_route_topk(logits, T, E, k, 0, 0, topk_idx, topk_w, (cudaStream_t)stream));
}

moe_status moe_route_topk_grouped(const float* logits, int64_t T, int32_t E, int32_t k,
                                  int32_t groups, int32_t max_groups, int32_t* topk_idx,
                                  float* topk_w, void* stream) {
    bool noop;
    moe_status st = check_route_groups(E, k, groups, max_groups);
    if (st == MOE_OK) st = check_route(logits, T, E, k, topk_idx, topk_w, &noop);
    if (st != MOE_OK || noop) return st;
    return cuda_status(launch_route_topk(logits, T, E, k, groups, max_groups, topk_idx, topk_w,
                                         (cudaStream_t)stream));
}

size_t moe_dispatch_layout_workspace_bytes(int64_t T, int32_t k, int32_t E) {
    if (T < 0 || k < 1 || E < 1) return 0;
    return layout_workspace_bytes(T, k, E);
}

moe_status moe_dispatch_layout(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                               int32_t W, int32_t* expert_counts, int32_t* expert_offsets,
                               int32_t* rank_offsets, int32_t* slot_of_pair,
                               int32_t* pair_of_slot, void* workspace, size_t workspace_bytes,
                               int32_t* dev_status, void* stream) {
    const moe_status st = check_layout(topk_idx, T, k, E, W, expert_counts, expert_offsets,
                                       rank_offsets, slot_of_pair, pair_of_slot, workspace,
                                       workspace_bytes, dev_status);
    if (st != MOE_OK) return st;
    return cuda_status(launch_dispatch_layout(topk_idx, T, k, E, W, -1, expert_counts,
                                              expert_offsets, rank_offsets, slot_of_pair,
                                              pair_of_slot, nullptr, workspace, dev_status,
                                              (cudaStream_t)stream));
}

moe_status moe_dispatch_layout_capacity(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                                        int32_t W, int32_t capacity, int32_t* expert_counts,
                                        int32_t* expert_offsets, int32_t* rank_offsets,
                                        int32_t* slot_of_pair, int32_t* pair_of_slot,
                                        int32_t* n_dropped, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_status,
                                        void* stream) {
    if (capacity < 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)E * capacity >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    moe_status st = check_layout(topk_idx, T, k, E, W, expert_counts, expert_offsets,
                                 rank_offsets, slot_of_pair, pair_of_slot, workspace,
                                 workspace_bytes, dev_status);
    if (st != MOE_OK) return st;
    if ((int64_t)E * capacity > 0 && !pair_of_slot) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_dispatch_layout(topk_idx, T, k, E, W, capacity, expert_counts,
                                              expert_offsets, rank_offsets, slot_of_pair,
                                              pair_of_slot, n_dropped, workspace, dev_status,
                                              (cudaStream_t)stream));
}

moe_status moe_permute(const void* x, moe_dtype x_dtype, int64_t T, int32_t H, int32_t k,
                       const int32_t* slot_of_pair, void* xp, moe_dtype xp_dtype,
                       float* xp_scales, void* stream) {
    bool noop;
    const moe_status st =
        check_permute(x, x_dtype, T, H, k, slot_of_pair, xp, xp_dtype, xp_scales, &noop);
    if (st != MOE_OK || noop) return st;
    return cuda_status(launch_permute(x, x_dtype, T, H, k, slot_of_pair, xp, xp_dtype, xp_scales,
                                      nullptr, (cudaStream_t)stream));
}

size_t moe_grouped_gemm_workspace_bytes(int64_t n_rows, int32_t H, int32_t I, moe_dtype xp_dtype,
                                        moe_dtype w_dtype) {
    (void)I;
    (void)w_dtype;
    return gemm_workspace_bytes(n_rows, H, xp_dtype);
}

moe_status moe_grouped_gemm(const void* xp, moe_dtype xp_dtype, const float* xp_scales,
                            const int32_t* expert_offsets, const int32_t* expert_counts,
                            int32_t expert_begin,
                            int32_t n_experts, int64_t n_rows, int32_t H, int32_t I,
                            const void* w13, const void* w2, moe_dtype w_dtype, void* h, void* y,
                            moe_dtype y_dtype, float* y_scales, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream) {
    bool noop;
    const moe_status st =
        check_gemm(xp, xp_dtype, xp_scales, expert_offsets, expert_begin, n_experts, n_rows, H,
                   I, w13, w2, w_dtype, h, y, y_dtype, y_scales, workspace, workspace_bytes,
                   dev_status, &noop);
    if (st != MOE_OK || noop) return st;
    return cuda_status(run_gemm(xp, xp_dtype, xp_scales, expert_offsets, expert_counts,
                                expert_begin, n_experts, n_rows, H, I, w13, w2, w_dtype, h, y,
                                y_dtype, y_scales, workspace, dev_status, (cudaStream_t)stream));
}

size_t moe_packed_weights_bytes(int32_t E, int32_t H, int32_t I, int32_t which) {
    if (E < 1 || H < 1 || I < 1 || (which != 0 && which != 1)) return 0;
    return packed_weights_bytes(E, H, I, which);
}

moe_status moe_pack_expert_weights(const void* w13, const void* w2, int32_t E, int32_t H,
                                   int32_t I, moe_dtype w_dtype, void* packed13, void* packed2,
                                   void* stream) {
    if (E < 1 || H < 1 || I < 1 || (H % 8) != 0 || (I % 8) != 0 || w_dtype != MOE_BF16)
        return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (!w13 && !w2) return MOE_ERR_INVALID_ARG;
    if ((w13 && (!packed13 || !aligned16(w13) || !aligned16(packed13))) ||
        (w2 && (!packed2 || !aligned16(w2) || !aligned16(packed2))))
        return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_pack_weights((const __nv_bfloat16*)w13, (const __nv_bfloat16*)w2, E,
                                           H, I, (__nv_bfloat16*)packed13, (__nv_bfloat16*)packed2,
                                           (cudaStream_t)stream));
}

moe_status moe_grouped_gemm_packed(const void* xp, moe_dtype xp_dtype, const float* xp_scales,
                                   const int32_t* expert_offsets, const int32_t* expert_counts,
                                   int32_t expert_begin, int32_t n_experts, int64_t n_rows,
                                   int32_t H, int32_t I, const void* packed13,
                                   const void* packed2, moe_dtype w_dtype, void* h, void* y,
                                   moe_dtype y_dtype, float* y_scales, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_status, void* stream) {
    if (w_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    bool noop;
    const moe_status st =
        check_gemm(xp, xp_dtype, xp_scales, expert_offsets, expert_begin, n_experts, n_rows, H,
                   I, packed13, packed2, w_dtype, h, y, y_dtype, y_scales, workspace,
                   workspace_bytes, dev_status, &noop);
    if (st != MOE_OK || noop) return st;
    return cuda_status(run_gemm(xp, xp_dtype, xp_scales, expert_offsets, expert_counts,
                                expert_begin, n_experts, n_rows, H, I, packed13, packed2, w_dtype,
                                h, y, y_dtype, y_scales, workspace, dev_status,
                                (cudaStream_t)stream, nullptr, nullptr, false, nullptr, true));
}

moe_status moe_combine(const void* y, moe_dtype y_dtype, const float* y_scales,
                       const int32_t* slot_of_pair, const float* topk_w, int64_t T, int32_t k,
                       int32_t H, void* out, moe_dtype out_dtype, void* stream) {
    bool noop;
    const moe_status st = check_combine(y, y_dtype, y_scales, slot_of_pair, topk_w, T, k, H, out,
                                        out_dtype, &noop);
    if (st != MOE_OK || noop) return st;
    return cuda_status(launch_combine(y, y_dtype, y_scales, slot_of_pair, topk_w, T, k, H, out,
                                      out_dtype, (cudaStream_t)stream));
}

moe_status moe_combine_rank(const void* y, moe_dtype y_dtype, const float* y_scales,
                            const int32_t* slot_of_pair, const float* topk_w, int64_t T,
                            int32_t k, int32_t H, const int32_t* rank_offsets, int32_t world,
                            int32_t rank, float* partial, void* stream) {
    bool noop;
    const moe_status st = check_combine(y, y_dtype, y_scales, slot_of_pair, topk_w, T, k, H,
                                        partial, MOE_F32, &noop);
    if (st != MOE_OK) return st;
    if (world < 1 || rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
    if (noop) return MOE_OK;
    if (!rank_offsets) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_combine(y, y_dtype, y_scales, slot_of_pair, topk_w, T, k, H, partial,
                                      MOE_F32, (cudaStream_t)stream, rank_offsets, rank));
}

moe_status moe_reduce_partials(const float* partials, int32_t n_partials, int64_t T, int32_t H,
                               void* out, moe_dtype out_dtype, void* stream) {
    if (n_partials < 1 || T < 0 || H < 1 || (H % 8) != 0 || !is_act_dtype(out_dtype))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!partials || !out || !aligned16(partials) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    return cuda_status(
        launch_reduce_partials(partials, n_partials, T * H, out, out_dtype, (cudaStream_t)stream));
}

// Rows of the permuted buffers: T*k (dropless) or E*capacity (fixed slabs).
static int64_t layer_slots(int64_t T, int32_t k, int32_t E, int32_t capacity) {
    return capacity < 0 ? T * k : (int64_t)E * capacity;
}

static moe_layer_options resolve(const moe_layer_options* o) {
    return o ? *o : moe_layer_options{-1, 0, 0, 0, 0, 0, 0};
}

static moe_status check_layer(const float* logits, const void* x, moe_dtype x_dtype, int64_t T,
                              int32_t H, int32_t E, int32_t k, int32_t W, int32_t I,
                              const void* w13, const void* w2, moe_dtype w_dtype,
                              moe_dtype payload_dtype, moe_dtype y_dtype,
                              const moe_layer_options& o, const moe_layer_buffers* b,
                              const void* out) {
    if (!b) return MOE_ERR_INVALID_ARG;
    const int32_t capacity = o.capacity;
    if (capacity >= 0 && (int64_t)E * capacity >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    bool noop;
    moe_status st = MOE_OK;
    if (o.route_groups != 0) st = check_route_groups(E, k, o.route_groups, o.route_max_groups);
    if (st == MOE_OK) st = check_route(logits, T, E, k, b->topk_idx, b->topk_w, &noop);
    if (st == MOE_OK)
        st = check_layout(b->topk_idx, T, k, E, W, b->expert_counts, b->expert_offsets,
                          b->rank_offsets, b->slot_of_pair, b->pair_of_slot,
                          b->layout_workspace, b->layout_workspace_bytes, b->dev_status);
    if (st == MOE_OK)
        st = check_permute(x, x_dtype, T, H, k, b->slot_of_pair, b->xp, payload_dtype,
                           b->xp_scales, &noop);
    if (st == MOE_OK)
        st = check_gemm(b->xp, payload_dtype, b->xp_scales, b->expert_offsets, 0, E,
                        layer_slots(T, k, E, capacity), H, I, w13, w2, w_dtype, b->h, b->y,
                        y_dtype, b->y_scales, b->gemm_workspace, b->gemm_workspace_bytes,
                        b->dev_status,
                        &noop);
    if (st == MOE_OK)
        st = check_combine(b->y, y_dtype, b->y_scales, b->slot_of_pair, b->topk_w, T, k, H, out,
                           x_dtype, &noop);
    // the all_reduce form: W fp32 partials of [T, H]
    if (st == MOE_OK && o.all_reduce_form != 0 && T > 0 && (!b->partials || !aligned16(b->partials)))
        st = MOE_ERR_INVALID_ARG;
    // packed weights and router weights in the GEMM: bf16 weights only
    if (st == MOE_OK && (o.packed_weights != 0 || o.weights_in_gemm != 0) && w_dtype != MOE_BF16)
        st = MOE_ERR_INVALID_ARG;
    // the fused gather's FP8 source, one bf16 row per token, lives in the
    // GEMM workspace
    if (st == MOE_OK && o.fused_gather != 0 && payload_dtype == MOE_E4M3 && T > 0 &&
        (b->gemm_workspace_bytes < (size_t)T * H * 2 || !b->gemm_workspace))
        st = MOE_ERR_INVALID_ARG;
    return st;
}

static cudaError_t launch_layer(const float* logits, const void* x, moe_dtype x_dtype, int64_t T,
                                int32_t H, int32_t E, int32_t k, int32_t W, int32_t I,
                                const void* w13, const void* w2, moe_dtype w_dtype,
                                moe_dtype payload_dtype, moe_dtype y_dtype,
                                const moe_layer_options& o, const moe_layer_buffers* b, void* out,
                                void* const* ev, cudaStream_t s) {
    const int32_t capacity = o.capacity;
    const int64_t n_slots = layer_slots(T, k, E, capacity);
    // Fused gather: the gate/up GEMM reads each routed row from a token-major
    // source (x itself for a bf16 payload; each token's FP8 round trip,
    // bf16(decode(q) * scale), for an FP8 payload) instead of a permuted copy.
    const bool gather = o.fused_gather != 0 && w_dtype == MOE_BF16 && n_slots > 0 &&
                        (o.packed_weights != 0 || grouped_gemm_tc_uses_swap(n_slots, E, y_dtype));
    const gemm_gather gsrc{payload_dtype == MOE_E4M3 ? (const __nv_bfloat16*)b->gemm_workspace
                                                     : (const __nv_bfloat16*)x,
                           b->pair_of_slot, k};
    auto mark = [&](int i) {
        return ev ? cudaEventRecord((cudaEvent_t)ev[i], s) : cudaSuccess;
    };
    cudaError_t e = mark(0);
    if (e == cudaSuccess && T > 0)
        e = launch_route_topk(logits, T, E, k, o.route_groups, o.route_max_groups, b->topk_idx,
                              b->topk_w, s);
    if (e == cudaSuccess) e = mark(1);
    if (e == cudaSuccess)
        e = launch_dispatch_layout(b->topk_idx, T, k, E, W, capacity < 0 ? -1 : capacity,
                                   b->expert_counts, b->expert_offsets, b->rank_offsets,
                                   b->slot_of_pair, b->pair_of_slot,
                                   capacity < 0 ? nullptr : b->n_dropped, b->layout_workspace,
                                   b->dev_status, s);
    if (e == cudaSuccess) e = mark(2);
    if (e == cudaSuccess && T > 0 && gather && payload_dtype == MOE_E4M3)
        e = launch_quantize_tokens_e4m3(x, x_dtype, T, H, (__nv_bfloat16*)b->gemm_workspace, s);
    else if (e == cudaSuccess && T > 0 && !gather)
        e = launch_permute(x, x_dtype, T, H, k, b->slot_of_pair, b->xp, payload_dtype,
                           b->xp_scales,
                           payload_dtype == MOE_E4M3 ? (__nv_bfloat16*)b->gemm_workspace : nullptr,
                           s);
    if (e == cudaSuccess) e = mark(3);
    if (e == cudaSuccess && T > 0 && n_slots > 0) {
        e = run_gemm(b->xp, payload_dtype, b->xp_scales, b->expert_offsets,
                     capacity < 0 ? nullptr : b->expert_counts, 0, E, n_slots, H, I, w13, w2,
                     w_dtype, b->h, b->y, y_dtype, b->y_scales, b->gemm_workspace, b->dev_status,
                     s, ev ? (cudaEvent_t)ev[4] : nullptr, ev ? (cudaEvent_t)ev[5] : nullptr,
                     /*a_ready=*/true, gather ? &gsrc : nullptr, o.packed_weights != 0,
                     o.weights_in_gemm != 0 ? b->topk_w : nullptr,
                     o.weights_in_gemm != 0 ? b->pair_of_slot : nullptr);
    } else if (e == cudaSuccess) {
        e = mark(4);
        if (e == cudaSuccess) e = mark(5);
    }
    if (e == cudaSuccess) e = mark(6);
    // with the router weights applied in the GEMM, the combine is a plain sum
    const float* comb_w = o.weights_in_gemm != 0 ? nullptr : b->topk_w;
    if (e == cudaSuccess && T > 0 && o.all_reduce_form != 0) {
        // each logical rank's partial over its own slab, then their sum in
        // rank order (on W GPUs: the all-reduce) rounded once
        for (int r = 0; r < W && e == cudaSuccess; ++r)
            e = launch_combine(b->y, y_dtype, b->y_scales, b->slot_of_pair, comb_w, T, k, H,
                               b->partials + (int64_t)r * T * H, MOE_F32, s, b->rank_offsets, r);
        if (e == cudaSuccess) e = launch_reduce_partials(b->partials, W, T * H, out, x_dtype, s);
    } else if (e == cudaSuccess && T > 0) {
        e = launch_combine(b->y, y_dtype, b->y_scales, b->slot_of_pair, comb_w, T, k, H, out,
                           x_dtype, s);
    }
    if (e == cudaSuccess) e = mark(7);
    return e;
}

moe_status moe_layer_forward(const float* logits, const void* x, moe_dtype x_dtype, int64_t T,
                             int32_t H, int32_t E, int32_t k, int32_t W, int32_t I,
                             const void* w13, const void* w2, moe_dtype w_dtype,
                             moe_dtype payload_dtype, moe_dtype y_dtype,
                             const moe_layer_options* opts, const moe_layer_buffers* b, void* out,
                             void* const* step_events, void* stream) {
    const moe_layer_options o = resolve(opts);
    const moe_status st = check_layer(logits, x, x_dtype, T, H, E, k, W, I, w13, w2, w_dtype,
                                      payload_dtype, y_dtype, o, b, out);
    if (st != MOE_OK) return st;
    return cuda_status(launch_layer(logits, x, x_dtype, T, H, E, k, W, I, w13, w2, w_dtype,
                                    payload_dtype, y_dtype, o, b, out, step_events,
                                    (cudaStream_t)stream));
}

moe_status moe_layer_forward_host(const float* logits_host, const void* x_host, void* out_host,
                                  float* logits_dev, void* x_dev, void* out_dev,
                                  moe_dtype x_dtype, int64_t T, int32_t H, int32_t E, int32_t k,
                                  int32_t W, int32_t I, const void* w13, const void* w2,
                                  moe_dtype w_dtype, moe_dtype payload_dtype, moe_dtype y_dtype,
                                  const moe_layer_options* opts, const moe_layer_buffers* b,
                                  void* const* step_events, void* stream) {
    const moe_layer_options o = resolve(opts);
    const moe_status st = check_layer(logits_dev, x_dev, x_dtype, T, H, E, k, W, I, w13, w2,
                                      w_dtype, payload_dtype, y_dtype, o, b, out_dev);
    if (st != MOE_OK) return st;
    if (T > 0 && (!logits_host || !x_host || !out_host)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t xb = (x_dtype == MOE_F32 ? 4 : 2) * (size_t)T * H;
    cudaError_t e = cudaSuccess;
    if (T > 0) {
        e = cudaMemcpyAsync(logits_dev, logits_host, sizeof(float) * (size_t)T * E,
                            cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, s);
    }
    if (e == cudaSuccess)
        e = launch_layer(logits_dev, x_dev, x_dtype, T, H, E, k, W, I, w13, w2, w_dtype,
                         payload_dtype, y_dtype, o, b, out_dev, step_events, s);
    if (e == cudaSuccess && T > 0)
        e = cudaMemcpyAsync(out_host, out_dev, xb, cudaMemcpyDeviceToHost, s);
    return cuda_status(e);
}

moe_status moe_check_status(int32_t* dev_status, void* stream) {
    if (!dev_status) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    if (v & MOE_DEV_TIMEOUT) return MOE_ERR_TIMEOUT;
    if (v & MOE_DEV_OVERFLOW) return MOE_ERR_OVERFLOW;
    if (v & MOE_DEV_BAD_INDEX) return MOE_ERR_BAD_INDEX;
    return MOE_OK;
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t moe_diag_layout_wait_timeout_workspace_bytes(void) { return layout_wait_selftest_bytes(); }

moe_status moe_diag_layout_wait_timeout(void* workspace, size_t workspace_bytes,
                                        uint64_t wait_limit_ns, int32_t* dev_status,
                                        void* stream) {
    if (!workspace || !dev_status || !aligned16(workspace) ||
        workspace_bytes < layout_wait_selftest_bytes())
        return MOE_ERR_INVALID_ARG;
    if (wait_limit_ns > kSpinLimitNs) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_layout_wait_selftest(workspace, wait_limit_ns, dev_status,
                                                   (cudaStream_t)stream));
}

const char* moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_BAD_INDEX: return "MOE_ERR_BAD_INDEX";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_OVERFLOW: return "MOE_ERR_OVERFLOW";
    }
    return "MOE_ERR_UNKNOWN";
}

}  // extern "C"
