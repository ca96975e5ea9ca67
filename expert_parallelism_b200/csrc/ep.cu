// ep.cu -- expert parallelism over W ranks: the dispatch plan from the
// exchanged counts, and the entry points that send each routed row to its
// expert's owner (dispatch) and bring the experts' outputs back (combine).
//
// Source: "Expert Parallelism" (aiwiki), "The two all-to-alls" (one
// all-to-all sends every token's row to the ranks that own its experts, a
// second one returns the outputs) and "Implementation" (a count exchange
// first tells each owner how many rows will arrive); "Expert parallelism and
// all-to-all", "Walking through one MoE layer", steps 2 and 4; ownership:
// "Expert parallelism" (Transformers docs), "How the sizes combine".
//
// Receive layout: an owner's buffer holds its experts one after the other,
// and inside an expert the rows of rank 0, then rank 1, ..., each in the
// sender's own slot order, so each local expert is one contiguous segment
// for the grouped GEMM.  A sender's rows for expert e are its slots
// [expert_offsets[e], expert_offsets[e+1]) and land, in order, from row
// send_base[e] of the owner's buffer.
//
// The data moves as plain stores (dispatch) and plain loads (combine)
// through a table of every rank's buffer: peer-mapped device pointers when
// the ranks are GPUs of one NVLink domain, or W buffers of one GPU when the
// ranks are run on one device.  No TMA and no cluster multicast touch
// another GPU's memory; the grouped GEMM reads only the local receive
// buffer.
#include <cuda.h>
#include <string.h>

#include "common.cuh"

namespace moe {

cudaError_t launch_permute_to(const void* x, moe_dtype xdt, int64_t T, int H, int k,
                              const int32_t* slot_of_pair, const PairRows& map,
                              const RankPtrs& dst, moe_dtype xpdt, __nv_bfloat16* a_bf16,
                              int32_t* dev_status, cudaStream_t s);
cudaError_t launch_combine_from(const RankPtrs& src, moe_dtype ydt, const int32_t* slot_of_pair,
                                const PairRows& map, const float* topk_w, int64_t T, int k, int H,
                                void* out, moe_dtype odt, int32_t* dev_status, cudaStream_t s,
                                const int32_t* rank_offsets, int rank);

constexpr int kPlanThreads = 1024;

// One CTA.  counts_all [W, E]: rows rank s routes to expert e.  For `rank`:
//   send_base[e] = (rows of owner(e)'s experts before e, all sources)
//                + (rows of e from ranks before `rank`),
//   recv_offsets[j] = rows of this rank's local experts before j, all
//                     sources (j = 0..Er).
// Negative counts are read as 0 and flagged (MOE_DEV_BAD_INDEX).
__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(const int32_t* __restrict__ counts_all,
                                                              int W, int E, int rank,
                                                              int32_t* __restrict__ send_base,
                                                              int32_t* __restrict__ recv_offsets,
                                                              int32_t* dev_status) {
    extern __shared__ int32_t s_tot[];   // [E]: rows of expert e over all sources
    const int Er = E / W;
    bool bad = false;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t tot = 0;
        for (int s = 0; s < W; ++s) {
            const int32_t c = counts_all[(int64_t)s * E + e];
            bad |= c < 0;
            tot += c > 0 ? c : 0;
        }
        s_tot[e] = tot;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(dev_status, MOE_DEV_BAD_INDEX);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int first = (e / Er) * Er;          // owner's first expert
        int32_t row = 0;
        for (int q = first; q < e; ++q) row += s_tot[q];
        for (int s = 0; s < rank; ++s) {
            const int32_t c = counts_all[(int64_t)s * E + e];
            row += c > 0 ? c : 0;
        }
        send_base[e] = row;
    }
    for (int j = threadIdx.x; j <= Er; j += blockDim.x) {
        int32_t row = 0;
        for (int q = rank * Er; q < rank * Er + j; ++q) row += s_tot[q];
        recv_offsets[j] = row;
    }
}

cudaError_t launch_ep_plan(const int32_t* counts_all, int W, int E, int rank, int32_t* send_base,
                           int32_t* recv_offsets, int32_t* dev_status, cudaStream_t s) {
    const size_t smem = (size_t)E * 4;
    ep_plan_kernel<<<1, kPlanThreads, smem, s>>>(counts_all, W, E, rank, send_base, recv_offsets,
                                                 dev_status);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool act_dtype(moe_dtype d) { return d == MOE_F32 || d == MOE_BF16; }

// Table of W buffers (and their block scales when `need_scales`), checked:
// every pointer non-null and 16-byte aligned.
bool fill_table(moe::RankPtrs& t, int W, void* const* rows, float* const* scales,
                bool need_scales) {
    t = moe::RankPtrs{};
    if (!rows || (need_scales && !scales)) return false;
    for (int r = 0; r < W; ++r) {
        if (!rows[r] || !aligned16(rows[r])) return false;
        t.rows[r] = rows[r];
        if (need_scales) {
            if (!scales[r] || !aligned16(scales[r])) return false;
            t.scales[r] = scales[r];
        }
    }
    return true;
}

moe_status check_ep_shape(int64_t T, int32_t H, int32_t k, int32_t E, int32_t W,
                          int64_t rows_capacity) {
    if (T < 0 || H < 1 || (H % 8) != 0 || k < 1 || E < 1 || W < 1 || (E % W) != 0 ||
        rows_capacity < 0)
        return MOE_ERR_INVALID_ARG;
    if (W > moe::kMaxEpRanks || E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK)
        return MOE_ERR_UNSUPPORTED;
    if (rows_capacity >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_ep_plan(const int32_t* counts_all, int32_t W, int32_t E, int32_t rank,
                       int32_t* send_base, int32_t* recv_offsets, int32_t* dev_status,
                       void* stream) {
    if (W < 1 || E < 1 || (E % W) != 0 || rank < 0 || rank >= W) return MOE_ERR_INVALID_ARG;
    if (W > moe::kMaxEpRanks || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (!counts_all || !send_base || !recv_offsets || !dev_status) return MOE_ERR_INVALID_ARG;
    return moe::report_cuda(moe::launch_ep_plan(counts_all, W, E, rank, send_base, recv_offsets,
                                                dev_status, (cudaStream_t)stream));
}

moe_status moe_ep_dispatch(const void* x, moe_dtype x_dtype, int64_t T, int32_t H, int32_t k,
                           const int32_t* topk_idx, const int32_t* slot_of_pair,
                           const int32_t* expert_offsets, const int32_t* send_base, int32_t E,
                           int32_t W, void* const* recv_rows, float* const* recv_scales,
                           moe_dtype payload_dtype, int64_t rows_capacity, int32_t* dev_status,
                           void* stream) {
    moe_status st = check_ep_shape(T, H, k, E, W, rows_capacity);
    if (st != MOE_OK) return st;
    if (!act_dtype(x_dtype) || (payload_dtype != x_dtype && payload_dtype != MOE_E4M3))
        return MOE_ERR_INVALID_ARG;
    const bool fp8 = payload_dtype == MOE_E4M3;
    if (fp8 && (H % 128) != 0) return MOE_ERR_INVALID_ARG;
    moe::RankPtrs dst;
    if (!fill_table(dst, W, recv_rows, recv_scales, fp8)) return MOE_ERR_INVALID_ARG;
    if (!topk_idx || !slot_of_pair || !expert_offsets || !send_base || !dev_status)
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    const moe::PairRows map{topk_idx, expert_offsets, send_base, E / W, rows_capacity};
    return moe::report_cuda(moe::launch_permute_to(x, x_dtype, T, H, k, slot_of_pair, map, dst,
                                                   payload_dtype, nullptr, dev_status,
                                                   (cudaStream_t)stream));
}

moe_status moe_ep_combine(void* const* y_rows, float* const* y_scales, moe_dtype y_dtype,
                          const int32_t* topk_idx, const int32_t* slot_of_pair,
                          const int32_t* expert_offsets, const int32_t* send_base,
                          const float* topk_w, int64_t T, int32_t k, int32_t H, int32_t E,
                          int32_t W, int64_t rows_capacity, void* out, moe_dtype out_dtype,
                          int32_t* dev_status, void* stream) {
    moe_status st = check_ep_shape(T, H, k, E, W, rows_capacity);
    if (st != MOE_OK) return st;
    if (!(act_dtype(y_dtype) || y_dtype == MOE_E4M3) || !act_dtype(out_dtype))
        return MOE_ERR_INVALID_ARG;
    const bool fp8 = y_dtype == MOE_E4M3;
    if (fp8 && (H % 128) != 0) return MOE_ERR_INVALID_ARG;
    moe::RankPtrs src;
    if (!fill_table(src, W, y_rows, y_scales, fp8)) return MOE_ERR_INVALID_ARG;
    if (!topk_idx || !slot_of_pair || !expert_offsets || !send_base || !dev_status)
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!topk_w || !out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const moe::PairRows map{topk_idx, expert_offsets, send_base, E / W, rows_capacity};
    return moe::report_cuda(moe::launch_combine_from(src, y_dtype, slot_of_pair, map, topk_w, T,
                                                     k, H, out, out_dtype, dev_status,
                                                     (cudaStream_t)stream, nullptr, 0));
}

}  // extern "C"

// ---------------------------------------------------------------- buffer sharing
// A rank hands its receive and output buffers to the other processes as
// CUDA IPC handles (the allocation's handle plus the buffer's offset inside
// it), and maps theirs the same way; the mapped addresses fill the buffer
// tables of moe_ep_dispatch and moe_ep_combine.  No multicast object is
// created.

namespace {

struct IpcRecord {
    cudaIpcMemHandle_t handle;
    uint64_t offset;
};

using MemGetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

MemGetAddressRangeFn mem_get_address_range() {
    static const MemGetAddressRangeFn fn = [] {
        void* q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &q, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            return (MemGetAddressRangeFn)q;
        return (MemGetAddressRangeFn) nullptr;
    }();
    return fn;
}

}  // namespace

extern "C" {

size_t moe_ipc_handle_bytes(void) { return sizeof(IpcRecord); }

moe_status moe_ipc_export(const void* ptr, void* record) {
    if (!ptr || !record) return MOE_ERR_INVALID_ARG;
    const MemGetAddressRangeFn range = mem_get_address_range();
    if (!range) return moe::report_cuda(cudaErrorInitializationError);
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, (CUdeviceptr)ptr) != CUDA_SUCCESS)
        return moe::report_cuda(cudaErrorInvalidValue);
    IpcRecord rec{};
    const cudaError_t e = cudaIpcGetMemHandle(&rec.handle, (void*)base);
    if (e != cudaSuccess) return moe::report_cuda(e);
    rec.offset = (uint64_t)((CUdeviceptr)ptr - base);
    memcpy(record, &rec, sizeof(rec));
    return MOE_OK;
}

moe_status moe_ipc_import(const void* record, void** ptr) {
    if (!record || !ptr) return MOE_ERR_INVALID_ARG;
    IpcRecord rec;
    memcpy(&rec, record, sizeof(rec));
    void* base = nullptr;
    const cudaError_t e =
        cudaIpcOpenMemHandle(&base, rec.handle, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return moe::report_cuda(e);
    *ptr = (char*)base + rec.offset;
    return MOE_OK;
}

moe_status moe_ipc_close(const void* record, void* ptr) {
    if (!record || !ptr) return MOE_ERR_INVALID_ARG;
    IpcRecord rec;
    memcpy(&rec, record, sizeof(rec));
    return moe::report_cuda(cudaIpcCloseMemHandle((char*)ptr - rec.offset));
}

}  // extern "C"
