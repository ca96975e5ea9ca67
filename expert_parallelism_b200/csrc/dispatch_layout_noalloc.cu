// dispatch_layout_noalloc.cu -- moe_dispatch_layout with its scratch in a
// fixed device array inside the library, for callers that cannot allocate.
//
// Some callers have no way to hand the library scratch memory: cudaMalloc
// may synchronise the device, it is not allowed while a stream is being
// captured into a graph, and some host frameworks keep every byte of
// device memory in their own allocator and give extensions no way to ask
// for more.  This entry point needs nothing but the inputs and outputs.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes.
// Every GPU that loads the library holds it until the process exits.  In
// host code the array's name is only a host-side stand-in, not a device
// address, so the set-up below asks the runtime for the real address once
// per device (with that device current) and passes it to the kernels.
#include <mutex>

#include "common.cuh"

namespace moe {
size_t layout_workspace_bytes(int64_t T, int k, int E);
cudaError_t launch_dispatch_layout(const int32_t*, int64_t, int, int, int, int, int32_t*,
                                   int32_t*, int32_t*, int32_t*, int32_t*, int32_t*, void*,
                                   int32_t*, cudaStream_t);
}  // namespace moe

// 2 MiB: enough for E * ceil(T*k / 2048) <= ~262,000, e.g. 256 experts and
// up to ~2 million routed pairs.
static constexpr size_t kNoAllocScratchBytes = 2u << 20;
static __device__ __align__(256) unsigned char g_layout_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device (nullptr on error).
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t moe_dispatch_layout_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

moe_status moe_dispatch_layout_noalloc(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                                       int32_t W, int32_t* expert_counts,
                                       int32_t* expert_offsets, int32_t* rank_offsets,
                                       int32_t* slot_of_pair, int32_t* pair_of_slot,
                                       int32_t* dev_status, void* stream) {
    if (T < 0 || k < 1 || E < 1 || W < 1 || W > E || (E % W) != 0) return MOE_ERR_INVALID_ARG;
    if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
    if (T * (int64_t)k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    if (!expert_counts || !expert_offsets || !rank_offsets || !dev_status)
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !slot_of_pair || !pair_of_slot)) return MOE_ERR_INVALID_ARG;
    if (moe::layout_workspace_bytes(T, k, E) > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
    void* scratch = scratch_on_current_device();
    if (!scratch) return MOE_ERR_CUDA;
    // The scratch keeps the previous call's contents; the first kernel of
    // the layout clears the look-back flags and the ticket itself, and the
    // rest is fully overwritten before it is read.
    const cudaError_t e = moe::launch_dispatch_layout(
        topk_idx, T, k, E, W, -1, expert_counts, expert_offsets, rank_offsets, slot_of_pair,
        pair_of_slot, nullptr, scratch, dev_status, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
