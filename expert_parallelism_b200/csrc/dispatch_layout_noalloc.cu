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
// per device (with that device current), again if the device's current
// context changes, and passes it to the kernels.
#include <cuda.h>

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

// What the set-up found on each device: the array's address, valid in the
// context that was current when it was looked up.
struct ScratchAddr {
    CUcontext ctx;
    void* ptr;
};
ScratchAddr g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent from the driver, through the runtime (looked up once).
CtxGetCurrentFn ctx_get_current() {
    static const CtxGetCurrentFn fn = [] {
        void* q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &q, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            return (CtxGetCurrentFn)q;
        return (CtxGetCurrentFn) nullptr;
    }();
    return fn;
}

// Device address of g_layout_scratch on the current device, looked up (with
// that device current) on the first call and again whenever the current
// context is not the one of the last lookup (after cudaDeviceReset, or with
// another context made current).  Returns the CUDA error of a failed lookup.
cudaError_t scratch_on_current_device(void** out) {
    *out = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const CtxGetCurrentFn get = ctx_get_current();
    if (!get) return cudaErrorInitializationError;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchAddr& s = g_scratch[dev];
    if (!s.ptr || !ctx || s.ctx != ctx) {
        // the lookup also brings up the runtime's context on this device
        // when none is current yet; the context is read again after it
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_layout_scratch);
        if (e != cudaSuccess) return e;
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorInitializationError;
        s.ctx = ctx;
        s.ptr = p;
    }
    *out = s.ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t moe_dispatch_layout_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

moe_status moe_dispatch_layout_noalloc(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E,
                                       int32_t W, int32_t* expert_counts,
                                       int32_t* expert_offsets, int32_t* rank_offsets,
                                       int32_t* slot_of_pair, int32_t* pair_of_slot,
                                       int32_t* dev_status, void* stream) {
    const moe_status st = moe::check_layout_args(topk_idx, T, k, E, W, expert_counts,
                                                 expert_offsets, rank_offsets, slot_of_pair,
                                                 pair_of_slot, dev_status);
    if (st != MOE_OK) return st;
    if (moe::layout_workspace_bytes(T, k, E) > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    cudaError_t e = scratch_on_current_device(&scratch);
    // The scratch keeps the previous call's contents; the first kernel of
    // the layout clears the look-back flags and the ticket itself, and the
    // rest is fully overwritten before it is read.
    if (e == cudaSuccess)
        e = moe::launch_dispatch_layout(topk_idx, T, k, E, W, -1, expert_counts, expert_offsets,
                                        rank_offsets, slot_of_pair, pair_of_slot, nullptr, scratch,
                                        dev_status, (cudaStream_t)stream);
    return moe::report_cuda(e);
}

}  // extern "C"
