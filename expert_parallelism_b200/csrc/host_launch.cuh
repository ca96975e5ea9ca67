// host_launch.cuh -- host-side helpers shared by the tensor-core GEMMs: the
// driver's tensor-map encoder (looked up once, thread-safe), a bf16 tiled
// tensor map with 128-byte swizzle, a CTA-pair cluster attribute, and a
// per-device cache for launch-geometry figures (each device keeps its own).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>

namespace moe {

// cuTensorMapEncodeTiled from the driver, through the runtime (the library
// links the runtime statically and does not link the driver library).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            return (PFN_cuTensorMapEncodeTiled_v12000)q;
        return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    }();
    return fn;
}

// Tiled bf16 tensor map of `rank` dimensions (innermost first), 128-byte
// swizzle, out-of-bounds elements read as zero.
inline bool make_bf16_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                          const cuuint64_t* strides_bytes, const cuuint32_t* box) {
    const auto fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint32_t elem[5] = {1, 1, 1, 1, 1};
    const CUresult r =
        fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
           strides_bytes, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Cluster of `ncta` CTAs along x as the launch's only attribute.
inline void set_cluster_attr(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int ncta) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ncta;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

inline int current_device_sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// One cached positive int per device (per instantiation of Tag): computed
// by `f` with that device current the first time it is asked for, then
// reused.  Concurrent first calls may both compute; they store the same
// value.
template <typename Tag>
struct PerDeviceInt {
    static constexpr int kMaxDevices = 64;
    template <typename F>
    static int get(F f) {
        static std::atomic<int> slot[kMaxDevices];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return f();
        int v = slot[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
        v = f();
        if (v > 0) slot[dev].store(v, std::memory_order_relaxed);
        return v;
    }
};

}  // namespace moe
