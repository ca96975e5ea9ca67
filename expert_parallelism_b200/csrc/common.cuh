// common.cuh -- shared device helpers for libmoe's sm_100a kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kWarp = 32;

// Bounded waits: every spin in this library gives up after this long
// (device globaltimer, nanoseconds), records MOE_DEV_TIMEOUT and returns.
constexpr uint64_t kSpinLimitNs = 2ull * 1000 * 1000 * 1000;

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void flag_status(int32_t* dev_status, int32_t bits) {
    if (dev_status) atomicOr(dev_status, bits);
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// 16-byte vector of a row: 4 fp32 or 8 bf16 elements.
template <typename T>
struct Vec16 {
    static constexpr int kN = 16 / sizeof(T);
};

__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32.
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
    return *reinterpret_cast<uint32_t*>(&p);
}

// Streaming loads/stores that do not allocate in L1.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// The FP8 payload rule, shared by the dispatch payload (permute) and the
// combine payload (the down GEMM's epilogue): for a block with largest
// magnitude amax, scale = amax / 448 (IEEE fp32 division; 1 for an all-zero
// block), and each value is encoded as e4m3(v / scale) (IEEE division, then
// the hardware's round-to-nearest-even, saturating conversion).
__device__ __forceinline__ float e4m3_block_scale(float amax) {
    const float s = __fdiv_rn(amax, 448.0f);
    return s == 0.0f ? 1.0f : s;
}

// Four e4m3 codes of a / scale .. d / scale, packed low byte first.
__device__ __forceinline__ uint32_t quant4_e4m3(float a, float b, float c, float d, float scale) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(a, scale), __fdiv_rn(b, scale)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(c, scale), __fdiv_rn(d, scale)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// The FP8 combine payload's encoding: four e4m3 codes of a * r .. d * r,
// r = 1 / scale (fp32 products, then the round-to-nearest-even,
// saturating conversion), packed low byte first.
__device__ __forceinline__ uint32_t quant4_e4m3_mul(float a, float b, float c, float d, float r) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(a, r), __fmul_rn(b, r)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(c, r), __fmul_rn(d, r)), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Two e4m3 codes (low byte first) decoded to fp32 (exact: e4m3 values are
// fp16 values).
__device__ __forceinline__ float2 decode2_e4m3(uint16_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// Source of the grouped GEMM's fused gather: row s of the gate/up operand
// is row pair_of_slot[s] / top_k of src (token-major, bf16); a slot holding
// no pair (-1) reads zeros.
struct gemm_gather {
    const __nv_bfloat16* src;
    const int32_t* pair_of_slot;
    int top_k;
};

// Where a routed pair's row lives.  For the single-GPU layout (send_base
// null) it is slot slot_of_pair[p] of the one local buffer (rank 0).  With an
// expert-parallel plan it is row send_base[e] + (slot - expert_offsets[e]) of
// the receive buffer of rank e / experts_per_rank, e = topk_idx[p]: the
// sender's slots for expert e, in order, are consecutive rows of e's owner.
struct PairRows {
    const int32_t* topk_idx;        // [T*k]: expert of each pair (plan only)
    const int32_t* expert_offsets;  // [E+1]: the sender's own layout (plan only)
    const int32_t* send_base;       // [E]: the plan, or null for the local layout
    int experts_per_rank;
    int64_t rows_capacity;          // rows of every rank's receive buffer (plan only)
};

// Resolves pair p in slot `slot` (>= 0) to (rank, row); false when the row
// would fall outside the receive buffer (the pair is then skipped).
__device__ __forceinline__ bool pair_row(const PairRows& m, int64_t p, int32_t slot, int& rank,
                                         int64_t& row) {
    if (!m.send_base) {
        rank = 0;
        row = slot;
        return true;
    }
    const int e = __ldg(m.topk_idx + p);
    rank = e / m.experts_per_rank;
    row = (int64_t)__ldg(m.send_base + e) + slot - __ldg(m.expert_offsets + e);
    return row >= 0 && row < m.rows_capacity;
}

// Base pointers of every rank's buffer (rank 0 only for the local layout;
// peer-mapped device pointers across W GPUs), passed by value as a
// __grid_constant__ kernel parameter.
constexpr int kMaxEpRanks = 64;
struct RankPtrs {
    void* rows[kMaxEpRanks];      // payload or y rows
    float* scales[kMaxEpRanks];   // FP8 block scales, or null
};

// Host-side count of kernel launches (reported by moe_launch_count).
void note_launches(int n);

// MOE_OK for cudaSuccess; otherwise prints the CUDA error and returns
// MOE_ERR_CUDA (every entry point reports CUDA failures this way).
moe_status report_cuda(cudaError_t e);

// The dispatch layout's argument rules other than the caller workspace.
moe_status check_layout_args(const int32_t* topk_idx, int64_t T, int32_t k, int32_t E, int32_t W,
                             const int32_t* expert_counts, const int32_t* expert_offsets,
                             const int32_t* rank_offsets, const int32_t* slot_of_pair,
                             const int32_t* pair_of_slot, const int32_t* dev_status);

}  // namespace moe
