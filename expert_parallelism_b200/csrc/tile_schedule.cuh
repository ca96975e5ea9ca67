// tile_schedule.cuh -- map a linear M-tile index onto (expert, first row)
// for a grouped GEMM whose per-expert row ranges come from device memory.
//
// Expert j (local index) owns rows [off[b + j], off[b + j + 1]) of the
// permuted buffer (or their first counts[b + j]) and contributes
// ceil(rows_j / BM) M-tiles.  A CTA builds
// the prefix sum of those tile counts in shared memory once, then finds
// the owner of any tile by binary search.  The host never reads the
// offsets, so the GEMM needs no device->host synchronisation.
#pragma once

#include "common.cuh"

namespace moe {

// Rows expert j (local index) computes: its segment [off[b+j], off[b+j+1]),
// cut to counts[b+j] rows when counts is given (fixed-capacity slabs whose
// tail rows hold no pair).  A decreasing offset pair counts as 0 rows.
__device__ __forceinline__ int32_t segment_rows(const int32_t* __restrict__ offsets,
                                                const int32_t* __restrict__ counts,
                                                int expert_begin, int j) {
    const int32_t span = offsets[expert_begin + j + 1] - offsets[expert_begin + j];
    const int32_t rows = counts ? min(span, counts[expert_begin + j]) : span;
    return rows > 0 ? rows : 0;
}

// Prefix sum over the local experts of units_of(rows_j) (the work units
// expert j contributes), into s_prefix[0..n_experts].  s_prefix must hold
// n_experts + 1 ints, s_warp_sums blockDim.x / 32.  Call with the whole CTA;
// contains __syncthreads().  Needs n_experts <= 8 * blockDim.x (1024 experts
// from 128 threads up).
template <typename UnitsOf>
__device__ __forceinline__ void build_unit_prefix(const int32_t* __restrict__ offsets,
                                                  const int32_t* __restrict__ counts,
                                                  int expert_begin, int n_experts, UnitsOf units_of,
                                                  int32_t* s_prefix, int32_t* s_warp_sums) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int per = (n_experts + nthr - 1) / nthr;   // experts per thread, <= 8
    const int j0 = tid * per;
    int32_t cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int32_t mine = 0;
    for (int i = 0; i < per && i < 8; ++i) {
        const int j = j0 + i;
        if (j < n_experts) {
            const int32_t rows = segment_rows(offsets, counts, expert_begin, j);
            cnt[i] = rows > 0 ? units_of(rows) : 0;
            mine += cnt[i];
        }
    }
    const int lane = tid & 31, warp = tid >> 5;
    int32_t incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp_sums[warp] = incl;
    __syncthreads();
    int32_t run = incl - mine;
    for (int w = 0; w < warp; ++w) run += s_warp_sums[w];
    if (tid == 0) s_prefix[0] = 0;
    for (int i = 0; i < per && i < 8; ++i) {
        const int j = j0 + i;
        if (j < n_experts) {
            run += cnt[i];
            s_prefix[j + 1] = run;
        }
    }
    __syncthreads();
}

struct CeilDiv {
    int32_t d;
    __device__ __forceinline__ int32_t operator()(int32_t rows) const { return (rows + d - 1) / d; }
};

// M-tiles of BM rows: expert j contributes ceil(rows_j / BM).
__device__ __forceinline__ void build_tile_prefix(const int32_t* __restrict__ offsets,
                                                  const int32_t* __restrict__ counts,
                                                  int expert_begin, int n_experts, int BM,
                                                  int32_t* s_prefix, int32_t* s_warp_sums) {
    build_unit_prefix(offsets, counts, expert_begin, n_experts, CeilDiv{BM}, s_prefix,
                      s_warp_sums);
}

// Local expert owning unit mt (0 <= mt < s_prefix[n_experts]).
__device__ __forceinline__ int find_tile_expert(const int32_t* s_prefix, int n_experts, int mt) {
    int lo = 0, hi = n_experts - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_prefix[mid] <= mt) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

}  // namespace moe
