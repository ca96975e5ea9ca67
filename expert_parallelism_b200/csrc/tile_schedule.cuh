// tile_schedule.cuh -- map a linear M-tile index onto (expert, first row)
// for a grouped GEMM whose per-expert row ranges come from device memory.
//
// Expert j (local index) owns rows [off[b + j], off[b + j + 1]) of the
// permuted buffer and contributes ceil(rows_j / BM) M-tiles.  A CTA builds
// the prefix sum of those tile counts in shared memory once, then finds
// the owner of any tile by binary search.  The host never reads the
// offsets, so the GEMM needs no device->host synchronisation.
#pragma once

#include "common.cuh"

namespace moe {

// s_prefix must hold n_experts + 1 ints, s_warp_sums blockDim.x / 32.  Call
// with the whole CTA; contains __syncthreads().  Needs n_experts <= 8 *
// blockDim.x (1024 experts from 128 threads up).
__device__ __forceinline__ void build_tile_prefix(const int32_t* __restrict__ offsets,
                                                  int expert_begin, int n_experts, int BM,
                                                  int32_t* s_prefix, int32_t* s_warp_sums) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int per = (n_experts + nthr - 1) / nthr;   // experts per thread, <= 8
    const int j0 = tid * per;
    int32_t cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int32_t mine = 0;
    for (int i = 0; i < per && i < 8; ++i) {
        const int j = j0 + i;
        if (j < n_experts) {
            const int32_t rows = offsets[expert_begin + j + 1] - offsets[expert_begin + j];
            cnt[i] = rows > 0 ? (rows + BM - 1) / BM : 0;   // a decreasing pair adds nothing
            mine += cnt[i];
        }
    }
    const int lane = tid & 31, warp = tid >> 5, nwarps = (nthr + 31) >> 5;
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
    (void)nwarps;
    __syncthreads();
}

// Local expert owning M-tile mt (0 <= mt < s_prefix[n_experts]).
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
