// route_topk.cu -- router top-k + softmax over the picks (one warp per token).
//
// Source: "Expert parallelism and all-to-all", "Walking through one MoE
// layer", step 1: every token gets a list of (expert, weight) picks.
//
// Each lane holds EPL = ceil(E/32) logits of its token (lane-strided, so
// the row load is coalesced).  k rounds of a warp-wide argmax over the
// key (logit descending, expert id ascending) pick the experts in order;
// the winner's lane marks it taken.  Lane j keeps pick j; the weights are
// a softmax over the k picks, max-subtracted (the first pick is the max).
//
// Group-limited mode ("Expert Parallelism" (aiwiki), "Hiding the latency":
// each token reaches at most M nodes): the experts form G <= 32 equal groups
// of consecutive ids; lane g ends up holding group g's score (its largest
// logit, a warp max per group); M rounds of a warp argmax over (score
// descending, group id ascending) keep M groups, and the experts of the
// other groups leave the candidate set before the top-k rounds.
#include "common.cuh"

namespace moe {

// G == 0 (or M >= G): plain top-k.  Otherwise G | E, G <= 32, 1 <= M < G.
template <int EPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         int64_t T, int E, int k, int G, int M,
                                                         int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + t * E;

    float v[EPL];
    uint32_t avail = 0;  // bit j: logit j of this lane is still a candidate
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
        const int e = j * kWarp + lane;
        v[j] = (e < E) ? __ldg(row + e) : 0.0f;
        if (e < E) avail |= 1u << j;
    }

    if (M < G) {
        const int per = E / G;
        float my_score = 0.0f;                  // lane g < G: group g's largest logit
        for (int g = 0; g < G; ++g) {
            float part = -INFINITY;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const int e = j * kWarp + lane;
                if (e < E && e / per == g) part = fmaxf(part, v[j]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                part = fmaxf(part, __shfl_xor_sync(0xffffffffu, part, off));
            if (lane == g) my_score = part;
        }
        uint32_t kept = 0;                      // bit g: group g kept
        for (int r = 0; r < M; ++r) {
            const bool cand = lane < G && !((kept >> lane) & 1u);
            float bs = my_score;
            int bg = cand ? lane : INT_MAX;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float os = __shfl_xor_sync(0xffffffffu, bs, off);
                const int og = __shfl_xor_sync(0xffffffffu, bg, off);
                const bool better =
                    (og != INT_MAX) && (bg == INT_MAX || os > bs || (os == bs && og < bg));
                if (better) {
                    bs = os;
                    bg = og;
                }
            }
            if (bg != INT_MAX) kept |= 1u << bg;
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = j * kWarp + lane;
            if (e < E && !((kept >> (e / per)) & 1u)) avail &= ~(1u << j);
        }
    }

    float my_v = 0.0f;
    int my_e = 0;
    for (int r = 0; r < k; ++r) {
        // this lane's best candidate: ids grow with j, so a strict '>' keeps
        // the lower id on equal logits
        float bv = 0.0f;
        int be = INT_MAX;  // INT_MAX = no candidate
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            if (((avail >> j) & 1u) && (be == INT_MAX || v[j] > bv)) {
                bv = v[j];
                be = j * kWarp + lane;
            }
        }
        // warp argmax under the same total order
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            const bool better = (oe != INT_MAX) &&
                                (be == INT_MAX || ov > bv || (ov == bv && oe < be));
            if (better) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & (kWarp - 1)) == lane) avail &= ~(1u << (be / kWarp));
        if (lane == r) {
            my_v = bv;
            my_e = be;
        }
    }

    const float m = __shfl_sync(0xffffffffu, my_v, 0);  // first pick = max logit
    const float z = (lane < k) ? expf(my_v - m) : 0.0f;
    float sum = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
        topk_idx[t * k + lane] = my_e;
        topk_w[t * k + lane] = __fdiv_rn(z, sum);
    }
}

cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int G, int M,
                              int32_t* idx, float* w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int warps_per_block = 8;
    const dim3 grid((unsigned)((T + warps_per_block - 1) / warps_per_block));
    const dim3 block(warps_per_block * kWarp);
    const int epl = (E + kWarp - 1) / kWarp;
    if (epl <= 1) route_topk_kernel<1><<<grid, block, 0, s>>>(logits, T, E, k, G, M, idx, w);
    else if (epl <= 2) route_topk_kernel<2><<<grid, block, 0, s>>>(logits, T, E, k, G, M, idx, w);
    else if (epl <= 4) route_topk_kernel<4><<<grid, block, 0, s>>>(logits, T, E, k, G, M, idx, w);
    else if (epl <= 8) route_topk_kernel<8><<<grid, block, 0, s>>>(logits, T, E, k, G, M, idx, w);
    else if (epl <= 16) route_topk_kernel<16><<<grid, block, 0, s>>>(logits, T, E, k, G, M, idx, w);
    else route_topk_kernel<32><<<grid, block, 0, s>>>(logits, T, E, k, G, M, idx, w);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
