// dispatch_layout.cu -- per-expert histogram, exclusive scan and stable
// expert-major slot assignment of the routed (token, expert) pairs.
//
// Source: "Expert Parallelism" (aiwiki), "Implementation": sort the local
// tokens by destination so each peer's rows form one slab, and count rows
// per rank; the sort is stable (ties by pair index).  Ranks own
// consecutive expert blocks ("Expert parallelism" (Transformers docs),
// "How the sizes combine"), so expert-major order is rank-major.
//
// Three launches on the caller's stream, no host synchronisation:
//   1. layout_hist     one CTA per tile of kTilePairs pairs: shared-memory
//                      atomic histogram -> counts[e * nt + b] (expert-major).
//   2. layout_scan     single-pass exclusive scan of counts[] in that
//                      expert-major order with decoupled look-back between
//                      chunks: base[e * nt + b] = slot of tile b's first
//                      pair routed to expert e.
//   3. layout_scatter  one CTA per tile: a stable in-tile rank per pair
//                      (warps walk their pairs in order, __match_any_sync
//                      groups equal experts inside each 32-pair step, warp
//                      counts are scanned across warps), slot = base +
//                      rank; writes slot_of_pair / pair_of_slot, and CTA 0
//                      writes the counts, offsets and rank offsets.
//
// Fixed-capacity mode (C >= 0; "Expert Parallelism" (aiwiki),
// "Implementation", closing note: fixed buffers make every size known in
// advance at the price of the tokens that do not fit): expert e owns the
// slab [e*C, (e+1)*C).  A pair's rank among its expert's pairs is its
// dropless slot minus the expert's dropless start; ranks below C keep that
// place in the slab, later pairs are dropped (slot -1).  The same three
// launches, the scatter doing the remap.
#include "common.cuh"

namespace moe {

constexpr int kLayoutThreads = 256;                       // 8 warps
constexpr int kLayoutWarps = kLayoutThreads / kWarp;
constexpr int kGroupsPerWarp = 8;                          // 8 x 32 pairs per warp
constexpr int kTilePairs = kLayoutWarps * kGroupsPerWarp * kWarp;  // 2048
constexpr int kScanThreads = 256;
constexpr int kScanItems = 16;
constexpr int kScanChunk = kScanThreads * kScanItems;      // 4096

// look-back status word: flag in the high 32 bits, value in the low 32
constexpr unsigned long long kFlagAggregate = 1ull << 32;
constexpr unsigned long long kFlagInclusive = 2ull << 32;

struct LayoutWorkspace {
    unsigned long long* status;  // [nchunks]
    int32_t* ticket;             // [1]
    int32_t* counts;             // [L]
    int32_t* base;               // [L]
    int64_t nt, L, nchunks;
};

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static LayoutWorkspace carve(void* ws, int64_t T, int k, int E) {
    LayoutWorkspace w;
    const int64_t N = T * k;
    w.nt = N > 0 ? (N + kTilePairs - 1) / kTilePairs : 1;
    w.L = (int64_t)E * w.nt;
    w.nchunks = (w.L + kScanChunk - 1) / kScanChunk;
    char* p = (char*)ws;
    w.status = (unsigned long long*)p;
    p += align_up((size_t)w.nchunks * 8, 16);
    w.ticket = (int32_t*)p;
    p += 16;
    w.counts = (int32_t*)p;
    p += align_up((size_t)w.L * 4, 16);
    w.base = (int32_t*)p;
    return w;
}

size_t layout_workspace_bytes(int64_t T, int k, int E) {
    LayoutWorkspace w = carve(nullptr, T, k, E);
    return align_up((size_t)w.nchunks * 8, 16) + 16 + 2 * align_up((size_t)w.L * 4, 16);
}

__global__ void __launch_bounds__(kLayoutThreads) layout_hist_kernel(
    const int32_t* __restrict__ idx, int64_t N, int E, int64_t nt,
    int32_t* __restrict__ counts, unsigned long long* __restrict__ status, int64_t nchunks,
    int32_t* __restrict__ ticket, int32_t* __restrict__ dev_status) {
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    if (blockIdx.x == 0) {
        for (int64_t c = threadIdx.x; c < nchunks; c += blockDim.x) status[c] = 0ull;
        if (threadIdx.x == 0) *ticket = 0;
    }
    __syncthreads();
    const int64_t b = blockIdx.x;
    const int64_t p0 = b * kTilePairs, p1 = min(N, p0 + kTilePairs);
    int bad = 0;
    for (int64_t p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        const int e = __ldg(idx + p);
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else bad = 1;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag_status(dev_status, MOE_DEV_BAD_INDEX);
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)e * nt + b] = hist[e];
}

// wait_limit_ns bounds each chunk's look-back wait (the library passes
// kSpinLimitNs); a chunk number at or past nchunks does nothing.
__global__ void __launch_bounds__(kScanThreads) layout_scan_kernel(
    const int32_t* __restrict__ counts, int32_t* __restrict__ base, int64_t L,
    unsigned long long* status, int64_t nchunks, int32_t* ticket, int32_t* dev_status,
    uint64_t wait_limit_ns) {
    __shared__ int32_t s_chunk, s_prefix;
    __shared__ int32_t s_warp[kScanThreads / kWarp];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // chunks are numbered in the order CTAs start, so every predecessor a
    // chunk waits for is already running: the look-back cannot deadlock
    if (tid == 0) s_chunk = atomicAdd(ticket, 1);
    __syncthreads();
    const int64_t c = s_chunk;
    if (c >= nchunks) return;
    const int64_t i0 = c * kScanChunk + (int64_t)tid * kScanItems;
    int32_t v[kScanItems];
    int32_t mine = 0;
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
        v[i] = (i0 + i < L) ? counts[i0 + i] : 0;
        mine += v[i];
    }
    // block-wide exclusive scan of the per-thread sums
    int32_t incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int32_t warp_excl = 0, total = 0;
    for (int w = 0; w < kScanThreads / kWarp; ++w) {
        if (w < warp) warp_excl += s_warp[w];
        total += s_warp[w];
    }
    if (tid == 0) {
        int32_t excl = 0;
        if (c == 0) {
            atomicExch(&status[0], kFlagInclusive | (uint32_t)total);
        } else {
            atomicExch(&status[c], kFlagAggregate | (uint32_t)total);
            const uint64_t deadline = global_timer_ns() + wait_limit_ns;
            int64_t j = c - 1;
            while (j >= 0) {
                const unsigned long long st = *((volatile unsigned long long*)&status[j]);
                const unsigned long long flag = st & 0xFFFFFFFF00000000ull;
                if (flag == 0ull) {
                    if (global_timer_ns() >= deadline) {
                        flag_status(dev_status, MOE_DEV_TIMEOUT);
                        break;
                    }
                    __nanosleep(64);
                    continue;
                }
                excl += (int32_t)(st & 0xFFFFFFFFull);
                if (flag == kFlagInclusive) break;
                --j;
            }
            atomicExch(&status[c], kFlagInclusive | (uint32_t)(excl + total));
        }
        s_prefix = excl;
    }
    __syncthreads();
    int32_t run = s_prefix + warp_excl + (incl - mine);
#pragma unroll
    for (int i = 0; i < kScanItems; ++i) {
        if (i0 + i < L) base[i0 + i] = run;
        run += v[i];
    }
}

// C < 0: dropless.  C >= 0: fixed slabs of C rows (pair_of_slot has E*C
// entries); n_dropped (may be null) receives the number of dropped pairs.
__global__ void __launch_bounds__(kLayoutThreads) layout_scatter_kernel(
    const int32_t* __restrict__ idx, int64_t N, int E, int W, int64_t nt,
    const int32_t* __restrict__ counts, const int32_t* __restrict__ base, int64_t L, int C,
    int32_t* __restrict__ expert_counts, int32_t* __restrict__ expert_offsets,
    int32_t* __restrict__ rank_offsets, int32_t* __restrict__ slot_of_pair,
    int32_t* __restrict__ pair_of_slot, int32_t* __restrict__ n_dropped) {
    extern __shared__ int32_t sm[];
    int32_t* wcount = sm;                      // [warps][E]: counts, then warp prefixes
    int32_t* s_base = sm + kLayoutWarps * E;   // [E]: base of this tile per expert
    int32_t* s_start = s_base + E;             // [E + 1]: dropless start of each expert
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t b = blockIdx.x;
    const int32_t total = base[L - 1] + counts[L - 1];
    const bool capped = C >= 0;

    for (int i = tid; i < kLayoutWarps * E; i += blockDim.x) wcount[i] = 0;
    for (int e = tid; e < E; e += blockDim.x) s_base[e] = base[(int64_t)e * nt + b];
    if (capped)
        for (int e = tid; e <= E; e += blockDim.x)
            s_start[e] = (e < E) ? base[(int64_t)e * nt] : total;
    __syncthreads();

    // pass 1: each warp walks its pairs in order; equal experts inside a
    // 32-pair step are ranked by lane, steps are ranked by a running count
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int64_t pw = b * kTilePairs + (int64_t)warp * (kGroupsPerWarp * kWarp);
    int32_t rank[kGroupsPerWarp];
    int32_t ex[kGroupsPerWarp];
#pragma unroll
    for (int g = 0; g < kGroupsPerWarp; ++g) {
        const int64_t p = pw + g * kWarp + lane;
        int e = (p < N) ? __ldg(idx + p) : -1;
        if (e < 0 || e >= E) e = -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int32_t c = (e >= 0) ? wcount[warp * E + e] : 0;
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1) wcount[warp * E + e] = c + __popc(peers);
        __syncwarp();
        rank[g] = c + __popc(peers & lt_mask);
        ex[g] = e;
    }
    __syncthreads();
    // exclusive prefix of the warp counts, per expert
    for (int e = tid; e < E; e += blockDim.x) {
        int32_t run = 0;
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int32_t t = wcount[w * E + e];
            wcount[w * E + e] = run;
            run += t;
        }
    }
    __syncthreads();
    // pass 2: slots
#pragma unroll
    for (int g = 0; g < kGroupsPerWarp; ++g) {
        const int64_t p = pw + g * kWarp + lane;
        if (p >= N) continue;
        const int e = ex[g];
        if (e < 0) {
            slot_of_pair[p] = -1;
            continue;
        }
        int32_t s = s_base[e] + wcount[warp * E + e] + rank[g];
        if (capped) {
            const int32_t pos = s - s_start[e];      // rank among the expert's pairs
            s = pos < C ? e * C + pos : -1;
        }
        slot_of_pair[p] = s;
        if (s >= 0) pair_of_slot[s] = (int32_t)p;
    }
    if (capped) {
        // slab rows past each expert's kept pairs
        const int64_t rows = (int64_t)E * C;
        for (int64_t s = b * blockDim.x + tid; s < rows; s += nt * blockDim.x) {
            const int e = (int)(s / C);
            const int32_t kept = min(s_start[e + 1] - s_start[e], C);
            if (s - (int64_t)e * C >= kept) pair_of_slot[s] = -1;
        }
        if (b == 0) {
            int32_t drop = 0;
            for (int e = tid; e < E; e += blockDim.x) {
                const int32_t cnt = s_start[e + 1] - s_start[e];
                expert_counts[e] = min(cnt, C);
                drop += max(cnt - C, 0);
            }
            for (int e = tid; e <= E; e += blockDim.x) expert_offsets[e] = e * C;
            for (int r = tid; r <= W; r += blockDim.x)
                rank_offsets[r] = (int32_t)((int64_t)r * E / W) * C;
            drop = __reduce_add_sync(0xffffffffu, drop);
            __syncthreads();                         // wcount is free again
            if (lane == 0) wcount[warp] = drop;
            __syncthreads();
            if (tid == 0 && n_dropped) {
                int32_t sum = 0;
                for (int w = 0; w < kLayoutWarps; ++w) sum += wcount[w];
                *n_dropped = sum;
            }
        }
        return;
    }
    // slots past the last routed row (only when ids were skipped)
    for (int64_t s = (int64_t)total + b * blockDim.x + tid; s < N; s += nt * blockDim.x)
        pair_of_slot[s] = -1;
    if (b == 0) {
        for (int e = tid; e <= E; e += blockDim.x) {
            const int32_t lo = (e < E) ? base[(int64_t)e * nt] : total;
            expert_offsets[e] = lo;
            if (e < E) {
                const int32_t hi = (e + 1 < E) ? base[(int64_t)(e + 1) * nt] : total;
                expert_counts[e] = hi - lo;
            }
        }
        for (int r = tid; r <= W; r += blockDim.x) {
            const int e = (int)((int64_t)r * E / W);
            rank_offsets[r] = (e < E) ? base[(int64_t)e * nt] : total;
        }
    }
}

cudaError_t launch_dispatch_layout(const int32_t* idx, int64_t T, int k, int E, int W, int C,
                                   int32_t* expert_counts, int32_t* expert_offsets,
                                   int32_t* rank_offsets, int32_t* slot_of_pair,
                                   int32_t* pair_of_slot, int32_t* n_dropped, void* workspace,
                                   int32_t* dev_status, cudaStream_t s) {
    const int64_t N = T * k;
    LayoutWorkspace w = carve(workspace, T, k, E);
    const size_t hist_smem = (size_t)E * 4;
    const size_t scatter_smem = ((size_t)(kLayoutWarps + 2) * E + 1) * 4;
    if (scatter_smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(
            layout_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)scatter_smem);
        if (err != cudaSuccess) return err;
    }
    layout_hist_kernel<<<(unsigned)w.nt, kLayoutThreads, hist_smem, s>>>(
        idx, N, E, w.nt, w.counts, w.status, w.nchunks, w.ticket, dev_status);
    layout_scan_kernel<<<(unsigned)w.nchunks, kScanThreads, 0, s>>>(
        w.counts, w.base, w.L, w.status, w.nchunks, w.ticket, dev_status, kSpinLimitNs);
    layout_scatter_kernel<<<(unsigned)w.nt, kLayoutThreads, scatter_smem, s>>>(
        idx, N, E, W, w.nt, w.counts, w.base, w.L, C, expert_counts, expert_offsets,
        rank_offsets, slot_of_pair, pair_of_slot, n_dropped);
    note_launches(3);
    return cudaGetLastError();
}

// Look-back state of a two-chunk scan in which chunk 0 never runs: the
// ticket starts at 1, so the one CTA launched becomes chunk 1 and waits for
// status[0], which nothing sets.  Counts are zero.
__global__ void layout_wait_selftest_init_kernel(unsigned long long* status, int32_t* ticket,
                                                 int32_t* counts, int64_t L) {
    for (int64_t i = threadIdx.x; i < L; i += blockDim.x) counts[i] = 0;
    if (threadIdx.x < 2) status[threadIdx.x] = 0ull;
    if (threadIdx.x == 0) *ticket = 1;
}

size_t layout_wait_selftest_bytes() {
    const int64_t L = 2 * kScanChunk;
    return align_up(2 * 8, 16) + 16 + 2 * align_up((size_t)L * 4, 16);
}

// The scan kernel itself, on that state, with the given wait limit: its
// look-back wait runs out and MOE_DEV_TIMEOUT is OR-ed into dev_status.
cudaError_t launch_layout_wait_selftest(void* workspace, uint64_t wait_limit_ns,
                                        int32_t* dev_status, cudaStream_t s) {
    const int64_t L = 2 * kScanChunk;
    char* p = (char*)workspace;
    unsigned long long* status = (unsigned long long*)p;
    p += align_up(2 * 8, 16);
    int32_t* ticket = (int32_t*)p;
    p += 16;
    int32_t* counts = (int32_t*)p;
    p += align_up((size_t)L * 4, 16);
    int32_t* base = (int32_t*)p;
    layout_wait_selftest_init_kernel<<<1, 256, 0, s>>>(status, ticket, counts, L);
    layout_scan_kernel<<<1, kScanThreads, 0, s>>>(counts, base, L, status, 2, ticket, dev_status,
                                                  wait_limit_ns);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace moe
