// grouped_gemm_tc_swap.cu -- bf16 grouped SwiGLU expert FFN on CTA pairs
// with the operands swapped: expert weights are the MMA's M operand and the
// routed rows its N operand, so an expert's rows are padded to a multiple of
// 16 instead of a whole tile, and each weight tile is streamed from memory
// once for all of an expert's rows (sm_100a).
//
// Source: "Expert parallelism and all-to-all", "Walking through one MoE
// layer", step 3 (each GPU runs its local experts on the rows it received
// as one grouped matrix multiply); weight layout as in "Expert parallelism"
// (Transformers docs), GroupedGemmParallel: W13[j] = [gate rows 0..I-1; up
// rows I..2I-1] x H, W2[j] = H x I.
//
// The product, transposed:
//   phase 1 (GLU):  h^T[f, s] = silu(W_gate[f] . A_s) * (W_up[f] . A_s)
//   phase 2:        y^T[n, s] = W2[n] . h_s
// A tile pairs 256 weight rows (128 staged by each CTA of the pair; MMA
// M = 256, tcgen05.mma.cta_group::2) with one "pass" over an expert's
// routed rows.  An expert with c rows takes
//   - one pass when c <= 256 + 64: a first chunk of min(c, 256) rows (MMA N
//     = the chunk rounded up to 16) and, past 256, a second chunk of the
//     rest (N <= 64), both multiplied from the same staged weights into two
//     accumulators;
//   - otherwise ceil(c / 256) passes of near-equal size (multiples of 16
//     rows, at most 256), which run side by side and share the weight
//     reads through L2.
// So the tensor core executes at most 15 padding rows per chunk, and no
// pass is much faster than the others reading the same weights (a pass
// that ran ahead would stop sharing them and re-read them from DRAM).
//
// Each CTA's tensor memory (512 columns) holds two 256-column accumulator
// slots used in ring order; a pass with two chunks takes both.  Each CTA
// receives its 128 weight rows (lanes) x the chunk's rows (columns).  Phase
// 1 stages, per CTA, 64 gate rows and the 64 matching up rows, so lanes
// 0..63 hold gate and 64..127 up for the same 64 features; the epilogue
// pairs them through shared memory.  Phase 2 stages 128 rows of W2 per CTA;
// its output y is fp32, bf16, or the FP8 combine payload: e4m3 codes of
// y * (1/scale) with one fp32 scale (amax / 448) per 128 features ("Expert
// parallelism and all-to-all", "Traffic math": 1-byte activations both ways).  A CTA's 128 weight rows are exactly
// one such block, so each block's amax is a max over one epilogue group's
// four warps.
//
// Rows come in expert segments [off[j], off[j+1]) read from device memory
// (tile_schedule.cuh).  Chunk rows past the segment are loaded (TMA
// zero-fills past n_rows), multiplied and discarded.
//
// Each CTA = 10 warps, one CTA per SM: warp 0 TMA producer, warp 1 tensor-
// memory allocation and (leader) MMA issue, warps 2-9 epilogue in two groups
// of four that take alternate 32-column pieces of an accumulator.  Tiles
// are (pass, weight tile) pairs, weight tile fastest, dealt round-robin over
// the persistent pairs.  Every wait is bounded; on timeout the kernel
// records MOE_DEV_TIMEOUT, lets in-flight copies and MMAs land, frees tensor
// memory and exits.  No TMA multicast is used.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_launch.cuh"
#include "tcgen05.cuh"
#include "tile_schedule.cuh"

namespace moe {
namespace tcs {

using namespace tc;

constexpr int kWRows = 128;          // weight rows per CTA (the pair: MMA M = 256)
constexpr int kMainN = 256;          // first chunk of a pass: routed rows at most
constexpr int kTailN = 64;           // second chunk of a one-pass expert: at most
constexpr int BK = 64;               // K per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int kEpiWarps = 8;
constexpr int kEpiGroups = kEpiWarps / 4;   // groups of 4 warps cover the 128 lanes
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kRowBytes = BK * 2;                               // one staged row: 128 bytes
constexpr int kWBytes = kWRows * kRowBytes;                     // 16 KB
constexpr int kTRows = (kMainN + kTailN) / 2;                   // routed rows per CTA per stage
constexpr int kTailOff = (kMainN / 2) * kRowBytes;              // second chunk's rows: 16 KB in
constexpr int kTBytes = kTRows * kRowBytes;                     // 20 KB
constexpr int kStages = 5;
constexpr int kSlotCols = 256;
constexpr int kTmemCols = 2 * kSlotCols;

// Fused gather (phase 1): the routed rows are read from a token-major
// source through pair_of_slot by two teams of four warps per CTA that take
// alternate k-steps; each thread owns one 16-byte piece (8 bf16) of ten of
// the stage's 160 rows.
constexpr int kGatherTeams = 2;
constexpr int kTeamWarps = 4;
constexpr int kGatherThreads = kGatherTeams * kTeamWarps * 32;
constexpr int kGatherWarp0 = kThreads / 32;                      // warps 10..17
constexpr int kGatherRows = kTRows * 8 / (kTeamWarps * 32);      // rows per thread per stage
constexpr int kMaxThreads = kThreads + kGatherThreads;
static_assert(kTRows * 8 % (kTeamWarps * 32) == 0, "gather pieces divide evenly");
template <bool GATHER>
constexpr int threads_of() { return GATHER ? kMaxThreads : kThreads; }

// Epilogue staging.  Phase 1: per group, 128 lanes x 32 chunk rows as fp32,
// row pitch 33 words (conflict-free both ways).  Phase 2: per warp 32 chunk
// rows x 32 outputs as fp32, row pitch 36 words (16-byte aligned rows).
constexpr int kGluPitch = 33;
constexpr int kGluGroupBytes = 128 * kGluPitch * 4;              // 16896 B
constexpr int kOutPitch = 36;
constexpr int kOutWarpBytes = 32 * kOutPitch * 4;                // 4608 B
constexpr int kEpiBytes = kEpiGroups * kGluGroupBytes > kEpiWarps * kOutWarpBytes
                              ? kEpiGroups * kGluGroupBytes
                              : kEpiWarps * kOutWarpBytes;

// FP8 y: per-token partial amax of each warp's 32 features, double-buffered
constexpr int kAmaxBytes = 2 * kEpiGroups * 4 * 32 * 4;

struct Smem {
    static constexpr int w = 0;
    static constexpr int t = w + kStages * kWBytes;
    static constexpr int bars = t + kStages * kTBytes;
    static constexpr int n_bars = 2 * kStages + 4;           // full, empty, tfull[2], tempty[2]
    static constexpr int misc = bars + n_bars * 8;           // tmem addr, abort flag
    static constexpr int prefix = misc + 16;                 // int32 [MOE_MAX_EXPERTS + 1]
    static constexpr int warp_sums = prefix + (MOE_MAX_EXPERTS + 1) * 4;
    static constexpr int epi = ((warp_sums + (kMaxThreads / 32) * 4 + 127) / 128) * 128;
    static constexpr int amax = epi + kEpiBytes;
    static constexpr int total = amax + kAmaxBytes;
    static constexpr size_t alloc = total + 1024;            // + alignment slack
};
static_assert(Smem::alloc <= 232448, "smem budget");
static_assert(kStages * kWBytes % 1024 == 0 && kTBytes % 1024 == 0 && kTailOff % 1024 == 0,
              "stage buffers stay 1024-byte aligned for the 128-byte swizzle");

struct Params {
    const int32_t* offsets;   // global expert offsets (device)
    const int32_t* counts;    // rows per expert (device) or null: the whole segments
    int expert_begin, n_experts;
    int K;                    // reduction length (H in phase 1, I in phase 2)
    int n_out;                // output columns (I in phase 1, H in phase 2); % 8 == 0
    int n_wtiles;             // weight tiles per pass
    int n_rows;               // rows of A and out: stores never go past it
    void* out;                // h (phase 1, bf16) or y (phase 2, OutT), row stride n_out
    float* out_scales;        // y's block scales [n_rows, n_out / 128] when OutT is e4m3
    int32_t* dev_status;
    // fused gather (phase 1 only): row s of A is row pair_of_slot[s] / top_k
    // of gather_src [*, K] (zeros for a slot holding no pair)
    const __nv_bfloat16* gather_src;
    const int32_t* pair_of_slot;
    int top_k;
    // weights in the packed layout (pack_weights.cu): one contiguous 16 KB
    // block per (expert, 64 or 128 weight rows, 64-column k-step)
    int packed;
    // phase 2 only, may be null: y row s is multiplied by
    // row_weights[pair_of_slot[s]] (0 for a slot holding no pair)
    const float* row_weights;
    const int32_t* weight_pairs;
};

// Router weight of routed row `row` (phase 2 with row weights), 0 past the
// pass or for a slot holding no pair.
__device__ __forceinline__ float row_weight(const Params& p, int64_t row, int row_end) {
    if (row >= row_end) return 0.0f;
    const int32_t pr = __ldg(p.weight_pairs + row);
    return pr >= 0 ? __ldg(p.row_weights + pr) : 0.0f;
}

// Passes an expert with `rows` routed rows takes.
struct PassesOf {
    __device__ __forceinline__ int32_t operator()(int32_t rows) const {
        return rows <= kMainN + kTailN ? 1 : (rows + kMainN - 1) / kMainN;
    }
};

// Tile t: expert j, pass rows [row0, row0 + rows), first chunk N = n0
// (rows row0 ..), second chunk N = n1 (rows row0 + 256 .., 0 if none),
// weight tile wt.
struct TileInfo {
    int j, row0, rows, n0, n1, wt;
};

__device__ __forceinline__ TileInfo tile_info(const Params& p, const int32_t* s_prefix, int t) {
    TileInfo ti;
    const int pass = t / p.n_wtiles;
    ti.wt = t - pass * p.n_wtiles;
    ti.j = find_tile_expert(s_prefix, p.n_experts, pass);
    const int seg0 = __ldg(p.offsets + p.expert_begin + ti.j);
    const int cnt = segment_rows(p.offsets, p.counts, p.expert_begin, ti.j);
    const int np = s_prefix[ti.j + 1] - s_prefix[ti.j];
    if (np == 1) {
        ti.row0 = seg0;
        ti.rows = cnt;
        ti.n0 = min(kMainN, (cnt + 15) & ~15);
        ti.n1 = cnt > kMainN ? ((cnt - kMainN + 15) & ~15) : 0;
    } else {
        // ceil(cnt / 16) groups of 16 rows dealt as evenly as possible
        const int pi = pass - s_prefix[ti.j];
        const int q = (cnt + 15) >> 4, base = q / np, extra = q - base * np;
        const int start = 16 * (pi * base + min(pi, extra));
        ti.row0 = seg0 + start;
        ti.rows = min(16 * (base + (pi < extra ? 1 : 0)), cnt - start);
        ti.n0 = (ti.rows + 15) & ~15;
        ti.n1 = 0;
    }
    return ti;
}

// Named barrier over one epilogue group (4 warps), id 1 + group.
__device__ __forceinline__ void group_bar(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + group) : "memory");
}

// Barrier over one epilogue group that also ANDs `ok` across it, so its
// warps leave the tile loop together (none is left waiting at group_bar).
__device__ __forceinline__ bool group_all(int group, bool ok) {
    uint32_t r;
    asm volatile(
        "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, %2, 128, p; "
        "selp.u32 %0, 1, 0, q; }"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(1 + group)
        : "memory");
    return r != 0;
}

// silu(g) = g / (1 + e^-g) with the fast exponential and division (a few
// ulp of fp32; the result is rounded to bf16).  e^-g = inf gives 0.
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Rows one TMA box stages for `rows` routed rows: the smallest of 8, 32
// and 128 that covers them.  One box per chunk: each TMA instruction has a
// large fixed cost, so a few extra rows (multiplied by nothing: the MMA reads
// only `rows` of them) are cheaper than several smaller boxes.
__device__ __forceinline__ int box_rows(int rows) { return rows <= 8 ? 8 : rows <= 32 ? 32 : 128; }

// Loads the box covering `rows` routed rows from row r0, K columns
// k0..k0+63, into shared memory at dst.
__device__ __forceinline__ void load_rows(uint32_t dst, const CUtensorMap* m128,
                                          const CUtensorMap* m32, const CUtensorMap* m8,
                                          uint32_t bar, int k0, int r0, int rows) {
    const int b = box_rows(rows);
    tma_load_2d<2>(dst, b == 128 ? m128 : b == 32 ? m32 : m8, bar, k0, r0);
}

// Clock record, summed over launches: per phase (gate/up, down), the SM
// cycles (clock64) and the nanoseconds (globaltimer) CTA 0 spent from its
// first instruction to its last.  Their ratio is the SM clock the kernel ran
// at, which the power cap can hold well below the nominal maximum while the
// tensor cores and the weight stream are both busy.
__device__ unsigned long long g_swap_clock[4];

template <bool GLU, typename OutT, bool GATHER>
__global__ void __launch_bounds__(threads_of<GATHER>(), 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmap_w,
                             const __grid_constant__ CUtensorMap tmap_t128,
                             const __grid_constant__ CUtensorMap tmap_t32,
                             const __grid_constant__ CUtensorMap tmap_t8, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();   // 0 = leader
    const bool leader = rank == 0;
    const int unit = blockIdx.x / 2, n_units = gridDim.x / 2;
    const bool clock_cta = blockIdx.x == 0 && threadIdx.x == 0;
    const long long clk0 = clock_cta ? clock64() : 0;
    const uint64_t ns0 = clock_cta ? global_timer_ns() : 0;

    const uint32_t bar0 = sbase + Smem::bars;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    uint32_t* s_tmem = (uint32_t*)(smem + Smem::misc);
    volatile int* s_abort = (volatile int*)(smem + Smem::misc + 4);
    int32_t* s_prefix = (int32_t*)(smem + Smem::prefix);
    int32_t* s_ws = (int32_t*)(smem + Smem::warp_sums);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // the leader's expect_tx (both CTAs' TMA bytes), and with the
            // fused gather one arrival per gathering warp of both CTAs
            mbar_init(full_bar(s), GATHER ? 1 + 2 * kTeamWarps : 1);
            mbar_init(empty_bar(s), 1);           // the leader's MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);                   // the leader's MMA commit
            mbar_init(tempty_bar(b), 2 * kEpiThreads);    // both CTAs' epilogue threads
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_t128);
        prefetch_tmap(&tmap_t32);
        prefetch_tmap(&tmap_t8);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    build_unit_prefix(p.offsets, p.counts, p.expert_begin, p.n_experts, PassesOf{}, s_prefix,
                      s_ws);
    tc_fence_before();
    cluster_sync();   // both CTAs' barriers exist before cross-CTA use
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int n_tiles = s_prefix[p.n_experts] * p.n_wtiles;
    const int nk = (p.K + BK - 1) / BK;
    bool aborted = false;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        // This CTA's weight box at k-step kb of a tile: W13 rows [f0, f0+64)
        // of gate and of up (one 4-D box), or 128 rows of W2.
        auto w_row = [&](const TileInfo& ti) {
            return GLU ? ti.wt * kWRows + (int)rank * (kWRows / 2)
                       : ti.wt * 2 * kWRows + (int)rank * kWRows;
        };
        int stage = 0;
        uint32_t phase = 0;
        for (int t = unit; t < n_tiles; t += n_units) {
            const TileInfo ti = tile_info(p, s_prefix, t);
            const int h0 = ti.n0 >> 1, h1 = ti.n1 >> 1;       // rows this CTA multiplies per chunk
            const uint32_t tx =
                GATHER ? 2u * (uint32_t)kWBytes
                       : 2u * (uint32_t)(kWBytes +
                                         (box_rows(h0) + (h1 ? box_rows(h1) : 0)) * kRowBytes);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, s_abort, p.dev_status)) {
                    aborted = true;
                    break;
                }
                const uint32_t fb = full_bar(stage);
                if (leader) mbar_arrive_expect_tx(fb, tx);
                const uint32_t cfb = map_to_rank(fb, 0);
                const uint32_t sw = sbase + Smem::w + stage * kWBytes;
                const uint32_t st = sbase + Smem::t + stage * kTBytes;
                const int k0 = kb * BK;
                if (p.packed)   // this CTA's row block of the tile: one 16 KB block
                    tma_load_3d<2>(sw, &tmap_w, cfb, 0, 0,
                                   (ti.j * 2 * p.n_wtiles + 2 * ti.wt + (int)rank) * nk + kb);
                else if (GLU)   // 64 gate rows, then the 64 matching up rows: one box
                    tma_load_4d<2>(sw, &tmap_w, cfb, k0, w_row(ti), 0, ti.j);
                else
                    tma_load_3d<2>(sw, &tmap_w, cfb, k0, w_row(ti), ti.j);
                if (!GATHER)
                    load_rows(st, &tmap_t128, &tmap_t32, &tmap_t8, cfb, k0,
                              ti.row0 + (int)rank * h0, h0);
                if (!GATHER && h1)
                    load_rows(st + kTailOff, &tmap_t128, &tmap_t32, &tmap_t8, cfb, k0,
                              ti.row0 + kMainN + (int)rank * h1, h1);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (aborted) break;
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        int stage = 0;
        uint32_t phase = 0;
        uint32_t nslot = 0;       // accumulator slots taken so far (ring of 2)
        for (int t = unit; t < n_tiles && !aborted; t += n_units) {
            const TileInfo ti = tile_info(p, s_prefix, t);
            const int ns = ti.n1 ? 2 : 1;
            for (int c = 0; c < ns && !aborted; ++c) {
                const uint32_t n = nslot + c;
                if (!mbar_wait(tempty_bar(n & 1), ((n >> 1) & 1) ^ 1u, s_abort, p.dev_status))
                    aborted = true;
            }
            if (aborted) break;
            tc_fence_after();
            const uint32_t d0 = tmem_base + (nslot & 1) * kSlotCols;
            const uint32_t d1 = tmem_base + ((nslot + 1) & 1) * kSlotCols;
            const uint32_t idesc0 = make_idesc(2 * kWRows, ti.n0);
            const uint32_t idesc1 = make_idesc(2 * kWRows, ti.n1 ? ti.n1 : 16);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(full_bar(stage), phase, s_abort, p.dev_status)) {
                    aborted = true;
                    break;
                }
                tc_fence_after();
                const uint32_t sw = sbase + Smem::w + stage * kWBytes;
                const uint32_t st = sbase + Smem::t + stage * kTBytes;
#pragma unroll
                for (int k = 0; k < BK / UMMA_K; ++k)
                    umma_bf16<2>(d0, smem_desc_sw128(sw + k * UMMA_K * 2),
                                 smem_desc_sw128(st + k * UMMA_K * 2), idesc0,
                                 (kb > 0 || k > 0) ? 1u : 0u);
                if (ti.n1) {
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        umma_bf16<2>(d1, smem_desc_sw128(sw + k * UMMA_K * 2),
                                     smem_desc_sw128(st + kTailOff + k * UMMA_K * 2), idesc1,
                                     (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit<2>(empty_bar(stage));   // stage free once these MMAs finish
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (aborted) break;
            for (int c = 0; c < ns; ++c) umma_commit<2>(tfull_bar((nslot + c) & 1));
            nslot += ns;
        }
    } else if (GATHER && warp >= kGatherWarp0) {
        // ------------------------------------------------ row gather (both CTAs)
        // Stage row q (q < 128: first chunk, q >= 128: second chunk) of this
        // CTA is the routed row in slot row0 + rank * h0 + q (or row0 + 256
        // + rank * h1 + q - 128); it is row pair_of_slot[slot] / top_k of the
        // source.  Rows are written in the 128-byte-swizzled layout a TMA box
        // would produce: 16-byte piece c of row q at q * 128 + ((c ^ (q % 8))
        // * 16).  Rows past the pass (padding) are zeros.  The copies are
        // cp.async: a team releases a k-step to the MMA (its copies landed,
        // proxy fence, one arrival per warp) only after issuing its next one,
        // so each team keeps two k-steps in flight -- four of the five stages
        // with both teams, and a k-step waits only on stages five back.
        const int gw = warp - kGatherWarp0;
        const uint32_t team = (uint32_t)(gw / kTeamWarps);
        const int lt = (gw % kTeamWarps) * 32 + lane;
        const int piece = lt & 7;                  // 16-byte piece of each row
        const int rb = lt >> 3;                    // rows rb, rb + 16, .., rb + 144
        uint32_t g = 0;                            // k-steps so far, both teams
        int pending = -1;                          // stage issued but not yet released
        // The release: every lane's copies of the k-step are complete in this
        // CTA's shared memory (cp.async.wait_group) and fenced to the async
        // proxy that the tensor core reads through; then lane 0 signals the
        // leader's full barrier.  The signal carries no data: the rows are
        // already in place when the leader, having seen the phase complete,
        // issues the MMA that reads them.  (A cluster-scope release here
        // stalled each warp about half a microsecond per k-step: gate/up on
        // dsv3 took 6.1 ms instead of 4.1.)
        auto release = [&](int stg) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_signal(map_to_rank(full_bar(stg), 0));
        };
        for (int t = unit; t < n_tiles && !aborted; t += n_units) {
            const TileInfo ti = tile_info(p, s_prefix, t);
            const int h0 = ti.n0 >> 1, h1 = ti.n1 >> 1;
            const __nv_bfloat16* src[kGatherRows];
            uint32_t need = 0;                     // bit m: row rb + 16 m is multiplied
#pragma unroll
            for (int m = 0; m < kGatherRows; ++m) {
                const int q = rb + 16 * m;
                const bool first = q < kMainN / 2;
                const int qi = first ? q : q - kMainN / 2;
                const bool used = qi < (first ? h0 : h1);
                const int ci = (int)rank * (first ? h0 : h1) + qi;        // row within the chunk
                const int lim = first ? min(ti.rows, kMainN) : ti.rows - kMainN;
                const int64_t slot = (int64_t)ti.row0 + (first ? 0 : kMainN) + ci;
                src[m] = nullptr;
                if (used) {
                    need |= 1u << m;
                    if (ci < lim && slot < p.n_rows) {
                        const int32_t pr = __ldg(p.pair_of_slot + slot);
                        if (pr >= 0)
                            src[m] = p.gather_src + (int64_t)(pr / p.top_k) * p.K + piece * 8;
                    }
                }
            }
            for (int kb = 0; kb < nk; ++kb, ++g) {
                if (g % kGatherTeams != team) continue;
                const int stage = (int)(g % kStages);
                const uint32_t phase = (g / kStages) & 1u;
                const bool ok = __all_sync(
                    0xffffffffu, mbar_wait(empty_bar(stage), phase ^ 1u, s_abort, p.dev_status));
                if (!ok) {
                    aborted = true;
                    break;
                }
                const int k0 = kb * BK;
                const bool kin = k0 + piece * 8 < p.K;
                const uint32_t st = sbase + Smem::t + stage * kTBytes;
#pragma unroll
                for (int m = 0; m < kGatherRows; ++m) {
                    const int q = rb + 16 * m;
                    if ((need >> m) & 1u) {
                        const bool live = src[m] != nullptr && kin;
                        cp_async16(st + q * kRowBytes + ((piece ^ (q & 7)) << 4),
                                   live ? (const void*)(src[m] + k0) : (const void*)p.gather_src,
                                   live ? 16u : 0u);
                    }
                }
                cp_async_commit();
                if (pending >= 0) {
                    cp_async_wait<1>();            // the previous k-step's copies landed
                    release(pending);
                }
                pending = stage;
            }
        }
        cp_async_wait<0>();
        if (!aborted && pending >= 0) release(pending);
    } else if (warp >= 2 && warp < 2 + kEpiWarps) {
        // ------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;                 // 0..7
        const int group = ew >> 2;               // takes every kEpiGroups-th 32-column piece
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const int lrow = quarter * 32 + lane;    // this thread's weight row in the CTA
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int gw = ew & 3;                   // warp within the group
        float* glu_stage = reinterpret_cast<float*>(smem + Smem::epi + group * kGluGroupBytes);
        float* out_stage = reinterpret_cast<float*>(smem + Smem::epi + ew * kOutWarpBytes);
        OutT* out = reinterpret_cast<OutT*>(p.out);
        constexpr bool kFP8 = sizeof(OutT) == 1;          // e4m3 codes + block scales
        float* s_amax = reinterpret_cast<float*>(smem + Smem::amax);
        uint32_t piece = 0;                               // FP8: amax buffer parity
        uint32_t nslot = 0;
        for (int t = unit; t < n_tiles && !aborted; t += n_units) {
            const TileInfo ti = tile_info(p, s_prefix, t);
            const int row_end = min(ti.row0 + ti.rows, p.n_rows);
            const int ns = ti.n1 ? 2 : 1;
            for (int c = 0; c < ns; ++c, ++nslot) {
                const int ncols = c == 0 ? ti.n0 : ti.n1;
                const int crow0 = ti.row0 + c * kMainN;      // chunk's first routed row
                bool ok = mbar_wait(tfull_bar(nslot & 1), (nslot >> 1) & 1, s_abort, p.dev_status);
                if (GLU || kFP8) ok = group_all(group, ok);
                if (!ok) {
                    aborted = true;
                    break;
                }
                tc_fence_after();
                const uint32_t tacc = tmem_base + lane_off + (nslot & 1) * kSlotCols;
#pragma unroll 1
                for (int col = 32 * group; col < ncols; col += 32 * kEpiGroups) {
                    float v[32];
                    tmem_ld32(tacc + (uint32_t)col, v);
                    tmem_ld_wait();
                    if (GLU) {
                        // lanes 0..63: gate of features f..f+63; 64..127: up of the same
                        group_bar(group);                 // previous piece's reads are done
#pragma unroll
                        for (int i = 0; i < 32; ++i) glu_stage[lrow * kGluPitch + i] = v[i];
                        group_bar(group);
                        // 32 chunk rows x 64 features: group warp gw takes rows
                        // 8*gw..8*gw+7; lane -> row (lane % 8), 8 features (lane / 8 + 4 * hf)
                        const int r = (lane & 7) + 8 * gw;
                        const int64_t row = crow0 + col + r;
                        const int f_cta = ti.wt * kWRows + (int)rank * (kWRows / 2);
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int piece = (lane >> 3) + 4 * hf;    // features 8*piece..+7
                            float hv[8];
#pragma unroll
                            for (int m = 0; m < 8; ++m) {
                                const float g = glu_stage[(8 * piece + m) * kGluPitch + r];
                                const float u = glu_stage[(64 + 8 * piece + m) * kGluPitch + r];
                                hv[m] = silu_fast(g) * u;
                            }
                            const int fcol = f_cta + 8 * piece;
                            if (row < row_end && fcol < p.n_out)
                                st_v4(out + row * p.n_out + fcol,
                                      make_uint4(pack_bf16x2(hv[0], hv[1]), pack_bf16x2(hv[2], hv[3]),
                                                 pack_bf16x2(hv[4], hv[5]), pack_bf16x2(hv[6], hv[7])));
                        }
                    } else if constexpr (kFP8) {
                        // this warp: 32 outputs (its lanes) x 32 chunk rows (v); lane l
                        // then takes chunk row l: its amax over this warp's 32
                        // outputs, the block amax over the group's four warps, and
                        // 32 codes (32 bytes) of the row's 128-wide block
                        if (p.row_weights) {   // the routed row's router weight, first
                            const float wl = row_weight(p, crow0 + col + lane, row_end);
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] *= __shfl_sync(0xffffffffu, wl, i);
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) out_stage[i * kOutPitch + lane] = v[i];
                        __syncwarp();
                        float rv[32];
                        float part = 0.0f;
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 f =
                                *reinterpret_cast<const float4*>(out_stage + lane * kOutPitch + 4 * q4);
                            rv[4 * q4 + 0] = f.x;
                            rv[4 * q4 + 1] = f.y;
                            rv[4 * q4 + 2] = f.z;
                            rv[4 * q4 + 3] = f.w;
                            part = fmaxf(part, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)),
                                                     fmaxf(fabsf(f.z), fabsf(f.w))));
                        }
                        float* amax_buf = s_amax + ((piece & 1) * kEpiGroups + group) * 128;
                        amax_buf[quarter * 32 + lane] = part;
                        group_bar(group);
                        const float amax = fmaxf(fmaxf(amax_buf[lane], amax_buf[32 + lane]),
                                                 fmaxf(amax_buf[64 + lane], amax_buf[96 + lane]));
                        const float scale = e4m3_block_scale(amax);
                        const float rs = __frcp_rn(scale);       // codes: e4m3(y * (1/scale))
                        const int64_t row = crow0 + col + lane;
                        const int blk0 = ti.wt * 2 * kWRows + (int)rank * kWRows;   // block start
                        if (row < row_end && blk0 < p.n_out) {
                            uint8_t* dst =
                                reinterpret_cast<uint8_t*>(out) + row * p.n_out + blk0 + quarter * 32;
                            st_v4(dst, make_uint4(quant4_e4m3_mul(rv[0], rv[1], rv[2], rv[3], rs),
                                                  quant4_e4m3_mul(rv[4], rv[5], rv[6], rv[7], rs),
                                                  quant4_e4m3_mul(rv[8], rv[9], rv[10], rv[11], rs),
                                                  quant4_e4m3_mul(rv[12], rv[13], rv[14], rv[15], rs)));
                            st_v4(dst + 16,
                                  make_uint4(quant4_e4m3_mul(rv[16], rv[17], rv[18], rv[19], rs),
                                             quant4_e4m3_mul(rv[20], rv[21], rv[22], rv[23], rs),
                                             quant4_e4m3_mul(rv[24], rv[25], rv[26], rv[27], rs),
                                             quant4_e4m3_mul(rv[28], rv[29], rv[30], rv[31], rs)));
                            if (quarter == 0) p.out_scales[row * (p.n_out / 128) + blk0 / 128] = scale;
                        }
                        ++piece;
                        __syncwarp();
                    } else {
                        // this warp: 32 outputs (its lanes) x 32 chunk rows (v)
                        if (p.row_weights) {   // y row = router weight x expert output
                            const float wl = row_weight(p, crow0 + col + lane, row_end);
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] *= __shfl_sync(0xffffffffu, wl, i);
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) out_stage[i * kOutPitch + lane] = v[i];
                        __syncwarp();
                        const int col0 = ti.wt * 2 * kWRows + (int)rank * kWRows + quarter * 32;
                        constexpr bool kF32 = sizeof(OutT) == 4;
                        constexpr int kLanesPerRow = kF32 ? 8 : 4;     // 16-byte stores
                        constexpr int kRowsPerStep = 32 / kLanesPerRow;
                        constexpr int kElems = 16 / (int)sizeof(OutT);
                        const int r_in = lane / kLanesPerRow, piece = lane % kLanesPerRow;
                        const int ocol = col0 + piece * kElems;
#pragma unroll
                        for (int r0 = 0; r0 < 32; r0 += kRowsPerStep) {
                            const int r = r0 + r_in;
                            const int64_t row = crow0 + col + r;
                            const float* src = out_stage + r * kOutPitch + piece * kElems;
                            uint4 d;
                            if (kF32) {
                                d = *reinterpret_cast<const uint4*>(src);
                            } else {
                                const float4 a = *reinterpret_cast<const float4*>(src);
                                const float4 b = *reinterpret_cast<const float4*>(src + 4);
                                d = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                               pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
                            }
                            if (row < row_end && ocol < p.n_out) st_v4(out + row * p.n_out + ocol, d);
                        }
                        __syncwarp();
                    }
                }
                tc_fence_before();
                mbar_arrive_signal(map_to_rank(tempty_bar(nslot & 1), 0));   // leader's barrier
            }
        }
    }
    __syncwarp();
    if (aborted || *s_abort) {
        // let copies and MMAs already issued land before shared and tensor
        // memory are released (bounded: 1 ms)
        const uint64_t until = global_timer_ns() + 1000ull * 1000;
        while (global_timer_ns() < until) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no cross-CTA access after this
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    if (clock_cta) {
        atomicAdd(&g_swap_clock[GLU ? 0 : 2], (unsigned long long)(clock64() - clk0));
        atomicAdd(&g_swap_clock[GLU ? 1 : 3], (unsigned long long)(global_timer_ns() - ns0));
    }
}

// ---------------------------------------------------------------- host side
static bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides_bytes, const cuuint32_t* box) {
    return make_bf16_map(m, base, rank, dims, strides_bytes, box);
}

// CTA pairs of this kernel that fit on the current device at once (one CTA
// per SM), cached per device.
template <bool GLU, typename OutT, bool GATHER>
static int resident_pairs(size_t smem) {
    struct Tag {};
    return PerDeviceInt<Tag>::get([smem] {
        int n = current_device_sm_count() / 2;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * n));
        cfg.blockDim = dim3(threads_of<GATHER>());
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        set_cluster_attr(cfg, attr, 2);
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, grouped_gemm_swap_kernel<GLU, OutT, GATHER>,
                                           &cfg) == cudaSuccess &&
            c > 0)
            n = c;
        return n;
    });
}

template <bool GLU, typename OutT, bool GATHER = false>
static cudaError_t launch_phase(const CUtensorMap& mw, const CUtensorMap* mt, const Params& p,
                                cudaStream_t s) {
    auto kern = grouped_gemm_swap_kernel<GLU, OutT, GATHER>;
    constexpr size_t smem = Smem::alloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * resident_pairs<GLU, OutT, GATHER>(smem)));
    cfg.blockDim = dim3(threads_of<GATHER>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    set_cluster_attr(cfg, attr, 2);
    return cudaLaunchKernelEx(&cfg, kern, mw, mt[0], mt[1], mt[2], p);
}

// Maps over a [n_rows, K] bf16 row operand: boxes of 64 x 128, 64 x 32 and
// 64 x 8 rows.
static bool make_row_maps(CUtensorMap* m, const void* base, int K, int64_t n_rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)n_rows};
    const cuuint64_t str[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box128[2] = {BK, 128};
    const cuuint32_t box32[2] = {BK, 32};
    const cuuint32_t box8[2] = {BK, 8};
    return make_map(&m[0], base, 2, dims, str, box128) &&
           make_map(&m[1], base, 2, dims, str, box32) && make_map(&m[2], base, 2, dims, str, box8);
}

}  // namespace tcs

// A [n_rows, H] bf16; W13 [n_exp, 2I, H]; W2 [n_exp, H, I]; h [n_rows, I]
// bf16; y [n_rows, H] in y_dtype (fp32, bf16, or e4m3 codes with fp32
// y_scales [n_rows, H/128]).  counts (may be null) cuts
// each expert's segment to its first counts[j] rows.  ev_mid (may be null)
// is recorded between the two phases.  With g (the fused gather) non-null,
// A is not read: row s of the gate/up operand is row pair_of_slot[s] / k of
// g.src [*, H] (16-byte aligned).  packed: w13 and w2 are in the packed
// layout of pack_weights.cu.  row_weights (may be null): y row s is written
// as row_weights[weight_pairs[s]] times the expert's output.
cudaError_t launch_grouped_gemm_tc_swap(const __nv_bfloat16* a, const int32_t* offsets,
                                        const int32_t* counts, int expert_begin, int n_experts,
                                        int64_t n_rows, int H, int I, const __nv_bfloat16* w13,
                                        const __nv_bfloat16* w2, __nv_bfloat16* h, void* y,
                                        moe_dtype y_dtype, float* y_scales, int32_t* dev_status,
                                        const gemm_gather* g, cudaEvent_t ev_mid,
                                        cudaStream_t s, bool packed, const float* row_weights,
                                        const int32_t* weight_pairs) {
    using namespace tcs;
    CUtensorMap mw1, mt1[3], mw2, mt2[3];
    const int nwt1 = (I + kWRows - 1) / kWRows, nwt2 = (H + 2 * kWRows - 1) / (2 * kWRows);
    // packed weights: [blocks][128 rows][64 columns], one 16 KB box per block
    auto packed_map = [&](CUtensorMap* m, const void* base, int64_t blocks) {
        const cuuint64_t dims[3] = {(cuuint64_t)BK, (cuuint64_t)kWRows, (cuuint64_t)blocks};
        const cuuint64_t str[2] = {(cuuint64_t)BK * 2, (cuuint64_t)kWBytes};
        const cuuint32_t box[3] = {BK, kWRows, 1};
        return make_map(m, base, 3, dims, str, box);
    };
    if (packed) {
        if (!packed_map(&mw1, w13, (int64_t)n_experts * 2 * nwt1 * ((H + BK - 1) / BK)) ||
            !packed_map(&mw2, w2, (int64_t)n_experts * 2 * nwt2 * ((I + BK - 1) / BK)))
            return cudaErrorInvalidValue;
    } else {   // W13 as [E, 2, I, H]: a box of 64 gate rows and the 64 matching up rows
        const cuuint64_t dims[4] = {(cuuint64_t)H, (cuuint64_t)I, 2, (cuuint64_t)n_experts};
        const cuuint64_t str[3] = {(cuuint64_t)H * 2, (cuuint64_t)I * H * 2,
                                   (cuuint64_t)2 * I * H * 2};
        const cuuint32_t box[4] = {BK, kWRows / 2, 2, 1};
        if (!make_map(&mw1, w13, 4, dims, str, box)) return cudaErrorInvalidValue;
    }
    if (!g && !make_row_maps(mt1, a, H, n_rows)) return cudaErrorInvalidValue;
    if (!packed) {   // W2 as [E, H, I]: a box of 128 rows
        const cuuint64_t dims[3] = {(cuuint64_t)I, (cuuint64_t)H, (cuuint64_t)n_experts};
        const cuuint64_t str[2] = {(cuuint64_t)I * 2, (cuuint64_t)H * I * 2};
        const cuuint32_t box[3] = {BK, kWRows, 1};
        if (!make_map(&mw2, w2, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    if (!make_row_maps(mt2, h, I, n_rows)) return cudaErrorInvalidValue;

    Params p1{offsets, counts, expert_begin, n_experts, H, I, nwt1,
              (int)n_rows, h, nullptr, dev_status, nullptr, nullptr, 0, packed ? 1 : 0,
              nullptr, nullptr};
    cudaError_t e;
    if (g) {
        p1.gather_src = g->src;
        p1.pair_of_slot = g->pair_of_slot;
        p1.top_k = g->top_k;
        const CUtensorMap unused[3] = {mw1, mw1, mw1};   // no row boxes: the rows are gathered
        e = launch_phase<true, __nv_bfloat16, true>(mw1, unused, p1, s);
    } else {
        e = launch_phase<true, __nv_bfloat16>(mw1, mt1, p1, s);
    }
    if (e == cudaSuccess && ev_mid) e = cudaEventRecord(ev_mid, s);
    if (e != cudaSuccess) return e;
    Params p2{offsets, counts, expert_begin, n_experts, I, H, nwt2,
              (int)n_rows, y, y_scales, dev_status, nullptr, nullptr, 0, packed ? 1 : 0,
              row_weights, weight_pairs};
    e = y_dtype == MOE_F32    ? launch_phase<false, float>(mw2, mt2, p2, s)
        : y_dtype == MOE_BF16 ? launch_phase<false, __nv_bfloat16>(mw2, mt2, p2, s)
                              : launch_phase<false, uint8_t>(mw2, mt2, p2, s);
    note_launches(2);
    return e;
}

}  // namespace moe

extern "C" moe_status moe_diag_gemm_clock(uint64_t* out, int32_t reset) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess && out)
        e = cudaMemcpyFromSymbol(out, moe::tcs::g_swap_clock, sizeof(moe::tcs::g_swap_clock));
    if (e == cudaSuccess && reset) {
        const unsigned long long zero[4] = {0, 0, 0, 0};
        e = cudaMemcpyToSymbol(moe::tcs::g_swap_clock, zero, sizeof(zero));
    }
    return moe::report_cuda(e);
}
