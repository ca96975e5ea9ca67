// grouped_gemm_tc.cu -- bf16 grouped SwiGLU expert FFN on the 5th-generation
// tensor cores (tcgen05 MMA on CTA pairs, accumulators in tensor memory,
// operands staged by TMA), for sm_100a.
//
// Source: "Expert parallelism and all-to-all", "Walking through one MoE
// layer", step 3: each GPU runs its local experts on the rows it received
// as one grouped matrix multiply.  Expert weights are stacked along the
// expert dimension ("Expert parallelism" (Transformers docs),
// GroupedGemmParallel): W13[j] = [gate rows 0..I-1; up rows I..2I-1] x H,
// W2[j] = H x I.
//
// Two launches of one persistent kernel:
//   phase 1 (GLU):  h[s, n0:n0+128] = silu(A_s W_gate^T) * (A_s W_up^T)
//   phase 2:        y[s, n0:n0+256] = h_s W2^T
// A tile is N=256 accumulator columns by M=128 rows (one CTA,
// tcgen05.mma.cta_group::1) or M=256 rows (a cluster of two CTAs,
// tcgen05.mma.cta_group::2: each CTA stages its own 128 rows of A and half
// of the 256 B rows, and each CTA's tensor memory receives its 128 rows x
// all 256 columns).  In phase 1 the B tile is 128 gate rows plus the 128
// matching up rows (with a pair, the leader stages the gate rows and the
// peer the up rows), so every accumulator holds gate in columns 0..127 and
// up in 128..255 and the epilogue fuses SwiGLU.  The pair halves each SM's
// shared-memory traffic per MMA; single CTAs pad each expert's rows to 128
// instead of 256.  The host picks by the average rows per expert.  No TMA
// multicast is used.
//
// Rows come in expert segments [off[j], off[j+1]) read from device memory
// (tile_schedule.cuh); a 256-row tile never mixes experts: rows past the
// segment end are computed from whatever TMA loads there and discarded.
//
// Each CTA = 6 warps, one CTA per SM:
//   warp 0      TMA producer (one thread): per stage A 128x64 and B
//               (256 or, with a pair, 128) x 64, 128-byte swizzle; with a
//               pair the bytes of both CTAs count on the leader's "full"
//               barrier.
//   warp 1      tensor-memory allocation (2 x 256 columns) and, in the
//               leader, the MMA issuer: 4 x tcgen05.mma (K=16) per stage,
//               tcgen05.commit to the "empty" barriers (both CTAs' with a
//               pair) and, after the last K step, to the "accumulator full"
//               barriers.
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes (warp w owns
//               lanes 32*(w%4)..), SwiGLU / conversion, stores staged
//               through shared memory into whole 128-byte lines; they
//               release the accumulator on the leader's barrier.
// Tiles are (M-tile, N-tile) pairs in M-major order, N fastest, dealt
// round-robin over the persistent clusters.  Every wait is bounded; on
// timeout the kernel records MOE_DEV_TIMEOUT, lets in-flight copies and
// MMAs land, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_launch.cuh"
#include "tcgen05.cuh"
#include "tile_schedule.cuh"

namespace moe {
namespace tc {

constexpr int BM_CTA = 128;         // rows of A per CTA (MMA M per CTA)
constexpr int BN = 256;             // accumulator columns per tile (MMA N)
constexpr int BK = 64;              // K per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;          // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;
constexpr int kABytes = BM_CTA * BK * 2;            // 16 KB
constexpr int kTmemCols = 2 * BN;                   // two accumulator buffers

// Per-configuration geometry: NCTA CTAs compute one tile of BM rows.
template <int NCTA>
struct Geo {
    static constexpr int BM = BM_CTA * NCTA;              // rows per tile
    static constexpr int B_ROWS = BN / NCTA;              // B rows staged per CTA
    static constexpr int kBBytes = B_ROWS * BK * 2;       // 32 KB or 16 KB
    static constexpr int kStageBytes = kABytes + kBBytes; // per CTA
    static constexpr int kStages = NCTA == 1 ? 4 : 6;     // ~192 KB ring
};

// Shared-memory layout (offsets inside a 1024-aligned block).  Each
// epilogue warp stages 32 rows x 32 outputs (OB bytes each), rows padded by
// 16 bytes.
template <int NCTA, int OB>
struct SmemLayout {
    using G = Geo<NCTA>;
    static constexpr int a = 0;
    static constexpr int b = a + G::kStages * kABytes;
    static constexpr int bars = b + G::kStages * G::kBBytes;
    // full[S], empty[S], tfull[2], tempty[2]
    static constexpr int n_bars = 2 * G::kStages + 4;
    static constexpr int misc = bars + n_bars * 8;                   // tmem addr, abort flag
    static constexpr int prefix = misc + 16;                         // int32 [MOE_MAX_EXPERTS+1]
    static constexpr int warp_sums = prefix + (MOE_MAX_EXPERTS + 1) * 4;
    static constexpr int pitch = 32 * OB + 16;
    static constexpr int stage_tile = 32 * pitch;
    static constexpr int epi = ((warp_sums + 32 * 4 + 127) / 128) * 128;
    static constexpr int total = epi + 4 * stage_tile;
    static constexpr size_t alloc = total + 1024;                    // + alignment slack
};
static_assert(SmemLayout<1, 4>::alloc <= 232448, "smem budget");
static_assert(SmemLayout<2, 4>::alloc <= 232448, "smem budget");


// ---------------------------------------------------------------- kernel
struct Params {
    const int32_t* offsets;   // global expert offsets (device)
    const int32_t* counts;    // rows per expert (device) or null: the whole segments
    int expert_begin, n_experts;
    int K;                    // reduction length (H in phase 1, I in phase 2)
    int n_out;                // output columns (I in phase 1, H in phase 2)
    int n_ntiles;             // N tiles per M tile
    int n_rows;               // rows of A and out: stores never go past it
    void* out;                // h (phase 1, bf16) or y (phase 2, OutT), row stride n_out
    int32_t* dev_status;
};

// Epilogue store of a warp's 32 rows x 32 columns (lane i holds row i's 32
// values).  The rows go through a padded shared-memory tile so that the
// global stores are whole 128-byte lines: for fp32 output 8 lanes write
// one row (4 rows per instruction), for bf16 output 4 lanes write one row
// (8 rows per instruction).  Rows past row_end and 16-byte pieces past
// n_out (n_out % 8 == 0) are skipped.
template <typename OutT>
__device__ __forceinline__ void store_tile32(uint8_t* stage, const float (&v)[32], int lane,
                                             OutT* out, int64_t row_base, int row_end,
                                             int col0, int n_out) {
    constexpr bool kF32 = sizeof(OutT) == 4;
    constexpr int kPitch = 32 * (int)sizeof(OutT) + 16;
    uint8_t* my = stage + lane * kPitch;
    if (kF32) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(my + q * 16) =
                make_uint4(__float_as_uint(v[q * 4 + 0]), __float_as_uint(v[q * 4 + 1]),
                           __float_as_uint(v[q * 4 + 2]), __float_as_uint(v[q * 4 + 3]));
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(my + q * 16) =
                make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]),
                           pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                           pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]),
                           pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]));
    }
    __syncwarp();
    constexpr int kLanesPerRow = kF32 ? 8 : 4;          // 16 bytes per lane
    constexpr int kRowsPerStep = 32 / kLanesPerRow;
    constexpr int kElemsPer16 = 16 / sizeof(OutT);
    const int r_in = lane / kLanesPerRow, piece = lane % kLanesPerRow;
    const int col = col0 + piece * kElemsPer16;
#pragma unroll
    for (int r0 = 0; r0 < 32; r0 += kRowsPerStep) {
        const int r = r0 + r_in;
        const int64_t row = row_base + r;
        const uint4 d = *reinterpret_cast<const uint4*>(stage + r * kPitch + piece * 16);
        if (row < row_end && col < n_out) st_v4(out + row * n_out + col, d);
    }
    __syncwarp();
}

template <bool GLU, typename OutT, int NCTA>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b, const Params p) {
    using G = Geo<NCTA>;
    using L = SmemLayout<NCTA, (int)sizeof(OutT)>;
    constexpr int kStages = G::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = NCTA == 2 ? cluster_ctarank() : 0u;   // 0 = leader
    const bool leader = rank == 0;
    const int unit = blockIdx.x / NCTA, n_units = gridDim.x / NCTA;

    const uint32_t bar0 = sbase + L::bars;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    uint32_t* s_tmem = (uint32_t*)(smem + L::misc);
    volatile int* s_abort = (volatile int*)(smem + L::misc + 4);
    int32_t* s_prefix = (int32_t*)(smem + L::prefix);
    int32_t* s_ws = (int32_t*)(smem + L::warp_sums);
    // expert offsets are read from global memory (L2-resident) once per tile
    auto off_at = [&](int j) { return __ldg(p.offsets + p.expert_begin + j); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);            // the leader's expect_tx (all CTAs' bytes)
            mbar_init(empty_bar(s), 1);           // the leader's MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);           // the leader's MMA commit
            mbar_init(tempty_bar(b), NCTA * 128); // every CTA's epilogue threads
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        if constexpr (NCTA == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(s_tmem)),
                         "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(s_tmem)),
                         "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    build_tile_prefix(p.offsets, p.counts, p.expert_begin, p.n_experts, G::BM, s_prefix,
                      s_ws);  // syncs
    tc_fence_before();
    if constexpr (NCTA == 2) cluster_sync();   // both CTAs' barriers exist before cross-CTA use
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int n_tiles = s_prefix[p.n_experts] * p.n_ntiles;
    const int nk = (p.K + BK - 1) / BK;
    bool aborted = false;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer (every CTA)
        int stage = 0;
        uint32_t phase = 0;
        for (int t = unit; t < n_tiles; t += n_units) {
            const int mt = t / p.n_ntiles, ntile = t - mt * p.n_ntiles;
            const int j = find_tile_expert(s_prefix, p.n_experts, mt);
            const int row0 = off_at(j) + (mt - s_prefix[j]) * G::BM + (int)rank * BM_CTA;
            const int n0 = ntile * (GLU ? BN / 2 : BN);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, s_abort, p.dev_status)) {
                    aborted = true;
                    break;
                }
                const uint32_t fb = full_bar(stage);
                if (leader) mbar_arrive_expect_tx(fb, NCTA * G::kStageBytes);
                const uint32_t cfb = NCTA == 2 ? map_to_rank(fb, 0) : fb;
                const uint32_t sa = sbase + L::a + stage * kABytes;
                const uint32_t sb = sbase + L::b + stage * G::kBBytes;
                tma_load_2d<NCTA>(sa, &tmap_a, cfb, kb * BK, row0);
                if (GLU) {
                    if constexpr (NCTA == 2) {  // leader: gate rows, peer: the matching up rows
                        tma_load_4d<NCTA>(sb, &tmap_b, cfb, kb * BK, n0, (int)rank, j);
                    } else {                    // gate rows, then the matching up rows
                        tma_load_4d<NCTA>(sb, &tmap_b, cfb, kb * BK, n0, 0, j);
                        tma_load_4d<NCTA>(sb + G::kBBytes / 2, &tmap_b, cfb, kb * BK, n0, 1, j);
                    }
                } else {
                    tma_load_3d<NCTA>(sb, &tmap_b, cfb, kb * BK, n0 + (int)rank * G::B_ROWS, j);
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (aborted) break;
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        constexpr uint32_t idesc = make_idesc(G::BM, BN);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = unit; t < n_tiles && !aborted; t += n_units) {
            if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, s_abort, p.dev_status)) {
                aborted = true;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(full_bar(stage), phase, s_abort, p.dev_status)) {
                    aborted = true;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = sbase + L::a + stage * kABytes;
                const uint32_t sb = sbase + L::b + stage * G::kBBytes;
#pragma unroll
                for (int k = 0; k < BK / UMMA_K; ++k) {
                    umma_bf16<NCTA>(d_tmem, smem_desc_sw128(sa + k * UMMA_K * 2),
                                    smem_desc_sw128(sb + k * UMMA_K * 2), idesc,
                                    (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit<NCTA>(empty_bar(stage));   // stage free once these MMAs finish
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (aborted) break;
            umma_commit<NCTA>(tfull_bar(acc));         // accumulator ready for the epilogue
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (every CTA)
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = unit; t < n_tiles; t += n_units) {
            const int mt = t / p.n_ntiles, ntile = t - mt * p.n_ntiles;
            const int j = find_tile_expert(s_prefix, p.n_experts, mt);
            const int row0 = off_at(j) + (mt - s_prefix[j]) * G::BM + (int)rank * BM_CTA;
            const int row_end =
                min(off_at(j) + segment_rows(p.offsets, p.counts, p.expert_begin, j), p.n_rows);
            const int n0 = ntile * (GLU ? BN / 2 : BN);
            if (!mbar_wait(tfull_bar(acc), acc_phase, s_abort, p.dev_status)) {
                aborted = true;
                break;
            }
            tc_fence_after();
            const int64_t row_base = row0 + quarter * 32;
            OutT* out = reinterpret_cast<OutT*>(p.out);
            uint8_t* stage = smem + L::epi + (warp - 2) * L::stage_tile;
            const uint32_t tacc = tmem_base + lane_off + (uint32_t)(acc * BN);
            constexpr int kOutCols = GLU ? BN / 2 : BN;
#pragma unroll 1
            for (int c = 0; c < kOutCols; c += 32) {
                float v[32];
                tmem_ld32(tacc + (uint32_t)c, v);
                if (GLU) {
                    float u[32];
                    tmem_ld32(tacc + (uint32_t)(BN / 2 + c), u);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * u[i];
                } else {
                    tmem_ld_wait();
                }
                store_tile32(stage, v, lane, out, row_base, row_end, n0 + c, p.n_out);
            }
            tc_fence_before();
            if constexpr (NCTA == 2)
                mbar_arrive_signal(map_to_rank(tempty_bar(acc), 0));   // the leader's barrier
            else
                mbar_arrive_signal(tempty_bar(acc));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
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
    if constexpr (NCTA == 2) cluster_sync();   // no cross-CTA access after this
    tc_fence_after();
    if (warp == 1) {
        if constexpr (NCTA == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                         "r"(kTmemCols)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                         "r"(kTmemCols)
                         : "memory");
    }
}

// ---------------------------------------------------------------- host side
static bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides_bytes, const cuuint32_t* box) {
    return make_bf16_map(m, base, rank, dims, strides_bytes, box);
}

// CTA groups of NCTA that fit on the current device at once (one CTA per
// SM), cached per device.
template <bool GLU, typename OutT, int NCTA>
static int resident_units(size_t smem) {
    struct Tag {};
    return PerDeviceInt<Tag>::get([smem] {
        int n = current_device_sm_count() / NCTA;
        if (NCTA > 1) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(n * NCTA));
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            set_cluster_attr(cfg, attr, NCTA);
            int c = 0;
            if (cudaOccupancyMaxActiveClusters(&c, grouped_gemm_tc_kernel<GLU, OutT, NCTA>,
                                               &cfg) == cudaSuccess &&
                c > 0)
                n = c;
        }
        return n;
    });
}

template <bool GLU, typename OutT, int NCTA>
static cudaError_t launch_phase(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p,
                                cudaStream_t s) {
    auto kern = grouped_gemm_tc_kernel<GLU, OutT, NCTA>;
    constexpr size_t smem = SmemLayout<NCTA, (int)sizeof(OutT)>::alloc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(NCTA * resident_units<GLU, OutT, NCTA>(smem)));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    set_cluster_attr(cfg, attr, NCTA);
    return cudaLaunchKernelEx(&cfg, kern, ma, mb, p);
}

template <int NCTA>
static cudaError_t run_gemm(const __nv_bfloat16* a, const int32_t* offsets,
                            const int32_t* counts, int expert_begin,
                            int n_experts, int64_t n_rows, int H, int I, const __nv_bfloat16* w13,
                            const __nv_bfloat16* w2, __nv_bfloat16* h, void* y, bool y_f32,
                            int32_t* dev_status, cudaEvent_t ev_mid, cudaStream_t s) {
    using G = Geo<NCTA>;
    CUtensorMap ma1, mb1, ma2, mb2;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)H, (cuuint64_t)n_rows};
        const cuuint64_t str[1] = {(cuuint64_t)H * 2};
        const cuuint32_t box[2] = {BK, BM_CTA};
        if (!make_map(&ma1, a, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    {   // W13 as [E, 2, I, H]: a box of 128 gate (index 0) or up (index 1) rows
        const cuuint64_t dims[4] = {(cuuint64_t)H, (cuuint64_t)I, 2, (cuuint64_t)n_experts};
        const cuuint64_t str[3] = {(cuuint64_t)H * 2, (cuuint64_t)I * H * 2,
                                   (cuuint64_t)2 * I * H * 2};
        const cuuint32_t box[4] = {BK, BN / 2, 1, 1};
        if (!make_map(&mb1, w13, 4, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)I, (cuuint64_t)n_rows};
        const cuuint64_t str[1] = {(cuuint64_t)I * 2};
        const cuuint32_t box[2] = {BK, BM_CTA};
        if (!make_map(&ma2, h, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)I, (cuuint64_t)H, (cuuint64_t)n_experts};
        const cuuint64_t str[2] = {(cuuint64_t)I * 2, (cuuint64_t)H * I * 2};
        const cuuint32_t box[3] = {BK, (cuuint32_t)G::B_ROWS, 1};
        if (!make_map(&mb2, w2, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    Params p1{offsets, counts, expert_begin, n_experts, H, I, (I + BN / 2 - 1) / (BN / 2),
              (int)n_rows, h, dev_status};
    cudaError_t e = launch_phase<true, __nv_bfloat16, NCTA>(ma1, mb1, p1, s);
    if (e == cudaSuccess && ev_mid) e = cudaEventRecord(ev_mid, s);
    if (e != cudaSuccess) return e;
    Params p2{offsets, counts, expert_begin, n_experts, I, H, (H + BN - 1) / BN, (int)n_rows, y,
              dev_status};
    e = y_f32 ? launch_phase<false, float, NCTA>(ma2, mb2, p2, s)
              : launch_phase<false, __nv_bfloat16, NCTA>(ma2, mb2, p2, s);
    note_launches(2);
    return e;
}

}  // namespace tc

cudaError_t launch_grouped_gemm_tc_swap(const __nv_bfloat16* a, const int32_t* offsets,
                                        const int32_t* counts, int expert_begin, int n_experts,
                                        int64_t n_rows, int H, int I, const __nv_bfloat16* w13,
                                        const __nv_bfloat16* w2, __nv_bfloat16* h, void* y,
                                        moe_dtype y_dtype, float* y_scales, int32_t* dev_status,
                                        const gemm_gather* g, cudaEvent_t ev_mid, cudaStream_t s,
                                        bool packed, const float* row_weights,
                                        const int32_t* weight_pairs);

// Kernel choice, from the average rows per expert (known on the host
// without reading the device offsets).  The operand-swapped pair kernel
// (grouped_gemm_tc_swap.cu) pads each expert's rows to a multiple of 16 and
// streams each weight tile once per pass; measured on B200 it is faster
// from ~100 rows per expert up (dsv3-shaped prefill: 18% on the step).
// With a handful of rows per expert (decode) both kernels just stream the
// weights, and the single-CTA kernel here does so ~4% faster (more weight
// bytes in flight per SM).
static bool gemm_use_swap(int64_t n_rows, int n_experts) {
    return n_rows >= (int64_t)16 * n_experts;
}

// Whether launch_grouped_gemm_tc runs the operand-swapped kernel, the one
// with the fused gather.
bool grouped_gemm_tc_uses_swap(int64_t n_rows, int n_experts, moe_dtype y_dtype) {
    return y_dtype == MOE_E4M3 || gemm_use_swap(n_rows, n_experts);
}

// A [n_rows, H] bf16 (the payload, or its dequantised copy); W13 [n_exp, 2I,
// H]; W2 [n_exp, H, I]; h [n_rows, I] bf16; y [n_rows, H] in y_dtype: fp32,
// bf16, or e4m3 codes with fp32 block scales y_scales [n_rows, H/128] (the
// operand-swapped kernel only).  counts (may be null) cuts each expert's
// segment to its first counts[j] rows.  g (may be null; the operand-swapped
// kernel only): the gate/up operand's rows are gathered from g->src instead
// of read from A.  ev_mid (may be null) is recorded between the two phases.
// packed: the weights are in pack_weights.cu's layout (operand-swapped
// kernel).  row_weights (may be null; operand-swapped kernel): y row s is
// scaled by row_weights[weight_pairs[s]].
cudaError_t launch_grouped_gemm_tc(const __nv_bfloat16* a, const int32_t* offsets,
                                   const int32_t* counts, int expert_begin, int n_experts,
                                   int64_t n_rows, int H, int I, const __nv_bfloat16* w13,
                                   const __nv_bfloat16* w2, __nv_bfloat16* h, void* y,
                                   moe_dtype y_dtype, float* y_scales, int32_t* dev_status,
                                   const gemm_gather* g, cudaEvent_t ev_mid, cudaStream_t s,
                                   bool packed, const float* row_weights,
                                   const int32_t* weight_pairs) {
    // packed weights and row weights: the operand-swapped kernel, at any size
    if (packed || row_weights || grouped_gemm_tc_uses_swap(n_rows, n_experts, y_dtype))
        return launch_grouped_gemm_tc_swap(a, offsets, counts, expert_begin, n_experts, n_rows, H,
                                           I, w13, w2, h, y, y_dtype, y_scales, dev_status, g,
                                           ev_mid, s, packed, row_weights, weight_pairs);
    if (g) return cudaErrorInvalidValue;
    return tc::run_gemm<1>(a, offsets, counts, expert_begin, n_experts, n_rows, H, I, w13, w2, h,
                           y, y_dtype == MOE_F32, dev_status, ev_mid, s);
}

}  // namespace moe
