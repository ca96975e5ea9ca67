// grouped_gemm_tc.cu -- bf16 grouped SwiGLU expert FFN on the 5th-generation
// tensor cores (tcgen05 MMA, accumulators in tensor memory, operands staged
// by TMA), for sm_100a.
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
//                   B tile = 128 gate rows + the 128 matching up rows, so one
//                   M=128 x N=256 accumulator holds gate in columns 0..127
//                   and up in 128..255; the epilogue fuses SwiGLU.
//   phase 2:        y[s, n0:n0+256] = h_s W2^T
// Rows come in expert segments [off[j], off[j+1]) read from device memory
// (tile_schedule.cuh); a 128-row M-tile never mixes experts: rows past the
// segment end are computed from whatever TMA loads there and discarded.
//
// CTA = 6 warps, one CTA per SM (the 4-stage smem ring takes ~200 KB):
//   warp 0      TMA producer (one thread): A tile 128x64 + B tile 256x64
//               per stage, 128-byte swizzle, mbarrier transaction counts.
//   warp 1      tensor-memory allocator and MMA issuer (one thread):
//               4 x tcgen05.mma (K=16) per stage into one of two
//               accumulator buffers (2 x 256 TMEM columns); tcgen05.commit
//               frees the smem stage and, after the last K step, hands the
//               buffer to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes (warp w owns
//               lanes 32*(w%4)..), SwiGLU / bf16 conversion, global stores;
//               double buffering overlaps them with the next tile's MMAs.
// Tiles are (M-tile, N-tile) pairs in M-major order, N fastest, dealt
// round-robin over the persistent CTAs: the CTAs running at one time share
// few experts' weights (read from HBM once) and A rows (reused from L2).
// Every wait is bounded; on timeout the kernel records MOE_DEV_TIMEOUT,
// drains what it has in flight (also bounded), frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tile_schedule.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;             // rows per tile (MMA M)
constexpr int BN = 256;             // accumulator columns per tile (MMA N)
constexpr int BK = 64;              // K per stage: one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;          // K per tcgen05.mma (kind::f16)
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kABytes = BM * BK * 2;               // 16 KB
constexpr int kBBytes = BN * BK * 2;               // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;     // 48 KB
constexpr int kTmemCols = 2 * BN;                  // two accumulator buffers

struct Smem {
    // offsets inside the 1024-aligned dynamic shared memory block
    static constexpr int a = 0;
    static constexpr int b = kStages * kABytes;
    static constexpr int bars = b + kStages * kBBytes;          // 8-byte barriers
    static constexpr int n_bars = 2 * kStages + 4 + 1;          // full, empty, tfull x2, tempty x2, drain
    static constexpr int misc = bars + n_bars * 8;               // tmem addr, abort flag
    static constexpr int prefix = misc + 16;                     // int32 [MOE_MAX_EXPERTS + 1]
    static constexpr int offs = prefix + (MOE_MAX_EXPERTS + 1) * 4;
    static constexpr int warp_sums = offs + (MOE_MAX_EXPERTS + 1) * 4;
    static constexpr int total = warp_sums + 32 * 4;
};
constexpr size_t kSmemBytes = Smem::total + 1024;   // + alignment slack

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
        "selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false (after flagging the CTA-wide abort) on timeout, or if another role
// aborted first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* dev_status, uint64_t limit_ns = kSpinLimitNs) {
    uint64_t deadline = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            if (*abort_flag) return false;
            const uint64_t now = global_timer_ns();
            if (deadline == 0) {
                deadline = now + limit_ns;
            } else if (now > deadline) {
                *abort_flag = 1;
                flag_status(dev_status, MOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Shared-memory matrix descriptor for a K-major, 128-byte-swizzled bf16
// tile whose rows are 128 bytes apart and whose 8-row groups are 1024 bytes
// apart (exactly what a TMA box of 64 x rows with SWIZZLE_128B writes).
// Fields: start address >> 4 [0,14), leading byte offset >> 4 [16,30)
// (1: unused for this layout), stride byte offset >> 4 [32,46) (1024 B),
// descriptor version 1 [46,48), layout SWIZZLE_128B = 2 [61,64).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at
// bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t make_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float silu(float g) { return __fdiv_rn(g, 1.0f + expf(-g)); }

// ---------------------------------------------------------------- kernel
struct Params {
    const int32_t* offsets;   // global expert offsets (device)
    int expert_begin, n_experts;
    int K;                    // reduction length (H in phase 1, I in phase 2)
    int n_out;                // output columns (I in phase 1, H in phase 2)
    int n_ntiles;             // N tiles per M tile
    int n_rows;               // rows of A and out: stores never go past it
    void* out;                // h (phase 1, bf16) or y (phase 2, OutT), row stride n_out
    int32_t* dev_status;
};

// 32 consecutive fp32 results of one row: 4 x 16-byte bf16 stores or
// 8 x 16-byte fp32 stores, skipping pieces past n_out (n_out % 8 == 0).
__device__ __forceinline__ void store_row32(__nv_bfloat16* orow, int col0, int n_out,
                                            const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int col = col0 + q * 8;
        if (col < n_out)
            st_v4(orow + col, make_uint4(pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]),
                                         pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]),
                                         pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]),
                                         pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7])));
    }
}
__device__ __forceinline__ void store_row32(float* orow, int col0, int n_out,
                                            const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int col = col0 + q * 4;
        if (col < n_out)
            st_v4(orow + col, make_uint4(__float_as_uint(v[q * 4 + 0]), __float_as_uint(v[q * 4 + 1]),
                                         __float_as_uint(v[q * 4 + 2]), __float_as_uint(v[q * 4 + 3])));
    }
}

template <bool GLU, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t bar0 = sbase + Smem::bars;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);
    uint32_t* s_tmem = (uint32_t*)(smem + Smem::misc);
    volatile int* s_abort = (volatile int*)(smem + Smem::misc + 4);
    int32_t* s_prefix = (int32_t*)(smem + Smem::prefix);
    int32_t* s_off = (int32_t*)(smem + Smem::offs);
    int32_t* s_ws = (int32_t*)(smem + Smem::warp_sums);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 128);
        }
        mbar_init(drain_bar, 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int j = threadIdx.x; j <= p.n_experts; j += blockDim.x)
        s_off[j] = p.offsets[p.expert_begin + j];
    build_tile_prefix(p.offsets, p.expert_begin, p.n_experts, BM, s_prefix, s_ws);  // syncs
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int n_tiles = s_prefix[p.n_experts] * p.n_ntiles;
    const int nk = (p.K + BK - 1) / BK;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0;
        int issued_phase[kStages];
        for (int s = 0; s < kStages; ++s) issued_phase[s] = -1;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            const int mt = t / p.n_ntiles, ntile = t - mt * p.n_ntiles;
            const int j = find_tile_expert(s_prefix, p.n_experts, mt);
            const int row0 = s_off[j] + (mt - s_prefix[j]) * BM;
            const int n0 = ntile * (GLU ? BN / 2 : BN);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, s_abort, p.dev_status)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = full_bar(stage);
                mbar_arrive_expect_tx(fb, kStageBytes);
                const uint32_t sa = sbase + Smem::a + stage * kABytes;
                const uint32_t sb = sbase + Smem::b + stage * kBBytes;
                tma_load_2d(sa, &tmap_a, fb, kb * BK, row0);
                if (GLU) {
                    tma_load_4d(sb, &tmap_b, fb, kb * BK, n0, 0, j);
                    tma_load_4d(sb + kBBytes / 2, &tmap_b, fb, kb * BK, n0, 1, j);
                } else {
                    tma_load_3d(sb, &tmap_b, fb, kb * BK, n0, j);
                }
                issued_phase[stage] = (int)phase;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {  // abort: let the copies already issued land before exiting
            for (int s = 0; s < kStages; ++s)
                if (issued_phase[s] >= 0)
                    mbar_wait(full_bar(s), (uint32_t)issued_phase[s], s_abort, p.dev_status,
                              200ull * 1000 * 1000);
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = make_idesc(BM, BN);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        bool issued_any = false;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, s_abort, p.dev_status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait(full_bar(stage), phase, s_abort, p.dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = sbase + Smem::a + stage * kABytes;
                const uint32_t sb = sbase + Smem::b + stage * kBBytes;
#pragma unroll
                for (int k = 0; k < BK / UMMA_K; ++k) {
                    umma_bf16(d_tmem, smem_desc_sw128(sa + k * UMMA_K * 2),
                              smem_desc_sw128(sb + k * UMMA_K * 2), idesc,
                              (kb > 0 || k > 0) ? 1u : 0u);
                }
                issued_any = true;
                umma_commit(empty_bar(stage));   // smem stage free once these MMAs finish
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            umma_commit(tfull_bar(acc));         // accumulator ready for the epilogue
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (!ok && issued_any) {  // abort: wait for the MMAs in flight before TMEM is freed
            umma_commit(drain_bar);
            mbar_wait(drain_bar, 0, s_abort, p.dev_status, 200ull * 1000 * 1000);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
            const int mt = t / p.n_ntiles, ntile = t - mt * p.n_ntiles;
            const int j = find_tile_expert(s_prefix, p.n_experts, mt);
            const int row0 = s_off[j] + (mt - s_prefix[j]) * BM;
            const int row_end = min(s_off[j + 1], p.n_rows);
            const int n0 = ntile * (GLU ? BN / 2 : BN);
            if (!mbar_wait(tfull_bar(acc), acc_phase, s_abort, p.dev_status)) break;
            tc_fence_after();
            const int row = row0 + quarter * 32 + lane;
            const bool row_ok = row < row_end;
            OutT* orow = reinterpret_cast<OutT*>(p.out) + (int64_t)row * p.n_out;
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
                if (row_ok) store_row32(orow, n0 + c, p.n_out, v);
            }
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

// Tiled bf16 tensor map, 128-byte swizzle, zero fill out of bounds.
static bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides_bytes, const cuuint32_t* box) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t elem[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                    dims, strides_bytes, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static int num_sms() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <bool GLU, typename OutT>
static cudaError_t launch_phase(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p,
                                cudaStream_t s) {
    auto kern = grouped_gemm_tc_kernel<GLU, OutT>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<num_sms(), kThreads, kSmemBytes, s>>>(ma, mb, p);
    return cudaGetLastError();
}

}  // namespace tc

// A [n_rows, H] bf16 (the payload, or its dequantised copy); W13 [n_exp, 2I,
// H]; W2 [n_exp, H, I]; h [n_rows, I] bf16; y [n_rows, H] in y_f32 ? fp32 : bf16.
cudaError_t launch_grouped_gemm_tc(const __nv_bfloat16* a, const int32_t* offsets,
                                   int expert_begin, int n_experts, int64_t n_rows, int H, int I,
                                   const __nv_bfloat16* w13, const __nv_bfloat16* w2,
                                   __nv_bfloat16* h, void* y, bool y_f32, int32_t* dev_status,
                                   cudaStream_t s) {
    using namespace tc;
    CUtensorMap ma1, mb1, ma2, mb2;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)H, (cuuint64_t)n_rows};
        const cuuint64_t str[1] = {(cuuint64_t)H * 2};
        const cuuint32_t box[2] = {BK, BM};
        if (!make_map(&ma1, a, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)H, (cuuint64_t)I, 2, (cuuint64_t)n_experts};
        const cuuint64_t str[3] = {(cuuint64_t)H * 2, (cuuint64_t)I * H * 2,
                                   (cuuint64_t)2 * I * H * 2};
        const cuuint32_t box[4] = {BK, BN / 2, 1, 1};
        if (!make_map(&mb1, w13, 4, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)I, (cuuint64_t)n_rows};
        const cuuint64_t str[1] = {(cuuint64_t)I * 2};
        const cuuint32_t box[2] = {BK, BM};
        if (!make_map(&ma2, h, 2, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)I, (cuuint64_t)H, (cuuint64_t)n_experts};
        const cuuint64_t str[2] = {(cuuint64_t)I * 2, (cuuint64_t)H * I * 2};
        const cuuint32_t box[3] = {BK, BN, 1};
        if (!make_map(&mb2, w2, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    Params p1{offsets, expert_begin, n_experts, H, I, (I + BN / 2 - 1) / (BN / 2), (int)n_rows,
              h, dev_status};
    cudaError_t e = launch_phase<true, __nv_bfloat16>(ma1, mb1, p1, s);
    if (e != cudaSuccess) return e;
    Params p2{offsets, expert_begin, n_experts, I, H, (H + BN - 1) / BN, (int)n_rows, y,
              dev_status};
    e = y_f32 ? launch_phase<false, float>(ma2, mb2, p2, s)
              : launch_phase<false, __nv_bfloat16>(ma2, mb2, p2, s);
    note_launches(2);
    return e;
}

}  // namespace moe
