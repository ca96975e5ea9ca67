// permute.cu -- write each token's hidden vector into the slots of its k
// pairs (expert-major slabs), optionally quantised to an FP8 e4m3 payload
// with one fp32 scale per 128-element block.
//
// Source: "Expert Parallelism" (aiwiki), "Implementation" (sent =
// x[order]: one contiguous slab per destination); "Expert parallelism and
// all-to-all", "Traffic math" (FP8 activations, 1 byte per element).
//
// The copy runs token-major: a CTA reads x[t] once (16-byte vector loads
// that do not allocate in L1) and stores it to its k slots, so HBM sees
// T*H*b bytes of reads and N*H*b' bytes of writes, the algorithmic
// minimum.  In FP8 mode 8 lanes own one 128-element block: they reduce
// amax with shuffles, divide by 448 (IEEE), and convert x/scale (IEEE
// division) with the hardware's round-to-nearest-even, saturating cvt.
#include "common.cuh"

namespace moe {

constexpr int kMaxTopK = MOE_MAX_TOPK;

// Destinations of token t's k pairs: the rank (-1: skipped) and the row in
// that rank's buffer, into shared memory.  Flags MOE_DEV_OVERFLOW for a
// plan row outside the receive buffers.
__device__ __forceinline__ void token_dests(const int32_t* __restrict__ slot_of_pair,
                                            const PairRows& map, int64_t t, int k,
                                            int* s_rank, int64_t* s_row, int32_t* dev_status) {
    if (threadIdx.x < k) {
        const int64_t p = t * k + threadIdx.x;
        const int32_t slot = slot_of_pair[p];
        int rank = -1;
        int64_t row = -1;
        if (slot >= 0 && !pair_row(map, p, slot, rank, row)) {
            rank = -1;
            flag_status(dev_status, MOE_DEV_OVERFLOW);
        }
        s_rank[threadIdx.x] = rank;
        s_row[threadIdx.x] = row;
    }
}

constexpr int kPermuteMaxThreads = 512;

template <typename T>
__global__ void __launch_bounds__(kPermuteMaxThreads) permute_copy_kernel(const T* __restrict__ x, int64_t T_,
                                                           int H, int k,
                                                           const int32_t* __restrict__ slot_of_pair,
                                                           const PairRows map,
                                                           const __grid_constant__ RankPtrs dst,
                                                           int32_t* dev_status) {
    __shared__ int s_rank[kMaxTopK];
    __shared__ int64_t s_row[kMaxTopK];
    const int nvec = H * (int)sizeof(T) / 16;
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        token_dests(slot_of_pair, map, t, k, s_rank, s_row, dev_status);
        __syncthreads();
        const char* src = reinterpret_cast<const char*>(x + t * H);
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
            const uint4 d = ld_nc_v4(src + (size_t)v * 16);
            for (int j = 0; j < k; ++j) {
                const int r = s_rank[j];
                if (r >= 0)
                    st_v4(reinterpret_cast<char*>(reinterpret_cast<T*>(dst.rows[r]) + s_row[j] * H) +
                              (size_t)v * 16,
                          d);
            }
        }
        __syncthreads();
    }
}

// 8 consecutive elements of a row as fp32.
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
    float a[4], b[4];
    unpack16(ld_nc_v4(p), a);
    unpack16(ld_nc_v4(p + 4), b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[i] = a[i];
        f[4 + i] = b[i];
    }
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
    unpack16(ld_nc_v4(p), f);
}

constexpr int kMaxBlocks = 64;           // scales staged in shared memory: H <= 8192

__device__ __forceinline__ void st_v2(void* p, uint32_t x, uint32_t y) {
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(x), "r"(y) : "memory");
}

// FP8 payload: one CTA per token (grid-stride).  8 lanes own a 128-element
// block, lane i its elements 8i..8i+7 and 64+8i..64+8i+7, so every store
// instruction of the 8 lanes covers whole 32-byte sectors (64 bytes of codes,
// 128 bytes of bf16): amax by shuffles, scale = amax / 448, and 8-byte
// stores of codes to each of the token's k destinations.  The
// token's scales are staged in shared memory and written as 16-byte vectors
// per destination once the row is done.  With `a` non-null (the layer call,
// local layout), the kernel also writes what the grouped GEMM consumes,
// bf16(decode(q) * scale) (an fp32 product rounded to bf16), to each slot's
// row of `a`, so the GEMM needs no separate dequantisation pass.  With
// dst.rows[0] null (the token-major form, for the GEMM's fused gather) only
// `a` is written, at the token's own row t: each token is quantised once and
// its k copies are the same row.
template <typename T>
__global__ void __launch_bounds__(kPermuteMaxThreads) permute_e4m3_kernel(
    const T* __restrict__ x, int64_t T_, int H, int k, const int32_t* __restrict__ slot_of_pair,
    const PairRows map, const __grid_constant__ RankPtrs dst, __nv_bfloat16* __restrict__ a,
    int32_t* dev_status) {
    __shared__ int s_rank[kMaxTopK];
    __shared__ int64_t s_row[kMaxTopK];
    __shared__ __align__(16) float s_scale[kMaxBlocks];
    const int nblk = H / 128;
    const int l8 = threadIdx.x & 7;                 // lane within the block's 8
    const int grp = threadIdx.x >> 3;               // block handled in this pass
    const int ngrp = blockDim.x >> 3;
    const bool tok_major = dst.rows[0] == nullptr;
    const bool vec_scales = !tok_major && (nblk % 4) == 0 && nblk <= kMaxBlocks;
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        if (!tok_major) token_dests(slot_of_pair, map, t, k, s_rank, s_row, dev_status);
        __syncthreads();
        const T* row = x + t * H;
        // whole warps iterate together so the 8-lane shuffles stay converged
        for (int g0 = 0; g0 < nblk; g0 += ngrp) {
            const int g = g0 + grp;
            const bool live = g < nblk;
            float f[16];
            float amax = 0.0f;
            if (live) {
                float a8[8], b8[8];
                load8(row + g * 128 + l8 * 8, a8);         // elements 8 l8 ..
                load8(row + g * 128 + 64 + l8 * 8, b8);    // elements 64 + 8 l8 ..
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    f[i] = a8[i];
                    f[8 + i] = b8[i];
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
            }
#pragma unroll
            for (int off = 4; off > 0; off >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            if (!live) continue;
            const float scale = e4m3_block_scale(amax);
            const uint4 q = make_uint4(quant4_e4m3(f[0], f[1], f[2], f[3], scale),
                                       quant4_e4m3(f[4], f[5], f[6], f[7], scale),
                                       quant4_e4m3(f[8], f[9], f[10], f[11], scale),
                                       quant4_e4m3(f[12], f[13], f[14], f[15], scale));
            for (int j = 0; j < k && !tok_major; ++j) {
                const int r = s_rank[j];
                if (r >= 0) {
                    uint8_t* d = reinterpret_cast<uint8_t*>(dst.rows[r]) + s_row[j] * H + g * 128;
                    st_v2(d + l8 * 8, q.x, q.y);
                    st_v2(d + 64 + l8 * 8, q.z, q.w);
                }
            }
            if (a) {
                // the GEMM's operand: each code decoded (exact) times the scale
                const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
                uint32_t bw[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 lo = decode2_e4m3((uint16_t)(qw[i] & 0xFFFFu));
                    const float2 hi = decode2_e4m3((uint16_t)(qw[i] >> 16));
                    bw[2 * i] = pack_bf16x2(__fmul_rn(lo.x, scale), __fmul_rn(lo.y, scale));
                    bw[2 * i + 1] = pack_bf16x2(__fmul_rn(hi.x, scale), __fmul_rn(hi.y, scale));
                }
                const uint4 b0 = make_uint4(bw[0], bw[1], bw[2], bw[3]);
                const uint4 b1 = make_uint4(bw[4], bw[5], bw[6], bw[7]);
                if (tok_major) {
                    __nv_bfloat16* d = a + t * H + g * 128;
                    st_v4(d + l8 * 8, b0);
                    st_v4(d + 64 + l8 * 8, b1);
                }
                for (int j = 0; j < k && !tok_major; ++j) {
                    if (s_rank[j] < 0) continue;
                    __nv_bfloat16* d = a + s_row[j] * H + g * 128;
                    st_v4(d + l8 * 8, b0);
                    st_v4(d + 64 + l8 * 8, b1);
                }
            }
            if (l8 == 0 && !tok_major) {
                if (vec_scales) {
                    s_scale[g] = scale;
                } else {
                    for (int j = 0; j < k; ++j)
                        if (s_rank[j] >= 0) dst.scales[s_rank[j]][s_row[j] * nblk + g] = scale;
                }
            }
        }
        if (vec_scales) {
            __syncthreads();
            const int nvec = nblk / 4;              // 16-byte pieces of one row's scales
            for (int i = threadIdx.x; i < k * nvec; i += blockDim.x) {
                const int j = i / nvec, v = i - j * nvec;
                const int r = s_rank[j];
                if (r >= 0)
                    st_v4(dst.scales[r] + s_row[j] * nblk + v * 4,
                          *reinterpret_cast<const uint4*>(s_scale + v * 4));
            }
        }
        __syncthreads();
    }
}

// Threads per CTA for `units` equal pieces of work per token (16-byte
// vectors, or 8 threads per 128-element FP8 block): as few equal rounds as
// a CTA of at most 512 threads allows, so no thread idles in the last one.
static int permute_threads(int units, int per_unit) {
    const int work = units * per_unit;
    const int rounds = (work + kPermuteMaxThreads - 1) / kPermuteMaxThreads;
    const int t = ((work + rounds - 1) / rounds + 31) / 32 * 32;
    return t < 32 ? 32 : t;
}

static unsigned permute_grid(int64_t T) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 8;  // 8 CTAs of 256 threads fill an SM
    return (unsigned)(T < cap ? T : cap);
}

static RankPtrs one_rank(void* rows, float* scales) {
    RankPtrs d{};
    d.rows[0] = rows;
    d.scales[0] = scales;
    return d;
}

// Every routed pair's payload row to its destination: slot_of_pair's slot of
// the local buffer (map.send_base null, dst.rows[0] = xp), or a row of its
// expert's owner under an expert-parallel plan.  a_bf16 (may be null; FP8
// payload, local layout only): also write the GEMM's bf16 operand
// bf16(decode(q) * scale) for every slot.
cudaError_t launch_permute_to(const void* x, moe_dtype xdt, int64_t T, int H, int k,
                              const int32_t* slot_of_pair, const PairRows& map,
                              const RankPtrs& dst, moe_dtype xpdt, __nv_bfloat16* a_bf16,
                              int32_t* dev_status, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const unsigned grid = permute_grid(T);
    if (xpdt == MOE_E4M3) {
        const int th = permute_threads(H / 128, 8);
        if (xdt == MOE_BF16)
            permute_e4m3_kernel<__nv_bfloat16><<<grid, th, 0, s>>>(
                (const __nv_bfloat16*)x, T, H, k, slot_of_pair, map, dst, a_bf16, dev_status);
        else
            permute_e4m3_kernel<float><<<grid, th, 0, s>>>((const float*)x, T, H, k, slot_of_pair,
                                                           map, dst, a_bf16, dev_status);
    } else if (xdt == MOE_BF16) {
        permute_copy_kernel<__nv_bfloat16><<<grid, permute_threads(H * 2 / 16, 1), 0, s>>>(
            (const __nv_bfloat16*)x, T, H, k, slot_of_pair, map, dst, dev_status);
    } else {
        permute_copy_kernel<float><<<grid, permute_threads(H * 4 / 16, 1), 0, s>>>(
            (const float*)x, T, H, k, slot_of_pair, map, dst, dev_status);
    }
    note_launches(1);
    return cudaGetLastError();
}

// The local layout: xp[slot_of_pair[t*k + j]] = x[t].
cudaError_t launch_permute(const void* x, moe_dtype xdt, int64_t T, int H, int k,
                           const int32_t* slot_of_pair, void* xp, moe_dtype xpdt,
                           float* xp_scales, __nv_bfloat16* a_bf16, cudaStream_t s) {
    const PairRows local{nullptr, nullptr, nullptr, 1, 0};
    return launch_permute_to(x, xdt, T, H, k, slot_of_pair, local, one_rank(xp, xp_scales), xpdt,
                             a_bf16, nullptr, s);
}

// Token-major FP8 round trip for the GEMM's fused gather: a[t] =
// bf16(decode(q) * scale) of x[t]'s FP8 payload, one row per token.
cudaError_t launch_quantize_tokens_e4m3(const void* x, moe_dtype xdt, int64_t T, int H,
                                       __nv_bfloat16* a, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const unsigned grid = permute_grid(T);
    const PairRows local{nullptr, nullptr, nullptr, 1, 0};
    const RankPtrs none = one_rank(nullptr, nullptr);
    const int th = permute_threads(H / 128, 8);
    if (xdt == MOE_BF16)
        permute_e4m3_kernel<__nv_bfloat16><<<grid, th, 0, s>>>(
            (const __nv_bfloat16*)x, T, H, 1, nullptr, local, none, a, nullptr);
    else
        permute_e4m3_kernel<float><<<grid, th, 0, s>>>((const float*)x, T, H, 1, nullptr, local,
                                                       none, a, nullptr);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
