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
// minimum.  In FP8 mode 16 lanes own one 128-element block: they reduce
// amax with shuffles, divide by 448 (IEEE), and convert x/scale (IEEE
// division) with the hardware's round-to-nearest-even, saturating cvt.
#include "common.cuh"

namespace moe {

constexpr int kMaxTopK = MOE_MAX_TOPK;

template <typename T>
__global__ void __launch_bounds__(256) permute_copy_kernel(const T* __restrict__ x, int64_t T_,
                                                           int H, int k,
                                                           const int32_t* __restrict__ slot_of_pair,
                                                           T* __restrict__ xp) {
    __shared__ int32_t s_slot[kMaxTopK];
    const int nvec = H * (int)sizeof(T) / 16;
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        if (threadIdx.x < k) s_slot[threadIdx.x] = slot_of_pair[t * k + threadIdx.x];
        __syncthreads();
        const char* src = reinterpret_cast<const char*>(x + t * H);
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
            const uint4 d = ld_nc_v4(src + (size_t)v * 16);
            for (int j = 0; j < k; ++j) {
                const int32_t s = s_slot[j];
                if (s >= 0) st_v4(reinterpret_cast<char*>(xp + (int64_t)s * H) + (size_t)v * 16, d);
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

template <typename T>
__global__ void __launch_bounds__(256) permute_e4m3_kernel(const T* __restrict__ x, int64_t T_,
                                                           int H, int k,
                                                           const int32_t* __restrict__ slot_of_pair,
                                                           uint8_t* __restrict__ xp,
                                                           float* __restrict__ xp_scales) {
    __shared__ int32_t s_slot[kMaxTopK];
    const int nblk = H / 128;
    const int half = (threadIdx.x >> 4) & 1;   // which 16-lane half of the warp
    const int l16 = threadIdx.x & 15;
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        if (threadIdx.x < k) s_slot[threadIdx.x] = slot_of_pair[t * k + threadIdx.x];
        __syncthreads();
        // whole warps iterate together so the 16-lane shuffles stay converged
        for (int g0 = 2 * warp; g0 < nblk; g0 += 2 * nwarps) {
            const int g = g0 + half;
            const bool live = g < nblk;
            float f[8];
            float amax = 0.0f;
            if (live) {
                load8(x + t * H + g * 128 + l16 * 8, f);
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            if (!live) continue;
            float scale = __fdiv_rn(amax, 448.0f);
            if (scale == 0.0f) scale = 1.0f;
            uint32_t packed[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(f[4 * i], scale), __fdiv_rn(f[4 * i + 1], scale)),
                    __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(f[4 * i + 2], scale), __fdiv_rn(f[4 * i + 3], scale)),
                    __NV_SATFINITE, __NV_E4M3);
                packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            const uint2 q = make_uint2(packed[0], packed[1]);
            for (int j = 0; j < k; ++j) {
                const int32_t s = s_slot[j];
                if (s < 0) continue;
                *reinterpret_cast<uint2*>(xp + (int64_t)s * H + g * 128 + l16 * 8) = q;
                if (l16 == 0) xp_scales[(int64_t)s * nblk + g] = scale;
            }
        }
        __syncthreads();
    }
}

static unsigned permute_grid(int64_t T) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t cap = (int64_t)sms * 8;  // 8 CTAs of 256 threads fill an SM
    return (unsigned)(T < cap ? T : cap);
}

cudaError_t launch_permute(const void* x, moe_dtype xdt, int64_t T, int H, int k,
                           const int32_t* slot_of_pair, void* xp, moe_dtype xpdt,
                           float* xp_scales, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const unsigned grid = permute_grid(T);
    if (xpdt == MOE_E4M3) {
        if (xdt == MOE_BF16)
            permute_e4m3_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
                (const __nv_bfloat16*)x, T, H, k, slot_of_pair, (uint8_t*)xp, xp_scales);
        else
            permute_e4m3_kernel<float><<<grid, 256, 0, s>>>((const float*)x, T, H, k,
                                                            slot_of_pair, (uint8_t*)xp, xp_scales);
    } else if (xdt == MOE_BF16) {
        permute_copy_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            (const __nv_bfloat16*)x, T, H, k, slot_of_pair, (__nv_bfloat16*)xp);
    } else {
        permute_copy_kernel<float><<<grid, 256, 0, s>>>((const float*)x, T, H, k, slot_of_pair,
                                                        (float*)xp);
    }
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
