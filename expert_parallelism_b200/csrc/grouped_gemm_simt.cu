// grouped_gemm_simt.cu -- fp32 grouped SwiGLU expert FFN on the CUDA cores,
// plus the FP8-payload dequantisation the tensor-core path consumes.
//
// Source: "Expert parallelism and all-to-all", "Walking through one MoE
// layer", step 3 (each GPU runs its local experts on the rows it received
// as one grouped matrix multiply).
//
// The fp32 workload needs fp32 products and sums (its tolerance is 1e-5 of
// the row RMS), which rules out the tensor cores' reduced-precision fp32
// input formats; it runs as a shared-memory tiled FFMA GEMM.  Each CTA
// owns a 64x64 output tile of one expert (rows from device offsets, see
// tile_schedule.cuh); each thread accumulates a 4x4 block in registers in
// ascending-K order.  The gate/up phase keeps two accumulators and applies
// silu(g) * u in the epilogue.
#include "common.cuh"
#include "tile_schedule.cuh"

namespace moe {

constexpr int kSimtBM = 64, kSimtBN = 64, kSimtBK = 16;

__device__ __forceinline__ float silu_f32(float g) { return __fdiv_rn(g, 1.0f + expf(-g)); }

// GLU: C[r, n] = silu(A_r . B[n]) * (A_r . B[I + n]), n < Nout (= I)
// else: C[r, n] = A_r . B[n], n < Nout
template <typename TA, typename TW, bool GLU>
__global__ void __launch_bounds__(256) simt_grouped_gemm_kernel(
    const TA* __restrict__ A, int K, const TW* __restrict__ B, int Nout,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts, int expert_begin,
    int n_experts, int64_t n_rows, TW* __restrict__ C) {
    __shared__ int32_t s_prefix[MOE_MAX_EXPERTS + 1];
    __shared__ int32_t s_ws[8];
    __shared__ float As[kSimtBK][kSimtBM + 4];
    __shared__ float Bg[kSimtBK][kSimtBN + 4];
    __shared__ float Bu[GLU ? kSimtBK : 1][kSimtBN + 4];

    build_tile_prefix(offsets, counts, expert_begin, n_experts, kSimtBM, s_prefix, s_ws);
    const int total_tiles = s_prefix[n_experts];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int n0 = blockIdx.x * kSimtBN;
    const int64_t brows = GLU ? 2 * (int64_t)Nout : (int64_t)Nout;

    for (int mt = blockIdx.y; mt < total_tiles; mt += gridDim.y) {
        const int j = find_tile_expert(s_prefix, n_experts, mt);
        const int64_t row0 = offsets[expert_begin + j] + (int64_t)(mt - s_prefix[j]) * kSimtBM;
        const int64_t row_end =
            min((int64_t)offsets[expert_begin + j] + segment_rows(offsets, counts, expert_begin, j),
                n_rows);
        const TW* Bj = B + (int64_t)j * brows * K;
        float acc_g[4][4], acc_u[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc_g[a][b] = acc_u[a][b] = 0.0f;

        for (int k0 = 0; k0 < K; k0 += kSimtBK) {
#pragma unroll
            for (int l = 0; l < 4; ++l) {
                const int id = threadIdx.x + l * 256;     // 0..1023 = 64 rows x 16 k
                const int r = id >> 4, kk = id & 15;
                const int64_t row = row0 + r;
                const int kg = k0 + kk;
                As[kk][r] = (row < row_end && kg < K) ? to_f32(A[row * K + kg]) : 0.0f;
                const int n = n0 + r;
                Bg[kk][r] = (n < Nout && kg < K) ? to_f32(Bj[(int64_t)n * K + kg]) : 0.0f;
                if (GLU)
                    Bu[kk][r] = (n < Nout && kg < K) ? to_f32(Bj[(int64_t)(Nout + n) * K + kg])
                                                     : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kSimtBK; ++kk) {
                float a[4], bg[4], bu[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    a[i] = As[kk][ty * 4 + i];
                    bg[i] = Bg[kk][tx * 4 + i];
                    if (GLU) bu[i] = Bu[kk][tx * 4 + i];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        acc_g[i][c] = fmaf(a[i], bg[c], acc_g[i][c]);
                        if (GLU) acc_u[i][c] = fmaf(a[i], bu[c], acc_u[i][c]);
                    }
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t row = row0 + ty * 4 + i;
            if (row >= row_end) continue;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int n = n0 + tx * 4 + c;
                if (n >= Nout) continue;
                const float v = GLU ? silu_f32(acc_g[i][c]) * acc_u[i][c] : acc_g[i][c];
                C[row * Nout + n] = from_f32<TW>(v);
            }
        }
    }
}

// A_s = bf16(decode(q) * scale) for the rows of experts [begin, begin+n).
__global__ void __launch_bounds__(256) dequant_e4m3_kernel(const uint8_t* __restrict__ q,
                                                           const float* __restrict__ scales,
                                                           const int32_t* __restrict__ offsets,
                                                           int expert_begin, int n_experts, int H,
                                                           int64_t n_rows,
                                                           __nv_bfloat16* __restrict__ out) {
    const int64_t r0 = max((int64_t)offsets[expert_begin], (int64_t)0);
    const int64_t r1 = min((int64_t)offsets[expert_begin + n_experts], n_rows);
    const int nblk = H / 128;
    const int64_t nv = (r1 - r0) * (H / 8);
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nv;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e0 = r0 * H + v * 8;
        const int64_t row = e0 / H;
        const int col = (int)(e0 - row * H);
        const float sc = scales[row * nblk + col / 128];
        const uint2 w = *reinterpret_cast<const uint2*>(q + e0);
        const uint32_t words[2] = {w.x, w.y};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int hpart = 0; hpart < 2; ++hpart) {
                const __nv_fp8x2_storage_t pr =
                    (__nv_fp8x2_storage_t)((words[i] >> (16 * hpart)) & 0xFFFFu);
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pr, __NV_E4M3);
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
                o[2 * i + hpart] = pack_bf16x2(__fmul_rn(f.x, sc), __fmul_rn(f.y, sc));
            }
        }
        st_v4(out + e0, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

static int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

cudaError_t launch_dequant_e4m3(const uint8_t* q, const float* scales, const int32_t* offsets,
                                int expert_begin, int n_experts, int64_t n_rows, int H,
                                __nv_bfloat16* out, cudaStream_t s) {
    const int64_t nv = n_rows * (H / 8);
    int64_t grid = (nv + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    dequant_e4m3_kernel<<<(unsigned)grid, 256, 0, s>>>(q, scales, offsets, expert_begin,
                                                        n_experts, H, n_rows, out);
    note_launches(1);
    return cudaGetLastError();
}

template <typename TA, typename TW>
static cudaError_t simt_two_phase(const TA* xp, const int32_t* offsets, const int32_t* counts,
                                  int expert_begin, int n_experts, int64_t n_rows, int H, int I,
                                  const TW* w13, const TW* w2, TW* h, TW* y, cudaEvent_t ev_mid,
                                  cudaStream_t s) {
    int64_t gy = (n_rows + kSimtBM - 1) / kSimtBM + n_experts;
    if (gy > 65535) gy = 65535;
    const dim3 g1((I + kSimtBN - 1) / kSimtBN, (unsigned)gy);
    simt_grouped_gemm_kernel<TA, TW, true><<<g1, 256, 0, s>>>(
        xp, H, w13, I, offsets, counts, expert_begin, n_experts, n_rows, h);
    if (ev_mid) cudaEventRecord(ev_mid, s);
    const dim3 g2((H + kSimtBN - 1) / kSimtBN, (unsigned)gy);
    simt_grouped_gemm_kernel<TW, TW, false><<<g2, 256, 0, s>>>(
        h, I, w2, H, offsets, counts, expert_begin, n_experts, n_rows, y);
    note_launches(2);
    return cudaGetLastError();
}

cudaError_t launch_grouped_gemm_simt_f32(const float* xp, const int32_t* offsets,
                                         const int32_t* counts, int expert_begin, int n_experts,
                                         int64_t n_rows, int H, int I, const float* w13,
                                         const float* w2, float* h, float* y, cudaEvent_t ev_mid,
                                         cudaStream_t s) {
    return simt_two_phase<float, float>(xp, offsets, counts, expert_begin, n_experts, n_rows, H,
                                        I, w13, w2, h, y, ev_mid, s);
}

}  // namespace moe

