// combine.cu -- un-permute plus the router-weighted sum of each token's k
// expert outputs back into its home row.
//
// Source: "Expert Parallelism" (aiwiki), "Implementation" (y[order] =
// back); "Expert parallelism and all-to-all", "Walking through one MoE
// layer", step 4 (the home GPU takes a weighted sum into the residual
// stream).
//
// One CTA per token (grid-stride).  Each thread owns 8 consecutive output
// elements; for every pick j it loads that piece of row y[slot_of_pair[t*k
// + j]] (16-byte vector loads, all k issued before the sums), accumulates
// w_j * y in fp32 with fused multiply-adds in j order, and rounds once.
//
// With the FP8 combine payload ("Expert parallelism and all-to-all",
// "Traffic math": 1-byte activations both ways) y holds e4m3 codes with one
// fp32 scale per 128 elements; a piece is 16 codes (one 16-byte load) and
// its block's scale.  A code q adds (w * scale) * decode(q): the pick's
// weight times the block scale is one fp32 product per piece, then each
// decoded code (exact in fp32) goes in with a fused multiply-add.
//
// The all_reduce form of the layer (Transformers docs, "Expert
// parallelism", "Choosing an implementation": no token moves, every rank
// runs its experts over the whole batch, and the ranks' outputs are summed
// by an all-reduce) uses the same kernel restricted to one rank's slab of
// slots, [rank_offsets[r], rank_offsets[r+1]) read on the device, writing
// an fp32 partial; reduce_partials_kernel sums the ranks' partials in rank
// order and rounds once.
#include "common.cuh"

namespace moe {

constexpr int kCombineMaxTopK = MOE_MAX_TOPK;
constexpr int kCombineMaxThreads = 256;

__device__ __forceinline__ void load8_row(const float* p, float (&f)[8]) {
    float a[4], b[4];
    unpack16(ld_nc_v4(p), a);
    unpack16(ld_nc_v4(p + 4), b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[i] = a[i];
        f[4 + i] = b[i];
    }
}
__device__ __forceinline__ void load8_row(const __nv_bfloat16* p, float (&f)[8]) {
    unpack16(ld_nc_v4(p), f);
}

__device__ __forceinline__ void store8(float* p, const float (&f)[8]) {
    st_v4(p, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                        __float_as_uint(f[3])));
    st_v4(p + 4, make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]),
                            __float_as_uint(f[7])));
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
    st_v4(p, make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                        pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
}

// One thread's piece of a y row: load() issues its global loads (all picks'
// loads are issued before any sum), add() folds w * piece into the fp32
// accumulators in element order.  fp32 / bf16 y: 8 elements (16 bytes),
// converted at load.  e4m3 y: 16 codes (16 bytes) and the block's scale,
// kept raw until add(), so four picks in flight hold 4 x 5 registers
// instead of 4 x 16.
template <typename TY>
struct Piece {
    static constexpr int N = 8;
    struct Raw {
        float f[8];
    };
    static __device__ __forceinline__ void load(const TY* y, const float*, int64_t s, int H, int c,
                                                Raw& r) {
        load8_row(y + s * H + c * 8, r.f);
    }
    static __device__ __forceinline__ void add(float (&acc)[8], const Raw& r, float w) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, r.f[i], acc[i]);
    }
};

template <>
struct Piece<uint8_t> {
    static constexpr int N = 16;
    struct Raw {
        uint4 q;
        float sc;
    };
    static __device__ __forceinline__ void load(const uint8_t* y, const float* y_scales, int64_t s,
                                                int H, int c, Raw& r) {
        r.q = ld_nc_v4(y + s * H + c * 16);
        r.sc = __ldg(y_scales + s * (H / 128) + (c * 16) / 128);
    }
    // The pick's weight times the block's scale (one fp32 product per 16
    // codes), then one fused multiply-add per code: an FP8-y combine of dsv3
    // ran 143 us this way against 158 us with a product per code.
    static __device__ __forceinline__ void add(float (&acc)[16], const Raw& r, float w) {
        const uint32_t q[4] = {r.q.x, r.q.y, r.q.z, r.q.w};
        const float ws = __fmul_rn(w, r.sc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = decode2_e4m3((uint16_t)(q[i] & 0xFFFFu));
            const float2 b = decode2_e4m3((uint16_t)(q[i] >> 16));
            acc[4 * i + 0] = fmaf(ws, a.x, acc[4 * i + 0]);
            acc[4 * i + 1] = fmaf(ws, a.y, acc[4 * i + 1]);
            acc[4 * i + 2] = fmaf(ws, b.x, acc[4 * i + 2]);
            acc[4 * i + 3] = fmaf(ws, b.y, acc[4 * i + 3]);
        }
    }
};

// rank_offsets null: every pick.  Otherwise only picks whose slot lies in
// [rank_offsets[rank], rank_offsets[rank + 1]) (the others add nothing).
// Pick j's row is found through `map` (the local slot of src.rows[0], or a
// row of its expert's owner under an expert-parallel plan).
template <typename TY, typename TO>
__global__ void __launch_bounds__(kCombineMaxThreads, 4) combine_kernel(const __grid_constant__ RankPtrs src,
                                                      const int32_t* __restrict__ slot_of_pair,
                                                      const PairRows map,
                                                      const float* __restrict__ topk_w, int64_t T,
                                                      int k, int H, TO* __restrict__ out,
                                                      const int32_t* __restrict__ rank_offsets,
                                                      int rank, int32_t* dev_status) {
    using P = Piece<TY>;
    constexpr int EPT = P::N;
    __shared__ int s_rank[kCombineMaxTopK];
    __shared__ int64_t s_row[kCombineMaxTopK];
    __shared__ float s_w[kCombineMaxTopK];
    const int nchunk = H / EPT;
    const int32_t lo = rank_offsets ? __ldg(rank_offsets + rank) : INT32_MIN;
    const int32_t hi = rank_offsets ? __ldg(rank_offsets + rank + 1) : INT32_MAX;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < k) {
            const int64_t p = t * k + threadIdx.x;
            const int32_t sl = slot_of_pair[p];
            int r = -1;
            int64_t row = -1;
            if (sl >= lo && sl < hi && sl >= 0 && !pair_row(map, p, sl, r, row)) {
                r = -1;
                flag_status(dev_status, MOE_DEV_OVERFLOW);
            }
            s_rank[threadIdx.x] = (sl >= lo && sl < hi) ? r : -1;
            s_row[threadIdx.x] = row;
            s_w[threadIdx.x] = topk_w ? topk_w[p] : 1.0f;   // null: unit weights
        }
        __syncthreads();
        for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
            float acc[EPT];
#pragma unroll
            for (int i = 0; i < EPT; ++i) acc[i] = 0.0f;
            int j = 0;
            // four picks at a time: their loads are in flight together
            for (; j + 4 <= k; j += 4) {
                typename P::Raw v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = s_rank[j + u];
                    if (r >= 0)
                        P::load((const TY*)src.rows[r], src.scales[r], s_row[j + u], H, c, v[u]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (s_rank[j + u] >= 0) P::add(acc, v[u], s_w[j + u]);
            }
            for (; j < k; ++j) {
                const int r = s_rank[j];
                if (r < 0) continue;
                typename P::Raw v;
                P::load((const TY*)src.rows[r], src.scales[r], s_row[j], H, c, v);
                P::add(acc, v, s_w[j]);
            }
#pragma unroll
            for (int h = 0; h < EPT / 8; ++h)
                store8(out + t * H + c * EPT + 8 * h, *reinterpret_cast<float(*)[8]>(acc + 8 * h));
        }
        __syncthreads();
    }
}

static int64_t sm_grid_cap() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return (int64_t)sms * 8;   // 8 CTAs of <= 256 threads per SM
}

// The combine over rows found through `map` in the buffers of `src`.
// rank_offsets (may be null): restrict to rank `rank`'s slab of slots.
cudaError_t launch_combine_from(const RankPtrs& src, moe_dtype ydt, const int32_t* slot_of_pair,
                                const PairRows& map, const float* topk_w, int64_t T, int k, int H,
                                void* out, moe_dtype odt, int32_t* dev_status, cudaStream_t s,
                                const int32_t* rank_offsets, int rank) {
    if (T == 0) return cudaSuccess;
    const int64_t cap = sm_grid_cap();
    const unsigned grid = (unsigned)(T < cap ? T : cap);
    // a token's pieces in as few equal rounds as a CTA of at most 256
    // threads allows (no thread idles in the last round).  Small CTAs, many
    // per SM, overlap one token's slot loads with another's rows: measured
    // on B200, an FP8-y combine of dsv3 took 156 us with 224-thread CTAs and
    // 175 us with 448-thread ones.
    const int ept = ydt == MOE_E4M3 ? 16 : 8;
    const int pieces = H / ept;
    const int rounds = (pieces + kCombineMaxThreads - 1) / kCombineMaxThreads;
    int threads = (((pieces + rounds - 1) / rounds) + 31) / 32 * 32;
    threads = threads < 32 ? 32 : threads;
#define MOE_COMBINE(TY, TO)                                                                  \
    combine_kernel<TY, TO><<<grid, threads, 0, s>>>(src, slot_of_pair, map, topk_w, T, k, H, \
                                                    (TO*)out, rank_offsets, rank, dev_status)
    if (ydt == MOE_E4M3 && odt == MOE_BF16) MOE_COMBINE(uint8_t, __nv_bfloat16);
    else if (ydt == MOE_E4M3) MOE_COMBINE(uint8_t, float);
    else if (ydt == MOE_BF16 && odt == MOE_BF16) MOE_COMBINE(__nv_bfloat16, __nv_bfloat16);
    else if (ydt == MOE_BF16) MOE_COMBINE(__nv_bfloat16, float);
    else if (odt == MOE_BF16) MOE_COMBINE(float, __nv_bfloat16);
    else MOE_COMBINE(float, float);
#undef MOE_COMBINE
    note_launches(1);
    return cudaGetLastError();
}

// The local layout: y rows at slot_of_pair's slots of y.
cudaError_t launch_combine(const void* y, moe_dtype ydt, const float* y_scales,
                           const int32_t* slot_of_pair, const float* topk_w, int64_t T, int k,
                           int H, void* out, moe_dtype odt, cudaStream_t s,
                           const int32_t* rank_offsets, int rank) {
    RankPtrs src{};
    src.rows[0] = const_cast<void*>(y);
    src.scales[0] = const_cast<float*>(y_scales);
    const PairRows local{nullptr, nullptr, nullptr, 1, 0};
    return launch_combine_from(src, ydt, slot_of_pair, local, topk_w, T, k, H, out, odt, nullptr,
                               s, rank_offsets, rank);
}

// out[i] = (((p[0][i] + p[1][i]) + p[2][i]) + ...) in fp32, rounded once to
// TO; each thread owns 8 consecutive elements (16-byte loads), n_elems % 8
// == 0.  With one partial it is the rounding after an all-reduce.
template <typename TO>
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float* __restrict__ p, int n,
                                                              int64_t n_elems,
                                                              TO* __restrict__ out) {
    const int64_t nvec = n_elems / 8;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nvec;
         v += (int64_t)gridDim.x * blockDim.x) {
        float acc[8];
        load8_row(p + v * 8, acc);
        for (int r = 1; r < n; ++r) {
            float f[8];
            load8_row(p + (int64_t)r * n_elems + v * 8, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], f[i]);
        }
        store8(out + v * 8, acc);
    }
}

cudaError_t launch_reduce_partials(const float* partials, int n, int64_t n_elems, void* out,
                                   moe_dtype odt, cudaStream_t s) {
    if (n_elems == 0) return cudaSuccess;
    const int64_t nvec = n_elems / 8;
    int64_t grid = (nvec + 255) / 256;
    const int64_t cap = sm_grid_cap();
    if (grid > cap) grid = cap;
    if (odt == MOE_BF16)
        reduce_partials_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, s>>>(
            partials, n, n_elems, (__nv_bfloat16*)out);
    else
        reduce_partials_kernel<float><<<(unsigned)grid, 256, 0, s>>>(partials, n, n_elems,
                                                                    (float*)out);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
