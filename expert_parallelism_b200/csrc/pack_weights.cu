// pack_weights.cu -- one-time re-layout of the stacked expert weights into
// 16 KB blocks that the grouped GEMM's weight loads read whole.
//
// In the stacked layout ("Expert parallelism" (Transformers docs),
// GroupedGemmParallel: W13 [E, 2I, H], W2 [E, H, I], K-major rows) one
// k-step of a weight tile is 128 rows x 128 bytes, 128 short pieces H*2
// (or I*2) bytes apart.  Packed, the same 128 x 64 tile is one contiguous
// 16 KB block, so each TMA load streams one run of DRAM.
//
//   W13 packed: block (e, fb, kb), fb < 2 * ceil(I/128), kb < ceil(H/64):
//     rows 0..63 = gate rows fb*64 .. fb*64+63, rows 64..127 = the matching
//     up rows (I + fb*64 ..), columns kb*64 .. kb*64+63; block index
//     (e * FB + fb) * KB + kb.
//   W2 packed: block (e, rb, kb), rb < 2 * ceil(H/256), kb < ceil(I/64):
//     rows rb*128 .. rb*128+127 of W2[e], columns kb*64 ..; block index
//     (e * RB + rb) * KB + kb.
// Inside a block: [128 rows][64 columns] bf16, rows 128 bytes apart.
// Rows and columns past the matrix are zero, and the row blocks run to a
// whole weight tile of the GEMM (128 gate/up features, 256 W2 rows), so no
// load of one expert reaches another's weights.
#include "common.cuh"

namespace moe {

struct PackGeo {
    int64_t blocks13, blocks2;   // per expert
    int FB, KB13, RB, KB2;
};

PackGeo pack_geo(int H, int I) {
    PackGeo g;
    g.FB = 2 * ((I + 127) / 128);
    g.KB13 = (H + 63) / 64;
    g.RB = 2 * ((H + 255) / 256);
    g.KB2 = (I + 63) / 64;
    g.blocks13 = (int64_t)g.FB * g.KB13;
    g.blocks2 = (int64_t)g.RB * g.KB2;
    return g;
}

// One thread per 16-byte piece (8 bf16) of a block: 1024 pieces per block.
__global__ void __launch_bounds__(256) pack_w13_kernel(const __nv_bfloat16* __restrict__ w13,
                                                       int64_t E, int H, int I, PackGeo g,
                                                       __nv_bfloat16* __restrict__ out) {
    const int64_t pieces = E * g.blocks13 * 1024;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < pieces;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = q >> 10;
        const int within = (int)(q & 1023);
        const int row = within >> 3, c8 = (within & 7) * 8;
        const int64_t e = b / g.blocks13;
        const int rest = (int)(b - e * g.blocks13);
        const int fb = rest / g.KB13, kb = rest - fb * g.KB13;
        const int f = fb * 64 + (row & 63);                // feature
        const int col = kb * 64 + c8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (f < I && col < H) {
            const int64_t src_row = (int64_t)e * 2 * I + (row < 64 ? f : I + f);
            v = ld_nc_v4(w13 + src_row * H + col);
        }
        st_v4(out + q * 8, v);
    }
}

__global__ void __launch_bounds__(256) pack_w2_kernel(const __nv_bfloat16* __restrict__ w2,
                                                      int64_t E, int H, int I, PackGeo g,
                                                      __nv_bfloat16* __restrict__ out) {
    const int64_t pieces = E * g.blocks2 * 1024;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < pieces;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = q >> 10;
        const int within = (int)(q & 1023);
        const int row = within >> 3, c8 = (within & 7) * 8;
        const int64_t e = b / g.blocks2;
        const int rest = (int)(b - e * g.blocks2);
        const int rb = rest / g.KB2, kb = rest - rb * g.KB2;
        const int n = rb * 128 + row;
        const int col = kb * 64 + c8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < H && col < I) v = ld_nc_v4(w2 + ((int64_t)e * H + n) * I + col);
        st_v4(out + q * 8, v);
    }
}

size_t packed_weights_bytes(int64_t E, int H, int I, int which) {
    const PackGeo g = pack_geo(H, I);
    return (size_t)E * (which == 0 ? g.blocks13 : g.blocks2) * 16384;
}

cudaError_t launch_pack_weights(const __nv_bfloat16* w13, const __nv_bfloat16* w2, int64_t E,
                                int H, int I, __nv_bfloat16* p13, __nv_bfloat16* p2,
                                cudaStream_t s) {
    const PackGeo g = pack_geo(H, I);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)(sms * 8);
    if (w13) pack_w13_kernel<<<grid, 256, 0, s>>>(w13, E, H, I, g, p13);
    if (w2) pack_w2_kernel<<<grid, 256, 0, s>>>(w2, E, H, I, g, p2);
    note_launches((w13 ? 1 : 0) + (w2 ? 1 : 0));
    return cudaGetLastError();
}

}  // namespace moe
