// One-time repack of Q8_0 expert weights into the tile-major form streamed by
// the GEMM and mat-vec kernels (layout in common.cuh).  Each thread produces
// one (expert, row, 64-column tile) piece: two 32-byte halves of u = q + 128
// and the two fp16 scales.  Padding rows / columns get u = 128 (q = 0), d = 0.
#include "common.cuh"

namespace moe {

__global__ void prepare_kernel(const uint8_t* __restrict__ src, int E, WLayout L, uint8_t* __restrict__ dst) {
    const int64_t total = (int64_t)E * L.n_out_pad * L.kt_count;
    const int nb = L.n_in / 32;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int kt = (int)(idx % L.kt_count);
        const int64_t er = idx / L.kt_count;
        const int row = (int)(er % L.n_out_pad);
        const int e = (int)(er / L.n_out_pad);
        const int mt = row / kTileM, r = row % kTileM;
        const int rows = L.rows(mt);
        uint8_t* blk = dst + L.block(e, mt, kt);
        uint16_t* d_out = (uint16_t*)(blk + (size_t)rows * kTileK + (size_t)r * 4);
        for (int h = 0; h < 2; ++h) {
            const int b = kt * 2 + h;  // Q8_0 block index along the row
            uint8_t* q_out = blk + (size_t)h * rows * 32 + (size_t)r * 32;
            uint16_t d = 0;
            uint32_t words[8];
            if (row < L.n_out && b < nb) {
                const uint8_t* s = src + (((int64_t)e * L.n_out + row) * nb + b) * 34;
                d = (uint16_t)(s[0] | (s[1] << 8));
                for (int w = 0; w < 8; ++w) {
                    uint32_t v = 0;
                    for (int j = 0; j < 4; ++j) v |= (uint32_t)(uint8_t)(s[2 + w * 4 + j] ^ 0x80u) << (8 * j);
                    words[w] = v;
                }
            } else {
                for (int w = 0; w < 8; ++w) words[w] = 0x80808080u;
            }
            uint4* o = (uint4*)q_out;
            o[0] = make_uint4(words[0], words[1], words[2], words[3]);
            o[1] = make_uint4(words[4], words[5], words[6], words[7]);
            d_out[h] = d;
        }
    }
}

moe_status launch_prepare(const void* src, int E, int n_out, int n_in, void* dst, cudaStream_t stream) {
    WLayout L(n_out, n_in);
    int64_t total = (int64_t)E * L.n_out_pad * L.kt_count;
    if (total == 0) return MOE_OK;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    prepare_kernel<<<(unsigned)blocks, 256, 0, stream>>>((const uint8_t*)src, E, L, (uint8_t*)dst);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
