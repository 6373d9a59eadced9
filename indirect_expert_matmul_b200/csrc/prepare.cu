// One-time repack of Q8_0 expert weights into the tile-major form streamed by
// the GEMM and mat-vec kernels (layout in common.cuh: 32-row sub-blocks inside
// each 128-row, 64-column block).  Each thread produces one (expert, row,
// 64-column tile) piece: two 32-byte halves of u = q + 128 and the two fp16
// scales.  Padding rows / columns get u = 128 (q = 0), d = 0.
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
        const int sb = r / kSubRows, rs = r % kSubRows, nr = sub_rows(L.rows(mt), sb);
        uint8_t* blk = dst + L.block(e, mt, kt) + (size_t)sb * L.sub_bytes();
        uint16_t* d_out = (uint16_t*)(blk + (size_t)nr * kTileK + (size_t)rs * 4);
        for (int h = 0; h < 2; ++h) {
            const int b = kt * 2 + h;  // Q8_0 block index along the row
            uint8_t* q_out = blk + (size_t)h * nr * 32 + (size_t)rs * 32;
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

// MXFP4: each thread produces one (expert, row, 64-column tile) piece from two
// 17-byte source blocks (scale byte X, then 16 bytes: element i of the block
// in the low nibble of byte i, element 16 + i in its high nibble): 32 bytes of
// codes, byte j holding column 2j (low nibble) and 2j + 1 (high nibble), and
// the two scale bytes.  Padding gets code 0 (zero) and scale 127 (one), never
// the NaN scale 255.
__global__ void prepare_mxfp4_kernel(const uint8_t* __restrict__ src, int E, WLayout L, uint8_t* __restrict__ dst) {
    const int64_t total = (int64_t)E * L.n_out_pad * L.kt_count;
    const int nb = L.n_in / 32;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int kt = (int)(idx % L.kt_count);
        const int64_t er = idx / L.kt_count;
        const int row = (int)(er % L.n_out_pad);
        const int e = (int)(er / L.n_out_pad);
        const int mt = row / kTileM, r = row % kTileM;
        const int sb = r / kSubRows, rs = r % kSubRows, nr = sub_rows(L.rows(mt), sb);
        uint8_t* blk = dst + L.block(e, mt, kt) + (size_t)sb * L.sub_bytes();
        __align__(16) uint8_t codes[32];
        uint8_t xs[2] = {127, 127};
        for (int h = 0; h < 2; ++h) {
            const int b = kt * 2 + h;  // source block index along the row
            const bool live = row < L.n_out && b < nb;
            const uint8_t* sblk = live ? src + (((int64_t)e * L.n_out + row) * nb + b) * 17 : nullptr;
            if (live) xs[h] = sblk[0];
            for (int j = 0; j < 16; ++j) {  // columns 32h + 2j, 32h + 2j + 1 = elements 2j, 2j + 1
                uint8_t lo = 0, hi = 0;
                if (live) {
                    const int i0 = 2 * j, i1 = 2 * j + 1;
                    lo = i0 < 16 ? (sblk[1 + i0] & 15) : (sblk[1 + i0 - 16] >> 4);
                    hi = i1 < 16 ? (sblk[1 + i1] & 15) : (sblk[1 + i1 - 16] >> 4);
                }
                codes[16 * h + j] = (uint8_t)(lo | (hi << 4));
            }
        }
        uint4* o = (uint4*)(blk + (size_t)rs * 32);
        o[0] = *(const uint4*)codes;
        o[1] = *(const uint4*)(codes + 16);
        blk[(size_t)nr * 32 + (size_t)rs * 2] = xs[0];
        blk[(size_t)nr * 32 + (size_t)rs * 2 + 1] = xs[1];
    }
}

moe_status launch_prepare(int wtype, const void* src, int E, int n_out, int n_in, void* dst, cudaStream_t stream) {
    WLayout L(n_out, n_in, wtype);
    int64_t total = (int64_t)E * L.n_out_pad * L.kt_count;
    if (total == 0) return MOE_OK;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (wtype == MOE_MXFP4)
        prepare_mxfp4_kernel<<<(unsigned)blocks, 256, 0, stream>>>((const uint8_t*)src, E, L, (uint8_t*)dst);
    else
        prepare_kernel<<<(unsigned)blocks, 256, 0, stream>>>((const uint8_t*)src, E, L, (uint8_t*)dst);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
