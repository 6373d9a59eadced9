// Shared definitions of the sm_100a MoE indirect-matmul library: status
// handling, workspace and repacked-weight layouts, and thin PTX wrappers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ----------------------------------------------------------------- limits
constexpr int kMaxExperts = 16384;
constexpr int64_t kMaxTokens = (int64_t)1 << 22;  // exclusive
constexpr int kMaxK = 1 << 10;                      // exclusive

// ------------------------------------------------------- device status word
// The first error sticks (compare-and-swap from MOE_OK).
__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }
__device__ __forceinline__ int read_status(const int* status) { return *(volatile const int*)status; }

// ------------------------------------------------------------ repacked weights
// Tile-major form: per expert, per 128-row tile mt, per 64-column tile kt, one
// block of rows(mt) rows, itself cut into sub-blocks of 32 rows (the last one
// 16 rows when rows(mt) is not a multiple of 32).  Any run of consecutive
// 32-row sub-blocks of one k-step is contiguous, so a row sub-tile of 32, 64
// or 128 rows is one copy per k-step.  A sub-block of nr rows holds, per type:
//  Q8_0  (68 bytes a row): nr*32 bytes of u = q + 128 for columns [0, 32) of
//        each row (32 bytes per row), then nr*32 bytes for columns [32, 64),
//        then nr*4 bytes of scales (two fp16 per row, one per 32-column half);
//  MXFP4 (34 bytes a row): nr*32 bytes of 4-bit E2M1 codes (32 bytes per row:
//        byte j holds column 2j in its low nibble and 2j+1 in its high
//        nibble), then nr*2 bytes of E8M0 scales (one per 32-column half).
// rows(mt) = min(128, n_out_pad - 128*mt), n_out_pad = round_up(n_out, 16).
constexpr int kTileM = 128;
constexpr int kTileK = 64;
constexpr int kRowBytes = kTileK + 4;  // Q8_0: 64 q bytes + 2 fp16 scales
constexpr int kRowBytesMx = 32 + 2;    // MXFP4: 64 codes + 2 scale bytes
constexpr int kSubRows = 32;           // rows of a sub-block

struct WLayout {
    int n_out, n_in, n_out_pad, kt_count, mt_count;
    int rb;  // bytes of one row of one k-step: kRowBytes (Q8_0) or kRowBytesMx (MXFP4)
    int64_t expert_bytes;
    __host__ __device__ WLayout() {}
    __host__ __device__ WLayout(int n_out_, int n_in_, int wtype = MOE_Q8_0) : n_out(n_out_), n_in(n_in_) {
        rb = wtype == MOE_MXFP4 ? kRowBytesMx : kRowBytes;
        n_out_pad = (n_out + 15) / 16 * 16;
        kt_count = (n_in + kTileK - 1) / kTileK;
        mt_count = (n_out_pad + kTileM - 1) / kTileM;
        expert_bytes = (int64_t)n_out_pad * kt_count * rb;
    }
    __host__ __device__ int rows(int mt) const {
        int r = n_out_pad - mt * kTileM;
        return r < kTileM ? r : kTileM;
    }
    // byte offset of block (e, mt, kt)
    __host__ __device__ int64_t block(int e, int mt, int kt) const {
        return e * expert_bytes + (int64_t)mt * kTileM * kt_count * rb + (int64_t)rows(mt) * kt * rb;
    }
    __host__ __device__ int sub_bytes() const { return kSubRows * rb; }  // one full sub-block
};

// Inside a k-step block of `rows` rows: row r lies in sub-block r / 32, which
// starts (r / 32) * sub_bytes() into the block and holds sub_rows(rows, r / 32) rows.
__host__ __device__ __forceinline__ int sub_rows(int rows, int sb) {
    const int r = rows - sb * kSubRows;
    return r < kSubRows ? r : kSubRows;
}


// ------------------------------------------------------------------ workspace
// Rows of the tile-major activation buffers of the grouped GEMM: every
// expert's sorted range starts on a multiple of 8 rows (so the 128-byte
// swizzle of an 8-row atom is position-independent), plus slack for a 16-row
// rounding of the last column tile.
inline int64_t tiled_rows(int64_t S, int n_groups) {
    return S + 8 * (S < n_groups ? S : n_groups) + 32;
}
// The row-id pass over several CTAs (up to kRidMaxCtas, for up to kRidMaxE
// experts) keeps its per-CTA counts, first positions and per-expert padding
// offsets in the workspace: 2 * kRidMaxCtas * E + E words.
constexpr int kRidMaxCtas = 64;
constexpr int kRidMaxE = 1024;
struct WsLayout {
    int64_t S, rows_pad, rows_pad_sh;
    size_t hdr, rid, src1, dst, sprow, bounds, active, tiles, pad, h, h_sh, xt, xt_sh, xs, xs_sh, total;
    static size_t up(size_t v) { return (v + 255) / 256 * 256; }
    WsLayout(int64_t n_tokens, int k, int n_experts, int n_in, int n_hidden, int n_hidden_sh, int x_type) {
        (void)x_type;
        S = n_tokens * k;
        rows_pad = tiled_rows(S, n_experts);
        rows_pad_sh = n_tokens + 32;
        const int64_t kin = (n_in + 63) / 64, khid = (n_hidden + 63) / 64, khs = (n_hidden_sh + 63) / 64;
        const size_t h_gemv = (size_t)S * n_hidden * 2, h_gemm = (size_t)rows_pad * khid * 128;
        const size_t hs_gemv = (size_t)n_tokens * n_hidden_sh * 2, hs_gemm = (size_t)rows_pad_sh * khs * 128;
        size_t o = 0;
        hdr = o; o += 256;
        src1 = o; o += up(S * 4);
        dst = o; o += up(S * 4);
        sprow = o; o += up(S * 4);  // tiled row of each slot t*k+s
        bounds = o; o += up((size_t)(n_experts + 1) * 4);
        rid = o; o += n_experts <= kRidMaxE ? up(((size_t)2 * kRidMaxCtas * n_experts + n_experts) * 4) : 0;
        active = o; o += up((size_t)(n_experts + 1) * 4);
        tiles = o; o += up((size_t)(n_experts + 1) * 4);
        pad = o; o += up((size_t)(n_experts + 1) * 4);
        h = o; o += up(h_gemv > h_gemm ? h_gemv : h_gemm);
        h_sh = o; o += up(hs_gemv > hs_gemm ? hs_gemv : hs_gemm);
        xt = o; o += up((size_t)rows_pad * kin * 128);
        xt_sh = o; o += n_hidden_sh > 0 ? up((size_t)rows_pad_sh * kin * 128) : 0;
        xs = o; o += up((size_t)rows_pad * 4);  // power-of-two scale of each tiled activation row
        xs_sh = o; o += n_hidden_sh > 0 ? up((size_t)rows_pad_sh * 4) : 0;
        total = o;
    }
};
// header words
constexpr int kHdrStatus = 0;
constexpr int kHdrActive = 1;
constexpr int kHdrTiles = 2;   // total column tiles of the grouped GEMM
constexpr int kHdrWaitSite = 3;  // first expired wait: 1<<30 | warp<<20 | shared address of its barrier
constexpr int kHdrDone = 4;      // CTAs of a finalising mat-vec launch that have finished
constexpr int kGemmBN = 192;   // column (token) tile of the grouped GEMM

// ---------------------------------------------------------------- profiling
void prof_begin(cudaStream_t s);                     // start of an operator call
void prof_mark(cudaStream_t s, const char* stage, int launches = 1);  // after the launch(es) of `stage`

// ------------------------------------------------------------------ dequant
// u = q + 128 as a byte; f = as_float(0x47000000 | u << 8) = 32768 + u exactly.
// fma(f, d, -32896*d) = (u - 128) * d = q * d, exact in fp32: q*d needs at most
// 7 + 11 significant bits and 32896*d at most 9 + 11, so neither the constant
// nor the single rounding of the fma loses anything.
__device__ __forceinline__ float magic_byte(uint32_t word, int byte) {
    uint32_t f;
    // select byte `byte` of word into bits 8..15 of 0x47000000
    const uint32_t sel = 0x7404u | ((uint32_t)byte << 4);
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(f) : "r"(word), "r"(0x47000000u), "r"(sel));
    return __uint_as_float(f);
}

}  // namespace moe
