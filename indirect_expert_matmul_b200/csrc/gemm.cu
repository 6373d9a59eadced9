// Grouped per-expert GEMM on the sm_100a tensor cores with the Q8_0
// dequantisation fused into the tile pipeline - the prompt-size path of
// GGML_OP_MUL_MAT_ID (the PR #283 article "ik_llama.cpp 的 CUDA 更优 MoE 实现",
// sections 2.1 and 6: gather src1 rows by ids_src1, multiply per expert, write
// dst rows by ids_dst), restated for Blackwell.
//
// Tile = (expert e, column tile j of up to 192 of the expert's sorted slots,
// row unit mt).  One persistent CTA per SM walks tiles in (e, j, mt) order, so
// CTAs running together share the gathered activations (and an expert's later
// column tiles find its weights in L2).  Every output element is produced by
// exactly one CTA with one fixed reduction order: the result is bit-identical
// from run to run.
//
// The dequantised weights (A) live in tensor memory, beside the two fp32
// accumulators; the activations (B) come from shared memory (128-byte-swizzled,
// K-major).  Shared-memory bandwidth (128 bytes a clock per SM, shared by the
// tensor core's operand reads and every copy and load) is what bounds a k-step
// when A too is staged there: A written and read back costs 64 KB a k-step on
// top of the raw weights and activations.  Warp roles (640 threads):
//   warp 0      weight producer: L2 prefetch and 1-D bulk copies of the
//               repacked int8+scale blocks of both A sources.
//   warp 1      TMEM allocation and the single thread issuing tcgen05.mma
//               (M=128, N=16..192, K=16 per instruction, A from tensor memory).
//               It touches no shared memory between k-steps: any shared-memory
//               access by the issuing thread (an mbarrier wait, even one that
//               passes, or a plain load) waits for its MMAs in flight to drain,
//               ~250 cycles a k-step, more than half the MMA time of a
//               96-column tile.
//   warp 3      the MMA warp's waits: the accumulators free at a tile's start,
//               then each k-step's A and B stages; it meets warp 1 at a named
//               barrier whose AND carries "ready" (false: abort).
//   warp 2      activation producer: one bulk copy per k-step of the
//               pre-swizzled, tile-major activation rows.
//   warps 4-19  four per tensor-memory lane quarter (warp % 4):
//               dequantisation, int8 q + fp16 d -> q*d rounded once to the
//               operand type, one row of one matrix a thread on alternate
//               k-steps, converted in registers before the stage is free and
//               then stored into tensor memory (a warp may only write its own
//               lane quarter); and the epilogue: tcgen05.ld of the
//               accumulators, SwiGLU of the gate/up pair to bf16 h, or fp32
//               rows scattered to dst by ids_dst.
// All waits are bounded; an expired wait sets MOE_ERR_TIMEOUT in the status
// word and every role leaves its loop.
#include "common.cuh"
#include "gemm_api.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kGemmThreads = 640;
constexpr int kWarpProdA = 0;   // weight blocks: L2 prefetch + bulk copies
constexpr int kWarpMma = 1;     // TMEM allocation + tcgen05.mma issue
constexpr int kWarpProdB = 2;   // activation tiles: bulk copies
constexpr int kWarpWait = 3;    // the MMA warp's mbarrier waits
constexpr uint32_t kBarIssue = 8;  // named barrier: warp 3 hands each k-step to warp 1 (64 threads)
constexpr int kWorkWarp0 = 4;   // warps 4-19: dequantisation and epilogue, four per lane quarter
constexpr int kWorkWarps = 16;
static_assert(kGemmBN <= 3 * 64, "a worker holds the output rows of three 16-column chunks");
constexpr uint32_t kBTileBytes = kGemmBN * kTileK * 2; // 24 KB
constexpr uint32_t kRawBytes = kTileM * kRowBytes;     // 8704
constexpr int kSmemGroups = 256;                       // schedule tables kept in shared memory up to this
constexpr int kPrefetchSteps = 8;                      // weight k-steps prefetched into L2 ahead of use
constexpr long long kWaitLimitCycles = 1ll << 32;      // ~2 s
constexpr uint32_t kSleepNs = 20000;                   // upper bound of one hardware wait
// Tensor memory (512 columns): two fp32 accumulators of kGemmBN columns, then
// kMA stages of the dequantised A operands, each two 128 x 64 matrices of
// 16-bit values (32 columns a matrix: lane = row, two K values a column).
constexpr uint32_t kAccCols = kGemmBN;
constexpr int kMA = 2;
constexpr uint32_t kACol0 = 2 * kAccCols;
static_assert(kACol0 + kMA * 64 <= 512, "accumulators and A stages fill tensor memory");
constexpr int kRS = 4;   // raw weight stages (int8 + scales of both matrices)
constexpr int kMB = 3;   // activation (B) stages
// Dequantisation warps take alternate k-steps by parity: with an even number
// of raw and A stages every stage is always filled and drained by the same
// group, so no group can mistake another phase of a stage for its own.
static_assert(kRS % 2 == 0 && kMA % 2 == 0, "ring stages are owned by one k-step parity");

struct Cfg {
    static constexpr uint32_t b_off = 0;
    static constexpr uint32_t raw_off = b_off + kMB * kBTileBytes;
    static constexpr uint32_t bar_off = raw_off + kRS * 2 * kRawBytes;
    static constexpr int n_bars = 2 * kRS + 2 * kMA + 2 * kMB + 3;
    static constexpr uint32_t misc_off = bar_off + n_bars * 8;
    static constexpr uint32_t smem_bytes = misc_off + 64 + 1024;  // + alignment slack
};

struct GemmParams {
    const uint8_t* A0;
    const uint8_t* A1;
    WLayout L;
    int n_groups;               // > 0: grouped by bounds / ntile_prefix; 0: one group of n_rows
    const int32_t* bounds;      // [n_groups + 1] sorted-position ranges
    const int32_t* ntile_prefix;// [n_groups + 1] column-tile prefix
    const int32_t* pad_start;   // [n_groups + 1] first row of each group in the tile-major buffers
    int n_rows;
    const uint8_t* B;           // activations, tile-major: [kt][b_rows][128 B], 128-byte swizzled
    int64_t b_rows;             // rows per k-plane of B
    const int32_t* dst_rows;    // output row of sorted position p (null: p)
    float* out;                 // single-matrix output
    uint8_t* h;                 // dual output (SwiGLU), tile-major like B: [kt][h_rows][128 B]
    int64_t h_rows;
    int out_ld;
    int* hdr;
    int bf16;                   // operand type: 1 bf16, 0 fp16
    int wtype;                  // A operand: MOE_Q8_0, or MOE_MXFP4 (bf16 operands)
    const float* col_scale;     // per tiled row of B (a tile column): factor the accumulator takes (null: 1)
    long long wait_limit;       // cycles a wait may take before the launch gives up (MOE_ERR_TIMEOUT)
    int stall_cta, stall_stage; // test only: that CTA's activation copy of that k-step is never issued (-1: off)
};

struct Tile {
    int e, mt, p0, n, p0pad;  // p0pad: first row of the tile in the tile-major buffers
};

__device__ __forceinline__ Tile decode_tile(int t, int mt_count, const GemmParams& p, const int* s_prefix,
                                            const int* s_bounds, const int* s_pad) {
    Tile r;
    const int q = t / mt_count;
    r.mt = t - q * mt_count;
    if (p.n_groups == 0) {
        r.e = 0;
        r.p0 = q * kGemmBN;
        r.p0pad = r.p0;
        r.n = min(kGemmBN, p.n_rows - r.p0);
        return r;
    }
    const bool in_smem = p.n_groups <= kSmemGroups;
    const int* pre = in_smem ? s_prefix : p.ntile_prefix;
    const int* bnd = in_smem ? s_bounds : p.bounds;
    const int* pad = in_smem ? s_pad : p.pad_start;
    // largest e with pre[e] <= q (empty experts share their successor's prefix)
    int lo = 0, hi = p.n_groups;  // invariant: pre[lo] <= q < pre[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (pre[mid] <= q) lo = mid; else hi = mid;
    }
    r.e = lo;
    const int j = q - pre[lo];
    r.p0 = bnd[lo] + j * kGemmBN;
    r.p0pad = pad[lo] + j * kGemmBN;
    r.n = min(kGemmBN, bnd[lo + 1] - r.p0);
    return r;
}

// Bounded wait by one lane; false when the kernel is aborting.  The lane
// sleeps in hardware between polls (suspend-time hint), so waiting roles do
// not take issue slots from the dequantisation warps.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                         long long limit) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (ptx::mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            *abort_flag = 1;
            const int site = (1 << 30) | ((int)(threadIdx.x >> 5) << 20) | (int)(ptx::smem_u32(bar) & 0xfffffu);
            atomicCAS(status + (kHdrWaitSite - kHdrStatus), 0, site);
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
}

// lane 0 waits, the warp learns the outcome
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          long long limit) {
    // every lane polls (no lane-0 branch); lanes that see different phases simply poll again
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (ptx::mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            if ((threadIdx.x & 31) == 0) {
                *abort_flag = 1;
                const int site = (1 << 30) | ((int)(threadIdx.x >> 5) << 20) | (int)(ptx::smem_u32(bar) & 0xfffffu);
                atomicCAS(status + (kHdrWaitSite - kHdrStatus), 0, site);
                set_status(status, MOE_ERR_TIMEOUT);
            }
            return false;
        }
    }
}

// Operand type is a template parameter: a runtime choice inside the unrolled
// dequantisation loop costs a compare and branch per packed pair.
template <int BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *(uint32_t*)&v;
    }
    __half2 v = __floats2half2_rn(lo, hi);
    return *(uint32_t*)&v;
}

// pack2 of a packed fp32 pair (low lane first)
template <int BF16>
__device__ __forceinline__ uint32_t pack2x(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return pack2<BF16>(lo, hi);
}

// Two A operands per tile share each activation tile: DUAL=1 gate and up of
// one 128-row tile (SwiGLU epilogue into h); DUAL=0 two consecutive 128-row
// tiles of one matrix (fp32 scatter to dst).  BF16: operand type bf16 (1) or
// fp16 (0), which must equal p.bf16.
// 16 quantised bytes (16 consecutive K values of one row) -> 8 packed pairs of
// operand values in K order, exact: q*d rounded once to the operand type.
// d2: the row's fp16 scale in both halves (fp16 route); dsc: the same as fp32.
template <int BF16>
__device__ __forceinline__ void dequant16(uint4 x, uint32_t d2, float dsc, uint32_t* pk) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    if (BF16) {
        const uint64_t dd = ptx::f2pack(dsc, dsc);
        const uint64_t nd = ptx::f2pack(-32896.0f * dsc, -32896.0f * dsc);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            pk[2 * j] = pack2x<BF16>(ptx::fma2(ptx::f2pack(magic_byte(w[j], 0), magic_byte(w[j], 1)), dd, nd));
            pk[2 * j + 1] = pack2x<BF16>(ptx::fma2(ptx::f2pack(magic_byte(w[j], 2), magic_byte(w[j], 3)), dd, nd));
        }
    } else {
        // {0x64, u} is the fp16 value 1024 + u; minus 1152 is q (exact); times d rounds once
        const __half2 off = __float2half2_rn(1152.0f);
        const __half2 d = *(const __half2*)&d2;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t lo, hi;
            asm("prmt.b32 %0, %1, %2, 0x7170;" : "=r"(lo) : "r"(w[j]), "r"(0x64646464u));
            asm("prmt.b32 %0, %1, %2, 0x7372;" : "=r"(hi) : "r"(w[j]), "r"(0x64646464u));
            const __half2 vlo = __hmul2(__hsub2(*(const __half2*)&lo, off), d);
            const __half2 vhi = __hmul2(__hsub2(*(const __half2*)&hi, off), d);
            pk[2 * j] = *(const uint32_t*)&vlo;
            pk[2 * j + 1] = *(const uint32_t*)&vhi;
        }
    }
}

// E8M0 scale byte -> 2^(x - 127) as a float (x = 0: 2^-127; x = 255: NaN).
__device__ __forceinline__ float e8m0_scale(uint32_t x) {
    return x == 0u ? __uint_as_float(0x00400000u) : x == 255u ? __uint_as_float(0x7fc00000u) : __uint_as_float(x << 23);
}

// 8 MXFP4 codes (one 32-bit word, code i in bits 4i..4i+3; consecutive
// columns) -> 4 packed pairs of bf16 operand values, exact: the pair
// conversion to f16 is exact (two significant bits), the power-of-two scale
// is exact in float, and the product has at most two significant bits.
__device__ __forceinline__ void dequant_mx8(uint32_t w, float s, uint32_t* pk) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 v = *(const __half2*)&h[i];
        const __nv_bfloat162 b = __floats2bfloat162_rn(__low2float(v) * s, __high2float(v) * s);
        pk[i] = *(const uint32_t*)&b;
    }
}

// WT: weight type of the A operand (MOE_Q8_0, or MOE_MXFP4 with BF16 = 1).
template <int DUAL, int BF16, int WT>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_kernel(const GemmParams p) {
    extern __shared__ uint8_t smem_dyn[];
    __shared__ int s_prefix[kSmemGroups + 1];
    __shared__ int s_bounds[kSmemGroups + 1];
    __shared__ int s_pad[kSmemGroups + 1];

    if (read_status(p.hdr + kHdrStatus) != 0) return;

    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_dyn + 1023) & ~(uintptr_t)1023);
    uint8_t* sB = smem + Cfg::b_off;
    uint8_t* sRaw = smem + Cfg::raw_off;
    const uint32_t raw_sa = ptx::smem_u32(sRaw);
    uint64_t* bars = (uint64_t*)(smem + Cfg::bar_off);
    uint64_t* raw_full = bars;
    uint64_t* raw_empty = raw_full + kRS;
    uint64_t* a_full = raw_empty + kRS;
    uint64_t* a_empty = a_full + kMA;
    uint64_t* b_full = a_empty + kMA;
    uint64_t* b_empty = b_full + kMB;
    uint64_t* tmem_full = b_empty + kMB;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* mma_drained = tmem_empty + 1;
    uint32_t* tmem_base_sh = (uint32_t*)(smem + Cfg::misc_off);
    volatile int* abort_flag = (volatile int*)(smem + Cfg::misc_off + 4);
    int* status = p.hdr + kHdrStatus;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const WLayout L = p.L;
    const int MT = L.mt_count, KT = L.kt_count;
    const int MU = DUAL ? MT : (MT + 1) / 2;  // row units per column tile

    // the two A sources of a tile: (block pointer at kt = 0, rows)
    auto source = [&](const Tile& tl, int i, const uint8_t*& ptr, int& rows, int& mt) {
        if (DUAL) {
            mt = tl.mt;
            rows = L.rows(mt);
            ptr = (i ? p.A1 : p.A0) + L.block(tl.e, mt, 0);
        } else {
            mt = 2 * tl.mt + i;
            rows = mt < MT ? L.rows(mt) : 0;
            ptr = p.A0 + (mt < MT ? L.block(tl.e, mt, 0) : 0);
        }
    };

    if (tid == 0) {
        for (int i = 0; i < kRS; ++i) {
            ptx::mbar_init(&raw_full[i], 1);
            ptx::mbar_init(&raw_empty[i], kWorkWarps / 2);
        }
        for (int i = 0; i < kMA; ++i) {
            ptx::mbar_init(&a_full[i], kWorkWarps / 2);
            ptx::mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < kMB; ++i) {
            ptx::mbar_init(&b_full[i], 1);
            ptx::mbar_init(&b_empty[i], 1);
        }
        ptx::mbar_init(tmem_full, 1);
        ptx::mbar_init(tmem_empty, kWorkWarps);
        ptx::mbar_init(mma_drained, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(tmem_base_sh, 512);
        ptx::tmem_relinquish();
    }
    if (p.n_groups > 0 && p.n_groups <= kSmemGroups) {
        for (int i = tid; i <= p.n_groups; i += kGemmThreads) {
            s_prefix[i] = p.ntile_prefix[i];
            s_bounds[i] = p.bounds[i];
            s_pad[i] = p.pad_start[i];
        }
    }
    const int n_coltiles = p.n_groups > 0 ? p.hdr[kHdrTiles] : (p.n_rows + kGemmBN - 1) / kGemmBN;
    const int total = n_coltiles * MU;
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_base_sh;

    if (warp == kWarpProdA) {
        // ---------------------------------------------------- weight producer
        // One lane streams both sources' weight blocks: an L2 prefetch runs
        // kPrefetchSteps k-steps ahead of the bulk copies into the raw ring.
        if (lane == 0) {
            int rs = 0;
            uint32_t rph = 0;
            uint32_t used = 0, par = 0;  // per-stage issue record, for draining
            int pf_t = blockIdx.x, pf_kt = 0, pf_tile = -1;
            const uint8_t* pf_a[2] = {nullptr, nullptr};
            uint32_t pf_b[2] = {0u, 0u};
            auto prefetch_one = [&]() {
                if (pf_t >= total) return;
                if (pf_tile != pf_t) {
                    const Tile tl = decode_tile(pf_t, MU, p, s_prefix, s_bounds, s_pad);
                    for (int i = 0; i < 2; ++i) {
                        int rows, mt;
                        source(tl, i, pf_a[i], rows, mt);
                        pf_b[i] = (uint32_t)rows * L.rb;
                    }
                    pf_tile = pf_t;
                }
                for (int i = 0; i < 2; ++i)
                    if (pf_b[i]) ptx::bulk_prefetch_l2(pf_a[i] + (size_t)pf_kt * pf_b[i], pf_b[i]);
                if (++pf_kt == KT) { pf_kt = 0; pf_t += gridDim.x; }
            };
            for (int i = 0; i < kPrefetchSteps; ++i) prefetch_one();
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile tl = decode_tile(t, MU, p, s_prefix, s_bounds, s_pad);
                const uint8_t* a[2];
                uint32_t nb[2];
                for (int i = 0; i < 2; ++i) {
                    int rows, mt;
                    source(tl, i, a[i], rows, mt);
                    nb[i] = (uint32_t)rows * L.rb;
                }
                for (int kt = 0; kt < KT; ++kt) {
                    prefetch_one();
                    ok = wait_bar(&raw_empty[rs], rph ^ 1, abort_flag, status, p.wait_limit);
                    if (!ok) break;
                    ptx::mbar_arrive_expect_tx(&raw_full[rs], nb[0] + nb[1]);
                    for (int i = 0; i < 2; ++i)
                        if (nb[i])
                            ptx::bulk_g2s(sRaw + (rs * 2 + i) * kRawBytes, a[i] + (size_t)kt * nb[i], nb[i],
                                          &raw_full[rs]);
                    used |= 1u << rs;
                    par = (par & ~(1u << rs)) | (rph << rs);
                    if (++rs == kRS) { rs = 0; rph ^= 1; }
                }
            }
            // let every copy issued land before the CTA can exit (bounded)
            volatile int never = 0;
            for (int s = 0; s < kRS; ++s)
                if (used >> s & 1) wait_bar(&raw_full[s], (par >> s) & 1, &never, status, p.wait_limit);
        }
    } else if (warp == kWarpProdB) {
        // ------------------------------------------------ activation producer
        // The rows of a column tile are contiguous and already swizzled in the
        // tile-major activation buffer: one bulk copy per k-step.
        if (lane == 0) {
            int bs = 0;
            uint32_t bph = 0;
            uint32_t used = 0, par = 0;
            bool ok = true;
            const size_t plane = (size_t)p.b_rows * 128u;
            int q = 0;  // k-steps of this CTA so far
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile tl = decode_tile(t, MU, p, s_prefix, s_bounds, s_pad);
                const uint32_t bytes = (uint32_t)((tl.n + 15) & ~15) * 128u;
                const uint8_t* src = p.B + (size_t)tl.p0pad * 128u;
                for (int kt = 0; kt < KT; ++kt, ++q) {
                    ok = wait_bar(&b_empty[bs], bph ^ 1, abort_flag, status, p.wait_limit);
                    if (!ok) break;
                    if (!((int)blockIdx.x == p.stall_cta && q == p.stall_stage)) {  // (test-only stall)
                        ptx::mbar_arrive_expect_tx(&b_full[bs], bytes);
                        ptx::bulk_g2s(sB + bs * kBTileBytes, src + kt * plane, bytes, &b_full[bs]);
                        used |= 1u << bs;
                        par = (par & ~(1u << bs)) | (bph << bs);
                    }
                    if (++bs == kMB) { bs = 0; bph ^= 1; }
                }
            }
            volatile int never = 0;
            for (int s = 0; s < kMB; ++s)
                if (used >> s & 1) wait_bar(&b_full[s], (par >> s) & 1, &never, status, p.wait_limit);
        }
    } else if (warp == kWarpMma) {
        // ----------------------------------------------------------------- MMA
        // A from tensor memory, B from shared memory; the two accumulators'
        // instructions interleave, sharing each B descriptor.  The whole warp
        // runs the loop (the named barrier takes whole warps); lane 0 issues.
        int as = 0, bs = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode_tile(t, MU, p, s_prefix, s_bounds, s_pad);
            const int n16 = (tl.n + 15) & ~15;
            const bool has1 = DUAL || (2 * tl.mt + 1 < MT);
            const uint32_t d0 = tmem_base, d1 = tmem_base + kAccCols;
            const uint32_t idesc = ptx::idesc_f16(BF16, n16, 128);
            for (int kt = 0; kt < KT; ++kt) {
                // warp 3 has seen this k-step's stages (and at kt = 0 the accumulators) ready
                ok = ptx::bar_red_and(kBarIssue, 64, true);
                if (!ok) break;
                ptx::tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = tmem_base + kACol0 + (uint32_t)as * 64u;  // 8 columns per K=16 slice
                    const uint32_t b = ptx::smem_u32(sB + bs * kBTileBytes);
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk) {
                        const uint32_t acc = (kt | kk) != 0;
                        const uint64_t bd = ptx::desc_k_sw128(b + kk * 32);
                        ptx::mma_f16_ts(d0, a0 + kk * 8, bd, idesc, acc);
                        if (has1) ptx::mma_f16_ts(d1, a0 + 32 + kk * 8, bd, idesc, acc);
                    }
                    ptx::mma_commit(&a_empty[as]);
                    ptx::mma_commit(&b_empty[bs]);
                }
                __syncwarp();
                if (++as == kMA) as = 0;
                if (++bs == kMB) bs = 0;
            }
            if (!ok) break;
            if (lane == 0) ptx::mma_commit(tmem_full);
            __syncwarp();
        }
        // every MMA issued has completed before the CTA can release tensor memory
        // (after an abort no epilogue waited for them); bounded like every wait
        if (lane == 0) {
            ptx::mma_commit(mma_drained);
            volatile int never = 0;
            wait_bar(mma_drained, 0, &never, status, p.wait_limit);
        }
        __syncwarp();
    } else if (warp == kWarpWait) {
        // ------------------------------------------------- the MMA warp's waits
        // The same k-step sequence as warp 1: wait (bounded) for what the k-step
        // needs, then meet warp 1 at the named barrier with the outcome.  Both
        // warps pass the barrier equally often: a failed wait is handed over,
        // and both leave their loops after it.
        int as = 0, bs = 0;
        uint32_t aph = 0, bph = 0, use = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            for (int kt = 0; kt < KT; ++kt) {
                bool ready = true;
                if (kt == 0) ready = warp_wait(tmem_empty, (use & 1) ^ 1, abort_flag, status, p.wait_limit);
                ready = ready && warp_wait(&a_full[as], aph, abort_flag, status, p.wait_limit) &&
                        warp_wait(&b_full[bs], bph, abort_flag, status, p.wait_limit);
                ok = ptx::bar_red_and(kBarIssue, 64, ready);
                if (!ok) break;
                if (++as == kMA) { as = 0; aph ^= 1; }
                if (++bs == kMB) { bs = 0; bph ^= 1; }
            }
            use += 1;
        }
    } else if (warp >= kWorkWarp0 && warp < kWorkWarp0 + kWorkWarps) {
        // ------------------------------------- dequantisation and epilogue warps
        // Four per tensor-memory lane quarter wq = warp % 4.  Dequantisation:
        // thread `lane` converts row 32 wq + lane of matrix `mat`, all 64
        // columns, in the k-steps of parity kpar, exactly (q*d rounded once to
        // the operand type), into registers as soon as the raw stage lands, and
        // stores them into the A stage of tensor memory once the MMAs of two
        // k-steps back have released it.  Epilogue: at the end of a tile each
        // drains a quarter of the 16-column chunks of its lanes.
        const int wq = warp & 3, wj = (warp - kWorkWarp0) >> 2;  // lane quarter; (parity, matrix) and chunk phase
        const int kpar = wj & 1, mat = wj >> 1;
        const int r = 32 * wq + lane;       // the thread's row of the tile: its tensor-memory lane
        const int first = (lane >> 2) & 1;  // alternate read order: conflict-free 16-byte loads
        const uint32_t lanes = (uint32_t)(32 * wq) << 16;
        const uint32_t a_dst = tmem_base + lanes + kACol0 + (uint32_t)mat * 32u;
        int rs = 0, as = 0;
        uint32_t rph = 0, aph = 0, use = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile tl = decode_tile(t, MU, p, s_prefix, s_bounds, s_pad);
            // output rows and column scales of this warp's epilogue chunks, fetched ahead of time
            int orow[3];
            float oscale[3];
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int col = (4 * q + wj) * 16 + (lane & 15);
                orow[q] = -1;
                oscale[q] = 1.0f;
                if (col < tl.n) {
                    if (!DUAL) orow[q] = p.dst_rows ? __ldg(p.dst_rows + tl.p0 + col) : tl.p0 + col;
                    if (p.col_scale) oscale[q] = __ldg(p.col_scale + tl.p0pad + col);
                }
            }
            int nr;
            {
                const uint8_t* dummy;
                int mt;
                source(tl, mat, dummy, nr, mt);
            }
            for (int kt = 0; kt < KT; ++kt) {
                if ((as & 1) == kpar) {  // the k-step count's parity, continued across tiles
                    ok = warp_wait(&raw_full[rs], rph, abort_flag, status, p.wait_limit);
                    if (!ok) break;
                    // the row's 64 operand values, packed in pairs in K order (padding rows: 0)
                    uint32_t pk[32];
                    if (nr > 0 && WT == MOE_MXFP4) {
                        // sub-block wq (nsr rows): 32 code bytes a row at sub + lane*32 (two 16-byte
                        // halves, read in alternating order), then two scale bytes a row at
                        // sub + nsr*32 + lane*2
                        uint4 h0 = make_uint4(0u, 0u, 0u, 0u), h1 = h0;
                        uint32_t xs = 0x7f7fu;  // padding rows: codes 0, scale 1
                        if (r < nr) {
                            const uint32_t raw = raw_sa + (uint32_t)(rs * 2 + mat) * kRawBytes;
                            const int nsr = sub_rows(nr, wq);
                            const uint32_t sub = raw + (uint32_t)wq * (uint32_t)L.sub_bytes();
                            const uint32_t q = sub + (uint32_t)lane * 32u;
                            const uint4 ca = ptx::lds128(q + first * 16), cb = ptx::lds128(q + (first ^ 1) * 16);
                            h0 = first ? cb : ca;
                            h1 = first ? ca : cb;
                            xs = ptx::lds16(sub + (uint32_t)nsr * 32u + (uint32_t)lane * 2u);
                        }
                        const float s0 = e8m0_scale(xs & 0xffu), s1 = e8m0_scale(xs >> 8);
                        const uint32_t w0[4] = {h0.x, h0.y, h0.z, h0.w}, w1[4] = {h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {  // word i of half h holds values 32h + 8i .. 32h + 8i + 7
                            dequant_mx8(w0[i], s0, pk + 4 * i);
                            dequant_mx8(w1[i], s1, pk + 16 + 4 * i);
                        }
                    } else if (nr > 0) {
                        uint4 x[4];
                        uint32_t sc = 0u;
#pragma unroll
                        for (int i = 0; i < 4; ++i) x[i] = make_uint4(0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u);
                        if (r < nr) {
                            // sub-block wq (nsr rows); block h, 16-byte chunk c at sub + h*nsr*32 +
                            // lane*32 + c*16; lanes alternate the chunk order so that the 16-byte
                            // loads are conflict-free
                            const uint32_t raw = raw_sa + (uint32_t)(rs * 2 + mat) * kRawBytes;
                            const int nsr = sub_rows(nr, wq);
                            const uint32_t sub = raw + (uint32_t)wq * (uint32_t)L.sub_bytes();
                            const uint32_t q = sub + (uint32_t)lane * 32u;
                            const uint32_t h1 = (uint32_t)nsr * 32u;
                            x[0] = ptx::lds128(q + first * 16);
                            x[1] = ptx::lds128(q + (first ^ 1) * 16);
                            x[2] = ptx::lds128(q + h1 + first * 16);
                            x[3] = ptx::lds128(q + h1 + (first ^ 1) * 16);
                            sc = ptx::lds32(sub + (uint32_t)nsr * kTileK + (uint32_t)lane * 4u);
                        }
                        uint32_t d0, d1;
                        asm("prmt.b32 %0, %1, %1, 0x1010;" : "=r"(d0) : "r"(sc));
                        asm("prmt.b32 %0, %1, %1, 0x3232;" : "=r"(d1) : "r"(sc));
                        const float f0 = BF16 ? __half2float(__ushort_as_half((unsigned short)(sc & 0xffffu))) : 0.f;
                        const float f1 = BF16 ? __half2float(__ushort_as_half((unsigned short)(sc >> 16))) : 0.f;
                        // chunk c of block h: K values 32h + 16c .. 32h + 16c + 15
                        dequant16<BF16>(first ? x[1] : x[0], d0, f0, pk + 0);
                        dequant16<BF16>(first ? x[0] : x[1], d0, f0, pk + 8);
                        dequant16<BF16>(first ? x[3] : x[2], d1, f1, pk + 16);
                        dequant16<BF16>(first ? x[2] : x[3], d1, f1, pk + 24);
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&raw_empty[rs]);  // its loads have been consumed
                    ok = warp_wait(&a_empty[as], aph ^ 1, abort_flag, status, p.wait_limit);
                    if (!ok) break;
                    if (nr > 0) {
                        ptx::tc_fence_after();
                        ptx::tmem_st_32x32b_x32(a_dst + (uint32_t)as * 64u, pk);
                        ptx::tmem_st_wait();
                        ptx::tc_fence_before();
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&a_full[as]);
                }
                if (++rs == kRS) { rs = 0; rph ^= 1; }
                if (++as == kMA) { as = 0; aph ^= 1; }
            }
            if (!ok) break;
            // ---- epilogue of this tile
            if (!warp_wait(tmem_full, use & 1, abort_flag, status, p.wait_limit)) break;
            use += 1;
            ptx::tc_fence_after();
            if (DUAL) {
                const int m = tl.mt * kTileM + 32 * wq + lane;
                const bool m_ok = m < L.n_out;
                // h goes to the tile-major swizzled buffer the down GEMM streams
                uint8_t* hplane = p.h + (size_t)(m >> 6) * p.h_rows * 128u + ((m & 7) << 1);
                const int mchunk = (m & 63) >> 3;
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const int c0 = (4 * q + wj) * 16;
                    if (c0 >= tl.n) break;
                    uint32_t v[16], u[16];
                    ptx::tmem_ld_32x32b_x16(tmem_base + lanes + c0, v);
                    ptx::tmem_ld_32x32b_x16(tmem_base + lanes + kAccCols + c0, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float sc = __shfl_sync(0xffffffffu, oscale[q], i);
                        if (c0 + i < tl.n && m_ok) {
                            const float g = __uint_as_float(v[i]) * sc, up = __uint_as_float(u[i]) * sc;
                            const float hv = __fdividef(g, 1.0f + __expf(-g)) * up;
                            const int prow = tl.p0pad + c0 + i;
                            *(__nv_bfloat16*)(hplane + (size_t)prow * 128u + ((mchunk ^ (prow & 7)) << 4)) =
                                __float2bfloat16_rn(hv);
                        }
                    }
                }
            } else {
                for (int i = 0; i < 2; ++i) {
                    const int mt2 = 2 * tl.mt + i;
                    if (mt2 >= MT) break;
                    const int m = mt2 * kTileM + 32 * wq + lane;
                    const bool m_ok = m < L.n_out;
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        const int c0 = (4 * q + wj) * 16;
                        if (c0 >= tl.n) break;
                        uint32_t v[16];
                        ptx::tmem_ld_32x32b_x16(tmem_base + lanes + (uint32_t)i * kAccCols + c0, v);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int rr = __shfl_sync(0xffffffffu, orow[q], j);
                            const float sc = __shfl_sync(0xffffffffu, oscale[q], j);
                            if (rr >= 0 && m_ok) p.out[(int64_t)rr * p.out_ld + m] = __uint_as_float(v[j]) * sc;
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(tmem_empty);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512);
    }
}

// Gather activation rows into the tile-major, 128-byte-swizzled layout the
// GEMM streams with one bulk copy per k-step: the row at sorted position p of
// group e (rank r inside the group) becomes row pad_start[e] + r; k-plane kt
// holds columns [64*kt, 64*kt + 64) as 128 bytes whose 16-byte chunk c sits at
// chunk c ^ (row % 8).  fp32 input is rounded to fp16; columns >= n_in are 0.
// Eight activations of row `row`, columns col .. col+7, as fp32 (zeros past n_in).
__device__ __forceinline__ void load8(const void* x, int x_type, int64_t row, int n_in, int col, float (&e)[8]) {
    if (col >= n_in) {
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = 0.f;
        return;
    }
    if (x_type == MOE_F32) {
        const float4* src = (const float4*)((const float*)x + row * n_in + col);
        const float4 a = __ldg(src), b = __ldg(src + 1);
        e[0] = a.x; e[1] = a.y; e[2] = a.z; e[3] = a.w;
        e[4] = b.x; e[5] = b.y; e[6] = b.z; e[7] = b.w;
        return;
    }
    const uint4 v = __ldg((const uint4*)((const uint16_t*)x + row * n_in + col));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = w[i] & 0xffffu, hi = w[i] >> 16;
        if (x_type == MOE_BF16) {
            e[2 * i] = __uint_as_float(lo << 16);
            e[2 * i + 1] = __uint_as_float(hi << 16);
        } else {
            e[2 * i] = __half2float(__ushort_as_half((unsigned short)lo));
            e[2 * i + 1] = __half2float(__ushort_as_half((unsigned short)hi));
        }
    }
}

// Gather activation rows into the tile-major, 128-byte-swizzled fp16 layout the
// GEMM streams with one bulk copy per k-step: the row at sorted position p of
// group e (rank r inside the group) becomes row pad_start[e] + r; k-plane kt
// holds columns [64*kt, 64*kt + 64) as 128 bytes whose 16-byte chunk c sits at
// chunk c ^ (row % 8); columns >= n_in are 0.  Each row is multiplied by the
// power of two 2^-e that puts its largest magnitude in [2^14, 2^15) - exact,
// and inside the fp16 range whatever the input type - and xs[row] = 2^e is what
// the GEMM epilogue multiplies that token's results by.
// OUT_BF16: write the rows as bf16 without scaling (xs = 1), the operand type
// of the MXFP4 GEMM.
__device__ __forceinline__ uint32_t pack_out(float a, float b, float sc, int out_bf16) {
    if (out_bf16) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *(const uint32_t*)&v;
    }
    const __half2 v = __floats2half2_rn(a * sc, b * sc);
    return *(const uint32_t*)&v;
}

template <int OUT_BF16>
__global__ void __launch_bounds__(256)
gather_tiled_kernel(const void* __restrict__ x, int x_type, int n_in, int KT, const int32_t* __restrict__ src_rows,
                    const int32_t* __restrict__ bounds, const int32_t* __restrict__ pad_start, int n_groups,
                    int64_t n_rows, int64_t rows_pad, uint8_t* __restrict__ xt, float* __restrict__ xs,
                    const int* __restrict__ hdr) {
    if (read_status(hdr + kHdrStatus) != 0) return;
    const int lane = threadIdx.x & 31;
    const int64_t S = n_groups > 0 ? bounds[n_groups] : n_rows;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t p = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); p < S; p += nw) {
        int64_t prow = p, srow = p;
        if (n_groups > 0) {
            int lo = 0, hi = n_groups;  // bounds[lo] <= p < bounds[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(bounds + mid) <= p) lo = mid; else hi = mid;
            }
            prow = __ldg(pad_start + lo) + (p - __ldg(bounds + lo));
            srow = src_rows ? __ldg(src_rows + p) : p;
        }
        float mx = 0.f;
        if (!OUT_BF16) {
            for (int seg = lane; seg < KT * 8; seg += 32) {
                float e[8];
                load8(x, x_type, srow, n_in, (seg >> 3) * 64 + (seg & 7) * 8, e);
#pragma unroll
                for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(e[i]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        int ex = 0;
        if (mx > 0.f && mx <= 3.402823466e38f) {
            ex = ilogbf(mx) - 14;
            ex = ex < -100 ? -100 : ex;
        }
        const float sc = ldexpf(1.0f, -ex);
        if (lane == 0) xs[prow] = ldexpf(1.0f, ex);
        for (int seg = lane; seg < KT * 8; seg += 32) {
            const int kt = seg >> 3, c = seg & 7;
            float e[8];
            load8(x, x_type, srow, n_in, kt * 64 + c * 8, e);
            uint32_t h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = pack_out(e[2 * i], e[2 * i + 1], sc, OUT_BF16);
            *(uint4*)(xt + ((size_t)kt * rows_pad + prow) * 128u + ((c ^ (int)(prow & 7)) << 4)) =
                make_uint4(h[0], h[1], h[2], h[3]);
        }
    }
}

// Broadcast gather, one warp per token: the token's row is read (and its scale
// found) once and written to the tiled rows of all k of its slots.
template <int OUT_BF16>
__global__ void __launch_bounds__(256)
gather_tokens_kernel(const void* __restrict__ x, int x_type, int n_in, int KT, const int32_t* __restrict__ slot_prow,
                     int k, int64_t n_tokens, int64_t rows_pad, uint8_t* __restrict__ xt, float* __restrict__ xs,
                     const int* __restrict__ hdr) {
    if (read_status(hdr + kHdrStatus) != 0) return;
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < n_tokens; t += nw) {
        const int32_t* pr = slot_prow + t * k;
        float mx = 0.f;
        if (!OUT_BF16) {
#pragma unroll 4
            for (int seg = lane; seg < KT * 8; seg += 32) {
                float e[8];
                load8(x, x_type, t, n_in, (seg >> 3) * 64 + (seg & 7) * 8, e);
#pragma unroll
                for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(e[i]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        int ex = 0;
        if (mx > 0.f && mx <= 3.402823466e38f) {
            ex = ilogbf(mx) - 14;
            ex = ex < -100 ? -100 : ex;
        }
        const float sc = ldexpf(1.0f, -ex);
        for (int j = lane; j < k; j += 32) xs[__ldg(pr + j)] = ldexpf(1.0f, ex);
#pragma unroll 2
        for (int seg = lane; seg < KT * 8; seg += 32) {
            const int kt = seg >> 3, c = seg & 7;
            float e[8];
            load8(x, x_type, t, n_in, kt * 64 + c * 8, e);
            uint32_t h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = pack_out(e[2 * i], e[2 * i + 1], sc, OUT_BF16);
            const uint4 v = make_uint4(h[0], h[1], h[2], h[3]);
            uint8_t* plane = xt + (size_t)kt * rows_pad * 128u;
            for (int j = 0; j < k; ++j) {
                const int prow = __ldg(pr + j);
                *(uint4*)(plane + (size_t)prow * 128u + ((c ^ (prow & 7)) << 4)) = v;
            }
        }
    }
}

// ------------------------------------------------------------------- host
static int sm_count() {
    static int dev_cached = -1, n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != dev_cached) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        dev_cached = dev;
    }
    return n > 0 ? n : 148;
}

// The test-only stall set by moe_testing_stall (csrc/gemv.cu): CTA, k-step and
// the wait limit in cycles; false when none is set.
bool testing_stall_state(int* cta, int* stage, long long* limit_cycles);

template <int DUAL, int BF16, int WT>
static moe_status launch_grouped(const GemmParams& in, int grid, cudaStream_t stream) {
    GemmParams p = in;
    p.wait_limit = kWaitLimitCycles;
    p.stall_cta = -1;
    p.stall_stage = 0;
    long long limit = 0;
    if (testing_stall_state(&p.stall_cta, &p.stall_stage, &limit)) p.wait_limit = limit;
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(grouped_gemm_kernel<DUAL, BF16, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Cfg::smem_bytes) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_dev = dev;
    }
    grouped_gemm_kernel<DUAL, BF16, WT><<<grid, kGemmThreads, Cfg::smem_bytes, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int DUAL>
static moe_status run_gemm(const GemmParams& p, int64_t max_coltiles, cudaStream_t stream) {
    const int64_t units = DUAL ? p.L.mt_count : (p.L.mt_count + 1) / 2;
    int64_t tiles = max_coltiles * units;
    if (tiles <= 0) return MOE_OK;
    const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
    if (p.wtype == MOE_MXFP4) return launch_grouped<DUAL, 1, MOE_MXFP4>(p, grid, stream);  // bf16 operands
    if (p.bf16) return launch_grouped<DUAL, 1, MOE_Q8_0>(p, grid, stream);
    return launch_grouped<DUAL, 0, MOE_Q8_0>(p, grid, stream);
}

static int64_t coltile_bound(int64_t S, int E) { return (S + kGemmBN - 1) / kGemmBN + (S < E ? S : E); }

// Broadcast mode (every slot of a token reads the token's row): per token.
static moe_status gather_tokens(const void* x, int x_type, int n_in, const int32_t* slot_prow, int k, int64_t n_tokens,
                                int64_t rows_pad, void* xt, float* xs, int* hdr, int out_bf16, cudaStream_t s) {
    const int KT = (n_in + kTileK - 1) / kTileK;
    int64_t blocks = (n_tokens + 7) / 8;
    if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
    if (blocks < 1) blocks = 1;
    if (out_bf16)
        gather_tokens_kernel<1><<<(unsigned)blocks, 256, 0, s>>>(x, x_type, n_in, KT, slot_prow, k, n_tokens, rows_pad,
                                                                 (uint8_t*)xt, xs, hdr);
    else
        gather_tokens_kernel<0><<<(unsigned)blocks, 256, 0, s>>>(x, x_type, n_in, KT, slot_prow, k, n_tokens, rows_pad,
                                                                 (uint8_t*)xt, xs, hdr);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static moe_status gather(const void* x, int x_type, int n_in, const int32_t* src_rows, const int32_t* bounds,
                         const int32_t* pad_start, int n_groups, int64_t rows, int64_t rows_pad, void* xt, float* xs,
                         int* hdr, int out_bf16, cudaStream_t s) {
    const int KT = (n_in + kTileK - 1) / kTileK;
    int64_t blocks = (rows + 7) / 8;
    if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
    if (blocks < 1) blocks = 1;
    if (out_bf16)
        gather_tiled_kernel<1><<<(unsigned)blocks, 256, 0, s>>>(x, x_type, n_in, KT, src_rows, bounds, pad_start,
                                                                n_groups, rows, rows_pad, (uint8_t*)xt, xs, hdr);
    else
        gather_tiled_kernel<0><<<(unsigned)blocks, 256, 0, s>>>(x, x_type, n_in, KT, src_rows, bounds, pad_start,
                                                                n_groups, rows, rows_pad, (uint8_t*)xt, xs, hdr);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_gemm_mul_mat_id(const GemmMulMatId& g, cudaStream_t stream) {
    const int mx = g.wtype == MOE_MXFP4;  // bf16 operands, unscaled activation rows
    moe_status st = g.x_rows * g.k == g.S
                        ? gather_tokens(g.x, g.x_type, g.n_in, g.slot_prow, g.k, g.x_rows, g.rows_pad, g.xt, g.xs,
                                        g.hdr, mx, stream)
                        : gather(g.x, g.x_type, g.n_in, g.ids_src1, g.bounds, g.pad_start, g.E, g.S, g.rows_pad, g.xt,
                                 g.xs, g.hdr, mx, stream);
    if (st) return st;
    prof_mark(stream, "gather");
    GemmParams p = {};
    p.A0 = g.W;
    p.L = WLayout(g.n_out, g.n_in, g.wtype);
    p.wtype = g.wtype;
    p.n_groups = g.E;
    p.bounds = g.bounds;
    p.ntile_prefix = g.ntile_prefix;
    p.pad_start = g.pad_start;
    p.B = (const uint8_t*)g.xt;
    p.b_rows = g.rows_pad;
    p.dst_rows = g.ids_dst;
    p.out = g.dst;
    p.out_ld = g.n_out;
    p.hdr = g.hdr;
    p.bf16 = mx;  // Q8_0: fp16 activation tiles (scaled rows); MXFP4: bf16
    p.col_scale = mx ? nullptr : g.xs;
    st = run_gemm<0>(p, coltile_bound(g.S, g.E), stream);
    prof_mark(stream, "gemm");
    return st;
}

moe_status launch_gemm_ffn(const GemmFfn& g, cudaStream_t stream) {
    const int mx = g.wtype == MOE_MXFP4;  // bf16 operands, unscaled activation rows
    const int kt_ff = (g.n_ff + kTileK - 1) / kTileK;
    moe_status st =
        gather_tokens(g.x, g.x_type, g.n_embd, g.slot_prow, g.k, g.T, g.rows_pad, g.xt, g.xs, g.hdr, mx, stream);
    if (st) return st;
    prof_mark(stream, "gather");
    if (g.n_ff % kTileK) {  // columns past n_ff of the last k-plane of h are read by the down GEMM: keep them 0
        if (cudaMemsetAsync((uint8_t*)g.h + (size_t)(kt_ff - 1) * g.rows_pad * 128u, 0, (size_t)g.rows_pad * 128u,
                            stream) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // gate/up -> h (tile-major, expert-sorted rows), SwiGLU in the epilogue
    GemmParams p = {};
    p.A0 = g.Wg;
    p.A1 = g.Wu;
    p.L = WLayout(g.n_ff, g.n_embd, g.wtype);
    p.wtype = g.wtype;
    p.n_groups = g.E;
    p.bounds = g.bounds;
    p.ntile_prefix = g.ntile_prefix;
    p.pad_start = g.pad_start;
    p.B = (const uint8_t*)g.xt;
    p.b_rows = g.rows_pad;
    p.h = (uint8_t*)g.h;
    p.h_rows = g.rows_pad;
    p.out_ld = g.n_ff;
    p.hdr = g.hdr;
    p.bf16 = mx;  // Q8_0: fp16 activation tiles (scaled rows); MXFP4: bf16
    p.col_scale = mx ? nullptr : g.xs;
    st = run_gemm<1>(p, coltile_bound(g.S, g.E), stream);
    if (st) return st;
    prof_mark(stream, "gemm_gate_up");
    const int kt_sh = (g.n_ff_shared + kTileK - 1) / kTileK;
    if (g.n_ff_shared > 0) {
        st = gather(g.x, g.x_type, g.n_embd, nullptr, nullptr, nullptr, 0, g.T, g.rows_pad_sh, g.xt_sh, g.xs_sh,
                    g.hdr, mx, stream);
        if (st) return st;
        if (g.n_ff_shared % kTileK) {
            if (cudaMemsetAsync((uint8_t*)g.h_sh + (size_t)(kt_sh - 1) * g.rows_pad_sh * 128u, 0,
                                (size_t)g.rows_pad_sh * 128u, stream) != cudaSuccess)
                return MOE_ERR_CUDA;
        }
        GemmParams q = {};
        q.A0 = g.Sg;
        q.A1 = g.Su;
        q.L = WLayout(g.n_ff_shared, g.n_embd, g.wtype);
        q.wtype = g.wtype;
        q.n_rows = (int)g.T;
        q.B = (const uint8_t*)g.xt_sh;
        q.b_rows = g.rows_pad_sh;
        q.h = (uint8_t*)g.h_sh;
        q.h_rows = g.rows_pad_sh;
        q.out_ld = g.n_ff_shared;
        q.hdr = g.hdr;
        q.bf16 = mx;
        q.col_scale = mx ? nullptr : g.xs_sh;
        st = run_gemm<1>(q, (g.T + kGemmBN - 1) / kGemmBN, stream);
        if (st) return st;
        prof_mark(stream, "gemm_shared_gate_up");
    }
    // down: B = h, contiguous per expert; the epilogue scatters rows to dst by ids_dst
    GemmParams d = {};
    d.A0 = g.Wd;
    d.L = WLayout(g.n_embd, g.n_ff, g.wtype);
    d.wtype = g.wtype;
    d.n_groups = g.E;
    d.bounds = g.bounds;
    d.ntile_prefix = g.ntile_prefix;
    d.pad_start = g.pad_start;
    d.B = (const uint8_t*)g.h;
    d.b_rows = g.rows_pad;
    d.dst_rows = g.ids_dst;
    d.out = g.dst;
    d.out_ld = g.n_embd;
    d.hdr = g.hdr;
    d.bf16 = 1;
    st = run_gemm<0>(d, coltile_bound(g.S, g.E), stream);
    if (st) return st;
    prof_mark(stream, "gemm_down");
    if (g.n_ff_shared > 0) {
        GemmParams q = {};
        q.A0 = g.Sd;
        q.L = WLayout(g.n_embd, g.n_ff_shared, g.wtype);
        q.wtype = g.wtype;
        q.n_rows = (int)g.T;
        q.B = (const uint8_t*)g.h_sh;
        q.b_rows = g.rows_pad_sh;
        q.out = g.dst_shared;
        q.out_ld = g.n_embd;
        q.hdr = g.hdr;
        q.bf16 = 1;
        st = run_gemm<0>(q, (g.T + kGemmBN - 1) / kGemmBN, stream);
        prof_mark(stream, "gemm_shared_down");
    }
    return st;
}

}  // namespace moe
