// Weight-streaming expert mat-vec for small token counts (decode), with the
// shared expert handled as more work items of the same launch - the fusion of
// llama.cpp PR #29184 ("CUDA: fuse shared experts into MMVQ", release b11370)
// restated for this library.
//
// Decode is bound by the weight stream; the kernel is built around keeping it
// moving:
//  - the down launch is a programmatic dependent of gate/up: its CTAs start as
//    gate/up's leave the SMs, their producers stream the down weights at once
//    and only their consumers wait for gate/up's h;
//  - a work item is (routed expert, row sub-tile of 32, 64 or 128 rows, or a
//    pair of full 128-row tiles for a single matrix) or (shared expert, row
//    sub-tile), always over the whole K, so no item needs another's partial
//    sums; the height is chosen per launch from an estimate of the fullest
//    CTA's stream (its items' bytes plus a fixed cost per item);
//  - one producer warp streams 34 KB stages (the item's rows for several
//    k-steps of each matrix: one tensor copy per matrix, or one bulk copy per
//    k-step and matrix where a tensor map does not apply) through a ring,
//    running ahead across items;
//  - 16 consumer warps on the tensor cores (mma.sync m16n8k16, fp16 in, fp32
//    out): A = 16 weight rows of quantised values, exact in fp16; B = up to 8
//    tokens' activations, each token scaled by a power of two into the fp16
//    range; each 32-column block's product is multiplied by its block scales
//    in fp32.  A warp owns one (matrix, 16-row group) and every W-th k-step;
//    the warps of a group are added in a fixed order, so results do not
//    depend on timing (with W = 1 on a single matrix the warp stores its
//    totals itself).  The consumers are bound by instruction issue, so the
//    per-stage bookkeeping is kept to additions and compares.
// The distinct routed experts come from ids directly: for up to 64 slots every
// warp finds them with ballots in its own registers (no block-wide pass before
// the first copy); for more slots a block-wide pass builds tables in shared
// memory.
//
// Modes: single matrix (mul_mat_id rows, or the down projection writing
// dst[t][s]), or dual gate/up with a SwiGLU epilogue writing bf16 h[t][s].
#include <atomic>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "gemv_args.cuh"
#include "moe_testing.h"
#include "ptx.cuh"

namespace moe {

constexpr int kGvConsumers = 512;
constexpr int kGvThreads = 32 + kGvConsumers;  // warp 0: producer
constexpr uint32_t kGvStage = 512 * kRowBytes;  // 34816 bytes: 512 (row, k-step) pieces of Q8_0
constexpr uint32_t kGvSmemBudget = 224 * 1024;
constexpr long long kGvWaitLimit = 1ll << 32;   // ~2 s
constexpr int kGvFast = 64;                     // slots up to which the experts come from warp ballots
constexpr int kGvXSteps = 32;                   // k-steps of the activation window (2048 columns)
constexpr uint32_t kGvXRow = kGvXSteps * kTileK * 2 + 16;  // bytes of one token's fp16 window row (+16: banks)
constexpr uint32_t kGvXBytes = kGvNT * kGvXRow + 2 * kGvNT * 4;  // window + per-token max and factor
constexpr uint32_t kGvRedBytes = (kGvConsumers / 32) * 32 * 4 * 4;  // 4 fp32 results a consumer thread

struct GvLay {
    uint32_t ring, x, red, tab, bars, misc, total;
};

// Shared memory: ring | activation window | reduction | tables (slow path) | barriers | misc.
__host__ __device__ inline GvLay gv_lay(int ns, int S, int n_experts) {
    GvLay m;
    uint32_t o = 0;
    m.ring = o; o += (uint32_t)ns * kGvStage;
    m.x = o; o += kGvXBytes;
    m.red = o; o += 2 * kGvRedBytes;  // two buffers: an item writes one while the last is still read
    m.tab = o;
    if (S > kGvFast) o += (uint32_t)(((n_experts + 31) / 32) * 2 + 2 + 2 * (S + 1) + 2 * S) * 4u;
    o = (o + 15u) & ~15u;
    m.bars = o; o += 2u * (uint32_t)ns * 8u;
    m.misc = o; o += 16u;
    m.total = o;
    return m;
}

// Bounded wait by one thread: false on expiry (status set, the wait's site
// recorded, abort raised) or when another thread raised abort.
__device__ __forceinline__ bool gv_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag,
                                        long long limit) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    // a short sleep between polls: the consumers are issue-bound, and a warp
    // that polls takes issue slots from the warps on its sub-partition
    while (!ptx::mbar_try_wait(bar, parity)) {
        __nanosleep(128);
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            *abort_flag = 1;
            const int site = (1 << 30) | ((int)(threadIdx.x >> 5) << 20) | (int)(ptx::smem_u32(bar) & 0xfffffu);
            atomicCAS(status + (kHdrWaitSite - kHdrStatus), 0, site);
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// gv_wait by lane 0; every lane of the warp gets its outcome.
__device__ __forceinline__ bool gv_warp_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag,
                                             long long limit) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = gv_wait(bar, parity, status, abort_flag, limit);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Named barrier 1 over the consumer warps; consumers_and also returns the AND
// of every consumer's flag, so exits decided from it are uniform.
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kGvConsumers) : "memory"); }
__device__ __forceinline__ bool consumers_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kGvConsumers)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float f2sum(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo + hi;
}

__device__ __forceinline__ float ld_x16(uint32_t bits16, int x_type) {
    return x_type == MOE_BF16 ? __uint_as_float(bits16 << 16) : __half2float(__ushort_as_half((unsigned short)bits16));
}

// E8M0 scale byte -> 2^(x - 127) as a float (x = 0: 2^-127, a float subnormal;
// x = 255: NaN).
__device__ __forceinline__ float e8m0_float(uint32_t x) {
    return x == 0u ? __uint_as_float(0x00400000u) : x == 255u ? __uint_as_float(0x7fc00000u) : __uint_as_float(x << 23);
}

// Eight E2M1 codes (a 32-bit word, code i in bits 4i..4i+3) -> their exact
// values as floats, by the sm_100a pair conversion to f16 (exact: two
// significant bits), then f16 -> float.
__device__ __forceinline__ void e2m1x8_to_float(uint32_t w, float (&v)[8]) {
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
        const __half2 p = *(const __half2*)&h[i];
        v[2 * i] = __low2float(p);
        v[2 * i + 1] = __high2float(p);
    }
}

// Exponent e such that m * 2^-e lies in [2^14, 2^15): the power of two that
// brings a token's largest magnitude to the top of the fp16 range (0 for zero
// or non-finite m; at least -100, so that 2^-e stays a finite float).
__device__ __forceinline__ int scale_exp(float m) {
    if (!(m > 0.f) || !(m <= 3.402823466e38f)) return 0;
    const int e = ilogbf(m) - 14;
    return e < -100 ? -100 : e;
}

// D += A * B on the tensor cores: A 16 x 16 fp16 (row major, four registers
// of two), B 16 x 8 fp16 (column major, two registers), D 16 x 8 fp32.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two stored Q8_0 bytes u = q + 128 (picked by the byte-permute selector:
// 0x7170 bytes 0 and 1, 0x7372 bytes 2 and 3) -> {q, q'} as fp16, exactly:
// the fp16 pattern {0x64, u} is 1024 + u, and 1024 + u - 1152 = q.
__device__ __forceinline__ uint32_t q8_h2(uint32_t w, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(w), "r"(0x64646464u), "r"(sel));
    const __half2 v = __hsub2(*(const __half2*)&r, __float2half2_rn(1152.0f));
    return *(const uint32_t*)&v;
}

// The two E2M1 codes of the low byte of w (low nibble first) -> fp16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_h2(uint32_t w) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
        : "=r"(r)
        : "r"(w));
    return r;
}

// Position of the n-th (0-based) set bit of m, for n < popc(m): a binary
// search that halves the window five times, stepping past the low half
// whenever it holds n or fewer set bits (straight-line popcounts; the
// find-n-th-set intrinsic measured about a microsecond a call under load).
__device__ __forceinline__ int select_bit(uint32_t m, int n) {
    int pos = 0;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const int c = __popc(m & ((1u << w) - 1u));
        const bool up = n >= c;
        n = up ? n - c : n;
        pos = up ? pos + w : pos;
        m = up ? m >> w : m;
    }
    return pos;
}

// n-th (0-based) set bit of a 64-bit mask given as two words.
__device__ __forceinline__ int nth_bit(uint32_t m0, uint32_t m1, int n) {
    const int c0 = __popc(m0);
    const bool lo = n < c0;
    return (lo ? 0 : 32) + select_bit(lo ? m0 : m1, lo ? n : n - c0);
}

// The distinct routed experts of this call, as one warp sees them.
//  fast (slots <= 64): v0/v1 = ids of slots lane and lane + 32 (-1 past the
//  end or out of range); fb0/fb1 = ballots of the slots that are the first
//  occurrence of their expert; distinct expert j = the expert of the j-th
//  first occurrence (slot order).
//  slow: tables in shared memory, distinct experts in ascending id order.
struct Routing {
    int v0, v1;
    uint32_t fb0, fb1;
    int n;
    const int* list_e;  // slow: [n] expert ids
    const int* off;     // slow: [n + 1] slot list offsets
    const int* slots;   // slow: slot list
    bool fast;

    // warp-collective in fast mode
    __device__ __forceinline__ int expert(int j) const {
        if (!fast) return list_e[j];
        const int s = nth_bit(fb0, fb1, j);
        const int a = __shfl_sync(0xffffffffu, v0, s & 31), b = __shfl_sync(0xffffffffu, v1, s & 31);
        return s < 32 ? a : b;
    }
};

// Warp-level distinct-expert scan for up to 64 slots (every lane of the warp).
// v0, v1: the ids of slots lane and lane + 32 (loaded by the caller; -1 past S).
__device__ __forceinline__ void routing_fast(Routing& R, int v0, int v1, int S, int E, int* status) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const bool bad = (lane < S && (v0 < 0 || v0 >= E)) || (lane + 32 < S && (v1 < 0 || v1 >= E));
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, MOE_ERR_BAD_ID);
    if (v0 >= E) v0 = -1;
    if (v1 >= E) v1 = -1;
    if (v0 < 0) v0 = -1;
    if (v1 < 0) v1 = -1;
    const uint32_t m0 = __match_any_sync(0xffffffffu, v0), m1 = __match_any_sync(0xffffffffu, v1);
    bool f0 = v0 >= 0 && (m0 & lt) == 0u;
    bool f1 = v1 >= 0 && (m1 & lt) == 0u;
    if (S > 32)  // an expert of the second half seen in the first is not new
        for (int i = 0; i < 32; ++i) {
            const int o = __shfl_sync(0xffffffffu, v0, i);
            if (o == v1) f1 = false;
        }
    R.v0 = v0;
    R.v1 = v1;
    R.fb0 = __ballot_sync(0xffffffffu, f0);
    R.fb1 = __ballot_sync(0xffffffffu, f1);
    R.n = __popc(R.fb0) + __popc(R.fb1);
    R.fast = true;
}

// Block-wide scan for more than 64 slots (every thread of the CTA): bitmap
// of the experts, per-word prefix, then a stable slot list per expert.
__device__ void routing_slow(Routing& R, const int32_t* ids, int S, int E, int* tab, int* status) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nw = (E + 31) / 32;
    uint32_t* bm = (uint32_t*)tab;        // [nw]
    int* wp = tab + nw;                   // [nw + 1]: distinct experts before word w
    int* nd = wp + nw + 1;                // [1]
    int* cnt = nd + 1;                    // [S + 1]
    int* off = cnt + S + 1;               // [S + 1]
    int* list = off + S + 1;              // [S]: slots grouped by distinct expert
    int* rank_sh = list + S;              // [S]: distinct index of each slot
    for (int w = tid; w < nw; w += blockDim.x) bm[w] = 0u;
    __syncthreads();
    for (int i = tid; i < S; i += blockDim.x) {
        const int v = __ldg(ids + i);
        if (v >= 0 && v < E) atomicOr(&bm[v >> 5], 1u << (v & 31));
        else set_status(status, MOE_ERR_BAD_ID);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of popcounts over the words
        int run = 0;
        for (int w0 = 0; w0 < nw; w0 += 32) {
            const int w = w0 + lane;
            const int c = w < nw ? __popc(bm[w]) : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nn = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nn;
            }
            if (w < nw) wp[w] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) { wp[nw] = run; *nd = run; }
    }
    __syncthreads();
    const int n = *nd;
    for (int j = tid; j <= n; j += blockDim.x) cnt[j] = 0;
    __syncthreads();
    for (int i = tid; i < S; i += blockDim.x) {
        const int v = __ldg(ids + i);
        int r = -1;
        if (v >= 0 && v < E) {
            r = wp[v >> 5] + __popc(bm[v >> 5] & ((1u << (v & 31)) - 1u));
            atomicAdd(&cnt[r], 1);
        }
        rank_sh[i] = r;
    }
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int j = j0 + lane;
            const int c = j < n ? cnt[j] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int nn = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += nn;
            }
            if (j < n) off[j] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) off[n] = run;
    }
    __syncthreads();
    // stable placement (ascending slot inside an expert), one warp per 32 slots in order
    if (warp == 0) {
        for (int base = 0; base < S; base += 32) {
            const int i = base + lane;
            const int r = i < S ? rank_sh[i] : -1;
            const uint32_t m = __match_any_sync(0xffffffffu, r);
            if (r >= 0) list[off[r] + __popc(m & ((1u << lane) - 1u))] = i;
            __syncwarp();
            if (r >= 0 && (m & ((1u << lane) - 1u)) == 0u) off[r] += __popc(m);
            __syncwarp();
        }
        __syncwarp();
        // restore the offsets (each was advanced by its count)
        for (int j = lane; j < n; j += 32) off[j] -= cnt[j];
    }
    // the expert id of distinct index j: the j-th set bit of the bitmap
    int* list_e = rank_sh;  // reuse: slot ranks are no longer needed after placement
    __syncthreads();
    for (int w = tid; w < nw; w += blockDim.x) {
        uint32_t bits = bm[w];
        int j = wp[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            list_e[j++] = w * 32 + b;
            bits &= bits - 1;
        }
    }
    __syncthreads();
    R.n = n;
    R.list_e = list_e;
    R.off = off;
    R.slots = list;
    R.fast = false;
}

// One work item.
struct GvItem {
    int side;    // 0 routed, 1 shared
    int e;       // expert of the weights
    int mt, r0;  // 128-row tile and first row of the sub-tile inside it
    int nrow;    // rows of the sub-tile (<= rsub); 0 = empty item (tail of the last tile)
    int nsl;     // slots (routed) or tokens (shared)
};

// The work of one CTA of 544 threads (a return ends the thread's part only).
template <int DUAL, int XB, int WT>
__device__ __forceinline__ void gemv_body(const GemvArgs& a) {
    extern __shared__ __align__(128) uint8_t sm[];
    constexpr int NMAT = DUAL + 1;
    int* status = a.hdr + kHdrStatus;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = a.n_tokens * a.k;
    const GvLay lay = gv_lay(a.ns, S, a.n_experts);
    uint8_t* ring = sm + lay.ring;
    float* red = (float*)(sm + lay.red);
    uint64_t* full = (uint64_t*)(sm + lay.bars);
    uint64_t* empty = full + a.ns;
    volatile int* abort_flag = (volatile int*)(sm + lay.misc);
    int* st_copy = (int*)(sm + lay.misc + 4);

    if (tid == 0) {
        for (int s = 0; s < a.ns; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kGvConsumers / 32);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    // Upstream dependency (this launch may start before the previous kernel of
    // the stream finished): nothing the previous kernel may write - ids,
    // activations, weights, the status - is read before this wait.
    if (a.pdl_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (a.pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // a sticky error stops the launch; one read, shared, so that the exit is
    // uniform (the other launch of the FFN may write the word meanwhile)
    // (the ids of a small call are loaded first, so that both loads are in flight together)
    int id0 = -1, id1 = -1;
    if (S <= kGvFast) {
        id0 = lane < S ? __ldg(a.ids + lane) : -1;
        id1 = lane + 32 < S ? __ldg(a.ids + lane + 32) : -1;
    }
    if (tid == 0) *st_copy = read_status(status);
    __syncthreads();
    if (*st_copy != 0) return;

    Routing R;
    if (S <= kGvFast) routing_fast(R, id0, id1, S, a.n_experts, status);
    else routing_slow(R, a.ids, S, a.n_experts, (int*)(sm + lay.tab), status);

    // A field of a side, read from the parameter space where it is used (taking
    // a kernel parameter's address, or copying a side whole, would cost local
    // memory or registers).
#define GV_SIDE(sh, field) ((sh) ? a.shared.field : a.routed.field)
    const int n_sh = a.has_shared ? a.shared.subs : 0;
    const int n_items = n_sh + R.n * a.routed.subs;
    // a contiguous range of items a CTA: consecutive items of one expert share
    // their tokens, so the activation window staged for one serves the next
    const int it_begin = (int)(((int64_t)blockIdx.x * n_items) / gridDim.x);
    const int it_end = (int)(((int64_t)(blockIdx.x + 1) * n_items) / gridDim.x);
    // items: the shared expert's sub-tiles first, then each distinct routed expert's
    auto item_of = [&](int it) {  // warp-collective in fast mode
        GvItem f;
        int u;
        if (it < n_sh) {
            f.side = 1;
            f.e = 0;
            u = it;
            f.nsl = a.n_tokens;
        } else {
            const int j = (it - n_sh) / a.routed.subs;
            u = (it - n_sh) - j * a.routed.subs;
            f.side = 0;
            f.e = R.expert(j);
            f.nsl = -1;  // counted by the consumers
        }
        const int rsub = f.side ? a.shared.rsub : a.routed.rsub;
        const WLayout L = f.side ? a.shared.L : a.routed.L;
        if (rsub > kTileM) {  // a pair of full tiles
            f.mt = 2 * u;
            f.r0 = 0;
        } else {
            const int per_tile = kTileM / rsub;
            f.mt = u / per_tile;
            f.r0 = (u - f.mt * per_tile) * rsub;
        }
        const int rows = L.n_out_pad - (f.mt * kTileM + f.r0);  // rows from the item's first to the end
        f.nrow = rows < rsub ? rows : rsub;
        if (f.nrow < 0) f.nrow = 0;
        return f;
    };

    if (warp == 0) {
        // ------------------------------------------------------- producer
        // Every lane runs the loop (the item decode is warp-collective); lane 0
        // issues the copies.  A stage holds kps k-steps of the sub-tile's rows
        // of each matrix: NMAT * kps copies of nrow * 68 bytes.
        // stage counter, its ring slot and the slot's phase (advanced together:
        // a division by the runtime ring depth per stage costs every warp)
        uint32_t sc = 0, slot = 0, ph = 0;
        bool ok = true;
        for (int it = it_begin; it < it_end && ok; ++it) {
            const GvItem f = item_of(it);
            if (f.nrow == 0) continue;
            int nsl = f.nsl;
            if (nsl < 0) {  // routed: slots of this expert
                if (R.fast)
                    nsl = __popc(__ballot_sync(0xffffffffu, R.v0 == f.e)) + __popc(__ballot_sync(0xffffffffu, R.v1 == f.e));
                else
                    nsl = R.off[(it - n_sh) / a.routed.subs + 1] - R.off[(it - n_sh) / a.routed.subs];
            }
            const int G = (nsl + kGvNT - 1) / kGvNT;
            const WLayout L = GV_SIDE(f.side, L);
            const int KT = L.kt_count, kps = GV_SIDE(f.side, kps);
            const uint8_t* W0 = GV_SIDE(f.side, W0);
            const uint8_t* W1 = GV_SIDE(f.side, W1);
            const uint32_t piece = (uint32_t)f.nrow * L.rb;
            for (int g = 0; g < G && ok; ++g)
                for (int k0 = 0; k0 < KT; k0 += kps, ++sc) {
                    const int s = (int)slot;
                    // (the first ns stages are fresh: nothing to wait for)
                    if (sc >= (uint32_t)a.ns &&
                        !gv_warp_wait(&empty[s], ph ^ 1u, status, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    const int nk = KT - k0 < kps ? KT - k0 : kps;
                    const bool stall = (int)blockIdx.x == a.stall_cta && (int)sc == a.stall_stage;  // test only
                    uint8_t* st_base = ring + (size_t)s * kGvStage;
                    if (GV_SIDE(f.side, tma)) {
                        // one tensor copy a matrix: kps k-steps of the sub-tile's lines (a
                        // last stage past KT reads zeros there and still lands kps pieces)
                        if (lane == 0 && !stall) {
                            ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)(NMAT * kps) * piece);
                            const int line0 = (f.r0 / kSubRows) * 17, tile = f.e * L.mt_count + f.mt;
#pragma unroll
                            for (int m = 0; m < NMAT; ++m)
                                ptx::tma_load_4d(st_base + (size_t)m * kps * piece,
                                                 f.side ? &a.shared.tm[m] : &a.routed.tm[m], 0, line0, k0, tile,
                                                 &full[s]);
                        }
                    } else {
                        // one bulk copy a (matrix, k-step), issued by as many lanes
                        if (lane == 0 && !stall) ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)(NMAT * nk) * piece);
                        __syncwarp();
                        if (lane < NMAT * nk && !stall) {
                            const int m = lane / nk, kk = lane - m * nk;
                            ptx::bulk_g2s(st_base + (size_t)(m * kps + kk) * piece,
                                          (m ? W1 : W0) + L.block(f.e, f.mt, k0 + kk) + (size_t)f.r0 * L.rb, piece,
                                          &full[s]);
                        }
                    }
                    __syncwarp();
                    if (++slot == (uint32_t)a.ns) {
                        slot = 0;
                        ph ^= 1u;
                    }
                }
        }
        // every copy issued lands before the CTA can exit (bounded; a stage the
        // test-only stall skipped has no copy to wait for)
        if (lane == 0) {
            volatile int never = 0;
            const uint32_t first = sc > (uint32_t)a.ns ? sc - a.ns : 0u;
            for (uint32_t q = first; q < sc; ++q)
                if (!((int)blockIdx.x == a.stall_cta && (int)q == a.stall_stage))
                    gv_wait(&full[q % a.ns], (q / a.ns) & 1u, status, &never, a.wait_limit);
        }
        return;
    }

    // ----------------------------------------------------------- consumers
    // Warp cw owns one (matrix, 16-row group) pair of the item and every W-th
    // k-step of each stage.  Per k-step it runs four m16n8k16 tensor-core
    // products: A = 16 weight rows x 16 columns (the quantised values
    // themselves, exact in fp16), B = the same 16 columns of the 8 token
    // columns (fp16, each token's window scaled by a power of two).  The
    // 16 columns of a product lie in one 32-column block, and thread t of a
    // fragment holds columns 8t .. 8t+3 (first product) or 8t+4 .. 8t+7
    // (second) of the block: the same permutation of K in A and B, so that a
    // thread's A values are one 8-byte load per row.  Each block's fp32 result
    // is multiplied by the rows' block scales and added in block order.
    const int ct = tid - 32, cw = ct >> 5;
    const int gq = lane >> 2, tq = lane & 3;  // fragment row group / token, thread in group
    uint8_t* sxb = sm + lay.x;                // [kGvNT][kGvXRow] fp16 activation window
    int* xmax = (int*)(sm + lay.x + kGvNT * kGvXRow);  // [kGvNT]: max |x| of the window (float bits)
    float* xsc = (float*)(xmax + kGvNT);               // [kGvNT]: the factor that undoes the scaling
    if (ct < kGvNT) xmax[ct] = 0;             // ordered before first use by the window barrier
    uint32_t slot = 0, ph = 0, rbuf = 0;  // ring slot and its phase, advanced per stage
    bool waited_primary = !a.pdl_secondary;

    int staged_side = -1, staged_e = -1;  // the item whose tokens the window holds (one group, one window)
    for (int it = it_begin; it < it_end; ++it) {
        const GvItem f = item_of(it);
        if (f.nrow == 0) continue;
        const WLayout L = GV_SIDE(f.side, L);
        const int rsub = GV_SIDE(f.side, rsub), kps = GV_SIDE(f.side, kps), KT = L.kt_count;
        // slot list of the item: routed fast = the ballot masks of its expert
        uint32_t mk0 = 0u, mk1 = 0u;
        int nsl = f.nsl, jrow = 0;
        if (f.side == 0) {
            if (R.fast) {
                mk0 = __ballot_sync(0xffffffffu, R.v0 == f.e);
                mk1 = __ballot_sync(0xffffffffu, R.v1 == f.e);
                nsl = __popc(mk0) + __popc(mk1);
            } else {
                jrow = (it - n_sh) / a.routed.subs;
                nsl = R.off[jrow + 1] - R.off[jrow];
            }
        }
        auto slot_of = [&](int q) {
            if (f.side == 1) return q;
            return R.fast ? nth_bit(mk0, mk1, q) : R.slots[R.off[jrow] + q];
        };
        // this warp's row group and k-step residue.  One matrix: 16 rows, the
        // fragment's rows 0-7 and 8-15 being rows rg16 + 0..7 and + 8..15.  Gate/up:
        // 8 rows of both matrices, the fragment's rows 0-7 from gate and 8-15 from
        // up, so that one thread holds both halves of its SwiGLU.
        const int GR = NMAT == 2 ? 8 : 16;  // rows of a group
        const int nrg = rsub / GR, P = nrg, W = (kGvConsumers / 32) / P;
        const int rg = cw % P, kr = cw / P;
        const bool live = GR * rg < f.nrow;
        // the row group's tile (a 256-row item spans two) and row inside it; a
        // k-step of a stage holds one piece per matrix, or per tile of a pair
        const int tt = (GR * rg) / kTileM, rin = (GR * rg) % kTileM;
        // the row group inside its piece: sub-block (r0 + rin) / 32 of the tile
        const int sbk = (f.r0 + rin) / kSubRows;
        const int nr = sub_rows(L.rows(f.mt + tt), sbk);
        const uint32_t roff = (uint32_t)((rin / kSubRows) * L.sub_bytes());
        const int rra = rin % kSubRows + gq;  // the fragment's row gq: row rra of the sub-block
        const uint32_t piece = (uint32_t)(f.nrow < kTileM ? f.nrow : kTileM) * L.rb;
        // the fragment's rows 8-15: the up piece's row rra (gate/up), or row rra + 8
        const uint32_t offb = NMAT == 2 ? (uint32_t)kps * piece : 8u * 32u;
        const int G = (nsl + kGvNT - 1) / kGvNT;
        for (int g = 0; g < G; ++g) {
            const int nt = nsl - g * kGvNT < kGvNT ? nsl - g * kGvNT : kGvNT;
            float tot[4] = {0.f, 0.f, 0.f, 0.f};  // rows rra, rra+8 x tokens 2tq, 2tq+1
            bool ok = true;
            // the window still holds this item's tokens (the previous item was the same
            // expert, in one token group and one window): no restaging
            const bool one = G == 1 && KT <= kGvXSteps;
            const bool reuse = one && staged_side == f.side && staged_e == f.e;
            for (int w0 = 0; w0 < KT; w0 += kGvXSteps) {
                const int nw = KT - w0 < kGvXSteps ? KT - w0 : kGvXSteps;
                if (!reuse) {
                    ok = consumers_and(ok && !*abort_flag);  // the previous window is no longer read
                    if (!ok) break;
                    if (!waited_primary) {
                        asm volatile("griddepcontrol.wait;" ::: "memory");
                        waited_primary = true;
                    }
                    // stage the nt tokens' activations of this window: each token's largest
                    // magnitude first, then the values times the power of two that puts it in
                    // [2^14, 2^15), rounded to fp16 (exact for 16-bit inputs in range)
                    const int cols = nw * kTileK, col0 = w0 * kTileK;
                    constexpr int VE = 16 / XB;  // elements per 16-byte vector
                    const int vpr = cols / VE;   // vectors per token row
                    const void* xg = GV_SIDE(f.side, x);
                    const int xt = GV_SIDE(f.side, x_type);
                    // every vector of the window is loaded once, into registers (at most 8
                    // tokens x 2048 columns: RV vectors a thread), then converted from there
                    constexpr int RV = XB == 4 ? 8 : 4;
                    uint4 v[RV];
                    int qv[RV];
    #pragma unroll
                    for (int r = 0; r < RV; ++r) {
                        const int idx = ct + r * kGvConsumers;
                        qv[r] = -1;
                        v[r] = make_uint4(0u, 0u, 0u, 0u);
                        if (idx < nt * vpr) {
                            const int q = idx / vpr, cc = (idx - q * vpr) * VE, col = col0 + cc;
                            const int sl = slot_of(g * kGvNT + q);
                            const int row = f.side == 1 ? sl : (a.routed.x_per_slot ? sl : sl / a.k);
                            qv[r] = q;
                            if (col < L.n_in)
                                v[r] = __ldg((const uint4*)((const uint8_t*)xg + ((size_t)row * L.n_in + col) * XB));
                        }
                    }
                    auto unpack = [&](const uint4& u, float (&e)[8]) {
                        if (XB == 4) {
                            e[0] = __uint_as_float(u.x); e[1] = __uint_as_float(u.y);
                            e[2] = __uint_as_float(u.z); e[3] = __uint_as_float(u.w);
                        } else {
                            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
    #pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                e[2 * b] = ld_x16(uw[b] & 0xffffu, xt);
                                e[2 * b + 1] = ld_x16(uw[b] >> 16, xt);
                            }
                        }
                    };
    #pragma unroll
                    for (int r = 0; r < RV; ++r) {
                        if (qv[r] < 0) continue;
                        float e[8];
                        unpack(v[r], e);
                        float mx = 0.f;
    #pragma unroll
                        for (int i = 0; i < VE; ++i) mx = fmaxf(mx, fabsf(e[i]));
                        if (mx > 0.f) atomicMax(&xmax[qv[r]], __float_as_int(mx));
                    }
                    consumers_sync();
    #pragma unroll
                    for (int r = 0; r < RV; ++r) {
                        if (qv[r] < 0) continue;
                        const int q = qv[r], idx = ct + r * kGvConsumers;
                        float e[8];
                        unpack(v[r], e);
                        const float sinv = ldexpf(1.0f, -scale_exp(__int_as_float(xmax[q])));
                        uint32_t hv[4];
    #pragma unroll
                        for (int i = 0; i < VE / 2; ++i) {
                            const __half2 hh = __floats2half2_rn(e[2 * i] * sinv, e[2 * i + 1] * sinv);
                            hv[i] = *(const uint32_t*)&hh;
                        }
                        uint8_t* dstx = sxb + (size_t)q * kGvXRow + (size_t)(idx - q * vpr) * VE * 2;
                        if (XB == 4) *(uint2*)dstx = make_uint2(hv[0], hv[1]);
                        else *(uint4*)dstx = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                    }
                    if (ct < kGvNT) xsc[ct] = ldexpf(1.0f, scale_exp(__int_as_float(xmax[ct])));
                    consumers_sync();
                    if (ct < kGvNT) xmax[ct] = 0;  // next written after the next window's first barrier
                }
                const float s0 = xsc[2 * tq], s1 = xsc[2 * tq + 1];  // tokens 2tq, 2tq + 1
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const uint8_t* xrow = sxb + (size_t)gq * kGvXRow + 16 * tq;  // token gq, columns 8tq..
                for (int k0 = w0; k0 < w0 + nw; k0 += kps) {
                    const int nk = KT - k0 < kps ? KT - k0 : kps;
                    const int s = (int)slot;
                    const uint32_t par = ph;
                    if (++slot == (uint32_t)a.ns) {
                        slot = 0;
                        ph ^= 1u;
                    }
                    if (!gv_warp_wait(&full[s], par, status, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    if (live) {
                        for (int kk = kr; kk < nk; kk += W) {
                            const uint8_t* pc = ring + (size_t)s * kGvStage + (size_t)(tt * kps + kk) * piece + roff;
                            const uint8_t* xk = xrow + (size_t)(k0 - w0 + kk) * kTileK * 2;
                            const uint4 xb[2] = {*(const uint4*)xk, *(const uint4*)(xk + 64)};
                            if (WT == MOE_MXFP4) {
                                // block b: bytes 16b + 4tq .. of the row (columns 32b + 8tq .. 32b + 8tq + 7)
                                const uint8_t* ca = pc + (size_t)rra * 32 + 4 * tq;
                                const uint32_t wa[2] = {*(const uint32_t*)ca, *(const uint32_t*)(ca + 16)};
                                const uint32_t wb[2] = {*(const uint32_t*)(ca + offb), *(const uint32_t*)(ca + offb + 16)};
                                const uint8_t* sp = pc + (size_t)nr * 32 + rra * 2;
                                const uint32_t sa = *(const uint16_t*)sp;
                                const uint32_t sb2 = *(const uint16_t*)(sp + (NMAT == 2 ? offb : 16u));
#pragma unroll
                                for (int b = 0; b < 2; ++b) {
                                    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                                    for (int j = 0; j < 2; ++j) {
                                        const uint32_t x0 = j ? xb[b].z : xb[b].x, x1 = j ? xb[b].w : xb[b].y;
                                        mma_16816(c, e2m1x2_h2(wa[b] >> (16 * j)), e2m1x2_h2(wb[b] >> (16 * j)),
                                                  e2m1x2_h2(wa[b] >> (16 * j + 8)), e2m1x2_h2(wb[b] >> (16 * j + 8)), x0, x1);
                                    }
                                    // E8M0 scales reach 2^127: the token factors come off first (exact
                                    // powers of two), so no partial sum leaves the range of the result
                                    const float da = e8m0_float((sa >> (8 * b)) & 0xffu), db = e8m0_float((sb2 >> (8 * b)) & 0xffu);
                                    acc[0] = fmaf(da, c[0] * s0, acc[0]);
                                    acc[1] = fmaf(da, c[1] * s1, acc[1]);
                                    acc[2] = fmaf(db, c[2] * s0, acc[2]);
                                    acc[3] = fmaf(db, c[3] * s1, acc[3]);
                                }
                            } else {
                                // block b: 8 bytes at 32 b nr + 32 row + 8 tq (columns 32b + 8tq .. 32b + 8tq + 7)
                                const uint8_t* qa = pc + (size_t)rra * 32 + 8 * tq;
                                const uint2 ua[2] = {*(const uint2*)qa, *(const uint2*)(qa + (size_t)nr * 32)};
                                const uint2 ub[2] = {*(const uint2*)(qa + offb), *(const uint2*)(qa + (size_t)nr * 32 + offb)};
                                const uint8_t* sp = pc + (size_t)nr * kTileK + rra * 4;
                                const uint32_t da2 = *(const uint32_t*)sp;
                                const uint32_t db2 = *(const uint32_t*)(sp + (NMAT == 2 ? offb : 32u));
#pragma unroll
                                for (int b = 0; b < 2; ++b) {
                                    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                                    for (int j = 0; j < 2; ++j) {
                                        const uint32_t wa = j ? ua[b].y : ua[b].x, wb = j ? ub[b].y : ub[b].x;
                                        const uint32_t x0 = j ? xb[b].z : xb[b].x, x1 = j ? xb[b].w : xb[b].y;
                                        mma_16816(c, q8_h2(wa, 0x7170u), q8_h2(wb, 0x7170u), q8_h2(wa, 0x7372u),
                                                  q8_h2(wb, 0x7372u), x0, x1);
                                    }
                                    const float da = __half2float(__ushort_as_half((unsigned short)(da2 >> (16 * b))));
                                    const float db = __half2float(__ushort_as_half((unsigned short)(db2 >> (16 * b))));
                                    acc[0] = fmaf(da, c[0], acc[0]);
                                    acc[1] = fmaf(da, c[1], acc[1]);
                                    acc[2] = fmaf(db, c[2], acc[2]);
                                    acc[3] = fmaf(db, c[3], acc[3]);
                                }
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&empty[s]);
                }
                // Q8_0: undo the window's token scaling (exact powers of two) into the
                // totals (fp16 block scales keep the scaled sums far inside the float range)
                if (WT == MOE_MXFP4) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) tot[i] += acc[i];
                } else {
                    tot[0] = fmaf(acc[0], s0, tot[0]);
                    tot[1] = fmaf(acc[1], s1, tot[1]);
                    tot[2] = fmaf(acc[2], s0, tot[2]);
                    tot[3] = fmaf(acc[3], s1, tot[3]);
                }
                // a failed wait is acted on at the next barrier, which every consumer reaches
            }
            staged_side = one ? f.side : -1;
            staged_e = f.e;
            if (W == 1) {
                // every k-step of the row group was this warp's: its totals are the
                // results, stored without a reduction or a barrier (a failed wait is
                // acted on at the next window's barrier, or ends with the range)
                if (ok && live) {
                    const int sl0 = 2 * tq < nt ? slot_of(g * kGvNT + 2 * tq) : 0;
                    const int sl1 = 2 * tq + 1 < nt ? slot_of(g * kGvNT + 2 * tq + 1) : 0;
                    if (DUAL) {  // tot[0..1]: gate, tot[2..3]: up, row GR rg + gq, tokens 2tq, 2tq + 1
                        const int r = GR * rg + gq, n = f.mt * kTileM + f.r0 + r;
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const float gt = tot[i], up = tot[2 + i];
                            if (r < f.nrow && n < L.n_out && 2 * tq + i < nt)
                                GV_SIDE(f.side, h)[(int64_t)(i ? sl1 : sl0) * L.n_out + n] =
                                    __float2bfloat16_rn(gt / (1.0f + expf(-gt)) * up);
                        }
                    } else {
#pragma unroll
                        for (int ii = 0; ii < 4; ++ii) {
                            const int r = GR * rg + gq + 8 * (ii >> 1), q = 2 * tq + (ii & 1);
                            const int n = f.mt * kTileM + f.r0 + r;
                            if (r < f.nrow && n < L.n_out && q < nt)
                                GV_SIDE(f.side, out)[(int64_t)((ii & 1) ? sl1 : sl0) * L.n_out + n] = tot[ii];
                        }
                    }
                }
                continue;
            }
            // per-warp totals, then each (row, token) adds its k-step residues in order
            float* rd = red + (rbuf & 1u) * (kGvRedBytes / 4);  // alternate buffers: no barrier after the reads
            ++rbuf;
#pragma unroll
            for (int i = 0; i < 4; ++i) rd[((kr * P + rg) * 32 + lane) * 4 + i] = tot[i];
            if (!consumers_and(ok && !*abort_flag)) return;  // uniform
            for (int idx = ct; idx < rsub * nt; idx += kGvConsumers) {
                const int r = idx % rsub, q = idx / rsub;
                const int n = f.mt * kTileM + f.r0 + r;
                if (r >= f.nrow || n >= L.n_out) continue;
                // (row, token) in the fragments of group r / GR: lane (r mod 8) * 4 + q / 2,
                // entry q mod 2 of the matrix's half (gate/up: gate 0-1, up 2-3; one
                // matrix: rows r mod 16 < 8 in 0-1, the others in 2-3)
                const int rgi = r / GR, rr = r % GR;
                const int ln = (rr & 7) * 4 + (q >> 1);
                float v[NMAT];
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const int ii = (NMAT == 2 ? 2 * m : (rr >> 3) * 2) + (q & 1);
                    float t = 0.f;
                    for (int k2 = 0; k2 < W; ++k2) t += rd[((k2 * P + rgi) * 32 + ln) * 4 + ii];
                    v[m] = t;
                }
                const int sl = slot_of(g * kGvNT + q);
                if (DUAL) {
                    const float gt = v[0], up = v[NMAT - 1];
                    GV_SIDE(f.side, h)[(int64_t)sl * L.n_out + n] = __float2bfloat16_rn(gt / (1.0f + expf(-gt)) * up);
                } else {
                    GV_SIDE(f.side, out)[(int64_t)sl * L.n_out + n] = v[0];
                }
            }
            // (the buffer just read is written again two groups later, after the next
            // group's barrier, which every consumer reaches only after these reads)
        }
    }
#undef GV_SIDE
}

// The call's status, once every CTA of the finalising launch has finished: the
// last CTA to finish copies the status word to status_out and clears the
// header words the launches use, so that the next call starts from zero with
// no memset or copy of its own (thread 0 of each CTA).
__device__ __forceinline__ void gemv_finalize(const GemvArgs& a) {
    // the primary launch's status writes are visible past this wait (a no-op
    // for a launch that is not a programmatic dependent)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __threadfence();  // this CTA's writes before its count
    int* hdr = a.hdr;
    if (atomicAdd(hdr + kHdrDone, 1) != (int)gridDim.x - 1) return;
    __threadfence();  // every other CTA's writes before the read
    const int st = read_status(hdr + kHdrStatus);
    if (a.status_out) *a.status_out = st;
    hdr[kHdrStatus] = 0;
    hdr[kHdrWaitSite] = 0;
    hdr[kHdrDone] = 0;
}

// One CTA of 544 threads an SM.
template <int DUAL, int XB, int WT>
__global__ void __launch_bounds__(kGvThreads, 1)
gemv_kernel(const __grid_constant__ GemvArgs a) {
    gemv_body<DUAL, XB, WT>(a);
    if (a.finalize) {
        __syncthreads();
        if (threadIdx.x == 0) gemv_finalize(a);
    }
}

// Rows per item of the routed side: 256 (a pair of full tiles, single-matrix
// sides only), 128, 64 or 32.  A CTA streams a contiguous range of items and
// the launch ends with its fullest CTA: ceil(items / SMs) items, each costing
// its bytes plus a fixed cost (decode, activation window, reduction) worth
// about 96 KB of stream (~2 us at one SM's share of HBM).  The height with the
// least such cost wins (the larger one on a tie); `experts` estimates the
// distinct experts.
static int pick_rsub(const WLayout& L, int nmat, int64_t experts, int64_t other_items, int sms, bool pairs) {
    constexpr int64_t kItemCost = 96 * 1024;
    int best = 32;
    int64_t best_cost = -1;
    for (int r : {256, 128, 64, 32}) {
        if (r > kTileM && !pairs) continue;
        const int64_t per_expert = r > kTileM ? L.mt_count / 2 : (int64_t)L.mt_count * (kTileM / r);
        const int64_t items = experts * per_expert + other_items;
        const int64_t per_cta = (items + sms - 1) / sms;
        const int64_t cost = per_cta * ((int64_t)r * L.kt_count * L.rb * nmat + kItemCost);
        if (best_cost < 0 || cost < best_cost) {
            best = r;
            best_cost = cost;
        }
    }
    return best;
}

// k-steps per ring stage: as many as fill kGvStage bytes with the sub-tile's
// rows of every matrix, at most 8 (the activation window of 8 tokens holds 8).
static int stage_ksteps(const WLayout& L, int rsub, int nmat) {
    const int k = (int)(kGvStage / ((uint32_t)L.rb * rsub * nmat));
    return k < 1 ? 1 : k > 8 ? 8 : k;
}

void gemv_plan_side(GemvSide& s, int dual) {
    s.rsub = kTileM;
    s.subs = s.L.mt_count;
    s.kps = stage_ksteps(s.L, kTileM, dual + 1);
}

template <int DUAL, int XB, int WT>
static moe_status launch_t(const GemvArgs& a, size_t smem, unsigned grid, int pdl_attr, cudaStream_t stream) {
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        // the largest shared-memory carveout: an SM configured for one launch's
        // CTA alone would have no room left for a CTA of the other launch
        if (cudaFuncSetAttribute(gemv_kernel<DUAL, XB, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kGvSmemBudget) != cudaSuccess ||
            cudaFuncSetAttribute(gemv_kernel<DUAL, XB, WT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return MOE_ERR_CUDA;
        attr_dev = dev;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_attr ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<DUAL, XB, WT>, a) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static int gv_sm_count() {
    static int dev_cached = -1, n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev != dev_cached) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        dev_cached = dev;
    }
    return n > 0 ? n : 148;
}

// cuTensorMapEncodeTiled from the driver, fetched once through the runtime.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::atomic<int> tried{0};
    if (!fn && !tried.exchange(1)) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)f;
    }
    return fn;
}

// Tensor maps of a side's weight matrices over the repacked layout seen as
// [expert x row tile][k-step][line][inner bytes] (uint8): a k-step block of a
// 128-row tile is 68 lines of inner = 32 rb / 17 bytes (128 for Q8_0, 64 for
// MXFP4), a 32-row sub-block 17 of them.  The box is a sub-tile's lines for
// kps k-steps of one tile.  Only when every row tile is full (one stride per
// dimension); otherwise the side keeps the per-k-step bulk copies.
static void plan_tensor_maps(GemvSide& sd, int n_experts, int nmat) {
    sd.tma = 0;
    const WLayout& L = sd.L;
    if (L.n_out_pad % kTileM != 0) return;
    const uint8_t* W[2] = {sd.W0, sd.W1};
    for (int m = 0; m < nmat; ++m)
        if (!W[m] || ((uintptr_t)W[m] & 15)) return;
    auto enc = tensor_map_encoder();
    if (!enc) return;
    const cuuint64_t inner = (cuuint64_t)L.rb * kSubRows / 17, blk = (cuuint64_t)kTileM * L.rb;
    cuuint64_t dims[4] = {inner, blk / inner, (cuuint64_t)L.kt_count, (cuuint64_t)n_experts * L.mt_count};
    cuuint64_t strides[3] = {inner, blk, blk * (cuuint64_t)L.kt_count};
    // a 256-row item: the full lines of two consecutive tiles
    const int rt = sd.rsub < kTileM ? sd.rsub : kTileM;
    cuuint32_t box[4] = {(cuuint32_t)inner, (cuuint32_t)(17 * (rt / kSubRows)), (cuuint32_t)sd.kps,
                         (cuuint32_t)(sd.rsub / rt)};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    for (int m = 0; m < nmat; ++m) {
        if (enc(&sd.tm[m], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(W[m]), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return;
    }
    sd.tma = 1;
}

// test-only stall (moe_testing_stall): CTA, stage, wait limit in microseconds
static std::atomic<int> g_stall_cta{-1}, g_stall_stage{0}, g_stall_wait_us{0};

static long long stall_limit_cycles() {
    int dev = 0, khz = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
    return (long long)g_stall_wait_us.load() * (khz > 0 ? khz : 2000000) / 1000;
}

// The stall as the grouped GEMM uses it: that CTA's activation copy of that
// k-step (counted over the CTA's tiles) is never issued.
bool testing_stall_state(int* cta, int* stage, long long* limit_cycles) {
    const int c = g_stall_cta.load();
    if (c < 0) return false;
    *cta = c;
    *stage = g_stall_stage.load();
    *limit_cycles = stall_limit_cycles();
    return true;
}

moe_status launch_gemv(const GemvArgs& in, cudaStream_t stream) {
    GemvArgs a = in;
    a.stall_cta = g_stall_cta.load();
    a.stall_stage = g_stall_stage.load();
    if (a.stall_cta >= 0) a.wait_limit = stall_limit_cycles();
    const int S = a.n_tokens * a.k;
    if (S > kGvMaxSlots || (a.wtype != MOE_Q8_0 && a.wtype != MOE_MXFP4)) return MOE_ERR_UNSUPPORTED;
    const bool f32 = a.routed.x_type == MOE_F32 || (a.has_shared && a.shared.x_type == MOE_F32);
    if (f32 && a.has_shared && a.routed.x_type != a.shared.x_type) return MOE_ERR_UNSUPPORTED;
    const int nmat = a.dual + 1;
    const int sms = gv_sm_count();
    // rows per item: 32 for the shared side (its items carry every token, so
    // they are the slowest per byte), then the routed side given those items
    int64_t sh_items = 0;
    if (a.has_shared) {
        a.shared.rsub = 32;
        a.shared.subs = a.shared.L.mt_count * (kTileM / a.shared.rsub);
        a.shared.kps = stage_ksteps(a.shared.L, a.shared.rsub, nmat);
        sh_items = a.shared.subs;
    }
    // tile pairs: one matrix, every tile full and an even count of them, the
    // copies by tensor map (the only copy path that fetches two tiles at once)
    const bool pairs = nmat == 1 && a.routed.L.n_out_pad % (2 * kTileM) == 0;
    auto plan_routed = [&](int rsub) {
        a.routed.rsub = rsub;
        a.routed.subs = rsub > kTileM ? a.routed.L.mt_count / 2 : a.routed.L.mt_count * (kTileM / rsub);
        a.routed.kps = stage_ksteps(a.routed.L, rsub, nmat);
        plan_tensor_maps(a.routed, a.n_experts, nmat);
    };
    // distinct experts expected of S slots drawn uniformly from E, E (1 - (1 - 1/E)^S),
    // at most max_distinct (the bound that sizes the grid)
    const double e_f = (double)a.n_experts;
    int64_t experts = (int64_t)(e_f * (1.0 - pow(1.0 - 1.0 / e_f, (double)S)) + 0.5);
    if (experts > a.max_distinct) experts = a.max_distinct;
    if (experts < 1) experts = 1;
    plan_routed(pick_rsub(a.routed.L, nmat, experts, sh_items, sms, pairs));
    if (a.routed.rsub > kTileM && !a.routed.tma) plan_routed(kTileM);
    if (a.wait_limit <= 0) a.wait_limit = kGvWaitLimit;
    if (a.has_shared) plan_tensor_maps(a.shared, 1, nmat);

    const uint32_t fixed = gv_lay(0, S, a.n_experts).total;
    int ns = (int)((kGvSmemBudget - fixed - 2 * 8 * 8) / kGvStage);
    if (ns > 8) ns = 8;
    if (ns < 2) return MOE_ERR_UNSUPPORTED;
    a.ns = ns;
    const size_t smem = gv_lay(ns, S, a.n_experts).total;
    if (smem > kGvSmemBudget) return MOE_ERR_UNSUPPORTED;

    const int64_t items_max = (int64_t)a.max_distinct * a.routed.subs + sh_items;
    if (items_max == 0) return MOE_OK;
    int64_t grid = sms;
    if (grid > items_max) grid = items_max;
    const int pdl_attr = a.pdl_wait || a.pdl_secondary;
    const unsigned g = (unsigned)grid;
    if (a.wtype == MOE_MXFP4) {
        if (a.dual)
            return f32 ? launch_t<1, 4, MOE_MXFP4>(a, smem, g, pdl_attr, stream)
                       : launch_t<1, 2, MOE_MXFP4>(a, smem, g, pdl_attr, stream);
        return f32 ? launch_t<0, 4, MOE_MXFP4>(a, smem, g, pdl_attr, stream)
                   : launch_t<0, 2, MOE_MXFP4>(a, smem, g, pdl_attr, stream);
    }
    if (a.dual)
        return f32 ? launch_t<1, 4, MOE_Q8_0>(a, smem, g, pdl_attr, stream)
                   : launch_t<1, 2, MOE_Q8_0>(a, smem, g, pdl_attr, stream);
    return f32 ? launch_t<0, 4, MOE_Q8_0>(a, smem, g, pdl_attr, stream)
               : launch_t<0, 2, MOE_Q8_0>(a, smem, g, pdl_attr, stream);
}

}  // namespace moe

extern "C" void moe_testing_stall(int cta, int stage, int wait_us) {
    moe::g_stall_stage.store(stage < 0 ? 0 : stage);
    moe::g_stall_wait_us.store(wait_us < 1 ? 1 : wait_us);
    moe::g_stall_cta.store(cta < 0 ? -1 : cta);
}
