// Deterministic row-id pass: a stable counting sort of the flat slots t*k+s by
// expert, emitting expert_bounds, ids_dst and ids_src1 (the three tables of
// the PR #283 article "ik_llama.cpp 的 CUDA 更优 MoE 实现", section 2.1) plus the
// list of experts that received at least one slot.
//
// One CTA of 32 warps.  The S slots are cut into n_chunks contiguous chunks,
// one per warp.  Pass 1: each warp counts its chunk's slots per expert into a
// private shared-memory row (warp match + one leader add per distinct expert,
// so no two threads update the same counter).  Pass 2: column prefix over the
// chunks and an exclusive prefix over experts give every (chunk, expert) its
// first output position.  Pass 3: each warp walks its chunk again in order and
// places slot i at  start[chunk][e] + (rank of i among equal experts so far).
// The result is unique (ascending (t, s) inside each expert), independent of
// scheduling, and uses no global atomics.
#include "common.cuh"
#include "warp_match.cuh"

namespace moe {

constexpr int kRowIdThreads = 1024;
constexpr int kRowIdWarps = kRowIdThreads / 32;
constexpr int kBatch = 8;  // 32-slot steps whose ids a warp loads at once

// Exclusive block-wide prefix sum of one value per thread (1024 threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sums[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        warp_sums[lane] = wi - w;  // exclusive warp offsets
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    int r = warp_sums[warp] + incl - v;
    __syncthreads();  // warp_sums reusable afterwards
    return r;
}

__global__ void __launch_bounds__(kRowIdThreads, 1)
row_ids_kernel(const int32_t* __restrict__ ids, int S, int k, int E, int mode, int n_chunks, int bn,
               int32_t* __restrict__ ids_src1, int32_t* __restrict__ ids_dst, int32_t* __restrict__ bounds,
               int32_t* __restrict__ active, int32_t* __restrict__ ntile_prefix, int32_t* __restrict__ pad_start,
               int32_t* __restrict__ slot_prow, int* __restrict__ hdr) {
    extern __shared__ int smem[];
    int* off = smem;                        // [n_chunks][E]
    int* cnt = off + (size_t)n_chunks * E;  // [E]
    int* pad_delta = cnt + E;               // [E]: pad_start[e] - bounds[e]
    __shared__ int warp_sums[32];
    __shared__ int totals[4];
    __shared__ int bad;

    if (read_status(hdr + kHdrStatus) != 0) return;  // sticky error: do nothing
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < n_chunks * E; i += blockDim.x) off[i] = 0;
    if (tid == 0) bad = 0;
    __syncthreads();

    const int L = (S + n_chunks - 1) / n_chunks;
    const int c0 = warp * L;
    const int c1 = min(S, c0 + L);
    const unsigned lt_mask = (1u << lane) - 1u;
    const int nb = E > 1 ? 32 - __clz(E - 1) : 1;  // bits of the largest id

    // pass 1: per-chunk histogram (the ids of kBatch 32-slot steps are loaded
    // together, so their load latencies overlap)
    if (warp < n_chunks) {
        int* row = off + (size_t)warp * E;
        int my_bad = 0;
        for (int b0 = c0; b0 < c1; b0 += 32 * kBatch) {
            int ev[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = b0 + 32 * j + lane;
                ev[j] = i < c1 ? __ldg(ids + i) : -1;
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = b0 + 32 * j + lane;
                int e = ev[j];
                if (i < c1 && (e < 0 || e >= E)) { my_bad = 1; e = -1; }
                unsigned m = match_by_ballots(e, nb);
                if (e >= 0 && (m & lt_mask) == 0) row[e] += __popc(m);
                __syncwarp();
            }
        }
        if (__any_sync(0xffffffffu, my_bad) && lane == 0) bad = 1;
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) set_status(hdr + kHdrStatus, MOE_ERR_BAD_ID);
        return;
    }

    // pass 2a: column prefix over chunks -> off[c][e] = count in chunks < c
    for (int e = tid; e < E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < n_chunks; ++c) {
            int v = off[(size_t)c * E + e];
            off[(size_t)c * E + e] = run;
            run += v;
        }
        cnt[e] = run;
    }
    __syncthreads();

    // pass 2b: exclusive prefix over experts (each thread owns a contiguous
    // segment of experts), the compacted list of non-empty experts, the
    // prefix of per-expert column-tile counts ceil(count / bn) for the GEMM,
    // and each expert's first row in the 8-row-aligned tile-major buffers
    const int seg = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(E, tid * seg), e1 = min(E, e0 + seg);
    int local = 0, local_act = 0, local_tiles = 0, local_pad = 0;
    for (int e = e0; e < e1; ++e) {
        local += cnt[e];
        local_act += cnt[e] > 0;
        local_tiles += (cnt[e] + bn - 1) / bn;
        local_pad += (cnt[e] + 7) & ~7;
    }
    int run = block_exclusive_scan(local, warp_sums, &totals[0]);
    int run_act = block_exclusive_scan(local_act, warp_sums, &totals[1]);
    int run_tiles = block_exclusive_scan(local_tiles, warp_sums, &totals[2]);
    int run_pad = block_exclusive_scan(local_pad, warp_sums, &totals[3]);
    for (int e = e0; e < e1; ++e) {
        int c = cnt[e];
        bounds[e] = run;
        ntile_prefix[e] = run_tiles;
        run_tiles += (c + bn - 1) / bn;
        pad_start[e] = run_pad;
        pad_delta[e] = run_pad - run;
        run_pad += (c + 7) & ~7;
        if (c > 0) active[run_act++] = e;
        cnt[e] = run;  // becomes the expert's first position
        run += c;
    }
    if (tid == 0) {
        bounds[E] = totals[0];
        ntile_prefix[E] = totals[2];
        pad_start[E] = totals[3];
        hdr[kHdrActive] = totals[1];
        hdr[kHdrTiles] = totals[2];
    }
    __syncthreads();
    for (int i = tid; i < n_chunks * E; i += blockDim.x) off[i] += cnt[i % E];
    __syncthreads();

    // pass 3: stable placement (ids loaded kBatch steps at a time, as in pass 1)
    if (warp < n_chunks) {
        int* row = off + (size_t)warp * E;
        for (int b0 = c0; b0 < c1; b0 += 32 * kBatch) {
            int ev[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = b0 + 32 * j + lane;
                ev[j] = i < c1 ? __ldg(ids + i) : -1;
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = b0 + 32 * j + lane;
                const int e = ev[j];
                unsigned m = match_by_ballots(e, nb);
                int p = 0;
                if (e >= 0) p = row[e] + __popc(m & lt_mask);
                __syncwarp();
                if (e >= 0) {
                    ids_dst[p] = i;
                    ids_src1[p] = (mode == MOE_BROADCAST) ? i / k : i;
                    if (slot_prow) slot_prow[i] = p + pad_delta[e];
                    if ((m & lt_mask) == 0) row[e] += __popc(m);
                }
                __syncwarp();
            }
        }
    }
}

// Shared memory needed for a given chunk count.
static size_t row_ids_smem(int n_chunks, int E) { return ((size_t)n_chunks + 2) * E * sizeof(int); }

moe_status launch_row_ids(const int32_t* ids, int64_t S, int k, int E, int mode, int32_t* ids_src1,
                          int32_t* ids_dst, int32_t* bounds, int32_t* active, int32_t* ntile_prefix,
                          int32_t* pad_start, int32_t* slot_prow, int bn, int* hdr, cudaStream_t stream) {
    const size_t budget = 200 * 1024;
    int n_chunks = kRowIdWarps;
    while (n_chunks > 1 && row_ids_smem(n_chunks, E) > budget) n_chunks >>= 1;
    if (row_ids_smem(n_chunks, E) > budget) return MOE_ERR_UNSUPPORTED;
    if (S < (int64_t)n_chunks * 32) {  // tiny inputs: fewer, fuller chunks
        n_chunks = (int)((S + 31) / 32);
        if (n_chunks < 1) n_chunks = 1;
    }
    size_t smem = row_ids_smem(n_chunks, E);
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(row_ids_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        attr_dev = dev;
    }
    row_ids_kernel<<<1, kRowIdThreads, smem, stream>>>(ids, (int)S, k, E, mode, n_chunks, bn, ids_src1, ids_dst,
                                                      bounds, active, ntile_prefix, pad_start, slot_prow, hdr);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
