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
//
// Larger calls (at least 16384 slots, at most kRidMaxE experts)
// spread the same three passes over G CTAs of 32 chunks each, in three
// launches: per-CTA counts; one CTA's prefix over CTAs and experts (the
// tables, each CTA's first position per expert); each CTA counting its chunks
// again and placing its slots.  The chunk order (CTA, warp) is slot order, so
// the tables are the same bit for bit as the one-CTA pass gives.
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

// Pass 1 for one warp: the ids of slots [c0, c1) counted per expert into
// row[E] (shared memory, this warp's own row).  Returns 1 on an id outside
// [0, E) (warp-uniform).
__device__ __forceinline__ int warp_count(const int32_t* __restrict__ ids, int c0, int c1, int E, int nb, int* row) {
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    int my_bad = 0;
    // (the ids of kBatch 32-slot steps are loaded together, so their load
    // latencies overlap)
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
    return __any_sync(0xffffffffu, my_bad);
}

// Pass 3 for one warp: slot i of [c0, c1) goes to row[e] + (its rank among the
// chunk's earlier slots of expert e); row[] holds the chunk's first positions
// and is advanced.
__device__ __forceinline__ void warp_place(const int32_t* __restrict__ ids, int c0, int c1, int k, int mode, int nb,
                                           int* row, const int* pad_delta, int32_t* __restrict__ ids_src1,
                                           int32_t* __restrict__ ids_dst, int32_t* __restrict__ slot_prow) {
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
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

// Pass 2b (every thread of a 1024-thread CTA): from the per-expert counts
// cnt[E] (shared), the exclusive prefix over experts - expert_bounds, the
// list of non-empty experts, the prefix of the GEMM's column-tile counts, each
// expert's first row in the 8-row-aligned tile-major buffers and the header
// totals; cnt[e] becomes the expert's first position, pad_delta[e] =
// pad_start[e] - bounds[e].
__device__ __forceinline__ void expert_prefix(int E, int bn, int* cnt, int* pad_delta, int* warp_sums, int* totals,
                                              int32_t* __restrict__ bounds, int32_t* __restrict__ active,
                                              int32_t* __restrict__ ntile_prefix, int32_t* __restrict__ pad_start,
                                              int* __restrict__ hdr) {
    const int tid = threadIdx.x;
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
    const int nb = E > 1 ? 32 - __clz(E - 1) : 1;  // bits of the largest id

    // pass 1: per-chunk histogram
    if (warp < n_chunks && warp_count(ids, c0, c1, E, nb, off + (size_t)warp * E) && lane == 0) bad = 1;
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

    // pass 2b: exclusive prefix over experts and the tables
    expert_prefix(E, bn, cnt, pad_delta, warp_sums, totals, bounds, active, ntile_prefix, pad_start, hdr);
    __syncthreads();
    for (int i = tid; i < n_chunks * E; i += blockDim.x) off[i] += cnt[i % E];
    __syncthreads();

    // pass 3: stable placement
    if (warp < n_chunks)
        warp_place(ids, c0, c1, k, mode, nb, off + (size_t)warp * E, pad_delta, ids_src1, ids_dst, slot_prow);
}

// ---------------------------------------------------------------- G CTAs
// CTA g owns slots [g S / G, (g + 1) S / G), its warp w the w-th of 32 equal
// chunks of that range.  scratch: cta_cnt [G][E] | cta_first [G][E] | pad_delta [E].
__device__ __forceinline__ void cta_chunk(int S, int g, int G, int warp, int& c0, int& c1) {
    const int s0 = (int)(((int64_t)g * S) / G), s1 = (int)(((int64_t)(g + 1) * S) / G);
    const int L = (s1 - s0 + kRowIdWarps - 1) / kRowIdWarps;
    c0 = min(s1, s0 + warp * L);
    c1 = min(s1, c0 + L);
}

// Launch 1: the CTA's count per expert (pass 1 of its 32 chunks, summed).
__global__ void __launch_bounds__(kRowIdThreads, 1)
rid_count_kernel(const int32_t* __restrict__ ids, int S, int E, int32_t* __restrict__ scratch, int* __restrict__ hdr) {
    extern __shared__ int smem[];
    int* off = smem;  // [32][E]
    __shared__ int bad;
    if (read_status(hdr + kHdrStatus) != 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kRowIdWarps * E; i += blockDim.x) off[i] = 0;
    if (tid == 0) bad = 0;
    __syncthreads();
    int c0, c1;
    cta_chunk(S, blockIdx.x, gridDim.x, warp, c0, c1);
    const int nb = E > 1 ? 32 - __clz(E - 1) : 1;
    if (warp_count(ids, c0, c1, E, nb, off + (size_t)warp * E) && lane == 0) bad = 1;
    __syncthreads();
    if (bad) {
        if (tid == 0) set_status(hdr + kHdrStatus, MOE_ERR_BAD_ID);
        return;
    }
    for (int e = tid; e < E; e += blockDim.x) {
        int t = 0;
        for (int w = 0; w < kRowIdWarps; ++w) t += off[w * E + e];
        scratch[(size_t)blockIdx.x * E + e] = t;
    }
}

// Launch 2 (one CTA): per expert, each CTA's count before it (column prefix),
// the expert totals, the tables of pass 2b, then each CTA's first position.
__global__ void __launch_bounds__(kRowIdThreads, 1)
rid_scan_kernel(int E, int G, int bn, int32_t* __restrict__ scratch, int32_t* __restrict__ bounds,
                int32_t* __restrict__ active, int32_t* __restrict__ ntile_prefix, int32_t* __restrict__ pad_start,
                int* __restrict__ hdr) {
    extern __shared__ int smem[];
    int* cnt = smem;  // [E]
    __shared__ int warp_sums[32];
    __shared__ int totals[4];
    if (read_status(hdr + kHdrStatus) != 0) return;
    const int32_t* __restrict__ cta_cnt = scratch;
    int32_t* __restrict__ cta_first = scratch + (size_t)G * E;
    int32_t* pad_delta = scratch + (size_t)2 * G * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int g0 = 0; g0 < G; g0 += 8) {  // eight loads in flight, then their prefix
            int v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = g0 + j < G ? cta_cnt[(size_t)(g0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (g0 + j < G) cta_first[(size_t)(g0 + j) * E + e] = run;
                run += v[j];
            }
        }
        cnt[e] = run;
    }
    __syncthreads();
    expert_prefix(E, bn, cnt, pad_delta, warp_sums, totals, bounds, active, ntile_prefix, pad_start, hdr);
    __syncthreads();
    for (int i = threadIdx.x; i < G * E; i += blockDim.x) cta_first[i] += cnt[i % E];
}

// Launch 3: the CTA's chunks counted again, each chunk's first positions from
// the CTA's, and the slots placed.
__global__ void __launch_bounds__(kRowIdThreads, 1)
rid_place_kernel(const int32_t* __restrict__ ids, int S, int k, int E, int mode, const int32_t* __restrict__ scratch,
                 int32_t* __restrict__ ids_src1, int32_t* __restrict__ ids_dst, int32_t* __restrict__ slot_prow,
                 const int* __restrict__ hdr) {
    extern __shared__ int smem[];
    int* off = smem;  // [32][E]
    if (read_status(hdr + kHdrStatus) != 0) return;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int G = gridDim.x;
    for (int i = tid; i < kRowIdWarps * E; i += blockDim.x) off[i] = 0;
    __syncthreads();
    int c0, c1;
    cta_chunk(S, blockIdx.x, G, warp, c0, c1);
    const int nb = E > 1 ? 32 - __clz(E - 1) : 1;
    warp_count(ids, c0, c1, E, nb, off + (size_t)warp * E);  // (ids were checked by launch 1)
    __syncthreads();
    const int32_t* cta_first = scratch + (size_t)G * E;
    for (int e = tid; e < E; e += blockDim.x) {
        int run = cta_first[(size_t)blockIdx.x * E + e];
        for (int w = 0; w < kRowIdWarps; ++w) {
            const int v = off[w * E + e];
            off[w * E + e] = run;
            run += v;
        }
    }
    __syncthreads();
    warp_place(ids, c0, c1, k, mode, nb, off + (size_t)warp * E, scratch + (size_t)2 * G * E, ids_src1, ids_dst,
               slot_prow);
}

// Shared memory needed for a given chunk count.
static size_t row_ids_smem(int n_chunks, int E) { return ((size_t)n_chunks + 2) * E * sizeof(int); }

moe_status launch_row_ids(const int32_t* ids, int64_t S, int k, int E, int mode, int32_t* ids_src1,
                          int32_t* ids_dst, int32_t* bounds, int32_t* active, int32_t* ntile_prefix,
                          int32_t* pad_start, int32_t* slot_prow, int bn, int* hdr, int32_t* rid_scratch,
                          cudaStream_t stream, int* launches) {
    // G CTAs of 32 chunks: about 2048 slots a CTA, from 8 CTAs on (below that
    // one CTA's pass costs less than two more launches)
    const int64_t G = S / 2048 < kRidMaxCtas ? S / 2048 : kRidMaxCtas;
    if (launches) *launches = 1;
    if (rid_scratch && E <= kRidMaxE && G >= 8) {
        if (launches) *launches = 3;
        const size_t smem = (size_t)kRowIdWarps * E * sizeof(int);
        static int attr_dev_g = -1;
        int dev = 0;
        cudaGetDevice(&dev);
        if (attr_dev_g != dev) {
            if (cudaFuncSetAttribute(rid_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(kRowIdWarps * kRidMaxE * sizeof(int))) != cudaSuccess ||
                cudaFuncSetAttribute(rid_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(kRowIdWarps * kRidMaxE * sizeof(int))) != cudaSuccess)
                return MOE_ERR_CUDA;
            attr_dev_g = dev;
        }
        rid_count_kernel<<<(unsigned)G, kRowIdThreads, smem, stream>>>(ids, (int)S, E, rid_scratch, hdr);
        rid_scan_kernel<<<1, kRowIdThreads, (size_t)E * sizeof(int), stream>>>(E, (int)G, bn, rid_scratch, bounds,
                                                                              active, ntile_prefix, pad_start, hdr);
        rid_place_kernel<<<(unsigned)G, kRowIdThreads, smem, stream>>>(ids, (int)S, k, E, mode, rid_scratch,
                                                                       ids_src1, ids_dst, slot_prow, hdr);
        return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
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
