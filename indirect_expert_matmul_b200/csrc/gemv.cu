// Weight-streaming expert mat-vec for small token counts (decode), with the
// shared expert handled as more work items of the same launch - the fusion of
// llama.cpp PR #29184 ("CUDA: fuse shared experts into MMVQ", release b11370)
// restated for this library.
//
// Decode is bound by the weight stream, so the kernel is built around moving
// the repacked weights in large contiguous pieces:
//  - a work item is (distinct routed expert, 128-row tile, K-chunk) or
//    (shared expert, 128-row tile, K-chunk); every k-step block of one
//    (expert, row tile) is contiguous in the repacked layout, so a stage of
//    up to two (dual) or four (single) k-steps of one matrix is a single bulk
//    copy of up to 34 KB;
//  - one producer warp streams the stages of the CTA's items through a ring
//    of shared-memory stages, ahead of the consumers and across items;
//  - 512 consumer threads dequantise (exact fp32 q*d) and take the dot
//    products with up to 8 tokens at a time: thread = (row, 16 columns);
//  - when there are fewer (expert, row tile) groups than SMs (a single decode
//    token), K is split into chunks; each chunk writes fp32 partial sums and
//    the CTA that finishes a group last adds the chunks in chunk order and
//    applies the epilogue.  Every sum has a fixed order, so results do not
//    depend on timing.
// A CTA finds the distinct experts and their slots from ids itself (bitmap +
// a per-CTA slot table), so the decode path needs no row-id launch.
//
// Modes: single matrix (mul_mat_id rows, or the down projection writing
// dst[t][s]), or dual gate/up with a SwiGLU epilogue writing bf16 h[t][s].
// The down launch is a programmatic dependent of the gate/up launch: its
// producer streams weights while gate/up finishes; its consumers wait for
// gate/up before reading h.
#include "common.cuh"
#include "gemv_args.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kGvConsumers = 512;
constexpr int kGvThreads = 32 + kGvConsumers;  // warp 0: producer
constexpr uint32_t kGvBlock = kTileM * kRowBytes;  // 8704: one k-step of a full row tile
constexpr uint32_t kGvSmemBudget = 200 * 1024;
constexpr long long kGvWaitLimit = 1ll << 32;

struct GvLay {
    uint32_t ring, x, red, bm, wp, tab, bars, misc, total;
};

__host__ __device__ inline GvLay gv_lay(const GemvArgs& a) {
    GvLay m;
    uint32_t o = 0;
    m.ring = o; o += (uint32_t)a.ns * a.stage_bytes;
    m.x = o; o += a.x_bytes;
    m.red = o; o += a.red_bytes;
    m.bm = o; o += a.bm_words * 4u;
    m.wp = o; o += (a.bm_words + 1u) * 4u;
    m.tab = o; o += a.tab_words * 4u;
    o = (o + 15u) & ~15u;
    m.bars = o; o += 2u * (uint32_t)a.ns * 8u;
    m.misc = o; o += 16u * 4u;
    m.total = o;
    return m;
}

// Packed fp32 pairs (two lanes of one 64-bit register): fma.rn.f32x2 does two
// independent round-to-nearest fp32 fmas, the same as two fmaf calls.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float f2sum(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo + hi;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ float ld_x16(uint32_t bits16, int x_type) {
    return x_type == MOE_BF16 ? __uint_as_float(bits16 << 16) : __half2float(__ushort_as_half((unsigned short)bits16));
}

// Bounded wait by one thread: false on expiry (status set, abort raised) or
// when another thread has raised abort.
__device__ __forceinline__ bool gv_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!ptx::mbar_try_wait_sleep(bar, parity, 20000)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kGvWaitLimit) {
            *abort_flag = 1;
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
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

// One work item.
struct GvItem {
    const GemvSide* sd;
    int shared;   // 1: shared expert
    int e;        // expert of the weights
    int mt;       // 128-row tile
    int c;        // K-chunk
    int kt0, nk;  // first k-step and k-steps of the chunk
    int rows;     // rows of the tile
    int nsl;      // slots (routed) or tokens (shared)
    int sbase;    // first entry of the expert's slots in the slot list
    int group;    // split-K counter index
};

template <int DUAL, int XB>
__global__ void __launch_bounds__(kGvThreads, 1)
gemv_kernel(const GemvArgs a) {
    extern __shared__ __align__(128) uint8_t sm[];
    constexpr int NMAT = DUAL + 1;
    int* status = a.hdr + kHdrStatus;
    if (!a.pdl_secondary) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (read_status(status) != 0) return;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const GvLay lay = gv_lay(a);
    uint8_t* ring = sm + lay.ring;
    uint8_t* sx = sm + lay.x;
    float* red = (float*)(sm + lay.red);
    uint32_t* bm = (uint32_t*)(sm + lay.bm);
    int* wp = (int*)(sm + lay.wp);
    int* tab = (int*)(sm + lay.tab);
    uint64_t* full = (uint64_t*)(sm + lay.bars);
    uint64_t* empty = full + a.ns;
    int* misc = (int*)(sm + lay.misc);
    volatile int* abort_flag = misc;   // misc[0]
    int* last_flag = misc + 1;
    const int S = a.n_tokens * a.k;
    const int nwords = (int)a.bm_words;

    // ---- the distinct routed experts: bitmap + per-word prefix of popcounts
    for (int w = tid; w < nwords; w += kGvThreads) bm[w] = 0u;
    if (tid == 0) {
        for (int s = 0; s < a.ns; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kGvConsumers / 32);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    int* ids_sh = tab + 2 * (a.max_distinct + 1) + S;  // ids, read from global memory once
    for (int i = tid; i < S; i += kGvThreads) {
        const int v = __ldg(a.ids + i);
        ids_sh[i] = v;
        if (v >= 0 && v < a.n_experts) atomicOr(&bm[v >> 5], 1u << (v & 31));
        else set_status(status, MOE_ERR_BAD_ID);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix, 32 words per step
        int run = 0;
        for (int w0 = 0; w0 < nwords; w0 += 32) {
            const int w = w0 + lane;
            const int c = w < nwords ? __popc(bm[w]) : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (w < nwords) wp[w] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) wp[nwords] = run;
    }
    __syncthreads();
    const int n_distinct = wp[nwords];
    // ---- slot table: the slots of distinct expert j are list[off[j] .. off[j+1])
    int* cnt = tab;                      // [n_distinct + 1]
    int* off = tab + (a.max_distinct + 1);
    int* list = off + (a.max_distinct + 1);
    auto rank_of = [&](int v) { return wp[v >> 5] + __popc(bm[v >> 5] & ((1u << (v & 31)) - 1u)); };
    for (int j = tid; j <= n_distinct; j += kGvThreads) cnt[j] = 0;
    __syncthreads();
    for (int i = tid; i < S; i += kGvThreads) {
        const int v = ids_sh[i];
        if (v >= 0 && v < a.n_experts) atomicAdd(&cnt[rank_of(v)], 1);
    }
    __syncthreads();
    if (warp == 0) {
        int run = 0;
        for (int j0 = 0; j0 < n_distinct; j0 += 32) {
            const int j = j0 + lane;
            const int c = j < n_distinct ? cnt[j] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (j < n_distinct) off[j] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) off[n_distinct] = run;
    }
    __syncthreads();
    for (int j = tid; j < n_distinct; j += kGvThreads) cnt[j] = 0;
    __syncthreads();
    for (int i = tid; i < S; i += kGvThreads) {  // order inside an expert is free: slots are independent
        const int v = ids_sh[i];
        if (v >= 0 && v < a.n_experts) {
            const int j = rank_of(v);
            list[off[j] + atomicAdd(&cnt[j], 1)] = i;
        }
    }
    __syncthreads();

    const GemvSide& R = a.routed;
    const GemvSide& Sh = a.shared;
    const int per_e = R.L.mt_count * R.chunks;
    const int n_items_r = n_distinct * per_e;
    const int n_items = n_items_r + (a.has_shared ? Sh.L.mt_count * Sh.chunks : 0);

    auto item_of = [&](int it) {
        GvItem f;
        if (it < n_items_r) {
            const int j = it / per_e, rem = it - j * per_e;
            f.sd = &R;
            f.shared = 0;
            f.mt = rem / R.chunks;
            f.c = rem - f.mt * R.chunks;
            int lo = 0, hi = nwords;  // wp[lo] <= j < wp[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (wp[mid] <= j) lo = mid; else hi = mid;
            }
            uint32_t bits = bm[lo];
            for (int q = j - wp[lo]; q > 0; --q) bits &= bits - 1;
            f.e = lo * 32 + __ffs(bits) - 1;
            f.sbase = off[j];
            f.nsl = off[j + 1] - off[j];
            f.group = R.group0 + j * R.L.mt_count + f.mt;
        } else {
            const int i2 = it - n_items_r;
            f.sd = &Sh;
            f.shared = 1;
            f.mt = i2 / Sh.chunks;
            f.c = i2 - f.mt * Sh.chunks;
            f.e = 0;
            f.sbase = 0;
            f.nsl = a.n_tokens;
            f.group = Sh.group0 + f.mt;
        }
        f.kt0 = f.c * f.sd->kc;
        f.nk = min(f.sd->kc, f.sd->L.kt_count - f.kt0);
        f.rows = f.sd->L.rows(f.mt);
        return f;
    };
    const int sk = a.sk, ns = a.ns;

    if (warp == 0) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            uint32_t sc = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const GvItem f = item_of(it);
                const GemvSide& sd = *f.sd;
                const int G = (f.nsl + kGvNT - 1) / kGvNT;
                for (int g = 0; g < G && ok; ++g)
                    for (int ks = 0; ks < f.nk; ks += sk, ++sc) {
                        const int nks = min(sk, f.nk - ks);
                        const int s = (int)(sc % (uint32_t)ns);
                        if (!gv_wait(&empty[s], ((sc / ns) & 1u) ^ 1u, status, abort_flag)) { ok = false; break; }
                        const uint32_t bytes = (uint32_t)nks * f.rows * kRowBytes;
                        ptx::mbar_arrive_expect_tx(&full[s], NMAT * bytes);
#pragma unroll
                        for (int m = 0; m < NMAT; ++m)
                            ptx::bulk_g2s(ring + (size_t)s * a.stage_bytes + (size_t)m * sk * kGvBlock,
                                          (m ? sd.W1 : sd.W0) + sd.L.block(f.e, f.mt, f.kt0 + ks), bytes, &full[s]);
                    }
            }
            // every copy issued lands before the CTA can exit (bounded)
            volatile int never = 0;
            const uint32_t first = sc > (uint32_t)ns ? sc - ns : 0u;
            for (uint32_t q = first; q < sc; ++q) gv_wait(&full[q % ns], (q / ns) & 1u, status, &never);
        }
        return;
    }

    // ----------------------------------------------------------- consumers
    // thread = (32-column half hh, row r, 16-column chunk c16): eight lanes read
    // four rows' 128 contiguous bytes, so the 16-byte shared loads do not conflict
    const int ct = tid - 32;
    const int c16 = ct & 1, r = (ct >> 1) & (kTileM - 1), hh = ct >> 8;
    const uint32_t xrow = (uint32_t)a.xw * kTileK;  // activation window row, elements
    uint32_t sc = 0;
    bool waited_primary = !a.pdl_secondary;

    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        const GvItem f = item_of(it);
        const GemvSide& sd = *f.sd;
        const WLayout L = sd.L;
        const int G = (f.nsl + kGvNT - 1) / kGvNT;
        const int S_side = f.shared ? a.n_tokens : S;
        auto slot_of = [&](int q) { return f.shared ? q : list[f.sbase + q]; };
        for (int g = 0; g < G; ++g) {
            const int nt = min(kGvNT, f.nsl - g * kGvNT);
            float acc[NMAT][kGvNT];
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int q = 0; q < kGvNT; ++q) acc[m][q] = 0.f;
            bool ok = true;
            for (int w0 = 0; w0 < f.nk; w0 += a.xw) {
                const int nw = min(a.xw, f.nk - w0);
                // the previous window's activations are no longer read; stop together on abort
                ok = consumers_and(ok && !*abort_flag);
                if (!ok) break;
                if (!waited_primary) {
                    asm volatile("griddepcontrol.wait;" ::: "memory");
                    waited_primary = true;
                }
                // stage the activations of the nt tokens for this window, as fp32
                const int cols = nw * kTileK, col0 = (f.kt0 + w0) * kTileK;
                constexpr int VE = 16 / XB;  // elements per 16-byte vector
                for (int idx = ct; idx < nt * cols / VE; idx += kGvConsumers) {
                    const int q = idx / (cols / VE), cc = (idx - q * (cols / VE)) * VE, col = col0 + cc;
                    const int sl = slot_of(g * kGvNT + q);
                    const int row = f.shared ? sl : (sd.x_per_slot ? sl : sl / a.k);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (col < L.n_in) v = __ldg((const uint4*)((const uint8_t*)sd.x + ((size_t)row * L.n_in + col) * XB));
                    float* dst = (float*)sx + (size_t)q * xrow + cc;
                    if (XB == 4) {
                        *(uint4*)dst = v;
                    } else {
                        const uint32_t uw[4] = {v.x, v.y, v.z, v.w};
                        float e[8];
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            e[2 * b] = ld_x16(uw[b] & 0xffffu, sd.x_type);
                            e[2 * b + 1] = ld_x16(uw[b] >> 16, sd.x_type);
                        }
                        *(float4*)dst = make_float4(e[0], e[1], e[2], e[3]);
                        *(float4*)(dst + 4) = make_float4(e[4], e[5], e[6], e[7]);
                    }
                }
                consumers_sync();
                for (int ks = w0; ks < w0 + nw; ks += sk, ++sc) {
                    const int nks = min(sk, f.nk - ks);
                    const int s = (int)(sc % (uint32_t)ns);
                    int okw = 1;
                    if (lane == 0) okw = gv_wait(&full[s], (sc / ns) & 1u, status, abort_flag);
                    if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
                    if (r < f.rows) {
                        for (int kk = 0; kk < nks; ++kk) {
                            // w = q*d for this thread's 16 columns of each matrix, as 8 packed pairs
                            uint64_t w2[NMAT][8];
#pragma unroll
                            for (int m = 0; m < NMAT; ++m) {
                                const uint8_t* blk = ring + (size_t)s * a.stage_bytes + (size_t)m * sk * kGvBlock +
                                                     (size_t)kk * f.rows * kRowBytes;
                                const uint4 qv = *(const uint4*)(blk + (size_t)hh * f.rows * 32 + r * 32 + c16 * 16);
                                const float d =
                                    __half2float(*(const __half*)(blk + (size_t)f.rows * kTileK + r * 4 + hh * 2));
                                const uint64_t dd = f2pack(d, d), nd = f2pack(-32896.0f * d, -32896.0f * d);
                                const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const uint32_t wd = qw[i >> 1];
                                    const int b0 = (2 * i) & 3;
                                    w2[m][i] = fma2(f2pack(magic_byte(wd, b0), magic_byte(wd, b0 + 1)), dd, nd);
                                }
                            }
                            const float* xk = (const float*)sx + (size_t)(ks - w0 + kk) * kTileK + hh * 32 + c16 * 16;
#pragma unroll
                            for (int q = 0; q < kGvNT; ++q) {
                                if (q >= nt) break;
                                const ulonglong2* xv = (const ulonglong2*)(xk + (size_t)q * xrow);
                                // two independent packed chains per matrix, added in a fixed order
                                uint64_t t0[NMAT], t1[NMAT];
#pragma unroll
                                for (int m = 0; m < NMAT; ++m) t0[m] = t1[m] = 0ull;
#pragma unroll
                                for (int v4 = 0; v4 < 4; ++v4) {
                                    const ulonglong2 u = xv[v4];
#pragma unroll
                                    for (int m = 0; m < NMAT; ++m) {
                                        t0[m] = fma2(w2[m][2 * v4], u.x, t0[m]);
                                        t1[m] = fma2(w2[m][2 * v4 + 1], u.y, t1[m]);
                                    }
                                }
#pragma unroll
                                for (int m = 0; m < NMAT; ++m) acc[m][q] += f2sum(t0[m]) + f2sum(t1[m]);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&empty[s]);
                }
            }
            // the two 16-column chunks (adjacent lanes; a + b == b + a), then the
            // two 32-column halves of each row, in a fixed order
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int q = 0; q < kGvNT; ++q) {
                    const float v = acc[m][q] + __shfl_xor_sync(0xffffffffu, acc[m][q], 1);
                    if (c16 == 0 && q < nt) red[((hh * kTileM + r) * kGvNT + q) * NMAT + m] = v;
                }
            if (!consumers_and(ok && !*abort_flag)) return;  // uniform
            if (hh == 0 && c16 == 0 && r < f.rows) {
                const int n = f.mt * kTileM + r;
                if (n < L.n_out)
                    for (int q = 0; q < nt; ++q) {
                        const int sl = slot_of(g * kGvNT + q);
                        float v[NMAT];
#pragma unroll
                        for (int m = 0; m < NMAT; ++m)
                            v[m] = red[((0 * kTileM + r) * kGvNT + q) * NMAT + m] +
                                   red[((1 * kTileM + r) * kGvNT + q) * NMAT + m];
                        if (sd.chunks > 1) {
                            float* pp = sd.part + (((size_t)f.c * S_side + sl) * L.n_out_pad + n) * NMAT;
#pragma unroll
                            for (int m = 0; m < NMAT; ++m) pp[m] = v[m];
                        } else if (DUAL) {
                            const float gt = v[0], up = v[NMAT - 1];
                            sd.h[(int64_t)sl * L.n_out + n] = __float2bfloat16_rn(gt / (1.0f + expf(-gt)) * up);
                        } else {
                            sd.out[(int64_t)sl * L.n_out + n] = v[0];
                        }
                    }
            }
            consumers_sync();  // red is free again
        }
        if (sd.chunks > 1) {
            // the last chunk of this (expert, row tile) to finish adds all chunks in order
            __threadfence();
            consumers_sync();
            if (ct == 0) *last_flag = atomicAdd(a.hdr + kHdrCnt0 + f.group, 1) == sd.chunks - 1;
            consumers_sync();
            if (*last_flag) {
                __threadfence();
                for (int idx = ct; idx < f.nsl * f.rows; idx += kGvConsumers) {
                    const int q = idx / f.rows, rr = idx - q * f.rows;
                    const int n = f.mt * kTileM + rr;
                    if (n >= L.n_out) continue;
                    const int sl = slot_of(q);
                    float v[NMAT];
#pragma unroll
                    for (int m = 0; m < NMAT; ++m) v[m] = 0.f;
                    for (int c = 0; c < sd.chunks; ++c) {
                        const volatile float* pp = sd.part + (((size_t)c * S_side + sl) * L.n_out_pad + n) * NMAT;
#pragma unroll
                        for (int m = 0; m < NMAT; ++m) v[m] += pp[m];
                    }
                    if (DUAL) {
                        const float gt = v[0], up = v[NMAT - 1];
                        sd.h[(int64_t)sl * L.n_out + n] = __float2bfloat16_rn(gt / (1.0f + expf(-gt)) * up);
                    } else {
                        sd.out[(int64_t)sl * L.n_out + n] = v[0];
                    }
                }
                if (ct == 0) atomicExch(a.hdr + kHdrCnt0 + f.group, 0);
            }
            consumers_sync();  // last_flag is free again
        }
    }
}

void gemv_plan_side(GemvSide& s, int dual) {
    (void)dual;
    s.kc = s.L.kt_count;
    s.chunks = 1;
    s.group0 = 0;
}

template <int DUAL, int XB>
static moe_status launch_t(const GemvArgs& a, size_t smem, unsigned grid, cudaStream_t stream) {
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        if (cudaFuncSetAttribute(gemv_kernel<DUAL, XB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kGvSmemBudget + 16 * 1024) != cudaSuccess)
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
    cfg.numAttrs = a.pdl_secondary ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<DUAL, XB>, a) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
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

moe_status launch_gemv(const GemvArgs& in, cudaStream_t stream) {
    GemvArgs a = in;
    const int S = a.n_tokens * a.k;
    if (S > kGvMaxSlots) return MOE_ERR_UNSUPPORTED;
    const int64_t groups_r = (int64_t)a.max_distinct * a.routed.L.mt_count;
    const int64_t groups_s = a.has_shared ? a.shared.L.mt_count : 0;
    if (groups_r + groups_s == 0) return MOE_OK;
    const bool f32 = a.routed.x_type == MOE_F32 || (a.has_shared && a.shared.x_type == MOE_F32);
    if (f32 && a.has_shared && a.routed.x_type != a.shared.x_type) return MOE_ERR_UNSUPPORTED;
    const int nmat = a.dual + 1;
    const int sms = gv_sm_count();

    // Split K when the (expert, row tile) groups alone cannot cover the SMs.
    // Shared-expert items carry every token, so that side is split further.
    // Split groups count arrivals in the header (kGvMaxGroups counters).
    GemvSide* sides[2] = {&a.routed, a.has_shared ? &a.shared : nullptr};
    for (GemvSide* s : sides)
        if (s) s->kc = s->L.kt_count, s->chunks = 1;
    const bool small = S <= kGvSplitSlots;
    int chunks_r = 1, chunks_s = 1;
    if (small) {
        // as many chunks as fit in one wave of CTAs (a second, partial wave would
        // double the time of the CTAs that run it)
        chunks_r = (int)(sms / (groups_r + groups_s));
        if (chunks_r < 1) chunks_r = 1;
        chunks_s = chunks_r > 2 * a.n_tokens ? chunks_r : 2 * a.n_tokens;
    }
    int counters = 0;
    auto split = [&](GemvSide* s, int64_t groups, int want) {
        if (!s || !s->part || want <= 1 || counters + groups > kGvMaxGroups) return;
        const int KT = s->L.kt_count;
        if (want > kGvMaxChunks) want = kGvMaxChunks;
        if (want > KT) want = KT;
        s->kc = (KT + want - 1) / want;
        s->chunks = (KT + s->kc - 1) / s->kc;
        s->group0 = counters;
        counters += (int)groups;
    };
    split(&a.routed, groups_r, chunks_r);
    if (a.has_shared) split(&a.shared, groups_s, chunks_s);

    // A stage carries ~34 KB whatever the mode (per-stage costs are fixed): two
    // k-steps of both matrices, or four of one.
    a.sk = a.dual ? 2 : 4;
    a.xw = 16;
    a.stage_bytes = (uint32_t)nmat * a.sk * kGvBlock;
    a.x_bytes = (uint32_t)kGvNT * a.xw * kTileK * 4;  // fp32 after staging
    a.red_bytes = (uint32_t)2 * kTileM * kGvNT * nmat * 4;
    a.bm_words = (uint32_t)((a.n_experts + 31) / 32);
    a.tab_words = (uint32_t)(2 * (a.max_distinct + 1) + 2 * S);  // cnt, off, slot list, ids
    a.ns = 1;
    const uint32_t fixed = gv_lay(a).total - a.stage_bytes;
    int ns = (int)((kGvSmemBudget - fixed) / a.stage_bytes);
    if (ns > 8) ns = 8;
    if (ns < 2) return MOE_ERR_UNSUPPORTED;
    a.ns = ns;
    const size_t smem = gv_lay(a).total;

    const int64_t items_max = groups_r * a.routed.chunks + groups_s * (a.has_shared ? a.shared.chunks : 0);
    int64_t grid = sms;
    if (grid > items_max) grid = items_max;
    if (a.dual)
        return f32 ? launch_t<1, 4>(a, smem, (unsigned)grid, stream) : launch_t<1, 2>(a, smem, (unsigned)grid, stream);
    return f32 ? launch_t<0, 4>(a, smem, (unsigned)grid, stream) : launch_t<0, 2>(a, smem, (unsigned)grid, stream);
}

}  // namespace moe
