/*
 * moe.h - C ABI of a B200 (sm_100a) library for the Mixture-of-Experts
 * indirect matrix multiplication, GGML_OP_MUL_MAT_ID.
 *
 * Source pages:
 *   [PR283]  "ik_llama.cpp 的 CUDA 更优 MoE 实现：以可复现的间接矩阵乘法换取
 *            Prompt Processing 性能跃升" - the article on ik_llama.cpp PR #283
 *            "CUDA: better MoE implementation" (sections 1.2, 2, 2.1, 5, 6).
 *   [b11370] "llama.cpp 發布 b11370，CUDA 後端將共享專家融合進 MMVQ" - release
 *            note of llama.cpp PR #29184 "CUDA: fuse shared experts into MMVQ".
 *   [cmoe]   "Optimalizace MoE modelů na slabém GPU: spuštění GPT-OSS-120B s
 *            6 GB VRAM až 30 t/s", section "Architektura Mixture of Experts"
 *            (the router before the path and the weighted combine after it).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is DEVICE memory owned by the caller, except the
 *    stream handle.  The library never allocates, frees or keeps a host copy
 *    of ids, so the host-buffer lifetime hazard discussed in [PR283] section 5
 *    (ids_host / rmapping leaving scope before an async copy) cannot arise.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns without synchronising.  Argument errors found on the
 *    host return a negative moe_status at once and enqueue nothing.
 *  - Errors found on the device (an id outside [0, n_experts), a bounded wait
 *    that expired) are written to a status word inside the caller's
 *    workspace.  The first error sticks: later kernels that see a non-zero
 *    status do nothing, and moe_get_status() reports it and clears it.
 *  - Results are a pure function of the inputs: no floating-point atomics, no
 *    order that depends on timing ([PR283] sections 1.1 and 2: the old
 *    atomic-increment copy made results irreproducible).
 *  - Layouts (row-major, innermost last):
 *      ids       int32 [n_tokens][k]           expert of (token t, slot s)
 *      x         [n_tokens][n_in]               MOE_BROADCAST
 *                [n_tokens][k][n_in]            MOE_PER_SLOT
 *      dst       float [n_tokens][k][n_out]
 *      weights   Q8_0 blocks [n_experts][n_out][n_in/32], 34 bytes each:
 *                fp16 scale d, then 32 int8 q; weight = d*q.  Stacked by
 *                expert as the page's [n_embd, n_embd_gate, n_experts]
 *                ([PR283] section 1.2).  Kernels read the repacked form made
 *                by moe_weights_prepare().
 *  - Limits ([PR283] section 2.1, mmq_id.cu#L128-L129, "32-bit packing
 *    safety"): n_tokens < 2^22, k < 2^10; also 1 <= k <= n_experts,
 *    n_tokens*k < 2^31 and n_experts <= 16384.  Violations return
 *    MOE_ERR_RANGE.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID = -1,     /* null pointer, bad enum, misaligned buffer, n_in % 32 != 0 */
    MOE_ERR_RANGE = -2,       /* a size outside the limits above */
    MOE_ERR_BAD_ID = -3,      /* device: some ids[t][s] outside [0, n_experts) */
    MOE_ERR_CUDA = -4,        /* a CUDA runtime call failed */
    MOE_ERR_TIMEOUT = -5,     /* device: a bounded wait inside a kernel expired */
    MOE_ERR_UNSUPPORTED = -6  /* a shape this build does not handle */
} moe_status;

typedef enum { MOE_BROADCAST = 0, MOE_PER_SLOT = 1 } moe_mode;
typedef enum { MOE_BF16 = 0, MOE_F16 = 1, MOE_F32 = 2 } moe_dtype;
/* Expert weight types.  Q8_0: 34-byte blocks (fp16 d, 32 int8 q; w = d*q).
 * MXFP4: 17-byte blocks of 32 weights (the OCP microscaling FP4 type that the
 * TensorSharp benchmark page lists for GPT-OSS, "Q8_0/MXFP4"): an E8M0 scale
 * byte X, then 16 bytes of 4-bit E2M1 codes, element i of the block in the low
 * nibble of byte i and element 16+i in its high nibble; w = 2^(X-127) * e2m1,
 * with E2M1 = sign, 2 exponent bits (bias 1), 1 mantissa bit (codes 0..7 are
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6).  X = 255 (NaN) and weights beyond the float
 * range give unspecified results. */
typedef enum { MOE_Q8_0 = 0, MOE_MXFP4 = 1 } moe_wtype;

typedef void *moe_stream; /* cudaStream_t */

/* Human-readable name of a status code (static string). */
MOE_API const char *moe_status_string(int status);

/* ------------------------------------------------------------------ memory */

/*
 * Bytes of workspace needed by one call with these sizes.  n_hidden is the
 * expert FFN width for moe_ffn (0 for moe_mul_mat_id / moe_row_ids);
 * n_hidden_shared the shared expert's width (0 = none); n_in the reduction
 * length of the first product.  The workspace holds the status word, the
 * row-id tables, the hidden activations of moe_ffn and, for MOE_F32 input,
 * an fp16 copy of x.  It must be 256-byte aligned.
 */
MOE_API size_t moe_workspace_size(int64_t n_tokens, int k, int n_experts, int n_in, int n_hidden,
                          int n_hidden_shared, moe_dtype x_type);

/* Zero the status word of a fresh workspace (enqueued on `stream`).  Call once
 * before the workspace's first use. */
MOE_API moe_status moe_workspace_init(void *workspace, moe_stream stream);

/*
 * Wait for `stream`, then read the workspace's status word and reset it to
 * MOE_OK.  Returns the device-side status of the calls enqueued before, or
 * MOE_ERR_CUDA if the stream itself failed.
 */
MOE_API moe_status moe_get_status(void *workspace, moe_stream stream);

/* ----------------------------------------------------------------- weights */

/* Bytes of the repacked weights for one stacked matrix.  Equal to the Q8_0
 * size (1.0625 bytes per weight) when n_out % 16 == 0 and n_in % 64 == 0;
 * otherwise padded with zero weights up to those multiples. */
MOE_API size_t moe_weights_prepared_size(int n_experts, int n_out, int n_in);

/*
 * One-time repack of Q8_0 blocks (layout above, 34-byte blocks, any 2-byte
 * alignment) into the tile-major form the kernels stream: per expert, per
 * 128-row tile, per 64-column tile, a 16-byte aligned block holding the rows'
 * int8 values (offset by +128) followed by their two fp16 scales.  The byte
 * count is unchanged (see above).  `prepared` must be 16-byte aligned and
 * moe_weights_prepared_size() bytes long; experts are stored one after the
 * other, so a matrix may be repacked in expert chunks (the operators need the
 * whole matrix 256-byte aligned).  Not part of the timed path.
 */
MOE_API moe_status moe_weights_prepare(const void *q8_0_blocks, int n_experts, int n_out, int n_in, void *prepared,
                               moe_stream stream);

/*
 * The same two calls for a given weight type: moe_weights_prepared_size(...)
 * and moe_weights_prepare(...) are these with MOE_Q8_0.  MOE_MXFP4 takes the
 * 17-byte blocks described at moe_wtype (any 1-byte alignment) and repacks
 * them the same tile-major way (0.53125 bytes per weight when n_out % 16 == 0
 * and n_in % 64 == 0).  MOE_ERR_INVALID for an unknown type.
 */
MOE_API size_t moe_weights_prepared_size_w(moe_wtype w_type, int n_experts, int n_out, int n_in);
MOE_API moe_status moe_weights_prepare_w(moe_wtype w_type, const void *blocks, int n_experts, int n_out, int n_in,
                                         void *prepared, moe_stream stream);

/* ------------------------------------------------------------------ row ids */

/*
 * The deterministic row-id pass ([PR283] sections 2.1 and 6: mmq_ids_helper /
 * compute_row_ids, replacing the atomic-increment k_copy_src1_to_contiguous of
 * section 2).  A stable counting sort of the flat slots t*k+s by expert:
 *   expert_bounds[e]  = number of slots whose expert is < e   (n_experts + 1
 *                       entries; expert_bounds[n_experts] = n_tokens*k)
 *   ids_dst[p]        = t*k+s of the p-th slot in (expert, t, s) order
 *   ids_src1[p]       = t (MOE_BROADCAST) or t*k+s (MOE_PER_SLOT)
 * ids_src1 / ids_dst hold n_tokens*k int32 each.  Out-of-range ids set
 * MOE_ERR_BAD_ID in the workspace status; the tables are then unspecified.
 */
MOE_API moe_status moe_row_ids(const int32_t *ids, int64_t n_tokens, int k, int n_experts, moe_mode mode,
                       int32_t *ids_src1, int32_t *ids_dst, int32_t *expert_bounds, void *workspace,
                       moe_stream stream);

/* --------------------------------------------------------------- operators */

/*
 * GGML_OP_MUL_MAT_ID ([PR283] section 1.2): for every token t and slot s,
 *   dst[t][s][:] = W[ids[t][s]] . x[r],   r = t (broadcast) or (t, s) (per_slot).
 * Runs the row-id pass, then either the grouped GEMM (tensor cores; gather of
 * x rows by ids_src1, Q8_0 dequantisation fused into the tiles, scatter to
 * dst by ids_dst) or, for n_tokens at or below the GEMV threshold, the
 * weight-streaming mat-vec kernel.  x_type MOE_BF16 computes with bf16
 * operands, MOE_F16 / MOE_F32 with fp16 operands; accumulation is fp32.
 * W_prepared comes from moe_weights_prepare(); dst is float [n_tokens][k][n_out].
 */
MOE_API moe_status moe_mul_mat_id(const void *W_prepared, int n_experts, int n_out, int n_in, const void *x,
                          moe_dtype x_type, const int32_t *ids, int64_t n_tokens, int k, moe_mode mode,
                          float *dst, void *workspace, moe_stream stream);

/*
 * Routed expert SwiGLU FFN with an optional always-on shared expert:
 *   g = mul_mat_id(Wg, x, broadcast), u = mul_mat_id(Wu, x, broadcast),
 *   h = silu(g) * u                  (stored as bf16 in expert-sorted order),
 *   dst[t][s][:]    = Wd[ids[t][s]] . h[(t, s)]      float [n_tokens][k][n_embd]
 *   dst_shared[t][:] = Sd . (silu(Sg . x[t]) * (Su . x[t]))  float [n_tokens][n_embd]
 * Gate and up are one pass with two accumulators ("fused_moe_up_gate",
 * [PR283] section 4.2).  The shared expert runs inside the same launches as
 * the routed experts ([b11370]: shared experts fused into the mat-vec pass).
 * Wg, Wu: prepared [n_experts][n_ff][n_embd]; Wd: prepared
 * [n_experts][n_embd][n_ff]; Sg, Su, Sd likewise with one expert and n_ff_shared
 * (all three NULL and n_ff_shared = 0 for no shared expert; dst_shared then
 * unused).
 */
MOE_API moe_status moe_ffn(const void *Wg, const void *Wu, const void *Wd, int n_experts, int n_embd, int n_ff,
                   const void *Sg, const void *Su, const void *Sd, int n_ff_shared, const void *x, moe_dtype x_type,
                   const int32_t *ids, int64_t n_tokens, int k, float *dst, float *dst_shared, void *workspace,
                   moe_stream stream);

/*
 * moe_mul_mat_id and moe_ffn for a given weight type (the plain entry points
 * are these with MOE_Q8_0); every weight pointer must hold that type's
 * prepared form.  MXFP4 weights decode exactly to float (and to bf16: an E2M1
 * value times a power of two has at most 2 significant bits), so the
 * tensor-core path multiplies bf16 operands: x is used as bf16 (exact for bf16
 * input, one rounding for fp16 / fp32 input).  The mat-vec path accumulates
 * exact fp32 products.  MOE_ERR_INVALID for an unknown type.
 */
MOE_API moe_status moe_mul_mat_id_w(moe_wtype w_type, const void *W_prepared, int n_experts, int n_out, int n_in,
                                    const void *x, moe_dtype x_type, const int32_t *ids, int64_t n_tokens, int k,
                                    moe_mode mode, float *dst, void *workspace, moe_stream stream);
MOE_API moe_status moe_ffn_w(moe_wtype w_type, const void *Wg, const void *Wu, const void *Wd, int n_experts,
                             int n_embd, int n_ff, const void *Sg, const void *Su, const void *Sd, int n_ff_shared,
                             const void *x, moe_dtype x_type, const int32_t *ids, int64_t n_tokens, int k, float *dst,
                             float *dst_shared, void *workspace, moe_stream stream);

/*
 * Decode-size moe_ffn that allocates nothing and takes no workspace.  The
 * method's description has no counterpart to this entry point: it serves
 * callers that cannot hand over scratch memory, such as a graph executor that
 * plans every buffer per tensor before running and gives each operation only
 * its inputs and outputs, with no allocator at hand while the graph runs.
 *
 * Computes what moe_ffn computes, on the mat-vec path, for
 *   n_tokens * k <= 64, n_ff <= 2048, n_ff_shared <= 2048
 * (MOE_ERR_RANGE beyond these, checked on the host before any CUDA call).
 * Scratch is one static device array in the library (256-byte status header +
 * 256 KB routed hidden activations + 256 KB shared hidden activations, about
 * 512 KB per device); no call allocates or frees memory.
 *   - A call is two kernel launches on `stream` (gate/up, then down), with no
 *     memset or copy: the status header is zero when the library is loaded,
 *     and every call leaves it zero - the last CTA of the down launch to
 *     finish copies the status word out and clears the header.  The hidden
 *     activations need no initial value (the gate/up kernel writes every
 *     element the down kernel reads).  If the down launch cannot be enqueued,
 *     the call enqueues a memset of the header before returning the error.
 *   - status_out (device int, may be NULL): receives the call's device status
 *     (MOE_OK, MOE_ERR_BAD_ID, MOE_ERR_TIMEOUT), written by that last CTA (for
 *     n_tokens == 0, by an asynchronous memset to MOE_OK); with NULL,
 *     device-side errors are not observable.
 *   - All calls on one device share the one scratch array: calls that may
 *     overlap in time (other streams, other host threads) race on it and give
 *     undefined results.  Order them on one stream or serialise them.
 *   - The first call on each device looks up the array's address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     outside any stream capture.
 */
MOE_API moe_status moe_ffn_decode_noalloc(const void *Wg, const void *Wu, const void *Wd, int n_experts, int n_embd,
                                          int n_ff, const void *Sg, const void *Su, const void *Sd, int n_ff_shared,
                                          const void *x, moe_dtype x_type, const int32_t *ids, int64_t n_tokens, int k,
                                          float *dst, float *dst_shared, int *status_out, moe_stream stream);

/* ------------------------------------------------------------------ router */

/*
 * Router - the step before the indirect matmul ("Optimalizace MoE modelů na
 * slabém GPU: spuštění GPT-OSS-120B s 6 GB VRAM až 30 t/s", section
 * "Architektura Mixture of Experts": a gating network picks k experts per
 * token).  For every token t:
 *   key[e]     = logits[t][e] + bias[e]      (one float addition; bias may be NULL)
 *   ids[t][:]  = the k largest keys in descending order, equal keys in
 *                ascending expert index      (int32 [n_tokens][k])
 *   weights[t][i] = softmax(logits[t])[ids[t][i]], divided by their sum over
 *                the k when normalize != 0   (float [n_tokens][k]).  The
 *                renormalised form is evaluated as the softmax over the k
 *                chosen logits (the same quantity), so it stays finite and
 *                sums to one even where the chosen experts' probabilities
 *                underflow in float (chosen logits far below the row's top).
 * logits: float [n_tokens][n_experts]; bias: float [n_experts] or NULL.  The
 * choice is a pure function of the float keys (bit-identical to any exact
 * evaluation of the rule above); the weights are within
 * (span + 8 + n_experts + k) * 2^-24 relative of the exact softmax, span being
 * the row's largest minus smallest logit.  NaN logits give unspecified ids.
 * Errors (host): MOE_ERR_INVALID for null pointers, 4-byte misalignment,
 * n_experts < 1 or k outside [1, n_experts]; MOE_ERR_RANGE for n_tokens >= 2^22,
 * n_experts > 1024 or k >= 1024.  n_tokens == 0 does nothing.
 */
MOE_API moe_status moe_route(const float *logits, const float *bias, int64_t n_tokens, int n_experts, int k,
                             int normalize, int32_t *ids, float *weights, moe_stream stream);

/* ----------------------------------------------------------------- combine */

/*
 * Weighted combine of each token's expert outputs - the step after the
 * indirect matmul in a MoE layer ("Optimalizace MoE modelů na slabém GPU:
 * spuštění GPT-OSS-120B s 6 GB VRAM až 30 t/s", section "Architektura Mixture
 * of Experts": a router picks k experts per token; the layer output weights
 * their outputs), plus the always-on shared expert ([b11370]):
 *   y[t][j] = sum_s weights[t][s] * dst[t][s][j]  (+ dst_shared[t][j])
 * dst: float [n_tokens][k][n] (moe_mul_mat_id / moe_ffn output); weights:
 * float [n_tokens][k] (the router's weights, any values); dst_shared: float
 * [n_tokens][n] or NULL; y: float [n_tokens][n], caller-owned, must not
 * overlap dst or weights (it may be dst_shared itself).  All pointers 4-byte
 * aligned; 16-byte alignment and n % 4 == 0 take the vector path.
 * Evaluation: per output one fused multiply-add per slot in ascending s, then
 * one add of the shared term - bit-identical from run to run; within
 * (k + 1 + shared) * 2^-24 * sum of the terms' magnitudes of the exact sum.
 * Errors (host, before any launch): MOE_ERR_INVALID for null pointers,
 * misalignment, k < 1 or n < 1; MOE_ERR_RANGE for n_tokens >= 2^22,
 * k >= 1024 or n >= 2^31.  n_tokens == 0 does nothing.
 */
MOE_API moe_status moe_combine(const float *dst, const float *weights, const float *dst_shared, int64_t n_tokens,
                               int k, int64_t n, float *y, moe_stream stream);

/* ------------------------------------------------------------------ tuning */

/* Token count at or below which the mat-vec path is used (default 24); the
 * analogue of ggml's mmq_id threshold ([PR283] section 2.1, ggml-cuda.cu#L2944).
 * The mat-vec path takes n_tokens*k <= 1024; larger calls use the GEMM. */
MOE_API void moe_set_gemv_threshold(int n_tokens);
MOE_API int moe_get_gemv_threshold(void);

/* Force a path for testing: 0 = by threshold, 1 = mat-vec (when n_tokens*k <=
 * 1024, else the GEMM), 2 = grouped GEMM. */
MOE_API void moe_set_path(int path);


/* -------------------------------------------------------------- profiling */

/*
 * Stage timing for benchmarks.  While enabled, every operator call records a
 * CUDA event on its own stream before its first kernel and after each kernel
 * launch; moe_profile_read() waits for those events and returns, per stage
 * name ("row_ids", "gemm_gate_up", "gemm_down", "gemv_gate_up", ...), the
 * number of launches and their summed device time in milliseconds.
 * moe_profile_enable(1) also discards earlier records.  At most 4096 events
 * are kept; later calls are not recorded.  Not thread-safe.
 */
MOE_API void moe_profile_enable(int enable);
MOE_API int moe_profile_read(const char **names, int *launches, double *total_ms, int max_stages);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
