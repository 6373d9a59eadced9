/*
 * CPU ORACLE for the indirect expert matmul (GGML_OP_MUL_MAT_ID).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file.  The library's own code
 * path never calls it, and this file shares no code, header or table with the
 * GPU library.
 *
 * It is the plain definition, written to be checked by eye:
 *   - fp64 accumulation in ascending reduction index, no blocking, no reordering;
 *   - OpenMP only across independent output elements, so a result never
 *     depends on the thread count.
 *
 * Source pages (cited as below):
 *   [PR283] "ik_llama.cpp 的 CUDA 更优 MoE 实现：以可复现的间接矩阵乘法换取
 *           Prompt Processing 性能跃升" (article on ik_llama.cpp PR #283,
 *           "CUDA: better MoE implementation"), sections 1.2, 2, 2.1, 5, 6.
 *   [b11370] "llama.cpp 發布 b11370，CUDA 後端將共享專家融合進 MMVQ"
 *           (release note of PR #29184 "CUDA: fuse shared experts into MMVQ").
 *   [cmoe]  "Optimalizace MoE modelů na slabém GPU: spuštění GPT-OSS-120B s 6 GB
 *           VRAM až 30 t/s", section "Architektura Mixture of Experts" (a router
 *           picks a few experts per token in every layer).
 *   [TS]    the TensorSharp vs llama.cpp MoE CPU-offload benchmark page
 *           (DeepSeek V4 / Gemma 4 / Qwen / GPT-OSS), per-model results: the
 *           benchmarked weight types include GPT-OSS "Q8_0/MXFP4".
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - Q8_0 block = fp16 scale d, then 32 int8 q; weight = d*q.
 *   - MXFP4 block (the OCP microscaling FP4 type; the pages list MXFP4 among
 *     the benchmarked weight types but print no bytes) = one E8M0 scale byte
 *     X, then 16 bytes of 4-bit E2M1 codes, element i of the block in the low
 *     nibble of byte i and element 16+i in its high nibble (the GGUF order
 *     of 4-bit blocks); weight = 2^(X-127) * e2m1(code).
 *   - x is [T][n_in] (broadcast) or [T][k][n_in] (per_slot); dst is
 *     [T][k][n_out]; W is [E][n_out][n_in] (the page's ne-order
 *     [n_embd, n_embd_gate, n_experts] read innermost-first).
 *   - Order inside an expert's range: ascending (token, slot) - a stable
 *     counting sort; expert_bounds has E+1 exclusive prefix entries.
 *   - ids_src1 = t (broadcast) or t*k+s (per_slot); ids_dst = t*k+s.
 *   - SwiGLU: h = silu(gate) * up, silu(z) = z / (1 + exp(-z)).
 *   - The shared expert is an always-on FFN on x[t] with its own weights,
 *     written to its own output.
 *   - Combine (the step after the path): y[t] = sum_s r[t][s] * dst[t][s] +
 *     dst_shared[t], the slots taken in ascending s.
 *   - Router (the step before it): softmax over all experts' logits; the k
 *     largest of logit + bias chosen (descending, ties to the lower index);
 *     weights = the chosen experts' probabilities, optionally renormalised.
 *
 * Tolerances returned beside every output element follow the bound
 * |gpu - oracle| <= 2e-3 * sum|w*x| + 1e-5; for the two-stage FFN the bound is
 * propagated through SwiGLU (see oracle_ffn_rows).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_OK = 0, OR_ERR_INVALID = -1, OR_ERR_RANGE = -2, OR_ERR_BAD_ID = -3 };
enum { OR_BROADCAST = 0, OR_PER_SLOT = 1 };
enum { OR_BF16 = 0, OR_F16 = 1, OR_F32 = 2 };
enum { OR_Q8_0 = 0, OR_MXFP4 = 1 }; /* weight types */

#define REL_TOL 2e-3
#define ABS_TOL 1e-5
#define SILU_SLOPE_MAX 1.1 /* max |d silu / dz| = 1.0998... */

/* ---------------------------------------------------------------- decoding */

/* IEEE binary16 bits -> exact double. */
static double f16_value(uint16_t b) {
    int sign = b >> 15, ex = (b >> 10) & 31, man = b & 1023;
    double v;
    if (ex == 0) v = ldexp((double)man, -24);
    else if (ex == 31) v = man ? NAN : INFINITY;
    else v = ldexp((double)(1024 + man), ex - 25);
    return sign ? -v : v;
}

/* bfloat16 bits -> exact double. */
static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Activation element i of a buffer of the given type, exact. */
static double x_value(const void *x, int x_type, int64_t i) {
    switch (x_type) {
    case OR_BF16: return bf16_value(((const uint16_t *)x)[i]);
    case OR_F16: return f16_value(((const uint16_t *)x)[i]);
    default: return (double)((const float *)x)[i];
    }
}

/* E2M1 (OCP microscaling FP4 element): bit 3 sign, bits 2-1 exponent (bias 1),
 * bit 0 mantissa.  Exponent 0 is the subnormal 0.5*m; otherwise
 * 2^(exponent-1) * (1 + m/2).  Codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static double e2m1_value(int code) {
    const int ex = (code >> 1) & 3, m = code & 1;
    const double mag = ex == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, ex - 1);
    return (code & 8) ? -mag : mag;
}

/* E8M0 (OCP microscaling scale): 2^(X-127); X = 255 encodes NaN. */
static double e8m0_value(uint8_t x) { return x == 255 ? NAN : ldexp(1.0, (int)x - 127); }

/* Dequantised weight W[e][n][j], exact in double:
 *   Q8_0  = d * q of its 34-byte block ([PR283] 2.1 names Q8_0 among the
 *           quantised types of the mmq_id path);
 *   MXFP4 = 2^(X-127) * e2m1(code) of its 17-byte block ([TS]'s GPT-OSS
 *           weights are "Q8_0/MXFP4"). */
static double w_value(const uint8_t *W, int wtype, int64_t n_out, int64_t n_in, int64_t e, int64_t n, int64_t j) {
    if (wtype == OR_MXFP4) {
        const uint8_t *blk = W + (((e * n_out + n) * (n_in / 32)) + j / 32) * 17;
        const int i = (int)(j % 32);
        const int code = i < 16 ? (blk[1 + i] & 15) : (blk[1 + i - 16] >> 4);
        return e8m0_value(blk[0]) * e2m1_value(code);
    }
    const uint8_t *blk = W + (((e * n_out + n) * (n_in / 32)) + j / 32) * 34;
    uint16_t d = (uint16_t)(blk[0] | (blk[1] << 8));
    int8_t q = (int8_t)blk[2 + (j % 32)];
    return f16_value(d) * (double)q;
}

/* ---------------------------------------------------------------- row ids */

/* Argument limits of the row-id pass.  [PR283] 2.1: n_tokens < 2^22 and
 * n_expert_used < 2^10 "for 32-bit packing safety" (mmq_id.cu#L128-L129);
 * k <= E and T*k < 2^31 are this library's readings. */
int oracle_check_args(int64_t n_tokens, int k, int n_experts) {
    if (n_tokens < 0 || k < 1 || n_experts < 1) return OR_ERR_INVALID;
    if (n_tokens >= (1 << 22) || k >= (1 << 10)) return OR_ERR_RANGE;
    if (k > n_experts) return OR_ERR_RANGE;
    if (n_tokens * (int64_t)k >= ((int64_t)1 << 31)) return OR_ERR_RANGE;
    return OR_OK;
}

/*
 * The deterministic row-id pass ([PR283] 2.1, 6): turn ids into
 *   expert_bounds[E+1]  - each expert's range in the expert-sorted order,
 *   ids_dst[S]          - for sorted position p, the flat dst row t*k+s,
 *   ids_src1[S]         - for sorted position p, the flat src1 row.
 * It replaces the atomic-increment copy of k_copy_src1_to_contiguous ([PR283]
 * 2), whose row order varied run to run.  Written as a stable counting sort:
 * count, exclusive prefix, then place in ascending (t, s).
 */
int oracle_row_ids(const int32_t *ids, int64_t n_tokens, int k, int n_experts, int mode,
                   int32_t *ids_src1, int32_t *ids_dst, int32_t *expert_bounds) {
    int rc = oracle_check_args(n_tokens, k, n_experts);
    if (rc) return rc;
    if (mode != OR_BROADCAST && mode != OR_PER_SLOT) return OR_ERR_INVALID;
    const int64_t S = n_tokens * k;
    for (int64_t i = 0; i < S; ++i)
        if (ids[i] < 0 || ids[i] >= n_experts) return OR_ERR_BAD_ID;

    int64_t *cnt = calloc((size_t)n_experts, sizeof(int64_t));
    int64_t *cur = malloc((size_t)n_experts * sizeof(int64_t));
    for (int64_t i = 0; i < S; ++i) cnt[ids[i]] += 1;              /* 1. count   */
    expert_bounds[0] = 0;                                          /* 2. prefix  */
    for (int e = 0; e < n_experts; ++e) expert_bounds[e + 1] = expert_bounds[e] + (int32_t)cnt[e];
    for (int e = 0; e < n_experts; ++e) cur[e] = expert_bounds[e];
    for (int64_t t = 0; t < n_tokens; ++t)                         /* 3. place   */
        for (int s = 0; s < k; ++s) {
            int e = ids[t * k + s];
            int64_t p = cur[e]++;
            ids_dst[p] = (int32_t)(t * k + s);
            ids_src1[p] = (int32_t)(mode == OR_BROADCAST ? t : t * k + s);
        }
    free(cnt);
    free(cur);
    return OR_OK;
}

/* ---------------------------------------------------------- mul_mat_id */

/* One output row: out[n] = sum_j W[e][n][j] * x[r][j] (ascending j, fp64), and
 * tol[n] = 2e-3 * sum_j |W[e][n][j] * x[r][j]| + 1e-5. */
static void dot_row(const uint8_t *W, int wtype, int64_t n_out, int64_t n_in, int64_t e, const void *x, int x_type,
                    int64_t r, double *out, double *tol) {
    for (int64_t n = 0; n < n_out; ++n) {
        double acc = 0.0, mag = 0.0;
        for (int64_t j = 0; j < n_in; ++j) {
            double prod = w_value(W, wtype, n_out, n_in, e, n, j) * x_value(x, x_type, r * n_in + j);
            acc += prod;
            mag += fabs(prod);
        }
        out[n] = acc;
        if (tol) tol[n] = REL_TOL * mag + ABS_TOL;
    }
}

/*
 * GGML_OP_MUL_MAT_ID by brute force ([PR283] 1.2): for every token t and slot
 * s, take expert e = ids[t][s] and multiply its weight matrix by the src1 row
 * of (t, s):  dst[t][s][:] = W[e] . x[r],  r = t (broadcast) or t*k+s.
 */
int oracle_mul_mat_id_brute(const uint8_t *W, int n_experts, int n_out, int n_in, const void *x, int x_type,
                            const int32_t *ids, int64_t n_tokens, int k, int mode, double *dst, double *tol,
                            int wtype) {
    int rc = oracle_check_args(n_tokens, k, n_experts);
    if (rc) return rc;
    if (n_in % 32) return OR_ERR_INVALID;
    const int64_t S = n_tokens * k;
    for (int64_t i = 0; i < S; ++i)
        if (ids[i] < 0 || ids[i] >= n_experts) return OR_ERR_BAD_ID;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < S; ++i) {
        int64_t t = i / k;
        int64_t r = (mode == OR_BROADCAST) ? t : i;
        dot_row(W, wtype, n_out, n_in, ids[i], x, x_type, r, dst + i * n_out, tol ? tol + i * n_out : NULL);
    }
    return OR_OK;
}

/*
 * The same operator computed the way the new scheme organises it ([PR283]
 * 2.1, 6): build the tables first, then walk each expert's range, read the
 * src1 row named by ids_src1 (gather) and write the result to the dst row
 * named by ids_dst (scatter).  Same fp64 order per element as the brute
 * force, so both must agree bit for bit.
 */
int oracle_mul_mat_id_grouped(const uint8_t *W, int n_experts, int n_out, int n_in, const void *x, int x_type,
                              const int32_t *ids, int64_t n_tokens, int k, int mode, double *dst, double *tol,
                              int wtype) {
    int rc = oracle_check_args(n_tokens, k, n_experts);
    if (rc) return rc;
    if (n_in % 32) return OR_ERR_INVALID;
    const int64_t S = n_tokens * k;
    int32_t *src1 = malloc((size_t)(S ? S : 1) * 4), *dstrow = malloc((size_t)(S ? S : 1) * 4);
    int32_t *bounds = malloc((size_t)(n_experts + 1) * 4);
    rc = oracle_row_ids(ids, n_tokens, k, n_experts, mode, src1, dstrow, bounds);
    if (rc == OR_OK) {
        for (int e = 0; e < n_experts; ++e) {
#pragma omp parallel for schedule(dynamic, 1)
            for (int64_t p = bounds[e]; p < bounds[e + 1]; ++p)
                dot_row(W, wtype, n_out, n_in, e, x, x_type, src1[p], dst + (int64_t)dstrow[p] * n_out,
                        tol ? tol + (int64_t)dstrow[p] * n_out : NULL);
        }
    }
    free(src1);
    free(dstrow);
    free(bounds);
    return rc;
}

/* Rows i of slot list `slots` only (for sampled checks at full size). */
int oracle_mul_mat_id_rows(const uint8_t *W, int n_experts, int n_out, int n_in, const void *x, int x_type,
                           const int32_t *ids, int64_t n_tokens, int k, int mode, const int64_t *slots,
                           int64_t n_slots, double *out, double *tol, int wtype) {
    int rc = oracle_check_args(n_tokens, k, n_experts);
    if (rc) return rc;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_slots; ++i) {
        int64_t sl = slots[i];
        int64_t r = (mode == OR_BROADCAST) ? sl / k : sl;
        dot_row(W, wtype, n_out, n_in, ids[sl], x, x_type, r, out + i * n_out, tol ? tol + i * n_out : NULL);
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ FFN */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * One expert FFN row block: y = Wd[e] . (silu(Wg[e] . x) * (Wu[e] . x)).
 * Gate/up use the token's src1 row (broadcast), down uses the slot's own h
 * row (per_slot): the "fused_moe_up_gate" forward of [PR283] 4.2 followed by
 * the down projection.
 *
 * Tolerance propagation (all element-wise, bounds not estimates):
 *   tol_g, tol_u  = 2e-3 * sum|w*x| + 1e-5                (per stage)
 *   dh           <= 1.1 * tol_g * (|u| + tol_u) + |silu(g)| * tol_u
 *                   (|silu'| <= 1.1; mean-value bound on silu(g')u' - silu(g)u)
 *   tol_h         = dh + 2^-9 * (|h| + dh)   (an implementation may store h
 *                   as bfloat16: relative rounding <= 2^-9)
 *   tol_y         = 2e-3 * sum|wd| (|h| + tol_h) + sum|wd| * tol_h + 1e-5
 */
static void ffn_row(const uint8_t *Wg, const uint8_t *Wu, const uint8_t *Wd, int wtype, int64_t e, int64_t n_embd,
                    int64_t n_ff, const void *x, int x_type, int64_t r, double *y, double *tol_y, double *h,
                    double *th) {
    for (int64_t f = 0; f < n_ff; ++f) {
        double g = 0, u = 0, mg = 0, mu = 0;
        for (int64_t j = 0; j < n_embd; ++j) {
            double xv = x_value(x, x_type, r * n_embd + j);
            double pg = w_value(Wg, wtype, n_ff, n_embd, e, f, j) * xv;
            double pu = w_value(Wu, wtype, n_ff, n_embd, e, f, j) * xv;
            g += pg; u += pu; mg += fabs(pg); mu += fabs(pu);
        }
        double tg = REL_TOL * mg + ABS_TOL, tu = REL_TOL * mu + ABS_TOL;
        double sg = silu(g);
        h[f] = sg * u;
        double dh = SILU_SLOPE_MAX * tg * (fabs(u) + tu) + fabs(sg) * tu;
        th[f] = dh + ldexp(fabs(h[f]) + dh, -9);
    }
    for (int64_t n = 0; n < n_embd; ++n) {
        double acc = 0, m1 = 0, m2 = 0;
        for (int64_t f = 0; f < n_ff; ++f) {
            double w = w_value(Wd, wtype, n_embd, n_ff, e, n, f);
            acc += w * h[f];
            m1 += fabs(w) * (fabs(h[f]) + th[f]);
            m2 += fabs(w) * th[f];
        }
        y[n] = acc;
        if (tol_y) tol_y[n] = REL_TOL * m1 + m2 + ABS_TOL;
    }
}

/*
 * MoE expert FFN over a list of flat slots t*k+s (or all of them when
 * slots == NULL):  y[slot] = FFN_{ids[slot]}(x[t]).
 * Optionally the shared expert ([b11370]: fused into the same mat-vec pass;
 * here its plain definition) over a list of tokens: y_sh[t] = FFN_shared(x[t]).
 */
int oracle_ffn_rows(const uint8_t *Wg, const uint8_t *Wu, const uint8_t *Wd, int n_experts, int n_embd, int n_ff,
                    const void *x, int x_type, const int32_t *ids, int64_t n_tokens, int k,
                    const int64_t *slots, int64_t n_slots, double *y, double *tol_y, int wtype) {
    int rc = oracle_check_args(n_tokens, k, n_experts);
    if (rc) return rc;
    if (n_embd % 32 || n_ff % 32) return OR_ERR_INVALID;
    int64_t count = slots ? n_slots : n_tokens * k;
    for (int64_t i = 0; i < count; ++i) {
        int64_t sl = slots ? slots[i] : i;
        if (ids[sl] < 0 || ids[sl] >= n_experts) return OR_ERR_BAD_ID;
    }
#pragma omp parallel
    {
        double *h = malloc((size_t)n_ff * sizeof(double)), *th = malloc((size_t)n_ff * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < count; ++i) {
            int64_t sl = slots ? slots[i] : i;
            ffn_row(Wg, Wu, Wd, wtype, ids[sl], n_embd, n_ff, x, x_type, sl / k, y + i * n_embd,
                    tol_y ? tol_y + i * n_embd : NULL, h, th);
        }
        free(h);
        free(th);
    }
    return OR_OK;
}

int oracle_shared_rows(const uint8_t *Sg, const uint8_t *Su, const uint8_t *Sd, int n_embd, int n_ff_shared,
                       const void *x, int x_type, const int64_t *tokens, int64_t n_tok, double *y, double *tol_y,
                       int wtype) {
    if (n_embd % 32 || n_ff_shared % 32) return OR_ERR_INVALID;
#pragma omp parallel
    {
        double *h = malloc((size_t)n_ff_shared * sizeof(double)), *th = malloc((size_t)n_ff_shared * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_tok; ++i)
            ffn_row(Sg, Su, Sd, wtype, 0, n_embd, n_ff_shared, x, x_type, tokens[i], y + i * n_embd,
                    tol_y ? tol_y + i * n_embd : NULL, h, th);
        free(h);
        free(th);
    }
    return OR_OK;
}

/* Hidden activations h = silu(g)*u of the listed slots (for pins on SwiGLU). */
int oracle_ffn_hidden(const uint8_t *Wg, const uint8_t *Wu, int n_experts, int n_embd, int n_ff, const void *x,
                      int x_type, const int32_t *ids, int64_t n_tokens, int k, const int64_t *slots,
                      int64_t n_slots, double *h_out, double *g_out, double *u_out, int wtype) {
    int rc = oracle_check_args(n_tokens, k, n_experts);
    if (rc) return rc;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_slots; ++i) {
        int64_t sl = slots[i], e = ids[sl], r = sl / k;
        for (int64_t f = 0; f < n_ff; ++f) {
            double g = 0, u = 0;
            for (int64_t j = 0; j < n_embd; ++j) {
                double xv = x_value(x, x_type, r * n_embd + j);
                g += w_value(Wg, wtype, n_ff, n_embd, e, f, j) * xv;
                u += w_value(Wu, wtype, n_ff, n_embd, e, f, j) * xv;
            }
            g_out[i * n_ff + f] = g;
            u_out[i * n_ff + f] = u;
            h_out[i * n_ff + f] = silu(g) * u;
        }
    }
    return OR_OK;
}

/* Dequantised weights of one expert as fp64 [n_out][n_in] (test helper). */
void oracle_dequant(const uint8_t *W, int n_out, int n_in, int e, double *out, int wtype) {
    for (int64_t n = 0; n < n_out; ++n)
        for (int64_t j = 0; j < n_in; ++j) out[n * n_in + j] = w_value(W, wtype, n_out, n_in, e, n, j);
}

/*
 * Weighted combine of a token's expert outputs ([cmoe], "Architektura Mixture
 * of Experts": the router picks k experts per token; the layer's output is
 * their outputs weighted by the router, plus the always-on shared expert of
 * [b11370]).  dst is [T][k][n] float, r is [T][k] float, dst_shared is [T][n]
 * float or NULL.  For every (t, j), in fp64 and ascending s:
 *   y[t][j]   = sum_s r[t][s] * dst[t][s][j]  (+ dst_shared[t][j])
 *   mag[t][j] = sum_s |r[t][s] * dst[t][s][j]| (+ |dst_shared[t][j]|)
 * mag is what a tolerance for a float evaluation of the same sum scales with.
 */
void oracle_combine(const float *dst, const float *r, const float *dst_shared, int64_t n_tokens, int k, int64_t n,
                    double *y, double *mag) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t) {
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0, m = 0.0;
            for (int s = 0; s < k; ++s) {
                const double term = (double)r[t * k + s] * (double)dst[(t * k + s) * n + j];
                acc += term;
                m += fabs(term);
            }
            if (dst_shared) {
                acc += (double)dst_shared[t * n + j];
                m += fabs((double)dst_shared[t * n + j]);
            }
            y[t * n + j] = acc;
            mag[t * n + j] = m;
        }
    }
}

/*
 * Router ([cmoe], "Architektura Mixture of Experts": a gating network picks k
 * of the experts for every token).  logits float [T][E]; bias float [E] or
 * NULL (a per-expert selection bias).  For every token t:
 *   key[e]  = logits[t][e] + bias[e], evaluated as one float addition - the
 *             selection is a decision on these float values, made from the
 *             same bits on both sides;
 *   ids[t]  = the k experts with the largest keys, in descending key order,
 *             equal keys taken in ascending expert index;
 *   p[e]    = exp(logits[t][e] - m) / sum_j exp(logits[t][j] - m), m = max_j
 *             logits[t][j] (softmax over all experts, fp64);
 *   w[t][i] = p[ids[t][i]], divided by sum_i p[ids[t][i]] when normalize != 0.
 * Returns 0, or -1 for k outside [1, E].
 */
int oracle_route(const float *logits, const float *bias, int64_t n_tokens, int n_experts, int k, int normalize,
                 int32_t *ids, double *w) {
    if (k < 1 || k > n_experts) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t) {
        const float *l = logits + t * n_experts;
        unsigned char *taken = (unsigned char *)calloc((size_t)n_experts, 1);
        for (int i = 0; i < k; ++i) {
            int best = -1;
            float bk = 0.0f;
            for (int e = 0; e < n_experts; ++e) {
                if (taken[e]) continue;
                const float key = bias ? l[e] + bias[e] : l[e];
                if (best < 0 || key > bk) { best = e; bk = key; }  /* ascending e keeps the lower index on ties */
            }
            taken[best] = 1;
            ids[t * k + i] = best;
        }
        free(taken);
        double m = l[0];
        for (int e = 1; e < n_experts; ++e) if (l[e] > m) m = l[e];
        double z = 0.0;
        for (int e = 0; e < n_experts; ++e) z += exp((double)l[e] - m);
        double sel = 0.0;
        for (int i = 0; i < k; ++i) {
            w[t * k + i] = exp((double)l[ids[t * k + i]] - m) / z;
            sel += w[t * k + i];
        }
        if (normalize)
            for (int i = 0; i < k; ++i) w[t * k + i] /= sel;
    }
    return 0;
}

/* Threads the parallel loops above use (timing runs report it), and a way to
 * set it to the host's cores when a launcher has capped it. */
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_num_threads(int n) { if (n > 0) omp_set_num_threads(n); }
