"""Pins of the CPU oracle to facts other than itself (no GPU).

Each check ties the oracle to something independent: a hand-worked example,
invariants of a stable counting sort, brute force over every tiny input,
dense special cases checked with numpy's float64 matmul, symmetries that must
hold exactly, and SwiGLU special values.  A dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
import workloads
from tests.fixtures import GOLDEN, hand_example, pack_q8_0, unpack_q8_0


def rand_q8(rng, E, n_out, n_in):
    q = rng.integers(-127, 128, size=(E, n_out, n_in), dtype=np.int64).astype(np.int8)
    d = rng.uniform(0.001, 0.01, size=(E, n_out, n_in // 32))
    return pack_q8_0(d, q)


def rand_ids_distinct(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32).reshape(T, k)


# ------------------------------------------------------------- hand example
@pytest.mark.parametrize("grouped", [False, True])
def test_hand_example_broadcast(grouped):
    g, W, xb, xs, ids = hand_example()
    dst, tol = oracle.mul_mat_id(W, xb, "f32", ids, "broadcast", grouped=grouped)
    assert np.array_equal(dst, np.array(g["dst_broadcast"], np.float64))
    assert np.all(tol > 0)


@pytest.mark.parametrize("grouped", [False, True])
def test_hand_example_per_slot(grouped):
    g, W, xb, xs, ids = hand_example()
    dst, _ = oracle.mul_mat_id(W, xs, "f32", ids, "per_slot", grouped=grouped)
    assert np.array_equal(dst, np.array(g["dst_per_slot"], np.float64))


def test_hand_example_tables():
    g, W, xb, xs, ids = hand_example()
    s1, dr, b = oracle.row_ids(ids, 2, "broadcast")
    assert b.tolist() == g["expert_bounds"]
    assert dr.tolist() == g["ids_dst"]
    assert s1.tolist() == g["ids_src1_broadcast"]
    s1, dr, b = oracle.row_ids(ids, 2, "per_slot")
    assert s1.tolist() == g["ids_src1_per_slot"]


# --------------------------------------------------------- row-id invariants
def check_invariants(ids, E, mode, src1, dst, bounds):
    T, k = ids.shape
    S = T * k
    flat = ids.reshape(-1)
    assert bounds[0] == 0 and bounds[E] == S
    assert np.all(np.diff(bounds) >= 0)
    assert np.array_equal(np.diff(bounds), np.bincount(flat, minlength=E)[:E])
    assert np.array_equal(np.sort(dst), np.arange(S))
    for e in range(E):
        seg = dst[bounds[e]:bounds[e + 1]]
        assert np.all(np.diff(seg) > 0)            # stable: ascending (t, s)
        assert np.all(flat[seg] == e)
    if mode == "per_slot":
        assert np.array_equal(src1, dst)
    else:
        assert np.array_equal(src1, dst // k)


@pytest.mark.parametrize("seed", range(12))
def test_row_ids_invariants_fuzz(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 300))
    k = int(rng.integers(1, min(E, 33) + 1))
    T = int(rng.integers(0, 700))
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)  # duplicates allowed
    for mode in ("broadcast", "per_slot"):
        src1, dst, bounds = oracle.row_ids(ids, E, mode)
        check_invariants(ids, E, mode, src1, dst, bounds)


def test_row_ids_brute_force_all_tiny():
    """Every id matrix with E <= 3, k <= 2, T <= 4 against numpy's stable sort."""
    for E in (1, 2, 3):
        for k in (1, 2):
            if k > E:
                continue
            for T in range(0, 5):
                for flat in itertools.product(range(E), repeat=T * k):
                    ids = np.array(flat, np.int32).reshape(T, k)
                    src1, dst, bounds = oracle.row_ids(ids, E, "broadcast")
                    order = np.argsort(ids.reshape(-1), kind="stable")
                    assert np.array_equal(dst, order)
                    assert np.array_equal(src1, order // k)
                    assert np.array_equal(bounds, np.searchsorted(np.sort(ids.reshape(-1)), np.arange(E + 1)))


def test_row_ids_limits():
    assert oracle.check_args((1 << 22) - 1, 1, 1) == oracle.OK
    assert oracle.check_args(1 << 22, 1, 1) == oracle.ERR_RANGE
    assert oracle.check_args(1, 1023, 1023) == oracle.OK
    assert oracle.check_args(1, 1024, 2000) == oracle.ERR_RANGE
    assert oracle.check_args(4, 3, 2) == oracle.ERR_RANGE
    assert oracle.check_args(4, 0, 2) == oracle.ERR_INVALID
    assert oracle.check_args((1 << 22) - 1, 1000, 1000) == oracle.ERR_RANGE  # T*k >= 2^31
    with pytest.raises(oracle.OracleError) as ei:
        oracle.row_ids(np.array([[0, 5]], np.int32), 3)
    assert ei.value.code == oracle.ERR_BAD_ID
    with pytest.raises(oracle.OracleError) as ei:
        oracle.row_ids(np.array([[-1]], np.int32), 3)
    assert ei.value.code == oracle.ERR_BAD_ID


# ----------------------------------------------------- grouped == brute force
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
@pytest.mark.parametrize("x_type", ["f32", "bf16"])
def test_grouped_equals_brute(mode, x_type):
    rng = np.random.default_rng(7)
    E, k, T, n_in, n_out = 5, 3, 23, 64, 48
    W = rand_q8(rng, E, n_out, n_in)
    ids = rand_ids_distinct(rng, T, E, k)
    rows = T if mode == "broadcast" else T * k
    x = workloads.activations(rows, n_in, x_type, seed=3, tensor=9)
    a, ta = oracle.mul_mat_id(W, x, x_type, ids, mode, grouped=False)
    b, tb = oracle.mul_mat_id(W, x, x_type, ids, mode, grouped=True)
    assert np.array_equal(a, b) and np.array_equal(ta, tb)
    slots = np.array([0, 5, T * k - 1])
    r, tr = oracle.mul_mat_id_rows(W, x, x_type, ids, slots, mode)
    assert np.array_equal(r, a.reshape(T * k, n_out)[slots])


# ---------------------------------------------------------- dense reductions
def test_single_expert_is_plain_gemm():
    rng = np.random.default_rng(11)
    n_in, n_out, T = 96, 40, 17
    W = rand_q8(rng, 1, n_out, n_in)
    x = rng.standard_normal((T, n_in)).astype(np.float32)
    ids = np.zeros((T, 1), np.int32)
    dst, tol = oracle.mul_mat_id(W, x, "f32", ids)
    w = unpack_q8_0(W)[0]                              # numpy's own decode
    ref = x.astype(np.float64) @ w.T                   # float64 library matmul
    assert np.allclose(dst[:, 0, :], ref, rtol=1e-12, atol=1e-12)
    mag = np.abs(x.astype(np.float64)) @ np.abs(w).T
    assert np.allclose(tol[:, 0, :], 2e-3 * mag + 1e-5, rtol=1e-12)


def test_oracle_dequant_matches_numpy_decode():
    rng = np.random.default_rng(2)
    W = rand_q8(rng, 3, 5, 64)
    for e in range(3):
        assert np.array_equal(oracle.dequant(W, e), unpack_q8_0(W)[e])


def test_all_ids_equal_is_dense_gemm_of_that_expert():
    rng = np.random.default_rng(12)
    E, n_in, n_out, T, k = 4, 64, 24, 9, 1
    W = rand_q8(rng, E, n_out, n_in)
    x = rng.standard_normal((T, n_in)).astype(np.float32)
    ids = np.full((T, k), 2, np.int32)
    dst, _ = oracle.mul_mat_id(W, x, "f32", ids)
    ref = x.astype(np.float64) @ unpack_q8_0(W)[2].T
    assert np.allclose(dst[:, 0], ref, rtol=1e-12, atol=1e-12)


def test_identical_experts_make_ids_irrelevant():
    rng = np.random.default_rng(13)
    n_in, n_out, T, k = 64, 16, 11, 3
    W1 = rand_q8(rng, 1, n_out, n_in)
    W = np.repeat(W1, 5, axis=0)
    x = rng.standard_normal((T, n_in)).astype(np.float32)
    a, _ = oracle.mul_mat_id(W, x, "f32", rand_ids_distinct(rng, T, 5, k))
    b, _ = oracle.mul_mat_id(W, x, "f32", rand_ids_distinct(rng, T, 5, k))
    assert np.array_equal(a, b)


def test_relabelling_experts_is_exact():
    rng = np.random.default_rng(14)
    E, n_in, n_out, T, k = 6, 64, 16, 10, 2
    W = rand_q8(rng, E, n_out, n_in)
    x = rng.standard_normal((T, n_in)).astype(np.float32)
    ids = rand_ids_distinct(rng, T, E, k)
    perm = rng.permutation(E)           # expert e becomes perm[e]
    Wp = np.empty_like(W)
    Wp[perm] = W
    a, _ = oracle.mul_mat_id(W, x, "f32", ids)
    b, _ = oracle.mul_mat_id(Wp, x, "f32", perm[ids].astype(np.int32))
    assert np.array_equal(a, b)


def test_transposed_operand_would_fail():
    """n_out != n_in and a non-symmetric W: out[n] must use row n of W."""
    rng = np.random.default_rng(15)
    W = rand_q8(rng, 1, 32, 64)
    x = np.zeros((1, 64), np.float32)
    x[0, 5] = 1.0
    dst, _ = oracle.mul_mat_id(W, x, "f32", np.zeros((1, 1), np.int32))
    assert np.array_equal(dst[0, 0], unpack_q8_0(W)[0][:, 5])


# ------------------------------------------------------------------- FFN
def silu(z):
    return z / (1.0 + np.exp(-z))


def test_ffn_single_expert_matches_numpy():
    rng = np.random.default_rng(21)
    n_embd, n_ff, T = 64, 96, 7
    Wg, Wu, Wd = rand_q8(rng, 1, n_ff, n_embd), rand_q8(rng, 1, n_ff, n_embd), rand_q8(rng, 1, n_embd, n_ff)
    x = rng.standard_normal((T, n_embd)).astype(np.float32)
    ids = np.zeros((T, 1), np.int32)
    y, tol = oracle.ffn(Wg, Wu, Wd, x, "f32", ids)
    xg = x.astype(np.float64)
    h = silu(xg @ unpack_q8_0(Wg)[0].T) * (xg @ unpack_q8_0(Wu)[0].T)
    ref = h @ unpack_q8_0(Wd)[0].T
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-9)
    assert np.all(tol > 2e-3 * (np.abs(h) @ np.abs(unpack_q8_0(Wd)[0]).T))


def test_ffn_routed_matches_composition_of_mul_mat_id():
    """FFN = down(per_slot) o SwiGLU o gate/up(broadcast), composed from the
    oracle's mul_mat_id and numpy's SwiGLU."""
    rng = np.random.default_rng(22)
    E, k, T, n_embd, n_ff = 4, 2, 6, 64, 64
    Wg, Wu, Wd = rand_q8(rng, E, n_ff, n_embd), rand_q8(rng, E, n_ff, n_embd), rand_q8(rng, E, n_embd, n_ff)
    x = rng.standard_normal((T, n_embd)).astype(np.float32)
    ids = rand_ids_distinct(rng, T, E, k)
    y, _ = oracle.ffn(Wg, Wu, Wd, x, "f32", ids)
    g, _ = oracle.mul_mat_id(Wg, x, "f32", ids, "broadcast")
    u, _ = oracle.mul_mat_id(Wu, x, "f32", ids, "broadcast")
    h = (silu(g) * u).reshape(T * k, n_ff)
    wd = unpack_q8_0(Wd)
    ref = np.stack([wd[ids.reshape(-1)[i]] @ h[i] for i in range(T * k)])
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-9)


def test_swiglu_special_values():
    rng = np.random.default_rng(23)
    n_embd, n_ff = 32, 32
    zero_gate = pack_q8_0(np.full((1, n_ff, 1), 0.01), np.zeros((1, n_ff, n_embd), np.int8))
    Wu = rand_q8(rng, 1, n_ff, n_embd)
    Wd = rand_q8(rng, 1, n_embd, n_ff)
    x = rng.standard_normal((3, n_embd)).astype(np.float32)
    ids = np.zeros((3, 1), np.int32)
    y, _ = oracle.ffn(zero_gate, Wu, Wd, x, "f32", ids)
    assert np.all(y == 0.0)                        # silu(0) = 0
    # large gate: silu(g) -> g (relative gap e^-g)
    big_gate = pack_q8_0(np.full((1, n_ff, 1), 2.0), np.full((1, n_ff, n_embd), 100, np.int8))
    xo = np.ones((1, n_embd), np.float32)
    h, g, u = oracle.ffn_hidden(big_gate, Wu, xo, "f32", np.zeros((1, 1), np.int32), np.array([0]))
    assert np.all(g == 6400.0)
    assert np.array_equal(h, g * u)
    # negative gate: silu(-40) ~ -40 e^-40 ~ 0
    neg_gate = pack_q8_0(np.full((1, n_ff, 1), 2.0 ** -6), np.full((1, n_ff, n_embd), -80, np.int8))
    h, g, u = oracle.ffn_hidden(neg_gate, Wu, xo, "f32", np.zeros((1, 1), np.int32), np.array([0]))
    assert np.all(g == -40.0)
    assert np.all(np.abs(h) <= np.abs(u) * 40 * np.exp(-40) * 1.0000001)


def test_shared_expert_equals_single_expert_routed_ffn():
    rng = np.random.default_rng(24)
    n_embd, n_ff, T = 64, 64, 5
    Sg, Su, Sd = rand_q8(rng, 1, n_ff, n_embd), rand_q8(rng, 1, n_ff, n_embd), rand_q8(rng, 1, n_embd, n_ff)
    x = workloads.activations(T, n_embd, "bf16", seed=1, tensor=5)
    a, ta = oracle.shared_ffn(Sg, Su, Sd, x, "bf16")
    b, tb = oracle.ffn(Sg, Su, Sd, x, "bf16", np.zeros((T, 1), np.int32))
    assert np.array_equal(a, b) and np.array_equal(ta, tb)


def test_ffn_tolerance_covers_bf16_h_rounding():
    """Rounding h to bfloat16 before the down projection stays inside tol."""
    rng = np.random.default_rng(25)
    E, k, T, n_embd, n_ff = 3, 2, 8, 64, 64
    Wg, Wu, Wd = rand_q8(rng, E, n_ff, n_embd), rand_q8(rng, E, n_ff, n_embd), rand_q8(rng, E, n_embd, n_ff)
    x = rng.standard_normal((T, n_embd)).astype(np.float32)
    ids = rand_ids_distinct(rng, T, E, k)
    y, tol = oracle.ffn(Wg, Wu, Wd, x, "f32", ids)
    h, _, _ = oracle.ffn_hidden(Wg, Wu, x, "f32", ids, np.arange(T * k))
    from tests.fixtures import bf16_bits_to_f64, f32_to_bf16_bits
    hb = bf16_bits_to_f64(f32_to_bf16_bits(h.astype(np.float32)))
    wd = unpack_q8_0(Wd)
    yb = np.stack([wd[ids.reshape(-1)[i]] @ hb[i] for i in range(T * k)])
    assert np.all(np.abs(yb - y) <= tol)


# ------------------------------------------------------- input generator
def test_workload_inputs_are_deterministic_and_shardable():
    wl = workloads.WORKLOADS["v3"]
    a = wl.ids(64)
    b = np.concatenate([wl.ids(32, t0=0), wl.ids(32, t0=32)])
    assert np.array_equal(a, b)
    for row in a:
        assert len(set(row.tolist())) == wl.k
    xa = wl.x(8)
    xb = np.concatenate([wl.x(4), wl.x(4, t0=4)])
    assert np.array_equal(xa, xb)
    sk = workloads.WORKLOADS["skew"]
    c = np.bincount(sk.ids(2048).reshape(-1), minlength=sk.n_experts)
    assert (c == 0).sum() >= sk.n_zero


# ----------------------------------------------------------- weighted combine
def _combine_inputs(T, k, n, seed):
    rng = np.random.default_rng(seed)
    dst = rng.normal(size=(T, k, n)).astype(np.float32)
    r = rng.uniform(0.05, 1.0, size=(T, k)).astype(np.float32)
    sh = rng.normal(size=(T, n)).astype(np.float32)
    return dst, r, sh


def test_combine_one_hot_weights_select_a_slot():
    # r = e_s picks slot s exactly; plus the shared term exactly (one fp64 add of two floats)
    dst, _, sh = _combine_inputs(5, 4, 33, 1)
    for s in range(4):
        r = np.zeros((5, 4), np.float32)
        r[:, s] = 1.0
        y, _ = oracle.combine(dst, r)
        assert np.array_equal(y, dst[:, s, :].astype(np.float64))
        y, _ = oracle.combine(dst, r, sh)
        assert np.array_equal(y, dst[:, s, :].astype(np.float64) + sh.astype(np.float64))


def test_combine_matches_numpy_einsum_and_is_linear():
    dst, r, sh = _combine_inputs(7, 6, 40, 2)
    y, mag = oracle.combine(dst, r, sh)
    ref = np.einsum("tk,tkn->tn", r.astype(np.float64), dst.astype(np.float64)) + sh.astype(np.float64)
    assert np.allclose(y, ref, rtol=0, atol=1e-12)
    ref_mag = np.einsum("tk,tkn->tn", np.abs(r.astype(np.float64)), np.abs(dst.astype(np.float64))) + np.abs(sh)
    assert np.allclose(mag, ref_mag, rtol=1e-14, atol=0)
    y2, _ = oracle.combine(dst, 2 * r, 2 * sh)  # scaling by 2 is exact in float
    assert np.array_equal(y2, 2 * y)


def test_combine_slot_order_and_tokens_are_not_mixed():
    # permuting the slots of one token together with their weights leaves y unchanged
    # up to fp64 reordering; token rows stay separate
    dst, r, _ = _combine_inputs(4, 5, 16, 3)
    perm = np.array([3, 0, 4, 1, 2])
    y, _ = oracle.combine(dst, r)
    yp, _ = oracle.combine(dst[:, perm, :], r[:, perm])
    assert np.allclose(y, yp, rtol=0, atol=1e-12)
    dst2 = dst.copy()
    dst2[1] += 1.0  # touching token 1 changes only row 1, by about sum_s r[1][s]
    y2, _ = oracle.combine(dst2, r)
    assert np.array_equal(np.delete(y2, 1, axis=0), np.delete(y, 1, axis=0))
    assert np.allclose(y2[1] - y[1], r[1].astype(np.float64).sum(), rtol=0, atol=1e-6)


def test_combine_edge_cases_and_tolerance():
    dst, r, sh = _combine_inputs(3, 1, 8, 4)
    y, mag = oracle.combine(dst, r)  # k = 1: one product, exact in fp64
    assert np.array_equal(y, r.astype(np.float64) * dst[:, 0, :].astype(np.float64))
    y0, _ = oracle.combine(np.zeros((0, 2, 8), np.float32), np.zeros((0, 2), np.float32))
    assert y0.shape == (0, 8)
    # the tolerance covers a float32 evaluation in the library's order
    dst, r, sh = _combine_inputs(6, 8, 64, 5)
    y, mag = oracle.combine(dst, r, sh)
    acc = np.zeros((6, 64), np.float32)
    for s in range(8):  # float32 multiply-add per slot (product exact in float64, one rounding)
        acc = (acc.astype(np.float64) + r[:, s:s + 1].astype(np.float64) * dst[:, s, :]).astype(np.float32)
    acc = (acc + sh).astype(np.float32)
    tol = oracle.combine_tolerance(mag, 8, True)
    assert np.all(np.abs(acc - y) <= tol)


def test_router_weights_are_seeded_and_normalised():
    a = workloads.router_weights(9, 8, 0)
    b = workloads.router_weights(9, 8, 0)
    assert np.array_equal(a, b) and a.dtype == np.float32
    assert np.allclose(a.sum(axis=1), 1.0, atol=1e-6) and np.all(a > 0)
    # rows are independent of how many tokens are generated (counter-based)
    assert np.array_equal(workloads.router_weights(4, 8, 0, t0=5), a[5:9])


# ------------------------------------------------------------------- router
def _np_route(logits, k, bias=None, normalize=True):
    # independent restatement with numpy: float32 keys, a stable sort, float64 softmax
    key = logits if bias is None else (logits + bias[None, :]).astype(np.float32)
    T, E = logits.shape
    order = np.array([np.lexsort((np.arange(E), -key[t].astype(np.float64)))[:k] for t in range(T)], np.int32)
    l64 = logits.astype(np.float64)
    p = np.exp(l64 - l64.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    w = np.take_along_axis(p, order, axis=1)
    if normalize:
        w = w / w.sum(axis=1, keepdims=True)
    return order, w


@pytest.mark.parametrize("normalize", [True, False])
@pytest.mark.parametrize("with_bias", [False, True])
def test_route_matches_numpy(normalize, with_bias):
    rng = np.random.default_rng(11)
    logits = rng.normal(size=(50, 40)).astype(np.float32)
    bias = rng.normal(scale=0.5, size=40).astype(np.float32) if with_bias else None
    ids, w, tol = oracle.route(logits, 6, bias, normalize)
    ref_ids, ref_w = _np_route(logits, 6, bias, normalize)
    assert np.array_equal(ids, ref_ids)
    assert np.allclose(w, ref_w, rtol=1e-13, atol=0)


def test_route_ties_bias_and_full_k():
    logits = np.zeros((3, 10), np.float32)
    ids, w, _ = oracle.route(logits, 4, normalize=False)
    assert np.array_equal(ids, np.tile(np.arange(4, dtype=np.int32), (3, 1)))  # equal keys: lower index first
    assert np.allclose(w, 0.1, rtol=1e-15)
    _, wn, _ = oracle.route(logits, 4)
    assert np.allclose(wn, 0.25, rtol=1e-15)
    # the bias moves the choice, not the probabilities
    bias = np.zeros(10, np.float32)
    bias[7] = 1.0
    ids_b, w_b, _ = oracle.route(logits, 2, bias, normalize=False)
    assert list(ids_b[0]) == [7, 0] and np.allclose(w_b, 0.1, rtol=1e-15)
    # k = E: every expert, probabilities summing to one
    rng = np.random.default_rng(3)
    l = rng.normal(size=(5, 12)).astype(np.float32)
    ids_f, w_f, _ = oracle.route(l, 12, normalize=False)
    assert all(sorted(r) == list(range(12)) for r in ids_f)
    assert np.allclose(w_f.sum(axis=1), 1.0, atol=1e-14)
    with pytest.raises(ValueError):
        oracle.route(l, 13)


def _wide_span_logits():
    # a row spanning ~200: the top expert far above the rest, and a bias that
    # makes the chosen experts ones whose probabilities are about e^-190 - far
    # below float32's smallest value, but not float64's
    logits = np.zeros((4, 16), np.float32)
    logits[:, 0] = 100.0
    logits[:, 1:] = np.linspace(-100.0, -90.0, 15, dtype=np.float32)[None, :] + np.arange(4, dtype=np.float32)[:, None]
    bias = np.zeros(16, np.float32)
    bias[0] = -1000.0  # expert 0 never chosen
    return logits, bias


def test_route_renormalised_weights_are_the_softmax_over_the_chosen_logits():
    # renormalising the chosen probabilities is the softmax over the chosen
    # logits alone (the common factor exp(-max) / sum cancels): checked against
    # that closed form, on a row whose chosen probabilities underflow in float32
    logits, bias = _wide_span_logits()
    ids, w, tol = oracle.route(logits, 4, bias)
    chosen = np.take_along_axis(logits.astype(np.float64), ids, axis=1)
    e = np.exp(chosen - chosen.max(axis=1, keepdims=True))
    assert np.all(ids != 0)
    assert np.allclose(w, e / e.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-15) and np.all(np.isfinite(tol))
    p32 = np.exp((chosen - 100.0).astype(np.float32))  # what a float32 softmax over all experts gives
    assert np.all(p32 == 0.0)


def test_route_tolerance_covers_a_float32_softmax():
    rng = np.random.default_rng(5)
    logits = (rng.normal(size=(40, 64)) * 3).astype(np.float32)
    ids, w, tol = oracle.route(logits, 8)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp((logits - m).astype(np.float32)).astype(np.float32)
    z = np.zeros((40, 1), np.float32)
    for j in range(64):  # float32 sum, one rounding per addition
        z = (z + e[:, j:j + 1]).astype(np.float32)
    p = (e / z).astype(np.float32)
    sel = np.take_along_axis(p, ids, axis=1)
    s = np.zeros((40, 1), np.float32)
    for i in range(8):
        s = (s + sel[:, i:i + 1]).astype(np.float32)
    w32 = (sel / s).astype(np.float32)
    assert np.all(np.abs(w32 - w) <= tol)


def test_float32_bounds_are_tight_enough_to_mean_something():
    # the combine and router bounds stay within a few hundred float32 units, so a
    # dropped term or a wrong weight (errors of order the values) cannot hide in them
    rng = np.random.default_rng(8)
    dst = rng.normal(size=(4, 8, 32)).astype(np.float32)
    r = rng.uniform(0.05, 1.0, size=(4, 8)).astype(np.float32)
    y, mag = oracle.combine(dst, r)
    tol = oracle.combine_tolerance(mag, 8, False)
    assert np.all(tol <= 1e-5 * mag + 1e-30)
    y_drop, _ = oracle.combine(dst[:, :7, :], r[:, :7])  # one slot missing
    assert np.any(np.abs(y_drop - y) > tol)
    logits = rng.normal(size=(6, 256)).astype(np.float32)
    ids, w, tol_w = oracle.route(logits, 8)
    assert np.all(tol_w <= 1e-4 * w)
    _, w_un, _ = oracle.route(logits, 8, normalize=False)  # forgetting the renormalisation
    assert np.all(np.abs(w_un - w) > tol_w)


# ------------------------------------------------------------------- MXFP4
def _golden_mxfp4():
    with open(os.path.join(GOLDEN, "mxfp4_blocks.json")) as f:
        return json.load(f)["blocks"]


def _np_decode_mxfp4(W):
    # independent restatement: the E2M1 magnitude table as the OCP MX
    # specification lists it, sign from bit 3, nibbles split low/high
    mag = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    X = W[..., 0].astype(np.int64)
    codes = np.concatenate([W[..., 1:] & 15, W[..., 1:] >> 4], axis=-1).astype(np.int64)
    v = np.where(codes & 8, -1.0, 1.0) * mag[codes & 7]
    scale = np.where(X == 255, np.nan, np.ldexp(1.0, X - 127))
    out = v * scale[..., None]
    return out.reshape(W.shape[:-2] + (W.shape[-2] * 32,))


def test_mxfp4_hand_worked_blocks():
    for blk in _golden_mxfp4():
        W = np.array(blk["bytes"], np.uint8).reshape(1, 1, 1, 17)
        got = oracle.dequant(W, 0)[0]
        if blk.get("nan"):
            assert np.isnan(got).all()
            continue
        if "values" in blk:
            want = np.array(blk["values"], np.float64)
        elif "values_pow2" in blk:
            m, e = blk["values_pow2"][0]
            want = np.full(32, np.ldexp(float(m), e))
        elif "values_pow2_halves" in blk:
            (m0, e0), (m1, e1) = blk["values_pow2_halves"]
            want = np.concatenate([np.full(16, np.ldexp(float(m0), e0)), np.full(16, np.ldexp(float(m1), e1))])
        else:
            a, b = blk["values_halves"]
            want = np.concatenate([np.full(16, float(a)), np.full(16, float(b))])
        assert np.array_equal(got, want), blk["note"]
        assert np.array_equal(np.signbit(got), np.signbit(want)), blk["note"]  # -0 stays -0


def test_mxfp4_decoder_matches_numpy_on_random_blocks():
    W = workloads.mxfp4_weights(3, 24, 96, 5, 9)
    for e in range(3):
        assert np.array_equal(oracle.dequant(W, e), _np_decode_mxfp4(W)[e])
    # the generator's scales put the weights in a plausible range, every code occurs
    w = _np_decode_mxfp4(W)
    assert 0.7 < np.abs(w).max() <= 6 * 2.0 ** -3 and np.unique(np.concatenate([W[..., 1:] & 15, W[..., 1:] >> 4])).size == 16


def test_mxfp4_mul_mat_id_is_a_dense_gemm_for_one_expert():
    W = workloads.mxfp4_weights(1, 40, 128, 6, 1)
    x = workloads.activations(7, 128, "f32", 6, 2)
    ids = np.zeros((7, 1), np.int32)
    dst, tol = oracle.mul_mat_id(W, x, "f32", ids)
    want = x.astype(np.float64) @ _np_decode_mxfp4(W)[0].T
    assert np.allclose(dst[:, 0, :], want, rtol=1e-13, atol=1e-13)
    assert np.all(tol > 1e-5)


def test_mxfp4_grouped_equals_brute_and_ffn_matches_numpy():
    E, k, T, n_embd, n_ff = 6, 2, 9, 64, 96
    ids = workloads.routing("uniform", T, E, k, 4)
    W = workloads.mxfp4_weights(E, n_ff, n_embd, 4, 3)
    x = workloads.activations(T, n_embd, "bf16", 4, 5)
    a, _ = oracle.mul_mat_id(W, x, "bf16", ids)
    b, _ = oracle.mul_mat_id(W, x, "bf16", ids, grouped=True)
    assert np.array_equal(a, b)
    Wg, Wu = W, workloads.mxfp4_weights(E, n_ff, n_embd, 4, 6)
    Wd = workloads.mxfp4_weights(E, n_embd, n_ff, 4, 7)
    y, _ = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    dg, du, dd = _np_decode_mxfp4(Wg), _np_decode_mxfp4(Wu), _np_decode_mxfp4(Wd)
    for i in range(T * k):
        t, e = i // k, ids.reshape(-1)[i]
        g, u = dg[e] @ xf[t], du[e] @ xf[t]
        h = g / (1.0 + np.exp(-g)) * u
        assert np.allclose(y[i], dd[e] @ h, rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.ffn(Wg, workloads.q8_0_weights(E, n_ff, n_embd, 4, 6), Wd, x, "bf16", ids)
