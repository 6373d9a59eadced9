"""moe_route - the router before the indirect matmul: the k largest
logit + bias per token (descending, ties to the lower expert) and their
softmax weights - against the oracle: ids bit-exact (a decision on the same
float32 keys on both sides), weights within the float32 bound; expert counts
that are not multiples of 32, the largest supported count, k = n_experts,
exact ties, the V3 routing shape with a bias; bit-identical reruns; host-side
argument errors; and the router's output driving moe_ffn and moe_combine.
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.gpu_util import check_close, prep, to_dev_x

pytestmark = pytest.mark.gpu


def _logits(T, E, seed, scale=1.0):
    return (workloads.activations(T, E, "f32", seed, 51) * scale).astype(np.float32)


@pytest.mark.parametrize("T,E,k", [(37, 200, 6), (8, 1024, 8), (9, 300, 5), (11, 96, 4), (5, 40, 40), (4096, 256, 8),
                                   (3, 7, 1)])
@pytest.mark.parametrize("normalize", [True, False])
def test_route_matches_oracle(T, E, k, normalize):
    logits = _logits(T, E, T + E, 2.0)
    bias = (workloads.activations(1, E, "f32", E, 52)[0] * 0.5).astype(np.float32) if E == 256 else None
    ref_ids, ref_w, tol = oracle.route(logits, k, bias, normalize)
    d_l = torch.from_numpy(logits).cuda()
    d_b = torch.from_numpy(bias).cuda() if bias is not None else None
    ids, w = moe.route(d_l, k, d_b, normalize)
    assert np.array_equal(ids.cpu().numpy(), ref_ids), "router ids differ from the oracle"
    check_close(w, ref_w, tol, f"router weights T={T} E={E} k={k}")
    ids2, w2 = moe.route(d_l, k, d_b, normalize)
    assert torch.equal(ids2, ids) and torch.equal(w2.view(torch.int32), w.view(torch.int32))


def test_route_renormalised_weights_stay_finite_when_probabilities_underflow():
    # chosen logits ~190 below the row's top: their float32 probabilities are 0,
    # yet the renormalised weights (the softmax over the chosen logits) are finite,
    # sum to one and match the oracle within the float32 bound
    from tests.test_oracle_pins import _wide_span_logits
    logits, bias = _wide_span_logits()
    ref_ids, ref_w, tol = oracle.route(logits, 4, bias)
    ids, w = moe.route(torch.from_numpy(logits).cuda(), 4, torch.from_numpy(bias).cuda())
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert torch.isfinite(w).all()
    check_close(w, ref_w, tol, "router weights, span 200")
    assert np.allclose(w.cpu().numpy().sum(axis=1), 1.0, atol=1e-6)


def test_route_exact_ties_take_the_lower_expert():
    logits = np.zeros((6, 96), np.float32)
    logits[:, 50] = 1.0
    ids, w = moe.route(torch.from_numpy(logits).cuda(), 5, normalize=False)
    assert np.array_equal(ids.cpu().numpy(), np.tile(np.array([50, 0, 1, 2, 3], np.int32), (6, 1)))
    ref_ids, ref_w, tol = oracle.route(logits, 5, normalize=False)
    check_close(w, ref_w, tol, "router ties")


def test_route_errors_and_empty():
    L = moe.lib()
    x = torch.zeros(64, dtype=torch.float32, device="cuda")
    i = torch.zeros(64, dtype=torch.int32, device="cuda")
    p = x.data_ptr
    assert L.moe_route(p(), None, 1, 8, 0, 1, i.data_ptr(), p(), None) == moe.ERR_INVALID
    assert L.moe_route(p(), None, 1, 8, 9, 1, i.data_ptr(), p(), None) == moe.ERR_INVALID
    assert L.moe_route(None, None, 1, 8, 2, 1, i.data_ptr(), p(), None) == moe.ERR_INVALID
    assert L.moe_route(p(), None, 1, 1025, 2, 1, i.data_ptr(), p(), None) == moe.ERR_RANGE
    assert L.moe_route(p(), None, 1 << 22, 8, 2, 1, i.data_ptr(), p(), None) == moe.ERR_RANGE
    assert L.moe_route(p() + 2, None, 1, 8, 2, 1, i.data_ptr(), p(), None) == moe.ERR_INVALID
    ids, w = moe.route(torch.zeros((0, 16), dtype=torch.float32, device="cuda"), 4)
    assert ids.shape == (0, 4) and w.shape == (0, 4)


def test_route_drives_ffn_and_combine():
    # the layer as the pages describe it: router -> expert FFN -> weighted combine
    E, k, T, n_embd, n_ff = 16, 4, 24, 256, 128
    logits = _logits(T, E, 9)
    ids, r = moe.route(torch.from_numpy(logits).cuda(), k)
    ref_ids, ref_r, tol_r = oracle.route(logits, k)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    Wg = workloads.q8_0_weights(E, n_ff, n_embd, 9, workloads.T_WG)
    Wu = workloads.q8_0_weights(E, n_ff, n_embd, 9, workloads.T_WU)
    Wd = workloads.q8_0_weights(E, n_embd, n_ff, 9, workloads.T_WD)
    x = workloads.activations(T, n_embd, "bf16", 9, workloads.T_X)
    dst, _ = moe.ffn(prep(Wg), prep(Wu), prep(Wd), E, n_embd, n_ff, to_dev_x(x, "bf16"), ids)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ref_ids)
    check_close(dst.reshape(T * k, n_embd), ref, tol, "ffn on routed ids")
    y = moe.combine(dst, r)
    y_ref, mag = oracle.combine(dst.cpu().numpy(), r.cpu().numpy())
    check_close(y, y_ref, oracle.combine_tolerance(mag, k, False), "combine of routed outputs")
