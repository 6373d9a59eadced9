"""moe_combine - the weighted combine y[t] = sum_s r[t][s]*dst[t][s] (+ shared[t])
that follows the indirect matmul - against the oracle element by element
within the float32 evaluation bound, on sizes that span many 256-thread
units with ragged tails, on both the vector (n % 4 == 0, 16-byte aligned) and
the scalar path, with and without the shared term; bit-identical reruns;
and host-side argument errors.  (The full V3 shape, on a real moe_ffn
output, is checked with the other full-size cases.)
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.gpu_util import check_close

pytestmark = pytest.mark.gpu


def _inputs(T, k, n, seed):
    dst = workloads.activations(T * k, n, "f32", seed, 41).reshape(T, k, n)
    r = workloads.router_weights(T, k, seed)
    sh = workloads.activations(T, n, "f32", seed, 42)
    return dst, r, sh


@pytest.mark.parametrize("T,k,n", [(37, 6, 1000), (37, 6, 1001), (5, 1, 260), (300, 8, 7168 // 8)])
@pytest.mark.parametrize("with_shared", [False, True])
def test_combine_matches_oracle(T, k, n, with_shared):
    dst, r, sh = _inputs(T, k, n, 3)
    y_ref, mag = oracle.combine(dst, r, sh if with_shared else None)
    tol = oracle.combine_tolerance(mag, k, with_shared)
    d_dst, d_r = torch.from_numpy(dst).cuda(), torch.from_numpy(r).cuda()
    d_sh = torch.from_numpy(sh).cuda() if with_shared else None
    y = moe.combine(d_dst, d_r, d_sh)
    check_close(y, y_ref, tol, f"combine T={T} k={k} n={n} shared={with_shared}")
    for _ in range(2):  # fixed order: bit-identical reruns
        assert torch.equal(moe.combine(d_dst, d_r, d_sh).view(torch.int32), y.view(torch.int32))


def test_combine_unaligned_pointers_take_the_scalar_path():
    T, k, n = 9, 3, 64
    dst, r, sh = _inputs(T, k, n, 5)
    y_ref, mag = oracle.combine(dst, r, sh)
    tol = oracle.combine_tolerance(mag, k, True)
    # views one float past 16-byte boundaries
    big = torch.zeros(T * k * n + 1, dtype=torch.float32, device="cuda")
    big[1:] = torch.from_numpy(dst.reshape(-1)).cuda()
    shb = torch.zeros(T * n + 1, dtype=torch.float32, device="cuda")
    shb[1:] = torch.from_numpy(sh.reshape(-1)).cuda()
    out = torch.zeros(T * n + 1, dtype=torch.float32, device="cuda")
    moe.combine(big[1:].view(T, k, n), torch.from_numpy(r).cuda(), shb[1:].view(T, n), out=out[1:].view(T, n))
    check_close(out[1:].view(T, n), y_ref, tol, "combine, unaligned")
    assert out[0].item() == 0.0  # nothing written before the output


def test_combine_in_place_into_the_shared_output():
    T, k, n = 11, 4, 128
    dst, r, sh = _inputs(T, k, n, 6)
    y_ref, mag = oracle.combine(dst, r, sh)
    d_sh = torch.from_numpy(sh).cuda()
    moe.combine(torch.from_numpy(dst).cuda(), torch.from_numpy(r).cuda(), d_sh, out=d_sh)
    check_close(d_sh, y_ref, oracle.combine_tolerance(mag, k, True), "combine into dst_shared")


def test_combine_edge_cases_and_errors():
    d = torch.zeros((0, 2, 8), dtype=torch.float32, device="cuda")
    assert moe.combine(d, torch.zeros((0, 2), dtype=torch.float32, device="cuda")).shape == (0, 8)
    L = moe.lib()
    y = torch.empty(8, dtype=torch.float32, device="cuda")
    x = torch.ones(8, dtype=torch.float32, device="cuda")
    assert L.moe_combine(x.data_ptr(), x.data_ptr(), None, 1, 0, 8, y.data_ptr(), None) == moe.ERR_INVALID
    assert L.moe_combine(x.data_ptr(), x.data_ptr(), None, 1, 1, 0, y.data_ptr(), None) == moe.ERR_INVALID
    assert L.moe_combine(None, x.data_ptr(), None, 1, 1, 8, y.data_ptr(), None) == moe.ERR_INVALID
    assert L.moe_combine(x.data_ptr(), x.data_ptr(), None, 1 << 22, 1, 8, y.data_ptr(), None) == moe.ERR_RANGE
    assert L.moe_combine(x.data_ptr(), x.data_ptr(), None, 1, 1024, 8, y.data_ptr(), None) == moe.ERR_RANGE
    assert L.moe_combine(x.data_ptr() + 2, x.data_ptr(), None, 1, 1, 4, y.data_ptr(), None) == moe.ERR_INVALID
