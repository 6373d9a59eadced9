"""MXFP4 expert weights (32 E2M1 codes sharing one E8M0 scale) on the GPU
against the oracle, element by element within |gpu - oracle| <= 2e-3 *
sum|w*x| + 1e-5 (propagated through SwiGLU for the FFN): moe_mul_mat_id in
both modes and moe_ffn with a shared expert, on the mat-vec path (decode
sizes) and the tensor-core GEMM path; the hand-worked blocks of
tests/golden/mxfp4_blocks.json reproduced exactly through a one-expert
product; bit-identical reruns.
"""
import json
import os

import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.fixtures import GOLDEN
from tests.gpu_util import check_close, paths, to_dev_x

pytestmark = pytest.mark.gpu

PATHS = [pytest.param(1, id="gemv"), pytest.param(2, id="gemm")]


def prep_mx(W: np.ndarray) -> torch.Tensor:
    E, n_out, nb, _ = W.shape
    return moe.weights_prepare(torch.from_numpy(np.ascontiguousarray(W)).cuda(), E, n_out, nb * 32, wtype="mxfp4")


@pytest.mark.parametrize("path", PATHS)
def test_hand_worked_blocks_exact(path):
    # each golden block as the single block of one weight row; x = one-hot columns
    # pick out every element: dst[t][0][row] = w[row][t] exactly
    blocks = [b for b in json.load(open(os.path.join(GOLDEN, "mxfp4_blocks.json")))["blocks"] if not b.get("nan")]
    W = np.zeros((1, 16, 1, 17), np.uint8)
    W[..., 0] = 127
    for i, b in enumerate(blocks):
        W[0, i, 0] = np.array(b["bytes"], np.uint8)
    x = np.eye(32, dtype=np.float32)
    ids = np.zeros((32, 1), np.int32)
    with paths(path):
        dst = moe.mul_mat_id(prep_mx(W), 1, 16, 32, to_dev_x(x, "f32"), torch.from_numpy(ids).cuda(), wtype="mxfp4")
    got = dst.cpu().numpy()[:, 0, :].T.astype(np.float64)  # [row][element]
    want = oracle.dequant(W, 0)
    # every value, from 6 * 2^-127 up to 2^127, is exact in float and in bf16
    assert np.array_equal(got[:len(blocks)], want[:len(blocks)])


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
@pytest.mark.parametrize("x_type", ["bf16", "f32"])
def test_mul_mat_id_mxfp4(path, mode, x_type):
    E, k, T, n_in, n_out = 24, 3, 7 if path == 1 else 90, 320, 208
    W = workloads.mxfp4_weights(E, n_out, n_in, 31, 1)
    ids = workloads.routing("uniform", T, E, k, 31)
    rows = T if mode == "broadcast" else T * k
    x = workloads.activations(rows, n_in, x_type, 31, 2)
    ref, tol = oracle.mul_mat_id(W, x, x_type, ids, mode)
    with paths(path):
        dst = moe.mul_mat_id(prep_mx(W), E, n_out, n_in, to_dev_x(x, x_type), torch.from_numpy(ids).cuda(), mode,
                             wtype="mxfp4")
    check_close(dst, ref, tol, f"mxfp4 mul_mat_id path {path} {mode} {x_type}")


@pytest.mark.parametrize("T", [1, 8, 40])
def test_ffn_mxfp4_with_shared_expert(T):
    wl = workloads.WORKLOADS["decode"]
    E, k, n_embd, n_ff, n_sh = wl.n_experts, wl.k, wl.n_in, wl.n_out, wl.n_ff_shared
    Wg = workloads.mxfp4_weights(E, n_ff, n_embd, 5, workloads.T_WG)
    Wu = workloads.mxfp4_weights(E, n_ff, n_embd, 5, workloads.T_WU)
    Wd = workloads.mxfp4_weights(E, n_embd, n_ff, 5, workloads.T_WD)
    Sg = workloads.mxfp4_weights(1, n_sh, n_embd, 5, workloads.T_SG)
    Su = workloads.mxfp4_weights(1, n_sh, n_embd, 5, workloads.T_SU)
    Sd = workloads.mxfp4_weights(1, n_embd, n_sh, 5, workloads.T_SD)
    x = workloads.activations(T, n_embd, "bf16", 5, workloads.T_X)
    ids = workloads.routing("uniform", T, E, k, 5)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    ref_sh, tol_sh = oracle.shared_ffn(Sg, Su, Sd, x, "bf16")
    args = (prep_mx(Wg), prep_mx(Wu), prep_mx(Wd), E, n_embd, n_ff, to_dev_x(x, "bf16"), torch.from_numpy(ids).cuda())
    shared = (prep_mx(Sg), prep_mx(Su), prep_mx(Sd), n_sh)
    dst, dsh = moe.ffn(*args, shared=shared, wtype="mxfp4")
    check_close(dst.reshape(T * k, n_embd), ref, tol, f"mxfp4 ffn T={T} routed")
    check_close(dsh, ref_sh, tol_sh, f"mxfp4 ffn T={T} shared")
    again, again_sh = moe.ffn(*args, shared=shared, wtype="mxfp4")
    assert torch.equal(again.view(torch.int32), dst.view(torch.int32))
    assert torch.equal(again_sh.view(torch.int32), dsh.view(torch.int32))
