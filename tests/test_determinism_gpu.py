"""Run-to-run bit identity of every GPU path: ten calls on the same inputs
give the same bits (the reproducibility the PR #283 article asks of the new
path: identical per-chunk perplexity under a fixed seed, sections 3.2 and
4.3), and a zero device status.

- The decode mat-vec path with the shared expert at 1, 4 and 8 tokens: at one
  token K is split across CTAs and the last CTA of each (expert, row tile)
  adds the chunks, so this is where an order that depended on arrival would
  show.  dst, dst_shared and the status are compared, through the workspace
  entry point and the one without a workspace.
- moe_mul_mat_id on the grouped GEMM in both modes at the full skewed-load
  shape (8192 tokens, Zipf popularity, empty and heavy experts).
- The Lite-shaped expert FFN on the grouped GEMM (512 tokens).
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import workloads
from tests.gpu_util import paths, prep, to_dev_x

pytestmark = pytest.mark.gpu

RUNS = 10


def _bits(t):
    return t.detach().contiguous().view(torch.int32).cpu().clone()


def _decode_inputs(T):
    wl = workloads.WORKLOADS["decode"]
    Wg = prep(workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG))
    Wu = prep(workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU))
    Wd = prep(workloads.q8_0_weights(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD))
    sh = (prep(workloads.q8_0_weights(1, wl.n_ff_shared, wl.n_in, wl.seed, workloads.T_SG)),
          prep(workloads.q8_0_weights(1, wl.n_ff_shared, wl.n_in, wl.seed, workloads.T_SU)),
          prep(workloads.q8_0_weights(1, wl.n_in, wl.n_ff_shared, wl.seed, workloads.T_SD)), wl.n_ff_shared)
    return wl, Wg, Wu, Wd, sh, to_dev_x(wl.x(T), "bf16"), torch.from_numpy(wl.ids(T)).cuda()


@pytest.mark.parametrize("T", [1, 4, 8])
def test_decode_ten_runs_bit_identical(T):
    wl, Wg, Wu, Wd, sh, x, ids = _decode_inputs(T)
    ws = moe.workspace(T, wl.k, wl.n_experts, wl.n_in, wl.n_out, wl.n_ff_shared)
    ref = ref_sh = None
    for run in range(RUNS):
        dst, dsh = moe.ffn(Wg, Wu, Wd, wl.n_experts, wl.n_in, wl.n_out, x, ids, shared=sh, ws=ws)
        assert moe.get_status(ws) == moe.OK, f"run {run}"
        if ref is None:
            ref, ref_sh = _bits(dst), _bits(dsh)
        else:
            assert torch.equal(_bits(dst), ref), f"T={T} run {run}: routed output differs"
            assert torch.equal(_bits(dsh), ref_sh), f"T={T} run {run}: shared output differs"
    # the entry point without a workspace: the same kernels, bit-identical across its own runs
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = None
    for run in range(RUNS):
        dst, dsh = moe.ffn_decode_noalloc(Wg, Wu, Wd, wl.n_experts, wl.n_in, wl.n_out, x, ids, shared=sh,
                                          status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.OK
        got = (_bits(dst), _bits(dsh))
        if first is None:
            first = got
        else:
            assert torch.equal(got[0], first[0]) and torch.equal(got[1], first[1]), f"noalloc T={T} run {run}"


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
def test_skew_mul_mat_id_ten_runs_bit_identical(mode):
    from tests.test_fullsize_gpu import prep_chunked
    wl = workloads.WORKLOADS["skew"]
    T = wl.n_tokens[0]
    W = prep_chunked(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    x = to_dev_x(wl.x(T, mode=mode), "bf16")
    ids = torch.from_numpy(wl.ids(T)).cuda()
    ws = moe.workspace(T, wl.k, wl.n_experts, wl.n_in, x_dtype=torch.bfloat16)
    out = torch.empty((T, wl.k, wl.n_out), dtype=torch.float32, device="cuda")
    ref = None
    with paths(2):
        for run in range(RUNS):
            moe.mul_mat_id(W, wl.n_experts, wl.n_out, wl.n_in, x, ids, mode, ws=ws, out=out)
            assert moe.get_status(ws) == moe.OK
            if ref is None:
                ref = out.clone()
            else:
                assert torch.equal(out.view(torch.int32), ref.view(torch.int32)), f"skew {mode} run {run}"
    del W
    torch.cuda.empty_cache()


def test_lite_ffn_gemm_ten_runs_bit_identical():
    wl = workloads.WORKLOADS["lite"]
    T = wl.n_tokens[0]
    Wg = prep(workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG))
    Wu = prep(workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU))
    Wd = prep(workloads.q8_0_weights(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD))
    x, ids = to_dev_x(wl.x(T), "bf16"), torch.from_numpy(wl.ids(T)).cuda()
    ws = moe.workspace(T, wl.k, wl.n_experts, wl.n_in, wl.n_out)
    ref = None
    with paths(2):
        for run in range(RUNS):
            dst, _ = moe.ffn(Wg, Wu, Wd, wl.n_experts, wl.n_in, wl.n_out, x, ids, ws=ws)
            assert moe.get_status(ws) == moe.OK
            if ref is None:
                ref = _bits(dst)
            else:
                assert torch.equal(_bits(dst), ref), f"lite run {run}"
    assert np.isfinite(dst.cpu().numpy()).all()
