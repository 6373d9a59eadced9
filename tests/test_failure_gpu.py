"""Failure detection on the GPU without a fault: a bounded wait inside the
mat-vec kernel, or inside the grouped GEMM, is made to run out (the test-only stall of include/
moe_testing.h: one CTA's weight producer skips one ring stage, no copy is
issued for it, and the waits give up after a millisecond).  The call must
report MOE_ERR_TIMEOUT with the expired wait's site recorded, the device must
stay usable, and the next call on a re-initialised workspace must be correct.
No trap, no fault, no unbounded spin is involved.
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.gpu_util import check_close, prep, to_dev_x

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("stage", [0, 3])
def test_expired_wait_reports_timeout_and_the_device_recovers(stage):
    wl = workloads.WORKLOADS["decode"]
    T = 1
    Wg = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG)
    Wu = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU)
    Wd = workloads.q8_0_weights(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD)
    x, ids = wl.x(T), wl.ids(T)
    args = (prep(Wg), prep(Wu), prep(Wd), wl.n_experts, wl.n_in, wl.n_out, to_dev_x(x, "bf16"),
            torch.from_numpy(ids).cuda())
    ws = moe.workspace(T, wl.k, wl.n_experts, wl.n_in, wl.n_out)
    lib = moe.lib()
    lib.moe_testing_stall(0, stage, 1000)  # CTA 0 skips a stage; waits give up after 1 ms
    try:
        moe.ffn(*args, ws=ws)
        st = moe.get_status(ws)  # synchronises
    finally:
        lib.moe_testing_stall(-1, 0, 0)
    assert st == moe.ERR_TIMEOUT
    site = int(ws[12:16].view(torch.int32).item())  # header word 3
    assert site >> 30 == 1, hex(site)
    assert 0 <= (site >> 20) & 0x3ff < 17  # a warp of the 544-thread mat-vec CTA
    # the device answers, and the same call on a re-initialised workspace is correct
    torch.cuda.synchronize()
    assert lib.moe_workspace_init(ws.data_ptr(), None) == moe.OK
    dst, _ = moe.ffn(*args, ws=ws)
    assert moe.get_status(ws) == moe.OK
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    check_close(dst.reshape(T * wl.k, wl.n_in), ref, tol, "decode after an expired wait")


@pytest.mark.parametrize("stage", [0, 5])
def test_expired_wait_in_the_grouped_gemm_reports_timeout_and_the_device_recovers(stage):
    # 32 tokens: above the mat-vec threshold, so both projections run on the
    # grouped GEMM; CTA 0's activation copy of its k-step `stage` is never issued
    wl = workloads.WORKLOADS["decode"]
    T = 32
    Wg = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG)
    Wu = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU)
    Wd = workloads.q8_0_weights(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD)
    x, ids = wl.x(T), wl.ids(T)
    args = (prep(Wg), prep(Wu), prep(Wd), wl.n_experts, wl.n_in, wl.n_out, to_dev_x(x, "bf16"),
            torch.from_numpy(ids).cuda())
    ws = moe.workspace(T, wl.k, wl.n_experts, wl.n_in, wl.n_out)
    lib = moe.lib()
    threshold = lib.moe_get_gemv_threshold()
    moe.set_gemv_threshold(8)  # the grouped GEMM path, whatever an earlier test set
    try:
        lib.moe_testing_stall(0, stage, 1000)  # waits give up after 1 ms
        try:
            moe.ffn(*args, ws=ws)
            st = moe.get_status(ws)  # synchronises
        finally:
            lib.moe_testing_stall(-1, 0, 0)
        assert st == moe.ERR_TIMEOUT
        site = int(ws[12:16].view(torch.int32).item())  # header word 3
        assert site >> 30 == 1, hex(site)
        assert 0 <= (site >> 20) & 0x3ff < 20  # a warp of the 640-thread GEMM CTA
        torch.cuda.synchronize()
        assert lib.moe_workspace_init(ws.data_ptr(), None) == moe.OK
        dst, _ = moe.ffn(*args, ws=ws)
        assert moe.get_status(ws) == moe.OK
    finally:
        moe.set_gemv_threshold(threshold)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    check_close(dst.reshape(T * wl.k, wl.n_in), ref, tol, "grouped GEMM after an expired wait")
