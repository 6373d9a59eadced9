"""moe_ffn_decode_noalloc - the decode FFN with its scratch in a static
device array - on the decode workload with a shared expert.  Two calls in a
row: each is within the oracle's per-element tolerance of the exact result,
each agrees with moe_ffn (the workspace entry point) within the sum of their
two distances to it, the second is bit-identical to the first (a stale
scratch array would show here), and each reports a zero device status.
Sizes past the static array's capacity are refused on the host.  This file
is named to be collected last so that it also runs after every other GPU
test in the same process.
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.gpu_util import prep, to_dev_x

pytestmark = pytest.mark.gpu


def _inputs(wl, T):
    Wg = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG)
    Wu = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU)
    Wd = workloads.q8_0_weights(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD)
    sh = (workloads.q8_0_weights(1, wl.n_ff_shared, wl.n_in, wl.seed, workloads.T_SG),
          workloads.q8_0_weights(1, wl.n_ff_shared, wl.n_in, wl.seed, workloads.T_SU),
          workloads.q8_0_weights(1, wl.n_in, wl.n_ff_shared, wl.seed, workloads.T_SD))
    return Wg, Wu, Wd, sh, wl.x(T), wl.ids(T)


@pytest.mark.parametrize("T", [1, 4, 8])
def test_noalloc_matches_workspace_entry_point(T):
    wl = workloads.WORKLOADS["decode"]
    Wg, Wu, Wd, sh, x, ids = _inputs(wl, T)
    exact, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    exact_sh, tol_sh = oracle.shared_ffn(*sh, x, "bf16")
    dWg, dWu, dWd = prep(Wg), prep(Wu), prep(Wd)
    shared = (prep(sh[0]), prep(sh[1]), prep(sh[2]), wl.n_ff_shared)
    xd, idd = to_dev_x(x, "bf16"), torch.from_numpy(ids).cuda()
    ref, ref_sh = moe.ffn(dWg, dWu, dWd, wl.n_experts, wl.n_in, wl.n_out, xd, idd, shared=shared)
    ref = ref.cpu().numpy().reshape(T * wl.k, wl.n_in).astype(np.float64)
    ref_sh = ref_sh.cpu().numpy().astype(np.float64)
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    first = None
    for call in range(2):  # two calls in a row share the one static scratch
        dst, dsh = moe.ffn_decode_noalloc(dWg, dWu, dWd, wl.n_experts, wl.n_in, wl.n_out, xd, idd, shared=shared,
                                          status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.OK, f"call {call}: {moe.status_string(int(status.item()))}"
        got = dst.cpu().numpy().reshape(T * wl.k, wl.n_in).astype(np.float64)
        got_sh = dsh.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - exact) <= tol), f"call {call}: routed rows outside the oracle's tolerance"
        assert np.all(np.abs(got_sh - exact_sh) <= tol_sh), f"call {call}: shared rows outside the oracle's tolerance"
        assert np.all(np.abs(got - ref) <= 2 * tol), f"call {call}: routed rows differ from moe_ffn beyond tolerance"
        assert np.all(np.abs(got_sh - ref_sh) <= 2 * tol_sh), f"call {call}: shared rows differ from moe_ffn"
        if first is None:
            first = (got.copy(), got_sh.copy())
        else:
            assert np.array_equal(got, first[0]) and np.array_equal(got_sh, first[1]), "calls differ bit for bit"


def test_noalloc_reports_bad_id():
    wl = workloads.WORKLOADS["decode"]
    Wg, Wu, Wd, _, x, ids = _inputs(wl, 1)
    ids = ids.copy()
    ids[0, 0] = wl.n_experts  # outside [0, n_experts)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.ffn_decode_noalloc(prep(Wg), prep(Wu), prep(Wd), wl.n_experts, wl.n_in, wl.n_out, to_dev_x(x, "bf16"),
                           torch.from_numpy(ids).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.ERR_BAD_ID


def test_noalloc_header_clears_itself_after_an_error():
    # the down launch's last CTA copies the status out and zeroes the header, so
    # a good call right after a failing one reports MOE_OK and computes exactly
    wl = workloads.WORKLOADS["decode"]
    Wg, Wu, Wd, _, x, ids = _inputs(wl, 4)
    dWg, dWu, dWd, xd = prep(Wg), prep(Wu), prep(Wd), to_dev_x(x, "bf16")
    bad = ids.copy()
    bad[1, 2] = -1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.ffn_decode_noalloc(dWg, dWu, dWd, wl.n_experts, wl.n_in, wl.n_out, xd, torch.from_numpy(bad).cuda(),
                           status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.ERR_BAD_ID
    dst, _ = moe.ffn_decode_noalloc(dWg, dWu, dWd, wl.n_experts, wl.n_in, wl.n_out, xd, torch.from_numpy(ids).cuda(),
                                    status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.OK
    exact, tol = oracle.ffn(Wg, Wu, Wd, x, "bf16", ids)
    got = dst.cpu().numpy().reshape(4 * wl.k, wl.n_in).astype(np.float64)
    assert np.all(np.abs(got - exact) <= tol)


def test_noalloc_refuses_sizes_past_its_scratch():
    wl = workloads.WORKLOADS["decode"]
    Wg, Wu, Wd, _, x, ids = _inputs(wl, 1)
    dWg, dWu, dWd, xd = prep(Wg), prep(Wu), prep(Wd), to_dev_x(x, "bf16")
    big_ids = torch.zeros((9, 8), dtype=torch.int32, device="cuda")  # 72 slots > 64
    big_x = torch.zeros((9, wl.n_in), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.ffn_decode_noalloc(dWg, dWu, dWd, wl.n_experts, wl.n_in, wl.n_out, big_x, big_ids)
    assert e.value.code == moe.ERR_RANGE
    # n_ff past 2048: the entry point refuses it on the host, before any weight is read
    ids_d = torch.from_numpy(ids).cuda()
    out = torch.empty((1, wl.k, wl.n_in), dtype=torch.float32, device="cuda")
    st = moe.lib().moe_ffn_decode_noalloc(dWg.data_ptr(), dWu.data_ptr(), dWd.data_ptr(), wl.n_experts, wl.n_in, 2080,
                                          None, None, None, 0, xd.data_ptr(), moe.BF16, ids_d.data_ptr(), 1, wl.k,
                                          out.data_ptr(), None, None, None)
    assert st == moe.ERR_RANGE
    # through the binding, weights too small for the stated n_ff are refused before the call
    with pytest.raises(ValueError):
        moe.ffn_decode_noalloc(dWg, dWu, dWd, wl.n_experts, wl.n_in, 2080, xd, ids_d)
