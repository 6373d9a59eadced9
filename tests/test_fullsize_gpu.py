"""Full-size parity in the launch configuration the benchmark times.

The DeepSeek-V3-shaped layer (256 experts, top-8, 7168 x 2048, 4096 tokens)
and the skewed-load stress case (128 experts, top-4 Zipf, 2880 x 2880, 8192
tokens, broadcast and per_slot) run whole on the GPU; the oracle computes
sampled output rows one by one (the first and last slot of every non-empty
expert plus random ones, so every expert's tiles are visited), element by
element within the tolerance.  The row-id tables are compared whole, and the
V3 output is checked bit-identical over 10 runs.
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.gpu_util import check_close, sample_slots, to_dev_x

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def prep_chunked(n_experts, n_out, n_in, seed, tensor, chunk=32):
    per = moe.weights_prepared_size(1, n_out, n_in)
    out = torch.empty(per * n_experts, dtype=torch.uint8, device="cuda")
    for e0 in range(0, n_experts, chunk):
        n_e = min(chunk, n_experts - e0)
        raw = torch.from_numpy(workloads.q8_0_weights_experts(e0, n_e, n_out, n_in, seed, tensor)).cuda()
        moe.weights_prepare(raw, n_e, n_out, n_in, out=out[e0 * per:(e0 + n_e) * per])
    return out


def sub_weights(experts, n_out, n_in, seed, tensor):
    return np.concatenate([workloads.q8_0_weights_experts(e, 1, n_out, n_in, seed, tensor) for e in experts])


@pytest.fixture(scope="module")
def v3_run():
    wl = workloads.WORKLOADS["v3"]
    T = wl.n_tokens[0]
    Wg = prep_chunked(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG)
    Wu = prep_chunked(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU)
    Wd = prep_chunked(wl.n_experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD)
    ids_np, x_np = wl.ids(T), wl.x(T)
    x, ids = to_dev_x(x_np, "bf16"), torch.from_numpy(ids_np).cuda()
    ws = moe.workspace(T, wl.k, wl.n_experts, wl.n_in, wl.n_out, 0, torch.bfloat16)
    dst, _ = moe.ffn(Wg, Wu, Wd, wl.n_experts, wl.n_in, wl.n_out, x, ids, ws=ws)
    assert moe.get_status(ws) == moe.OK
    yield wl, ids_np, x_np, (Wg, Wu, Wd, x, ids, ws), dst
    del Wg, Wu, Wd
    torch.cuda.empty_cache()


def test_v3_sampled_rows_within_tolerance(v3_run):
    wl, ids_np, x_np, _, dst = v3_run
    T = wl.n_tokens[0]
    slots = sample_slots(ids_np, wl.n_experts, per_expert=2)
    flat = ids_np.reshape(-1)
    experts = sorted(set(int(flat[s]) for s in slots))
    remap = np.zeros(wl.n_experts, np.int32)
    remap[experts] = np.arange(len(experts))
    Wg = sub_weights(experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WG)
    Wu = sub_weights(experts, wl.n_out, wl.n_in, wl.seed, workloads.T_WU)
    Wd = sub_weights(experts, wl.n_in, wl.n_out, wl.seed, workloads.T_WD)
    ref, tol = oracle.ffn(Wg, Wu, Wd, x_np, "bf16", remap[ids_np], slots)
    got = dst.reshape(T * wl.k, wl.n_in)[torch.from_numpy(slots).cuda()]
    check_close(got, ref, tol, "v3 moe_ffn")


def test_v3_combine_sampled_tokens(v3_run):
    wl, _, _, _, dst = v3_run
    T = wl.n_tokens[0]
    r = workloads.router_weights(T, wl.k, wl.seed)
    y = moe.combine(dst, torch.from_numpy(r).cuda())
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 62, replace=False)]))
    sel = torch.from_numpy(toks).cuda()
    y_ref, mag = oracle.combine(dst[sel].cpu().numpy(), r[toks])
    check_close(y[sel], y_ref, oracle.combine_tolerance(mag, wl.k, False), "combine V3")


def test_v3_ten_runs_bit_identical(v3_run):
    wl, _, _, (Wg, Wu, Wd, x, ids, ws), dst = v3_run
    ref = dst.clone()
    for _ in range(9):
        again, _ = moe.ffn(Wg, Wu, Wd, wl.n_experts, wl.n_in, wl.n_out, x, ids, ws=ws)
        assert torch.equal(again.view(torch.int32), ref.view(torch.int32))
    assert moe.get_status(ws) == moe.OK


def test_v3_tables_bit_exact(v3_run):
    wl, ids_np, _, (_, _, _, _, ids, _), _ = v3_run
    s1, d, b = moe.row_ids(ids, wl.n_experts, "broadcast")
    o1, od, ob = oracle.row_ids(ids_np, wl.n_experts, "broadcast")
    assert np.array_equal(s1.cpu().numpy(), o1)
    assert np.array_equal(d.cpu().numpy(), od)
    assert np.array_equal(b.cpu().numpy(), ob)


@pytest.mark.parametrize("mode", ["broadcast", "per_slot"])
def test_skew_full_size_sampled(mode):
    wl = workloads.WORKLOADS["skew"]
    T = wl.n_tokens[0]
    W = prep_chunked(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    ids_np, x_np = wl.ids(T), wl.x(T, mode=mode)
    counts = np.bincount(ids_np.reshape(-1), minlength=wl.n_experts)
    assert (counts == 0).sum() >= wl.n_zero and counts.max() > 4 * 256  # heavy experts span many tiles
    dst = moe.mul_mat_id(W, wl.n_experts, wl.n_out, wl.n_in, to_dev_x(x_np, "bf16"),
                         torch.from_numpy(ids_np).cuda(), mode)
    slots = sample_slots(ids_np, wl.n_experts, per_expert=3, seed=1)
    flat = ids_np.reshape(-1)
    experts = sorted(set(int(flat[s]) for s in slots))
    remap = np.zeros(wl.n_experts, np.int32)
    remap[experts] = np.arange(len(experts))
    Ws = sub_weights(experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    ref, tol = oracle.mul_mat_id_rows(Ws, x_np, "bf16", remap[ids_np], slots, mode)
    got = dst.reshape(T * wl.k, wl.n_out)[torch.from_numpy(slots).cuda()]
    check_close(got, ref, tol, f"skew {mode}")
