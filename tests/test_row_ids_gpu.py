"""Row-id pass on the GPU against the oracle: bit-exact tables.

The tables of the PR #283 article ("ik_llama.cpp 的 CUDA 更优 MoE 实现",
section 2.1) are unique once the order inside an expert is fixed to ascending
(token, slot), so the comparison is exact equality.
"""
import numpy as np
import pytest
import torch

import indirect_expert_matmul_b200 as moe
import oracle
import workloads
from tests.fixtures import hand_example

pytestmark = pytest.mark.gpu


def gpu_tables(ids_np, E, mode):
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).cuda()
    ws = moe.workspace(ids.shape[0], ids.shape[1], E, 0)
    s1, d, b = moe.row_ids(ids, E, mode, ws=ws)
    assert moe.get_status(ws) == moe.OK
    return s1.cpu().numpy(), d.cpu().numpy(), b.cpu().numpy()


def assert_tables_equal(ids_np, E, mode):
    a = gpu_tables(ids_np, E, mode)
    b = oracle.row_ids(ids_np, E, mode)
    for name, x, y in zip(("ids_src1", "ids_dst", "expert_bounds"), a, b):
        assert np.array_equal(x, y), f"{name} differs (E={E}, shape={ids_np.shape}, mode={mode})"


def test_hand_example_tables():
    g, W, xb, xs, ids = hand_example()
    s1, d, b = gpu_tables(ids, 2, "broadcast")
    assert b.tolist() == g["expert_bounds"]
    assert d.tolist() == g["ids_dst"]
    assert s1.tolist() == g["ids_src1_broadcast"]
    s1, _, _ = gpu_tables(ids, 2, "per_slot")
    assert s1.tolist() == g["ids_src1_per_slot"]


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_workload_tables_bit_exact(name):
    wl = workloads.WORKLOADS[name]
    for T in wl.n_tokens:
        ids = wl.ids(T)
        for mode in ("broadcast", "per_slot"):
            assert_tables_equal(ids, wl.n_experts, mode)


@pytest.mark.parametrize("seed", range(16))
def test_fuzz_bit_exact(seed):
    rng = np.random.default_rng(100 + seed)
    E = int(rng.choice([1, 2, 3, 7, 64, 256, 1000, 5000]))
    k = int(rng.integers(1, min(E, 40) + 1))
    T = int(rng.choice([0, 1, 2, 5, 31, 33, 300, 1025, 4099]))
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)  # duplicates allowed
    assert_tables_equal(ids, E, "broadcast" if seed % 2 else "per_slot")


def test_skewed_and_single_expert():
    # every slot on one expert; and an expert list with most experts empty
    assert_tables_equal(np.full((777, 4), 3, np.int32), 8, "broadcast")
    rng = np.random.default_rng(5)
    ids = rng.choice([0, 511], size=(1000, 2)).astype(np.int32)
    assert_tables_equal(ids, 512, "per_slot")


def test_large_token_count():
    rng = np.random.default_rng(6)
    ids = rng.integers(0, 256, size=(65536, 8)).astype(np.int32)
    assert_tables_equal(ids, 256, "broadcast")


def test_bad_id_sets_status_and_recovers():
    E = 4
    ids = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")
    ws = moe.workspace(2, 2, E, 0)
    moe.row_ids(ids, E, "broadcast", ws=ws)
    assert moe.get_status(ws) == moe.ERR_BAD_ID
    ids2 = torch.tensor([[0, 1], [2, -1]], dtype=torch.int32, device="cuda")
    moe.row_ids(ids2, E, "broadcast", ws=ws)
    assert moe.get_status(ws) == moe.ERR_BAD_ID
    # status was cleared by the read: a good call now succeeds
    good = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    s1, d, b = moe.row_ids(good, E, "broadcast", ws=ws)
    assert moe.get_status(ws) == moe.OK
    assert b.cpu().tolist() == [0, 1, 2, 3, 4]


def test_sticky_error_blocks_later_kernels():
    E = 4
    ws = moe.workspace(2, 2, E, 0)
    moe.row_ids(torch.tensor([[0, 7], [1, 2]], dtype=torch.int32, device="cuda"), E, ws=ws)
    s1, d, b = moe.row_ids(torch.tensor([[0, 1], [1, 2]], dtype=torch.int32, device="cuda"), E, ws=ws)
    torch.cuda.synchronize()
    assert moe.get_status(ws) == moe.ERR_BAD_ID   # second call did nothing


def test_host_argument_errors():
    ids = torch.zeros((2, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.row_ids(ids, 1)                 # k > E
    assert e.value.code == moe.ERR_RANGE
    big = torch.zeros((1, 1024), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.row_ids(big, 2000)              # k >= 2^10
    assert e.value.code == moe.ERR_RANGE


def test_repeatable_ten_runs():
    wl = workloads.WORKLOADS["v3"]
    ids = wl.ids(4096)
    ref = gpu_tables(ids, wl.n_experts, "broadcast")
    for _ in range(9):
        again = gpu_tables(ids, wl.n_experts, "broadcast")
        for x, y in zip(ref, again):
            assert np.array_equal(x, y)


@pytest.mark.parametrize("E", [1024, 1025])
def test_many_ctas_at_the_expert_limit(E):
    # 8192 x 8 slots: the pass runs over 32 CTAs up to 1024 experts (32 chunk rows
    # of E counters in shared memory), and in one CTA past that
    rng = np.random.default_rng(7)
    ids = rng.integers(0, E, size=(8192, 8)).astype(np.int32)
    assert_tables_equal(ids, E, "per_slot")


def test_many_ctas_one_heavy_expert():
    # every slot but a few on expert 3: one column of per-CTA counts carries all
    rng = np.random.default_rng(8)
    ids = np.full((4096, 8), 3, dtype=np.int32)
    ids[rng.integers(0, 4096, 50), rng.integers(0, 8, 50)] = 200
    assert_tables_equal(ids, 256, "broadcast")


def test_many_ctas_bad_id_reports_status():
    ids = np.zeros((4096, 8), dtype=np.int32)
    ids[3000, 5] = 256  # outside [0, 256), counted by the CTA that owns slot 24005
    t = torch.from_numpy(ids).cuda()
    ws = moe.workspace(4096, 8, 256, 0)
    moe.row_ids(t, 256, "broadcast", ws=ws)
    assert moe.get_status(ws) == moe.ERR_BAD_ID
