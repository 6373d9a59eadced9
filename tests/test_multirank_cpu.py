"""Multi-rank host logic on CPU (gloo, world size 2): token sharding needs no
data-path collective - each rank's shard, computed alone, equals the same rows
of the unsharded computation - and the step time is the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from indirect_expert_matmul_b200.dist import token_shard


def test_token_shard_partitions_the_batch():
    for T in (0, 1, 7, 4096, 4097):
        for W in (1, 2, 3, 8):
            spans = [token_shard(T, r, W) for r in range(W)]
            assert spans[0][0] == 0
            for (a, n), (b, _) in zip(spans, spans[1:]):
                assert a + n == b
            assert sum(n for _, n in spans) == T
            assert max(n for _, n in spans) - min(n for _, n in spans) <= 1
    with pytest.raises(ValueError):
        token_shard(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    import oracle
    import workloads
    from indirect_expert_matmul_b200.dist import max_over_ranks, token_shard

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = workloads.WORKLOADS["tiny"]
    T_total = 50
    t0, T = token_shard(T_total, rank, world)
    W = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)  # replicated
    ids = wl.ids(T, t0=t0)
    x = wl.x(T, t0=t0)
    dst, _ = oracle.mul_mat_id(W, x, "f32", ids)
    # gather shards to rank 0 (test only: the operator itself needs no collective)
    parts = [None] * world
    dist.all_gather_object(parts, (t0, ids, dst))
    slow = max_over_ranks(0.5 + rank)
    if rank == 0:
        np.savez(os.path.join(out_dir, "shards.npz"),
                 ids=np.concatenate([p[1] for p in sorted(parts, key=lambda p: p[0])]),
                 dst=np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])]), slow=slow)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_match_unsharded(tmp_path):
    import oracle
    import workloads

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    got = np.load(tmp_path / "shards.npz")
    wl = workloads.WORKLOADS["tiny"]
    W = workloads.q8_0_weights(wl.n_experts, wl.n_out, wl.n_in, wl.seed, workloads.T_W)
    ids = wl.ids(50)
    dst, _ = oracle.mul_mat_id(W, wl.x(50), "f32", ids)
    assert np.array_equal(got["ids"], ids)
    assert np.array_equal(got["dst"], dst)       # bit-identical: tokens are independent
    assert float(got["slow"]) == 1.5              # max over ranks


# ------------------------------------------------------- expert parallelism
def _ep_rank_main(rank, world, port, out_dir, what):
    import torch
    import torch.distributed as dist

    import oracle
    import workloads
    from indirect_expert_matmul_b200.dist import token_shard
    from indirect_expert_matmul_b200.expert_parallel import ep_forward, expert_range

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    e0, e1 = expert_range(EP_E, rank, world)
    t0, T = token_shard(EP_T, rank, world)
    ids_all = workloads.routing("uniform", EP_T, EP_E, EP_K, 21)
    if what == "mul_mat_id":
        W = workloads.q8_0_weights(EP_E, EP_NOUT, EP_NIN, 21, workloads.T_W)[e0:e1]  # this rank's experts only
        x = workloads.activations(EP_T, EP_NIN, "f32", 21, workloads.T_X)[t0:t0 + T]
        n_out = EP_NOUT

        def compute(xr, ir):
            out, _ = oracle.mul_mat_id(W, xr.numpy(), "f32", ir.numpy())
            return torch.from_numpy(out.astype(np.float32))
        x_t = torch.from_numpy(np.ascontiguousarray(x))
    else:  # the routed SwiGLU FFN, bf16 activations (bit patterns carried as int32)
        Wg = workloads.q8_0_weights(EP_E, EP_NFF, EP_NIN, 21, workloads.T_WG)[e0:e1]
        Wu = workloads.q8_0_weights(EP_E, EP_NFF, EP_NIN, 21, workloads.T_WU)[e0:e1]
        Wd = workloads.q8_0_weights(EP_E, EP_NIN, EP_NFF, 21, workloads.T_WD)[e0:e1]
        x = workloads.activations(EP_T, EP_NIN, "bf16", 21, workloads.T_X)[t0:t0 + T]
        n_out = EP_NIN

        def compute(xr, ir):
            out, _ = oracle.ffn(Wg, Wu, Wd, xr.numpy().astype(np.uint16), "bf16", ir.numpy())
            return torch.from_numpy(out.astype(np.float32))
        x_t = torch.from_numpy(np.ascontiguousarray(x).astype(np.int32))
    dst = ep_forward(x_t, torch.from_numpy(ids_all[t0:t0 + T].copy()), EP_T, EP_E, n_out, compute)
    np.save(os.path.join(out_dir, f"ep_{rank}.npy"), dst.numpy())
    dist.barrier()
    dist.destroy_process_group()


EP_E, EP_K, EP_T, EP_NIN, EP_NOUT, EP_NFF = 10, 3, 23, 96, 40, 64


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("what", ["mul_mat_id", "ffn"])
def test_expert_parallel_matches_unsharded(tmp_path, world, what):
    """Experts split into contiguous ranges across gloo ranks, tokens sharded:
    after the all-to-all every rank holds exactly the unsharded oracle's rows
    for its tokens, bit for bit (each slot is computed once, from the same
    weights and activation row, and the exchange does no arithmetic)."""
    import oracle
    import workloads

    mp.start_processes(_ep_rank_main, args=(world, _free_port(), str(tmp_path), what), nprocs=world,
                       start_method="spawn")
    got = np.concatenate([np.load(tmp_path / f"ep_{r}.npy") for r in range(world)])
    ids = workloads.routing("uniform", EP_T, EP_E, EP_K, 21)
    if what == "mul_mat_id":
        W = workloads.q8_0_weights(EP_E, EP_NOUT, EP_NIN, 21, workloads.T_W)
        ref, _ = oracle.mul_mat_id(W, workloads.activations(EP_T, EP_NIN, "f32", 21, workloads.T_X), "f32", ids)
        ref = ref.reshape(EP_T, EP_K, EP_NOUT)
    else:
        Wg = workloads.q8_0_weights(EP_E, EP_NFF, EP_NIN, 21, workloads.T_WG)
        Wu = workloads.q8_0_weights(EP_E, EP_NFF, EP_NIN, 21, workloads.T_WU)
        Wd = workloads.q8_0_weights(EP_E, EP_NIN, EP_NFF, 21, workloads.T_WD)
        ref, _ = oracle.ffn(Wg, Wu, Wd, workloads.activations(EP_T, EP_NIN, "bf16", 21, workloads.T_X), "bf16", ids)
        ref = ref.reshape(EP_T, EP_K, EP_NIN)
    assert got.shape == ref.shape
    assert np.array_equal(got, ref.astype(np.float32))


def test_expert_ranges_partition_the_experts():
    from indirect_expert_matmul_b200.expert_parallel import expert_range, owned_slot_range
    import oracle
    import workloads
    for E in (1, 8, 10, 256):
        for W in (1, 2, 3, 8):
            if W > E:
                continue
            rs = [expert_range(E, r, W) for r in range(W)]
            assert rs[0][0] == 0 and rs[-1][1] == E
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
    # a contiguous expert range owns a contiguous range of sorted positions
    ids = workloads.routing("uniform", 40, 10, 3, 5)
    _, ids_dst, bounds = oracle.row_ids(ids, 10)
    for W in (2, 3):
        for r in range(W):
            e0, e1 = expert_range(10, r, W)
            p0, p1 = owned_slot_range(bounds, e0, e1)
            flat = ids.reshape(-1)
            assert sorted(ids_dst[p0:p1].tolist()) == [i for i in range(flat.size) if e0 <= flat[i] < e1]
