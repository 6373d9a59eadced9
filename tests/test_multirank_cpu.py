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
