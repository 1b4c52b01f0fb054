"""The N > 1 path on CPU: two `gloo` ranks (world size 2) run independent
replicas over their share of a batch.  Because the (batch, head) slices of the
forward pass share nothing, sharding the batch needs no exchange on the data
path; these tests check the sharding arithmetic, the max-over-ranks timing
reduction and that concatenating the ranks' results (computed here by the
fp64 oracle on each rank's shard) reproduces the single-process result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from efficient_vision_attention_b200 import replicas


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("n,world", [(10, 2), (1, 2), (7, 3), (64, 8), (3, 4)])
def test_shard_covers_every_item_once(n, world):
    seen = []
    sizes = []
    for r in range(world):
        b, e = replicas.shard(n, world, r)
        seen.extend(range(b, e))
        sizes.append(e - b)
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_single_process_helpers():
    assert replicas.dist_env()[0] >= 1
    assert replicas.max_over_ranks(3.5, None) == 3.5
    assert replicas.rank_seed(3, 0) == 3 and replicas.rank_seed(3, 1) != 3


def _worker(rank, world, port, q_path, out_dir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import oracle
    dist = replicas.init("gloo", timeout_s=60)
    data = np.load(q_path)
    q, k, v = data["q"], data["k"], data["v"]
    b0, b1 = replicas.shard(q.shape[0], world, rank)
    o = oracle.agent_attn(q[b0:b1], k[b0:b1], v[b0:b1], 6, 6, 3, 2, 0.4) if b1 > b0 else \
        np.zeros((0,) + q.shape[1:])
    np.save(os.path.join(out_dir, f"o{rank}.npy"), o)
    # the step time of the job is the slowest rank's
    t = replicas.max_over_ranks(1.0 + rank, dist)
    np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([t]))
    replicas.barrier(dist)
    replicas.finalize(dist)


def test_two_gloo_ranks_reproduce_the_single_process_result(tmp_path):
    world = 2
    rng = np.random.default_rng(3)
    B, H, N, d = 5, 2, 36, 8
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    path = os.path.join(tmp_path, "qkv.npz")
    np.savez(path, q=q, k=k, v=v)
    mp.start_processes(_worker, args=(world, free_port(), path, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import oracle
    full = oracle.agent_attn(q, k, v, 6, 6, 3, 2, 0.4)
    parts = [np.load(os.path.join(tmp_path, f"o{r}.npy")) for r in range(world)]
    np.testing.assert_array_equal(np.concatenate(parts), full)
    for r in range(world):
        assert float(np.load(os.path.join(tmp_path, f"t{r}.npy"))[0]) == float(world)
