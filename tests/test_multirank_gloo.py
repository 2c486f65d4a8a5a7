"""Data-parallel host path on CPU with two gloo ranks: each rank computes the backward
of its own sequences (with the CPU oracle standing in for the GPU kernels), the product's
helpers sum dU across ranks and take the slowest rank's time, and the result must equal
the single-process backward of the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

B, T, D, G, W, R = 4, 40, 16, 2, 3, 5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch():
    import dsc_inputs as di
    t = di.make(di.small(B, T, D, G, W, R, "f32", seed=21), "cpu", ("x", "z", "U", "dy"))
    return {k: v.double().numpy() for k, v in t.items()}


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist

    import oracle
    from dynamic_short_convolutions_causal_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        f = _batch()
        seqs = dp.shard_sequences(B, rank, world)
        sl = slice(seqs.start, seqs.stop)
        dx, dz, dU = oracle.bwd_lowrank(f["x"][sl], f["z"][sl], f["U"], f["dy"][sl], G, W)
        dU_t = torch.from_numpy(dU.copy())
        dp.allreduce_weight_grad(dU_t)
        slowest = dp.max_over_ranks(float(rank + 1))
        out[rank] = (seqs.start, seqs.stop, dx, dz, dU_t.numpy(), slowest)
    finally:
        dist.destroy_process_group()


def test_two_rank_data_parallel_backward_matches_single_process():
    import oracle
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    f = _batch()
    rdx, rdz, rdU = oracle.bwd_lowrank(f["x"], f["z"], f["U"], f["dy"], G, W)
    covered = []
    for rank in range(world):
        lo, hi, dx, dz, dU, slowest = out[rank]
        covered += list(range(lo, hi))
        np.testing.assert_allclose(dx, rdx[lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dz, rdz[lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dU, rdU, rtol=1e-12, atol=1e-12)   # summed over both ranks
        assert slowest == float(world)
    assert covered == list(range(B))


@pytest.mark.parametrize("Bn,world", [(8, 2), (5, 2), (7, 3), (1, 2)])
def test_shard_sequences_partitions_the_batch(Bn, world):
    from dynamic_short_convolutions_causal_b200 import dp
    seen = []
    for r in range(world):
        seen += list(dp.shard_sequences(Bn, r, world))
    assert seen == list(range(Bn))
