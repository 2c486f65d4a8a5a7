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


# ------------------------------------------------------------------ sequence sharding
# A sequence of P*T tokens split into P shards of T on P gloo ranks.  The product's
# helpers move the (W-1)-row halos (sp.exchange_prev / sp.exchange_next) and sum dU
# (dp.allreduce_weight_grad); each rank's shard computation uses the CPU oracle as the
# stand-in for the GPU kernels + halo fix-ups: the shard's outputs are the oracle's on
# the shard extended by the halos it received, which must equal the unsharded results.
SB, ST, SD, SG, SW, SR = 2, 9, 12, 3, 4, 5       # shard length 9 >= W-1 = 3


def _seq_batch(P):
    import dsc_inputs as di
    t = di.make(di.small(SB, ST * P, SD, SG, SW, SR, "f32", seed=33), "cpu", ("x", "z", "U", "dy"))
    return {k: v.double().numpy() for k, v in t.items()}


def _sp_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist

    import oracle
    from dynamic_short_convolutions_causal_b200 import dp, sp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        f = _seq_batch(world)
        tok = sp.shard_tokens(ST * world, rank, world)
        sl = slice(tok.start, tok.stop)
        x, z, dy = (torch.from_numpy(f[k][:, sl].copy()) for k in ("x", "z", "dy"))
        x_prev = sp.exchange_prev(x, SW)
        dy_next, z_next = sp.exchange_next(dy, z, SW)
        h = SW - 1
        # forward of the shard given the halo: rows of x before it (zeros on the first shard)
        xp = x_prev.numpy() if x_prev is not None else np.zeros((SB, h, SD))
        y = oracle.fwd_lowrank(np.concatenate([xp, x.numpy()], 1),
                               np.concatenate([np.zeros((SB, h, SR)), z.numpy()], 1), f["U"], SG, SW)[:, h:]
        # backward: dx sees the next shard's dy and z; dz and dU see the previous shard's x
        dyn = dy_next.numpy() if dy_next is not None else np.zeros((SB, h, SD))
        zn = z_next.numpy() if z_next is not None else np.zeros((SB, h, SR))
        dx = oracle.bwd_lowrank(np.concatenate([x.numpy(), np.zeros((SB, h, SD))], 1),
                                np.concatenate([z.numpy(), zn], 1), f["U"],
                                np.concatenate([dy.numpy(), dyn], 1), SG, SW)[0][:, :ST]
        _, dz, dU = oracle.bwd_lowrank(np.concatenate([xp, x.numpy()], 1),
                                       np.concatenate([np.zeros((SB, h, SR)), z.numpy()], 1), f["U"],
                                       np.concatenate([np.zeros((SB, h, SD)), dy.numpy()], 1), SG, SW)
        dU_t = torch.from_numpy(dU.copy())
        dp.allreduce_weight_grad(dU_t)
        got = {k: (v.numpy() if v is not None else None) for k, v in
               (("x_prev", x_prev), ("dy_next", dy_next), ("z_next", z_next))}
        out[rank] = (tok.start, tok.stop, got, y, dx, dz[:, h:], dU_t.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharded_step_matches_unsharded(world):
    import oracle
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_sp_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    f = _seq_batch(world)
    ry = oracle.fwd_lowrank(f["x"], f["z"], f["U"], SG, SW)
    rdx, rdz, rdU = oracle.bwd_lowrank(f["x"], f["z"], f["U"], f["dy"], SG, SW)
    h = SW - 1
    for rank in range(world):
        lo, hi, got, y, dx, dz, dU = out[rank]
        assert (lo, hi) == (rank * ST, (rank + 1) * ST)
        # the halos are the neighbours' rows, exactly
        if rank == 0:
            assert got["x_prev"] is None
        else:
            np.testing.assert_array_equal(got["x_prev"], f["x"][:, lo - h:lo])
        if rank == world - 1:
            assert got["dy_next"] is None and got["z_next"] is None
        else:
            np.testing.assert_array_equal(got["dy_next"], f["dy"][:, hi:hi + h])
            np.testing.assert_array_equal(got["z_next"], f["z"][:, hi:hi + h])
        np.testing.assert_allclose(y, ry[:, lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dx, rdx[:, lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dz, rdz[:, lo:hi], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dU, rdU, rtol=1e-12, atol=1e-12)


def test_shard_shorter_than_halo_is_rejected():
    """A one-hop halo needs shards of at least W-1 tokens; shorter ones fail before any
    message is sent."""
    from dynamic_short_convolutions_causal_b200 import sp
    x = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        sp.exchange_prev(x, 4, seq_ranks=[0, 1])
    with pytest.raises(ValueError):
        sp.exchange_next(x, torch.zeros(1, 2, 3), 4, seq_ranks=[0, 1])
    with pytest.raises(ValueError):
        sp.shard_tokens(10, 0, 3)
