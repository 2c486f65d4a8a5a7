"""Sequence sharding on one GPU: a sequence of P*T tokens is split into P shards of T,
each shard runs through dsc_fwd_lowrank / dsc_bwd_lowrank as if it were a whole
sequence, then through the halo fix-ups (dsc_fwd_lowrank_halo / dsc_bwd_lowrank_halo)
with the (W-1)-row halos cut from the whole tensors (what the neighbouring ranks would
send).  Reassembled, y, dx and dz, and dU summed over the shards, must match the oracle
on the whole sequence.  The shards run one after another: no kernel waits on another."""
import numpy as np
import pytest
import torch

import dsc_inputs as di
import oracle
from parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def dsc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dynamic_short_convolutions_causal_b200 as m
    return m


CASES = [
    # B, P, T (shard), D, G, W, R, dtype
    (2, 2, 100, 128, 1, 4, 32, "bf16"),     # tensor-core kernels on each shard
    (2, 3, 70, 192, 4, 8, 64, "bf16"),
    (1, 2, 300, 256, 64, 3, 16, "bf16"),
    (1, 4, 2, 64, 1, 4, 16, "bf16"),        # shards shorter than W-1: halos span shards
    (2, 3, 37, 48, 3, 5, 8, "f32"),         # CUDA-core kernels
    (2, 2, 20, 64, 2, 1, 8, "bf16"),        # W = 1: nothing to fix
]


def _rows(t, lo, hi):
    """Rows [lo, hi) of t [B, L, C] along the sequence, zero outside [0, L)."""
    B, L, C = t.shape
    out = torch.zeros((B, hi - lo, C), dtype=t.dtype, device=t.device)
    a, b = max(lo, 0), min(hi, L)
    if a < b:
        out[:, a - lo:b - lo] = t[:, a:b]
    return out.contiguous()


@pytest.mark.parametrize("B,P,T,D,G,W,R,dt", CASES)
def test_sequence_shards_match_whole_sequence(dsc, B, P, T, D, G, W, R, dt):
    wl = di.small(B, P * T, D, G, W, R, dt, seed=500 + P * T)
    t = {k: v.to(DEV) for k, v in di.make(wl, "cpu", ("x", "z", "U", "dy")).items()}
    x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
    h = W - 1
    ys, dxs, dzs = [], [], []
    dU = torch.zeros((R, (D // G) * W), dtype=torch.float32, device=DEV)
    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R, x.dtype), DEV)
    for r in range(P):
        lo, hi = r * T, (r + 1) * T
        xs, zs, dys = (a[:, lo:hi].contiguous() for a in (x, z, dy))
        x_prev = _rows(x, lo - h, lo) if (r > 0 and h > 0) else None
        dy_next = _rows(dy, hi, hi + h) if (r < P - 1 and h > 0) else None
        z_next = _rows(z, hi, hi + h) if (r < P - 1 and h > 0) else None
        y = torch.full_like(xs, float("nan"))
        dsc.dsc_fwd_lowrank(xs, zs, U, y, G, W)
        dsc.dsc_fwd_lowrank_halo(xs, zs, U, x_prev, y, G, W)
        dx = torch.full_like(xs, float("nan"))
        dz = torch.full((B, T, R), float("nan"), dtype=torch.float32, device=DEV)
        dUs = torch.full_like(dU, float("nan"))
        dsc.dsc_bwd_lowrank(xs, zs, U, dys, dx, dz, dUs, ws, G, W)
        dsc.dsc_bwd_lowrank_halo(x_prev, zs, U, dys, dy_next, z_next, dx, dz, dUs, G, W)
        ys.append(y)
        dxs.append(dx)
        dzs.append(dz)
        dU += dUs
    torch.cuda.synchronize()
    ry = oracle.fwd_lowrank(f64(x), f64(z), f64(U), G, W)
    rdx, rdz, rdU = oracle.bwd_lowrank(f64(x), f64(z), f64(U), f64(dy), G, W)
    assert_close(torch.cat(ys, 1), ry, dt, "y")
    assert_close(torch.cat(dxs, 1), rdx, dt, "dx")
    assert_close(torch.cat(dzs, 1), rdz, dt, "dz", reduction=True)
    assert_close(dU, rdU, dt, "dU", reduction=True)


def test_halo_calls_reject_a_lone_next_halo(dsc):
    B, T, D, G, W, R = 1, 8, 64, 1, 4, 16
    z = torch.zeros((B, T, R), dtype=torch.bfloat16, device=DEV)
    U = torch.zeros((R, D * W), dtype=torch.bfloat16, device=DEV)
    dy = torch.zeros((B, T, D), dtype=torch.bfloat16, device=DEV)
    dx = torch.zeros_like(dy)
    dz = torch.zeros((B, T, R), dtype=torch.float32, device=DEV)
    dU = torch.zeros((R, D * W), dtype=torch.float32, device=DEV)
    dyn = torch.zeros((B, W - 1, D), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(dsc.DscError):
        dsc.dsc_bwd_lowrank_halo(None, z, U, dy, dyn, None, dx, dz, dU, G, W)
