"""RoPE fused with the low-rank op (dsc_fwd_lowrank_rope / dsc_bwd_lowrank_rope) against
the oracle's rotated op, element by element, on seeded inputs on the tensor-core path:
the rotated channel range covering part of D (Q and K of a stacked [Q | K | V]), all of
it, or none; heads of 16 to 128 channels; ragged tails and several slices."""
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


def rope_table(T, dh, base=10000.0):
    """(cos, sin) of the standard RoPE angles t * base^(-2i/dh), fp32 [T, dh/2, 2] (the
    oracle's layout; the library takes it pair-major, [dh/2, T, 2])."""
    inv = base ** (-np.arange(0, dh, 2, dtype=np.float64) / dh)
    th = np.arange(T, dtype=np.float64)[:, None] * inv[None, :]
    return torch.from_numpy(np.stack([np.cos(th), np.sin(th)], axis=-1).astype(np.float32))


CASES = [
    # B, T, D, G, W, R, dh, n_rot
    (2, 300, 192, 1, 4, 32, 64, 128),       # Q, K rotated, V not
    (1, 260, 256, 4, 8, 64, 32, 128),
    (2, 129, 128, 1, 3, 16, 128, 128),      # every channel rotated
    (2, 200, 384, 2, 4, 32, 128, 256),      # two thirds, as in a stacked QKV
    (1, 77, 128, 16, 2, 32, 16, 64),        # grouped filters, small heads
    (2, 150, 128, 1, 4, 32, 64, 0),         # nothing rotated: the plain op
    (1, 140, 128, 1, 6, 16, 32, 128),       # 6 taps: products stored as computed
    (2, 100, 256, 32, 4, 32, 64, 128),      # one filter per 32 channels (virtual groups)
]


@pytest.mark.parametrize("B,T,D,G,W,R,dh,n_rot", CASES)
def test_lowrank_rope_fwd_bwd(dsc, B, T, D, G, W, R, dh, n_rot):
    assert dsc.dsc_lowrank_path(B, T, D, G, W, R) == 3
    wl = di.small(B, T, D, G, W, R, "bf16", seed=900 + T)
    t = {k: v.to(DEV) for k, v in di.make(wl, "cpu", ("x", "z", "U", "dy")).items()}
    x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
    cs_t = rope_table(T, dh)
    cs = cs_t.permute(1, 0, 2).contiguous().to(DEV)
    y = torch.full_like(x, float("nan"))
    dsc.dsc_fwd_lowrank_rope(x, z, U, cs, y, G, W, dh, n_rot)
    torch.cuda.synchronize()
    csd = f64(cs_t)
    assert_close(y, oracle.fwd_lowrank_rope(f64(x), f64(z), f64(U), csd, G, W, dh, n_rot), "bf16", "y")
    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R), DEV)
    dx = torch.full_like(x, float("nan"))
    dz = torch.full((B, T, R), float("nan"), dtype=torch.float32, device=DEV)
    dU = torch.full((R, (D // G) * W), float("nan"), dtype=torch.float32, device=DEV)
    dsc.dsc_bwd_lowrank_rope(x, z, U, cs, dy, dx, dz, dU, ws, G, W, dh, n_rot)
    torch.cuda.synchronize()
    rdx, rdz, rdU = oracle.bwd_lowrank_rope(f64(x), f64(z), f64(U), csd, f64(dy), G, W, dh, n_rot)
    assert_close(dx, rdx, "bf16", "dx")
    assert_close(dz, rdz, "bf16", "dz", reduction=True)
    assert_close(dU, rdU, "bf16", "dU", reduction=True)


def test_rope_off_equals_plain_op(dsc):
    """n_rot = 0 gives exactly the plain entry points' results."""
    B, T, D, G, W, R = 2, 140, 128, 1, 4, 32
    t = {k: v.to(DEV) for k, v in di.make(di.small(B, T, D, G, W, R, "bf16", seed=5), "cpu",
                                          ("x", "z", "U", "dy")).items()}
    cs = rope_table(T, 64).permute(1, 0, 2).contiguous().to(DEV)
    y0 = torch.empty_like(t["x"])
    y1 = torch.empty_like(t["x"])
    dsc.dsc_fwd_lowrank(t["x"], t["z"], t["U"], y0, G, W)
    dsc.dsc_fwd_lowrank_rope(t["x"], t["z"], t["U"], cs, y1, G, W, 64, 0)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
