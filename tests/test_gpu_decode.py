"""GPU parity of the decode step (one new token per sequence with a rolling window of
the W-1 previous inputs) against the CPU oracle, through the C ABI: single steps
from random windows, and sequences stepped token by token from a zero window."""
import numpy as np
import pytest
import torch

import dsc_inputs as di
import oracle
from parity import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dynamic_short_convolutions_causal_b200 as m
    return m


DEV = "cuda"


def _draw(shape, std, dt, gen):
    return (torch.randn(shape, generator=gen) * std).to(di.torch_dtype(dt))


DECODE = [
    # B, D, G, W, R, dtype
    # CUDA cores (fewer than 8 sequences, or shapes the tensor-core kernel does not take)
    (1, 6144, 1, 4, 32, "bf16"),       # the stacked-QKV width, one sequence
    (8, 6144, 1, 4, 32, "bf16"),       # from here on bf16 with D % 64 == 0: tensor cores
    (64, 256, 4, 8, 64, "bf16"),
    (37, 96, 3, 5, 8, "bf16"),         # ragged sequence block, G not a power of two
    (3, 40, 8, 3, 16, "f32"),          # D not a multiple of the 32-channel block
    (5, 64, 1, 1, 4, "bf16"),          # W = 1: no window
    (2, 128, 64, 2, 48, "bf16"),
    # up to 4 sequences with rank <= 32: U read straight from global memory
    (4, 256, 4, 2, 8, "f32"),
    (2, 512, 16, 4, 16, "bf16"),
    (2, 96, 1, 4, 8, "bf16"),          # a last block of 32 channels
    (3, 104, 1, 4, 24, "bf16"),        # a last block of 40 channels
    (4, 128, 2, 8, 32, "f32"),         # 8 taps, fp32
    (2, 64, 1, 1, 16, "bf16"),         # W = 1: no window
    # tensor-core decode (the forward kernel with one row per sequence)
    (256, 6144, 1, 4, 32, "bf16"),     # two full 128-sequence tiles
    (130, 128, 2, 8, 16, "bf16"),      # a ragged second tile, W = 8
    (200, 512, 8, 3, 64, "bf16"),
    (129, 192, 16, 6, 32, "bf16"),
    (33, 128, 1, 2, 16, "bf16"),       # W = 2: the window is x_t alone
    (40, 64, 1, 1, 16, "bf16"),        # W = 1
]


@pytest.mark.parametrize("B,D,G,W,R,dt", DECODE)
def test_decode_step_matches_oracle(dsc, B, D, G, W, R, dt):
    gen = torch.Generator().manual_seed(B * 7 + D + W)
    N = (D // G) * W
    x = _draw((B, D), 1.0, dt, gen)
    z = _draw((B, R), 1.0, dt, gen)
    U = _draw((R, N), R ** -0.5, dt, gen)
    w = _draw((B, D // G, W), 0.5, dt, gen)
    st0 = _draw((B, W - 1, D), 1.0, dt, gen)
    for lowrank in (True, False):
        xs, st = x.to(DEV), st0.clone().to(DEV)
        y = torch.full_like(xs, float("nan"))
        if lowrank:
            dsc.dsc_decode_step_lowrank(xs, z.to(DEV), U.to(DEV), st if W > 1 else None, y, G, W)
            ry, rst = oracle.decode_lowrank(f64(x), f64(z), f64(U), f64(st0), G, W)
        else:
            dsc.dsc_decode_step(xs, w.to(DEV), st if W > 1 else None, y, G)
            ry, rst = oracle.decode(f64(x), f64(w), f64(st0), G)
        torch.cuda.synchronize()
        assert_close(y, ry, dt, "y_t (lowrank=%s)" % lowrank)
        # the window moves by exact copies: bitwise
        assert np.array_equal(f64(st), rst), "window after the step (lowrank=%s)" % lowrank


@pytest.mark.parametrize("B,T,D,G,W,R", [(3, 20, 128, 2, 4, 16), (2, 9, 64, 1, 7, 32), (9, 12, 128, 1, 4, 32),
                                         (130, 6, 64, 4, 5, 16)])
def test_decode_steps_reproduce_forward(dsc, B, T, D, G, W, R):
    """Stepping from a zero window through T tokens gives the fused forward's outputs."""
    wl = di.small(B, T, D, G, W, R, "bf16", seed=T)
    t = {k: v.to(DEV) for k, v in di.make(wl, "cpu", ("x", "z", "U")).items()}
    y_ref = torch.empty_like(t["x"])
    dsc.dsc_fwd_lowrank(t["x"], t["z"], t["U"], y_ref, G, W)
    st = torch.zeros((B, W - 1, D), dtype=t["x"].dtype, device=DEV)
    ys = []
    for s in range(T):
        y = torch.empty((B, D), dtype=t["x"].dtype, device=DEV)
        dsc.dsc_decode_step_lowrank(t["x"][:, s].contiguous(), t["z"][:, s].contiguous(), t["U"], st, y, G, W)
        ys.append(y)
    torch.cuda.synchronize()
    yd = torch.stack(ys, dim=1)
    ro = oracle.fwd_lowrank(f64(t["x"]), f64(t["z"]), f64(t["U"]), G, W)
    assert_close(yd, ro, "bf16", "stepped y")
    assert_close(y_ref, ro, "bf16", "forward y")
    assert np.array_equal(f64(st), f64(t["x"][:, T - (W - 1):])), "window holds the last W-1 inputs"
