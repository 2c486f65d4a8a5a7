"""The chunked whole-tensor oracle driver (tests/fullsize.py) against the oracle run
on the whole problem at once, on small inputs, so that its chunking, causal halos and
zeroed-dy sums are checked before the GPU tests rely on it at the full sizes."""
import numpy as np
import pytest
import torch

import dsc_inputs as di
import fullsize
import oracle


def _f(t):
    return t.to(torch.float64).numpy()


@pytest.mark.parametrize("B,T,D,G,W,R,chunk", [(2, 37, 16, 1, 4, 5, 8), (1, 50, 24, 4, 8, 3, 7),
                                               (2, 9, 8, 2, 3, 2, 16), (1, 12, 8, 1, 1, 2, 5)])
def test_lowrank_chunks_equal_whole(B, T, D, G, W, R, chunk):
    t = di.make(di.small(B, T, D, G, W, R, "bf16", seed=T), "cpu", ("x", "z", "U", "dy"))
    y, dx, dz, dU = fullsize.lowrank(t["x"], t["z"], t["U"], t["dy"], G, W, chunk=chunk)
    ry = oracle.fwd_lowrank(_f(t["x"]), _f(t["z"]), _f(t["U"]), G, W)
    rdx, rdz, rdU = oracle.bwd_lowrank(_f(t["x"]), _f(t["z"]), _f(t["U"]), _f(t["dy"]), G, W)
    np.testing.assert_allclose(y, ry, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(dx, rdx, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(dz, rdz, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(dU, rdU, rtol=1e-12, atol=1e-12)


def test_explicit_chunks_equal_whole():
    t = di.make(di.small(2, 41, 16, 4, 5, 0, "bf16", seed=1), "cpu", ("x", "w"))
    y = fullsize.explicit_fwd(t["x"], t["w"], 4, chunk=6)
    np.testing.assert_allclose(y, oracle.fwd(_f(t["x"]), _f(t["w"]), 4), rtol=1e-6, atol=1e-6)


def test_static_chunks_equal_whole():
    t = di.make(di.small(2, 33, 16, 1, 6, 0, "bf16", seed=2), "cpu", ("x", "dy", "ws"))
    y, dx, dw = fullsize.static(t["x"], t["ws"], t["dy"], chunk=5)
    ry = oracle.static_fwd(_f(t["x"]), _f(t["ws"]))
    rdx, rdw = oracle.static_bwd(_f(t["x"]), _f(t["ws"]), _f(t["dy"]))
    np.testing.assert_allclose(y, ry, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(dx, rdx, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(dw, rdw, rtol=1e-12, atol=1e-12)
