"""The tensor-core kernels' give-up path, exercised without faulting or hanging anything.

Every wait in those kernels is bounded; a wait that runs out makes the CTA record a
fault code, leave its loops, let its in-flight copies land and free its tensor memory.
dsc_test_arm_wait_timeout() makes one launch withhold a tile's loads with a short wait
limit, so a consumer's wait runs out.  The call must return, the fault word must be set
and then clear, and the next ordinary call must be correct."""
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


B, T, D, G, W, R = 2, 300, 192, 1, 4, 32


def _inputs():
    return {k: v.cuda() for k, v in di.make(di.small(B, T, D, G, W, R, "bf16", seed=21), "cpu",
                                            ("x", "z", "U", "dy")).items()}


def _fwd(dsc, t):
    y = torch.empty_like(t["x"])
    dsc.dsc_fwd_lowrank(t["x"], t["z"], t["U"], y, G, W)
    return y


def _bwd(dsc, t):
    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R), "cuda")
    dx = torch.empty_like(t["x"])
    dz = torch.empty((B, T, R), dtype=torch.float32, device="cuda")
    dU = torch.empty((R, D * W), dtype=torch.float32, device="cuda")
    dsc.dsc_bwd_lowrank(t["x"], t["z"], t["U"], t["dy"], dx, dz, dU, ws, G, W)
    return dx, dz, dU


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_wait_runs_out_and_the_next_call_is_correct(dsc, which):
    assert dsc.dsc_lowrank_path(B, T, D, G, W, R) == 3
    assert dsc.dsc_device_fault(True) == 0
    t = _inputs()
    dsc.lib.dsc_test_arm_wait_timeout(2000)          # 2 ms limit, one tile withheld
    (_fwd if which == "fwd" else _bwd)(dsc, t)       # returns; outputs undefined
    torch.cuda.synchronize()
    assert dsc.dsc_device_fault(True) != 0, "the withheld tile should make a wait run out"
    assert dsc.dsc_device_fault() == 0, "the fault word clears on reset"
    f = lambda a: f64(a)
    if which == "fwd":
        assert_close(_fwd(dsc, t), oracle.fwd_lowrank(f(t["x"]), f(t["z"]), f(t["U"]), G, W), "bf16", "y")
    else:
        dx, dz, dU = _bwd(dsc, t)
        rdx, rdz, rdU = oracle.bwd_lowrank(f(t["x"]), f(t["z"]), f(t["U"]), f(t["dy"]), G, W)
        assert_close(dx, rdx, "bf16", "dx")
        assert_close(dz, rdz, "bf16", "dz", reduction=True)
        assert_close(dU, rdU, "bf16", "dU", reduction=True)
    torch.cuda.synchronize()
    assert dsc.dsc_device_fault() == 0
