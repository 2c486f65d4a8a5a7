"""dsc_static_bwd_noalloc: the static-convolution backward for callers that cannot
allocate device memory (it takes its scratch from a fixed array inside the library).

Checked through the C ABI against dsc_static_bwd with a caller-provided workspace, on
two calls in a row (the array keeps the previous call's contents, which must not
leak into the next result).  Collected last so that a run stopping at the first
failure has already run every other test."""
import ctypes

import pytest
import torch

import dsc_inputs as di
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dynamic_short_convolutions_causal_b200 as m
    return m


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(dsc, x, w, dy, dx, dw):
    B, T, D = x.shape
    st = dsc.lib.dsc_static_bwd_noalloc(_p(x), _p(w), _p(dy), _p(dx), _p(dw), B, T, D, w.shape[-1],
                                        dsc._dt(x), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("B,T,D,W,dt", [(2, 300, 192, 4, "bf16"), (2, 8192, 8192, 8, "bf16"),
                                        (3, 70, 32, 3, "f32")])
def test_noalloc_matches_workspace_version_twice(dsc, B, T, D, W, dt):
    need = dsc.dsc_static_bwd_workspace_bytes(B, T, D, W, di.torch_dtype(dt))
    assert need <= dsc.lib.dsc_static_bwd_noalloc_max_scratch_bytes()
    for call, seed in enumerate((5, 6)):            # two calls in a row, different inputs
        t = di.make(di.small(B, T, D, 1, W, 0, dt, seed=seed), "cuda", ("x", "dy", "ws"))
        x, dy, w = t["x"], t["dy"], t["ws"]
        ref_dx = torch.empty_like(x)
        ref_dw = torch.empty((D, W), dtype=torch.float32, device="cuda")
        ws = dsc.workspace(need, "cuda")
        dsc.dsc_static_bwd(x, w, dy, ref_dx, ref_dw, ws)
        dx = torch.full_like(x, float("nan"))
        dw = torch.full((D, W), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(dsc, x, w, dy, dx, dw) == 0, dsc.lib.dsc_last_error()
        torch.cuda.synchronize()
        assert_close(dx, ref_dx.double().cpu().numpy(), dt, "dx (call %d)" % call)
        assert_close(dw, ref_dw.double().cpu().numpy(), dt, "dw (call %d)" % call, reduction=True)


def test_noalloc_rejects_sizes_beyond_the_array(dsc):
    B, T, D, W = 16, 8192, 8192, 8         # needs 64 MiB of partials
    need = dsc.dsc_static_bwd_workspace_bytes(B, T, D, W, torch.bfloat16)
    assert need > dsc.lib.dsc_static_bwd_noalloc_max_scratch_bytes()
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")   # never touched: rejected first
    st = dsc.lib.dsc_static_bwd_noalloc(_p(x), _p(x), _p(x), _p(x), _p(x), B, T, D, W, 1, None)
    assert st == 2
    assert b"scratch" in dsc.lib.dsc_last_error()
