"""GPU parity: every entry point of libdsc.so against the CPU oracle, element by
element, on seeded inputs (sizes that span several tiles, ragged tails, edge cases),
and every output tensor whole at the full workload sizes.

All calls go through the C ABI (the binding only marshals arguments)."""
import numpy as np
import pytest
import torch

import dsc_inputs as di
import oracle
import fullsize
from parity import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsc():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import dynamic_short_convolutions_causal_b200 as m
    return m


DEV = "cuda"


def _guarded(shape, dtype, fill=float("nan"), guard=256):
    """An output tensor inside a larger buffer whose guard bands hold a canary."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * guard,), fill, dtype=dtype, device=DEV)
    buf[:guard] = 4096.0
    buf[-guard:] = 4096.0
    return buf, buf[guard:guard + n].view(*shape)


def _check_guard(buf, guard=256):
    assert torch.all(buf[:guard] == 4096.0) and torch.all(buf[-guard:] == 4096.0), \
        "a kernel wrote outside its output"


def _gen(wl, parts):
    return {k: v.to(DEV) for k, v in di.make(wl, "cpu", parts).items()}


# ------------------------------------------------------------------ explicit filters
EXPLICIT = [
    # B, T, D, G, W, dtype
    (1, 64, 64, 8, 4, "f32"),          # the small fp32 workload's shape
    (2, 300, 192, 1, 4, "bf16"),
    (3, 77, 256, 64, 3, "bf16"),
    (1, 5, 64, 8, 8, "bf16"),
    (2, 1, 16, 2, 1, "bf16"),
    (2, 45, 24, 3, 5, "bf16"),
    (2, 33, 96, 96, 2, "f32"),
    (1, 130, 40, 5, 7, "f32"),
    # one-pass explicit backward, packed bf16: ring windows with a ragged last chunk
    # (W=4: the open rows' slots depend on T mod 4; W=2), and shifted windows (W=8)
    (1, 131, 128, 16, 4, "bf16"),
    (2, 260, 64, 8, 2, "bf16"),
    (2, 300, 128, 8, 8, "bf16"),
]


@pytest.mark.parametrize("B,T,D,G,W,dt", EXPLICIT)
def test_explicit_fwd_bwd(dsc, B, T, D, G, W, dt):
    wl = di.small(B, T, D, G, W, 0, dt, seed=B * 1000 + T)
    t = _gen(wl, ("x", "w", "dy"))
    buf, y = _guarded((B, T, D), t["x"].dtype)
    dsc.dsc_fwd(t["x"], t["w"], y, G)
    torch.cuda.synchronize()
    _check_guard(buf)
    assert_close(y, oracle.fwd(f64(t["x"]), f64(t["w"]), G), dt, "y")
    bdx, dx = _guarded((B, T, D), t["x"].dtype)
    bdw, dw = _guarded((B, T, D // G, W), torch.float32)
    dsc.dsc_bwd(t["x"], t["w"], t["dy"], dx, dw, G)
    torch.cuda.synchronize()
    _check_guard(bdx)
    _check_guard(bdw)
    rdx, rdw = oracle.bwd(f64(t["x"]), f64(t["w"]), f64(t["dy"]), G)
    assert_close(dx, rdx, dt, "dx")
    assert_close(dw, rdw, dt, "dw", reduction=True)


def test_small_fp32_workload_exact_bound(dsc):
    """The fp32 explicit workload (seed 0) at its full size: max|err| <= 1e-5."""
    wl = di.WORKLOADS["explicit_fp32_small"]
    t = _gen(wl, ("x", "w"))
    y = torch.empty_like(t["x"])
    dsc.dsc_fwd(t["x"], t["w"], y, wl.G)
    ref = oracle.fwd(f64(t["x"]), f64(t["w"]), wl.G)
    assert np.max(np.abs(f64(y) - ref)) <= 1e-5


# ------------------------------------------------------------------ static filters
STATIC = [
    (2, 300, 192, 4, "bf16"), (1, 1000, 64, 8, "bf16"), (2, 3, 16, 5, "bf16"),
    (3, 70, 32, 1, "f32"), (2, 257, 128, 3, "f32"),
]


@pytest.mark.parametrize("B,T,D,W,dt", STATIC)
def test_static_fwd_bwd(dsc, B, T, D, W, dt):
    wl = di.small(B, T, D, 1, W, 0, dt, seed=7 + T)
    t = _gen(wl, ("x", "dy", "ws"))
    buf, y = _guarded((B, T, D), t["x"].dtype)
    dsc.dsc_static_fwd(t["x"], t["ws"], y)
    torch.cuda.synchronize()
    _check_guard(buf)
    assert_close(y, oracle.static_fwd(f64(t["x"]), f64(t["ws"])), dt, "y")
    dx = torch.full_like(t["x"], float("nan"))
    dw = torch.full((D, W), float("nan"), dtype=torch.float32, device=DEV)
    ws = dsc.workspace(dsc.dsc_static_bwd_workspace_bytes(B, T, D, W, t["x"].dtype), DEV)
    dsc.dsc_static_bwd(t["x"], t["ws"], t["dy"], dx, dw, ws)
    rdx, rdw = oracle.static_bwd(f64(t["x"]), f64(t["ws"]), f64(t["dy"]))
    assert_close(dx, rdx, dt, "dx")
    assert_close(dw, rdw, dt, "dw", reduction=True)


# ------------------------------------------------------------------ low-rank
LOWRANK = [
    # B, T, D, G, W, R, dtype
    (2, 300, 192, 1, 4, 32, "bf16"),
    (2, 257, 256, 4, 8, 64, "bf16"),
    (1, 130, 128, 2, 3, 16, "bf16"),
    (3, 50, 64, 64, 2, 16, "bf16"),
    (2, 200, 128, 1, 4, 1, "bf16"),
    (1, 9, 64, 1, 5, 3, "bf16"),
    (2, 3, 64, 1, 4, 32, "bf16"),
    (1, 1, 64, 2, 6, 32, "bf16"),
    (2, 140, 320, 8, 7, 48, "bf16"),
    (2, 70, 64, 1, 4, 32, "f32"),
    (1, 100, 48, 3, 3, 8, "f32"),
    # shapes aimed at the tensor-core kernels
    (1, 4096, 2048, 1, 4, 16, "bf16"),   # many tiles per CTA: ring wrap-around, slice changes
    (2, 1000, 512, 1, 8, 64, "bf16"),    # 512 filter columns: two MMA N-chunks, one accumulator
    (2, 300, 256, 16, 2, 32, "bf16"),    # G = 16
    (2, 129, 128, 32, 4, 64, "bf16"),    # G = 32
    (1, 200, 128, 64, 8, 32, "bf16"),    # G = 64
    (2, 77, 128, 8, 1, 16, "bf16"),      # W = 1
    (3, 2048, 384, 2, 3, 32, "bf16"),    # G = 2, W = 3
    (2, 500, 256, 4, 4, 16, "bf16"),     # backward: 64 filter columns, padded dU^T block
    (2, 260, 128, 1, 3, 32, "bf16"),     # backward: 192 filter columns, padded dU^T block
    (1, 300, 128, 2, 8, 32, "bf16"),     # backward: G = 2, W = 8
    # tensor-core backward with grouped filters (tap blocks padded to 16 columns; for
    # G >= 32 one virtual group per 16 channels, summed into dU)
    (2, 500, 512, 64, 4, 32, "bf16"),
    (2, 300, 384, 32, 3, 16, "bf16"),
    (1, 260, 256, 8, 5, 64, "bf16"),
    (2, 129, 192, 16, 8, 64, "bf16"),
    (3, 70, 128, 8, 2, 16, "bf16"),
]


@pytest.mark.parametrize("B,T,D,G,W,R,dt", LOWRANK)
def test_lowrank_fwd_bwd(dsc, B, T, D, G, W, R, dt):
    wl = di.small(B, T, D, G, W, R, dt, seed=R * 100 + T)
    t = _gen(wl, ("x", "z", "U", "dy"))
    x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
    buf, y = _guarded((B, T, D), x.dtype)
    dsc.dsc_fwd_lowrank(x, z, U, y, G, W)
    torch.cuda.synchronize()
    _check_guard(buf)
    assert_close(y, oracle.fwd_lowrank(f64(x), f64(z), f64(U), G, W), dt, "y")

    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R, x.dtype), DEV)
    bdx, dx = _guarded((B, T, D), x.dtype)
    bdz, dz = _guarded((B, T, R), torch.float32)
    bdU, dU = _guarded((R, (D // G) * W), torch.float32)
    dsc.dsc_bwd_lowrank(x, z, U, dy, dx, dz, dU, ws, G, W)
    torch.cuda.synchronize()
    for b in (bdx, bdz, bdU):
        _check_guard(b)
    rdx, rdz, rdU = oracle.bwd_lowrank(f64(x), f64(z), f64(U), f64(dy), G, W)
    assert_close(dx, rdx, dt, "dx")
    assert_close(dz, rdz, dt, "dz", reduction=True)
    assert_close(dU, rdU, dt, "dU", reduction=True)


def test_tensor_core_path_is_selected(dsc):
    """The bf16 workloads of the benchmark run on the tcgen05 kernels (forward: bit 0,
    backward: bit 1)."""
    for name in ("lowrank_qkv", "lowrank_mlp"):
        wl = di.WORKLOADS[name]
        assert dsc.dsc_lowrank_path(wl.B, wl.T, wl.D, wl.G, wl.W, wl.R) == 3, name


def test_grouped_filters_take_the_tensor_core_backward(dsc):
    """G = 8..64 with R in {16, 32, 64} and D a multiple of 64: the tcgen05 backward
    (bit 1), which keeps w and dw on chip."""
    for (B, T, D, G, W, R) in [(2, 500, 512, 64, 4, 32), (2, 300, 384, 32, 3, 16), (1, 260, 256, 8, 5, 64),
                               (2, 129, 192, 16, 8, 64), (2, 300, 256, 16, 2, 32), (1, 200, 128, 64, 8, 32)]:
        assert dsc.dsc_lowrank_path(B, T, D, G, W, R) & 2, (B, T, D, G, W, R)


def test_no_device_fault_recorded(dsc):
    assert dsc.dsc_device_fault() == 0


def test_lowrank_deterministic(dsc):
    B, T, D, G, W, R = 2, 300, 192, 1, 4, 32
    t = _gen(di.small(B, T, D, G, W, R, "bf16", seed=3), ("x", "z", "U", "dy"))
    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R), DEV)
    outs = []
    for _ in range(2):
        y = torch.empty_like(t["x"])
        dx = torch.empty_like(t["x"])
        dz = torch.empty((B, T, R), dtype=torch.float32, device=DEV)
        dU = torch.empty((R, D * W), dtype=torch.float32, device=DEV)
        dsc.dsc_fwd_lowrank(t["x"], t["z"], t["U"], y, G, W)
        dsc.dsc_bwd_lowrank(t["x"], t["z"], t["U"], t["dy"], dx, dz, dU, ws, G, W)
        outs.append((y, dx, dz, dU))
    # y, dx and dU are summed in fixed orders; dz of the tensor-core backward adds the
    # slice groups' sums with fp32 reductions in L2, in arrival order
    for name, a, b in zip(("y", "dx", "dz", "dU"), *outs):
        if name == "dz" and dsc.dsc_lowrank_path(B, T, D, G, W, R) & 2:
            assert torch.max(torch.abs(a - b)) <= 1e-5 * torch.max(torch.abs(a)), "dz differs beyond rounding"
        else:
            assert torch.equal(a, b), "repeated call differs bitwise: " + name


def test_failed_call_launches_nothing(dsc):
    x = torch.randn(2, 8, 64, device=DEV, dtype=torch.bfloat16)
    w = torch.randn(2, 8, 64, 9, device=DEV, dtype=torch.bfloat16)   # W = 9: unsupported
    y = torch.full_like(x, float("nan"))
    with pytest.raises(dsc.DscError):
        dsc.dsc_fwd(x, w, y, 1)
    torch.cuda.synchronize()
    assert torch.isnan(y).all()


# ------------------------------------------------------------------ full sizes, whole tensors
# Every output tensor is compared with the oracle element by element at the workload's
# full size, in the launch configuration the benchmark times.  The oracle runs on token
# chunks with their causal halos (tests/fullsize.py), which gives each chunk's outputs
# exactly; the reported numbers are the per-tensor errors of the stated tolerance rule.
def _report(name, errs):
    print("full-size parity %s: %s" % (name, ", ".join("%s %.3e" % kv for kv in errs.items())))


@pytest.mark.parametrize("name", ["tied_qkv"])
def test_full_size_explicit_fwd(dsc, name):
    wl = di.WORKLOADS[name]
    t = di.make(wl, DEV, ("x", "w"))
    y = torch.empty_like(t["x"])
    dsc.dsc_fwd(t["x"], t["w"], y, wl.G)
    torch.cuda.synchronize()
    h = {k: v.cpu() for k, v in t.items()}
    yh = y.cpu()
    del t, y
    torch.cuda.empty_cache()
    ry = fullsize.explicit_fwd(h["x"], h["w"], wl.G)
    _report(name, {"y": assert_close(yh, ry, wl.dtype, "y")})


@pytest.mark.parametrize("name", ["lowrank_qkv", "lowrank_mlp"])
def test_full_size_lowrank(dsc, name):
    wl = di.WORKLOADS[name]
    G, W, R = wl.G, wl.W, wl.R
    t = di.make(wl, DEV, ("x", "z", "U", "dy"))
    x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
    y = torch.empty_like(x)
    dsc.dsc_fwd_lowrank(x, z, U, y, G, W)
    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(wl.B, wl.T, wl.D, G, W, R), DEV)
    dx = torch.empty_like(x)
    dz = torch.empty((wl.B, wl.T, R), dtype=torch.float32, device=DEV)
    dU = torch.empty((R, wl.N), dtype=torch.float32, device=DEV)
    dsc.dsc_bwd_lowrank(x, z, U, dy, dx, dz, dU, ws, G, W)
    torch.cuda.synchronize()
    assert dsc.dsc_device_fault() == 0
    h = {k: v.cpu() for k, v in t.items()}
    g = {"y": y.cpu(), "dx": dx.cpu(), "dz": dz.cpu(), "dU": dU.cpu()}
    del t, x, z, U, dy, y, dx, dz, dU, ws
    torch.cuda.empty_cache()
    ry, rdx, rdz, rdU = fullsize.lowrank(h["x"], h["z"], h["U"], h["dy"], G, W)
    errs = {"y": assert_close(g["y"], ry, wl.dtype, "y"),
            "dx": assert_close(g["dx"], rdx, wl.dtype, "dx"),
            "dz": assert_close(g["dz"], rdz, wl.dtype, "dz", reduction=True),
            "dU": assert_close(g["dU"], rdU, wl.dtype, "dU", reduction=True)}
    _report(name, errs)
    # invariant: sum(dU * U) == sum(dz * z) (both are sum_t <dw_t, w_t>)
    pu = g["dU"].double() * h["U"].double()
    pz = g["dz"].double() * h["z"].double()
    a, bsum = float(pu.sum()), float(pz.sum())
    scale = float(pu.abs().sum()) + float(pz.abs().sum())
    assert abs(a - bsum) <= 1e-3 * scale, (a, bsum, scale)


def test_full_size_static(dsc):
    wl = di.WORKLOADS["lowrank_mlp"]
    t = di.make(wl, DEV, ("x", "dy", "ws"))
    x, dy, w = t["x"], t["dy"], t["ws"]
    y = torch.empty_like(x)
    dsc.dsc_static_fwd(x, w, y)
    dx = torch.empty_like(x)
    dw = torch.empty((wl.D, wl.W), dtype=torch.float32, device=DEV)
    ws = dsc.workspace(dsc.dsc_static_bwd_workspace_bytes(wl.B, wl.T, wl.D, wl.W), DEV)
    dsc.dsc_static_bwd(x, w, dy, dx, dw, ws)
    torch.cuda.synchronize()
    h = {k: v.cpu() for k, v in t.items()}
    g = {"y": y.cpu(), "dx": dx.cpu(), "dw": dw.cpu()}
    del t, x, dy, w, y, dx, dw, ws
    torch.cuda.empty_cache()
    ry, rdx, rdw = fullsize.static(h["x"], h["ws"], h["dy"])
    _report("static " + wl.name, {
        "y": assert_close(g["y"], ry, wl.dtype, "y"),
        "dx": assert_close(g["dx"], rdx, wl.dtype, "dx"),
        "dw": assert_close(g["dw"], rdw, wl.dtype, "dw", reduction=True)})
