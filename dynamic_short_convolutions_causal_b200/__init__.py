"""Python binding of libdsc.so, the B200 (sm_100a) causal dynamic short convolution.

Argument marshalling only: every function here derives the sizes from torch tensor
shapes, checks devices and dtypes, and calls the C entry point of the same name on the
current CUDA stream.  All arithmetic runs in the library's CUDA kernels; there is no
CPU or PyTorch fallback.  Importing this module fails loudly when libdsc.so is
missing (build it with ``python dynamic_short_convolutions_causal_b200/build.py``).

Operation ("Convolucoes Curtas Dinamicas Melhoram Transformers", Metodologia >
Convolucoes Curtas Dinamicas): y_t = x_t + sum_{k<W} w(t)_k * x_{t-k}, with explicit,
low-rank (w = z U, formed on chip) or static filters; see include/dsc.h.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "DscError", "lib", "lib_path", "dsc_fwd", "dsc_fwd_lowrank", "dsc_bwd_lowrank",
    "dsc_bwd_lowrank_workspace_bytes", "dsc_bwd", "dsc_static_fwd", "dsc_static_bwd",
    "dsc_static_bwd_workspace_bytes", "dsc_static_bwd_noalloc", "dsc_lowrank_path",
    "dsc_decode_step", "dsc_decode_step_lowrank", "dsc_fwd_lowrank_halo", "dsc_bwd_lowrank_halo",
    "dsc_fwd_lowrank_rope", "dsc_bwd_lowrank_rope",
    "DSC_F32", "DSC_BF16",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libdsc.so")

DSC_OK, DSC_ERR_INVALID_ARG, DSC_ERR_UNSUPPORTED, DSC_ERR_CUDA = 0, 1, 2, 3
DSC_F32, DSC_BF16 = 0, 1


class DscError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__("%s (status %d)" % (detail, status))
        self.status = status


def _load():
    if not os.path.exists(lib_path):
        raise ImportError(
            "libdsc.so not found at %s: build it with "
            "`python dynamic_short_convolutions_causal_b200/build.py`" % lib_path)
    L = ctypes.CDLL(lib_path)
    vp, i, sz, fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    sigs = {
        "dsc_fwd": (i, [vp, vp, vp, i, i, i, i, i, i, vp]),
        "dsc_fwd_lowrank": (i, [vp, vp, vp, vp, i, i, i, i, i, i, i, vp]),
        "dsc_bwd_lowrank_workspace_bytes": (sz, [i, i, i, i, i, i, i]),
        "dsc_bwd_lowrank": (i, [vp, vp, vp, vp, vp, fp, fp, vp, sz, i, i, i, i, i, i, i, vp]),
        "dsc_bwd": (i, [vp, vp, vp, vp, fp, i, i, i, i, i, i, vp]),
        "dsc_static_fwd": (i, [vp, vp, vp, i, i, i, i, i, vp]),
        "dsc_static_bwd_workspace_bytes": (sz, [i, i, i, i, i]),
        "dsc_static_bwd": (i, [vp, vp, vp, vp, fp, vp, sz, i, i, i, i, i, vp]),
        "dsc_static_bwd_noalloc": (i, [vp, vp, vp, vp, fp, i, i, i, i, i, vp]),
        "dsc_static_bwd_noalloc_max_scratch_bytes": (sz, []),
        "dsc_lowrank_path": (i, [i, i, i, i, i, i, i]),
        "dsc_decode_step": (i, [vp, vp, vp, vp, i, i, i, i, i, vp]),
        "dsc_decode_step_lowrank": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]),
        "dsc_fwd_lowrank_halo": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]),
        "dsc_bwd_lowrank_halo": (i, [vp, vp, vp, vp, vp, vp, vp, fp, fp, i, i, i, i, i, i, i, vp]),
        "dsc_fwd_lowrank_rope": (i, [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, vp]),
        "dsc_bwd_lowrank_rope": (i, [vp, vp, vp, vp, vp, vp, fp, fp, vp, sz, i, i, i, i, i, i, i, i, i, vp]),
        "dsc_device_fault": (ctypes.c_uint, [i]),
        "dsc_test_arm_wait_timeout": (None, [ctypes.c_uint]),
        "dsc_status_string": (ctypes.c_char_p, [i]),
        "dsc_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sigs.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def _check(status: int):
    if status != DSC_OK:
        raise DscError(status, (lib.dsc_last_error() or b"").decode() or
                       lib.dsc_status_string(status).decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSC_BF16
    if t.dtype == torch.float32:
        return DSC_F32
    raise TypeError("dsc: unsupported dtype %s (bf16 or fp32)" % t.dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("dsc: tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("dsc: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _same(ref, *ts):
    for t in ts:
        if t.device != ref.device:
            raise ValueError("dsc: all tensors must be on %s" % ref.device)


def dsc_fwd(x, w, y, G: int):
    """y = x + dynconv(x; w); x, y [B,T,D], w [B,T,D/G,W] (same dtype)."""
    B, T, D = x.shape
    W = w.shape[-1]
    _same(x, w, y)
    with torch.cuda.device(x.device):
        _check(lib.dsc_fwd(_ptr(x), _ptr(w), _ptr(y), B, T, D, G, W, _dt(x), _stream(x)))
    return y


def dsc_fwd_lowrank(x, z, U, y, G: int, W: int):
    """y = x + dynconv(x; w = z U formed on chip); z [B,T,R], U [R,(D/G)*W]."""
    B, T, D = x.shape
    R = z.shape[-1]
    _same(x, z, U, y)
    with torch.cuda.device(x.device):
        _check(lib.dsc_fwd_lowrank(_ptr(x), _ptr(z), _ptr(U), _ptr(y), B, T, D, G, W, R, _dt(x),
                                   _stream(x)))
    return y


def dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R, dtype=torch.bfloat16) -> int:
    dt = DSC_BF16 if dtype == torch.bfloat16 else DSC_F32
    return int(lib.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R, dt))


def dsc_bwd_lowrank(x, z, U, dy, dx, dz, dU, workspace, G: int, W: int):
    """dx [B,T,D] (x's dtype), dz [B,T,R] fp32, dU [R,(D/G)*W] fp32 (overwritten).
    ``workspace`` is a device tensor of at least dsc_bwd_lowrank_workspace_bytes()."""
    B, T, D = x.shape
    R = z.shape[-1]
    _same(x, z, U, dy, dx, dz, dU)
    if dz.dtype != torch.float32 or dU.dtype != torch.float32:
        raise TypeError("dsc_bwd_lowrank: dz and dU must be fp32")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(x.device):
        _check(lib.dsc_bwd_lowrank(_ptr(x), _ptr(z), _ptr(U), _ptr(dy), _ptr(dx), _ptr(dz),
                                   _ptr(dU), _ptr(workspace), ws_bytes, B, T, D, G, W, R, _dt(x),
                                   _stream(x)))
    return dx, dz, dU


def dsc_bwd(x, w, dy, dx, dw, G: int):
    """Explicit-filter backward: dx [B,T,D] (x's dtype), dw [B,T,D/G,W] fp32."""
    B, T, D = x.shape
    W = w.shape[-1]
    _same(x, w, dy, dx, dw)
    if dw.dtype != torch.float32:
        raise TypeError("dsc_bwd: dw must be fp32")
    with torch.cuda.device(x.device):
        _check(lib.dsc_bwd(_ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), B, T, D, G, W, _dt(x),
                           _stream(x)))
    return dx, dw


def dsc_static_fwd(x, w, y):
    """y = x + depthwise causal conv with fixed filters w [D,W]."""
    B, T, D = x.shape
    W = w.shape[-1]
    _same(x, w, y)
    with torch.cuda.device(x.device):
        _check(lib.dsc_static_fwd(_ptr(x), _ptr(w), _ptr(y), B, T, D, W, _dt(x), _stream(x)))
    return y


def dsc_static_bwd_workspace_bytes(B, T, D, W, dtype=torch.bfloat16) -> int:
    dt = DSC_BF16 if dtype == torch.bfloat16 else DSC_F32
    return int(lib.dsc_static_bwd_workspace_bytes(B, T, D, W, dt))


def dsc_static_bwd(x, w, dy, dx, dw, workspace):
    """dx [B,T,D] (x's dtype) and dw [D,W] fp32 summed over all tokens."""
    B, T, D = x.shape
    W = w.shape[-1]
    _same(x, w, dy, dx, dw, workspace)
    ws_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(x.device):
        _check(lib.dsc_static_bwd(_ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), _ptr(workspace),
                                  ws_bytes, B, T, D, W, _dt(x), _stream(x)))
    return dx, dw


def dsc_static_bwd_noalloc(x, w, dy, dx, dw):
    """dsc_static_bwd with the library's fixed scratch array instead of a workspace
    (for callers that cannot allocate device memory; see include/dsc.h)."""
    B, T, D = x.shape
    W = w.shape[-1]
    _same(x, w, dy, dx, dw)
    with torch.cuda.device(x.device):
        _check(lib.dsc_static_bwd_noalloc(_ptr(x), _ptr(w), _ptr(dy), _ptr(dx), _ptr(dw), B, T, D,
                                          W, _dt(x), _stream(x)))
    return dx, dw


def dsc_decode_step(x_t, w_t, state, y_t, G: int):
    """One decode step with explicit filters: x_t, y_t [B,D], w_t [B,D/G,W], state
    [B,W-1,D] (oldest row first, updated in place; may be None when W = 1)."""
    B, D = x_t.shape
    W = w_t.shape[-1]
    _same(x_t, w_t, y_t, *([state] if state is not None else []))
    with torch.cuda.device(x_t.device):
        _check(lib.dsc_decode_step(_ptr(x_t), _ptr(w_t), _ptr(state), _ptr(y_t), B, D, G, W, _dt(x_t),
                                   _stream(x_t)))
    return y_t


def dsc_decode_step_lowrank(x_t, z_t, U, state, y_t, G: int, W: int):
    """One decode step with w_t = z_t U: z_t [B,R], U [R,(D/G)*W]; see dsc_decode_step."""
    B, D = x_t.shape
    R = z_t.shape[-1]
    _same(x_t, z_t, U, y_t, *([state] if state is not None else []))
    with torch.cuda.device(x_t.device):
        _check(lib.dsc_decode_step_lowrank(_ptr(x_t), _ptr(z_t), _ptr(U), _ptr(state), _ptr(y_t), B, D, G,
                                           W, R, _dt(x_t), _stream(x_t)))
    return y_t


def dsc_fwd_lowrank_halo(x, z, U, x_prev, y, G: int, W: int):
    """Sequence shard fix-up after dsc_fwd_lowrank: recompute y rows t < W-1 with the W-1
    tokens before the shard, x_prev [B,W-1,D] (oldest first; None for the first shard)."""
    B, T, D = x.shape
    R = z.shape[-1]
    _same(x, z, U, y, *([x_prev] if x_prev is not None else []))
    with torch.cuda.device(x.device):
        _check(lib.dsc_fwd_lowrank_halo(_ptr(x), _ptr(z), _ptr(U), _ptr(x_prev), _ptr(y), B, T, D, G, W, R,
                                        _dt(x), _stream(x)))
    return y


def dsc_bwd_lowrank_halo(x_prev, z, U, dy, dy_next, z_next, dx, dz, dU, G: int, W: int):
    """Sequence shard fix-up after dsc_bwd_lowrank: recompute dx rows t >= T-(W-1) with the
    W-1 tokens after the shard (dy_next [B,W-1,D], z_next [B,W-1,R]; None for the last
    shard) and add the x_prev terms to dz rows t < W-1 and to dU (fp32, in place)."""
    B, T, D = dy.shape
    R = z.shape[-1]
    _same(dy, z, U, dx, dz, dU, *[t for t in (x_prev, dy_next, z_next) if t is not None])
    if dz.dtype != torch.float32 or dU.dtype != torch.float32:
        raise TypeError("dsc_bwd_lowrank_halo: dz and dU must be fp32")
    with torch.cuda.device(dy.device):
        _check(lib.dsc_bwd_lowrank_halo(_ptr(x_prev), _ptr(z), _ptr(U), _ptr(dy), _ptr(dy_next), _ptr(z_next),
                                        _ptr(dx), _ptr(dz), _ptr(dU), B, T, D, G, W, R, _dt(dy), _stream(dy)))
    return dx, dz, dU


def dsc_fwd_lowrank_rope(x, z, U, cs, y, G: int, W: int, dh: int, n_rot: int):
    """dsc_fwd_lowrank followed by RoPE of the first n_rot channels of y (heads of dh,
    adjacent pairs); cs fp32 [dh/2, T, 2] holds (cos, sin) per pair and position."""
    B, T, D = x.shape
    R = z.shape[-1]
    _same(x, z, U, y, cs)
    if cs.dtype != torch.float32:
        raise TypeError("dsc_fwd_lowrank_rope: cs must be fp32")
    with torch.cuda.device(x.device):
        _check(lib.dsc_fwd_lowrank_rope(_ptr(x), _ptr(z), _ptr(U), _ptr(cs), _ptr(y), B, T, D, G, W, R, dh, n_rot,
                                        _dt(x), _stream(x)))
    return y


def dsc_bwd_lowrank_rope(x, z, U, cs, dy_rot, dx, dz, dU, workspace, G: int, W: int, dh: int, n_rot: int):
    """Backward of dsc_fwd_lowrank_rope given dy_rot, the gradient of the rotated output;
    same outputs and workspace as dsc_bwd_lowrank."""
    B, T, D = x.shape
    R = z.shape[-1]
    _same(x, z, U, cs, dy_rot, dx, dz, dU)
    if dz.dtype != torch.float32 or dU.dtype != torch.float32 or cs.dtype != torch.float32:
        raise TypeError("dsc_bwd_lowrank_rope: dz, dU and cs must be fp32")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(x.device):
        _check(lib.dsc_bwd_lowrank_rope(_ptr(x), _ptr(z), _ptr(U), _ptr(cs), _ptr(dy_rot), _ptr(dx), _ptr(dz),
                                        _ptr(dU), _ptr(workspace), ws_bytes, B, T, D, G, W, R, dh, n_rot, _dt(x),
                                        _stream(x)))
    return dx, dz, dU


def dsc_device_fault(reset: bool = False) -> int:
    """Fault word of the current device (nonzero: a kernel gave up on a wait)."""
    return int(lib.dsc_device_fault(1 if reset else 0))


def dsc_lowrank_path(B, T, D, G, W, R, dtype=torch.bfloat16) -> int:
    """Bit 0: forward on tensor cores, bit 1: backward on tensor cores; -1: invalid."""
    dt = DSC_BF16 if dtype == torch.bfloat16 else DSC_F32
    return int(lib.dsc_lowrank_path(B, T, D, G, W, R, dt))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned device scratch buffer of at least ``nbytes`` bytes."""
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)
