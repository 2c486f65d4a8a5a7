"""CPU oracle for the causal dynamic short convolution -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  The product library never loads it and shares
no code with it.

The arithmetic lives in ``dsc_oracle.c`` (plain single-threaded C, double precision),
written from "Convolucoes Curtas Dinamicas Melhoram Transformers"
(gist.science/pt/paper/2606.03825), section "Metodologia > Convolucoes Curtas
Dinamicas" (Mecanismo, Parametrizacao, Posicionamento).  This module only compiles
that file with gcc, loads it with ctypes and marshals numpy float64 arrays.

Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsc_oracle.c")
_LIB = os.path.join(_HERE, "libdsc_oracle.so")
_lock = threading.Lock()
_default = None

_GCC_FLAGS = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c99", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile dsc_oracle.c into libdsc_oracle.so (gcc -O2, strict IEEE double)."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
            return _LIB
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.run(_GCC_FLAGS + ["-o", tmp, _SRC], check=True)
        os.replace(tmp, _LIB)
        return _LIB


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    sig = {
        "oracle_fwd": (None, [dp, dp, dp, i, i, i, i, i]),
        "oracle_lowrank_weights": (None, [dp, dp, dp, i, i, i, i, i, i]),
        "oracle_fwd_lowrank": (i, [dp, dp, dp, dp, i, i, i, i, i, i]),
        "oracle_bwd": (None, [dp, dp, dp, dp, dp, i, i, i, i, i]),
        "oracle_bwd_lowrank": (i, [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i]),
        "oracle_static_fwd": (None, [dp, dp, dp, i, i, i, i]),
        "oracle_static_bwd": (None, [dp, dp, dp, dp, dp, i, i, i, i]),
        "oracle_decode": (None, [dp, dp, dp, dp, dp, i, i, i, i]),
        "oracle_decode_lowrank": (i, [dp, dp, dp, dp, dp, dp, i, i, i, i, i]),
        "oracle_rope": (None, [dp, dp, i, i, i, i, i, i]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def _in(a, shape):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if tuple(a.shape) != tuple(shape):
        raise ValueError("oracle: expected shape %s, got %s" % (shape, a.shape))
    return a


def _p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check_dims(B, T, D, G, W, R=1):
    if min(B, T, D, G, W, R) < 1 or D % G:
        raise ValueError("oracle: bad sizes B=%d T=%d D=%d G=%d W=%d R=%d" % (B, T, D, G, W, R))


class Oracle:
    """numpy front end over one compiled copy of the oracle source."""

    def __init__(self, lib):
        self._l = lib

    def fwd(self, x, w, G):
        """y = x + sum_k w(t)_k * x_{t-k}; x [B,T,D], w [B,T,D/G,W]."""
        x = np.asarray(x)
        B, T, D = x.shape
        W = np.asarray(w).shape[-1]
        _check_dims(B, T, D, G, W)
        x = _in(x, (B, T, D))
        w = _in(w, (B, T, D // G, W))
        y = np.empty_like(x)
        self._l.oracle_fwd(_p(x), _p(w), _p(y), B, T, D, G, W)
        return y

    def lowrank_weights(self, z, U, D, G, W):
        """w = reshape(z U, [B,T,D/G,W]) by a plain triple loop."""
        z = np.asarray(z)
        B, T, R = z.shape
        _check_dims(B, T, D, G, W, R)
        z = _in(z, (B, T, R))
        U = _in(U, (R, (D // G) * W))
        w = np.empty((B, T, D // G, W), dtype=np.float64)
        self._l.oracle_lowrank_weights(_p(z), _p(U), _p(w), B, T, D, G, W, R)
        return w

    def fwd_lowrank(self, x, z, U, G, W):
        """y = x + dynconv(x; w = z U); x [B,T,D], z [B,T,R], U [R,(D/G)*W]."""
        x = np.asarray(x)
        B, T, D = x.shape
        R = np.asarray(z).shape[-1]
        _check_dims(B, T, D, G, W, R)
        x = _in(x, (B, T, D))
        z = _in(z, (B, T, R))
        U = _in(U, (R, (D // G) * W))
        y = np.empty_like(x)
        if self._l.oracle_fwd_lowrank(_p(x), _p(z), _p(U), _p(y), B, T, D, G, W, R):
            raise MemoryError("oracle_fwd_lowrank")
        return y

    def bwd(self, x, w, dy, G):
        """Backward of fwd: returns (dx [B,T,D], dw [B,T,D/G,W])."""
        x = np.asarray(x)
        B, T, D = x.shape
        W = np.asarray(w).shape[-1]
        _check_dims(B, T, D, G, W)
        x = _in(x, (B, T, D))
        w = _in(w, (B, T, D // G, W))
        dy = _in(dy, (B, T, D))
        dx = np.empty_like(x)
        dw = np.empty_like(w)
        self._l.oracle_bwd(_p(x), _p(w), _p(dy), _p(dx), _p(dw), B, T, D, G, W)
        return dx, dw

    def bwd_lowrank(self, x, z, U, dy, G, W):
        """Backward of fwd_lowrank: returns (dx [B,T,D], dz [B,T,R], dU [R,(D/G)*W])."""
        x = np.asarray(x)
        B, T, D = x.shape
        R = np.asarray(z).shape[-1]
        _check_dims(B, T, D, G, W, R)
        N = (D // G) * W
        x = _in(x, (B, T, D))
        z = _in(z, (B, T, R))
        U = _in(U, (R, N))
        dy = _in(dy, (B, T, D))
        dx = np.empty_like(x)
        dz = np.empty_like(z)
        dU = np.empty_like(U)
        if self._l.oracle_bwd_lowrank(_p(x), _p(z), _p(U), _p(dy), _p(dx), _p(dz), _p(dU),
                                      B, T, D, G, W, R):
            raise MemoryError("oracle_bwd_lowrank")
        return dx, dz, dU

    def static_fwd(self, x, ws):
        """y = x + depthwise causal conv with fixed filters ws [D,W]."""
        x = np.asarray(x)
        B, T, D = x.shape
        W = np.asarray(ws).shape[-1]
        _check_dims(B, T, D, 1, W)
        x = _in(x, (B, T, D))
        ws = _in(ws, (D, W))
        y = np.empty_like(x)
        self._l.oracle_static_fwd(_p(x), _p(ws), _p(y), B, T, D, W)
        return y

    def static_bwd(self, x, ws, dy):
        """Backward of static_fwd: returns (dx [B,T,D], dws [D,W])."""
        x = np.asarray(x)
        B, T, D = x.shape
        W = np.asarray(ws).shape[-1]
        _check_dims(B, T, D, 1, W)
        x = _in(x, (B, T, D))
        ws = _in(ws, (D, W))
        dy = _in(dy, (B, T, D))
        dx = np.empty_like(x)
        dws = np.empty_like(ws)
        self._l.oracle_static_bwd(_p(x), _p(ws), _p(dy), _p(dx), _p(dws), B, T, D, W)
        return dx, dws


    def decode(self, x_t, w_t, state, G):
        """One decode step with explicit filters: x_t [B,D], w_t [B,D/G,W], state
        [B,W-1,D] (oldest row first).  Returns (y_t [B,D], new state [B,W-1,D])."""
        x_t = np.asarray(x_t)
        B, D = x_t.shape
        W = np.asarray(w_t).shape[-1]
        _check_dims(B, 1, D, G, W)
        x_t = _in(x_t, (B, D))
        w_t = _in(w_t, (B, D // G, W))
        state = _in(state, (B, W - 1, D))
        y = np.empty_like(x_t)
        st = np.empty_like(state)
        self._l.oracle_decode(_p(x_t), _p(w_t), _p(state), _p(y), _p(st), B, D, G, W)
        return y, st

    def decode_lowrank(self, x_t, z_t, U, state, G, W):
        """One decode step with w_t = z_t U: x_t [B,D], z_t [B,R], U [R,(D/G)*W],
        state [B,W-1,D].  Returns (y_t [B,D], new state [B,W-1,D])."""
        x_t = np.asarray(x_t)
        B, D = x_t.shape
        R = np.asarray(z_t).shape[-1]
        _check_dims(B, 1, D, G, W, R)
        x_t = _in(x_t, (B, D))
        z_t = _in(z_t, (B, R))
        U = _in(U, (R, (D // G) * W))
        state = _in(state, (B, W - 1, D))
        y = np.empty_like(x_t)
        st = np.empty_like(state)
        if self._l.oracle_decode_lowrank(_p(x_t), _p(z_t), _p(U), _p(state), _p(y), _p(st),
                                         B, D, G, W, R):
            raise MemoryError("oracle_decode_lowrank")
        return y, st

    def rope(self, y, cs, dh, n_rot, transpose=False):
        """RoPE of the first n_rot channels of y [B,T,D] (heads of dh channels, adjacent
        pairs rotated; cs [T, dh/2, 2] holds cos, sin); returns a rotated copy.
        transpose=True rotates by the opposite angle (the transpose)."""
        y = np.asarray(y)
        B, T, D = y.shape
        if dh < 2 or dh % 2 or n_rot % dh or not 0 <= n_rot <= D:
            raise ValueError("oracle.rope: bad dh=%d n_rot=%d for D=%d" % (dh, n_rot, D))
        out = _in(y, (B, T, D)).copy()
        cs = _in(cs, (T, dh // 2, 2))
        self._l.oracle_rope(_p(out), _p(cs), B, T, D, dh, n_rot, 1 if transpose else 0)
        return out

    def fwd_lowrank_rope(self, x, z, U, cs, G, W, dh, n_rot):
        """RoPE(x + dynconv(x; w = z U)): the op followed by the rotation of its Q and K
        channels (Posicionamento: the convolution sits before RoPE)."""
        return self.rope(self.fwd_lowrank(x, z, U, G, W), cs, dh, n_rot)

    def bwd_lowrank_rope(self, x, z, U, cs, dy_rot, G, W, dh, n_rot):
        """Backward of fwd_lowrank_rope given the gradient of its rotated output:
        bwd_lowrank with dy = RoPE^T(dy_rot).  Returns (dx, dz, dU)."""
        return self.bwd_lowrank(x, z, U, self.rope(dy_rot, cs, dh, n_rot, transpose=True), G, W)


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_bind(ctypes.CDLL(build())))
    return _default


def from_source(text: str, workdir: str) -> Oracle:
    """Compile a variant of the oracle source (used by the pin tests to plant a
    mistake on the CPU and check that some pin catches it)."""
    src = os.path.join(workdir, "variant.c")
    lib = os.path.join(workdir, "libvariant.so")
    with open(src, "w") as f:
        f.write(text)
    subprocess.run(_GCC_FLAGS + ["-o", lib, src], check=True)
    return Oracle(_bind(ctypes.CDLL(lib)))


def fwd(x, w, G):
    return default().fwd(x, w, G)


def lowrank_weights(z, U, D, G, W):
    return default().lowrank_weights(z, U, D, G, W)


def fwd_lowrank(x, z, U, G, W):
    return default().fwd_lowrank(x, z, U, G, W)


def bwd(x, w, dy, G):
    return default().bwd(x, w, dy, G)


def bwd_lowrank(x, z, U, dy, G, W):
    return default().bwd_lowrank(x, z, U, dy, G, W)


def static_fwd(x, ws):
    return default().static_fwd(x, ws)


def static_bwd(x, ws, dy):
    return default().static_bwd(x, ws, dy)


def decode(x_t, w_t, state, G):
    return default().decode(x_t, w_t, state, G)


def rope(y, cs, dh, n_rot, transpose=False):
    return default().rope(y, cs, dh, n_rot, transpose)


def fwd_lowrank_rope(x, z, U, cs, G, W, dh, n_rot):
    return default().fwd_lowrank_rope(x, z, U, cs, G, W, dh, n_rot)


def bwd_lowrank_rope(x, z, U, cs, dy_rot, G, W, dh, n_rot):
    return default().bwd_lowrank_rope(x, z, U, cs, dy_rot, G, W, dh, n_rot)


def decode_lowrank(x_t, z_t, U, state, G, W):
    return default().decode_lowrank(x_t, z_t, U, state, G, W)
