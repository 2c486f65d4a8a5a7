"""Whole-tensor oracle results at the full workload sizes, computed in token chunks.

Every output of the convolution at token t depends on a few neighbouring tokens only
(y_t and dz_t on tokens t-W+1..t, dx_t on tokens t..t+W-1), so the oracle run on a
chunk of tokens plus its causal halo gives that chunk's outputs exactly.  The weight
gradients (dU, static dw) are sums over tokens: each chunk's sub-problem has dy set
to zero outside the chunk, so it contributes exactly that chunk's terms, and the
chunk sums are added in float64.

The chunks run on a thread pool: the oracle is plain C called through ctypes, which
releases the GIL, so the threads use separate host cores.  Reference values are kept
as float32 arrays (a relative rounding of 6e-8, far below the 2e-2 bf16 bound).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle


def _threads():
    return max(1, min(32, os.cpu_count() or 1))


def _chunks(B, T, size):
    return [(b, t0, min(T, t0 + size)) for b in range(B) for t0 in range(0, T, size)]


def _h(t, b, a, e):
    """Rows [a, e) of sequence b of a host tensor, as float64 with a batch axis of 1."""
    return t[b:b + 1, a:e].to(torch.float64).numpy()


def _run(jobs, fn):
    with ThreadPoolExecutor(_threads()) as ex:
        return list(ex.map(fn, jobs))


def lowrank(x, z, U, dy, G, W, chunk=256):
    """y, dx, dz (float32 arrays) and dU (float64) of the low-rank op at any size.
    x, z, dy: host tensors [B,T,*] (bf16 or fp32); U: host tensor [R, N]."""
    B, T, D = x.shape
    R = z.shape[-1]
    Uh = U.to(torch.float64).numpy()
    y = np.empty((B, T, D), np.float32)
    dx = np.empty((B, T, D), np.float32)
    dz = np.empty((B, T, R), np.float32)

    def job(c):
        b, t0, t1 = c
        a = max(0, t0 - W + 1)
        e = min(T, t1 + W - 1)
        y[b, t0:t1] = oracle.fwd_lowrank(_h(x, b, a, t1), _h(z, b, a, t1), Uh, G, W)[0, t0 - a:]
        d = _h(dy, b, a, t1)
        d[:, :t0 - a] = 0.0                    # tokens before the chunk contribute nothing
        _, rdz, rdU = oracle.bwd_lowrank(_h(x, b, a, t1), _h(z, b, a, t1), Uh, d, G, W)
        dz[b, t0:t1] = rdz[0, t0 - a:]
        rdx, _, _ = oracle.bwd_lowrank(_h(x, b, t0, e), _h(z, b, t0, e), Uh, _h(dy, b, t0, e), G, W)
        dx[b, t0:t1] = rdx[0, :t1 - t0]
        return rdU

    dU = np.zeros_like(Uh)
    for part in _run(_chunks(B, T, chunk), job):
        dU += part
    return y, dx, dz, dU


def explicit_fwd(x, w, G, chunk=512):
    """y (float32) of the explicit-filter forward at any size."""
    B, T, D = x.shape
    W = w.shape[-1]
    y = np.empty((B, T, D), np.float32)

    def job(c):
        b, t0, t1 = c
        a = max(0, t0 - W + 1)
        y[b, t0:t1] = oracle.fwd(_h(x, b, a, t1), _h(w, b, a, t1), G)[0, t0 - a:]

    _run(_chunks(B, T, chunk), job)
    return y


def static(x, ws, dy, chunk=512):
    """y, dx (float32) and dw (float64) of the static convolution at any size."""
    B, T, D = x.shape
    W = ws.shape[-1]
    wh = ws.to(torch.float64).numpy()
    y = np.empty((B, T, D), np.float32)
    dx = np.empty((B, T, D), np.float32)

    def job(c):
        b, t0, t1 = c
        a = max(0, t0 - W + 1)
        e = min(T, t1 + W - 1)
        y[b, t0:t1] = oracle.static_fwd(_h(x, b, a, t1), wh)[0, t0 - a:]
        d = _h(dy, b, a, t1)
        d[:, :t0 - a] = 0.0
        _, rdw = oracle.static_bwd(_h(x, b, a, t1), wh, d)
        rdx, _ = oracle.static_bwd(_h(x, b, t0, e), wh, _h(dy, b, t0, e))
        dx[b, t0:t1] = rdx[0, :t1 - t0]
        return rdw

    dw = np.zeros_like(wh)
    for part in _run(_chunks(B, T, chunk), job):
        dw += part
    return y, dx, dw
