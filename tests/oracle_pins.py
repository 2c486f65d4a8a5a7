"""Pins for the CPU oracle: checks against what the pages and the mathematics fix,
independent of the oracle's own code.

Each pin takes an ``Oracle`` instance and raises AssertionError when it disagrees.
They are run on the real oracle (tests/test_oracle_pins.py) and on copies with a
planted mistake (tests/test_oracle_mutants.py), where at least one must fail.

What each pin rests on ("Convolucoes Curtas Dinamicas Melhoram Transformers",
gist.science/pt/paper/2606.03825, "Metodologia > Convolucoes Curtas Dinamicas"):
  * hand_example  -- values worked out by hand from the Mecanismo formula
                     (tests/golden/hand_example_T3_D2_W2.json).
  * identity      -- W=1, w=1: y_t = x_t + x_t = 2x exactly (Mecanismo + residual).
  * numpy_convolve -- time-constant filters are the static depthwise causal
                     convolution the method generalises ("Contribuicoes Chave" 1);
                     checked against numpy.convolve, a library routine.
  * tying         -- one filter shared by G consecutive channels (Parametrizacao 2)
                     equals G=1 with each filter repeated over its G channels.
  * lowrank       -- w = z U (Parametrizacao 1; the fused kernel of "Implementacao
                     de Treinamento Eficiente" forms zU on chip) equals the explicit
                     op fed numpy's matmul.
  * causality     -- y_t depends on x_{t'} only for t-W < t' <= t and on its own
                     sequence only (the op is causal and short).
  * impulse       -- a unit impulse produces exactly the filter taps.
  * finite differences / adjoint -- the backward is the adjoint of the forward's
                     Jacobian; y is linear in each argument separately, so central
                     differences are exact up to rounding.
  * invariant     -- sum(dU*U) == sum(dz*z) (both equal sum_t <dw_t, w_t>).
  * rope          -- the op sits before RoPE on the Q and K projections
                     ("Posicionamento"); RoPE (original form: adjacent channel pairs
                     of each head rotated by their angle) is checked against numpy's
                     complex multiplication, its transpose against the inverse and
                     the adjoint identity, and the fused backward against central
                     differences of the rotated forward.
  * decode        -- one decode step (a token with its W-1 predecessors held in a
                     rolling window; "Significancia e Alegacoes" notes that inference
                     still needs engineering) is the forward at the last position of
                     the sequence [window rows, x_t]; stepping through a sequence from
                     a zero window gives the pinned forward's outputs token by token,
                     and the window then holds the last W-1 inputs.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "hand_example_T3_D2_W2.json")


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, "%s: shape %s vs %s" % (what, a.shape, b.shape)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b)))) if b.size else 1.0
    assert err <= tol * scale, "%s: max|err| = %.3e (tol %.1e)" % (what, err, tol * scale)


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- hand example
def pin_hand_example(orc):
    g = json.load(open(GOLDEN))
    x = np.array(g["x"], dtype=np.float64)[None]
    dy = np.array(g["dy"], dtype=np.float64)[None]
    W = g["sizes"]["W"]
    e = g["explicit"]
    w = np.array(e["w"], dtype=np.float64)[None]
    _close(orc.fwd(x, w, e["G"]), np.array(e["y"])[None], 0, "hand explicit y")
    dx, dw = orc.bwd(x, w, dy, e["G"])
    _close(dx, np.array(e["dx"])[None], 0, "hand explicit dx")
    _close(dw, np.array(e["dw"])[None], 0, "hand explicit dw")
    lr = g["lowrank"]
    z = np.array(lr["z"], dtype=np.float64)[None]
    U = np.array(lr["U"], dtype=np.float64)
    _close(orc.fwd_lowrank(x, z, U, lr["G"], W), np.array(lr["y"])[None], 0, "hand lowrank y")
    dx, dz, dU = orc.bwd_lowrank(x, z, U, dy, lr["G"], W)
    _close(dx, np.array(lr["dx"])[None], 0, "hand lowrank dx")
    _close(dz, np.array(lr["dz"])[None], 0, "hand lowrank dz")
    _close(dU, np.array(lr["dU"]), 0, "hand lowrank dU")
    st = g["static"]
    ws = np.array(st["ws"], dtype=np.float64)
    _close(orc.static_fwd(x, ws), np.array(st["y"])[None], 0, "hand static y")
    dx, dws = orc.static_bwd(x, ws, dy)
    _close(dx, np.array(st["dx"])[None], 0, "hand static dx")
    _close(dws, np.array(st["dws"]), 0, "hand static dws")


# ---------------------------------------------------------------- closed forms
def pin_identity_filter_doubles(orc):
    r = _rng(1)
    B, T, D = 2, 9, 12
    x = r.standard_normal((B, T, D))
    for G in (1, 3, 12):
        w = np.ones((B, T, D // G, 1))
        assert np.array_equal(orc.fwd(x, w, G), 2 * x), "explicit W=1 w=1 must give 2x"
        z = np.ones((B, T, 1))
        U = np.ones((1, D // G))
        assert np.array_equal(orc.fwd_lowrank(x, z, U, G, 1), 2 * x), "lowrank W=1 w=1 must give 2x"
    assert np.array_equal(orc.static_fwd(x, np.ones((D, 1))), 2 * x), "static W=1 w=1 must give 2x"


def _np_static(x, ws):
    """y = x + causal depthwise conv by numpy.convolve (full mode, first T samples)."""
    B, T, D = x.shape
    y = x.copy()
    for b in range(B):
        for c in range(D):
            y[b, :, c] += np.convolve(x[b, :, c], ws[c])[:T]
    return y


def pin_numpy_convolve(orc):
    r = _rng(2)
    for (B, T, D, W) in [(2, 11, 6, 4), (1, 3, 5, 5), (3, 1, 4, 2), (1, 17, 3, 8)]:
        x = r.standard_normal((B, T, D))
        ws = r.standard_normal((D, W))
        ref = _np_static(x, ws)
        _close(orc.static_fwd(x, ws), ref, 1e-12, "static vs numpy.convolve")
        # explicit dynamic filters held constant over t (G=1): the static op
        w = np.broadcast_to(ws[None, None], (B, T, D, W))
        _close(orc.fwd(x, w, 1), ref, 1e-12, "time-constant explicit vs numpy.convolve")
        # low-rank with z_t constant: w_t = 1 * U row
        z = np.ones((B, T, 1))
        U = ws.reshape(1, D * W)
        _close(orc.fwd_lowrank(x, z, U, 1, W), ref, 1e-12, "time-constant lowrank vs numpy.convolve")


def pin_static_bwd_numpy(orc):
    """dws[c,k] = sum_t dy_t[c] x_{t-k}[c] (numpy.correlate) and dx via the flipped
    convolution (numpy.convolve of dy with reversed taps), both library routines."""
    r = _rng(3)
    B, T, D, W = 2, 10, 5, 4
    x = r.standard_normal((B, T, D))
    dy = r.standard_normal((B, T, D))
    ws = r.standard_normal((D, W))
    dx, dws = orc.static_bwd(x, ws, dy)
    ref_dws = np.zeros((D, W))
    ref_dx = dy.copy()
    for b in range(B):
        for c in range(D):
            full = np.correlate(dy[b, :, c], x[b, :, c], mode="full")  # index T-1+k: sum_t dy[t] x[t-k]
            ref_dws[c] += full[T - 1:T - 1 + W] if T >= W else np.pad(full[T - 1:], (0, W - T))
            ref_dx[b, :, c] += np.convolve(dy[b, ::-1, c], ws[c])[:T][::-1]
    _close(dws, ref_dws, 1e-12, "static dws vs numpy.correlate")
    _close(dx, ref_dx, 1e-12, "static dx vs numpy.convolve")


# ---------------------------------------------------------------- structure
def pin_tying(orc):
    r = _rng(4)
    B, T, D, W = 2, 8, 12, 3
    x = r.standard_normal((B, T, D))
    dy = r.standard_normal((B, T, D))
    for G in (2, 3, 4, 6, 12):
        wg = r.standard_normal((B, T, D // G, W))
        w1 = np.repeat(wg, G, axis=2)       # filter g serves channels g*G .. g*G+G-1
        _close(orc.fwd(x, wg, G), orc.fwd(x, w1, 1), 1e-13, "tied fwd vs repeated G=1")
        dxg, dwg = orc.bwd(x, wg, dy, G)
        dx1, dw1 = orc.bwd(x, w1, dy, 1)
        _close(dxg, dx1, 1e-13, "tied dx vs repeated G=1")
        _close(dwg, dw1.reshape(B, T, D // G, G, W).sum(axis=3), 1e-12, "tied dw vs summed G=1")


def pin_lowrank_equals_explicit(orc):
    r = _rng(5)
    for (B, T, D, G, W, R) in [(2, 9, 8, 1, 4, 3), (1, 6, 12, 3, 2, 5), (2, 5, 8, 8, 3, 2)]:
        N = (D // G) * W
        x = r.standard_normal((B, T, D))
        z = r.standard_normal((B, T, R))
        U = r.standard_normal((R, N))
        dy = r.standard_normal((B, T, D))
        w = np.matmul(z, U).reshape(B, T, D // G, W)   # library matmul; column j = g*W+k
        _close(orc.lowrank_weights(z, U, D, G, W), w, 1e-13, "lowrank_weights vs numpy matmul")
        _close(orc.fwd_lowrank(x, z, U, G, W), orc.fwd(x, w, G), 1e-12, "fused vs explicit fwd")
        dx, dz, dU = orc.bwd_lowrank(x, z, U, dy, G, W)
        dxe, dwe = orc.bwd(x, w, dy, G)
        _close(dx, dxe, 1e-12, "lowrank dx vs explicit dx")
        dwf = dwe.reshape(B, T, N)
        _close(dz, np.matmul(dwf, U.T), 1e-12, "dz vs dw U^T (numpy)")
        _close(dU, np.einsum("btr,btj->rj", z, dwf), 1e-12, "dU vs z^T dw (numpy)")


def pin_causality(orc):
    r = _rng(6)
    B, T, D, G, W, R = 2, 12, 6, 2, 4, 3
    N = (D // G) * W
    x = r.standard_normal((B, T, D))
    z = r.standard_normal((B, T, R))
    U = r.standard_normal((R, N))
    w = r.standard_normal((B, T, D // G, W))
    y0 = orc.fwd_lowrank(x, z, U, G, W)
    e0 = orc.fwd(x, w, G)
    for tp in (0, 5, T - 1):
        x2 = x.copy()
        x2[1, tp] += 10.0
        z2 = z.copy()
        z2[1, tp] += 3.0
        y2 = orc.fwd_lowrank(x2, z2, U, G, W)
        e2 = orc.fwd(x2, w, G)
        # earlier tokens, and tokens W or more steps later, are bitwise unchanged
        for arr0, arr2 in ((y0, y2), (e0, e2)):
            assert np.array_equal(arr0[1, :tp], arr2[1, :tp]), "future input leaked into the past"
            assert np.array_equal(arr0[1, tp + W:], arr2[1, tp + W:]), "filter reached further than W-1"
            assert np.array_equal(arr0[0], arr2[0]), "one sequence leaked into another"
            assert not np.array_equal(arr0[1, tp], arr2[1, tp]), "perturbation had no effect"


def pin_impulse_response(orc):
    r = _rng(7)
    B, T, D, G, W = 1, 10, 4, 2, 4
    w = r.standard_normal((B, T, D // G, W))
    for t0 in (0, 3, 8):
        for c in range(D):
            x = np.zeros((B, T, D))
            x[0, t0, c] = 1.0
            y = orc.fwd(x, w, G)
            exp = np.zeros((B, T, D))
            exp[0, t0, c] = 1.0
            for k in range(W):
                if t0 + k < T:
                    exp[0, t0 + k, c] += w[0, t0 + k, c // G, k]
            assert np.array_equal(y, exp), "impulse response must be 1 + w_t0[.,0], then w_{t0+k}[.,k]"


def pin_short_sequences(orc):
    """T < W, T = 1: taps past the sequence start contribute nothing."""
    r = _rng(8)
    for T in (1, 2, 3):
        B, D, G, W, R = 2, 4, 1, 6, 2
        x = r.standard_normal((B, T, D))
        z = r.standard_normal((B, T, R))
        U = r.standard_normal((R, D * W))
        w = np.matmul(z, U).reshape(B, T, D, W)
        exp = x.copy()
        for t in range(T):
            for k in range(t + 1):
                exp[:, t] += w[:, t, :, k] * x[:, t - k]
        _close(orc.fwd_lowrank(x, z, U, G, W), exp, 1e-12, "short sequence")


# ---------------------------------------------------------------- backward
def _fd_check(loss, params, grads, what, tol=1e-9):
    """Central differences with step 1: exact for a loss linear in each argument."""
    for name, p in params.items():
        g = np.zeros_like(p)
        flat = p.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + 1.0
            lp = loss()
            flat[i] = old - 1.0
            lm = loss()
            flat[i] = old
            g.reshape(-1)[i] = (lp - lm) / 2.0
        _close(grads[name], g, tol, "%s d%s vs finite differences" % (what, name))


def pin_fd_lowrank(orc):
    r = _rng(9)
    for (G, W) in ((1, 1), (1, 3), (2, 4), (2, 3)):
        B, T, D, R = 2, 7, 8, 3
        N = (D // G) * W
        x = r.standard_normal((B, T, D))
        z = r.standard_normal((B, T, R))
        U = r.standard_normal((R, N))
        dy = r.standard_normal((B, T, D))
        loss = lambda: float(np.sum(dy * orc.fwd_lowrank(x, z, U, G, W)))
        dx, dz, dU = orc.bwd_lowrank(x, z, U, dy, G, W)
        _fd_check(loss, {"x": x, "z": z, "U": U}, {"x": dx, "z": dz, "U": dU},
                  "lowrank G=%d W=%d" % (G, W))


def pin_fd_explicit(orc):
    r = _rng(10)
    for (G, W) in ((1, 2), (2, 4), (4, 3)):
        B, T, D = 2, 6, 8
        x = r.standard_normal((B, T, D))
        w = r.standard_normal((B, T, D // G, W))
        dy = r.standard_normal((B, T, D))
        loss = lambda: float(np.sum(dy * orc.fwd(x, w, G)))
        dx, dw = orc.bwd(x, w, dy, G)
        _fd_check(loss, {"x": x, "w": w}, {"x": dx, "w": dw}, "explicit G=%d W=%d" % (G, W))


def pin_fd_static(orc):
    r = _rng(11)
    B, T, D, W = 2, 6, 5, 3
    x = r.standard_normal((B, T, D))
    ws = r.standard_normal((D, W))
    dy = r.standard_normal((B, T, D))
    loss = lambda: float(np.sum(dy * orc.static_fwd(x, ws)))
    dx, dws = orc.static_bwd(x, ws, dy)
    _fd_check(loss, {"x": x, "ws": ws}, {"x": dx, "ws": dws}, "static")


def pin_adjoint_and_invariant(orc):
    """<dy, J v> = <J^T dy, v> for random directions, and sum(dU*U) = sum(dz*z)."""
    r = _rng(12)
    B, T, D, G, W, R = 3, 20, 16, 4, 4, 5
    N = (D // G) * W
    x = r.standard_normal((B, T, D))
    z = r.standard_normal((B, T, R))
    U = r.standard_normal((R, N))
    dy = r.standard_normal((B, T, D))
    dx, dz, dU = orc.bwd_lowrank(x, z, U, dy, G, W)
    vx = r.standard_normal(x.shape)
    # y is linear in x: J_x v = f(v) restricted to the conv part plus v
    jv = orc.fwd_lowrank(vx, z, U, G, W)
    lhs, rhs = float(np.sum(dy * jv)), float(np.sum(dx * vx))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)), "adjoint in x: %r vs %r" % (lhs, rhs)
    # y - x is bilinear in (x, z): directional derivative along z is f(x; vz U) - x
    vz = r.standard_normal(z.shape)
    jz = orc.fwd_lowrank(x, vz, U, G, W) - x
    lhs, rhs = float(np.sum(dy * jz)), float(np.sum(dz * vz))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)), "adjoint in z: %r vs %r" % (lhs, rhs)
    vU = r.standard_normal(U.shape)
    jU = orc.fwd_lowrank(x, z, vU, G, W) - x
    lhs, rhs = float(np.sum(dy * jU)), float(np.sum(dU * vU))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)), "adjoint in U: %r vs %r" % (lhs, rhs)
    a, b = float(np.sum(dU * U)), float(np.sum(dz * z))
    assert abs(a - b) <= 1e-10 * max(1.0, abs(a)), "sum(dU*U) %r != sum(dz*z) %r" % (a, b)


# ---------------------------------------------------------------- decode step
def pin_decode_is_forward_at_last_position(orc):
    """A window of W-1 rows (oldest first) and x_t, run through the forward as a
    W-token sequence whose last token carries the step's filters, gives y_t."""
    r = _rng(13)
    for (B, D, G, W, R) in [(2, 8, 1, 4, 3), (3, 12, 3, 5, 2), (1, 6, 6, 2, 4), (2, 4, 2, 1, 2)]:
        NG = D // G
        state = r.standard_normal((B, W - 1, D))
        x_t = r.standard_normal((B, D))
        xs = np.concatenate([state, x_t[:, None]], axis=1)           # [B, W, D]
        w_full = r.standard_normal((B, W, NG, W))
        y, st = orc.decode(x_t, w_full[:, -1], state, G)
        _close(y, orc.fwd(xs, w_full, G)[:, -1], 1e-13, "explicit decode vs forward")
        _close(st, xs[:, 1:], 0, "window after the step")
        z_full = r.standard_normal((B, W, R))
        U = r.standard_normal((R, NG * W))
        y, st = orc.decode_lowrank(x_t, z_full[:, -1], U, state, G, W)
        _close(y, orc.fwd_lowrank(xs, z_full, U, G, W)[:, -1], 1e-13, "lowrank decode vs forward")
        _close(st, xs[:, 1:], 0, "window after the step (lowrank)")


def pin_decode_steps_match_forward(orc):
    """Stepping from a zero window reproduces the forward token by token (T = 1
    included), and after n steps the window holds x_{n-W+1..n-1} (zeros before 0)."""
    r = _rng(14)
    B, T, D, G, W, R = 2, 9, 8, 2, 4, 3
    NG = D // G
    x = r.standard_normal((B, T, D))
    z = r.standard_normal((B, T, R))
    U = r.standard_normal((R, NG * W))
    w = r.standard_normal((B, T, NG, W))
    ref_lr = orc.fwd_lowrank(x, z, U, G, W)
    ref_ex = orc.fwd(x, w, G)
    s_lr = np.zeros((B, W - 1, D))
    s_ex = np.zeros((B, W - 1, D))
    for t in range(T):
        y, s_lr = orc.decode_lowrank(x[:, t], z[:, t], U, s_lr, G, W)
        _close(y, ref_lr[:, t], 1e-13, "lowrank decode step %d" % t)
        y, s_ex = orc.decode(x[:, t], w[:, t], s_ex, G)
        _close(y, ref_ex[:, t], 1e-13, "explicit decode step %d" % t)
        pad = np.concatenate([np.zeros((B, W - 1, D)), x[:, :t + 1]], axis=1)
        _close(s_lr, pad[:, -(W - 1):] if W > 1 else pad[:, :0], 0, "window after step %d" % t)


# ---------------------------------------------------------------- RoPE after the op
def _angles(r, T, dh):
    th = r.uniform(-np.pi, np.pi, size=(T, dh // 2))
    return th, np.stack([np.cos(th), np.sin(th)], axis=-1)


def pin_rope_complex(orc):
    """Pair (2i, 2i+1) of each rotated head, read as the complex number y_2i + i y_2i+1,
    is multiplied by exp(i theta_{t,i}); channels past n_rot are untouched."""
    r = _rng(31)
    for (D, dh, n_rot) in ((12, 4, 8), (16, 8, 16), (6, 2, 0)):
        B, T = 2, 5
        y = r.standard_normal((B, T, D))
        th, cs = _angles(r, T, dh)
        got = orc.rope(y, cs, dh, n_rot)
        for c0 in range(0, n_rot, dh):
            zc = y[:, :, c0:c0 + dh:2] + 1j * y[:, :, c0 + 1:c0 + dh:2]
            ref = zc * np.exp(1j * th)[None]
            _close(got[:, :, c0:c0 + dh:2], ref.real, 1e-14, "rope real part")
            _close(got[:, :, c0 + 1:c0 + dh:2], ref.imag, 1e-14, "rope imaginary part")
        assert np.array_equal(got[:, :, n_rot:], y[:, :, n_rot:]), "rope touched channels past n_rot"


def pin_rope_transpose(orc):
    """The transpose undoes the rotation and satisfies <R a, b> = <a, R^T b>."""
    r = _rng(32)
    B, T, D, dh, n_rot = 2, 6, 16, 8, 8
    a = r.standard_normal((B, T, D))
    b = r.standard_normal((B, T, D))
    _, cs = _angles(r, T, dh)
    _close(orc.rope(orc.rope(a, cs, dh, n_rot), cs, dh, n_rot, transpose=True), a, 1e-14, "rope^T rope")
    lhs = float(np.sum(orc.rope(a, cs, dh, n_rot) * b))
    rhs = float(np.sum(a * orc.rope(b, cs, dh, n_rot, transpose=True)))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), "rope adjoint %.6e vs %.6e" % (lhs, rhs)


def pin_fd_lowrank_rope(orc):
    """The fused backward (bwd_lowrank of the un-rotated gradient) is the gradient of
    <dy_rot, RoPE(fwd_lowrank)>, by central differences (linear in x, z and U)."""
    r = _rng(33)
    B, T, D, G, W, R, dh, n_rot = 2, 5, 8, 2, 3, 2, 4, 4
    N = (D // G) * W
    x = r.standard_normal((B, T, D))
    z = r.standard_normal((B, T, R))
    U = r.standard_normal((R, N))
    dy = r.standard_normal((B, T, D))
    _, cs = _angles(r, T, dh)
    loss = lambda: float(np.sum(dy * orc.fwd_lowrank_rope(x, z, U, cs, G, W, dh, n_rot)))
    dx, dz, dU = orc.bwd_lowrank_rope(x, z, U, cs, dy, G, W, dh, n_rot)
    _fd_check(loss, {"x": x, "z": z, "U": U}, {"x": dx, "z": dz, "U": dU}, "lowrank + rope")


PINS = [
    pin_hand_example,
    pin_identity_filter_doubles,
    pin_numpy_convolve,
    pin_static_bwd_numpy,
    pin_tying,
    pin_lowrank_equals_explicit,
    pin_causality,
    pin_impulse_response,
    pin_short_sequences,
    pin_fd_lowrank,
    pin_fd_explicit,
    pin_fd_static,
    pin_adjoint_and_invariant,
    pin_decode_is_forward_at_last_position,
    pin_decode_steps_match_forward,
    pin_rope_complex,
    pin_rope_transpose,
    pin_fd_lowrank_rope,
]
