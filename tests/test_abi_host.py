"""Host-only checks of the C ABI: the library loads, exports every symbol that
include/dsc.h declares, and rejects bad arguments before launching anything.

Every call below carries at least one invalid argument, so none of them reaches a
kernel launch (these tests need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsc.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSC_API\s+[\w\s\*]+?\b(dsc_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def dsc():
    import dynamic_short_convolutions_causal_b200 as m
    return m


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("dsc_fwd", "dsc_fwd_lowrank", "dsc_bwd_lowrank", "dsc_bwd_lowrank_workspace_bytes",
              "dsc_static_fwd", "dsc_static_bwd", "dsc_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(dsc):
    out = subprocess.run(["nm", "-D", "--defined-only", dsc.lib_path], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(dsc_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, "declared but not exported: %s" % missing
    for n in _declared():
        assert hasattr(ctypes.CDLL(dsc.lib_path), n)


def test_status_strings(dsc):
    for s in range(4):
        assert dsc.lib.dsc_status_string(s).decode().startswith("DSC_")


FAKE = ctypes.c_void_p(4096)      # a 16-byte aligned non-null address, never dereferenced
ODD = ctypes.c_void_p(4096 + 2)   # misaligned


def _fwd(dsc, x=FAKE, w=FAKE, y=FAKE, B=2, T=8, D=64, G=1, W=4, dt=1):
    return dsc.lib.dsc_fwd(x, w, y, B, T, D, G, W, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), 1), (dict(y=None), 1), (dict(B=0), 1), (dict(T=-1), 1), (dict(D=0), 1),
    (dict(G=3), 1), (dict(G=0), 1), (dict(W=0), 1), (dict(W=9), 2), (dict(D=12, G=1), 2),
    (dict(x=ODD), 2), (dict(w=ODD), 2), (dict(dt=7), 1), (dict(B=1 << 20, T=1 << 12), 2),
])
def test_dsc_fwd_validation(dsc, kw, status):
    assert _fwd(dsc, **kw) == status
    assert dsc.lib.dsc_last_error().decode()


def _lr(dsc, x=FAKE, z=FAKE, U=FAKE, y=FAKE, B=2, T=8, D=64, G=1, W=4, R=32, dt=1):
    return dsc.lib.dsc_fwd_lowrank(x, z, U, y, B, T, D, G, W, R, dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(z=None), 1), (dict(U=None), 1), (dict(R=0), 1), (dict(R=257), 2), (dict(U=ODD), 2),
    (dict(D=60, G=1, dt=1), 2), (dict(D=66, G=1, dt=0), 2), (dict(D=64, G=5), 1),
])
def test_dsc_fwd_lowrank_validation(dsc, kw, status):
    assert _lr(dsc, **kw) == status


def test_dsc_bwd_lowrank_validation(dsc):
    L = dsc.lib
    B, T, D, G, W, R = 2, 8, 64, 1, 4, 32
    need = L.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R, 1)
    if need:
        # workspace too small
        assert L.dsc_bwd_lowrank(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1,
                                 B, T, D, G, W, R, 1, None) == 2
        # missing workspace
        assert L.dsc_bwd_lowrank(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, need,
                                 B, T, D, G, W, R, 1, None) == 1
    assert L.dsc_bwd_lowrank(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1 << 40,
                             B, T, D, G, W, R, 1, None) == 1
    assert L.dsc_bwd_lowrank(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ODD, FAKE, 1 << 40,
                             B, T, D, G, W, R, 1, None) == 2
    assert L.dsc_bwd_lowrank_workspace_bytes(0, T, D, G, W, R, 1) == 0


def test_static_validation(dsc):
    L = dsc.lib
    B, T, D, W = 2, 8, 64, 4
    need = L.dsc_static_bwd_workspace_bytes(B, T, D, W, 1)
    assert need > 0
    assert L.dsc_static_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, B, T, D, W, 1, None) == 2
    assert L.dsc_static_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, need, B, T, D, W, 1, None) == 1
    assert L.dsc_static_fwd(FAKE, FAKE, FAKE, B, T, D, 9, 1, None) == 2
    assert L.dsc_bwd(FAKE, FAKE, FAKE, FAKE, None, B, T, D, 1, W, 1, None) == 1


def test_lowrank_path_query(dsc):
    L = dsc.lib
    assert L.dsc_lowrank_path(0, 8, 64, 1, 4, 32, 1) == -1
    assert L.dsc_lowrank_path(2, 8, 64, 1, 4, 32, 0) == 0      # fp32: CUDA cores
    assert L.dsc_lowrank_path(2, 8, 64, 1, 4, 3, 1) == 0       # R=3: CUDA cores
    assert L.dsc_lowrank_path(2, 8, 64, 1, 4, 32, 1) in (0, 1, 2, 3)


def test_halo_validation(dsc):
    """The sequence-shard fix-ups check their arguments before launching anything."""
    L = dsc.lib
    B, T, D, G, W, R = 2, 8, 64, 1, 4, 32
    # a next-shard halo needs both dy_next and z_next
    assert L.dsc_bwd_lowrank_halo(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE,
                                  B, T, D, G, W, R, 1, None) == 1
    assert L.dsc_bwd_lowrank_halo(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE,
                                  B, T, D, G, W, R, 1, None) == 1
    # required tensors, alignment, sizes
    assert L.dsc_bwd_lowrank_halo(FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, FAKE,
                                  B, T, D, G, W, R, 1, None) == 1
    assert L.dsc_bwd_lowrank_halo(ODD, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE,
                                  B, T, D, G, W, R, 1, None) == 2
    assert L.dsc_fwd_lowrank_halo(FAKE, FAKE, FAKE, FAKE, None, B, T, D, G, W, R, 1, None) == 1
    assert L.dsc_fwd_lowrank_halo(FAKE, FAKE, FAKE, ODD, FAKE, B, T, D, G, W, R, 1, None) == 2
    assert L.dsc_fwd_lowrank_halo(FAKE, FAKE, FAKE, FAKE, FAKE, B, T, D, G, 9, R, 1, None) == 2


def test_rope_validation(dsc):
    """RoPE head size, rotated range, table pointer and path are checked before any launch."""
    L = dsc.lib
    B, T, D, G, W, R = 2, 8, 128, 1, 4, 32
    fwd = lambda cs, dh, n_rot, dt=1: L.dsc_fwd_lowrank_rope(FAKE, FAKE, FAKE, cs, FAKE, B, T, D, G, W, R, dh, n_rot,
                                                             dt, None)
    assert fwd(FAKE, 8, 64) == 1            # dh not a multiple of 16
    assert fwd(FAKE, 64, 96) == 1           # n_rot not a multiple of dh
    assert fwd(FAKE, 64, 192) == 1          # n_rot > D
    assert fwd(None, 64, 64) == 1           # no table
    assert fwd(ODD, 64, 64) == 2            # misaligned table
    assert fwd(FAKE, 64, 64, dt=0) == 2     # fp32: not on the tensor-core path
    need = L.dsc_bwd_lowrank_workspace_bytes(B, T, D, G, W, R, 1)
    bwd = lambda ws_bytes: L.dsc_bwd_lowrank_rope(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws_bytes,
                                                  B, T, D, G, W, R, 64, 64, 1, None)
    if need:
        assert bwd(need - 1) == 2
    assert L.dsc_bwd_lowrank_rope(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 40,
                                  B, T, D, G, W, R, 64, 64, 1, None) == 1
