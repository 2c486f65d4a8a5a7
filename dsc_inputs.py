"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module holds shapes, value distributions and seeds only; none of the method's
arithmetic lives here.  Every tensor is drawn as float32 from a seeded
``torch.Generator`` in the order the workload lists it, scaled by its standard
deviation, then cast to the working dtype (bf16 rounding happens once, here, so the
device path and the CPU oracle read identical values).

Workloads ("Convolucoes Curtas Dinamicas Melhoram Transformers", section
"Implementacao de Treinamento Eficiente": the method is applied to the stacked Q/K/V
projections and, in a variant, after every linear layer; the 2B-parameter model it
is measured on is stood in for by its activation shapes):

  explicit_fp32_small  x [1,64,64] ~N(0,1); w [1,64,8,4] ~N(0,1/4); G=8, W=4; fp32
  tied_qkv             x [8,2048,6144] ~N(0,1); w [8,2048,96,4] ~N(0,1/4); G=64; bf16
  lowrank_qkv          x [8,2048,6144]; z [8,2048,32] ~N(0,1); U [32,24576] ~N(0,1/32);
                       G=1, W=4; dy ~N(0,1); bf16
  lowrank_mlp          x [2,8192,8192]; z [2,8192,64]; U [64,16384] ~N(0,1/64); G=4, W=8;
                       dy ~N(0,1); static filters ws [8192,8] ~N(0,1/8); bf16

"N(0, v)" is read as variance v (standard deviation sqrt(v)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    D: int
    G: int
    W: int
    R: int = 0              # 0: explicit filters (no low-rank generator)
    dtype: str = "bf16"     # "bf16" or "f32"
    seed: int = 0
    w_var: float = 0.25     # variance of explicit filters
    u_var: float = 0.0      # variance of U (defaults to 1/R)
    ws_var: float = 0.125   # variance of static filters
    notes: str = field(default="", compare=False)

    @property
    def NG(self) -> int:
        return self.D // self.G

    @property
    def N(self) -> int:
        return self.NG * self.W

    @property
    def tokens(self) -> int:
        return self.B * self.T


WORKLOADS = {
    "explicit_fp32_small": Workload("explicit_fp32_small", 1, 64, 64, 8, 4, 0, "f32", 0, 0.25),
    "tied_qkv": Workload("tied_qkv", 8, 2048, 6144, 64, 4, 0, "bf16", 1, 0.25),
    "lowrank_qkv": Workload("lowrank_qkv", 8, 2048, 6144, 1, 4, 32, "bf16", 2, u_var=1 / 32),
    "lowrank_mlp": Workload("lowrank_mlp", 2, 8192, 8192, 4, 8, 64, "bf16", 4, u_var=1 / 64,
                            ws_var=1 / 8),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _draw(gen, shape, std, dtype, device):
    t = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make(wl: Workload, device="cpu", parts=("x", "w", "z", "U", "dy", "ws")) -> dict:
    """Draw the workload's tensors.  ``parts`` selects which are drawn; the draw
    order is fixed (x, w, z, U, dy, ws) so a given seed always yields the same
    values for the parts that are drawn together."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    dt = torch_dtype(wl.dtype)
    out = {}
    shapes = {
        "x": ((wl.B, wl.T, wl.D), 1.0),
        "w": ((wl.B, wl.T, wl.NG, wl.W), math.sqrt(wl.w_var)),
        "z": ((wl.B, wl.T, wl.R), 1.0),
        "U": ((wl.R, wl.N), math.sqrt(wl.u_var if wl.u_var > 0 else 1.0 / max(wl.R, 1))),
        "dy": ((wl.B, wl.T, wl.D), 1.0),
        "ws": ((wl.D, wl.W), math.sqrt(wl.ws_var)),
    }
    for name in ("x", "w", "z", "U", "dy", "ws"):
        if name not in parts:
            continue
        if name in ("z", "U") and wl.R == 0:
            continue
        shape, std = shapes[name]
        out[name] = _draw(gen, shape, std, dt, device)
    return out


def small(B, T, D, G, W, R=0, dtype="bf16", seed=0, **kw) -> Workload:
    """An ad-hoc workload with the same distributions as the named ones."""
    return Workload("adhoc", B, T, D, G, W, R, dtype, seed, **kw)


def scaled(wl: Workload, **changes) -> Workload:
    return replace(wl, **changes)
