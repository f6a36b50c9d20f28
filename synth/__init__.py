"""Seeded synthetic inputs for the group-scale search workloads.

This module only draws random tensors of the workloads' shapes, value
distributions and outlier structure.  It holds none of the quantization
arithmetic: both the CUDA path and the CPU oracle are fed from here, and
neither depends on the other.

Workloads (weights W are O x I row-major, groups run along I):

* ``c0``  int3-g64 symmetric, one fp32 matrix 256 x 512, Student-t(4)*0.02,
          2 rows with 5 entries (1 % of 512) scaled x25; activations
          128 x 512 fp32, x = N(0,1) * c_j, c_j ~ LogNormal(0,1).
* ``c1``  int4-g128 asymmetric, bf16 4096 x 4096, N(0, 0.02), 4 input columns
          (0.1 %) scaled x10; activations 2048 x 4096 bf16.
* ``c2``  int3-g64 symmetric MoE stack, 64 experts of bf16 2048 x 7168,
          Student-t(4)*0.015, 10 rows per expert (0.5 %) scaled x15; per-expert
          activations 512 x 7168 bf16; plus one 2048 x 7208 tail matrix.
* ``c3``  int4-g128 asymmetric, the 7 linears of a 27B-dense layer
          (q 5120x5120, k 1024x5120, v 1024x5120, o 5120x5120,
          gate 17408x5120, up 17408x5120, down 5120x17408), N(0, 0.02) with
          round(0.001*I) outlier columns x10; activations 65536 tokens at 4
          input sites (qkv-in, o-in, gate/up-in: 5120; down-in: 17408).
* ``c4``  NVFP4-g16, 128 experts of bf16 1856 x 2688, Student-t(4)*0.02;
          per-expert activations 512 x 2688 bf16.

Random numbers come from ``torch.Generator`` seeded per tensor from
(seed, workload, tensor index), so a tensor is reproducible on its own and
independent of the order in which others are drawn.  A ``scale`` argument
shrinks the matrix and token counts for fast tests while keeping the
distributions and the tail structure.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List

import torch

__all__ = ["Unit", "Site", "Workload", "make", "WORKLOADS", "student_t", "lognormal_channels"]


def _gen(device, seed: int, *tags) -> torch.Generator:
    key = zlib.crc32(repr((seed,) + tuple(tags)).encode())
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(key))
    return g


def student_t(shape, nu: int, gen: torch.Generator, device) -> torch.Tensor:
    """Student-t(nu) samples for integer nu: Z / sqrt(chi2_nu / nu)."""
    z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        chi2 += torch.randn(shape, generator=gen, device=device, dtype=torch.float32).square()
    return z / torch.sqrt(chi2 / nu)


def lognormal_channels(n: int, gen: torch.Generator, device) -> torch.Tensor:
    """Per-channel activation scales c_j ~ LogNormal(0, 1)."""
    return torch.exp(torch.randn(n, generator=gen, device=device, dtype=torch.float32))


@dataclasses.dataclass
class Site:
    """Calibration activations feeding one or more matrices: X is [n_mat, T, I]."""
    name: str
    X: torch.Tensor


@dataclasses.dataclass
class Unit:
    """A batch of same-shaped weight matrices W [n_mat, O, I] quantized alike."""
    name: str
    fmt: str            # "int3_g64_sym" | "int4_g128_asym" | "nvfp4_g16"
    W: torch.Tensor
    site: str           # name of the Site whose imatrix weights this unit
    timed: bool = True  # False for parity-only extras (the C2 tail matrix)


@dataclasses.dataclass
class Workload:
    name: str
    units: List[Unit]
    sites: Dict[str, Site]

    @property
    def n_weights(self) -> int:
        return sum(u.W.numel() for u in self.units if u.timed)


def _scaled(n: int, scale: float, multiple: int = 1, minimum: int = 1) -> int:
    v = max(minimum, int(round(n * scale)))
    return max(multiple, (v // multiple) * multiple)


def _activations(n_mat, T, I, dtype, gen, device) -> torch.Tensor:
    X = torch.empty((n_mat, T, I), dtype=dtype, device=device)
    for e in range(n_mat):
        c = lognormal_channels(I, gen, device)
        x = torch.randn((T, I), generator=gen, device=device, dtype=torch.float32) * c
        X[e] = x.to(dtype)
    return X


def _dims(name: str, scale: float):
    """Shapes of a workload at ``scale``: (matrices E, rows O, columns I,
    tokens T); c3's per-linear shapes are scaled the same way from
    C3_LINEARS / C3_SITES."""
    if name == "c0":
        return 1, 256, 512, 128
    if name == "c1":
        return 1, _scaled(4096, scale, 8), _scaled(4096, scale, 128), _scaled(2048, scale, 8)
    if name == "c2":
        return (_scaled(64, scale, 1), _scaled(2048, scale, 8),
                7168 if scale >= 1 else _scaled(7168, scale, 64, 128), _scaled(512, scale, 8))
    if name == "c3":
        return 1, None, None, _scaled(8 * 8192, scale, 8)
    if name == "c4":
        return (_scaled(128, scale, 1), _scaled(1856, scale, 8),
                2688 if scale >= 1 else _scaled(2688, scale, 16, 32), _scaled(512, scale, 8))
    raise KeyError(name)


def _c0(device, seed, scale, max_mats=None):
    g = _gen(device, seed, "c0", "W")
    _, O, I, T = _dims("c0", scale)
    W = student_t((O, I), 4, g, device) * 0.02
    rows = torch.randperm(O, generator=g, device=device)[:2]
    n_out = max(1, round(0.01 * I))
    for r in rows.tolist():
        cols = torch.randperm(I, generator=g, device=device)[:n_out]
        W[r, cols] *= 25.0
    X = _activations(1, T, I, torch.float32, _gen(device, seed, "c0", "X"), device)
    return Workload("c0", [Unit("w", "int3_g64_sym", W.unsqueeze(0), "x")], {"x": Site("x", X)})


def _c1(device, seed, scale, max_mats=None):
    g = _gen(device, seed, "c1", "W")
    _, O, I, T = _dims("c1", scale)
    W = torch.randn((O, I), generator=g, device=device) * 0.02
    cols = torch.randperm(I, generator=g, device=device)[: max(1, round(0.001 * I))]
    W[:, cols] *= 10.0
    X = _activations(1, T, I, torch.bfloat16, _gen(device, seed, "c1", "X"), device)
    return Workload("c1", [Unit("w", "int4_g128_asym", W.to(torch.bfloat16).unsqueeze(0), "x")],
                    {"x": Site("x", X)})


def _c2(device, seed, scale, max_mats=None):
    E, O, I, T = _dims("c2", scale)
    E = E if max_mats is None else min(E, max_mats)
    g = _gen(device, seed, "c2", "W")
    W = torch.empty((E, O, I), dtype=torch.bfloat16, device=device)
    n_rows = max(1, round(0.005 * O))
    for e in range(E):
        w = student_t((O, I), 4, g, device) * 0.015
        rows = torch.randperm(O, generator=g, device=device)[:n_rows]
        w[rows] *= 15.0
        W[e] = w.to(torch.bfloat16)
    X = _activations(E, T, I, torch.bfloat16, _gen(device, seed, "c2", "X"), device)
    # parity-only tail matrix: I = 7168 + 40 (the last 64-group holds 40 weights)
    gt = _gen(device, seed, "c2", "tail")
    It = I + 40
    wt = student_t((O, It), 4, gt, device) * 0.015
    rows = torch.randperm(O, generator=gt, device=device)[:n_rows]
    wt[rows] *= 15.0
    Xt = _activations(1, T, It, torch.bfloat16, _gen(device, seed, "c2", "Xtail"), device)
    units = [Unit("experts", "int3_g64_sym", W, "x"),
             Unit("tail", "int3_g64_sym", wt.to(torch.bfloat16).unsqueeze(0), "xtail", timed=False)]
    return Workload("c2", units, {"x": Site("x", X), "xtail": Site("xtail", Xt)})


C3_LINEARS = [  # name, O, I, input site
    ("q", 5120, 5120, "qkv_in"), ("k", 1024, 5120, "qkv_in"), ("v", 1024, 5120, "qkv_in"),
    ("o", 5120, 5120, "o_in"), ("gate", 17408, 5120, "gateup_in"), ("up", 17408, 5120, "gateup_in"),
    ("down", 5120, 17408, "down_in"),
]
C3_SITES = [("qkv_in", 5120), ("o_in", 5120), ("gateup_in", 5120), ("down_in", 17408)]


def _c3(device, seed, scale, max_mats=None):
    T = _dims("c3", scale)[3]
    units = []
    for name, O, I, site in C3_LINEARS:
        g = _gen(device, seed, "c3", "W", name)
        Os, Is = _scaled(O, scale, 8), _scaled(I, scale, 128)
        w = torch.randn((Os, Is), generator=g, device=device) * 0.02
        cols = torch.randperm(Is, generator=g, device=device)[: max(1, round(0.001 * Is))]
        w[:, cols] *= 10.0
        units.append(Unit(name, "int4_g128_asym", w.to(torch.bfloat16).unsqueeze(0), site))
    sites = {}
    for name, I in C3_SITES:
        Is = _scaled(I, scale, 128)
        sites[name] = Site(name, _activations(1, T, Is, torch.bfloat16,
                                              _gen(device, seed, "c3", "X", name), device))
    return Workload("c3", units, sites)


def _c4(device, seed, scale, max_mats=None):
    E, O, I, T = _dims("c4", scale)
    E = E if max_mats is None else min(E, max_mats)
    g = _gen(device, seed, "c4", "W")
    W = torch.empty((E, O, I), dtype=torch.bfloat16, device=device)
    for e in range(E):
        W[e] = (student_t((O, I), 4, g, device) * 0.02).to(torch.bfloat16)
    X = _activations(E, T, I, torch.bfloat16, _gen(device, seed, "c4", "X"), device)
    return Workload("c4", [Unit("experts", "nvfp4_g16", W, "x")], {"x": Site("x", X)})


WORKLOADS = {"c0": _c0, "c1": _c1, "c2": _c2, "c3": _c3, "c4": _c4}

DESCRIPTIONS = {
    "c0": "int3-g64 sym, fp32 W 256x512 (t4*0.02, 2 outlier rows), X 128x512",
    "c1": "int4-g128 asym, bf16 W 4096x4096 (N(0,0.02), 0.1% cols x10), X 2048x4096",
    "c2": "int3-g64 sym MoE, 64 x bf16 2048x7168 (t4*0.015, 0.5% rows x15), X 64x512x7168",
    "c3": "int4-g128 asym, 7 linears of a 27B-dense layer, X 4 sites x 65536 tokens",
    "c4": "NVFP4-g16, 128 x bf16 1856x2688 (t4*0.02), X 128x512x2688",
}


def make(name: str, device="cpu", seed: int = 0, scale: float = 1.0, max_mats=None) -> Workload:
    """Build workload ``name`` on ``device``; ``scale`` < 1 shrinks it for
    tests; ``max_mats`` draws only the first experts of a MoE workload (the
    same values as the first experts of the whole draw on that device)."""
    return WORKLOADS[name](device, seed, scale, max_mats)


def layout(name: str, scale: float = 1.0):
    """The workload's shapes without drawing anything: ``units`` as
    (name, fmt, (E, O, I), site, timed) and ``sites`` as name -> (E, T, I, dtype)."""
    E, O, I, T = _dims(name, scale)
    if name == "c0":
        return {"units": [("w", "int3_g64_sym", (1, O, I), "x", True)], "sites": {"x": (1, T, I, "f32")}}
    if name == "c1":
        return {"units": [("w", "int4_g128_asym", (1, O, I), "x", True)], "sites": {"x": (1, T, I, "bf16")}}
    if name == "c2":
        return {"units": [("experts", "int3_g64_sym", (E, O, I), "x", True),
                          ("tail", "int3_g64_sym", (1, O, I + 40), "xtail", False)],
                "sites": {"x": (E, T, I, "bf16"), "xtail": (1, T, I + 40, "bf16")}}
    if name == "c3":
        units = [(n, "int4_g128_asym", (1, _scaled(o, scale, 8), _scaled(i, scale, 128)), s, True)
                 for n, o, i, s in C3_LINEARS]
        return {"units": units, "sites": {n: (1, T, _scaled(i, scale, 128), "bf16") for n, i in C3_SITES}}
    if name == "c4":
        return {"units": [("experts", "nvfp4_g16", (E, O, I), "x", True)], "sites": {"x": (E, T, I, "bf16")}}
    raise KeyError(name)


def random_groups(n_groups: int, group: int, dist: str, seed: int, device="cpu",
                  dtype=torch.float32, outlier_frac: float = 0.0,
                  outlier_mult: float = 10.0) -> torch.Tensor:
    """A [n_groups, group] weight block for unit tests (t4 or normal entries)."""
    g = _gen(device, seed, "groups", dist, n_groups, group)
    if dist == "t4":
        w = student_t((n_groups, group), 4, g, device) * 0.02
    else:
        w = torch.randn((n_groups, group), generator=g, device=device) * 0.02
    if outlier_frac > 0:
        mask = torch.rand((n_groups, group), generator=g, device=device) < outlier_frac
        w = torch.where(mask, w * outlier_mult, w)
    return w.to(dtype)


def random_imatrix(n: int, seed: int, device="cpu") -> torch.Tensor:
    """A positive per-column importance vector shaped like E[x^2] with LogNormal scales."""
    g = _gen(device, seed, "imatrix", n)
    c = lognormal_channels(n, g, device)
    return (c * c * (0.5 + torch.rand(n, generator=g, device=device))).to(torch.float32)
