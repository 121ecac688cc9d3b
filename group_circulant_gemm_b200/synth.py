"""Seeded synthetic inputs for EQ-Linear workloads.

This module only draws random numbers and casts them; it holds none of the
layer's arithmetic, so both the CUDA path and the float64 oracle can be fed the
same arrays.  Recipe (same for every workload):

* ``numpy.random.default_rng(seed)``, float64 normal draws in the fixed order
  X, W, bias, dY (the bias of a bias-free workload is drawn and then zeroed, so
  the later draws do not move; dY is drawn last, only when asked for), then
  cast to the workload dtype with round-to-nearest.
* ``X ~ N(0, 1)`` of shape ``[N, C*T]`` (feature index ``c*T + t``).
* ``W ~ N(0, 1/(C*T))`` of shape ``[D, C, T]`` (variance ``1/(C*T)``).
* ``bias ~ N(0, 0.01)`` (variance 0.01) of shape ``[D]``, or zeros.
* ``dY ~ N(0, 1)`` of shape ``[N, D*T]`` (upstream gradient).

The named shapes are ViT/Swin-style projections: N = images x tokens rows,
C -> D channels per group element, T = group order.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    N: int
    C: int
    D: int
    dtype: str  # "f32" or "f16"
    bias: bool = True
    seed: int = 1234

    @property
    def np_dtype(self):
        return np.float32 if self.dtype == "f32" else np.float16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the layer's benchmark plan, seeds 1234 + index.
WORKLOADS = {
    "p4_small_f32": Workload("p4_small_f32", 4, 256, 16, 16, "f32", True, 1234),
    "p4_vitb_proj_f32": Workload("p4_vitb_proj_f32", 4, 12608, 192, 192, "f32", False, 1235),
    "p4_vitb_fc1_f16": Workload("p4_vitb_fc1_f16", 4, 12608, 192, 768, "f16", True, 1236),
    "p4_vitb_fc2_f16": Workload("p4_vitb_fc2_f16", 4, 12608, 768, 192, "f16", True, 1236),
    "p4_vith_fc1_f16": Workload("p4_vith_fc1_f16", 4, 8224, 320, 1280, "f16", True, 1237),
    "c8_1024_f16": Workload("c8_1024_f16", 8, 16384, 128, 128, "f16", True, 1238),
}


def make_inputs(w: Workload, need_dy: bool = False, rows: int | None = None):
    """Return dict(X, W, bias, dY) as numpy arrays of the workload dtype.

    ``rows`` truncates N (the draws are made for the full N first so a
    truncated X is a prefix of the full one)."""
    rng = np.random.default_rng(w.seed)
    N, C, D, T = w.N, w.C, w.D, w.T
    X = rng.standard_normal((N, C * T))
    W = rng.standard_normal((D, C, T)) * np.sqrt(1.0 / (C * T))
    b = rng.standard_normal((D,)) * np.sqrt(0.01)
    if not w.bias:
        b = np.zeros((D,))
    dY = rng.standard_normal((N, D * T)) if need_dy else None
    if rows is not None:
        X = X[:rows]
        dY = None if dY is None else dY[:rows]
    dt = w.np_dtype
    out = {
        "X": np.ascontiguousarray(X.astype(dt)),
        "W": np.ascontiguousarray(W.astype(dt)),
        "bias": np.ascontiguousarray(b.astype(dt)),
    }
    if dY is not None:
        out["dY"] = np.ascontiguousarray(dY.astype(dt))
    return out


def make_arrays(seed: int, T: int, N: int, C: int, D: int, dtype: str = "f32",
                bias: bool = True, need_dy: bool = False):
    """Ad-hoc shape with the same recipe (used for edge-case tests)."""
    return make_inputs(Workload("adhoc", T, N, C, D, dtype, bias, seed), need_dy=need_dy)
