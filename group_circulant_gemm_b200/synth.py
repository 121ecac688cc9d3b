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
    # the ViT-B MLP pair over the dihedral group D4 (8 elements): 768 -> 3072 -> 768
    # features as 96 -> 384 -> 96 channels per group element
    "p4m_vitb_fc1_f16": Workload("p4m_vitb_fc1_f16", 8, 12608, 96, 384, "f16", True, 1239),
    "p4m_vitb_fc2_f16": Workload("p4m_vitb_fc2_f16", 8, 12608, 384, 96, "f16", True, 1239),
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


@dataclass(frozen=True)
class ConvWorkload:
    """A group-circulant convolution: N images of H x W pixels, C -> D channels per
    group element, KH x KW taps, stride 1, zero padding (ph, pw)."""
    name: str
    T: int
    N: int
    H: int
    W: int
    C: int
    D: int
    KH: int
    KW: int
    ph: int
    pw: int
    dtype: str = "f16"
    seed: int = 1300
    backward: bool = False  # a training step: forward, dX and dWc

    @property
    def Ho(self) -> int:
        return self.H + 2 * self.ph - self.KH + 1

    @property
    def Wo(self) -> int:
        return self.W + 2 * self.pw - self.KW + 1

    def with_(self, **kw) -> "ConvWorkload":
        return replace(self, **kw)


# A ResNet-stage shape for p4 feature maps (64 images, 56 x 56, 64 -> 64
# channels per group element, 3 x 3): the pages measure no convolution, so this
# is a plain choice of a common CNN stage, not a published benchmark.
CONV_WORKLOADS = {
    "p4_conv3x3_f16": ConvWorkload("p4_conv3x3_f16", 4, 64, 56, 56, 64, 64, 3, 3, 1, 1, "f16",
                                   1300),
    "p4_conv3x3_fwd_bwd_f16": ConvWorkload("p4_conv3x3_fwd_bwd_f16", 4, 64, 56, 56, 64, 64, 3,
                                           3, 1, 1, "f16", 1300, True),
}


def make_conv_inputs(w: ConvWorkload, images: int | None = None, need_dy: bool = False):
    """dict(X [N, H, W, C*T], Wc [KH, KW, D, C, T], bias [D], and with need_dy
    dY [N, Ho, Wo, D*T]) with the layer's recipe: float64 normal draws in the
    order X, Wc, bias, dY from default_rng(seed), Wc ~ N(0, 1/(C*T*KH*KW)),
    bias ~ N(0, 0.01), dY ~ N(0, 1), cast to the dtype.  ``images`` keeps a
    prefix of the images (drawn in full first)."""
    rng = np.random.default_rng(w.seed)
    X = rng.standard_normal((w.N, w.H, w.W, w.C * w.T))
    Wc = rng.standard_normal((w.KH, w.KW, w.D, w.C, w.T)) * np.sqrt(
        1.0 / (w.C * w.T * w.KH * w.KW))
    b = rng.standard_normal((w.D,)) * np.sqrt(0.01)
    dY = rng.standard_normal((w.N, w.Ho, w.Wo, w.D * w.T)) if need_dy else None
    if images is not None:
        X = X[:images]
        dY = None if dY is None else dY[:images]
    dt = np.float16 if w.dtype == "f16" else np.float32
    out = {"X": np.ascontiguousarray(X.astype(dt)), "Wc": np.ascontiguousarray(Wc.astype(dt)),
           "bias": np.ascontiguousarray(b.astype(dt))}
    if dY is not None:
        out["dY"] = np.ascontiguousarray(dY.astype(dt))
    return out


# Extreme group vectors for the FP16 range tests: for each group order, sign
# patterns that put the largest possible magnitude into one frequency
# (constant, alternating, and the sign patterns of the first harmonics).  Plain
# integer tables: a planted group is amplitude * pattern.
RANGE_PATTERNS = {
    3: [[1, 1, 1], [1, -1, -1], [0, 1, -1]],
    4: [[1, 1, 1, 1], [1, -1, 1, -1], [1, 0, -1, 0], [0, -1, 0, 1], [1, 1, -1, -1]],
    8: [[1] * 8, [1, -1] * 4, [1, 1, 0, -1, -1, -1, 0, 1], [0, -1, -1, -1, 0, 1, 1, 1],
        [1, 0, -1, 0] * 2, [1, -1, 0, 1, -1, 1, 0, -1], [1, 1, -1, -1] * 2],
}


def make_range_inputs(seed: int, T: int, N: int, C: int, D: int,
                      x=(1.0, 0.0), w=(1.0, 0.0), dy=(1.0, 0.0), need_dy: bool = False,
                      dtype: str = "f16"):
    """Inputs that reach the edge of the FP16 range.

    Each of X [N, C*T], W [D, C, T], dY [N, D*T] is given as (fill, amp): every
    entry is first drawn as fill * U(-1, 1) (W's fill also times 1/sqrt(C*T)),
    then about one group vector in four is replaced by amp * (a random pattern
    of RANGE_PATTERNS[T]) * (random sign), so that a group's DFT reaches T * amp.
    bias ~ N(0, 0.01).  Draw order: X, W, bias, dY, each array's uniform fill,
    then its group mask, pattern choice and signs.  Cast with round-to-nearest."""
    rng = np.random.default_rng(seed)
    pats = np.asarray(RANGE_PATTERNS[T], dtype=np.float64)

    def draw(shape_groups, fill, amp):
        a = rng.uniform(-1.0, 1.0, shape_groups + (T,)) * fill
        mask = rng.uniform(0.0, 1.0, shape_groups) < 0.25
        which = rng.integers(0, len(pats), shape_groups)
        sign = np.where(rng.uniform(0.0, 1.0, shape_groups) < 0.5, -1.0, 1.0)
        if amp > 0:
            a = np.where(mask[..., None], amp * sign[..., None] * pats[which], a)
        return a

    X = draw((N, C), *x).reshape(N, C * T)
    W = draw((D, C), w[0] / np.sqrt(C * T), w[1])
    b = rng.standard_normal((D,)) * np.sqrt(0.01)
    dY = draw((N, D), *dy).reshape(N, D * T) if need_dy else None
    dt = np.float32 if dtype == "f32" else np.float16
    out = {"X": np.ascontiguousarray(X.astype(dt)), "W": np.ascontiguousarray(W.astype(dt)),
           "bias": np.ascontiguousarray(b.astype(dt))}
    if dY is not None:
        out["dY"] = np.ascontiguousarray(dY.astype(dt))
    return out
