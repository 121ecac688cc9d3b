"""Float64 CPU oracle for the Flash EQ-Linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and the
two share no code: the arithmetic lives in ``eqlinear_oracle.c`` (plain C,
float64, OpenMP), loaded here through ctypes.

What each function computes, and the passage of the "Flash EQ-Linear" summary
(gist.science/ko/paper/2607.21271) it follows:

* :func:`forward` -- the operator's plain definition,
  ``Y[n,d,s] = bias[d] + sum_{c,t} W[d,c,(t-s) mod T] X[n,c,t]``, input feature
  index ``c*T+t`` ("Key insight": group-circulant weights; "Contributions" item 2:
  the fast method is exact, so the definition is the oracle).
* :func:`backward_input`, :func:`backward_weight` -- the gradients of that
  definition ("Implementation", bullet 1 names backward kernels but no formula).
* :func:`forward_spectral` -- the method's own route ("Algorithmic approach"
  items 1-3): DFT over the group axis, per-frequency products on the
  non-redundant half of the spectrum, inverse DFT, with a counter of real MACs
  ("Specialisation for p4", bullet 3: 6 real GEMMs, 16/6 fewer MACs).
* :func:`p4_transform_matrices` -- the real 4x4 DFT / inverse-DFT pair for the
  p4 group ("Specialisation for p4", bullets 1-2: coefficients 0, +-1, +-1/2).
* :func:`d4_forward` -- the layer over the dihedral group D4 (p4m), the
  reflection group named in "Limitations and future work" (no formula given):
  the group cross-correlation ``Y[n,d,g] = bias[d] + sum_{c,h} W[d,c,g^-1 h]
  X[n,c,h]`` with elements ``g = a + 4b`` for ``r^a m^b``.
* :func:`conv_forward` -- the group-circulant convolution ("Limitations and
  future work" names equivariant convolution as the next operator; no formula
  is given): the EQ-Linear's channel mixing at every tap of a KH x KW kernel,
  stride 1, zero padding.

Every function is pinned by tests/test_oracle_pins.py against values fixed by
something other than this code (dense replicated matmul, numpy FFT, closed
forms, hand-worked examples, exact MAC counts).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eqlinear_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile eqlinear_oracle.c into liboracle.so (gcc, -O3, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lp = ctypes.POINTER(ctypes.c_int64)
            for name in ("eqlo_forward", "eqlo_forward_spectral"):
                fn = getattr(lib, name)
                fn.argtypes = [ctypes.c_int, i64, i64, i64, dp, dp, dp, dp]
                fn.restype = i64
            lib.eqlo_backward_input.argtypes = [ctypes.c_int, i64, i64, i64, dp, dp, dp]
            lib.eqlo_backward_input.restype = i64
            lib.eqlo_backward_weight.argtypes = [ctypes.c_int, i64, i64, i64, dp, dp, dp, dp]
            lib.eqlo_backward_weight.restype = i64
            lib.eqlo_backward_weight_pairs.argtypes = [ctypes.c_int, i64, i64, i64, dp, dp,
                                                       i64, lp, lp, dp]
            lib.eqlo_backward_weight_pairs.restype = None
            lib.eqlo_gelu.argtypes = [i64, dp]
            lib.eqlo_gelu.restype = None
            lib.eqlo_p4_transform_matrices.argtypes = [dp, dp]
            lib.eqlo_p4_transform_matrices.restype = None
            lib.eqlo_conv_forward.argtypes = [ctypes.c_int, i64, i64, i64, i64, i64,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, dp, dp, dp, dp]
            lib.eqlo_conv_forward.restype = i64
            lib.eqlo_d4_forward.argtypes = [i64, i64, i64, dp, dp, dp, dp]
            lib.eqlo_d4_forward.restype = i64
            lib.eqlo_d4_backward_input.argtypes = [i64, i64, i64, dp, dp, dp]
            lib.eqlo_d4_backward_input.restype = i64
            lib.eqlo_d4_backward_weight.argtypes = [i64, i64, i64, dp, dp, dp, dp]
            lib.eqlo_d4_backward_weight.restype = i64
            ci = ctypes.c_int
            lib.eqlo_conv_backward_input.argtypes = [ci, i64, i64, i64, i64, i64, ci, ci, ci, ci,
                                                     dp, dp, dp]
            lib.eqlo_conv_backward_input.restype = None
            lib.eqlo_conv_backward_weight.argtypes = [ci, i64, i64, i64, i64, i64, ci, ci, ci,
                                                      ci, dp, dp, dp, dp]
            lib.eqlo_conv_backward_weight.restype = None
            lib.eqlo_set_threads.argtypes = [ctypes.c_int]
            lib.eqlo_set_threads.restype = None
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shapes(T: int, X: np.ndarray, W: np.ndarray):
    D, C, TW = W.shape
    if TW != T:
        raise ValueError(f"W has group axis {TW}, expected T={T}")
    if X.ndim != 2 or X.shape[1] != C * T:
        raise ValueError(f"X must be [N, C*T] = [N, {C * T}], got {X.shape}")
    return X.shape[0], C, D


def forward(T: int, X, W, bias=None, return_macs: bool = False, act: str = "none"):
    """Y[N, D*T] in float64 from X[N, C*T], W[D, C, T], bias[D] or None;
    act="gelu" applies the exact GELU to every output feature (EQ-MLP block)."""
    if act not in ("none", "gelu"):
        raise ValueError(f"unknown activation {act!r}")
    lib = _load()
    X, W = _f64(X), _f64(W)
    N, C, D = _shapes(T, X, W)
    b = None if bias is None else _f64(bias)
    Y = np.empty((N, D * T), dtype=np.float64)
    macs = lib.eqlo_forward(T, N, C, D, _ptr(X), _ptr(W), _ptr(b), _ptr(Y))
    if act == "gelu":
        lib.eqlo_gelu(Y.size, _ptr(Y))
    return (Y, macs) if return_macs else Y


def gelu(y):
    """The activation alone, elementwise, in float64 (for pins and composition)."""
    lib = _load()
    y = _f64(y).copy()
    lib.eqlo_gelu(y.size, _ptr(y))
    return y


def forward_spectral(T: int, X, W, bias=None, return_macs: bool = False):
    """Same output as :func:`forward`, computed through the DFT route."""
    if T > 126:
        raise ValueError("forward_spectral supports T <= 126")
    lib = _load()
    X, W = _f64(X), _f64(W)
    N, C, D = _shapes(T, X, W)
    b = None if bias is None else _f64(bias)
    Y = np.empty((N, D * T), dtype=np.float64)
    macs = lib.eqlo_forward_spectral(T, N, C, D, _ptr(X), _ptr(W), _ptr(b), _ptr(Y))
    return (Y, macs) if return_macs else Y


def backward_input(T: int, dY, W):
    """dX[N, C*T] from dY[N, D*T] and W[D, C, T]."""
    lib = _load()
    dY, W = _f64(dY), _f64(W)
    D, C, _ = W.shape
    if dY.ndim != 2 or dY.shape[1] != D * T:
        raise ValueError(f"dY must be [N, {D * T}]")
    N = dY.shape[0]
    dX = np.empty((N, C * T), dtype=np.float64)
    lib.eqlo_backward_input(T, N, C, D, _ptr(dY), _ptr(W), _ptr(dX))
    return dX


def backward_weight(T: int, X, dY, D: int):
    """(dW[D, C, T], dbias[D]) from X[N, C*T] and dY[N, D*T]."""
    lib = _load()
    X, dY = _f64(X), _f64(dY)
    N = X.shape[0]
    C = X.shape[1] // T
    if X.shape[1] != C * T or dY.shape != (N, D * T):
        raise ValueError("shape mismatch")
    dW = np.empty((D, C, T), dtype=np.float64)
    db = np.empty((D,), dtype=np.float64)
    lib.eqlo_backward_weight(T, N, C, D, _ptr(X), _ptr(dY), _ptr(dW), _ptr(db))
    return dW, db


def backward_weight_pairs(T: int, X, dY, D: int, d_idx, c_idx):
    """dW[d_i, c_i, :] for sampled pairs, shape [len(d_idx), T]."""
    lib = _load()
    X, dY = _f64(X), _f64(dY)
    N = X.shape[0]
    C = X.shape[1] // T
    d_idx = np.ascontiguousarray(np.asarray(d_idx, dtype=np.int64))
    c_idx = np.ascontiguousarray(np.asarray(c_idx, dtype=np.int64))
    if d_idx.shape != c_idx.shape or d_idx.ndim != 1:
        raise ValueError("d_idx and c_idx must be 1-D and the same length")
    if (d_idx < 0).any() or (d_idx >= D).any() or (c_idx < 0).any() or (c_idx >= C).any():
        raise ValueError("pair index out of range")
    out = np.empty((d_idx.shape[0], T), dtype=np.float64)
    lp = ctypes.POINTER(ctypes.c_int64)
    lib.eqlo_backward_weight_pairs(T, N, C, D, _ptr(X), _ptr(dY), d_idx.shape[0],
                                   d_idx.ctypes.data_as(lp), c_idx.ctypes.data_as(lp),
                                   _ptr(out))
    return out


def p4_transform_matrices():
    """(F, G): real 4x4 forward DFT (rows Re0, Re2, Re1, Im1) and its inverse."""
    lib = _load()
    F = np.empty((4, 4), dtype=np.float64)
    G = np.empty((4, 4), dtype=np.float64)
    lib.eqlo_p4_transform_matrices(_ptr(F), _ptr(G))
    return F, G


def d4_forward(X, W, bias=None, return_macs: bool = False, act: str = "none"):
    """Y[N, D*8] in float64 from X[N, C*8], W[D, C, 8], bias[D] or None: the layer
    over D4, feature index c*8 + g with g = a + 4b for r^a m^b."""
    if act not in ("none", "gelu"):
        raise ValueError(act)
    X, W = _f64(X), _f64(W)
    D, C, G = W.shape
    if G != 8 or X.ndim != 2 or X.shape[1] != C * 8:
        raise ValueError("X must be [N, C*8] and W [D, C, 8]")
    N = X.shape[0]
    b = None if bias is None else _f64(bias)
    Y = np.empty((N, D * 8), dtype=np.float64)
    macs = _load().eqlo_d4_forward(N, C, D, _ptr(X), _ptr(W), _ptr(b), _ptr(Y))
    if act == "gelu":
        _load().eqlo_gelu(Y.size, _ptr(Y))
    return (Y, macs) if return_macs else Y


def d4_backward_input(dY, W):
    """dX[N, C*8] in float64 from dY[N, D*8] and W[D, C, 8]: the gradient of
    d4_forward with respect to X."""
    dY, W = _f64(dY), _f64(W)
    D, C, G = W.shape
    if G != 8 or dY.ndim != 2 or dY.shape[1] != D * 8:
        raise ValueError("dY must be [N, D*8] and W [D, C, 8]")
    N = dY.shape[0]
    dX = np.empty((N, C * 8), dtype=np.float64)
    _load().eqlo_d4_backward_input(N, C, D, _ptr(dY), _ptr(W), _ptr(dX))
    return dX


def d4_backward_weight(X, dY, D: int):
    """(dW[D, C, 8], dbias[D]) in float64 from X[N, C*8] and dY[N, D*8]: the
    gradients of d4_forward with respect to W and the bias."""
    X, dY = _f64(X), _f64(dY)
    N = X.shape[0]
    C = X.shape[1] // 8
    if X.shape[1] != C * 8 or dY.shape != (N, D * 8):
        raise ValueError("shape mismatch")
    dW = np.empty((D, C, 8), dtype=np.float64)
    db = np.empty((D,), dtype=np.float64)
    _load().eqlo_d4_backward_weight(N, C, D, _ptr(X), _ptr(dY), _ptr(dW), _ptr(db))
    return dW, db


def conv_forward(T: int, X, Wc, bias=None, pad=(0, 0), return_macs: bool = False):
    """Y[N, Ho, Wo, D*T] in float64 from X[N, H, W, C*T], Wc[KH, KW, D, C, T],
    bias[D] or None, zero padding pad = (ph, pw), stride 1."""
    X, Wc = _f64(X), _f64(Wc)
    KH, KW, D, C, TW = Wc.shape
    if TW != T or X.ndim != 4 or X.shape[3] != C * T:
        raise ValueError("X must be [N, H, W, C*T] and Wc [KH, KW, D, C, T]")
    N, H, Wd = X.shape[:3]
    ph, pw = pad
    Ho, Wo = H + 2 * ph - KH + 1, Wd + 2 * pw - KW + 1
    if Ho <= 0 or Wo <= 0:
        raise ValueError("empty output")
    b = None if bias is None else _f64(bias)
    Y = np.empty((N, Ho, Wo, D * T), dtype=np.float64)
    macs = _load().eqlo_conv_forward(T, N, H, Wd, C, D, KH, KW, ph, pw, _ptr(X), _ptr(Wc),
                                     _ptr(b), _ptr(Y))
    return (Y, macs) if return_macs else Y


_threads_override = None



def conv_backward_input(T: int, dY, Wc, H: int, W: int, pad=(0, 0)):
    """dX[N, H, W, C*T] in float64 from dY[N, Ho, Wo, D*T] and Wc[KH, KW, D, C, T]:
    the gradient of conv_forward with respect to X (input size H x W)."""
    dY, Wc = _f64(dY), _f64(Wc)
    KH, KW, D, C, TW = Wc.shape
    N, Ho, Wo = dY.shape[:3]
    ph, pw = pad
    if TW != T or dY.shape[3] != D * T or Ho != H + 2 * ph - KH + 1 or Wo != W + 2 * pw - KW + 1:
        raise ValueError("shape mismatch")
    dX = np.empty((N, H, W, C * T), dtype=np.float64)
    _load().eqlo_conv_backward_input(T, N, H, W, C, D, KH, KW, ph, pw, _ptr(dY), _ptr(Wc),
                                     _ptr(dX))
    return dX


def conv_backward_weight(T: int, X, dY, KH: int, KW: int, pad=(0, 0)):
    """(dWc[KH, KW, D, C, T], dbias[D]) in float64 from X[N, H, W, C*T] and
    dY[N, Ho, Wo, D*T]: the gradients of conv_forward."""
    X, dY = _f64(X), _f64(dY)
    N, H, W = X.shape[:3]
    C = X.shape[3] // T
    ph, pw = pad
    Ho, Wo = H + 2 * ph - KH + 1, W + 2 * pw - KW + 1
    D = dY.shape[3] // T
    if dY.shape != (N, Ho, Wo, D * T) or X.shape[3] != C * T:
        raise ValueError("shape mismatch")
    dWc = np.empty((KH, KW, D, C, T), dtype=np.float64)
    db = np.empty((D,), dtype=np.float64)
    _load().eqlo_conv_backward_weight(T, N, H, W, C, D, KH, KW, ph, pw, _ptr(X), _ptr(dY),
                                      _ptr(dWc), _ptr(db))
    return dWc, db

def set_threads(n: int | None) -> None:
    """Run the parallel loops on n threads (None: back to the default count).
    Timing only: every loop writes disjoint outputs, so results do not change."""
    global _threads_override
    _load().eqlo_set_threads(int(n) if n else _default_threads())
    _threads_override = int(n) if n else None


def _default_threads() -> int:
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        try:
            return max(1, int(env.split(",")[0]))
        except ValueError:
            pass
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_model() -> str:
    """The host CPU's model name (first 'model name' line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def threads_used() -> int:
    """Threads OpenMP will use for the parallel loops (OMP_NUM_THREADS or cores)."""
    if _threads_override:
        return _threads_override
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        try:
            return max(1, int(env.split(",")[0]))
        except ValueError:
            pass
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
