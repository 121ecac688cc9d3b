"""ctypes binding of libeqlinear.so, with the C ABI's own names.

Every function here only marshals arguments (tensor -> device pointer, stream ->
handle) and checks the returned status; all computation happens in the CUDA
library.  There is no fallback: if the shared library is missing or was built
for another architecture, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeqlinear.so")

EQL_OK, EQL_ERR_INVALID_ARG, EQL_ERR_UNSUPPORTED, EQL_ERR_ALIGNMENT = 0, 1, 2, 3
EQL_ERR_WORKSPACE, EQL_ERR_CUDA, EQL_ERR_TIMEOUT = 4, 5, 6
EQL_F32, EQL_F16 = 0, 1
EQL_KERNEL_AUTO, EQL_KERNEL_SIMT, EQL_KERNEL_TCGEN05 = 0, 1, 2

EXPORTED = (
    "eqlinear_version", "eqlinear_status_string", "eqlinear_plan_create",
    "eqlinear_plan_destroy", "eqlinear_plan_set_kernel", "eqlinear_forward_kernel_name",
    "eqlinear_backward_weight_kernel_name", "eqlinear_prepared_weight_bytes",
    "eqlinear_prepare_weights", "eqlinear_forward", "eqlinear_forward_act",
    "eqlinear_spectral_bytes", "eqlinear_forward_to_spectral", "eqlinear_forward_from_spectral",
    "eqlinear_backward_input",
    "eqlinear_backward_weight_workspace_bytes", "eqlinear_backward_weight",
    "eqlinear_get_status", "eqlinear_backward_weight_noalloc",
    "eqlinear_backward_weight_f32", "eqlinear_cast_from_f32",
    "eqlinear_chain_workspace_bytes", "eqlinear_forward_chain",
    "eqlinear_conv_prepared_weight_bytes", "eqlinear_conv_prepare_weights",
    "eqlinear_conv_workspace_bytes", "eqlinear_conv_forward",
    "eqlinear_conv_backward_workspace_bytes", "eqlinear_conv_backward_input",
    "eqlinear_conv_backward_weight",
    "eqlinear_plan_create_dihedral4",
    "eqlinear_forward_save_spectrum", "eqlinear_backward_input_save_spectrum",
    "eqlinear_backward_weight_from_spectra", "eqlinear_backward_weight_from_spectra_f32",
    "eqlinear_backward_weight_tiled", "eqlinear_backward_weight_tiled_f32",
    "eqlinear_tiled_spectrum_bytes", "eqlinear_group_dft", "eqlinear_forward_tiled",
    "eqlinear_forward_tiled_next", "eqlinear_backward_input_tiled",
    "eqlinear_chain_tiled_workspace_bytes", "eqlinear_forward_chain_tiled",
)


class EqLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.eqlinear_status_string(status).decode()}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m group_circulant_gemm_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    sig = {
        "eqlinear_version": ([], i32),
        "eqlinear_status_string": ([i32], ctypes.c_char_p),
        "eqlinear_plan_create": ([i32, i32, i32, i32, ctypes.POINTER(vp)], i32),
        "eqlinear_plan_create_dihedral4": ([i32, i32, i32, ctypes.POINTER(vp)], i32),
        "eqlinear_plan_destroy": ([vp], None),
        "eqlinear_plan_set_kernel": ([vp, i32], i32),
        "eqlinear_forward_kernel_name": ([vp, i64], ctypes.c_char_p),
        "eqlinear_backward_weight_kernel_name": ([vp, i64], ctypes.c_char_p),
        "eqlinear_prepared_weight_bytes": ([vp], sz),
        "eqlinear_prepare_weights": ([vp, vp, vp, vp], i32),
        "eqlinear_forward": ([vp, vp, i64, vp, vp, vp, vp], i32),
        "eqlinear_forward_act": ([vp, vp, i64, vp, vp, i32, vp, vp], i32),
        "eqlinear_spectral_bytes": ([vp, i64], ctypes.c_size_t),
        "eqlinear_forward_to_spectral": ([vp, vp, i64, vp, vp, i32, vp, vp], i32),
        "eqlinear_forward_from_spectral": ([vp, vp, i64, vp, vp, i32, vp, vp], i32),
        "eqlinear_tiled_spectrum_bytes": ([vp, i64, i32], sz),
        "eqlinear_group_dft": ([vp, vp, i64, i32, vp, vp], i32),
        "eqlinear_forward_tiled": ([vp, vp, i64, vp, vp, i32, vp, vp], i32),
        "eqlinear_forward_tiled_next": ([vp, vp, i64, vp, vp, i32, vp, vp], i32),
        "eqlinear_backward_input_tiled": ([vp, vp, i64, vp, vp, vp], i32),
        "eqlinear_chain_tiled_workspace_bytes": ([vp, vp, i64], sz),
        "eqlinear_forward_chain_tiled": ([vp, vp, vp, i64, vp, vp, i32, vp, vp, vp, vp, vp, sz,
                                          vp], i32),
        "eqlinear_backward_input": ([vp, vp, i64, vp, vp, vp], i32),
        "eqlinear_backward_weight_workspace_bytes": ([vp, i64], sz),
        "eqlinear_backward_weight": ([vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "eqlinear_get_status": ([vp, vp], i32),
        "eqlinear_backward_weight_noalloc": ([vp, vp, vp, i64, vp, vp, vp], i32),
        "eqlinear_backward_weight_f32": ([vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "eqlinear_cast_from_f32": ([vp, vp, i64, vp, vp], i32),
        "eqlinear_forward_save_spectrum": ([vp, vp, i64, vp, vp, i32, vp, vp, vp], i32),
        "eqlinear_backward_input_save_spectrum": ([vp, vp, i64, vp, vp, vp, vp], i32),
        "eqlinear_backward_weight_from_spectra": ([vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "eqlinear_backward_weight_tiled": ([vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "eqlinear_backward_weight_tiled_f32": ([vp, vp, vp, i64, vp, vp, vp, sz, vp], i32),
        "eqlinear_backward_weight_from_spectra_f32": ([vp, vp, vp, i64, vp, vp, vp, sz, vp],
                                                      i32),
        "eqlinear_chain_workspace_bytes": ([vp, vp, i64], sz),
        "eqlinear_conv_prepared_weight_bytes": ([vp, i32, i32], sz),
        "eqlinear_conv_prepare_weights": ([vp, i32, i32, vp, vp, vp], i32),
        "eqlinear_conv_workspace_bytes": ([vp, i64, i32, i32], sz),
        "eqlinear_conv_forward": ([vp, vp, i64, i32, i32, i32, i32, i32, i32, vp, vp, i32, vp,
                                   vp, sz, vp], i32),
        "eqlinear_conv_backward_workspace_bytes": ([vp, i64, i32, i32, i32, i32, i32, i32], sz),
        "eqlinear_conv_backward_input": ([vp, vp, i64, i32, i32, i32, i32, i32, i32, vp, vp,
                                          vp, sz, vp], i32),
        "eqlinear_conv_backward_weight": ([vp, vp, i64, i32, i32, vp, i32, i32, i32, i32, vp,
                                           vp, vp, sz, vp], i32),
        "eqlinear_forward_chain": ([vp, vp, vp, i64, vp, vp, i32, vp, vp, i32, vp, vp, vp, sz,
                                    vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def _check(status: int, where: str) -> None:
    if status != EQL_OK:
        raise EqLinearError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --- the C ABI, name for name --------------------------------------------------

def eqlinear_version() -> int:
    return _lib.eqlinear_version()


def eqlinear_status_string(status: int) -> str:
    return _lib.eqlinear_status_string(status).decode()


def eqlinear_plan_create(T: int, C: int, D: int, dtype: int) -> int:
    out = ctypes.c_void_p()
    _check(_lib.eqlinear_plan_create(T, C, D, dtype, ctypes.byref(out)), "eqlinear_plan_create")
    return out.value


def eqlinear_plan_create_dihedral4(C: int, D: int, dtype: int) -> int:
    out = ctypes.c_void_p()
    _check(_lib.eqlinear_plan_create_dihedral4(C, D, dtype, ctypes.byref(out)),
           "eqlinear_plan_create_dihedral4")
    return out.value


def eqlinear_plan_destroy(plan: int) -> None:
    _lib.eqlinear_plan_destroy(plan)


def eqlinear_plan_set_kernel(plan: int, which: int) -> None:
    _check(_lib.eqlinear_plan_set_kernel(plan, which), "eqlinear_plan_set_kernel")


def eqlinear_forward_kernel_name(plan: int, N: int) -> str:
    return _lib.eqlinear_forward_kernel_name(plan, N).decode()


def eqlinear_backward_weight_kernel_name(plan: int, N: int) -> str:
    return _lib.eqlinear_backward_weight_kernel_name(plan, N).decode()


def eqlinear_prepared_weight_bytes(plan: int) -> int:
    return _lib.eqlinear_prepared_weight_bytes(plan)


def eqlinear_prepare_weights(plan: int, W, W_hat, stream=None) -> None:
    _check(_lib.eqlinear_prepare_weights(plan, _ptr(W), _ptr(W_hat), _stream(stream)),
           "eqlinear_prepare_weights")


def eqlinear_forward(plan: int, X, N: int, W_hat, bias, Y, stream=None) -> None:
    _check(_lib.eqlinear_forward(plan, _ptr(X), N, _ptr(W_hat), _ptr(bias), _ptr(Y),
                                 _stream(stream)), "eqlinear_forward")


ACT = {"none": 0, "gelu": 1}


def eqlinear_forward_act(plan: int, X, N: int, W_hat, bias, act: int, Y, stream=None) -> None:
    _check(_lib.eqlinear_forward_act(plan, _ptr(X), N, _ptr(W_hat), _ptr(bias), act, _ptr(Y),
                                     _stream(stream)), "eqlinear_forward_act")


def eqlinear_spectral_bytes(plan: int, N: int) -> int:
    return _lib.eqlinear_spectral_bytes(plan, N)


def eqlinear_forward_to_spectral(plan: int, X, N: int, W_hat, bias, act: int, Xhat,
                                 stream=None) -> None:
    _check(_lib.eqlinear_forward_to_spectral(plan, _ptr(X), N, _ptr(W_hat), _ptr(bias), act,
                                             _ptr(Xhat), _stream(stream)),
           "eqlinear_forward_to_spectral")


def eqlinear_forward_from_spectral(plan: int, Xhat, N: int, W_hat, bias, act: int, Y,
                                   stream=None) -> None:
    _check(_lib.eqlinear_forward_from_spectral(plan, _ptr(Xhat), N, _ptr(W_hat), _ptr(bias), act,
                                               _ptr(Y), _stream(stream)),
           "eqlinear_forward_from_spectral")


def eqlinear_tiled_spectrum_bytes(plan: int, N: int, channels: int) -> int:
    return _lib.eqlinear_tiled_spectrum_bytes(plan, N, channels)


def eqlinear_group_dft(plan: int, X, N: int, channels: int, Xt, stream=None) -> None:
    _check(_lib.eqlinear_group_dft(plan, _ptr(X), N, channels, _ptr(Xt), _stream(stream)),
           "eqlinear_group_dft")


def eqlinear_forward_tiled(plan: int, Xt, N: int, W_hat, bias, act: int, Y,
                           stream=None) -> None:
    _check(_lib.eqlinear_forward_tiled(plan, _ptr(Xt), N, _ptr(W_hat), _ptr(bias), act, _ptr(Y),
                                       _stream(stream)),
           "eqlinear_forward_tiled")


def eqlinear_forward_tiled_next(plan: int, Xt, N: int, W_hat, bias, act: int, Yt,
                                stream=None) -> None:
    _check(_lib.eqlinear_forward_tiled_next(plan, _ptr(Xt), N, _ptr(W_hat), _ptr(bias), act,
                                            _ptr(Yt), _stream(stream)),
           "eqlinear_forward_tiled_next")


def eqlinear_chain_tiled_workspace_bytes(first: int, second: int, N: int) -> int:
    return _lib.eqlinear_chain_tiled_workspace_bytes(first, second, N)


def eqlinear_forward_chain_tiled(first: int, second: int, Xt, N: int, W1_hat, bias1, act1: int,
                                 W2_hat, bias2, Ht, Y, workspace, workspace_bytes: int,
                                 stream=None) -> None:
    _check(_lib.eqlinear_forward_chain_tiled(first, second, _ptr(Xt), N, _ptr(W1_hat),
                                             _ptr(bias1), act1, _ptr(W2_hat), _ptr(bias2),
                                             _ptr(Ht), _ptr(Y), _ptr(workspace), workspace_bytes,
                                             _stream(stream)),
           "eqlinear_forward_chain_tiled")


def eqlinear_backward_input_tiled(plan: int, dYt, N: int, W_hat, dX, stream=None) -> None:
    _check(_lib.eqlinear_backward_input_tiled(plan, _ptr(dYt), N, _ptr(W_hat), _ptr(dX),
                                              _stream(stream)),
           "eqlinear_backward_input_tiled")


def eqlinear_backward_input(plan: int, dY, N: int, W_hat, dX, stream=None) -> None:
    _check(_lib.eqlinear_backward_input(plan, _ptr(dY), N, _ptr(W_hat), _ptr(dX),
                                        _stream(stream)), "eqlinear_backward_input")


def eqlinear_backward_weight_workspace_bytes(plan: int, N: int) -> int:
    return _lib.eqlinear_backward_weight_workspace_bytes(plan, N)


def eqlinear_backward_weight(plan: int, X, dY, N: int, dW, dbias, workspace,
                             workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_backward_weight(plan, _ptr(X), _ptr(dY), N, _ptr(dW), _ptr(dbias),
                                         _ptr(workspace), workspace_bytes, _stream(stream)),
           "eqlinear_backward_weight")


def eqlinear_backward_weight_f32(plan: int, X, dY, N: int, dW, dbias, workspace,
                                 workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_backward_weight_f32(plan, _ptr(X), _ptr(dY), N, _ptr(dW), _ptr(dbias),
                                             _ptr(workspace), workspace_bytes, _stream(stream)),
           "eqlinear_backward_weight_f32")


def eqlinear_forward_save_spectrum(plan: int, X, N: int, W_hat, bias, act: int, Y, Xhat,
                                   stream=None) -> None:
    _check(_lib.eqlinear_forward_save_spectrum(plan, _ptr(X), N, _ptr(W_hat), _ptr(bias), act,
                                               _ptr(Y), _ptr(Xhat), _stream(stream)),
           "eqlinear_forward_save_spectrum")


def eqlinear_backward_input_save_spectrum(plan: int, dY, N: int, W_hat, dX, dYhat,
                                          stream=None) -> None:
    _check(_lib.eqlinear_backward_input_save_spectrum(plan, _ptr(dY), N, _ptr(W_hat), _ptr(dX),
                                                      _ptr(dYhat), _stream(stream)),
           "eqlinear_backward_input_save_spectrum")


def eqlinear_backward_weight_from_spectra(plan: int, Xhat, dYhat, N: int, dW, dbias, workspace,
                                          workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_backward_weight_from_spectra(plan, _ptr(Xhat), _ptr(dYhat), N, _ptr(dW),
                                                      _ptr(dbias), _ptr(workspace),
                                                      workspace_bytes, _stream(stream)),
           "eqlinear_backward_weight_from_spectra")


def eqlinear_backward_weight_tiled(plan: int, Xt, dYt, N: int, dW, dbias, workspace,
                                   workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_backward_weight_tiled(plan, _ptr(Xt), _ptr(dYt), N, _ptr(dW),
                                               _ptr(dbias), _ptr(workspace), workspace_bytes,
                                               _stream(stream)),
           "eqlinear_backward_weight_tiled")


def eqlinear_backward_weight_tiled_f32(plan: int, Xt, dYt, N: int, dW, dbias, workspace,
                                       workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_backward_weight_tiled_f32(plan, _ptr(Xt), _ptr(dYt), N, _ptr(dW),
                                                   _ptr(dbias), _ptr(workspace), workspace_bytes,
                                                   _stream(stream)),
           "eqlinear_backward_weight_tiled_f32")


def eqlinear_backward_weight_from_spectra_f32(plan: int, Xhat, dYhat, N: int, dW, dbias,
                                              workspace, workspace_bytes: int,
                                              stream=None) -> None:
    _check(_lib.eqlinear_backward_weight_from_spectra_f32(plan, _ptr(Xhat), _ptr(dYhat), N,
                                                          _ptr(dW), _ptr(dbias), _ptr(workspace),
                                                          workspace_bytes, _stream(stream)),
           "eqlinear_backward_weight_from_spectra_f32")


def eqlinear_cast_from_f32(plan: int, src, count: int, dst, stream=None) -> None:
    _check(_lib.eqlinear_cast_from_f32(plan, _ptr(src), count, _ptr(dst), _stream(stream)),
           "eqlinear_cast_from_f32")


def eqlinear_chain_workspace_bytes(first: int, second: int, N: int) -> int:
    return _lib.eqlinear_chain_workspace_bytes(first, second, N)


def eqlinear_forward_chain(first: int, second: int, X, N: int, W1_hat, bias1, act1: int, W2_hat,
                           bias2, spectral_intermediate: int, H, Y, workspace,
                           workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_forward_chain(first, second, _ptr(X), N, _ptr(W1_hat), _ptr(bias1),
                                       act1, _ptr(W2_hat), _ptr(bias2), spectral_intermediate,
                                       _ptr(H), _ptr(Y), _ptr(workspace), workspace_bytes,
                                       _stream(stream)),
           "eqlinear_forward_chain")


def eqlinear_conv_prepared_weight_bytes(plan: int, KH: int, KW: int) -> int:
    return _lib.eqlinear_conv_prepared_weight_bytes(plan, KH, KW)


def eqlinear_conv_prepare_weights(plan: int, KH: int, KW: int, Wc, Wc_hat, stream=None) -> None:
    _check(_lib.eqlinear_conv_prepare_weights(plan, KH, KW, _ptr(Wc), _ptr(Wc_hat),
                                              _stream(stream)),
           "eqlinear_conv_prepare_weights")


def eqlinear_conv_workspace_bytes(plan: int, N: int, H: int, W: int) -> int:
    return _lib.eqlinear_conv_workspace_bytes(plan, N, H, W)


def eqlinear_conv_forward(plan: int, X, N: int, H: int, W: int, KH: int, KW: int, pad_h: int,
                          pad_w: int, Wc_hat, bias, act: int, Y, workspace, workspace_bytes: int,
                          stream=None) -> None:
    _check(_lib.eqlinear_conv_forward(plan, _ptr(X), N, H, W, KH, KW, pad_h, pad_w,
                                      _ptr(Wc_hat), _ptr(bias), act, _ptr(Y), _ptr(workspace),
                                      workspace_bytes, _stream(stream)),
           "eqlinear_conv_forward")


def eqlinear_conv_backward_workspace_bytes(plan: int, N: int, H: int, W: int, KH: int, KW: int,
                                           pad_h: int, pad_w: int) -> int:
    return _lib.eqlinear_conv_backward_workspace_bytes(plan, N, H, W, KH, KW, pad_h, pad_w)


def eqlinear_conv_backward_input(plan: int, dY, N: int, H: int, W: int, KH: int, KW: int,
                                 pad_h: int, pad_w: int, Wc_hat, dX, workspace,
                                 workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_conv_backward_input(plan, _ptr(dY), N, H, W, KH, KW, pad_h, pad_w,
                                             _ptr(Wc_hat), _ptr(dX), _ptr(workspace),
                                             workspace_bytes, _stream(stream)),
           "eqlinear_conv_backward_input")


def eqlinear_conv_backward_weight(plan: int, X, N: int, H: int, W: int, dY, KH: int, KW: int,
                                  pad_h: int, pad_w: int, dWc, dbias, workspace,
                                  workspace_bytes: int, stream=None) -> None:
    _check(_lib.eqlinear_conv_backward_weight(plan, _ptr(X), N, H, W, _ptr(dY), KH, KW, pad_h,
                                              pad_w, _ptr(dWc), _ptr(dbias), _ptr(workspace),
                                              workspace_bytes, _stream(stream)),
           "eqlinear_conv_backward_weight")


def eqlinear_backward_weight_noalloc(plan: int, X, dY, N: int, dW, dbias, stream=None) -> None:
    """dW/dbias with the library's own built-in scratch (no workspace argument)."""
    _check(_lib.eqlinear_backward_weight_noalloc(plan, _ptr(X), _ptr(dY), N, _ptr(dW),
                                                 _ptr(dbias), _stream(stream)),
           "eqlinear_backward_weight_noalloc")


def eqlinear_get_status(plan: int, stream=None) -> int:
    return _lib.eqlinear_get_status(plan, _stream(stream))


def raw_status(fn_name: str, *args) -> int:
    """Call an ABI function and return its raw status (for error-path tests)."""
    return getattr(_lib, fn_name)(*args)
