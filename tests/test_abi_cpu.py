"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/eqlinear.h declares, and rejects bad arguments before it
touches CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "eqlinear.h")) as f:
        text = f.read()
    return set(re.findall(r"EQL_API[^;(]*?\b(eqlinear_\w+)\s*\(", text, flags=re.S))


@pytest.fixture(scope="module")
def native():
    from group_circulant_gemm_b200 import build
    build.build()
    from group_circulant_gemm_b200 import native as n
    return n


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("eqlinear_plan_create", "eqlinear_prepare_weights", "eqlinear_forward",
                     "eqlinear_backward_input", "eqlinear_backward_weight"):
        assert required in names


def test_library_exports_every_declared_symbol(native):
    lib = ctypes.CDLL(native.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol(native):
    assert set(native.EXPORTED) == _declared()
    for name in _declared():
        assert callable(getattr(native, name))


def test_library_targets_sm100a_only(native):
    """The build line asks for sm_100a code only (checked from the build flags,
    not by inspecting the binary)."""
    from group_circulant_gemm_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "compute_90" not in flags and "sm_90" not in flags


def test_status_strings(native):
    assert native.eqlinear_version() >= 100
    for s in range(7):
        assert native.eqlinear_status_string(s).startswith("EQL_")
    assert "UNKNOWN" in native.eqlinear_status_string(99)


def test_plan_create_rejects_bad_args_without_cuda(native):
    out = ctypes.c_void_p()
    bad = [(0, 4, 4, 0), (4, 0, 4, 0), (4, 4, -1, 0), (4, 4, 4, 7)]
    for T, C, D, dt in bad:
        assert native.raw_status("eqlinear_plan_create", T, C, D, dt, ctypes.byref(out)) == \
            native.EQL_ERR_INVALID_ARG
    assert native.raw_status("eqlinear_plan_create", 9, 4, 4, 0, ctypes.byref(out)) == \
        native.EQL_ERR_UNSUPPORTED
    assert native.raw_status("eqlinear_plan_create", 4, 4, 4, 0, None) == native.EQL_ERR_INVALID_ARG


def test_null_plan_calls_are_rejected(native):
    assert native.raw_status("eqlinear_forward", None, None, 4, None, None, None, None) == \
        native.EQL_ERR_INVALID_ARG
    assert native.raw_status("eqlinear_backward_input", None, None, 4, None, None, None) == \
        native.EQL_ERR_INVALID_ARG
    assert native.raw_status("eqlinear_get_status", None, None) == native.EQL_ERR_INVALID_ARG
    # the training-with-saved-spectra entries
    assert native.raw_status("eqlinear_forward_save_spectrum", None, None, 4, None, None, 0,
                             None, None, None) == native.EQL_ERR_INVALID_ARG
    assert native.raw_status("eqlinear_backward_input_save_spectrum", None, None, 4, None, None,
                             None, None) == native.EQL_ERR_INVALID_ARG
    for name in ("eqlinear_backward_weight_from_spectra",
                 "eqlinear_backward_weight_from_spectra_f32"):
        assert native.raw_status(name, None, None, None, 4, None, None, None, 0, None) == \
            native.EQL_ERR_INVALID_ARG
    assert native.eqlinear_prepared_weight_bytes(None) == 0
    assert native.eqlinear_backward_weight_workspace_bytes(None, 10) == 0
    native.eqlinear_plan_destroy(None)


def test_plan_create_without_gpu_reports_cuda_error(native):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    out = ctypes.c_void_p()
    assert native.raw_status("eqlinear_plan_create", 4, 16, 16, 0, ctypes.byref(out)) == \
        native.EQL_ERR_CUDA


FREQUENCY_DOMAIN_AND_CONV_CALLS = (
    "eqlinear_group_dft", "eqlinear_forward_tiled", "eqlinear_forward_tiled_next",
    "eqlinear_backward_input_tiled", "eqlinear_forward_chain_tiled",
    "eqlinear_backward_weight_tiled", "eqlinear_backward_weight_tiled_f32",
    "eqlinear_conv_prepare_weights", "eqlinear_conv_forward", "eqlinear_conv_backward_input",
    "eqlinear_conv_backward_weight", "eqlinear_forward_chain",
)
SIZE_QUERIES = (
    "eqlinear_tiled_spectrum_bytes", "eqlinear_chain_tiled_workspace_bytes",
    "eqlinear_conv_backward_workspace_bytes", "eqlinear_conv_prepared_weight_bytes",
    "eqlinear_conv_workspace_bytes", "eqlinear_chain_workspace_bytes",
)


def _null_args(fn):
    # null for every pointer (the plans included), 1 for every count and flag
    return [None if t is ctypes.c_void_p else 1 for t in fn.argtypes]


def test_frequency_domain_and_convolution_entries_reject_a_null_plan(native):
    lib = ctypes.CDLL(native.LIB_PATH)
    for name in FREQUENCY_DOMAIN_AND_CONV_CALLS:
        fn = getattr(native._lib, name)
        assert fn(*_null_args(fn)) == native.EQL_ERR_INVALID_ARG, name
        assert hasattr(lib, name)
    for name in SIZE_QUERIES:
        fn = getattr(native._lib, name)
        assert fn(*_null_args(fn)) == 0, name
