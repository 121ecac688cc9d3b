"""The allocation-free weight gradient, checked against the allocating one.

eqlinear_backward_weight_noalloc serves callers that cannot give the library a
workspace (their device memory belongs to another allocator or is fixed at
start-up, or they must not call cudaMalloc/cudaFree on their hot path, since
those calls can synchronise the device).  It keeps its partial sums in a
built-in 16 MiB scratch array instead.  This file is named so that pytest
collects it last; it must pass alone in a fresh process and after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

from group_circulant_gemm_b200 import native
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3}
TDT = {"f32": torch.float32, "f16": torch.float16}


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("T,N,C,D,dtype", [(4, 2000, 64, 96, "f16"), (3, 333, 20, 12, "f32"),
                                           (4, 8224, 320, 1280, "f16")])
def test_noalloc_matches_workspace_entry_two_calls(T, N, C, D, dtype):
    plan = native.eqlinear_plan_create(T, C, D, native.EQL_F16 if dtype == "f16" else native.EQL_F32)
    try:
        for call in range(2):  # two calls in a row: the second sees the first's leftovers
            inp = make_inputs(Workload("na", T, N, C, D, dtype, True, 900 + call), need_dy=True)
            X = torch.from_numpy(inp["X"]).cuda()
            dY = torch.from_numpy(inp["dY"]).cuda()
            dW_ref = torch.empty((D, C, T), dtype=TDT[dtype], device="cuda")
            db_ref = torch.empty((D,), dtype=TDT[dtype], device="cuda")
            nb = native.eqlinear_backward_weight_workspace_bytes(plan, N)
            ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
            native.eqlinear_backward_weight(plan, X, dY, N, dW_ref, db_ref, ws, nb)
            dW = torch.full((D, C, T), float("nan"), dtype=TDT[dtype], device="cuda")
            db = torch.full((D,), float("nan"), dtype=TDT[dtype], device="cuda")
            native.eqlinear_backward_weight_noalloc(plan, X, dY, N, dW, db)
            torch.cuda.synchronize()
            assert native.eqlinear_get_status(plan) == native.EQL_OK
            assert _rel(dW, dW_ref) <= TOL[dtype], (call, _rel(dW, dW_ref))
            assert _rel(db, db_ref) <= TOL[dtype]
    finally:
        native.eqlinear_plan_destroy(plan)


def test_noalloc_rejects_plans_beyond_its_scratch():
    # T*C*D + D = 4*1024*1025 + 1025 floats > 4,194,304: rejected before launch
    plan = native.eqlinear_plan_create(4, 1024, 1025, native.EQL_F16)
    try:
        X = torch.zeros(16, dtype=torch.float16, device="cuda")
        s = native.raw_status("eqlinear_backward_weight_noalloc", plan, X.data_ptr(), X.data_ptr(),
                              1, X.data_ptr(), None, None)
        assert s == native.EQL_ERR_WORKSPACE
    finally:
        native.eqlinear_plan_destroy(plan)


@pytest.mark.parametrize("T,N,C,D,dtype", [(4, 700, 32, 48, "f16"), (5, 257, 16, 24, "f32"),
                                           (4, 513, 16, 16, "f32")])
def test_noalloc_against_the_oracle(T, N, C, D, dtype):
    """Directly against the float64 oracle (not only against the other entry)."""
    import oracle
    plan = native.eqlinear_plan_create(T, C, D, native.EQL_F16 if dtype == "f16" else native.EQL_F32)
    try:
        inp = make_inputs(Workload("nao", T, N, C, D, dtype, True, 950 + T), need_dy=True)
        X = torch.from_numpy(inp["X"]).cuda()
        dY = torch.from_numpy(inp["dY"]).cuda()
        dW = torch.empty((D, C, T), dtype=TDT[dtype], device="cuda")
        db = torch.empty((D,), dtype=TDT[dtype], device="cuda")
        native.eqlinear_backward_weight_noalloc(plan, X, dY, N, dW, db)
        torch.cuda.synchronize()
        assert native.eqlinear_get_status(plan) == native.EQL_OK
        ref_w, ref_b = oracle.backward_weight(T, inp["X"], inp["dY"], D)
        assert _rel(dW, torch.from_numpy(ref_w)) <= TOL[dtype]
        assert _rel(db, torch.from_numpy(ref_b)) <= TOL[dtype]
    finally:
        native.eqlinear_plan_destroy(plan)


def test_noalloc_without_bias_and_with_no_rows():
    plan = native.eqlinear_plan_create(4, 32, 48, native.EQL_F16)
    try:
        inp = make_inputs(Workload("nab", 4, 300, 32, 48, "f16", True, 977), need_dy=True)
        X = torch.from_numpy(inp["X"]).cuda()
        dY = torch.from_numpy(inp["dY"]).cuda()
        # dbias = NULL: dW only, the same as the workspace entry without dbias
        nb = native.eqlinear_backward_weight_workspace_bytes(plan, 300)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        dW_ref = torch.empty((48, 32, 4), dtype=torch.float16, device="cuda")
        native.eqlinear_backward_weight(plan, X, dY, 300, dW_ref, None, ws, nb)
        dW = torch.full((48, 32, 4), float("nan"), dtype=torch.float16, device="cuda")
        native.eqlinear_backward_weight_noalloc(plan, X, dY, 300, dW, None)
        torch.cuda.synchronize()
        assert _rel(dW, dW_ref) <= TOL["f16"]
        # N = 0 after a call that left partial sums in the scratch: dW and dbias are zero
        dW0 = torch.full((48, 32, 4), 5.0, dtype=torch.float16, device="cuda")
        db0 = torch.full((48,), 5.0, dtype=torch.float16, device="cuda")
        native.eqlinear_backward_weight_noalloc(plan, None, None, 0, dW0, db0)
        torch.cuda.synchronize()
        assert float(dW0.abs().sum()) == 0.0 and float(db0.abs().sum()) == 0.0
        assert native.eqlinear_get_status(plan) == native.EQL_OK
    finally:
        native.eqlinear_plan_destroy(plan)


def test_noalloc_rejects_a_plan_forced_to_tensor_cores():
    plan = native.eqlinear_plan_create(4, 64, 64, native.EQL_F16)
    try:
        native.eqlinear_plan_set_kernel(plan, native.EQL_KERNEL_TCGEN05)
        X = torch.zeros(16 * 256, dtype=torch.float16, device="cuda")
        s = native.raw_status("eqlinear_backward_weight_noalloc", plan, X.data_ptr(), X.data_ptr(),
                              16, X.data_ptr(), None, None)
        assert s == native.EQL_ERR_UNSUPPORTED
    finally:
        native.eqlinear_plan_destroy(plan)
