"""Failure detection without a GPU fault: a bounded wait that runs out.

With EQL_DEBUG_DROP_W_STAGE set when the plan is created, the tensor-core
kernel's first CTA never issues one weight copy.  Every wait in the kernel is
bounded (about 2 s), so the MMA thread gives up, sets the plan's status word,
the CTA drains what it issued and returns; the host then reads EQL_ERR_TIMEOUT
from eqlinear_get_status and the CUDA context stays usable.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _run(w, inp):
    from group_circulant_gemm_b200 import EqLinearPlan
    p = EqLinearPlan(w.T, w.C, w.D, torch.float16, kernel="tcgen05")
    wh = p.prepare_weights(torch.from_numpy(inp["W"]).cuda())
    Y = p.forward(torch.from_numpy(inp["X"]).cuda(), wh, torch.from_numpy(inp["bias"]).cuda())
    return p, Y


def test_dropped_weight_stage_times_out_and_context_survives():
    from group_circulant_gemm_b200 import native as n
    w = Workload("fault", 4, 1024, 64, 256, "f16", True, 41)
    inp = make_inputs(w)
    os.environ["EQL_DEBUG_DROP_W_STAGE"] = "1"
    try:
        p, _ = _run(w, inp)
    finally:
        del os.environ["EQL_DEBUG_DROP_W_STAGE"]
    assert p.status() == n.EQL_ERR_TIMEOUT
    assert p.status() == n.EQL_OK  # the word is cleared once read
    # the same process keeps working: a fresh plan computes the right answer
    p2, Y = _run(w, inp)
    assert p2.status() == n.EQL_OK
    ref = oracle.forward(4, inp["X"], inp["W"], inp["bias"])
    rel = np.max(np.abs(Y.double().cpu().numpy() - ref)) / np.max(np.abs(ref))
    assert rel <= 2e-3
