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


def test_chained_launch_row_wait_times_out_and_recovers():
    """The chained two-layer launch waits (bounded) for the layer-1 tiles of a row
    before a layer-2 tile reads them.  Starting the task counter past the first
    layer-1 tile (a workspace the host planted) leaves row 0's layer-2 tile waiting
    for a tile nobody computes: the wait gives up after ~2 s, the status word
    reports EQL_ERR_TIMEOUT, the kernel's last CTA still clears the counters, and
    the next call with the same workspace is correct."""
    from group_circulant_gemm_b200 import EqLinearPlan, forward_chain
    from group_circulant_gemm_b200 import native as n
    N, C0, C1, C2 = 20 * 128, 64, 128, 64
    w1 = Workload("chf1", 4, N, C0, C1, "f16", True, 51)
    w2 = Workload("chf2", 4, N, C1, C2, "f16", True, 52)
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1 = EqLinearPlan(4, C0, C1, torch.float16)
    p2 = EqLinearPlan(4, C1, C2, torch.float16)
    wh1 = p1.prepare_weights(torch.from_numpy(in1["W"]).cuda())
    wh2 = p2.prepare_weights(torch.from_numpy(in2["W"]).cuda())
    X = torch.from_numpy(in1["X"]).cuda()
    b1, b2 = torch.from_numpy(in1["bias"]).cuda(), torch.from_numpy(in2["bias"]).cuda()
    ws = torch.zeros(n.eqlinear_chain_workspace_bytes(p1.handle, p2.handle, N),
                     dtype=torch.uint8, device="cuda")
    ws.view(torch.int32)[0] = 1  # skip task 0: the layer-1 tile of row 0
    forward_chain(p1, p2, X, wh1, b1, wh2, b2, workspace=ws)
    assert p1.status() == n.EQL_ERR_TIMEOUT
    assert int(ws.view(torch.int32).abs().sum().item()) == 0
    H, Y = forward_chain(p1, p2, X, wh1, b1, wh2, b2, workspace=ws)
    assert p1.status() == n.EQL_OK
    Y_ref = p2.forward(p1.forward(X, wh1, b1), wh2, b2)
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
