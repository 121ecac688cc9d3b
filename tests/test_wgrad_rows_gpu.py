"""Full-size weight gradient with every output checked (GPU required).

The tensor-core weight gradient cuts the (tile, 32-row stage) space into equal
contiguous ranges, one per CTA (stream-K). A range can therefore end inside a
tile's rows, and the finalize adds the pieces in a fixed order.

dW and dbias are sums over rows ("Algorithmic approach": the backward is the
same per-frequency product, transposed, reduced over N). So the full-size launch
on inputs that are zero except on a row set S gives exactly the gradient of the
rows in S. The float64 oracle computes that for every (d, c, t) from S alone.

S holds:
  * one row of every 32-row stage, at an offset that walks through all 32
    positions of a stage;
  * the last 40 rows, the short end of the last row block.
A stage that is lost, counted twice, or read at the wrong row changes outputs.
That holds at a range seam, at a 128-channel tile edge and at the ragged end.

Both the transforming kernel and the variant that multiplies the saved spectra
run at the ViT-H fc1 training shape (N = 8224, 320 -> 1280) that the bench
times. All of dW and dbias are compared (FP16 bar 2e-3 of max|ref|).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL16 = 2e-3
N, C, D = 8224, 320, 1280


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _rows():
    k = np.arange(N // 32)
    per_stage = 32 * k + (7 * k) % 32
    return np.unique(np.concatenate([per_stage, np.arange(N - 40, N)]))


@pytest.fixture(scope="module")
def sparse_case():
    from group_circulant_gemm_b200 import EqLinearPlan
    inp = make_inputs(Workload("wr", 4, N, C, D, "f16", True, 6100), need_dy=True)
    S = _rows()
    X = np.zeros_like(inp["X"])
    dY = np.zeros_like(inp["dY"])
    X[S], dY[S] = inp["X"][S], inp["dY"][S]
    ref_dW, ref_db = oracle.backward_weight(4, inp["X"][S], inp["dY"][S], D)
    p = EqLinearPlan(4, C, D, torch.float16)
    assert p.backward_weight_kernel_name(N) == "tcgen05"
    Wh = p.prepare_weights(_dev(inp["W"]))
    return p, Wh, _dev(X), _dev(dY), ref_dW, ref_db


def test_row_set_covers_every_stage_and_the_end():
    S = _rows()
    assert len(np.unique(S // 32)) == N // 32 + (1 if N % 32 else 0)
    assert len(np.unique(S % 32)) == 32
    assert S.max() == N - 1


def test_transforming_weight_gradient_every_output(sparse_case):
    p, _, X, dY, ref_dW, ref_db = sparse_case
    dW, db = p.backward_weight(X, dY)
    assert p.status() == 0
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16


def test_weight_gradient_from_spectra_every_output(sparse_case):
    p, Wh, X, dY, ref_dW, ref_db = sparse_case
    _, Xhat = p.forward_save_spectrum(X, Wh)
    _, dYhat = p.backward_input_save_spectrum(dY, Wh)
    dW, db = p.backward_weight_from_spectra(Xhat, dYhat)
    assert p.status() == 0
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16
