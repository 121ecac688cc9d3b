"""Data-parallel weight gradient on one GPU (GPU required).

A batch split by rows across ranks has dW = the sum over ranks of each rank's dW.
The ranks are emulated here as row shards processed one after another on the
same GPU (no kernel waits on another), each writing its FP32 sums with
eqlinear_backward_weight_f32; the shards' buffers are added in FP32 (what the
all-reduce does) and eqlinear_cast_from_f32 rounds the total once.  The result
is compared with the float64 oracle on the whole batch.
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.parallel import row_shard
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3}
TDT = {"f32": torch.float32, "f16": torch.float16}


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(w, kernel="auto"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(w.T, w.C, w.D, TDT[w.dtype], kernel=kernel)


CASES = [
    # T, N, C, D, dtype, kernel
    (4, 2000, 144, 272, "f16", "tcgen05"),
    (4, 777, 64, 48, "f16", "simt"),
    (4, 500, 24, 40, "f32", "simt"),
    (3, 301, 7, 9, "f32", "simt"),
    (8, 300, 16, 32, "f16", "simt"),
]


@pytest.mark.parametrize("T,N,C,D,dtype,kernel", CASES)
def test_f32_gradient_rounds_to_the_plan_dtype_result(T, N, C, D, dtype, kernel):
    """backward_weight_f32 then cast_from_f32 gives exactly backward_weight's bits,
    and the FP32 sums themselves meet the oracle."""
    w = Workload("dpcast", T, N, C, D, dtype, True, 900 + N)
    inp = make_inputs(w, need_dy=True)
    p = _plan(w, kernel)
    assert p.backward_weight_kernel_name(N) == kernel
    X, dY = _dev(inp["X"]), _dev(inp["dY"])
    dW, db = p.backward_weight(X, dY)
    buf32 = p.backward_weight_f32(X, dY)
    buf = p.cast_from_f32(buf32)
    dW2, db2 = p.split_grad(buf)
    assert p.status() == 0
    bits = torch.int16 if dtype == "f16" else torch.int32
    assert torch.equal(dW2.contiguous().view(bits).cpu(), dW.view(bits).cpu())
    assert torch.equal(db2.contiguous().view(bits).cpu(), db.view(bits).cpu())
    rdW, rdb = oracle.backward_weight(T, inp["X"], inp["dY"], D)
    w32, b32 = p.split_grad(buf32)
    assert _rel(w32.double().cpu().numpy(), rdW) <= TOL[dtype]
    assert _rel(b32.double().cpu().numpy(), rdb) <= TOL[dtype]


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
def test_emulated_ranks_sum_to_the_full_batch_gradient(world, kernel):
    w = Workload("dpsum", 4, 3001, 80, 144, "f16", True, 4242)
    inp = make_inputs(w, need_dy=True)
    p = _plan(w, kernel)
    total = p.grad_buffer(torch.float32)
    for r in range(world):
        a, b = row_shard(w.N, world, r)
        part = p.backward_weight_f32(_dev(inp["X"][a:b]), _dev(inp["dY"][a:b]))
        total += part  # the all-reduce's FP32 sum
    dW, db = p.split_grad(p.cast_from_f32(total))
    assert p.status() == 0
    rdW, rdb = oracle.backward_weight(4, inp["X"], inp["dY"], w.D)
    assert _rel(dW.double().cpu().numpy(), rdW) <= TOL["f16"]
    assert _rel(db.double().cpu().numpy(), rdb) <= TOL["f16"]


def test_cast_from_f32_rounds_to_nearest_even():
    from group_circulant_gemm_b200 import EqLinearPlan
    p = EqLinearPlan(4, 16, 16, torch.float16)
    rng = np.random.default_rng(5)
    vals = np.concatenate([
        rng.standard_normal(100000) * np.exp2(rng.integers(-30, 17, 100000)),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 5.96e-8, 2.98e-8, 2.99e-8,
         1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, np.inf, -np.inf],
    ]).astype(np.float32)
    src = _dev(vals)
    got = p.cast_from_f32(src).cpu()
    want = torch.from_numpy(vals).to(torch.float16)  # IEEE round-to-nearest-even on the host
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    # a source 4 bytes past a 16-byte boundary takes the one-element path
    got1 = p.cast_from_f32(src[1:]).cpu()
    assert torch.equal(got1.view(torch.int16), want[1:].view(torch.int16))
    nan = p.cast_from_f32(_dev(np.array([np.nan], dtype=np.float32))).cpu()
    assert torch.isnan(nan).all()


def test_cast_from_f32_edges():
    from group_circulant_gemm_b200 import EqLinearPlan, native
    p = EqLinearPlan(4, 16, 16, torch.float16)
    empty = torch.empty(0, dtype=torch.float32, device="cuda")
    assert p.cast_from_f32(empty).numel() == 0
    src = torch.zeros(64, dtype=torch.float32, device="cuda")
    # overlapping source and destination are rejected
    assert native.raw_status("eqlinear_cast_from_f32", p.handle, src.data_ptr(), 64,
                             src.data_ptr() + 8, None) == native.EQL_ERR_INVALID_ARG
    assert native.raw_status("eqlinear_cast_from_f32", p.handle, src.data_ptr(), -1,
                             src.data_ptr(), None) == native.EQL_ERR_INVALID_ARG
    q = EqLinearPlan(4, 16, 16, torch.float32)
    x = torch.arange(10, dtype=torch.float32, device="cuda")
    assert torch.equal(q.cast_from_f32(x), x)
    # an FP32 plan may cast in place (nothing to do)
    assert native.raw_status("eqlinear_cast_from_f32", q.handle, x.data_ptr(), 10,
                             x.data_ptr(), None) == native.EQL_OK
    assert torch.equal(x, torch.arange(10, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("world", [2, 3])
def test_emulated_ranks_from_saved_spectra(world):
    """The training step's form: each rank saves the spectra of its rows in the
    forward and dX calls and writes FP32 sums from them; the FP32 total, cast
    once, meets the oracle on the whole batch."""
    w = Workload("dpspec", 4, 2501, 128, 192, "f16", True, 4343)
    inp = make_inputs(w, need_dy=True)
    p = _plan(w)
    Wh = p.prepare_weights(_dev(inp["W"]))
    total = p.grad_buffer(torch.float32)
    for r in range(world):
        a, b = row_shard(w.N, world, r)
        _, xhat = p.forward_save_spectrum(_dev(inp["X"][a:b]), Wh)
        _, ghat = p.backward_input_save_spectrum(_dev(inp["dY"][a:b]), Wh)
        total += p.backward_weight_from_spectra_f32(xhat, ghat)
    dW, db = p.split_grad(p.cast_from_f32(total))
    assert p.status() == 0
    rdW, rdb = oracle.backward_weight(4, inp["X"], inp["dY"], w.D)
    assert _rel(dW.double().cpu().numpy(), rdW) <= TOL["f16"]
    assert _rel(db.double().cpu().numpy(), rdb) <= TOL["f16"]
