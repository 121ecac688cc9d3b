"""Two chained layers in one launch (eqlinear_forward_chain), GPU required.

The chained call runs every tile with the same arithmetic as the one-layer
kernels, so H and Y must equal the two separate calls bit for bit; Y is also
checked against the float64 oracle of the two layers composed (on the FP16
intermediate the GPU produced, and end to end).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plans(C0, C1, C2):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(4, C0, C1, torch.float16), EqLinearPlan(4, C1, C2, torch.float16)


def _setup(N, C0, C1, C2, seed):
    w1 = Workload("ch1", 4, N, C0, C1, "f16", True, seed)
    w2 = Workload("ch2", 4, N, C1, C2, "f16", True, seed + 1)
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1, p2 = _plans(C0, C1, C2)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    return in1, in2, p1, p2, Wh1, Wh2


CASES = [
    # N, C0, C1, C2, act, spectral
    (333, 192, 768, 192, "none", False),
    (333, 192, 768, 192, "gelu", True),
    (1, 32, 64, 48, "none", False),
    (129, 16, 16, 32, "gelu", False),
    (300, 48, 144, 80, "none", True),
    (1000, 64, 384, 64, "gelu", False),
    (4097, 80, 208, 16, "none", True),
]


@pytest.mark.parametrize("N,C0,C1,C2,act,spectral", CASES)
def test_chain_equals_two_calls_bitwise(N, C0, C1, C2, act, spectral):
    from group_circulant_gemm_b200 import forward_chain
    in1, in2, p1, p2, Wh1, Wh2 = _setup(N, C0, C1, C2, 2100 + N + C1)
    X, b1, b2 = _dev(in1["X"]), _dev(in1["bias"]), _dev(in2["bias"])
    H, Y = forward_chain(p1, p2, X, Wh1, b1, Wh2, b2, act=act, spectral=spectral)
    if spectral:
        H_ref = p1.forward_to_spectral(X, Wh1, b1, act=act)
        Y_ref = p2.forward_from_spectral(H_ref, Wh2, b2)
    else:
        H_ref = p1.forward(X, Wh1, b1, act=act)
        Y_ref = p2.forward(H_ref, Wh2, b2)
    assert p1.status() == 0 and p2.status() == 0
    assert torch.equal(H.view(torch.int16), H_ref.view(torch.int16))
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    if not spectral:
        # against the oracle: layer 2 on the FP16 H the GPU produced, and end to end
        Hh = H.double().cpu().numpy()
        ref_y = oracle.forward(4, Hh, in2["W"], in2["bias"])
        assert _rel(Y.double().cpu().numpy(), ref_y) <= TOL16
        ref_h = oracle.forward(4, in1["X"], in1["W"], in1["bias"], act=act)
        assert _rel(Hh, ref_h) <= TOL16


def test_chain_full_size_vitb_bitwise():
    """ViT-B MLP shape (N = 12608, 192 -> 768 -> 192), the bench's launch."""
    from group_circulant_gemm_b200 import forward_chain
    N, C0, C1, C2 = 12608, 192, 768, 192
    in1, in2, p1, p2, Wh1, Wh2 = _setup(N, C0, C1, C2, 2500)
    X, b1, b2 = _dev(in1["X"]), _dev(in1["bias"]), _dev(in2["bias"])
    for spectral in (False, True):
        H, Y = forward_chain(p1, p2, X, Wh1, b1, Wh2, b2, spectral=spectral)
        if spectral:
            H_ref = p1.forward_to_spectral(X, Wh1, b1)
            Y_ref = p2.forward_from_spectral(H_ref, Wh2, b2)
        else:
            H_ref = p1.forward(X, Wh1, b1)
            Y_ref = p2.forward(H_ref, Wh2, b2)
        assert p1.status() == 0
        assert torch.equal(H.view(torch.int16), H_ref.view(torch.int16))
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    # sampled rows against the oracle, end to end through both layers
    rows = np.concatenate([np.arange(0, 3), np.arange(6000, 6003), np.arange(N - 3, N)])
    ref = oracle.forward(4, oracle.forward(4, in1["X"][rows], in1["W"], in1["bias"]).astype(
        np.float16).astype(np.float64), in2["W"], in2["bias"])
    H, Y = forward_chain(p1, p2, X, Wh1, b1, Wh2, b2)
    assert _rel(Y.double().cpu().numpy()[rows], ref) <= TOL16


def test_chain_repeated_calls_reuse_the_workspace():
    from group_circulant_gemm_b200 import forward_chain
    in1, in2, p1, p2, Wh1, Wh2 = _setup(777, 64, 128, 64, 2600)
    X, b1, b2 = _dev(in1["X"]), _dev(in1["bias"]), _dev(in2["bias"])
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    outs = [forward_chain(p1, p2, X, Wh1, b1, Wh2, b2, workspace=ws)[1] for _ in range(5)]
    assert p1.status() == 0
    for y in outs[1:]:
        assert torch.equal(y, outs[0])
    # the counters are back to zero after every call, also for another N
    assert int(ws.view(torch.int32).abs().sum().item()) == 0
    X2 = X[:200].contiguous()
    _, y2 = forward_chain(p1, p2, X2, Wh1, b1, Wh2, b2, workspace=ws)
    _, y2_ref = forward_chain(p1, p2, X2, Wh1, b1, Wh2, b2)
    assert torch.equal(y2, y2_ref)
    assert int(ws.view(torch.int32).abs().sum().item()) == 0


def test_chain_error_paths():
    from group_circulant_gemm_b200 import EqLinearPlan, native
    p1, p2 = _plans(32, 64, 32)
    bad = EqLinearPlan(4, 48, 32, torch.float16)      # C does not chain
    p8 = EqLinearPlan(8, 64, 32, torch.float16)       # T = 8: no chained kernel
    f32 = EqLinearPlan(4, 64, 32, torch.float32)
    N = 10
    X = torch.zeros(N, 32 * 4, dtype=torch.float16, device="cuda")
    Wh1 = p1.prepare_weights(torch.zeros(64, 32, 4, dtype=torch.float16, device="cuda"))
    Wh2 = p2.prepare_weights(torch.zeros(32, 64, 4, dtype=torch.float16, device="cuda"))
    H = torch.empty(N, 64 * 4, dtype=torch.float16, device="cuda")
    Y = torch.empty(N, 32 * 4, dtype=torch.float16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")

    def call(a, b, workspace=ws, nbytes=256, spectral=0, act=0, x=X):
        return native.raw_status("eqlinear_forward_chain", a.handle, b.handle, x.data_ptr(), N,
                                 Wh1.data_ptr(), None, act, Wh2.data_ptr(), None, spectral,
                                 H.data_ptr(), Y.data_ptr(),
                                 workspace.data_ptr() if workspace is not None else None,
                                 nbytes, None)
    assert call(p1, p2) == native.EQL_OK
    assert call(p1, bad) == native.EQL_ERR_INVALID_ARG
    assert call(p1, p8) == native.EQL_ERR_UNSUPPORTED
    assert call(p1, f32) == native.EQL_ERR_UNSUPPORTED
    assert call(p1, p2, nbytes=0) == native.EQL_ERR_WORKSPACE
    assert call(p1, p2, workspace=None) == native.EQL_ERR_WORKSPACE
    assert call(p1, p2, spectral=2) == native.EQL_ERR_INVALID_ARG
    assert call(p1, p2, act=7) == native.EQL_ERR_INVALID_ARG
    Xo = torch.zeros(N * 32 * 4 + 1, dtype=torch.float16, device="cuda")[1:]
    assert call(p1, p2, x=Xo) == native.EQL_ERR_ALIGNMENT
    assert native.eqlinear_chain_workspace_bytes(p1.handle, bad.handle, N) == 0
    assert native.eqlinear_chain_workspace_bytes(p1.handle, p2.handle, N) >= 8
    p2.set_kernel("simt")
    assert call(p1, p2) == native.EQL_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert p1.status() == 0
