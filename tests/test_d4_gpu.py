"""The layer over the dihedral group D4 on the GPU against the float64 oracle
(oracle.d4_forward), GPU required.  Element g = a + 4b for r^a m^b; error metric
max|gpu - oracle| / max|oracle| <= 2e-3 (FP16)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _inputs(N, C, D, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((N, C * 8)).astype(np.float16)
    W = (rng.standard_normal((D, C, 8)) / np.sqrt(C * 8)).astype(np.float16)
    b = (rng.standard_normal(D) * 0.1).astype(np.float16)
    return X, W, b


def _plan(C, D, dtype=torch.float16):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(8, C, D, dtype, group="dihedral4")


def _run(p, X, W, b, act="none"):
    Wh = p.prepare_weights(torch.from_numpy(W).cuda())
    Y = p.forward(torch.from_numpy(X).cuda(), Wh, torch.from_numpy(b).cuda(), act=act)
    assert p.status() == 0
    return Y.double().cpu().numpy()


CASES = [
    # N, C, D, act
    (300, 16, 16, "none"),
    (129, 48, 80, "gelu"),
    (1000, 128, 128, "none"),
    (1, 16, 32, "none"),
    (4097, 64, 208, "none"),
    (700, 96, 384, "gelu"),
]


@pytest.mark.parametrize("N,C,D,act", CASES)
def test_d4_forward_matches_oracle(N, C, D, act):
    X, W, b = _inputs(N, C, D, 4000 + N + C + D)
    p = _plan(C, D)
    assert p.forward_kernel_name(N) == "tcgen05"
    ref = oracle.d4_forward(X, W, b, act=act)
    assert _rel(_run(p, X, W, b, act), ref) <= TOL16


def _perm(k):
    """h -> k^-1 h on indices g = a + 4b (r^a m^b; m r m = r^-1)."""
    def mul(g, h):
        a, bb, c, e = g & 3, g >> 2, h & 3, h >> 2
        return ((a + (-c if bb else c)) & 3) + 4 * (bb ^ e)

    def inv(g):
        a, bb = g & 3, g >> 2
        return (a if bb else (-a) & 3) + 4 * bb
    ki = inv(k)
    return [mul(ki, h) for h in range(8)]


@pytest.mark.parametrize("k", [1, 4, 6])
def test_d4_equivariance_on_gpu(k):
    """Acting on the input's group axis by k acts on the output's the same way
    (k = 1: a quarter turn, 4: the mirror, 6: a mirror composed with a half turn)."""
    N, C, D = 640, 32, 48
    X, W, b = _inputs(N, C, D, 4100)
    p = _plan(C, D)
    perm = _perm(k)
    Y = _run(p, X, W, b).reshape(N, D, 8)
    Xk = np.ascontiguousarray(X.reshape(N, C, 8)[:, :, perm].reshape(N, C * 8))
    Yk = _run(p, Xk, W, b).reshape(N, D, 8)
    assert _rel(Yk, Y[:, :, perm]) <= 1e-3


def test_d4_rotation_subgroup_matches_p4_oracle():
    N, C, D = 333, 32, 64
    X, W, b = _inputs(N, C, D, 4200)
    X.reshape(N, C, 8)[:, :, 4:] = 0
    W[:, :, 4:] = 0
    p = _plan(C, D)
    Y = _run(p, X, W, b).reshape(N, D, 8)
    p4 = oracle.forward(4, X.reshape(N, C, 8)[:, :, :4].reshape(N, C * 4), W[:, :, :4], b)
    assert _rel(Y[:, :, :4].reshape(N, D * 4), p4) <= TOL16


def test_d4_unsupported_paths():
    from group_circulant_gemm_b200 import native
    p = _plan(16, 16)
    X = torch.zeros(4, 16 * 8, dtype=torch.float16, device="cuda")
    Wh = p.prepare_weights(torch.zeros(16, 16, 8, dtype=torch.float16, device="cuda"))
    dX = torch.empty_like(X)
    # dX runs through the tiled entries (eqlinear_backward_input_tiled); dW on CUDA cores
    assert native.raw_status("eqlinear_backward_input", p.handle, X.data_ptr(), 4, Wh.data_ptr(),
                             dX.data_ptr(), None) == native.EQL_ERR_UNSUPPORTED
    assert p.backward_weight_kernel_name(4) == "simt"
    f32 = _plan(16, 16, torch.float32)
    assert native.eqlinear_prepared_weight_bytes(f32.handle) == 0
    p.set_kernel("simt")
    Y = torch.empty(4, 16 * 8, dtype=torch.float16, device="cuda")
    assert native.raw_status("eqlinear_forward", p.handle, X.data_ptr(), 4, Wh.data_ptr(), None,
                             Y.data_ptr(), None) == native.EQL_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        from group_circulant_gemm_b200 import EqLinearPlan
        EqLinearPlan(4, 16, 16, torch.float16, group="dihedral4")
