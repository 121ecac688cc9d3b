"""Pins for the float64 oracle: each test fixes it to something other than itself.

Passages (Flash EQ-Linear summary, gist.science/ko/paper/2607.21271):
  * "Problem definition": the naive layer replicates the shared weights into a
    dense matrix and calls a dense linear kernel -> brute-force dense pin.
  * "Key insight": group-circulant weight, circular structure over the group
    axis -> hand-worked values, equivariance.
  * "Algorithmic approach" items 1-3 and "Contributions" item 2: DFT
    convolution theorem, exactness -> numpy FFT pin, spectral route equality.
  * "Algorithmic approach" item 3 and "Specialisation for p4" bullet 3: MAC
    counts NDC -> about 2NDC/T and 16/6 -> exact integer MAC counts.
  * "Specialisation for p4" bullets 1-2: dyadic transform coefficients.
"""
import json
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
TS = [1, 2, 3, 4, 5, 8]


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def _dense_replicated(W):
    """The naive layer's dense (D*T) x (C*T) matrix, built by explicit loops:
    row (d,s) holds the parameter set W[d,c,:] cyclically shifted by s."""
    D, C, T = W.shape
    M = np.zeros((D * T, C * T))
    for d in range(D):
        for s in range(T):
            for c in range(C):
                shifted = np.roll(W[d, c, :], s)  # shifted[t] = W[d,c,(t-s) mod T]
                M[d * T + s, c * T:(c + 1) * T] = shifted
    return M


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --- hand-worked values -------------------------------------------------------

def test_handworked_golden(oracle_mod):
    with open(os.path.join(HERE, "golden", "p4_handworked.json")) as f:
        cases = json.load(f)["cases"]
    for cs in cases:
        T = cs["T"]
        X = np.array(cs["X"], dtype=np.float64)
        W = np.array(cs["W"], dtype=np.float64)
        b = np.array(cs["bias"], dtype=np.float64)
        Y = oracle_mod.forward(T, X, W, b)
        np.testing.assert_array_equal(Y, np.array(cs["Y"]), err_msg=cs["name"])
        Ys = oracle_mod.forward_spectral(T, X, W, b)
        np.testing.assert_allclose(Ys, np.array(cs["Y"]), atol=1e-12, err_msg=cs["name"])
        if "dY" in cs:
            dY = np.array(cs["dY"], dtype=np.float64)
            np.testing.assert_array_equal(oracle_mod.backward_input(T, dY, W), np.array(cs["dX"]))
            dW, db = oracle_mod.backward_weight(T, X, dY, W.shape[0])
            np.testing.assert_array_equal(dW, np.array(cs["dW"]))
            np.testing.assert_array_equal(db, np.array(cs["dbias"]))


# --- brute force against the replicated dense matrix -------------------------

@pytest.mark.parametrize("T", TS)
def test_forward_matches_replicated_dense(oracle_mod, T):
    N, C, D = 5, 3, 4
    X, W, b = _rand(1, N, C * T), _rand(2, D, C, T), _rand(3, D)
    M = _dense_replicated(W)
    ref = X @ M.T + np.repeat(b, T)[None, :]
    assert _rel(oracle_mod.forward(T, X, W, b), ref) < 1e-13
    assert _rel(oracle_mod.forward(T, X, W, None), X @ M.T) < 1e-13


@pytest.mark.parametrize("T", TS)
def test_backward_matches_autograd_of_dense(oracle_mod, T):
    """Gradients of the naive dense layer via torch autograd (float64, CPU)."""
    N, C, D = 6, 3, 2
    X, W, b, dY = _rand(4, N, C * T), _rand(5, D, C, T), _rand(6, D), _rand(7, N, D * T)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    # replicate: index tensor idx[d*T+s, c*T+t] -> flat index of W[d,c,(t-s) mod T]
    idx = np.zeros((D * T, C * T), dtype=np.int64)
    for d in range(D):
        for s in range(T):
            for c in range(C):
                for t in range(T):
                    idx[d * T + s, c * T + t] = (d * C + c) * T + (t - s) % T
    M = Wt.reshape(-1)[torch.tensor(idx)]
    Y = Xt @ M.T + bt.repeat_interleave(T)[None, :]
    Y.backward(torch.tensor(dY))
    assert _rel(oracle_mod.backward_input(T, dY, W), Xt.grad.numpy()) < 1e-13
    dW, db = oracle_mod.backward_weight(T, X, dY, D)
    assert _rel(dW, Wt.grad.numpy()) < 1e-13
    assert _rel(db, bt.grad.numpy()) < 1e-13
    pairs_d, pairs_c = np.array([0, 1, 1]), np.array([2, 0, 1])
    sub = oracle_mod.backward_weight_pairs(T, X, dY, D, pairs_d, pairs_c)
    assert _rel(sub, Wt.grad.numpy()[pairs_d, pairs_c, :]) < 1e-13


# --- adjoint identities (exact bilinear algebra) ------------------------------

@pytest.mark.parametrize("T", [3, 4, 8])
def test_adjoint_identities(oracle_mod, T):
    """<forward(X) - b, G> = <X, backward_input(G)> = <W, backward_weight(X,G)>."""
    N, C, D = 7, 5, 3
    X, W, G = _rand(8, N, C * T), _rand(9, D, C, T), _rand(10, N, D * T)
    Y = oracle_mod.forward(T, X, W, None)
    lhs = np.sum(Y * G)
    assert abs(lhs - np.sum(X * oracle_mod.backward_input(T, G, W))) < 1e-11 * (1 + abs(lhs))
    dW, db = oracle_mod.backward_weight(T, X, G, D)
    assert abs(lhs - np.sum(W * dW)) < 1e-11 * (1 + abs(lhs))
    np.testing.assert_allclose(db, G.reshape(N, D, T).sum(axis=(0, 2)), rtol=1e-13)


# --- convolution theorem with numpy's FFT -------------------------------------

@pytest.mark.parametrize("T", TS)
def test_convolution_theorem_numpy_fft(oracle_mod, T):
    N, C, D = 4, 3, 5
    X, W, b = _rand(11, N, C * T), _rand(12, D, C, T), _rand(13, D)
    Xh = np.fft.fft(X.reshape(N, C, T), axis=-1)          # [N,C,T]
    Wh = np.fft.fft(W, axis=-1)                             # [D,C,T]
    Yh = np.einsum("dck,nck->ndk", np.conj(Wh), Xh)
    ref = np.real(np.fft.ifft(Yh, axis=-1)).reshape(N, D * T) + np.repeat(b, T)[None, :]
    assert _rel(oracle_mod.forward(T, X, W, b), ref) < 1e-13
    assert _rel(oracle_mod.forward_spectral(T, X, W, b), ref) < 1e-13


def test_dft_round_trip_numpy():
    x = _rand(14, 100, 8)
    assert np.max(np.abs(np.real(np.fft.ifft(np.fft.fft(x, axis=-1), axis=-1)) - x)) < 1e-14


# --- equivariance -------------------------------------------------------------

@pytest.mark.parametrize("T", TS)
def test_equivariance_every_shift(oracle_mod, T):
    """Rolling every input group vector by r rolls every output group vector by r
    ("Contributions" item 2: rotation equivariance is preserved)."""
    N, C, D = 3, 4, 2
    X, W, b = _rand(15, N, C * T), _rand(16, D, C, T), _rand(17, D)
    Y = oracle_mod.forward(T, X, W, b).reshape(N, D, T)
    dX = oracle_mod.backward_input(T, Y.reshape(N, D * T), W).reshape(N, C, T)
    for r in range(T):
        Xr = np.roll(X.reshape(N, C, T), r, axis=-1).reshape(N, C * T)
        Yr = oracle_mod.forward(T, Xr, W, b).reshape(N, D, T)
        np.testing.assert_allclose(Yr, np.roll(Y, r, axis=-1), rtol=0, atol=1e-12)
        Gr = np.roll(Y, r, axis=-1).reshape(N, D * T)
        dXr = oracle_mod.backward_input(T, Gr, W).reshape(N, C, T)
        np.testing.assert_allclose(dXr, np.roll(dX, r, axis=-1), rtol=0, atol=1e-12)


# --- special cases with closed forms ------------------------------------------

def test_T1_is_plain_linear(oracle_mod):
    N, C, D = 9, 6, 4
    X, W, b = _rand(18, N, C), _rand(19, D, C, 1), _rand(20, D)
    assert _rel(oracle_mod.forward(1, X, W, b), X @ W[:, :, 0].T + b) < 1e-14


@pytest.mark.parametrize("T", [2, 4, 8])
def test_delta_weight_is_per_element_linear(oracle_mod, T):
    """W[:,:,u] = delta_{u0} A: each group element s sees the plain map A."""
    N, C, D = 5, 3, 4
    A, X = _rand(21, D, C), _rand(22, N, C * T)
    W = np.zeros((D, C, T))
    W[:, :, 0] = A
    Y = oracle_mod.forward(T, X, W, None).reshape(N, D, T)
    Xg = X.reshape(N, C, T)
    for s in range(T):
        np.testing.assert_allclose(Y[:, :, s], Xg[:, :, s] @ A.T, atol=1e-13)


@pytest.mark.parametrize("T", [3, 4, 8])
def test_group_constant_input(oracle_mod, T):
    """x[c,t] = v[c] for all t gives y[d,s] = sum_c (sum_u W[d,c,u]) v[c] + b[d]."""
    N, C, D = 4, 5, 3
    v, W, b = _rand(23, N, C), _rand(24, D, C, T), _rand(25, D)
    X = np.repeat(v, T, axis=1)
    Y = oracle_mod.forward(T, X, W, b).reshape(N, D, T)
    ref = v @ W.sum(axis=2).T + b
    for s in range(T):
        np.testing.assert_allclose(Y[:, :, s], ref, atol=1e-12)


# --- MAC counts ---------------------------------------------------------------

@pytest.mark.parametrize("T", TS)
def test_mac_counts(oracle_mod, T):
    N, C, D = 3, 5, 7
    X, W = _rand(26, N, C * T), _rand(27, D, C, T)
    _, direct = oracle_mod.forward(T, X, W, None, return_macs=True)
    _, spectral = oracle_mod.forward_spectral(T, X, W, None, return_macs=True)
    assert direct == N * C * D * T * T
    gemms = (2 * T - 2) if T % 2 == 0 else (2 * T - 1)
    if T == 1:
        gemms = 1
    assert spectral == N * C * D * gemms
    if T == 4:  # "Specialisation for p4": 16 vs 6 real GEMM-equivalents, ~2.67x
        assert direct * 6 == spectral * 16
        assert abs(direct / spectral - 2.6667) < 1e-3
    if T >= 2:  # "Algorithmic approach" item 3 with widths DT, CT: NDC -> ~2NDC/T
        naive = N * (D * T) * (C * T)
        approx = 2 * N * (D * T) * (C * T) / T
        assert abs(spectral - approx) <= 2 * N * C * D


# --- p4 transforms are dyadic -------------------------------------------------

def test_p4_transform_dyadic_and_inverse(oracle_mod):
    F, G = oracle_mod.p4_transform_matrices()
    allowed = {0.0, 1.0, -1.0, 0.5, -0.5, 0.25, -0.25}
    assert set(np.unique(F)).issubset({0.0, 1.0, -1.0})
    assert set(np.unique(G)).issubset(allowed)
    np.testing.assert_array_equal(G @ F, np.eye(4))
    # rows of F against numpy's DFT of the unit vectors
    E = np.fft.fft(np.eye(4), axis=0)  # column t = DFT of e_t
    np.testing.assert_allclose(F[0], np.real(E[0]), atol=1e-15)
    np.testing.assert_allclose(F[1], np.real(E[2]), atol=1e-15)
    np.testing.assert_allclose(F[2], np.real(E[1]), atol=1e-15)
    np.testing.assert_allclose(F[3], np.imag(E[1]), atol=1e-15)
    # each coefficient is exact in fp16
    assert np.array_equal(F.astype(np.float16).astype(np.float64), F)
    assert np.array_equal(G.astype(np.float16).astype(np.float64), G)


# --- planted mistakes are caught ---------------------------------------------

def test_pins_catch_planted_index_mistake(oracle_mod):
    """A wrong-direction shift (s-t instead of t-s), computed here on the CPU,
    is equivariant too but fails the hand-worked and FFT pins."""
    T = 4
    X = np.array([[1.0, 2, 3, 4]])
    W = np.array([[[1.0, 2, 0, 0]]])
    wrong = np.array([[sum(W[0, 0, (s - t) % T] * X[0, t] for t in range(T)) for s in range(T)]])
    assert not np.allclose(wrong, oracle_mod.forward(T, X, W, None))
    np.testing.assert_array_equal(oracle_mod.forward(T, X, W, None), [[5, 8, 11, 6]])


# --- the EQ-MLP block's activation (exact GELU) ------------------------------------

def test_gelu_matches_normal_cdf_closed_form(oracle_mod):
    """GELU(y) = y * Phi(y): pinned to scipy's normal CDF, an independent routine."""
    from scipy.special import ndtr
    y = np.concatenate([np.linspace(-8.0, 8.0, 161), [0.0, 1.0, -1.0, 1e-8, -30.0, 30.0]])
    ref = y * ndtr(y)
    got = oracle_mod.gelu(y)
    assert np.max(np.abs(got - ref)) <= 1e-14
    assert got[-6] == 0.0 and abs(got[-5] - 0.8413447460685429) < 1e-15
    assert abs(got[-2]) < 1e-190  # GELU(-30) = -30 * Phi(-30), about -1.5e-196
    assert got[-1] == 30.0


def test_forward_gelu_is_gelu_of_forward_and_equivariant(oracle_mod):
    rng = np.random.default_rng(21)
    T, N, C, D = 4, 9, 5, 6
    X = rng.standard_normal((N, C * T))
    W = rng.standard_normal((D, C, T)) / np.sqrt(C * T)
    b = 0.1 * rng.standard_normal(D)
    from scipy.special import ndtr
    plain = oracle_mod.forward(T, X, W, b)
    Y = oracle_mod.forward(T, X, W, b, act="gelu")
    assert np.max(np.abs(Y - plain * ndtr(plain))) <= 1e-14
    for r in range(T):
        Xr = np.roll(X.reshape(N, C, T), r, axis=2).reshape(N, C * T)
        Yr = oracle_mod.forward(T, Xr, W, b, act="gelu")
        assert np.max(np.abs(Yr - np.roll(Y.reshape(N, D, T), r, axis=2).reshape(N, D * T))) <= 1e-12
