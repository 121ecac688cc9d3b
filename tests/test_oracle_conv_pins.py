"""Pins for the oracle's group-circulant convolution (conv_forward).

The pages name equivariant convolution as the natural next operator for the
per-frequency method ("Limitations and future work") and give no formula; the
reading (the EQ-Linear's group-circulant channel mixing at every tap of a
KH x KW kernel, stride 1, zero padding) is pinned here to things other than the
oracle's own loop:
  * a library routine: torch's conv2d (float64, CPU) with the naive layer's
    replicated dense kernel ("Problem definition": the naive layer replicates the
    shared weights into a dense matrix) at every tap;
  * the 1 x 1 kernel is the EQ-Linear layer (its oracle is pinned separately);
  * cyclic-shift equivariance of the group axis ("Key insight") and translation
    equivariance away from the border;
  * exact multiply-add counts taken inside the image.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def _dense_kernel(Wc):
    """[D*T, C*T, KH, KW] with entry ((d,s),(c,t),i,j) = Wc[i,j,d,c,(t-s) mod T], built
    by rolling each parameter vector (np.roll(v, s)[t] = v[(t-s) mod T])."""
    KH, KW, D, C, T = Wc.shape
    K = np.zeros((D * T, C * T, KH, KW))
    for i in range(KH):
        for j in range(KW):
            for d in range(D):
                for c in range(C):
                    for s in range(T):
                        K[d * T + s, c * T:(c + 1) * T, i, j] = np.roll(Wc[i, j, d, c], s)
    return K


CASES = [
    # T, N, H, W, C, D, KH, KW, ph, pw
    (4, 2, 5, 6, 3, 2, 3, 3, 1, 1),
    (4, 1, 7, 4, 2, 3, 5, 5, 2, 2),
    (3, 2, 4, 5, 2, 2, 3, 1, 1, 0),
    (8, 1, 3, 3, 1, 2, 3, 3, 1, 1),
    (4, 1, 6, 6, 2, 2, 3, 3, 0, 0),
    (2, 3, 4, 4, 3, 1, 2, 2, 1, 0),
]


@pytest.mark.parametrize("T,N,H,W,C,D,KH,KW,ph,pw", CASES)
def test_conv_matches_torch_conv2d_on_dense_kernel(oracle_mod, T, N, H, W, C, D, KH, KW, ph,
                                                   pw):
    X = _rand(1, N, H, W, C * T)
    Wc = _rand(2, KH, KW, D, C, T)
    b = _rand(3, D)
    Y = oracle_mod.conv_forward(T, X, Wc, b, pad=(ph, pw))
    ref = F.conv2d(torch.from_numpy(X).permute(0, 3, 1, 2), torch.from_numpy(_dense_kernel(Wc)),
                   torch.from_numpy(np.repeat(b, T)), padding=(ph, pw))
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert Y.shape == ref.shape
    assert _rel(Y, ref) < 1e-13


@pytest.mark.parametrize("T", [1, 3, 4, 8])
def test_conv_1x1_is_the_eq_linear_layer(oracle_mod, T):
    N, H, W, C, D = 2, 3, 5, 4, 3
    X = _rand(4, N, H, W, C * T)
    Wc = _rand(5, 1, 1, D, C, T)
    b = _rand(6, D)
    Y = oracle_mod.conv_forward(T, X, Wc, b)
    lin = oracle_mod.forward(T, X.reshape(-1, C * T), Wc[0, 0], b).reshape(N, H, W, D * T)
    assert _rel(Y, lin) < 1e-14


@pytest.mark.parametrize("T", [3, 4, 8])
def test_conv_group_equivariance(oracle_mod, T):
    N, H, W, C, D = 1, 5, 4, 3, 2
    X = _rand(7, N, H, W, C * T)
    Wc = _rand(8, 3, 3, D, C, T)
    b = _rand(9, D)
    Y = oracle_mod.conv_forward(T, X, Wc, b, pad=(1, 1)).reshape(N, H, W, D, T)
    for r in range(1, T):
        Xr = np.roll(X.reshape(N, H, W, C, T), r, axis=4).reshape(N, H, W, C * T)
        Yr = oracle_mod.conv_forward(T, Xr, Wc, b, pad=(1, 1)).reshape(N, H, W, D, T)
        assert _rel(Yr, np.roll(Y, r, axis=4)) < 1e-13


def test_conv_translation_equivariance_inside(oracle_mod):
    T, N, H, W, C, D = 4, 1, 9, 10, 2, 2
    X = _rand(10, N, H, W, C * T)
    X[:, :, -2:, :] = 0.0  # content leaves room on the right
    X[:, -2:, :, :] = 0.0  # and at the bottom
    Wc = _rand(11, 3, 3, D, C, T)
    Y = oracle_mod.conv_forward(T, X, Wc, None, pad=(1, 1))
    Xs = np.zeros_like(X)
    Xs[:, 2:, 1:, :] = X[:, :-2, :-1, :]  # shift down 2, right 1
    Ys = oracle_mod.conv_forward(T, Xs, Wc, None, pad=(1, 1))
    assert _rel(Ys[:, 2:, 1:, :], Y[:, :-2, :-1, :]) < 1e-13


def test_conv_mac_counts_exact(oracle_mod):
    T, N, H, W, C, D, KH, KW, ph, pw = 4, 2, 5, 7, 3, 2, 3, 3, 1, 1
    X = _rand(12, N, H, W, C * T)
    Wc = _rand(13, KH, KW, D, C, T)
    _, macs = oracle_mod.conv_forward(T, X, Wc, None, pad=(ph, pw), return_macs=True)
    # taps inside the image per output pixel, counted independently
    inside = 0
    for oy in range(H):
        for ox in range(W):
            inside += sum(1 for i in range(KH) for j in range(KW)
                          if 0 <= oy + i - ph < H and 0 <= ox + j - pw < W)
    assert macs == N * inside * D * T * C * T


def test_conv_pins_catch_a_planted_direction_mistake(oracle_mod):
    """A convolution with (s - t) instead of (t - s), computed here on the CPU, fails
    the torch pin that the oracle passes."""
    T, N, H, W, C, D = 4, 1, 4, 4, 2, 2
    X = _rand(14, N, H, W, C * T)
    Wc = _rand(15, 3, 3, D, C, T)
    ref = F.conv2d(torch.from_numpy(X).permute(0, 3, 1, 2), torch.from_numpy(_dense_kernel(Wc)),
                   padding=1).permute(0, 2, 3, 1).numpy()
    wrong = oracle_mod.conv_forward(T, X, Wc[..., (-np.arange(T)) % T], None, pad=(1, 1))
    assert _rel(wrong, ref) > 1e-3
    assert _rel(oracle_mod.conv_forward(T, X, Wc, None, pad=(1, 1)), ref) < 1e-13


@pytest.mark.parametrize("T,N,H,W,C,D,KH,KW,ph,pw", CASES)
def test_conv_gradients_match_autograd_of_torch_conv2d(oracle_mod, T, N, H, W, C, D, KH, KW,
                                                       ph, pw):
    """dX, dWc and dbias against torch autograd (float64) of conv2d on the
    replicated dense kernel, whose entries are gathered from Wc by rolling the
    parameter vectors (a differentiable function of Wc)."""
    X = _rand(11, N, H, W, C * T)
    Wc = _rand(12, KH, KW, D, C, T)
    b = _rand(13, D)
    Ho, Wo = H + 2 * ph - KH + 1, W + 2 * pw - KW + 1
    dY = _rand(14, N, Ho, Wo, D * T)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(Wc, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    # dense kernel [D*T, C*T, KH, KW]: entry ((d,s),(c,t)) = Wc[.., d, c, (t - s) mod T]
    idx = torch.tensor([[(t - s) % T for t in range(T)] for s in range(T)])  # [s, t]
    K = Wt[:, :, :, :, idx]                               # [KH, KW, D, C, s, t]
    K = K.permute(2, 4, 3, 5, 0, 1).reshape(D * T, C * T, KH, KW)
    Y = F.conv2d(Xt.permute(0, 3, 1, 2), K, bt.repeat_interleave(T), padding=(ph, pw))
    Y.permute(0, 2, 3, 1).backward(torch.tensor(dY))
    dX = oracle_mod.conv_backward_input(T, dY, Wc, H, W, pad=(ph, pw))
    assert _rel(dX, Xt.grad.numpy()) < 1e-12
    dW, db = oracle_mod.conv_backward_weight(T, X, dY, KH, KW, pad=(ph, pw))
    assert _rel(dW, Wt.grad.numpy()) < 1e-12
    assert _rel(db, bt.grad.numpy()) < 1e-12
