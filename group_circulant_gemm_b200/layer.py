"""Torch-tensor convenience wrapper over the C ABI (allocation + marshalling only).

PyTorch provides device memory and streams; every arithmetic step runs in
libeqlinear.so through the functions of :mod:`group_circulant_gemm_b200.native`.
"""
from __future__ import annotations

import torch

from . import native as _n

_DT = {torch.float32: _n.EQL_F32, torch.float16: _n.EQL_F16}
_KERNEL = {"auto": _n.EQL_KERNEL_AUTO, "simt": _n.EQL_KERNEL_SIMT,
           "tcgen05": _n.EQL_KERNEL_TCGEN05}


class EqLinearPlan:
    """A plan for the EQ-Linear layer of group order T, C -> D channels.

    ``group="dihedral4"`` makes the layer over the dihedral group D4 instead of
    the cyclic group (T must be 8; forward only, FP16)."""

    def __init__(self, T: int, C: int, D: int, dtype: torch.dtype, kernel: str = "auto",
                 group: str = "cyclic"):
        if dtype not in _DT:
            raise ValueError(f"unsupported dtype {dtype}")
        self.T, self.C, self.D, self.dtype, self.group = T, C, D, dtype, group
        if group == "dihedral4":
            if T != 8:
                raise ValueError("D4 has eight elements: T must be 8")
            self.handle = _n.eqlinear_plan_create_dihedral4(C, D, _DT[dtype])
        elif group == "cyclic":
            self.handle = _n.eqlinear_plan_create(T, C, D, _DT[dtype])
        else:
            raise ValueError(f"unknown group {group}")
        self.set_kernel(kernel)

    def set_kernel(self, kernel: str) -> None:
        _n.eqlinear_plan_set_kernel(self.handle, _KERNEL[kernel])
        self.kernel = kernel

    def close(self) -> None:
        if getattr(self, "handle", None):
            _n.eqlinear_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, t: torch.Tensor, shape, name: str) -> None:
        if not t.is_cuda or t.dtype != self.dtype or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor of {self.dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")

    def forward_kernel_name(self, N: int) -> str:
        return _n.eqlinear_forward_kernel_name(self.handle, N)

    def backward_weight_kernel_name(self, N: int) -> str:
        return _n.eqlinear_backward_weight_kernel_name(self.handle, N)

    def prepare_weights(self, W: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        self._check(W, (self.D, self.C, self.T), "W")
        nbytes = _n.eqlinear_prepared_weight_bytes(self.handle)
        if out is None:
            out = torch.empty(nbytes // W.element_size(), dtype=self.dtype, device=W.device)
        _n.eqlinear_prepare_weights(self.handle, W, out)
        return out

    def forward(self, X, W_hat, bias=None, out=None, act: str = "none") -> torch.Tensor:
        """Y = act(EQ-Linear(X) + bias); act is "none" or "gelu" (fused in the epilogue)."""
        N = X.shape[0]
        self._check(X, (N, self.C * self.T), "X")
        if bias is not None:
            self._check(bias, (self.D,), "bias")
        if act not in _n.ACT:
            raise ValueError(f"unknown activation {act!r}")
        if out is None:
            out = torch.empty((N, self.D * self.T), dtype=self.dtype, device=X.device)
        if act == "none":
            _n.eqlinear_forward(self.handle, X, N, W_hat, bias, out)
        else:
            _n.eqlinear_forward_act(self.handle, X, N, W_hat, bias, _n.ACT[act], out)
        return out

    def forward_to_spectral(self, X, W_hat, bias=None, act: str = "none",
                            out=None) -> torch.Tensor:
        """act(EQ-Linear(X) + bias) as the next p4 layer's input planes [4, N, D]."""
        N = X.shape[0]
        self._check(X, (N, self.C * self.T), "X")
        if bias is not None:
            self._check(bias, (self.D,), "bias")
        if out is None:
            out = torch.empty((4, N, self.D), dtype=self.dtype, device=X.device)
        self._check(out, (4, N, self.D), "out")
        _n.eqlinear_forward_to_spectral(self.handle, X, N, W_hat, bias, _n.ACT[act], out)
        return out

    def forward_from_spectral(self, Xhat, W_hat, bias=None, act: str = "none",
                              out=None) -> torch.Tensor:
        """EQ-Linear forward of an input given as spectral planes [4, N, C]."""
        N = Xhat.shape[1]
        self._check(Xhat, (4, N, self.C), "Xhat")
        if bias is not None:
            self._check(bias, (self.D,), "bias")
        if out is None:
            out = torch.empty((N, self.D * self.T), dtype=self.dtype, device=Xhat.device)
        _n.eqlinear_forward_from_spectral(self.handle, Xhat, N, W_hat, bias, _n.ACT[act], out)
        return out

    # --- the frequency-domain form on tiled planes (see eqlinear_group_dft)

    def tiled_shape(self, N: int, channels: int):
        """Shape of tiled planes of N rows, Np = N rounded up to a multiple of 128.
        FP16: (4 planes, channels/16 blocks, Np rows, 16 halves per row in the
        swizzled order of the header); 8 planes at T = 8 (cyclic or D4).  FP32: (8
        planes = the TF32 hi parts of the four, then the lo parts, channels/8
        blocks, Np rows, 8 floats per row)."""
        Np = (N + 127) // 128 * 128
        if self.dtype == torch.float32:
            return (8, channels // 8, Np, 8)
        if self.T == 8:
            return (8, channels // 16, Np, 16)
        return (4, channels // 16, Np, 16)

    def group_dft(self, X, out=None) -> torch.Tensor:
        """Tiled planes of X [N, c*4] (c = C for an input, D for an upstream gradient)."""
        N = X.shape[0]
        c = X.shape[1] // self.T
        if c not in (self.C, self.D) or X.shape[1] != c * self.T:
            raise ValueError(f"X must be [N, C*T] or [N, D*T], got {tuple(X.shape)}")
        self._check(X, (N, c * self.T), "X")
        if out is None:
            out = torch.empty(self.tiled_shape(N, c), dtype=self.dtype, device=X.device)
        self._check(out, self.tiled_shape(N, c), "out")
        _n.eqlinear_group_dft(self.handle, X, N, c, out)
        return out

    def forward_tiled(self, Xt, N: int, W_hat, bias=None, act: str = "none",
                      out=None) -> torch.Tensor:
        """Y [N, D*T] from the tiled planes of X."""
        self._check(Xt, self.tiled_shape(N, self.C), "Xt")
        if bias is not None:
            self._check(bias, (self.D,), "bias")
        if out is None:
            out = torch.empty((N, self.D * self.T), dtype=self.dtype, device=Xt.device)
        self._check(out, (N, self.D * self.T), "out")
        _n.eqlinear_forward_tiled(self.handle, Xt, N, W_hat, bias, _n.ACT[act], out)
        return out

    def forward_tiled_next(self, Xt, N: int, W_hat, bias=None, act: str = "none",
                           out=None) -> torch.Tensor:
        """The tiled planes of act(Y) (the next p4 layer's input) from those of X."""
        self._check(Xt, self.tiled_shape(N, self.C), "Xt")
        if bias is not None:
            self._check(bias, (self.D,), "bias")
        if out is None:
            out = torch.empty(self.tiled_shape(N, self.D), dtype=self.dtype, device=Xt.device)
        self._check(out, self.tiled_shape(N, self.D), "out")
        _n.eqlinear_forward_tiled_next(self.handle, Xt, N, W_hat, bias, _n.ACT[act], out)
        return out

    def backward_input_tiled(self, dYt, N: int, W_hat, out=None) -> torch.Tensor:
        """dX [N, C*T] from the tiled planes of dY."""
        self._check(dYt, self.tiled_shape(N, self.D), "dYt")
        if out is None:
            out = torch.empty((N, self.C * self.T), dtype=self.dtype, device=dYt.device)
        self._check(out, (N, self.C * self.T), "out")
        _n.eqlinear_backward_input_tiled(self.handle, dYt, N, W_hat, out)
        return out

    def backward_weight_tiled(self, Xt, dYt, N: int, dW=None, dbias=None, workspace=None,
                              want_bias=True):
        """(dW [D, C, T], dbias [D]) from the tiled planes of X and dY (group_dft of each)."""
        self._check(Xt, self.tiled_shape(N, self.C), "Xt")
        self._check(dYt, self.tiled_shape(N, self.D), "dYt")
        if dW is None:
            dW = torch.empty((self.D, self.C, self.T), dtype=self.dtype, device=Xt.device)
        if dbias is None and want_bias:
            dbias = torch.empty((self.D,), dtype=self.dtype, device=Xt.device)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(N), 16), dtype=torch.uint8,
                                    device=Xt.device)
        _n.eqlinear_backward_weight_tiled(self.handle, Xt, dYt, N, dW, dbias, workspace,
                                          workspace.numel() * workspace.element_size())
        return dW, dbias

    def backward_weight_tiled_f32(self, Xt, dYt, N: int, buf=None, workspace=None):
        """backward_weight_f32 from the tiled planes of X and dY."""
        self._check(Xt, self.tiled_shape(N, self.C), "Xt")
        self._check(dYt, self.tiled_shape(N, self.D), "dYt")
        if buf is None:
            buf = self.grad_buffer(torch.float32, Xt.device)
        if buf.dtype != torch.float32 or buf.numel() != self.grad_offset() + self.D:
            raise ValueError("buf must be a flat FP32 gradient buffer of this plan")
        dW, db = self.split_grad(buf)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(N), 16), dtype=torch.uint8,
                                    device=Xt.device)
        _n.eqlinear_backward_weight_tiled_f32(self.handle, Xt, dYt, N, dW, db, workspace,
                                              workspace.numel() * workspace.element_size())
        return buf

    def backward_input(self, dY, W_hat, out=None) -> torch.Tensor:
        N = dY.shape[0]
        self._check(dY, (N, self.D * self.T), "dY")
        if out is None:
            out = torch.empty((N, self.C * self.T), dtype=self.dtype, device=dY.device)
        _n.eqlinear_backward_input(self.handle, dY, N, W_hat, out)
        return out

    def workspace_bytes(self, N: int) -> int:
        return _n.eqlinear_backward_weight_workspace_bytes(self.handle, N)

    def backward_weight(self, X, dY, dW=None, dbias=None, workspace=None, want_bias=True):
        N = X.shape[0]
        self._check(X, (N, self.C * self.T), "X")
        self._check(dY, (N, self.D * self.T), "dY")
        if dW is None:
            dW = torch.empty((self.D, self.C, self.T), dtype=self.dtype, device=X.device)
        if dbias is None and want_bias:
            dbias = torch.empty((self.D,), dtype=self.dtype, device=X.device)
        nb = self.workspace_bytes(N)
        if workspace is None:
            workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=X.device)
        _n.eqlinear_backward_weight(self.handle, X, dY, N, dW, dbias, workspace,
                                    workspace.numel() * workspace.element_size())
        return dW, dbias

    # --- training with saved spectra (the weight gradient runs no transform)

    def forward_save_spectrum(self, X, W_hat, bias=None, act: str = "none", out=None,
                              Xhat=None):
        """(forward(X), Xhat): Xhat [4, N, C] is X's group spectrum, kept for
        backward_weight_from_spectra."""
        N = X.shape[0]
        self._check(X, (N, self.C * self.T), "X")
        if bias is not None:
            self._check(bias, (self.D,), "bias")
        if out is None:
            out = torch.empty((N, self.D * self.T), dtype=self.dtype, device=X.device)
        if Xhat is None:
            Xhat = torch.empty((4, N, self.C), dtype=self.dtype, device=X.device)
        self._check(out, (N, self.D * self.T), "out")
        self._check(Xhat, (4, N, self.C), "Xhat")
        _n.eqlinear_forward_save_spectrum(self.handle, X, N, W_hat, bias, _n.ACT[act], out, Xhat)
        return out, Xhat

    def backward_input_save_spectrum(self, dY, W_hat, out=None, dYhat=None):
        """(backward_input(dY), dYhat): dYhat [4, N, D] is dY's group spectrum."""
        N = dY.shape[0]
        self._check(dY, (N, self.D * self.T), "dY")
        if out is None:
            out = torch.empty((N, self.C * self.T), dtype=self.dtype, device=dY.device)
        if dYhat is None:
            dYhat = torch.empty((4, N, self.D), dtype=self.dtype, device=dY.device)
        self._check(out, (N, self.C * self.T), "out")
        self._check(dYhat, (4, N, self.D), "dYhat")
        _n.eqlinear_backward_input_save_spectrum(self.handle, dY, N, W_hat, out, dYhat)
        return out, dYhat

    def backward_weight_from_spectra(self, Xhat, dYhat, dW=None, dbias=None, workspace=None,
                                     want_bias=True):
        N = Xhat.shape[1]
        self._check(Xhat, (4, N, self.C), "Xhat")
        self._check(dYhat, (4, N, self.D), "dYhat")
        if dW is None:
            dW = torch.empty((self.D, self.C, self.T), dtype=self.dtype, device=Xhat.device)
        if dbias is None and want_bias:
            dbias = torch.empty((self.D,), dtype=self.dtype, device=Xhat.device)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(N), 16), dtype=torch.uint8,
                                    device=Xhat.device)
        _n.eqlinear_backward_weight_from_spectra(self.handle, Xhat, dYhat, N, dW, dbias,
                                                 workspace,
                                                 workspace.numel() * workspace.element_size())
        return dW, dbias

    def backward_weight_from_spectra_f32(self, Xhat, dYhat, buf=None, workspace=None):
        """backward_weight_f32 from the saved spectra."""
        N = Xhat.shape[1]
        self._check(Xhat, (4, N, self.C), "Xhat")
        self._check(dYhat, (4, N, self.D), "dYhat")
        if buf is None:
            buf = self.grad_buffer(torch.float32, Xhat.device)
        if buf.dtype != torch.float32 or buf.numel() != self.grad_offset() + self.D:
            raise ValueError("buf must be a flat FP32 gradient buffer of this plan")
        dW, db = self.split_grad(buf)
        if workspace is None:
            workspace = torch.empty(max(self.workspace_bytes(N), 16), dtype=torch.uint8,
                                    device=Xhat.device)
        _n.eqlinear_backward_weight_from_spectra_f32(self.handle, Xhat, dYhat, N, dW, db,
                                                     workspace,
                                                     workspace.numel() * workspace.element_size())
        return buf

    # --- group-circulant convolution (KH x KW taps, stride 1, zero padding)

    def conv_prepare_weights(self, Wc: torch.Tensor, out: torch.Tensor | None = None):
        """Wc [KH, KW, D, C, T] -> prepared convolution weights."""
        KH, KW = int(Wc.shape[0]), int(Wc.shape[1])
        self._check(Wc, (KH, KW, self.D, self.C, self.T), "Wc")
        nbytes = _n.eqlinear_conv_prepared_weight_bytes(self.handle, KH, KW)
        if nbytes == 0:
            raise ValueError("this plan has no convolution kernel (T = 4, FP16, C and D "
                             "multiples of 16)")
        if out is None:
            out = torch.empty(nbytes // Wc.element_size(), dtype=self.dtype, device=Wc.device)
        _n.eqlinear_conv_prepare_weights(self.handle, KH, KW, Wc, out)
        return out

    def conv_forward(self, X, Wc_hat, KH: int, KW: int, bias=None, pad=(0, 0), act="none",
                     out=None, workspace=None) -> torch.Tensor:
        """X [N, H, W, C*T] -> Y [N, Ho, Wo, D*T]."""
        N, H, W = (int(v) for v in X.shape[:3])
        self._check(X, (N, H, W, self.C * self.T), "X")
        ph, pw = pad
        Ho, Wo = H + 2 * ph - KH + 1, W + 2 * pw - KW + 1
        if out is None:
            out = torch.empty((N, Ho, Wo, self.D * self.T), dtype=self.dtype, device=X.device)
        nb = _n.eqlinear_conv_workspace_bytes(self.handle, N, H, W)
        if workspace is None:
            workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=X.device)
        _n.eqlinear_conv_forward(self.handle, X, N, H, W, KH, KW, ph, pw, Wc_hat, bias,
                                 _n.ACT[act], out, workspace,
                                 workspace.numel() * workspace.element_size())
        return out

    def _conv_bwd_workspace(self, N, H, W, KH, KW, ph, pw, workspace, device):
        nb = _n.eqlinear_conv_backward_workspace_bytes(self.handle, N, H, W, KH, KW, ph, pw)
        if nb == 0:
            raise ValueError("no convolution backward for this plan and shape")
        if workspace is None:
            workspace = torch.empty(nb, dtype=torch.uint8, device=device)
        return workspace

    def conv_backward_input(self, dY, Wc_hat, KH: int, KW: int, H: int, W: int, pad=(0, 0),
                            out=None, workspace=None) -> torch.Tensor:
        """dY [N, Ho, Wo, D*T] -> dX [N, H, W, C*T] (the flipped kernel of adjoint taps)."""
        N = int(dY.shape[0])
        ph, pw = pad
        Ho, Wo = H + 2 * ph - KH + 1, W + 2 * pw - KW + 1
        self._check(dY, (N, Ho, Wo, self.D * self.T), "dY")
        if out is None:
            out = torch.empty((N, H, W, self.C * self.T), dtype=self.dtype, device=dY.device)
        workspace = self._conv_bwd_workspace(N, H, W, KH, KW, ph, pw, workspace, dY.device)
        _n.eqlinear_conv_backward_input(self.handle, dY, N, H, W, KH, KW, ph, pw, Wc_hat, out,
                                        workspace, workspace.numel() * workspace.element_size())
        return out

    def conv_backward_weight(self, X, dY, KH: int, KW: int, pad=(0, 0), workspace=None,
                             dW=None, dbias=None):
        """X [N, H, W, C*T], dY [N, Ho, Wo, D*T] -> (dWc [KH, KW, D, C, T], dbias [D])."""
        N, H, W = (int(v) for v in X.shape[:3])
        self._check(X, (N, H, W, self.C * self.T), "X")
        ph, pw = pad
        Ho, Wo = H + 2 * ph - KH + 1, W + 2 * pw - KW + 1
        self._check(dY, (N, Ho, Wo, self.D * self.T), "dY")
        if dW is None:
            dW = torch.empty((KH, KW, self.D, self.C, self.T), dtype=self.dtype, device=X.device)
        self._check(dW, (KH, KW, self.D, self.C, self.T), "dW")
        db = dbias
        if db is None:
            db = torch.empty(self.D, dtype=self.dtype, device=X.device)
        self._check(db, (self.D,), "dbias")
        workspace = self._conv_bwd_workspace(N, H, W, KH, KW, ph, pw, workspace, X.device)
        _n.eqlinear_conv_backward_weight(self.handle, X, N, H, W, dY, KH, KW, ph, pw, dW, db,
                                         workspace, workspace.numel() * workspace.element_size())
        return dW, db

    # --- data-parallel weight gradient: FP32 per-rank sums, one reduction, one cast

    def grad_offset(self) -> int:
        """Element offset of dbias in a flat gradient buffer (dW first, padded to 8)."""
        return (self.D * self.C * self.T + 7) // 8 * 8

    def grad_buffer(self, dtype: torch.dtype = torch.float32, device="cuda") -> torch.Tensor:
        """A zeroed flat buffer holding dW [D, C, T] then dbias [D], so one
        collective reduces both."""
        return torch.zeros(self.grad_offset() + self.D, dtype=dtype, device=device)

    def split_grad(self, buf: torch.Tensor):
        """(dW, dbias) views of a flat gradient buffer."""
        off = self.grad_offset()
        return buf[:self.D * self.C * self.T].view(self.D, self.C, self.T), buf[off:off + self.D]

    def backward_weight_f32(self, X, dY, buf=None, workspace=None) -> torch.Tensor:
        """This rank's dW and dbias as FP32 sums in a flat buffer (before the cast)."""
        N = X.shape[0]
        self._check(X, (N, self.C * self.T), "X")
        self._check(dY, (N, self.D * self.T), "dY")
        if buf is None:
            buf = self.grad_buffer(torch.float32, X.device)
        if buf.dtype != torch.float32 or buf.numel() != self.grad_offset() + self.D:
            raise ValueError("buf must be a flat FP32 gradient buffer of this plan")
        dW, db = self.split_grad(buf)
        nb = self.workspace_bytes(N)
        if workspace is None:
            workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=X.device)
        _n.eqlinear_backward_weight_f32(self.handle, X, dY, N, dW, db, workspace,
                                        workspace.numel() * workspace.element_size())
        return buf

    def cast_from_f32(self, src: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """Round an FP32 tensor to the plan dtype on the GPU (nearest-even)."""
        if not src.is_cuda or src.dtype != torch.float32 or not src.is_contiguous():
            raise ValueError("src must be a contiguous CUDA FP32 tensor")
        if out is None:
            out = torch.empty(tuple(src.shape), dtype=self.dtype, device=src.device)
        if out.dtype != self.dtype or out.numel() != src.numel() or not out.is_contiguous():
            raise ValueError("out must be a contiguous tensor of the plan dtype, same size")
        _n.eqlinear_cast_from_f32(self.handle, src, src.numel(), out)
        return out

    def status(self) -> int:
        return _n.eqlinear_get_status(self.handle)


def forward_chain(first: EqLinearPlan, second: EqLinearPlan, X, W1_hat, bias1, W2_hat, bias2,
                  act: str = "none", spectral: bool = False, H=None, Y=None, workspace=None):
    """Two chained layers in one launch: H = act(first(X)), Y = second(H).

    Returns (H, Y); H is [N, D1*T], or the spectral planes [4, N, D1] when
    ``spectral``.  Bitwise equal to the two separate calls.  A ``workspace``
    passed in must be zero-filled before its first use (each call leaves it
    zero).
    """
    N = X.shape[0]
    first._check(X, (N, first.C * first.T), "X")
    if second.C != first.D:
        raise ValueError("the second layer's input width must be the first layer's output width")
    shape_h = (4, N, first.D) if spectral else (N, first.D * first.T)
    if H is None:
        H = torch.empty(shape_h, dtype=first.dtype, device=X.device)
    if Y is None:
        Y = torch.empty((N, second.D * second.T), dtype=second.dtype, device=X.device)
    nb = _n.eqlinear_chain_workspace_bytes(first.handle, second.handle, N)
    if workspace is None:
        # counters that must start at zero; each call leaves them zero again
        workspace = torch.zeros(max(nb, 16), dtype=torch.uint8, device=X.device)
    _n.eqlinear_forward_chain(first.handle, second.handle, X, N, W1_hat, bias1, _n.ACT[act],
                              W2_hat, bias2, 1 if spectral else 0, H, Y, workspace,
                              workspace.numel() * workspace.element_size())
    return H, Y



def forward_chain_tiled(first: EqLinearPlan, second: EqLinearPlan, Xt, N: int, W1_hat, bias1,
                        W2_hat, bias2, act: str = "none", Ht=None, Y=None, workspace=None):
    """Two chained layers on tiled planes in one launch: Ht = tiled planes of
    act(first(X)), Y = second(H) [N, D2*T], from Xt = first.group_dft(X).
    Bitwise equal to first.forward_tiled_next then second.forward_tiled.  A
    ``workspace`` passed in must be zero-filled before its first use (each call
    leaves it zero)."""
    first._check(Xt, first.tiled_shape(N, first.C), "Xt")
    if second.C != first.D:
        raise ValueError("the second layer's input width must be the first layer's output width")
    if Ht is None:
        Ht = torch.empty(first.tiled_shape(N, first.D), dtype=first.dtype, device=Xt.device)
    if Y is None:
        Y = torch.empty((N, second.D * second.T), dtype=second.dtype, device=Xt.device)
    nb = _n.eqlinear_chain_tiled_workspace_bytes(first.handle, second.handle, N)
    if workspace is None:
        workspace = torch.zeros(max(nb, 16), dtype=torch.uint8, device=Xt.device)
    _n.eqlinear_forward_chain_tiled(first.handle, second.handle, Xt, N, W1_hat, bias1,
                                    _n.ACT[act], W2_hat, bias2, Ht, Y, workspace,
                                    workspace.numel() * workspace.element_size())
    return Ht, Y
