"""Tensor-level API over the C ABI: torch tensors in, torch tensors out.

PyTorch provides device memory and the current CUDA stream; every step of the computation runs
in libqlora_nf4.so.  All tensors must be contiguous CUDA tensors on the current device.
"""

from dataclasses import dataclass

import torch

from . import abi


def _ptr(t):
    return t.data_ptr() if t is not None else None


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _need(t, dtype, shape, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


@dataclass
class NF4Weight:
    """A packed NF4 base weight W0 [N, K] (device tensors owned by this object)."""
    q: torch.Tensor                      # [N, K/2] uint8
    absmax: torch.Tensor                 # [N*K/64] fp32 (first-level absmax)
    absmax_q8: torch.Tensor = None       # [N*K/64] uint8 (double-quantised)
    absmax_scale: torch.Tensor = None    # [ceil(N*K/64/256)] fp32
    N: int = 0
    K: int = 0
    double_quant: bool = False

    def c_struct(self):
        return abi.Nf4Weight(
            _ptr(self.q), None if self.double_quant else _ptr(self.absmax),
            _ptr(self.absmax_q8) if self.double_quant else None,
            _ptr(self.absmax_scale) if self.double_quant else None,
            self.N, self.K, 1 if self.double_quant else 0)


def nf4_pack(W, double_quant=False):
    """Quantise a bf16 weight [N, K] to NF4 (qlora_nf4_pack)."""
    N, K = W.shape
    _need(W, torch.bfloat16, (N, K), "W")
    dev = W.device
    q = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    nb = N * (K // 64)
    absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    q8 = scale = None
    if double_quant:
        q8 = torch.empty(nb, dtype=torch.uint8, device=dev)
        scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    abi.qlora_nf4_pack(W.data_ptr(), N, K, double_quant, q.data_ptr(), absmax.data_ptr(),
                       _ptr(q8), _ptr(scale), _stream())
    return NF4Weight(q, absmax, q8, scale, N, K, bool(double_quant))


def nf4_dequant(w: NF4Weight):
    """bf16 [N, K] dequantised weight (test / diagnostic export, qlora_nf4_dequant)."""
    out = torch.empty((w.N, w.K), dtype=torch.bfloat16, device=w.q.device)
    abi.qlora_nf4_dequant(w.c_struct(), out.data_ptr(), _stream())
    return out


def workspace_bytes(M, N, K, r):
    return abi.qlora_workspace_bytes(M, N, K, r)


def alloc_workspace(M, N, K, r, device):
    n = workspace_bytes(M, N, K, r)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def forward(X, w: NF4Weight, A, B, alpha, H=None, XA=None, ws=None, save_xa=True):
    """h = X deq(W0)^T + (alpha/r) (X A^T) B^T.  Returns (h, XA_saved), XA_saved None when
    save_xa is False (the backward then recomputes it)."""
    M, K = X.shape
    r = A.shape[0]
    _need(X, torch.bfloat16, (M, w.K), "X")
    _need(A, torch.bfloat16, (r, w.K), "A")
    _need(B, torch.bfloat16, (w.N, r), "B")
    if H is None:
        H = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if XA is None and save_xa:
        XA = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = alloc_workspace(M, w.N, w.K, r, X.device)
    abi.qlora_linear_fwd(X.data_ptr(), w.c_struct(), A.data_ptr(), B.data_ptr(), M, r, alpha,
                         H.data_ptr(), _ptr(XA) if save_xa else None, ws.data_ptr(), ws.numel(),
                         _stream())
    return H, (XA if save_xa else None)


def backward(dY, X, w: NF4Weight, A, B, XA, alpha, need_dx=True, dX=None, dA=None, dB=None,
             ws=None):
    """Hand-derived gradients.  Returns (dX or None, dA fp32 [r, K], dB fp32 [N, r]).  XA None:
    recomputed from X."""
    M = X.shape[0]
    r = A.shape[0]
    _need(dY, torch.bfloat16, (M, w.N), "dY")
    _need(X, torch.bfloat16, (M, w.K), "X")
    if XA is not None:
        _need(XA, torch.bfloat16, (M, r), "XA")
    dev = X.device
    if need_dx and dX is None:
        dX = torch.empty((M, w.K), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, w.K), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((w.N, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(M, w.N, w.K, r, dev)
    abi.qlora_linear_bwd(dY.data_ptr(), X.data_ptr(), w.c_struct(), A.data_ptr(), B.data_ptr(),
                         _ptr(XA), M, r, alpha, _ptr(dX) if need_dx else None,
                         dA.data_ptr(), dB.data_ptr(), ws.data_ptr(), ws.numel(), _stream())
    return (dX if need_dx else None), dA, dB


def grouped_workspace_bytes(M, N, K, r, n_groups):
    return abi.qlora_grouped_workspace_bytes(M, N, K, r, n_groups)


def alloc_grouped_workspace(M, N, K, r, n_groups, device):
    n = grouped_workspace_bytes(M, N, K, r, n_groups)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def grouped_forward(X, w: NF4Weight, A, B, group_rows, alpha, H=None, XA=None, ws=None,
                    save_xa=True):
    """Adapters packed along W0's rows (qlora_grouped_fwd).  w: NF4 [sum N_g, K]; A [n r, K];
    B [sum N_g, r].  Returns (H [M, sum N_g], XA_saved [M, n r] or None)."""
    M = X.shape[0]
    n = len(group_rows)
    r = A.shape[0] // n
    _need(X, torch.bfloat16, (M, w.K), "X")
    _need(A, torch.bfloat16, (n * r, w.K), "A")
    _need(B, torch.bfloat16, (w.N, r), "B")
    if H is None:
        H = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if XA is None and save_xa:
        XA = torch.empty((M, n * r), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = alloc_grouped_workspace(M, w.N, w.K, r, n, X.device)
    abi.qlora_grouped_fwd(X.data_ptr(), w.c_struct(), A.data_ptr(), B.data_ptr(), group_rows, M,
                          r, alpha, H.data_ptr(), _ptr(XA) if save_xa else None, ws.data_ptr(),
                          ws.numel(), _stream())
    return H, (XA if save_xa else None)


def gate_up_swiglu_forward(X, w: NF4Weight, A, B, alpha, GU=None, XA=None, act=None, ws=None,
                           save_xa=True):
    """Packed gate/up forward with its SwiGLU (qlora_grouped_fwd_swiglu): w NF4 [2I, K] (gate
    rows, then up rows); A [2r, K]; B [2I, r].  Returns (GU [M, 2I], XA [M, 2r] or None,
    act [M, I] = silu(g) * u)."""
    M = X.shape[0]
    r = A.shape[0] // 2
    I = w.N // 2
    _need(X, torch.bfloat16, (M, w.K), "X")
    _need(A, torch.bfloat16, (2 * r, w.K), "A")
    _need(B, torch.bfloat16, (w.N, r), "B")
    if GU is None:
        GU = torch.empty((M, w.N), dtype=torch.bfloat16, device=X.device)
    if XA is None and save_xa:
        XA = torch.empty((M, 2 * r), dtype=torch.bfloat16, device=X.device)
    if act is None:
        act = torch.empty((M, I), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = alloc_grouped_workspace(M, w.N, w.K, r, 2, X.device)
    abi.qlora_grouped_fwd_swiglu(X.data_ptr(), w.c_struct(), A.data_ptr(), B.data_ptr(), M, r,
                                 alpha, GU.data_ptr(), _ptr(XA) if save_xa else None,
                                 act.data_ptr(), ws.data_ptr(), ws.numel(), _stream())
    return GU, (XA if save_xa else None), act


def grouped_backward(dY, X, w: NF4Weight, A, B, XA, group_rows, alpha, need_dx=True, dX=None,
                     dA=None, dB=None, ws=None):
    """Backward of grouped_forward.  Returns (dX or None, dA fp32 [n r, K], dB fp32 [N, r])."""
    M = X.shape[0]
    n = len(group_rows)
    r = A.shape[0] // n
    _need(dY, torch.bfloat16, (M, w.N), "dY")
    _need(X, torch.bfloat16, (M, w.K), "X")
    if XA is not None:
        _need(XA, torch.bfloat16, (M, n * r), "XA")
    dev = X.device
    if need_dx and dX is None:
        dX = torch.empty((M, w.K), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((n * r, w.K), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((w.N, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_grouped_workspace(M, w.N, w.K, r, n, dev)
    abi.qlora_grouped_bwd(dY.data_ptr(), X.data_ptr(), w.c_struct(), A.data_ptr(), B.data_ptr(),
                          _ptr(XA), group_rows, M, r, alpha, _ptr(dX) if need_dx else None,
                          dA.data_ptr(), dB.data_ptr(), ws.data_ptr(), ws.numel(), _stream())
    return (dX if need_dx else None), dA, dB


def swiglu_forward(g, u, a=None):
    if a is None:
        a = torch.empty_like(g)
    abi.qlora_swiglu_fwd(g.data_ptr(), u.data_ptr(), a.data_ptr(), g.numel(), _stream())
    return a


def swiglu_backward(g, u, da, dg=None, du=None):
    if dg is None:
        dg = torch.empty_like(g)
    if du is None:
        du = torch.empty_like(g)
    abi.qlora_swiglu_bwd(g.data_ptr(), u.data_ptr(), da.data_ptr(), dg.data_ptr(), du.data_ptr(),
                         g.numel(), _stream())
    return dg, du


def swiglu_packed_forward(gu, a=None):
    """a = silu(g) u for a packed gate/up output gu [M, 2I] (g first)."""
    M, I2 = gu.shape
    if a is None:
        a = torch.empty((M, I2 // 2), dtype=gu.dtype, device=gu.device)
    abi.qlora_swiglu_packed_fwd(gu.data_ptr(), a.data_ptr(), M, I2 // 2, _stream())
    return a


def swiglu_packed_backward(gu, da, dgu=None):
    """dgu [M, 2I]: dg and du in the packed layer's column order."""
    if dgu is None:
        dgu = torch.empty_like(gu)
    M, I2 = gu.shape
    abi.qlora_swiglu_packed_bwd(gu.data_ptr(), da.data_ptr(), dgu.data_ptr(), M, I2 // 2,
                                _stream())
    return dgu


def lm_head_ce(X, w: NF4Weight, labels, chunk=1024, need_dx=True, dX=None, token_loss=None,
               ws=None):
    """Chunked LM head + cross-entropy (qlora_lm_head_ce): X [M, K] bf16, w the NF4 head
    [V, K], labels [M] int32 (outside [0, V): ignored).  Returns (loss [1] fp32, token_loss
    [M] fp32, dX [M, K] bf16 or None)."""
    M = X.shape[0]
    _need(X, torch.bfloat16, (M, w.K), "X")
    _need(labels, torch.int32, (M,), "labels")
    dev = X.device
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    if token_loss is None:
        token_loss = torch.empty(M, dtype=torch.float32, device=dev)
    if need_dx and dX is None:
        dX = torch.empty((M, w.K), dtype=torch.bfloat16, device=dev)
    if ws is None:
        n = abi.qlora_lm_head_ce_workspace_bytes(M, w.N, w.K, chunk)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    abi.qlora_lm_head_ce(X.data_ptr(), w.c_struct(), labels.data_ptr(), M, chunk,
                         loss.data_ptr(), token_loss.data_ptr(), _ptr(dX) if need_dx else None,
                         ws.data_ptr(), ws.numel(), _stream())
    return loss, token_loss, (dX if need_dx else None)


def device_error():
    """Synchronising: the device error word (0 = none), cleared after reading."""
    return abi.qlora_device_error()
