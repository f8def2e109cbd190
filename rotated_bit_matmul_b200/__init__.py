"""B200 (sm_100a) rotated low-bit linear: HARP's inference hot path.

"HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme LLM
Quantization" wraps every linear layer in two butterfly transforms (log2 w stages
of 2x2 Givens-times-Hadamard blocks after a random sign diagonal, initialised to the
randomized Hadamard transform) around a low-bit quantized weight matrix:
y = U^T dequant(Q(U W V^T)) V x, with V x and U^T applied online.

This package is a thin torch-facing binding of libharp.so (C ABI in include/harp.h).
The functions keep the C names; they marshal tensors into device pointers and the
current CUDA stream and raise HarpError on a non-OK status. All arithmetic runs in
the library's kernels; there is no Python or CPU fallback.
"""
from __future__ import annotations

import ctypes
import math

from ._lib import (HARP_BF16, HARP_F16, HARP_F32, HarpError, call, load)  # noqa: F401

__all__ = ["HarpError", "harp_butterfly_fwd", "harp_butterfly_inv", "harp_quantize_weights", "HarpLayer",
           "HarpStack", "HarpMixedRadix", "rotate_weights_device", "harp_quantize_angles", "harp_calib_fit", "harp_device_status",
           "harp_test_set_faults", "load"]


def _torch():
    import torch
    return torch


def _dt(t) -> int:
    torch = _torch()
    return {torch.float32: HARP_F32, torch.bfloat16: HARP_BF16, torch.float16: HARP_F16}[t.dtype]


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _contig(t):
    return t.contiguous() if t is not None else None


def _stream():
    return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("rotated_bit_matmul_b200 works on CUDA tensors only")


def harp_device_status() -> None:
    """Raises HarpError if a kernel reported a device-side failure (clears it)."""
    call("harp_device_status", _stream())


def harp_test_set_faults(wait_limit_us: int = 0, gemv_skip_stage: int = -1, decode_barrier: int = -1) -> None:
    """Testing hook for the failure paths (process-wide; the defaults switch it off): a short
    bound on device-side waits, a weight-ring stage the dequant-GEMV's first CTA never
    issues, a grid barrier of the fused decode step that can never complete."""
    call("harp_test_set_faults", int(wait_limit_us), int(gemv_skip_stage), int(decode_barrier))


def _bfly(name, x, theta, sign, w, out_dtype=None, out=None):
    torch = _torch()
    _need_cuda(x, theta, sign)
    x2 = x.reshape(-1, x.shape[-1]) if x.dim() > 1 else x.reshape(1, -1)
    if not x2.is_contiguous():
        x2 = x2.contiguous()
    n = x2.shape[1]
    if out is None:
        out = torch.empty(x2.shape, dtype=out_dtype or x.dtype, device=x.device)
    call(name, n, int(w), x2.shape[0], _p(theta), _p(sign), _p(x2), _dt(x2), _p(out), _dt(out), _stream())
    return out.reshape(x.shape)


def harp_butterfly_fwd(x, theta, sign, w, out_dtype=None, out=None):
    """F(theta, s, w) x over the last dimension. theta fp32 [log2 w, n/2] (None: Theta = 0,
    the fixed randomized Hadamard transform), sign int8 [n]."""
    return _bfly("harp_butterfly_fwd", x, theta, sign, w, out_dtype, out)


def harp_butterfly_inv(x, theta, sign, w, out_dtype=None, out=None):
    """F(theta, s, w)^T x over the last dimension."""
    return _bfly("harp_butterfly_inv", x, theta, sign, w, out_dtype, out)


def harp_quantize_weights(W_rot, bits: int, group: int = 64):
    """Quantizes a rotated fp32 [n_out, n_in] matrix; returns (codes uint8, scale_zero int32)."""
    torch = _torch()
    _need_cuda(W_rot)
    W_rot = W_rot.contiguous()
    n_out, n_in = W_rot.shape
    codes = torch.empty(n_out * n_in * bits // 8, dtype=torch.uint8, device=W_rot.device)
    sz = torch.empty(n_out * (n_in // group), dtype=torch.int32, device=W_rot.device)
    call("harp_quantize_weights", n_out, n_in, int(bits), int(group), _p(W_rot), _p(codes), _p(sz), _stream())
    return codes, sz


def harp_quantize_angles(theta):
    """int8 storage of a butterfly's angle offsets theta fp32 [m, n/2]: returns (q int8
    [m, n/2], delta fp32 [m]) with delta_t = max |theta_t| / 127 and q = RNE(theta / delta_t)."""
    torch = _torch()
    _need_cuda(theta)
    th = theta.float().contiguous()
    m, half = th.shape
    q = torch.empty((m, half), dtype=torch.int8, device=th.device)
    d = torch.empty(max(m, 4), dtype=torch.float32, device=th.device)  # 16-byte allocation
    call("harp_quantize_angles", int(m), int(half), _p(th), _p(q), _p(d), _stream())
    return q, d[:m]


def rotate_weights_device(W, theta_V, sign_V, w_in, theta_U, sign_U, w_out):
    """W' = U W V^T on the device: rows through F_V, then columns through F_U^T."""
    _need_cuda(W)
    Wr = harp_butterfly_fwd(W.float().contiguous(), theta_V, sign_V, w_in)
    Wt = Wr.t().contiguous()
    harp_butterfly_inv(Wt, theta_U, sign_U, w_out, out=Wt)
    return Wt.t().contiguous()


def harp_calib_fit(W, bits, w_in, w_out, theta_V, sign_V, theta_U, sign_U, H=None, lambda_bd=0.0, grad=False,
                   group=64):
    """The per-layer fitting loss L_fit = L_diag + lambda_bd R_bd (wraps harp_calib_fit).

    Returns a device fp64 tensor [L_fit, L_diag, R_bd]; with grad=True also the fp32
    gradients in theta_V and theta_U (shaped [log2 w, n/2]). theta None: Theta = 0.
    H: the fp32 [n_in, n_in] input Hessian proxy, or None for the identity."""
    torch = _torch()
    _need_cuda(W, theta_V, sign_V, theta_U, sign_U, H)
    W = W.float().contiguous()
    n_out, n_in = W.shape
    Hc = H.float().contiguous() if H is not None else None
    n = ctypes.c_size_t()
    call("harp_calib_workspace_size", n_out, n_in, int(bits), int(w_in), int(w_out), int(H is not None), int(grad),
         ctypes.byref(n))
    ws = torch.empty(n.value, dtype=torch.uint8, device=W.device)
    loss = torch.empty(3, dtype=torch.float64, device=W.device)
    gV = torch.empty((log2i(w_in), n_in // 2), dtype=torch.float32, device=W.device) if grad else None
    gU = torch.empty((log2i(w_out), n_out // 2), dtype=torch.float32, device=W.device) if grad else None
    call("harp_calib_fit", n_out, n_in, int(bits), int(group), int(w_in), int(w_out), _p(W), _p(_contig(theta_V)),
         _p(sign_V.contiguous()), _p(_contig(theta_U)), _p(sign_U.contiguous()), _p(Hc), float(lambda_bd), _p(loss),
         _p(gV), _p(gU), _p(ws), ws.numel(), _stream())
    return (loss, gV, gU) if grad else loss


class HarpLayer:
    """A rotated low-bit linear on the device (wraps harp_create_layer). theta_V or theta_U
    None makes that side the fixed randomized Hadamard transform (Theta = 0)."""

    def __init__(self, n_in, n_out, bits, w_in, w_out, theta_V, sign_V, theta_U, sign_U, codes, scale_zero,
                 group=64):
        _need_cuda(theta_V, sign_V, theta_U, sign_U, codes, scale_zero)
        self._fields(n_in, n_out, bits, w_in, w_out, codes, scale_zero, group)
        h = ctypes.c_void_p()
        call("harp_create_layer", ctypes.byref(h), self.n_in, self.n_out, self.bits, self.group, self.w_in,
             self.w_out, _p(_contig(theta_V)), _p(sign_V.contiguous()), _p(_contig(theta_U)),
             _p(sign_U.contiguous()), _p(codes), _p(scale_zero), _stream())
        self.handle = h

    @classmethod
    def int8_angles(cls, n_in, n_out, bits, w_in, w_out, q_V, delta_V, sign_V, q_U, delta_U, sign_U, codes,
                    scale_zero, group=64):
        """A layer keeping its angles in int8 (wraps harp_create_layer_q8): q int8
        [log2 w, n/2] and delta fp32 [log2 w] per side, as harp_quantize_angles returns
        them; q None makes that side Theta = 0."""
        _need_cuda(q_V, delta_V, sign_V, q_U, delta_U, sign_U, codes, scale_zero)
        self = cls.__new__(cls)
        self._fields(n_in, n_out, bits, w_in, w_out, codes, scale_zero, group)
        h = ctypes.c_void_p()
        call("harp_create_layer_q8", ctypes.byref(h), self.n_in, self.n_out, self.bits, self.group, self.w_in,
             self.w_out, _p(_contig(q_V)), _p(_contig(delta_V)), _p(sign_V.contiguous()), _p(_contig(q_U)),
             _p(_contig(delta_U)), _p(sign_U.contiguous()), _p(codes), _p(scale_zero), _stream())
        self.handle = h
        return self

    @classmethod
    def mixed_radix(cls, V, U, bits, codes, scale_zero, group=64):
        """A layer whose sides are mixed-radix butterflies (wraps harp_create_layer_mr): V and U
        are HarpMixedRadix plans of lengths n_in and n_out; the layer borrows them (they must
        outlive it) as it borrows codes and scale_zero."""
        _need_cuda(codes, scale_zero)
        self = cls.__new__(cls)
        self._fields(V.d, U.d, bits, 0, 0, codes, scale_zero, group)
        self._plans = (V, U)
        h = ctypes.c_void_p()
        call("harp_create_layer_mr", ctypes.byref(h), self.n_in, self.n_out, self.bits, self.group, V.handle,
             U.handle, _p(codes), _p(scale_zero), _stream())
        self.handle = h
        return self

    def _fields(self, n_in, n_out, bits, w_in, w_out, codes, scale_zero, group):
        self.handle = None
        self.n_in, self.n_out, self.bits, self.group = int(n_in), int(n_out), int(bits), int(group)
        self.w_in, self.w_out = int(w_in), int(w_out)
        # the library borrows codes and scale_zero: keep them alive with the handle
        self.codes, self.scale_zero = codes, scale_zero
        self._ws = {}
        self.device = codes.device

    def workspace_bytes(self, batch: int) -> int:
        n = ctypes.c_size_t()
        call("harp_linear_workspace_size", self.handle, int(batch), ctypes.byref(n))
        return n.value

    def workspace(self, batch: int):
        ws = self._ws.get(batch)
        if ws is None:
            ws = _torch().empty(max(self.workspace_bytes(batch), 256), dtype=_torch().uint8, device=self.device)
            self._ws[batch] = ws
        return ws

    def __call__(self, x, out_dtype=None, out=None, workspace=None):
        torch = _torch()
        _need_cuda(x)
        x2 = x.reshape(-1, self.n_in).contiguous()
        if out is None:
            out = torch.empty((x2.shape[0], self.n_out), dtype=out_dtype or x.dtype, device=x.device)
        ws = workspace if workspace is not None else self.workspace(x2.shape[0])
        call("harp_linear_fwd", self.handle, x2.shape[0], _p(x2), _dt(x2), _p(out), _dt(out), _p(ws),
             ws.numel(), _stream())
        return out

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            call("harp_destroy_layer", self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class HarpMixedRadix:
    """A mixed-radix butterfly (wraps harp_mr_plan_*): d = prod(radices), stage t mixing the
    coordinates that differ in mixed-radix digit t with Q(theta) G_b blocks (Givens for
    b = 2, Cayley times the base mixer above). theta: fp32, stage after stage, group after
    group; gauss: one b x b fp32 Gaussian per stage (None when every radix is a power of two)."""

    def __init__(self, radices, theta, sign, gauss=None):
        _need_cuda(theta, sign, gauss)
        self.radices = [int(b) for b in radices]
        self.d = int(math.prod(self.radices))
        want = sum((self.d // b) * (1 if b == 2 else b * (b - 1) // 2) for b in self.radices)
        if theta.numel() != want:
            raise ValueError(f"theta has {theta.numel()} parameters, the schedule needs {want}")
        if gauss is not None and gauss.numel() != sum(b * b for b in self.radices):
            raise ValueError("gauss needs one b x b matrix per stage")
        r = (ctypes.c_int * len(self.radices))(*self.radices)
        h = ctypes.c_void_p()
        self.handle = None
        call("harp_mr_plan_create", ctypes.byref(h), self.d, len(self.radices), r, _p(theta.float().contiguous()),
             _p(sign.contiguous()), _p(gauss.float().contiguous() if gauss is not None else None), _stream())
        self.handle = h

    def _apply(self, name, x, out_dtype, out):
        torch = _torch()
        _need_cuda(x)
        x2 = x.reshape(-1, self.d).contiguous()
        if out is None:
            out = torch.empty(x2.shape, dtype=out_dtype or x.dtype, device=x.device)
        call(name, self.handle, x2.shape[0], _p(x2), _dt(x2), _p(out), _dt(out), _stream())
        return out.reshape(x.shape)

    def fwd(self, x, out_dtype=None, out=None):
        return self._apply("harp_mr_butterfly_fwd", x, out_dtype, out)

    def inv(self, x, out_dtype=None, out=None):
        return self._apply("harp_mr_butterfly_inv", x, out_dtype, out)

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            call("harp_mr_plan_destroy", self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class HarpStack:
    """Llama-shaped decode stack of rotated linears (wraps harp_stack_create/step)."""

    def __init__(self, layers, hidden, ffn, n_heads, n_kv_heads, head_dim, eps=1e-5):
        self.layers = list(layers)
        assert len(self.layers) % 7 == 0
        arr = (ctypes.c_void_p * len(self.layers))(*[l.handle.value for l in self.layers])
        h = ctypes.c_void_p()
        call("harp_stack_create", ctypes.byref(h), len(self.layers) // 7, int(hidden), int(ffn), int(n_heads),
             int(n_kv_heads), int(head_dim), ctypes.c_float(eps), arr, _stream())
        self.handle = h
        self.hidden = int(hidden)
        self._ws = {}
        self.device = self.layers[0].device

    def workspace_bytes(self, batch: int) -> int:
        n = ctypes.c_size_t()
        call("harp_stack_workspace_size", self.handle, int(batch), ctypes.byref(n))
        return n.value

    def uses_fused_step(self, batch: int = 1) -> bool:
        """True when a step of this batch runs the single-kernel fused decode path (when the
        stack's shapes keep it on the per-linear path, harp_last_error says why)."""
        return bool(load().harp_stack_uses_fused_step(self.handle, int(batch)))

    def fused_reason(self) -> str:
        """Why the fused decode step is not taken ('' when it is)."""
        lib = load()
        return "" if lib.harp_stack_uses_fused_step(self.handle, 1) else lib.harp_last_error().decode()

    def workspace(self, batch: int):
        ws = self._ws.get(batch)
        if ws is None:
            ws = _torch().empty(self.workspace_bytes(batch), dtype=_torch().uint8, device=self.device)
            self._ws[batch] = ws
        return ws

    def step(self, x, out_dtype=None, out=None, workspace=None):
        torch = _torch()
        _need_cuda(x)
        x2 = x.reshape(-1, self.hidden).contiguous()
        if out is None:
            out = torch.empty(x2.shape, dtype=out_dtype or torch.float32, device=x.device)
        ws = workspace if workspace is not None else self.workspace(x2.shape[0])
        call("harp_stack_step", self.handle, x2.shape[0], _p(x2), _dt(x2), _p(out), _dt(out), _p(ws), ws.numel(),
             _stream())
        return out

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            call("harp_stack_destroy", self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def log2i(w: int) -> int:
    m = int(math.log2(w))
    assert 1 << m == w
    return m
