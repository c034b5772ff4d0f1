"""Tensor-level binding of the C ABI: same names as the C entry points.

Argument marshalling only: check that tensors are contiguous CUDA tensors of the
expected dtype, allocate outputs that the caller did not pass (torch is used for
device memory and streams), pass ``data_ptr()`` values and the current CUDA stream
to libbitlinear.so.  Every step of the computation runs in the library's kernels.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib

_DT = {torch.float32: _lib.BL_F32, torch.bfloat16: _lib.BL_BF16}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _cuda(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def workspace_bytes(T: int, N: int, K: int) -> int:
    return int(_lib.lib().bitlinear_workspace_bytes(T, N, K))


def workspace(T: int, N: int, K: int, device) -> torch.Tensor:
    return torch.empty(workspace_bytes(T, N, K), dtype=torch.uint8, device=device)


def bitlinear_quant_weight(W: torch.Tensor, want_i8: bool = True, want_bf16: bool = True,
                           want_packed: bool = True, ws: Optional[torch.Tensor] = None, out=None):
    """Returns dict(gamma [1] f32, wq_i8 [N,K] i8, wq_bf16 [N,K] bf16, packed [N,K/4] u8)."""
    _cuda(W, "W", torch.float32)
    N, K = W.shape
    dev = W.device
    o = dict(out or {})
    o.setdefault("gamma", torch.empty(1, dtype=torch.float32, device=dev))
    if want_i8:
        o.setdefault("wq_i8", torch.empty(N, K, dtype=torch.int8, device=dev))
    if want_bf16:
        o.setdefault("wq_bf16", torch.empty(N, K, dtype=torch.bfloat16, device=dev))
    if want_packed:
        o.setdefault("packed", torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
    if ws is None:
        ws = workspace(1, N, K, dev)
    _lib.call("bitlinear_quant_weight", W.data_ptr(), N, K, _ptr(o.get("wq_i8")), _ptr(o.get("wq_bf16")),
              _ptr(o.get("packed")), o["gamma"].data_ptr(), ws.data_ptr(), ws.numel(), _stream(dev))
    return o


def bitlinear_quant_weight_noalloc(W: torch.Tensor, gamma: torch.Tensor, wq_i8: Optional[torch.Tensor] = None,
                                   wq_bf16: Optional[torch.Tensor] = None, packed: Optional[torch.Tensor] = None):
    """bitlinear_quant_weight without a workspace: the caller passes every output and the
    library uses its built-in scratch (see include/bitlinear.h)."""
    _cuda(W, "W", torch.float32)
    N, K = W.shape
    _lib.call("bitlinear_quant_weight_noalloc", W.data_ptr(), N, K, _ptr(wq_i8), _ptr(wq_bf16), _ptr(packed),
              gamma.data_ptr(), _stream(W.device))
    return gamma


def bitlinear_act_quant(X: torch.Tensor, apply_rmsnorm: bool = True, g: Optional[torch.Tensor] = None,
                        eps: float = 1e-6, want_xdq: bool = True, out=None):
    """Returns dict(xq [T,K] i8, sx [T] f32, rinv [T] f32 or None, xdq [T,K] X.dtype or None)."""
    _cuda(X, "X")
    T, K = X.shape
    dev = X.device
    if g is not None:
        _cuda(g, "g", torch.float32)
    o = dict(out or {})
    o.setdefault("xq", torch.empty(T, K, dtype=torch.int8, device=dev))
    o.setdefault("sx", torch.empty(T, dtype=torch.float32, device=dev))
    if apply_rmsnorm:
        o.setdefault("rinv", torch.empty(T, dtype=torch.float32, device=dev))
    if want_xdq:
        o.setdefault("xdq", torch.empty(T, K, dtype=X.dtype, device=dev))
    _lib.call("bitlinear_act_quant", X.data_ptr(), _dt(X), T, K, 1 if apply_rmsnorm else 0, _ptr(g), float(eps),
              o["xq"].data_ptr(), o["sx"].data_ptr(), _ptr(o.get("rinv")), _ptr(o.get("xdq")), _stream(dev))
    return o


def bitlinear_linear(xq: torch.Tensor, sx: torch.Tensor, wq_i8: torch.Tensor, gamma: torch.Tensor,
                     out_dtype=torch.bfloat16, want_acc: bool = False, y: Optional[torch.Tensor] = None,
                     acc: Optional[torch.Tensor] = None):
    _cuda(xq, "xq", torch.int8)
    _cuda(wq_i8, "wq_i8", torch.int8)
    T, K = xq.shape
    N = wq_i8.shape[0]
    dev = xq.device
    if y is None:
        y = torch.empty(T, N, dtype=out_dtype, device=dev)
    if want_acc and acc is None:
        acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    _lib.call("bitlinear_linear", xq.data_ptr(), sx.data_ptr(), T, K, wq_i8.data_ptr(), gamma.data_ptr(), N,
              y.data_ptr(), _dt(y), _ptr(acc), _stream(dev))
    return y, acc


def bitlinear_forward(X: torch.Tensor, wq_i8: torch.Tensor, gamma: torch.Tensor, g: Optional[torch.Tensor] = None,
                      eps: float = 1e-6, want_acc: bool = False, want_xdq: bool = True, out=None):
    """Returns dict(y, xq, sx, rinv, xdq, acc)."""
    _cuda(X, "X")
    _cuda(wq_i8, "wq_i8", torch.int8)
    T, K = X.shape
    N = wq_i8.shape[0]
    dev = X.device
    o = dict(out or {})
    o.setdefault("y", torch.empty(T, N, dtype=X.dtype, device=dev))
    o.setdefault("xq", torch.empty(T, K, dtype=torch.int8, device=dev))
    o.setdefault("sx", torch.empty(T, dtype=torch.float32, device=dev))
    o.setdefault("rinv", torch.empty(T, dtype=torch.float32, device=dev))
    if want_xdq:
        o.setdefault("xdq", torch.empty(T, K, dtype=X.dtype, device=dev))
    if want_acc:
        o.setdefault("acc", torch.empty(T, N, dtype=torch.int32, device=dev))
    _lib.call("bitlinear_forward", X.data_ptr(), _dt(X), T, K, _ptr(g), float(eps), wq_i8.data_ptr(),
              gamma.data_ptr(), N, o["y"].data_ptr(), o["xq"].data_ptr(), o["sx"].data_ptr(), o["rinv"].data_ptr(),
              _ptr(o.get("xdq")), _ptr(o.get("acc")), _stream(dev))
    return o


def bitlinear_forward_qat(X: torch.Tensor, W: torch.Tensor, g: Optional[torch.Tensor] = None, eps: float = 1e-6,
                          want_bf16: bool = True, want_packed: bool = True, want_acc: bool = False,
                          want_xdq: bool = True, ws: Optional[torch.Tensor] = None, out=None):
    """Quantisation-aware forward from the fp32 latent weight (weight and activation
    quantisation, then the linear).  Returns dict(gamma, wq_i8, wq_bf16, packed, y, xq, sx,
    rinv, xdq, acc) -- the union of bitlinear_quant_weight's and bitlinear_forward's."""
    _cuda(X, "X")
    _cuda(W, "W", torch.float32)
    T, K = X.shape
    N = W.shape[0]
    dev = X.device
    o = dict(out or {})
    o.setdefault("gamma", torch.empty(1, dtype=torch.float32, device=dev))
    o.setdefault("wq_i8", torch.empty(N, K, dtype=torch.int8, device=dev))
    if want_bf16:
        o.setdefault("wq_bf16", torch.empty(N, K, dtype=torch.bfloat16, device=dev))
    if want_packed:
        o.setdefault("packed", torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
    o.setdefault("y", torch.empty(T, N, dtype=X.dtype, device=dev))
    o.setdefault("xq", torch.empty(T, K, dtype=torch.int8, device=dev))
    o.setdefault("sx", torch.empty(T, dtype=torch.float32, device=dev))
    o.setdefault("rinv", torch.empty(T, dtype=torch.float32, device=dev))
    if want_xdq:
        o.setdefault("xdq", torch.empty(T, K, dtype=X.dtype, device=dev))
    if want_acc:
        o.setdefault("acc", torch.empty(T, N, dtype=torch.int32, device=dev))
    if ws is None:
        ws = workspace(T, N, K, dev)
    _lib.call("bitlinear_forward_qat", X.data_ptr(), _dt(X), T, K, _ptr(g), float(eps), W.data_ptr(), N,
              o["wq_i8"].data_ptr(), _ptr(o.get("wq_bf16")), _ptr(o.get("packed")), o["gamma"].data_ptr(),
              o["y"].data_ptr(), o["xq"].data_ptr(), o["sx"].data_ptr(), o["rinv"].data_ptr(), _ptr(o.get("xdq")),
              _ptr(o.get("acc")), ws.data_ptr(), ws.numel(), _stream(dev))
    return o


def bitlinear_backward_input(dY: torch.Tensor, X: torch.Tensor, rinv: torch.Tensor, wq_bf16: torch.Tensor,
                             gamma: torch.Tensor, g: Optional[torch.Tensor] = None, want_dg: bool = True,
                             ws: Optional[torch.Tensor] = None, dX: Optional[torch.Tensor] = None,
                             dg: Optional[torch.Tensor] = None):
    _cuda(dY, "dY")
    _cuda(X, "X", dY.dtype)
    _cuda(wq_bf16, "wq_bf16", torch.bfloat16)
    T, N = dY.shape
    K = X.shape[1]
    dev = dY.device
    if dX is None:
        dX = torch.empty(T, K, dtype=torch.float32, device=dev)
    if want_dg and dg is None:
        dg = torch.empty(K, dtype=torch.float32, device=dev)
    if ws is None and dg is not None:
        ws = workspace(T, N, K, dev)
    _lib.call("bitlinear_backward_input", dY.data_ptr(), X.data_ptr(), _dt(dY), T, K, N, _ptr(g), rinv.data_ptr(),
              wq_bf16.data_ptr(), gamma.data_ptr(), dX.data_ptr(), _ptr(dg), _ptr(ws),
              0 if ws is None else ws.numel(), _stream(dev))
    return dX, dg


def bitlinear_grad_input(dY: torch.Tensor, wq_bf16: torch.Tensor, gamma: torch.Tensor,
                         dXhat: Optional[torch.Tensor] = None):
    """dX_hat = gamma * dY . W_q  (fp32 [T, K])."""
    _cuda(dY, "dY")
    _cuda(wq_bf16, "wq_bf16", torch.bfloat16)
    T, N = dY.shape
    K = wq_bf16.shape[1]
    if dXhat is None:
        dXhat = torch.empty(T, K, dtype=torch.float32, device=dY.device)
    _lib.call("bitlinear_grad_input", dY.data_ptr(), _dt(dY), T, K, N, wq_bf16.data_ptr(), gamma.data_ptr(),
              dXhat.data_ptr(), _stream(dY.device))
    return dXhat


def bitlinear_rmsnorm_backward(X: torch.Tensor, rinv: torch.Tensor, dX_inout: torch.Tensor,
                               g: Optional[torch.Tensor] = None, want_dg: bool = True,
                               ws: Optional[torch.Tensor] = None, dg: Optional[torch.Tensor] = None):
    """In place: dX_inout holds dX_hat on entry and dX on return."""
    _cuda(X, "X")
    _cuda(dX_inout, "dX_inout", torch.float32)
    T, K = X.shape
    dev = X.device
    if want_dg and dg is None:
        dg = torch.empty(K, dtype=torch.float32, device=dev)
    if ws is None and dg is not None:
        ws = workspace(T, 16, K, dev)
    _lib.call("bitlinear_rmsnorm_backward", X.data_ptr(), _dt(X), T, K, _ptr(g), rinv.data_ptr(),
              dX_inout.data_ptr(), _ptr(dg), _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev))
    return dX_inout, dg


def bitlinear_backward_weight(dY: torch.Tensor, xdq: torch.Tensor, dW: Optional[torch.Tensor] = None):
    _cuda(dY, "dY")
    _cuda(xdq, "xdq", dY.dtype)
    T, N = dY.shape
    K = xdq.shape[1]
    if dW is None:
        dW = torch.empty(N, K, dtype=torch.float32, device=dY.device)
    _lib.call("bitlinear_backward_weight", dY.data_ptr(), xdq.data_ptr(), _dt(dY), T, K, N, dW.data_ptr(),
              _stream(dY.device))
    return dW


def bitlinear_backward(dY, X, xdq, rinv, wq_bf16, gamma, g=None, want_dg=True, ws=None, dX=None, dW=None, dg=None):
    _cuda(dY, "dY")
    T, N = dY.shape
    K = X.shape[1]
    dev = dY.device
    if dX is None:
        dX = torch.empty(T, K, dtype=torch.float32, device=dev)
    if dW is None:
        dW = torch.empty(N, K, dtype=torch.float32, device=dev)
    if want_dg and dg is None:
        dg = torch.empty(K, dtype=torch.float32, device=dev)
    if ws is None and dg is not None:
        ws = workspace(T, N, K, dev)
    _lib.call("bitlinear_backward", dY.data_ptr(), X.data_ptr(), xdq.data_ptr(), _dt(dY), T, K, N, _ptr(g),
              rinv.data_ptr(), wq_bf16.data_ptr(), gamma.data_ptr(), dX.data_ptr(), dW.data_ptr(), _ptr(dg),
              _ptr(ws), 0 if ws is None else ws.numel(), _stream(dev))
    return dX, dW, dg


def ternary_pack(wq_i8: torch.Tensor, packed: Optional[torch.Tensor] = None):
    _cuda(wq_i8, "wq_i8", torch.int8)
    N, K = wq_i8.shape
    if packed is None:
        packed = torch.empty(N, K // 4, dtype=torch.uint8, device=wq_i8.device)
    _lib.call("ternary_pack", wq_i8.data_ptr(), N, K, packed.data_ptr(), _stream(wq_i8.device))
    return packed


def ternary_gemv(packed: torch.Tensor, gamma: torch.Tensor, K: int, xq: torch.Tensor, sx: torch.Tensor,
                 want_acc: bool = False, y: Optional[torch.Tensor] = None, acc: Optional[torch.Tensor] = None):
    _cuda(packed, "packed", torch.uint8)
    _cuda(xq, "xq", torch.int8)
    N = packed.shape[0]
    B = xq.shape[0]
    dev = packed.device
    if y is None:
        y = torch.empty(B, N, dtype=torch.float32, device=dev)
    if want_acc and acc is None:
        acc = torch.empty(B, N, dtype=torch.int32, device=dev)
    _lib.call("ternary_gemv", packed.data_ptr(), gamma.data_ptr(), N, K, xq.data_ptr(), sx.data_ptr(), B,
              y.data_ptr(), _ptr(acc), _stream(dev))
    return y, acc


# ----------------------------------------------------------------------------------
# quantiser variants (per-row weight scale, zero threshold, per-tensor activation scale)
# ----------------------------------------------------------------------------------

def bitlinear_quant_weight_rows(W: torch.Tensor, want_i8: bool = True, want_bf16: bool = True,
                                want_packed: bool = True, out=None):
    """Per-row scale. Returns dict(gamma_rows [N] f32, wq_i8 [N,K] i8, wq_bf16 [N,K] bf16
    (= W_q * bf16(gamma_n)), packed [N,K/4] u8)."""
    _cuda(W, "W", torch.float32)
    N, K = W.shape
    dev = W.device
    o = dict(out or {})
    o.setdefault("gamma_rows", torch.empty(N, dtype=torch.float32, device=dev))
    if want_i8:
        o.setdefault("wq_i8", torch.empty(N, K, dtype=torch.int8, device=dev))
    if want_bf16:
        o.setdefault("wq_bf16", torch.empty(N, K, dtype=torch.bfloat16, device=dev))
    if want_packed:
        o.setdefault("packed", torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
    _lib.call("bitlinear_quant_weight_rows", W.data_ptr(), N, K, _ptr(o.get("wq_i8")), _ptr(o.get("wq_bf16")),
              _ptr(o.get("packed")), o["gamma_rows"].data_ptr(), _stream(dev))
    return o


def bitlinear_quant_weight_tau(W: torch.Tensor, tau_factor: float = 0.7, want_i8: bool = True,
                               want_bf16: bool = True, want_packed: bool = True,
                               ws: Optional[torch.Tensor] = None, out=None):
    """Zero threshold tau = tau_factor * gamma; outputs as bitlinear_quant_weight."""
    _cuda(W, "W", torch.float32)
    N, K = W.shape
    dev = W.device
    o = dict(out or {})
    o.setdefault("gamma", torch.empty(1, dtype=torch.float32, device=dev))
    if want_i8:
        o.setdefault("wq_i8", torch.empty(N, K, dtype=torch.int8, device=dev))
    if want_bf16:
        o.setdefault("wq_bf16", torch.empty(N, K, dtype=torch.bfloat16, device=dev))
    if want_packed:
        o.setdefault("packed", torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
    if ws is None:
        ws = workspace(1, N, K, dev)
    _lib.call("bitlinear_quant_weight_tau", W.data_ptr(), N, K, float(tau_factor), _ptr(o.get("wq_i8")),
              _ptr(o.get("wq_bf16")), _ptr(o.get("packed")), o["gamma"].data_ptr(), ws.data_ptr(), ws.numel(),
              _stream(dev))
    return o


def bitlinear_act_quant_tensor(X: torch.Tensor, apply_rmsnorm: bool = True, g: Optional[torch.Tensor] = None,
                               eps: float = 1e-6, want_xdq: bool = True, ws: Optional[torch.Tensor] = None,
                               out=None):
    """Per-tensor scale; returns as bitlinear_act_quant (sx holds the one scale T times)."""
    _cuda(X, "X")
    T, K = X.shape
    dev = X.device
    if g is not None:
        _cuda(g, "g", torch.float32)
    o = dict(out or {})
    o.setdefault("xq", torch.empty(T, K, dtype=torch.int8, device=dev))
    o.setdefault("sx", torch.empty(T, dtype=torch.float32, device=dev))
    if apply_rmsnorm:
        o.setdefault("rinv", torch.empty(T, dtype=torch.float32, device=dev))
    if want_xdq:
        o.setdefault("xdq", torch.empty(T, K, dtype=X.dtype, device=dev))
    if ws is None:
        ws = workspace(T, 16, K, dev)
    _lib.call("bitlinear_act_quant_tensor", X.data_ptr(), _dt(X), T, K, 1 if apply_rmsnorm else 0, _ptr(g),
              float(eps), o["xq"].data_ptr(), o["sx"].data_ptr(), _ptr(o.get("rinv")), _ptr(o.get("xdq")),
              ws.data_ptr(), ws.numel(), _stream(dev))
    return o


def bitlinear_linear_rows(xq: torch.Tensor, sx: torch.Tensor, wq_i8: torch.Tensor, gamma_rows: torch.Tensor,
                          out_dtype=torch.bfloat16, want_acc: bool = False, y: Optional[torch.Tensor] = None,
                          acc: Optional[torch.Tensor] = None):
    _cuda(xq, "xq", torch.int8)
    _cuda(wq_i8, "wq_i8", torch.int8)
    T, K = xq.shape
    N = wq_i8.shape[0]
    dev = xq.device
    if y is None:
        y = torch.empty(T, N, dtype=out_dtype, device=dev)
    if want_acc and acc is None:
        acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    _lib.call("bitlinear_linear_rows", xq.data_ptr(), sx.data_ptr(), T, K, wq_i8.data_ptr(), gamma_rows.data_ptr(),
              N, y.data_ptr(), _dt(y), _ptr(acc), _stream(dev))
    return y, acc


def bitlinear_linear_packed(xq: torch.Tensor, sx: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                            K: int, out_dtype=torch.bfloat16, want_acc: bool = False,
                            y: Optional[torch.Tensor] = None, acc: Optional[torch.Tensor] = None,
                            ws: Optional[torch.Tensor] = None):
    """int8 x packed-ternary linear (few tokens); ws (up to 8 x 4*T*N bytes) lets K be split."""
    _cuda(xq, "xq", torch.int8)
    _cuda(packed, "packed", torch.uint8)
    T = xq.shape[0]
    N = packed.shape[0]
    dev = xq.device
    if y is None:
        y = torch.empty(T, N, dtype=out_dtype, device=dev)
    if want_acc and acc is None:
        acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    _lib.call("bitlinear_linear_packed", xq.data_ptr(), sx.data_ptr(), T, K, packed.data_ptr(), gamma.data_ptr(),
              N, y.data_ptr(), _dt(y), _ptr(acc), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
              _stream(dev))
    return y, acc


def ternary_gemv_rows(packed: torch.Tensor, gamma_rows: torch.Tensor, K: int, xq: torch.Tensor, sx: torch.Tensor,
                      want_acc: bool = False, y: Optional[torch.Tensor] = None, acc: Optional[torch.Tensor] = None):
    _cuda(packed, "packed", torch.uint8)
    _cuda(xq, "xq", torch.int8)
    N = packed.shape[0]
    B = xq.shape[0]
    dev = packed.device
    if y is None:
        y = torch.empty(B, N, dtype=torch.float32, device=dev)
    if want_acc and acc is None:
        acc = torch.empty(B, N, dtype=torch.int32, device=dev)
    _lib.call("ternary_gemv_rows", packed.data_ptr(), gamma_rows.data_ptr(), N, K, xq.data_ptr(), sx.data_ptr(), B,
              y.data_ptr(), _ptr(acc), _stream(dev))
    return y, acc


# ----------------------------------------------------------------------------------
# optimizer step (clip -> AdamW -> clamp), optionally re-quantising W for the next step
# ----------------------------------------------------------------------------------

def bitlinear_optimizer_step(W: torch.Tensor, dW: torch.Tensor, m: torch.Tensor, v: torch.Tensor,
                             step: torch.Tensor, lr: float = 1e-3, betas=(0.9, 0.95), eps: float = 1e-6,
                             weight_decay: float = 0.01, max_norm: float = 1.0, requantize: bool = False,
                             ws: Optional[torch.Tensor] = None, out=None):
    """Updates W, m, v (fp32) and step (int32 [1]) in place.  With requantize, returns
    dict(gamma, wq_i8, wq_bf16, packed) of the updated W (keys from ``out`` are reused)."""
    for t, name in ((W, "W"), (dW, "dW"), (m, "m"), (v, "v")):
        _cuda(t, name, torch.float32)
    _cuda(step, "step", torch.int32)
    N, K = W.shape
    dev = W.device
    o = dict(out or {})
    if requantize:
        o.setdefault("gamma", torch.empty(1, dtype=torch.float32, device=dev))
        o.setdefault("wq_i8", torch.empty(N, K, dtype=torch.int8, device=dev))
        o.setdefault("wq_bf16", torch.empty(N, K, dtype=torch.bfloat16, device=dev))
        o.setdefault("packed", torch.empty(N, K // 4, dtype=torch.uint8, device=dev))
    if ws is None:
        ws = workspace(1, N, K, dev)
    _lib.call("bitlinear_optimizer_step", W.data_ptr(), dW.data_ptr(), m.data_ptr(), v.data_ptr(), N, K,
              float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay), float(max_norm),
              step.data_ptr(), _ptr(o.get("wq_i8")), _ptr(o.get("wq_bf16")), _ptr(o.get("packed")),
              _ptr(o.get("gamma")), ws.data_ptr(), ws.numel(), _stream(dev))
    return o


def check_device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    dev = device if device is not None else torch.cuda.current_device()
    return int(_lib.lib().bl_check_device_status(_stream(dev)))


def set_wait_limit_ns(ns: int) -> None:
    _lib.lib().bl_set_wait_limit_ns(int(ns))


def launch_count() -> int:
    return int(_lib.lib().bl_launch_count())


def selftest_bounded_wait(limit_ns: int, device=None) -> None:
    dev = device if device is not None else torch.cuda.current_device()
    _lib.call("bl_selftest_bounded_wait", int(limit_ns), _stream(dev))


def read_peak_probe(buf: torch.Tensor, pattern: str = "gemv", sink: Optional[torch.Tensor] = None) -> int:
    """Launch the read-bandwidth probe on buf (uint8 [rows x row_bytes], rows a multiple of 16,
    row_bytes of 64) on the current stream; returns the bytes the launch reads.  Time it with
    CUDA events for the rate."""
    _cuda(buf, "buf", torch.uint8)
    rows, row_bytes = buf.shape
    if sink is None:
        sink = torch.zeros(4, dtype=torch.int32, device=buf.device)
    _lib.call("bl_read_peak_probe", buf.data_ptr(), rows, row_bytes, {"gemv": 0, "coalesced": 1}[pattern],
              sink.data_ptr(), _stream(buf.device))
    return rows * row_bytes


def mma_peak_probe(kind: str = "int8", pair: bool = True, iters: int = 20000, device=None) -> float:
    """Launch the tensor-pipe peak probe on the current stream (tcgen05.mma from fixed
    shared-memory operands, no global traffic).  Returns 2 x the multiply-adds of the
    launch; time the launch with CUDA events for the rate."""
    import ctypes
    dev = device if device is not None else torch.cuda.current_device()
    ops = ctypes.c_double(0.0)
    _lib.call("bl_mma_peak_probe", {"int8": 0, "bf16": 1, "imma_sync": 2}[kind], 1 if pair else 0, int(iters),
              ctypes.byref(ops), _stream(dev))
    return float(ops.value)
