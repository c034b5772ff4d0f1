"""CPU oracle of the BitLinear hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may import this package.  The product (``bit_ternary_qat_b200``) never
imports it and shares no code with it.

The arithmetic lives in ``bitlinear_oracle.c`` (plain C, fp32 with
round-half-to-even, fp64 reductions); this module only builds it with gcc and
marshals numpy / torch arrays into it.  Every function documents the page section
it restates in the C source.

Functions with no independent pin would be listed here as "parity unpinned";
every function below is pinned: the layer's steps by ``tests/test_oracle_pins.py``, the
quantiser variants by ``tests/test_oracle_variants.py`` and the optimizer step by
``tests/test_oracle_optimizer.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-frounding-math", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/liboracle.so (idempotent)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int64
            F = ctypes.c_float
            L.ora_num_threads.restype = ctypes.c_int
            L.ora_round_bf16.argtypes = [P, I, P]
            L.ora_bf16_to_f32.argtypes = [P, I, P]
            L.ora_rmsnorm_rinv.argtypes = [P, I, I, F, P]
            L.ora_act_quant.argtypes = [P, I, I, P, P, P, P, P]
            L.ora_absmean_gamma.argtypes = [P, I]
            L.ora_absmean_gamma.restype = F
            L.ora_ternary_round.argtypes = [P, I, F, P]
            L.ora_pack.argtypes = [P, I, I, P]
            L.ora_unpack.argtypes = [P, I, I, P]
            L.ora_int_gemm.argtypes = [P, P, I, I, I, P, I, P]
            L.ora_linear_epilogue.argtypes = [P, I, I, F, P, P]
            L.ora_grad_input_hat.argtypes = [P, P, F, I, I, I, P, I, P]
            L.ora_grad_weight.argtypes = [P, P, I, I, I, P, I, P]
            L.ora_rmsnorm_backward.argtypes = [P, P, P, P, I, I, P, I, P, P]
            L.ora_gemv.argtypes = [P, F, I, I, P, P, I, P, P]
            L.ora_absmean_gamma_rows.argtypes = [P, I, I, P]
            L.ora_ternary_round_rows.argtypes = [P, I, I, P, P]
            L.ora_ternary_tau.argtypes = [P, I, F, F, P]
            L.ora_act_quant_tensor.argtypes = [P, I, I, P, P, P, P, P]
            L.ora_linear_epilogue_rows.argtypes = [P, I, I, P, P, P]
            D = ctypes.c_double
            L.ora_optimizer_step.argtypes = [P, P, P, P, I, D, D, D, D, D, D, I]
            L.ora_optimizer_step.restype = D
            _lib = L
    return _lib


# ----------------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------------

def _f32(a) -> np.ndarray:
    """Exact conversion to a contiguous float32 numpy array (bf16 -> f32 is exact)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu()
            if a.dtype != torch.float32:
                a = a.to(torch.float32)
            return np.ascontiguousarray(a.numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _arr(a, dtype) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows: Optional[Sequence[int]]):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, int(r.size)


def num_threads() -> int:
    return int(lib().ora_num_threads())


# ----------------------------------------------------------------------------------
# the path, step by step
# ----------------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """fp32 -> bf16 (round-to-nearest-even) as uint16 bit patterns."""
    x = _f32(x)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().ora_round_bf16(_p(x), x.size, _p(out))
    return out


def bf16_bits_to_f32(h) -> np.ndarray:
    h = _arr(h, np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    lib().ora_bf16_to_f32(_p(h), h.size, _p(out))
    return out


def rmsnorm_rinv(X, eps: float) -> np.ndarray:
    X = _f32(X)
    T, K = X.shape
    r = np.empty(T, dtype=np.float32)
    lib().ora_rmsnorm_rinv(_p(X), T, K, eps, _p(r))
    return r


def act_quant(X, rinv=None, g=None):
    """Returns (x_q int8 [T,K], s fp32 [T], x_dq fp32 [T,K])."""
    X = _f32(X)
    T, K = X.shape
    r = None if rinv is None else _f32(rinv)
    gg = None if g is None else _f32(g)
    xq = np.empty((T, K), dtype=np.int8)
    s = np.empty(T, dtype=np.float32)
    xdq = np.empty((T, K), dtype=np.float32)
    lib().ora_act_quant(_p(X), T, K, _p(r), _p(gg), _p(xq), _p(s), _p(xdq))
    return xq, s, xdq


def absmean_gamma(W) -> float:
    W = _f32(W)
    return float(lib().ora_absmean_gamma(_p(W), W.size))


def ternary_round(W, gamma: float) -> np.ndarray:
    W = _f32(W)
    out = np.empty(W.shape, dtype=np.int8)
    lib().ora_ternary_round(_p(W), W.size, float(gamma), _p(out))
    return out


def quant_weight(W):
    """(gamma, W_q int8)."""
    gamma = absmean_gamma(W)
    return gamma, ternary_round(W, gamma)


def pack(wq) -> np.ndarray:
    wq = _arr(wq, np.int8)
    N, K = wq.shape
    out = np.empty((N, K // 4), dtype=np.uint8)
    lib().ora_pack(_p(wq), N, K, _p(out))
    return out


def unpack(packed, K: int) -> np.ndarray:
    packed = _arr(packed, np.uint8)
    N = packed.shape[0]
    out = np.empty((N, K), dtype=np.int8)
    lib().ora_unpack(_p(packed), N, K, _p(out))
    return out


def int_gemm(xq, wq, rows=None) -> np.ndarray:
    xq = _arr(xq, np.int8)
    wq = _arr(wq, np.int8)
    T, K = xq.shape
    N = wq.shape[0]
    r, nr = _rows(rows)
    R = nr if r is not None else T
    acc = np.empty((R, N), dtype=np.int32)
    lib().ora_int_gemm(_p(xq), _p(wq), T, N, K, _p(r), nr, _p(acc))
    return acc


def linear_epilogue(acc, gamma: float, s_rows) -> np.ndarray:
    acc = _arr(acc, np.int32)
    s_rows = _f32(s_rows)
    R, N = acc.shape
    y = np.empty((R, N), dtype=np.float32)
    lib().ora_linear_epilogue(_p(acc), R, N, float(gamma), _p(s_rows), _p(y))
    return y


def grad_input_hat(dY, wq, gamma: float, rows=None) -> np.ndarray:
    dY = _f32(dY)
    wq = _arr(wq, np.int8)
    T, N = dY.shape
    K = wq.shape[1]
    r, nr = _rows(rows)
    R = nr if r is not None else T
    out = np.empty((R, K), dtype=np.float32)
    lib().ora_grad_input_hat(_p(dY), _p(wq), float(gamma), T, N, K, _p(r), nr, _p(out))
    return out


def grad_weight(dY, xdq, wrows=None) -> np.ndarray:
    dY = _f32(dY)
    xdq = _f32(xdq)
    T, N = dY.shape
    K = xdq.shape[1]
    r, nr = _rows(wrows)
    R = nr if r is not None else N
    out = np.empty((R, K), dtype=np.float32)
    lib().ora_grad_weight(_p(dY), _p(xdq), T, N, K, _p(r), nr, _p(out))
    return out


def rmsnorm_backward(X, rinv, g, dxhat_rows, rows=None, want_dg: bool = True):
    """dxhat_rows holds dX_hat for the selected rows (all rows when rows is None)."""
    X = _f32(X)
    rinv = _f32(rinv)
    gg = None if g is None else _f32(g)
    dh = _f32(dxhat_rows)
    T, K = X.shape
    r, nr = _rows(rows)
    R = nr if r is not None else T
    dX = np.empty((R, K), dtype=np.float32)
    dg = np.empty(K, dtype=np.float32) if want_dg else None
    lib().ora_rmsnorm_backward(_p(X), _p(rinv), _p(gg), _p(dh), T, K, _p(r), nr, _p(dX), _p(dg))
    return dX, dg


def gemv(packed, gamma: float, K: int, xq, s):
    packed = _arr(packed, np.uint8)
    xq = _arr(xq, np.int8)
    s = _f32(s)
    N = packed.shape[0]
    B = xq.shape[0]
    acc = np.empty((B, N), dtype=np.int32)
    y = np.empty((B, N), dtype=np.float32)
    lib().ora_gemv(_p(packed), float(gamma), N, K, _p(xq), _p(s), B, _p(acc), _p(y))
    return acc, y


# ----------------------------------------------------------------------------------
# page variants of the quantisers (P4 §9 per-row scale, P2 tau = 0.7 scale, P5 §5.1
# per-tensor activation scale)
# ----------------------------------------------------------------------------------

def absmean_gamma_rows(W) -> np.ndarray:
    """gamma_n = max(mean_k |W[n, k]|, 1e-5), fp64 sum per row."""
    W = _f32(W)
    N, K = W.shape
    g = np.empty(N, dtype=np.float32)
    lib().ora_absmean_gamma_rows(_p(W), N, K, _p(g))
    return g


def ternary_round_rows(W, gamma_rows) -> np.ndarray:
    W = _f32(W)
    N, K = W.shape
    g = _f32(gamma_rows)
    out = np.empty((N, K), dtype=np.int8)
    lib().ora_ternary_round_rows(_p(W), N, K, _p(g), _p(out))
    return out


def quant_weight_rows(W):
    """(gamma_rows fp32 [N], W_q int8 [N, K])."""
    g = absmean_gamma_rows(W)
    return g, ternary_round_rows(W, g)


def ternary_tau(W, gamma: float, tau_factor: float) -> np.ndarray:
    """W_q = 0 where |W| < fl32(tau_factor * gamma), sign(W) elsewhere."""
    W = _f32(W)
    out = np.empty(W.shape, dtype=np.int8)
    lib().ora_ternary_tau(_p(W), W.size, float(gamma), float(tau_factor), _p(out))
    return out


def act_quant_tensor(X, rinv=None, g=None):
    """Per-tensor scale: (x_q int8 [T,K], s fp32 [T] (one value repeated), x_dq fp32 [T,K])."""
    X = _f32(X)
    T, K = X.shape
    r = None if rinv is None else _f32(rinv)
    gg = None if g is None else _f32(g)
    xq = np.empty((T, K), dtype=np.int8)
    s = np.empty(T, dtype=np.float32)
    xdq = np.empty((T, K), dtype=np.float32)
    lib().ora_act_quant_tensor(_p(X), T, K, _p(r), _p(gg), _p(xq), _p(s), _p(xdq))
    return xq, s, xdq


def linear_epilogue_rows(acc, gamma_rows, s_rows) -> np.ndarray:
    acc = _arr(acc, np.int32)
    g = _f32(gamma_rows)
    s_rows = _f32(s_rows)
    R, N = acc.shape
    y = np.empty((R, N), dtype=np.float32)
    lib().ora_linear_epilogue_rows(_p(acc), R, N, _p(g), _p(s_rows), _p(y))
    return y


# ----------------------------------------------------------------------------------
# optimizer step: clip -> AdamW -> clamp (returns new arrays; the inputs are untouched)
# ----------------------------------------------------------------------------------

def optimizer_step(W, dW, m, v, t: int, lr: float = 1e-3, betas=(0.9, 0.95), eps: float = 1e-6,
                   weight_decay: float = 0.01, max_norm: float = 1.0):
    """(W', m', v', c) after step t (1-based); c is the clip coefficient applied to dW."""
    W2 = _f32(W).copy()
    m2 = _f32(m).copy()
    v2 = _f32(v).copy()
    g = _f32(dW)
    assert W2.shape == g.shape == m2.shape == v2.shape
    c = lib().ora_optimizer_step(_p(W2), _p(g), _p(m2), _p(v2), W2.size, float(lr), float(betas[0]),
                                 float(betas[1]), float(eps), float(weight_decay), float(max_norm), int(t))
    return W2, m2, v2, float(c)


# ----------------------------------------------------------------------------------
# composite steps (forward / backward of one BitLinear), as the pages chain them
# ----------------------------------------------------------------------------------

def forward(X, W, g=None, eps: float = 1e-6, out_dtype: str = "f32", rinv=None, gamma=None):
    """One BitLinear forward (P3 §3.1): RMSNorm -> act quant -> weight quant -> linear.

    ``rinv`` / ``gamma`` may be given to re-run the quantisers conditional on another
    implementation's reduction results.  Returns a dict of every intermediate.
    y is fp32, or bf16 bits (uint16) when out_dtype == "bf16"; x_dq likewise.
    """
    if rinv is None:
        rinv = rmsnorm_rinv(X, eps)
    xq, s, xdq = act_quant(X, rinv, g)
    if gamma is None:
        gamma = absmean_gamma(W)
    wq = ternary_round(W, gamma)
    acc = int_gemm(xq, wq)
    y = linear_epilogue(acc, gamma, s)
    out = dict(rinv=_f32(rinv), xq=xq, s=s, xdq=xdq, gamma=float(gamma), wq=wq, acc=acc, y=y)
    if out_dtype == "bf16":
        out["y_bf16"] = round_bf16(y)
        out["xdq_bf16"] = round_bf16(xdq)
        out["xdq_saved"] = bf16_bits_to_f32(out["xdq_bf16"])
    else:
        out["xdq_saved"] = xdq
    return out


def backward(X, dY, fwd: dict, g=None):
    """STE backward of one BitLinear (P3 §3.2; P5 §3.2): returns (dX, dW, dg, dX_hat)."""
    dxhat = grad_input_hat(dY, fwd["wq"], fwd["gamma"])
    dW = grad_weight(dY, fwd["xdq_saved"])
    dX, dg = rmsnorm_backward(X, fwd["rinv"], g, dxhat)
    return dX, dW, dg, dxhat
