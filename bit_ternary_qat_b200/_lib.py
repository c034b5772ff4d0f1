"""ctypes loader of libbitlinear.so (the C ABI declared in include/bitlinear.h).

Loads the in-tree library built by ``bit_ternary_qat_b200.build``.  There is no
fallback: if the library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

BL_OK = 0
STATUS_NAMES = {
    0: "BL_OK", 1: "BL_ERR_INVALID_ARG", 2: "BL_ERR_UNSUPPORTED_SHAPE", 3: "BL_ERR_MISALIGNED",
    4: "BL_ERR_WORKSPACE", 5: "BL_ERR_CUDA", 6: "BL_ERR_TIMEOUT", 7: "BL_ERR_DEVICE",
}
BL_F32 = 0
BL_BF16 = 1

# Every symbol the header declares, with its ctypes signature.
P = ctypes.c_void_p
I64 = ctypes.c_int64
U64 = ctypes.c_uint64
F = ctypes.c_float
INT = ctypes.c_int
SZ = ctypes.c_size_t
SIGNATURES = {
    "bl_abi_version": (INT, []),
    "bl_last_error": (ctypes.c_char_p, []),
    "bitlinear_workspace_bytes": (SZ, [I64, I64, I64]),
    "bl_check_device_status": (INT, [P]),
    "bl_set_wait_limit_ns": (None, [U64]),
    "bl_launch_count": (U64, []),
    "bitlinear_quant_weight": (INT, [P, I64, I64, P, P, P, P, P, SZ, P]),
    "bitlinear_quant_weight_noalloc": (INT, [P, I64, I64, P, P, P, P, P]),
    "bitlinear_act_quant": (INT, [P, INT, I64, I64, INT, P, F, P, P, P, P, P]),
    "bitlinear_linear": (INT, [P, P, I64, I64, P, P, I64, P, INT, P, P]),
    "bitlinear_forward": (INT, [P, INT, I64, I64, P, F, P, P, I64, P, P, P, P, P, P, P]),
    "bitlinear_forward_qat": (INT, [P, INT, I64, I64, P, F, P, I64, P, P, P, P, P, P, P, P, P, P, P, SZ, P]),
    "bitlinear_backward_input": (INT, [P, P, INT, I64, I64, I64, P, P, P, P, P, P, P, SZ, P]),
    "bitlinear_backward_weight": (INT, [P, P, INT, I64, I64, I64, P, P]),
    "bitlinear_grad_input": (INT, [P, INT, I64, I64, I64, P, P, P, P]),
    "bitlinear_rmsnorm_backward": (INT, [P, INT, I64, I64, P, P, P, P, P, SZ, P]),
    "bitlinear_backward": (INT, [P, P, P, INT, I64, I64, I64, P, P, P, P, P, P, P, P, SZ, P]),
    "ternary_pack": (INT, [P, I64, I64, P, P]),
    "ternary_gemv": (INT, [P, P, I64, I64, P, P, I64, P, P, P]),
    "bl_selftest_bounded_wait": (INT, [U64, P]),
    "bl_mma_peak_probe": (INT, [INT, INT, INT, P, P]),
    "bl_read_peak_probe": (INT, [P, I64, I64, INT, P, P]),
    "bitlinear_quant_weight_rows": (INT, [P, I64, I64, P, P, P, P, P]),
    "bitlinear_quant_weight_tau": (INT, [P, I64, I64, F, P, P, P, P, P, SZ, P]),
    "bitlinear_act_quant_tensor": (INT, [P, INT, I64, I64, INT, P, F, P, P, P, P, P, SZ, P]),
    "bitlinear_linear_rows": (INT, [P, P, I64, I64, P, P, I64, P, INT, P, P]),
    "ternary_gemv_rows": (INT, [P, P, I64, I64, P, P, I64, P, P, P]),
    "bitlinear_linear_packed": (INT, [P, P, I64, I64, P, P, I64, P, INT, P, P, SZ, P]),
    "bitlinear_optimizer_step": (INT, [P, P, P, P, I64, I64, F, F, F, F, F, F, P, P, P, P, P, P, SZ, P]),
}


class BitLinearError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load (once) and return the ctypes handle; raises if the library is not built."""
    global _lib
    with _lock:
        if _lib is None:
            path = lib_path()
            if not os.path.exists(path):
                raise ImportError(
                    f"{path} is not built; run `python -m bit_ternary_qat_b200.build` "
                    "(nvcc, sm_100a). There is no CPU fallback.")
            L = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def call(name: str, *args) -> None:
    """Call an entry point that returns bl_status; raise BitLinearError unless BL_OK."""
    L = lib()
    st = getattr(L, name)(*args)
    if st != BL_OK:
        raise BitLinearError(name, st, L.bl_last_error().decode(errors="replace"))


def status(name: str, *args) -> int:
    """Call an entry point and return its raw bl_status (tests of validation paths)."""
    return int(getattr(lib(), name)(*args))


def last_error() -> str:
    return lib().bl_last_error().decode(errors="replace")
