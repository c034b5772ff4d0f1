"""C-ABI checks that need no GPU: the library builds for sm_100a, exports every symbol
include/bitlinear.h declares, and rejects invalid calls on the host before launching
anything (so these calls never reach the device)."""
import ctypes
import os
import re
import subprocess

import pytest

from bit_ternary_qat_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^BL_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_header_declares_expected_entry_points():
    syms = header_symbols()
    for name in ["bitlinear_quant_weight", "bitlinear_forward", "bitlinear_backward", "ternary_pack",
                 "ternary_gemv", "bitlinear_act_quant", "bitlinear_linear", "bitlinear_backward_input",
                 "bitlinear_backward_weight", "bl_last_error", "bitlinear_workspace_bytes"]:
        assert name in syms, name


def test_library_exports_every_header_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [s for s in header_symbols() if s not in exported]
    assert not missing, missing
    # the binding knows every symbol too
    assert set(header_symbols()) == set(_lib.SIGNATURES)
    # and nothing else of ours leaks out of the library (hidden visibility)
    ours = {s for s in exported if s.startswith(("bl_", "bitlinear_", "ternary_"))}
    assert ours == set(header_symbols())


def test_abi_version_and_workspace(L):
    assert L.bl_abi_version() == 1
    assert L.bitlinear_workspace_bytes(4096, 2048, 2048) >= 296 * 2048 * 4
    assert L.bitlinear_workspace_bytes(1, 16, 32) % 256 == 0


FAKE = 1 << 20          # a 16-byte aligned fake device address: never dereferenced on the host
ODD = FAKE + 4          # misaligned


@pytest.mark.parametrize("args,expected", [
    # (W, N, K, Wq_i8, Wq_bf16, packed, gamma, ws, ws_bytes, stream)
    ((None, 16, 32, None, None, None, FAKE, FAKE, 1 << 20, None), 1),          # null W
    ((FAKE, 16, 32, None, None, None, None, FAKE, 1 << 20, None), 1),          # null gamma
    ((FAKE, 16, 48, None, None, None, FAKE, FAKE, 1 << 20, None), 2),          # K % 32
    ((FAKE, 24, 32, None, None, None, FAKE, FAKE, 1 << 20, None), 2),          # N % 16
    ((FAKE, 0, 32, None, None, None, FAKE, FAKE, 1 << 20, None), 1),           # N = 0
    ((ODD, 16, 32, None, None, None, FAKE, FAKE, 1 << 20, None), 3),           # misaligned
    ((FAKE, 16, 32, None, None, None, FAKE, FAKE, 8, None), 4),                # workspace too small
])
def test_quant_weight_validation(L, args, expected):
    assert _lib.status("bitlinear_quant_weight", *args) == expected
    assert len(_lib.last_error()) > 0


def test_forward_validation(L):
    ok = dict(X=FAKE, dt=1, T=8, K=64, g=None, eps=1e-6, wq=FAKE, gamma=FAKE, N=32, Y=FAKE, xq=FAKE, sx=FAKE,
              rinv=FAKE, xdq=None, acc=None, st=None)

    def call(**kw):
        a = dict(ok, **kw)
        return _lib.status("bitlinear_forward", *a.values())
    assert call(dt=7) == 1
    assert call(X=None) == 1
    assert call(rinv=None) == 1
    assert call(T=0) == 1
    assert call(K=40) == 2
    assert call(N=8) == 2
    assert call(Y=ODD) == 3
    assert call(eps=-1.0) == 1
    assert call(K=16384 + 32) == 2          # row kernels hold a row in registers


def test_backward_and_gemv_validation(L):
    # bitlinear_backward_input with dg requested but no workspace
    st = _lib.status("bitlinear_backward_input", FAKE, FAKE, 1, 8, 64, 32, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                     None, 0, None)
    assert st == 1
    st = _lib.status("bitlinear_backward_input", FAKE, FAKE, 1, 8, 64, 32, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                     FAKE, 16, None)
    assert st == 4
    # GEMV batch limits
    assert _lib.status("ternary_gemv", FAKE, FAKE, 32, 64, FAKE, FAKE, 0, FAKE, None, None) == 2
    assert _lib.status("ternary_gemv", FAKE, FAKE, 32, 64, FAKE, FAKE, 17, FAKE, None, None) == 2
    assert _lib.status("ternary_gemv", FAKE, FAKE, 32, 1 << 17, FAKE, FAKE, 1, FAKE, None, None) == 2
    assert _lib.status("ternary_pack", FAKE, 16, 33, FAKE, None) == 2
    assert _lib.status("ternary_gemv", FAKE, FAKE, 32, 96, FAKE, FAKE, 1, FAKE, None, None) == 2   # K % 64
    assert _lib.status("bl_selftest_bounded_wait", 0, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "lib_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.lib()


def test_variant_and_optimizer_validation(L):
    """Host-side rejections of the entry points beyond the step (nothing reaches a device)."""
    # per-row weight quantiser: (W, N, K, Wq_i8, Wq_bf16, packed, gamma_rows, stream)
    assert _lib.status("bitlinear_quant_weight_rows", None, 16, 32, None, None, None, FAKE, None) == 1
    assert _lib.status("bitlinear_quant_weight_rows", FAKE, 16, 32, None, None, None, None, None) == 1
    assert _lib.status("bitlinear_quant_weight_rows", FAKE, 16, 48, None, None, None, FAKE, None) == 2
    assert _lib.status("bitlinear_quant_weight_rows", FAKE, 16, 32, ODD, None, None, FAKE, None) == 3
    # zero threshold: (W, N, K, tau, Wq_i8, Wq_bf16, packed, gamma, ws, ws_bytes, stream)
    for bad in (-0.5, float("nan"), float("inf")):
        assert _lib.status("bitlinear_quant_weight_tau", FAKE, 16, 32, bad, None, None, None, FAKE, FAKE, 1 << 20,
                           None) == 1
    assert _lib.status("bitlinear_quant_weight_tau", FAKE, 16, 32, 0.7, None, None, None, FAKE, FAKE, 8, None) == 4
    # per-tensor activation scale: (X, dt, T, K, norm, g, eps, Xq, sx, rinv, Xdq, ws, ws_bytes, stream)
    assert _lib.status("bitlinear_act_quant_tensor", FAKE, 1, 8, 64, 1, None, 1e-6, FAKE, FAKE, None, None, FAKE,
                       1 << 20, None) == 1                                      # rinv needed with RMSNorm
    assert _lib.status("bitlinear_act_quant_tensor", FAKE, 1, 8, 64, 0, None, 1e-6, FAKE, FAKE, None, None, FAKE,
                       16, None) == 4                                           # block maxima do not fit
    assert _lib.status("bitlinear_act_quant_tensor", FAKE, 1, 8, 64, 0, None, 1e-6, FAKE, FAKE, None, None, None,
                       1 << 20, None) == 1
    assert L.bitlinear_workspace_bytes(8, 16, 64) >= 4 * 1184
    # per-row linear and GEMV
    assert _lib.status("bitlinear_linear_rows", FAKE, FAKE, 8, 64, FAKE, None, 32, FAKE, 1, None, None) == 1
    assert _lib.status("bitlinear_linear_rows", FAKE, FAKE, 8, 40, FAKE, FAKE, 32, FAKE, 1, None, None) == 2
    assert _lib.status("ternary_gemv_rows", FAKE, FAKE, 32, 64, FAKE, FAKE, 17, FAKE, None, None) == 2
    assert _lib.status("ternary_gemv_rows", FAKE, FAKE, 32, 96, FAKE, FAKE, 1, FAKE, None, None) == 2
    # packed-weight linear: (Xq, sx, T, K, packed, gamma, N, Y, y_dt, acc, ws, ws_bytes, stream)
    assert _lib.status("bitlinear_linear_packed", FAKE, FAKE, 8, 96, FAKE, FAKE, 32, FAKE, 1, None, None, 0,
                       None) == 2                                               # K % 64
    assert _lib.status("bitlinear_linear_packed", FAKE, FAKE, 8, 128, None, FAKE, 32, FAKE, 1, None, None, 0,
                       None) == 1
    assert _lib.status("bitlinear_linear_packed", FAKE, FAKE, 8, 128, FAKE, FAKE, 32, FAKE, 1, ODD, None, 0,
                       None) == 3
    # optimizer: (W, dW, m, v, N, K, lr, b1, b2, eps, wd, max_norm, step, Wq_i8, Wq_bf16, packed, gamma, ws,
    #             ws_bytes, stream)
    ok = [FAKE, FAKE, FAKE, FAKE, 16, 32, 1e-3, 0.9, 0.95, 1e-6, 0.01, 1.0, FAKE, None, None, None, None, FAKE,
          1 << 20, None]

    def opt(**kw):
        a = list(ok)
        names = ["W", "dW", "m", "v", "N", "K", "lr", "b1", "b2", "eps", "wd", "mn", "step", "wq", "wbf", "pk",
                 "gamma", "ws", "ws_bytes", "st"]
        for k, val in kw.items():
            a[names.index(k)] = val
        return _lib.status("bitlinear_optimizer_step", *a)
    assert opt(step=None) == 1
    assert opt(m=None) == 1
    assert opt(lr=-1.0) == 1
    assert opt(b1=1.0) == 1
    assert opt(eps=0.0) == 1
    assert opt(wd=float("nan")) == 1
    assert opt(wq=FAKE) == 1                       # next codes without gamma
    assert opt(ws_bytes=64) == 4
    assert opt(K=48) == 2
    assert opt(W=ODD) == 3
    assert L.bitlinear_workspace_bytes(1, 16, 32) >= 2 * 8 * 1184 + 16


def test_status_values_match_header():
    """The numeric bl_status values of the header, which differ from a plain
    OK / invalid / shape / CUDA / timeout list by the misalignment, workspace and device
    codes, are the ones the binding decodes."""
    text = open(HEADER).read()
    body = text[text.index("typedef enum {"):text.index("} bl_status;")]
    vals = {name: int(v) for name, v in re.findall(r"\b(BL_\w+)\s*=\s*(\d+)", body)}
    assert vals == {"BL_OK": 0, "BL_ERR_INVALID_ARG": 1, "BL_ERR_UNSUPPORTED_SHAPE": 2, "BL_ERR_MISALIGNED": 3,
                    "BL_ERR_WORKSPACE": 4, "BL_ERR_CUDA": 5, "BL_ERR_TIMEOUT": 6, "BL_ERR_DEVICE": 7}
    assert {v: k for k, v in vals.items()} == _lib.STATUS_NAMES


@pytest.mark.parametrize("rows,row_bytes,pattern,status", [(16, 64, 2, 1), (16, 64, -1, 1), (8, 64, 0, 2), (24, 64, 1, 2),
                                                         (16, 32, 0, 2), (16, 96, 0, 2), (0, 64, 0, 2),
                                                         (1 << 30, 1 << 14, 0, 2)])
def test_read_probe_validation(L, rows, row_bytes, pattern, status):
    """The read probe rejects a bad pattern or shape before touching the (fake, aligned) pointers."""
    fake = 1 << 20
    assert _lib.status("bl_read_peak_probe", fake, rows, row_bytes, pattern, fake, None) == status
    assert len(_lib.last_error()) > 0


def test_read_probe_null_and_misaligned(L):
    assert _lib.status("bl_read_peak_probe", None, 16, 64, 0, 1 << 20, None) == 1
    assert _lib.status("bl_read_peak_probe", 1 << 20, 16, 64, 0, None, None) == 1
    assert _lib.status("bl_read_peak_probe", (1 << 20) + 8, 16, 64, 0, 1 << 20, None) == 3


@pytest.mark.parametrize("kind,pair,iters", [(3, 0, 10), (-1, 0, 10), (0, 2, 10), (0, 0, 0), (1, 1, (1 << 20) + 1)])
def test_peak_probe_validation(L, kind, pair, iters):
    assert _lib.status("bl_mma_peak_probe", kind, pair, iters, None, None) == 1
    assert len(_lib.last_error()) > 0
