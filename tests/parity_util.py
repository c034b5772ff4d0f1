"""Comparison helpers shared by the GPU parity tests (no layer arithmetic here)."""
import numpy as np
import torch

# Tolerances of the float outputs (max relative error = max|gpu - oracle| / max|oracle|
# over the whole tensor): 2e-3 where the layer runs in bf16, 1e-4 where it runs in fp32.
TOL = {"bf16": 2e-3, "f32": 1e-4}


def np_(t):
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()
    return np.asarray(t)


def f32_of(t):
    """fp32 values of a tensor (bf16 is widened exactly)."""
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().float().numpy()
    return np.asarray(t, dtype=np.float32)


def ulp_diff(a, b):
    """|a - b| in units of fp32 ulps (a, b same-sign finite fp32 arrays)."""
    ai = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


def max_rel_err(gpu, ora):
    gpu = np.asarray(gpu, dtype=np.float64)
    ora = np.asarray(ora, dtype=np.float64)
    den = np.max(np.abs(ora))
    if den == 0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(gpu - ora)) / den)


def sample_rows(n, k=24, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, n - 1, n // 2}
    rows.update(rng.integers(0, n, size=k).tolist())
    return sorted(r for r in rows if 0 <= r < n)
