"""Seeded random shapes for the int8 x packed-ternary linear.

Tokens 1-300, K a multiple of 64 up to 4096, N a multiple of 16 up to 40000 (log-uniform), so
that the launches cover both kernels (the decode GEMV up to 16 tokens, CTA pairs above), one
to several work units per CTA pair, short and long units, ragged row / token / K tiles, and
the K split when a workspace is given.  Every output of every shape is compared bit for bit
with the linear on the int8 codes of the same weight (itself checked against the oracle by the
parity tests), and 128 weight rows of every shape (the first 32, the last 64 and 32 drawn at
random) with the oracle's contraction and epilogue.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import np_

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _shapes(n=24, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        lo, hi = ((1, 17), (17, 65), (65, 301))[i % 3]
        T = int(rng.integers(lo, hi))
        K = 64 * int(rng.integers(1, 65))
        N = 16 * max(1, int(round(np.exp(rng.uniform(0.0, np.log(2500.0))))))
        out.append((T, K, N))
    return out


# and more weight tiles than CTA pairs with short units (one to three stages of two k-blocks)
_MULTI_UNIT = [(100, 320, 30000), (250, 192, 25008), (20, 128, 45008), (150, 704, 40000)]


@pytest.mark.parametrize("T,K,N", _shapes() + _MULTI_UNIT)
def test_linear_packed_random_shapes(bl, T, K, N):
    rng = np.random.default_rng(T * 1000003 + K * 1009 + N)
    xq = rng.integers(-128, 128, size=(T, K)).astype(np.int8)
    wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    packed = oracle.pack(wq)
    s = rng.uniform(5, 300, size=T).astype(np.float32)
    gamma = 0.0173
    xq_d, s_d, g_d = torch.from_numpy(xq).to(DEV), torch.from_numpy(s).to(DEV), torch.tensor([gamma], device=DEV)
    y8, acc8 = bl.bitlinear_linear(xq_d, s_d, torch.from_numpy(wq).to(DEV), g_d, want_acc=True)
    p_d = torch.from_numpy(packed).to(DEV)
    ws = torch.empty(8 * T * N * 4, dtype=torch.uint8, device=DEV)
    for w in (None, ws):
        yp, accp = bl.bitlinear_linear_packed(xq_d, s_d, p_d, g_d, K, want_acc=True, ws=w)
        torch.cuda.synchronize()
        assert bl.check_device_status() == 0
        assert torch.equal(accp, acc8), (T, K, N, w is not None)
        assert torch.equal(yp.view(torch.int16), y8.view(torch.int16)), (T, K, N, w is not None)
    rows = np.unique(np.r_[0:min(32, N), max(0, N - 64):N, rng.integers(0, N, size=32)])
    acc_o = oracle.int_gemm(xq, oracle.unpack(packed[rows], K))
    assert np.array_equal(np_(acc8)[:, rows], acc_o)
    assert np.array_equal(np_(y8)[:, rows], oracle.round_bf16(oracle.linear_epilogue(acc_o, gamma, s)))
