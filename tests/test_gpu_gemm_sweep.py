"""Seeded random shapes for the layer's three GEMMs: the int8 x ternary linear, the grad-input
GEMM dX_hat = gamma dY . W_q and the weight-gradient GEMM dW = dY^T . X_dq (both bf16).

Tokens 1-6000 and N 16-16000 (log-uniform), K a multiple of 32 up to 8192, so that the 2-SM
GEMMs see one tile to several waves of pair tiles, ragged rows, columns and K, split tails and
short contractions.  The linear's int32 sums and outputs are compared exactly with the oracle
on sampled token rows (every column); the backward GEMMs on sampled rows of dX_hat and dW with
the oracle's fp64-accumulated contraction, within the bf16 tolerance of the parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import TOL, max_rel_err, np_

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _shapes(n=18, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        T = max(1, int(round(np.exp(rng.uniform(0.0, np.log(6000.0))))))
        K = 32 * int(rng.integers(1, 257))
        N = 16 * max(1, int(round(np.exp(rng.uniform(0.0, np.log(1000.0))))))
        if T * N * K <= 4e10:
            out.append((T, K, N))
    return out


# and several waves of pair tiles in each GEMM
_WAVES = [(3000, 1024, 9008), (5000, 2048, 2064), (1500, 4000, 5008), (6000, 512, 3008)]


@pytest.mark.parametrize("T,K,N", _shapes() + _WAVES)
def test_gemms_random_shapes(bl, T, K, N):
    rng = np.random.default_rng(T * 7919 + K * 31 + N)
    xq = rng.integers(-127, 128, size=(T, K)).astype(np.int8)
    wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s = rng.uniform(10, 200, size=T).astype(np.float32)
    gamma = np.float32(0.0173)
    g_d = torch.tensor([gamma], device=DEV)
    xq_d, s_d, wq_d = (torch.from_numpy(a).to(DEV) for a in (xq, s, wq))
    y, acc = bl.bitlinear_linear(xq_d, s_d, wq_d, g_d, want_acc=True)

    dY = torch.from_numpy(rng.standard_normal((T, N)).astype(np.float32) * 1e-2).to(torch.bfloat16)
    xdq = (torch.from_numpy(xq).float() / torch.from_numpy(s)[:, None]).to(torch.bfloat16)
    dY_d, xdq_d = dY.to(DEV), xdq.to(DEV)
    dXh = bl.bitlinear_grad_input(dY_d, wq_d.to(torch.bfloat16), g_d)
    dW = bl.bitlinear_backward_weight(dY_d, xdq_d)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0

    trows = np.unique(np.r_[0, T - 1, rng.integers(0, T, size=4)])
    acc_o = oracle.int_gemm(xq, wq, rows=trows)
    assert np.array_equal(np_(acc)[trows], acc_o)
    assert np.array_equal(np_(y)[trows], oracle.round_bf16(oracle.linear_epilogue(acc_o, gamma, s[trows])))

    dY32 = dY.float().numpy()
    dxh_o = oracle.grad_input_hat(dY32, wq, float(gamma), rows=trows)
    assert max_rel_err(np_(dXh)[trows], dxh_o) <= TOL["bf16"]
    wrows = np.unique(np.r_[0, N - 1, rng.integers(0, N, size=4)])
    dw_o = oracle.grad_weight(dY32, xdq.float().numpy(), wrows=wrows)
    assert max_rel_err(np_(dW)[wrows], dw_o) <= TOL["bf16"]
