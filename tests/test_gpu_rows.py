"""GPU parity of the two per-token row kernels at every block-size family they choose from
the row length, up to the maximum d_in of 16384: the RMSNorm backward (persistent rows,
128 / 256 / 512 / 1024 threads, one or two row buffers) and the activation quantiser
(warp-per-row and block-per-row kernels).

The RMSNorm backward gets dX_hat directly (random fp32) and the forward's r.  Its output dX
and the gain gradient dg are checked against the oracle's textbook derivative (fp64
accumulation) within the fp32 tolerance, for bf16 and fp32 X, with and without a gain.
The quantiser's codes, scales and X_dq are compared bit for bit with the oracle (given the
GPU's r, which must be within 1 ulp of the oracle's).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_ternary_qat_b200 import synth
from parity_util import TOL, max_rel_err, np_, ulp_diff

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# K per launch family: bf16 rows of 16-byte vectors of 4 fp32 dX columns each; the launcher
# picks the smallest block of 128 / 256 / 512 / 1024 threads with at most four vectors per thread
ROW_K = [32, 2080, 4096, 8192, 11008, 12288, 16384]


@pytest.mark.parametrize("K", ROW_K)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("gain", [False, True])
def test_rmsnorm_backward_every_block_size(bl, K, dtype, gain):
    T = 37 if K >= 8192 else 301          # rows stride over the persistent grid unevenly
    li = synth.random_case(T, K, 16, seed=K + T, dtype=dtype, with_gain=gain)
    X = li.X.to(DEV)
    g = None if li.g is None else li.g.to(DEV)
    a = bl.bitlinear_act_quant(X, g=g, want_xdq=False)
    dxh = torch.randn(T, K, generator=synth.generator(K + 1)) * 1e-2
    dX, dg = bl.bitlinear_rmsnorm_backward(X, a["rinv"], dxh.to(DEV).contiguous(), g=g)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    r = np_(a["rinv"])
    assert ulp_diff(r, oracle.rmsnorm_rinv(li.X, 1e-6)).max() <= 1
    dX_o, dg_o = oracle.rmsnorm_backward(li.X, r, li.g, dxh.numpy())
    assert max_rel_err(np_(dX), dX_o) <= TOL["f32"]
    assert max_rel_err(np_(dg), dg_o) <= TOL["f32"]


def test_rmsnorm_backward_single_row_and_dg_absent(bl):
    """T = 1 (a grid of one block) and a call without dg (no partial rows written)."""
    li = synth.random_case(1, 11008, 16, seed=5, dtype="bf16")
    X = li.X.to(DEV)
    a = bl.bitlinear_act_quant(X, want_xdq=False)
    dxh = torch.randn(1, 11008, generator=synth.generator(6))
    dX = dxh.to(DEV).contiguous()
    bl.bitlinear_rmsnorm_backward(X, a["rinv"], dX, want_dg=False)
    torch.cuda.synchronize()
    dX_o, _ = oracle.rmsnorm_backward(li.X, np_(a["rinv"]), None, dxh.numpy(), want_dg=False)
    assert max_rel_err(np_(dX), dX_o) <= TOL["f32"]


@pytest.mark.parametrize("K", [8192, 12288, 16384])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("gain", [False, True])
def test_act_quant_longest_rows(bl, K, dtype, gain):
    li = synth.random_case(19, K, 16, seed=K, dtype=dtype, with_gain=gain)
    o = bl.bitlinear_act_quant(li.X.to(DEV), g=None if li.g is None else li.g.to(DEV))
    torch.cuda.synchronize()
    r = np_(o["rinv"])
    assert ulp_diff(r, oracle.rmsnorm_rinv(li.X, 1e-6)).max() <= 1
    xq, s, xdq = oracle.act_quant(li.X, r, li.g)
    assert np.array_equal(np_(o["sx"]), s)
    assert np.array_equal(np_(o["xq"]), xq)
    want = oracle.round_bf16(xdq) if dtype == "bf16" else xdq
    assert np.array_equal(np_(o["xdq"]), want)
