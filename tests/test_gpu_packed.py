"""GPU parity of the int8 x packed-ternary linear (few tokens) against the oracle, on both of
its kernels: the decode GEMV's (up to 16 tokens) and the 2-SM tile on CTA pairs (17 tokens or
more, and up to 16 tokens whose activation rows do not fit the GEMV's shared memory, such as
16 x 65536; 256 weight rows x up to 256 tokens, ragged in rows, tokens and K).

The accumulators are exact int32 and compared bit for bit with the oracle's contraction of
the unpacked codes (reserved code 11 decodes to 0); Y = fl(acc * fl(gamma / s_t)) is
compared bit for bit with the oracle's epilogue (rounded to bf16 for a bf16 output), with
and without the K split (whose int32 partial sums are added in any order, exactly).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_ternary_qat_b200 import synth
from parity_util import np_, sample_rows

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gpu(a):
    if isinstance(a, np.ndarray):
        a = torch.from_numpy(a)
    return a.to(DEV).contiguous()


def _case(T, K, N, seed, raw_bytes=False):
    rng = np.random.default_rng(seed)
    xq = rng.integers(-128, 128, size=(T, K)).astype(np.int8)
    if raw_bytes:
        packed = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)     # includes reserved 11 codes
    else:
        packed = oracle.pack(rng.integers(-1, 2, size=(N, K)).astype(np.int8))
    s = rng.uniform(5, 300, size=T).astype(np.float32)
    return xq, packed, s


def _check(bl, xq, packed, s, gamma, out, split):
    T, K = xq.shape
    N = packed.shape[0]
    ws = torch.empty(8 * T * N * 4, dtype=torch.uint8, device=DEV) if split else None
    y, acc = bl.bitlinear_linear_packed(_gpu(xq), _gpu(s), _gpu(packed), _gpu(torch.tensor([gamma])), K,
                                        out_dtype=torch.bfloat16 if out == "bf16" else torch.float32,
                                        want_acc=True, ws=ws)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    wq = oracle.unpack(packed, K)
    rows = None if T * N * K <= 2 ** 31 else sample_rows(T, 6, seed=T)
    acc_o = oracle.int_gemm(xq, wq, rows=rows)
    acc_g = np_(acc) if rows is None else np_(acc)[rows]
    assert np.array_equal(acc_g, acc_o)
    y_o = oracle.linear_epilogue(acc_o, gamma, s if rows is None else s[rows])
    y_g = np_(y) if rows is None else np_(y)[rows]
    assert np.array_equal(y_g, oracle.round_bf16(y_o) if out == "bf16" else y_o)
    return y, acc


@pytest.mark.parametrize("T,K,N", [(1, 64, 16), (7, 4096, 11008), (16, 8192, 28672), (64, 2048, 2048),
                                   (129, 1024, 400), (300, 512, 1040), (33, 192, 2064), (8, 2048, 400),
                                   (3, 1024, 272), (32, 4096, 2048), (20, 1024, 400), (16, 65536, 64),
                                   (17, 1024, 272), (96, 640, 512), (200, 1088, 1008), (257, 512, 608),
                                   (40, 256, 40000), (64, 4096, 11008), (256, 4096, 11008),
                                   (256, 4096, 4096), (192, 4096, 4096), (100, 2048, 1024)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("split", [False, True])
def test_linear_packed_parity(bl, T, K, N, out, split):
    xq, packed, s = _case(T, K, N, seed=T + K + N)
    _check(bl, xq, packed, s, 0.0173, out, split)


def test_linear_packed_reserved_codes_decode_to_zero(bl):
    xq, packed, s = _case(24, 512, 272, seed=5, raw_bytes=True)
    assert np.any(((packed[:, :, None] >> np.array([0, 2, 4, 6])) & 3) == 3)
    _check(bl, xq, packed, s, 0.02, "f32", False)
    _check(bl, xq, packed, s, 0.02, "bf16", True)


def test_linear_packed_matches_int8_linear(bl):
    """Same layer through the quantisers: the packed path gives the int8 path's Y bit for bit."""
    li = synth.random_case(48, 4096, 4096, seed=17, dtype="bf16")
    qw = bl.bitlinear_quant_weight(_gpu(li.W))
    aq = bl.bitlinear_act_quant(_gpu(li.X))
    y8, acc8 = bl.bitlinear_linear(aq["xq"], aq["sx"], qw["wq_i8"], qw["gamma"], want_acc=True)
    yp, accp = bl.bitlinear_linear_packed(aq["xq"], aq["sx"], qw["packed"], qw["gamma"], 4096, want_acc=True)
    torch.cuda.synchronize()
    assert torch.equal(acc8, accp)
    assert torch.equal(y8.view(torch.int16), yp.view(torch.int16))


@pytest.mark.parametrize("T,K,N", [(17, 1024, 272), (64, 4096, 11008), (100, 640, 4112), (256, 512, 1040),
                                   (40, 256, 40000)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_linear_packed_without_accumulators(bl, T, K, N, out):
    """Y alone (no int32 copy requested): the CTA-pair epilogue stages bf16 output in four 2 KB
    tiles per warp instead of two 4 KB ones; Y must equal the path with the copy bit for bit."""
    xq, packed, s = _case(T, K, N, seed=3 * T + K)
    args = (_gpu(xq), _gpu(s), _gpu(packed), _gpu(torch.tensor([0.0173])), K)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    y_only, none = bl.bitlinear_linear_packed(*args, out_dtype=dt)
    assert none is None
    y, acc = bl.bitlinear_linear_packed(*args, out_dtype=dt, want_acc=True)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    assert torch.equal(y_only.view(torch.int16 if out == "bf16" else torch.int32),
                       y.view(torch.int16 if out == "bf16" else torch.int32))
    rows = sample_rows(T, 6, seed=T)
    acc_o = oracle.int_gemm(xq, oracle.unpack(packed, K), rows=rows)
    y_o = oracle.linear_epilogue(acc_o, 0.0173, s[rows])
    assert np.array_equal(np_(y_only)[rows], oracle.round_bf16(y_o) if out == "bf16" else y_o)


@pytest.mark.parametrize("T,K,N", [(256, 512, 20480), (200, 1024, 40000), (64, 256, 40000)])
def test_linear_packed_short_last_units(bl, T, K, N):
    """More weight tiles than CTA pairs, with short units (one, two or four stages of two
    k-blocks): a pair's decoder warps finish decoding its last unit while an earlier unit's
    accumulators are still open, and then take part in the last unit's epilogue.  One 256-column
    accumulator (200 and 256 tokens) or two (64 tokens).  Every token is checked on the first
    weight tile and on the last 4096 rows, which hold the pairs' second and third units."""
    xq, packed, s = _case(T, K, N, seed=T + K + N)
    gamma = 0.0173
    y, acc = bl.bitlinear_linear_packed(_gpu(xq), _gpu(s), _gpu(packed), _gpu(torch.tensor([gamma])), K,
                                        want_acc=True)
    torch.cuda.synchronize()
    assert bl.check_device_status() == 0
    sel = np.r_[0:256, N - 4096:N]
    acc_o = oracle.int_gemm(xq, oracle.unpack(packed[sel], K))
    assert np.array_equal(np_(acc)[:, sel], acc_o)
    assert np.array_equal(np_(y)[:, sel], oracle.round_bf16(oracle.linear_epilogue(acc_o, gamma, s)))


def test_linear_packed_split_with_single_k_block_stages(bl):
    """K = 5440 (42.5 k-blocks) at 20 tokens on 512 rows: two pair tiles, so K is split -- five
    ways by the launcher's rule (8 / 9 / 8 / 9 / 9 k-blocks); the splits of 9 k-blocks end in a
    one-k-block stage, the last of them on the half k-block of the K tail."""
    xq, packed, s = _case(20, 5440, 512, seed=11)
    for out in ("bf16", "f32"):
        _check(bl, xq, packed, s, 0.0173, out, True)
        _check(bl, xq, packed, s, 0.0173, out, False)
