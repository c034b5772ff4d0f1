"""NEXT-3, a zero-skip / sparsity-aware GEMV, was evaluated and not built.

The source is page 5, "1.58-bit量化技术…", §4.1-§4.2: the reserved code 11 and a circuit that
skips zeros.  This test measures what skipping all-zero groups could save on the codes the
oracle produces from the synthetic weights (the normal weights of the 2048 x 2048 and 7B-layer
workloads, and the Student-t weights of the 7B MLP workload).

A GPU moves the packed codes from HBM in 32-byte sectors (128 codes).  Skipping saves HBM
bytes only for sectors that are entirely zero, and instructions only for groups that are.
The codes are independent draws, so a group of g codes is all zero with probability p0^g.
"""
import numpy as np

import oracle
from bit_ternary_qat_b200 import synth


def _zero_group_fractions(W: np.ndarray):
    _, wq = oracle.quant_weight(W)
    p0 = float((wq == 0).mean())
    packed = oracle.pack(wq)                      # code 00 = 0: an all-zero group packs to zero
    bytes4 = float((packed == 0).mean())                                   # 4 codes
    words16 = float((packed.view(np.uint32) == 0).mean())                  # 16 codes
    sectors128 = float((packed.reshape(-1, 32) == 0).all(axis=1).mean())   # 128 codes
    return p0, bytes4, words16, sectors128


def test_all_zero_groups_are_too_rare_to_skip():
    gen = synth.generator(5)
    for name, W in (("normal", synth.normal((2048, 4096), synth.W_STD, gen)),
                    ("student_t3", synth.student_t3((2048, 4096), synth.W_STD, gen))):
        p0, bytes4, words16, sectors128 = _zero_group_fractions(W.numpy())
        # a normal weight's codes are zero where |w| < gamma / 2 = sigma sqrt(2 / pi) / 2:
        # P(|Z| < 0.399) = 0.310
        if name == "normal":
            assert abs(p0 - 0.310) < 0.005, p0
        assert 0.2 < p0 < 0.5, (name, p0)
        # independent codes: all-zero groups at the binomial rate p0^g
        assert abs(bytes4 - p0 ** 4) < 0.003, (name, bytes4, p0 ** 4)
        assert words16 < 10 * p0 ** 16 + 1e-5, (name, words16)
        # not one 32-byte sector of 8.4 M codes is all zero: skipping saves no HBM bytes, and
        # a byte-granular skip would spare p0^4 of the decode work (0.9 % normal, 2.1 %
        # Student-t) at the cost of a branch per byte
        assert sectors128 == 0.0, (name, sectors128)
        assert bytes4 < 0.025
