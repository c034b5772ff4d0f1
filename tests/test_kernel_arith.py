"""Host-side checks of the exact-arithmetic shortcuts the CUDA kernels take.

The kernels avoid per-element divisions and float<->int conversions while reproducing
the oracle's fp32 results bit for bit.  These tests check the identities they rely on
with exact rational arithmetic (fractions) or exact fp32 emulation (numpy float32 ops
are IEEE round-to-nearest-even), independently of any GPU:

* act quant: fl(q / s) == fl(y1 + fl(q - s*y1) * c) with c = fl(1/s), y0 = fl(q*c),
  y1 = fl(y0 + fl(q - s*y0) * c) (one reciprocal per row, two FMA corrections), for
  every q in [-128, 127];
* the same two-correction quotient for fl(gamma_n / s_t) (per-column linear epilogue);
* act quant: round-half-to-even of v via fl(v + 1.5*2^23) for |v| <= 128;
* weight quant: the ternary code equals sign(w) * [|w| >= w*] with w* found by the
  32-wide window search around gamma/2;
* decode GEMV: sum_k dec(c_k) x_k == sum_j dp4a(lo_j, x_j) - dp4a(hi_j, x_j) with the
  interleaved activation words.
"""
import math
from fractions import Fraction

import numpy as np
import pytest


def rn32(x: Fraction) -> Fraction:
    """Round a rational to the nearest fp32 value, ties to even (normal range)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    scale = Fraction(2) ** (23 - e)
    m = round(a * scale)            # Python rounds half to even
    return sign * Fraction(m) / scale


def f32(x: Fraction) -> np.float32:
    return np.float32(float(x))


def test_markstein_quotient_is_correctly_rounded():
    rng = np.random.default_rng(0)
    # s = fl(127 / m) over a wide range of row absmax values m, plus the clamp value
    ms = np.concatenate([10.0 ** rng.uniform(-5, 4, size=150), [1e-5, 1.0, 2.0, 127.0, 1e4]])
    for m in ms:
        s = Fraction(np.float32(np.float32(127.0) / np.float32(max(np.float32(m), np.float32(1e-5)))).item())
        c = rn32(Fraction(1) / s)
        for qi in range(0, 129):
            for q in (Fraction(qi), Fraction(-qi)):
                if q < -128 or q > 127:
                    continue
                y0 = rn32(q * c)
                y1 = rn32(y0 + rn32(q - s * y0) * c)
                e1 = rn32(q - s * y1)
                assert q - s * y1 == e1         # y1 is faithful: the second residual is exact
                y = rn32(y1 + e1 * c)
                assert y == rn32(q / s), (float(q), float(s))


def test_markstein_weight_scale_quotient_is_correctly_rounded():
    """The per-column linear epilogue computes fl(gamma_n / s_t) the same way, with the
    weight scale as the numerator: gamma in [1e-5, 1e2] (the quantiser's floor upwards),
    s_t over the activation quantiser's whole range."""
    rng = np.random.default_rng(2)
    gammas = np.concatenate([10.0 ** rng.uniform(-5, 2, size=400), [1e-5, 0.02, 1.0, 100.0]])
    ms = np.concatenate([10.0 ** rng.uniform(-5, 4, size=400), [1e-5, 1e-5, 1.0, 1e4]])
    for gv, m in zip(gammas, ms):
        a = Fraction(np.float32(max(np.float32(gv), np.float32(1e-5))).item())
        s = Fraction(np.float32(np.float32(127.0) / np.float32(max(np.float32(m), np.float32(1e-5)))).item())
        c = rn32(Fraction(1) / s)
        y0 = rn32(a * c)
        y1 = rn32(y0 + rn32(a - s * y0) * c)
        e1 = rn32(a - s * y1)
        assert a - s * y1 == e1
        assert rn32(y1 + e1 * c) == rn32(a / s), (float(a), float(s))


def test_magic_constant_rounds_half_to_even():
    magic = np.float32(12582912.0)
    v = np.concatenate([np.arange(-128, 128.5, 0.5, dtype=np.float32),
                        np.random.default_rng(1).uniform(-128, 128, 200000).astype(np.float32),
                        np.nextafter(np.arange(-128, 129, dtype=np.float32) + np.float32(0.5), np.float32(0)),
                        np.nextafter(np.arange(-128, 129, dtype=np.float32) + np.float32(0.5), np.float32(1e9))])
    t = (v + magic).astype(np.float32)
    q = t.view(np.int32) - 0x4B400000
    assert np.array_equal(q, np.rint(v).astype(np.int32))
    assert np.array_equal((t - magic).astype(np.float32), np.rint(v))


def _threshold_window(gamma: np.float32) -> np.float32:
    """The kernel's search: 32 lanes test the bit patterns gamma/2 - 16 + lane; the first
    pattern above 0.5 is the threshold unless the window fails to bracket it, in which case
    a bisection over the whole positive range runs."""
    def above(bits):
        return np.float32(np.uint32(bits).view(np.float32)) / gamma > np.float32(0.5)
    c = int(np.float32(np.float32(0.5) * gamma).view(np.uint32))
    mask = [above(c - 16 + lane) for lane in range(32)]
    if any(mask) and not mask[0]:
        return np.uint32(c - 16 + mask.index(True)).view(np.float32)
    lo, hi = 0, 0x7F7FFFFF
    while hi - lo > 1:
        mid = lo + ((hi - lo) >> 1)
        if above(mid):
            hi = mid
        else:
            lo = mid
    return np.uint32(hi).view(np.float32)


def test_ternary_threshold_equals_round_clamp():
    rng = np.random.default_rng(2)
    for gamma in [np.float32(1e-5), np.float32(0.0159), np.float32(0.265625), np.float32(3.7)] + \
            [np.float32(g) for g in 10.0 ** rng.uniform(-5, 2, 40)]:
        thr = _threshold_window(gamma)
        # dense neighbourhood of the threshold and random weights
        b = int(thr.view(np.uint32))
        near = np.arange(b - 64, b + 64, dtype=np.uint32).view(np.float32)
        w = np.concatenate([near, -near, rng.normal(0, float(gamma), 4096).astype(np.float32),
                            np.array([0.0, -0.0, 1.5 * gamma, -2.5 * gamma], dtype=np.float32)])
        ref = np.clip(np.rint((w / gamma).astype(np.float32)), -1, 1).astype(np.int8)
        got = np.where(w >= thr, 1, np.where(w <= -thr, -1, 0)).astype(np.int8)
        assert np.array_equal(got, ref), float(gamma)


def _ternary_fields(w):
    """(w & 0x55..) | 0xAA.. minus (w >> 1) & 0x55.., in 32-bit arithmetic."""
    return (((w & 0x55555555) | 0xAAAAAAAA) - ((w >> 1) & 0x55555555)) & 0xFFFFFFFF


def test_gemv_field_identity():
    """The GEMV's two in-word identities, emulated on the integers.

    Every 2-bit field of F equals dec(code) + 2 (the reserved 11 included), and masking F
    with 0x03030303 << 2j leaves bytes f_j * 4^j; then
    sum_j D_j / 4^j - 2 sum x == sum dec * x with D_j the byte dot products.
    """
    rng = np.random.default_rng(3)
    dec_of = {0: 0, 1: 1, 2: -1, 3: 0}
    # exhaustive over one byte of four codes, in each byte position of the word
    for byte in range(256):
        for pos in range(4):
            w = byte << (8 * pos)
            f = _ternary_fields(w)
            for j in range(4):
                c = (byte >> (2 * j)) & 3
                assert (f >> (8 * pos + 2 * j)) & 3 == dec_of[c] + 2
    for trial in range(20):
        K = 64 * (1 + trial)
        codes = rng.integers(0, 4, size=K)           # includes the reserved 11
        x = rng.integers(-128, 128, size=K).astype(np.int64)
        if trial == 0:
            x[:] = -128                              # extreme activations
        dec = np.where(codes == 1, 1, np.where(codes == 2, -1, 0))
        ref = int(np.sum(dec * x))
        # 16 codes per 32-bit word, code k at bits 2*(k % 16) of word k // 16
        words = [sum(int(codes[16 * g + e]) << (2 * e) for e in range(16)) for g in range(K // 16)]
        D = [0, 0, 0, 0]
        for g, w in enumerate(words):
            F = _ternary_fields(w)
            for j in range(4):
                xs = [int(x[16 * g + 4 * i + j]) for i in range(4)]    # interleaved activation word
                m = F & (0x03030303 << (2 * j))
                a = [(m >> (8 * i)) & 0xFF for i in range(4)]           # u8 entries of the mma A register
                assert all(v % (4 ** j) == 0 and 4 ** j <= v <= 3 * 4 ** j for v in a)
                D[j] += sum(av * xv for av, xv in zip(a, xs))
        assert all(D[j] % (4 ** j) == 0 for j in range(4))
        got = sum(D[j] >> (2 * j) for j in range(4)) - 2 * int(np.sum(x))
        assert got == ref


def _byte_perm(a: int, b: int, sel: int) -> int:
    """CUDA __byte_perm: byte i of the result is byte (sel >> 4i) & 7 of the 8-byte value b:a."""
    x = (b << 32) | a
    out = 0
    for i in range(4):
        k = (sel >> (4 * i)) & 7
        out |= ((x >> (8 * k)) & 0xFF) << (8 * i)
    return out


def test_codes_from_rounding_sum_bits():
    """The activation quantiser reads the int8 code off the low byte of
    fl(v + 1.5*2^23) and the table index off that byte with bit 7 flipped."""
    magic = np.float32(1.5 * 2 ** 23)
    for q in range(-127, 128):
        for frac in (0.0, 0.25, -0.25, 0.5 if q % 2 == 0 else 0.0):
            v = np.float32(q + frac)
            t = np.float32(v + magic)                   # fp32 addition, round to nearest even
            bits = int(np.array([t], dtype=np.float32).view(np.uint32)[0])
            assert (bits & 0xFF) == (q & 0xFF)
            assert ((bits & 0xFF) ^ 0x80) == q + 128
    # gathering the low bytes of four words into one
    words = [0x4B4000FB, 0x4B400005, 0x4B3FFF80, 0x4B40007F]
    got = _byte_perm(_byte_perm(words[0], words[1], 0x0040), _byte_perm(words[2], words[3], 0x0040), 0x5410)
    assert got == 0x7F8005FB


def _pk_decode_word(w: int):
    """Emulation of the packed GEMM's decoder: byte-permute lookups of the codes in the table
    {0, +1, -1, 0}, then two permutes that interleave even and odd codes."""
    tab = 0x00FF0100
    se = w & 0x33333333
    so = (w >> 2) & 0x33333333
    e_lo = _byte_perm(tab, 0, se & 0xFFFF)
    e_hi = _byte_perm(tab, 0, (se >> 16) & 0xFFFF)
    o_lo = _byte_perm(tab, 0, so & 0xFFFF)
    o_hi = _byte_perm(tab, 0, (so >> 16) & 0xFFFF)
    words = [_byte_perm(e_lo, o_lo, 0x5140), _byte_perm(e_lo, o_lo, 0x7362),
             _byte_perm(e_hi, o_hi, 0x5140), _byte_perm(e_hi, o_hi, 0x7362)]
    out = []
    for x in words:
        for i in range(4):
            b = (x >> (8 * i)) & 0xFF
            out.append(b - 256 if b >= 128 else b)
    return out


def test_packed_gemm_decoder_matches_code_table():
    """16 codes per word, code i in bits 2i..2i+1: 00 -> 0, 01 -> +1, 10 -> -1, 11 -> 0."""
    rng = np.random.default_rng(9)
    words = [0, 0xFFFFFFFF, 0x55555555, 0xAAAAAAAA, 0x1B1B1B1B] + rng.integers(0, 2 ** 32, 3000).tolist()
    for w in words:
        w = int(w)
        ref = []
        for i in range(16):
            c = (w >> (2 * i)) & 3
            ref.append((c & 1) - (c >> 1) if c != 3 else 0)
        assert _pk_decode_word(w) == ref, hex(w)


def test_packed_gemm_decoder_addresses():
    """The pair kernel's decoders: a group of four warps (warps 6 + 4 g .. 9 + 4 g) covers the
    four TMEM lane quarters (warp % 4), so thread (warp, lane) owns weight row
    32 (warp % 4) + lane.  For k-block jj of a 128-byte-swizzled packed stage it reads the row's
    logical 16-byte chunks 2 jj and 2 jj + 1 at chunk (c ^ (row % 8)); over the stage's four
    k-blocks every physical chunk of every row is read exactly once, and word i of a k-block
    (codes 16 i .. 16 i + 15) lands in TMEM columns 4 i .. 4 i + 3 of that k-block's 32."""
    for g in range(4):
        rows = sorted(32 * (w % 4) + lane for w in range(6 + 4 * g, 10 + 4 * g) for lane in range(32))
        assert rows == list(range(128))
    reads = {}
    for row in range(128):
        sw = row & 7
        for jj in range(4):
            for half in range(2):
                logical = 2 * jj + half
                phys = logical ^ sw
                assert 0 <= phys < 8
                reads[(row, phys)] = reads.get((row, phys), 0) + 1
                # the 16 bytes of this chunk are words 4 half .. 4 half + 3 of k-block jj; word
                # q covers codes 16 q .. 16 q + 15 and goes to columns 4 q .. 4 q + 3
                for q in range(4 * half, 4 * half + 4):
                    byte0 = 32 * jj + 4 * q                  # byte of the logical packed row
                    assert byte0 // 16 == logical
                    assert [4 * q + e for e in range(4)] == list(range(4 * q, 4 * q + 4))
    assert len(reads) == 128 * 8 and set(reads.values()) == {1}

