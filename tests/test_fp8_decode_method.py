"""The FP8 decoder's arithmetic, emulated on the CPU for every input, against the oracle's E4M3
decoder.

The GPU decoder places a code's 7 magnitude bits at bits 4-10 of a bf16 and its sign at bit
15, then multiplies by the bf16 2^(s - 7) (s the scale byte) with one round-to-nearest bf16
multiply.  Here that is done in fp64 from the bit patterns (the bf16 values, the exact product,
and bf16 rounding of the product), for all 254 finite codes and every scale byte, to pin the
header's input contract: the result equals code * 2^(s - 127) exactly for s in 7..134.  The
GPU tests check the kernel itself bit for bit against the bf16 path on the oracle's decoding.
"""
import math

import numpy as np

import oracle


def bf16_value(bits: int) -> float:
    """The number a bf16 bit pattern stands for (1 sign, 8 exponent bits bias 127, 7 mantissa
    bits; exponent field 0 is subnormal)."""
    sign = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0xFF:
        return float("nan") if m else sign * math.inf
    if e == 0:
        return sign * (m / 128.0) * 2.0 ** -126
    return sign * (1.0 + m / 128.0) * 2.0 ** (e - 127)


def round_to_bf16(x: float) -> float:
    """x rounded to the nearest bf16 value (ties to even), overflow to infinity."""
    if x == 0.0 or math.isnan(x) or math.isinf(x):
        return x
    m, e = math.frexp(abs(x))          # x = m * 2^e, m in [0.5, 1)
    e -= 1                              # x = (2m) * 2^e with 2m in [1, 2)
    if e > 127:
        return math.copysign(math.inf, x)
    step = 2.0 ** (max(e, -126) - 7)    # spacing of bf16 values at this binade
    q = abs(x) / step
    r = math.floor(q)
    frac = q - r
    if frac > 0.5 or (frac == 0.5 and r % 2 == 1):
        r += 1
    y = r * step
    if y >= 2.0 ** 128:
        return math.copysign(math.inf, x)
    return math.copysign(y, x)


def kernel_decode(code: int, s: int) -> float:
    placed = ((code & 0x7F) << 4) | ((code & 0x80) << 8)
    mult = bf16_value(((s + 120) << 7) & 0x7F80)
    return round_to_bf16(bf16_value(placed) * mult)


FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_bit_placement_reads_as_code_times_2_pow_minus_120():
    for c in FINITE:
        placed = ((c & 0x7F) << 4) | ((c & 0x80) << 8)
        assert bf16_value(placed) == oracle.e4m3_value(c) * 2.0 ** -120, hex(c)


def test_decode_is_exact_for_scale_bytes_7_to_134():
    for s in range(7, 135):
        for c in FINITE:
            want = oracle.e4m3_value(c) * 2.0 ** (s - 127)
            got = kernel_decode(c, s)
            assert got == want, (hex(c), s, got, want)


def test_outside_the_contract_the_decode_is_not_exact():
    # scale byte 135 would need the bf16 factor 2^128: not finite
    assert kernel_decode(0x38, 135) != oracle.e4m3_value(0x38) * 2.0 ** 8
    # at scale byte 0 the smallest subnormal code lands below bf16's smallest subnormal
    want = oracle.e4m3_value(0x01) * 2.0 ** -127
    assert want < 2.0 ** -133 and kernel_decode(0x01, 0) != want


def test_the_workload_checkpoint_stays_inside_the_contract():
    from workloads import make_fp8, make_small
    routed, shared = make_fp8(make_small(8, 256, 4, 2, 128, 1, seed=3))
    for t in (routed.gate_scale, routed.up_scale, routed.down_scale, shared.gate_scale):
        b = t.numpy()
        assert b.min() >= 7 and b.max() <= 134, (b.min(), b.max())
    for t in (routed.gate, routed.up, routed.down):
        c = t.numpy()
        assert not np.any((c & 0x7F) == 0x7F)    # no NaN codes


def prmt(a: int, b: int, sel: int) -> int:
    """PRMT in its default mode: result byte i is byte (nibble i of sel) & 7 of the eight
    bytes b:a (a bytes 0-3, b bytes 4-7); bit 3 of the nibble replicates that byte's sign."""
    src = (b << 32) | a
    out = 0
    for i in range(4):
        nib = (sel >> (4 * i)) & 0xF
        byte = (src >> (8 * (nib & 7))) & 0xFF
        if nib & 8:
            byte = 0xFF if byte & 0x80 else 0x00
        out |= byte << (8 * i)
    return out


def word_planes(w: int):
    """The word-level decoder's integer steps: byte planes of the low and high bf16 bytes,
    interleaved into the pairs (code 0, code 1) and (code 2, code 3)."""
    lo = (w << 4) & 0xF0F0F0F0
    hi = ((w >> 4) & 0x07070707) | (w & 0x80808080)
    return prmt(lo, hi, 0x5140), prmt(lo, hi, 0x7362)


def pair_bits(w: int, sel: int) -> int:
    """The pair decoder's integer steps: PRMT of two code bytes to bits 8-15 and 24-31 (zero
    elsewhere), magnitude shifted down by 4, sign kept."""
    x8 = prmt(w, 0, sel)
    return ((x8 >> 4) & 0x07F007F0) | (x8 & 0x80008000)


def test_word_decoder_places_every_code_like_the_pair_decoder():
    """Both integer routes give, for every code in every byte position of a word, the bf16
    half whose bits read as code * 2^-120 (the bit placement pinned above), so the one bf16
    multiply that follows gives the same exact weights."""
    rng = np.random.default_rng(11)
    words = [int(c) * 0x01010101 for c in range(256)]
    words += [int(v) for v in rng.integers(0, 2 ** 32, size=4096, dtype=np.uint64)]
    for pos in range(4):                       # each code once in each byte, others random
        for c in range(256):
            words.append((int(rng.integers(0, 2 ** 32)) & ~(0xFF << (8 * pos)) | (c << (8 * pos)))
                         & 0xFFFFFFFF)
    for w in words:
        p01, p23 = word_planes(w)
        assert p01 == pair_bits(w, 0x1404) and p23 == pair_bits(w, 0x3424), hex(w)
        codes = [(w >> (8 * i)) & 0xFF for i in range(4)]
        halves = [p01 & 0xFFFF, p01 >> 16, p23 & 0xFFFF, p23 >> 16]
        for c, h in zip(codes, halves):
            assert h == ((c & 0x7F) << 4) | ((c & 0x80) << 8), (hex(w), hex(c), hex(h))
