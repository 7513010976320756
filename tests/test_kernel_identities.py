"""CPU checks of the exact binary32 identities the step kernel's arithmetic
rests on (the kernel itself runs only on the GPU; its results are checked
against the oracle by the -m gpu parity tests).  Each identity is checked
over every case it is used for, with float32 values and exact rational
arithmetic standing in for one fused multiply-add."""
from fractions import Fraction

import numpy as np

KMAGIC = np.float32(12582912.0)          # 1.5 * 2^23: adding it rounds to an integer


def f32(x):
    return np.float32(x)


def bits(x):
    return int(np.frombuffer(np.float32(x).tobytes(), np.uint32)[0])


def from_bits(b):
    return np.frombuffer(np.uint32(b).tobytes(), np.float32)[0]


def fma_exact(a, b, c):
    """a*b + c computed exactly (Fraction), and whether its binary32 rounding
    loses nothing."""
    v = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    r = f32(float(v))
    return v, Fraction(float(r)) == v, r


def test_zero_excluded_decode_from_nibbles_in_place():
    # A nibble k at bit p (0, 4, 8, 12) of the code word, or-ed into kMagic's
    # mantissa, is kMagic + k 2^p; one fma with scale 2^-(p+4) and offset
    # 1/16 - kMagic 2^-(p+4) gives (k + 1)/16, exactly.
    for p in (0, 4, 8, 12):
        scale = f32(2.0 ** -(p + 4))
        off = f32(f32(0.0625) - KMAGIC * scale)
        assert Fraction(float(off)) == Fraction(1, 16) - Fraction(12582912) * Fraction(2) ** -(p + 4)
        for k in range(16):
            x = from_bits(bits(KMAGIC) | (k << p))
            assert Fraction(float(x)) == 12582912 + k * 2 ** p
            v, exact, r = fma_exact(x, scale, off)
            assert exact and v == Fraction(k + 1, 16)


def test_zero_excluded_code_from_the_clamped_magic_sum():
    # t2 = fma(x, 16, kMagic) = kMagic + rint(16x) for x in [0, 1]; clamped at
    # kMagic + 1 it is kMagic + k + 1; t2 - 1 has kMagic's bit pattern plus k,
    # and fma(t2, 1/16, -kMagic/16) is (k + 1)/16, all exact.
    nmagic16 = f32(-KMAGIC / f32(16.0))
    assert Fraction(float(nmagic16)) == Fraction(-12582912, 16)
    xs = np.concatenate([np.linspace(0, 1, 40001, dtype=np.float32),
                         np.array([0.0, 1 / 32, 3 / 32, 0.5, 1.0], np.float32)])
    for x in xs:
        v, _, t2 = fma_exact(x, f32(16.0), KMAGIC)
        r = round(Fraction(float(x)) * 16)               # half to even, like the fma's rounding
        assert t2 == f32(12582912 + r)
        tm = max(t2, f32(KMAGIC + 1))
        k = max(r, 1) - 1
        assert bits(f32(tm - f32(1.0))) == bits(KMAGIC) + k
        v, exact, q = fma_exact(tm, f32(1 / 16), nmagic16)
        assert exact and v == Fraction(k + 1, 16)


def test_nf4_bucket_row_offset_is_the_masked_bit_pattern():
    # fma(x, 4096, kMagic + 4096) = kMagic + r with r = round(4096 x + 4096) in
    # [0, 8192] for |x| <= 1 + 2^-23; its bits masked with 0x3F80 are
    # 128 floor(r / 128), the byte offset of bucket row floor(r / 128).
    m4096 = f32(KMAGIC + f32(4096.0))
    xs = np.concatenate([np.linspace(-1, 1, 200001, dtype=np.float32),
                         np.array([np.nextafter(np.float32(1), np.float32(2)),
                                   -np.nextafter(np.float32(1), np.float32(2))], np.float32)])
    for x in xs[::7]:
        _, _, y = fma_exact(x, f32(4096.0), m4096)
        r = bits(y) - bits(KMAGIC)
        assert 0 <= r <= 8192
        assert (bits(y) & 0x3F80) == 128 * (r // 128)


def test_philox_quad_counter_never_carries_within_a_block():
    # A group at value offset off (a multiple of 8, off + 7 < 128) of a block
    # starting at element e0 (a multiple of 128) draws from quads
    # (e0 + off)/4 and (e0 + off)/4 + 1; formed as (e0 >> 2) + (off >> 2) (+1)
    # in the low 32-bit word, they never carry into the high word.
    rng = np.random.default_rng(0)
    e0s = [0, 128, (1 << 34) - 128, (1 << 34), (1 << 39) - 4096, (1 << 36) + 896 - 896 % 128]
    e0s += [int(x) * 128 for x in rng.integers(0, 1 << 32, size=200)]
    for e0 in e0s:
        assert e0 % 128 == 0
        for off in range(0, 128, 8):
            for c in (0, 1):
                quad = (e0 + off) // 4 + c
                lo = ((e0 >> 2) & 0xFFFFFFFF) + (off >> 2) + c
                assert lo < (1 << 32)
                assert (quad & 0xFFFFFFFF) == lo and (quad >> 32) == (e0 >> 34)
