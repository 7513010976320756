"""Pins of the oracle's ZE-EDEN second-moment code (CPU only).

ZE-EDEN rounds v/s to the nearest zero-excluded code point (k+1)/16 and
multiplies the block scale by ||x||^2 / max(<x,Q(x)>, 1e-12 s^2) ("ZIP-SR /
ZE-EDEN: 4-bit AdamW state quantization", Core equation)."""
import numpy as np
import pytest

import oracle
from workloads import bf16_bits, bf16_to_f32


def test_codes_are_nearest_zero_excluded_points():
    for x in np.linspace(0, 1, 2001, dtype=np.float32):
        k = oracle.zeeden_code(float(x))
        pts = (np.arange(16) + 1) / 16.0
        d = np.abs(pts - float(x))
        assert d[k] == d.min()
    assert oracle.zeeden_code(0.0) == 0            # zero maps to the floor 1/16
    assert oracle.zeeden_code(1.0) == 15
    # ties at 16x = j + 1/2 go to even j
    assert oracle.zeeden_code(2.5 / 16) == 1        # 16x = 2.5 -> 2 -> k = 1
    assert oracle.zeeden_code(3.5 / 16) == 3        # 16x = 3.5 -> 4 -> k = 3


def test_factor_hand_computed_two_elements():
    # x = (1, 0.3): Q = (1, 5/16) ; ||x||^2 = 1.09 ; <x,Q> = 1 + 0.09375
    c = oracle.zeeden_factor(np.float32([1.0, 0.3]) ** 2,
                             np.float32([1.0 * 1.0, 0.3 * 0.3125]))
    assert c == pytest.approx(1.09 / 1.09375, rel=1e-6)


def test_factor_is_one_on_the_grid():
    x = (np.arange(16, dtype=np.float32) + 1) / 16
    c = oracle.zeeden_factor(x * x, x * x)
    assert c == 1.0


def _block(g, vcode=1, t=1, b2=0.999):
    sc = oracle.make_scalars(1e-3, 0.9, b2, 1e-8, t=t)
    gb = bf16_bits(np.asarray(g, np.float32))
    n = len(gb)
    w = np.zeros(128, np.float32)
    gpad = np.zeros(128, np.uint16)
    gpad[:n] = gb
    mc = np.zeros(64, np.uint8)
    vc = np.zeros(64, np.uint8)
    ms = np.zeros(1, np.float32)
    vs = np.zeros(1, np.float32)
    oracle.lib().oracle_block4(sc, np.float32(1.0), vcode, 0, 0, 0, n, w, gpad, mc, ms, vc, vs)
    codes = np.empty(128, np.int64)
    codes[0::2] = vc & 15
    codes[1::2] = vc >> 4
    v1 = (np.float32(sc.omb2) * (bf16_to_f32(gb) ** 2)).astype(np.float32)
    return codes[:n], vs[0], v1, codes


@pytest.mark.parametrize("n", [128, 77, 1])
def test_block_scale_equals_page_formula(n):
    """The stored scale is s * ||x||^2 / max(<x,Q(x)>, 1e-12 s^2) with x the
    block's v values and Q(x) their code points times s, all in binary64,
    within 1e-6 relative (binary32 rounding of the sums)."""
    rng = np.random.default_rng(n)
    g = rng.standard_normal(n).astype(np.float32) * np.float32(1e-3)
    codes, scale, v1, allc = _block(g)
    s = float(v1.max())
    x = v1.astype(np.float64)
    q = (codes + 1) / 16.0 * s
    ref = s * (x @ x) / max(x @ q, 1e-12 * s * s)
    assert scale == pytest.approx(ref, rel=1e-6)
    assert np.all(allc[n:] == 0)        # empty slots stay code 0
    # EDEN projection identity: the rescaled reconstruction projects onto x
    c = scale / s
    assert (x @ (c * q)) == pytest.approx(x @ x, rel=1e-6)


def test_zero_block_stores_zero_bytes():
    codes, scale, _, allc = _block(np.zeros(128, np.float32))
    assert scale == 0.0 and np.all(allc == 0)


def test_tiny_values_use_the_floor_code():
    g = np.full(128, 1e-9, np.float32)
    g[0] = 1e-3
    codes, scale, v1, _ = _block(g)
    assert codes[0] == 15
    assert np.all(codes[1:] == 0)            # floor (k+1)/16 with k = 0, never zero
    assert scale > 0


def test_factor_floor_matches_page_units():
    """The floor 1e-12 s^2 in the pages' units becomes 1e-12 after dividing
    the block by s; on a block whose <x,Q> falls below it both give the same
    scale factor."""
    xx = np.zeros(128, np.float32)
    xq = np.zeros(128, np.float32)
    xx[0] = 1e-14
    xq[0] = 1e-15
    c = oracle.zeeden_factor(xx, xq)
    assert c == pytest.approx(1e-14 / 1e-12, rel=1e-6)
