"""Pins of the oracle's state-space v variants (CPU only): round-to-nearest
and stochastic rounding on the zero-inclusive code {k/15 s}, and the
zero-excluded code {(k+1)/16 s} without the EDEN rescale.  These are the
quantisers the pages set the two methods against ("ZIP-SR 4-bit AdamW --
Preconditioner-space stochastic rounding", car / stochastic rounding paragraph
and worked example: state-space rules on the zero-inclusive code; memory
paragraph: a zero-excluded code with a positive floor)."""
import json
import os

import numpy as np
import pytest

import oracle
from workloads import bf16_bits

U_STEP = 2.0 ** -23


def _p_low(fn, x, lo_code):
    """Fraction of the 2^23 uniforms giving the lower code (monotone in u)."""
    lo, hi = 0, 1 << 23
    while lo < hi:
        j = (lo + hi) // 2
        if fn(x, j * U_STEP) == lo_code:
            lo = j + 1
        else:
            hi = j
    return lo / 2.0 ** 23


def test_zi_rtn_is_nearest_code_point():
    _, _, vz, _ = oracle.tables()
    pts = vz.astype(np.float64)
    mids = ((pts[:-1] + pts[1:]) / 2).astype(np.float32)
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.uniform(0, 1, 3000), vz, mids, np.nextafter(mids, 2)]).astype(np.float32)
    for x in xs:
        c = oracle.zi_rtn(float(x))
        d = np.abs(pts - float(x))
        assert abs(d[c] - d.min()) <= 2 * np.spacing(np.float32(1.0))
    for k, m in enumerate(mids):                       # on a threshold: low
        assert oracle.zi_rtn(float(m)) == k


@pytest.mark.parametrize("x", [0.0, 1e-6, 0.01, 1 / 30, 0.2, 0.5, 0.77, 0.999, 1.0])
def test_zi_sr_unbiased_by_enumeration(x):
    _, _, vz, _ = oracle.tables()
    x = float(np.float32(x))
    a = oracle.zi_sr(x, 0.0)
    b = oracle.zi_sr(x, 1.0 - U_STEP)
    if a == b:
        assert float(vz[a]) == x or x in (0.0, 1.0)
        return
    p = _p_low(oracle.zi_sr, x, a)
    mean = p * float(vz[a]) + (1 - p) * float(vz[b])
    assert abs(mean - x) <= U_STEP * float(vz[b] - vz[a]) + 1e-7


def test_worked_example_state_space_rounding(golden_dir):
    """The same near-zero cell as the ZIP-SR pin: state-space stochastic
    rounding stores zero with probability (b - v)/b = 75%, the expected next
    multiplier is about 75 million, 74 times the exact one."""
    ex = json.load(open(os.path.join(golden_dir, "worked_example_near_zero.json")))
    inp, pr = ex["inputs"], ex["printed"]
    s = np.float32(15 * inp["b"])
    v = np.float32(inp["v"])
    x = float(np.float32(v * (np.float32(1) / s)))
    assert oracle.zi_sr(x, 0.0) == 0 and oracle.zi_sr(x, 1 - U_STEP) == 1
    p_zero = _p_low(oracle.zi_sr, x, 0)
    assert round(p_zero, 2) == pr["state_space_p_zero"]
    sc = oracle.make_scalars(1e-3, 0.9, 0.95, inp["eps"], t=100000)
    _, _, vz, _ = oracle.tables()
    b = float(np.float32(vz[1] * s))

    def mult(vs):
        den, _, _, _ = oracle.update_elem(sc, 1.0, 0.0, 0.0, vs, 0.0)
        return 1.0 / den
    e = p_zero * mult(0.0) + (1 - p_zero) * mult(b)
    assert abs(e - pr["state_space_expected_multiplier"]) <= 0.05 * pr["state_space_expected_multiplier"]
    assert round(e / mult(float(v))) == pr["state_space_overshoot_factor"]


def _block(vcode, g, t=1):
    sc = oracle.make_scalars(1e-3, 0.9, 0.999, 1e-8, t=t, seed=7)
    gb = bf16_bits(np.asarray(g, np.float32))
    w = np.zeros(128, np.float32)
    mc = np.zeros(64, np.uint8)
    vc = np.zeros(64, np.uint8)
    ms = np.zeros(1, np.float32)
    vs = np.zeros(1, np.float32)
    oracle.lib().oracle_block4(sc, np.float32(1.0), vcode, 0, 0, 0, 128, w, gb, mc, ms, vc, vs)
    codes = np.empty(128, np.int64)
    codes[0::2] = vc & 15
    codes[1::2] = vc >> 4
    return codes, vs[0], sc


def test_ze_floor_is_nearest_zero_excluded_without_rescale():
    g = np.random.default_rng(1).standard_normal(128).astype(np.float32) * np.float32(1e-3)
    codes, scale, sc = _block(oracle.VCODE_ZE_FLOOR, g)
    v1 = (np.float32(sc.omb2) * (bf16_bits(g).astype(np.uint32) << 16).view(np.float32) ** 2)
    assert scale == v1.max()                          # the block maximum, unrescaled
    inv = np.float32(1) / scale
    for i in range(128):
        assert codes[i] == oracle.zeeden_code(float(np.float32(v1[i]) * inv))
    codes_e, scale_e, _ = _block(oracle.VCODE_ZEEDEN, g)
    assert np.array_equal(codes, codes_e) and scale_e != scale


def test_zero_inclusive_variants_share_scale_and_top_code():
    """ZIP-SR and the two state-space variants use the same k/15 code and the
    same block scale: all three store the block maximum as the scale and code
    15 for the element that holds it."""
    g = np.zeros(128, np.float32)
    g[:8] = np.float32(1e-3) * np.arange(1, 9, dtype=np.float32)
    out = {}
    for vc in (oracle.VCODE_ZIPSR, oracle.VCODE_ZI_RTN, oracle.VCODE_ZI_SR):
        out[vc] = _block(vc, g)[:2]
    for vc, (codes, scale) in out.items():
        assert codes[7] == 15 and scale == out[oracle.VCODE_ZIPSR][1]
        assert np.all(codes[8:] == 0)                 # v = 0 stays on the zero point
