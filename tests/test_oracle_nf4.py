"""Pins of the oracle's NF4 first-moment codebook and its round-to-nearest
(CPU only).  NF4 is named, not listed, by the pages ("A New Approach to 4-bit
AdamW Optimizer Quantization", Two Complementary Technical Approaches); the
construction is QLoRA's normal-quantile one."""
import numpy as np
import pytest
from scipy.special import ndtri

import oracle


def scipy_nf4():
    """The same construction through scipy's inverse normal CDF."""
    offset = 0.9677083
    pos = ndtri(np.linspace(offset, 0.5, 9)[:-1])
    neg = -ndtri(np.linspace(offset, 0.5, 8)[:-1])
    vals = np.sort(np.concatenate([pos, [0.0], neg]))
    return vals / vals.max()


def test_levels_match_library_quantiles():
    ours = oracle.nf4_levels_f64()
    ref = scipy_nf4()
    np.testing.assert_allclose(ours, ref, rtol=0, atol=1e-14)
    nf4, _, _, _ = oracle.tables()
    assert np.array_equal(nf4, ref.astype(np.float32))


def test_level_structure():
    nf4, mid, _, _ = oracle.tables()
    assert nf4[0] == -1.0 and nf4[7] == 0.0 and nf4[15] == 1.0
    assert np.all(np.diff(nf4) > 0)
    assert (nf4 < 0).sum() == 7 and (nf4 > 0).sum() == 8
    assert np.all(nf4[:-1] < mid) and np.all(mid < nf4[1:])
    # the published NF4 values, to the 4 digits they are commonly quoted with
    approx = [-1.0, -0.6962, -0.5251, -0.3949, -0.2844, -0.1848, -0.0911, 0.0,
              0.0796, 0.1609, 0.2461, 0.3379, 0.4407, 0.5626, 0.7230, 1.0]
    np.testing.assert_allclose(nf4, approx, atol=6e-5)


def test_rtn_is_nearest_level():
    """Brute force: the code is the nearest level in exact arithmetic, except
    within one ulp of a midpoint where the binary32 threshold decides."""
    nf4, mid, _, _ = oracle.tables()
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.uniform(-1, 1, 4000), nf4, mid,
                         np.nextafter(mid, 2), np.nextafter(mid, -2)]).astype(np.float32)
    for x in xs:
        c = oracle.nf4_rtn(float(x))
        d = np.abs(nf4.astype(np.float64) - float(x))
        near = np.min(np.abs(mid.astype(np.float64) - float(x)))
        if near > 2 * np.spacing(np.float32(abs(x) + 1e-30)):
            assert c == int(np.argmin(d))
        else:
            assert abs(d[c] - d.min()) <= 4 * np.spacing(np.float32(1.0))


def test_rtn_threshold_ties_go_low():
    _, mid, _, _ = oracle.tables()
    for j, m in enumerate(mid):
        assert oracle.nf4_rtn(float(m)) == j
        assert oracle.nf4_rtn(float(np.nextafter(m, np.float32(2)))) == j + 1


@pytest.mark.parametrize("x", [-1.0, -0.8, -0.3, -0.05, 0.0, 0.02, 0.3, 0.65, 0.99, 1.0])
def test_state_space_sr_unbiased_by_enumeration(x):
    """LM-head first-moment stochastic rounding ("A New Approach ...",
    Stochastic rounding): over all 2^23 uniforms E[Q(x)] = x.  The decision
    is monotone in u, so the count of low outcomes is found by bisection."""
    nf4, _, _, _ = oracle.tables()
    x = float(np.float32(x))
    lo_code = oracle.nf4_sr(x, 0.0)
    hi_code = oracle.nf4_sr(x, 1.0 - 2.0 ** -23)
    assert hi_code - lo_code in (0, 1)
    if lo_code == hi_code:
        assert float(nf4[lo_code]) == x
        return
    lo, hi = 0, 1 << 23          # first j that rounds up
    while lo < hi:
        j = (lo + hi) // 2
        if oracle.nf4_sr(x, j * 2.0 ** -23) == lo_code:
            lo = j + 1
        else:
            hi = j
    p_low = lo / 2.0 ** 23
    mean = p_low * float(nf4[lo_code]) + (1 - p_low) * float(nf4[hi_code])
    assert abs(mean - x) <= 2.0 ** -23 * float(nf4[hi_code] - nf4[lo_code]) + 1e-7
