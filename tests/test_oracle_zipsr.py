"""Pins of the oracle's ZIP-SR second-moment rounding (CPU only).

ZIP-SR keeps the lower of two code points a < b with probability
[h(v)-h(b)]/[h(a)-h(b)], h(v) = 1/(sqrt(v/(1-b2^t)) + eps) ("ZIP-SR / ZE-EDEN:
4-bit AdamW state quantization", Core equation), so E[h(Q(v))] = h(v).
"""
import json
import os

import numpy as np
import pytest

import oracle

U_STEP = 2.0 ** -23
N_U = 1 << 23
W_STEP = 2.0 ** -32


def f32(x):
    return float(np.float32(x))


def p_low_exact(x, dv, R, eps):
    """Fraction of the 2^32 draw words for which ZIP-SR keeps the lower code
    point, with the uniform ZIP-SR draws from a word (oracle.uniform32).  The
    decision is monotone in the word; bisection finds the threshold."""
    k_lo = oracle.zipsr_decide(x, dv, R, eps, oracle.uniform32(0))
    k_hi = oracle.zipsr_decide(x, dv, R, eps, oracle.uniform32(0xFFFFFFFF))
    if k_lo == k_hi:
        return (1.0 if k_lo == oracle.zipsr_bracket(x) else 0.0), k_lo
    lo, hi = 0, 1 << 32
    while lo < hi:
        j = (lo + hi) // 2
        if oracle.zipsr_decide(x, dv, R, eps, oracle.uniform32(j)) == k_lo:
            lo = j + 1
        else:
            hi = j
    return lo * W_STEP, k_lo


def p_low_exact_u23(x, dv, R, eps):
    """The same fraction for a 23-bit uniform (j 2^-23, j < 2^23): the
    granularity the ZIP-SR draw had before it took the whole word."""
    k_lo = oracle.zipsr_decide(x, dv, R, eps, 0.0)
    k_hi = oracle.zipsr_decide(x, dv, R, eps, 1.0 - U_STEP)
    if k_lo == k_hi:
        return (1.0 if k_lo == oracle.zipsr_bracket(x) else 0.0), k_lo
    lo, hi = 0, N_U
    while lo < hi:
        j = (lo + hi) // 2
        if oracle.zipsr_decide(x, dv, R, eps, j * U_STEP) == k_lo:
            lo = j + 1
        else:
            hi = j
    return lo / N_U, k_lo


def h64(v, rs_bc2, eps):
    return 1.0 / (np.sqrt(v) * rs_bc2 + eps)


def test_worked_example_near_zero_cell(golden_dir):
    """The worked example of "ZIP-SR 4-bit AdamW -- Preconditioner-space
    stochastic rounding" (quiet-gradient paragraph): v = 1e-12 between the
    code points 0 and b = 4e-12, eps = 1e-8, beta2 = 0.95, bias correction
    ignored.  Checked at the two significant figures the page prints."""
    ex = json.load(open(os.path.join(golden_dir, "worked_example_near_zero.json")))
    inp, pr = ex["inputs"], ex["printed"]
    eps = f32(inp["eps"])
    v = f32(inp["v"])
    # block scale s with b = s/15; x = v/s lies in the zero cell
    s = f32(15 * inp["b"])
    _, _, vz, vzs = oracle.tables()
    b = f32(np.float32(vz[1]) * np.float32(s))
    assert abs(b - inp["b"]) / inp["b"] < 1e-6
    rs_bc2 = 1.0
    R = f32(np.float32(np.sqrt(np.float32(s))) * np.float32(rs_bc2))
    dv = f32(np.float32(np.sqrt(np.float32(v))) * np.float32(rs_bc2) + np.float32(eps))
    x = f32(np.float32(v) * (np.float32(1.0) / np.float32(s)))
    assert oracle.zipsr_bracket(x) == 0

    p_zero, k = p_low_exact(x, dv, R, eps)
    assert k == 0
    # page: "about 0.5%", closed form eps(1 - sqrt(v/b))/(sqrt(v) + eps)
    closed = inp["eps"] * (1 - np.sqrt(inp["v"] / inp["b"])) / (np.sqrt(inp["v"]) + inp["eps"])
    assert abs(p_zero - closed) < 1e-5
    assert round(p_zero, 3) == pr["zipsr_p_zero"]

    # next-step multipliers through the oracle's own update (g = 0, b2 = 0.95)
    sc = oracle.make_scalars(1e-3, 0.9, 0.95, eps, t=100000)
    assert sc.rs_bc2 == 1.0

    def next_mult(v_stored):
        den, _, _, _ = oracle.update_elem(sc, 1.0, 0.0, 0.0, v_stored, 0.0)
        return 1.0 / den

    m_exact, m_b, m_zero = next_mult(v), next_mult(b), next_mult(0.0)

    def sig2(a, b_):
        return abs(a - b_) <= 0.05 * abs(b_)
    assert sig2(m_exact, pr["next_multiplier_exact_v"])
    assert sig2(m_b, pr["next_multiplier_b_stored"])
    assert m_zero == pytest.approx(pr["next_multiplier_zero_stored"], rel=1e-6)
    # state-space rounding stores zero with probability (b - v)/b
    p_ss = (b - v) / b
    e_ss = p_ss * m_zero + (1 - p_ss) * m_b
    assert p_ss == pytest.approx(pr["state_space_p_zero"], abs=1e-6)
    assert sig2(e_ss, pr["state_space_expected_multiplier"])
    assert round(e_ss / m_exact) == pr["state_space_overshoot_factor"]
    # ZIP-SR's expected next multiplier is about the exact one
    e_zip = p_zero * m_zero + (1 - p_zero) * m_b
    assert sig2(e_zip, pr["zipsr_expected_multiplier"])
    assert abs(e_zip - m_exact) / m_exact < 0.02


CASES = []
for s in [6e-11, 1e-8, 3e-7, 1e-4, 2.5e-2]:
    for xv in [0.0, 1e-6, 0.003, 0.02, 1 / 15, 0.07, 0.2, 0.5, 0.81, 14 / 15, 0.99, 1.0]:
        for rs in [1.0, 31.6]:
            CASES.append((s, xv, rs))


@pytest.mark.parametrize("s,xv,rs_bc2", CASES)
def test_exact_expectation_of_h(s, xv, rs_bc2):
    """Enumerating every draw word: the oracle's canonical binary32
    probability equals the pages' formula in binary64 within 1e-6 plus the
    binary32 conditioning of the cell, and the expected preconditioner
    equals h(v) (the preconditioner-space unbiasedness ZIP-SR is built on)."""
    eps = f32(1e-8)
    s = f32(s)
    rs_bc2 = f32(rs_bc2)
    _, _, vz, vzs = oracle.tables()
    v = f32(np.float32(xv) * np.float32(s))
    inv = np.float32(1.0) / np.float32(s)
    x = f32(np.float32(v) * inv)
    R = f32(np.sqrt(np.float32(s)) * np.float32(rs_bc2))
    dv = f32(np.float32(np.sqrt(np.float32(v))) * np.float32(rs_bc2) + np.float32(eps))
    k = oracle.zipsr_bracket(x)
    assert float(vz[k]) <= x and (k == 14 or x < float(vz[k + 1]))
    p, _ = p_low_exact(x, dv, R, eps)
    # the pages' probability in binary64 with the code points' d values
    da = float(vzs[k]) * R + eps
    db = float(vzs[k + 1]) * R + eps
    if db == da:
        return  # flat preconditioner: the state-space fallback applies
    p_ref = (1 / dv - 1 / db) / (1 / da - 1 / db)
    p_ref = min(max(p_ref, 0.0), 1.0)
    # binary32 conditioning: da and db are each rounded once (half an ulp of
    # d); p moves by that over (db - da).  Plus the draw granularity.
    cond = 4 * 2.0 ** -24 * db / (db - da)
    # the draw: 2^-32 granularity near zero, 2^-23 relative above 2^-8
    grain = W_STEP + 2.0 ** -22 * p_ref
    assert abs(p - p_ref) < 1e-6 * p_ref + grain + cond
    # E[h(Q)] = h(v): with d-values of the code points, in binary64
    e_h = p * (1 / da) + (1 - p) * (1 / db)
    assert abs(e_h - 1 / dv) <= (1e-6 * p_ref + grain + cond) * abs(1 / da - 1 / db) + 1e-12 / dv


def test_zero_and_top_are_deterministic():
    eps = f32(1e-8)
    R = f32(np.sqrt(np.float32(1e-6)))
    assert oracle.zipsr_decide(0.0, eps, R, eps, 0.999) == 0
    assert oracle.zipsr_decide(1.0, R + eps, R, eps, 0.0) == 15


@pytest.mark.parametrize("v_frac", [0.004, 0.03, 0.5])
def test_monte_carlo_unbiased_in_h(v_frac):
    """10^6 draws through the oracle's whole block step: the mean of the
    stored preconditioner 1/(sqrt(Q(v)) rs_bc2 + eps) matches h(v) within
    4 sigma, while the state-space mean of the code point would not near zero.
    One element carries the block maximum; 127 carry v."""
    _, _, vz, vzs = oracle.tables()
    b1, b2, eps = np.float32(0.9), np.float32(0.999), np.float32(1e-8)
    # zero state: v1 = (1-b2) g^2 ; choose g so that v1 spans the near-zero cell
    g_max = np.float32(3e-5)
    g_small = np.float32(g_max * np.sqrt(np.float32(v_frac)))
    from workloads import bf16_bits, bf16_to_f32
    g = np.full(128, g_small, np.float32)
    g[0] = g_max
    gb = bf16_bits(g)
    gf = bf16_to_f32(gb)
    omb2 = np.float32(1.0) - b2
    v1 = (omb2 * (gf * gf)).astype(np.float32)
    hs, h_true = [], None
    n_rep = 8000
    for rep in range(n_rep):
        sc = oracle.make_scalars(1e-3, b1, b2, eps, t=1, seed=rep)
        w = np.zeros(128, np.float32)
        mc = np.zeros(64, np.uint8)
        vc = np.zeros(64, np.uint8)
        ms = np.zeros(1, np.float32)
        vs = np.zeros(1, np.float32)
        oracle.lib().oracle_block4(sc, np.float32(1.0), 0, 0, 0, 0, 128, w, gb, mc, ms, vc, vs)
        codes = np.empty(128, np.int64)
        codes[0::2] = vc & 15
        codes[1::2] = vc >> 4
        rs = np.float64(sc.rs_bc2)
        R = np.sqrt(np.float64(vs[0])) * rs
        h_code = 1.0 / (np.sqrt(vz[codes[1:]].astype(np.float64)) * R + float(eps))
        hs.append(h_code)
        if h_true is None:
            h_true = 1.0 / (np.sqrt(np.float64(v1[1])) * rs + float(eps))
    hs = np.concatenate(hs)
    assert hs.size >= 10 ** 6
    mean, sd = hs.mean(), hs.std() / np.sqrt(hs.size)
    assert abs(mean - h_true) < 4 * sd + 1e-6 * h_true


def test_bracket_at_and_below_code_points():
    """The ZIP-SR bracket of a value exactly on code point k is [k, k+1] (k
    for the top one, 14), and one binary32 step below it is [k-1, k]."""
    _, _, vz, _ = oracle.tables()
    for k in range(1, 16):
        assert oracle.zipsr_bracket(float(vz[k])) == min(k, 14)
        below = float(np.nextafter(vz[k], np.float32(-1)))
        assert oracle.zipsr_bracket(below) == k - 1
    assert oracle.zipsr_bracket(0.0) == 0


# ---------------------------------------------------------------------------
# ZIP-SR deciding on the whole 32-bit draw (v code 5)
# ---------------------------------------------------------------------------

W_STEP = 2.0 ** -32


def p_low_exact_u32(x, dv, R, eps):
    """Fraction of the 2^32 draw words for which the 32-bit decision keeps the
    lower code point (the decision is monotone in the word; bisection)."""
    k_lo = oracle.zipsr_decide_u32(x, dv, R, eps, 0)
    k_hi = oracle.zipsr_decide_u32(x, dv, R, eps, 0xFFFFFFFF)
    if k_lo == k_hi:
        return (1.0 if k_lo == oracle.zipsr_bracket(x) else 0.0), k_lo
    lo, hi = 0, 1 << 32
    while lo < hi:
        j = (lo + hi) // 2
        if oracle.zipsr_decide_u32(x, dv, R, eps, j) == k_lo:
            lo = j + 1
        else:
            hi = j
    return lo * W_STEP, k_lo


@pytest.mark.parametrize("s,xv,rs_bc2", CASES[::3])
def test_u32_decision_exact_expectation(s, xv, rs_bc2):
    """Over all 2^32 words the 32-bit decision's probability equals the pages'
    formula in binary64 within 2^-32 plus the binary32 conditioning of the
    cell, so E[h(Q)] = h(v) to that resolution."""
    eps = f32(1e-8)
    s = f32(s)
    rs_bc2 = f32(rs_bc2)
    _, _, vz, vzs = oracle.tables()
    v = f32(np.float32(xv) * np.float32(s))
    x = f32(np.float32(v) * (np.float32(1.0) / np.float32(s)))
    R = f32(np.sqrt(np.float32(s)) * np.float32(rs_bc2))
    dv = f32(np.float32(np.sqrt(np.float32(v))) * np.float32(rs_bc2) + np.float32(eps))
    k = oracle.zipsr_bracket(x)
    p, _ = p_low_exact_u32(x, dv, R, eps)
    da = float(vzs[k]) * R + eps
    db = float(vzs[k + 1]) * R + eps
    if db == da:
        return
    p_ref = min(max((1 / dv - 1 / db) / (1 / da - 1 / db), 0.0), 1.0)
    cond = 4 * 2.0 ** -24 * db / (db - da)
    assert abs(p - p_ref) < 1e-6 * cond + W_STEP + cond
    # the binary32 terms B and rhs fix the probability to binary32 precision:
    # p is rhs/B rounded up to a multiple of 2^-32
    B = f32(np.float32(np.float32(db) - np.float32(da)) * np.float32(dv))
    rhs = f32(np.float32(np.float32(db) - np.float32(dv)) * np.float32(da))
    if B > 0 and 0 <= rhs < B:
        assert p == pytest.approx(np.ceil(rhs / B * 2.0 ** 32) * W_STEP, abs=2 * W_STEP)


@pytest.mark.parametrize("v_hat", [1e-2, 3e-3, 1e-3])
def test_zero_cell_has_no_23_bit_bias(v_hat):
    """Values in the cell next to zero where the pages' probability of zero
    is below 2^-23 (b = 2 v, eps = 1e-8, no bias correction).  A 23-bit
    uniform keeps zero with probability 2^-23 at least, several times too
    often, and pushes E[h] far above h(v) (h(0) = 1/eps is huge); ZIP-SR's
    draw from the whole word and the binary64 option (v code 5) both realise
    the probability to within 2^-32 plus 2^-22 relative, so
    |E[h] - h(v)| <= 2^-32 (h(0) - h(b)) + the cell's binary32 conditioning."""
    eps = f32(1e-8)
    s = f32(15 * 2 * v_hat)                         # b = s/15 = 2 v
    v = f32(v_hat)
    x = f32(np.float32(v) * (np.float32(1.0) / np.float32(s)))
    R = f32(np.sqrt(np.float32(s)))
    dv = f32(np.float32(np.sqrt(np.float32(v))) + np.float32(eps))
    assert oracle.zipsr_bracket(x) == 0
    _, _, vz, vzs = oracle.tables()
    da, db = float(vzs[0]) * R + eps, float(vzs[1]) * R + eps
    p_ref = (1 / dv - 1 / db) / (1 / da - 1 / db)
    assert p_ref < 2.0 ** -23
    p23, _ = p_low_exact_u23(x, dv, R, eps)
    p0, _ = p_low_exact(x, dv, R, eps)              # ZIP-SR (v code 0)
    p5, _ = p_low_exact_u32(x, dv, R, eps)          # binary64 option (v code 5)
    assert p23 == U_STEP                            # rounded up to one granule
    cond = 4 * 2.0 ** -24 * db / (db - da) * p_ref
    for p in (p0, p5):
        assert abs(p - p_ref) < 2 * W_STEP + 2.0 ** -22 * p_ref + cond
    e_h = lambda p: p / da + (1 - p) / db          # noqa: E731
    assert e_h(p23) - 1 / dv > 0.5 * (U_STEP - p_ref) * (1 / da - 1 / db)
    for p in (p0, p5):
        assert abs(e_h(p) - 1 / dv) <= (2 * W_STEP + 2.0 ** -22 * p_ref + cond) * (1 / da - 1 / db)
    assert abs(e_h(p0) - 1 / dv) < 1e-3 / dv


def test_block_decisions_follow_the_page_probability_on_the_word():
    """The block step's ZIP-SR codes, element by element: with the draw word
    w of each element (Philox, pinned by its known answers) and the pages'
    keep probability p computed in binary64 from the block's binary32
    quantities, an element whose w 2^-32 lies clearly below p keeps the lower
    code point and one clearly above takes the upper; near-ties (within the
    binary32 conditioning) are skipped.  A decision taken on other bits of
    the word, or on a mis-scaled uniform, fails this."""
    from workloads import bf16_bits, bf16_to_f32
    _, _, vz, vzs = oracle.tables()
    b1, b2, eps = np.float32(0.9), np.float32(0.999), np.float32(1e-8)
    rng = np.random.default_rng(7)
    decisive = 0
    for rep in range(40):
        g = (rng.standard_normal(128) * 1e-3 * np.exp(rng.uniform(-3, 0, 128))).astype(np.float32)
        gb = bf16_bits(g)
        gf = bf16_to_f32(gb)
        seed, tid = 1000 + rep, 3
        sc = oracle.make_scalars(1e-3, b1, b2, eps, t=1, seed=seed)
        w = np.zeros(128, np.float32)
        mc, vc = np.zeros(64, np.uint8), np.zeros(64, np.uint8)
        ms, vs = np.zeros(1, np.float32), np.zeros(1, np.float32)
        oracle.lib().oracle_block4(sc, np.float32(1.0), 0, 0, tid, 0, 128, w, gb, mc, ms, vc, vs)
        codes = np.empty(128, np.int64)
        codes[0::2] = vc & 15
        codes[1::2] = vc >> 4
        # the canonical binary32 quantities of the block (zero prior state)
        omb2 = np.float32(1.0) - b2
        v1 = (omb2 * (gf * gf)).astype(np.float32)
        av = np.float32(v1.max())
        inv = np.float32(1.0) / av
        rs = np.float32(sc.rs_bc2)
        R = np.float32(np.sqrt(av) * rs)
        for i in range(128):
            x = np.float32(v1[i] * inv)
            dv = np.float32(np.float32(np.sqrt(v1[i]) * rs) + eps)
            k = oracle.zipsr_bracket(float(x))
            da = float(np.float32(np.float32(vzs[k]) * R + eps))   # fma: exact enough here
            db = float(np.float32(np.float32(vzs[k + 1]) * R + eps))
            if db == da:
                continue
            p = min(max((1 / float(dv) - 1 / db) / (1 / da - 1 / db), 0.0), 1.0)
            u = oracle.draw_word(seed, 1, tid, 0, i) * 2.0 ** -32
            tol = 1e-5 * db / (db - da) + 2.0 ** -22
            if abs(u - p) <= tol:
                continue
            decisive += 1
            assert codes[i] == (k if u < p else k + 1), (rep, i, u, p, k, codes[i])
    assert decisive > 3000


def test_u32_decision_ends_are_deterministic():
    eps = f32(1e-8)
    R = f32(np.sqrt(np.float32(1e-6)))
    for w in (0, 0x12345678, 0xFFFFFFFF):
        assert oracle.zipsr_decide_u32(0.0, eps, R, eps, w) == 0
        assert oracle.zipsr_decide_u32(1.0, R + eps, R, eps, w) == 15
