"""Pins of the oracle's counter-based generator (CPU only)."""
import os

import numpy as np

import oracle


def _kat(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "philox4x32_10_kat.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if not line:
                continue
            words = [int(x, 16) for x in line]
            rows.append((words[0:4], words[4:6], words[6:10]))
    return rows


def test_known_answer_vectors(golden_dir):
    rows = _kat(golden_dir)
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = oracle.philox4x32_10(ctr, key)
        assert [int(x) for x in got] == want


def test_draw_keying_fields_each_change_the_word():
    base = oracle.draw_word(7, 5, 3, 0, 1000)
    assert oracle.draw_word(8, 5, 3, 0, 1000) != base          # seed
    assert oracle.draw_word(7, 6, 3, 0, 1000) != base          # step
    assert oracle.draw_word(7, 5, 4, 0, 1000) != base          # tensor
    assert oracle.draw_word(7, 5, 3, 1, 1000) != base          # stream
    assert oracle.draw_word(7, 5, 3, 0, 1001) != base          # element


def test_draw_is_word_e_mod_4_of_one_call():
    seed, t, tid, stream = (0x1234567890ABCDEF, 77, 9, 1)
    for e in [0, 1, 2, 3, 4, 4099, (1 << 34) + 6]:
        q = e >> 2
        out = oracle.philox4x32_10([q & 0xFFFFFFFF, q >> 32, t, tid * 2 + stream],
                                   [seed & 0xFFFFFFFF, seed >> 32])
        assert oracle.draw_word(seed, t, tid, stream, e) == int(out[e & 3])


def test_uniform_range_and_granularity():
    """u is the word's low 23 bits times 2^-23."""
    assert oracle.uniform(0) == 0.0
    assert oracle.uniform(0xFFFFFFFF) == 1.0 - 2.0 ** -23
    assert oracle.uniform(1) == 2.0 ** -23
    assert oracle.uniform(1 << 23) == 0.0
    assert oracle.uniform(0x12345678) == (0x12345678 & 0x7FFFFF) * 2.0 ** -23


def test_uniform_moments():
    # 2^16 draws: mean 1/2 and variance 1/12 within 5 sigma.
    n = 1 << 16
    u = np.array([oracle.uniform(oracle.draw_word(1, 1, 0, 0, e)) for e in range(n)])
    assert abs(u.mean() - 0.5) < 5 * np.sqrt(1 / 12 / n)
    assert abs(u.var() - 1 / 12) < 5 * np.sqrt(1 / 180 / n)
