"""Pins of the oracle's counter-based generator (CPU only)."""
import ctypes
import ctypes.util
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


def test_uniform32_rounds_the_whole_word():
    """ZIP-SR's uniform is the whole word rounded to the nearest binary32
    (ties to even), times 2^-32: exact below 2^24, relative rounding above."""
    assert oracle.uniform32(0) == 0.0
    assert oracle.uniform32(1) == 2.0 ** -32
    assert oracle.uniform32(12345) == 12345 * 2.0 ** -32
    assert oracle.uniform32((1 << 24) - 1) == ((1 << 24) - 1) * 2.0 ** -32
    assert oracle.uniform32((1 << 24) + 1) == 2.0 ** -8           # tie to even: down
    assert oracle.uniform32((1 << 24) + 3) == ((1 << 24) + 4) * 2.0 ** -32   # tie: up to even
    assert oracle.uniform32(0x80000000) == 0.5
    assert oracle.uniform32(0x80000080) == 0.5                    # 2^31 + 2^7: tie, even
    assert oracle.uniform32(0x80000081) == 0.5 + 2.0 ** -24
    assert oracle.uniform32(0xFFFFFFFF) == 1.0                    # rounds up to 2^32
    assert oracle.uniform32(0xFFFFFF7F) == 1.0 - 2.0 ** -24
    rng = np.random.default_rng(5)
    for w in rng.integers(0, 1 << 32, 2000, dtype=np.uint64):
        w = int(w)
        u = oracle.uniform32(w)
        # the nearest binary32 to w: no binary32 is closer
        f = np.float32(u * 2.0 ** 32)
        assert float(f) == u * 2.0 ** 32
        assert abs(float(f) - w) <= abs(float(np.nextafter(f, np.float32(np.inf))) - w)
        assert abs(float(f) - w) <= abs(float(np.nextafter(f, np.float32(0))) - w)


def test_uniform_moments():
    # 2^16 draws: mean 1/2 and variance 1/12 within 5 sigma.
    n = 1 << 16
    words = [oracle.draw_word(1, 1, 0, 0, e) for e in range(n)]
    for u in (np.array([oracle.uniform(w) for w in words]),
              np.array([oracle.uniform32(w) for w in words])):
        assert abs(u.mean() - 0.5) < 5 * np.sqrt(1 / 12 / n)
        assert abs(u.var() - 1 / 12) < 5 * np.sqrt(1 / 180 / n)


def _curand():
    for cand in ("/usr/local/cuda/lib64/libcurand.so", ctypes.util.find_library("curand")):
        if cand:
            try:
                return ctypes.CDLL(cand)
            except OSError:
                pass
    return None


def _curand_quads(L, seed, nquads, first_quad):
    """Words of cuRAND's host Philox4x32-10 generator (it runs on the CPU)."""
    gen = ctypes.c_void_p()
    assert L.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0   # PHILOX4_32_10
    try:
        assert L.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert L.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(4 * first_quad)) == 0
        buf = (ctypes.c_uint32 * (4 * nquads))()
        assert L.curandGenerate(gen, buf, 4 * nquads) == 0
    finally:
        L.curandDestroyGenerator(gen)
    return np.array(buf, dtype=np.uint32).reshape(-1, 4)


def test_matches_the_curand_library_generator():
    """cuRAND's Philox4x32-10 (host generator, library code run on the CPU):
    key = (seed lo, seed hi), and its output quad q is the block of counter
    (q >> 16 as a 64-bit value in words 0-1, q & 0xFFFF in word 2, 0 in
    word 3).  Seeds and offsets make every key bit and counter words 0-2
    matter; word 3 is covered by the known-answer vectors."""
    L = _curand()
    assert L is not None, "libcurand from the CUDA toolkit is needed"
    for seed in (0, 1, 0x0123456789ABCDEF, (1 << 64) - 1):
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for q0 in (0, 65536 * 3 + 17, (1 << 48) + 5 * 65536 + 9, (1 << 61) + 65530):
            w = _curand_quads(L, seed, 12, q0)
            for i in range(12):
                q = q0 + i
                ctr = [(q >> 16) & 0xFFFFFFFF, (q >> 48) & 0xFFFFFFFF, q & 0xFFFF, 0]
                assert [int(x) for x in oracle.philox4x32_10(ctr, key)] == [int(x) for x in w[i]], \
                    (hex(seed), q)
