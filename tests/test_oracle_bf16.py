"""Pins of the oracle's bf16 weight storage (CPU only).

bf16 weights are a lower-memory option of the library, not part of the pages:
the step reads them exactly, computes in binary32 as for fp32 weights, and
stores the result rounded to the nearest bf16, ties to even (IEEE 754)."""
import numpy as np
import torch

import oracle


def _edge_values():
    rng = np.random.default_rng(3)
    # wide random spread of magnitudes and both signs
    with np.errstate(over="ignore"):           # a few overflow to +-inf, kept on purpose
        x = (rng.standard_normal(20000) * np.exp(rng.uniform(-90, 88, 20000))).astype(np.float32)
    bits = rng.integers(0, 1 << 16, 4000, dtype=np.uint32) << 16
    # exact ties with an even and an odd kept bit, just below and just above
    ties = np.concatenate([bits | 0x8000, bits | 0x7FFF, bits | 0x8001,
                           (bits | 0x18000) & 0xFFFFFFFF])
    specials = np.array([0x00000000, 0x80000000, 0x00000001, 0x00008000, 0x00018000,
                         0x007FFFFF, 0x00800000, 0x7F7FFFFF, 0xFF7FFFFF, 0x7F7F8000,
                         0x7F800000, 0xFF800000, 0x3F808000, 0x3F818000], np.uint32)
    allbits = np.concatenate([x.view(np.uint32), ties.astype(np.uint32), specials])
    keep = (allbits & 0x7FFFFFFF) <= 0x7F800000          # no NaNs here
    return allbits[keep].view(np.float32)


def test_round_matches_the_library_conversion():
    """torch's float32 -> bfloat16 conversion rounds to nearest even."""
    x = _edge_values()
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.round_bf16(x), want)


def test_round_is_the_nearest_bf16_by_brute_force():
    x = _edge_values()
    x = x[np.isfinite(x) & (np.abs(x) < 3.3e38)]
    b = oracle.round_bf16(x).astype(np.int64)

    def val(bb):
        return ((bb.astype(np.uint32) & 0xFFFF) << 16).view(np.float32).astype(np.float64)
    d0 = np.abs(val(b) - x.astype(np.float64))
    for step in (-1, 1):                  # the neighbours in the same sign's ordering
        nb = b + step
        ok = ((nb & 0x7FFF) <= 0x7F7F) & ((nb & 0x8000) == (b & 0x8000))
        dn = np.abs(val(nb) - x.astype(np.float64))
        assert (d0[ok] <= dn[ok]).all()
        tie = ok & (d0 == dn)
        assert (b[tie] % 2 == 0).all()    # ties keep the even pattern


def test_nan_stays_nan():
    b = oracle.f32_to_bf16(float("nan"))
    assert (b & 0x7F80) == 0x7F80 and (b & 0x7F) != 0


def test_bf16_weight_step_is_the_fp32_step_rounded():
    """The moments do not depend on w, and the update is computed in binary32
    from the exactly widened weight, so each step of the bf16 path equals the
    fp32 path's step from the same (bf16) weights, rounded."""
    specs = [dict(numel=128 * 40 + 9, tensor_id=1, flags=0, weight_decay=0.1),
             dict(numel=5000, tensor_id=2, flags=oracle.T_NORM, weight_decay=0.0),
             dict(numel=4096, tensor_id=3, flags=oracle.T_LM_HEAD, weight_decay=0.1)]
    for vcode in (0, 1):
        rng = np.random.default_rng(vcode)
        wb = [oracle.round_bf16((rng.standard_normal(s["numel"]) * 0.02).astype(np.float32))
              for s in specs]
        bf = oracle.OracleAdamW4(vcode=vcode, seed=4, total_steps=3,
                                 tensors=[dict(s, flags=s["flags"] | oracle.T_BF16_PARAM)
                                          for s in specs])
        f32 = oracle.OracleAdamW4(vcode=vcode, seed=4, total_steps=3, tensors=specs)
        for t in range(3):
            g = [np.asarray(torch.from_numpy((rng.standard_normal(s["numel"]) * 1e-3)
                                             .astype(np.float32)).to(torch.bfloat16)
                            .view(torch.int16).numpy().view(np.uint16)) for s in specs]
            wf = [(w.astype(np.uint32) << 16).view(np.float32) for w in wb]
            f32.step(wf, g)
            bf.step(wb, g)
            for a, b in zip(wb, wf):
                assert np.array_equal(a, oracle.round_bf16(b))
            assert bf.export_state() == f32.export_state()
