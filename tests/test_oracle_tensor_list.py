"""The oracle over a tensor list: threads, partial blocks, checkpoints (CPU)."""
import numpy as np
import pytest

import oracle
from workloads import bf16_bits


def _run(ts, steps, nthreads=1, vcode=0, total_steps=0, seed=11):
    o = oracle.OracleAdamW4(vcode=vcode, seed=seed, total_steps=total_steps, tensors=ts,
                            nthreads=nthreads)
    rng = np.random.default_rng(1)
    ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
    for s in range(steps):
        gs = [bf16_bits((rng.standard_normal(t["numel"]) * 1e-3).astype(np.float32)) for t in ts]
        o.step(ws, gs)
    return o, ws


TS = [dict(numel=4096 + 37, tensor_id=3, weight_decay=0.1),
      dict(numel=4095, tensor_id=5, weight_decay=0.1),
      dict(numel=128 * 40, tensor_id=8, flags=oracle.T_LM_HEAD, weight_decay=0.0),
      dict(numel=9000, tensor_id=9, flags=oracle.T_NORM, weight_decay=0.1)]


@pytest.mark.parametrize("vcode", [0, 1])
def test_threads_do_not_change_results(vcode):
    a, wa = _run(TS, 3, 1, vcode)
    b, wb = _run(TS, 3, 4, vcode)
    assert a.export_state() == b.export_state()
    for x, y in zip(wa, wb):
        assert np.array_equal(x, y)


def test_classification():
    o = oracle.OracleAdamW4(tensors=TS)
    assert [t.fp32 for t in o.tensors] == [False, True, False, True]


def test_partial_block_padding_codes_are_zero():
    o, _ = _run(TS[:1], 2)
    t = o.tensors[0]
    last = t.nb - 1
    valid = t.numel - last * 128                       # 37 valid slots
    mc = t.mcodes[last * 64:(last + 1) * 64]
    vc = t.vcodes[last * 64:(last + 1) * 64]
    assert valid == 37
    assert mc[19] >> 4 == 0 and np.all(mc[20:] == 0)   # slot 37 is the high nibble of byte 18
    assert vc[19] >> 4 == 0 and np.all(vc[20:] == 0)


def test_checkpoint_resume_is_bit_exact():
    ts = TS
    rng = np.random.default_rng(2)
    w0 = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
    grads = [[bf16_bits((rng.standard_normal(t["numel"]) * 1e-3).astype(np.float32))
              for t in ts] for _ in range(6)]
    a = oracle.OracleAdamW4(tensors=ts, total_steps=6)
    wa = [w.copy() for w in w0]
    for g in grads:
        a.step(wa, g)
    b = oracle.OracleAdamW4(tensors=ts, total_steps=6)
    wb = [w.copy() for w in w0]
    for g in grads[:3]:
        b.step(wb, g)
    blob = b.export_state()
    c = oracle.OracleAdamW4(tensors=ts, total_steps=6)
    c.import_state(blob)
    assert c.t == 3
    for g in grads[3:]:
        c.step(wb, g)
    assert c.export_state() == a.export_state()
    for x, y in zip(wa, wb):
        assert np.array_equal(x, y)


def test_lm_head_phase_changes_only_the_head_m_codes():
    """Over the final 10% the LM-head m is rounded stochastically; the other
    tensors and the head's v are untouched by the switch."""
    ts = [dict(numel=128 * 32, tensor_id=0, flags=oracle.T_LM_HEAD),
          dict(numel=128 * 32, tensor_id=1)]
    runs = []
    for T in (0, 10):
        o = oracle.OracleAdamW4(tensors=ts, total_steps=T)
        o.t = 9
        rng = np.random.default_rng(4)
        ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
        gs = [bf16_bits((rng.standard_normal(t["numel"]) * 1e-3).astype(np.float32)) for t in ts]
        o.step(ws, gs)                     # t = 10 > 0.9 T when T = 10
        runs.append(o)
    a, b = runs
    assert not np.array_equal(a.tensors[0].mcodes, b.tensors[0].mcodes)
    assert np.array_equal(a.tensors[0].vcodes, b.tensors[0].vcodes)
    assert np.array_equal(a.tensors[1].mcodes, b.tensors[1].mcodes)


def test_nibble_layout_of_the_codes():
    """Element 2i sits in the low nibble of byte i and 2i+1 in the high one
    (the checkpoint layout).  A block whose only nonzero first moment is
    element 1 (byte 0 = 0xF7: element 0 on the NF4 zero level, element 1 on
    +1) moves weight 1 and leaves weight 0 alone when the gradients are zero."""
    s = oracle.make_scalars(1e-3, 0.9, 0.999, 1e-8, t=5)
    w0 = np.full(128, 0.25, np.float32)
    w = w0.copy()
    g = np.zeros(128, np.uint16)
    mc = np.full(64, 0x77, np.uint8)
    mc[0] = 0xF7
    vc = np.zeros(64, np.uint8)
    ms = np.ones(1, np.float32)
    vs = np.zeros(1, np.float32)
    oracle.lib().oracle_block4(s, np.float32(1.0), 0, 0, 0, 0, 128, w, g, mc, ms, vc, vs)
    assert w[0] == w0[0] and np.all(w[2:] == w0[2:])
    assert w[1] < w0[1] - 1.0
