"""Device status and the kernel's fast-path ranges (needs a B200).

1. Non-finite weights: a step whose updated weights include a NaN or an
   infinity (from a non-finite grad or weight) runs to the end and records it;
   adamw4_sync then returns ADAMW4_ENONFINITE once and clears it.  The faults
   are made on the host (NaN / inf values written into the input buffers);
   nothing faults on the GPU.
2. Fast-path boundaries: the kernel takes the square root and the division
   from the fast sequences only for lanes whose |m1| and v1 lie inside their
   ranges, and the block reciprocals and square root only inside theirs.
   Blocks built around each limit (tiny and huge moment scales, zero first
   moments, a scale in the lowest binade of normal numbers, an eps that turns
   the fast path off) must still give the oracle's bits.
"""
import struct

import numpy as np
import pytest

import oracle
import workloads
from gpu_common import CudaRun, binding

pytestmark = pytest.mark.gpu


def _list():
    return [dict(numel=128 * 40, tensor_id=1, flags=0, weight_decay=0.1),
            dict(numel=128 * 9 + 17, tensor_id=2, flags=0, weight_decay=0.1),
            dict(numel=700, tensor_id=3, flags=0, weight_decay=0.0)]      # fp32 state


@pytest.mark.parametrize("vcode", [0, 1])
def test_nonfinite_weight_is_reported_once(vcode):
    B = binding()
    ts = _list()
    rng = np.random.default_rng(0)
    ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
    run = CudaRun(ts, ws, vcode=vcode)
    try:
        def grads(poison=None):
            gs = [workloads.bf16_bits((rng.standard_normal(t["numel"]) * 1e-3).astype(np.float32))
                  for t in ts]
            if poison is not None:
                i, j, bits = poison
                gs[i][j] = bits
            return gs

        import torch
        run.step(grads())
        run.opt.sync()                                       # finite: OK
        blob0, w0 = run.blob(), run.weights()

        def restore():
            # a non-finite value also reaches the moments of its block; put
            # back the state and the weights from before the poisoned step
            run.opt.load_state_blob(blob0)
            for p, w in zip(run.params, w0):
                p.copy_(torch.from_numpy(w).cuda())

        for poison in ((0, 1000, 0x7FC0),                    # NaN grad, 4-bit tensor
                       (1, 128 * 9 + 3, 0xFF80),             # -inf grad, ragged block
                       (2, 5, 0x7F80)):                      # +inf grad, fp32-state tensor
            run.step(grads(poison))
            with pytest.raises(B.AdamW4Error) as err:
                run.opt.sync()
            assert err.value.code == B.ADAMW4_ENONFINITE
            run.opt.sync()                                   # read and cleared
            assert not np.isfinite(run.weights()[poison[0]]).all()
            restore()
        run.step(grads())
        run.opt.sync()                                       # finite again: OK
        # an infinite weight (finite grads) is reported too
        restore()
        run.params[0][77] = float("inf")
        run.step(grads())
        with pytest.raises(B.AdamW4Error) as err:
            run.opt.sync()
        assert err.value.code == B.ADAMW4_ENONFINITE
    finally:
        run.close()


def _blob(ts, vcode, t, scales, rng_seed=0, seed=0):
    """A checkpoint blob (for an optimizer with key `seed`) whose 4-bit blocks
    carry the given (m scale, v scale) pairs in turn, with codes spread over
    the whole grid (m codes include the NF4 zero level, ZIP-SR v codes include
    0)."""
    rng = np.random.default_rng(rng_seed)
    parts = []
    k = 0
    for tt in ts:
        n, tid = tt["numel"], tt["tensor_id"]
        if oracle.is_fp32_state(n, tt["flags"]):
            m = (rng.standard_normal(n) * 1e-4).astype(np.float32)
            v = (rng.random(n) * 1e-7).astype(np.float32)
            parts += [struct.pack("<IIq", tid, 1, n), m.tobytes(), v.tobytes()]
            continue
        nb = (n + 127) // 128
        mc = rng.integers(0, 16, nb * 128).astype(np.uint8)
        vc = rng.integers(0, 16, nb * 128).astype(np.uint8)
        mc[n:] = 0
        vc[n:] = 0
        ms = np.empty(nb, np.float32)
        vs = np.empty(nb, np.float32)
        for b in range(nb):
            ms[b], vs[b] = scales[k % len(scales)]
            k += 1
        parts += [struct.pack("<IIq", tid, 0, n), (mc[0::2] | (mc[1::2] << 4)).tobytes(),
                  (vc[0::2] | (vc[1::2] << 4)).tobytes(), ms.tobytes(), vs.tobytes()]
    payload = b"".join(parts)
    return b"ADAMW4S1" + struct.pack("<IIqQQ", len(ts), vcode, t, seed, len(payload)) + payload


# (m scale, v scale) of successive blocks, around the limits of the fast
# ranges: |m1| in [2^-60, 2^100 eps], v1 in [2^-100, 2^64], block reciprocal
# for scales in [2^-125, 2^125], block square root in [2^-100, 2^100]
SCALES = [(1e-3, 1e-6),            # ordinary: every lane fast
          (1e-20, 1e-6),           # |m1| below 2^-60 (~8.7e-19)
          (1.2e-18, 1e-6),         # |m1| straddles 2^-60 across lanes
          (1e-3, 1e-32),           # v1 below 2^-100 (~7.9e-31)
          (1e-3, 1.3e-30),         # v1 straddles 2^-100
          (1e-3, 1e21),            # v1 above 2^64 (~1.8e19)
          (1e-3, 2e19),            # v1 straddles 2^64
          (1e23, 1e-6),            # |m1| above 2^100 eps (~1.3e22 at eps 1e-8)
          (1.5e-38, 1.5e-38),      # block scales in [2^-126, 2^-125): IEEE reciprocal
          (1e38, 1e31),            # block scales above 2^125 and 2^100
          (0.0, 0.0),              # zero block
          (1e-3, 0.0)]             # v zero: every v1 = (1-b2) g^2 only


@pytest.mark.parametrize("vcode", [0, 1, 5])
@pytest.mark.parametrize("eps", [1e-8, 2.0 ** -60, 1e-30], ids=["eps1e-8", "eps2^-60", "eps1e-30"])
def test_fast_path_boundaries_match_the_oracle(vcode, eps):
    ts = _list()
    ts.append(dict(numel=128 * 24, tensor_id=4, flags=0, weight_decay=0.1))
    rng = np.random.default_rng(3)
    ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
    blob = _blob(ts, vcode, 5, SCALES, rng_seed=vcode)

    def grads(s):
        r = np.random.default_rng(50 + s)
        out = []
        for t in ts:
            g = (r.standard_normal(t["numel"]) * 1e-3).astype(np.float32)
            g[r.random(t["numel"]) < 0.2] = 0.0           # exact zeros: m1 may vanish
            g[r.random(t["numel"]) < 0.05] *= 1e-14        # squares near 2^-100
            out.append(workloads.bf16_bits(g))
        return out
    import gpu_common
    gpu = gpu_common.CudaRun(ts, ws, vcode=vcode, eps=eps, blob=blob)
    ref = gpu_common.oracle_for(ts, vcode=vcode, eps=eps)
    ref.import_state(blob)
    wr = [w.copy() for w in ws]
    try:
        for s in range(1, 4):
            gs = grads(s)
            old = [w.copy() for w in wr]
            gpu.step(gs)
            ref.step(wr, gs)
            wg = gpu.weights()
            for i, (a, b, o) in enumerate(zip(wg, wr, old)):
                gpu_common.assert_weights_close(a, b, o, f"v{vcode} eps {eps} step {s} tensor {i}")
            gpu_common.assert_state_equal(gpu.blob(), ref.export_state(), vcode,
                                          f"v{vcode} eps {eps} step {s}")
    finally:
        gpu.close()
