"""bf16 weights on one B200 (parity through the C ABI).

Tensors flagged ADAMW4_T_BF16_PARAM keep bf16 weights: the kernel widens them
exactly, steps in binary32 and stores the nearest bf16.  A mixed list (bf16
and fp32 weights, 4-bit and fp32 state, ragged tails, an LM head in its
final-10% phase, denormal weights) against the oracle, bit for bit."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_common import assert_state_equal, assert_weights_close, binding, oracle_for

pytestmark = pytest.mark.gpu

BF = oracle.T_BF16_PARAM
SPECS = [dict(numel=128 * 500 + 3, tensor_id=1, flags=BF, weight_decay=0.1),
         dict(numel=128 * 300, tensor_id=2, flags=0, weight_decay=0.1),
         dict(numel=4096, tensor_id=3, flags=BF | oracle.T_LM_HEAD, weight_decay=0.0),
         dict(numel=5000, tensor_id=4, flags=BF | oracle.T_NORM, weight_decay=0.0),
         dict(numel=1000, tensor_id=5, flags=BF, weight_decay=0.1),
         dict(numel=128 * 64, tensor_id=6, flags=BF, weight_decay=0.1),
         dict(numel=128 * 40 + 77, tensor_id=7, flags=0, weight_decay=0.05)]
STEPS = 3


def _inputs():
    rng = np.random.default_rng(11)
    ws = []
    for s in SPECS:
        w = (rng.standard_normal(s["numel"]) * 0.02).astype(np.float32)
        if s["tensor_id"] == 6:
            w[:2048] = (rng.standard_normal(2048) * 1e-39).astype(np.float32)   # denormal
        ws.append(oracle.round_bf16(w) if s["flags"] & BF else w)
    gs = [[workloads.bf16_bits((np.random.default_rng(70 * t + i).standard_normal(s["numel"])
                                * 1e-3).astype(np.float32)) for i, s in enumerate(SPECS)]
          for t in range(STEPS)]
    return ws, gs


def _device(torch, w):
    if w.dtype == np.uint16:
        return torch.from_numpy(w.view(np.int16).copy()).cuda().view(torch.bfloat16)
    return torch.from_numpy(w.copy()).cuda()


def _host(torch, p):
    if p.dtype == torch.bfloat16:
        return p.view(torch.int16).cpu().numpy().view(np.uint16)
    return p.cpu().numpy()


@pytest.mark.parametrize("vcode", [0, 1, 2, 3, 4, 5])
def test_bf16_weights_match_the_oracle(vcode):
    import torch
    B = binding()
    ws, gs = _inputs()
    params = [_device(torch, w) for w in ws]
    grads = [torch.zeros(s["numel"], dtype=torch.bfloat16, device="cuda") for s in SPECS]
    opt = B.AdamW4(params, grads, [dict(s, flags=s["flags"] & ~BF) for s in SPECS], vcode=vcode,
                   seed=8, total_steps=STEPS)
    ref = oracle_for(SPECS, vcode=vcode, seed=8, total_steps=STEPS)
    wref = [w.copy() for w in ws]
    try:
        for t in range(STEPS):
            for g, hg in zip(grads, gs[t]):
                g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
            opt.step()
            old = [w.copy() for w in wref]
            ref.step(wref, gs[t])
            torch.cuda.synchronize()
            for i, (p, s) in enumerate(zip(params, SPECS)):
                got = _host(torch, p)
                if s["flags"] & BF:
                    diff = np.nonzero(got != wref[i])[0]
                    assert diff.size == 0, (f"step {t + 1} tensor {i}: {diff.size} bf16 weights "
                                            f"differ, first at {diff[0]}: gpu {got[diff[0]]:#06x} "
                                            f"oracle {wref[i][diff[0]]:#06x}")
                else:
                    assert_weights_close(got, wref[i], old[i], f"step {t + 1} tensor {i}")
            assert_state_equal(opt.state_dict_blob(), ref.export_state(), vcode, f"step {t + 1}")
    finally:
        opt.close()


def test_bf16_weights_through_host_buffers():
    """adamw4_step_host copies bf16 weights back as 2-byte values."""
    import torch
    B = binding()
    ws, gs = _inputs()
    params = [_device(torch, w) for w in ws]
    grads = [torch.zeros(s["numel"], dtype=torch.bfloat16, device="cuda") for s in SPECS]
    opt = B.AdamW4(params, grads, SPECS, vcode=0, seed=8, total_steps=STEPS)
    ref = oracle_for(SPECS, vcode=0, seed=8, total_steps=STEPS)
    wref = [w.copy() for w in ws]
    try:
        hg = [np.ascontiguousarray(g) for g in gs[0]]
        hp = [np.zeros_like(w) for w in ws]
        B.adamw4_step_host(opt.handle, 1e-3, [g.ctypes.data for g in hg],
                           [p.ctypes.data for p in hp], None)
        ref.step(wref, gs[0])
        for i, s in enumerate(SPECS):
            if s["flags"] & BF:
                assert np.array_equal(hp[i], wref[i]), f"tensor {i}"
                assert np.array_equal(hp[i], _host(torch, params[i])), f"tensor {i}"
            else:
                assert_weights_close(hp[i], wref[i], ws[i], f"tensor {i}")
    finally:
        opt.close()
