"""Pins of the oracle's AdamW arithmetic, step scalars and ordering (CPU only)."""
import numpy as np
import pytest
import torch

import oracle
from workloads import bf16_bits, bf16_to_f32


def test_step_scalars_closed_form():
    s = oracle.make_scalars(2e-3, 0.9, 0.999, 1e-8, t=7, total_steps=100)
    b1, b2 = float(np.float32(0.9)), float(np.float32(0.999))
    assert s.step_size == np.float32(float(np.float32(2e-3)) / (1 - b1 ** 7))
    assert s.rs_bc2 == np.float32(1 / np.sqrt(1 - b2 ** 7))
    assert s.omb1 == np.float32(1 - b1) and s.omb2 == np.float32(1 - b2)
    assert not s.lm_sr_active


@pytest.mark.parametrize("t,T,on", [(90, 100, False), (91, 100, True), (100, 100, True),
                                    (900, 1000, False), (901, 1000, True), (5, 0, False)])
def test_final_ten_percent_phase(t, T, on):
    """"final 10% of training" (ZIP-SR 4-bit AdamW, ZE-EDEN paragraph): on
    when 10 t > 9 T."""
    assert bool(oracle.make_scalars(1e-3, 0.9, 0.999, 1e-8, t=t, total_steps=T).lm_sr_active) == on


def test_fp32_state_path_matches_torch_adamw():
    """With every tensor on fp32 state the oracle is plain AdamW; it must
    agree with torch.optim.AdamW (fp32, CPU, foreach=False) on w to 1e-6
    relative (to the larger of the old and new |w|) at every one of 10 steps (the two order their binary32
    operations differently, so not bit for bit)."""
    rng = np.random.default_rng(0)
    n = 3000
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    o = oracle.OracleAdamW4(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
                            tensors=[dict(numel=n, tensor_id=0, weight_decay=0.1)])
    assert o.tensors[0].fp32
    p = torch.nn.Parameter(torch.from_numpy(w0.copy()))
    # the ABI's hyper-parameters are binary32: give torch the same values
    f = lambda x: float(np.float32(x))
    opt = torch.optim.AdamW([p], lr=f(1e-3), betas=(f(0.9), f(0.999)), eps=f(1e-8),
                            weight_decay=f(0.1), foreach=False)
    w = w0.copy()
    for _ in range(10):
        gb = bf16_bits((rng.standard_normal(n) * 1e-3).astype(np.float32))
        before = w.copy()
        o.step([w], [gb])
        p.grad = torch.from_numpy(bf16_to_f32(gb).copy())
        opt.step()
        wt = p.detach().numpy()
        scale = np.maximum(np.abs(before), np.abs(wt)).astype(np.float64)
        assert np.all(np.abs(w.astype(np.float64) - wt) <= 1e-6 * scale)
        # the update itself agrees to 1e-4 relative, up to a few ulps of w
        ulp = np.spacing(np.abs(before)).astype(np.float64)
        upd_o = w.astype(np.float64) - before
        upd_t = wt.astype(np.float64) - before
        assert np.all(np.abs(upd_o - upd_t) <= 1e-4 * np.abs(upd_t) + 4 * ulp)
        # continue both from torch's weights and moments
        w = wt.astype(np.float32).copy()
        o.tensors[0].m = opt.state[p]["exp_avg"].numpy().astype(np.float32).copy()
        o.tensors[0].v = opt.state[p]["exp_avg_sq"].numpy().astype(np.float32).copy()


def test_update_elem_values():
    s = oracle.make_scalars(1e-3, 0.9, 0.999, 1e-8, t=1)
    den, w, m1, v1 = oracle.update_elem(s, 1.0, 1e-3, 0.0, 0.0, 0.5)
    # t = 1: m-hat = g, v-hat = g^2, so the step is lr * g / (|g| + eps)
    assert m1 == pytest.approx(1e-4, rel=1e-6)
    assert v1 == pytest.approx(1e-9, rel=1e-6)
    assert w == pytest.approx(0.5 - 1e-3 * 1e-3 / (1e-3 + 1e-8), rel=1e-7)
    assert den == pytest.approx(1e-3 + 1e-8, rel=1e-6)


def test_weights_updated_before_quantising():
    """"Update weights before quantizing the working moments" (ZIP-SR /
    ZE-EDEN, Core equation): the quantiser cannot change w at step t, only
    from step t+1 on.  ZIP-SR and ZE-EDEN give identical w after one step from
    zero state and differ after the second."""
    rng = np.random.default_rng(3)
    n = 8192
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    gs = [bf16_bits((rng.standard_normal(n) * 1e-3).astype(np.float32)) for _ in range(2)]
    ws = []
    for vcode in (0, 1):
        o = oracle.OracleAdamW4(vcode=vcode, tensors=[dict(numel=n, tensor_id=0,
                                                           weight_decay=0.1)])
        w = w0.copy()
        o.step([w], [gs[0]])
        w1 = w.copy()
        o.step([w], [gs[1]])
        ws.append((w1, w.copy()))
    assert np.array_equal(ws[0][0], ws[1][0])
    assert not np.array_equal(ws[0][1], ws[1][1])


def test_quantised_path_tracks_fp32_adamw():
    """A 4-bit run stays close to the fp32 run over 20 steps: the relative
    gap of the accumulated update is small (a coarse sanity bound, not a
    claim of the pages)."""
    rng = np.random.default_rng(5)
    n = 128 * 64
    w0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    runs = {}
    for name, flags in (("q", 0), ("f", 4)):
        for vcode in (0, 1):
            o = oracle.OracleAdamW4(vcode=vcode, tensors=[dict(numel=n, tensor_id=0,
                                                               flags=flags, weight_decay=0.0)])
            w = w0.copy()
            r = np.random.default_rng(9)
            for _ in range(20):
                o.step([w], [bf16_bits((r.standard_normal(n) * 1e-3).astype(np.float32))])
            runs[(name, vcode)] = w - w0
    for vcode in (0, 1):
        d = runs[("q", vcode)] - runs[("f", vcode)]
        assert np.linalg.norm(d) < 0.25 * np.linalg.norm(runs[("f", vcode)])
