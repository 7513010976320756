"""GPU parity: the CUDA path through the C ABI against the oracle, element by
element, on seeded synthetic inputs (needs a B200)."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_common import (CudaRun, assert_state_equal, assert_weights_close, binding, oracle_for,
                        parse_blob, run_both)

pytestmark = pytest.mark.gpu


def _grads_fn(name, ts):
    return lambda s: workloads.host_grads(name, ts, s)


def test_single_65k_zipsr_10_steps():
    """65,536 elements (512 blocks), 10 steps, ZIP-SR, NF4 m; 10% of the
    coordinates carry gradients 1e-4 smaller so v visits the near-zero cell."""
    ts = workloads.tensor_list("single-65k")
    ws = workloads.host_weights("single-65k", ts)
    run_both(ts, ws, _grads_fn("single-65k", ts), 10, vcode=0, check_every_step=True,
             what="single-65k")


@pytest.mark.parametrize("vcode", [2, 3, 4, 5])
def test_single_65k_state_space_variants_10_steps(vcode):
    """The state-space variants (zero-inclusive nearest and stochastic
    rounding, zero-excluded floor without rescale) on the 65,536-element
    workload with its near-zero coordinates, 10 steps."""
    ts = workloads.tensor_list("single-65k")
    ws = workloads.host_weights("single-65k", ts)
    run_both(ts, ws, _grads_fn("single-65k", ts), 10, vcode=vcode, seed=12,
             check_every_step=True, what=f"single-65k v{vcode}")


def test_single_4m_zeeden_20_steps():
    """4,194,304 elements (32,768 blocks), 20 steps, ZE-EDEN, per-block
    gradient scales log-uniform over three decades."""
    ts = workloads.tensor_list("single-4m")
    ws = workloads.host_weights("single-4m", ts)
    run_both(ts, ws, _grads_fn("single-4m", ts), 20, vcode=1, what="single-4m")


RAGGED = [1, 7, 100, 4095, 4096, 4097, 4096 + 5, 4096 + 37, 4096 + 120, 128 * 37 + 64, 8192]


# ZIP-SR, ZE-EDEN, the three state-space variants, and ZIP-SR on 32-bit draws
ALL_VCODES = [0, 1, 2, 3, 4, 5]


@pytest.mark.parametrize("vcode", ALL_VCODES)
def test_ragged_mixed_tensor_list(vcode):
    """Every tail shape: whole blocks, a last lane with 1..7 values, lanes with
    nothing, fp32-state tensors below 4096 and flagged NORM / FP32_STATE,
    per-tensor weight decay, an LM head inside its final-10% phase."""
    ts = []
    for i, n in enumerate(RAGGED):
        ts.append(dict(numel=n, tensor_id=100 + 3 * i, flags=0, weight_decay=0.01 * i))
    ts.append(dict(numel=5000, tensor_id=7, flags=workloads.T_NORM, weight_decay=0.0))
    ts.append(dict(numel=4224, tensor_id=8, flags=workloads.T_FP32_STATE, weight_decay=0.1))
    ts.append(dict(numel=128 * 50 + 3, tensor_id=9, flags=workloads.T_LM_HEAD, weight_decay=0.1))
    rng = np.random.default_rng(vcode)
    ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]

    def grads(s):
        r = np.random.default_rng(1000 + s)
        return [workloads.bf16_bits((r.standard_normal(t["numel"]) * 1e-3
                                     * 10.0 ** r.uniform(-4, 0)).astype(np.float32)) for t in ts]
    run_both(ts, ws, grads, 6, vcode=vcode, seed=0xDEADBEEFCAFE, total_steps=6,
             check_every_step=True, what=f"ragged v{vcode}")


@pytest.mark.parametrize("vcode", ALL_VCODES)
def test_degenerate_values(vcode):
    """All-zero gradients (blocks stay exactly zero, then decay onto code
    points), gradients whose squares are subnormal, single huge outliers in a
    block, and lr = 0."""
    n = 128 * 24
    ts = [dict(numel=n, tensor_id=1, weight_decay=0.1), dict(numel=n, tensor_id=2, weight_decay=0.0)]
    rng = np.random.default_rng(5)
    ws = [(rng.standard_normal(n) * 0.02).astype(np.float32) for _ in ts]

    def grads(s):
        r = np.random.default_rng(s)
        out = []
        for _ in ts:
            g = (r.standard_normal(n) * 1e-3).astype(np.float32)
            if s in (3, 4):
                g[:] = 0                               # quiet steps: x on code points
            g[0:128] = 0                               # an all-zero block, always
            g[128:256] = np.float32(1e-21)             # g^2 subnormal
            g[256:384] *= np.float32(1e-6)
            g[300] = np.float32(5.0)                   # outlier
            out.append(workloads.bf16_bits(g))
        return out
    run_both(ts, ws, grads, 6, vcode=vcode, check_every_step=True, what=f"degenerate v{vcode}")
    # lr = 0 leaves the weights unchanged (decay 1 - 0*wd = 1)
    gpu = CudaRun(ts, ws, vcode=vcode)
    try:
        gpu.step(grads(1), lr=0.0)
        for a, b in zip(gpu.weights(), ws):
            assert np.array_equal(a, b)
    finally:
        gpu.close()


def test_empty_tensor_list():
    import torch
    B = binding()
    cfg = B.adamw4_config(1e-3, 0.9, 0.999, 1e-8, 0, 0, 0)
    h = B.adamw4_create(cfg, [], 0)
    B.adamw4_step(h, 1e-3, None)
    torch.cuda.synchronize()
    assert B.adamw4_get_step(h) == 1
    assert B.adamw4_state_bytes(h) == 0
    B.adamw4_destroy(h)


def test_checkpoint_resume_bit_exact():
    ts = workloads.tensor_list("single-65k") + [dict(numel=3000, tensor_id=1, flags=0,
                                                     weight_decay=0.1)]
    ws = [(np.random.default_rng(i).standard_normal(t["numel"]) * 0.02).astype(np.float32)
          for i, t in enumerate(ts)]
    gfn = lambda s: [workloads.bf16_bits((np.random.default_rng(50 + s).standard_normal(
        t["numel"]) * 1e-3).astype(np.float32)) for t in ts]
    a = CudaRun(ts, ws)
    for s in range(1, 7):
        a.step(gfn(s))
    wa, ba = a.weights(), a.blob()
    a.close()
    b = CudaRun(ts, ws)
    for s in range(1, 4):
        b.step(gfn(s))
    mid, wmid = b.blob(), b.weights()
    b.close()
    c = CudaRun(ts, wmid, blob=mid)
    assert c.opt.t == 3
    for s in range(4, 7):
        c.step(gfn(s))
    assert c.blob() == ba
    for x, y in zip(c.weights(), wa):
        assert np.array_equal(x, y)
    c.close()


def test_state_bytes_match_layout():
    B = binding()
    ts = workloads.tensor_list("microlm-p4")
    ws = [np.zeros(t["numel"], np.float32) for t in ts]
    g = CudaRun(ts, ws)
    try:
        assert g.opt.state_bytes() == 157952
        assert g.opt.state_bytes() == oracle_for(ts).state_bytes()
    finally:
        g.close()


def test_host_buffer_step_matches_device_step():
    """adamw4_step_host (grads from pinned host memory, params copied back)
    gives exactly what the device-resident step gives."""
    import torch
    B = binding()
    ts = workloads.tensor_list("single-65k") + [dict(numel=1000, tensor_id=5, flags=0,
                                                     weight_decay=0.1)]
    ws = [(np.random.default_rng(i).standard_normal(t["numel"]) * 0.02).astype(np.float32)
          for i, t in enumerate(ts)]
    gs = [workloads.bf16_bits((np.random.default_rng(9).standard_normal(t["numel"]) * 1e-3)
                              .astype(np.float32)) for t in ts]
    a = CudaRun(ts, ws)
    a.step(gs)
    wa = a.weights()
    a.close()
    b = CudaRun(ts, ws)
    hg = [torch.from_numpy(g.view(np.int16)).pin_memory() for g in gs]
    hp = [torch.empty(t["numel"], dtype=torch.float32).pin_memory() for t in ts]
    B.adamw4_step_host(b.opt.handle, 1e-3, [x.data_ptr() for x in hg], [x.data_ptr() for x in hp],
                       torch.cuda.current_stream().cuda_stream)
    for x, y in zip(hp, wa):
        assert np.array_equal(x.numpy(), y)
    b.close()


def test_pipeline_wait_timeout_is_reported_and_context_survives():
    """Failure detection without a GPU fault: the test hook marks the kernel's
    pipeline stages as filled without issuing copies, so every stage wait runs
    out after its one-second limit; adamw4_sync reports ADAMW4_ETIMEOUT and the
    next step on the same handle and context completes normally."""
    import torch
    B = binding()
    ts = workloads.tensor_list("single-65k")
    ws = workloads.host_weights("single-65k", ts)
    g = CudaRun(ts, ws)
    try:
        B.adamw4_inject_fault(g.opt.handle, B.ADAMW4_FAULT_STALL_PIPELINE)
        g.step(workloads.host_grads("single-65k", ts, 1))
        with pytest.raises(B.AdamW4Error) as err:
            g.opt.sync()
        assert err.value.code == B.ADAMW4_ETIMEOUT
        g.opt.sync()                      # the status word was cleared
        g.step(workloads.host_grads("single-65k", ts, 2))
        g.opt.sync()
        assert all(np.isfinite(w).all() for w in g.weights())
    finally:
        g.close()


def test_pipelined_host_step_cuts_tensors_anywhere():
    """adamw4_step_host pipelines pieces of whole units; with 7-unit pieces
    every tensor of a mixed list (ragged, fp32-state, bf16 weights) is cut at
    several places.  Weights and state equal the one-launch device step."""
    import os
    import torch
    B = binding()
    ts = [dict(numel=65536, tensor_id=0, flags=0, weight_decay=0.1),
          dict(numel=1000, tensor_id=5, flags=0, weight_decay=0.1),
          dict(numel=4096 + 37, tensor_id=6, flags=workloads.T_LM_HEAD, weight_decay=0.0),
          dict(numel=5000, tensor_id=7, flags=workloads.T_NORM, weight_decay=0.0),
          dict(numel=128 * 50 + 3, tensor_id=8, flags=B.ADAMW4_T_BF16_PARAM, weight_decay=0.1)]
    bf = [bool(t["flags"] & B.ADAMW4_T_BF16_PARAM) for t in ts]

    def weights0():
        out = []
        for i, t in enumerate(ts):
            w = torch.from_numpy((np.random.default_rng(i).standard_normal(t["numel"]) * 0.02)
                                 .astype(np.float32))
            out.append(w.to(torch.bfloat16) if bf[i] else w)
        return out
    gs = [workloads.bf16_bits((np.random.default_rng(9 + i).standard_normal(t["numel"]) * 1e-3)
                              .astype(np.float32)) for i, t in enumerate(ts)]

    def run(host):
        params = [w.cuda() for w in weights0()]
        grads = [torch.zeros(t["numel"], dtype=torch.bfloat16, device="cuda") for t in ts]
        opt = B.AdamW4(params, grads, ts, vcode=0, seed=3, total_steps=2)
        hp = [torch.empty(t["numel"], dtype=torch.int16 if bf[i] else torch.float32).pin_memory()
              for i, t in enumerate(ts)]
        hg = [torch.from_numpy(g.view(np.int16)).pin_memory() for g in gs]
        for _ in range(2):
            if host:
                B.adamw4_step_host(opt.handle, 1e-3, [x.data_ptr() for x in hg],
                                   [x.data_ptr() for x in hp],
                                   torch.cuda.current_stream().cuda_stream)
            else:
                for g, x in zip(grads, hg):
                    g.view(torch.int16).copy_(x)
                opt.step()
        torch.cuda.synchronize()
        dev_w = [p.view(torch.int16).cpu().numpy() if bf[i] else p.cpu().numpy()
                 for i, p in enumerate(params)]
        blob = opt.state_dict_blob()
        opt.close()
        return dev_w, [x.numpy() for x in hp], blob

    ref_w, _, ref_blob = run(False)
    os.environ["ADAMW4_HOST_CHUNK_UNITS"] = "7"
    try:
        dev_w, host_w, blob = run(True)
    finally:
        del os.environ["ADAMW4_HOST_CHUNK_UNITS"]
    assert blob == ref_blob
    for i in range(len(ts)):
        assert dev_w[i].tobytes() == ref_w[i].tobytes(), f"tensor {i} (device)"
        assert host_w[i].tobytes() == ref_w[i].tobytes(), f"tensor {i} (host copy)"
