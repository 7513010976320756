"""The allocation-free step, for callers that must not allocate device memory
(programs whose memory belongs to a pooling allocator or a fixed arena, loops
where cudaMalloc's device synchronisation is not acceptable).  It keeps the
step kernel's scratch -- the descriptor table and the status word -- in a
static device array instead of allocating it.

Checked through the C ABI against the handle-based step: two calls in a row on
the same inputs must give the same weights and packed state, within the
tolerances the other parity tests use.  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest

import workloads
from gpu_common import assert_state_equal, assert_weights_close, binding, parse_blob

pytestmark = pytest.mark.gpu


def _layout(ts):
    """Byte sizes of the caller-owned state buffers, as the header describes."""
    nb4, n32 = 0, 0
    for t in ts:
        nb = (t["numel"] + 127) // 128
        if t["numel"] < 4096 or t["flags"] & (workloads.T_NORM | workloads.T_FP32_STATE):
            n32 += nb * 128
        else:
            nb4 += nb
    return nb4, n32


def _blob_from_buffers(ts, bufs, t, vcode, seed):
    """The checkpoint-layout view of caller-owned buffers (host copies)."""
    import struct
    mc, vc, ms, vs, m32, v32 = (b.cpu().numpy() for b in bufs)
    parts, b4, e32 = [], 0, 0
    for tt in ts:
        n = tt["numel"]
        nb = (n + 127) // 128
        if n < 4096 or tt["flags"] & (workloads.T_NORM | workloads.T_FP32_STATE):
            parts += [struct.pack("<IIq", tt["tensor_id"], 1, n), m32[e32:e32 + n].tobytes(),
                      v32[e32:e32 + n].tobytes()]
            e32 += nb * 128
        else:
            parts += [struct.pack("<IIq", tt["tensor_id"], 0, n),
                      mc[b4 * 64:(b4 + nb) * 64].tobytes(), vc[b4 * 64:(b4 + nb) * 64].tobytes(),
                      ms[b4:b4 + nb].tobytes(), vs[b4:b4 + nb].tobytes()]
            b4 += nb
    payload = b"".join(parts)
    return b"ADAMW4S1" + struct.pack("<IIqQQ", len(ts), vcode, t, seed, len(payload)) + payload


@pytest.mark.parametrize("vcode", [0, 1])
def test_noalloc_step_matches_handle_step_twice(vcode):
    import torch
    B = binding()
    ts = [dict(numel=65536, tensor_id=0, flags=0, weight_decay=0.1),
          dict(numel=4096 + 37, tensor_id=4, flags=0, weight_decay=0.0),
          dict(numel=3000, tensor_id=5, flags=0, weight_decay=0.1),
          dict(numel=5000, tensor_id=6, flags=workloads.T_NORM, weight_decay=0.0),
          dict(numel=128 * 40, tensor_id=7, flags=workloads.T_LM_HEAD, weight_decay=0.1)]
    rng = np.random.default_rng(vcode)
    w0 = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
    grads = [[workloads.bf16_bits((np.random.default_rng(10 * s + i).standard_normal(t["numel"])
                                   * 1e-3).astype(np.float32)) for i, t in enumerate(ts)]
             for s in (1, 2)]
    seed, total = 77, 2
    dev = torch.device("cuda", 0)

    # handle-based step, twice
    params = [torch.from_numpy(w.copy()).to(dev) for w in w0]
    gbuf = [torch.zeros(t["numel"], dtype=torch.bfloat16, device=dev) for t in ts]
    opt = B.AdamW4(params, gbuf, ts, vcode=vcode, seed=seed, total_steps=total)
    for gs in grads:
        for g, hg in zip(gbuf, gs):
            g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
        opt.step()
    torch.cuda.synchronize()
    ref_w = [p.cpu().numpy() for p in params]
    ref_blob = opt.state_dict_blob()
    opt.close()

    # allocation-free step, twice, on buffers this test owns
    params2 = [torch.from_numpy(w.copy()).to(dev) for w in w0]
    gbuf2 = [torch.zeros(t["numel"], dtype=torch.bfloat16, device=dev) for t in ts]
    nb4, n32 = _layout(ts)
    bufs = [torch.zeros(nb4 * 64, dtype=torch.uint8, device=dev),
            torch.zeros(nb4 * 64, dtype=torch.uint8, device=dev),
            torch.zeros(max(nb4, 1), dtype=torch.float32, device=dev),
            torch.zeros(max(nb4, 1), dtype=torch.float32, device=dev),
            torch.zeros(max(n32, 4), dtype=torch.float32, device=dev),
            torch.zeros(max(n32, 4), dtype=torch.float32, device=dev)]
    sb = B.adamw4_state_buffers(*[b.data_ptr() for b in bufs])
    cfg = B.adamw4_config(1e-3, 0.9, 0.999, 1e-8, vcode, seed, total)
    descs = [B.adamw4_tensor(p.data_ptr(), g.data_ptr(), t["numel"], t["tensor_id"], t["flags"],
                             t["weight_decay"]) for p, g, t in zip(params2, gbuf2, ts)]
    stream = torch.cuda.current_stream().cuda_stream
    for step, gs in enumerate(grads, start=1):
        for g, hg in zip(gbuf2, gs):
            g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
        B.adamw4_step_noalloc(cfg, descs, sb, step, 1e-3, 0, stream)
        torch.cuda.synchronize()
        # after each call the weights follow the same arithmetic as the handle path
        assert all(np.isfinite(p.cpu().numpy()).all() for p in params2)
    for i, p in enumerate(params2):
        assert_weights_close(p.cpu().numpy(), ref_w[i], w0[i], f"noalloc tensor {i}")
    got_blob = _blob_from_buffers(ts, bufs, 2, vcode, seed)
    assert_state_equal(got_blob, ref_blob, vcode, "noalloc")


def test_noalloc_rejects_too_many_tensors():
    import torch
    B = binding()
    n = B.ADAMW4_NOALLOC_MAX_TENSORS + 1
    base = torch.zeros(16 * n, dtype=torch.float32, device="cuda")
    gb = torch.zeros(16 * n, dtype=torch.bfloat16, device="cuda")
    descs = [B.adamw4_tensor(base.data_ptr() + 64 * i, gb.data_ptr() + 32 * i, 16, i, 0, 0.0)
             for i in range(n)]
    sb = B.adamw4_state_buffers(0, 0, 0, 0, base.data_ptr(), base.data_ptr())
    cfg = B.adamw4_config(1e-3, 0.9, 0.999, 1e-8, 0, 0, 0)
    with pytest.raises(B.AdamW4Error) as err:
        B.adamw4_step_noalloc(cfg, descs, sb, 1, 1e-3, 0, None)
    assert err.value.code == B.ADAMW4_ERANGE


def test_noalloc_bf16_weights_and_pieces():
    """The same descriptor fields as the handle path: bf16 weights and a piece
    of a tensor (elem_offset, QUANT_STATE) give the handle step's bits."""
    import torch
    B = binding()
    BF, Q = B.ADAMW4_T_BF16_PARAM, B.ADAMW4_T_QUANT_STATE
    ts = [dict(numel=128 * 90 + 5, tensor_id=1, flags=BF, weight_decay=0.1, elem_offset=0),
          dict(numel=1280, tensor_id=2, flags=Q, weight_decay=0.1, elem_offset=128 * 700),
          dict(numel=5000, tensor_id=3, flags=BF | workloads.T_NORM, weight_decay=0.0,
               elem_offset=0)]
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(5)

    def make_params():
        out = []
        for t in ts:
            w = torch.from_numpy((np.random.default_rng(t["tensor_id"]).standard_normal(
                t["numel"]) * 0.02).astype(np.float32)).to(dev)
            out.append(w.to(torch.bfloat16) if t["flags"] & BF else w)
        return out
    grads = [workloads.bf16_bits((rng.standard_normal(t["numel"]) * 1e-3).astype(np.float32))
             for t in ts]
    gbuf = [torch.from_numpy(g.view(np.int16)).to(dev).view(torch.bfloat16) for g in grads]

    params = make_params()
    opt = B.AdamW4(params, gbuf, ts, vcode=0, seed=3)
    opt.step()
    torch.cuda.synchronize()
    ref = [p.view(torch.int16).cpu().numpy() if p.dtype == torch.bfloat16 else p.cpu().numpy()
           for p in params]
    ref_blob = opt.state_dict_blob()
    opt.close()

    params2 = make_params()
    nb4 = sum((t["numel"] + 127) // 128 for t in ts if not t["flags"] & workloads.T_NORM)
    n32 = 5120
    bufs = [torch.zeros(nb4 * 64, dtype=torch.uint8, device=dev),
            torch.zeros(nb4 * 64, dtype=torch.uint8, device=dev),
            torch.zeros(nb4, dtype=torch.float32, device=dev),
            torch.zeros(nb4, dtype=torch.float32, device=dev),
            torch.zeros(n32, dtype=torch.float32, device=dev),
            torch.zeros(n32, dtype=torch.float32, device=dev)]
    sb = B.adamw4_state_buffers(*[b.data_ptr() for b in bufs])
    cfg = B.adamw4_config(1e-3, 0.9, 0.999, 1e-8, 0, 3, 0)
    descs = [B.adamw4_tensor(p.data_ptr(), g.data_ptr(), t["numel"], t["tensor_id"], t["flags"],
                             t["weight_decay"], t["elem_offset"])
             for p, g, t in zip(params2, gbuf, ts)]
    B.adamw4_step_noalloc(cfg, descs, sb, 1, 1e-3, 0, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    for i, p in enumerate(params2):
        got = p.view(torch.int16).cpu().numpy() if p.dtype == torch.bfloat16 else p.cpu().numpy()
        assert got.tobytes() == ref[i].tobytes(), f"tensor {i}"
    st = parse_blob(ref_blob)["tensors"]
    mc, vc, ms, vs, m32, v32 = (b.cpu().numpy() for b in bufs)
    b4 = 0
    for t, r in zip(ts, st):
        if r["fp32"]:
            assert r["m"].tobytes() == m32[:t["numel"]].tobytes()
            assert r["v"].tobytes() == v32[:t["numel"]].tobytes()
            continue
        nb = (t["numel"] + 127) // 128
        assert r["mcodes"].tobytes() == mc[b4 * 64:(b4 + nb) * 64].tobytes()
        assert r["vcodes"].tobytes() == vc[b4 * 64:(b4 + nb) * 64].tobytes()
        assert r["mscale"].tobytes() == ms[b4:b4 + nb].tobytes()
        assert r["vscale"].tobytes() == vs[b4:b4 + nb].tobytes()
        b4 += nb


def _small_noalloc_case(B, dev, vcode=0):
    """One 4-bit tensor and one fp32-state tensor on caller-owned buffers."""
    import torch
    ts = [dict(numel=128 * 64, tensor_id=1, flags=0, weight_decay=0.1),
          dict(numel=900, tensor_id=2, flags=0, weight_decay=0.0)]
    rng = np.random.default_rng(11)
    params = [torch.from_numpy((rng.standard_normal(t["numel"]) * 0.02).astype(np.float32)).to(dev)
              for t in ts]
    grads = [torch.from_numpy(workloads.bf16_bits((rng.standard_normal(t["numel"]) * 1e-3)
                                                  .astype(np.float32)).view(np.int16)).to(dev)
             .view(torch.bfloat16) for t in ts]
    nb4, n32 = _layout(ts)
    bufs = [torch.zeros(nb4 * 64, dtype=torch.uint8, device=dev),
            torch.zeros(nb4 * 64, dtype=torch.uint8, device=dev),
            torch.zeros(nb4, dtype=torch.float32, device=dev),
            torch.zeros(nb4, dtype=torch.float32, device=dev),
            torch.zeros(n32, dtype=torch.float32, device=dev),
            torch.zeros(n32, dtype=torch.float32, device=dev)]
    sb = B.adamw4_state_buffers(*[b.data_ptr() for b in bufs])
    cfg = B.adamw4_config(1e-3, 0.9, 0.999, 1e-8, vcode, 9, 0)
    descs = [B.adamw4_tensor(p.data_ptr(), g.data_ptr(), t["numel"], t["tensor_id"], t["flags"],
                             t["weight_decay"]) for p, g, t in zip(params, grads, ts)]
    return params, grads, bufs, sb, cfg, descs


def _clear_status(B, stream):
    """Reads and clears the status word (earlier calls may have set it)."""
    try:
        B.adamw4_noalloc_sync(0, stream)
    except B.AdamW4Error:
        pass


def test_noalloc_status_reports_timeout_and_nonfinite_weights():
    """The device status word of the allocation-free step, read through
    adamw4_noalloc_sync: a stage stall armed on the host for one call (the
    kernel's bounded waits run out after about a second each; nothing faults)
    gives ADAMW4_ETIMEOUT; a NaN grad written on the host gives
    ADAMW4_ENONFINITE; each is reported once, and a clean call then reads
    ADAMW4_OK.  The context stays usable throughout."""
    import torch
    B = binding()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream().cuda_stream
    params, grads, bufs, sb, cfg, descs = _small_noalloc_case(B, dev)
    B.adamw4_step_noalloc(cfg, descs, sb, 1, 1e-3, 0, stream)
    _clear_status(B, stream)
    B.adamw4_step_noalloc(cfg, descs, sb, 2, 1e-3, 0, stream)
    B.adamw4_noalloc_sync(0, stream)                          # clean: OK

    B.adamw4_inject_fault(None, B.ADAMW4_FAULT_STALL_PIPELINE)
    B.adamw4_step_noalloc(cfg, descs, sb, 3, 1e-3, 0, stream)
    with pytest.raises(B.AdamW4Error) as err:
        B.adamw4_noalloc_sync(0, stream)
    assert err.value.code == B.ADAMW4_ETIMEOUT
    B.adamw4_noalloc_sync(0, stream)                          # cleared

    grads[0][100] = float("nan")
    B.adamw4_step_noalloc(cfg, descs, sb, 4, 1e-3, 0, stream)
    with pytest.raises(B.AdamW4Error) as err:
        B.adamw4_noalloc_sync(0, stream)
    assert err.value.code == B.ADAMW4_ENONFINITE
    B.adamw4_noalloc_sync(0, stream)                          # cleared
    # the context is still usable: a small device computation works
    assert float(torch.ones(4, device=dev).sum()) == 4.0


def test_noalloc_status_needs_a_used_device():
    B = binding()
    with pytest.raises(B.AdamW4Error) as err:
        B.adamw4_noalloc_sync(63, None)
    assert err.value.code == -1
