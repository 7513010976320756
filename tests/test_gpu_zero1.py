"""ZeRO-1 sharding on one B200 (parity through the C ABI).

The kernel steps pieces of tensors (``elem_offset``, ``QUANT_STATE``) exactly
as it steps whole tensors: the shards of an emulated W-rank layout, one handle
per (rank, chunk) on this GPU, give the whole-list handle's weights and state
bit for bit, and the whole-list handle matches the oracle.  The sharded
optimizer itself runs over NCCL with one rank (its collectives reduce to
copies), chunked, against the whole-list handle."""
import datetime
import socket

import numpy as np
import pytest

import workloads
from gpu_common import assert_state_equal, assert_weights_close, binding, oracle_for

pytestmark = pytest.mark.gpu

SPECS = [dict(numel=128 * 300 + 5, tensor_id=3, flags=0, weight_decay=0.1),
         dict(numel=4096, tensor_id=9, flags=2, weight_decay=0.0),
         dict(numel=3000, tensor_id=11, flags=0, weight_decay=0.1),
         dict(numel=128 * 1000, tensor_id=12, flags=0, weight_decay=0.1),
         dict(numel=5000, tensor_id=13, flags=1, weight_decay=0.0),
         dict(numel=128 * 77 + 77, tensor_id=14, flags=0, weight_decay=0.05)]
STEPS = 3           # with total_steps = 3 the LM head's final-10% phase is step 3


def _host_inputs():
    rng = np.random.default_rng(1)
    ws = [(rng.standard_normal(s["numel"]) * 0.02).astype(np.float32) for s in SPECS]
    gs = [[workloads.bf16_bits((np.random.default_rng(50 * t + i).standard_normal(s["numel"])
                                * 1e-3).astype(np.float32)) for i, s in enumerate(SPECS)]
          for t in range(STEPS)]
    return ws, gs


def _flat_fill(torch, layout, flat, arrays):
    for i, a in enumerate(arrays):
        src = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        dst = layout.tensor_view(flat.view(torch.int16) if a.dtype == np.uint16 else flat, i)
        dst.copy_(src)


def _whole(torch, B, ws, vcode):
    params = [torch.from_numpy(w.copy()).cuda() for w in ws]
    grads = [torch.zeros(s["numel"], dtype=torch.bfloat16, device="cuda") for s in SPECS]
    opt = B.AdamW4(params, grads, SPECS, vcode=vcode, seed=21, total_steps=STEPS)
    return params, grads, opt


@pytest.mark.parametrize("vcode", [0, 1, 2, 3, 4, 5])
@pytest.mark.parametrize("world,chunks", [(2, 1), (3, 2), (8, 3)])
def test_emulated_shards_equal_the_whole_list(vcode, world, chunks):
    import torch
    B = binding()
    from bit_quantized_optimizer_b200.zero1 import FlatLayout, merge_state, piece_spec
    ws, gs = _host_inputs()
    L = FlatLayout([s["numel"] for s in SPECS], world, chunks)
    fp = torch.zeros(L.padded, dtype=torch.float32, device="cuda")
    fg = torch.zeros(L.padded, dtype=torch.bfloat16, device="cuda")
    _flat_fill(torch, L, fp, ws)
    handles = {}
    for r in range(world):
        for k in range(chunks):
            ps = L.pieces(r, k)
            if ps:
                handles[(r, k)] = B.AdamW4([fp[p.flat:p.flat + p.numel] for p in ps],
                                           [fg[p.flat:p.flat + p.numel] for p in ps],
                                           [piece_spec(SPECS[p.tensor], p) for p in ps],
                                           vcode=vcode, seed=21, total_steps=STEPS)
    params, grads, whole = _whole(torch, B, ws, vcode)
    ref = oracle_for(SPECS, vcode=vcode, seed=21, total_steps=STEPS)
    wref = [w.copy() for w in ws]
    try:
        for t in range(STEPS):
            _flat_fill(torch, L, fg, gs[t])
            for g, hg in zip(grads, gs[t]):
                g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
            for h in handles.values():
                h.step()
            whole.step()
            old = [w.copy() for w in wref]
            ref.step(wref, gs[t])
        torch.cuda.synchronize()
        for i, p in enumerate(params):
            a = L.tensor_view(fp, i).cpu().numpy()
            b = p.cpu().numpy()
            assert a.tobytes() == b.tobytes(), f"tensor {i}: sharded and whole weights differ"
            assert_weights_close(b, wref[i], old[i], f"whole list tensor {i}")
        merged = merge_state(L, SPECS, {rk: h.state_dict_blob() for rk, h in handles.items()})
        assert merged == whole.state_dict_blob()
        assert_state_equal(merged, ref.export_state(), vcode, "sharded")
    finally:
        for h in handles.values():
            h.close()
        whole.close()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("vcode", [0, 1])
def test_zero1_over_nccl_one_rank(vcode):
    import torch
    import torch.distributed as dist
    B = binding()
    from bit_quantized_optimizer_b200.zero1 import FlatLayout, ZeroAdamW4
    assert not dist.is_initialized()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        ws, gs = _host_inputs()
        L = FlatLayout([s["numel"] for s in SPECS], 1, 3)
        fp = torch.zeros(L.padded, dtype=torch.float32, device="cuda")
        fg = torch.zeros(L.padded, dtype=torch.bfloat16, device="cuda")
        _flat_fill(torch, L, fp, ws)
        opt = ZeroAdamW4(fp, fg, L, SPECS, vcode=vcode, seed=21, total_steps=STEPS)
        params, grads, whole = _whole(torch, B, ws, vcode)
        for t in range(STEPS):
            _flat_fill(torch, L, fg, gs[t])
            for g, hg in zip(grads, gs[t]):
                g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
            opt.step()
            whole.step()
        torch.cuda.synchronize()
        for i, p in enumerate(params):
            assert L.tensor_view(fp, i).cpu().numpy().tobytes() == p.cpu().numpy().tobytes()
        blob = opt.consolidated_state()
        assert blob == whole.state_dict_blob()
        # resume in another chunking from the consolidated checkpoint
        L2 = FlatLayout([s["numel"] for s in SPECS], 1, 2)
        fp2 = torch.zeros(L2.padded, dtype=torch.float32, device="cuda")
        fg2 = torch.zeros(L2.padded, dtype=torch.bfloat16, device="cuda")
        for i in range(len(SPECS)):
            L2.tensor_view(fp2, i).copy_(L.tensor_view(fp, i))
        opt2 = ZeroAdamW4(fp2, fg2, L2, SPECS, vcode=vcode, seed=21, total_steps=STEPS)
        opt2.load_consolidated_state(blob)
        assert opt2.t == STEPS
        _flat_fill(torch, L2, fg2, gs[0])
        for g, hg in zip(grads, gs[0]):
            g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
        opt2.step()
        whole.step()
        torch.cuda.synchronize()
        for i, p in enumerate(params):
            assert L2.tensor_view(fp2, i).cpu().numpy().tobytes() == p.cpu().numpy().tobytes()
        assert opt2.consolidated_state() == whole.state_dict_blob()
        opt.close()
        opt2.close()
        whole.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("vcode", [0, 1, 3, 5])
def test_pieces_at_large_element_offsets(vcode):
    """Pieces far into their tensors: elem_offset 2^36 + 896 and 2^39 - 4096
    (the largest allowed).  The Philox counter's high words are then in use
    (element index / 4 >= 2^32); the kernel matches the oracle stepping the
    same pieces by their blocks' indices in the whole tensor."""
    import torch
    B = binding()
    from oracle_pieces import OraclePieces
    Q = B.ADAMW4_T_QUANT_STATE
    pspecs = [dict(numel=128 * 50 + 3, tensor_id=3, flags=Q, weight_decay=0.1,
                   elem_offset=(1 << 36) + 896),
              dict(numel=4096, tensor_id=4, flags=Q | B.ADAMW4_T_LM_HEAD, weight_decay=0.0,
                   elem_offset=(1 << 39) - 4096)]
    rng = np.random.default_rng(3)
    ws = [(rng.standard_normal(s["numel"]) * 0.02).astype(np.float32) for s in pspecs]
    params = [torch.from_numpy(w.copy()).cuda() for w in ws]
    grads = [torch.zeros(s["numel"], dtype=torch.bfloat16, device="cuda") for s in pspecs]
    opt = B.AdamW4(params, grads, pspecs, vcode=vcode, seed=99, total_steps=3)
    cp = [torch.from_numpy(w.copy()) for w in ws]
    cg = [torch.zeros(s["numel"], dtype=torch.bfloat16) for s in pspecs]
    ref = OraclePieces(cp, cg, pspecs, vcode=vcode, seed=99, total_steps=3)
    try:
        for t in range(3):
            for i, s in enumerate(pspecs):
                hg = workloads.bf16_bits((np.random.default_rng(10 * t + i).standard_normal(
                    s["numel"]) * 1e-3).astype(np.float32))
                grads[i].view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
                cg[i].view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
            opt.step()
            ref.step(1e-3)
        torch.cuda.synchronize()
        for p, c in zip(params, cp):
            assert p.cpu().numpy().tobytes() == c.numpy().tobytes()
        assert opt.state_dict_blob() == ref.state_dict_blob()
    finally:
        opt.close()


@pytest.mark.parametrize("vcode", [0, 1])
def test_emulated_shards_with_bf16_weights(vcode):
    """The same emulation with bf16 weights in the flat buffer: the pieces'
    handles keep bf16 weights and equal the whole-list handle bit for bit."""
    import torch
    B = binding()
    from bit_quantized_optimizer_b200.zero1 import FlatLayout, merge_state, piece_spec
    ws, gs = _host_inputs()
    L = FlatLayout([s["numel"] for s in SPECS], 3, 2)
    fp = torch.zeros(L.padded, dtype=torch.bfloat16, device="cuda")
    fg = torch.zeros(L.padded, dtype=torch.bfloat16, device="cuda")
    for i, w in enumerate(ws):
        L.tensor_view(fp, i).copy_(torch.from_numpy(w))
    handles = {}
    for r in range(3):
        for k in range(2):
            ps = L.pieces(r, k)
            if ps:
                handles[(r, k)] = B.AdamW4([fp[p.flat:p.flat + p.numel] for p in ps],
                                           [fg[p.flat:p.flat + p.numel] for p in ps],
                                           [piece_spec(SPECS[p.tensor], p) for p in ps],
                                           vcode=vcode, seed=21, total_steps=STEPS)
    params = [torch.from_numpy(w).to(torch.bfloat16).cuda() for w in ws]
    grads = [torch.zeros(s["numel"], dtype=torch.bfloat16, device="cuda") for s in SPECS]
    whole = B.AdamW4(params, grads, SPECS, vcode=vcode, seed=21, total_steps=STEPS)
    try:
        for t in range(STEPS):
            _flat_fill(torch, L, fg, gs[t])
            for g, hg in zip(grads, gs[t]):
                g.view(torch.int16).copy_(torch.from_numpy(hg.view(np.int16)))
            for h in handles.values():
                h.step()
            whole.step()
        torch.cuda.synchronize()
        for i, p in enumerate(params):
            a = L.tensor_view(fp, i).view(torch.int16).cpu().numpy()
            assert a.tobytes() == p.view(torch.int16).cpu().numpy().tobytes(), f"tensor {i}"
        merged = merge_state(L, SPECS, {rk: h.state_dict_blob() for rk, h in handles.items()})
        assert merged == whole.state_dict_blob()
    finally:
        for h in handles.values():
            h.close()
        whole.close()
