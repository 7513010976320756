"""ZeRO-1 sharding on CPU: the flat layout, the checkpoint merge, the oracle on
pieces, and the sharded step over gloo ranks (world sizes 2, 3 and 4).

The invariant: the sharded step (reduce-scatter, step of each rank's pieces,
all-gather) gives the same weights and state, bit for bit, as the oracle's
step of the whole tensor list on the reduced gradient.  Blocks and draws are
keyed by the element's index in its whole tensor, so nothing in the method
depends on where a tensor is cut (at block boundaries)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads
from bit_quantized_optimizer_b200 import ADAMW4_T_QUANT_STATE, is_fp32_state
from bit_quantized_optimizer_b200.zero1 import FlatLayout, merge_state, piece_spec, split_state
from gpu_common import parse_blob
from oracle_pieces import OraclePieces

# Ragged tensors, a tensor that many shards cut, a small fp32 tensor, a large
# normalisation tensor (fp32 pieces), and an LM head whose final-10% phase
# starts at step 3 of 3.
SPECS = [dict(numel=128 * 37 + 5, tensor_id=3, flags=0, weight_decay=0.1),
         dict(numel=4096, tensor_id=9, flags=2, weight_decay=0.0),
         dict(numel=3000, tensor_id=11, flags=0, weight_decay=0.1),
         dict(numel=128 * 64, tensor_id=12, flags=0, weight_decay=0.1),
         dict(numel=5000, tensor_id=13, flags=1, weight_decay=0.0),
         dict(numel=128 * 9 + 77, tensor_id=14, flags=0, weight_decay=0.05)]
TOTAL_STEPS = 3


def _pieces_of(layout):
    return {(r, k): layout.pieces(r, k) for r in range(layout.world)
            for k in range(layout.chunks)}


@pytest.mark.parametrize("world,chunks", [(1, 1), (2, 1), (2, 3), (3, 2), (8, 1), (8, 4)])
def test_layout_cuts_every_tensor_into_block_aligned_pieces(world, chunks):
    numels = [s["numel"] for s in SPECS] + [1, 127, 129, 100_000]
    L = FlatLayout(numels, world, chunks)
    assert L.shard % 128 == 0 and L.padded == L.shard * world * chunks >= L.used
    for i, (off, n) in enumerate(zip(L.offsets, numels)):
        assert off % 128 == 0
        if i:
            assert off >= L.offsets[i - 1] + numels[i - 1]
    seen = [np.zeros(n, np.int32) for n in numels]
    for (r, k), ps in _pieces_of(L).items():
        lo, hi = L.shard_range(r, k)
        for p in ps:
            assert p.elem_offset % 128 == 0 and p.numel > 0
            assert lo <= p.flat and p.flat + p.numel <= hi
            assert p.flat == L.offsets[p.tensor] + p.elem_offset
            # a piece ends on a block boundary or at its tensor's end
            end = p.elem_offset + p.numel
            assert end % 128 == 0 or end == numels[p.tensor]
            seen[p.tensor][p.elem_offset:end] += 1
    for s in seen:
        assert (s == 1).all()


def test_piece_spec_keeps_the_whole_tensors_class():
    L = FlatLayout([s["numel"] for s in SPECS], 8, 2)
    for (r, k), ps in _pieces_of(L).items():
        for p in ps:
            spec = SPECS[p.tensor]
            ps_ = piece_spec(spec, p)
            assert ps_["tensor_id"] == spec["tensor_id"]
            assert ps_["elem_offset"] == p.elem_offset and ps_["numel"] == p.numel
            whole = is_fp32_state(spec["numel"], spec["flags"])
            assert is_fp32_state(ps_["numel"], ps_["flags"]) == whole
            assert bool(ps_["flags"] & ADAMW4_T_QUANT_STATE) == (not whole)


@pytest.mark.parametrize("world,chunks", [(2, 1), (3, 2), (8, 3)])
def test_split_then_merge_is_the_identity(world, chunks):
    blob = workloads.synthetic_state_blob(SPECS, 0, 17, seed=5, is_fp32=is_fp32_state)
    L = FlatLayout([s["numel"] for s in SPECS], world, chunks)
    parts = {rk: split_state(L, SPECS, blob, *rk) for rk, ps in _pieces_of(L).items() if ps}
    assert merge_state(L, SPECS, parts) == blob
    # and across layouts: cut for one, merged back through another
    L2 = FlatLayout([s["numel"] for s in SPECS], 2, 1)
    parts2 = {rk: split_state(L2, SPECS, merge_state(L, SPECS, parts), *rk)
              for rk, ps in _pieces_of(L2).items() if ps}
    assert merge_state(L2, SPECS, parts2) == blob


def test_merge_rejects_missing_pieces():
    blob = workloads.synthetic_state_blob(SPECS, 1, 2, seed=1, is_fp32=is_fp32_state)
    L = FlatLayout([s["numel"] for s in SPECS], 2, 2)
    parts = {rk: split_state(L, SPECS, blob, *rk) for rk, ps in _pieces_of(L).items() if ps}
    parts.pop(next(iter(parts)))
    with pytest.raises(ValueError):
        merge_state(L, SPECS, parts)


def _inputs(world, steps=TOTAL_STEPS):
    rng = np.random.default_rng(0)
    ws = [(rng.standard_normal(s["numel"]) * 0.02).astype(np.float32) for s in SPECS]
    # rank r's gradients at each step; they are summed across the ranks
    gs = [[[(np.random.default_rng(1000 * t + 10 * r + i).standard_normal(s["numel"])
             * 1e-3).astype(np.float32) for i, s in enumerate(SPECS)]
           for r in range(world)] for t in range(steps)]
    return ws, gs


def _flat(layout, arrays, dtype):
    f = torch.zeros(layout.padded, dtype=dtype)
    for i, a in enumerate(arrays):
        layout.tensor_view(f, i).copy_(torch.from_numpy(a).to(dtype))
    return f


@pytest.mark.parametrize("vcode", [0, 1, 3, 5])
def test_oracle_pieces_equal_the_whole_step(vcode):
    """No collectives: the pieces of an 8 x 3 layout stepped one by one give the
    whole step's bits (weights and merged state)."""
    ws, gs = _inputs(1)
    L = FlatLayout([s["numel"] for s in SPECS], 8, 3)
    cfg = dict(vcode=vcode, seed=77, total_steps=TOTAL_STEPS)
    full = oracle.OracleAdamW4(tensors=SPECS, **cfg)
    wf = [w.copy() for w in ws]
    fp = _flat(L, ws, torch.float32)
    fg = torch.zeros(L.padded, dtype=torch.bfloat16)
    steppers = {rk: OraclePieces([fp[p.flat:p.flat + p.numel] for p in ps],
                                 [fg[p.flat:p.flat + p.numel] for p in ps],
                                 [piece_spec(SPECS[p.tensor], p) for p in ps], **cfg)
                for rk, ps in _pieces_of(L).items() if ps}
    for t in range(TOTAL_STEPS):
        g = [workloads.bf16_bits(x) for x in gs[t][0]]
        full.step(wf, g)
        for i, gi in enumerate(g):
            L.tensor_view(fg.view(torch.int16), i).copy_(torch.from_numpy(gi.view(np.int16)))
        for st in steppers.values():
            st.step(full.lr)
    for i in range(len(SPECS)):
        assert L.tensor_view(fp, i).numpy().tobytes() == wf[i].tobytes()
    merged = merge_state(L, SPECS, {rk: st.state_dict_blob() for rk, st in steppers.items()})
    assert merged == full.export_state()


# ---------------------------------------------------------------------------
# gloo ranks
# ---------------------------------------------------------------------------

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _wbits(t):
    """Weights as comparable bytes: fp32, or bf16 bit patterns."""
    return (t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16
            else t.numpy()).copy()


def _rank(rank, world, port, root, vcode, chunks, out, bf16=False):
    import sys
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from bit_quantized_optimizer_b200.zero1 import FlatLayout, ZeroAdamW4
        from oracle_pieces import OraclePieces
        cfg = dict(vcode=vcode, seed=77, total_steps=TOTAL_STEPS)
        ws, gs = _inputs(world)
        L = FlatLayout([s["numel"] for s in SPECS], world, chunks)
        wdt = torch.bfloat16 if bf16 else torch.float32
        fp, fg = _flat(L, ws, wdt), torch.zeros(L.padded, dtype=torch.bfloat16)

        def make(p, g, s):
            return OraclePieces(p, g, s, **cfg)
        opt = ZeroAdamW4(fp, fg, L, SPECS, make_stepper=make, **cfg)
        reduced = []
        for t in range(TOTAL_STEPS - 1):
            fg.copy_(_flat(L, gs[t][rank], torch.bfloat16))
            opt.step()
            full_g = torch.empty_like(fg)
            for k in range(chunks):      # the reduced gradient, gathered for the check
                dist.all_gather_into_tensor(full_g[L.chunk_range(k)[0]:L.chunk_range(k)[1]],
                                            opt.grad_shard[k * L.shard:(k + 1) * L.shard])
            reduced.append(full_g.view(torch.int16).numpy().copy())
        blob = opt.consolidated_state()
        # resume the last step from the merged checkpoint in another layout
        L2 = FlatLayout([s["numel"] for s in SPECS], world, chunks + 1)
        fp2 = torch.zeros(L2.padded, dtype=wdt)
        for i in range(len(SPECS)):
            L2.tensor_view(fp2, i).copy_(L.tensor_view(fp, i))
        fg2 = torch.zeros(L2.padded, dtype=torch.bfloat16)
        opt2 = ZeroAdamW4(fp2, fg2, L2, SPECS, make_stepper=make, **cfg)
        opt2.load_consolidated_state(blob)
        fg2.copy_(_flat(L2, gs[-1][rank], torch.bfloat16))
        opt2.step()
        full_g = torch.empty_like(fg2)
        for k in range(chunks + 1):
            dist.all_gather_into_tensor(full_g[L2.chunk_range(k)[0]:L2.chunk_range(k)[1]],
                                        opt2.grad_shard[k * L2.shard:(k + 1) * L2.shard])
        reduced.append(full_g.view(torch.int16).numpy().copy())
        final = opt2.consolidated_state()
        weights = [_wbits(L2.tensor_view(fp2, i)) for i in range(len(SPECS))]
        out.put((rank, reduced, blob, final, weights, opt2.t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,vcode,chunks,bf16", [(2, 0, 1, False), (2, 1, 2, False),
                                                      (2, 4, 3, False), (3, 0, 2, False),
                                                      (4, 5, 2, False), (2, 0, 2, True)])
def test_gloo_ranks_equal_the_whole_step(world, vcode, chunks, bf16):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, root, vcode, chunks, q, bf16))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r[0], r[1:]) for r in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    red0, blob0, final0, w0, t0 = res[0]
    for r in range(1, world):
        red, blob, final, w, t = res[r]
        assert blob == blob0 and final == final0 and t == t0 == TOTAL_STEPS
        for a, b in zip(w0, w):
            assert a.tobytes() == b.tobytes()
        for a, b in zip(red0, red):
            assert a.tobytes() == b.tobytes()
    # the whole list on one process, on the reduced gradients
    ws, _ = _inputs(world)
    specs = [dict(s, flags=s["flags"] | (oracle.T_BF16_PARAM if bf16 else 0)) for s in SPECS]
    full = oracle.OracleAdamW4(tensors=specs, vcode=vcode, seed=77, total_steps=TOTAL_STEPS)
    wf = [oracle.round_bf16(w) if bf16 else w.copy() for w in ws]
    for t in range(TOTAL_STEPS):
        L = FlatLayout([s["numel"] for s in SPECS], world, chunks if t < TOTAL_STEPS - 1
                       else chunks + 1)
        g = [L.tensor_view(torch.from_numpy(red0[t]), i).numpy().view(np.uint16).copy()
             for i in range(len(SPECS))]
        full.step(wf, g)
        if t == TOTAL_STEPS - 2:
            assert blob0 == full.export_state()
    assert final0 == full.export_state()
    for a, b in zip(w0, wf):
        assert a.tobytes() == b.tobytes()
    st = parse_blob(final0)
    assert st["t"] == TOTAL_STEPS and len(st["tensors"]) == len(SPECS)


def _rank_dies(rank, world, port, root, out):
    import sys
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import time
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    from bit_quantized_optimizer_b200.zero1 import FlatLayout, ZeroAdamW4
    from oracle_pieces import OraclePieces
    L = FlatLayout([s["numel"] for s in SPECS], world, 2)
    fp, fg = torch.zeros(L.padded), torch.zeros(L.padded, dtype=torch.bfloat16)
    opt = ZeroAdamW4(fp, fg, L, SPECS, vcode=0, seed=1,
                     make_stepper=lambda p, g, s: OraclePieces(p, g, s, vcode=0, seed=1,
                                                               total_steps=0))
    opt.step()                             # one good step on both ranks
    dist.barrier()
    if rank == 1:
        os._exit(0)                        # leaves between steps, nothing in flight
    time.sleep(0.5)
    t0 = time.monotonic()
    try:
        opt.step()
        out.put(("no error", time.monotonic() - t0))
    except Exception as e:                 # the survivor's next collective fails
        out.put((type(e).__name__, time.monotonic() - t0))


def test_a_lost_rank_surfaces_as_an_error_on_the_survivor():
    """Failure detection on the host: rank 1 leaves between steps; rank 0's
    next sharded step raises (peer gone or the 5 s process-group timeout)
    instead of hanging."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, 2, port, root, q)) for r in range(2)]
    for p in procs:
        p.start()
    what, took = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert what != "no error"
    assert took < 30
