"""The multi-rank path on CPU with gloo (world size 2).

bench.py --gpus N runs one replica of the step per rank with no data-path
collective; the only cross-rank operations are a barrier and the maximum of
the timed duration.  Those run here under gloo.  The same ranks also show that
the step shards without any exchange: each rank steps half of a tensor list
through the oracle, and the union equals a single-process step bit for bit,
because every draw is keyed by (seed, step, tensor, element)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


TS = [dict(numel=128 * 37 + 5, tensor_id=3, flags=0, weight_decay=0.1),
      dict(numel=4096, tensor_id=9, flags=2, weight_decay=0.0),
      dict(numel=3000, tensor_id=11, flags=0, weight_decay=0.1),
      dict(numel=128 * 64, tensor_id=12, flags=0, weight_decay=0.1),
      dict(numel=5000, tensor_id=13, flags=1, weight_decay=0.0)]


def _inputs():
    import workloads
    rng = np.random.default_rng(0)
    ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in TS]
    gs = [[workloads.bf16_bits((np.random.default_rng(100 * s + i).standard_normal(t["numel"])
                                * 1e-3).astype(np.float32)) for i, t in enumerate(TS)]
          for s in range(3)]
    return ws, gs


def _rank(rank, world, port, root, vcode, out):
    import sys
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        bench.barrier(world)
        got = bench.max_over_ranks(10.0 + rank, world)
        value = bench.weak_scaling_value(world, 1000, got)
        # tensors dealt out round-robin: rank r steps tensors r, r + world, ...
        mine = list(range(rank, len(TS), world))
        ws, gs = _inputs()
        o = oracle.OracleAdamW4(vcode=vcode, seed=5, total_steps=3,
                                tensors=[TS[i] for i in mine])
        wmine = [ws[i].copy() for i in mine]
        for g in gs:
            o.step(wmine, [g[i] for i in mine])
        parts = [None] * world
        dist.all_gather_object(parts, (mine, [w.tobytes() for w in wmine], o.export_state()))
        if rank == 0:
            out.put((got, value, parts))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("vcode", [0, 1])
def test_two_gloo_ranks(vcode):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, root, vcode, q)) for r in range(2)]
    for p in procs:
        p.start()
    got, value, parts = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == 11.0                               # max over the ranks' 10.0, 11.0
    assert value == pytest.approx(2 * 1000 / 11e-3 / 1e9)
    # single process, whole list
    ws, gs = _inputs()
    full = oracle.OracleAdamW4(vcode=vcode, seed=5, total_steps=3, tensors=TS)
    wfull = [w.copy() for w in ws]
    for g in gs:
        full.step(wfull, g)
    from gpu_common import parse_blob
    ref = parse_blob(full.export_state())["tensors"]
    seen = set()
    for mine, wbytes, blob in parts:
        st = parse_blob(blob)["tensors"]
        for k, i in enumerate(mine):
            seen.add(i)
            assert np.frombuffer(wbytes[k], np.float32).tobytes() == wfull[i].tobytes()
            for key in ref[i]:
                a, b = st[k][key], ref[i][key]
                assert (a == b).all() if isinstance(a, np.ndarray) else a == b
    assert seen == set(range(len(TS)))
