"""The benchmark's multi-GPU path on CPU: `bench.zero1_setup` (the ZeRO-1 job
that `bench.py --gpus N` times for N > 1) over two gloo ranks, with the oracle
stepping each rank's pieces in place of the CUDA handle.  The sharded job must
give, bit for bit, the oracle's whole-list step on the reduced gradients, and
every rank must end with the same weights."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

SPECS = [dict(numel=128 * 37 + 5, tensor_id=3, flags=0, weight_decay=0.1),
         dict(numel=3000, tensor_id=11, flags=0, weight_decay=0.1),
         dict(numel=128 * 64, tensor_id=12, flags=0, weight_decay=0.1),
         dict(numel=5000, tensor_id=13, flags=1, weight_decay=0.0)]
STEPS = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, root, vcode, chunks, out):
    import sys
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from oracle_pieces import OraclePieces
        layout, fp, fg, opt = bench.zero1_setup(
            SPECS, world, rank, chunks, torch.float32, "cpu", vcode,
            make_stepper=lambda p, g, s: OraclePieces(p, g, s, vcode=vcode, seed=0,
                                                      total_steps=0))
        w0 = [layout.tensor_view(fp, i).numpy().copy() for i in range(len(SPECS))]
        reduced = []
        for _ in range(STEPS):
            opt.step()
            full_g = torch.empty_like(fg)
            for k in range(chunks):       # the reduced gradient, gathered for the check
                lo, hi = layout.chunk_range(k)
                dist.all_gather_into_tensor(full_g[lo:hi],
                                            opt.grad_shard[k * layout.shard:(k + 1) * layout.shard])
            reduced.append(full_g.view(torch.int16).numpy().copy())
        blob = opt.consolidated_state()
        weights = [layout.tensor_view(fp, i).numpy().copy() for i in range(len(SPECS))]
        out.put((rank, w0, reduced, blob, weights))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("vcode,chunks", [(0, 1), (1, 3)])
def test_bench_zero1_job_equals_the_whole_step(vcode, chunks):
    import oracle
    from bit_quantized_optimizer_b200.zero1 import FlatLayout
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, root, vcode, chunks, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r[0], r[1:]) for r in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w0, red0, blob0, wf0 = res[0]
    w1, red1, blob1, wf1 = res[1]
    # the same starting weights on both ranks (seed 0), the same results
    for a, b in zip(w0, w1):
        assert a.tobytes() == b.tobytes()
    assert blob0 == blob1
    for a, b in zip(wf0, wf1):
        assert a.tobytes() == b.tobytes()
    # the oracle's whole step on the reduced gradients
    L = FlatLayout([s["numel"] for s in SPECS], world, chunks)
    full = oracle.OracleAdamW4(tensors=SPECS, vcode=vcode, seed=0)
    wf = [w.copy() for w in w0]
    for t in range(STEPS):
        g = [L.tensor_view(torch.from_numpy(red0[t]), i).numpy().view(np.uint16).copy()
             for i in range(len(SPECS))]
        full.step(wf, g)
    assert blob0 == full.export_state()
    for a, b in zip(wf0, wf):
        assert a.tobytes() == b.tobytes()
