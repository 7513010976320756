"""Benchmark of the fused 4-bit AdamW step (ZIP-SR / ZE-EDEN) on B200.

One step = one pass of the whole path over the GPT-style 2.7B tensor list (32
layers, d 2560, FFN 10,240, vocab 50,304, context 2048, untied head; 195
4-bit tensors, 194 fp32-state tensors): decode, moment update, weight update,
requantise and pack, as one kernel launch.  Inputs are synthetic and resident
in HBM (19.7 GB > L2, so no L2 flush is needed between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--vcode zipsr|zeeden]
                    [--impl ours|reference]

At N = 1 the line's headline is the v code chosen (ZIP-SR by default); the
other method (ZE-EDEN, or ZIP-SR) is timed the same way on the same inputs
and reported under "by_vcode".

With N > 1 (under torch.distributed.run) the ranks run the ZeRO-1 sharded
step: they share one copy of the workload, and each steps 1/N of it between a
reduce-scatter of the bf16 gradients and an all-gather of the fp32 weights
over NCCL (strong scaling; `--zero1` selects it at N = 1 too, as a one-rank
group whose collectives are local copies).  `--replicas` times N independent
replicas instead (no collective, weak scaling).
`--impl reference` times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

WORKLOAD = "gpt-2.7b"        # the benchmark workload; --workload picks a profiling case
VCODES = {"zipsr": 0, "zeeden": 1, "zi_rtn": 2, "zi_sr": 3, "ze_floor": 4, "zipsr_u32": 5}
METRIC = "fused 4-bit AdamW step Gparams/s; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
# the device code of the step (the C ABI around it is in adamw4.cu)
KERNEL_SRCS = [os.path.join(ROOT, "bit_quantized_optimizer_b200", "csrc", f)
               for f in ("adamw4_kernel.cuh", "exact_math.cuh")]


def is_fp32_state(numel, flags):
    """The library's state class of a tensor (fp32 m, v or 4-bit codes)."""
    import bit_quantized_optimizer_b200 as B
    return B.is_fp32_state(numel, flags)


def algorithmic_bytes(ts, wbytes=4):
    """HBM bytes one step must move: per 4-bit value, w read+write (2 x 4, or
    2 x 2 for bf16 weights), bf16 grad read (2); per 128-value block, m and v
    codes (64 B each) and scales (4 B each), read and written; per fp32-state
    value w read+write, grad read, and m, v (4 + 4 each) read and written."""
    b = 0
    for t in ts:
        n = t["numel"]
        if is_fp32_state(n, t["flags"]):
            b += (2 * wbytes + 2 + 16) * n
        else:
            b += (2 * wbytes + 2) * n + 2 * 136 * ((n + 127) // 128)
    return b


def variant_name(args):
    return args.vcode + ("_bf16w" if args.bf16_params else "")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sha():
    """sha256 of the step kernel's device sources (the profile records carry
    it, so that counters taken on other source are not reported)."""
    h = hashlib.sha256()
    for f in KERNEL_SRCS:
        h.update(open(f, "rb").read())
    return h.hexdigest()


def profile_record(vcode_name):
    """The committed ncu summary of the step kernel for this workload and
    v code, if it was taken on the current kernel source; else {}."""
    p = os.path.join(ROOT, "profiles", f"adamw4_step_{WORKLOAD}_{vcode_name}_traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return {}
    return d if d.get("kernel_source_sha256") == kernel_sha() else {}


def traffic_record(vcode_name):
    """DRAM bytes per launch (ncu), or None."""
    return profile_record(vcode_name).get("traffic_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    Q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5:
            time.sleep(0.02)
        self.skip = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [l.split(",") for l in self.lines[max(self.skip - 1, 0):] if l.count(",") >= 6]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[3:7]):
                if v.strip().lower() in ("active", "1", "yes"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].strip().replace(".", "").isdigit()
                else None, "reasons": sorted(reasons), "samples": len(rows)}


def dist_setup(n_gpus):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        # one line per rank on stderr (stdout carries rank 0's JSON line only)
        print(f"bench: rank {rank} of {ws} on cuda:{local} ({torch.cuda.get_device_name(local)}), "
              f"process group {dist.get_backend()}", file=sys.stderr, flush=True)
    else:
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    """The maximum of a per-rank number (a device-timed duration) over all
    ranks; NCCL reduces a CUDA tensor, gloo a CPU one."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world_size, params_per_rank, max_ms_per_step):
    """Whole-job throughput in Gparams/s: every rank steps its own replica of
    the workload, and the job takes as long as the slowest rank."""
    return world_size * params_per_rank / (max_ms_per_step * 1e-3) / 1e9


def cpu_baseline(ts, params, grads, vcode, target_s=10.0, per_tensor_cap=1 << 18):
    """The oracle on the host cores over a bounded sample of the workload: the
    first up-to-256K values of every tensor of the list (about 40M params),
    one step repeated until about `target_s` seconds have passed."""
    import torch
    import oracle
    sub, ws, gs = [], [], []
    for t, p, g in zip(ts, params, grads):
        n = min(t["numel"], per_tensor_cap)
        tt = dict(t)
        tt["numel"] = n
        if p.dtype == torch.bfloat16:
            tt["flags"] = tt["flags"] | oracle.T_BF16_PARAM
            ws.append(p[:n].view(torch.int16).cpu().numpy().view(np.uint16).copy())
        else:
            ws.append(p[:n].cpu().numpy().copy())
        sub.append(tt)
        gs.append(g[:n].view(torch.int16).cpu().numpy().view(np.uint16).copy())
    nthreads = max(1, oracle.max_threads())
    o = oracle.OracleAdamW4(vcode=vcode, tensors=sub, nthreads=nthreads)
    nparams = sum(t["numel"] for t in sub)
    steps, t0 = 0, time.perf_counter()
    while True:
        o.step(ws, gs)
        steps += 1
        el = time.perf_counter() - t0
        if el >= target_s:
            break
    # the same oracle on one thread, on the first up-to-16K values of every
    # tensor (about 3 s)
    cap1 = 1 << 14
    sub1 = [dict(t, numel=min(t["numel"], cap1)) for t in sub]
    o1 = oracle.OracleAdamW4(vcode=vcode, tensors=sub1, nthreads=1)
    ws1 = [w[:t["numel"]].copy() for w, t in zip(ws, sub1)]
    gs1 = [g[:t["numel"]].copy() for g, t in zip(gs, sub1)]
    n1 = sum(t["numel"] for t in sub1)
    steps1, t1 = 0, time.perf_counter()
    while True:
        o1.step(ws1, gs1)
        steps1 += 1
        el1 = time.perf_counter() - t1
        if el1 >= target_s / 3:
            break
    return {"value": nparams * steps / el / 1e9, "unit": "Gparams/s", "cores": nthreads,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"first <= {per_tensor_cap} values of each of the {len(sub)} tensors of the "
                      f"{WORKLOAD} list ({nparams} params), {steps} step(s), {el:.1f} s, "
                      f"{nthreads} OpenMP threads",
            "single_thread": {"value": n1 * steps1 / el1 / 1e9, "unit": "Gparams/s", "cores": 1,
                              "sample": f"first <= {cap1} values of each tensor ({n1} params), "
                                        f"{steps1} step(s), {el1:.1f} s"}}


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or platform.machine()


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    vcode = VCODES[args.vcode]
    ts = workloads.tensor_list(WORKLOAD)
    # per step: the first up-to-64K values of every tensor (about 12M params);
    # inputs from the host generator, state zero-initialised
    cap = 1 << 16
    sub = []
    for t in ts:
        tt = dict(t)
        tt["numel"] = min(t["numel"], cap)
        sub.append(tt)
    wts = workloads.host_weights(WORKLOAD, sub)
    grs = workloads.host_grads(WORKLOAD, sub, 1)
    nthreads = max(1, oracle.max_threads())
    o = oracle.OracleAdamW4(vcode=vcode, tensors=sub, nthreads=nthreads)
    nparams = sum(t["numel"] for t in sub)
    for _ in range(args.warmup):
        o.step(wts, grs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.step(wts, grs)
    el = time.perf_counter() - t0
    value = nparams * args.steps / el / 1e9
    sample = (f"first <= {cap} values of each of the {len(sub)} tensors of the {WORKLOAD} list "
              f"({nparams} params) per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Gparams/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "vcode": args.vcode, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "Gparams/s", "cores": nthreads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "Gparams/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def e2e_run(B, opt, ts, grads, nparams, stream, ws_, args):
    """Same metric end to end through the C ABI with host buffers, every step:
    adamw4_step_host copies the step's inputs (the bf16 grads) from pinned
    host memory to the device, pipelined with the step over pieces of the
    list, and adamw4_sync reads the step's result back (its 4-byte device
    status word: OK, or a non-finite weight); the weights stay resident on
    the device, as in training.  `with_weights_d2h` repeats it with the
    updated weights also copied back to pinned host memory every step."""
    import torch
    e2e_steps = max(1, min(3, args.steps))
    wbytes = 2 if args.bf16_params else 4
    hg = torch.empty(nparams, dtype=torch.int16).pin_memory()
    hp = torch.empty(nparams, dtype=torch.int16 if wbytes == 2 else torch.float32).pin_memory()
    offs = np.cumsum([0] + [t["numel"] for t in ts])
    gptrs = [hg.data_ptr() + 2 * int(o) for o in offs[:-1]]
    pptrs = [hp.data_ptr() + wbytes * int(o) for o in offs[:-1]]
    for g, o, t in zip(grads, offs[:-1], ts):
        hg[int(o):int(o) + t["numel"]].copy_(g.view(torch.int16).cpu())

    def timed(params_host):
        B.adamw4_step_host(opt.handle, 1e-3, gptrs, params_host, stream.cuda_stream)   # warm
        B.adamw4_sync(opt.handle, stream.cuda_stream)
        barrier(ws_)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            B.adamw4_step_host(opt.handle, 1e-3, gptrs, params_host, stream.cuda_stream)
            B.adamw4_sync(opt.handle, stream.cuda_stream)
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws_)

    ms = timed(None)
    ms_w = timed(pptrs)
    del hg, hp
    return {"value": ws_ * nparams / (ms * 1e-3) / 1e9, "unit": "Gparams/s",
            "h2d_bytes_per_step": 2 * nparams, "d2h_bytes_per_step": 4, "steps": e2e_steps,
            "with_weights_d2h": {"value": ws_ * nparams / (ms_w * 1e-3) / 1e9,
                                 "unit": "Gparams/s", "h2d_bytes_per_step": 2 * nparams,
                                 "d2h_bytes_per_step": 4 + wbytes * nparams}}


def timed_steps(opt, args, stream, ws_, local):
    """W untimed steps, then K steps bracketed by CUDA events on the launching
    stream (per launch and in total), a barrier and a synchronize on both
    sides, with nvidia-smi sampling the clocks meanwhile.  Returns (max over
    ranks of the total ms, max over ranks of the mean launch ms, clocks)."""
    import torch
    for _ in range(args.warmup):
        opt.step(stream=stream.cuda_stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(ws_)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        opt.step(stream=stream.cuda_stream)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(ws_)
    clk = clocks.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), ws_)
    avg_launch_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev])), ws_)
    return total_ms, avg_launch_ms, clk


def run_ours(args):
    import torch
    ws_, rank, local = dist_setup(args.gpus)
    import bit_quantized_optimizer_b200 as B
    B.lib()  # fail loudly if the extension is missing
    ts = workloads.tensor_list(WORKLOAD)
    params, grads = workloads.device_inputs(WORKLOAD, ts, seed=rank)
    if args.bf16_params:                  # bf16 weights: the nearest bf16 of the same draw
        for i in range(len(params)):
            params[i] = params[i].to(torch.bfloat16)
    torch.cuda.synchronize()
    nparams = sum(t["numel"] for t in ts)
    alg_bytes = algorithmic_bytes(ts, 2 if args.bf16_params else 4)
    stream = torch.cuda.current_stream()
    peak, peak_kind = peaks()

    # the headline v code, then the other method on the same inputs
    names = [args.vcode]
    if not args.no_companion and args.vcode in ("zipsr", "zeeden"):
        names.append("zeeden" if args.vcode == "zipsr" else "zipsr")
    by_vcode, opt_head = {}, None
    for name in names:
        opt = B.AdamW4(params, grads, ts, lr=1e-3, vcode=VCODES[name], seed=rank)
        total_ms, avg_launch_ms, clk = timed_steps(opt, args, stream, ws_, local)
        ms = total_ms / args.steps
        achieved = alg_bytes / (avg_launch_ms * 1e-3) / 1e9
        vname = name + ("_bf16w" if args.bf16_params else "")
        by_vcode[name] = {"ms_per_step": ms, "value": weak_scaling_value(ws_, nparams, ms),
                          "unit": "Gparams/s", "launch_ms": avg_launch_ms, "hbm_gbs": achieved,
                          "frac": achieved / peak, "traffic": traffic_record(vname),
                          "issue": profile_record(vname).get("issue"), "clocks": clk,
                          "gpu_launches": args.steps}
        if name == args.vcode:
            opt_head = opt
        else:
            opt.close()
    head = by_vcode[args.vcode]
    grid, block, units = B.adamw4_launch_info(opt_head.handle)
    resident = (4 if not args.bf16_params else 2) * nparams + 2 * nparams + opt_head.state_bytes()

    # e2e through the C ABI with host buffers: grads H2D, step, params D2H
    e2e = None
    if not args.no_e2e:
        e2e = e2e_run(B, opt_head, ts, grads, nparams, stream, ws_, args)

    cpu = None
    if rank == 0 and ws_ == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(ts, params, grads, VCODES[args.vcode])

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": head["value"],
            "unit": "Gparams/s",
            "n_gpus": ws_,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "vcode": args.vcode, "params": nparams,
                       "weights": "bf16" if args.bf16_params else "fp32",
                       "tensors": len(ts), "algorithmic_bytes_per_step": alg_bytes,
                       "parallelism": f"replicas x{ws_} (no data-path collective)",
                       "l2": f"inputs {resident / 1e9:.1f} GB > 126 MB L2; no flush",
                       "grid": grid, "block": block, "units": units},
            "hbm_gbs": head["hbm_gbs"],
            "roofline": {"bound": "hbm", "achieved": head["hbm_gbs"], "peak": peak, "unit": "GB/s",
                         "frac": head["frac"], "peak_kind": peak_kind,
                         "traffic": head["traffic"],
                         # the step is bound by instruction issue, not HBM: ncu figures
                         "issue": head["issue"]},
            "by_vcode": by_vcode,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": head["clocks"],
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    opt_head.close()
    if ws_ > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def zero1_setup(ts, world, rank, chunks, wdtype, device, vcode, make_stepper=None):
    """The ZeRO-1 job's inputs and optimizer on one rank: flat buffers in the
    layout of `chunks` chunks over `world` ranks, the same weights on every
    rank (seed 0), the rank's own gradients (seed rank + 1), and a
    ZeroAdamW4 over them (its steppers from `make_stepper`, default the CUDA
    handle).  Returns (layout, flat params, flat grads, optimizer)."""
    import torch
    from bit_quantized_optimizer_b200.zero1 import FlatLayout, ZeroAdamW4
    layout = FlatLayout([t["numel"] for t in ts], world, chunks)
    fp = torch.zeros(layout.padded, dtype=wdtype, device=device)
    fg = torch.zeros(layout.padded, dtype=torch.bfloat16, device=device)
    params, _ = workloads.device_inputs(WORKLOAD, ts, device=device, seed=0)
    for i, p in enumerate(params):
        layout.tensor_view(fp, i).copy_(p)
    del params, _
    _, grads = workloads.device_inputs(WORKLOAD, ts, device=device, seed=rank + 1)
    for i, g in enumerate(grads):
        layout.tensor_view(fg, i).copy_(g)
    del grads, _
    opt = ZeroAdamW4(fp, fg, layout, ts, lr=1e-3, vcode=vcode, seed=0, make_stepper=make_stepper)
    return layout, fp, fg, opt


def run_zero1(args):
    """The ZeRO-1 step: reduce-scatter (bf16, sum) -> the step kernel on the
    rank's shard, one handle per chunk -> all-gather (fp32), chunked so the
    collectives of one chunk run under the step of another.  value = the
    workload's params / the max over ranks of the device time per step (the
    total work is fixed: strong scaling).  The roofline is the step kernel's,
    from CUDA events around its launches (the rank's shard's algorithmic
    bytes over their mean duration); e2e adds, every step, the copy of the
    rank's grads from pinned host memory and of the updated weights back."""
    import datetime
    import torch
    import torch.distributed as dist
    ws_, rank, local = dist_setup(args.gpus)
    if ws_ == 1:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", 0))
    import bit_quantized_optimizer_b200 as B
    from bit_quantized_optimizer_b200.zero1 import piece_spec
    B.lib()  # fail loudly if the extension is missing
    vcode = VCODES[args.vcode]
    ts = workloads.tensor_list(WORKLOAD)
    wdt = torch.bfloat16 if args.bf16_params else torch.float32
    layout, fp, fg, opt = zero1_setup(ts, ws_, rank, args.chunks, wdt, "cuda", vcode)
    torch.cuda.synchronize()
    nparams = sum(t["numel"] for t in ts)
    # the algorithmic bytes of this rank's pieces (its share of the step kernel)
    mine = [piece_spec(ts[p.tensor], p) for k in range(layout.chunks)
            for p in layout.pieces(rank, k)]
    alg_rank = algorithmic_bytes(mine, fp.element_size())
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        opt.step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    opt.kernel_events = []
    barrier(ws_)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        opt.step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(ws_)
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), ws_) / args.steps
    kernel_ms = sum(a.elapsed_time(b) for a, b in opt.kernel_events) / args.steps
    kernel_ms = max_over_ranks(kernel_ms, ws_)
    opt.kernel_events = None
    launches = sum(1 for s_ in opt.steppers if s_ is not None)

    e2e = None
    if not args.no_e2e:
        # grads of this rank H2D into the flat buffer, the step, weights D2H
        e2e_steps = max(1, min(3, args.steps))
        hg = torch.empty(fg.numel(), dtype=torch.int16).pin_memory()
        hp = torch.empty(fp.numel(), dtype=fp.dtype).pin_memory()
        hg.copy_(fg.view(torch.int16))
        barrier(ws_)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            fg.view(torch.int16).copy_(hg, non_blocking=True)
            opt.step()
            hp.copy_(fp, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws_)
        e2e = {"value": nparams / (e2e_ms * 1e-3) / 1e9, "unit": "Gparams/s",
               "h2d_bytes_per_step": 2 * fg.numel(), "d2h_bytes_per_step":
               fp.element_size() * fp.numel(), "steps": e2e_steps}
        del hg, hp
    if rank == 0:
        peak, peak_kind = peaks()
        achieved = alg_rank / (kernel_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": nparams / (ms * 1e-3) / 1e9, "unit": "Gparams/s",
            "n_gpus": ws_, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "vcode": args.vcode, "params": nparams,
                       "tensors": len(ts), "parallelism": f"zero1 x{ws_}",
                       "weights": "bf16" if args.bf16_params else "fp32",
                       "chunks": args.chunks, "shard_elems_per_chunk": layout.shard,
                       "reduce_scatter_bytes_per_rank": 2 * layout.padded,
                       "all_gather_bytes_per_rank": fp.element_size() * layout.padded,
                       "algorithmic_bytes_per_step": algorithmic_bytes(ts, fp.element_size()),
                       "algorithmic_bytes_per_rank": alg_rank,
                       "l2": "inputs 19.7 GB > 126 MB L2; no flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind, "traffic": None,
                         "kernel_ms_per_step": kernel_ms,
                         "of": "the step kernel's launches on rank 0's shard (CUDA events)"},
            "e2e": e2e,
            "gpu_launches": args.steps * launches,
            "clocks": clk,
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    opt.close()
    dist.destroy_process_group()
    return 0


def run_sweep(args):
    """Single tensors of 4096 * 4^k values, k = 0..8 (4 K to 256 M): the
    step's time per launch with L2 flushed before every timed launch (a
    256 MB write between launches, outside the timed interval), for ZIP-SR
    and ZE-EDEN (or the v code chosen with --no-companion).  One JSON line per
    size and code; a profiling aid beside the headline line."""
    import torch
    import bit_quantized_optimizer_b200 as B
    torch.cuda.set_device(0)
    B.lib()
    names = [args.vcode] if args.no_companion else ["zipsr", "zeeden"]
    sweep_floor(args)
    for name in names:
        sweep_one(args, B, name)
    return 0


def sweep_floor(args):
    """The timing floor of the sweep's method: the same flush and event
    bracket around a one-element fill (one tiny library kernel), so that the
    step's fixed cost per launch can be read as the part above this."""
    import torch
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    tiny = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        tiny.fill_(0.0)
    times = []
    for _ in range(max(args.steps // 10, 5)):
        flush.fill_(1.0)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        tiny.fill_(2.0)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    print(json.dumps({"sweep": "floor", "what": "one-element fill, same flush and event bracket",
                      "us": float(np.median(times)) * 1e3,
                      "us_p10": float(np.percentile(times, 10)) * 1e3,
                      "us_p90": float(np.percentile(times, 90)) * 1e3}), flush=True)


def sweep_one(args, B, name):
    import torch
    vcode = VCODES[name]
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for n in [4096 * 4 ** k for k in range(9)]:
        ts = [dict(numel=n, tensor_id=0, flags=0, weight_decay=0.1)]
        gen = torch.Generator(device="cuda").manual_seed(n)
        w = torch.empty(n, device="cuda").normal_(0.0, 0.02, generator=gen)
        g = torch.empty(n, device="cuda").normal_(0.0, 1e-3, generator=gen).to(torch.bfloat16)
        opt = B.AdamW4([w], [g], ts, vcode=vcode)
        for _ in range(args.warmup):
            opt.step()
        times = []
        for _ in range(max(args.steps // 10, 5)):
            flush.fill_(1.0)                       # evict the tensor's data from L2
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            opt.step()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = float(np.median(times))
        alg = algorithmic_bytes(ts)
        peak, _ = peaks()
        print(json.dumps({"sweep": name, "numel": n, "ms_per_launch": ms,
                          "us_p10": float(np.percentile(times, 10)) * 1e3,
                          "us_p90": float(np.percentile(times, 90)) * 1e3,
                          "gparams": n / (ms * 1e-3) / 1e9, "hbm_gbs": alg / (ms * 1e-3) / 1e9,
                          "frac": alg / (ms * 1e-3) / 1e9 / peak, "l2": "flushed before each launch"}),
              flush=True)
        opt.close()
        del w, g


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--vcode", choices=list(VCODES), default="zipsr",
                    help="second-moment code: the two methods, or a state-space variant")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--bf16-params", action="store_true",
                    help="keep every tensor's weights in bf16 (ADAMW4_T_BF16_PARAM)")
    ap.add_argument("--zero1", action="store_true",
                    help="time the ZeRO-1 sharded step (reduce-scatter, step, all-gather); "
                         "the default for N > 1")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1: time N independent replicas (no collective) instead")
    ap.add_argument("--no-companion", action="store_true",
                    help="time only the chosen v code (not also the other method)")
    ap.add_argument("--sweep", action="store_true",
                    help="time single tensors of 4K..256M values (L2 flushed per launch)")
    ap.add_argument("--chunks", type=int, default=4,
                    help="ZeRO-1 pipeline chunks (collectives of one overlap the step of another)")
    ap.add_argument("--workload", default=WORKLOAD, choices=["gpt-2.7b", "llama-1.1b", "gpt-130m"],
                    help="tensor list (the benchmark is gpt-2.7b; the others are profiling cases)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)     # at least three untimed steps
    globals()["WORKLOAD"] = args.workload
    if args.impl == "reference":
        return run_reference(args)
    if args.zero1 or (int(os.environ.get("WORLD_SIZE", "1")) > 1 and not args.replicas):
        return run_zero1(args)
    if args.sweep:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
