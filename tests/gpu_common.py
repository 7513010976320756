"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, then compare element by element.

Tolerances (stated with the workloads): codes bit-exact; m scales and ZIP-SR v
scales bit-exact (both are a maximum of identical binary32 values); ZE-EDEN v
scales within 1e-6 relative; weights within 1e-6 relative to the larger of the
old and new |w|.  Both sides follow one binary32 evaluation order, so all of
these are expected to hold with zero difference; the tolerances are the
stated bar, not slack that is needed.
"""
import struct

import numpy as np

import oracle
import workloads

B = None


def binding():
    global B
    if B is None:
        import bit_quantized_optimizer_b200 as mod
        from bit_quantized_optimizer_b200 import build
        build.build()
        mod.lib()
        B = mod
    return B


def parse_blob(blob):
    """Splits a checkpoint blob into per-tensor dicts of numpy arrays."""
    n, vcode, t, seed, plen = struct.unpack_from("<IIqQQ", blob, 8)
    off = 40
    out = []
    for _ in range(n):
        tid, kind, numel = struct.unpack_from("<IIq", blob, off)
        off += 16
        d = dict(tensor_id=tid, fp32=bool(kind), numel=numel)
        if kind:
            d["m"] = np.frombuffer(blob, np.float32, numel, off); off += 4 * numel
            d["v"] = np.frombuffer(blob, np.float32, numel, off); off += 4 * numel
        else:
            nb = (numel + 127) // 128
            d["mcodes"] = np.frombuffer(blob, np.uint8, nb * 64, off); off += nb * 64
            d["vcodes"] = np.frombuffer(blob, np.uint8, nb * 64, off); off += nb * 64
            d["mscale"] = np.frombuffer(blob, np.float32, nb, off); off += 4 * nb
            d["vscale"] = np.frombuffer(blob, np.float32, nb, off); off += 4 * nb
        out.append(d)
    return dict(t=t, vcode=vcode, seed=seed, tensors=out)


def assert_weights_close(w_gpu, w_ref, w_old, what=""):
    w_gpu = np.asarray(w_gpu, np.float64)
    w_ref = np.asarray(w_ref, np.float64)
    scale = np.maximum(np.abs(w_ref), np.abs(np.asarray(w_old, np.float64)))
    with np.errstate(invalid="ignore"):            # equal infinities subtract to NaN
        same = (w_gpu == w_ref) | (np.isnan(w_gpu) & np.isnan(w_ref))
        bad = ~same & ~(np.abs(w_gpu - w_ref) <= 1e-6 * scale)
    assert not bad.any(), (f"{what}: {bad.sum()} weights differ beyond 1e-6, first at "
                           f"{np.argmax(bad)}: gpu {w_gpu[bad][0]!r} oracle {w_ref[bad][0]!r}")


def assert_state_equal(blob_gpu, blob_ref, vcode, what=""):
    a, b = parse_blob(blob_gpu), parse_blob(blob_ref)
    assert a["t"] == b["t"]
    for x, y in zip(a["tensors"], b["tensors"]):
        tag = f"{what} tensor {x['tensor_id']}"
        assert x["fp32"] == y["fp32"]
        if x["fp32"]:
            np.testing.assert_allclose(x["m"], y["m"], rtol=1e-6, atol=0, err_msg=tag + " m")
            np.testing.assert_allclose(x["v"], y["v"], rtol=1e-6, atol=0, err_msg=tag + " v")
            continue
        for k in ("mcodes", "vcodes"):
            diff = np.nonzero(x[k] != y[k])[0]
            assert diff.size == 0, (f"{tag} {k}: {diff.size} bytes differ, first byte {diff[0]} "
                                    f"(block {diff[0] // 64}) gpu {x[k][diff[0]]:#04x} "
                                    f"oracle {y[k][diff[0]]:#04x}")
        assert np.array_equal(x["mscale"], y["mscale"]), tag + " m scales"
        if vcode != 1:             # only ZE-EDEN rescales (a division); the others store s
            assert np.array_equal(x["vscale"], y["vscale"]), tag + " v scales"
        else:
            np.testing.assert_allclose(x["vscale"], y["vscale"], rtol=1e-6, atol=0,
                                       err_msg=tag + " v scales")


class CudaRun:
    """The CUDA path over a tensor list with host-provided inputs."""

    def __init__(self, ts, host_ws, vcode=0, seed=0, total_steps=0, lr=1e-3, beta1=0.9,
                 beta2=0.999, eps=1e-8, blob=None, t0=None):
        import torch
        Bm = binding()
        self.torch = torch
        # uint16 host arrays are bf16 weights (tensors flagged ADAMW4_T_BF16_PARAM)
        self.params = [torch.from_numpy(np.ascontiguousarray(w).view(np.int16)).cuda()
                       .view(torch.bfloat16) if w.dtype == np.uint16 else
                       torch.from_numpy(np.ascontiguousarray(w)).cuda() for w in host_ws]
        self.grads = [torch.zeros(t["numel"], dtype=torch.bfloat16, device="cuda") for t in ts]
        self.opt = Bm.AdamW4(self.params, self.grads, ts, lr=lr, betas=(beta1, beta2), eps=eps,
                             vcode=vcode, seed=seed, total_steps=total_steps)
        if blob is not None:
            self.opt.load_state_blob(blob)
        if t0 is not None:
            self.opt.t = t0

    def set_grads(self, host_grads):
        for g, hg in zip(self.grads, host_grads):
            g.view(self.torch.int16).copy_(self.torch.from_numpy(hg.view(np.int16)))

    def step(self, host_grads=None, lr=None):
        if host_grads is not None:
            self.set_grads(host_grads)
        self.opt.step(lr)

    def weights(self):
        self.torch.cuda.synchronize()
        return [p.view(self.torch.int16).cpu().numpy().view(np.uint16)
                if p.dtype == self.torch.bfloat16 else p.cpu().numpy() for p in self.params]

    def blob(self):
        return self.opt.state_dict_blob()

    def close(self):
        self.opt.close()


def oracle_for(ts, vcode=0, seed=0, total_steps=0, nthreads=None, lr=1e-3, beta1=0.9,
               beta2=0.999, eps=1e-8):
    if nthreads is None:
        nthreads = max(1, oracle.max_threads())
    return oracle.OracleAdamW4(lr=lr, beta1=beta1, beta2=beta2, eps=eps, vcode=vcode, seed=seed,
                               total_steps=total_steps, tensors=ts, nthreads=nthreads)


def run_both(ts, host_ws, grads_fn, steps, vcode=0, seed=0, total_steps=0, blob=None, t0=None,
             check_every_step=False, what=""):
    """Steps the CUDA path and the oracle `steps` times from the same inputs
    and compares state and weights (after every step if asked, else at the
    end).  grads_fn(step) returns the host bf16 grads of that step."""
    gpu = CudaRun(ts, host_ws, vcode=vcode, seed=seed, total_steps=total_steps, blob=blob, t0=t0)
    ref = oracle_for(ts, vcode=vcode, seed=seed, total_steps=total_steps)
    if blob is not None:
        ref.import_state(blob)
    if t0 is not None:
        ref.t = t0
    ws = [w.copy() for w in host_ws]
    try:
        for s in range(1, steps + 1):
            gs = grads_fn(s)
            old = [w.copy() for w in ws]
            gpu.step(gs)
            ref.step(ws, gs)
            if check_every_step or s == steps:
                wg = gpu.weights()
                for i, (a, b, o) in enumerate(zip(wg, ws, old)):
                    if a.dtype == np.uint16:          # bf16 weights: bit for bit
                        assert np.array_equal(a, b), f"{what} step {s} tensor {i} (bf16)"
                    else:
                        assert_weights_close(a, b, o, f"{what} step {s} tensor {i}")
                assert_state_equal(gpu.blob(), ref.export_state(), vcode, f"{what} step {s}")
        return gpu, ref, ws
    finally:
        gpu.close()


def sampled_blocks(ts, per_tensor=6, head_extra=192, seed=0):
    """Blocks to check per quantised tensor: the first, the last (the ragged
    one if any) and a few random ones; more on the LM head; and, in a tensor
    past 2^31 elements, the blocks on either side of element 2^31."""
    rng = np.random.default_rng(seed)
    out = {}
    for i, t in enumerate(ts):
        if oracle.is_fp32_state(t["numel"], t["flags"]):
            continue
        nb = (t["numel"] + 127) // 128
        k = per_tensor + (head_extra if t["flags"] & workloads.T_LM_HEAD else 0)
        sel = {0, nb - 1} | set(rng.integers(0, nb, size=min(k, nb)).tolist())
        if nb > (1 << 24) + 1:
            sel |= {(1 << 24) - 1, 1 << 24, (1 << 24) + 1}
        out[i] = np.array(sorted(sel), np.int64)
    return out


def _gather_blocks(vec, numel, blocks, dtype):
    """Host copy of whole 128-slot blocks of a device vector (zero padded)."""
    import torch
    idx = (blocks[:, None] * 128 + np.arange(128)[None, :]).reshape(-1)
    valid = idx < numel
    out = np.zeros(idx.size, dtype)
    src = vec[torch.from_numpy(idx[valid]).to(vec.device)].cpu()
    if dtype == np.uint16:
        out[valid] = src.view(torch.int16).numpy().view(np.uint16)
    else:
        out[valid] = src.numpy()
    return out, valid


def sampled_parity(name, vcode, steps, t0=0, total_steps=0, prewarm=False, seed=0, what=""):
    """Full-size run of the CUDA path with device-generated inputs; the oracle
    recomputes the sampled blocks (and every fp32-state tensor) for the same
    steps.  Returns the number of blocks checked."""
    import torch
    ts = workloads.tensor_list(name)
    params, grads = workloads.device_inputs(name, ts, seed=seed)
    blob = (workloads.synthetic_state_blob(ts, vcode, t0, seed=seed, is_fp32=oracle.is_fp32_state)
            if prewarm else None)
    sel = sampled_blocks(ts, seed=seed)
    # oracle inputs, taken from the input buffers before any step runs
    ref_in = {}
    for i, blocks in sel.items():
        w, valid = _gather_blocks(params[i], ts[i]["numel"], blocks, np.float32)
        g, _ = _gather_blocks(grads[i], ts[i]["numel"], blocks, np.uint16)
        ref_in[i] = dict(blocks=blocks, w=w, w0=w.copy(), g=g, valid=valid)
    fp_idx = [i for i, t in enumerate(ts) if oracle.is_fp32_state(t["numel"], t["flags"])]
    fp_w = {i: params[i].cpu().numpy().copy() for i in fp_idx}
    fp_g = {i: grads[i].view(torch.int16).cpu().numpy().view(np.uint16).copy() for i in fp_idx}

    ref = oracle_for(ts, vcode=vcode, seed=0, total_steps=total_steps)
    if blob is not None:
        ref.import_state(blob)
        pb = parse_blob(blob)
        for i, d in ref_in.items():
            tb = pb["tensors"][i]
            bl = d["blocks"]
            d["mc"] = np.concatenate([tb["mcodes"][b * 64:(b + 1) * 64] for b in bl]).copy()
            d["vc"] = np.concatenate([tb["vcodes"][b * 64:(b + 1) * 64] for b in bl]).copy()
            d["ms"] = tb["mscale"][bl].copy()
            d["vs"] = tb["vscale"][bl].copy()
    else:
        ref.t = t0
        for d in ref_in.values():
            nsel = len(d["blocks"])
            d["mc"] = np.zeros(nsel * 64, np.uint8)
            d["vc"] = np.zeros(nsel * 64, np.uint8)
            d["ms"] = np.zeros(nsel, np.float32)
            d["vs"] = np.zeros(nsel, np.float32)

    B_ = binding()
    opt = B_.AdamW4(params, grads, ts, lr=1e-3, vcode=vcode, seed=0, total_steps=total_steps)
    try:
        if blob is not None:
            opt.load_state_blob(blob)
        else:
            opt.t = t0
        t_start = ref.t
        for s in range(steps):
            opt.step()
            ref.t = t_start + s + 1
            for i, d in ref_in.items():
                ref.step_blocks(i, d["blocks"], d["w"], d["g"], d["mc"], d["ms"], d["vc"], d["vs"],
                                advance=False)
            ref.step([fp_w[i] for i in fp_idx], [fp_g[i] for i in fp_idx], only=fp_idx,
                     advance=False)
        torch.cuda.synchronize()
        got = parse_blob(opt.state_dict_blob())
        checked = 0
        for i, d in ref_in.items():
            wg, valid = _gather_blocks(params[i], ts[i]["numel"], d["blocks"], np.float32)
            assert_weights_close(wg[valid], d["w"][valid], d["w0"][valid], f"{what} tensor {i}")
            tb = got["tensors"][i]
            for j, b in enumerate(d["blocks"]):
                for key, arr in (("mcodes", d["mc"]), ("vcodes", d["vc"])):
                    a = tb[key][b * 64:(b + 1) * 64]
                    e = arr[j * 64:(j + 1) * 64]
                    assert np.array_equal(a, e), f"{what} tensor {i} block {b} {key}"
                assert tb["mscale"][b] == d["ms"][j], f"{what} tensor {i} block {b} m scale"
                if vcode != 1:
                    assert tb["vscale"][b] == d["vs"][j], f"{what} tensor {i} block {b} v scale"
                else:
                    assert abs(tb["vscale"][b] - d["vs"][j]) <= 1e-6 * abs(d["vs"][j]), \
                        f"{what} tensor {i} block {b} v scale"
                checked += 1
        for i in fp_idx:
            st = ref.tensors[i]
            assert_weights_close(params[i].cpu().numpy(), fp_w[i], fp_w[i], f"{what} fp32 {i}")
            np.testing.assert_allclose(got["tensors"][i]["m"], st.m, rtol=1e-6, atol=0)
            np.testing.assert_allclose(got["tensors"][i]["v"], st.v, rtol=1e-6, atol=0)
        return checked
    finally:
        opt.close()
        del params, grads
        torch.cuda.empty_cache()


def teacher_forced_parity(name, vcode, steps, seed=0, what="", total_steps=0):
    """Runs the CUDA path for `steps` steps over a full-size list (device
    inputs, one seeded grad set reused every step, zero initial state), then
    checks the last step teacher-forced: the state and weights the GPU holds
    after step `steps` - 1 are given to the oracle, which computes step
    `steps` on sampled blocks of every 4-bit tensor and on every fp32-state
    tensor; the GPU's own step `steps` must match it.  Returns (blocks
    checked, shares of the sampled v codes that are 0 and 1 after step
    `steps` - 1).  total_steps: the run length that sets the LM head's
    final-10% phase (0: never)."""
    import torch
    ts = workloads.tensor_list(name)
    params, grads = workloads.device_inputs(name, ts, seed=seed)
    sel = sampled_blocks(ts, seed=seed + 1)
    fp_idx = [i for i, t in enumerate(ts) if oracle.is_fp32_state(t["numel"], t["flags"])]
    B_ = binding()
    opt = B_.AdamW4(params, grads, ts, lr=1e-3, vcode=vcode, seed=0, total_steps=total_steps)
    try:
        for _ in range(steps - 1):
            opt.step()
        torch.cuda.synchronize()
        before = parse_blob(opt.state_dict_blob())
        assert before["t"] == steps - 1
        ref = oracle_for(ts, vcode=vcode, seed=0, total_steps=total_steps)
        ref.t = steps - 1
        d_in = {}
        zero_codes, one_codes, n_codes = 0, 0, 0
        for i, blocks in sel.items():
            w, valid = _gather_blocks(params[i], ts[i]["numel"], blocks, np.float32)
            g, _ = _gather_blocks(grads[i], ts[i]["numel"], blocks, np.uint16)
            tb = before["tensors"][i]
            vc = np.concatenate([tb["vcodes"][b * 64:(b + 1) * 64] for b in blocks]).copy()
            nib = np.stack([vc & 15, vc >> 4], axis=1).reshape(-1)[:valid.size][valid]
            zero_codes += int((nib == 0).sum())
            one_codes += int((nib == 1).sum())
            n_codes += nib.size
            d_in[i] = dict(blocks=blocks, w=w, w0=w.copy(), g=g, valid=valid,
                           mc=np.concatenate([tb["mcodes"][b * 64:(b + 1) * 64] for b in blocks]).copy(),
                           vc=vc, ms=tb["mscale"][blocks].copy(), vs=tb["vscale"][blocks].copy())
        fp_w = {i: params[i].cpu().numpy().copy() for i in fp_idx}
        fp_g = {i: grads[i].view(torch.int16).cpu().numpy().view(np.uint16).copy() for i in fp_idx}
        for i in fp_idx:
            st = ref.tensors[i]
            st.m = before["tensors"][i]["m"].copy()
            st.v = before["tensors"][i]["v"].copy()
        del before
        # step `steps`: the GPU, and the oracle from the GPU's state
        opt.step()
        ref.t = steps
        for i, d in d_in.items():
            ref.step_blocks(i, d["blocks"], d["w"], d["g"], d["mc"], d["ms"], d["vc"], d["vs"],
                            advance=False)
        old_fp = {i: fp_w[i].copy() for i in fp_idx}
        ref.step([fp_w[i] for i in fp_idx], [fp_g[i] for i in fp_idx], only=fp_idx, advance=False)
        torch.cuda.synchronize()
        after = parse_blob(opt.state_dict_blob())
        checked = 0
        for i, d in d_in.items():
            wg, valid = _gather_blocks(params[i], ts[i]["numel"], d["blocks"], np.float32)
            assert_weights_close(wg[valid], d["w"][valid], d["w0"][valid], f"{what} tensor {i}")
            tb = after["tensors"][i]
            for j, b in enumerate(d["blocks"]):
                for key, arr in (("mcodes", d["mc"]), ("vcodes", d["vc"])):
                    assert np.array_equal(tb[key][b * 64:(b + 1) * 64], arr[j * 64:(j + 1) * 64]), \
                        f"{what} tensor {i} block {b} {key}"
                assert tb["mscale"][b] == d["ms"][j], f"{what} tensor {i} block {b} m scale"
                if vcode != 1:
                    assert tb["vscale"][b] == d["vs"][j], f"{what} tensor {i} block {b} v scale"
                else:
                    assert abs(tb["vscale"][b] - d["vs"][j]) <= 1e-6 * abs(d["vs"][j]), \
                        f"{what} tensor {i} block {b} v scale"
                checked += 1
        for i in fp_idx:
            st = ref.tensors[i]
            assert_weights_close(params[i].cpu().numpy(), fp_w[i], old_fp[i], f"{what} fp32 {i}")
            np.testing.assert_allclose(after["tensors"][i]["m"], st.m, rtol=1e-6, atol=0)
            np.testing.assert_allclose(after["tensors"][i]["v"], st.v, rtol=1e-6, atol=0)
        return checked, zero_codes / max(n_codes, 1), one_codes / max(n_codes, 1)
    finally:
        opt.close()
        del params, grads
        torch.cuda.empty_cache()
