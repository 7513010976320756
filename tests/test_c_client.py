"""A plain C program drives the library through the C ABI alone (no Python in
the loop) -- CPU: it compiles and links against libadamw4.so; GPU: its
results equal the oracle's."""
import os
import shutil
import struct
import subprocess

import numpy as np
import pytest

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_quantized_optimizer_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    from bit_quantized_optimizer_b200 import build
    build.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    assert cc, "a C compiler is needed"
    exe = str(tmp_path / "c_client")
    cmd = [cc, "-std=c11", "-O2", "-Wall", "-Wextra", os.path.join(ROOT, "tests", "c_client.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", PKG, "-ladamw4", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{PKG}:{os.path.join(CUDA, 'lib64')}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_client_builds_against_the_library(tmp_path):
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
@pytest.mark.parametrize("vcode", [0, 1])
def test_c_client_matches_the_oracle(vcode, tmp_path):
    from gpu_common import assert_state_equal, assert_weights_close, oracle_for
    exe = _compile(tmp_path)
    ts = [dict(numel=128 * 60 + 9, tensor_id=2, flags=0, weight_decay=0.1),
          dict(numel=4096, tensor_id=3, flags=workloads.T_LM_HEAD, weight_decay=0.0),
          dict(numel=777, tensor_id=4, flags=0, weight_decay=0.1)]
    steps, seed, total = 3, 12345, 3
    rng = np.random.default_rng(vcode)
    ws = [(rng.standard_normal(t["numel"]) * 0.02).astype(np.float32) for t in ts]
    gs = [[workloads.bf16_bits((rng.standard_normal(t["numel"]) * 1e-3).astype(np.float32))
           for t in ts] for _ in range(steps)]
    inp, out = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        f.write(struct.pack("<iiiiQq", len(ts), steps, vcode, 0, seed, total))
        for t in ts:
            f.write(struct.pack("<qIIfi", t["numel"], t["tensor_id"], t["flags"],
                                t["weight_decay"], 0))
        for w in ws:
            f.write(w.tobytes())
        for g in gs:
            for x in g:
                f.write(x.tobytes())
    r = subprocess.run([exe, str(inp), str(out)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
    data = open(out, "rb").read()
    off, got = 0, []
    for t in ts:
        got.append(np.frombuffer(data, np.float32, t["numel"], off))
        off += 4 * t["numel"]
    (blen,) = struct.unpack_from("<q", data, off)
    blob = data[off + 8:off + 8 + blen]

    ref = oracle_for(ts, vcode=vcode, seed=seed, total_steps=total)
    wref = [w.copy() for w in ws]
    for g in gs:
        old = [w.copy() for w in wref]
        ref.step(wref, g)
    for i, (a, b, o) in enumerate(zip(got, wref, old)):
        assert_weights_close(a, b, o, f"C client tensor {i}")
    assert_state_equal(blob, ref.export_state(), vcode, "C client")
