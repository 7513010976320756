"""The checked build (-DADAMW4_CHECKED: every unit's element and state range
tested on the device, in place of a memory checker) finds nothing on a mixed
tensor list -- ragged and fp32-state tensors, bf16 weights, a piece of a
larger tensor, an LM head in its final-10% phase, all five v codes -- and
gives the same bits as the normal build."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _run(lib):
    env = dict(os.environ, ADAMW4_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_run.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_checked_build_finds_nothing_and_matches():
    from bit_quantized_optimizer_b200 import build
    normal = build.build()
    checked = build.build(checked=True)
    a, b = _run(normal), _run(checked)
    assert a["lib"] == normal and b["lib"] == checked
    assert a["hashes"] == b["hashes"]
