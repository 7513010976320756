"""The 1-D quadratic diagnostic: the oracle shows the qualitative split the
pages describe (CPU), and the GPU run equals the oracle's (parity).

The pages give no constants for the construction; these are this library's
(see ``bit_quantized_optimizer_b200/quadratic.py``).  What is checked is the
shape of the result: after the gradient vanishes, state-space rounding of v
(to zero, where h = 1/eps) throws the 1-D weight orders of magnitude further
than exact AdamW, while preconditioner-space rounding (ZIP-SR) and the
zero-excluded codes stay within a small factor of it."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_optimizer_b200 import quadratic as Q


def oracle_run(cfg, method):
    w = Q.initial_weights(cfg)
    o = oracle.OracleAdamW4(lr=cfg["lr"], beta1=cfg["beta1"], beta2=cfg["beta2"], eps=cfg["eps"],
                            vcode=0 if method == Q.EXACT else method, seed=cfg["seed"],
                            tensors=[Q.spec(method, w.size)], nthreads=oracle.max_threads())
    out = [w[0::Q.BLOCK].copy()]
    for step in range(cfg["steps"]):
        prod = Q.curvatures(cfg, step) * w                 # binary32 product
        g = torch.from_numpy(prod).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        o.step([w], [g])
        out.append(w[0::Q.BLOCK].copy())
    return np.stack(out)


def test_state_space_rounding_throws_the_weight_after_the_gradient_vanishes():
    cfg = Q.default_config(replicas=512, steps=60, pulse=5)
    runs = {m: oracle_run(cfg, m) for m in (Q.EXACT, 0, 1, 3, 4)}
    s = {m: Q.summary(r, runs[Q.EXACT], cfg["pulse"]) for m, r in runs.items()}
    exact = abs(s[Q.EXACT]["drift_mean"])
    assert exact > 0
    # state space: the stored v rounds to zero and h = 1/eps takes over
    assert abs(s[3]["drift_median"]) > 1e3 * exact
    # preconditioner space and the zero-excluded codes stay within a factor of 20
    for m in (0, 1, 4):
        assert s[m]["drift_p99"] < 20 * exact, (m, s[m])


@pytest.mark.gpu
def test_gpu_run_equals_the_oracle_run():
    from gpu_common import binding
    binding()
    cfg = Q.default_config(replicas=64, steps=25, pulse=5)
    for m in Q.METHODS:
        got = Q.run(cfg, m)
        want = oracle_run(cfg, m)
        assert got.tobytes() == want.tobytes(), Q.NAMES[m]
