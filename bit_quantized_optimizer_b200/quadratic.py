"""One-dimensional quadratic diagnostic: state-space against
preconditioner-space rounding of the second moment.

"A New Approach to 4-bit AdamW Optimizer Quantization: Rounding in
Preconditioner Space" (kongchang.com), sections *Preconditioner* and *The
Blind Spot of State-Space Rounding*, describes a one-dimensional quadratic on
which the two rounding spaces give qualitatively different trajectories.  It
gives no constants; this module is this library's version of it.

- ``replicas`` independent copies, each one 128-value block of one tensor.
  Value 0 of a block is the 1-D problem f(w) = a w^2 / 2, started at
  ``w_small``.  Values 1..127 are companions, f = b w^2 / 2 started at
  N(0, 1), which keep the block's scale up.
- Every step the gradient is curvature x w in binary32, rounded to the
  nearest bf16 (ties to even); then one optimizer step.
- After ``pulse`` steps the 1-D problem's curvature is switched off: its
  gradient is exactly 0 from then on, its second moment decays towards the
  code cell next to zero, and its first moment keeps pushing.  This is the
  next-gradient-near-zero situation of the near-zero worked example in
  "ZIP-SR 4-bit AdamW -- Preconditioner-space stochastic rounding".  With
  ``pulse`` = ``steps`` the gradient never vanishes.
- Methods: exact AdamW (the same kernel with fp32 state, ``FP32_STATE``),
  ZIP-SR, ZE-EDEN and the three state-space quantisers (``vcode`` 0..4).

``run`` steps a method on the GPU and returns the 1-D problems' weights after
every step; ``summary`` reduces them to the diagnostic's numbers.
"""
from __future__ import annotations

import numpy as np

from . import ADAMW4_T_FP32_STATE, AdamW4

BLOCK = 128
EXACT = "exact"        # fp32-state AdamW, the reference trajectory
METHODS = (EXACT, 0, 1, 2, 3, 4)
NAMES = {EXACT: "fp32 AdamW", 0: "ZIP-SR", 1: "ZE-EDEN", 2: "zero-incl. nearest",
         3: "zero-incl. state-space SR", 4: "zero-excl. floor"}


def default_config(**kw):
    c = dict(replicas=4096, steps=100, pulse=5, a=1.0, b=1.0, w_small=1.0, lr=1e-3, beta1=0.9,
             beta2=0.999, eps=1e-8, seed=0)
    c.update(kw)
    return c


def initial_weights(cfg) -> np.ndarray:
    """fp32 weights of all replicas: w_small at value 0 of each block, the
    companions N(0, 1) (numpy PCG64 with the config's seed)."""
    rng = np.random.default_rng(cfg["seed"])
    w = rng.standard_normal(cfg["replicas"] * BLOCK).astype(np.float32)
    w[0::BLOCK] = np.float32(cfg["w_small"])
    return w


def curvatures(cfg, step) -> np.ndarray:
    """Curvature of every value at step `step` (0-based): a for the 1-D
    problems while step < pulse, then 0; b for the companions."""
    c = np.full(cfg["replicas"] * BLOCK, np.float32(cfg["b"]), np.float32)
    c[0::BLOCK] = np.float32(cfg["a"]) if step < cfg["pulse"] else np.float32(0.0)
    return c


def spec(method, numel) -> dict:
    return dict(numel=numel, tensor_id=1, weight_decay=0.0,
                flags=ADAMW4_T_FP32_STATE if method == EXACT else 0)


def run(cfg, method, device="cuda"):
    """Steps `method` on the GPU; returns the 1-D problems' weights after
    every step, shape (steps + 1, replicas), row 0 the start."""
    import torch
    w = torch.from_numpy(initial_weights(cfg)).to(device)
    on = torch.from_numpy(curvatures(cfg, 0)).to(device)
    off = torch.from_numpy(curvatures(cfg, cfg["pulse"])).to(device)
    g = torch.empty(w.numel(), dtype=torch.bfloat16, device=device)
    opt = AdamW4([w], [g], [spec(method, w.numel())], lr=cfg["lr"],
                 betas=(cfg["beta1"], cfg["beta2"]), eps=cfg["eps"],
                 vcode=0 if method == EXACT else method, seed=cfg["seed"])
    out = [w[0::BLOCK].cpu().numpy().copy()]
    try:
        for step in range(cfg["steps"]):
            curv = on if step < cfg["pulse"] else off
            g.copy_(torch.mul(curv, w))        # binary32 product, nearest-even bf16
            opt.step()
            out.append(w[0::BLOCK].cpu().numpy().copy())
    finally:
        opt.close()
    return np.stack(out)


def summary(traj, exact, pulse):
    """The 1-D weights' drift after the pulse (w_T - w_pulse) over the
    replicas -- mean, median, 99th percentile and maximum of its size -- and
    the mean distance from the exact trajectory over all steps."""
    d = traj[-1] - traj[pulse]
    a = np.abs(d)
    return dict(drift_mean=float(d.mean()), drift_median=float(np.median(d)),
                drift_p99=float(np.quantile(a, 0.99)), drift_max=float(a.max()),
                mean_abs_dev=float(np.abs(traj - exact).mean()))


def table(cfg=None):
    """The diagnostic over every method: rows of (name, summary)."""
    cfg = cfg or default_config()
    runs = {m: run(cfg, m) for m in METHODS}
    return [(NAMES[m], summary(runs[m], runs[EXACT], cfg["pulse"])) for m in METHODS]


if __name__ == "__main__":
    for pulse in (5, 100):
        cfg = default_config(pulse=pulse)
        print(f"1-D quadratic: {cfg['replicas']} replicas, {cfg['steps']} steps, gradient on for "
              f"{pulse}, a={cfg['a']}, b={cfg['b']}, w0={cfg['w_small']}, lr={cfg['lr']}, "
              f"betas=({cfg['beta1']}, {cfg['beta2']}), eps={cfg['eps']}")
        print(f"  {'method':28s} {'drift mean':>12s} {'median':>12s} {'p99 |d|':>11s} "
              f"{'max |d|':>11s} {'mean |w-w_ex|':>14s}")
        for name, r in table(cfg):
            print(f"  {name:28s} {r['drift_mean']:12.4e} {r['drift_median']:12.4e} "
                  f"{r['drift_p99']:11.3e} {r['drift_max']:11.3e} {r['mean_abs_dev']:14.4e}")
