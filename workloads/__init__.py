"""Seeded synthetic inputs for the fused 4-bit AdamW step.

This module makes inputs only: tensor lists of the model shapes named below,
fp32 weights, bf16 gradients (as uint16 bit patterns) and synthetic packed
optimizer state.  It holds none of the optimizer's arithmetic; the oracle and
the CUDA path both consume what it makes.

Workloads (all synthetic; no dataset or checkpoint is involved):
  single-65k   one tensor of 65,536 elements, 10 steps, ZIP-SR.  w ~ N(0, 0.02^2);
               g ~ N(0, (1e-3)^2) fresh each step, with a fixed 10% of the
               coordinates scaled by 1e-4 so that v reaches the near-zero cell.
  single-4m    one tensor of 4,194,304 elements, 20 steps, ZE-EDEN; per block a
               sigma drawn log-uniform in [1e-5, 1e-2] once, g ~ N(0, sigma^2)
               fresh each step.
  gpt-130m     GPT-2-style tensor list: 12 layers, d 768, FFN 3072, vocab
               50,304, context 1024, tied head; LayerNorm tensors fp32.  g ~
               N(0, (1e-3 * 10^(-l/11))^2) for layer l; one step at t = 1000
               from pre-warmed synthetic state; ZIP-SR.
  llama-1.1b   Llama-style: 22 layers, d 2048, SwiGLU FFN 5632, vocab 32,000,
               grouped k/v projections 2048 -> 256, untied head, RMSNorm fp32;
               g = 1e-3 * Student-t(3); ZE-EDEN with the LM-head final-10% phase
               (T = 1000, steps 901..).
  gpt-2.7b     GPT-style: 32 layers, d 2560, FFN 10,240, vocab 50,304, context
               2048, untied head; g ~ N(0, (1e-3)^2); ZIP-SR and ZE-EDEN.
  microlm-p4   a 2-layer byte-level GPT (d 64, context 64, FFN 256, untied
               head): the smallest GPT whose fp32 and 4-bit persistent moment
               bytes equal the two figures of the WikiText-2 table of "ZIP-SR /
               ZE-EDEN: 4-bit AdamW state quantization" (Local reproduction).
Hyper-parameters for all: lr 1e-3, beta1 0.9, beta2 0.999, eps 1e-8, weight
decay 0.1 on every tensor, seed 0.
"""
from __future__ import annotations

import numpy as np

T_NORM = 1
T_LM_HEAD = 2
T_FP32_STATE = 4

HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, seed=0)


# ----------------------------------------------------------------------------
# bf16 bit patterns
# ----------------------------------------------------------------------------

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Rounds fp32 values to bf16 (nearest, ties to even) and returns the bit
    patterns as uint16.  Inputs are finite."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# Tensor lists
# ----------------------------------------------------------------------------

def _t(name, numel, flags=0, layer=-1):
    return dict(name=name, numel=int(numel), flags=flags, layer=layer)


def gpt_tensors(n_layer, d, ffn, vocab, ctx, tied):
    ts = [_t("wte", vocab * d), _t("wpe", ctx * d)]
    for l in range(n_layer):
        ts += [_t(f"h{l}.ln1.w", d, T_NORM, l), _t(f"h{l}.ln1.b", d, T_NORM, l),
               _t(f"h{l}.attn.qkv.w", d * 3 * d, 0, l), _t(f"h{l}.attn.qkv.b", 3 * d, 0, l),
               _t(f"h{l}.attn.proj.w", d * d, 0, l), _t(f"h{l}.attn.proj.b", d, 0, l),
               _t(f"h{l}.ln2.w", d, T_NORM, l), _t(f"h{l}.ln2.b", d, T_NORM, l),
               _t(f"h{l}.mlp.fc.w", d * ffn, 0, l), _t(f"h{l}.mlp.fc.b", ffn, 0, l),
               _t(f"h{l}.mlp.proj.w", ffn * d, 0, l), _t(f"h{l}.mlp.proj.b", d, 0, l)]
    ts += [_t("lnf.w", d, T_NORM), _t("lnf.b", d, T_NORM)]
    if not tied:
        ts.append(_t("lm_head", vocab * d, T_LM_HEAD))
    else:
        ts[0]["flags"] |= T_LM_HEAD   # the tied embedding is the head
    return ts


def llama_tensors(n_layer, d, ffn, vocab, kv_dim):
    ts = [_t("embed", vocab * d)]
    for l in range(n_layer):
        ts += [_t(f"l{l}.attn_norm", d, T_NORM, l),
               _t(f"l{l}.q", d * d, 0, l), _t(f"l{l}.k", d * kv_dim, 0, l),
               _t(f"l{l}.v", d * kv_dim, 0, l), _t(f"l{l}.o", d * d, 0, l),
               _t(f"l{l}.mlp_norm", d, T_NORM, l),
               _t(f"l{l}.gate", d * ffn, 0, l), _t(f"l{l}.up", d * ffn, 0, l),
               _t(f"l{l}.down", ffn * d, 0, l)]
    ts += [_t("norm", d, T_NORM), _t("lm_head", vocab * d, T_LM_HEAD)]
    return ts


def with_ids(ts, weight_decay=HYPER["weight_decay"]):
    out = []
    for i, t in enumerate(ts):
        t = dict(t)
        t["tensor_id"] = i
        t["weight_decay"] = weight_decay
        out.append(t)
    return out


TENSOR_LISTS = {
    "gpt-130m": lambda: with_ids(gpt_tensors(12, 768, 3072, 50304, 1024, tied=True)),
    "llama-1.1b": lambda: with_ids(llama_tensors(22, 2048, 5632, 32000, 256)),
    "gpt-2.7b": lambda: with_ids(gpt_tensors(32, 2560, 10240, 50304, 2048, tied=False)),
    "microlm-p4": lambda: with_ids(gpt_tensors(2, 64, 256, 256, 64, tied=False)),
    "single-65k": lambda: with_ids([_t("w", 65536)]),
    "single-4m": lambda: with_ids([_t("w", 4194304)]),
    # one 4-bit tensor past 2^31 elements (ragged tail), an LM head and a norm
    "huge-2g": lambda: with_ids([_t("w", (1 << 31) + 300), _t("head", 128 * 4096, T_LM_HEAD),
                                 _t("ln", 5000, T_NORM)]),
}

WORKLOADS = {
    "single-65k": dict(vcode=0, steps=10, t0=0, total_steps=0),
    "single-4m": dict(vcode=1, steps=20, t0=0, total_steps=0),
    "gpt-130m": dict(vcode=0, steps=1, t0=999, total_steps=0),
    "llama-1.1b": dict(vcode=1, steps=10, t0=900, total_steps=1000),
    "gpt-2.7b": dict(vcode=0, steps=100, t0=0, total_steps=0),
}


def tensor_list(name):
    return TENSOR_LISTS[name]()


# ----------------------------------------------------------------------------
# Host generation (numpy PCG64)
# ----------------------------------------------------------------------------

def _rng(*key):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _layer_scale(t, n_layer):
    if t.get("layer", -1) < 0:
        return 1.0
    return 10.0 ** (-t["layer"] / max(n_layer - 1, 1))


def host_weights(name, ts, seed=0):
    """fp32 weights ~ N(0, 0.02^2), one stream per tensor."""
    return [(_rng(seed, 1, t["tensor_id"]).standard_normal(t["numel"], np.float32)
             * np.float32(0.02)).astype(np.float32) for t in ts]


def host_grads(name, ts, step, seed=0):
    """bf16 gradients of step `step` (1-based) for the named workload."""
    out = []
    n_layer = 1 + max([t.get("layer", -1) for t in ts] + [0])
    for t in ts:
        n = t["numel"]
        r = _rng(seed, 2, t["tensor_id"], step)
        if name == "single-65k":
            mask = _rng(seed, 3, t["tensor_id"]).random(n) < 0.1
            g = r.standard_normal(n, np.float32) * np.float32(1e-3)
            g[mask] *= np.float32(1e-4)
        elif name == "single-4m":
            nb = (n + 127) // 128
            lo, hi = np.log(1e-5), np.log(1e-2)
            sig = np.exp(_rng(seed, 4, t["tensor_id"]).uniform(lo, hi, nb)).astype(np.float32)
            g = r.standard_normal(n, np.float32) * np.repeat(sig, 128)[:n]
        elif name == "gpt-130m":
            g = r.standard_normal(n, np.float32) * np.float32(1e-3 * _layer_scale(t, n_layer))
        elif name == "llama-1.1b":
            g = (r.standard_t(3, n) * 1e-3).astype(np.float32)
        else:
            g = r.standard_normal(n, np.float32) * np.float32(1e-3)
        out.append(bf16_bits(g))
    return out


def synthetic_state_blob(ts, vcode, t, seed=0, sigma=1e-3, is_fp32=None):
    """A packed state blob in the checkpoint layout with synthetic contents:
    m codes spread around the NF4 zero level, v codes skewed to small values
    (ZIP-SR blocks include zeros), positive scales of the size a gradient of
    scale `sigma` gives.  `is_fp32(numel, flags)` picks the fp32 tensors.
    Returns bytes."""
    import struct
    parts = []
    for tt in ts:
        n, tid, fl = tt["numel"], tt["tensor_id"], tt["flags"]
        r = _rng(seed, 5, tid)
        if is_fp32(n, fl):
            m = (r.standard_normal(n, np.float32) * np.float32(0.3 * sigma)).astype(np.float32)
            v = (np.float32(sigma * sigma)
                 * (0.5 + 0.5 * r.chisquare(1, n))).astype(np.float32)
            parts += [struct.pack("<IIq", tid, 1, n), m.tobytes(), v.tobytes()]
            continue
        nb = (n + 127) // 128
        mc = np.clip(np.rint(7.5 + 2.2 * r.standard_normal(nb * 128)), 0, 15).astype(np.uint8)
        if vcode == 0:
            vc = np.minimum(r.geometric(0.25, nb * 128) - 1, 15).astype(np.uint8)
        else:
            vc = np.minimum(r.geometric(0.3, nb * 128) - 1, 15).astype(np.uint8)
        pad = nb * 128 - n
        if pad:
            mc[n:] = 0
            vc[n:] = 0
        mpk = (mc[0::2] | (mc[1::2] << 4)).astype(np.uint8)
        vpk = (vc[0::2] | (vc[1::2] << 4)).astype(np.uint8)
        ms = (np.float32(3.0 * 0.3 * sigma) * (0.5 + r.random(nb))).astype(np.float32)
        vs = (np.float32(sigma * sigma) * (1.0 + 4.0 * r.random(nb))).astype(np.float32)
        parts += [struct.pack("<IIq", tid, 0, n), mpk.tobytes(), vpk.tobytes(), ms.tobytes(),
                  vs.tobytes()]
    payload = b"".join(parts)
    return b"ADAMW4S1" + struct.pack("<IIqQQ", len(ts), vcode, t, seed, len(payload)) + payload


# ----------------------------------------------------------------------------
# Device generation (torch, seeded CUDA generator) for the full-size lists
# ----------------------------------------------------------------------------

def device_inputs(name, ts, device="cuda", seed=0, dtype_grad_bits=True):
    """Allocates and fills fp32 weights and bf16 gradients on the device with
    a seeded torch generator: w ~ N(0, 0.02^2); g as `host_grads` describes
    for the workload (Student-t(3) for llama-1.1b, layer-scaled normals for
    gpt-130m, N(0, (1e-3)^2) otherwise).  Each tensor is its own allocation.
    Returns (params, grads) as lists of torch tensors (float32 / bfloat16)."""
    import torch
    gen = torch.Generator(device=device)
    params, grads = [], []
    n_layer = 1 + max([t.get("layer", -1) for t in ts] + [0])
    for t in ts:
        n = t["numel"]
        gen.manual_seed((seed * 1000003 + 2 * t["tensor_id"]) & 0x7FFFFFFFFFFF)
        w = torch.empty(n, dtype=torch.float32, device=device)
        w.normal_(0.0, 0.02, generator=gen)
        gen.manual_seed((seed * 1000003 + 2 * t["tensor_id"] + 1) & 0x7FFFFFFFFFFF)
        g = torch.empty(n, dtype=torch.float32, device=device)
        if name == "llama-1.1b":
            # Student-t(3) = N / sqrt(chi2_3 / 3), chi2_3 = sum of three squared normals
            g.normal_(0.0, 1.0, generator=gen)
            c = torch.empty(n, dtype=torch.float32, device=device)
            acc = torch.zeros(n, dtype=torch.float32, device=device)
            for _ in range(3):
                c.normal_(0.0, 1.0, generator=gen)
                acc.addcmul_(c, c)
            g.mul_(torch.rsqrt(acc / 3.0)).mul_(1e-3)
            del c, acc
        elif name == "gpt-130m":
            g.normal_(0.0, 1e-3 * _layer_scale(t, n_layer), generator=gen)
        else:
            g.normal_(0.0, 1e-3, generator=gen)
        params.append(w)
        grads.append(g.to(torch.bfloat16))
        del g
    return params, grads
