"""The oracle stepping pieces of tensors (test infrastructure).

A piece is the part [elem_offset, elem_offset + numel) of a tensor, as the
ZeRO-1 sharding hands it to one rank.  4-bit pieces go through the oracle's
block-list entry with the blocks' indices in the whole tensor, so every block
and every draw is keyed exactly as in a step of the whole tensor; fp32 pieces
go through its elementwise fp32 step.  The object has the stepper interface
``ZeroAdamW4`` expects: step(lr), state_dict_blob(), load_state_blob(blob).
"""
import ctypes
import struct

import numpy as np
import torch

import oracle

T_QUANT_STATE = 8


def _np_f32(t):
    return t.detach().numpy()


def _is_bf16(t):
    return t.dtype == torch.bfloat16


def _np_u16(t):
    return t.detach().view(torch.int16).numpy().view(np.uint16)


class OraclePieces:
    def __init__(self, params, grads, pspecs, *, vcode, seed, total_steps, lr=1e-3,
                 betas=(0.9, 0.999), eps=1e-8):
        self.params, self.grads = list(params), list(grads)
        self.specs = [dict(s) for s in pspecs]
        self.vcode, self.seed, self.total_steps = int(vcode), int(seed), int(total_steps)
        self.betas, self.eps, self.lr = betas, eps, lr
        self.t = 0
        self.state = []
        for s in self.specs:
            n = s["numel"]
            if s["flags"] & T_QUANT_STATE:
                nb = (n + 127) // 128
                self.state.append(dict(kind=0, nb=nb, mcodes=np.zeros(nb * 64, np.uint8),
                                       vcodes=np.zeros(nb * 64, np.uint8),
                                       mscale=np.zeros(nb, np.float32),
                                       vscale=np.zeros(nb, np.float32)))
            else:
                self.state.append(dict(kind=1, m=np.zeros(n, np.float32),
                                       v=np.zeros(n, np.float32)))

    def step(self, lr):
        L = oracle.lib()
        self.t += 1
        s = oracle.make_scalars(np.float32(lr), np.float32(self.betas[0]),
                                np.float32(self.betas[1]), np.float32(self.eps), self.t,
                                self.total_steps, self.seed)
        for p, g, spec, st in zip(self.params, self.grads, self.specs, self.state):
            # bf16 weights: widened exactly, stepped in binary32, stored rounded
            w = ((_np_u16(p).astype(np.uint32) << 16).view(np.float32) if _is_bf16(p)
                 else _np_f32(p))
            gb = _np_u16(g)
            n, e0 = spec["numel"], spec["elem_offset"]
            if st["kind"] == 1:
                L.oracle_step_fp32(ctypes.byref(s), spec["weight_decay"], n, w, gb,
                                   st["m"], st["v"])
                if _is_bf16(p):
                    _np_u16(p)[:] = oracle.round_bf16(w)
                continue
            nb = st["nb"]
            blocks = np.arange(e0 // 128, e0 // 128 + nb, dtype=np.int64)
            w_sel = np.zeros(nb * 128, np.float32)
            g_sel = np.zeros(nb * 128, np.uint16)
            w_sel[:n], g_sel[:n] = w, gb
            m_sr = int(bool(spec["flags"] & oracle.T_LM_HEAD) and s.lm_sr_active)
            # a piece ends on a block boundary unless it ends the tensor, so
            # e0 + n stands for the tensor's numel in the ragged-block test
            L.oracle_step_blocks4(ctypes.byref(s), spec["weight_decay"], self.vcode, m_sr,
                                  spec["tensor_id"], e0 + n, nb, blocks, w_sel, g_sel,
                                  st["mcodes"], st["mscale"], st["vcodes"], st["vscale"])
            if _is_bf16(p):
                _np_u16(p)[:] = oracle.round_bf16(w_sel[:n])
            else:
                w[:] = w_sel[:n]

    def state_dict_blob(self) -> bytes:
        parts = []
        for spec, st in zip(self.specs, self.state):
            parts.append(struct.pack("<IIq", spec["tensor_id"], st["kind"], spec["numel"]))
            keys = ("mcodes", "vcodes", "mscale", "vscale") if st["kind"] == 0 else ("m", "v")
            parts += [st[k].tobytes() for k in keys]
        payload = b"".join(parts)
        return b"ADAMW4S1" + struct.pack("<IIqQQ", len(self.specs), self.vcode, self.t,
                                         self.seed, len(payload)) + payload

    def load_state_blob(self, blob: bytes):
        n, vcode, t, seed, plen = struct.unpack_from("<IIqQQ", blob, 8)
        assert n == len(self.specs) and vcode == self.vcode and seed == self.seed
        off = 40
        for spec, st in zip(self.specs, self.state):
            tid, kind, numel = struct.unpack_from("<IIq", blob, off)
            off += 16
            assert (tid, kind, numel) == (spec["tensor_id"], st["kind"], spec["numel"])
            keys = ((("mcodes", np.uint8), ("vcodes", np.uint8), ("mscale", np.float32),
                     ("vscale", np.float32)) if kind == 0 else
                    (("m", np.float32), ("v", np.float32)))
            for k, dt in keys:
                cnt = st[k].size
                st[k] = np.frombuffer(blob, dt, cnt, off).copy()
                off += cnt * np.dtype(dt).itemsize
        self.t = t
