"""CPU oracle of the fused 4-bit AdamW step (ZIP-SR / ZE-EDEN).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg use it; the product library never does.  The arithmetic lives in
``adamw4_oracle.c`` (plain scalar C, binary32 canonical form); this module
builds it with gcc, binds it with ctypes and drives it over a tensor list with
the same classification, state layout and checkpoint format as the C ABI.

Pages followed (title -- section):
  "ZIP-SR / ZE-EDEN: 4-bit AdamW state quantization" (daiwk.github.io)
      -- Method flowchart; Core equation; Local reproduction notes
  "ZIP-SR 4-bit AdamW -- Preconditioner-space stochastic rounding"
      (learnaivisually.com) -- memory paragraph, worked example, ZE-EDEN
      paragraph
"""
from __future__ import annotations

import ctypes
import os
import struct
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "adamw4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_adamw4.so")

BLOCK = 128
MIN_QUANT_NUMEL = 4096
VCODE_ZIPSR = 0
VCODE_ZEEDEN = 1
VCODE_ZI_RTN = 2      # zero-inclusive code, state-space round-to-nearest
VCODE_ZI_SR = 3       # zero-inclusive code, state-space stochastic rounding
VCODE_ZE_FLOOR = 4    # zero-excluded code, no rescale
VCODE_ZIPSR_U32 = 5   # ZIP-SR deciding on the whole 32-bit draw
T_NORM = 1
T_LM_HEAD = 2
T_FP32_STATE = 4
T_BF16_PARAM = 16      # weights stored as bf16 (a library option, not the pages')
STREAM_V = 0
STREAM_M = 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-fopenmp", "-Wall", "-Wextra", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class Scalars(ctypes.Structure):
    _fields_ = [("step_size", ctypes.c_float), ("rs_bc2", ctypes.c_float),
                ("b1", ctypes.c_float), ("omb1", ctypes.c_float),
                ("b2", ctypes.c_float), ("omb2", ctypes.c_float),
                ("eps", ctypes.c_float), ("lr", ctypes.c_float),
                ("t", ctypes.c_int64), ("seed", ctypes.c_uint64),
                ("lm_sr_active", ctypes.c_int)]


_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    S = ctypes.POINTER(Scalars)
    c = ctypes
    L.oracle_philox4x32_10.argtypes = [_u32p, _u32p, _u32p]
    L.oracle_draw_word.restype = c.c_uint32
    L.oracle_draw_word.argtypes = [c.c_uint64, c.c_int64, c.c_uint32, c.c_uint32, c.c_uint64]
    L.oracle_uniform.restype = c.c_float
    L.oracle_uniform.argtypes = [c.c_uint32]
    L.oracle_uniform32.restype = c.c_float
    L.oracle_uniform32.argtypes = [c.c_uint32]
    L.oracle_nf4_levels_f64.argtypes = [_f64p]
    L.oracle_tables.argtypes = [_f32p, _f32p, _f32p, _f32p]
    L.oracle_make_scalars.argtypes = [c.c_float, c.c_float, c.c_float, c.c_float,
                                      c.c_int64, c.c_int64, c.c_uint64, S]
    L.oracle_decay.restype = c.c_float
    L.oracle_decay.argtypes = [c.c_float, c.c_float]
    L.oracle_update_elem.restype = c.c_float
    L.oracle_update_elem.argtypes = [S, c.c_float, c.c_float, c.c_float, c.c_float,
                                     c.POINTER(c.c_float), c.POINTER(c.c_float),
                                     c.POINTER(c.c_float)]
    L.oracle_nf4_rtn.restype = c.c_int
    L.oracle_nf4_rtn.argtypes = [c.c_float]
    L.oracle_nf4_sr.restype = c.c_int
    L.oracle_nf4_sr.argtypes = [c.c_float, c.c_float]
    L.oracle_zipsr_bracket.restype = c.c_int
    L.oracle_zipsr_bracket.argtypes = [c.c_float]
    L.oracle_zi_rtn.restype = c.c_int
    L.oracle_zi_rtn.argtypes = [c.c_float]
    L.oracle_zi_sr.restype = c.c_int
    L.oracle_zi_sr.argtypes = [c.c_float, c.c_float]
    L.oracle_zipsr_decide.restype = c.c_int
    L.oracle_zipsr_decide.argtypes = [c.c_float] * 5
    L.oracle_zipsr_decide_u32.restype = c.c_int
    L.oracle_zipsr_decide_u32.argtypes = [c.c_float] * 4 + [c.c_uint32]
    L.oracle_zeeden_code.restype = c.c_int
    L.oracle_zeeden_code.argtypes = [c.c_float]
    L.oracle_zeeden_factor.restype = c.c_float
    L.oracle_zeeden_factor.argtypes = [_f32p, _f32p]
    L.oracle_block4.argtypes = [S, c.c_float, c.c_int, c.c_int, c.c_uint32, c.c_uint64,
                                c.c_int, _f32p, _u16p, _u8p, _f32p, _u8p, _f32p]
    L.oracle_step_tensor4.argtypes = [S, c.c_float, c.c_int, c.c_int, c.c_uint32,
                                      c.c_int64, _f32p, _u16p, _u8p, _f32p, _u8p,
                                      _f32p, c.c_int]
    L.oracle_step_blocks4.argtypes = [S, c.c_float, c.c_int, c.c_int, c.c_uint32,
                                      c.c_int64, c.c_int64, _i64p, _f32p, _u16p, _u8p,
                                      _f32p, _u8p, _f32p]
    L.oracle_step_fp32.argtypes = [S, c.c_float, c.c_int64, _f32p, _u16p, _f32p, _f32p]
    L.oracle_f32_to_bf16.restype = c.c_uint16
    L.oracle_f32_to_bf16.argtypes = [c.c_float]
    L.oracle_round_bf16.argtypes = [_f32p, _u16p, c.c_int64]
    L.oracle_max_threads.restype = c.c_int
    return L


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def build_variant(source_text: str, out_path: str) -> str:
    """Compiles a modified copy of the oracle source (used by the tests that
    plant mistakes in the oracle to show that the pins catch them)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    cmd = ["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", src, "-o", out_path, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return out_path


class use_library:
    """Context manager: route every oracle call to the library at `path`."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        lib()
        self.saved = _lib
        _lib = _bind(ctypes.CDLL(self.path))
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def source() -> str:
    with open(_SRC) as f:
        return f.read()


# ----------------------------------------------------------------------------
# Thin wrappers over the C stages (used by the pins).
# ----------------------------------------------------------------------------

def philox4x32_10(ctr, key) -> np.ndarray:
    out = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(np.ascontiguousarray(ctr, np.uint32),
                               np.ascontiguousarray(key, np.uint32), out)
    return out


def draw_word(seed: int, t: int, tensor_id: int, stream: int, e: int) -> int:
    return int(lib().oracle_draw_word(seed, t, tensor_id, stream, e))


def uniform(word: int) -> float:
    return float(lib().oracle_uniform(word))


def uniform32(word: int) -> float:
    """The ZIP-SR uniform: the whole word rounded to binary32, times 2^-32."""
    return float(lib().oracle_uniform32(word))


def nf4_levels_f64() -> np.ndarray:
    out = np.zeros(16, np.float64)
    lib().oracle_nf4_levels_f64(out)
    return out


def tables():
    nf4 = np.zeros(16, np.float32)
    mid = np.zeros(15, np.float32)
    vz = np.zeros(16, np.float32)
    vzs = np.zeros(16, np.float32)
    lib().oracle_tables(nf4, mid, vz, vzs)
    return nf4, mid, vz, vzs


def make_scalars(lr, beta1, beta2, eps, t, total_steps=0, seed=0) -> Scalars:
    s = Scalars()
    lib().oracle_make_scalars(lr, beta1, beta2, eps, t, total_steps, seed, ctypes.byref(s))
    return s


def nf4_rtn(x: float) -> int:
    return int(lib().oracle_nf4_rtn(x))


def nf4_sr(x: float, u: float) -> int:
    return int(lib().oracle_nf4_sr(x, u))


def zipsr_bracket(x: float) -> int:
    return int(lib().oracle_zipsr_bracket(x))


def zi_rtn(x: float) -> int:
    return int(lib().oracle_zi_rtn(x))


def zi_sr(x: float, u: float) -> int:
    return int(lib().oracle_zi_sr(x, u))


def zipsr_decide(x: float, dv: float, R: float, eps: float, u: float) -> int:
    return int(lib().oracle_zipsr_decide(x, dv, R, eps, u))


def zipsr_decide_u32(x: float, dv: float, R: float, eps: float, word: int) -> int:
    return int(lib().oracle_zipsr_decide_u32(x, dv, R, eps, word))


def zeeden_code(x: float) -> int:
    return int(lib().oracle_zeeden_code(x))


def zeeden_factor(xx: np.ndarray, xq: np.ndarray) -> float:
    a = np.zeros(BLOCK, np.float32)
    b = np.zeros(BLOCK, np.float32)
    a[: len(xx)] = xx
    b[: len(xq)] = xq
    return float(lib().oracle_zeeden_factor(a, b))


def update_elem(s: Scalars, decay: float, g: float, m0: float, v0: float, w: float):
    wc, m1, v1 = ctypes.c_float(w), ctypes.c_float(), ctypes.c_float()
    den = lib().oracle_update_elem(ctypes.byref(s), decay, g, m0, v0, ctypes.byref(wc),
                                   ctypes.byref(m1), ctypes.byref(v1))
    return float(den), wc.value, m1.value, v1.value


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# ----------------------------------------------------------------------------
# The step over a tensor list, with the C ABI's semantics.
# ----------------------------------------------------------------------------

def is_fp32_state(numel: int, flags: int) -> bool:
    """fp32 state for normalisation layers, forced tensors and tensors under
    4096 elements ("ZIP-SR 4-bit AdamW", memory paragraph; "ZIP-SR / ZE-EDEN:
    4-bit AdamW state quantization", Local reproduction notes)."""
    return numel < MIN_QUANT_NUMEL or bool(flags & (T_NORM | T_FP32_STATE))


def f32_to_bf16(x: float) -> int:
    return int(lib().oracle_f32_to_bf16(x))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """binary32 array -> bf16 bit patterns (nearest, ties to even)."""
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.size, np.uint16)
    lib().oracle_round_bf16(x, out, x.size)
    return out


class TensorState:
    def __init__(self, numel: int, tensor_id: int, flags: int, weight_decay: float):
        self.numel = int(numel)
        self.tensor_id = int(tensor_id)
        self.flags = int(flags)
        self.bf16w = bool(self.flags & T_BF16_PARAM)
        self.weight_decay = float(weight_decay)
        self.fp32 = is_fp32_state(self.numel, self.flags)
        if self.fp32:
            self.m = np.zeros(self.numel, np.float32)
            self.v = np.zeros(self.numel, np.float32)
        else:
            nb = (self.numel + BLOCK - 1) // BLOCK
            self.nb = nb
            self.mcodes = np.zeros(nb * 64, np.uint8)
            self.vcodes = np.zeros(nb * 64, np.uint8)
            self.mscale = np.zeros(nb, np.float32)
            self.vscale = np.zeros(nb, np.float32)

    def state_bytes(self) -> int:
        return 8 * self.numel if self.fp32 else 136 * self.nb


class OracleAdamW4:
    """The whole step over a tensor list: params are fp32 numpy arrays
    (updated in place), grads are uint16 arrays of bf16 bit patterns."""

    def __init__(self, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, vcode=VCODE_ZIPSR, seed=0,
                 total_steps=0, tensors=(), nthreads=1):
        self.lr = np.float32(lr)
        self.beta1 = np.float32(beta1)
        self.beta2 = np.float32(beta2)
        self.eps = np.float32(eps)
        self.vcode = int(vcode)
        self.seed = int(seed)
        self.total_steps = int(total_steps)
        self.nthreads = int(nthreads)
        ids = [int(t["tensor_id"]) for t in tensors]
        if len(set(ids)) != len(ids):
            raise ValueError("tensor ids must be unique")
        self.tensors = [TensorState(t["numel"], t["tensor_id"], t.get("flags", 0),
                                    t.get("weight_decay", 0.0)) for t in tensors]
        self.t = 0

    def state_bytes(self) -> int:
        return sum(ts.state_bytes() for ts in self.tensors)

    def scalars(self, lr) -> Scalars:
        return make_scalars(np.float32(lr), self.beta1, self.beta2, self.eps, self.t,
                            self.total_steps, self.seed)

    def m_sr(self, ts: TensorState, s: Scalars) -> int:
        return int(bool(ts.flags & T_LM_HEAD) and s.lm_sr_active)

    def step(self, params, grads, lr=None, only=None, advance=True):
        """One step over every tensor, or over the tensors listed in `only`
        (then params/grads hold just those, in that order).  With
        advance=False the step counter is not incremented first.  The params
        of a T_BF16_PARAM tensor are uint16 arrays of bf16 bit patterns: read
        exactly, stepped in binary32, stored rounded to the nearest bf16."""
        L = lib()
        if advance:
            self.t += 1
        s = self.scalars(self.lr if lr is None else lr)
        idx = range(len(self.tensors)) if only is None else list(only)
        for i, w_in, g in zip(idx, params, grads):
            ts = self.tensors[i]
            if ts.bf16w:
                assert w_in.dtype == np.uint16
                w = (w_in.astype(np.uint32) << 16).view(np.float32)
            else:
                w = w_in
            assert w.dtype == np.float32 and g.dtype == np.uint16 and w.size == ts.numel
            if ts.fp32:
                L.oracle_step_fp32(ctypes.byref(s), ts.weight_decay, ts.numel, w, g, ts.m, ts.v)
            else:
                L.oracle_step_tensor4(ctypes.byref(s), ts.weight_decay, self.vcode,
                                      self.m_sr(ts, s), ts.tensor_id, ts.numel, w, g,
                                      ts.mcodes, ts.mscale, ts.vcodes, ts.vscale, self.nthreads)
            if ts.bf16w:
                w_in[:] = round_bf16(w)

    def step_blocks(self, index: int, blocks, w_sel, g_sel, mc_sel, ms_sel, vc_sel, vs_sel,
                    lr=None, advance=True):
        """Steps selected blocks of tensor `index` only (arrays hold just those
        blocks, 128 slots each).  Blocks are independent, so this equals the
        full step restricted to them."""
        L = lib()
        if advance:
            self.t += 1
        s = self.scalars(self.lr if lr is None else lr)
        ts = self.tensors[index]
        assert not ts.bf16w, "step_blocks takes fp32 weights"
        blocks = np.ascontiguousarray(blocks, np.int64)
        L.oracle_step_blocks4(ctypes.byref(s), ts.weight_decay, self.vcode, self.m_sr(ts, s),
                              ts.tensor_id, ts.numel, len(blocks), blocks, w_sel, g_sel, mc_sel,
                              ms_sel, vc_sel, vs_sel)

    # -- checkpoint blob (layout documented with the C ABI) --------------------
    def export_state(self) -> bytes:
        parts = []
        for ts in self.tensors:
            if ts.fp32:
                parts.append(struct.pack("<IIq", ts.tensor_id, 1, ts.numel))
                parts += [ts.m.tobytes(), ts.v.tobytes()]
            else:
                parts.append(struct.pack("<IIq", ts.tensor_id, 0, ts.numel))
                parts += [ts.mcodes.tobytes(), ts.vcodes.tobytes(), ts.mscale.tobytes(),
                          ts.vscale.tobytes()]
        payload = b"".join(parts)
        head = b"ADAMW4S1" + struct.pack("<IIqQQ", len(self.tensors), self.vcode, self.t,
                                         self.seed, len(payload))
        return head + payload

    def import_state(self, blob: bytes):
        if blob[:8] != b"ADAMW4S1":
            raise ValueError("bad magic")
        n, vcode, t, seed, plen = struct.unpack_from("<IIqQQ", blob, 8)
        if n != len(self.tensors) or vcode != self.vcode or seed != self.seed:
            raise ValueError("blob does not match this optimizer")
        if len(blob) != 40 + plen:
            raise ValueError("bad length")
        off = 40
        for ts in self.tensors:
            tid, kind, numel = struct.unpack_from("<IIq", blob, off)
            off += 16
            if tid != ts.tensor_id or kind != int(ts.fp32) or numel != ts.numel:
                raise ValueError("tensor mismatch")

            def take(count, dtype):
                nonlocal off
                nbytes = count * np.dtype(dtype).itemsize
                a = np.frombuffer(blob, dtype, count, off).copy()
                off += nbytes
                return a
            if ts.fp32:
                ts.m = take(ts.numel, np.float32)
                ts.v = take(ts.numel, np.float32)
            else:
                ts.mcodes = take(ts.nb * 64, np.uint8)
                ts.vcodes = take(ts.nb * 64, np.uint8)
                ts.mscale = take(ts.nb, np.float32)
                ts.vscale = take(ts.nb, np.float32)
        self.t = t
