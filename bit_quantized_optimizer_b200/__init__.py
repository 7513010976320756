"""Python binding of the fused 4-bit AdamW step (ZIP-SR / ZE-EDEN) for B200.

Argument marshalling only: every step of the method runs in the CUDA kernels
of ``libadamw4.so`` (built in-tree by ``build.py``).  There is no fallback: if
the library is missing or cannot load, importing the functions raises.

The functions carry the C ABI's names (``include/adamw4.h``); ``AdamW4``
wraps them for torch tensors (fp32 params, bf16 grads on one CUDA device).
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["ADAMW4_V_ZIPSR", "ADAMW4_V_ZEEDEN", "ADAMW4_V_ZI_RTN", "ADAMW4_V_ZI_SR",
           "ADAMW4_V_ZE_FLOOR", "ADAMW4_V_ZIPSR_U32", "ADAMW4_T_NORM", "ADAMW4_T_LM_HEAD",
           "ADAMW4_T_FP32_STATE", "ADAMW4_T_QUANT_STATE", "ADAMW4_T_BF16_PARAM", "AdamW4Error", "adamw4_tensor", "adamw4_config", "lib",
           "adamw4_create", "adamw4_step", "adamw4_step_host", "adamw4_destroy",
           "adamw4_get_step", "adamw4_set_step", "adamw4_state_bytes", "adamw4_state_export",
           "adamw4_state_import", "adamw4_launch_info", "adamw4_last_error", "adamw4_sync",
           "adamw4_inject_fault", "ADAMW4_ETIMEOUT", "ADAMW4_FAULT_STALL_PIPELINE", "AdamW4",
           "adamw4_state_buffers", "adamw4_step_noalloc", "adamw4_noalloc_sync",
           "ADAMW4_NOALLOC_MAX_TENSORS", "ADAMW4_ENONFINITE", "ADAMW4_ERANGE", "ADAMW4_ECHECK",
           "is_fp32_state", "adamw4_tensor_state_kind", "LIB_PATH"]

# ADAMW4_LIBRARY selects another build of the same library (the checked one)
LIB_PATH = os.environ.get("ADAMW4_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libadamw4.so")

ADAMW4_OK = 0
ADAMW4_V_ZIPSR = 0
ADAMW4_V_ZEEDEN = 1
ADAMW4_V_ZI_RTN = 2      # zero-inclusive code, state-space nearest
ADAMW4_V_ZI_SR = 3       # zero-inclusive code, state-space stochastic rounding
ADAMW4_V_ZE_FLOOR = 4    # zero-excluded code, nearest, no rescale
ADAMW4_V_ZIPSR_U32 = 5   # ZIP-SR deciding on the whole 32-bit draw
ADAMW4_T_NORM = 1
ADAMW4_T_LM_HEAD = 2
ADAMW4_T_FP32_STATE = 4
ADAMW4_T_QUANT_STATE = 8   # 4-bit state below 4096 elements (a piece of a larger tensor)
ADAMW4_T_BF16_PARAM = 16   # bf16 weights (rounded to nearest even after each update)
MIN_QUANT_NUMEL = 4096
BLOCK = 128

ADAMW4_ENONFINITE = -6
ADAMW4_ETIMEOUT = -7
ADAMW4_ECHECK = -8
ADAMW4_ERANGE = -9
ADAMW4_NOALLOC_MAX_TENSORS = 1024
ADAMW4_FAULT_STALL_PIPELINE = 1

STATUS = {0: "ADAMW4_OK", -1: "ADAMW4_EINVAL", -2: "ADAMW4_EALIGN", -3: "ADAMW4_ENOMEM",
          -4: "ADAMW4_ECUDA", -5: "ADAMW4_ESTATE", -6: "ADAMW4_ENONFINITE",
          -7: "ADAMW4_ETIMEOUT", -8: "ADAMW4_ECHECK", -9: "ADAMW4_ERANGE"}


class AdamW4Error(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class adamw4_tensor(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad_bf16", ctypes.c_void_p),
                ("numel", ctypes.c_int64), ("tensor_id", ctypes.c_uint32),
                ("flags", ctypes.c_uint32), ("weight_decay", ctypes.c_float),
                ("elem_offset", ctypes.c_int64)]


class adamw4_state_buffers(ctypes.Structure):
    """Caller-owned device buffers of the packed state (allocation-free step)."""
    _fields_ = [("mcodes", ctypes.c_void_p), ("vcodes", ctypes.c_void_p),
                ("mscale", ctypes.c_void_p), ("vscale", ctypes.c_void_p),
                ("m32", ctypes.c_void_p), ("v32", ctypes.c_void_p)]


class adamw4_config(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("vcode", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("total_steps", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libadamw4.so; raises if it is absent (build it with build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run bit_quantized_optimizer_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        c = ctypes
        H = c.c_void_p
        L.adamw4_create.argtypes = [c.POINTER(adamw4_config), c.POINTER(adamw4_tensor), c.c_int,
                                    c.c_int, c.POINTER(H)]
        L.adamw4_step.argtypes = [H, c.c_float, c.c_void_p]
        L.adamw4_step_host.argtypes = [H, c.c_float, c.POINTER(c.c_void_p),
                                       c.POINTER(c.c_void_p), c.c_void_p]
        L.adamw4_destroy.argtypes = [H]
        L.adamw4_get_step.argtypes = [H, c.POINTER(c.c_int64)]
        L.adamw4_set_step.argtypes = [H, c.c_int64]
        L.adamw4_state_bytes.argtypes = [H]
        L.adamw4_state_bytes.restype = c.c_int64
        L.adamw4_state_export.argtypes = [H, c.c_void_p, c.c_int64, c.POINTER(c.c_int64)]
        L.adamw4_state_import.argtypes = [H, c.c_void_p, c.c_int64]
        L.adamw4_launch_info.argtypes = [H, c.POINTER(c.c_int), c.POINTER(c.c_int),
                                         c.POINTER(c.c_int64)]
        L.adamw4_sync.argtypes = [H, c.c_void_p]
        L.adamw4_inject_fault.argtypes = [H, c.c_int]
        L.adamw4_step_noalloc.argtypes = [c.POINTER(adamw4_config), c.POINTER(adamw4_tensor),
                                          c.c_int, c.POINTER(adamw4_state_buffers), c.c_int64,
                                          c.c_float, c.c_int, c.c_void_p]
        L.adamw4_noalloc_sync.argtypes = [c.c_int, c.c_void_p]
        L.adamw4_tensor_state_kind.argtypes = [c.POINTER(adamw4_tensor)]
        L.adamw4_tensor_state_kind.restype = c.c_int
        L.adamw4_last_error.argtypes = [H]
        L.adamw4_last_error.restype = c.c_char_p
        for f in ("adamw4_create", "adamw4_step", "adamw4_step_host", "adamw4_destroy",
                  "adamw4_get_step", "adamw4_set_step", "adamw4_state_export",
                  "adamw4_state_import", "adamw4_launch_info", "adamw4_sync",
                  "adamw4_inject_fault", "adamw4_step_noalloc", "adamw4_noalloc_sync"):
            getattr(L, f).restype = c.c_int
        _lib = L
    return _lib


def adamw4_last_error(h=None) -> str:
    return lib().adamw4_last_error(h).decode()


def _check(rc, h=None):
    if rc != ADAMW4_OK:
        raise AdamW4Error(rc, adamw4_last_error(h))


def adamw4_create(cfg: adamw4_config, tensors, device: int = 0):
    arr = (adamw4_tensor * max(len(tensors), 1))(*tensors)
    h = ctypes.c_void_p()
    _check(lib().adamw4_create(ctypes.byref(cfg), arr, len(tensors), device, ctypes.byref(h)))
    return h


def adamw4_step(h, lr: float, stream=None):
    _check(lib().adamw4_step(h, lr, stream), h)


def adamw4_step_host(h, lr: float, grads_host, params_host, stream=None):
    """grads_host / params_host: sequences of host addresses (or None)."""
    g = (ctypes.c_void_p * len(grads_host))(*grads_host) if grads_host is not None else None
    p = (ctypes.c_void_p * len(params_host))(*params_host) if params_host is not None else None
    _check(lib().adamw4_step_host(h, lr, g, p, stream), h)


def adamw4_destroy(h):
    _check(lib().adamw4_destroy(h))


def adamw4_get_step(h) -> int:
    t = ctypes.c_int64()
    _check(lib().adamw4_get_step(h, ctypes.byref(t)), h)
    return t.value


def adamw4_set_step(h, t: int):
    _check(lib().adamw4_set_step(h, t), h)


def adamw4_state_bytes(h) -> int:
    b = lib().adamw4_state_bytes(h)
    if b < 0:
        raise AdamW4Error(-1, "unknown handle")
    return b


def adamw4_state_export(h) -> bytes:
    used = ctypes.c_int64()
    _check(lib().adamw4_state_export(h, None, 0, ctypes.byref(used)), h)
    buf = ctypes.create_string_buffer(used.value)
    _check(lib().adamw4_state_export(h, buf, used.value, ctypes.byref(used)), h)
    return buf.raw


def adamw4_state_import(h, blob: bytes):
    _check(lib().adamw4_state_import(h, blob, len(blob)), h)


def adamw4_sync(h, stream=None):
    _check(lib().adamw4_sync(h, stream), h)


def adamw4_inject_fault(h, fault: int):
    """Arms a test fault for the next step of handle h (h None: for the next
    adamw4_step_noalloc call)."""
    _check(lib().adamw4_inject_fault(h, fault), h)


def adamw4_step_noalloc(cfg: adamw4_config, tensors, state: adamw4_state_buffers, t: int,
                        lr: float, device: int = 0, stream=None):
    """The allocation-free step (see include/adamw4.h): no handle, caller-owned
    state buffers, step number t.  Raises AdamW4Error with the status code."""
    arr = (adamw4_tensor * max(len(tensors), 1))(*tensors)
    rc = lib().adamw4_step_noalloc(ctypes.byref(cfg), arr, len(tensors), ctypes.byref(state), t,
                                   lr, device, stream)
    if rc != ADAMW4_OK:
        raise AdamW4Error(rc, "adamw4_step_noalloc failed")


def adamw4_noalloc_sync(device: int = 0, stream=None):
    """Waits for the stream and reads and clears the allocation-free step's
    status word on the device; raises AdamW4Error(ADAMW4_ETIMEOUT /
    ADAMW4_ENONFINITE) when a call reported a failure."""
    rc = lib().adamw4_noalloc_sync(device, stream)
    if rc != ADAMW4_OK:
        raise AdamW4Error(rc, "adamw4_noalloc_sync: status word set")


def adamw4_launch_info(h):
    g, b, u = ctypes.c_int(), ctypes.c_int(), ctypes.c_int64()
    _check(lib().adamw4_launch_info(h, ctypes.byref(g), ctypes.byref(b), ctypes.byref(u)), h)
    return g.value, b.value, u.value


def adamw4_tensor_state_kind(numel: int, flags: int, elem_offset: int = 0) -> int:
    """The library's state class of a descriptor: 1 fp32 state, 0 4-bit."""
    t = adamw4_tensor(1, 1, numel, 0, flags, 0.0, elem_offset)
    k = lib().adamw4_tensor_state_kind(ctypes.byref(t))
    if k < 0:
        raise AdamW4Error(k, "invalid descriptor (numel, flags or elem_offset)")
    return k


def is_fp32_state(numel: int, flags: int) -> bool:
    """Whether the library keeps fp32 state for such a tensor (asked of the
    library: fp32 for NORM / FP32_STATE tensors, and below 4096 elements
    unless flagged QUANT_STATE)."""
    return adamw4_tensor_state_kind(numel, flags) == 1


class AdamW4:
    """Optimizer over torch tensors: fp32 (or bf16) params and bf16 grads
    (contiguous, 16-byte aligned, on one CUDA device).  ``specs`` is a list of
    dicts with tensor_id, flags, weight_decay and (for a piece of a larger
    tensor) elem_offset, parallel to ``params``.  A bf16 param sets
    ADAMW4_T_BF16_PARAM for its tensor."""

    def __init__(self, params, grads, specs, lr=1e-3, betas=(0.9, 0.999), eps=1e-8,
                 vcode=ADAMW4_V_ZIPSR, seed=0, total_steps=0):
        import torch
        self.params, self.grads = list(params), list(grads)
        dev = self.params[0].device.index if self.params else 0
        ts = []
        for p, g, s in zip(self.params, self.grads, specs):
            if p.dtype not in (torch.float32, torch.bfloat16) or g.dtype != torch.bfloat16:
                raise TypeError("params must be float32 or bfloat16 and grads bfloat16")
            if not (p.is_contiguous() and g.is_contiguous()) or p.numel() != g.numel():
                raise ValueError("params and grads must be contiguous and of equal size")
            flags = int(s.get("flags", 0)) & ~ADAMW4_T_BF16_PARAM
            if p.dtype == torch.bfloat16:
                flags |= ADAMW4_T_BF16_PARAM
            ts.append(adamw4_tensor(p.data_ptr(), g.data_ptr(), p.numel(), s["tensor_id"],
                                    flags, s.get("weight_decay", 0.0), s.get("elem_offset", 0)))
        self.cfg = adamw4_config(lr, betas[0], betas[1], eps, vcode, seed, total_steps)
        self.lr = lr
        self.handle = adamw4_create(self.cfg, ts, dev)

    def step(self, lr=None, stream=None):
        import torch
        s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        adamw4_step(self.handle, self.lr if lr is None else lr, s)

    @property
    def t(self) -> int:
        return adamw4_get_step(self.handle)

    @t.setter
    def t(self, value: int):
        adamw4_set_step(self.handle, value)

    def state_bytes(self) -> int:
        return adamw4_state_bytes(self.handle)

    def sync(self, stream=None):
        """Waits for the stream; raises AdamW4Error(ADAMW4_ETIMEOUT) if a step
        kernel on it stopped on a pipeline wait, AdamW4Error(ADAMW4_ENONFINITE)
        if a step produced a non-finite weight."""
        import torch
        s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        adamw4_sync(self.handle, s)

    def state_dict_blob(self) -> bytes:
        return adamw4_state_export(self.handle)

    def load_state_blob(self, blob: bytes):
        adamw4_state_import(self.handle, blob)

    def close(self):
        if self.handle is not None:
            adamw4_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
