"""The C ABI library: builds, loads, exports every declared entry point, and
rejects bad input on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

import bit_quantized_optimizer_b200 as B
from bit_quantized_optimizer_b200 import build as B_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B_build.build()
    return B.lib()


def declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(adamw4_[a-z_0-9]+)\s*\(", txt))
    return sorted(names)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "adamw4_create" in names and "adamw4_step" in names and "adamw4_destroy" in names
    for n in names:
        assert hasattr(L, n), n


def _cfg(**kw):
    c = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, vcode=0, seed=0, total_steps=0)
    c.update(kw)
    return B.adamw4_config(c["lr"], c["beta1"], c["beta2"], c["eps"], c["vcode"], c["seed"],
                           c["total_steps"])


def _create(cfg, ts):
    arr = (B.adamw4_tensor * max(len(ts), 1))(*ts)
    h = ctypes.c_void_p()
    rc = B.lib().adamw4_create(ctypes.byref(cfg), arr, len(ts), 0, ctypes.byref(h))
    return rc, h


P0 = 0x7F0000000000   # fake, aligned device addresses: validation never dereferences them


@pytest.mark.parametrize("kw,code", [(dict(beta1=1.0), -1), (dict(beta2=-0.1), -1),
                                     (dict(eps=0.0), -1), (dict(vcode=6), -1), (dict(vcode=-1), -1),
                                     (dict(total_steps=-1), -1), (dict(lr=float("nan")), -1)])
def test_bad_config(L, kw, code):
    rc, _ = _create(_cfg(**kw), [B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 0, 0.0)])
    assert rc == code
    assert B.adamw4_last_error()


@pytest.mark.parametrize("t,code,msg", [
    (B.adamw4_tensor(0, P0, 4096, 0, 0, 0.0), -1, "NULL"),
    (B.adamw4_tensor(P0, 0, 4096, 0, 0, 0.0), -1, "NULL"),
    (B.adamw4_tensor(P0 + 4, P0 + (1 << 30), 4096, 0, 0, 0.0), -2, "aligned"),
    (B.adamw4_tensor(P0, P0 + (1 << 30) + 8, 4096, 0, 0, 0.0), -2, "aligned"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 0, 0, 0, 0.0), -1, "numel"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), -5, 0, 0, 0.0), -1, "numel"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 0, float("inf")), -1, "weight_decay"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 32, 0.0), -1, "unknown flag"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 1 << 16, 0.0), -1, "unknown flag"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 8 | 1, 0.0), -1, "QUANT_STATE"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 8 | 4, 0.0), -1, "QUANT_STATE"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 0, 0.0, 64), -1, "elem_offset"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 0, 0.0, -128), -1, "elem_offset"),
    (B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 0, 0.0, 1 << 39), -1, "elem_offset"),
])
def test_bad_tensor(L, t, code, msg):
    rc, _ = _create(_cfg(), [t])
    assert rc == code
    assert msg in B.adamw4_last_error()


def test_duplicate_ids_and_overlaps(L):
    a = B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 7, 0, 0.0)
    b = B.adamw4_tensor(P0 + (1 << 20), P0 + (1 << 31), 4096, 7, 0, 0.0)
    rc, _ = _create(_cfg(), [a, b])
    assert rc == -1 and "duplicate" in B.adamw4_last_error()
    # param of b inside param of a
    b = B.adamw4_tensor(P0 + 1024, P0 + (1 << 31), 4096, 8, 0, 0.0)
    rc, _ = _create(_cfg(), [a, b])
    assert rc == -1 and "overlaps" in B.adamw4_last_error()
    # grad of b inside param of a
    b = B.adamw4_tensor(P0 + (1 << 20), P0 + 4096, 4096, 8, 0, 0.0)
    rc, _ = _create(_cfg(), [a, b])
    assert rc == -1 and "overlaps" in B.adamw4_last_error()
    # grads may alias each other (read only)
    b = B.adamw4_tensor(P0 + (1 << 20), P0 + (1 << 30), 4096, 8, 0, 0.0)
    os.environ["ADAMW4_FAIL_ALLOC"] = "1"
    try:
        rc, _ = _create(_cfg(), [a, b])
    finally:
        del os.environ["ADAMW4_FAIL_ALLOC"]
    assert rc == -3 and "injected" in B.adamw4_last_error()


def test_unknown_handles_are_rejected(L):
    bogus = ctypes.c_void_p(0x1234)
    assert L.adamw4_step(bogus, 1e-3, None) == -1
    assert L.adamw4_destroy(bogus) == -1
    assert L.adamw4_destroy(None) == -1
    assert L.adamw4_state_bytes(bogus) == -1
    t = ctypes.c_int64()
    assert L.adamw4_get_step(bogus, ctypes.byref(t)) == -1
    assert L.adamw4_set_step(bogus, 3) == -1
    assert L.adamw4_state_import(bogus, b"x", 1) == -1


def test_null_out_pointer(L):
    cfg = _cfg()
    arr = (B.adamw4_tensor * 1)(B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 0, 0, 0.0))
    assert L.adamw4_create(ctypes.byref(cfg), arr, 1, 0, None) == -1


def test_piece_descriptors_pass_validation(L):
    """A block-aligned piece (elem_offset a multiple of 128, below 2^39) with
    QUANT_STATE gets past validation: the fake addresses then stop it at the
    injected allocation failure, before any device work."""
    t = B.adamw4_tensor(P0, P0 + (1 << 30), 256, 0, 8 | 2, 0.0, (1 << 39) - 128)
    os.environ["ADAMW4_FAIL_ALLOC"] = "1"
    try:
        rc, _ = _create(_cfg(), [t])
    finally:
        del os.environ["ADAMW4_FAIL_ALLOC"]
    assert rc == -3 and "injected" in B.adamw4_last_error()


def test_descriptor_layout_matches_the_header():
    assert ctypes.sizeof(B.adamw4_tensor) == 48
    assert B.adamw4_tensor.elem_offset.offset == 40


def test_bf16_params_span_two_bytes_per_weight(L):
    """A bf16 weight tensor of 4096 values ends 8 KB after its start; the same
    tensor with fp32 weights would overlap a param placed there."""
    b = B.adamw4_tensor(P0 + 8192, P0 + (1 << 31), 4096, 2, 16, 0.0)
    a32 = B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 1, 0, 0.0)
    rc, _ = _create(_cfg(), [a32, b])
    assert rc == -1 and "overlaps" in B.adamw4_last_error()
    a16 = B.adamw4_tensor(P0, P0 + (1 << 30), 4096, 1, 16, 0.0)
    os.environ["ADAMW4_FAIL_ALLOC"] = "1"
    try:
        rc, _ = _create(_cfg(), [a16, b])
    finally:
        del os.environ["ADAMW4_FAIL_ALLOC"]
    assert rc == -3 and "injected" in B.adamw4_last_error()


def _header_enums():
    txt = open(os.path.join(ROOT, "include", "adamw4.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    vals = {}
    for name, val in re.findall(r"\b(ADAMW4_[A-Z0-9_]+)\s*=\s*(-?[0-9]+)u?\b", txt):
        vals[name] = int(val)
    for name, val in re.findall(r"#define\s+(ADAMW4_[A-Z0-9_]+)\s+([0-9]+)", txt):
        vals[name] = int(val)
    return vals


def test_binding_constants_match_the_header():
    """Every status code, v code, flag and size the header defines has the same
    value in the Python binding, and every status code has a name there."""
    vals = _header_enums()
    assert len(vals) >= 20
    for name, v in vals.items():
        if hasattr(B, name):
            assert getattr(B, name) == v, name
    for name in ("ADAMW4_V_ZIPSR", "ADAMW4_V_ZEEDEN", "ADAMW4_V_ZI_RTN", "ADAMW4_V_ZI_SR",
                 "ADAMW4_V_ZE_FLOOR", "ADAMW4_V_ZIPSR_U32", "ADAMW4_T_NORM", "ADAMW4_T_LM_HEAD",
                 "ADAMW4_T_FP32_STATE", "ADAMW4_T_QUANT_STATE", "ADAMW4_T_BF16_PARAM",
                 "ADAMW4_NOALLOC_MAX_TENSORS", "ADAMW4_ETIMEOUT", "ADAMW4_ECHECK",
                 "ADAMW4_ENONFINITE", "ADAMW4_ERANGE"):
        assert name in vals and getattr(B, name) == vals[name], name
    codes = {v for n, v in vals.items() if n in (
        "ADAMW4_OK", "ADAMW4_EINVAL", "ADAMW4_EALIGN", "ADAMW4_ENOMEM", "ADAMW4_ECUDA",
        "ADAMW4_ESTATE", "ADAMW4_ENONFINITE", "ADAMW4_ERANGE", "ADAMW4_ETIMEOUT",
        "ADAMW4_ECHECK")}
    assert codes == set(B.STATUS)
    assert B.MIN_QUANT_NUMEL == vals["ADAMW4_MIN_QUANT_NUMEL"] and B.BLOCK == vals["ADAMW4_BLOCK"]


def _noalloc(L, ts, sb, n=None):
    arr = (B.adamw4_tensor * max(len(ts), 1))(*ts)
    return L.adamw4_step_noalloc(ctypes.byref(_cfg()), arr, len(ts) if n is None else n,
                                 ctypes.byref(sb), 1, ctypes.c_float(1e-3), 0, None)




def _no_gpu():
    """These checks hand the library fake device addresses: on a machine with
    a GPU a descriptor list that passed validation would be launched on
    them, so they run only where no GPU is visible."""
    try:
        import torch
        return not torch.cuda.is_available()
    except Exception:
        return True


@pytest.mark.skipif(not _no_gpu(), reason="host-validation check with fake device addresses")
def test_noalloc_rejects_missing_state_buffers(L):
    """The allocation-free step refuses, on the host and before any CUDA call,
    a NULL state buffer that its tensor list needs: the codes and scales for a
    4-bit tensor, the fp32 moments for an fp32-state tensor."""
    q = B.adamw4_tensor(P0, P0 + (1 << 20), 8192, 1, 0, 0.0)          # 4-bit state
    f = B.adamw4_tensor(P0 + (2 << 20), P0 + (3 << 20), 1000, 2, 0, 0.0)   # fp32 state
    S = P0 + (8 << 20)
    full = [S, S + 4096, S + 8192, S + 12288, S + 16384, S + 20480]
    for missing in range(4):                       # any of the four 4-bit buffers
        bufs = list(full)
        bufs[missing] = 0
        assert _noalloc(L, [q], B.adamw4_state_buffers(*bufs)) == -1
    for missing in (4, 5):                         # either fp32 moment buffer
        bufs = list(full)
        bufs[missing] = 0
        assert _noalloc(L, [f], B.adamw4_state_buffers(*bufs)) == -1
    # the buffers a list does not use may be NULL: validation passes, and the
    # call then fails only on the missing GPU (a CUDA error, not EINVAL)
    assert _noalloc(L, [q], B.adamw4_state_buffers(S, S + 4096, S + 8192, S + 12288, 0, 0)) == -4
    assert _noalloc(L, [f], B.adamw4_state_buffers(0, 0, 0, 0, S + 16384, S + 20480)) == -4


def test_tensor_state_kind_follows_the_documented_rule(L):
    """adamw4_tensor_state_kind (which the binding's is_fp32_state asks) gives
    the classification the header documents: fp32 for NORM / FP32_STATE, 4-bit
    for QUANT_STATE, else fp32 below 4096 elements; invalid descriptors are
    refused."""
    N, F, Q, H = (B.ADAMW4_T_NORM, B.ADAMW4_T_FP32_STATE, B.ADAMW4_T_QUANT_STATE,
                  B.ADAMW4_T_LM_HEAD)
    cases = [(1, 0, 1), (100, 0, 1), (4095, 0, 1), (4096, 0, 0), (8192, 0, 0), (8192, N, 1),
             (8192, F, 1), (100, Q, 0), (4095, Q, 0), (4096, H, 0), (4000, H, 1),
             (1 << 33, 0, 0), (1 << 33, N, 1), (4096, B.ADAMW4_T_BF16_PARAM, 0)]
    for numel, flags, want in cases:
        assert B.adamw4_tensor_state_kind(numel, flags) == want, (numel, flags)
        assert B.is_fp32_state(numel, flags) == bool(want)
    for numel, flags, off in [(0, 0, 0), (-5, 0, 0), (4096, 1 << 9, 0), (4096, Q | N, 0),
                              (4096, 0, 100), (4096, 0, 1 << 39)]:
        with pytest.raises(B.AdamW4Error):
            B.adamw4_tensor_state_kind(numel, flags, off)
