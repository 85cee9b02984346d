"""The C ABI without a GPU: the library loads, exports exactly what
include/la.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from linear_attention_11_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "la.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(la_[a-z0-9_]+)\s*\(", src))


def test_header_declares_binding_names():
    assert _declared() == set(api.EXPORTS)


def test_library_exports_every_declared_symbol(lib_path):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.split()[-1].startswith("la_")}
    assert exported == _declared()
    lib = ctypes.CDLL(lib_path)
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings_and_version(la):
    assert la.la_status_string(0) == "LA_OK"
    assert la.la_status_string(4) == "LA_ERR_TIMEOUT"
    assert la.la_status_string(99) == "LA_ERR_UNKNOWN"
    assert la.api.load_library().la_version() == 1


# Argument checks that return before any CUDA call (no device needed).
def _raw(la):
    return la.api.load_library()


def test_forward_rejects_null_pointers(la):
    lib = _raw(la)
    assert lib.la_forward(None, None, None, None, 1, 1, 1, 16, 128, 64, None) == 1
    assert lib.la_forward_ws(None, None, None, None, None, 1, 1, 1, 16, 128, 64, None, 0, None) == 1


def test_decode_rejects_bad_shapes(la):
    lib = _raw(la)
    p = ctypes.c_void_p(256)
    assert lib.la_decode_step(p, p, p, p, p, 1, 3, 2, 128, None) == 1   # Hq % Hkv
    assert lib.la_decode_step(p, p, p, p, p, 0, 2, 2, 128, None) == 1   # B <= 0
    assert lib.la_decode_step(p, p, p, p, p, 1, 2, 2, 96, None) == 2    # d unsupported
    assert lib.la_decode_step(p, p, p, p, p, 1, 66, 1, 128, None) == 2  # group too large
    q = ctypes.c_void_p(256 + 4)                                          # misaligned
    assert lib.la_decode_step(p, q, p, p, p, 1, 2, 2, 128, None) == 1


def test_f32_rejects_bad_shapes(la):
    lib = _raw(la)
    p = ctypes.c_void_p(4096)
    assert lib.la_forward_f32(p, p, p, p, None, 1, 2, 2, 16, 96, 64, None) == 2   # d
    assert lib.la_forward_f32(p, p, p, p, None, 1, 2, 2, 16, 64, 32, None) == 2   # chunk
    assert lib.la_forward_f32(p, p, p, p, None, 1, 2, 2, 0, 64, 64, None) == 1    # N
    assert lib.la_forward_f32(p, p, p, p, None, 1, 3, 2, 16, 64, 64, None) == 1   # Hq % Hkv


def test_selftest_and_status_reject_bad_arguments(la):
    lib = _raw(la)
    assert lib.la_selftest_wait(0, None) == 1
    assert lib.la_device_status(None, 0) == 1


def test_backward_rejects_null_and_misaligned_pointers(la):
    lib = _raw(la)
    p, m = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 8)
    shape = (1, 2, 2, 16, 128, 64, None)
    assert lib.la_backward(None, p, p, p, None, None, p, p, p, None, *shape) == 1  # q
    assert lib.la_backward(p, p, p, None, None, None, p, p, p, None, *shape) == 1  # dO
    assert lib.la_backward(p, p, p, p, None, None, p, p, None, None, *shape) == 1  # dv
    assert lib.la_backward(p, p, p, m, None, None, p, p, p, None, *shape) == 1     # dO misaligned
    assert lib.la_backward(p, p, p, p, None, m, p, p, p, None, *shape) == 1        # dSf misaligned
    assert lib.la_backward(p, p, p, p, None, None, p, p, p, m, *shape) == 1        # dS0 misaligned


def test_state_prefix_rejects_bad_arguments(la):
    lib = _raw(la)
    per = 1 * 2 * 128 * 128 * 4                  # bytes of one segment's states
    states, S = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 3 * per)
    assert lib.la_state_prefix(states, None, S, 3, 3, 1, 2, 128, None) == 1   # seg >= nseg
    assert lib.la_state_prefix(states, None, S, 3, -1, 1, 2, 128, None) == 1  # seg < 0
    assert lib.la_state_prefix(states, None, S, 0, 0, 1, 2, 128, None) == 1   # nseg < 1
    assert lib.la_state_prefix(None, None, S, 3, 1, 1, 2, 128, None) == 1    # states null
    inside = ctypes.c_void_p((1 << 20) + per)                                  # S within states
    assert lib.la_state_prefix(states, None, inside, 3, 1, 1, 2, 128, None) == 1
    odd = ctypes.c_void_p((1 << 20) + 3 * per + 4)                             # misaligned S
    assert lib.la_state_prefix(states, None, odd, 3, 1, 1, 2, 128, None) == 1
