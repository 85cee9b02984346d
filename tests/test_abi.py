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
