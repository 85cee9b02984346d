"""fp64 CPU oracle for causal Lightning Attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it and
shares no code with it; the only code both sides use is the seeded input
generator in ``linear_attention_11_b200.synth``, which holds none of the
method's arithmetic.

The arithmetic lives in ``la_oracle.c`` (plain C, fp64, every function citing
the passage it follows).  This module compiles it with gcc on first use and
marshals numpy / torch-CPU arrays into it.

Functions
---------
quadratic(q, k, v)        masked form, all rows:  O[t] = sum_{s<=t} (q_t.k_s) v_s
rows(q, k, v, rows)       the same sum at selected (b, h, t) rows only
recurrent(q, k, v, S0)    token recurrence S += k^T v; o = q S; returns (O, S)
state(k, v)               S = K^T V (scalar loops)
state_gemm(k, v)          S = K^T V (one fp64 matmul per head, for long sequences)
decode(S, q, k, v)        one decode step on a copy of S; returns (o, S_new)
backward(q, k, v, dO, S0, dSf, form)   gradients (dq, dk, dv, dS0) of the prefill
                          for output gradient dO and final-state gradient dSf

Inputs may be torch CPU tensors (float32 or bfloat16) or numpy arrays
(float32, or uint16 holding bfloat16 bits).  Outputs are float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB = os.path.join(_HERE, "_la_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle (plain -O2: no fast-math, no reassociation)."""
    cmd = ["gcc", "-O2", "-std=c99", "-Wall", "-shared", "-fPIC", "-o", out, src, "-lpthread"]
    subprocess.run(cmd, check=True)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.la_oracle_quadratic.argtypes = [P, P, P, I, I, I, I, L, I, P, I]
    lib.la_oracle_rows.argtypes = [P, P, P, I, I, I, I, L, I, P, L, P, I]
    lib.la_oracle_recurrent.argtypes = [P, P, P, I, I, I, I, L, I, P, P, P, P, I]
    lib.la_oracle_state.argtypes = [P, P, I, I, I, L, I, P, I]
    lib.la_oracle_decode.argtypes = [P, P, P, P, I, I, I, I, I, P, I]
    for f in (lib.la_oracle_backward_quadratic, lib.la_oracle_backward_recurrent):
        f.argtypes = [P, P, P, P, I, I, I, I, L, I, P, P, P, P, P, P, I]
    for f in (lib.la_oracle_quadratic, lib.la_oracle_rows, lib.la_oracle_recurrent,
              lib.la_oracle_state, lib.la_oracle_decode, lib.la_oracle_backward_quadratic,
              lib.la_oracle_backward_recurrent):
        f.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Return the ctypes handle, building the shared object if it is missing."""
    global _lib
    if path is not None:
        return _bind(path)
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
                build()
            _lib = _bind(_LIB)
    return _lib


def threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def _as_array(x):
    """Return (contiguous numpy array, dtype code) without changing any value."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"oracle takes float32 or bfloat16, got {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, F32
    raise TypeError(f"oracle takes float32 or bf16 bits (uint16), got {x.dtype}")


def _prep(q, k, v):
    (qa, qt), (ka, kt), (va, vt) = _as_array(q), _as_array(k), _as_array(v)
    if not (qt == kt == vt):
        raise TypeError("q, k, v must share one dtype")
    B, Hq, N, d = qa.shape
    Bk, Hkv, Nk, dk = ka.shape
    if (Bk, Nk, dk) != (B, N, d) or va.shape != ka.shape or Hq % Hkv:
        raise ValueError("shapes: q [B,Hq,N,d], k/v [B,Hkv,N,d], Hq % Hkv == 0")
    return qa, ka, va, qt, (B, Hq, Hkv, N, d)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def quadratic(q, k, v, nthreads: int | None = None) -> np.ndarray:
    qa, ka, va, dt, (B, Hq, Hkv, N, d) = _prep(q, k, v)
    o = np.empty((B, Hq, N, d), np.float64)
    rc = load().la_oracle_quadratic(_ptr(qa), _ptr(ka), _ptr(va), dt, B, Hq, Hkv, N, d, _ptr(o),
                                    nthreads or threads())
    if rc:
        raise ValueError(f"la_oracle_quadratic rc={rc}")
    return o


def rows(q, k, v, rows_bht, nthreads: int | None = None) -> np.ndarray:
    qa, ka, va, dt, (B, Hq, Hkv, N, d) = _prep(q, k, v)
    r = np.ascontiguousarray(np.asarray(rows_bht, dtype=np.int64).reshape(-1, 3))
    out = np.empty((r.shape[0], d), np.float64)
    rc = load().la_oracle_rows(_ptr(qa), _ptr(ka), _ptr(va), dt, B, Hq, Hkv, N, d, _ptr(r),
                               r.shape[0], _ptr(out), nthreads or threads())
    if rc:
        raise ValueError(f"la_oracle_rows rc={rc}")
    return out


def recurrent(q, k, v, S0=None, want_o: bool = True, o_dtype=np.float64,
              nthreads: int | None = None):
    """Token recurrence.  Returns (O or None, S_final) as float64 (O float32 if asked)."""
    qa, ka, va, dt, (B, Hq, Hkv, N, d) = _prep(q, k, v)
    S = np.empty((B, Hkv, d, d), np.float64)
    s0 = None
    if S0 is not None:
        s0 = np.ascontiguousarray(np.asarray(S0, dtype=np.float64).reshape(B, Hkv, d, d))
    o = o32 = None
    if want_o:
        if o_dtype == np.float32:
            o32 = np.empty((B, Hq, N, d), np.float32)
        else:
            o = np.empty((B, Hq, N, d), np.float64)
    rc = load().la_oracle_recurrent(
        _ptr(qa), _ptr(ka), _ptr(va), dt, B, Hq, Hkv, N, d,
        _ptr(s0) if s0 is not None else None,
        _ptr(o) if o is not None else None,
        _ptr(o32) if o32 is not None else None,
        _ptr(S), nthreads or threads())
    if rc:
        raise ValueError(f"la_oracle_recurrent rc={rc}")
    return (o if o is not None else o32), S


def state(k, v, nthreads: int | None = None) -> np.ndarray:
    (ka, kt), (va, vt) = _as_array(k), _as_array(v)
    if kt != vt or ka.shape != va.shape:
        raise ValueError("k, v must match")
    B, Hkv, N, d = ka.shape
    S = np.empty((B, Hkv, d, d), np.float64)
    rc = load().la_oracle_state(_ptr(ka), _ptr(va), kt, B, Hkv, N, d, _ptr(S), nthreads or threads())
    if rc:
        raise ValueError(f"la_oracle_state rc={rc}")
    return S


def state_gemm(k, v) -> np.ndarray:
    """S = K^T V for each (b, kv head) as one fp64 library GEMM per head.

    The same definition as ``state`` ("MiniMax-01与Lightning Attention",
    section 2.2: kv_sum over the sequence axis) with numpy's matmul as the
    summation step; used for very long sequences where the scalar loop would
    take minutes."""
    (ka, kt), (va, vt) = _as_array(k), _as_array(v)
    if kt != vt or ka.shape != va.shape:
        raise ValueError("k, v must match")
    B, Hkv, N, d = ka.shape
    S = np.empty((B, Hkv, d, d), np.float64)
    for b in range(B):
        for g in range(Hkv):
            kd, vd = _widen(ka[b, g], kt), _widen(va[b, g], vt)
            S[b, g] = kd.T @ vd
    return S


def _widen(a, dt):
    """Exact widening of fp32 values or bf16 bits to float64."""
    if dt == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def decode(S, q, k, v, nthreads: int | None = None, inplace: bool = False):
    """One step.  q [B,Hq,d]; k, v [B,Hkv,d].  Returns (o, S_new).

    S_new is a float64 copy of S after the update, or S itself when ``inplace``
    and S is already a C-contiguous float64 array."""
    (qa, qt), (ka, kt), (va, vt) = _as_array(q), _as_array(k), _as_array(v)
    if not (qt == kt == vt):
        raise TypeError("q, k, v must share one dtype")
    B, Hq, d = qa.shape
    Hkv = ka.shape[1]
    if inplace and isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous:
        Sn = S
    else:
        Sn = np.array(np.asarray(S, dtype=np.float64).reshape(B, Hkv, d, d), copy=True, order="C")
    o = np.empty((B, Hq, d), np.float64)
    rc = load().la_oracle_decode(_ptr(Sn), _ptr(qa), _ptr(ka), _ptr(va), qt, B, Hq, Hkv, d, _ptr(o),
                                 nthreads or threads())
    if rc:
        raise ValueError(f"la_oracle_decode rc={rc}")
    return o, Sn


def backward(q, k, v, dO, S0=None, dSf=None, form: str = "recurrent", nthreads: int | None = None):
    """Gradients of the prefill: returns (dq, dk, dv, dS0) as float64 arrays.

    form "quadratic" writes the sums out; "recurrent" runs a forward sweep for
    dq and a reverse sweep for dk, dv (see la_oracle.c)."""
    qa, ka, va, dt, (B, Hq, Hkv, N, d) = _prep(q, k, v)
    (da, ddt) = _as_array(dO)
    if ddt != dt or da.shape != qa.shape:
        raise ValueError("dO must match q in dtype and shape")
    f = {"quadratic": load().la_oracle_backward_quadratic,
         "recurrent": load().la_oracle_backward_recurrent}[form]
    s0 = None if S0 is None else np.ascontiguousarray(np.asarray(S0, np.float64).reshape(B, Hkv, d, d))
    dsf = None if dSf is None else np.ascontiguousarray(np.asarray(dSf, np.float64).reshape(B, Hkv, d, d))
    dq = np.empty((B, Hq, N, d), np.float64)
    dk = np.empty((B, Hkv, N, d), np.float64)
    dv = np.empty((B, Hkv, N, d), np.float64)
    dS0 = np.empty((B, Hkv, d, d), np.float64)
    rc = f(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), dt, B, Hq, Hkv, N, d,
           _ptr(s0) if s0 is not None else None, _ptr(dsf) if dsf is not None else None,
           _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dS0), nthreads or threads())
    if rc:
        raise ValueError(f"la_oracle_backward rc={rc}")
    return dq, dk, dv, dS0
