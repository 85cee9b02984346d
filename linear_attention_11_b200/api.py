"""Thin ctypes binding of ``include/la.h``: same names, argument marshalling only.

Each function takes torch CUDA tensors, passes their device pointers, sizes and
the current CUDA stream to the C ABI, and raises ``LAError`` on a non-zero
status.  No arithmetic of the method happens here; there is no CPU fallback.
The shared library is loaded on first use and a missing build is an error.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIBNAME = "liblightning_b200.so"
_lock = threading.Lock()
_lib = None

STATUS = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_CUDA",
          4: "LA_ERR_TIMEOUT", 5: "LA_ERR_WORKSPACE"}

# Every symbol include/la.h declares.
EXPORTS = ("la_status_string", "la_version", "la_forward", "la_forward_state",
           "la_forward_workspace_bytes", "la_forward_ws", "la_forward_noalloc",
           "la_forward_host", "la_prefill_fused_workspace_bytes", "la_prefill_fused",
           "la_prefill_plan", "la_backward", "la_segment_state", "la_state_prefix",
           "la_prefill_span_states", "la_prefill_scan", "la_prefill_main", "la_forward_f32",
           "la_decode_step", "la_decode_steps", "la_device_status", "la_selftest_wait",
           "la_shutdown")


class LAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class la_plan(ctypes.Structure):
    _fields_ = [("nspan", ctypes.c_int32), ("tile", ctypes.c_int32),
                ("heads_per_tile", ctypes.c_int32), ("tiles_total", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_int64)]


def library_path() -> str:
    return os.environ.get("LA_LIBRARY", os.path.join(_HERE, _LIBNAME))


def _declare(lib):
    P, I, L, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    PP = ctypes.POINTER(la_plan)
    sig = {
        "la_status_string": ([I], ctypes.c_char_p),
        "la_version": ([], I),
        "la_forward": ([P, P, P, P, I, I, I, L, I, I, P], I),
        "la_forward_state": ([P, P, P, P, P, I, I, I, L, I, I, P], I),
        "la_forward_workspace_bytes": ([I, I, I, L, I, I], S),
        "la_forward_ws": ([P, P, P, P, P, I, I, I, L, I, I, P, S, P], I),
        "la_forward_noalloc": ([P, P, P, P, P, I, I, I, L, I, I, P], I),
        "la_forward_host": ([P, P, P, P, P, I, I, I, L, I, I, L, P], I),
        "la_prefill_fused_workspace_bytes": ([I, I, I, L, I, I, I], S),
        "la_prefill_fused": ([P, P, P, P, P, I, I, I, L, I, I, I, I, P, S, P], I),
        "la_prefill_plan": ([I, I, I, L, I, I, PP], I),
        "la_prefill_span_states": ([P, P, I, I, L, I, PP, P, P], I),
        "la_prefill_scan": ([P, P, I, I, I, PP, P], I),
        "la_prefill_main": ([P, P, P, P, P, I, I, I, L, I, PP, P], I),
        "la_forward_f32": ([P, P, P, P, P, I, I, I, L, I, I, P], I),
        "la_backward": ([P, P, P, P, P, P, P, P, P, P, I, I, I, L, I, I, P], I),
        "la_segment_state": ([P, P, P, I, I, L, I, I, P], I),
        "la_state_prefix": ([P, P, P, I, I, I, I, I, P], I),
        "la_decode_step": ([P, P, P, P, P, I, I, I, I, P], I),
        "la_decode_steps": ([P, P, P, P, P, I, I, I, I, I, P], I),
        "la_device_status": ([ctypes.POINTER(ctypes.c_uint), I], I),
        "la_selftest_wait": ([L, P], I),
        "la_shutdown": ([], None),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


def load_library(path: str | None = None):
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or library_path()
            if not os.path.exists(p):
                raise RuntimeError(
                    f"CUDA library not built: {p} is missing "
                    "(run `python -m linear_attention_11_b200.build`)")
            _lib = _declare(ctypes.CDLL(p))
    return _lib


def _check(fn: str, code: int):
    if code != 0:
        raise LAError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _on_device(t) -> bool:
    return t.is_cuda


def _need(fn, name, t, dtype=None, device=True):
    """Reject what the library would misread: host memory where device memory
    is expected (or the reverse), another element type, or a strided view."""
    if t is None:
        return
    if _on_device(t) != device:
        raise ValueError(f"{fn}: {name} must be a {'CUDA' if device else 'host'} tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{fn}: {name} must be {dtype}, not {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{fn}: {name} must be contiguous")


def _qkv(fn, q, k, v, o=None, dtype=torch.bfloat16, device=True):
    """q, o [B,Hq,N,d] and k, v [B,Hkv,N,d] of one dtype -> (B, Hq, Hkv, N, d)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(fn, name, t, dtype, device)
    if (q.dim() != 4 or k.dim() != 4 or k.shape != v.shape or k.shape[0] != q.shape[0]
            or k.shape[2:] != q.shape[2:] or (o is not None and o.shape != q.shape)):
        raise ValueError(f"{fn}: expected q, o [B,Hq,N,d] and k, v [B,Hkv,N,d]; got q "
                         f"{tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}"
                         + ("" if o is None else f", o {tuple(o.shape)}"))
    B, Hq, N, d = q.shape
    return B, Hq, k.shape[1], N, d


def _state(fn, name, S, B, Hkv, d):
    """S [B,Hkv,d,d] fp32 on the device (or None)."""
    _need(fn, name, S, torch.float32)
    if S is not None and tuple(S.shape) != (B, Hkv, d, d):
        raise ValueError(f"{fn}: {name} must be [{B},{Hkv},{d},{d}], not {tuple(S.shape)}")


def la_status_string(code: int) -> str:
    return load_library().la_status_string(code).decode()


def la_forward(q, k, v, o=None, chunk: int = 64, stream=None):
    """O for q [B,Hq,N,d], k, v [B,Hkv,N,d] (bf16, CUDA); zero initial state."""
    B, Hq, Hkv, N, d = _qkv("la_forward", q, k, v, o)
    if o is None:
        o = torch.empty_like(q)
    _check("la_forward", load_library().la_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, Hkv, N, d, chunk, _stream(stream)))
    return o


def la_forward_state(q, k, v, S=None, o=None, chunk: int = 64, stream=None):
    """As la_forward; S [B,Hkv,d,d] fp32 (in: initial state, out: final state)."""
    B, Hq, Hkv, N, d = _qkv("la_forward_state", q, k, v, o)
    _state("la_forward_state", "S", S, B, Hkv, d)
    if o is None:
        o = torch.empty_like(q)
    _check("la_forward_state", load_library().la_forward_state(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, Hq, Hkv, N, d, chunk, _stream(stream)))
    return o


def la_forward_workspace_bytes(B, Hq, Hkv, N, d, chunk) -> int:
    return int(load_library().la_forward_workspace_bytes(B, Hq, Hkv, N, d, chunk))


def la_forward_ws(q, k, v, o, S, workspace, chunk: int = 64, stream=None):
    B, Hq, Hkv, N, d = _qkv("la_forward_ws", q, k, v, o)
    _state("la_forward_ws", "S", S, B, Hkv, d)
    _need("la_forward_ws", "workspace", workspace)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("la_forward_ws", load_library().la_forward_ws(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, Hq, Hkv, N, d, chunk,
        _ptr(workspace), nbytes, _stream(stream)))
    return o


def la_forward_noalloc(q, k, v, S=None, o=None, chunk: int = 64, stream=None):
    """As la_forward_state, with the library's fixed device scratch instead of
    an allocation (for callers that cannot allocate device memory)."""
    B, Hq, Hkv, N, d = _qkv("la_forward_noalloc", q, k, v, o)
    _state("la_forward_noalloc", "S", S, B, Hkv, d)
    if o is None:
        o = torch.empty_like(q)
    _check("la_forward_noalloc", load_library().la_forward_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, Hq, Hkv, N, d, chunk, _stream(stream)))
    return o


def la_forward_host(q, k, v, o=None, S=None, chunk: int = 64, piece: int = 0, stream=None):
    """Prefill from and to pinned host tensors (q, k, v, o on the CPU, pinned);
    S, if given, is a CUDA tensor.  Asynchronous on `stream`."""
    B, Hq, Hkv, N, d = _qkv("la_forward_host", q, k, v, o, device=False)
    _state("la_forward_host", "S", S, B, Hkv, d)
    if o is None:
        o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    _check("la_forward_host", load_library().la_forward_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, Hq, Hkv, N, d, chunk, piece,
        _stream(stream)))
    return o


def la_prefill_fused_workspace_bytes(B, Hq, Hkv, N, d, chunk, nspan=0) -> int:
    return int(load_library().la_prefill_fused_workspace_bytes(B, Hq, Hkv, N, d, chunk, nspan))


def la_prefill_fused(q, k, v, o, S, workspace, chunk: int = 64, nspan: int = 0,
                     lookahead: int = 0, stream=None):
    """The single-pass prefill with an explicit span count and lookahead (0 = automatic)."""
    B, Hq, Hkv, N, d = _qkv("la_prefill_fused", q, k, v, o)
    _state("la_prefill_fused", "S", S, B, Hkv, d)
    _need("la_prefill_fused", "workspace", workspace)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("la_prefill_fused", load_library().la_prefill_fused(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, Hq, Hkv, N, d, chunk, nspan, lookahead,
        _ptr(workspace), nbytes, _stream(stream)))
    return o


def la_prefill_plan(B, Hq, Hkv, N, d, chunk) -> la_plan:
    plan = la_plan()
    _check("la_prefill_plan", load_library().la_prefill_plan(B, Hq, Hkv, N, d, chunk,
                                                             ctypes.byref(plan)))
    return plan


def la_prefill_span_states(k, v, plan: la_plan, ws, stream=None):
    B, _, Hkv, N, d = _qkv("la_prefill_span_states", k, k, v)
    _need("la_prefill_span_states", "ws", ws)
    _check("la_prefill_span_states", load_library().la_prefill_span_states(
        _ptr(k), _ptr(v), B, Hkv, N, d, ctypes.byref(plan), _ptr(ws), _stream(stream)))


def la_prefill_scan(ws, S, plan: la_plan, B, Hkv, d, stream=None):
    _need("la_prefill_scan", "ws", ws)
    _state("la_prefill_scan", "S", S, B, Hkv, d)
    _check("la_prefill_scan", load_library().la_prefill_scan(
        _ptr(ws), _ptr(S), B, Hkv, d, ctypes.byref(plan), _stream(stream)))


def la_prefill_main(q, k, v, o, ws, plan: la_plan, stream=None):
    B, Hq, Hkv, N, d = _qkv("la_prefill_main", q, k, v, o)
    _need("la_prefill_main", "ws", ws)
    _check("la_prefill_main", load_library().la_prefill_main(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ws), B, Hq, Hkv, N, d, ctypes.byref(plan),
        _stream(stream)))


def la_segment_state(k, v, S=None, chunk: int = 64, stream=None):
    """K^T V of one segment's k, v [B,Hkv,N,d] (bf16, CUDA) -> S [B,Hkv,d,d] fp32."""
    B, _, Hkv, N, d = _qkv("la_segment_state", k, k, v)
    _state("la_segment_state", "S", S, B, Hkv, d)
    if S is None:
        S = torch.empty(B, Hkv, d, d, dtype=torch.float32, device=k.device)
    _check("la_segment_state", load_library().la_segment_state(
        _ptr(k), _ptr(v), _ptr(S), B, Hkv, N, d, chunk, _stream(stream)))
    return S


def la_state_prefix(states, seg: int, S0=None, S=None, stream=None):
    """S0 (or 0) + sum of states[:seg]; states [nseg,B,Hkv,d,d] fp32 (CUDA)."""
    _need("la_state_prefix", "states", states, torch.float32)
    if states.dim() != 5 or states.shape[3] != states.shape[4]:
        raise ValueError(f"la_state_prefix: states must be [nseg,B,Hkv,d,d], not "
                         f"{tuple(states.shape)}")
    nseg, B, Hkv, d, _ = states.shape
    _state("la_state_prefix", "S0", S0, B, Hkv, d)
    _state("la_state_prefix", "S", S, B, Hkv, d)
    if S is None:
        S = torch.empty(B, Hkv, d, d, dtype=torch.float32, device=states.device)
    _check("la_state_prefix", load_library().la_state_prefix(
        _ptr(states), _ptr(S0), _ptr(S), nseg, seg, B, Hkv, d, _stream(stream)))
    return S


def la_backward(q, k, v, dO, S0=None, dSf=None, want_dS0: bool = False, chunk: int = 64,
                stream=None):
    """Gradients (dq, dk, dv, dS0 or None) of the prefill for output gradient dO
    and final-state gradient dSf (CUDA tensors; S0 the forward's initial state)."""
    B, Hq, Hkv, N, d = _qkv("la_backward", q, k, v, dO)
    _state("la_backward", "S0", S0, B, Hkv, d)
    _state("la_backward", "dSf", dSf, B, Hkv, d)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dS0 = torch.empty(B, Hkv, d, d, dtype=torch.float32, device=q.device) if want_dS0 else None
    _check("la_backward", load_library().la_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(S0), _ptr(dSf), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(dS0), B, Hq, Hkv, N, d, chunk, _stream(stream)))
    return dq, dk, dv, dS0


def la_forward_f32(q, k, v, o=None, S=None, chunk: int = 64, stream=None):
    B, Hq, Hkv, N, d = _qkv("la_forward_f32", q, k, v, o, dtype=torch.float32)
    _state("la_forward_f32", "S", S, B, Hkv, d)
    if o is None:
        o = torch.empty_like(q)
    _check("la_forward_f32", load_library().la_forward_f32(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, Hq, Hkv, N, d, chunk, _stream(stream)))
    return o


def la_decode_step(S, q, k, v, o=None, stream=None):
    """One decode step: S [B,Hkv,d,d] fp32 updated in place; returns o [B,Hq,d]."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need("la_decode_step", name, t, torch.bfloat16)
    if (q.dim() != 3 or k.shape != v.shape or k.dim() != 3 or k.shape[0] != q.shape[0]
            or k.shape[2] != q.shape[2] or (o is not None and o.shape != q.shape)):
        raise ValueError(f"la_decode_step: expected q, o [B,Hq,d] and k, v [B,Hkv,d]; got q "
                         f"{tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    B, Hq, d = q.shape
    _state("la_decode_step", "S", S, B, k.shape[1], d)
    if S is None:
        raise ValueError("la_decode_step: S is required")
    if o is None:
        o = torch.empty_like(q)
    _check("la_decode_step", load_library().la_decode_step(
        _ptr(S), _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, k.shape[1], d, _stream(stream)))
    return o


def la_decode_steps(S, q, k, v, o=None, stream=None):
    """Several decode steps: q [B,Hq,steps,d], k, v [B,Hkv,steps,d]; S updated in place."""
    B, Hq, Hkv, steps, d = _qkv("la_decode_steps", q, k, v, o)
    _state("la_decode_steps", "S", S, B, Hkv, d)
    if S is None:
        raise ValueError("la_decode_steps: S is required")
    if o is None:
        o = torch.empty_like(q)
    _check("la_decode_steps", load_library().la_decode_steps(
        _ptr(S), _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Hq, k.shape[1], d, steps, _stream(stream)))
    return o


def la_device_status(clear: bool = True):
    """(status code, device flags).  Synchronises the current device."""
    flags = ctypes.c_uint(0)
    code = load_library().la_device_status(ctypes.byref(flags), 1 if clear else 0)
    return code, flags.value


def la_selftest_wait(timeout_ns: int, stream=None):
    _check("la_selftest_wait", load_library().la_selftest_wait(timeout_ns, _stream(stream)))


def la_shutdown():
    load_library().la_shutdown()
