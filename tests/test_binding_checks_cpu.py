"""Argument checks of the Python binding, without a GPU: a fake library
stands in for the CUDA one, and host tensors stand in for device tensors
(the device predicate is patched), so every entry point can be called.
Well-formed calls reach the library; host tensors where device ones are
expected (and the reverse), other dtypes, strided views and inconsistent
shapes raise ValueError before any call; the library's own errors still come
back as LAError."""
import pytest
import torch

from linear_attention_11_b200 import api

bf16, f32 = torch.bfloat16, torch.float32


class FakeLib:
    def __init__(self):
        self.calls, self.code = [], 0

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return self.code
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(api, "load_library", lambda path=None: lib)
    monkeypatch.setattr(api, "_stream", lambda stream: None)
    monkeypatch.setattr(api, "_on_device", lambda t: getattr(t, "on_host", False) is False)
    return lib


def host(t):
    t.on_host = True
    return t


def qkv(B=1, Hq=4, Hkv=2, N=8, d=128, dtype=bf16):
    return (torch.zeros(B, Hq, N, d, dtype=dtype), torch.zeros(B, Hkv, N, d, dtype=dtype),
            torch.zeros(B, Hkv, N, d, dtype=dtype))


def S(B=1, Hkv=2, d=128):
    return torch.zeros(B, Hkv, d, d, dtype=f32)


def test_well_formed_calls_reach_the_library(fake):
    q, k, v = qkv()
    api.la_forward(q, k, v)
    api.la_forward_state(q, k, v, S=S())
    api.la_forward_ws(q, k, v, torch.empty_like(q), S(), torch.zeros(64, dtype=torch.uint8))
    api.la_forward_noalloc(q, k, v, S=S())
    api.la_prefill_fused(q, k, v, torch.empty_like(q), None, torch.zeros(16))
    api.la_prefill_span_states(k, v, api.la_plan(), torch.zeros(16))
    api.la_prefill_scan(torch.zeros(16), S(), api.la_plan(), 1, 2, 128)
    api.la_prefill_main(q, k, v, torch.empty_like(q), None, api.la_plan())
    api.la_segment_state(k, v)
    api.la_state_prefix(torch.zeros(3, 1, 2, 128, 128), 1, S0=S())
    api.la_backward(q, k, v, torch.zeros_like(q), S0=S(), dSf=S(), want_dS0=True)
    qf, kf, vf = qkv(d=64, dtype=f32)
    api.la_forward_f32(qf, kf, vf, S=S(d=64))
    api.la_decode_step(S(), q[:, :, 0].contiguous(), k[:, :, 0].contiguous(),
                       v[:, :, 0].contiguous())
    api.la_decode_steps(S(), q, k, v)
    qh, kh, vh = (host(t) for t in qkv())
    api.la_forward_host(qh, kh, vh, o=host(torch.empty_like(qh)), S=S())
    assert fake.calls == ["la_forward", "la_forward_state", "la_forward_ws", "la_forward_noalloc",
                          "la_prefill_fused", "la_prefill_span_states", "la_prefill_scan",
                          "la_prefill_main", "la_segment_state", "la_state_prefix",
                          "la_backward", "la_forward_f32", "la_decode_step", "la_decode_steps",
                          "la_forward_host"]


def test_library_errors_still_raise_laerror(fake):
    """Arguments the binding passes on (aliasing, chunk, head size, empty
    shapes) are the library's to reject."""
    fake.code = 1
    q, k, v = qkv()
    with pytest.raises(api.LAError):
        api.la_forward(q, k, v, o=q)
    q0 = torch.zeros(1, 2, 0, 128, dtype=bf16)
    with pytest.raises(api.LAError):
        api.la_forward(q0, q0.clone(), q0.clone())
    q64 = torch.zeros(1, 2, 64, 64, dtype=bf16)
    with pytest.raises(api.LAError):
        api.la_forward(q64, q64.clone(), q64.clone(), chunk=32)
    qt = torch.zeros(0, 1, 128, dtype=bf16)
    with pytest.raises(api.LAError):
        api.la_decode_step(torch.zeros(0, 1, 128, 128), qt, qt.clone(), qt.clone())
    with pytest.raises(api.LAError):
        api.la_state_prefix(torch.zeros(5, 1, 2, 128, 128), 5)


def test_host_memory_where_device_memory_is_expected(fake):
    q, k, v = qkv()
    with pytest.raises(ValueError, match="CUDA"):
        api.la_forward(host(q), k, v)
    with pytest.raises(ValueError, match="CUDA"):
        api.la_forward_state(q, k, v, S=host(S()))
    with pytest.raises(ValueError, match="CUDA"):
        api.la_backward(q, k, v, host(torch.zeros_like(q)))
    with pytest.raises(ValueError, match="host"):
        api.la_forward_host(q, k, v)          # device tensors on the host path
    assert fake.calls == []


def test_wrong_dtype_view_or_shape(fake):
    q, k, v = qkv()
    with pytest.raises(ValueError, match="bfloat16"):
        api.la_forward(q.float(), k, v)
    with pytest.raises(ValueError, match="float32"):
        api.la_forward_state(q, k, v, S=S().double())
    with pytest.raises(ValueError, match="contiguous"):
        api.la_forward(q.transpose(2, 3), k, v)
    with pytest.raises(ValueError, match="expected q"):
        api.la_forward(q, k, v[:, :, :4].contiguous())       # N differs
    with pytest.raises(ValueError, match="expected q"):
        api.la_forward(q, k, v, o=torch.zeros(1, 4, 9, 128, dtype=bf16))
    with pytest.raises(ValueError, match="must be \\[1,2,128,128\\]"):
        api.la_forward_state(q, k, v, S=S(Hkv=4))
    with pytest.raises(ValueError, match="expected q"):
        api.la_decode_step(S(), q[:, :, 0].contiguous(), k[:, :, 0, :64].contiguous(),
                           v[:, :, 0, :64].contiguous())
    with pytest.raises(ValueError, match="required"):
        api.la_decode_steps(None, q, k, v)
    with pytest.raises(ValueError, match="nseg"):
        api.la_state_prefix(torch.zeros(2, 128, 128), 0)
    assert fake.calls == []
