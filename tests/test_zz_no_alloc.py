"""la_forward_noalloc: the prefill for callers that cannot allocate device
memory (allocator callbacks, frameworks that own all device memory, paths that
must not block in the driver's allocator).  It takes its workspace (span
states, or the counters of the single-span launch) from a fixed device array
inside the library.

Checked through the C ABI against la_forward_state, the entry point that
allocates its workspace, on two calls in a row with different inputs (the
second call reuses whatever the first left in the shared array).  This file
sorts last so that a run stopping at the first failure has already run every
other test.
"""
import ctypes

import pytest
import torch

from linear_attention_11_b200 import synth

from _compare import STATE_REL_L2, assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _call_noalloc(lib, q, k, v, o, S, chunk):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.la_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  S.data_ptr() if S is not None else None, B, Hq, Hkv, N, d,
                                  chunk, stream)


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", [(1, 8, 2, 1500, 64), (2, 4, 4, 777, 128)])
def test_noalloc_matches_allocating_entry_point(la, B, Hq, Hkv, N, chunk):
    lib = la.api.load_library()
    for call, seed in enumerate((201, 202)):
        q, k, v = (t.to(DEV) for t in synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, seed))
        S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(seed)) / 128
        S_ref, S_new = S0.to(DEV), S0.to(DEV)
        o_ref = la.la_forward_state(q, k, v, S=S_ref, chunk=chunk)
        o_new = torch.empty_like(q)
        assert _call_noalloc(lib, q, k, v, o_new, S_new, chunk) == 0
        torch.cuda.synchronize()
        assert_bf16_close(o_new.cpu(), o_ref.cpu(), f"call {call}: O")
        assert_f32_close(S_new.cpu(), S_ref.cpu(), f"call {call}: final state", tol=STATE_REL_L2)
    assert la.la_device_status()[0] == 0


def test_noalloc_one_span_beyond_span_state_limit(la):
    """1024 kv heads would need 64 MiB of span states (over the 32 MiB
    array) even at one span each; with one span the call runs as the single
    chunk-loop launch, which needs only 4 KiB of counters, in place on S."""
    lib = la.api.load_library()
    B, Hq, Hkv, N, chunk = 256, 16, 4, 80, 64
    assert la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).nspan == 1
    q, k, v = (t.to(DEV) for t in synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, 203))
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(204)) / 128
    S_ref, S_new = S0.to(DEV), S0.to(DEV)
    o_ref = la.la_forward_state(q, k, v, S=S_ref, chunk=chunk)
    o_new = torch.empty_like(q)
    assert _call_noalloc(lib, q, k, v, o_new, S_new, chunk) == 0
    torch.cuda.synchronize()
    assert torch.equal(o_new, o_ref)
    assert torch.equal(S_new, S_ref)
    assert la.la_device_status()[0] == 0
