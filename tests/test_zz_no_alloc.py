"""la_forward_noalloc: the prefill for callers that cannot allocate device
memory (allocator callbacks, frameworks that own all device memory, paths that
must not block in the driver's allocator).  It takes its span-state workspace
from a fixed device array inside the library.

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


def test_noalloc_rejects_problems_beyond_its_scratch(la):
    lib = la.api.load_library()
    # B * Hkv = 1024 kv heads need 64 MiB for a single span each: over the 32 MiB limit.
    q = torch.zeros(1, 1024, 1, 128, dtype=torch.bfloat16, device=DEV)
    k, v, o = torch.zeros_like(q), torch.zeros_like(q), torch.empty_like(q)
    assert _call_noalloc(lib, q, k, v, o, None, 64) == 5  # LA_ERR_WORKSPACE
