"""la_forward_noalloc: the prefill for callers that cannot allocate device
memory at call time -- code running inside an allocator or memory-pool
callback (where a nested allocation would re-enter the allocator), frameworks
that own every device byte and reject foreign allocations, and paths that must
not block in the driver's allocator.  Its workspace (the span states) is a
fixed device array inside the library.

Checked through the C ABI on two calls in a row with different inputs (the
second call reuses whatever the first left in the shared array): against the
fp64 oracle, and against la_forward_state (the entry point that allocates its
workspace) within the same tolerance.  One shape plans more span states than
the array holds, so the entry point lowers the span count; another plans one
span per sequence, which needs no workspace.  A last test checks the defining
property: after a warm-up call, a call changes neither the device's free
memory nor the default memory pool's reservation.

This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import STATE_REL_L2, assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCRATCH_BYTES = 32 << 20  # the array's size, as include/la.h states it


def _call_noalloc(lib, q, k, v, o, S, chunk):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.la_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                  S.data_ptr() if S is not None else None, B, Hq, Hkv, N, d,
                                  chunk, stream)


def _two_calls(la, B, Hq, Hkv, N, chunk, seeds):
    """Two calls in a row, each against the oracle and against la_forward_state."""
    lib = la.api.load_library()
    for call, seed in enumerate(seeds):
        q, k, v = synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, seed)
        S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(seed)) / 128
        ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy(), o_dtype=np.float32)
        qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
        S_alloc, S_new = S0.to(DEV), S0.to(DEV)
        o_alloc = la.la_forward_state(qd, kd, vd, S=S_alloc, chunk=chunk)
        o_new = torch.full_like(qd, float("nan"))
        assert _call_noalloc(lib, qd, kd, vd, o_new, S_new, chunk) == 0
        torch.cuda.synchronize()
        got_o, got_S = o_new.cpu(), S_new.cpu()
        assert_bf16_close(got_o, ref_o, f"call {call}: O vs oracle")
        assert_f32_close(got_S, ref_S, f"call {call}: final state vs oracle", tol=STATE_REL_L2)
        assert_bf16_close(got_o, o_alloc.cpu(), f"call {call}: O vs la_forward_state")
        assert_f32_close(got_S, S_alloc.cpu(), f"call {call}: state vs la_forward_state",
                         tol=STATE_REL_L2)
    assert la.la_device_status()[0] == 0


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", [(1, 8, 2, 1500, 64), (2, 4, 4, 777, 128)])
def test_noalloc_two_calls(la, B, Hq, Hkv, N, chunk):
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk)
    assert plan.nspan > 1 and plan.workspace_bytes <= SCRATCH_BYTES
    _two_calls(la, B, Hq, Hkv, N, chunk, (201, 202))


def test_noalloc_lowers_span_count_past_the_array(la):
    """171 kv groups of 384 tokens: the planner takes three spans each, 513
    span states (32.06 MiB), one more than the array holds, so the entry
    point runs the span scheme with two spans instead."""
    B, Hq, Hkv, N, chunk = 57, 12, 3, 384, 128
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk)
    assert plan.nspan == 3
    assert plan.workspace_bytes > SCRATCH_BYTES
    assert SCRATCH_BYTES // (B * Hkv * 128 * 128 * 4) == 2  # the lowered span count
    _two_calls(la, B, Hq, Hkv, N, chunk, (205, 206))


def test_noalloc_one_span_per_sequence(la):
    """1024 kv groups of 80 tokens: one span each, so the call is the single
    chunk-loop launch that reads the state and writes it back in place; it
    uses none of the array and equals la_forward_state bit for bit."""
    lib = la.api.load_library()
    B, Hq, Hkv, N, chunk = 256, 16, 4, 80, 64
    assert la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).nspan == 1
    q, k, v = synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, 203)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(204)) / 128
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy(), o_dtype=np.float32)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    S_ref, S_new = S0.to(DEV), S0.to(DEV)
    o_ref = la.la_forward_state(qd, kd, vd, S=S_ref, chunk=chunk)
    o_new = torch.empty_like(qd)
    assert _call_noalloc(lib, qd, kd, vd, o_new, S_new, chunk) == 0
    torch.cuda.synchronize()
    assert_bf16_close(o_new.cpu(), ref_o, "O vs oracle")
    assert_f32_close(S_new.cpu(), ref_S, "final state vs oracle", tol=STATE_REL_L2)
    assert torch.equal(o_new, o_ref)
    assert torch.equal(S_new, S_ref)
    assert la.la_device_status()[0] == 0


def _pool_reserved(dev):
    from cuda.bindings import runtime as rt
    err, pool = rt.cudaDeviceGetDefaultMemPool(dev)
    assert err == rt.cudaError_t.cudaSuccess
    err, val = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrReservedMemCurrent)
    assert err == rt.cudaError_t.cudaSuccess
    return int(val)


def test_noalloc_allocates_nothing_after_warm_up(la):
    """After one warm-up call (which may load modules), a multi-span call
    leaves the device's free memory and the default pool's reservation as
    they were, with the pool trimmed to nothing beforehand."""
    lib = la.api.load_library()
    B, Hq, Hkv, N, chunk = 1, 8, 2, 4096, 64
    assert la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).nspan > 1
    q, k, v = (t.to(DEV) for t in synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, 207))
    S = torch.zeros(B, Hkv, 128, 128, device=DEV)
    o = torch.empty_like(q)
    assert _call_noalloc(lib, q, k, v, o, S, chunk) == 0  # warm-up
    torch.cuda.synchronize()
    lib.la_shutdown()  # trims the default pool
    torch.cuda.synchronize()
    dev = torch.cuda.current_device()
    free0, reserved0 = torch.cuda.mem_get_info(dev)[0], _pool_reserved(dev)
    for _ in range(2):
        assert _call_noalloc(lib, q, k, v, o, S, chunk) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0
    assert _pool_reserved(dev) == reserved0
    assert la.la_device_status()[0] == 0
