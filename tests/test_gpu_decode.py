"""Decode step on the GPU against the fp64 oracle's decode step."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("B,Hq,Hkv,d", [(3, 4, 2, 128), (2, 6, 3, 64), (1, 32, 1, 128), (5, 1, 1, 64)])
def test_decode_small(la, B, Hq, Hkv, d):
    w = synth.Decode("t", B, Hq, Hkv, d, 5, 9)
    S = synth.decode_state(w)
    Sref = S.double().numpy().copy()
    Sd = S.to(DEV)
    for step in range(w.steps):
        q, k, v = synth.decode_token(w, step)
        o_ref, Sref = oracle.decode(Sref, q, k, v)
        o = la.la_decode_step(Sd, q.to(DEV), k.to(DEV), v.to(DEV))
        torch.cuda.synchronize()
        assert_bf16_close(o.cpu(), o_ref, f"o step {step}")
    assert_f32_close(Sd.cpu(), Sref, "state", tol=1e-6)


def test_decode_continues_prefill(la):
    """Prefill N tokens, then decode the next ones: rows equal one longer prefill."""
    B, Hq, Hkv, N, extra = 1, 4, 2, 300, 6
    q, k, v = synth.random_qkv(B, Hq, Hkv, N + extra, 128, torch.bfloat16, 77)
    ref_o, ref_S = oracle.recurrent(q, k, v)
    S = torch.zeros(B, Hkv, 128, 128, device=DEV)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    la.la_forward_state(*(t[:, :, :N].contiguous() for t in (qd, kd, vd)), S=S, chunk=64)
    for t in range(N, N + extra):
        o = la.la_decode_step(S, qd[:, :, t].contiguous(), kd[:, :, t].contiguous(),
                              vd[:, :, t].contiguous())
        torch.cuda.synchronize()
        assert_bf16_close(o.cpu(), ref_o[:, :, t], f"decode row {t}")
    assert_f32_close(S.cpu(), ref_S, "state after decode", tol=1e-6)


def test_decode_full_b256_64_steps(la):
    """The decode workload: B=256, Hq=64/Hkv=16, d=128, 64 consecutive steps."""
    w = synth.DECODE_B256
    S = synth.decode_state(w)
    Sref = np.ascontiguousarray(S.double().numpy())
    Sd = S.to(DEV)
    worst = 0.0
    for step in range(w.steps):
        q, k, v = synth.decode_token(w, step)
        o_ref, Sref = oracle.decode(Sref, q, k, v, inplace=True)
        o = la.la_decode_step(Sd, q.to(DEV), k.to(DEV), v.to(DEV))
        torch.cuda.synchronize()
        rel, _ = assert_bf16_close(o.cpu(), o_ref, f"o step {step}")
        worst = max(worst, rel)
    assert_f32_close(Sd.cpu(), Sref, "state after 64 steps", tol=1e-6)


# ------------------------------------------------------------------ several steps per launch
def _stack_steps(w, steps, B=None):
    toks = [synth.decode_token(w, t, B=B) for t in range(steps)]
    q = torch.stack([t[0] for t in toks], dim=2).contiguous()  # [B, Hq, steps, d]
    k = torch.stack([t[1] for t in toks], dim=2).contiguous()  # [B, Hkv, steps, d]
    v = torch.stack([t[2] for t in toks], dim=2).contiguous()
    return q, k, v


@pytest.mark.parametrize("B,Hq,Hkv,d,steps", [(3, 4, 2, 128, 5), (2, 6, 3, 64, 17), (1, 32, 1, 128, 3),
                                               (4, 8, 8, 128, 1), (2, 2, 1, 64, 40),
                                               # groups of 3, 6, 12: passes of 2, 4, 8 heads
                                               # with a shorter last pass
                                               (2, 9, 3, 128, 7), (1, 12, 2, 128, 9),
                                               (1, 24, 2, 64, 6)])
def test_decode_steps_matches_recurrence(la, B, Hq, Hkv, d, steps):
    w = synth.Decode("t", B, Hq, Hkv, d, steps, 13)
    S0 = synth.decode_state(w)
    q, k, v = _stack_steps(w, steps)
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy())
    S = S0.to(DEV)
    o = la.la_decode_steps(S, q.to(DEV), k.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    assert_bf16_close(o.cpu(), ref_o, "o")
    assert_f32_close(S.cpu(), ref_S, "state", tol=1e-6)


def test_decode_steps_equals_single_steps(la):
    """64 steps of the decode workload in one launch: the state is bitwise the
    state of 64 single-step launches (the same fp32 FMA per element, in token
    order); the outputs agree within bf16 rounding (their dot products are
    summed in a different order)."""
    w = synth.DECODE_B256
    S0 = synth.decode_state(w)
    q, k, v = _stack_steps(w, w.steps)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    S_multi = S0.to(DEV)
    o_multi = la.la_decode_steps(S_multi, qd, kd, vd)
    S_single = S0.to(DEV)
    outs = [la.la_decode_step(S_single, qd[:, :, t].contiguous(), kd[:, :, t].contiguous(),
                              vd[:, :, t].contiguous()) for t in range(w.steps)]
    torch.cuda.synchronize()
    assert torch.equal(S_multi, S_single)
    assert_bf16_close(o_multi.cpu(), torch.stack(outs, dim=2).cpu(), "o, one launch vs 64")
