"""Backward of the bf16 prefill on the GPU (tensor-core passes through the C
ABI) against the fp64 backward oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import STATE_REL_L2, assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _inputs(B, Hq, Hkv, N, seed, states):
    q, k, v = synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, seed)
    dO = synth.random_qkv(B, Hq, Hq, N, 128, torch.bfloat16, seed + 1)[0]
    g = torch.Generator().manual_seed(seed + 2)
    S0 = torch.randn(B, Hkv, 128, 128, generator=g) / 128 if states else None
    dSf = torch.randn(B, Hkv, 128, 128, generator=g) / 128 if states else None
    return q, k, v, dO, S0, dSf


def _check(la, q, k, v, dO, S0, dSf, chunk, form, what):
    ref = oracle.backward(q, k, v, dO,
                          S0=None if S0 is None else S0.double().numpy(),
                          dSf=None if dSf is None else dSf.double().numpy(), form=form)
    dev = [t.to(DEV) for t in (q, k, v, dO)]
    got = la.la_backward(*dev, S0=None if S0 is None else S0.to(DEV),
                         dSf=None if dSf is None else dSf.to(DEV), want_dS0=True, chunk=chunk)
    torch.cuda.synchronize()
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        assert_bf16_close(g.cpu(), r, f"{what} {name}")
    assert_f32_close(got[3].cpu(), ref[3], f"{what} dS0", tol=STATE_REL_L2)
    assert la.la_device_status()[1] == 0


SMALL = [
    # B, Hq, Hkv, N, chunk, with states
    (1, 2, 2, 300, 64, False),
    (2, 4, 2, 777, 64, True),
    (1, 8, 2, 1000, 128, True),
    (1, 1, 1, 129, 64, True),
    (1, 4, 1, 64, 64, False),
    (1, 3, 1, 385, 128, True),
    (1, 2, 1, 1, 64, True),
    (64, 4, 4, 200, 64, True),   # one span per group, CTAs with two groups
    (3, 8, 1, 2000, 128, True),  # eight query heads per group, many spans
]


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk,states", SMALL)
def test_backward_small(la, B, Hq, Hkv, N, chunk, states):
    q, k, v, dO, S0, dSf = _inputs(B, Hq, Hkv, N, 600 + N + Hq, states)
    _check(la, q, k, v, dO, S0, dSf, chunk, "quadratic", f"{B}x{Hq}/{Hkv}x{N}")


def test_backward_full_gqa_32k(la):
    w = synth.GQA_32K
    q, k, v = synth.prefill_inputs(w)
    dO = synth.random_qkv(w.B, w.Hq, w.Hq, w.N, w.d, torch.bfloat16, 77)[0]
    _check(la, q, k, v, dO, None, None, 64, "recurrent", w.name)
