"""Seeded random shapes across the scheduling regimes of the bf16 prefill
(span counts from 1 up, sub-span parts, one-launch with staged or row-by-row
states, 64- and 128-token tiles, groups of 1-8 query heads, ragged N), each
with and without an initial state, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import STATE_REL_L2, assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _cases(n=24, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        G = int(rng.choice([1, 2, 3, 4, 8]))
        Hkv = int(rng.integers(1, 5))
        B = int(rng.choice([1, 2, 3, 8, 24, 48]))
        N = int(rng.choice([1, 17, 64, 100, 255, 640, 1111, 2048]))
        chunk = int(rng.choice([64, 128]))
        # keep the fp64 oracle to a few seconds: tokens x heads bounded
        if B * Hkv * G * N > 300_000:
            continue
        cases.append((B, G * Hkv, Hkv, N, chunk, bool(rng.integers(0, 2)), int(rng.integers(1 << 30))))
    return cases


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk,with_s0,seed", _cases())
def test_prefill_random_shapes(la, B, Hq, Hkv, N, chunk, with_s0, seed):
    q, k, v = synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, seed)
    S0 = (torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(seed + 1)) / 128
          if with_s0 else torch.zeros(B, Hkv, 128, 128))
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy(), o_dtype=np.float32)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    o_plain = la.la_forward(qd, kd, vd, chunk=chunk) if not with_s0 else None
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    what = f"B{B} Hq{Hq}/Hkv{Hkv} N{N} chunk {chunk} S0 {with_s0}"
    assert_bf16_close(o.cpu(), ref_o, "O " + what)
    assert_f32_close(S.cpu(), ref_S, "final state " + what, tol=STATE_REL_L2)
    if o_plain is not None:
        assert torch.equal(o_plain, o), "la_forward vs la_forward_state from zero: " + what
