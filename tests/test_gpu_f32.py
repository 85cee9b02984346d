"""fp32 prefill (CUDA-core kernel) against the fp64 oracle at rel-L2 <= 1e-4."""
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_causal_f32_b1_h2_n1024_d64(la):
    w = synth.PR1_F32
    q, k, v = synth.prefill_inputs(w)
    ref_o, ref_S = oracle.quadratic(q, k, v), oracle.state(k, v)
    S = torch.zeros(1, 2, 64, 64, device=DEV)
    o = la.la_forward_f32(q.to(DEV), k.to(DEV), v.to(DEV), S=S, chunk=64)
    torch.cuda.synchronize()
    assert_f32_close(o.cpu(), ref_o, "O")
    assert_f32_close(S.cpu(), ref_S, "final state")


@pytest.mark.parametrize("B,Hq,Hkv,N,d,chunk", [
    (1, 1, 1, 1, 64, 64), (2, 4, 2, 333, 64, 128), (1, 6, 3, 200, 128, 64), (1, 2, 1, 129, 128, 128)])
def test_f32_shapes_with_state(la, B, Hq, Hkv, N, d, chunk):
    q, k, v = synth.random_qkv(B, Hq, Hkv, N, d, torch.float32, seed=N + d)
    S0 = torch.randn(B, Hkv, d, d, generator=torch.Generator().manual_seed(3)) / d
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy())
    S = S0.to(DEV)
    o = la.la_forward_f32(q.to(DEV), k.to(DEV), v.to(DEV), S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert_f32_close(o.cpu(), ref_o, "O")
    assert_f32_close(S.cpu(), ref_S, "final state")
