"""Sequence sharding, emulated on one GPU: a sequence cut into ragged
segments (one per would-be rank); each segment's K^T V, the prefix of the
segments before it, and the segment's prefill from that state, all through
the C ABI, against the fp64 oracle on the whole sequence."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import STATE_REL_L2, assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("B,Hq,Hkv,cuts,chunk,with_s0", [
    (2, 8, 2, [0, 400, 777, 1300, 1500], 64, True),
    (1, 4, 4, [0, 129, 1000], 128, False),
    (3, 6, 3, [0, 1, 65, 300], 64, True),
])
def test_sequence_sharding_emulated(la, B, Hq, Hkv, cuts, chunk, with_s0):
    N = cuts[-1]
    q, k, v = synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, seed=1500 + N)
    S0 = (torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(1501)) / 128
          if with_s0 else None)
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy() if with_s0 else None,
                                    o_dtype=np.float32)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    segs = list(zip(cuts[:-1], cuts[1:]))
    # each rank's segment state, stacked as the all-gather lays them out
    states = torch.stack([la.la_segment_state(kd[:, :, a:b].contiguous(),
                                              vd[:, :, a:b].contiguous(), chunk=chunk)
                          for a, b in segs])
    torch.cuda.synchronize()
    for r, (a, b) in enumerate(segs):
        ref = oracle.state_gemm(k[:, :, a:b], v[:, :, a:b])
        assert_f32_close(states[r].cpu(), ref, f"segment {r} state", tol=STATE_REL_L2)
    outs, S = [], None
    S0d = S0.to(DEV) if with_s0 else None
    for r, (a, b) in enumerate(segs):
        S = la.la_state_prefix(states, r, S0=S0d)
        outs.append(la.la_forward_state(*(t[:, :, a:b].contiguous() for t in (qd, kd, vd)), S=S,
                                        chunk=chunk))
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    assert_bf16_close(torch.cat(outs, dim=2).cpu(), ref_o, "O of the sharded sequence")
    assert_f32_close(S.cpu(), ref_S, "final state (last segment)", tol=STATE_REL_L2)


def test_state_prefix_is_exact_on_integers(la):
    """S0 + sum of the first r states, for small-integer states: exact in fp32."""
    g = torch.Generator().manual_seed(1600)
    states = torch.randint(-8, 9, (5, 2, 3, 128, 128), generator=g).float()
    S0 = torch.randint(-8, 9, (2, 3, 128, 128), generator=g).float()
    sd, s0d = states.to(DEV), S0.to(DEV)
    for r in range(5):
        got = la.la_state_prefix(sd, r, S0=s0d)
        want = S0 + states[:r].sum(0)
        assert torch.equal(got.cpu(), want)
    assert torch.equal(la.la_state_prefix(sd, 0).cpu(), torch.zeros_like(S0))
    with pytest.raises(la.LAError) as e:
        la.la_state_prefix(sd, 5)
    assert e.value.code == 1
