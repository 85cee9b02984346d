"""The library's calls are stream-ordered (workspace from the stream-ordered
pool, launches on the given stream), so they can be captured in a CUDA graph
and replayed: a prefill with a state and 8 decode steps, captured once,
replayed, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import STATE_REL_L2, assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("B,Hq,Hkv,N", [(1, 8, 2, 1000), (40, 16, 4, 64)])
def test_prefill_and_decode_steps_replay_from_a_cuda_graph(la, B, Hq, Hkv, N):
    steps = 8
    q, k, v = synth.random_qkv(B, Hq, Hkv, N, 128, torch.bfloat16, seed=1700 + N)
    toks = [synth.random_qkv(B, Hq, Hkv, 1, 128, torch.bfloat16, seed=1800 + i) for i in range(steps)]
    ref_o, ref_S = oracle.recurrent(q, k, v, o_dtype=np.float32)
    ref_steps = []
    S_ref = ref_S
    for tq, tk, tv in toks:
        o_t, S_ref = oracle.decode(S_ref, tq[:, :, 0].contiguous(), tk[:, :, 0].contiguous(),
                                   tv[:, :, 0].contiguous())
        ref_steps.append(o_t)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    td = [tuple(t[:, :, 0].contiguous().to(DEV) for t in tok) for tok in toks]
    S = torch.zeros(B, Hkv, 128, 128, dtype=torch.float32, device=DEV)
    o = torch.empty_like(qd)
    od = [torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=DEV) for _ in range(steps)]
    s = torch.cuda.Stream()

    def work():
        la.la_forward_state(qd, kd, vd, S=S, o=o, chunk=64, stream=s)
        for i, (tq, tk, tv) in enumerate(td):
            la.la_decode_step(S, tq, tk, tv, o=od[i], stream=s)

    with torch.cuda.stream(s):
        work()  # first calls outside capture (one-time setup of the library)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        work()
    for _ in range(2):  # replays start from a zero state
        S.zero_()
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert_bf16_close(o.cpu(), ref_o, "prefill O (graph replay)")
        for i in range(steps):
            assert_bf16_close(od[i].cpu(), ref_steps[i], f"decode step {i} (graph replay)")
        assert_f32_close(S.cpu(), S_ref, "state after the steps", tol=STATE_REL_L2)
    del g
    assert la.la_device_status()[1] == 0
