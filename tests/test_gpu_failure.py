"""Failure detection without a GPU fault: a bounded device wait on a flag that
nothing sets runs out, records the timeout bit, and the context stays usable."""
import pytest
import torch

from linear_attention_11_b200 import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports(la):
    la.la_device_status(clear=True)
    la.api.la_selftest_wait(50_000_000)  # 50 ms of device time
    code, flags = la.la_device_status(clear=True)
    assert code == 4 and flags & 1
    # cleared, and the device still runs work
    code, flags = la.la_device_status(clear=True)
    assert code == 0 and flags == 0
    q, k, v = (t.cuda() for t in synth.random_qkv(1, 2, 2, 256, 128, torch.bfloat16, 1))
    o = la.la_forward(q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert la.la_device_status()[0] == 0
