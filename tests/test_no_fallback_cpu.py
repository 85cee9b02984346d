"""The product path has no CPU fallback: without the built CUDA library, or
with tensors that are not on a CUDA device, calls raise instead of computing
anything on the host.  Run in fresh interpreters so that a library loaded by
other tests cannot stand in."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code):
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                          timeout=300, cwd=ROOT)


def test_missing_library_raises():
    r = _run("import linear_attention_11_b200.api as api\n"
             "try:\n"
             "    api.load_library('/nonexistent/liblightning_b200.so')\n"
             "except RuntimeError as e:\n"
             "    print('raised:', e)\n")
    assert r.returncode == 0, r.stderr[-2000:]
    assert "raised: CUDA library not built" in r.stdout


def test_host_tensors_do_not_compute():
    r = _run("import torch, linear_attention_11_b200 as la\n"
             "from linear_attention_11_b200 import synth\n"
             "q, k, v = synth.random_qkv(1, 2, 2, 64, 128, torch.bfloat16, 0)\n"
             "try:\n"
             "    la.la_forward(q, k, v, chunk=64)\n"
             "    print('computed')\n"
             "except Exception as e:\n"
             "    print('raised:', type(e).__name__)\n")
    assert r.returncode == 0, r.stderr[-2000:]
    assert "raised:" in r.stdout and "computed" not in r.stdout
