"""Comparison helpers shared by the GPU parity tests.

Tolerances: fp32 inputs, rel-L2 <= 1e-4; bf16 inputs with fp32 accumulation,
rel-L2 <= 1e-2 and max-abs <= 2e-2 * max|reference| over the whole tensor.
"""
import numpy as np
import torch

F32_REL_L2 = 1e-4
BF16_REL_L2 = 1e-2
BF16_MAX_ABS = 2e-2
# The fp32 state of the bf16 path is a sum of up to 2^20 exact bf16 products
# in fp32 (tensor-core accumulation inside spans, then the span scan).  Its
# rounding error grows with the number of sequential fp32 additions (about
# tiles-per-span + spans, a few hundred at 1M tokens): u_fp32 * 300 ~ 2e-5.
# The state is held to 1e-4, a hundred times tighter than the 1e-2 allowed
# for bf16-input results.
STATE_REL_L2 = 1e-4


def as64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().float().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def errors(got, ref):
    g, r = as64(got), as64(ref)
    diff = g - r
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(r), 1e-300))
    mx = float(np.max(np.abs(diff))) if diff.size else 0.0
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    return rel, mx, scale


def assert_bf16_close(got, ref, what=""):
    rel, mx, scale = errors(got, ref)
    assert np.all(np.isfinite(as64(got))), f"{what}: non-finite values"
    assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
    assert mx <= BF16_MAX_ABS * scale, f"{what}: max-abs {mx:.3e} > {BF16_MAX_ABS} * {scale:.3e}"
    return rel, mx


def assert_f32_close(got, ref, what="", tol=F32_REL_L2):
    rel, mx, scale = errors(got, ref)
    assert np.all(np.isfinite(as64(got))), f"{what}: non-finite values"
    assert rel <= tol, f"{what}: rel-L2 {rel:.3e} > {tol}"
    return rel


class RunningBF16Check:
    """The bf16 bounds over a tensor compared piece by piece: rel-L2 and
    max-abs are accumulated over all pieces and checked once, so the bound
    is the same as for the whole tensor at once."""

    def __init__(self):
        self.d2 = self.r2 = self.mx = self.scale = 0.0
        self.finite = True
        self.count = 0

    def update(self, got, ref):
        g, r = as64(got), as64(ref)
        diff = g - r
        self.finite &= bool(np.all(np.isfinite(g)))
        self.d2 += float(np.sum(diff * diff))
        self.r2 += float(np.sum(r * r))
        if diff.size:
            self.mx = max(self.mx, float(np.max(np.abs(diff))))
            self.scale = max(self.scale, float(np.max(np.abs(r))))
        self.count += diff.size

    def check(self, what=""):
        rel = float(np.sqrt(self.d2) / max(np.sqrt(self.r2), 1e-300))
        assert self.finite, f"{what}: non-finite values"
        assert rel <= BF16_REL_L2, f"{what}: rel-L2 {rel:.3e} > {BF16_REL_L2}"
        assert self.mx <= BF16_MAX_ABS * self.scale, \
            f"{what}: max-abs {self.mx:.3e} > {BF16_MAX_ABS} * {self.scale:.3e}"
        return rel, self.mx
