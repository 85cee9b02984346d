"""Pins for the fp64 backward oracle (no GPU).

The forward O and final state are linear in each of q, k, v and S0 taken on
its own (O = sum (q.k) v + q S0, S = S0 + sum k^T v).  So for the loss
L = <O, dO> + <S_final, dSf> a central difference with step 1 is the exact
partial derivative, and with small-integer inputs every sum is exact in fp64:
the finite-difference gradient of the FORWARD oracle must equal the backward
oracle bit for bit.  Planted mistakes in the backward code must break a pin.
"""
import os
import shutil
import tempfile

import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth


def _ints(rng, *shape, lo=-2, hi=3):
    return torch.tensor(rng.integers(lo, hi, size=shape).astype(np.float32))


def _loss(q, k, v, S0, dO, dSf):
    o, S = oracle.recurrent(q, k, v, S0=S0)
    return float(np.sum(o * dO.double().numpy()) + np.sum(S * dSf))


def _fd_gradients(q, k, v, S0, dO, dSf):
    """Central differences of the forward oracle, step 1 (exact: the loss is
    linear in each argument on its own)."""
    grads = []
    for which, x in (("q", q), ("k", k), ("v", v)):
        g = np.zeros(x.shape)
        flat = x.view(-1)
        for i in range(flat.numel()):
            old = float(flat[i])
            flat[i] = old + 1
            lp = _loss(q, k, v, S0, dO, dSf)
            flat[i] = old - 1
            lm = _loss(q, k, v, S0, dO, dSf)
            flat[i] = old
            g.reshape(-1)[i] = (lp - lm) / 2
        grads.append(g)
    gS = np.zeros(S0.shape)
    for i in range(S0.size):
        old = S0.reshape(-1)[i]
        S0.reshape(-1)[i] = old + 1
        lp = _loss(q, k, v, S0, dO, dSf)
        S0.reshape(-1)[i] = old - 1
        lm = _loss(q, k, v, S0, dO, dSf)
        S0.reshape(-1)[i] = old
        gS.reshape(-1)[i] = (lp - lm) / 2
    grads.append(gS)
    return grads


def pin_finite_differences_exact():
    rng = np.random.default_rng(40)
    for (B, Hq, Hkv, N, d) in [(1, 2, 1, 5, 3), (2, 1, 1, 4, 2), (1, 3, 3, 3, 2)]:
        q, k, v = _ints(rng, B, Hq, N, d), _ints(rng, B, Hkv, N, d), _ints(rng, B, Hkv, N, d)
        dO = _ints(rng, B, Hq, N, d)
        S0 = rng.integers(-2, 3, size=(B, Hkv, d, d)).astype(np.float64)
        dSf = rng.integers(-2, 3, size=(B, Hkv, d, d)).astype(np.float64)
        want = _fd_gradients(q, k, v, S0, dO, dSf)
        for form in ("quadratic", "recurrent"):
            got = oracle.backward(q, k, v, dO, S0=S0, dSf=dSf, form=form)
            for name, g, w in zip(("dq", "dk", "dv", "dS0"), got, want):
                assert np.array_equal(g, w), (form, name, B, Hq, Hkv, N, d)


def pin_forms_agree():
    for (B, Hq, Hkv, N, d, seed) in [(1, 4, 2, 37, 8, 41), (2, 3, 1, 20, 4, 42), (1, 1, 1, 1, 5, 43)]:
        q, k, v = synth.random_qkv(B, Hq, Hkv, N, d, torch.float32, seed)
        dO = synth.random_qkv(B, Hq, Hq, N, d, torch.float32, seed + 100)[0]
        S0 = np.random.default_rng(seed).standard_normal((B, Hkv, d, d))
        dSf = np.random.default_rng(seed + 1).standard_normal((B, Hkv, d, d))
        a = oracle.backward(q, k, v, dO, S0=S0, dSf=dSf, form="quadratic")
        b = oracle.backward(q, k, v, dO, S0=S0, dSf=dSf, form="recurrent")
        for x, y in zip(a, b):
            assert np.linalg.norm(x - y) <= 1e-12 * max(np.linalg.norm(x), 1e-300)


def pin_dq_is_forward_with_swapped_roles():
    # dq_t = do_t S0^T + sum_{s<=t} (do_t . v_s) k_s: the forward oracle with
    # queries dO, keys V, values K and initial state S0^T.
    q, k, v = synth.random_qkv(1, 4, 2, 29, 8, torch.float32, 44)
    dO = synth.random_qkv(1, 4, 4, 29, 8, torch.float32, 45)[0]
    S0 = np.random.default_rng(46).standard_normal((1, 2, 8, 8))
    dq = oracle.backward(q, k, v, dO, S0=S0, form="quadratic")[0]
    fwd, _ = oracle.recurrent(dO, v, k, S0=np.swapaxes(S0, -1, -2))
    assert np.linalg.norm(dq - fwd) <= 1e-12 * np.linalg.norm(fwd)


def pin_no_state_gradient_defaults():
    # dSf = None is dSf = 0 and S0 = None is S0 = 0
    q, k, v = synth.random_qkv(1, 2, 1, 11, 4, torch.float32, 47)
    dO = synth.random_qkv(1, 2, 2, 11, 4, torch.float32, 48)[0]
    a = oracle.backward(q, k, v, dO)
    b = oracle.backward(q, k, v, dO, S0=np.zeros((1, 1, 4, 4)), dSf=np.zeros((1, 1, 4, 4)))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


PINS = [pin_finite_differences_exact, pin_forms_agree, pin_dq_is_forward_with_swapped_roles,
        pin_no_state_gradient_defaults]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


MUTANTS = [
    ("dk-strict-causal", "      for (int64_t t = s; t < N; ++t) {", "      for (int64_t t = s + 1; t < N; ++t) {"),
    ("dq-drops-diagonal", "      for (int64_t s = 0; s <= t; ++s) {\n        double a = 0.0;\n        for (int64_t j = 0; j < d; ++j)\n          a += elem(J->dO",
     "      for (int64_t s = 0; s < t; ++s) {\n        double a = 0.0;\n        for (int64_t j = 0; j < d; ++j)\n          a += elem(J->dO"),
    ("dsf-untransposed", "a += elem(J->v, kb + s * d + j, J->dtype) * dSf[i * d + j]; /* (v dSf^T)_i */",
     "a += elem(J->v, kb + s * d + j, J->dtype) * dSf[j * d + i]; /* (v dSf^T)_i */"),
    ("dq-s0-untransposed", "a += elem(J->dO, qb + t * d + j, J->dtype) * S0[i * d + j];",
     "a += elem(J->dO, qb + t * d + j, J->dtype) * S0[j * d + i];"),
    ("reverse-read-before-update",
     "        a += vt[j] * St[i * d + j]; /* (v G^T)_i */",
     "        a += vt[j] * (St[i * d + j] - elem(J->q, (b * J->Hq + g * G) * N * d + s * d + i, J->dtype) * elem(J->dO, (b * J->Hq + g * G) * N * d + s * d + j, J->dtype)); /* (v G^T)_i */"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistakes(name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "la_oracle.c")).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    tmp = tempfile.mkdtemp(prefix="la_bmut_")
    try:
        path = os.path.join(tmp, "mut.c")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        so = oracle.build(path, os.path.join(tmp, "mut.so"))
        saved = oracle._lib
        oracle._lib = oracle.load(so)
        failed = []
        try:
            for pin in PINS:
                try:
                    pin()
                except (AssertionError, ValueError):
                    failed.append(pin.__name__)
        finally:
            oracle._lib = saved
        assert failed, f"mutant {name} passed every pin"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
