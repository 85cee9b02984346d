"""Pins for the fp64 CPU oracle (no GPU).

Each check ties the oracle to something other than its own code: hand-worked
fixtures, closed forms, a library GEMM, invariants of the definition, and an
independent chunked restatement of the pages' sketch.  ``test_planted_mistakes``
compiles mutated copies of the oracle source and requires every mutation to be
caught by at least one of these checks.
"""
import json
import os
import shutil
import tempfile

import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _t(x, shape):
    return torch.tensor(np.asarray(x, dtype=np.float32).reshape(shape))


def _rand(B, Hq, Hkv, N, d, seed, dtype=torch.float32):
    return synth.random_qkv(B, Hq, Hkv, N, d, dtype, seed)


def _f64(x):
    return x.double().numpy()


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- the pins
# Each pin is a plain function so that the planted-mistake test can run the
# whole set against a mutated oracle.

def pin_hand_mha():
    g = _load("hand_mha_n3_d2.json")
    q, k, v = (_t(g[n], (1, 1, 3, 2)) for n in ("q", "k", "v"))
    want_o, want_s = np.array(g["O"], float), np.array(g["S"], float)
    o = oracle.quadratic(q, k, v)[0, 0]
    assert np.array_equal(o, want_o), o
    o_r, S = oracle.recurrent(q, k, v)
    assert np.array_equal(o_r[0, 0], want_o), o_r
    assert np.array_equal(S[0, 0], want_s), S
    assert np.array_equal(oracle.state(k, v)[0, 0], want_s)
    r = oracle.rows(q, k, v, [(0, 0, 2), (0, 0, 0)])
    assert np.array_equal(r, want_o[[2, 0]])


def pin_hand_gqa():
    g = _load("hand_gqa_n2_d2.json")
    q = _t(g["q"], (1, 2, 2, 2))
    k, v = _t(g["k"], (1, 1, 2, 2)), _t(g["v"], (1, 1, 2, 2))
    want = np.array(g["O"], float)
    assert np.array_equal(oracle.quadratic(q, k, v)[0], want)
    o_r, S = oracle.recurrent(q, k, v)
    assert np.array_equal(o_r[0], want)
    assert np.array_equal(S[0, 0], np.array(g["S"], float))


def pin_hand_decode():
    g = _load("hand_decode_d2.json")
    S0 = np.array(g["S0"], float).reshape(1, 1, 2, 2)
    q, k, v = _t(g["q"], (1, 1, 2)), _t(g["k"], (1, 1, 2)), _t(g["v"], (1, 1, 2))
    o, S = oracle.decode(S0, q, k, v)
    assert np.array_equal(o[0, 0], np.array(g["o"], float)), o
    assert np.array_equal(S[0, 0], np.array(g["S"], float)), S


def pin_d1_prefix_sum():
    # d = 1: O_t = q_t * sum_{s<=t} k_s v_s, an inclusive prefix sum.
    q, k, v = _rand(2, 3, 3, 37, 1, seed=11)
    want = _f64(q) * np.cumsum(_f64(k) * _f64(v), axis=2)
    assert _rel(oracle.quadratic(q, k, v), want) < 1e-13
    assert _rel(oracle.recurrent(q, k, v)[0], want) < 1e-13


def pin_state_is_ktv():
    # S = K^T V as a library GEMM (numpy einsum over the sequence axis).
    q, k, v = _rand(2, 4, 2, 53, 8, seed=12)
    want = np.einsum("bgsi,bgsj->bgij", _f64(k), _f64(v))
    assert _rel(oracle.state(k, v), want) < 1e-13
    assert _rel(oracle.recurrent(q, k, v, want_o=False)[1], want) < 1e-13
    kb, vb = k.bfloat16(), v.bfloat16()
    wantb = np.einsum("bgsi,bgsj->bgij", _f64(kb), _f64(vb))
    assert _rel(oracle.state_gemm(kb, vb), wantb) < 1e-13
    assert _rel(oracle.state(kb, vb), wantb) < 1e-13


def pin_last_row_noncausal():
    # The last causal row sees every token: it equals the non-causal form
    # q_{N-1} (K^T V) (section 2.2 of the page-4 notes, with phi = identity).
    q, k, v = _rand(1, 4, 2, 41, 8, seed=13)
    S = np.einsum("bgsi,bgsj->bgij", _f64(k), _f64(v))
    G = 2
    want = np.stack([_f64(q)[0, h, -1] @ S[0, h // G] for h in range(4)])
    assert _rel(oracle.quadratic(q, k, v)[0, :, -1], want) < 1e-13
    assert _rel(oracle.recurrent(q, k, v)[0][0, :, -1], want) < 1e-13


def pin_first_row_single_token():
    # Row 0 sees only token 0: (q0.k0) v0.
    q, k, v = _rand(1, 2, 1, 9, 4, seed=14)
    qa, ka, va = _f64(q)[0], _f64(k)[0, 0], _f64(v)[0, 0]
    want = np.stack([(qa[h, 0] @ ka[0]) * va[0] for h in range(2)])
    assert _rel(oracle.quadratic(q, k, v)[0, :, 0], want) < 1e-14


def pin_forms_agree():
    for (B, Hq, Hkv, N, d, seed) in [(1, 1, 1, 1, 3, 21), (2, 4, 2, 67, 16, 22), (1, 6, 3, 130, 8, 23)]:
        q, k, v = _rand(B, Hq, Hkv, N, d, seed)
        a = oracle.quadratic(q, k, v)
        b, _ = oracle.recurrent(q, k, v)
        assert _rel(b, a) < 1e-12, (B, Hq, Hkv, N, d)


def pin_gqa_is_repeated_mha():
    q, k, v = _rand(2, 6, 2, 33, 8, seed=24)
    G = 3
    kr, vr = k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    assert _rel(oracle.quadratic(q, k, v), oracle.quadratic(q, kr, vr)) < 1e-15
    o1, S1 = oracle.recurrent(q, k, v)
    o2, S2 = oracle.recurrent(q, kr, vr)
    assert _rel(o1, o2) < 1e-15
    assert _rel(S2[:, ::G], S1) < 1e-15


def pin_bilinear():
    # Small-integer inputs keep every input sum exact, so the identities hold
    # to fp64 rounding.
    rng = np.random.default_rng(25)

    def ints(*shape):
        return torch.tensor(rng.integers(-3, 4, size=shape).astype(np.float32))

    q, k, v = ints(1, 2, 29, 8), ints(1, 2, 29, 8), ints(1, 2, 29, 8)
    q2, v2 = ints(1, 2, 29, 8), ints(1, 2, 29, 8)
    base = oracle.quadratic(q, k, v)
    assert _rel(oracle.quadratic(q * 2, k, v), 2 * base) < 1e-15
    assert _rel(oracle.quadratic(q, k, v * -4), -4 * base) < 1e-15
    # additive in v and in q
    assert _rel(oracle.quadratic(q, k, v + v2), base + oracle.quadratic(q, k, v2)) < 1e-14
    assert _rel(oracle.quadratic(q + q2, k, v), base + oracle.quadratic(q2, k, v)) < 1e-14


def _chunked_numpy(q, k, v, C):
    """The chunkwise scheme of the page-5 sketch, restated in numpy fp64.

    Per block: inter = Q_b S; intra = tril(Q_b K_b^T) V_b; O_b = inter + intra;
    then S += K_b^T V_b.  Query head h reads kv head h // G."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(Hq):
            S = np.zeros((d, d))
            for s0 in range(0, N, C):
                s1 = min(s0 + C, N)
                qb, kb, vb = q[b, h, s0:s1], k[b, h // G, s0:s1], v[b, h // G, s0:s1]
                out[b, h, s0:s1] = qb @ S + np.tril(qb @ kb.T) @ vb
                S = S + kb.T @ vb
    return out


def pin_chunk_independence():
    q, k, v = _rand(1, 4, 2, 100, 8, seed=27)
    o = oracle.quadratic(q, k, v)
    for C in (1, 7, 32, 64, 100, 128):
        assert _rel(_chunked_numpy(q, k, v, C), o) < 1e-12, C


def pin_update_first_tile_differs():
    # Negative pin: the tile sketch of the page-4 notes (section 2.3) updates
    # the state with the whole tile before reading it, which lets a token see
    # later tokens of its own tile.  With tile 1 it is the causal result; with
    # any larger tile it must differ from the oracle.
    q, k, v = _rand(1, 2, 2, 64, 8, seed=28)
    qa, ka, va = _f64(q), _f64(k), _f64(v)
    o = oracle.quadratic(q, k, v)

    def update_first(T):
        out = np.zeros_like(qa)
        for h in range(2):
            S = np.zeros((8, 8))
            for s0 in range(0, 64, T):
                S = S + ka[0, h, s0:s0 + T].T @ va[0, h, s0:s0 + T]
                out[0, h, s0:s0 + T] = qa[0, h, s0:s0 + T] @ S
        return out

    assert _rel(update_first(1), o) < 1e-12
    for T in (2, 16, 64):
        assert _rel(update_first(T), o) > 1e-2, T


def pin_rows_match_full():
    q, k, v = _rand(2, 4, 2, 70, 16, seed=29)
    full = oracle.quadratic(q, k, v)
    sel = [(0, 0, 0), (1, 3, 69), (0, 2, 31), (1, 1, 32), (0, 3, 64)]
    got = oracle.rows(q, k, v, sel)
    want = np.stack([full[b, h, t] for b, h, t in sel])
    assert np.array_equal(got, want)


def pin_initial_state_and_resume():
    q, k, v = _rand(1, 4, 2, 60, 8, seed=30)
    S0 = np.random.default_rng(0).standard_normal((1, 2, 8, 8))
    o0, Sz = oracle.recurrent(q, k, v)
    o1, S1 = oracle.recurrent(q, k, v, S0=S0)
    # The initial state adds q_t S0 to every row and S0 to the final state.
    add = np.einsum("bhti,bhij->bhtj", _f64(q), np.repeat(S0, 2, axis=1))
    assert _rel(o1, o0 + add) < 1e-12
    assert _rel(S1, Sz + S0) < 1e-13
    # Split at 23 and resume from the carried state.
    oa, Sa = oracle.recurrent(q[:, :, :23], k[:, :, :23], v[:, :, :23], S0=S0)
    ob, Sb = oracle.recurrent(q[:, :, 23:], k[:, :, 23:], v[:, :, 23:], S0=Sa)
    assert _rel(np.concatenate([oa, ob], axis=2), o1) < 1e-13
    assert _rel(Sb, S1) < 1e-13


def pin_decode_matches_prefill():
    q, k, v = _rand(2, 4, 2, 12, 8, seed=31)
    o_ref, S_ref = oracle.recurrent(q, k, v)
    S = np.zeros((2, 2, 8, 8))
    for t in range(12):
        o, S = oracle.decode(S, q[:, :, t], k[:, :, t], v[:, :, t])
        assert _rel(o, o_ref[:, :, t]) < 1e-13, t
    assert _rel(S, S_ref) < 1e-13


def pin_bf16_widening():
    # bf16 inputs are widened exactly: the result equals the fp32 path on the
    # same (bf16-representable) values.
    q, k, v = _rand(1, 2, 1, 40, 8, seed=32, dtype=torch.bfloat16)
    a = oracle.quadratic(q, k, v)
    b = oracle.quadratic(q.float(), k.float(), v.float())
    assert np.array_equal(a, b)
    o, S = oracle.recurrent(q, k, v)
    o2, S2 = oracle.recurrent(q.float(), k.float(), v.float())
    assert np.array_equal(o, o2) and np.array_equal(S, S2)


PINS = [pin_hand_mha, pin_hand_gqa, pin_hand_decode, pin_d1_prefix_sum, pin_state_is_ktv,
        pin_last_row_noncausal, pin_first_row_single_token, pin_forms_agree,
        pin_gqa_is_repeated_mha, pin_bilinear, pin_chunk_independence,
        pin_update_first_tile_differs, pin_rows_match_full, pin_initial_state_and_resume,
        pin_decode_matches_prefill, pin_bf16_widening]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_thread_count_does_not_change_results():
    q, k, v = _rand(2, 4, 2, 50, 8, seed=33)
    assert np.array_equal(oracle.quadratic(q, k, v, nthreads=1), oracle.quadratic(q, k, v, nthreads=5))
    a = oracle.recurrent(q, k, v, nthreads=1)
    b = oracle.recurrent(q, k, v, nthreads=3)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_float32_output_option():
    q, k, v = _rand(1, 2, 2, 30, 8, seed=34)
    o64, S = oracle.recurrent(q, k, v)
    o32, S2 = oracle.recurrent(q, k, v, o_dtype=np.float32)
    assert o32.dtype == np.float32
    assert np.array_equal(o32, o64.astype(np.float32)) and np.array_equal(S, S2)


def test_rejects_bad_arguments():
    q, k, v = _rand(1, 3, 2, 5, 4, seed=35)
    with pytest.raises(ValueError):
        oracle.quadratic(q, k, v)  # Hq % Hkv != 0
    q, k, v = _rand(1, 2, 2, 5, 4, seed=35)
    with pytest.raises(ValueError):
        oracle.rows(q, k, v, [(0, 0, 5)])  # t out of range


# ------------------------------------------------ planted mistakes
# (name, exact source text, replacement).  Each mutant is a plausible slip:
# a dropped diagonal, a transposed operand, a wrong head map, a wrong
# widening, a read placed before the update.
MUTANTS = [
    ("drop-diagonal-quadratic", "for (int64_t s = 0; s <= t; ++s) { /* causal",
     "for (int64_t s = 0; s < t; ++s) { /* causal"),
    ("drop-diagonal-rows", "  for (int64_t s = 0; s <= t; ++s) {\n    double a = 0.0;",
     "  for (int64_t s = 0; s < t; ++s) {\n    double a = 0.0;"),
    ("gqa-map-modulo", "const int64_t b = unit / J->Hq, h = unit % J->Hq, g = h / G;",
     "const int64_t b = unit / J->Hq, h = unit % J->Hq, g = h % J->Hkv;"),
    ("transposed-state-update", "for (int64_t j = 0; j < d; ++j) S[i * d + j] += kt[i] * vt[j];",
     "for (int64_t j = 0; j < d; ++j) S[i * d + j] += kt[j] * vt[i];"),
    ("transposed-state-read", "for (int64_t j = 0; j < d; ++j) ot[j] += qi * S[i * d + j];",
     "for (int64_t j = 0; j < d; ++j) ot[j] += qi * S[j * d + i];"),
    ("bf16-widening-shift", "((uint32_t)((const uint16_t *)p)[i]) << 16;",
     "((uint32_t)((const uint16_t *)p)[i]) << 15;"),
    ("decode-transposed", "for (int64_t j = 0; j < d; ++j) Sg[i * d + j] += ki * elem(J->v, kv + j, J->dtype);",
     "for (int64_t j = 0; j < d; ++j) Sg[j * d + i] += ki * elem(J->v, kv + j, J->dtype);"),
    ("state-q-for-k", "const double ki = elem(J->k, kbase + s * d + i, J->dtype);",
     "const double ki = elem(J->v, kbase + s * d + i, J->dtype);"),
    ("recurrent-read-before-update",
     "    for (int64_t i = 0; i < d; ++i) /* S += k_t^T v_t */\n"
     "      for (int64_t j = 0; j < d; ++j) S[i * d + j] += kt[i] * vt[j];\n"
     "    if (!J->o && !J->o32) continue;\n",
     "    if (t > 0) for (int64_t i = 0; i < d; ++i)\n"
     "      for (int64_t j = 0; j < d; ++j) S[i * d + j] += kt[i] * vt[j] * 0.0;\n"
     "    if (!J->o && !J->o32) { for (int64_t i = 0; i < d; ++i) for (int64_t j = 0; j < d; ++j) S[i * d + j] += kt[i] * vt[j]; continue; }\n"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistakes(name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "la_oracle.c")).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    tmp = tempfile.mkdtemp(prefix="la_mut_")
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
