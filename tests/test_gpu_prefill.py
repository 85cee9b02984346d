"""bf16 prefill on the GPU (tcgen05 kernels, called through the C ABI) against
the fp64 oracle.

Stage by stage first (span states, scan, main pass), then whole calls on small
ragged shapes that span several tiles, then the full-size workloads in the
launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_11_b200 import synth

from _compare import (STATE_REL_L2, RunningBF16Check, assert_bf16_close, assert_f32_close,
                      errors)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _qkv(B, Hq, Hkv, N, seed, d=128):
    return synth.random_qkv(B, Hq, Hkv, N, d, torch.bfloat16, seed)


def _cuda(*ts):
    return [t.to(DEV) for t in ts]


def _span_bounds(plan, j):
    b = (j * plan.tiles_total) // plan.nspan * plan.tile
    e = ((j + 1) * plan.tiles_total) // plan.nspan * plan.tile
    return b, e


@pytest.mark.parametrize("Hq,Hkv,N,chunk", [(2, 2, 700, 64), (4, 2, 1000, 64), (4, 1, 520, 128)])
def test_span_states_and_scan(la, Hq, Hkv, N, chunk):
    B = 2
    q, k, v = _qkv(B, Hq, Hkv, N, seed=100 + N)
    kd, vd = _cuda(k, v)
    for nspan in (1, 3, None):
        plan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk)
        if nspan is not None:
            plan.nspan = min(nspan, plan.tiles_total)
            plan.workspace_bytes = B * Hkv * plan.nspan * 128 * 128 * 4
        ws = torch.empty(B, Hkv, plan.nspan, 128, 128, dtype=torch.float32, device=DEV)
        la.api.la_prefill_span_states(kd, vd, plan, ws)
        torch.cuda.synchronize()
        got = ws.cpu()
        for j in range(plan.nspan):
            b0, b1 = _span_bounds(plan, j)
            ref = oracle.state_gemm(k[:, :, b0:min(b1, N)], v[:, :, b0:min(b1, N)])
            assert_f32_close(got[:, :, j], ref, f"span state {j}/{plan.nspan}", tol=STATE_REL_L2)
        # scan with an initial state
        S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(5))
        S = S0.to(DEV)
        la.api.la_prefill_scan(ws, S, plan, B, Hkv, 128)
        torch.cuda.synchronize()
        got = ws.cpu()
        for j in range(plan.nspan):
            b0, _ = _span_bounds(plan, j)
            ref = S0.double().numpy() + (oracle.state_gemm(k[:, :, :b0], v[:, :, :b0]) if b0 else 0)
            assert_f32_close(got[:, :, j], ref, f"entering state {j}", tol=STATE_REL_L2)
        ref = S0.double().numpy() + oracle.state_gemm(k, v)
        assert_f32_close(S.cpu(), ref, "final state", tol=STATE_REL_L2)


SMALL = [
    # B, Hq, Hkv, N, chunk  -- tile = 64 needs an even group; other cases use 128-token tiles
    (1, 1, 1, 1, 64),
    (1, 2, 2, 63, 64),
    (1, 2, 1, 64, 64),
    (1, 2, 1, 65, 64),
    (2, 2, 2, 300, 64),      # single-head groups at chunk 64: two chunks per tile
    (2, 4, 2, 777, 64),      # two query heads per tile, ragged tail
    (1, 8, 2, 1000, 64),     # GQA 4:1
    (1, 8, 2, 1000, 128),
    (1, 3, 1, 385, 64),      # odd group -> 128-token tiles
    (3, 6, 3, 129, 128),
    (1, 4, 4, 2048, 128),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", SMALL)
def test_forward_small(la, B, Hq, Hkv, N, chunk):
    q, k, v = _qkv(B, Hq, Hkv, N, seed=N * 7 + Hq)
    ref = oracle.quadratic(q, k, v)
    qd, kd, vd = _cuda(q, k, v)
    o = la.la_forward(qd, kd, vd, chunk=chunk)
    torch.cuda.synchronize()
    assert_bf16_close(o.cpu(), ref, f"O {B}x{Hq}/{Hkv}x{N} chunk {chunk}")
    assert la.la_device_status()[1] == 0


@pytest.mark.parametrize("nspan", [1, 2, 5, 16])
def test_span_count_does_not_change_result(la, nspan):
    B, Hq, Hkv, N, chunk = 1, 4, 2, 1024, 64
    q, k, v = _qkv(B, Hq, Hkv, N, seed=31)
    ref = oracle.quadratic(q, k, v)
    qd, kd, vd = _cuda(q, k, v)
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk)
    plan.nspan = nspan
    plan.workspace_bytes = B * Hkv * nspan * 128 * 128 * 4
    ws = torch.empty(plan.workspace_bytes // 4, dtype=torch.float32, device=DEV)
    o = torch.empty_like(qd)
    la.api.la_prefill_span_states(kd, vd, plan, ws)
    la.api.la_prefill_scan(ws, None, plan, B, Hkv, 128)
    la.api.la_prefill_main(qd, kd, vd, o, ws, plan)
    torch.cuda.synchronize()
    assert_bf16_close(o.cpu(), ref, f"nspan={nspan}")


def test_state_in_out_and_resume(la):
    B, Hq, Hkv, N, chunk = 2, 4, 2, 900, 64
    q, k, v = _qkv(B, Hq, Hkv, N, seed=41)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(42)) / 128
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy())
    qd, kd, vd = _cuda(q, k, v)
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert_bf16_close(o.cpu(), ref_o, "O with initial state")
    assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)
    # the same sequence in two pieces, carrying the state
    cut = 333
    S2 = S0.to(DEV)
    o1 = la.la_forward_state(*(t[:, :, :cut].contiguous() for t in (qd, kd, vd)), S=S2, chunk=chunk)
    o2 = la.la_forward_state(*(t[:, :, cut:].contiguous() for t in (qd, kd, vd)), S=S2, chunk=chunk)
    torch.cuda.synchronize()
    assert_bf16_close(torch.cat([o1, o2], dim=2).cpu(), ref_o, "resumed O")
    assert_f32_close(S2.cpu(), ref_S, "resumed final state", tol=STATE_REL_L2)


def test_chunk_sizes_agree(la):
    q, k, v = _cuda(*_qkv(1, 8, 2, 1500, seed=51))
    a = la.la_forward(q, k, v, chunk=64)
    b = la.la_forward(q, k, v, chunk=128)
    torch.cuda.synchronize()
    assert_bf16_close(a.cpu(), b.cpu(), "chunk 64 vs 128")


def test_forward_ws_and_workspace_errors(la):
    B, Hq, Hkv, N = 1, 4, 2, 500
    q, k, v = _cuda(*_qkv(B, Hq, Hkv, N, seed=61))
    nbytes = la.api.la_forward_workspace_bytes(B, Hq, Hkv, N, 128, 64)
    assert nbytes > 0
    ws = torch.empty(nbytes // 4, dtype=torch.float32, device=DEV)
    o = torch.empty_like(q)
    la.api.la_forward_ws(q, k, v, o, None, ws, chunk=64)
    ref = la.la_forward(q, k, v, chunk=64)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)
    small = torch.empty(nbytes // 8, dtype=torch.float32, device=DEV)
    with pytest.raises(la.LAError) as e:
        la.api.la_forward_ws(q, k, v, o, None, small, chunk=64)
    assert e.value.code == 5


def test_argument_errors_on_device(la):
    q, k, v = _cuda(*_qkv(1, 2, 2, 64, seed=71))
    with pytest.raises(la.LAError) as e:
        la.la_forward(q, k, v, o=q)  # output aliases an input
    assert e.value.code == 1
    with pytest.raises(la.LAError) as e:
        la.la_forward(q, k, v, chunk=32)
    assert e.value.code == 2
    q64 = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(la.LAError) as e:
        la.la_forward(q64, q64.clone(), q64.clone())
    assert e.value.code == 2
    raw = la.api.load_library()
    base = torch.zeros(1 << 16, dtype=torch.bfloat16, device=DEV)
    mis = base.data_ptr() + 2  # not 16-byte aligned
    rc = raw.la_forward(mis, k.data_ptr(), v.data_ptr(), base.data_ptr() + 4096 * 2, 1, 2, 2, 64,
                        128, 64, None)
    assert rc == 1


# ------------------------------------------------------------------ full size
def _full(la, w, chunk):
    q, k, v = synth.prefill_inputs(w)
    qd, kd, vd = _cuda(q, k, v)
    S = torch.zeros(w.B, w.Hkv, 128, 128, dtype=torch.float32, device=DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    oc = o.cpu()
    del o, qd, kd, vd
    ref_o, ref_S = oracle.recurrent(q, k, v, o_dtype=np.float32)
    assert_bf16_close(oc, ref_o, f"{w.name} chunk {chunk}")
    assert_f32_close(S.cpu(), ref_S, f"{w.name} final state", tol=STATE_REL_L2)


def test_full_mha_8k(la):
    _full(la, synth.MHA_8K, 64)


@pytest.mark.parametrize("chunk", [64, 128])
def test_full_gqa_32k(la, chunk):
    _full(la, synth.GQA_32K, chunk)


def _boundary_rows(la, w, chunk, count, seed=0):
    """Rows t at every place a GPU schedule changes hands -- the first and
    last tokens, both sides of chunk boundaries near the start, middle and
    end, and both sides of every span boundary of the plan -- plus random
    rows, at least `count` in all."""
    N = w.N
    plan = la.api.la_prefill_plan(w.B, w.Hq, w.Hkv, N, w.d, chunk)
    ts = {0, 1, chunk - 1, chunk, chunk + 1, 2 * chunk - 1, 2 * chunk, N // 2 - 1, N // 2,
          N - chunk - 1, N - chunk, N - 1}
    for j in range(1, plan.nspan):
        b, _ = _span_bounds(plan, j)
        ts.update({b - 1, b})
    rng = np.random.default_rng(seed)
    while len(ts) < count:
        ts.add(int(rng.integers(0, N)))
    ts = sorted(t for t in ts if 0 <= t < N)
    return [(int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq)), t) for t in ts]


def test_full_long_1m(la):
    """All 8 x 2^20 output rows against the token recurrence (run in pieces of
    2^17 tokens, each starting from the fp64 state the previous piece ended
    with, which is the same recurrence), the final state against the
    recurrence and K^T V, and >= 64 rows at chunk and span boundaries
    against the masked quadratic sum."""
    w, chunk = synth.LONG_1M, 128
    q, k, v = synth.prefill_inputs(w)
    qd, kd, vd = _cuda(q, k, v)
    S = torch.zeros(w.B, w.Hkv, 128, 128, dtype=torch.float32, device=DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    oc = o.cpu()
    Sc = S.cpu()
    del o, qd, kd, vd, S
    torch.cuda.empty_cache()

    piece = 1 << 17
    run = RunningBF16Check()
    S64 = None
    for a in range(0, w.N, piece):
        b = min(w.N, a + piece)
        ref_o, S64 = oracle.recurrent(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], S0=S64,
                                      o_dtype=np.float32)
        run.update(oc[:, :, a:b], ref_o)
        del ref_o
    assert run.count == w.B * w.Hq * w.N * w.d
    run.check(f"{w.name} chunk {chunk}, all rows vs the recurrence")
    assert_f32_close(Sc, S64, f"{w.name} final state vs the recurrence", tol=STATE_REL_L2)
    assert_f32_close(Sc, oracle.state_gemm(k, v), f"{w.name} final state vs K^T V",
                     tol=STATE_REL_L2)

    sel = _boundary_rows(la, w, chunk, 64)
    assert len(sel) >= 64
    ref = oracle.rows(q, k, v, sel)
    got = torch.stack([oc[b, h, t] for b, h, t in sel])
    assert_bf16_close(got, ref, f"{w.name} rows at chunk and span boundaries")


# ------------------------------------------------------------------ fused kernel
@pytest.mark.parametrize("Hq,Hkv,chunk", [(4, 2, 64), (2, 2, 64), (4, 1, 128), (6, 3, 64)])
@pytest.mark.parametrize("nspan,lookahead", [(1, 0), (2, 1), (3, 2), (7, 1), (7, 3), (7, 99),
                                             (0, 0), (-1, 1), (-1, 4)])
def test_fused_span_counts(la, Hq, Hkv, chunk, nspan, lookahead):
    """The single-pass kernel for span counts 1, 2, 3, 7, automatic (0) and
    one span per tile (-1), state items 1 to all rounds ahead, with an
    initial state; two calls on one workspace."""
    B, N = 2, 1100
    q, k, v = _qkv(B, Hq, Hkv, N, seed=300 + Hq * 10 + Hkv + chunk)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(7)) / 128
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy())
    qd, kd, vd = _cuda(q, k, v)
    if nspan == -1:
        nspan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).tiles_total
    nbytes = la.api.la_prefill_fused_workspace_bytes(B, Hq, Hkv, N, 128, chunk, nspan)
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    for call in range(2):
        S = S0.to(DEV)
        o = torch.full_like(qd, float("nan"))
        la.api.la_prefill_fused(qd, kd, vd, o, S, ws, chunk=chunk, nspan=nspan, lookahead=lookahead)
        torch.cuda.synchronize()
        assert_bf16_close(o.cpu(), ref_o, f"O nspan={nspan} call {call}")
        assert_f32_close(S.cpu(), ref_S, f"final state nspan={nspan} call {call}", tol=STATE_REL_L2)
    assert la.la_device_status()[1] == 0


def test_fused_rejects_bad_span_count(la):
    q, k, v = _cuda(*_qkv(1, 2, 2, 256, seed=9))
    tiles = la.api.la_prefill_plan(1, 2, 2, 256, 128, 64).tiles_total
    assert la.api.la_prefill_fused_workspace_bytes(1, 2, 2, 256, 128, 64, tiles + 1) == 0
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(la.LAError) as e:
        la.api.la_prefill_fused(q, k, v, torch.empty_like(q), None, ws, chunk=64, nspan=tiles + 1)
    assert e.value.code == 1
    with pytest.raises(la.LAError) as e:
        la.api.la_prefill_fused(q, k, v, torch.empty_like(q), None, ws[:64], chunk=64, nspan=1)
    assert e.value.code == 5


# ------------------------------------------------------------------ host buffers
@pytest.mark.parametrize("N,piece,with_state", [(1000, 0, False), (1000, 128, True), (777, 300, True),
                                                (64, 0, False)])
def test_forward_host_pipelined(la, N, piece, with_state):
    """Pinned host inputs and output, pieces pipelined against the compute:
    the same result as the oracle, and the carried state as the final state."""
    B, Hq, Hkv = 2, 4, 2
    q, k, v = _qkv(B, Hq, Hkv, N, seed=500 + N + piece)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(8)) / 128
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy() if with_state else None)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    S = S0.to(DEV) if with_state else None
    o = la.la_forward_host(qh, kh, vh, S=S, chunk=64, piece=piece)
    torch.cuda.synchronize()
    assert_bf16_close(o, ref_o, f"O N={N} piece={piece}")
    if with_state:
        assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)


# ------------------------------------------------------------------ one span per kv head
# With many (batch, kv head) sequences and short N the plan has one span each,
# and la_forward / la_forward_state / la_forward_ws run the persistent chunk
# loop alone (one CTA per SM walks whole kv groups): it reads the initial
# state and writes the final one from tensor memory, in place.
def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


PERSISTENT = [
    # B, Hq, Hkv, N, chunk
    (40, 16, 4, 100, 64),    # T=64, two tiles per chunk step, ragged tail
    (40, 16, 4, 300, 64),    # several chunk steps per item
    (40, 16, 4, 100, 128),   # T=128, four tiles per chunk step
    (160, 4, 4, 130, 64),    # single-head groups: 128-token tiles
    (50, 18, 3, 77, 64),     # group of 6: three tiles per chunk step
    (100, 8, 2, 1, 64),      # one token
    (37, 32, 4, 64, 64),     # 148 sequences: one item per CTA
    (300, 2, 1, 65, 128),    # 300 items over the SMs, uneven rounds
]
FEWER_THAN_SMS = [
    (30, 16, 4, 100, 64),    # 120 sequences: some SMs idle, one item each
    (30, 16, 4, 100, 128),
    (64, 6, 2, 64, 64),      # group of 3 -> 128-token tiles
]


def _state_in_out(la, B, Hq, Hkv, N, chunk, seed):
    q, k, v = _qkv(B, Hq, Hkv, N, seed=seed)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(N)) / 128
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy())
    qd, kd, vd = _cuda(q, k, v)
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    o0 = la.la_forward(qd, kd, vd, chunk=chunk)  # zero state, no state out
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    assert_bf16_close(o.cpu(), ref_o, f"O {B}x{Hq}/{Hkv}x{N}")
    assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)
    assert_bf16_close(o0.cpu(), oracle.recurrent(q, k, v)[0], "O from zero state")


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", PERSISTENT)
def test_persistent_state_in_out(la, B, Hq, Hkv, N, chunk):
    assert B * Hkv >= _sms()
    assert la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).nspan == 1
    _state_in_out(la, B, Hq, Hkv, N, chunk, seed=700 + B + N)


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", FEWER_THAN_SMS)
def test_one_span_fewer_sequences_than_sms(la, B, Hq, Hkv, N, chunk):
    assert B * Hkv < _sms()
    assert la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).nspan == 1
    _state_in_out(la, B, Hq, Hkv, N, chunk, seed=750 + B + N)


@pytest.mark.parametrize("B,Hq,Hkv,N", [(48, 8, 2, 200), (160, 8, 2, 130), (200, 8, 2, 64)])
def test_one_launch_path_matches_staged_scheme(la, B, Hq, Hkv, N):
    """The one-launch path and the three stages with the same one-span plan
    compute the same outputs bit for bit (same entering state, same tile
    arithmetic in the same order); the final states agree to fp32 rounding
    of the two sums (accumulated in tensor memory vs. span sum + scan).
    The last shape has two tiles per item, where states are staged through
    shared memory."""
    chunk = 64
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk)
    assert plan.nspan == 1
    qd, kd, vd = _cuda(*_qkv(B, Hq, Hkv, N, seed=801))
    S0 = (torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(802)) / 128).to(DEV)
    S_a = S0.clone()
    o_a = la.la_forward_state(qd, kd, vd, S=S_a, chunk=chunk)
    ws = torch.empty(plan.workspace_bytes // 4, dtype=torch.float32, device=DEV)
    S_b = S0.clone()
    o_b = torch.empty_like(qd)
    la.api.la_prefill_span_states(kd, vd, plan, ws)
    la.api.la_prefill_scan(ws, S_b, plan, B, Hkv, 128)
    la.api.la_prefill_main(qd, kd, vd, o_b, ws, plan)
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_b)
    assert_f32_close(S_a.cpu(), S_b.cpu().double().numpy(), "final states", tol=1e-6)


def test_single_span_workspace(la):
    """With one span per sequence la_forward_ws needs no workspace (a nominal
    256 bytes, contents irrelevant); the state carries across two in-place
    calls on consecutive pieces."""
    for B, Hq, Hkv, N in ((30, 16, 4, 96), (40, 16, 4, 96)):
        chunk = 64
        assert la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk).nspan == 1
        nbytes = la.api.la_forward_workspace_bytes(B, Hq, Hkv, N, 128, chunk)
        assert nbytes == 256
        q, k, v = _qkv(B, Hq, Hkv, 2 * N, seed=901)
        ref_o, ref_S = oracle.recurrent(q, k, v)
        qd, kd, vd = _cuda(q, k, v)
        ws = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device=DEV)  # not zero on entry
        S = torch.zeros(B, Hkv, 128, 128, dtype=torch.float32, device=DEV)
        outs = []
        for piece in range(2):
            sl = slice(piece * N, (piece + 1) * N)
            o = torch.empty_like(qd[:, :, sl])
            la.api.la_forward_ws(*(t[:, :, sl].contiguous() for t in (qd, kd, vd)), o, S, ws,
                                 chunk=chunk)
            outs.append(o)
        torch.cuda.synchronize()
        assert_bf16_close(torch.cat(outs, dim=2).cpu(), ref_o, f"O in two pieces, B={B}")
        assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)


@pytest.mark.parametrize("chunk", [64, 128])
def test_multi_token_decode_shape(la, chunk):
    """64 known tokens for each of 256 sequences (64 query / 16 kv heads)
    through the one-launch path, continuing from a decode state: every output
    and the final state against the oracle's recurrence."""
    w = synth.DECODE_B256
    B, Hq, Hkv, T = w.B, w.Hq, w.Hkv, 64
    S0 = synth.decode_state(w)
    q, k, v = synth.random_qkv(B, Hq, Hkv, T, 128, torch.bfloat16, w.seed + 1000)
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy(), o_dtype=np.float32)
    qd, kd, vd = _cuda(q, k, v)
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    assert_bf16_close(o.cpu(), ref_o, "multi-token O")
    assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)


def test_span_parts(la):
    """Few sequences and spans (64 kv heads, 2 spans): each span's state is
    computed by several CTAs (sub-spans) and the scan folds them in; entering
    states, outputs and the final state against the oracle."""
    B, Hq, Hkv, N, chunk = 4, 16, 16, 2048, 64
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, 128, chunk)
    assert plan.nspan == 2
    assert la.api.la_forward_workspace_bytes(B, Hq, Hkv, N, 128, chunk) > plan.workspace_bytes
    q, k, v = _qkv(B, Hq, Hkv, N, seed=1201)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(1202)) / 128
    ref_o, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy(), o_dtype=np.float32)
    qd, kd, vd = _cuda(q, k, v)
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    o0 = la.la_forward(qd, kd, vd, chunk=chunk)
    torch.cuda.synchronize()
    assert la.la_device_status()[1] == 0
    assert_bf16_close(o.cpu(), ref_o, "O")
    assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)
    assert_bf16_close(o0.cpu(), oracle.recurrent(q, k, v, o_dtype=np.float32)[0], "O from zero")


# ------------------------------------------------------------------ degenerate inputs
def test_empty_inputs_are_rejected(la):
    """N = 0 or B = 0: nothing to compute; the ABI rejects the shape."""
    for shape in ((1, 2, 0, 128), (0, 2, 64, 128)):
        q = torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
        with pytest.raises(la.LAError) as e:
            la.la_forward(q, q.clone(), q.clone(), chunk=64)
        assert e.value.code == 1
    S = torch.zeros(0, 1, 128, 128, dtype=torch.float32, device=DEV)
    qt = torch.zeros(0, 1, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(la.LAError) as e:
        la.la_decode_step(S, qt, qt.clone(), qt.clone())
    assert e.value.code == 1


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", [(2, 8, 2, 1000, 64), (1, 2, 2, 300, 128), (200, 4, 2, 64, 64)])
def test_zero_keys_leave_only_the_state_term(la, B, Hq, Hkv, N, chunk):
    """K = 0: every score and every state update vanishes, so O = Q S0 and
    the final state is S0 bit for bit (on every path: span scheme, one launch,
    staged states)."""
    q, _, v = _qkv(B, Hq, Hkv, N, seed=1301 + N)
    k = torch.zeros(B, Hkv, N, 128, dtype=torch.bfloat16)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(1302)) / 128
    ref_o, _ = oracle.recurrent(q, k, v, S0=S0.double().numpy(), o_dtype=np.float32)
    qd, kd, vd = _cuda(q, k, v)
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert_bf16_close(o.cpu(), ref_o, "O = Q S0")
    assert torch.equal(S.cpu(), S0)


@pytest.mark.parametrize("B,Hq,Hkv,N,chunk", [(2, 8, 2, 1000, 64), (200, 4, 2, 64, 64)])
def test_zero_queries_give_zero_output(la, B, Hq, Hkv, N, chunk):
    """Q = 0: O is exactly zero; the state still takes every K^T V."""
    _, k, v = _qkv(B, Hq, Hkv, N, seed=1401 + N)
    q = torch.zeros(B, Hq, N, 128, dtype=torch.bfloat16)
    S0 = torch.randn(B, Hkv, 128, 128, generator=torch.Generator().manual_seed(1402)) / 128
    _, ref_S = oracle.recurrent(q, k, v, S0=S0.double().numpy())
    qd, kd, vd = _cuda(q, k, v)
    S = S0.to(DEV)
    o = la.la_forward_state(qd, kd, vd, S=S, chunk=chunk)
    torch.cuda.synchronize()
    assert not torch.any(o)
    assert_f32_close(S.cpu(), ref_S, "final state", tol=STATE_REL_L2)
