"""Benchmark of the causal Lightning Attention prefill (and decode step) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa32k|mha8k|long1m] [--chunk 64|128]

One JSON line on rank 0.  A step is one la_forward call over the whole
workload (span states, state scan, chunk loop = every prefill stage).  The
default workload is the grouped-query MiniMax-01-shaped layer: B=1, 128 query
heads over 32 kv heads, N=32768, d=128, chunk 64, bf16 (q, k ~ N(0,1)/sqrt(d),
v ~ N(0,1), seed 2).  Its inputs (2.7 GB) exceed L2, so no flush is needed.

  value      Mtok/s with inputs resident in HBM (tokens = B*N positions, all heads)
  e2e        the same metric through the public call with pinned host buffers,
             host->device copies of q, k, v and the device->host copy of O
             inside the timed region
  roofline   the main chunk-loop kernel: algorithmic Q+K+V+O bytes / its
             CUDA-event duration, against the measured HBM copy bandwidth
  decode     the decode step on B=256, Hq=64/Hkv=16, d=128, 64 steps: GB/s
  workloads  the suite's other prefill workloads (mha B4 H16 N8K chunk 64, gqa
             at chunk 128, long B1 H8 N1M chunk 128): step time, Mtok/s and
             fraction of roofline of the step and of the chunk-loop kernel
  cpu_baseline  the fp64 CPU oracle (recurrent form) on a bounded sample

Multi-GPU (torchrun): every rank runs its own copy of the workload (independent
sequences, no collective on the data path): weak scaling; the reported time is
the max over ranks.  ``--impl reference`` times the CPU oracle on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_11_b200 import synth  # noqa: E402

# the headline metric: prefill Mtok/s (value), its roofline fraction
# (roofline), and the decode step's GB/s (decode)
METRIC = "causal lightning-attn prefill Mtok/s & % roofline; decode-step GB/s, 1 B200"

WORKLOADS = {"gqa32k": synth.GQA_32K, "mha8k": synth.MHA_8K, "long1m": synth.LONG_1M}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="gqa32k")
    ap.add_argument("--chunk", type=int, default=None)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads of the suite (mha 8K, gqa chunk 128, long 1M)")
    ap.add_argument("--cpu-sample-tokens", type=int, default=None)
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override N (smaller case of the same workload, for profiling)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the GPU works."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001
            self._nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def max_over_ranks(t: float, dist=None, device=None) -> float:
    """The largest of every rank's value (a scalar all-reduce; no data path)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return t
    tt = torch.tensor([t], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def throughput_mtok(world: int, B: int, N: int, steps: int, seconds: float) -> float:
    """Whole-job Mtok/s: every rank processes its own B x N tokens per step."""
    return world * B * N * steps / seconds / 1e6


def timed(fn, steps, stream):
    """Device time of `steps` calls of fn on `stream`, with clock samples."""
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dev = torch.cuda.current_device()
    with ClockSampler(dev) as clk:
        start.record(stream)
        for _ in range(steps):
            fn()
        end.record(stream)
        while not end.query():
            time.sleep(0.001)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3, clk.summary()


def kernel_source_sha256():
    """Hash of the chunk-loop kernel's source (its file and the device headers
    it includes) with // comments and whitespace removed, the key under which
    ncu figures of it are committed."""
    csrc = os.path.join(ROOT, "linear_attention_11_b200", "csrc")
    h = hashlib.sha256()
    for name in ("la_prefill_persist.cu", "la_tile.cuh", "la_ptx.cuh"):
        text = open(os.path.join(csrc, name), encoding="utf-8").read()
        code = re.sub(r"//[^\n]*", "", text)  # no string literal in these files holds "//"
        h.update("".join(code.split()).encode())
    return h.hexdigest()


def traffic_from_profile():
    """DRAM bytes per launch of the chunk-loop kernel on the benchmark workload
    from the committed ncu figure (profiles/prefill_persist_traffic.json), if
    the kernel source is unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "prefill_persist_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("kernel_source_sha256") == kernel_source_sha256():
            return int(rec["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError, TypeError):
        pass
    return None


# ------------------------------------------------------------------ CPU oracle
def cpu_baseline(w, tokens=None, target_s=10.0):
    """The fp64 oracle (recurrent form), as it stands, on a sequence of n tokens
    drawn with the workload's recipe, all heads.  Without tokens, n is
    grown from a 256-token probe to about target_s seconds of work.
    Returns (tokens/s, sample description, threads used, seconds)."""
    import numpy as np

    import oracle
    cores = oracle.threads()
    units = w.B * w.Hkv
    n = sample_tokens(w, target_s) if tokens is None else tokens
    q, k, v = synth.prefill_inputs(w, N=n)
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v, o_dtype=np.float32)
    dt = time.perf_counter() - t0
    sample = (f"{n} of {w.N} tokens drawn with the workload recipe, B={w.B}, all {w.Hq} query "
              f"heads; {units} independent (batch, kv head) units over {min(cores, units)} threads")
    return w.B * n / dt, sample, min(cores, units), dt


def bench_workload(la, w, chunk, steps, dev, stream, pk):
    """One more workload of the suite on this GPU: the whole prefill step
    (la_forward, every stage) and its chunk-loop kernel alone, each timed
    with CUDA events, against the HBM roofline of its Q, K, V, O bytes."""
    q, k, v = synth.prefill_inputs(w)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    del q, k, v
    o = torch.empty_like(qd)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d

    def step():
        la.la_forward(qd, kd, vd, o=o, chunk=chunk, stream=stream)

    for _ in range(3):
        step()
    t, clk = timed(step, steps, stream)
    t /= steps
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, d, chunk)
    ws = torch.empty(max(1, plan.workspace_bytes // 4), dtype=torch.float32, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(max(3, min(steps, 10)))]
    for i in range(len(ev) + 2):
        la.api.la_prefill_span_states(kd, vd, plan, ws, stream=stream)
        la.api.la_prefill_scan(ws, None, plan, B, Hkv, d, stream=stream)
        if i >= 2:
            ev[i - 2][0].record(stream)
        la.api.la_prefill_main(qd, kd, vd, o, ws, plan, stream=stream)
        if i >= 2:
            ev[i - 2][1].record(stream)
    torch.cuda.synchronize()
    t_main = statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3
    alg = 2 * (2 * B * Hq * N * d + 2 * B * Hkv * N * d)
    flops = B * Hq * N * (4 * chunk * d + 4 * d * d)
    t_roof = max(alg / (pk["hbm_gbs"] * 1e9), flops / (pk["bf16_tflops"] * 1e12))
    del qd, kd, vd, o, ws
    torch.cuda.empty_cache()
    return {"workload": w.name, "chunk": chunk, "steps": steps, "ms_per_step": t * 1e3,
            "mtok_s": B * N / t / 1e6, "algorithmic_bytes": alg,
            "step_frac_of_roofline": t_roof / t, "chunk_loop_ms": t_main * 1e3,
            "chunk_loop_frac_of_hbm": alg / t_main / 1e9 / pk["hbm_gbs"],
            "nspan": plan.nspan, "clocks": clk,
            "roofline": "slower of Q+K+V+O bytes at the measured HBM peak and the chunk-form "
                        "FLOPs N(4Cd+4d^2) per query head at the measured bf16 peak (HBM here)"}


# ------------------------------------------------------------------ arms
def bench_config(w, chunk, world):
    """The workload as both arms name it (N ranks: N replicas of it)."""
    return {"workload": w.name, "global_batch": w.B * world, "seq_len": w.N, "chunk": chunk,
            "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (no flush)"}


def sample_tokens(w, target_s):
    """Tokens of the workload the oracle covers in about target_s seconds
    (grown from a 256-token probe, at most the whole sequence)."""
    import numpy as np

    import oracle
    q, k, v = synth.prefill_inputs(w, N=256)
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v, o_dtype=np.float32)
    dt0 = time.perf_counter() - t0
    return int(min(w.N, max(256, 256 * target_s / max(dt0, 1e-3))))


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    steps, warm = args.steps, args.warmup
    # the same sample as the in-line cpu_baseline (the whole sequence when it
    # takes up to ~10 s), shortened only to keep the whole run near 150 s
    n = args.cpu_sample_tokens or sample_tokens(w, min(10.0, 150.0 / max(1, steps + warm)))
    cores = min(oracle.threads(), w.B * w.Hkv)
    q, k, v = synth.prefill_inputs(w, N=n)
    per = []
    for i in range(warm + steps):
        t0 = time.perf_counter()
        oracle.recurrent(q, k, v, o_dtype=np.float32)
        if i >= warm:
            per.append(time.perf_counter() - t0)
    dt = sum(per)
    value = w.B * n * steps / dt / 1e6
    line = {"impl": "reference", "metric": METRIC,
            "value": value, "unit": "Mtok/s", "n_gpus": args.gpus, "steps": steps,
            "warmup": warm, "ms_per_step": 1e3 * dt / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(w, args.chunk or w.chunks[0], args.gpus),
            "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: the first {n} tokens of the workload "
                                       f"(B={w.B}, all {w.Hq} query heads), fp64 recurrent form"},
            "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, w):
    import linear_attention_11_b200 as la

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    chunk = args.chunk or w.chunks[0]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    q, k, v = synth.prefill_inputs(w)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    o = torch.empty_like(qd)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d

    def step():
        la.la_forward(qd, kd, vd, o=o, chunk=chunk, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if dist:
            dist.barrier()
        torch.cuda.synchronize()

    barrier()
    t, clocks = timed(step, args.steps, stream)
    barrier()
    t = max_over_ranks(t, dist, dev)
    value = throughput_mtok(world, B, N, args.steps, t)

    # --- per-kernel timing of the main chunk-loop pass (stages called apart)
    plan = la.api.la_prefill_plan(B, Hq, Hkv, N, d, chunk)
    ws = torch.empty(plan.workspace_bytes // 4, dtype=torch.float32, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(max(3, min(args.steps, 20)))]
    for i in range(len(ev) + 2):
        la.api.la_prefill_span_states(kd, vd, plan, ws, stream=stream)
        la.api.la_prefill_scan(ws, None, plan, B, Hkv, d, stream=stream)
        if i >= 2:
            ev[i - 2][0].record(stream)
        la.api.la_prefill_main(qd, kd, vd, o, ws, plan, stream=stream)
        if i >= 2:
            ev[i - 2][1].record(stream)
    torch.cuda.synchronize()
    t_main = statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3
    elt = 2
    alg_bytes = elt * (2 * B * Hq * N * d + 2 * B * Hkv * N * d)
    # chunk-form FLOPs per query head: N (4 C d + 4 d^2)
    flops_chunk_form = B * Hq * N * (4 * chunk * d + 4 * d * d)
    pk = peaks()
    achieved = alg_bytes / t_main / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": (traffic_from_profile() if (w is synth.GQA_32K and chunk == 64) else None),
                "kernel": "prefill_persist_kernel", "launch_ms": t_main * 1e3,
                "algorithmic_bytes_per_launch": alg_bytes, "peak_source": pk["source"]}
    step_frac = (alg_bytes / (t / args.steps) / 1e9) / pk["hbm_gbs"]

    # --- the schemes weighed against the span-parallel two-pass prefill
    def ev_mean(fn, reps=5):
        for _ in range(2):
            fn()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b2.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b2) / reps / 1e3

    seq = la.api.la_prefill_plan(B, Hq, Hkv, N, d, chunk)
    seq.nspan = 1
    seq.workspace_bytes = B * Hkv * d * d * 4
    ws1 = torch.zeros(seq.workspace_bytes // 4, dtype=torch.float32, device=dev)
    t_seq = ev_mean(lambda: la.api.la_prefill_main(qd, kd, vd, o, ws1, seq, stream=stream), 2)
    fb = la.api.la_prefill_fused_workspace_bytes(B, Hq, Hkv, N, d, chunk, 0)
    wsf = torch.empty(fb, dtype=torch.uint8, device=dev)
    t_fused = ev_mean(lambda: la.api.la_prefill_fused(qd, kd, vd, o, None, wsf, chunk=chunk,
                                                      stream=stream))
    # the same step captured once in a CUDA graph and replayed (launch costs
    # of the host call removed): informational
    gs = torch.cuda.Stream()
    with torch.cuda.stream(gs):
        la.la_forward(qd, kd, vd, o=o, chunk=chunk, stream=gs)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=gs):
        la.la_forward(qd, kd, vd, o=o, chunk=chunk, stream=gs)
    t_graph = ev_mean(graph.replay, 10)
    del graph
    alternatives = {
        "two_pass_span_parallel_ms": 1e3 * t / args.steps,
        "cuda_graph_replay_ms": 1e3 * t_graph,
        "sequential_chunk_loop_ms": 1e3 * t_seq,
        "single_pass_fused_ms": 1e3 * t_fused,
        "note": "sequential = one span per (batch, kv head): one CTA walks every chunk of "
                "the kv group; "
                "fused = span states and chunk loops in one persistent kernel",
    }
    del ws1, wsf

    # --- backward of the same workload (training): dq, dk, dv from dO
    backward = None
    if not args.no_backward:
        dOd = synth.random_qkv(B, Hq, Hq, N, d, torch.bfloat16, 77)[0].to(dev)
        for _ in range(2):
            la.la_backward(qd, kd, vd, dOd, chunk=chunk, stream=stream)
        reps = max(3, min(args.steps, 10))
        tb, bclk = timed(lambda: la.la_backward(qd, kd, vd, dOd, chunk=chunk, stream=stream), reps,
                         stream)
        tb /= reps
        bbytes = elt * (3 * B * Hq * N * d + 4 * B * Hkv * N * d)  # q, dO, dq + k, v, dk, dv
        # chunk-form FLOPs: the dq pass as the forward; the dk, dv walk per
        # query-head token 2 scores + 2 products over 128-row chunks (8*128*d)
        # and the state update (2 d^2), per kv token K_c D and V_c D^T (4 d^2)
        bflops = (B * Hq * N * (4 * chunk * d + 4 * d * d)
                  + B * Hq * N * (8 * 128 * d + 2 * d * d) + B * Hkv * N * 4 * d * d)
        t_hbm = bbytes / (pk["hbm_gbs"] * 1e9)
        t_tc = bflops / (pk["bf16_tflops"] * 1e12)
        backward = {"ms_per_step": tb * 1e3, "mtok_s": world * B * N / tb / 1e6,
                    "algorithmic_gb_s": bbytes / tb / 1e9,
                    "frac_of_hbm_roofline": bbytes / tb / 1e9 / pk["hbm_gbs"],
                    "tflops_chunk_form": bflops / tb / 1e12,
                    "bound": "tensor" if t_tc > t_hbm else "hbm",
                    "frac_of_roofline": max(t_hbm, t_tc) / tb,
                    "bytes": bbytes, "flops": bflops, "clocks": bclk,
                    "passes": "dq causal (grouped) + one anti-causal dk, dv walk per kv group"}
        del dOd

    # --- end to end: pinned host buffers, copies inside the timed region.
    # The public host-buffer call pipelines the copies against the compute;
    # copies around the device call (serial) are reported beside it.
    e2e = None
    if not args.no_e2e:
        e2e_steps = args.e2e_steps or max(3, min(args.steps, 10))
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        oh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)

        def e2e_step():
            la.la_forward_host(qh, kh, vh, o=oh, chunk=chunk, stream=stream)

        e2e_step()
        barrier()
        te, _ = timed(e2e_step, e2e_steps, stream)
        barrier()
        te = max_over_ranks(te, dist, dev)
        qe, ke, ve = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)

        def serial_step():
            qe.copy_(qh, non_blocking=True)
            ke.copy_(kh, non_blocking=True)
            ve.copy_(vh, non_blocking=True)
            la.la_forward(qe, ke, ve, o=o, chunk=chunk, stream=stream)
            oh.copy_(o, non_blocking=True)

        serial_step()
        ts, _ = timed(serial_step, e2e_steps, stream)
        e2e = {"value": throughput_mtok(world, B, N, e2e_steps, te), "unit": "Mtok/s",
               "h2d_bytes_per_step": elt * (q.numel() + k.numel() + v.numel()),
               "d2h_bytes_per_step": elt * q.numel(), "steps": e2e_steps,
               "api": "la_forward_host (pinned host q, k, v in; O out; copies pipelined)",
               "ms_per_step": 1e3 * te / e2e_steps,
               "serial_copies_mtok_s": throughput_mtok(world, B, N, e2e_steps, ts)}
        del qh, kh, vh, oh, qe, ke, ve

    # --- decode step
    decode = None
    if not args.no_decode:
        del qd, kd, vd, o, ws
        torch.cuda.empty_cache()
        dw = synth.DECODE_B256
        S = synth.decode_state(dw).to(dev)
        toks = [tuple(t.to(dev) for t in synth.decode_token(dw, i)) for i in range(dw.steps)]
        od = torch.empty(dw.B, dw.Hq, dw.d, dtype=torch.bfloat16, device=dev)
        for i in range(3):
            la.la_decode_step(S, *toks[i], o=od, stream=stream)
        it = iter(range(10**9))

        def dstep():
            i = next(it) % dw.steps
            la.la_decode_step(S, *toks[i], o=od, stream=stream)

        td, dclk = timed(dstep, dw.steps, stream)
        per = td / dw.steps
        dbytes = 4 * 2 * dw.B * dw.Hkv * dw.d * dw.d + 2 * (2 * dw.B * dw.Hq * dw.d +
                                                             2 * dw.B * dw.Hkv * dw.d)
        decode = {"metric": "decode-step HBM bandwidth", "value": dbytes / per / 1e9,
                  "unit": "GB/s", "us_per_step": per * 1e6, "steps": dw.steps,
                  "frac_of_hbm_peak": dbytes / per / 1e9 / pk["hbm_gbs"],
                  "bytes_per_step": dbytes, "workload": dw.name, "clocks": dclk}
        # the same 64 tokens per sequence in one launch (state kept on chip)
        qs = torch.stack([t[0] for t in toks], dim=2).contiguous()
        ks = torch.stack([t[1] for t in toks], dim=2).contiguous()
        vs = torch.stack([t[2] for t in toks], dim=2).contiguous()
        os_ = torch.empty_like(qs)
        for _ in range(3):
            la.la_decode_steps(S, qs, ks, vs, o=os_, stream=stream)
        reps = 10
        tm, _ = timed(lambda: la.la_decode_steps(S, qs, ks, vs, o=os_, stream=stream), reps, stream)
        tm /= reps
        mbytes = 4 * 2 * dw.B * dw.Hkv * dw.d * dw.d + 2 * dw.steps * (2 * dw.B * dw.Hq * dw.d +
                                                                       2 * dw.B * dw.Hkv * dw.d)
        flops = 2 * dw.steps * dw.B * dw.Hkv * dw.d * dw.d * (1 + dw.G)
        decode["multi_step"] = {
            "us_per_call": tm * 1e6, "tokens_per_call": dw.steps,
            "us_per_token_step": tm * 1e6 / dw.steps,
            "speedup_vs_single_steps": per * dw.steps / tm,
            "gb_s": mbytes / tm / 1e9, "fp32_tflop_s": flops / tm / 1e12,
            "note": "fp32 FMA recurrence, state in registers; bound by fp32 ALU throughput"}
        # the same tokens through the chunked tensor-core form: one span per
        # (sequence, kv head), so la_forward_state is a single chunk-loop
        # launch reading S and writing the final S (plus a counter reset)
        for _ in range(3):
            la.la_forward_state(qs, ks, vs, S=S, o=os_, chunk=64, stream=stream)
        tc, tclk = timed(lambda: la.la_forward_state(qs, ks, vs, S=S, o=os_, chunk=64,
                                                     stream=stream), reps, stream)
        tc /= reps
        decode["multi_step_tensor_core"] = {
            "us_per_call": tc * 1e6, "tokens_per_call": dw.steps,
            "us_per_token_step": tc * 1e6 / dw.steps,
            "speedup_vs_single_steps": per * dw.steps / tc,
            "gb_s": mbytes / tc / 1e9, "frac_of_hbm_peak": mbytes / tc / 1e9 / pk["hbm_gbs"],
            "bytes_per_call": mbytes, "clocks": tclk,
            "api": "la_forward_state on [B,H,64,d] with S in/out (chunk 64)",
            "note": "bf16 operands, fp32 state in tensor memory; outputs within the bf16 "
                    "tolerance of the oracle, not bitwise equal to single steps"}

    # --- the other workloads of the suite (prefill step and chunk loop each)
    workloads = None
    if not args.no_workloads:
        workloads = []
        for ow, oc in ((synth.MHA_8K, 64), (synth.GQA_32K, 128), (synth.LONG_1M, 128)):
            if ow is w and oc == chunk:
                continue
            reps = max(3, min(args.steps, 10 if ow is synth.LONG_1M else 20))
            workloads.append(bench_workload(la, ow, oc, reps, dev, stream, pk))

    line = {
        "metric": METRIC,
        "value": value, "unit": "Mtok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(w, chunk, world),
        "clocks": clocks,
        "gpu_launches": 3 * args.steps,  # span states, scan, chunk loop per step
        "roofline": roofline,
        "step_hbm_frac": step_frac,
        "alternatives": alternatives,
        "tflops_chunk_form": flops_chunk_form / (t / args.steps) / 1e12,
        "e2e": e2e,
        "backward": backward,
        "decode": decode,
        "workloads": workloads,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, sample, cores, dt = cpu_baseline(w, args.cpu_sample_tokens)
        line["cpu_baseline"] = {"value": tok_s / 1e6, "unit": "Mtok/s", "cores": cores,
                                "kind": "oracle", "sample": sample, "seconds": dt}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    w = WORKLOADS[args.workload]
    if args.seq_len:
        import dataclasses
        w = dataclasses.replace(w, N=args.seq_len, name=f"{w.name.split(' N')[0]} N{args.seq_len} d{w.d}")
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
