"""Benchmark: effective prefill TFLOP/s (and speedup over the same kernel with
every window open, alpha = inf) on the largest single-GPU workload: one
Qwen2.5-7B-shaped attention layer (batch 1, 28 query / 4 kv heads, d = 128,
theta = 1e7, alpha = 1) of 131072 tokens, prefilled causally in 16 query chunks
of 8192 against all earlier keys.  The 8k layer with its alpha sweep, the 32k
pair-energy layer and the 1M-key decode (GB/s) are reported as extra keys.

One step = the whole prefill hot path on one input: RoPE of k into the cache
(fp64 angles), then per query chunk RoPE of its queries and the windowed
prefill (windowed QK on the tensor cores, online softmax, P.V, epilogue, the
skipped-pair counter).  Effective FLOPs count only the query-key pairs inside
their window (4 FLOP per active pair) plus P.V (2d FLOP per causal element);
the exponentials are not counted.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own independent layer (weak scaling; no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rope_frequency_sparse_b200 import atf, synth  # noqa: E402

HEADLINE = "layer_128k_chunked"
METRIC = "effective prefill TFLOP/s (alpha=1; active query-key pairs + P.V counted)"
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ accounting (host integers)

def window_table(d, theta, alpha, windows=None):
    """W_i as Python ints: from the library (our arm) or from `windows` (the
    reference arm passes the oracle's table, so that arm loads no CUDA code)."""
    if windows is not None:
        return [int(x) for x in windows(d, theta, alpha)]
    return [int(x) for x in atf.atf_windows(d, theta, alpha)]


def prefill_flops(w: synth.Workload, alpha: float, seq: int | None = None, windows=None) -> tuple[int, int, int]:
    """(effective FLOPs, dense FLOPs, skipped pairs) of a causal prefill over `seq` tokens."""
    S = w.seq if seq is None else seq
    P = S * (S + 1) // 2
    W = window_table(w.d, w.theta, alpha, windows)
    skipped = sum((S - 1 - x) * (S - x) // 2 for x in W if x < S - 1)
    active = (w.d // 2) * P - skipped
    eff = w.batch * w.q_heads * (4 * active + 2 * w.d * P)
    dense = w.batch * w.q_heads * (4 * (w.d // 2) * P + 2 * w.d * P)
    return eff, dense, w.q_heads * skipped * w.batch


def row_flops(w: synth.Workload, alpha: float, m: int, windows=None) -> int:
    W = window_table(w.d, w.theta, alpha, windows)
    active = sum(min(m, x) + 1 for x in W)  # pairs i with (m - n) <= W_i over n = 0..m
    return 4 * active + 2 * w.d * (m + 1)


def causal_elements(w: synth.Workload, seq: int | None = None) -> int:
    """Query-key elements (m, n <= m) of the prefill, all heads: one exponential each."""
    S = w.seq if seq is None else seq
    return w.batch * w.q_heads * S * (S + 1) // 2


def decode_moved_bytes(w: synth.Workload, alpha: float) -> int:
    """Bytes the decode kernel reads and writes at full caches: every value row, and
    per 128-key tile each 8-pair key chunk (32 bytes per key) that some key of the
    tile still needs (chunk c while its widest pair's window W_{8c+7} reaches the
    tile's nearest key), plus q and out."""
    N = w.seq
    W = window_table(w.d, w.theta, alpha)
    nc = w.d // 16
    keys = 0
    for t in range((N + 127) // 128):
        nearest = N - 1 - min(N - 1, 128 * t + 127)  # distance of the tile's last (nearest) key
        n_t = min(128, N - 128 * t)
        keys += n_t * sum(1 for c in range(nc) if W[8 * c + 7] >= nearest)
    qo = 2 * w.batch * w.q_heads * w.d * 2
    return w.batch * w.kv_heads * (keys * 32 + N * w.d * 2) + qo


def decode_bytes(w: synth.Workload, alpha: float) -> tuple[int, int]:
    """(active bytes, dense bytes) of one decode step at full caches (pair granularity)."""
    N = w.seq
    W = window_table(w.d, w.theta, alpha)
    a_dec = sum(min(N - 1, x) + 1 for x in W)  # active (key, pair) per (b, kv head)
    qo = 2 * w.batch * w.q_heads * w.d * 2
    active = w.batch * w.kv_heads * (4 * a_dec + 2 * w.d * N) + qo
    dense = w.batch * w.kv_heads * (4 * N * w.d) + qo
    return active, dense


# ------------------------------------------------------------------ measurement helpers

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def flush_l2(buf):
    buf.fill_(1)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def recorded_traffic(kernel_file: str, profile_name: str):
    """DRAM bytes per launch recorded from an ncu capture, if the kernel source is
    unchanged since (the profile states the sha256 of the source it measured)."""
    path = os.path.join(ROOT, "profiles", profile_name)
    src = os.path.join(ROOT, "rope_frequency_sparse_b200", "csrc", kernel_file)
    try:
        text = open(path).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    m_sha = re.search(r"source sha256:\s*([0-9a-f]{64})", text)
    m_bytes = re.search(r"dram bytes per full-size launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_bytes or m_sha.group(1) != sha:
        return None
    return float(m_bytes.group(1))


# ------------------------------------------------------------------ the timed step

class PrefillStep:
    """Device-resident inputs and scratch for one windowed prefill step."""

    def __init__(self, w: synth.Workload, seed: int, device):
        q, k, v = synth.prefill_inputs(w, seed=seed)
        self.w = w
        self.host = (q, k, v)
        self.q, self.k, self.v = q.to(device), k.to(device), v.to(device)
        self.out = torch.empty_like(self.q)
        B, S, Hq, d = self.q.shape
        Hkv = self.k.shape[2]
        self.ws_bytes = atf.atf_prefill_workspace_bytes(B, S, S, Hq, Hkv, d, atf.ATF_BF16, 0)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.q_rot = self.ws[: B * S * Hq * d * 2].view(torch.bfloat16).view(B, S, Hq, d)
        off = ((B * S * Hq * d * 2 + 255) // 256) * 256
        self.k_rot = self.ws[off: off + B * S * Hkv * d * 2].view(torch.bfloat16).view(B, S, Hkv, d)
        self.cnt = torch.zeros(1, dtype=torch.int64, device=device)

    def run(self, alpha, stream, ev=None, pairing=0):
        """RoPE q, RoPE k, windowed prefill: 3 kernel launches.  ev = (e0, e1, e2)
        brackets the RoPE part and the prefill kernel.  pairing 1 reads q, k as
        rotate-half (NeoX-style) pairs."""
        w = self.w
        B, S, Hq, d = self.q.shape
        Hkv = self.k.shape[2]
        mode = 2 if pairing == atf.ATF_PAIRS_ROTATE_HALF else 1
        if ev:
            ev[0].record(stream)
        atf.atf_rope_layout(self.q, self.q_rot, None, B, S, Hq, d, 0, w.theta, mode, atf.ATF_BF16, stream)
        atf.atf_rope_layout(self.k, self.k_rot, None, B, S, Hkv, d, 0, w.theta, mode, atf.ATF_BF16, stream)
        if ev:
            ev[1].record(stream)
        atf.atf_prefill_ex(self.q_rot, self.k_rot, self.v, self.out, B, S, S, Hq, Hkv, d, 0, atf.ATF_BF16, 1,
                           w.theta, alpha, self.cnt, None, 0, stream)
        if ev:
            ev[2].record(stream)


class ChunkedPrefillStep:
    """Device-resident inputs and scratch for the chunked prefill of a long layer:
    keys rotated once into a cache, then per query chunk its queries rotated at
    their offset and attended against all earlier keys."""

    def __init__(self, w: synth.Workload, seed: int, device):
        q, k, v = synth.prefill_inputs(w, seed=seed)
        self.w = w
        self.host = (q, k, v)
        self.q, self.k, self.v = q.to(device), k.to(device), v.to(device)
        B, S, Hq, d = self.q.shape
        self.k_rot = torch.empty_like(self.k)
        self.q_rot = torch.empty((B, w.q_chunk, Hq, d), dtype=self.q.dtype, device=device)
        self.out = torch.empty_like(self.q)
        self.cnt = torch.zeros(1, dtype=torch.int64, device=device)
        self.n_chunks = S // w.q_chunk

    def n_events(self):
        return 2 + 2 * self.n_chunks

    def run(self, alpha, stream, ev=None, count=True):
        """RoPE k, then per chunk RoPE q + windowed prefill: 1 + 2 x chunks launches.
        ev = (step start, step end, then start/end of each chunk's prefill kernel)."""
        w = self.w
        B, S, Hq, d = self.q.shape
        Hkv = self.k.shape[2]
        C = w.q_chunk
        if ev:
            ev[0].record(stream)
        atf.atf_rope_layout(self.k, self.k_rot, None, B, S, Hkv, d, 0, w.theta, 1, atf.ATF_BF16, stream)
        for c in range(self.n_chunks):
            c0 = c * C
            atf.atf_rope_layout(self.q[:, c0:c0 + C], self.q_rot, None, B, C, Hq, d, c0, w.theta, 1, atf.ATF_BF16,
                                stream)
            if ev:
                ev[2 + 2 * c].record(stream)
            atf.atf_prefill_ex(self.q_rot, self.k_rot, self.v, self.out[:, c0:c0 + C], B, C, c0 + C, Hq, Hkv, d, c0,
                               atf.ATF_BF16, 1, w.theta, alpha, self.cnt if count else None, None, 0, stream)
            if ev:
                ev[3 + 2 * c].record(stream)
        if ev:
            ev[1].record(stream)

    @staticmethod
    def times(evs):
        """(mean ms per step, mean ms of the prefill kernels per step) of timed steps."""
        step = [e[0].elapsed_time(e[1]) for e in evs]
        kern = [sum(e[2 + 2 * c].elapsed_time(e[3 + 2 * c]) for c in range((len(e) - 2) // 2)) for e in evs]
        return sum(step) / len(step), sum(kern) / len(kern)


def time_steps(fn, steps, warmup, stream, flush_buf, n_events=3):
    """Run warmup + steps; per-step CUDA events (the L2 flush between steps is
    outside the events).  Returns list of per-step event-lists."""
    for _ in range(warmup):
        flush_l2(flush_buf)
        fn(None)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(steps)]
    for i in range(steps):
        flush_l2(flush_buf)
        fn(evs[i])
    torch.cuda.synchronize()
    return evs


def graphed_step(call, stream):
    """Capture `call` (the library calls of one step, issued on torch's current
    stream) in a CUDA graph and return a step function for time_steps that
    replays it between the step's two events.  The host's argument checks and
    descriptor encoding then stay outside the timed region, as in a serving loop
    that replays a captured decode step; the device work is the same launches."""
    call()  # first-call set-up (kernel attributes) outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()

    def step(ev):
        if ev:
            ev[0].record(stream)
        graph.replay()
        if ev:
            ev[1].record(stream)

    step.graph = graph
    return step


def time_interleaved(fns, steps, warmup, stream, flush_buf, n_events):
    """Warm up every step function, then run `steps` rounds of all of them in turn,
    so that they see the same clocks and power state; per-step CUDA events (the L2
    flush between steps outside them).  Returns one list of event-lists per fn."""
    for _ in range(warmup):
        for fn in fns:
            flush_l2(flush_buf)
            fn(None)
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(n_events)] for _ in range(steps)] for _ in fns]
    for i in range(steps):
        for f, fn in enumerate(fns):
            flush_l2(flush_buf)
            fn(evs[f][i])
    torch.cuda.synchronize()
    return evs


def dist_max(x: float) -> float:
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return x


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


# ------------------------------------------------------------------ CPU oracle baseline

def cpu_oracle_sample(w: synth.Workload, alpha: float, target_s: float = 12.0, seed=synth.DEFAULT_SEED,
                      inputs=None):
    """Time the fp64 oracle on a bounded sample of query rows of the workload (the
    rows of a chunked workload are the same rows of the unchunked prefill)."""
    import oracle  # test infrastructure: the CPU baseline only

    win = lambda d, theta, a: oracle.windows(d, theta, a)[0]  # noqa: E731
    q, k, v = inputs if inputs is not None else synth.prefill_inputs(w, seed=seed)
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    n_rows = 2
    while True:
        rows = np.sort(rng.choice(w.seq, size=n_rows, replace=False))
        t0 = time.perf_counter()
        oracle.prefill(q, k, v, w.theta, alpha, rows=rows, nthreads=cores)
        dt = time.perf_counter() - t0
        if dt >= target_s or n_rows >= w.seq:
            break
        n_rows = min(w.seq, max(n_rows * 2, int(n_rows * target_s / max(dt, 1e-3))))
    flops = w.batch * w.q_heads * sum(row_flops(w, alpha, int(m), win) for m in rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} random query rows x {w.q_heads} heads of {w.name} (alpha={alpha}), each "
                      f"against all its earlier keys; {dt:.1f} s wall; includes the oracle's one-time fp64 "
                      "rotation of all keys",
            "seconds": dt}


# ------------------------------------------------------------------ arms

def headline_config(w: synth.Workload, world: int) -> dict:
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seq, "query_chunk": w.q_chunk,
            "q_heads": w.q_heads, "kv_heads": w.kv_heads, "d": w.d, "theta": w.theta, "alpha": 1.0,
            "parallelism": f"independent layers x{world}",
            "l2": "inputs (1.2 GB) larger than L2, and a 256 MiB write between steps outside the CUDA events"}


def run_reference(args, rank):
    """The fp64 CPU oracle as it stands, on this arm's workload and metric (no
    CUDA code is loaded: FLOPs are counted with the oracle's own window table)."""
    if rank != 0:
        return
    w = synth.WORKLOADS[HEADLINE]
    inputs = synth.prefill_inputs(w)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, 1.0, target_s=2.0, inputs=inputs)
    vals, samples = [], []
    for _ in range(args.steps):
        smp = cpu_oracle_sample(w, 1.0, target_s=5.0, inputs=inputs)
        vals.append(smp["value"])
        samples.append(smp)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
            "config": headline_config(w, 1),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": samples[-1]["cores"], "kind": "oracle",
                             "sample": samples[-1]["sample"]},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    s = stream
    peaks, peak_kind = measured_peaks()
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    w = synth.WORKLOADS[HEADLINE]
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    step = ChunkedPrefillStep(w, synth.DEFAULT_SEED + rank, device)
    nev = step.n_events()

    # ---- headline: alpha = 1, timed region bracketed by barrier + sync
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        t_wall = time.perf_counter()
        evs = time_steps(lambda ev: step.run(1.0, s, ev), args.steps, args.warmup, stream, flush_buf, n_events=nev)
        t_wall = time.perf_counter() - t_wall
    barrier()
    torch.cuda.synchronize()
    atf.atf_check(s)
    ms_step, ms_kern = ChunkedPrefillStep.times(evs)
    ms_step, ms_kern = dist_max(ms_step), dist_max(ms_kern)
    eff, dense_flops, skipped = prefill_flops(w, 1.0)
    value = world * eff / (ms_step * 1e-3) / 1e12
    cnt_per_step = int(step.cnt.item()) // (args.steps + args.warmup)

    # ---- the same step with every window open (the dense specialisation) and with
    # alpha = 0.5, interleaved step by step with alpha = 1 so that all three see the
    # same clocks: the windowed kernel draws less power and keeps higher clocks under
    # the power cap, which a back-to-back comparison would credit to the method
    with ClockSampler(local_rank) as clocks_i:
        ev_i = time_interleaved([lambda ev: step.run(1.0, s, ev, count=False),
                                 lambda ev: step.run(math.inf, s, ev, count=False),
                                 lambda ev: step.run(0.5, s, ev, count=False)],
                                max(3, args.steps // 2), args.warmup, stream, flush_buf, nev)
    (ms_one, ms_one_kern), (ms_dense, ms_dense_kern), (ms_half, ms_half_kern) = (
        tuple(dist_max(x) for x in ChunkedPrefillStep.times(e)) for e in ev_i)
    eff_half = prefill_flops(w, 0.5)[0]
    per_alpha = {"0.5": {"tflops": eff_half / (ms_half * 1e-3) / 1e12, "ms": ms_half, "kernel_ms": ms_half_kern,
                         "speedup_vs_dense": ms_dense / ms_half},
                 "1.0": {"tflops": eff / (ms_one * 1e-3) / 1e12, "ms": ms_one, "kernel_ms": ms_one_kern,
                         "speedup_vs_dense": ms_dense / ms_one},
                 "inf": {"tflops": dense_flops / (ms_dense * 1e-3) / 1e12, "ms": ms_dense, "kernel_ms": ms_dense_kern},
                 "note": "the three steps interleaved (one of each per round), clocks in clocks_interleaved"}

    # ---- end to end through the C ABI from pinned host buffers: atf_prefill_host
    # uploads q, k, v, rotates and attends query chunks of 8192 rows as they land,
    # and downloads each chunk's output, copies overlapped with each other and with
    # the kernels
    q_h, k_h, v_h = (t.pin_memory() for t in step.host)
    out_h = torch.empty_like(q_h).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = out_h.numel() * out_h.element_size()
    B, S, Hq, d = step.q.shape
    Hkv = step.k.shape[2]
    hws_bytes = atf.atf_prefill_host_workspace_bytes(B, S, S, Hq, Hkv, d, 0)
    del step.out
    torch.cuda.empty_cache()
    hws = torch.empty(hws_bytes, dtype=torch.uint8, device=device)

    def e2e_step(ev):
        if ev:
            ev[0].record(stream)
        atf.atf_prefill_host(q_h, k_h, v_h, out_h, B, S, S, Hq, Hkv, d, 0, 0, w.theta, 1.0, hws, hws_bytes,
                             w.q_chunk, None, s)
        if ev:
            ev[1].record(stream)

    evs_e = time_steps(e2e_step, min(args.steps, 5), args.warmup, stream, flush_buf, n_events=2)
    ms_e2e = dist_max(sum(e[0].elapsed_time(e[1]) for e in evs_e) / len(evs_e))
    e2e_val = world * eff / (ms_e2e * 1e-3) / 1e12
    atf.atf_check(s)
    del hws, step
    torch.cuda.empty_cache()

    extra = {}
    if world == 1 and not args.no_extra:
        extra = run_extra(args, device, stream, flush_buf, peaks)

    ck = clocks.summary()
    sm_mhz = ck.get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    tflops_kern = eff / (ms_kern * 1e-3) / 1e12
    exps = causal_elements(w)
    ex2_rate = exps / (ms_kern * 1e-3)
    ex2_peak = 16 * n_sm * sm_mhz * 1e6
    traffic = recorded_traffic("prefill_tc.cu", "prefill_tc_layer_128k_chunk.md")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded numpy PCG64 N(0,1) -> bf16)",
        "config": headline_config(w, world),
        "speedup_vs_dense": ms_dense / ms_one,
        "kernel_speedup_vs_dense": ms_dense_kern / ms_one_kern,
        "per_alpha": per_alpha,
        "skipped_pairs_per_step": cnt_per_step, "skipped_pairs_closed_form": skipped,
        "roofline": {"bound": "tensor", "achieved": tflops_kern, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tflops_kern / peaks["bf16_tflops"], "traffic": traffic,
                     "kernel": "prefill_tc_kernel<128,sparse>, 16 launches per step", "kernel_ms": ms_kern,
                     "peak_kind": f"{peak_kind} bf16 burst",
                     "peak_sustained": peaks.get("bf16_tflops_sustained"),
                     "frac_sustained": tflops_kern / peaks["bf16_tflops_sustained"]
                     if peaks.get("bf16_tflops_sustained") else None,
                     "dense_kernel_tflops": dense_flops / (ms_dense_kern * 1e-3) / 1e12},
        "sfu_ex2_roof": {"exponentials_per_step": exps, "achieved_per_s": ex2_rate, "peak_per_s": ex2_peak,
                         "frac": ex2_rate / ex2_peak, "sm_mhz": sm_mhz,
                         "peak_basis": f"16 ex2 per clock per SM (measured) x {n_sm} SMs x the median SM clock "
                                       "sampled during the timed steps"},
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": ms_e2e,
                "call": "atf_prefill_host (pinned host buffers, query chunks of 8192 rows, two copy streams)"},
        "gpu_launches": (1 + 2 * (w.seq // w.q_chunk)) * args.steps,  # rope(k), then rope(q) + prefill per chunk
        "clocks": ck,
        "clocks_interleaved": clocks_i.summary(),
        "wall_s_timed_region": t_wall,
    }
    line.update(extra)
    if world == 1 and rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = {k2: v2 for k2, v2 in cpu_oracle_sample(w, 1.0).items() if k2 != "seconds"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_extra(args, device, stream, flush_buf, peaks):
    """Secondary workloads: the 8k layer (alpha sweep against the dense kernel,
    and rotate-half pairs), 32k pair-energy prefill, 1M-key decode, split-KV
    decode, FASA-style decode, KV-cache append."""
    s = stream
    out = {}
    # the 8k layer: alpha sweep, each against the same step with every window open
    w8 = synth.WORKLOADS["layer_8k"]
    st8 = PrefillStep(w8, synth.DEFAULT_SEED, device)
    res8 = {}
    for a in w8.alphas:
        ev8 = time_steps(lambda ev: st8.run(a, s, ev), 10, 3, stream, flush_buf)
        ms8 = sum(e[0].elapsed_time(e[2]) for e in ev8) / len(ev8)
        ms8k = sum(e[1].elapsed_time(e[2]) for e in ev8) / len(ev8)
        f8 = prefill_flops(w8, a)[0] if not math.isinf(a) else prefill_flops(w8, a)[1]
        res8[str(a)] = {"tflops": f8 / (ms8 * 1e-3) / 1e12, "ms": ms8, "kernel_ms": ms8k,
                        "kernel_tflops": f8 / (ms8k * 1e-3) / 1e12}
    res8["speedup_vs_dense_alpha1"] = res8["inf"]["ms"] / res8["1.0"]["ms"]
    res8["kernel_speedup_vs_dense_alpha1"] = res8["inf"]["kernel_ms"] / res8["1.0"]["kernel_ms"]
    res8["kernel_frac_of_peak_alpha1"] = res8["1.0"]["kernel_tflops"] / peaks["bf16_tflops"]
    ev2 = time_steps(lambda ev: st8.run(1.0, s, ev, pairing=atf.ATF_PAIRS_ROTATE_HALF), 5, 3, stream, flush_buf)
    ms2 = sum(e[0].elapsed_time(e[2]) for e in ev2) / 5
    ms2r = sum(e[0].elapsed_time(e[1]) for e in ev2) / 5
    res8["rotate_half_alpha1"] = {"tflops": prefill_flops(w8, 1.0)[0] / (ms2 * 1e-3) / 1e12, "ms": ms2,
                                  "rope_ms": ms2r}
    out["layer_8k"] = res8
    del st8
    torch.cuda.empty_cache()
    # 32k tokens, pair-energy-scaled q/k
    w3 = synth.WORKLOADS["layer_32k_pair_energy"]
    st3 = PrefillStep(w3, synth.DEFAULT_SEED, device)
    ev3 = time_steps(lambda ev: st3.run(1.0, s, ev), 3, 2, stream, flush_buf)
    ev3d = time_steps(lambda ev: st3.run(math.inf, s, ev), 3, 1, stream, flush_buf)
    ms3 = sum(e[0].elapsed_time(e[2]) for e in ev3) / 3
    ms3k = sum(e[1].elapsed_time(e[2]) for e in ev3) / 3
    ms3d = sum(e[0].elapsed_time(e[2]) for e in ev3d) / 3
    eff3 = prefill_flops(w3, 1.0)[0]
    out["layer_32k_pair_energy"] = {"tflops": eff3 / (ms3 * 1e-3) / 1e12, "ms": ms3,
                                    "kernel_frac_of_peak": eff3 / (ms3k * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                    "speedup_vs_dense": ms3d / ms3}
    del st3
    torch.cuda.empty_cache()

    # decode: 4 sequences x 1,048,576 cached keys (device-generated seeded normals)
    w5 = synth.WORKLOADS["decode_1m"]
    g = torch.Generator(device=device)
    g.manual_seed(synth.DEFAULT_SEED)
    N = w5.seq
    kc = torch.randn((w5.batch, w5.kv_heads, w5.d // 16, N, 16), generator=g, device=device).to(torch.bfloat16)
    v5 = torch.randn((w5.batch, N, w5.kv_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    q5 = torch.randn((w5.batch, w5.q_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    o5 = torch.empty_like(q5)
    kv_len = np.full(w5.batch, N, dtype=np.int64)
    ws_b = atf.atf_decode_workspace_bytes(w5.batch, w5.q_heads, w5.kv_heads, N, w5.d)
    ws5 = torch.empty(ws_b, dtype=torch.uint8, device=device)

    def dec(alpha):  # on torch's current stream (the capture stream while a graph is captured)
        atf.atf_decode(q5, kc, v5, o5, w5.batch, kv_len, N, w5.q_heads, w5.kv_heads, w5.d, w5.theta, alpha, ws5,
                       ws_b, None, None)

    dec_w = graphed_step(lambda: dec(1.0), stream)
    dec_d = graphed_step(lambda: dec(math.inf), stream)
    ev5 = time_steps(dec_w, 10, 3, stream, flush_buf, n_events=2)
    ev5d = time_steps(dec_d, 10, 3, stream, flush_buf, n_events=2)
    ms5 = sum(e[0].elapsed_time(e[1]) for e in ev5) / 10
    ms5d = sum(e[0].elapsed_time(e[1]) for e in ev5d) / 10
    del dec_w, dec_d
    act, dense_b = decode_bytes(w5, 1.0)
    moved = decode_moved_bytes(w5, 1.0)
    gbs = act / (ms5 * 1e-3) / 1e9
    out["decode_1m"] = {"GBps_active": gbs, "ms": ms5, "ms_dense": ms5d, "speedup_vs_dense": ms5d / ms5,
                        "active_bytes": act, "dense_bytes": dense_b, "moved_bytes": moved,
                        "GBps_moved": moved / (ms5 * 1e-3) / 1e9,
                        "frac_moved": moved / (ms5 * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "timing": "CUDA graph of the atf_decode call (main kernel + split combine) replayed between "
                                  "the events; L2 flushed between steps",
                        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs / peaks["hbm_gbs"],
                                     "traffic": recorded_traffic("decode.cu", "decode_1m.md")},
                        "data": "seeded torch CUDA normals (torch.Generator), bf16"}

    # split-KV decode: the cache of every sequence split by key position across
    # `world` ranks (traffic-balanced ranges), each rank's partial decode timed on
    # its own copy of its range, plus the merge of the world partials
    from rope_frequency_sparse_b200 import splitkv
    skv = {}
    part = torch.empty((w5.batch, w5.q_heads, w5.d + 2), dtype=torch.float32, device=device)
    for world in (2, 4, 8):
        ranges = splitkv.shard_ranges(N, world, w5.d, w5.theta, 1.0)
        worst = 0.0
        for r in (0, world - 1):  # the ranges farthest from and nearest to the query
            lo, hi = ranges[r]
            kc_r = kc[:, :, :, lo:hi, :].contiguous()
            v_r = v5[:, lo:hi].contiguous()
            need = atf.atf_decode_workspace_bytes(w5.batch, w5.q_heads, w5.kv_heads, hi - lo, w5.d)
            ws_r = torch.empty(need, dtype=torch.uint8, device=device)

            def prt():
                atf.atf_decode_partial(q5, kc_r, v_r, part, w5.batch, [hi - lo] * w5.batch, [lo] * w5.batch,
                                       [N - 1] * w5.batch, hi - lo, w5.q_heads, w5.kv_heads, w5.d, w5.theta, 1.0,
                                       ws_r, need, None, None)

            prt_step = graphed_step(prt, stream)
            evp = time_steps(prt_step, 10, 3, stream, flush_buf, n_events=2)
            del prt_step
            worst = max(worst, sum(e[0].elapsed_time(e[1]) for e in evp) / 10)
            del kc_r, v_r, ws_r
        parts = torch.zeros((world, w5.batch, w5.q_heads, w5.d + 2), dtype=torch.float32, device=device)

        def mrg(ev):
            if ev:
                ev[0].record(stream)
            atf.atf_decode_merge(parts, world, w5.batch, w5.q_heads, w5.d, o5, s)
            if ev:
                ev[1].record(stream)

        evm = time_steps(mrg, 10, 3, stream, flush_buf, n_events=2)
        ms_m = sum(e[0].elapsed_time(e[1]) for e in evm) / 10
        skv[str(world)] = {"ms_rank_partial_max": worst, "ms_merge": ms_m,
                           "speedup_vs_one_gpu_decode_excl_exchange": ms5 / (worst + ms_m),
                           "exchange_bytes_per_rank": w5.batch * w5.q_heads * (w5.d + 2) * 4}
    out["split_kv_decode_1m"] = dict(skv, note="per-rank partials timed one at a time on one GPU (the first and "
                                               "last key ranges); the all-gather of the partials between GPUs is "
                                               "not measured here")

    # FASA-style decode on the same cache: token scores on the 16 lowest-frequency
    # pairs (two 8-pair chunks), 2048 keys kept per query head, attention on those
    mask16, budget = 0xFFFF << 48, 2048
    fws_b = atf.atf_fasa_workspace_bytes(w5.batch, w5.q_heads, N, budget, w5.d)
    fws = torch.empty(fws_b, dtype=torch.uint8, device=device)

    def fas():  # on torch's current stream (the capture stream while a graph is captured)
        atf.atf_fasa_decode(q5, kc, v5, o5, w5.batch, kv_len, N, w5.q_heads, w5.kv_heads, w5.d, mask16, budget,
                            None, None, fws, fws_b, None)

    fas_step = graphed_step(fas, stream)
    ev8 = time_steps(fas_step, 10, 3, stream, flush_buf, n_events=2)
    del fas_step
    ms8 = sum(e[0].elapsed_time(e[1]) for e in ev8) / 10
    # algorithmic bytes: the dominant pairs of every key (4 B per pair, key and kv
    # head), the kept keys' K and V rows, q and out; "moved" adds the sampled keys'
    # dominant chunks read again by the threshold sample (one key in 32)
    alg8 = (w5.batch * w5.kv_heads * N * 16 * 4 + w5.batch * w5.q_heads * budget * w5.d * 2 * 2
            + 2 * w5.batch * w5.q_heads * w5.d * 2)
    moved8 = alg8 + w5.batch * w5.kv_heads * N * 16 * 4 // 32
    gbs8 = alg8 / (ms8 * 1e-3) / 1e9
    out["fasa_1m"] = {"ms": ms8, "speedup_vs_windowed_decode": ms5 / ms8, "speedup_vs_dense_decode": ms5d / ms8,
                      "timing": "CUDA graph of the atf_fasa_decode call (seven launches) replayed between the events; "
                                "L2 flushed between steps",
                      "GBps_algorithmic": gbs8, "GBps_moved": moved8 / (ms8 * 1e-3) / 1e9,
                      "algorithmic_bytes": alg8, "moved_bytes": moved8,
                      "config": f"{w5.batch} x {N} cached keys, 28/4 heads, d=128, 16 dominant pairs, "
                                f"budget {budget} keys per query head",
                      "roofline": {"bound": "hbm", "achieved": gbs8, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                   "frac": gbs8 / peaks["hbm_gbs"]}}

    # KV-cache append into the same caches: a bulk append of 32768 new tokens per
    # sequence (varlen positions) and a decode step's one new token per sequence
    n_bulk = 32768
    kn = torch.randn((w5.batch * n_bulk, w5.kv_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    vn = torch.randn((w5.batch * n_bulk, w5.kv_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    pos_bulk = [0, N // 3, N // 2, N - n_bulk][: w5.batch]

    def app(ev, n, pos):
        if ev:
            ev[0].record(stream)
        atf.atf_kv_append(kn, vn, kc, v5, w5.batch, [n] * w5.batch, pos, N, w5.kv_heads, w5.d, w5.theta, 0, s)
        if ev:
            ev[1].record(stream)

    ev6 = time_steps(lambda ev: app(ev, n_bulk, pos_bulk), 10, 3, stream, flush_buf, n_events=2)
    ms6 = sum(e[0].elapsed_time(e[1]) for e in ev6) / 10
    bytes6 = 4 * w5.batch * n_bulk * w5.kv_heads * w5.d * 2  # read k, v; write both caches
    ev7 = time_steps(lambda ev: app(ev, 1, [N - 1] * w5.batch), 10, 3, stream, flush_buf, n_events=2)
    us7 = sum(e[0].elapsed_time(e[1]) for e in ev7) / 10 * 1e3
    out["kv_append"] = {"GBps_bulk": bytes6 / (ms6 * 1e-3) / 1e9, "ms_bulk": ms6,
                        "bulk": f"{w5.batch} sequences x {n_bulk} new tokens, 28/4 heads, d=128",
                        "roofline": {"bound": "hbm", "achieved": bytes6 / (ms6 * 1e-3) / 1e9,
                                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": bytes6 / (ms6 * 1e-3) / 1e9 / peaks["hbm_gbs"]},
                        "us_decode_step_append": us7}
    atf.atf_check(s)
    return out


def run_chunk_profile(args):
    """Only the last query chunk of the 131072-token layer (the heaviest launch of
    the headline step): ROWS query rows ending at position 131071 against all
    131072 keys, windowed (alpha = 1) then dense, W + K prefill launches each, for
    ncu captures.  Inputs are seeded device normals of the workload's shapes."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w = synth.WORKLOADS[HEADLINE]
    S, C = w.seq, args.profile_chunk
    g = torch.Generator(device=device)
    g.manual_seed(synth.DEFAULT_SEED)
    q = torch.randn((1, C, w.q_heads, w.d), generator=g, device=device).to(torch.bfloat16)
    k = torch.randn((1, S, w.kv_heads, w.d), generator=g, device=device).to(torch.bfloat16)
    v = torch.randn((1, S, w.kv_heads, w.d), generator=g, device=device).to(torch.bfloat16)
    s = torch.cuda.current_stream()
    q_rot, k_rot, out = torch.empty_like(q), torch.empty_like(k), torch.empty_like(q)
    atf.atf_rope_layout(k, k_rot, None, 1, S, w.kv_heads, w.d, 0, w.theta, 1, atf.ATF_BF16, s)
    atf.atf_rope_layout(q, q_rot, None, 1, C, w.q_heads, w.d, S - C, w.theta, 1, atf.ATF_BF16, s)
    res = {}
    for alpha in (1.0, math.inf):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for it in range(args.warmup + args.steps):
            if it == args.warmup:
                e0.record(s)
            atf.atf_prefill_ex(q_rot, k_rot, v, out, 1, C, S, w.q_heads, w.kv_heads, w.d, S - C, atf.ATF_BF16, 1,
                               w.theta, alpha, None, None, 0, s)
        e1.record(s)
        atf.atf_check(s)
        res[str(alpha)] = e0.elapsed_time(e1) / max(args.steps, 1)
    print(json.dumps({"profile": "prefill_chunk", "query_rows": C, "keys": S, "launches_per_alpha":
                      args.warmup + args.steps, "ms_per_launch": res}))


def run_decode_profile(args):
    """Only the decode step (alpha = 1) with a shortened cache, for ncu captures:
    the decode_1m shapes with KEYS cached keys per sequence, W + K launches."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w5 = synth.WORKLOADS["decode_1m"]
    N = args.profile_decode
    g = torch.Generator(device=device)
    g.manual_seed(synth.DEFAULT_SEED)
    kc = torch.randn((w5.batch, w5.kv_heads, w5.d // 16, N, 16), generator=g, device=device).to(torch.bfloat16)
    v5 = torch.randn((w5.batch, N, w5.kv_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    q5 = torch.randn((w5.batch, w5.q_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    o5 = torch.empty_like(q5)
    kv_len = np.full(w5.batch, N, dtype=np.int64)
    ws_b = atf.atf_decode_workspace_bytes(w5.batch, w5.q_heads, w5.kv_heads, N, w5.d)
    ws5 = torch.empty(ws_b, dtype=torch.uint8, device=device)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for it in range(args.warmup + args.steps):
        if it == args.warmup:
            e0.record(s)
        atf.atf_decode(q5, kc, v5, o5, w5.batch, kv_len, N, w5.q_heads, w5.kv_heads, w5.d, w5.theta, 1.0, ws5,
                       ws_b, None, s)
    e1.record(s)
    atf.atf_check(s)
    print(json.dumps({"profile": "decode", "keys": N, "batch": w5.batch, "launches": args.warmup + args.steps,
                      "ms_per_step": e0.elapsed_time(e1) / max(args.steps, 1)}))


def run_fasa_profile(args):
    """Only the FASA-style decode with a shortened cache, for ncu captures: one
    sequence of KEYS cached keys, 28/4 heads, d = 128, the 16 lowest-frequency
    pairs dominant, 2048 keys kept per query head; W + K calls."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w5 = synth.WORKLOADS["decode_1m"]
    N, B = args.profile_fasa, 1
    g = torch.Generator(device=device)
    g.manual_seed(synth.DEFAULT_SEED)
    kc = torch.randn((B, w5.kv_heads, w5.d // 16, N, 16), generator=g, device=device).to(torch.bfloat16)
    v5 = torch.randn((B, N, w5.kv_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    q5 = torch.randn((B, w5.q_heads, w5.d), generator=g, device=device).to(torch.bfloat16)
    o5 = torch.empty_like(q5)
    budget = 2048
    ws_b = atf.atf_fasa_workspace_bytes(B, w5.q_heads, N, budget, w5.d)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=device)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for it in range(args.warmup + args.steps):
        if it == args.warmup:
            e0.record(s)
        atf.atf_fasa_decode(q5, kc, v5, o5, B, [N], N, w5.q_heads, w5.kv_heads, w5.d, 0xFFFF << 48, budget, None,
                            None, ws, ws_b, s)
    e1.record(s)
    atf.atf_check(s)
    print(json.dumps({"profile": "fasa", "keys": N, "batch": B, "calls": args.warmup + args.steps,
                      "ms_per_call": e0.elapsed_time(e1) / max(args.steps, 1)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="only the headline workload")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--profile-decode", type=int, metavar="KEYS", default=0,
                    help="run only the decode step with KEYS cached keys per sequence (for ncu captures)")
    ap.add_argument("--profile-chunk", type=int, metavar="ROWS", default=0,
                    help="run only the last ROWS query rows of the 131072-token layer (for ncu captures)")
    ap.add_argument("--profile-fasa", type=int, metavar="KEYS", default=0,
                    help="run only the FASA-style decode on one sequence of KEYS keys (for ncu captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.profile_decode:
        run_decode_profile(args)
        return
    if args.profile_chunk:
        run_chunk_profile(args)
        return
    if args.profile_fasa:
        run_fasa_profile(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
