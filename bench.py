"""Benchmark of the Gated DeltaNet mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (one "step"): one decode token through the GDN layers of a
Qwen3.5-0.8B-shaped model -- 18 independent layer states, batch 32, 16 key and
16 value heads, d_k = d_v = 128, bf16 q/k/v/z and outputs, fp32 state,
S_0 ~ N(0, 0.02).  Each step launches the decode kernel once per layer (18
launches, replayed from one CUDA graph per step).  Inputs are seeded and
synthetic, drawn on the GPU; the 18 layer states (604 MB) rotate through HBM,
far more than the 126 MB L2, so no step finds its state in L2.

Metric: GB/s of algorithmic bytes (per (sequence, value head) and token: the
fp32 state read and written once, q/k per key head, v/z/g/beta read once, the
output written once).  The JSON line also carries the roofline of the decode
kernel, a clock record of the timed region, an end-to-end figure through the
same C ABI with inputs copied from pinned host memory every step, the
chunked-prefill throughput (Qwen3.5-0.8B-shaped prefill: 4 x 4096 tokens,
16 heads), and the fp64 CPU oracle timed on this host on a bounded sample.

With N > 1 (torchrun), every rank runs the same workload on its own GPU
(weak scaling: the batch grows with N, no data exchange between ranks); the
timed region is bracketed by barriers and the maximum over ranks is used.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Workload: Qwen3.5-0.8B-shaped GDN decode.
LAYERS, BATCH, H_K, H_V, D = 18, 32, 16, 16, 128
SLOTS = 512  # distinct per-step inputs (the workload's 512 decode steps), cycled
IN_BYTES, OUT_BYTES = 2, 2
# Chunked prefill (reported beside the headline): Qwen3.5-0.8B-shaped prompt batch.
P_SEQS, P_LEN, P_H, P_CHUNK = 4, 4096, 16, 64

HEADLINE = "GDN decode state-update GB/s"


def decode_bytes_per_layer_step(B, H_k, H_v, d, in_b=IN_BYTES, out_b=OUT_BYTES) -> int:
    per_value_head = 2 * d * d * 4 + 2 * d * in_b + 2 * 4 + d * out_b  # state r+w, v, z, g, beta, out
    per_key_head = 2 * d * in_b                                       # q, k
    return B * H_v * per_value_head + B * H_k * per_key_head


def decode_bytes_per_layer_call(B, H_k, H_v, d, T, in_b=IN_BYTES, out_b=OUT_BYTES) -> int:
    """Algorithmic bytes of one multi-token call over B sequences x T tokens:
    the state once, the per-token inputs and outputs T times."""
    state = B * H_v * 2 * d * d * 4
    per_token = decode_bytes_per_layer_step(B, H_k, H_v, d, in_b, out_b) - state
    return state + T * per_token


def prefill_flops_per_token_head(C, d, gva: bool) -> int:
    # K K^T, Q K^T, U, W, P Delta at 2 C d each; W S^T, Q S^T, state update at 2 d^2 each.
    kk_qk = 0 if gva else 4 * C * d
    return kk_qk + 6 * C * d + 6 * d * d


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def captured_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu capture of `kernel`, or None if
    there is none or the kernel's source has changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    return rec["dram_bytes_per_launch"] if digest.startswith(rec["sha256_prefix"]) else None


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return None
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.strip().split(", ") for r in f if r.strip()]
        os.unlink(self.file.name)
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        loaded = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()
                  and r[3].replace(".", "").isdigit() and float(r[3]) > 200.0] or sm
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded)}


# ----------------------------------------------------------------- decode

class DecodeBench:
    def __init__(self, device, seed=1, B=BATCH, layers=LAYERS, slots=SLOTS):
        import linear_attention_recurrence_10_b200 as gdr
        from linear_attention_recurrence_10_b200 import synth
        self.gdr = gdr
        self.B, self.L, self.T = B, layers, slots
        x = synth.make_decode_inputs(layers, slots, B, H_K, H_V, D, seed=seed, s0_std=0.02,
                                     device=device)
        self.x = x
        self.state = x.s0.clone()
        self.out = torch.empty(layers, B, H_V, D, device=device, dtype=torch.bfloat16)
        self.graphs = []
        self.overlap = layers > 1
        self.bytes_per_step = layers * decode_bytes_per_layer_step(B, H_K, H_V, D)
        self.launches_per_step = layers

    def launch_layer(self, l, t, x=None, out=None):
        x = x or self.x
        out = self.out if out is None else out
        # Consecutive launches touch different layers' states, so each may
        # start loading its state while the previous layer's kernel drains.
        self.gdr.decode_step(x.q[l, t], x.k[l, t], x.v[l, t], x.g[l, t], x.beta[l, t],
                             self.state[l], out[l], z=x.z[l, t], norm_w=x.w,
                             overlap_state_load=self.overlap)

    def launch_step(self, t, x=None, out=None):
        for l in range(self.L):
            self.launch_layer(l, t, x, out)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.launch_step(0)  # load the library and kernels before capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for t in range(self.T):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.launch_step(t)
            self.graphs.append(g)
        torch.cuda.synchronize()

    def run(self, first, n):
        for s in range(first, first + n):
            self.graphs[s % self.T].replay()


class DecodeE2E:
    """Same steps through the same C ABI, with every step's inputs copied in from
    pinned host memory and its outputs copied back.

    Each step is one CUDA graph (how a serving loop replays a decode step
    without paying the Python binding's per-call cost): on a side stream it
    copies the NEXT step's inputs into the other of two device input buffers,
    while on the main stream its own 18 library calls read the inputs the
    previous step copied, then its output is copied back.  So every step moves
    one step's inputs and outputs, and the copies overlap the kernels."""

    def __init__(self, bench: DecodeBench, host_slots=16):
        self.b = bench
        x = bench.x
        # An even number of slots, so that a slot fixes its input buffer.
        n = max(1, min(host_slots, bench.T))
        idx = list(range(n)) + ([0] if n % 2 else [])
        self.host_slots = len(idx)
        pin = lambda t: t[:, idx].transpose(0, 1).contiguous().cpu().pin_memory()
        # host tensors [slot, L, ...]
        self.h = {n: pin(getattr(x, n)) for n in ("q", "k", "v", "z", "g", "beta")}
        dev = x.q.device
        self.d = [{n: torch.empty_like(t[0], device=dev) for n, t in self.h.items()}
                  for _ in range(2)]
        self.h_out = torch.empty(bench.out.shape, dtype=bench.out.dtype).pin_memory()
        self.h2d_bytes = sum(t[0].numel() * t[0].element_size() for t in self.h.values())
        self.d2h_bytes = self.h_out.numel() * self.h_out.element_size()
        import types
        self.view = [types.SimpleNamespace(
            q=d["q"].unsqueeze(1), k=d["k"].unsqueeze(1), v=d["v"].unsqueeze(1),
            z=d["z"].unsqueeze(1), g=d["g"].unsqueeze(1), beta=d["beta"].unsqueeze(1), w=x.w)
            for d in self.d]

    def _copy_in(self, slot):
        for n, t in self.h.items():
            self.d[slot % 2][n].copy_(t[slot], non_blocking=True)

    def _enqueue(self, slot):
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self._copy_in((slot + 1) % self.host_slots)
        self.b.launch_step(0, x=self.view[slot % 2])
        self.h_out.copy_(self.b.out, non_blocking=True)
        main.wait_stream(self.side)

    def capture(self):
        self.side = torch.cuda.Stream()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self._copy_in(0)
            self._enqueue(0)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graphs = []
        for slot in range(self.host_slots):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._enqueue(slot)
            self.graphs.append(g)
        torch.cuda.synchronize()
        self._copy_in(0)  # the first replayed step's inputs
        torch.cuda.synchronize()

    def step(self, s):
        self.graphs[s % self.host_slots].replay()


def time_region(fn, n, ranks):
    """CUDA-event time of fn() over a barrier-bracketed region; max over ranks (ms)."""
    if ranks > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    torch.cuda.synchronize()
    if ranks > 1:
        torch.distributed.barrier()
    from linear_attention_recurrence_10_b200.ranks import max_over_ranks
    return max_over_ranks(e0.elapsed_time(e1), ranks, device="cuda")


def decode_batch_sweep(device, batches=(1, 2, 4, 8, 16, 32), steps=64, warmup=4, slots=32,
                       world=1):
    """The headline step (18 layers, 16/16 heads, d=128) at each batch size.
    Where the 18 layer states (18 x B x 1 MiB) total less than twice the L2,
    L2 is flushed (a 256 MB write) before every step and each step is timed
    on its own with CUDA events, so no step finds its state in L2; larger
    batches rotate more state than L2 holds and are timed as one region."""
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    res = {}
    for B in batches:
        bench = DecodeBench(device, seed=20 + B, B=B, slots=slots)
        bench.capture()
        bench.run(0, warmup)
        state_bytes = LAYERS * B * H_V * D * D * 4
        flushed = state_bytes < 2 * l2
        if flushed:
            ms = 0.0
            for s in range(steps):
                flush.zero_()
                ms += time_region(lambda: bench.run(warmup + s, 1), 1, world)
        else:
            ms = time_region(lambda: bench.run(warmup, steps), steps, world)
        res[str(B)] = {"value": bench.bytes_per_step * steps / (ms * 1e-3) / 1e9, "unit": "GB/s",
                       "us_per_launch": ms * 1e3 / (steps * LAYERS),
                       "l2": "flushed before every step" if flushed else "states exceed L2"}
        del bench
        torch.cuda.empty_cache()
    return res


def decode_variants(device, B, steps=64, warmup=4, slots=32, T=4, world=1):
    """Two more views of the headline decode workload (18 layers x B, 16/16
    heads, d=128), each timed on its own inputs with the states rotating
    through HBM:
    - layer-folded: the 18 layers' states as one batch of 18*B rows, one
      launch per step (the kernel without per-launch ramp and tail);
    - multi-token: T tokens per sequence per call (gdr_decode_multi), 18
      launches per call, the state read and written once per call."""
    import linear_attention_recurrence_10_b200 as gdr
    from linear_attention_recurrence_10_b200 import synth
    res = {}
    # Layer-folded single launch.
    x = synth.make_decode_inputs(LAYERS, slots, B, H_K, H_V, D, seed=11, s0_std=0.02, device=device)
    fold = lambda t: t.transpose(0, 1).contiguous().view(slots, LAYERS * B, *t.shape[3:])
    q, k, v, z, g, beta = (fold(t) for t in (x.q, x.k, x.v, x.z, x.g, x.beta))
    state = x.s0.view(LAYERS * B, H_V, D, D)
    out = torch.empty(LAYERS * B, H_V, D, device=device, dtype=torch.bfloat16)
    del x

    def fold_step(s):
        t = s % slots
        gdr.decode_step(q[t], k[t], v[t], g[t], beta[t], state, out, z=z[t], norm_w=None)

    for s in range(warmup):
        fold_step(s)
    ms = time_region(lambda: [fold_step(warmup + s) for s in range(steps)], steps, world)
    nbytes = LAYERS * decode_bytes_per_layer_step(B, H_K, H_V, D)
    res["layer_folded"] = {
        "value": nbytes * steps / (ms * 1e-3) / 1e9, "unit": "GB/s", "steps": steps,
        "us_per_launch": ms * 1e3 / steps, "launch": f"one launch per step over {LAYERS}x{B} rows",
        "tokens_per_s": B * steps / (ms * 1e-3)}
    del q, k, v, z, g, beta, state, out
    # Multi-token calls.
    x = synth.make_decode_inputs(LAYERS, slots * T, B, H_K, H_V, D, seed=12, s0_std=0.02,
                                 device=device)
    # [L, calls, T, B, ...] -> [L, calls, B, T, ...]: each call's rows are b*T + t.
    per_call = lambda t: t.view(LAYERS, slots, T, B, *t.shape[3:]).transpose(2, 3).contiguous() \
        .view(LAYERS, slots, B * T, *t.shape[3:])
    q, k, v, z, g, beta = (per_call(t) for t in (x.q, x.k, x.v, x.z, x.g, x.beta))
    state = x.s0
    out = torch.empty(B * T, H_V, D, device=device, dtype=torch.bfloat16)
    del x

    def enqueue_call(c):
        for l in range(LAYERS):
            gdr.decode_multi(q[l, c], k[l, c], v[l, c], g[l, c], beta[l, c], state[l], out,
                             n_tokens=T, z=z[l, c], overlap_state_load=True)

    # One CUDA graph per call, as for the headline (the binding's per-call host
    # cost would otherwise exceed the kernels' time).
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        enqueue_call(0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for c in range(slots):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            enqueue_call(c)
        graphs.append(gr)

    def multi_call(s):
        graphs[s % slots].replay()

    for s in range(warmup):
        multi_call(s)
    ms = time_region(lambda: [multi_call(warmup + s) for s in range(steps)], steps, world)
    nbytes = LAYERS * decode_bytes_per_layer_call(B, H_K, H_V, D, T)
    res["batch_sweep"] = decode_batch_sweep(device, world=world)
    res["multi_token"] = {
        "value": nbytes * steps / (ms * 1e-3) / 1e9, "unit": "GB/s", "tokens_per_call": T,
        "tokens_per_s": B * T * steps / (ms * 1e-3), "us_per_launch": ms * 1e3 / (steps * LAYERS),
        "launch": f"{LAYERS} launches per call, {T} tokens per sequence each, one CUDA graph per call"}
    del graphs
    return res


# ---------------------------------------------------------------- prefill

def prefill_measure(device, reps=5, world=1):
    import linear_attention_recurrence_10_b200 as gdr
    from linear_attention_recurrence_10_b200 import synth
    inp = synth.make_inputs([P_LEN] * P_SEQS, P_H, P_H, D, seed=2, device=device)
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device=device)
    out = torch.empty(inp.n_tok, P_H, D, device=device, dtype=torch.bfloat16)
    final = torch.empty(P_SEQS, P_H, D, D, device=device)
    ws_bytes = gdr.prefill_workspace_size(inp.q, inp.k, inp.v, inp.g, inp.beta, cu, out,
                                          cu_seqlens_host=inp.cu_seqlens, z=inp.z, chunk=P_CHUNK)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)

    def call():
        gdr.prefill_chunked(inp.q, inp.k, inp.v, inp.g, inp.beta, cu, out,
                            cu_seqlens_host=inp.cu_seqlens, z=inp.z, norm_w=inp.w,
                            final_state=final, chunk=P_CHUNK, workspace=ws)

    for _ in range(2):
        call()
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    times = []
    for _ in range(reps):
        flush.zero_()  # evict L2 between repetitions
        times.append(time_region(call, 1, world))  # max over ranks
    ms = statistics.median(times)
    n_tok = inp.n_tok * world
    flops = n_tok * P_H * prefill_flops_per_token_head(P_CHUNK, D, gva=False)
    per_gpu_tflops = flops / world / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    return {"metric": "chunked-prefill tokens/s", "value": n_tok / (ms * 1e-3), "unit": "tokens/s",
            "ms": ms, "workload": f"Qwen3.5-0.8B-shaped prefill: {P_SEQS} x {P_LEN} tokens, "
                                  f"{P_H}/{P_H} heads, d={D}, bf16, chunk {P_CHUNK}, S_0=0",
            "n_gpus": world, "scaling": "weak",
            "tflops": tflops, "tc_frac": per_gpu_tflops / peaks["bf16_tflops"],
            "tc_peak_tflops": peaks["bf16_tflops"], "flops_per_token_head":
                prefill_flops_per_token_head(P_CHUNK, D, gva=False),
            "l2": "flushed (256 MB write) before each repetition", "reps": reps}


# ------------------------------------------------------------- CPU oracle

def oracle_sample(n_tokens=512, seed=1, threads=None):
    """Time the fp64 oracle on one layer of the decode workload: B sequences x
    16 heads x n_tokens steps, on every host core."""
    import numpy as np
    import oracle
    from linear_attention_recurrence_10_b200 import synth
    threads = threads or os.cpu_count() or 1
    inp = synth.make_inputs([n_tokens] * BATCH, H_K, H_V, D, seed=seed, s0_std=0.02)
    f = lambda t: t.to(torch.float64).numpy()
    args = dict(q=f(inp.q), k=f(inp.k), v=f(inp.v), g=f(inp.g), beta=f(inp.beta),
                cu_seqlens=np.array(inp.cu_seqlens), z=f(inp.z), s0=f(inp.s0), w=f(inp.w))
    t0 = time.perf_counter()
    oracle.gdr_recurrent(**args, threads=threads)
    dt = time.perf_counter() - t0
    nbytes = n_tokens * decode_bytes_per_layer_step(BATCH, H_K, H_V, D)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": dt,
            "sample": f"one layer of the decode workload: {BATCH} sequences x {H_V} heads x "
                      f"{n_tokens} tokens, fp64 recurrence, {threads} threads"}


def run_reference(args, rank, world):
    """The fp64 oracle as the reference arm: each step is one decode token of one
    layer for a sample of the batch's (sequence, head) pairs, on the host cores."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    from linear_attention_recurrence_10_b200 import synth
    threads = os.cpu_count() or 1
    inp = synth.make_inputs([SLOTS] * BATCH, H_K, H_V, D, seed=1, s0_std=0.02)
    f = lambda t: t.to(torch.float64).numpy()
    q, k, v, z = (f(t).reshape(BATCH, SLOTS, -1, D) for t in (inp.q, inp.k, inp.v, inp.z))
    g, beta = (f(t).reshape(BATCH, SLOTS, H_V) for t in (inp.g, inp.beta))
    state = f(inp.s0)
    w = f(inp.w)
    cu = np.arange(BATCH + 1, dtype=np.int64)
    lib = oracle.load()

    def step(s):
        nonlocal state
        t = s % SLOTS
        r = oracle.gdr_recurrent(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], cu, z=z[:, t],
                                 s0=state, w=w, threads=threads, lib=lib)
        state = r.state

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(args.warmup + s)
    dt = time.perf_counter() - t0
    nbytes = args.steps * decode_bytes_per_layer_step(BATCH, H_K, H_V, D)
    value = nbytes / dt / 1e9
    sample = (f"one decode token of one layer per step: {BATCH} sequences x {H_V} heads, "
              f"fp64 recurrence, {threads} threads")
    line = {"impl": "reference", "metric": HEADLINE, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "Qwen3.5-0.8B-shaped GDN decode (oracle sample)",
                       "global_batch": BATCH, "seq_len": 1, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=8192)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--batch", type=int, default=BATCH)
    ap.add_argument("--slots", type=int, default=SLOTS,
                    help="distinct per-step inputs, cycled (fewer holds less device memory)")
    ap.add_argument("--e2e-steps", type=int, default=1024)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-variants", action="store_true")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the chunked-prefill measurement and print its JSON (profiling)")
    ap.add_argument("--prefill-reps", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    from linear_attention_recurrence_10_b200.ranks import rank_env, weak_scaling_rate
    env = rank_env()
    world, rank, local = env.world, env.rank, env.local
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=device,
                                             timeout=datetime.timedelta(seconds=120))

    from linear_attention_recurrence_10_b200 import build
    build.build(quiet=True)
    if args.prefill_only:
        pre = prefill_measure(device, reps=args.prefill_reps, world=world)
        if rank == 0:
            print(json.dumps(pre), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    bench = DecodeBench(device, seed=1 + rank, B=args.batch, slots=args.slots)
    bench.capture()
    bench.run(0, args.warmup)
    torch.cuda.synchronize()
    visible = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    gpu_index = int(visible[local]) if local < len(visible) and visible[local].isdigit() else local
    with ClockSampler(gpu_index) as clocks:
        ms = time_region(lambda: bench.run(args.warmup, args.steps), args.steps, world)
    clock_info = clocks.summary()

    peaks = load_peaks()
    gbs = weak_scaling_rate(bench.bytes_per_step * args.steps, world, ms) / 1e9
    per_launch_ms = ms / (args.steps * bench.launches_per_step)
    per_launch_bytes = decode_bytes_per_layer_step(args.batch, H_K, H_V, D)
    achieved = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9

    # End to end through the same ABI with host buffers.
    e2e = DecodeE2E(bench)
    e2e.capture()
    for s in range(4):
        e2e.step(s)
    ms_e2e = time_region(lambda: [e2e.step(4 + s) for s in range(args.e2e_steps)],
                         args.e2e_steps, world)  # consecutive with the warm-up steps
    e2e_gbs = weak_scaling_rate(bench.bytes_per_step * args.e2e_steps, world, ms_e2e) / 1e9

    # Free the headline's inputs before the extra decode views allocate theirs.
    launches_per_step, h2d_bytes, d2h_bytes = bench.launches_per_step, e2e.h2d_bytes, e2e.d2h_bytes
    del e2e, bench
    torch.cuda.empty_cache()
    variants = None if args.no_decode_variants else decode_variants(device, args.batch, world=world)
    prefill = None if args.no_prefill else prefill_measure(device, reps=args.prefill_reps,
                                                           world=world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample()

    line = {
        "metric": HEADLINE, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": f"Qwen3.5-0.8B-shaped GDN decode: {LAYERS} layers x B={args.batch}, "
                        f"{H_K}/{H_V} heads, d={D}, bf16 q/k/v/z/out, fp32 state and math",
            "global_batch": args.batch * world, "seq_len": 1, "layers": LAYERS,
            "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2: {LAYERS} layer states "
                  f"({LAYERS * args.batch * H_V * D * D * 4 / 1e6:.0f} MB) rotate every step",
            "launch": "one CUDA graph per step (one decode launch per layer)"},
        "tokens_per_s": weak_scaling_rate(args.batch * args.steps, world, ms),
        "hbm_frac": gbs / world / peaks["hbm_gbs"],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": captured_traffic("decode_kernel<128, bf16, bf16, false>"),
                     "kernel": "decode_kernel<128, bf16, bf16, false>",
                     "bytes_per_launch": per_launch_bytes, "us_per_launch": per_launch_ms * 1e3,
                     "peak_source": peaks["source"] + " (hbm_gbs, of measured copy bandwidth)"},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes, "steps": args.e2e_steps,
                "launch": "one CUDA graph per step: the 18 library calls on inputs the previous "
                          "step copied from pinned host memory, the next step's inputs copied "
                          "in meanwhile, the outputs copied back",
                "ms_per_step": ms_e2e / args.e2e_steps},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clock_info,
        "decode_variants": variants,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
