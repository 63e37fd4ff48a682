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
SLOTS = 512  # the workload's decode steps: the reference arm's distinct per-step inputs
# Device-resident per-step input sets of the decode benchmarks, cycled: 32 sets
# of the 18 layers' inputs are 0.3 GB, well past L2, so every step reads its
# inputs (and all 18 states) from DRAM.  512 sets (4.7 GB of inputs beside
# 1.2 GB of state) made each launch 7-12% slower through the footprint alone,
# which a serving loop writing each step's inputs into the same buffers does
# not have.
INPUT_SETS = 32
IN_BYTES, OUT_BYTES = 2, 2
# Chunked prefill (reported beside the headline): Qwen3.5-0.8B-shaped prompt batch.
P_SEQS, P_LEN, P_H, P_CHUNK = 4, 4096, 16, 64
# Qwen3.6-35B-A3B-shaped GVA decode: 30 GDN layers' states, batch 64, 16 key /
# 32 value heads, 256 distinct decode steps.
GVA_LAYERS, GVA_B, GVA_HK, GVA_HV, GVA_STEPS = 30, 64, 16, 32, 256
# Qwen3.6-35B-A3B-shaped gated full-attention decode: its 10 attention layers
# (one mixer in four of 40), batch 64, 16 query / 2 key-value heads, head_dim
# 256, 4096 cached tokens per sequence, rotary embedding on 64 dims, theta 1e7.
ATT_LAYERS, ATT_B, ATT_HQ, ATT_HKV, ATT_D, ATT_CTX, ATT_ROT = 10, 64, 16, 2, 256, 4096, 64
# Qwen3.6-35B-A3B-shaped routed-expert MoE block at decode: hidden 2048, 256
# experts, top 8, expert and shared intermediate 512; 8 layers' weights (12.7 GB
# in bf16) rotate, one token per step (the pages' single-sequence decode).
MOE_LAYERS, MOE_H, MOE_E, MOE_K, MOE_I, MOE_SI = 8, 2048, 256, 8, 512, 512
# Long-context GVA prefill: 8 sequences of U{1024..32768} tokens (seed 4),
# 16 key / 32 value heads, exp(g) in [0.9, 1).
LC_SEQS, LC_LO, LC_HI, LC_HK, LC_HV, LC_SEED = 8, 1024, 32768, 16, 32, 4

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


def prefill_flops_per_token_head(C, d, hv_per_hk: int = 1) -> int:
    """Algorithmic FLOPs per (token, value head): K K^T, Q K^T, U, W, P Delta at
    2 C d each, W S^T, Q S^T and the state update at 2 d^2 each; K K^T and
    Q K^T belong to the key head, so value heads sharing it share them."""
    return 4 * C * d // hv_per_hk + 6 * C * d + 6 * d * d


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
    """One decode token through `layers` independent layer states per step, one
    library call per layer, replayed from one CUDA graph per step."""

    def __init__(self, device, seed=1, B=BATCH, layers=LAYERS, slots=INPUT_SETS, H_k=H_K, H_v=H_V):
        import linear_attention_recurrence_10_b200 as gdr
        from linear_attention_recurrence_10_b200 import synth
        self.gdr = gdr
        self.B, self.L, self.T = B, layers, slots
        x = synth.make_decode_inputs(layers, slots, B, H_k, H_v, D, seed=seed, s0_std=0.02,
                                     device=device)
        self.x = x
        self.state = x.s0.clone()
        self.out = torch.empty(layers, B, H_v, D, device=device, dtype=torch.bfloat16)
        self.graphs = []
        self.overlap = layers > 1
        self.bytes_per_launch = decode_bytes_per_layer_step(B, H_k, H_v, D)
        self.bytes_per_step = layers * self.bytes_per_launch
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


class DecodeMultiBench:
    """The headline layers with T tokens per sequence per call (gdr_decode_multi):
    each call-step runs the 18 layers once, every launch with
    GDR_DECODE_OVERLAP_STATE_LOAD, replayed from one CUDA graph per call-step.
    The state is read and written once per call whatever T."""

    def __init__(self, device, seed=12, B=BATCH, layers=LAYERS, slots=32, T=4):
        import linear_attention_recurrence_10_b200 as gdr
        from linear_attention_recurrence_10_b200 import synth
        self.gdr = gdr
        self.B, self.L, self.T, self.slots = B, layers, T, slots
        x = synth.make_decode_inputs(layers, slots * T, B, H_K, H_V, D, seed=seed, s0_std=0.02,
                                     device=device)
        # [L, calls, T, B, ...] -> [L, calls, B, T, ...]: each call's rows are b*T + t.
        per_call = lambda t: t.view(layers, slots, T, B, *t.shape[3:]).transpose(2, 3) \
            .contiguous().view(layers, slots, B * T, *t.shape[3:])
        self.q, self.k, self.v, self.z, self.g, self.beta = (
            per_call(t) for t in (x.q, x.k, x.v, x.z, x.g, x.beta))
        self.w = x.w
        self.state = x.s0
        self.out = torch.empty(layers, B * T, H_V, D, device=device, dtype=torch.bfloat16)
        self.graphs = []
        self.bytes_per_call = layers * decode_bytes_per_layer_call(B, H_K, H_V, D, T)

    def enqueue_call(self, c):
        for l in range(self.L):
            self.gdr.decode_multi(self.q[l, c], self.k[l, c], self.v[l, c], self.g[l, c],
                                  self.beta[l, c], self.state[l], self.out[l], n_tokens=self.T,
                                  z=self.z[l, c], overlap_state_load=True)

    def capture(self):
        # The binding's per-call host cost would otherwise exceed the kernels' time.
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.enqueue_call(0)  # load the library and kernels before capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        for c in range(self.slots):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                self.enqueue_call(c)
            self.graphs.append(gr)
        torch.cuda.synchronize()

    def run(self, first, n):
        for s in range(first, first + n):
            self.graphs[s % self.slots].replay()


class DecodeE2E:
    """Same steps through the same C ABI, with every step's inputs copied in from
    pinned host memory and its outputs copied back.

    Each step is one CUDA graph (how a serving loop replays a decode step
    without paying the Python binding's per-call cost): on a side stream it
    copies the NEXT step's inputs into the other of two device input buffers
    and the PREVIOUS step's output back to the host, while on the main stream
    its own 18 library calls read the inputs the previous step copied and
    write the other of two device output buffers.  So every step moves one
    step's inputs and one step's output, and the copies overlap the kernels."""

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
        self.d_out = [torch.empty_like(bench.out) for _ in range(2)]
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
        # The side stream starts once the previous step's kernels are done: its
        # inputs buffer may be refilled and its output read back.  (An even
        # slot count makes a slot's parity its step's.)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self._copy_in((slot + 1) % self.host_slots)
            self.h_out.copy_(self.d_out[(slot + 1) % 2], non_blocking=True)
        self.b.launch_step(0, x=self.view[slot % 2], out=self.d_out[slot % 2])
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
    mb = DecodeMultiBench(device, seed=12, B=B, slots=slots, T=T)
    mb.capture()
    mb.run(0, warmup)
    ms = time_region(lambda: mb.run(warmup, steps), steps, world)
    nbytes = mb.bytes_per_call
    del mb
    torch.cuda.empty_cache()
    res["batch_sweep"] = decode_batch_sweep(device, world=world)
    res["multi_token"] = {
        "value": nbytes * steps / (ms * 1e-3) / 1e9, "unit": "GB/s", "tokens_per_call": T,
        "tokens_per_s": B * T * steps / (ms * 1e-3), "us_per_launch": ms * 1e3 / (steps * LAYERS),
        "launch": f"{LAYERS} launches per call, {T} tokens per sequence each, one CUDA graph per call"}
    return res


# ---------------------------------------------------------------- prefill

def prefill_measure(device, lens=None, H_k=P_H, H_v=P_H, seed=2, g_mode="softplus",
                    workload=None, reps=5, world=1):
    """Median time of one chunked prefill over the packed sequences `lens` (default:
    the Qwen3.5-0.8B-shaped 4 x 4096 prompt batch), L2 flushed before every
    repetition; tokens/s and algorithmic TFLOP/s against the bf16 peak."""
    import linear_attention_recurrence_10_b200 as gdr
    from linear_attention_recurrence_10_b200 import synth
    lens = lens or [P_LEN] * P_SEQS
    inp = synth.make_inputs(lens, H_k, H_v, D, seed=seed, g_mode=g_mode, device=device)
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device=device)
    out = torch.empty(inp.n_tok, H_v, D, device=device, dtype=torch.bfloat16)
    final = torch.empty(len(lens), H_v, D, D, device=device)
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
    fpt = prefill_flops_per_token_head(P_CHUNK, D, H_v // H_k)
    flops = n_tok * H_v * fpt
    per_gpu_tflops = flops / world / (ms * 1e-3) / 1e12
    peaks = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    workload = workload or (f"Qwen3.5-0.8B-shaped prefill: {P_SEQS} x {P_LEN} tokens, "
                            f"{H_k}/{H_v} heads, d={D}, bf16, chunk {P_CHUNK}, S_0=0")
    return {"metric": "chunked-prefill tokens/s", "value": n_tok / (ms * 1e-3), "unit": "tokens/s",
            "ms": ms, "workload": workload, "tokens": inp.n_tok, "n_gpus": world,
            "scaling": "weak", "tflops": tflops, "tc_frac": per_gpu_tflops / peaks["bf16_tflops"],
            "tc_peak_tflops": peaks["bf16_tflops"], "flops_per_token_head": fpt,
            "roofline": {"bound": "tensor", "achieved": per_gpu_tflops,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": per_gpu_tflops / peaks["bf16_tflops"], "traffic": None,
                         "peak_source": peaks["source"] + " bf16 GEMM, burst (bf16_tflops)"},
            "l2": "flushed (256 MB write) before each repetition", "reps": reps}


def long_context_prefill_measure(device, reps=3, world=1):
    """Long-context GVA prefill: 8 sequences of U{1024..32768} tokens (seed 4),
    16 key / 32 value heads, d=128, bf16, chunk 64, exp(g) in [0.9, 1), S_0 = 0."""
    from linear_attention_recurrence_10_b200 import synth
    lens = synth.lengths(LC_SEQS, LC_SEED, LC_LO, LC_HI)
    return prefill_measure(
        device, lens, LC_HK, LC_HV, seed=LC_SEED, g_mode="long", reps=reps, world=world,
        workload=f"long-context GVA prefill: {LC_SEQS} sequences of U{{{LC_LO}..{LC_HI}}} tokens "
                 f"({sum(lens)} in all), {LC_HK}/{LC_HV} heads, d={D}, bf16, chunk {P_CHUNK}, "
                 f"exp(g) in [0.9, 1), S_0=0")


def attn_decode_bytes_per_layer(B, H_q, H_kv, d, ctx, out_b=OUT_BYTES) -> int:
    """Algorithmic bytes of one gated-attention decode step of one layer: the
    cache rows read (ctx cached + the appended one, keys and values), the new
    key and value read and appended, q and gate read, the output written."""
    cache = B * H_kv * (ctx + 1) * 2 * d * 2
    new_kv = B * H_kv * 2 * d * 2 * 2
    q_gate = B * H_q * 2 * d * 2
    return cache + new_kv + q_gate + B * H_q * d * out_b


def attn_decode_measure(device, steps=16, warmup=4, world=1, layers=ATT_LAYERS):
    """Qwen3.6-35B-A3B-shaped gated full-attention decode: 10 layers' KV caches
    (64 x 2 heads x 4097 rows x 256, bf16: 5.4 GB in all) rotate through HBM;
    one step runs the 10 layers' decode calls from one CUDA graph."""
    import linear_attention_recurrence_10_b200 as gdr
    from linear_attention_recurrence_10_b200 import synth
    L, B, Hq, Hkv, d, ctx = layers, ATT_B, ATT_HQ, ATT_HKV, ATT_D, ATT_CTX
    nrm = lambda shape, name: synth.normal(shape, 9, name, device=device).to(torch.bfloat16)
    q, gate = nrm((L, B, Hq, d), "att_q"), nrm((L, B, Hq, d), "att_gate")
    k, v = nrm((L, B, Hkv, d), "att_k"), nrm((L, B, Hkv, d), "att_v")
    kc = torch.empty(L, B, Hkv, ctx + 1, d, device=device, dtype=torch.bfloat16)
    vc = torch.empty_like(kc)
    for l in range(L):  # the cached rows, drawn layer by layer
        kc[l] = nrm((B, Hkv, ctx + 1, d), f"att_kc{l}")
        vc[l] = nrm((B, Hkv, ctx + 1, d), f"att_vc{l}")
    cache_len = torch.full((B,), ctx, dtype=torch.int32, device=device)
    out = torch.empty(L, B, Hq, d, device=device, dtype=torch.bfloat16)
    n = gdr.attn_decode_workspace_size(q[0], gate[0], k[0], v[0], kc[0], vc[0], cache_len, out[0],
                                       kv_bound=ctx, rot_dim=ATT_ROT)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)

    def step():
        for l in range(L):
            gdr.attn_decode_step(q[l], gate[l], k[l], v[l], kc[l], vc[l], cache_len, out[l],
                                 kv_bound=ctx, rot_dim=ATT_ROT, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        graph.replay()
    ms = time_region(lambda: [graph.replay() for _ in range(steps)], steps, world)
    status = int(ws[:4].view(torch.int32).item())
    from linear_attention_recurrence_10_b200.ranks import weak_scaling_rate
    per_layer = attn_decode_bytes_per_layer(B, Hq, Hkv, d, ctx)
    peaks = load_peaks()
    achieved = per_layer * L * steps / (ms * 1e-3) / 1e9
    res = {"metric": "gated-attention decode GB/s", "unit": "GB/s",
           "value": weak_scaling_rate(per_layer * L * steps, world, ms) / 1e9,
           "steps": steps, "ms_per_step": ms / steps, "status_word": status,
           "tokens_per_s": weak_scaling_rate(B * steps, world, ms),
           "workload": f"Qwen3.6-35B-A3B-shaped gated attention decode: {L} layers x B={B}, "
                       f"{Hq}/{Hkv} heads, head_dim {d}, {ctx} cached tokens, RoPE on {ATT_ROT} "
                       f"dims, bf16 cache and outputs",
           "l2": f"inputs larger than L2: {L} layers' caches "
                 f"({2 * kc.numel() * 2 / 1e9:.1f} GB) rotate every step",
           "launch": "one CUDA graph per step: rope/append and attend per layer (one work item "
                     "per (sequence, kv head): the attend kernel stores the gated output, no "
                     "combine)",
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                        "traffic": captured_traffic("attend_kernel"), "kernel": "attend_kernel",
                        "bytes_per_layer": per_layer,
                        "us_per_layer": ms * 1e3 / (steps * L),
                        "peak_source": peaks["source"] + " copy bandwidth (hbm_gbs)"}}
    del graph, q, gate, k, v, kc, vc, out, ws
    torch.cuda.empty_cache()
    return res


def moe_bytes_per_layer(n_tok, n_active, E=MOE_E, H=MOE_H, I=MOE_I, SI=MOE_SI, out_b=OUT_BYTES) -> int:
    """Algorithmic bytes of one MoE decode step of one layer: the router and
    shared-gate rows, the gate/up and down weights of the n_active experts the
    tokens chose and of the shared expert (bf16), the tokens in, the outputs out."""
    return (E * H + H) * 2 + n_active * 3 * I * H * 2 + 3 * SI * H * 2 + n_tok * H * (2 + out_b)


def moe_decode_measure(device, B=1, steps=32, warmup=4, world=1, slots=16, layers=MOE_LAYERS):
    """Qwen3.6-35B-A3B-shaped MoE decode: 8 layers' expert weights rotate through
    HBM; each step runs B tokens through the 8 layers (one CUDA graph per step,
    five kernels per layer).  The bytes are counted from each step's routing:
    only the experts some token chose are read."""
    import linear_attention_recurrence_10_b200 as gdr
    from linear_attention_recurrence_10_b200 import synth
    L, H, E, K, I, SI = layers, MOE_H, MOE_E, MOE_K, MOE_I, MOE_SI
    nrm = lambda shape, name, std: (synth.normal(shape, 10, name, device=device) * std).to(torch.bfloat16)
    layers = []
    for l in range(L):
        layers.append(dict(
            w_router=nrm((E, H), f"moe_r{l}", H ** -0.5),
            w_gate_up=nrm((E, 2 * I, H), f"moe_gu{l}", H ** -0.5),
            w_down=nrm((E, H, I), f"moe_d{l}", I ** -0.5),
            shared=(nrm((2 * SI, H), f"moe_sgu{l}", H ** -0.5), nrm((H, SI), f"moe_sd{l}", SI ** -0.5),
                    nrm((H,), f"moe_sg{l}", H ** -0.5))))
    x = nrm((slots, L, B, H), "moe_x", 1.0)
    out = torch.empty(L, B, H, device=device, dtype=torch.bfloat16)
    idx = torch.empty(slots, L, B, K, dtype=torch.int32, device=device)
    w0 = layers[0]
    n = gdr.moe_workspace_size(x[0, 0], w0["w_router"], w0["w_gate_up"], w0["w_down"], out[0],
                               top_k=K, shared=w0["shared"])
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)

    def step(sl):
        for l, w in enumerate(layers):
            gdr.moe_decode(x[sl, l], w["w_router"], w["w_gate_up"], w["w_down"], out[l], top_k=K,
                           shared=w["shared"], topk_idx=idx[sl, l], workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for sl in range(slots):
            step(sl)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    routing = idx.cpu()
    per_step = [sum(moe_bytes_per_layer(B, len(set(routing[sl, l].flatten().tolist())))
                    for l in range(L)) for sl in range(slots)]
    graphs = []
    for sl in range(slots):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            step(sl)
        graphs.append(gr)
    for s_ in range(warmup):
        graphs[s_ % slots].replay()
    ms = time_region(lambda: [graphs[(warmup + s_) % slots].replay() for s_ in range(steps)], steps,
                     world)
    nbytes = sum(per_step[(warmup + s_) % slots] for s_ in range(steps))
    from linear_attention_recurrence_10_b200.ranks import weak_scaling_rate
    peaks = load_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    res = {"metric": "MoE decode GB/s (routed experts read)", "unit": "GB/s",
           "value": weak_scaling_rate(nbytes, world, ms) / 1e9, "steps": steps,
           "ms_per_step": ms / steps, "us_per_layer": ms * 1e3 / (steps * L),
           "tokens_per_s": weak_scaling_rate(B * steps, world, ms),
           "bytes_per_step": nbytes / steps,
           "workload": f"Qwen3.6-35B-A3B-shaped MoE decode: {L} layers x B={B} tokens, hidden {H}, "
                       f"{E} experts top-{K}, intermediate {I}, shared expert {SI}, bf16 weights",
           "l2": f"inputs larger than L2: {L} layers' weights "
                 f"({L * (E * 3 * I * H + 3 * SI * H + E * H) * 2 / 1e9:.1f} GB) rotate; each step "
                 f"reads ~{nbytes / steps / 1e6:.0f} MB",
           "launch": "one CUDA graph per step: 5 kernels per layer (router, route, gate_up, down, "
                     "combine)",
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                        "peak_source": peaks["source"] + " copy bandwidth (hbm_gbs)"}}
    del graphs, layers, x, out, ws
    torch.cuda.empty_cache()
    return res


def gva_decode_measure(device, steps=32, warmup=4, world=1):
    """Qwen3.6-35B-A3B-shaped GVA decode: B=64, 16 key / 32 value heads, 30 layer
    states (4.0 GB, rotating through HBM), 256 distinct steps cycled; one CUDA
    graph of 30 decode launches per step."""
    b = DecodeBench(device, seed=3, B=GVA_B, layers=GVA_LAYERS, slots=GVA_STEPS, H_k=GVA_HK,
                    H_v=GVA_HV)
    b.capture()
    b.run(0, warmup)
    ms = time_region(lambda: b.run(warmup, steps), steps, world)
    from linear_attention_recurrence_10_b200.ranks import weak_scaling_rate
    per_launch_ms = ms / (steps * b.L)
    achieved = b.bytes_per_launch / (per_launch_ms * 1e-3) / 1e9
    peaks = load_peaks()
    res = {"metric": HEADLINE, "value": weak_scaling_rate(b.bytes_per_step * steps, world, ms) / 1e9,
           "unit": "GB/s", "steps": steps, "ms_per_step": ms / steps,
           "tokens_per_s": weak_scaling_rate(GVA_B * steps, world, ms),
           "workload": f"Qwen3.6-35B-A3B-shaped GVA decode: {GVA_LAYERS} layers x B={GVA_B}, "
                       f"{GVA_HK}/{GVA_HV} heads, d={D}, bf16 q/k/v/z/out, fp32 state",
           "l2": f"inputs larger than L2: {GVA_LAYERS} layer states "
                 f"({GVA_LAYERS * GVA_B * GVA_HV * D * D * 4 / 1e9:.1f} GB) rotate every step",
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                        "bytes_per_launch": b.bytes_per_launch,
                        "us_per_launch": per_launch_ms * 1e3,
                        "peak_source": peaks["source"] + " copy bandwidth (hbm_gbs)"}}
    del b
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------- CPU oracle

def oracle_sample(n_tokens=512, seed=1, threads=None, reps=30):
    """Time the fp64 oracle on one layer of the decode workload: B sequences x
    16 heads x n_tokens steps, on every host core, `reps` times over (about ten
    seconds of CPU work with the defaults)."""
    import numpy as np
    import oracle
    from linear_attention_recurrence_10_b200 import synth
    threads = threads or os.cpu_count() or 1
    inp = synth.make_inputs([n_tokens] * BATCH, H_K, H_V, D, seed=seed, s0_std=0.02)
    f = lambda t: t.to(torch.float64).numpy()
    args = dict(q=f(inp.q), k=f(inp.k), v=f(inp.v), g=f(inp.g), beta=f(inp.beta),
                cu_seqlens=np.array(inp.cu_seqlens), z=f(inp.z), s0=f(inp.s0), w=f(inp.w))
    lib = oracle.load()
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.gdr_recurrent(**args, threads=threads, lib=lib)
    dt = time.perf_counter() - t0
    nbytes = reps * n_tokens * decode_bytes_per_layer_step(BATCH, H_K, H_V, D)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": dt,
            "sample": f"one layer of the decode workload: {BATCH} sequences x {H_V} heads x "
                      f"{n_tokens} tokens, fp64 recurrence, {threads} threads, {reps} times"}


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
    ap.add_argument("--slots", type=int, default=INPUT_SETS,
                    help="device-resident per-step input sets of the decode, cycled")
    ap.add_argument("--e2e-steps", type=int, default=1024)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-variants", action="store_true")
    ap.add_argument("--no-gva-decode", action="store_true")
    ap.add_argument("--no-attn-decode", action="store_true")
    ap.add_argument("--no-moe", action="store_true")
    ap.add_argument("--moe-only", action="store_true",
                    help="run only the MoE decode measurements and print their JSON")
    ap.add_argument("--moe-layers", type=int, default=MOE_LAYERS,
                    help="layers' expert weights rotated in the MoE measurement (fewer for profiling)")
    ap.add_argument("--attn-only", action="store_true",
                    help="run only the gated-attention decode measurement and print its JSON")
    ap.add_argument("--attn-layers", type=int, default=ATT_LAYERS,
                    help="layers' caches rotated in the attention measurement (fewer for profiling)")
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
    if args.moe_only:
        res = {"B1": moe_decode_measure(device, B=1, world=world, layers=args.moe_layers),
               "B8": moe_decode_measure(device, B=8, world=world, layers=args.moe_layers)}
        if rank == 0:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.attn_only:
        res = attn_decode_measure(device, world=world, layers=args.attn_layers)
        if rank == 0:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.prefill_only:
        pre = prefill_measure(device, reps=args.prefill_reps, world=world)
        pre["long_context_prefill"] = long_context_prefill_measure(device, world=world)
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
    gva = None if args.no_gva_decode else gva_decode_measure(device, world=world)
    attn = None if args.no_attn_decode else attn_decode_measure(device, world=world)
    moe = None if args.no_moe else {"B1": moe_decode_measure(device, B=1, world=world),
                                    "B8": moe_decode_measure(device, B=8, world=world)}
    prefill = None if args.no_prefill else prefill_measure(device, reps=args.prefill_reps,
                                                           world=world)
    long_prefill = None if args.no_prefill else long_context_prefill_measure(device, world=world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample()
        one = oracle_sample(n_tokens=32, threads=1, reps=30)
        cpu["single_thread"] = {"value": one["value"], "unit": one["unit"], "cores": 1,
                                "seconds": one["seconds"], "sample": one["sample"]}

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
                  f"({LAYERS * args.batch * H_V * D * D * 4 / 1e6:.0f} MB) rotate every step; "
                  f"per-step inputs cycle through {args.slots} device-resident sets",
            "launch": "one CUDA graph per step (one decode launch per layer)"},
        "tokens_per_s": weak_scaling_rate(args.batch * args.steps, world, ms),
        "hbm_frac": gbs / world / peaks["hbm_gbs"],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": captured_traffic("decode_rb_kernel<bf16, bf16>"),
                     "kernel": "decode_rb_kernel<bf16, bf16>",
                     "bytes_per_launch": per_launch_bytes, "us_per_launch": per_launch_ms * 1e3,
                     "peak_source": peaks["source"] + " copy bandwidth (hbm_gbs)"},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes, "steps": args.e2e_steps,
                "launch": "one CUDA graph per step: the 18 library calls on inputs the previous "
                          "step copied from pinned host memory, while a side stream copies the "
                          "next step's inputs in and the previous step's outputs back (two "
                          "device output buffers)",
                "ms_per_step": ms_e2e / args.e2e_steps},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clock_info,
        "decode_variants": variants,
        "gva_decode": gva,
        "attn_decode": attn,
        "moe_decode": moe,
        "prefill": prefill,
        "long_context_prefill": long_prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
