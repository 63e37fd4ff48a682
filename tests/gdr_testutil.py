"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding, run the fp64 oracle on the same seeded inputs, compare.

Error metric: relative L2, |x - x_ref|_2 / |x_ref|_2 over the compared tensor.
Bars (the mixer's stated acceptance): bf16 inputs -> outputs <= 2e-3 and
final fp32 state <= 1e-3; fp32 inputs -> 1e-5.  Outputs are compared in fp32
(out_dtype fp32): rounding y to bf16 alone would cost ~1.6e-3 of the 2e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import linear_attention_recurrence_10_b200 as gdr
import oracle
from linear_attention_recurrence_10_b200 import synth

TOL = {torch.bfloat16: dict(out=2e-3, state=1e-3), torch.float32: dict(out=1e-5, state=1e-5)}


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def sub_problem(inp: synth.Inputs, seq: int, hv: int):
    """Inputs of one (sequence, value head) for the oracle: 1 key head, 1 value head."""
    t0, t1 = inp.cu_seqlens[seq], inp.cu_seqlens[seq + 1]
    hk = hv * inp.H_k // inp.H_v
    return dict(
        q=f64(inp.q[t0:t1, hk:hk + 1]), k=f64(inp.k[t0:t1, hk:hk + 1]),
        v=f64(inp.v[t0:t1, hv:hv + 1]), z=f64(inp.z[t0:t1, hv:hv + 1]),
        g=f64(inp.g[t0:t1, hv:hv + 1]), beta=f64(inp.beta[t0:t1, hv:hv + 1]),
        s0=None if inp.s0 is None else f64(inp.s0[seq:seq + 1, hv:hv + 1]),
        w=f64(inp.w), cu_seqlens=[0, t1 - t0])


def oracle_full(inp: synth.Inputs, threads=8, **kw):
    return oracle.gdr_recurrent(
        q=f64(inp.q), k=f64(inp.k), v=f64(inp.v), g=f64(inp.g), beta=f64(inp.beta),
        cu_seqlens=inp.cu_seqlens, z=f64(inp.z), s0=f64(inp.s0), w=f64(inp.w), threads=threads,
        **kw)


def run_decode(inp: synth.Inputs, T: int, *, out_dtype=torch.float32, with_z=True,
               in_place=True, **kw):
    """T decode steps over B = n_seq sequences of T tokens each (teacher forced:
    step t reads token t of every sequence from the seeded inputs)."""
    dev = "cuda"
    B = inp.n_seq
    d = inp.d
    x = inp.to(dev)
    q = x.q.view(B, T, inp.H_k, d)
    k = x.k.view(B, T, inp.H_k, d)
    v = x.v.view(B, T, inp.H_v, d)
    z = x.z.view(B, T, inp.H_v, d)
    g = x.g.view(B, T, inp.H_v)
    beta = x.beta.view(B, T, inp.H_v)
    state = (x.s0.clone() if x.s0 is not None
             else torch.zeros(B, inp.H_v, d, d, device=dev, dtype=torch.float32))
    bufs = [state, state if in_place else torch.empty_like(state)]
    out = torch.empty(B, T, inp.H_v, d, device=dev, dtype=out_dtype)
    for t in range(T):
        src, dst = bufs[t % 2], bufs[(t + 1) % 2]
        gdr.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], src, out[:, t],
                        z=z[:, t] if with_z else None, norm_w=x.w, state_out=dst, **kw)
    final = bufs[T % 2]
    torch.cuda.synchronize()
    return out.reshape(B * T, inp.H_v, d), final


def run_prefill(inp: synth.Inputs, *, chunk=64, out_dtype=torch.float32, with_z=True,
                initial_state="inputs", **kw):
    dev = "cuda"
    x = inp.to(dev)
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device=dev)
    out = torch.empty(inp.n_tok, inp.H_v, inp.d, device=dev, dtype=out_dtype)
    s0 = x.s0 if initial_state == "inputs" else initial_state
    final = torch.empty(inp.n_seq, inp.H_v, inp.d, inp.d, device=dev, dtype=torch.float32)
    gdr.prefill_chunked(x.q, x.k, x.v, x.g, x.beta, cu, out, cu_seqlens_host=inp.cu_seqlens,
                        z=x.z if with_z else None, norm_w=x.w, initial_state=s0,
                        final_state=final, chunk=chunk, **kw)
    torch.cuda.synchronize()
    return out, final
