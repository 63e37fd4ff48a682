"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding, run the fp64 oracle on the same seeded inputs, compare.

Error metric: relative L2, |x - x_ref|_2 / |x_ref|_2 over the compared tensor.
Bars (the mixer's stated acceptance): bf16 inputs -> outputs <= 2e-3 and
final fp32 state <= 1e-3; fp32 inputs -> 1e-5.  Outputs are compared in fp32
(out_dtype fp32): rounding y to bf16 alone would cost ~1.6e-3 of the 2e-3.

A relative L2 over millions of elements cannot see one bad element, so every
comparison also bounds each element:

    max_i |x_i - ref_i| <= ELEM_C * tol * RMS(ref)   (+ one bf16 ulp of |ref_i|
                                                      when x was stored as bf16)

ELEM_C = 128.  Errors are not Gaussian with one scale: where the tensor cores
see the state as bf16, the error of o_t = S_t q_t is relative to |S_t||q_t|,
not to o_t, so a token whose output is small against its state carries a
relative error many times the tensor's, and RMSNormGated scales that token back
up to full size.  The largest of up to 2^26 elements then sits well past the
Gaussian sqrt(2 ln 2^26) ~ 6 times the RMS error.  Measured on the tensor-core
prefill: 13-28x the output bar in most tests, 82x for one token of the
4 x 4096 prompt batch (rel-L2 there 0.14x the bar); decode and attention stay
under 11x.  128 x the output bar is a quarter of the tensor's RMS: an element
wrong by a quarter of the tensor's typical size or more fails.
When GDR_TEST_ERRLOG names a file, every comparison appends its figures to it.
"""
from __future__ import annotations

import json
import os

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


ELEM_C = 128.0


def max_err_ratio(x, ref, bf16_ulp=False) -> float:
    """max_i |x_i - ref_i| / (tol-free scale): the largest element error over
    RMS(ref), after subtracting one bf16 ulp of |ref_i| when ``bf16_ulp``."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    err = np.abs(x - ref)
    if bf16_ulp:
        err = np.maximum(err - np.abs(ref) * 2.0 ** -8, 0.0)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(err.max() / (rms if rms > 0 else 1.0))


def assert_close(x, ref, tol, what="", bf16_ulp=False):
    """Relative L2 <= tol and every element within ELEM_C * tol * RMS(ref)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, f"{what}: shape {x.shape} vs {ref.shape}"
    assert np.isfinite(x).all(), f"{what}: non-finite values"
    e = rel_l2(x, ref)
    m = max_err_ratio(x, ref, bf16_ulp)
    log = os.environ.get("GDR_TEST_ERRLOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "?"), "what": what,
                                "tol": tol, "rel_l2": e, "max_over_rms": m,
                                "n": int(x.size)}) + "\n")
    assert e <= tol, f"{what} rel-L2 {e:.3e} > {tol:.1e}"
    assert m <= ELEM_C * tol, f"{what} max element error {m:.3e} x RMS > {ELEM_C * tol:.1e}"
    return e, m


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


def oracle_sequence(inp: synth.Inputs, seq: int, threads=8, **kw):
    """The oracle on one whole sequence (every head) of a packed problem."""
    t0, t1 = inp.cu_seqlens[seq], inp.cu_seqlens[seq + 1]
    return oracle.gdr_recurrent(
        q=f64(inp.q[t0:t1]), k=f64(inp.k[t0:t1]), v=f64(inp.v[t0:t1]), g=f64(inp.g[t0:t1]),
        beta=f64(inp.beta[t0:t1]), cu_seqlens=[0, t1 - t0], z=f64(inp.z[t0:t1]),
        s0=None if inp.s0 is None else f64(inp.s0[seq:seq + 1]), w=f64(inp.w),
        threads=threads, **kw)


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
